// Query kernel of the ARL2 hybrid layer and the growing-KV-cache baseline: the launch of
// query_cta (arl2_query_body.cuh, which describes the kernel), and its host-side plan.
#include "arl2_query_body.cuh"

namespace arl2 {
namespace {

template <bool kHybrid>
__global__ void __launch_bounds__(kThreads, 1)
    arl2_query_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_o,
                      const __grid_constant__ QueryArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  query_cta<kHybrid>(tm_q, tm_k, tm_v, tm_w, tm_s, tm_o, a, smem_raw);
}

}  // namespace

size_t query_smem_bytes() { return kSmemBytes; }

cudaError_t query_setup() {
  cudaError_t e = cudaFuncSetAttribute(arl2_query_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(arl2_query_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemBytes));
}

QueryPlan plan_query(int B, int H, int T, int kv_len, int num_sms) {
  QueryPlan p{};
  p.nq = (T + kRows - 1) / kRows;
  p.nkv = (kv_len + kRows - 1) / kRows;
  p.units = static_cast<long long>(B) * H * p.nq * p.nkv;
  p.qtiles = static_cast<long long>(B) * H * p.nq;
  long long ctas = std::max<long long>(1, std::min<long long>(num_sms, p.units));
  while (true) {
    // Key tile 0 of a query tile weighs more than the others: its segment also computes the
    // readout and finishes the tile (merge, normalisation, store), which costs about as much
    // as two and a half key tiles on the B200. The weight applies only while every CTA's
    // weighted share spans a whole unit of the largest weight, so no range is empty.
    const long long wtot = p.qtiles * (4ll * p.nkv + kHeadWeight);
    p.head_w = wtot / ctas >= 4 + kHeadWeight + 1 ? kHeadWeight : 0;
    // Largest number of CTAs sharing one query tile under this grid.
    int worst = 1;
    for (long long Q = 0; Q < p.qtiles; ++Q) {
      const long long first = Q * p.nkv, last = first + p.nkv - 1;
      const int c0 = split_owner(first, p.units, p.nkv, p.head_w, static_cast<int>(ctas));
      const int c1 = split_owner(last, p.units, p.nkv, p.head_w, static_cast<int>(ctas));
      worst = std::max(worst, c1 - c0 + 1);
    }
    if (worst <= kMaxSegs || ctas == 1) {
      p.max_segs = worst;
      break;
    }
    ctas = std::max<long long>(1, ctas * 3 / 4);
  }
  p.num_ctas = static_cast<int>(ctas);
  return p;
}

size_t query_flag_count(const QueryPlan& p) { return static_cast<size_t>(p.qtiles) * p.max_segs; }

size_t query_scratch_floats(const QueryPlan& p) {
  const size_t slots = static_cast<size_t>(p.qtiles) * p.max_segs;
  return slots * kRows * kDP + slots * 2 * kRows;
}

cudaError_t launch_query(bool hybrid, const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                         const CUtensorMap& tm_w, const CUtensorMap& tm_s, const CUtensorMap& tm_o, const QueryArgs& a,
                         cudaStream_t stream, bool dependent) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(a.num_ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  if (hybrid)
    return cudaLaunchKernelEx(&cfg, arl2_query_kernel<true>, tm_q, tm_k, tm_v, tm_w, tm_s, tm_o, a);
  return cudaLaunchKernelEx(&cfg, arl2_query_kernel<false>, tm_q, tm_k, tm_v, tm_w, tm_s, tm_o, a);
}

}  // namespace arl2
