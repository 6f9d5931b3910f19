// Gate producer of the ARL2 hybrid layer: the per-token forget gate and rate computed from
// the token's hidden state ("Attend Locally, Remember Linearly", technical summary of arXiv
// 2605.16579, §2.1: alpha and beta are per-token learned projections). This library reads
// them as a linear projection per head plus a bias, through a sigmoid:
//     alpha[b, h, t] = sigmoid(x[b, t, :] . Wa[h, :] + ba[h])
//     beta[b, h, t]  = sigmoid(x[b, t, :] . Wb[h, :] + bb[h])
// Together that is one small GEMM, z = x Wg^T with Wg = [Wa; Wb] of 2H rows, then a
// per-column bias and a sigmoid. x is as large as one of q, k, v, so the kernel reads it once
// for all heads.
//
// One cluster of S CTAs per (batch, 128-token tile); CTA s of the cluster takes a slice of
// the model width D (its 64-column panels) and accumulates its partial z on the tensor cores
// (tcgen05, M = 128 tokens, N = 2H rounded up to 16, fp32 in TMEM). Each CTA then sends each
// token row of its partial to the CTA of the cluster that owns that row (distributed shared
// memory); after one cluster barrier each CTA sums its rows over the S partials in a fixed
// order (the result does not depend on timing), adds the bias, applies the sigmoid and
// writes alpha and beta.
//
// Roles (192 threads): warp 0 TMA (x and Wg panels through a 4-stage ring), warp 1 TMEM
// owner and MMA issuer (one elected lane issues), warps 2-5 thread = token row (TMEM lane).
// Every thread takes part in the owner phase.
#include <algorithm>

#include "arl2_device.cuh"
#include "arl2_kernels.h"

namespace arl2 {
namespace {

constexpr int kThreadsG = 192;
constexpr int kGStages = 4;
constexpr int kMaxSplit = 8;                   // CTAs per cluster (slices of D)
constexpr uint32_t kXPanel = kRows * 128;      // 128 token rows x 64 bf16 columns, 128-byte swizzled
constexpr uint32_t kWPanel = kMaxGateCols * 128;   // up to kMaxGateCols rows x 64 bf16 columns
constexpr uint32_t kStageBytes = kXPanel + kWPanel;
constexpr uint32_t kRecvOff = kGStages * kStageBytes;   // [S][rows per CTA][kMaxGateCols] fp32
constexpr uint32_t kRecvBytes = (kRows + kMaxSplit) * kMaxGateCols * 4;   // rpc * S <= kRows + S - 1 rows
constexpr uint32_t kCtlOff = kRecvOff + kRecvBytes;
enum : int {
  kBarFull = 0,     // +stage (4)
  kBarEmpty = 4,    // +stage (4)
  kBarZ = 8,        // the partial z is complete in TMEM
  kNumBarsG = 9
};
constexpr uint32_t kCtlBytes = 128;   // barriers, tmem slot, abort flag
constexpr uint32_t kSmemBytesG = kCtlOff + kCtlBytes;
constexpr uint32_t kSmemAllocG = kSmemBytesG + 1024;
static_assert(kNumBarsG * 8 + 16 <= kCtlBytes, "control block");
static_assert(kSmemAllocG <= 232448, "shared memory per CTA");
static_assert(kMaxGateCols % 16 == 0 && kMaxGateCols <= 256, "MMA N");

__device__ __forceinline__ uint64_t desc_panel(uint32_t addr, int s) {   // K-step s (16 columns) of a 64-column panel
  return sdesc_sw128(addr + s * 32, 16, 1024);
}

__global__ void __launch_bounds__(kThreadsG, 1)
    arl2_gates_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ GateArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) { return base + kCtlOff + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kCtlOff + kNumBarsG * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kCtlOff + kNumBarsG * 8 + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = static_cast<int>(gridDim.x);
  const int rank = static_cast<int>(cluster_rank());   // equals blockIdx.x: the cluster spans x
  const int tile = blockIdx.y, b = blockIdx.z;
  const int npan = (a.D + 63) / 64;
  const int ppc = (npan + S - 1) / S;                  // panels per CTA
  const int p0 = min(npan, rank * ppc), np = min(npan, p0 + ppc) - p0;
  const int ncols = a.ncols;                           // 2H rounded up to 16 (the MMA's N)
  const Guard g{abort_flag, a.err, a.timeout_ns};

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBarsG; ++i) mbar_init(bar(i), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_w);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), a.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // x panels are this frame's activations, read once: evict-first in L2.
    const uint64_t stream_policy = l2_evict_first_policy();
    const bool lead = elect_one();
    for (int i = 0; i < np; ++i) {
      const int s = i % kGStages;
      if (i >= kGStages && !mbar_wait_warp(bar(kBarEmpty + s), ((i - kGStages) / kGStages) & 1, g)) break;
      if (lead) {
        const uint32_t st = base + s * kStageBytes;
        mbar_expect_tx(bar(kBarFull + s), kXPanel + static_cast<uint32_t>(ncols) * 128);
        tma_load_3d_hint(st, &tm_x, bar(kBarFull + s), 64 * (p0 + i), tile * kRows, b, stream_policy);
        tma_load_2d(st + kXPanel, &tm_w, bar(kBarFull + s), 64 * (p0 + i), 0);
      }
      __syncwarp();
    }
    for (int s = 0; s < kGStages; ++s) {
      const int uses = np > s ? (np - s + kGStages - 1) / kGStages : 0;
      if (uses) mbar_wait_drain(bar(kBarFull + s), (uses - 1) & 1);
    }
  } else if (warp == 1) {
    const bool lead = elect_one();
    const uint32_t idesc = idesc_bf16(128, ncols, false, false);
    bool ok = true;
    for (int i = 0; i < np && ok; ++i) {
      const int s = i % kGStages;
      ok = mbar_wait_warp(bar(kBarFull + s), (i / kGStages) & 1, g);
      if (!ok) break;
      tc_fence_after();
      if (lead) {
        const uint32_t st = base + s * kStageBytes;
        for (int k = 0; k < 4; ++k)
          mma_bf16(tmem, desc_panel(st, k), desc_panel(st + kXPanel, k), idesc, (i > 0 || k > 0) ? 1u : 0u);
        mma_commit(bar(kBarEmpty + s));
      }
      __syncwarp();
    }
    if (lead) mma_commit(bar(kBarZ));   // arrives once every MMA issued above is done
    __syncwarp();
  }
  // Every thread: wait for this CTA's partial (a CTA with no panel has nothing in TMEM).
  bool ok = np == 0 || mbar_wait_warp(bar(kBarZ), 0, g);
  tc_fence_after();

  // Send the partial's rows to their owners: CTA o owns token rows [o rpc, (o + 1) rpc) of
  // the tile and receives, from each CTA j, [j][row - o rpc][column] floats.
  const int rpc = (kRows + S - 1) / S;
  const int ng = a.ngates;   // 2H valid columns
  if (warp >= 2) {
    const uint32_t r = static_cast<uint32_t>(warp & 3) * 32 + lane;   // token row == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp & 3) * 32 << 16;
    const int owner = static_cast<int>(r) / rpc;
    const uint32_t dst = peer_smem(base + kRecvOff + ((rank * rpc + (static_cast<int>(r) - owner * rpc)) * kMaxGateCols) * 4u,
                                   owner);
    for (int c = 0; c < ncols; c += 16) {
      uint32_t z[16];
      if (np > 0 && ok) {
        tmem_ld16_wait(tmem + lane_off + c, z);
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) z[e] = 0u;
      }
#pragma unroll
      for (int e = 0; e < 16; e += 4)
        if (c + e < ng)
          st_cluster_v4(dst + (c + e) * 4u, make_float4(__uint_as_float(z[e]), __uint_as_float(z[e + 1]),
                                                       __uint_as_float(z[e + 2]), __uint_as_float(z[e + 3])));
    }
  }
  tc_fence_before();
  cluster_sync();   // every partial row is in its owner's shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, a.tmem_cols);
  }
  if (!ok || *abort_flag) return;

  // Owner: rows [rank rpc, rank rpc + rpc) of the tile; item (gate column j, row), rows fastest
  // so that the alpha / beta stores of a warp are contiguous in t.
  const float* recv = reinterpret_cast<const float*>(gbase + kRecvOff);
  const int r0 = rank * rpc;
  const int nrows = max(0, min(rpc, kRows - r0));
  for (int it = threadIdx.x; it < ng * nrows; it += kThreadsG) {
    const int j = it / nrows, rr = it % nrows;
    const int t = tile * kRows + r0 + rr;
    if (t >= a.T) continue;
    float z = a.bias[j];
    for (int src = 0; src < S; ++src) z += recv[(src * rpc + rr) * kMaxGateCols + j];
    const float gate = 1.f / (1.f + expf(-z));
    const int h = j < a.H ? j : j - a.H;
    float* out = j < a.H ? a.alpha : a.beta;
    out[(static_cast<size_t>(b) * a.H + h) * a.T + t] = gate;
  }
}

}  // namespace

cudaError_t gates_setup() {
  return cudaFuncSetAttribute(arl2_gates_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemAllocG));
}

int gate_split(int D) {
  const int npan = (D + 63) / 64;
  return std::max(1, std::min(kMaxSplit, npan));
}

cudaError_t launch_gates(const CUtensorMap& tm_x, const CUtensorMap& tm_w, const GateArgs& a, cudaStream_t stream) {
  const int S = gate_split(a.D);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(S, (a.T + kRows - 1) / kRows, a.B);
  cfg.blockDim = dim3(kThreadsG);
  cfg.dynamicSmemBytes = kSmemAllocG;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, arl2_gates_kernel, tm_x, tm_w, a);
}

}  // namespace arl2
