// Allocation-free form of the clean-pass commit (arl2_frame_commit_noalloc in arl2.h).
//
// Some callers cannot call cudaMalloc. Examples:
//   - a serving engine that reserved all of device memory for its own pool at start-up;
//   - a real-time frame loop that must not take the allocator's locks or its implicit
//     synchronisation;
//   - an embedding that only ever hands the library pointers into memory it owns.
// For them this file offers the commit without a context: the caller passes the inputs
// (k, v, the gates, phi_k, phi_v, S_{N-1}) and the output (S_N). The scratch the commit
// needs lives in one file-scope device array of fixed size, g_commit_scratch. It holds:
//   - the bf16 copy of S_{N-1} the MMAs read;
//   - a discarded bf16 copy of S_N (the kernel writes one for the context's queries);
//   - the chunk groups' partial sums of the update and of alpha (64 KiB per group and
//     (batch, head)), which the groups of a cluster reduce after one barrier.
// The caller passes a device status word: a kernel whose bounded wait ran out reports it
// there, and there is no other place it could be read back without a context.
// The array is part of the library's device image, so every GPU that loads the library
// holds ARL2_NOALLOC_SCRATCH_BYTES of it until the process exits.
//
// In host code the array's name is only a host-side stand-in. Its device address is
// looked up once per device, with that device current, by cudaGetSymbolAddress on the
// first call made on the device. That first call should therefore come before any stream
// capture. Every call on a device shares the one array and leaves its contents behind.
// Each call writes everything it reads back before reading it. Calls that overlap on the
// GPU (on different streams, say) race on the array and must not be made.
#include <mutex>

#include "../../include/arl2.h"
#include "arl2_kernels.h"

namespace {

constexpr size_t kScratchBytes = ARL2_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;
constexpr unsigned long long kTimeoutNs = 1000000000ull;

__device__ __align__(256) unsigned char g_commit_scratch[kScratchBytes];

std::mutex g_mu;
unsigned char* g_scratch_dev[kMaxDevices] = {};

// Device address of g_commit_scratch on the current device `dev` (looked up once per device).
arl2_status scratch_on_device(int dev, unsigned char** out) {
  if (dev < 0 || dev >= kMaxDevices) return ARL2_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_dev[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_commit_scratch) != cudaSuccess || !p) return ARL2_ERR_CUDA;
    g_scratch_dev[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_scratch_dev[dev];
  return ARL2_OK;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned(const void* p, uintptr_t a) { return p && (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" arl2_status arl2_frame_commit_noalloc(int B, int H, int T, int d, const arl2_bf16* k, const arl2_bf16* v,
                                                 const float* alpha, const float* beta, const arl2_bf16* Wk,
                                                 const arl2_bf16* Wv, const float* S_prev, float* S_next,
                                                 unsigned int* status, arl2_stream stream) {
  if (B < 1 || H < 1 || T < 1 || d < 1) return ARL2_ERR_INVALID_ARG;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(Wk, 16) || !aligned(Wv, 16) || !aligned(S_prev, 16) ||
      !aligned(S_next, 16) || !aligned(alpha, 4) || !aligned(beta, 4) || !aligned(status, 4))
    return ARL2_ERR_INVALID_ARG;
  if ((d != 32 && d != 64 && d != 128) || T > 4096 || static_cast<long long>(B) * H > 65535)
    return ARL2_ERR_UNSUPPORTED;
  int dev = 0, sms = 0;
  const arl2_status ds = static_cast<arl2_status>(arl2::prepare_device(&dev, &sms));
  if (ds != ARL2_OK) return ds;

  // The same work split as a context's commit.
  int cpg = 1, ngroups = 1;
  arl2::commit_split(T, H, B, sms, &cpg, &ngroups);

  // Scratch layout: S_{N-1} bf16 | S_N bf16 (discarded) | partial U | partial alpha sums.
  const size_t bh = static_cast<size_t>(B) * H, dd = static_cast<size_t>(d) * d;
  const size_t off_sprev = 0;
  const size_t off_snext = off_sprev + round256(bh * dd * 2);
  const size_t off_part = off_snext + round256(bh * dd * 2);
  const size_t part_floats = arl2::commit_scratch_floats(B, H, ngroups);
  const size_t needed = off_part + round256(part_floats * 4);
  if (needed > kScratchBytes) return ARL2_ERR_UNSUPPORTED;

  unsigned char* scratch = nullptr;
  const arl2_status ss = scratch_on_device(dev, &scratch);
  if (ss != ARL2_OK) return ss;
  uint16_t* s_prev_bf16 = reinterpret_cast<uint16_t*>(scratch + off_sprev);
  uint16_t* s_next_bf16 = reinterpret_cast<uint16_t*>(scratch + off_snext);

  CUtensorMap tm_k, tm_v, tm_wk, tm_wv, tm_s;
  if (!arl2::encode_act_map(&tm_k, k, B, T, H, d) || !arl2::encode_act_map(&tm_v, v, B, T, H, d) ||
      !arl2::encode_mat_map(&tm_wk, Wk, H, d) || !arl2::encode_mat_map(&tm_wv, Wv, H, d) ||
      !arl2::encode_mat_map(&tm_s, s_prev_bf16, B * H, d))
    return ARL2_ERR_CUDA;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // bf16 copy of S_{N-1} for the K'S MMA (no fp32 copy: the commit reads S_prev itself).
  if (arl2::launch_state_import(S_prev, nullptr, s_prev_bf16, bh * dd, st) != cudaSuccess) return ARL2_ERR_CUDA;

  arl2::CommitArgs a{};
  a.alpha = alpha;
  a.beta = beta;
  a.T = T;
  a.B = B;
  a.H = H;
  a.d = d;
  a.chunks_per_group = cpg;
  a.ngroups = ngroups;
  a.state_slot = 0;
  a.inv_T = 1.0f / static_cast<float>(T);
  a.err = status;
  a.timeout_ns = kTimeoutNs;
  arl2::ReduceArgs r{};
  r.S_old = S_prev;
  r.S_new = S_next;
  r.S_new_bf16 = s_next_bf16;
  r.part_u = reinterpret_cast<float*>(scratch + off_part);
  r.part_alpha = r.part_u + part_floats - bh * ngroups;
  r.d = d;
  r.inv_T = a.inv_T;
  return arl2::launch_commit(tm_k, tm_v, tm_wk, tm_wv, tm_s, a, r, st, false) == cudaSuccess ? ARL2_OK
                                                                                       : ARL2_ERR_CUDA;
}
