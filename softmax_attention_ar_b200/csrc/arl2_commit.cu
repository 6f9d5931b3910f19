// Commit kernels of the ARL2 hybrid layer: the clean-pass gated-delta state update
// ("Attend Locally, Remember Linearly", technical summary of arXiv 2605.16579, §2.1 state
// update and §2.2 clean-pass update), read with an explicit transpose:
//     K' = rownorm(K Wk_h),  V' = V Wv_h,  abar = mean_t alpha_t
//     S_N = abar S_{N-1} + K'^T diag(beta / T) (V' - K' S_{N-1})
//
// Kernel 1 (one CTA per group of 128-token chunks of one (batch, head)) runs the chain
// per chunk on the tensor cores, with TMEM accumulators:
//     Kp = K Wk, Vp = V Wv            (MMA)
//     K' = Kp / max(|Kp|, 1e-12)      (thread = token row; bf16 into shared memory)
//     KS = K' S_{N-1}                 (MMA, state from its bf16 copy)
//     R  = (Vp - KS) beta_t / T       (thread = token row; bf16 into shared memory)
//     U += K'^T R                     (MMA, both operands MN-major; accumulates over chunks)
// and writes its partial U (fp32) and partial sum of alpha to scratch.
// Kernel 2 adds the partials in a fixed order (deterministic, no atomics) and writes
// S_N = abar S_{N-1} + U into the other state buffer, with its bf16 copy.
//
// Roles of kernel 1 (192 threads): warp 0 TMA, warp 1 TMEM owner + MMA issuer (lane 0),
// warps 2-5 row warps (thread = token row for K'/R, = state row k for the U write-out).
// TMEM: Kp at 0, Vp at 128, KS at 256, U at 384. Shared memory: Wk | Wv | S | K0 K1 | V0 V1.
#include <algorithm>

#include "arl2_device.cuh"
#include "arl2_kernels.h"

namespace arl2 {
namespace {

constexpr uint32_t kWkOff = 0;
constexpr uint32_t kWvOff = kTileBytes;
constexpr uint32_t kSOff = 2 * kTileBytes;
constexpr uint32_t kKOff = 3 * kTileBytes;   // two buffers
constexpr uint32_t kVOff = 5 * kTileBytes;   // two buffers
constexpr uint32_t kBarOff = 7 * kTileBytes;
enum : int {
  kBarW = 0,
  kBarKVFull = 1,   // +buffer
  kBarKVEmpty = 3,  // +buffer
  kBarProj = 5,     // Kp, Vp in TMEM
  kBarKn = 6,       // K' bf16 in shared memory (128 arrivals)
  kBarKS = 7,       // K'S in TMEM
  kBarR = 8,        // R bf16 in shared memory (128 arrivals)
  kBarU = 9,        // U complete
  kBarFinal = 10,
  kNumBars = 11
};
constexpr uint32_t kMiscOff = kBarOff + 256;
constexpr uint32_t kSmemBytes = kMiscOff + 64 + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColKp = 0, kColVp = 128, kColKS = 256, kColU = 384;
constexpr float kNormEps = 1e-12f;

struct Smem {
  uint32_t base;
  __device__ uint32_t bar(int i) const { return base + kBarOff + 8u * i; }
  __device__ uint32_t wk() const { return base + kWkOff; }
  __device__ uint32_t wv() const { return base + kWvOff; }
  __device__ uint32_t s() const { return base + kSOff; }
  __device__ uint32_t k(int i) const { return base + kKOff + i * kTileBytes; }
  __device__ uint32_t v(int i) const { return base + kVOff + i * kTileBytes; }
};

__device__ void producer(const Smem& sm, const CUtensorMap* tm_k, const CUtensorMap* tm_v, const CUtensorMap* tm_wk,
                         const CUtensorMap* tm_wv, const CUtensorMap* tm_s, const CommitArgs& a, int c0, int nc,
                         int h, int b, const Guard& g) {
  uint32_t n[2] = {0, 0};
  const int slot = a.state_slot * a.B * a.H + b * a.H + h;
  mbar_expect_tx(sm.bar(kBarW), 3 * kTileBytes);
  for (int p = 0; p < 2; ++p) {
    tma_load_3d(sm.wk() + p * kPanelBytes, tm_wk, sm.bar(kBarW), 64 * p, 0, h);
    tma_load_3d(sm.wv() + p * kPanelBytes, tm_wv, sm.bar(kBarW), 64 * p, 0, h);
    tma_load_3d(sm.s() + p * kPanelBytes, tm_s, sm.bar(kBarW), 64 * p, 0, slot);
  }
  for (int i = 0; i < nc; ++i) {
    const int s = i & 1;
    if (i >= 2 && !mbar_wait(sm.bar(kBarKVEmpty + s), ((i - 2) >> 1) & 1, g)) break;
    mbar_expect_tx(sm.bar(kBarKVFull + s), 2 * kTileBytes);
    const int row = (c0 + i) * kRows;
    for (int p = 0; p < 2; ++p) {
      tma_load_4d(sm.k(s) + p * kPanelBytes, tm_k, sm.bar(kBarKVFull + s), 64 * p, h, row, b);
      tma_load_4d(sm.v(s) + p * kPanelBytes, tm_v, sm.bar(kBarKVFull + s), 64 * p, h, row, b);
    }
    ++n[s];
  }
  mbar_wait_drain(sm.bar(kBarW), 0);
  for (int s = 0; s < 2; ++s)
    if (n[s]) mbar_wait_drain(sm.bar(kBarKVFull + s), (n[s] - 1) & 1);
}

__device__ void mma_issuer(const Smem& sm, uint32_t tmem, int nc, const Guard& g) {
  constexpr uint32_t id_kmn = idesc_bf16(128, 128, false, true);   // A K-major, B MN-major
  constexpr uint32_t id_mnmn = idesc_bf16(128, 128, true, true);   // A MN-major, B MN-major
  if (!mbar_wait(sm.bar(kBarW), 0, g)) return;
  for (int i = 0; i < nc; ++i) {
    const int st = i & 1;
    if (!mbar_wait(sm.bar(kBarKVFull + st), (i >> 1) & 1, g)) return;
    tc_fence_after();
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_bf16(tmem + kColKp, desc_kmajor(sm.k(st), s), desc_mnmajor(sm.wk(), s), id_kmn, s > 0);
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_bf16(tmem + kColVp, desc_kmajor(sm.v(st), s), desc_mnmajor(sm.wv(), s), id_kmn, s > 0);
    mma_commit(sm.bar(kBarProj));
    if (!mbar_wait(sm.bar(kBarKn), i & 1, g)) return;
    tc_fence_after();
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_bf16(tmem + kColKS, desc_kmajor(sm.k(st), s), desc_mnmajor(sm.s(), s), id_kmn, s > 0);
    mma_commit(sm.bar(kBarKS));
    if (!mbar_wait(sm.bar(kBarR), i & 1, g)) return;
    tc_fence_after();
#pragma unroll
    for (int s = 0; s < 8; ++s)
      mma_bf16(tmem + kColU, desc_mnmajor(sm.k(st), s), desc_mnmajor(sm.v(st), s), id_mnmn, (i > 0 || s > 0) ? 1u : 0u);
    mma_commit(sm.bar(kBarKVEmpty + st));
  }
  mma_commit(sm.bar(kBarU));
}

__device__ void row_role(const Smem& sm, uint32_t tmem, const CommitArgs& a, int c0, int nc, int h, int b,
                         int warp, int lane, float* red, const Guard& g) {
  const int quarter = warp & 3;
  const uint32_t r = quarter * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const size_t bh = static_cast<size_t>(b) * a.H + h;
  const float* alpha = a.alpha + bh * a.T;
  const float* beta = a.beta + bh * a.T;
  float asum = 0.f;
  bool ok = true;
  for (int i = 0; i < nc && ok; ++i) {
    const int st = i & 1;
    const int t = (c0 + i) * kRows + static_cast<int>(r);
    const bool valid = t < a.T;
    // K' = Kp / max(|Kp|, eps) -> bf16, over the K tile (its MMA has finished).
    if (!mbar_wait_warp(sm.bar(kBarProj), i & 1, g)) { ok = false; break; }
    tc_fence_after();
    {
      uint32_t kv[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + kColKp + 32u * c, kv[c]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(kv[c]);
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) ss = fmaf(__uint_as_float(kv[c][e]), __uint_as_float(kv[c][e]), ss);
      const float inv = 1.f / fmaxf(sqrtf(ss), kNormEps);
      const uint32_t tile = sm.k(st);
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t* x = kv[c] + 8 * q;
          st_shared_v4(tile + swz_chunk(r, 4 * c + q),
                       pack_bf16x2(__uint_as_float(x[0]) * inv, __uint_as_float(x[1]) * inv),
                       pack_bf16x2(__uint_as_float(x[2]) * inv, __uint_as_float(x[3]) * inv),
                       pack_bf16x2(__uint_as_float(x[4]) * inv, __uint_as_float(x[5]) * inv),
                       pack_bf16x2(__uint_as_float(x[6]) * inv, __uint_as_float(x[7]) * inv));
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(sm.bar(kBarKn));
    // R = (Vp - K'S) * beta_t / T -> bf16, over the V tile (its MMA has finished).
    const float coef = valid ? beta[t] * a.inv_T : 0.f;
    if (valid) asum += alpha[t];
    if (!mbar_wait_warp(sm.bar(kBarKS), i & 1, g)) { ok = false; break; }
    tc_fence_after();
    const uint32_t tile = sm.v(st);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t vp[32], ks[32];
      tmem_ld32(tmem + lane_off + kColVp + 32u * c, vp);
      tmem_ld32(tmem + lane_off + kColKS + 32u * c, ks);
      tmem_wait_ld();
      reg_fence(vp);
      reg_fence(ks);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float y[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = (__uint_as_float(vp[8 * q + e]) - __uint_as_float(ks[8 * q + e])) * coef;
        st_shared_v4(tile + swz_chunk(r, 4 * c + q), pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]),
                     pack_bf16x2(y[4], y[5]), pack_bf16x2(y[6], y[7]));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(sm.bar(kBarR));
  }

  // Partial sum of alpha over this group's tokens: warp shuffles, then a fixed-order sum.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) asum += __shfl_xor_sync(0xffffffffu, asum, o);
  if (lane == 0) red[quarter] = asum;
  named_bar_sync(1, 128);
  const size_t pg = bh * a.ngroups + blockIdx.x;
  if (r == 0 && ok) a.alpha_part[pg] = red[0] + red[1] + red[2] + red[3];
  if (!ok) return;

  // Row k = r of the partial U, columns < d.
  if (!mbar_wait_warp(sm.bar(kBarU), 0, g)) return;
  tc_fence_after();
  float* dst = a.part + (pg * a.d + r) * a.d;
  for (int c = 0; 32 * c < a.d; ++c) {
    uint32_t u[32];
    tmem_ld32(tmem + lane_off + kColU + 32u * c, u);
    tmem_wait_ld();
    reg_fence(u);
    if (static_cast<int>(r) < a.d) {
      float4* d4 = reinterpret_cast<float4*>(dst + 32 * c);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        d4[q] = make_float4(__uint_as_float(u[4 * q]), __uint_as_float(u[4 * q + 1]), __uint_as_float(u[4 * q + 2]),
                            __uint_as_float(u[4 * q + 3]));
    }
  }
}

__global__ void __launch_bounds__(192, 1)
    arl2_commit_partial_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                               const __grid_constant__ CUtensorMap tm_wk, const __grid_constant__ CUtensorMap tm_wv,
                               const __grid_constant__ CUtensorMap tm_s, const CommitArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const Smem sm{base};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kMiscOff + 4);
  float* red = reinterpret_cast<float*>(gbase + kMiscOff + 16);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int nchunks = (a.T + kRows - 1) / kRows;
  const int c0 = blockIdx.x * a.chunks_per_group;
  const int nc = min(a.chunks_per_group, nchunks - c0);
  const Guard g{abort_flag, a.err, a.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(sm.bar(kBarW), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(sm.bar(kBarKVFull + s), 1);
      mbar_init(sm.bar(kBarKVEmpty + s), 1);
    }
    mbar_init(sm.bar(kBarProj), 1);
    mbar_init(sm.bar(kBarKn), 128);
    mbar_init(sm.bar(kBarKS), 1);
    mbar_init(sm.bar(kBarR), 128);
    mbar_init(sm.bar(kBarU), 1);
    mbar_init(sm.bar(kBarFinal), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_wk);
    prefetch_tmap(&tm_wv);
    prefetch_tmap(&tm_s);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) producer(sm, &tm_k, &tm_v, &tm_wk, &tm_wv, &tm_s, a, c0, nc, h, b, g);
  } else if (warp == 1) {
    if (lane == 0) {
      mma_issuer(sm, tmem, nc, g);
      mma_commit(sm.bar(kBarFinal));
    }
    __syncwarp();
  } else {
    row_role(sm, tmem, a, c0, nc, h, b, warp, lane, red, g);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    mbar_wait_drain(sm.bar(kBarFinal), 0);
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// S_new = abar * S_old + sum_g part_g, four consecutive elements per thread. The partials
// are loaded in batches of 8 (all in flight at once) and added in group order, so the sum
// does not depend on the batching.
__global__ void __launch_bounds__(256) arl2_commit_reduce_kernel(const ReduceArgs a) {
  const int bh = blockIdx.y;
  const int dd = a.d * a.d;
  const int e = (blockIdx.x * 256 + threadIdx.x) * 4;
  if (e >= dd) return;
  const float* ap = a.alpha_part + static_cast<size_t>(bh) * a.ngroups;
  float asum = 0.f;
  for (int g0 = 0; g0 < a.ngroups; g0 += 8) {
    float x[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = (g0 + j < a.ngroups) ? ap[g0 + j] : 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (g0 + j < a.ngroups) asum += x[j];
  }
  const float abar = asum * a.inv_T;
  const size_t off = static_cast<size_t>(bh) * dd + e;
  const float4 s = *reinterpret_cast<const float4*>(a.S_old + off);
  float4 acc = make_float4(abar * s.x, abar * s.y, abar * s.z, abar * s.w);
  const float* pp = a.part + static_cast<size_t>(bh) * a.ngroups * dd + e;
  for (int g0 = 0; g0 < a.ngroups; g0 += 8) {
    float4 u[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      u[j] = (g0 + j < a.ngroups) ? *reinterpret_cast<const float4*>(pp + static_cast<size_t>(g0 + j) * dd)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (g0 + j < a.ngroups) {
        acc.x += u[j].x;
        acc.y += u[j].y;
        acc.z += u[j].z;
        acc.w += u[j].w;
      }
    }
  }
  *reinterpret_cast<float4*>(a.S_new + off) = acc;
  *reinterpret_cast<uint2*>(a.S_new_bf16 + off) = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
}

__global__ void arl2_state_import_kernel(const float* __restrict__ src, float* __restrict__ S,
                                         uint16_t* __restrict__ S_bf16, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float x = src[i];
    S[i] = x;
    __nv_bfloat16 y = __float2bfloat16_rn(x);
    S_bf16[i] = *reinterpret_cast<uint16_t*>(&y);
  }
}

}  // namespace

size_t commit_smem_bytes() { return kSmemBytes; }

cudaError_t commit_setup() {
  return cudaFuncSetAttribute(arl2_commit_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemBytes));
}

cudaError_t launch_commit(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_wk,
                          const CUtensorMap& tm_wv, const CUtensorMap& tm_s, const CommitArgs& a,
                          const ReduceArgs& r, cudaStream_t stream, bool dependent) {
  // As a programmatic dependent, the partial kernel may start while the preceding kernel (a
  // query) still runs: it reads S_{N-1}, k, v and the gates, none of which a query writes, and
  // writes only its own scratch. The reduce kernel, which writes S_N, is launched normally.
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(a.ngroups, a.H, a.B);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, arl2_commit_partial_kernel, tm_k, tm_v, tm_wk, tm_wv, tm_s, a);
  if (e != cudaSuccess) return e;
  const dim3 rgrid((r.d * r.d / 4 + 255) / 256, r.BH);
  arl2_commit_reduce_kernel<<<rgrid, 256, 0, stream>>>(r);
  return cudaGetLastError();
}

cudaError_t launch_state_import(const float* src, float* S, uint16_t* S_bf16, size_t n, cudaStream_t stream) {
  const int blocks = static_cast<int>(std::min<size_t>((n + 255) / 256, 4096));
  arl2_state_import_kernel<<<blocks, 256, 0, stream>>>(src, S, S_bf16, n);
  return cudaGetLastError();
}

}  // namespace arl2
