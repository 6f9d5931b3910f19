// Query kernel of the ARL2 hybrid layer, and the growing-KV-cache baseline that shares it.
//
// Computes, for one 128-row query tile of one (batch, head) per CTA
// ("Attend Locally, Remember Linearly", technical summary of arXiv 2605.16579, §2.1):
//     O = softmax(Q K^T / sqrt(d)) V  +  (Q Wq_h) S_{N-1}
// The intra-frame branch is unmasked inside the frame; the inter-frame branch reads the
// state of the previous frame and never writes it (§2.2, frame-level access). With
// kHybrid = false the kernel is the baseline the layer replaces (§1): softmax attention of
// the newest frame over every cached key, with no state branch.
//
// Roles (192 threads, one CTA per SM):
//   warp 0     TMA producer: Q tile (+ Wq_h and the bf16 state copy), then K/V tiles into
//              a two-stage ring; K and V stages are released separately.
//   warp 1     TMEM owner; lane 0 issues every tcgen05.mma and commit.
//   warps 2-5  softmax warpgroup; thread = query row = TMEM lane. Also converts Q' to bf16
//              for the readout MMA and writes the output.
// TMEM (512 columns): S tiles at 0 and 128 (double-buffered), O at 256, Q' / O_inter at 384.
// Shared memory: Q | K0 K1 | V0 V1 | P0 P1 (32 KiB tiles). P0/P1 hold Wq_h and the state
// during the prologue, then Q' (bf16), then the probabilities of each KV tile.
//
// Online softmax: scores are kept in log2 units; the running max m is raised only when a
// tile's max exceeds it by more than 8 (a factor 256), so O in TMEM is rescaled rarely.
// Probabilities therefore stay below 2^8, well inside bf16 and fp32 range, and the final
// O / l is exact whichever max was used.
#include "arl2_device.cuh"
#include "arl2_kernels.h"

namespace arl2 {
namespace {

constexpr uint32_t kQOff = 0;
constexpr uint32_t kKOff = kTileBytes;          // two stages
constexpr uint32_t kVOff = 3 * kTileBytes;      // two stages
constexpr uint32_t kPOff = 5 * kTileBytes;      // two buffers
constexpr uint32_t kBarOff = 7 * kTileBytes;
enum : int {
  kBarQ = 0,
  kBarKFull = 1,    // +stage
  kBarVFull = 3,
  kBarKEmpty = 5,
  kBarVEmpty = 7,
  kBarSFull = 9,    // +S buffer
  kBarPFull = 11,   // +P buffer
  kBarPFree = 13,   // +P buffer: the P.V MMA that read it is done
  kBarQp = 15,      // Q' = Q Wq is in TMEM
  kBarQpReady = 16, // Q' bf16 is in shared memory
  kBarOFull = 17,
  kBarFinal = 18,
  kNumBars = 19
};
constexpr uint32_t kMiscOff = kBarOff + 256;
constexpr uint32_t kSmemBytes = kMiscOff + 16 + 1024;  // + slack for 1 KiB alignment
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColO = 256, kColOI = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Smem {
  uint32_t base;
  __device__ uint32_t bar(int i) const { return base + kBarOff + 8u * i; }
  __device__ uint32_t q() const { return base + kQOff; }
  __device__ uint32_t k(int s) const { return base + kKOff + s * kTileBytes; }
  __device__ uint32_t v(int s) const { return base + kVOff + s * kTileBytes; }
  __device__ uint32_t p(int s) const { return base + kPOff + s * kTileBytes; }
};

template <bool kHybrid>
__device__ void producer(const Smem& sm, const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                         const CUtensorMap* tm_w, const CUtensorMap* tm_s, const QueryArgs& a, int q0, int h, int b,
                         int nkv, const Guard& g) {
  uint32_t nk[2] = {0, 0}, nv[2] = {0, 0};
  mbar_expect_tx(sm.bar(kBarQ), (kHybrid ? 3 : 1) * kTileBytes);
  for (int p = 0; p < 2; ++p) tma_load_4d(sm.q() + p * kPanelBytes, tm_q, sm.bar(kBarQ), 64 * p, h, q0, b);
  if (kHybrid) {
    const int slot = a.state_slot * a.B * a.H + b * a.H + h;
    for (int p = 0; p < 2; ++p) {
      tma_load_3d(sm.p(0) + p * kPanelBytes, tm_w, sm.bar(kBarQ), 64 * p, 0, h);
      tma_load_3d(sm.p(1) + p * kPanelBytes, tm_s, sm.bar(kBarQ), 64 * p, 0, slot);
    }
  }
  for (int j = 0; j < nkv; ++j) {
    const int s = j & 1;
    if (j >= 2 && !mbar_wait(sm.bar(kBarKEmpty + s), ((j - 2) >> 1) & 1, g)) break;
    mbar_expect_tx(sm.bar(kBarKFull + s), kTileBytes);
    for (int p = 0; p < 2; ++p)
      tma_load_4d(sm.k(s) + p * kPanelBytes, tm_k, sm.bar(kBarKFull + s), 64 * p, h, j * kRows, b);
    ++nk[s];
    if (j >= 2 && !mbar_wait(sm.bar(kBarVEmpty + s), ((j - 2) >> 1) & 1, g)) break;
    mbar_expect_tx(sm.bar(kBarVFull + s), kTileBytes);
    for (int p = 0; p < 2; ++p)
      tma_load_4d(sm.v(s) + p * kPanelBytes, tm_v, sm.bar(kBarVFull + s), 64 * p, h, j * kRows, b);
    ++nv[s];
  }
  // Every load issued must land before the CTA may exit (matters only after an abort).
  mbar_wait_drain(sm.bar(kBarQ), 0);
  for (int s = 0; s < 2; ++s) {
    if (nk[s]) mbar_wait_drain(sm.bar(kBarKFull + s), (nk[s] - 1) & 1);
    if (nv[s]) mbar_wait_drain(sm.bar(kBarVFull + s), (nv[s] - 1) & 1);
  }
}

template <bool kHybrid>
__device__ void mma_issuer(const Smem& sm, uint32_t tmem, int nkv, const Guard& g) {
  constexpr uint32_t id_kk = idesc_bf16(128, 128, false, false);   // A, B K-major
  constexpr uint32_t id_kmn = idesc_bf16(128, 128, false, true);   // A K-major, B MN-major
  const uint32_t tO = tmem + kColO, tOI = tmem + kColOI;
  if (!mbar_wait(sm.bar(kBarQ), 0, g)) return;
  tc_fence_after();
  if (kHybrid) {
    // Q' = Q Wq_h (phi_q), then O_inter = Q' S_{N-1}.
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_bf16(tOI, desc_kmajor(sm.q(), s), desc_mnmajor(sm.p(0), s), id_kmn, s > 0);
    mma_commit(sm.bar(kBarQp));
    if (!mbar_wait(sm.bar(kBarQpReady), 0, g)) return;
    tc_fence_after();
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_bf16(tOI, desc_kmajor(sm.p(0), s), desc_mnmajor(sm.p(1), s), id_kmn, s > 0);
  }
  auto issue_qk = [&](int j) -> bool {
    const int st = j & 1;
    if (!mbar_wait(sm.bar(kBarKFull + st), (j >> 1) & 1, g)) return false;
    tc_fence_after();
    const uint32_t tS = tmem + kColS0 + 128u * st;
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_bf16(tS, desc_kmajor(sm.q(), s), desc_kmajor(sm.k(st), s), id_kk, s > 0);
    mma_commit(sm.bar(kBarKEmpty + st));
    mma_commit(sm.bar(kBarSFull + st));
    return true;
  };
  if (!issue_qk(0)) return;
  if (nkv > 1 && !issue_qk(1)) return;
  for (int j = 0; j < nkv; ++j) {
    const int st = j & 1;
    const uint32_t ph = (j >> 1) & 1;
    if (!mbar_wait(sm.bar(kBarPFull + st), ph, g)) return;
    if (!mbar_wait(sm.bar(kBarVFull + st), ph, g)) return;
    tc_fence_after();
#pragma unroll
    for (int s = 0; s < 8; ++s)
      mma_bf16(tO, desc_kmajor(sm.p(st), s), desc_mnmajor(sm.v(st), s), id_kmn, (j > 0 || s > 0) ? 1u : 0u);
    mma_commit(sm.bar(kBarPFree + st));
    mma_commit(sm.bar(kBarVEmpty + st));
    if (j + 2 < nkv && !issue_qk(j + 2)) return;
  }
  mma_commit(sm.bar(kBarOFull));
}

// Row r of a 128-column fp32 TMEM block -> bf16 row r of a swizzled shared tile.
__device__ __forceinline__ void tmem_row_to_smem_bf16(uint32_t taddr, uint32_t tile, uint32_t r) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t v[32];
    tmem_ld32(taddr + 32u * c, v);
    tmem_wait_ld();
    reg_fence(v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t* x = v + 8 * j;
      st_shared_v4(tile + swz_chunk(r, 4 * c + j), pack_bf16x2(__uint_as_float(x[0]), __uint_as_float(x[1])),
                   pack_bf16x2(__uint_as_float(x[2]), __uint_as_float(x[3])),
                   pack_bf16x2(__uint_as_float(x[4]), __uint_as_float(x[5])),
                   pack_bf16x2(__uint_as_float(x[6]), __uint_as_float(x[7])));
    }
  }
}

template <bool kHybrid>
__device__ void softmax_role(const Smem& sm, uint32_t tmem, const QueryArgs& a, int q0, int h, int b, int nkv,
                             int warp, int lane, const Guard& g) {
  const int quarter = warp & 3;
  const uint32_t r = quarter * 32 + lane;                  // tile row == TMEM lane
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tO = tmem + lane_off + kColO;
  const uint32_t tOI = tmem + lane_off + kColOI;

  if (kHybrid) {
    if (!mbar_wait_warp(sm.bar(kBarQp), 0, g)) return;
    tc_fence_after();
    tmem_row_to_smem_bf16(tOI, sm.p(0), r);
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(sm.bar(kBarQpReady));
  }

  float m = -INFINITY, l = 0.f;
  for (int j = 0; j < nkv; ++j) {
    const int st = j & 1;
    if (!mbar_wait_warp(sm.bar(kBarSFull + st), (j >> 1) & 1, g)) return;
    tc_fence_after();
    uint32_t sv[4][32];
    const uint32_t tS = tmem + lane_off + kColS0 + 128u * st;
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32u * c, sv[c]);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 4; ++c) reg_fence(sv[c]);

    const int valid = a.kv_len - j * kRows;   // >= 1
    float mt = -INFINITY;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float x = __uint_as_float(sv[c][i]) * a.scale_log2;
        if (valid < kRows && 32 * c + i >= valid) x = -INFINITY;
        sv[c][i] = __float_as_uint(x);
        mt = fmaxf(mt, x);
      }
    }
    float m_new = m;
    bool rescale = false;
    if (j == 0) {
      m_new = mt;
    } else if (mt > m + kRescaleThreshold) {
      m_new = mt;
      rescale = true;
    }
    if (__any_sync(0xffffffffu, rescale)) {
      // O holds the sum up to tile j-1: wait for that P.V MMA, then scale this row of O.
      if (!mbar_wait_warp(sm.bar(kBarPFree + ((j - 1) & 1)), ((j - 1) >> 1) & 1, g)) return;
      tc_fence_after();
      const float corr = rescale ? ex2_approx(m - m_new) : 1.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t ov[32];
        tmem_ld32(tO + 32u * c, ov);
        tmem_wait_ld();
        reg_fence(ov);
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * corr);
        tmem_st32(tO + 32u * c, ov);
      }
      tmem_wait_st();
      l *= corr;
    }
    m = m_new;
    // P buffer st was last read by the P.V MMA of tile j-2.
    if (j >= 2 && !mbar_wait_warp(sm.bar(kBarPFree + st), ((j - 2) >> 1) & 1, g)) return;
    const uint32_t tile = sm.p(st);
    float rowsum = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float p[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          p[e] = ex2_approx(__uint_as_float(sv[c][8 * q + e]) - m);
          rowsum += p[e];
        }
        st_shared_v4(tile + swz_chunk(r, 4 * c + q), pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]),
                     pack_bf16x2(p[4], p[5]), pack_bf16x2(p[6], p[7]));
      }
    }
    l += rowsum;
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(sm.bar(kBarPFull + st));
  }

  // Epilogue: O = O_acc / l (+ O_inter), bf16, rows < T only.
  if (!mbar_wait_warp(sm.bar(kBarOFull), 0, g)) return;
  tc_fence_after();
  const float inv_l = 1.f / l;
  const int t = q0 + static_cast<int>(r);
  for (int c = 0; 32 * c < a.d; ++c) {
    uint32_t ov[32], iv[32];
    tmem_ld32(tO + 32u * c, ov);
    if (kHybrid) tmem_ld32(tOI + 32u * c, iv);
    tmem_wait_ld();
    reg_fence(ov);
    if (kHybrid) reg_fence(iv);
    if (t < a.T) {
      uint4* dst = reinterpret_cast<uint4*>(a.o + ((static_cast<size_t>(b) * a.T + t) * a.H + h) * a.d + 32 * c);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float y[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          y[e] = __uint_as_float(ov[8 * q + e]) * inv_l;
          if (kHybrid) y[e] += __uint_as_float(iv[8 * q + e]);
        }
        dst[q] = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                            pack_bf16x2(y[6], y[7]));
      }
    }
  }
}

template <bool kHybrid>
__global__ void __launch_bounds__(192, 1)
    arl2_query_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_s, const QueryArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const Smem sm{base};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kMiscOff + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * kRows, h = blockIdx.y, b = blockIdx.z;
  const int nkv = (a.kv_len + kRows - 1) / kRows;
  const Guard g{abort_flag, a.err, a.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(sm.bar(kBarQ), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(sm.bar(kBarKFull + s), 1);
      mbar_init(sm.bar(kBarVFull + s), 1);
      mbar_init(sm.bar(kBarKEmpty + s), 1);
      mbar_init(sm.bar(kBarVEmpty + s), 1);
      mbar_init(sm.bar(kBarSFull + s), 1);
      mbar_init(sm.bar(kBarPFull + s), 128);
      mbar_init(sm.bar(kBarPFree + s), 1);
    }
    mbar_init(sm.bar(kBarQp), 1);
    mbar_init(sm.bar(kBarQpReady), 128);
    mbar_init(sm.bar(kBarOFull), 1);
    mbar_init(sm.bar(kBarFinal), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    if (kHybrid) {
      prefetch_tmap(&tm_w);
      prefetch_tmap(&tm_s);
    }
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) producer<kHybrid>(sm, &tm_q, &tm_k, &tm_v, &tm_w, &tm_s, a, q0, h, b, nkv, g);
  } else if (warp == 1) {
    if (lane == 0) {
      mma_issuer<kHybrid>(sm, tmem, nkv, g);
      mma_commit(sm.bar(kBarFinal));   // arrives once every MMA issued above has finished
    }
    __syncwarp();
  } else {
    softmax_role<kHybrid>(sm, tmem, a, q0, h, b, nkv, warp, lane, g);
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

}  // namespace

size_t query_smem_bytes() { return kSmemBytes; }

cudaError_t query_setup() {
  cudaError_t e = cudaFuncSetAttribute(arl2_query_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(arl2_query_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemBytes));
}

cudaError_t launch_query(bool hybrid, const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                         const CUtensorMap& tm_w, const CUtensorMap& tm_s, const QueryArgs& a, cudaStream_t stream) {
  const dim3 grid((a.T + kRows - 1) / kRows, a.H, a.B);
  if (hybrid)
    arl2_query_kernel<true><<<grid, 192, kSmemBytes, stream>>>(tm_q, tm_k, tm_v, tm_w, tm_s, a);
  else
    arl2_query_kernel<false><<<grid, 192, kSmemBytes, stream>>>(tm_q, tm_k, tm_v, tm_w, tm_s, a);
  return cudaGetLastError();
}

}  // namespace arl2
