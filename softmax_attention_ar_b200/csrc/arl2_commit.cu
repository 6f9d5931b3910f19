// Commit kernel of the ARL2 hybrid layer: the clean-pass gated-delta state update
// ("Attend Locally, Remember Linearly", technical summary of arXiv 2605.16579, §2.1 state
// update and §2.2 clean-pass update), read with an explicit transpose:
//     K' = rownorm(K Wk_h),  V' = V Wv_h,  abar = mean_t alpha_t
//     S_N = abar S_{N-1} + K'^T diag(beta / T) (V' - K' S_{N-1})
//
// One cluster of G CTAs per (batch, head); CTA g of the cluster takes a group of 128-token
// chunks and runs, per chunk, this chain on the tensor cores with TMEM accumulators:
//     Kp = K Wk, Vp = V Wv            (MMA)
//     K' = Kp / max(|Kp|, 1e-12)      (thread = token row; bf16 over the K tile in shared memory)
//     Vp -= K' S_{N-1}                (MMA with the B operand negated, S from its bf16 copy)
//     R  = Vp beta_t / T              (thread = token row; bf16 over the V tile)
//     U += K'^T R                     (MMA, both operands MN-major; accumulates over the chunks)
// Chunk i+1's K projection runs while the rows normalise chunk i (Kp is double-buffered).
// Then every CTA pushes each row of its U, and its sum of alpha, to the CTA of the cluster
// that owns that row of S_N (distributed shared memory), and each CTA sums its rows in a
// fixed order (the result does not depend on timing) and writes S_N in fp32 and bf16. One
// launch, no scratch in global memory.
//
// Roles (192 threads): warp 0 TMA, warp 1 TMEM owner and MMA issuer (warp-wide loop, one
// elected lane issues), warps 2-5 row warps (thread = token row for K' and R, = state row k
// for the U staging).
// TMEM: Kp of even chunks at 0, Vp at 128, U at 256, Kp of odd chunks at 384.
// Shared memory: Wk | Wv | S | K0 K1 | V0 V1 (32 KiB tiles), then a control block. After
// every MMA is done the Wk, Wv and S tiles hold the receive buffer of the reduction.
#include <algorithm>

#include "arl2_device.cuh"
#include "arl2_kernels.h"

namespace arl2 {
namespace {

constexpr int kThreadsC = 192;
constexpr int kMaxCluster = 8;             // CTAs per (batch, head); the host keeps ngroups at or below this
constexpr uint32_t kWkOff = 0;
constexpr uint32_t kWvOff = kTileBytes;
constexpr uint32_t kSOff = 2 * kTileBytes;
constexpr uint32_t kKOff = 3 * kTileBytes;   // two stages
constexpr uint32_t kVOff = 5 * kTileBytes;   // two stages
// Receive buffer of the cluster reduction, over Wk | Wv | S: [G][32 column quads][rows per
// CTA] float4, at most (128 + G - 1) * 512 bytes.
constexpr uint32_t kRecvOff = kWkOff;
constexpr uint32_t kCtlOff = 7 * kTileBytes;
enum : int {
  kBarW = 0,          // Wk, Wv landed
  kBarKVFull = 1,     // +stage (2)
  kBarKVEmpty = 3,    // +stage
  kBarProjK = 5,      // +Kp buffer (2): Kp of the chunk in TMEM
  kBarKn = 7,         // K' bf16 over the K tile (one arrival per row warp)
  kBarKS = 8,         // Vp - K'S in TMEM
  kBarR = 9,          // R bf16 over the V tile (one arrival per row warp)
  kBarU = 10,         // U complete
  kBarFinal = 11,     // every MMA done (drain before TMEM is freed)
  kBarS = 12,         // the bf16 copy of S_{N-1} landed
  kNumBars = 13
};
constexpr uint32_t kCtlMisc = 128;           // tmem slot, abort flag, alpha sums, status
constexpr uint32_t kSmemBytes = kCtlOff + kCtlMisc + 64;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;   // room to align the base to 1 KiB
static_assert(kNumBars * 8 <= kCtlMisc, "barriers must fit their slot");
static_assert(kSmemAlloc <= 232448, "shared memory per CTA");
static_assert(kRecvOff + (kDP + kMaxCluster - 1) * kDP * 4 <= kKOff, "the receive buffer must fit Wk, Wv and S");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColKp0 = 0, kColVp = 128, kColU = 256, kColKp1 = 384;
constexpr float kNormEps = 1e-12f;
constexpr int kRowWarps = 4;

struct Smem {
  uint32_t base;
  __device__ uint32_t bar(int i) const { return base + kCtlOff + 8u * i; }
  __device__ uint32_t wk() const { return base + kWkOff; }
  __device__ uint32_t wv() const { return base + kWvOff; }
  __device__ uint32_t s() const { return base + kSOff; }
  __device__ uint32_t k(int i) const { return base + kKOff + i * kTileBytes; }
  __device__ uint32_t v(int i) const { return base + kVOff + i * kTileBytes; }
};
__device__ __forceinline__ uint32_t col_kp(int i) { return (i & 1) ? kColKp1 : kColKp0; }

// Warp 0 (warp-wide, lead lane issues): Wk and Wv once, the first K and V chunk tiles, then
// the bf16 S once, then the remaining K and V chunk tiles through two stages. S_{N-1} is the
// previous commit's output; when this grid was launched as a programmatic dependent of the
// kernel before it, that output is visible only after griddepcontrol.wait, so S waits for
// it and goes out after the first chunk (the projections do not need S).
__device__ void producer(const Smem& sm, const CUtensorMap* tm_k, const CUtensorMap* tm_v, const CUtensorMap* tm_wk,
                         const CUtensorMap* tm_wv, const CUtensorMap* tm_s, const CommitArgs& a, int c0, int nc,
                         int h, int b, bool lead, const Guard& g) {
  uint32_t n[2] = {0, 0};
  const int slot = a.state_slot * a.B * a.H + b * a.H + h;
  if (lead) {
    mbar_expect_tx(sm.bar(kBarW), 2 * kTileBytes);
    for (int p = 0; p < 2; ++p) {
      tma_load_3d(sm.wk() + p * kPanelBytes, tm_wk, sm.bar(kBarW), 64 * p, 0, h);
      tma_load_3d(sm.wv() + p * kPanelBytes, tm_wv, sm.bar(kBarW), 64 * p, 0, h);
    }
  }
  auto load_s = [&]() {
    griddep_wait();
    if (lead) {
      mbar_expect_tx(sm.bar(kBarS), kTileBytes);
      for (int p = 0; p < 2; ++p) tma_load_3d(sm.s() + p * kPanelBytes, tm_s, sm.bar(kBarS), 64 * p, 0, slot);
    }
    __syncwarp();
  };
  if (nc == 0) load_s();
  for (int i = 0; i < nc; ++i) {
    const int s = i & 1;
    if (i >= 2 && !mbar_wait_warp(sm.bar(kBarKVEmpty + s), ((i - 2) >> 1) & 1, g)) break;
    const int row = (c0 + i) * kRows;
    if (lead) {
      mbar_expect_tx(sm.bar(kBarKVFull + s), 2 * kTileBytes);
      for (int p = 0; p < 2; ++p) {
        tma_load_4d(sm.k(s) + p * kPanelBytes, tm_k, sm.bar(kBarKVFull + s), 64 * p, h, row, b);
        tma_load_4d(sm.v(s) + p * kPanelBytes, tm_v, sm.bar(kBarKVFull + s), 64 * p, h, row, b);
      }
    }
    ++n[s];
    if (i == 0) load_s();
  }
  mbar_wait_drain(sm.bar(kBarW), 0);
  mbar_wait_drain(sm.bar(kBarS), 0);
  for (int s = 0; s < 2; ++s)
    if (n[s]) mbar_wait_drain(sm.bar(kBarKVFull + s), (n[s] - 1) & 1);
}

// Warp 1 (warp-wide, lead lane issues every MMA and commit).
__device__ void mma_issuer(const Smem& sm, uint32_t tmem, int nc, bool lead, const Guard& g) {
  constexpr uint32_t id_kmn = idesc_bf16(128, 128, false, true);            // A K-major, B MN-major
  constexpr uint32_t id_kmn_neg = idesc_bf16(128, 128, false, true, true);  // ... B negated
  constexpr uint32_t id_mnmn = idesc_bf16(128, 128, true, true);            // A MN-major, B MN-major
  auto proj_k = [&](int i) {   // Kp of chunk i from K stage i % 2
    if (lead) {
      mma8_ss<false, true>(tmem + col_kp(i), desc_kmajor(sm.k(i & 1), 0), desc_mnmajor(sm.wk(), 0), id_kmn, 0u);
      mma_commit(sm.bar(kBarProjK + (i & 1)));
    }
  };
  auto proj_v = [&](int i) {   // Vp of chunk i from V stage i % 2
    if (lead) mma8_ss<false, true>(tmem + kColVp, desc_kmajor(sm.v(i & 1), 0), desc_mnmajor(sm.wv(), 0), id_kmn, 0u);
  };
  if (nc > 0) {
    if (!mbar_wait_warp(sm.bar(kBarW), 0, g)) return;
    if (!mbar_wait_warp(sm.bar(kBarKVFull), 0, g)) return;
    tc_fence_after();
    proj_k(0);
    proj_v(0);
  }
  for (int i = 0; i < nc; ++i) {
    const int st = i & 1;
    if (i + 1 < nc) {
      // The next chunk's K projection: its Kp buffer was read out (K' of chunk i-1) before
      // this warp issued chunk i-1's K'S.
      if (!mbar_wait_warp(sm.bar(kBarKVFull + ((i + 1) & 1)), ((i + 1) >> 1) & 1, g)) return;
      tc_fence_after();
      proj_k(i + 1);
    }
    // Vp -= K'S: K' (bf16) over the K tile, S from its bf16 copy, B negated.
    if (i == 0 && !mbar_wait_warp(sm.bar(kBarS), 0, g)) return;
    if (!mbar_wait_warp(sm.bar(kBarKn), i & 1, g)) return;
    tc_fence_after();
    if (lead) {
      mma8_ss<false, true>(tmem + kColVp, desc_kmajor(sm.k(st), 0), desc_mnmajor(sm.s(), 0), id_kmn_neg, 1u);
      mma_commit(sm.bar(kBarKS));
    }
    // U += K'^T R, then the next chunk's V projection (Vp was read out into R).
    if (!mbar_wait_warp(sm.bar(kBarR), i & 1, g)) return;
    tc_fence_after();
    if (lead) {
      mma8_ss<true, true>(tmem + kColU, desc_mnmajor(sm.k(st), 0), desc_mnmajor(sm.v(st), 0), id_mnmn, i > 0 ? 1u : 0u);
      mma_commit(sm.bar(kBarKVEmpty + st));
    }
    if (i + 1 < nc) proj_v(i + 1);
  }
  if (lead) mma_commit(sm.bar(kBarU));
}

// Warps 2-5: K' and R per chunk (thread = token row), then wait for U. Returns false if a
// wait gave up.
__device__ bool row_role(const Smem& sm, uint32_t tmem, const CommitArgs& a, int c0, int nc, int h, int b, int warp,
                         int lane, float* warp_sums, const Guard& g) {
  const int quarter = warp & 3;
  const uint32_t r = quarter * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const size_t bh = static_cast<size_t>(b) * a.H + h;
  const float* alpha = a.alpha + bh * a.T;
  const float* beta = a.beta + bh * a.T;
  float asum = 0.f;
  // This row's gates, loaded one chunk ahead so that their latency hides behind the
  // previous chunk's work.
  auto gate_at = [&](int i, float& coef, float& al) {
    const int t = (c0 + i) * kRows + static_cast<int>(r);
    const bool valid = i < nc && t < a.T;
    coef = valid ? beta[t] * a.inv_T : 0.f;
    al = valid ? alpha[t] : 0.f;
  };
  float coef_next, alpha_next;
  gate_at(0, coef_next, alpha_next);
  for (int i = 0; i < nc; ++i) {
    const int st = i & 1;
    const float coef = coef_next;
    asum += alpha_next;
    gate_at(i + 1, coef_next, alpha_next);
    // K' = Kp / max(|Kp|, eps) -> bf16, over the K tile (its MMA has finished).
    if (!mbar_wait_warp(sm.bar(kBarProjK + st), (i >> 1) & 1, g)) return false;
    tc_fence_after();
    {
      uint32_t kv[4][32];
      tmem_ld32x2_wait(tmem + lane_off + col_kp(i), kv[0], tmem + lane_off + col_kp(i) + 32u, kv[1]);
      tmem_ld32x2_wait(tmem + lane_off + col_kp(i) + 64u, kv[2], tmem + lane_off + col_kp(i) + 96u, kv[3]);
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
    warp_arrive(sm.bar(kBarKn));
    // R = (Vp - K'S) * beta_t / T -> bf16, over the V tile (its MMA has finished).
    if (!mbar_wait_warp(sm.bar(kBarKS), i & 1, g)) return false;
    tc_fence_after();
    const uint32_t tile = sm.v(st);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t vp[32];
      tmem_ld32_wait(tmem + lane_off + kColVp + 32u * c, vp);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float y[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = __uint_as_float(vp[8 * q + e]) * coef;
        st_shared_v4(tile + swz_chunk(r, 4 * c + q), pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]),
                     pack_bf16x2(y[4], y[5]), pack_bf16x2(y[6], y[7]));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    warp_arrive(sm.bar(kBarR));
  }
  // This CTA's sum of alpha: warp shuffles here, the four warps in a fixed order later.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) asum += __shfl_xor_sync(0xffffffffu, asum, o);
  if (lane == 0) warp_sums[quarter] = asum;

  // U is complete (every MMA of this CTA is done); the tail pushes it to its owners.
  if (!mbar_wait_warp(sm.bar(kBarU), 0, g)) return false;
  tc_fence_after();
  return true;
}

__global__ void __launch_bounds__(kThreadsC, 1)
    arl2_commit_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_wk, const __grid_constant__ CUtensorMap tm_wv,
                       const __grid_constant__ CUtensorMap tm_s, const CommitArgs a, const ReduceArgs rd) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // Align the base to 1 KiB. The offset is the same in every CTA of the cluster (same
  // kernel, same dynamic shared memory), so a peer's staging sits at the same address.
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const Smem sm{base};
  uint8_t* ctl = gbase + kCtlOff;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + kCtlMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + kCtlMisc + 4);
  float* alpha_cta = reinterpret_cast<float*>(ctl + kCtlMisc + 8);
  volatile int* rows_failed = reinterpret_cast<volatile int*>(ctl + kCtlMisc + 12);
  float* warp_sums = reinterpret_cast<float*>(ctl + kCtlMisc + 16);
  float* recv_alpha = reinterpret_cast<float*>(ctl + kCtlMisc + 32);   // [G] alpha sums pushed by the CTAs
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int G = static_cast<int>(gridDim.x);   // CTAs of the cluster = chunk groups
  const uint32_t rank = cluster_rank();         // equals blockIdx.x: the cluster spans x
  const int nchunks = (a.T + kRows - 1) / kRows;
  const int c0 = static_cast<int>(rank) * a.chunks_per_group;
  const int nc = max(0, min(a.chunks_per_group, nchunks - c0));
  const Guard g{abort_flag, a.err, a.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(sm.bar(kBarW), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(sm.bar(kBarKVFull + s), 1);
      mbar_init(sm.bar(kBarKVEmpty + s), 1);
      mbar_init(sm.bar(kBarProjK + s), 1);
    }
    mbar_init(sm.bar(kBarKn), kRowWarps);
    mbar_init(sm.bar(kBarKS), 1);
    mbar_init(sm.bar(kBarR), kRowWarps);
    mbar_init(sm.bar(kBarU), 1);
    mbar_init(sm.bar(kBarFinal), 1);
    mbar_init(sm.bar(kBarS), 1);
    *abort_flag = 0;
    *rows_failed = 0;
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
    producer(sm, &tm_k, &tm_v, &tm_wk, &tm_wv, &tm_s, a, c0, nc, h, b, elect_one(), g);
  } else if (warp == 1) {
    const bool lead = elect_one();
    mma_issuer(sm, tmem, nc, lead, g);
    if (lead) mma_commit(sm.bar(kBarFinal));
    __syncwarp();
  } else {
    const bool ok = row_role(sm, tmem, a, c0, nc, h, b, warp, lane, warp_sums, g);
    if (!__all_sync(0xffffffffu, ok) && lane == 0) *rows_failed = 1;
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) *alpha_cta = (warp_sums[0] + warp_sums[1]) + (warp_sums[2] + warp_sums[3]);

  // ---- S_N from the whole cluster's U. The rows of S_N are split among the CTAs; every
  // CTA pushes each of its U rows to the CTA that owns it (remote stores into the owner's
  // receive buffer over its Wk/Wv/S tiles, free once that CTA's MMAs are done), then every
  // CTA sums its rows locally in a fixed order. Every thread of every CTA takes both cluster
  // barriers on every path, so no CTA can leave its peers waiting. A CTA that gave up wrote
  // its error bit; the state of that call is then undefined.
  const int d = rd.d;
  const int rows_per = (d + G - 1) / G;
  const bool ok_here = !*abort_flag && !*rows_failed;
  cluster_sync();   // 1: every CTA's MMAs are done (its receive buffer is free)
  if (ok_here) {
    if (warp >= 2) {
      const uint32_t r = static_cast<uint32_t>(warp & 3) * 32 + lane;
      const uint32_t lane_off = static_cast<uint32_t>(warp & 3) * 32 << 16;
      // Rows r < d only: then the owner r / rows_per is a rank of the cluster (< G).
      const bool row_ok = static_cast<int>(r) < d;
      const int owner = row_ok ? static_cast<int>(r) / rows_per : 0;
      const int lr = static_cast<int>(r) - owner * rows_per;
      // Receive layout [source rank][column quad][row of the owner]: a warp's consecutive
      // rows store to consecutive 16-byte slots of one owner.
      const uint32_t dst = row_ok ? peer_smem(sm.base + kRecvOff + (rank * 32u * rows_per + lr) * 16u, owner) : 0u;
      for (int c = 0; c < 4; ++c) {
        if (32 * c >= d) break;
        uint32_t u[32];
        if (nc > 0) {
          tmem_ld32_wait(tmem + lane_off + kColU + 32u * c, u);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) u[e] = 0u;
        }
        if (row_ok) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            st_cluster_v4(dst + (8u * c + q) * rows_per * 16u,
                          make_float4(__uint_as_float(u[4 * q]), __uint_as_float(u[4 * q + 1]),
                                      __uint_as_float(u[4 * q + 2]), __uint_as_float(u[4 * q + 3])));
        }
      }
    } else if (threadIdx.x < static_cast<unsigned>(G)) {
      // Threads 0..G-1: this CTA's alpha sum into slot `rank` of CTA threadIdx.x.
      st_cluster_f32(peer_smem(smem_u32(recv_alpha + rank), threadIdx.x), *alpha_cta);
    }
  }
  // This CTA's rows of S_{N-1} go to L2 ahead of the barrier (no other CTA writes them). The
  // reduction below is a plain rolled loop: it runs once per launch, and when its code is
  // not cached (the commit runs once per frame) a long unrolled body costs more in
  // instruction fetch than it saves.
  const int quads = d / 4;
  const int k0 = static_cast<int>(rank) * rows_per, k1 = min(d, k0 + rows_per);
  const int items = (k1 > k0 ? k1 - k0 : 0) * quads;
  const size_t bh = static_cast<size_t>(b) * a.H + h;
  const size_t dd = static_cast<size_t>(d) * d;
  if (ok_here) {
    const int lines = (d + 31) / 32;   // 128-byte lines per row
    for (int i = threadIdx.x; i < (k1 - k0) * lines; i += kThreadsC)
      prefetch_l2(rd.S_old + bh * dd + static_cast<size_t>(k0 + i / lines) * d + 32 * (i % lines));
  }
  cluster_sync();   // 2: every push has landed
  if (ok_here) {
    float asum = 0.f;
    for (int j = 0; j < G; ++j) asum += recv_alpha[j];
    const float abar = asum * rd.inv_T;
    const float* S_old = rd.S_old + bh * dd;
    float* S_new = rd.S_new + bh * dd;
    uint16_t* S_new_bf16 = rd.S_new_bf16 + bh * dd;
    const float4* recv = reinterpret_cast<const float4*>(gbase + kRecvOff);
    // Up to kBatch items a thread per pass, their S_{N-1} loads issued together so that one
    // L2 round trip covers them all (at 480p a single pass covers every item).
    constexpr int kBatch = 4;
#pragma unroll 1
    for (int it0 = threadIdx.x; it0 < items; it0 += kBatch * kThreadsC) {
      float4 so[kBatch];
#pragma unroll
      for (int e = 0; e < kBatch; ++e) {
        const int it = it0 + e * kThreadsC;
        if (it < items) {
          const int lr = it / quads, q = it % quads;
          so[e] = *reinterpret_cast<const float4*>(S_old + static_cast<size_t>(k0 + lr) * d + 4 * q);
        }
      }
#pragma unroll
      for (int e = 0; e < kBatch; ++e) {
        const int it = it0 + e * kThreadsC;
        if (it >= items) break;
        const int lr = it / quads, q = it % quads, k = k0 + lr;
        float4 acc = make_float4(abar * so[e].x, abar * so[e].y, abar * so[e].z, abar * so[e].w);
#pragma unroll 1
        for (int j = 0; j < G; ++j) {
          const float4 u = recv[(j * 32 + q) * rows_per + lr];
          acc.x += u.x;
          acc.y += u.y;
          acc.z += u.z;
          acc.w += u.w;
        }
        *reinterpret_cast<float4*>(S_new + static_cast<size_t>(k) * d + 4 * q) = acc;
        *reinterpret_cast<uint2*>(S_new_bf16 + static_cast<size_t>(k) * d + 4 * q) =
            make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
      }
    }
  }

  if (warp == 1) {
    tc_fence_after();
    mbar_wait_drain(sm.bar(kBarFinal), 0);
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

__global__ void arl2_state_import_kernel(const float* __restrict__ src, float* __restrict__ S,
                                         uint16_t* __restrict__ S_bf16, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float x = src[i];
    if (S) S[i] = x;
    __nv_bfloat16 y = __float2bfloat16_rn(x);
    S_bf16[i] = *reinterpret_cast<uint16_t*>(&y);
  }
}

}  // namespace

size_t commit_smem_bytes() { return kSmemAlloc; }

void commit_split(int T, int H, int B, int sms, int* chunks_per_group, int* ngroups) {
  const int nchunks = (T + kRows - 1) / kRows;
  const long long total = static_cast<long long>(nchunks) * H * B;
  int cpg = static_cast<int>(std::max<long long>(1, (total + sms - 1) / sms));   // about one CTA per SM
  cpg = std::max(cpg, (nchunks + kMaxCluster - 1) / kMaxCluster);                  // at most kMaxCluster groups
  cpg = std::min(cpg, nchunks);
  int ng = (nchunks + cpg - 1) / cpg;
  cpg = (nchunks + ng - 1) / ng;   // even out the groups
  ng = (nchunks + cpg - 1) / cpg;  // and leave none empty
  *chunks_per_group = cpg;
  *ngroups = ng;
}

cudaError_t commit_setup() {
  return cudaFuncSetAttribute(arl2_commit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemAlloc));
}

cudaError_t launch_commit(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_wk,
                          const CUtensorMap& tm_wv, const CUtensorMap& tm_s, const CommitArgs& a,
                          const ReduceArgs& r, cudaStream_t stream, bool dependent) {
  // One cluster of a.ngroups CTAs per (batch, head). As a programmatic dependent the kernel
  // may start while the preceding kernel (a query) still runs: it reads S_{N-1}, k, v and the
  // gates, none of which a query writes, and writes only the other state buffer.
  if (a.ngroups < 1 || a.ngroups > kMaxCluster) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(a.ngroups, a.H, a.B);
  cfg.blockDim = dim3(kThreadsC);
  cfg.dynamicSmemBytes = kSmemAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = a.ngroups;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, arl2_commit_kernel, tm_k, tm_v, tm_wk, tm_wv, tm_s, a, r);
}

cudaError_t launch_state_import(const float* src, float* S, uint16_t* S_bf16, size_t n, cudaStream_t stream) {
  const int blocks = static_cast<int>(std::min<size_t>((n + 255) / 256, 4096));
  arl2_state_import_kernel<<<blocks, 256, 0, stream>>>(src, S, S_bf16, n);
  return cudaGetLastError();
}

}  // namespace arl2
