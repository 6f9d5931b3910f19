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
// The first K projection starts as soon as W_k and the first K tile have landed; chunk i+1's
// K projection runs while the rows normalise chunk i (Kp is double-buffered).
//
// Reduction through L2. Every CTA writes its partial U (fp32, column-quad-major so that a
// warp's stores are contiguous) and its sum of alpha to a scratch slot of its own, then the
// cluster meets once at a barrier (release/acquire: the partials are visible after it). CTA
// g then owns a block of columns of S_N: it bulk-copies that block of every group's partial
// into shared memory, sums the G partials of each element in a fixed order (the result does
// not depend on timing), adds abar S_{N-1} and writes S_N in fp32 and bf16. The scratch is
// private to the launch's own clusters and is fully written before it is read, so it never
// needs clearing.
//
// Roles (192 threads): warp 0 TMA, warp 1 TMEM owner and MMA issuer (warp-wide loop, one
// elected lane issues), warps 2-5 row warps (thread = token row for K' and R, = state row k
// for writing U). Every thread takes part in the owner phase.
// TMEM: Kp of even chunks at 0, Vp at 128, U at 256, Kp of odd chunks at 384.
// Shared memory: Wk | Wv | S | K0 K1 | V0 V1 (32 KiB tiles), then a control block.
#include <algorithm>

#include "arl2_commit_rows.cuh"
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
constexpr uint32_t kCtlOff = 7 * kTileBytes;
enum : int {
  kBarWk = 0,         // Wk landed
  kBarWv = 1,         // Wv landed
  kBarS = 2,          // the bf16 copy of S_{N-1} landed
  kBarKFull = 3,      // +stage (2): K chunk tile landed
  kBarVFull = 5,      // +stage (2): V chunk tile landed
  kBarKVEmpty = 7,    // +stage (2): the chunk's last MMA (K'^T R) is done with its K and V tiles
  kBarProjK = 9,      // +Kp buffer (2): Kp of the chunk in TMEM
  kBarKn = 11,        // K' bf16 over the K tile (one arrival per row warp)
  kBarKS = 12,        // Vp - K'S in TMEM
  kBarR = 13,         // R bf16 over the V tile (one arrival per row warp)
  kBarU = 14,         // U complete
  kBarFinal = 15,     // every MMA done (drain before TMEM is freed)
  kBarOwn = 16,       // the owned columns of every group's partial landed in shared memory
  kNumBars = 17
};
constexpr uint32_t kCtlMisc = 192;           // tmem slot, abort flag, rows-failed flag, warp alpha sums
constexpr uint32_t kSmemBytes = kCtlOff + kCtlMisc + 64;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;   // room to align the base to 1 KiB
static_assert(kNumBars * 8 <= kCtlMisc, "barriers must fit their slot");
static_assert(kSmemAlloc <= 232448, "shared memory per CTA");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColKp0 = 0, kColVp = 128, kColU = 256, kColKp1 = 384;
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

// Warp 0 (warp-wide, lead lane issues). Order: Wk and the first K tile (the first MMA needs
// only these), Wv and the first V tile, the second chunk's tiles, then the bf16 S, then the
// remaining chunks through two stages. S_{N-1} is the previous commit's output; when this
// grid was launched as a programmatic dependent of the kernel before it, that output is
// visible only after griddepcontrol.wait, so the S load waits for it. The K and V tiles are
// this frame's activations, read once: they are loaded with an evict-first L2 policy.
__device__ void producer(const Smem& sm, const CUtensorMap* tm_k, const CUtensorMap* tm_v, const CUtensorMap* tm_wk,
                         const CUtensorMap* tm_wv, const CUtensorMap* tm_s, const CommitArgs& a, int c0, int nc,
                         int h, int b, bool lead, const Guard& g) {
  uint32_t nk[2] = {0, 0};
  const int slot = a.state_slot * a.B * a.H + b * a.H + h;
  const uint64_t stream_policy = l2_evict_first_policy();
  auto load_tile = [&](const CUtensorMap* map, uint32_t dst, int bar, int i) {
    if (lead) {
      mbar_expect_tx(sm.bar(bar), kTileBytes);
      for (int p = 0; p < 2; ++p)
        tma_load_4d_hint(dst + p * kPanelBytes, map, sm.bar(bar), 64 * p, h, (c0 + i) * kRows, b, stream_policy);
    }
  };
  auto load_weight = [&](const CUtensorMap* map, uint32_t dst, int bar, int c2) {
    if (lead) {
      mbar_expect_tx(sm.bar(bar), kTileBytes);
      for (int p = 0; p < 2; ++p) tma_load_3d(dst + p * kPanelBytes, map, sm.bar(bar), 64 * p, 0, c2);
    }
  };
  auto load_chunk = [&](int i) {
    load_tile(tm_k, sm.k(i & 1), kBarKFull + (i & 1), i);
    load_tile(tm_v, sm.v(i & 1), kBarVFull + (i & 1), i);
    ++nk[i & 1];
  };
  load_weight(tm_wk, sm.wk(), kBarWk, h);
  if (nc > 0) load_tile(tm_k, sm.k(0), kBarKFull, 0);
  load_weight(tm_wv, sm.wv(), kBarWv, h);
  if (nc > 0) {
    load_tile(tm_v, sm.v(0), kBarVFull, 0);
    ++nk[0];
  }
  if (nc > 1) load_chunk(1);
  griddep_wait();
  load_weight(tm_s, sm.s(), kBarS, slot);
  __syncwarp();
  for (int i = 2; i < nc; ++i) {
    if (!mbar_wait_warp(sm.bar(kBarKVEmpty + (i & 1)), ((i - 2) >> 1) & 1, g)) break;
    load_chunk(i);
  }
  // Every load issued must land before the CTA may exit (matters only after an abort).
  mbar_wait_drain(sm.bar(kBarWk), 0);
  mbar_wait_drain(sm.bar(kBarWv), 0);
  mbar_wait_drain(sm.bar(kBarS), 0);
  for (int s = 0; s < 2; ++s)
    if (nk[s]) {
      mbar_wait_drain(sm.bar(kBarKFull + s), (nk[s] - 1) & 1);
      mbar_wait_drain(sm.bar(kBarVFull + s), (nk[s] - 1) & 1);
    }
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
  auto chunk_ready = [&](int bar0, int i) { return mbar_wait_warp(sm.bar(bar0 + (i & 1)), (i >> 1) & 1, g); };
  if (nc > 0) {
    if (!mbar_wait_warp(sm.bar(kBarWk), 0, g) || !chunk_ready(kBarKFull, 0)) return;
    tc_fence_after();
    proj_k(0);
    if (!mbar_wait_warp(sm.bar(kBarWv), 0, g) || !chunk_ready(kBarVFull, 0)) return;
    tc_fence_after();
    proj_v(0);
  }
  for (int i = 0; i < nc; ++i) {
    const int st = i & 1;
    if (i + 1 < nc) {
      // The next chunk's K projection: its Kp buffer was read out (K' of chunk i-1) before
      // this warp issued chunk i-1's K'S.
      if (!chunk_ready(kBarKFull, i + 1)) return;
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
    if (i + 1 < nc) {
      if (!chunk_ready(kBarVFull, i + 1)) return;
      tc_fence_after();
      proj_v(i + 1);
    }
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
    commit_rows_normalise(tmem + lane_off + col_kp(i), sm.k(st), r);
    fence_proxy_async_smem();
    tc_fence_before();
    warp_arrive(sm.bar(kBarKn));
    // R = (Vp - K'S) * beta_t / T -> bf16, over the V tile (its MMA has finished).
    if (!mbar_wait_warp(sm.bar(kBarKS), i & 1, g)) return false;
    tc_fence_after();
    commit_rows_residual(tmem + lane_off + kColVp, sm.v(st), r, coef);
    fence_proxy_async_smem();
    tc_fence_before();
    warp_arrive(sm.bar(kBarR));
  }
  // This CTA's sum of alpha: warp shuffles here, the four warps in a fixed order later.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) asum += __shfl_xor_sync(0xffffffffu, asum, o);
  if (lane == 0) warp_sums[quarter] = asum;

  // U is complete (every MMA of this CTA is done).
  if (!mbar_wait_warp(sm.bar(kBarU), 0, g)) return false;
  tc_fence_after();
  return true;
}

// Scratch slot of (batch-head bh, group g): [32 column quads][128 rows] float4.
__device__ __forceinline__ float4* part_slot(float* part_u, size_t bh, int G, int g) {
  return reinterpret_cast<float4*>(part_u) + (bh * G + g) * (32 * kRows);
}

__global__ void __launch_bounds__(kThreadsC, 1)
    arl2_commit_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_wk, const __grid_constant__ CUtensorMap tm_wv,
                       const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CommitArgs a,
                       const __grid_constant__ ReduceArgs rd) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const Smem sm{base};
  uint8_t* ctl = gbase + kCtlOff;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + kCtlMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + kCtlMisc + 4);
  volatile int* rows_failed = reinterpret_cast<volatile int*>(ctl + kCtlMisc + 8);
  float* warp_sums = reinterpret_cast<float*>(ctl + kCtlMisc + 16);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int G = static_cast<int>(gridDim.x);   // CTAs of the cluster = chunk groups
  const int rank = static_cast<int>(cluster_rank());   // equals blockIdx.x: the cluster spans x
  const int nchunks = (a.T + kRows - 1) / kRows;
  const int c0 = rank * a.chunks_per_group;
  const int nc = max(0, min(a.chunks_per_group, nchunks - c0));
  const Guard g{abort_flag, a.err, a.timeout_ns};
  const size_t bh = static_cast<size_t>(b) * a.H + h;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(sm.bar(i), (i == kBarKn || i == kBarR) ? kRowWarps : 1);
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
  __syncwarp();   // the producer ends in per-lane drains: one arrival per warp at the barrier
  tc_fence_before();
  __syncthreads();
  const int d = rd.d;
  const bool ok_here = !*abort_flag && !*rows_failed;

  // This CTA's partial U and alpha sum into its scratch slot (a CTA with no chunk writes
  // zeros). A CTA that gave up wrote its error bit and skips the write; the state of that
  // call is then undefined.
  if (ok_here) {
    float4* slot = part_slot(rd.part_u, bh, G, rank);
    if (warp >= 2) {
      const uint32_t r = static_cast<uint32_t>(warp & 3) * 32 + lane;   // state row k == TMEM lane
      const uint32_t lane_off = static_cast<uint32_t>(warp & 3) * 32 << 16;
      tc_fence_after();
      for (int c = 0; c < 4; ++c) {
        if (32 * c >= d) break;
        uint32_t u[32];
        if (nc > 0) {
          tmem_ld32_wait(tmem + lane_off + kColU + 32u * c, u);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) u[e] = 0u;
        }
        if (static_cast<int>(r) < d) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            slot[(8 * c + q) * kRows + r] = make_float4(__uint_as_float(u[4 * q]), __uint_as_float(u[4 * q + 1]),
                                                       __uint_as_float(u[4 * q + 2]), __uint_as_float(u[4 * q + 3]));
        }
      }
    } else if (threadIdx.x == 0) {
      rd.part_alpha[bh * G + rank] = (warp_sums[0] + warp_sums[1]) + (warp_sums[2] + warp_sums[3]);
    }
  }
  // CTA `rank` owns column quads [q0, q1) of S_N, every row. Its columns of S_{N-1} go to L2
  // ahead of the barrier (no other CTA writes them): for each row, the 128-byte lines that
  // hold the first and last of its columns.
  const int quads = d / 4;
  const int qpo = (quads + G - 1) / G;   // column quads owned per CTA
  const int q0 = min(quads, rank * qpo), q1 = min(quads, q0 + qpo);
  const int nq_own = q1 - q0;
  const size_t dd = static_cast<size_t>(d) * d;
  if (ok_here && nq_own > 0) {
    for (int i = threadIdx.x; i < 2 * d; i += kThreadsC) {
      const int k = i >> 1, col = (i & 1) ? 4 * q1 - 1 : 4 * q0;
      prefetch_l2(rd.S_old + bh * dd + static_cast<size_t>(k) * d + col);
    }
  }
  // The partials were written through the generic proxy and are read below by bulk copies
  // (the async proxy); the cluster barrier's release/acquire makes them visible.
  fence_proxy_async_global();
  tc_fence_before();
  cluster_sync();   // every CTA's partial is written and visible
  if (warp == 1) {   // every TMEM read of this CTA happened before the barrier
    tc_fence_after();
    mbar_wait_drain(sm.bar(kBarFinal), 0);
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (!ok_here) return;

  // Owner phase. The G partial blocks of the owned columns (contiguous in the column-quad-
  // major slots: nq_own x 128 float4 each, one bulk copy per group; many small copies would
  // cost far more than these few large ones) come into shared memory over the chunk tiles
  // that are idle now, while each thread loads the S_{N-1} values and the alpha sums it
  // needs; then every item (row k, quad q; rows fastest) sums the G partials in a fixed
  // order, adds abar S_{N-1} and writes S_N in fp32 and bf16.
  const uint32_t own_bytes = static_cast<uint32_t>(nq_own) * kRows * 16;
  const uint32_t recv = sm.k(0);
  if (nq_own > 0 && warp == 0) {
    if (lane == 0) {
      fence_proxy_async_global();
      mbar_expect_tx(sm.bar(kBarOwn), own_bytes * G);
    }
    __syncwarp();
    for (int j = lane; j < G; j += 32)
      bulk_load(recv + j * own_bytes, part_slot(rd.part_u, bh, G, j) + static_cast<size_t>(q0) * kRows, own_bytes,
                sm.bar(kBarOwn));
  }
  float al[kMaxCluster];
#pragma unroll
  for (int j = 0; j < kMaxCluster; ++j) al[j] = j < G ? __ldcg(rd.part_alpha + bh * G + j) : 0.f;
  float asum = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxCluster; ++j) asum += al[j];
  const float abar = asum * rd.inv_T;
  const float* S_old = rd.S_old + bh * dd;
  float* S_new = rd.S_new + bh * dd;
  uint16_t* S_new_bf16 = rd.S_new_bf16 + bh * dd;
  const float4* own = reinterpret_cast<const float4*>(gbase + (recv - base));
  const int items = d * nq_own;
  constexpr int kBatch = 4;   // items a thread loads S_{N-1} for before it sums them
  bool landed = false;
#pragma unroll 1
  for (int it0 = threadIdx.x; it0 < items; it0 += kBatch * kThreadsC) {
    float4 so[kBatch];
#pragma unroll
    for (int e = 0; e < kBatch; ++e) {
      const int it = it0 + e * kThreadsC;
      if (it < items)
        so[e] = *reinterpret_cast<const float4*>(S_old + static_cast<size_t>(it % d) * d + 4 * (q0 + it / d));
    }
    if (!landed) {
      if (!mbar_wait(sm.bar(kBarOwn), 0, g)) break;
      landed = true;
    }
#pragma unroll
    for (int e = 0; e < kBatch; ++e) {
      const int it = it0 + e * kThreadsC;
      if (it >= items) break;
      const int k = it % d, qo = it / d;
      float4 acc = make_float4(abar * so[e].x, abar * so[e].y, abar * so[e].z, abar * so[e].w);
#pragma unroll
      for (int j = 0; j < kMaxCluster; ++j) {
        if (j < G) {
          const float4 u = own[(j * nq_own + qo) * kRows + k];
          acc.x += u.x;
          acc.y += u.y;
          acc.z += u.z;
          acc.w += u.w;
        }
      }
      const size_t o = static_cast<size_t>(k) * d + 4 * (q0 + qo);
      *reinterpret_cast<float4*>(S_new + o) = acc;
      *reinterpret_cast<uint2*>(S_new_bf16 + o) = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
    }
  }
  // The copies must land before the CTA may exit (matters only after a time-out).
  if (nq_own > 0 && warp == 0) mbar_wait_drain(sm.bar(kBarOwn), 0);
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

size_t commit_scratch_floats(int B, int H, int ngroups) {
  const size_t slots = static_cast<size_t>(B) * H * ngroups;
  return slots * 32 * kRows * 4 + slots;   // partial U, then the alpha sums
}

cudaError_t commit_setup() {
  return cudaFuncSetAttribute(arl2_commit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemAlloc));
}

cudaError_t launch_commit(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_wk,
                          const CUtensorMap& tm_wv, const CUtensorMap& tm_s, const CommitArgs& a,
                          const ReduceArgs& r, cudaStream_t stream, bool dependent) {
  // One cluster of a.ngroups CTAs per (batch, head). As a programmatic dependent the kernel
  // may start while the preceding kernel (a query) still runs: it reads k, v and the gates,
  // which a query does not write, before griddepcontrol.wait, and S_{N-1} after it; it writes
  // only the other state buffer and its own scratch.
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
