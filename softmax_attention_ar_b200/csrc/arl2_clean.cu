// Fused clean pass of the ARL2 hybrid layer: the clean pass's query and the frame's commit in
// one launch ("Attend Locally, Remember Linearly", technical summary of arXiv 2605.16579,
// §2.2 clean-pass update: the last, clean forward pass of a frame reads S_{N-1} like every
// pass, and its K, V and gates then write S_N, once per frame).
//     O   = softmax(Q K^T / sqrt(d)) V + (Q Wq_h) S_{N-1}
//     S_N = abar S_{N-1} + K'^T diag(beta / T) (V' - K' S_{N-1}),  K' = rownorm(K Wk_h), V' = V Wv_h
//
// The grid holds two kinds of CTA, all resident at once (one per SM):
//   - CTAs [Pc, Pc + Pq) run the query kernel's persistent stream-K split over Pq CTAs,
//     unchanged (query_cta).
//   - CTAs [0, Pc) run the commit as a stream of chunk units. They come first, so that they
//     take the first SMs the kernel before them frees: each runs a longer serial chain than a
//     query CTA. The B*H*nchunks units
//     (128-token chunks, (batch, head)-major) are cut into Pc contiguous ranges of equal
//     length; a range falls into segments, one per (batch, head) it touches. A segment runs
//     the commit chain on the tensor cores, chunk after chunk, with U accumulating in TMEM:
//         Kp = K Wk, Vp = V Wv; K' = Kp / max(|Kp|, 1e-12); Vp -= K' S; R = Vp beta/T; U += K'^T R
//     A segment that covers every chunk of its head writes S_N = abar S_{N-1} + U straight
//     from TMEM. The segments of a head split between CTAs (a few: the ranges are long) each
//     write their partial U and alpha sum to a scratch slot of their own, then count
//     themselves in on the head's arrival counter (fence, then an atomic increment that
//     wraps at the head's segment count). The last to arrive sums the slots in segment
//     order, so the result does not depend on which one that is, and writes S_N. No commit
//     CTA ever waits for another CTA.
// Why two kinds of CTA rather than the commit inside the query CTAs: a query CTA holds all 512
// TMEM columns and nearly all of shared memory for its rings, and a chunk's chain (four
// 128x128x128 MMAs and two row passes) would stall its softmax pipeline. Both kinds run at
// the same time, so each K and V tile comes from DRAM once and is an L2 hit for the other
// kind. The host picks Pc from a cost model so that both kinds finish together.
//
// Commit CTA roles (the launch's 384 threads): warp 0 TMA, warp 1 TMEM owner and MMA issuer
// (warp-wide loop, one elected lane issues), warps 4-7 the row passes (thread = token row for
// K' and R), warps 8-11 the segments' epilogues (thread = state row). Warps 2 and 3 have no
// work.
// TMEM: Kp of even chunks at 0, Vp at 128, U at 256, Kp of odd chunks at 384.
// Shared memory (the query CTAs' allocation): Wk | Wv | S | K0 K1 | V0 V1 (32 KiB tiles) from
// the 1 KiB-aligned base, then a control block.
#include "arl2_commit_rows.cuh"
#include "arl2_query_body.cuh"

namespace arl2 {
namespace {

constexpr uint32_t kQuerySmemBytes = kSmemBytes;   // the launch's dynamic shared memory

namespace cs {

constexpr uint32_t kWkOff = 0;
constexpr uint32_t kWvOff = kTileBytes;
constexpr uint32_t kSOff = 2 * kTileBytes;
constexpr uint32_t kKOff = 3 * kTileBytes;   // two stages
constexpr uint32_t kVOff = 5 * kTileBytes;   // two stages
constexpr uint32_t kCtlOff = 7 * kTileBytes;
enum : int {
  kBarWk = 0,         // the segment's Wk_h landed (once per segment)
  kBarWv = 1,         // its Wv_h
  kBarS = 2,          // its bf16 copy of S_{N-1}
  kBarKFull = 3,      // +stage (2): K chunk tile landed
  kBarVFull = 5,      // +stage (2): V chunk tile landed
  kBarKVEmpty = 7,    // +stage (2): the chunk's last MMA (K'^T R) is done with its K and V tiles
  kBarProjK = 9,      // +Kp buffer (2): Kp of the chunk in TMEM
  kBarKn = 11,        // K' bf16 over the K tile (one arrival per row warp)
  kBarKS = 12,        // Vp - K'S in TMEM
  kBarR = 13,         // R bf16 over the V tile (one arrival per row warp)
  kBarU = 14,         // every MMA of the segment is done: U complete, its W, S and tiles free
  kBarUFree = 15,     // the segment's epilogue has read U out of TMEM (one arrival per epilogue warp)
  kBarFinal = 16,     // every MMA done and every row and epilogue warp finished with TMEM (before it is freed)
  kBarEpi = 17,       // rendezvous of the epilogue warps (one arrival per epilogue warp)
  kBarASum = 18,      // the segment's alpha sums are in shared memory (one arrival per row warp)
  kNumBars = 19
};
constexpr uint32_t kCtlMisc = 192;   // tmem slot, abort flag, last-arrival flag, row warps' alpha sums (2 x 4)
constexpr uint32_t kCtlBytes = kCtlMisc + 64;
static_assert(kNumBars * 8 <= kCtlMisc, "barriers must fit their slot");
static_assert(kCtlOff + kCtlBytes <= kQuerySmemBytes, "the commit CTAs fit the query CTAs' shared memory");
constexpr uint32_t kColKp0 = 0, kColVp = 128, kColU = 256, kColKp1 = 384;
constexpr int kFirstRowWarp = 4;   // warps 4-7: the chain's row passes
constexpr int kRowWarps = 4;
constexpr int kFirstEpiWarp = 8;   // warps 8-11: the segments' epilogues
constexpr int kEpiWarps = 4;

struct Smem {
  uint32_t base;
  __device__ uint32_t bar(int i) const { return base + kCtlOff + 8u * i; }
  __device__ uint32_t wk() const { return base + kWkOff; }
  __device__ uint32_t wv() const { return base + kWvOff; }
  __device__ uint32_t s() const { return base + kSOff; }
  __device__ uint32_t k(int i) const { return base + kKOff + i * kTileBytes; }
  __device__ uint32_t v(int i) const { return base + kVOff + i * kTileBytes; }
};
__device__ __forceinline__ uint32_t col_kp(int j) { return (j & 1) ? kColKp1 : kColKp0; }

// The commit CTA's range of chunk units and its walk over segments. 32-bit arithmetic: the
// host keeps units x commit CTAs below 2^31 (B*H <= 65535 heads of at most 32 chunks, at
// most a few hundred CTAs), so no 64-bit division runs on the device.
struct Walk {
  int u, u1;
  int nchunks;
  __device__ Walk(const CommitStreamArgs& a, int c)
      : u(c * static_cast<int>(a.units) / a.num_ctas),
        u1((c + 1) * static_cast<int>(a.units) / a.num_ctas),
        nchunks(a.nchunks) {}
  // The next segment: (batch, head) bh = b*H + h and its chunks [c0, c0 + nc).
  __device__ bool next(int& bh, int& c0, int& nc) {
    if (u >= u1) return false;
    bh = u / nchunks;
    c0 = u - bh * nchunks;
    const int end = min(u1, (bh + 1) * nchunks);
    nc = end - u;
    u = end;
    return true;
  }
};
// The commit CTA (0-based) whose range holds chunk unit x: the largest c with c*U/P <= x.
__device__ __forceinline__ int cta_of(int x, const CommitStreamArgs& a) {
  return ((x + 1) * a.num_ctas - 1) / static_cast<int>(a.units);
}

// Warp 0 (warp-wide, lead lane issues). Per segment: Wk, Wv and S of its head, and its chunk
// tiles through two stages. The first segment loads Wk and its first chunk before anything
// else (the first MMA needs only those) and S_{N-1} after griddepcontrol.wait (it is the output
// of the grid before this one when that is a commit). A later segment loads its first chunk,
// then waits until the previous segment's MMAs are done before it overwrites W and S.
__device__ void producer(const Smem& sm, const CUtensorMap* tm_k, const CUtensorMap* tm_v, const CUtensorMap* tm_wk,
                         const CUtensorMap* tm_wv, const CUtensorMap* tm_s, const CommitStreamArgs& a, int cta,
                         bool lead, const Guard& g) {
  const uint64_t stream_policy = l2_evict_first_policy();
  uint32_t nk[2] = {0, 0};
  int nseg = 0, gi = 0;
  int nw = 0;   // segments whose Wk, Wv and S loads were issued
  Walk w(a, cta);
  int bh, c0, nc;
  while (w.next(bh, c0, nc)) {
    const int b = bh / a.H, h = bh - b * a.H;
    auto load_chunk = [&](int i) -> bool {   // chunk i of the segment, CTA chunk gi + i
      const int j = gi + i, st = j & 1;
      if (j >= 2 && !mbar_wait_warp(sm.bar(kBarKVEmpty + st), ((j - 2) >> 1) & 1, g)) return false;
      if (lead) {
        mbar_expect_tx(sm.bar(kBarKFull + st), kTileBytes);
        for (int p = 0; p < 2; ++p)
          tma_load_4d_hint(sm.k(st) + p * kPanelBytes, tm_k, sm.bar(kBarKFull + st), 64 * p, h, (c0 + i) * kRows, b,
                           stream_policy);
        mbar_expect_tx(sm.bar(kBarVFull + st), kTileBytes);
        for (int p = 0; p < 2; ++p)
          tma_load_4d_hint(sm.v(st) + p * kPanelBytes, tm_v, sm.bar(kBarVFull + st), 64 * p, h, (c0 + i) * kRows, b,
                           stream_policy);
      }
      __syncwarp();
      ++nk[st];
      return true;
    };
    auto load_weight = [&](const CUtensorMap* map, uint32_t dst, int bar, int c2) {
      if (lead) {
        mbar_expect_tx(sm.bar(bar), kTileBytes);
        for (int p = 0; p < 2; ++p) tma_load_3d(dst + p * kPanelBytes, map, sm.bar(bar), 64 * p, 0, c2);
      }
      __syncwarp();
    };
    const int slot = a.state_slot * a.B * a.H + bh;
    bool ok = true;
    int rest = 1;
    if (nseg == 0) {
      load_weight(tm_wk, sm.wk(), kBarWk, h);
      ok = load_chunk(0);
      load_weight(tm_wv, sm.wv(), kBarWv, h);
      if (nc > 1) {
        ok = ok && load_chunk(1);
        rest = 2;
      }
      griddep_wait();
      load_weight(tm_s, sm.s(), kBarS, slot);
      ++nw;
    } else {
      ok = load_chunk(0) && mbar_wait_warp(sm.bar(kBarU), (nseg - 1) & 1, g);
      if (ok) {
        load_weight(tm_wk, sm.wk(), kBarWk, h);
        load_weight(tm_wv, sm.wv(), kBarWv, h);
        load_weight(tm_s, sm.s(), kBarS, slot);
        ++nw;
      }
    }
    for (int i = rest; ok && i < nc; ++i) ok = load_chunk(i);
    if (!ok) break;
    gi += nc;
    ++nseg;
  }
  // Every load issued must land before the CTA may exit (matters only after an abort).
  if (nw > 0) {
    mbar_wait_drain(sm.bar(kBarWk), (nw - 1) & 1);
    mbar_wait_drain(sm.bar(kBarWv), (nw - 1) & 1);
    mbar_wait_drain(sm.bar(kBarS), (nw - 1) & 1);
  }
  for (int s = 0; s < 2; ++s)
    if (nk[s]) {
      mbar_wait_drain(sm.bar(kBarKFull + s), (nk[s] - 1) & 1);
      mbar_wait_drain(sm.bar(kBarVFull + s), (nk[s] - 1) & 1);
    }
}

// Warp 1 (warp-wide, lead lane issues every MMA and commit). Per segment the chain of the
// commit kernel; the first U MMA of a segment (which overwrites U) waits until the previous
// segment's epilogue has read U.
__device__ void mma_issuer(const Smem& sm, uint32_t tmem, const CommitStreamArgs& a, int cta, bool lead,
                           const Guard& g) {
  constexpr uint32_t id_kmn = idesc_bf16(128, 128, false, true);            // A K-major, B MN-major
  constexpr uint32_t id_kmn_neg = idesc_bf16(128, 128, false, true, true);  // ... B negated
  constexpr uint32_t id_mnmn = idesc_bf16(128, 128, true, true);            // A MN-major, B MN-major
  auto proj_k = [&](int j) {   // Kp of CTA chunk j from K stage j % 2
    if (lead) {
      mma8_ss<false, true>(tmem + col_kp(j), desc_kmajor(sm.k(j & 1), 0), desc_mnmajor(sm.wk(), 0), id_kmn, 0u);
      mma_commit(sm.bar(kBarProjK + (j & 1)));
    }
  };
  auto proj_v = [&](int j) {   // Vp of CTA chunk j from V stage j % 2
    if (lead) mma8_ss<false, true>(tmem + kColVp, desc_kmajor(sm.v(j & 1), 0), desc_mnmajor(sm.wv(), 0), id_kmn, 0u);
  };
  auto chunk_ready = [&](int bar0, int j) { return mbar_wait_warp(sm.bar(bar0 + (j & 1)), (j >> 1) & 1, g); };
  int nseg = 0, gi = 0;
  Walk w(a, cta);
  int bh, c0, nc;
  while (w.next(bh, c0, nc)) {
    const uint32_t sp = nseg & 1;
    if (!mbar_wait_warp(sm.bar(kBarWk), sp, g) || !chunk_ready(kBarKFull, gi)) return;
    tc_fence_after();
    proj_k(gi);
    if (!mbar_wait_warp(sm.bar(kBarWv), sp, g) || !chunk_ready(kBarVFull, gi)) return;
    tc_fence_after();
    proj_v(gi);
    for (int i = 0; i < nc; ++i) {
      const int j = gi + i, st = j & 1;
      if (i + 1 < nc) {
        // The next chunk's K projection: its Kp buffer was read out (K' of chunk j-1) before
        // this warp issued chunk j-1's K'S.
        if (!chunk_ready(kBarKFull, j + 1)) return;
        tc_fence_after();
        proj_k(j + 1);
      }
      if (i == 0 && !mbar_wait_warp(sm.bar(kBarS), sp, g)) return;
      if (!mbar_wait_warp(sm.bar(kBarKn), j & 1, g)) return;
      tc_fence_after();
      if (lead) {
        mma8_ss<false, true>(tmem + kColVp, desc_kmajor(sm.k(st), 0), desc_mnmajor(sm.s(), 0), id_kmn_neg, 1u);
        mma_commit(sm.bar(kBarKS));
      }
      if (!mbar_wait_warp(sm.bar(kBarR), j & 1, g)) return;
      if (i == 0 && nseg > 0 && !mbar_wait_warp(sm.bar(kBarUFree), (nseg - 1) & 1, g)) return;
      tc_fence_after();
      if (lead) {
        mma8_ss<true, true>(tmem + kColU, desc_mnmajor(sm.k(st), 0), desc_mnmajor(sm.v(st), 0), id_mnmn,
                            i > 0 ? 1u : 0u);
        mma_commit(sm.bar(kBarKVEmpty + st));
      }
      if (i + 1 < nc) {
        if (!chunk_ready(kBarVFull, j + 1)) return;
        tc_fence_after();
        proj_v(j + 1);
      }
    }
    if (lead) mma_commit(sm.bar(kBarU));
    __syncwarp();
    gi += nc;
    ++nseg;
  }
}

// Rendezvous of the four epilogue warps through an mbarrier (release/acquire at CTA scope, so
// their shared-memory writes before it are visible after it), with a bounded wait. phase
// counts the rendezvous this warp took; every epilogue warp takes the same ones.
__device__ __forceinline__ bool epi_sync(const Smem& sm, uint32_t& phase, const Guard& g) {
  warp_arrive(sm.bar(kBarEpi));
  const bool ok = mbar_wait_warp(sm.bar(kBarEpi), phase & 1, g);
  ++phase;
  return ok;
}

// Scratch slot of segment `piece` of head bh: [32 column quads][128 rows] float4.
__device__ __forceinline__ float4* part_slot(const CommitStreamArgs& a, size_t bh, int piece) {
  return reinterpret_cast<float4*>(a.part_u) + (bh * a.max_pieces + piece) * (32 * kRows);
}

// Warps 4-7: per segment and chunk, K' and R (thread = token row), and the segment's alpha
// sum, which goes to shared memory (slot by segment parity) for the epilogue warps.
__device__ void row_role(const Smem& sm, uint32_t tmem, const CommitStreamArgs& a, int cta, int warp, int lane,
                         volatile float* warp_sums, const Guard& g) {
  const int quarter = warp & 3;
  const int r = quarter * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  int nseg = 0, gi = 0;
  Walk w(a, cta);
  int bh, c0, nc;
  while (w.next(bh, c0, nc)) {
    const float* alpha = a.alpha + static_cast<size_t>(bh) * a.T;
    const float* beta = a.beta + static_cast<size_t>(bh) * a.T;
    float asum = 0.f;
    auto gate_at = [&](int i, float& coef, float& al) {   // one chunk ahead, to hide the latency
      const int t = (c0 + i) * kRows + r;
      const bool valid = i < nc && t < a.T;
      coef = valid ? beta[t] * a.inv_T : 0.f;
      al = valid ? alpha[t] : 0.f;
    };
    float coef_next, alpha_next;
    gate_at(0, coef_next, alpha_next);
    for (int i = 0; i < nc; ++i) {
      const int j = gi + i, st = j & 1;
      const float coef = coef_next;
      asum += alpha_next;
      gate_at(i + 1, coef_next, alpha_next);
      if (!mbar_wait_warp(sm.bar(kBarProjK + st), (j >> 1) & 1, g)) return;
      tc_fence_after();
      commit_rows_normalise(tmem + lane_off + col_kp(j), sm.k(st), r);
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(sm.bar(kBarKn));
      if (!mbar_wait_warp(sm.bar(kBarKS), j & 1, g)) return;
      tc_fence_after();
      commit_rows_residual(tmem + lane_off + kColVp, sm.v(st), r, coef);
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(sm.bar(kBarR));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) asum += __shfl_xor_sync(0xffffffffu, asum, o);
    if (lane == 0) warp_sums[(nseg & 1) * 4 + quarter] = asum;
    warp_arrive(sm.bar(kBarASum));
    gi += nc;
    ++nseg;
  }
}

// Warps 8-11: per segment, once its U is complete (thread = state row r = TMEM lane), S_N of a
// whole head straight from TMEM, or a split head's partial, its arrival and, for the last
// arrival, the reduction. They have their own registers, so the loads of a row stay in flight
// together, and the row warps move on to the next segment meanwhile. Every epilogue warp takes
// every rendezvous and arrives on its head's counter for every split segment in its range,
// also after an abort, so that the counters stay in step with the launches.
__device__ void epilogue_role(const Smem& sm, uint32_t tmem, const CommitStreamArgs& a, int cta, int warp, int lane,
                              volatile int* last_flag, volatile float* warp_sums, const Guard& g) {
  const int quarter = warp & 3;
  const int r = quarter * 32 + lane;   // 0..127: warps 8-11 hold TMEM lane quarters 0-3
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  bool alive = true;
  uint32_t ephase = 0;
  // S_{N-1} is the previous grid's output, and the counters may be the previous grid's.
  griddep_wait();
  int nseg = 0;
  Walk w(a, cta);
  int bh, c0, nc;
  while (w.next(bh, c0, nc)) {
    const int first = bh * a.nchunks;
    const int cta_first = cta_of(first, a);
    const int npieces = cta_of(first + a.nchunks - 1, a) - cta_first + 1;
    alive = alive && mbar_wait_warp(sm.bar(kBarASum), nseg & 1, g);
    const float seg_alpha = (warp_sums[(nseg & 1) * 4 + 0] + warp_sums[(nseg & 1) * 4 + 1]) +
                            (warp_sums[(nseg & 1) * 4 + 2] + warp_sums[(nseg & 1) * 4 + 3]);
    const size_t row0 = bh * a.d * a.d + static_cast<size_t>(r) * a.d;
    const float4* s_old = reinterpret_cast<const float4*>(a.S_old + row0);
    float4* s_new = reinterpret_cast<float4*>(a.S_new + row0);
    uint2* s_new_bf16 = reinterpret_cast<uint2*>(a.S_new_bf16 + row0);
    // S_N columns [32 c, 32 c + 32) of row r from 8 float4 of S_{N-1} and of the update.
    auto write_block = [&](int c, float abar, const float4 (&so)[8], const float4 (&u)[8]) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 x = make_float4(fmaf(abar, so[q].x, u[q].x), fmaf(abar, so[q].y, u[q].y),
                                     fmaf(abar, so[q].z, u[q].z), fmaf(abar, so[q].w, u[q].w));
        s_new[8 * c + q] = x;
        s_new_bf16[8 * c + q] = make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
      }
    };
    float4 so[8];
    if (alive && npieces == 1 && r < a.d) {   // the first block of S_{N-1} loads while the MMAs finish
#pragma unroll
      for (int q = 0; q < 8; ++q) so[q] = __ldcg(s_old + q);
    }
    alive = alive && mbar_wait_warp(sm.bar(kBarU), nseg & 1, g);
    tc_fence_after();
    if (npieces == 1) {
      // The whole head: S_N = abar S_{N-1} + U from TMEM, the next block of S_{N-1} in flight
      // while one is written.
      if (alive) {
        const float abar = seg_alpha * a.inv_T;
        for (int c = 0; 32 * c < a.d; ++c) {
          uint32_t w32[32];
          tmem_ld32_wait(tmem + lane_off + kColU + 32u * c, w32);
          float4 u[8];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            u[q] = make_float4(__uint_as_float(w32[4 * q]), __uint_as_float(w32[4 * q + 1]),
                               __uint_as_float(w32[4 * q + 2]), __uint_as_float(w32[4 * q + 3]));
          if (r < a.d) {
            float4 nx[8];
            if (32 * (c + 1) < a.d) {
#pragma unroll
              for (int q = 0; q < 8; ++q) nx[q] = __ldcg(s_old + 8 * (c + 1) + q);
            }
            write_block(c, abar, so, u);
#pragma unroll
            for (int q = 0; q < 8; ++q) so[q] = nx[q];
          }
        }
      }
      tc_fence_before();
      warp_arrive(sm.bar(kBarUFree));
    } else {
      // A split head: this segment's partial to its slot, then the arrival count.
      const int piece = cta - cta_first;
      if (alive) {
        float4* slot = part_slot(a, bh, piece);
        for (int c = 0; 32 * c < a.d; ++c) {
          uint32_t w32[32];
          tmem_ld32_wait(tmem + lane_off + kColU + 32u * c, w32);
          if (r < a.d) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              slot[(8 * c + q) * kRows + r] = make_float4(__uint_as_float(w32[4 * q]), __uint_as_float(w32[4 * q + 1]),
                                                         __uint_as_float(w32[4 * q + 2]),
                                                         __uint_as_float(w32[4 * q + 3]));
          }
        }
        if (r == 0) a.part_alpha[static_cast<size_t>(bh) * a.max_pieces + piece] = seg_alpha;
      }
      tc_fence_before();
      warp_arrive(sm.bar(kBarUFree));
      __threadfence();   // this thread's partial is visible at GPU scope before the arrival
      alive = epi_sync(sm, ephase, g) && alive;
      if (r == 0) {
        const unsigned old = atomicInc(a.counters + bh, static_cast<unsigned>(npieces - 1));
        __threadfence();
        *last_flag = (old == static_cast<unsigned>(npieces - 1)) ? 1 : 0;
      }
      alive = epi_sync(sm, ephase, g) && alive;
      if (*last_flag && alive) {
        // The last arrival: S_N = abar S_{N-1} + the partials summed in segment order. Per
        // column block, the loads of S_{N-1} and of the first two partials are in flight
        // together.
        __threadfence();   // the other segments' partials are visible to this thread
        float asum_all = 0.f;
        for (int p = 0; p < npieces; ++p) asum_all += __ldcg(a.part_alpha + static_cast<size_t>(bh) * a.max_pieces + p);
        const float abar = asum_all * a.inv_T;
        const float4* parts = part_slot(a, bh, 0);
        if (r < a.d) {
#pragma unroll 1
          for (int c = 0; 32 * c < a.d; ++c) {
            float4 acc[8], x[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              so[q] = __ldcg(s_old + 8 * c + q);
              acc[q] = __ldcg(parts + (8 * c + q) * kRows + r);
              x[q] = __ldcg(parts + (32 + 8 * c + q) * kRows + r);   // npieces >= 2 here
            }
            for (int p = 1; p < npieces; ++p) {
              if (p > 1) {
#pragma unroll
                for (int q = 0; q < 8; ++q) x[q] = __ldcg(parts + (32 * p + 8 * c + q) * kRows + r);
              }
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                acc[q].x += x[q].x;
                acc[q].y += x[q].y;
                acc[q].z += x[q].z;
                acc[q].w += x[q].w;
              }
            }
            write_block(c, abar, so, acc);
          }
        }
      }
      alive = epi_sync(sm, ephase, g) && alive;   // the last-arrival flag is reused by the next segment
    }
    ++nseg;
  }
}

// One commit CTA of the fused clean pass.
__device__ __forceinline__ void commit_cta(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_wk,
                                           const CUtensorMap& tm_wv, const CUtensorMap& tm_s,
                                           const CommitStreamArgs& a, uint8_t* smem_raw) {
  const uint32_t base = smem_u32(smem_raw);
  if (base & 1023u) {   // the swizzled tiles need a 1 KiB-aligned base: report, do nothing
    if (threadIdx.x == 0) atomicOr(a.err, kErrLayoutBit);
    return;
  }
  const Smem sm{base};
  uint8_t* ctl = smem_raw + kCtlOff;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + kCtlMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + kCtlMisc + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(ctl + kCtlMisc + 8);
  volatile float* warp_sums = reinterpret_cast<volatile float*>(ctl + kCtlMisc + 16);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = static_cast<int>(blockIdx.x);
  const Guard g{abort_flag, a.err, a.timeout_ns};

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i)
      mbar_init(sm.bar(i), (i == kBarKn || i == kBarR || i == kBarASum) ? kRowWarps
                           : (i == kBarUFree || i == kBarEpi)              ? kEpiWarps
                           : i == kBarFinal                                ? 1 + kRowWarps + kEpiWarps
                                                                           : 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_wk);
    prefetch_tmap(&tm_wv);
    prefetch_tmap(&tm_s);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // No early trigger here: a kernel launched behind this one starts its CTAs once these have
  // exited. The commit CTAs run the longest serial chains of the launch; letting the next
  // query in early would give its last CTAs (in launch order) the SMs these CTAs hold only at
  // their end, and delay that whole query.

  if (warp == 0) {
    producer(sm, &tm_k, &tm_v, &tm_wk, &tm_wv, &tm_s, a, cta, elect_one(), g);
  } else if (warp == 1) {
    const bool lead = elect_one();
    mma_issuer(sm, tmem, a, cta, lead, g);
    if (lead) mma_commit(sm.bar(kBarFinal));   // arrives once every MMA issued above has finished
    __syncwarp();
  } else if (warp >= kFirstRowWarp && warp < kFirstRowWarp + kRowWarps) {
    row_role(sm, tmem, a, cta, warp, lane, warp_sums, g);
    tc_fence_before();
    warp_arrive(sm.bar(kBarFinal));   // this warp's TMEM accesses are done, however the role ended
  } else if (warp >= kFirstEpiWarp && warp < kFirstEpiWarp + kEpiWarps) {
    epilogue_role(sm, tmem, a, cta, warp, lane, last_flag, warp_sums, g);
    tc_fence_before();
    warp_arrive(sm.bar(kBarFinal));
  }
  __syncwarp();   // roles end in per-lane drains: one arrival per warp at the barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    mbar_wait_drain(sm.bar(kBarFinal), 0);
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace cs

__global__ void __launch_bounds__(kThreads, 1)
    arl2_clean_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_wq,
                      const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ CUtensorMap tm_o,
                      const __grid_constant__ CUtensorMap tm_wk, const __grid_constant__ CUtensorMap tm_wv,
                      const __grid_constant__ QueryArgs qa, const __grid_constant__ CommitStreamArgs ca) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (static_cast<int>(blockIdx.x) < ca.num_ctas)
    cs::commit_cta(tm_k, tm_v, tm_wk, tm_wv, tm_s, ca, smem_raw);
  else
    query_cta<true>(tm_q, tm_k, tm_v, tm_wq, tm_s, tm_o, qa, smem_raw);
}

// Cost model of the split, in microseconds of one CTA's work, fitted to B200 timings of the
// fused kernel and the standalone query at 480p and larger shapes: a query CTA spends about
// 1.24 us per (query tile, key tile) unit plus about 3 us per segment (epilogue, readout,
// merge) and 8 us of start-up and tail; a commit CTA about 5.5 us per 128-token chunk (its
// four-MMA chain with two row passes between, next to the query CTAs), 3 us per segment, 2 us
// for a split head's reduction and 4 us of start-up.
double query_cta_cost(long long units, int ctas) {
  const double per = static_cast<double>((units + ctas - 1) / ctas);
  return 8.0 + 1.24 * per + 3.0 * 2.0;
}
double commit_cta_cost(long long cunits, int nchunks, int ctas) {
  const long long per = (cunits + ctas - 1) / ctas;
  const long long segs = (per + nchunks - 1) / nchunks + 1;
  return 4.0 + 5.5 * static_cast<double>(per) + 3.0 * static_cast<double>(segs) + 2.0;
}

}  // namespace

CleanPlan plan_clean(int B, int H, int T, int num_sms, int commit_ctas) {
  CleanPlan p{};
  p.nchunks = (T + kRows - 1) / kRows;
  p.cunits = static_cast<long long>(B) * H * p.nchunks;
  const long long qunits = static_cast<long long>(B) * H * p.nchunks * p.nchunks;
  const int max_pc = static_cast<int>(std::max<long long>(1, std::min<long long>(num_sms - 1, p.cunits)));
  int pc = commit_ctas;
  if (pc <= 0) {
    double best = 0.0;
    for (int c = 1; c <= max_pc; ++c) {
      const double cost = std::max(query_cta_cost(qunits, num_sms - c), commit_cta_cost(p.cunits, p.nchunks, c));
      if (c == 1 || cost < best) {
        best = cost;
        pc = c;
      }
    }
  }
  pc = std::max(1, std::min(pc, max_pc));
  p.commit_ctas = pc;
  p.q = plan_query(B, H, T, T, std::max(1, num_sms - pc));
  // Segments per head, at most: the commit CTAs whose ranges hold its first and last chunk.
  auto cta_of = [&](long long x) { return static_cast<int>(((x + 1) * pc - 1) / p.cunits); };
  p.max_pieces = 1;
  for (long long bh = 0; bh < static_cast<long long>(B) * H; ++bh) {
    const long long first = bh * p.nchunks;
    p.max_pieces = std::max(p.max_pieces, cta_of(first + p.nchunks - 1) - cta_of(first) + 1);
  }
  return p;
}

size_t clean_scratch_floats(const CleanPlan& p) {
  const size_t slots = static_cast<size_t>(p.cunits / p.nchunks) * p.max_pieces;
  return slots * 32 * kRows * 4 + slots;
}

cudaError_t clean_setup() {
  return cudaFuncSetAttribute(arl2_clean_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kQuerySmemBytes));
}

cudaError_t launch_clean(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                         const CUtensorMap& tm_wq, const CUtensorMap& tm_s, const CUtensorMap& tm_o,
                         const CUtensorMap& tm_wk, const CUtensorMap& tm_wv, const QueryArgs& qa,
                         const CommitStreamArgs& ca, cudaStream_t stream, bool dependent) {
  if (qa.first_cta != ca.num_ctas || ca.num_ctas < 1 || ca.units < ca.num_ctas ||
      (ca.units + 1) * ca.num_ctas >= (1ll << 31))
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(qa.num_ctas + ca.num_ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kQuerySmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, arl2_clean_kernel, tm_q, tm_k, tm_v, tm_wq, tm_s, tm_o, tm_wk, tm_wv, qa, ca);
}

}  // namespace arl2
