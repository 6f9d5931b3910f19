// Query kernel of the ARL2 hybrid layer, and the growing-KV-cache baseline that shares it.
//
// For every 128-row query tile of every (batch, head) it computes ("Attend Locally,
// Remember Linearly", technical summary of arXiv 2605.16579, §2.1):
//     O = softmax(Q K^T / sqrt(d)) V  +  (Q Wq_h) S_{N-1}
// The intra-frame branch is unmasked inside the frame. The inter-frame branch reads the
// state of the previous frame and never writes it (§2.2, frame-level access). With
// kHybrid = false the kernel is the baseline the layer replaces (§1): softmax attention of
// the newest frame over every cached key, with no state branch.
//
// Work split (persistent, stream-K). The work is U = B*H*nq*nkv units, each one
// (query tile, key tile) pair, ordered key tile fastest. CTA c of P takes the units
// [c*U/P, (c+1)*U/P), so every SM gets the same number of tile pairs. A CTA's range falls
// into segments, each a key range of one query tile:
//   - A segment that covers a whole query tile writes O directly.
//   - Otherwise the CTA writes a partial record (O_acc, running max m and sum l) to scratch
//     and bumps the tile's counter. The segment holding key tile 0 also stores O_inter.
//   - The CTA that brings the counter to the segment count merges every record of that
//     tile in key order and writes O. It then resets the counter. The merge order is
//     fixed, so the result does not depend on which CTA merges it.
//
// Roles (192 threads, one CTA per SM):
//   warp 0     TMA producer. Per segment: the Q tile, plus Wq_h and the bf16 state copy when
//              the segment starts the tile. Then K/V tiles into two-stage rings, where K and
//              V stages are released separately.
//   warp 1     TMEM owner; lane 0 issues every tcgen05.mma and commit.
//   warps 2-5  softmax warpgroup: thread = query row = TMEM lane. These threads also pack
//              Q' to bf16 for the readout MMA, and write outputs and partial records.
// TMEM (512 columns):
//   - cols 0 and 128: the two S tiles, double-buffered. P (bf16, 64 columns) overwrites
//     its own S tile and feeds the P.V MMA straight from TMEM.
//   - col 256: O. At the start of a segment that starts a tile, it briefly holds Q' packed
//     to bf16 for the readout MMA.
//   - col 384: Q' (fp32), then O_inter.
// Shared memory: Q | K0 K1 | V0 V1 | Wq | S (32 KiB tiles).
//
// Online softmax: scores are kept in log2 units. The running max m is raised only when a
// tile's max exceeds it by more than 8 (a factor of 256), so O in TMEM is rescaled rarely.
// Probabilities stay below 2^8. A quarter of the exponentials run on the FMA pipe
// (exp2_poly) and the rest on the MUFU unit, which would otherwise pace the loop.
#include <algorithm>

#include "arl2_device.cuh"
#include "arl2_kernels.h"

namespace arl2 {
namespace {

constexpr uint32_t kQOff = 0;
constexpr uint32_t kKOff = kTileBytes;          // two stages
constexpr uint32_t kVOff = 3 * kTileBytes;      // two stages
constexpr uint32_t kWOff = 5 * kTileBytes;
constexpr uint32_t kSOff = 6 * kTileBytes;
constexpr uint32_t kBarOff = 7 * kTileBytes;
enum : int {
  kBarQFull = 0,     // Q (+ Wq, S) of a segment landed
  kBarQEmpty = 1,    // the segment's QK^T MMAs are done with Q
  kBarWSEmpty = 2,   // the readout MMAs are done with Wq, S
  kBarKFull = 3,     // +stage
  kBarVFull = 5,
  kBarKEmpty = 7,
  kBarVEmpty = 9,
  kBarSFull = 11,    // +S buffer
  kBarPFull = 13,    // +S buffer: P written over it (128 arrivals)
  kBarPVDone = 15,   // +S buffer: the P.V MMA that read it is done
  kBarQp = 17,       // Q' = Q Wq is in TMEM
  kBarQpReady = 18,  // Q' bf16 is packed in TMEM (128 arrivals)
  kBarOFull = 19,    // the segment's MMAs are all done
  kBarOEmpty = 20,   // the segment's O / O_inter were read (128 arrivals)
  kBarFinal = 21,
  kBarGroup = 22,    // bounded rendezvous of the softmax warpgroup (128 arrivals)
  kNumBars = 23
};
static_assert(kNumBars * 8 <= 256, "barriers must fit their shared-memory slot");
constexpr int kMaxSegs = 8;        // the host plan keeps segments per query tile at or below this

// Rendezvous of the 128 softmax threads with a bounded wait (no hang if a warp aborted).
__device__ __forceinline__ bool group_sync(uint32_t bar, uint32_t& phase, const Guard& g) {
  mbar_arrive(bar);
  const bool ok = mbar_wait(bar, phase & 1, g);
  ++phase;
  return __all_sync(0xffffffffu, ok);
}
constexpr uint32_t kMiscOff = kBarOff + 256;
constexpr uint32_t kSmemBytes = kMiscOff + 32 + 1024;  // + slack for 1 KiB alignment
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColO = 256, kColOI = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Smem {
  uint32_t base;
  __device__ uint32_t bar(int i) const { return base + kBarOff + 8u * i; }
  __device__ uint32_t q() const { return base + kQOff; }
  __device__ uint32_t k(int s) const { return base + kKOff + s * kTileBytes; }
  __device__ uint32_t v(int s) const { return base + kVOff + s * kTileBytes; }
  __device__ uint32_t w() const { return base + kWOff; }
  __device__ uint32_t s() const { return base + kSOff; }
};

// One segment of a CTA's unit range: key tiles [kb, ke) of query tile Q.
struct Seg {
  int Q, kb, ke;
  int b, h, qt;
  bool head, tail;
};

struct Sched {
  long long u, u1;
  int nq, nkv, H;
  __device__ Sched(const QueryArgs& a, int c) : nq(a.nq), nkv(a.nkv), H(a.H) {
    u = static_cast<long long>(c) * a.units / a.num_ctas;
    u1 = static_cast<long long>(c + 1) * a.units / a.num_ctas;
  }
  __device__ bool next(Seg& s) {
    if (u >= u1) return false;
    s.Q = static_cast<int>(u / nkv);
    s.kb = static_cast<int>(u % nkv);
    s.ke = static_cast<int>(min(static_cast<long long>(nkv), s.kb + (u1 - u)));
    u = static_cast<long long>(s.Q) * nkv + s.ke;
    const int bh = s.Q / nq;
    s.qt = s.Q % nq;
    s.b = bh / H;
    s.h = bh % H;
    s.head = s.kb == 0;
    s.tail = s.ke == nkv;
    return true;
  }
};

// The CTA whose unit range holds unit u.
__device__ __forceinline__ int owner(long long u, const QueryArgs& a) {
  return static_cast<int>(((u + 1) * a.num_ctas - 1) / a.units);
}

template <bool kHybrid>
__device__ void producer(const Smem& sm, const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                         const CUtensorMap* tm_w, const CUtensorMap* tm_s, const QueryArgs& a, const Guard& g) {
  uint32_t nk[2] = {0, 0}, nv[2] = {0, 0};
  uint32_t nseg = 0, nhead = 0, tile = 0;
  Sched sch(a, blockIdx.x);
  Seg sg;
  bool ok = true;
  while (ok && sch.next(sg)) {
    const bool rd = kHybrid && sg.head;
    if (nseg > 0 && !mbar_wait(sm.bar(kBarQEmpty), (nseg - 1) & 1, g)) break;
    if (rd && nhead > 0 && !mbar_wait(sm.bar(kBarWSEmpty), (nhead - 1) & 1, g)) break;
    mbar_expect_tx(sm.bar(kBarQFull), (rd ? 3 : 1) * kTileBytes);
    for (int p = 0; p < 2; ++p)
      tma_load_4d(sm.q() + p * kPanelBytes, tm_q, sm.bar(kBarQFull), 64 * p, sg.h, sg.qt * kRows, sg.b);
    if (rd) {
      const int slot = a.state_slot * a.B * a.H + sg.b * a.H + sg.h;
      for (int p = 0; p < 2; ++p) {
        tma_load_3d(sm.w() + p * kPanelBytes, tm_w, sm.bar(kBarQFull), 64 * p, 0, sg.h);
        tma_load_3d(sm.s() + p * kPanelBytes, tm_s, sm.bar(kBarQFull), 64 * p, 0, slot);
      }
      ++nhead;
    }
    ++nseg;
    for (int j = sg.kb; j < sg.ke; ++j, ++tile) {
      const int s = tile & 1;
      if (tile >= 2 && !mbar_wait(sm.bar(kBarKEmpty + s), ((tile - 2) >> 1) & 1, g)) {
        ok = false;
        break;
      }
      mbar_expect_tx(sm.bar(kBarKFull + s), kTileBytes);
      for (int p = 0; p < 2; ++p)
        tma_load_4d(sm.k(s) + p * kPanelBytes, tm_k, sm.bar(kBarKFull + s), 64 * p, sg.h, j * kRows, sg.b);
      ++nk[s];
      if (tile >= 2 && !mbar_wait(sm.bar(kBarVEmpty + s), ((tile - 2) >> 1) & 1, g)) {
        ok = false;
        break;
      }
      mbar_expect_tx(sm.bar(kBarVFull + s), kTileBytes);
      for (int p = 0; p < 2; ++p)
        tma_load_4d(sm.v(s) + p * kPanelBytes, tm_v, sm.bar(kBarVFull + s), 64 * p, sg.h, j * kRows, sg.b);
      ++nv[s];
    }
  }
  // Every load issued must land before the CTA may exit (matters only after an abort).
  if (nseg > 0) mbar_wait_drain(sm.bar(kBarQFull), (nseg - 1) & 1);
  for (int s = 0; s < 2; ++s) {
    if (nk[s]) mbar_wait_drain(sm.bar(kBarKFull + s), (nk[s] - 1) & 1);
    if (nv[s]) mbar_wait_drain(sm.bar(kBarVFull + s), (nv[s] - 1) & 1);
  }
}

template <bool kHybrid>
__device__ void mma_issuer(const Smem& sm, uint32_t tmem, const QueryArgs& a, const Guard& g) {
  constexpr uint32_t id_kk = idesc_bf16(128, 128, false, false);   // A, B K-major
  constexpr uint32_t id_kmn = idesc_bf16(128, 128, false, true);   // A K-major (smem or TMEM), B MN-major
  const uint32_t tO = tmem + kColO, tOI = tmem + kColOI;
  uint32_t nseg = 0, nhead = 0, tile = 0;
  Sched sch(a, blockIdx.x);
  Seg sg;
  auto issue_qk = [&](uint32_t t) -> bool {
    const int st = t & 1;
    if (!mbar_wait(sm.bar(kBarKFull + st), (t >> 1) & 1, g)) return false;
    tc_fence_after();
    const uint32_t tS = tmem + kColS0 + 128u * st;
#pragma unroll
    for (int s = 0; s < 8; ++s) mma_bf16(tS, desc_kmajor(sm.q(), s), desc_kmajor(sm.k(st), s), id_kk, s > 0);
    mma_commit(sm.bar(kBarKEmpty + st));
    mma_commit(sm.bar(kBarSFull + st));
    return true;
  };
  while (sch.next(sg)) {
    const bool rd = kHybrid && sg.head;
    const uint32_t t0 = tile, n = sg.ke - sg.kb;
    if (!mbar_wait(sm.bar(kBarQFull), nseg & 1, g)) return;
    tc_fence_after();
    // The first two score tiles only need free S buffers; they overlap the previous
    // segment's epilogue.
    if (!issue_qk(t0)) return;
    if (n > 1 && !issue_qk(t0 + 1)) return;
    // O and O_inter of the previous segment must have been read before they are rewritten.
    if (nseg > 0 && !mbar_wait(sm.bar(kBarOEmpty), (nseg - 1) & 1, g)) return;
    tc_fence_after();
    if (rd) {
      // Q' = Q Wq_h (phi_q) into the O_inter columns.
#pragma unroll
      for (int s = 0; s < 8; ++s) mma_bf16(tOI, desc_kmajor(sm.q(), s), desc_mnmajor(sm.w(), s), id_kmn, s > 0);
      mma_commit(sm.bar(kBarQp));
    }
    if (n <= 2) mma_commit(sm.bar(kBarQEmpty));
    if (rd) {
      // O_inter = Q' S_{N-1}, with Q' packed to bf16 in the O columns.
      if (!mbar_wait(sm.bar(kBarQpReady), nhead & 1, g)) return;
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < 8; ++s) mma_bf16_ts(tOI, tO + 8u * s, desc_mnmajor(sm.s(), s), id_kmn, s > 0);
      mma_commit(sm.bar(kBarWSEmpty));
      ++nhead;
    }
    for (uint32_t i = 0; i < n; ++i) {
      const uint32_t t = t0 + i;
      const int st = t & 1;
      const uint32_t ph = (t >> 1) & 1;
      if (!mbar_wait(sm.bar(kBarPFull + st), ph, g)) return;
      if (!mbar_wait(sm.bar(kBarVFull + st), ph, g)) return;
      tc_fence_after();
      const uint32_t tP = tmem + kColS0 + 128u * st;
#pragma unroll
      for (int s = 0; s < 8; ++s)
        mma_bf16_ts(tO, tP + 8u * s, desc_mnmajor(sm.v(st), s), id_kmn, (i > 0 || s > 0) ? 1u : 0u);
      mma_commit(sm.bar(kBarPVDone + st));
      mma_commit(sm.bar(kBarVEmpty + st));
      if (i + 2 < n) {
        if (!issue_qk(t + 2)) return;
        if (i + 3 == n) mma_commit(sm.bar(kBarQEmpty));
      }
    }
    mma_commit(sm.bar(kBarOFull));
    tile += n;
    ++nseg;
  }
}

// Softmax of one 128-key tile for this thread's row: scores sv (raw fp32) -> P (bf16) in
// TMEM over the same columns. Returns the row sum of P; m is the log2-unit max in use.
__device__ __forceinline__ float tile_probs(uint32_t (&sv)[4][32], float m, float scale_log2, uint32_t tP) {
  const float neg_m = -m;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  // Two halves of 64 score columns; each becomes 32 packed bf16 pairs stored to TMEM at
  // once, so only one half's packed words are live.
#pragma unroll
  for (int hlf = 0; hlf < 2; ++hlf) {
    uint32_t pk[32];   // pk[w]: score columns 64*hlf + 2w, 64*hlf + 2w + 1
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int c = 2 * hlf + cc;
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        float p2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int col = i + e;
          const float x = fmaf(__uint_as_float(sv[c][col]), scale_log2, neg_m);
          // Every fourth column on the FMA pipe, the rest on MUFU.
          p2[e] = ((col & 3) == 3) ? exp2_poly(x) : ex2_approx(x);
          acc[col & 7] += p2[e];
        }
        pk[16 * cc + (i >> 1)] = pack_bf16x2(p2[0], p2[1]);
      }
    }
    tmem_st32(tP + 32u * hlf, pk);
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += acc[i];
  return s;
}

template <bool kHybrid>
__device__ void softmax_role(const Smem& sm, uint32_t tmem, const QueryArgs& a, int warp, int lane,
                             volatile int* bcast, const Guard& g) {
  const int quarter = warp & 3;
  const uint32_t r = quarter * 32 + lane;                  // tile row == TMEM lane
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tO = tmem + lane_off + kColO;
  const uint32_t tOI = tmem + lane_off + kColOI;
  const int d = a.d;
  uint32_t nseg = 0, nhead = 0, tile = 0, gphase = 0;
  Sched sch(a, blockIdx.x);
  Seg sg;
  while (sch.next(sg)) {
    const bool rd = kHybrid && sg.head;
    const uint32_t t0 = tile, n = sg.ke - sg.kb;
    if (rd) {
      // Q' (fp32, O_inter columns) -> bf16 pairs in the O columns, the readout MMA's A operand.
      if (!mbar_wait_warp(sm.bar(kBarQp), nhead & 1, g)) return;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t x[32], pk[16];
        tmem_ld32(tOI + 32u * c, x);
        tmem_wait_ld();
        reg_fence(x);
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(x[2 * i]), __uint_as_float(x[2 * i + 1]));
        tmem_st16(tO + 16u * c, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(sm.bar(kBarQpReady));
      ++nhead;
    }

    float m = -INFINITY, l = 0.f;
    for (uint32_t i = 0; i < n; ++i) {
      const uint32_t t = t0 + i;
      const int st = t & 1;
      if (!mbar_wait_warp(sm.bar(kBarSFull + st), (t >> 1) & 1, g)) return;
      tc_fence_after();
      uint32_t sv[4][32];
      const uint32_t tS = tmem + lane_off + kColS0 + 128u * st;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32u * c, sv[c]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(sv[c]);

      // Tile max of the raw scores (eight independent chains); keys >= kv_len are masked.
      const int valid = a.kv_len - (sg.kb + static_cast<int>(i)) * kRows;   // >= 1
      if (valid < kRows) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (32 * c + e >= valid) sv[c][e] = __float_as_uint(-INFINITY);
      }
      float mx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx[e] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) mx[e & 7] = fmaxf(mx[e & 7], __uint_as_float(sv[c][e]));
      const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                             fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * a.scale_log2;
      float m_new = m;
      bool rescale = false;
      if (i == 0) {
        m_new = mt;
      } else if (mt > m + kRescaleThreshold) {
        m_new = mt;
        rescale = true;
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // O holds the sum up to tile t-1: wait for that P.V MMA, then scale this row of O.
        if (!mbar_wait_warp(sm.bar(kBarPVDone + ((t - 1) & 1)), ((t - 1) >> 1) & 1, g)) return;
        tc_fence_after();
        const float corr = rescale ? ex2_approx(m - m_new) : 1.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[32];
          tmem_ld32(tO + 32u * c, ov);
          tmem_wait_ld();
          reg_fence(ov);
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * corr);
          tmem_st32(tO + 32u * c, ov);
        }
        l *= corr;
      }
      m = m_new;
      l += tile_probs(sv, m, a.scale_log2, tS);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(sm.bar(kBarPFull + st));
    }
    tile += n;

    // ---- end of segment: every MMA of it is done.
    if (!mbar_wait_warp(sm.bar(kBarOFull), nseg & 1, g)) return;
    tc_fence_after();
    const int t_row = sg.qt * kRows + static_cast<int>(r);
    const bool row_ok = t_row < a.T;
    uint16_t* out_row = a.o + ((static_cast<size_t>(sg.b) * a.T + t_row) * a.H + sg.h) * d;
    if (sg.head && sg.tail) {
      const float inv_l = 1.f / l;
      for (int c = 0; 16 * c < d; ++c) {
        uint32_t ov[16], iv[16];
        tmem_ld16(tO + 16u * c, ov);
        if (kHybrid) tmem_ld16(tOI + 16u * c, iv);
        tmem_wait_ld();
        reg_fence16(ov);
        if (kHybrid) reg_fence16(iv);
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(out_row + 16 * c);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
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
      tc_fence_before();
      mbar_arrive(sm.bar(kBarOEmpty));
    } else {
      // Partial record of this segment: O_acc, m, l (and O_inter if it holds key tile 0).
      const long long first = static_cast<long long>(sg.Q) * a.nkv;
      const int c_first = owner(first, a);
      const int nsegs = owner(first + a.nkv - 1, a) - c_first + 1;
      const int slot = sg.Q * a.max_segs + (static_cast<int>(blockIdx.x) - c_first);
      float* po = a.part_o + (static_cast<size_t>(slot) * kRows + r) * kDP;
      float* poi = a.part_oi + (static_cast<size_t>(sg.Q) * kRows + r) * kDP;
      for (int c = 0; 16 * c < d; ++c) {
        uint32_t ov[16], iv[16];
        tmem_ld16(tO + 16u * c, ov);
        if (kHybrid && sg.head) tmem_ld16(tOI + 16u * c, iv);
        tmem_wait_ld();
        reg_fence16(ov);
        if (kHybrid && sg.head) reg_fence16(iv);
        float4* d4 = reinterpret_cast<float4*>(po + 16 * c);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          d4[q] = make_float4(__uint_as_float(ov[4 * q]), __uint_as_float(ov[4 * q + 1]),
                              __uint_as_float(ov[4 * q + 2]), __uint_as_float(ov[4 * q + 3]));
        if (kHybrid && sg.head) {
          float4* i4 = reinterpret_cast<float4*>(poi + 16 * c);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            i4[q] = make_float4(__uint_as_float(iv[4 * q]), __uint_as_float(iv[4 * q + 1]),
                                __uint_as_float(iv[4 * q + 2]), __uint_as_float(iv[4 * q + 3]));
        }
      }
      a.part_ml[(static_cast<size_t>(slot) * 2) * kRows + r] = m;
      a.part_ml[(static_cast<size_t>(slot) * 2 + 1) * kRows + r] = l;
      // TMEM is read: the next segment's MMAs may reuse O and O_inter.
      tc_fence_before();
      mbar_arrive(sm.bar(kBarOEmpty));
      // Publish, then count this segment in; the CTA completing the count merges.
      __threadfence();
      if (!group_sync(sm.bar(kBarGroup), gphase, g)) return;
      if (r == 0) {
        const int prev = atomicAdd(a.cnt + sg.Q, 1);
        *bcast = (prev == nsegs - 1) ? 1 : 0;
      }
      if (!group_sync(sm.bar(kBarGroup), gphase, g)) return;
      if (*bcast) {
        __threadfence();
        float M = -INFINITY;
        for (int s = 0; s < nsegs; ++s)
          M = fmaxf(M, __ldcg(a.part_ml + (static_cast<size_t>(sg.Q * a.max_segs + s) * 2) * kRows + r));
        float L = 0.f, wgt[kMaxSegs];
        for (int s = 0; s < nsegs && s < kMaxSegs; ++s) {
          const size_t sl = static_cast<size_t>(sg.Q * a.max_segs + s);
          wgt[s] = ex2_approx(__ldcg(a.part_ml + (sl * 2) * kRows + r) - M);
          L += wgt[s] * __ldcg(a.part_ml + (sl * 2 + 1) * kRows + r);
        }
        const float inv_L = 1.f / L;
        for (int c = 0; 8 * c < d; ++c) {
          float y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) y[e] = 0.f;
          for (int s = 0; s < nsegs && s < kMaxSegs; ++s) {
            const float4* src = reinterpret_cast<const float4*>(
                a.part_o + (static_cast<size_t>(sg.Q * a.max_segs + s) * kRows + r) * kDP + 8 * c);
            const float4 u0 = __ldcg(src), u1 = __ldcg(src + 1);
            y[0] += wgt[s] * u0.x;
            y[1] += wgt[s] * u0.y;
            y[2] += wgt[s] * u0.z;
            y[3] += wgt[s] * u0.w;
            y[4] += wgt[s] * u1.x;
            y[5] += wgt[s] * u1.y;
            y[6] += wgt[s] * u1.z;
            y[7] += wgt[s] * u1.w;
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) y[e] *= inv_L;
          if (kHybrid) {
            const float4* src = reinterpret_cast<const float4*>(poi + 8 * c);
            const float4 u0 = __ldcg(src), u1 = __ldcg(src + 1);
            y[0] += u0.x;
            y[1] += u0.y;
            y[2] += u0.z;
            y[3] += u0.w;
            y[4] += u1.x;
            y[5] += u1.y;
            y[6] += u1.z;
            y[7] += u1.w;
          }
          if (row_ok)
            *reinterpret_cast<uint4*>(out_row + 8 * c) = make_uint4(
                pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]), pack_bf16x2(y[6], y[7]));
        }
        if (r == 0) a.cnt[sg.Q] = 0;   // ready for the next launch
      }
    }
    ++nseg;
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
  volatile int* bcast = reinterpret_cast<volatile int*>(gbase + kMiscOff + 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Guard g{abort_flag, a.err, a.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(sm.bar(kBarQFull), 1);
    mbar_init(sm.bar(kBarQEmpty), 1);
    mbar_init(sm.bar(kBarWSEmpty), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(sm.bar(kBarKFull + s), 1);
      mbar_init(sm.bar(kBarVFull + s), 1);
      mbar_init(sm.bar(kBarKEmpty + s), 1);
      mbar_init(sm.bar(kBarVEmpty + s), 1);
      mbar_init(sm.bar(kBarSFull + s), 1);
      mbar_init(sm.bar(kBarPFull + s), 128);
      mbar_init(sm.bar(kBarPVDone + s), 1);
    }
    mbar_init(sm.bar(kBarQp), 1);
    mbar_init(sm.bar(kBarQpReady), 128);
    mbar_init(sm.bar(kBarOFull), 1);
    mbar_init(sm.bar(kBarOEmpty), 128);
    mbar_init(sm.bar(kBarFinal), 1);
    mbar_init(sm.bar(kBarGroup), 128);
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
    if (lane == 0) producer<kHybrid>(sm, &tm_q, &tm_k, &tm_v, &tm_w, &tm_s, a, g);
  } else if (warp == 1) {
    if (lane == 0) {
      mma_issuer<kHybrid>(sm, tmem, a, g);
      mma_commit(sm.bar(kBarFinal));   // arrives once every MMA issued above has finished
    }
    __syncwarp();
  } else {
    softmax_role<kHybrid>(sm, tmem, a, warp, lane, bcast, g);
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

QueryPlan plan_query(int B, int H, int T, int kv_len, int num_sms) {
  QueryPlan p{};
  p.nq = (T + kRows - 1) / kRows;
  p.nkv = (kv_len + kRows - 1) / kRows;
  p.units = static_cast<long long>(B) * H * p.nq * p.nkv;
  p.qtiles = static_cast<long long>(B) * H * p.nq;
  long long ctas = std::max<long long>(1, std::min<long long>(num_sms, p.units));
  while (true) {
    // Largest number of CTAs sharing one query tile under this grid.
    int worst = 1;
    for (long long Q = 0; Q < p.qtiles; ++Q) {
      const long long first = Q * p.nkv, last = first + p.nkv - 1;
      const long long c0 = ((first + 1) * ctas - 1) / p.units;
      const long long c1 = ((last + 1) * ctas - 1) / p.units;
      worst = std::max<int>(worst, static_cast<int>(c1 - c0 + 1));
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

size_t query_scratch_floats(const QueryPlan& p) {
  const size_t slots = static_cast<size_t>(p.qtiles) * p.max_segs;
  return slots * kRows * kDP + slots * 2 * kRows + static_cast<size_t>(p.qtiles) * kRows * kDP;
}

cudaError_t launch_query(bool hybrid, const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                         const CUtensorMap& tm_w, const CUtensorMap& tm_s, const QueryArgs& a, cudaStream_t stream) {
  const dim3 grid(a.num_ctas);
  if (hybrid)
    arl2_query_kernel<true><<<grid, 192, kSmemBytes, stream>>>(tm_q, tm_k, tm_v, tm_w, tm_s, a);
  else
    arl2_query_kernel<false><<<grid, 192, kSmemBytes, stream>>>(tm_q, tm_k, tm_v, tm_w, tm_s, a);
  return cudaGetLastError();
}

}  // namespace arl2
