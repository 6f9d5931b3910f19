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
//   - Otherwise the CTA writes a partial record (O_acc, running max m, sum l) to scratch
//     and bumps the tile's counter.
//   - The CTA that brings the counter to the segment count merges every record of that
//     tile in key order and writes O. It then resets the counter. The merge order is
//     fixed, so the result does not depend on which CTA merges it.
//   - The segment holding key tile 0 computes the readout O_inter first and stores it
//     (fp32) in the tile's scratch record; whoever finishes the tile adds it.
// Scratch records are column-quad-major, so every scratch access of a warp is coalesced.
//
// Roles (384 threads, one CTA per SM):
//   warp 0      K producer: per segment the Q tile, then K tiles into a three-stage ring.
//               When a segment starts a tile, Wq_h first goes through the ring like a tile.
//   warp 1      TMEM owner; lane 0 issues every tcgen05.mma and commit.
//   warp 2      V producer: V tiles into a three-stage ring. When a segment starts a tile,
//               the bf16 state copy S_h goes first, through the ring.
//   warps 4-11  two softmax warpgroups. Thread = query row = TMEM lane; warps 4-7 own
//               score and output columns 0-63, warps 8-11 columns 64-127. A thread reads
//               and writes only its own half-row; warps w and w+4 (same rows, same SM
//               sub-partition) swap half-row maxima through shared memory each tile.
//               These threads also pack Q' for the readout MMA and write outputs and
//               partial records.
// TMEM (512 columns):
//   - cols 0, 128, 256: three S tiles. The score MMA of tile t+2 is queued right behind
//     the P.V MMA of tile t and writes the buffer last read two MMA groups earlier, so no
//     MMA group overwrites TMEM columns that the group just ahead of it still reads (that
//     stalls the tensor pipe). P (bf16) overwrites its own S tile, scores 0-63 packed into
//     columns 0-31 and scores 64-127 into columns 64-95, and feeds the P.V MMA straight
//     from TMEM.
//   - col 384: O. At the start of a segment that starts a tile, it first holds Q' (fp32,
//     then packed to bf16 for the readout MMA, whose result goes to a free S tile).
// Shared memory: Q | K0 K1 K2 | V0 V1 V2 (32 KiB tiles) from its 1 KiB-aligned base, then a
// small control block (mbarriers, flags, the row-sum exchange).
//
// Online softmax: scores are kept in log2 units. The running max m is raised only when a
// tile's max exceeds it by more than 8 (a factor of 256), so O in TMEM is rescaled rarely.
// Probabilities stay below 2^8. Three column pairs in eight take their exponentials on
// the FMA pipe (exp2_poly2) and the rest on the MUFU unit; scaling, sums and the
// polynomial use the paired fp32 instructions.
#include <algorithm>

#include "arl2_device.cuh"
#include "arl2_kernels.h"

namespace arl2 {
namespace {

constexpr int kStages = 3;      // K and V ring depth
constexpr int kSBufs = 3;       // score tiles in TMEM
constexpr int kThreads = 384;
constexpr int kSoftmaxThreads = 256;
enum : int {
  kBarQFull = 0,      // Q of a segment landed
  kBarQEmpty = 1,     // the segment's MMAs are done with Q
  kBarKFull = 2,      // +stage (3)
  kBarKEmpty = 5,
  kBarVFull = 8,
  kBarVEmpty = 11,
  kBarSFull = 14,     // +S buffer (3): scores of a tile are in TMEM
  kBarPFull = 17,     // +S buffer: P written over them (256 arrivals)
  kBarPVDone = 20,    // +S buffer: the P.V MMA that read P is done
  kBarQp = 23,        // Q' = Q Wq is in TMEM (O columns)
  kBarQpReady = 24,   // Q' is packed to bf16 (256 arrivals)
  kBarOIReady = 25,   // O_inter is in TMEM (a free S buffer)
  kBarOIFree = 26,    // O_inter was read out (256 arrivals)
  kBarOFull = 27,     // the segment's MMAs are all done
  kBarOEmpty = 28,    // the segment's O was read (256 arrivals)
  kBarFinal = 29,
  kBarGroup = 30,     // bounded rendezvous of the softmax threads (256 arrivals)
  kBarPair = 31,      // +row quarter (4): the two warps of those rows swapped half-row maxima
  kBarNever = 35,     // never signalled: target of the failure-detection test hook
  kNumBars = 36
};
// Tiles at the (1 KiB-aligned) base of dynamic shared memory, then the control block.
constexpr uint32_t kQOff = 0;
constexpr uint32_t kKOff = kTileBytes;
constexpr uint32_t kVOff = kKOff + kStages * kTileBytes;
constexpr uint32_t kTileRegion = kVOff + kStages * kTileBytes;
constexpr uint32_t kCtlBars = 0;
constexpr uint32_t kCtlMisc = 320;           // tmem slot, abort flag, merge flag
// [2 slots][2 halves][128] fp32: per-tile half-row maxima (slot = tile parity); slot 0
// also carries the end-of-segment row sums.
constexpr uint32_t kCtlX = 384;
constexpr uint32_t kCtlBytes = kCtlX + 2 * 2 * 128 * 4;
static_assert(kNumBars * 8 <= kCtlMisc, "barriers must fit their slot");
constexpr uint32_t kSmemBytes = kTileRegion + kCtlBytes;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kMaxSegs = 8;                // the host plan keeps segments per query tile at or below this

struct Smem {
  uint32_t ctl, tiles;
  __device__ uint32_t bar(int i) const { return ctl + kCtlBars + 8u * i; }
  __device__ uint32_t q() const { return tiles + kQOff; }
  __device__ uint32_t k(int s) const { return tiles + kKOff + s * kTileBytes; }
  __device__ uint32_t v(int s) const { return tiles + kVOff + s * kTileBytes; }
};

// Rendezvous of the 256 softmax threads with a bounded wait (no hang if a warp aborted).
__device__ __forceinline__ bool group_sync(uint32_t bar, uint32_t& phase, const Guard& g) {
  mbar_arrive(bar);
  const bool ok = mbar_wait(bar, phase & 1, g);
  ++phase;
  return __all_sync(0xffffffffu, ok);
}

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

// Ring slot g: stage g % 3, used for the (g / 3)-th time. S buffers cycle the same way.
__device__ __forceinline__ int ring_stage(uint32_t g) { return static_cast<int>(g % kStages); }
__device__ __forceinline__ uint32_t ring_phase(uint32_t g) { return (g / kStages) & 1; }
__device__ __forceinline__ int sbuf(uint32_t t) { return static_cast<int>(t % kSBufs); }
__device__ __forceinline__ uint32_t sphase(uint32_t t) { return (t / kSBufs) & 1; }

// K producer (kIsK) or V producer. Per segment: [the readout operand (Wq or S) when the
// segment starts a tile], then its key tiles, all through this producer's ring. The K
// producer also loads each segment's Q tile.
template <bool kHybrid, bool kIsK>
__device__ void producer(const Smem& sm, const CUtensorMap* tm_q, const CUtensorMap* tm_kv, const CUtensorMap* tm_rd,
                         const QueryArgs& a, const Guard& g, bool lead) {
  const int full0 = kIsK ? kBarKFull : kBarVFull, empty0 = kIsK ? kBarKEmpty : kBarVEmpty;
  uint32_t nissued[kStages] = {0, 0, 0};
  uint32_t nseg = 0, ring = 0;
  Sched sch(a, blockIdx.x);
  Seg sg;
  bool ok = true;
  auto slot_wait = [&](uint32_t gidx) -> bool {
    return gidx < kStages || mbar_wait_warp(sm.bar(empty0 + ring_stage(gidx)), ring_phase(gidx - kStages), g);
  };
  auto tile_addr = [&](int s) { return kIsK ? sm.k(s) : sm.v(s); };
  while (ok && sch.next(sg)) {
    if (kIsK) {
      if (nseg > 0 && !mbar_wait_warp(sm.bar(kBarQEmpty), (nseg - 1) & 1, g)) break;
      if (lead) {
        mbar_expect_tx(sm.bar(kBarQFull), kTileBytes);
        for (int p = 0; p < 2; ++p)
          tma_load_4d(sm.q() + p * kPanelBytes, tm_q, sm.bar(kBarQFull), 64 * p, sg.h, sg.qt * kRows, sg.b);
      }
    }
    ++nseg;
    if (kHybrid && sg.head) {
      if (!slot_wait(ring)) break;
      const int s = ring_stage(ring);
      const int c2 = kIsK ? sg.h : a.state_slot * a.B * a.H + sg.b * a.H + sg.h;
      if (lead) {
        mbar_expect_tx(sm.bar(full0 + s), kTileBytes);
        for (int p = 0; p < 2; ++p) tma_load_3d(tile_addr(s) + p * kPanelBytes, tm_rd, sm.bar(full0 + s), 64 * p, 0, c2);
      }
      ++nissued[s];
      ++ring;
    }
    for (int j = sg.kb; j < sg.ke; ++j, ++ring) {
      if (!slot_wait(ring)) {
        ok = false;
        break;
      }
      const int s = ring_stage(ring);
      if (lead) {
        mbar_expect_tx(sm.bar(full0 + s), kTileBytes);
        for (int p = 0; p < 2; ++p)
          tma_load_4d(tile_addr(s) + p * kPanelBytes, tm_kv, sm.bar(full0 + s), 64 * p, sg.h, j * kRows, sg.b);
      }
      ++nissued[s];
    }
  }
  // Every load issued must land before the CTA may exit (matters only after an abort).
  if (kIsK && nseg > 0) mbar_wait_drain(sm.bar(kBarQFull), (nseg - 1) & 1);
  for (int s = 0; s < kStages; ++s)
    if (nissued[s]) mbar_wait_drain(sm.bar(full0 + s), (nissued[s] - 1) & 1);
}



template <bool kHybrid>
__device__ void mma_issuer(const Smem& sm, uint32_t tmem, const QueryArgs& a, const Guard& g, bool lead) {
  constexpr uint32_t id_kk = idesc_bf16(128, 128, false, false);   // A, B K-major
  constexpr uint32_t id_kmn = idesc_bf16(128, 128, false, true);   // A K-major (smem or TMEM), B MN-major
  const uint32_t tO = tmem + kColO;
  const uint32_t kPacked[8] = {0, 8, 16, 24, 64, 72, 80, 88};   // see the TMEM layout above
  uint32_t nseg = 0, nhead = 0, tile = 0, ring = 0;
  Sched sch(a, blockIdx.x);
  Seg sg;
  // Score tile t (S buffer t % 3) from the K tile in ring slot r. The buffer's previous
  // tile (t - 3) was consumed by a P.V MMA issued earlier, so in-order execution keeps it.
  auto issue_qk = [&](uint32_t t, uint32_t r) -> bool {
    const int sb = sbuf(t), ks = ring_stage(r);
    if (!mbar_wait_warp(sm.bar(kBarKFull + ks), ring_phase(r), g)) return false;
    tc_fence_after();
    const uint32_t tS = tmem + 128u * sb;
    if (lead) {
      mma8_ss<false, false>(tS, desc_kmajor(sm.q(), 0), desc_kmajor(sm.k(ks), 0), id_kk, 0u);
      mma_commit(sm.bar(kBarKEmpty + ks));
      mma_commit(sm.bar(kBarSFull + sb));
    }
    return true;
  };
  while (sch.next(sg)) {
    const bool rd = kHybrid && sg.head;
    const uint32_t t0 = tile, n = sg.ke - sg.kb;
    const uint32_t r_rd = ring, r0 = ring + (rd ? 1 : 0);   // readout operands' slot, first key tile's slot
    // Score tiles issued before the P.V loop: two. Afterwards the scores of tile t + 2 are
    // issued right behind the P.V MMA of tile t: they go to the buffer whose P was read by
    // the P.V MMA before that one, so adjacent MMA groups never touch the same TMEM columns
    // (an MMA that overwrites columns the MMA just ahead of it still reads stalls the pipe).
    const uint32_t npre = min(n, 2u);
    if (!mbar_wait_warp(sm.bar(kBarQFull), nseg & 1, g)) return;
    tc_fence_after();
    for (uint32_t i = 0; i < npre; ++i)
      if (!issue_qk(t0 + i, r0 + i)) return;
    // O of the previous segment must have been read before it is rewritten.
    if (nseg > 0 && !mbar_wait_warp(sm.bar(kBarOEmpty), (nseg - 1) & 1, g)) return;
    tc_fence_after();
    if (rd) {
      // Q' = Q Wq_h (phi_q) into the O columns; Wq_h sits in K slot r_rd.
      const int ws = ring_stage(r_rd);
      if (!mbar_wait_warp(sm.bar(kBarKFull + ws), ring_phase(r_rd), g)) return;
      tc_fence_after();
      if (lead) {
        mma8_ss<false, true>(tO, desc_kmajor(sm.q(), 0), desc_mnmajor(sm.k(ws), 0), id_kmn, 0u);
        mma_commit(sm.bar(kBarKEmpty + ws));
        mma_commit(sm.bar(kBarQp));
      }
    }
    if (lead && n <= npre) mma_commit(sm.bar(kBarQEmpty));
    if (rd) {
      // O_inter = Q' S_{N-1}: Q' packed to bf16 in the O columns, S_h in V slot r_rd, the
      // result in the S buffer of tile t0 + 2 (free until that tile's scores are issued).
      const int ss = ring_stage(r_rd);
      if (!mbar_wait_warp(sm.bar(kBarQpReady), nhead & 1, g)) return;
      if (!mbar_wait_warp(sm.bar(kBarVFull + ss), ring_phase(r_rd), g)) return;
      tc_fence_after();
      const uint32_t tX = tmem + 128u * sbuf(t0 + 2);
      if (lead) {
        mma8_ts(tX, tO, kPacked, desc_mnmajor(sm.v(ss), 0), id_kmn, 0u);
        mma_commit(sm.bar(kBarVEmpty + ss));
        mma_commit(sm.bar(kBarOIReady));
      }
      // Whatever tile next scores into that buffer (this segment's or a later one's) must
      // wait for the read-out. It costs nothing here: the first P.V of the segment needs
      // the softmax threads, which read O_inter out first.
      if (!mbar_wait_warp(sm.bar(kBarOIFree), nhead & 1, g)) return;
      tc_fence_after();
      ++nhead;
    }
    const uint32_t nissued = npre;   // score tiles issued ahead of the P.V loop
    for (uint32_t i = 0; i < n; ++i) {
      const uint32_t t = t0 + i, r = r0 + i;
      const int sb = sbuf(t), vs = ring_stage(r);
      if (!mbar_wait_warp(sm.bar(kBarPFull + sb), sphase(t), g)) return;
      if (!mbar_wait_warp(sm.bar(kBarVFull + vs), ring_phase(r), g)) return;
      tc_fence_after();
      const uint32_t tP = tmem + 128u * sb;
      if (lead) {
        mma8_ts(tO, tP, kPacked, desc_mnmajor(sm.v(vs), 0), id_kmn, i > 0 ? 1u : 0u);
        mma_commit(sm.bar(kBarPVDone + sb));
        mma_commit(sm.bar(kBarVEmpty + vs));
      }
      if (i + nissued < n) {
        if (!issue_qk(t + nissued, r + nissued)) return;
        if (lead && i + nissued + 1 == n) mma_commit(sm.bar(kBarQEmpty));
      }
    }
    if (lead) mma_commit(sm.bar(kBarOFull));
    tile += n;
    ring = r0 + n;
    ++nseg;
  }
}

// Max of this half's 64 score columns (raw units), with keys at or beyond `valid` masked
// to -inf. Three-input maxima, four independent chains.
__device__ __forceinline__ float half_max(uint32_t (&sv)[2][32], int col0, int valid) {
  if (valid < col0 + 64) {
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (col0 + 32 * c + e >= valid) sv[c][e] = __float_as_uint(-INFINITY);
  }
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int e = 0; e < 32; e += 2)
      mx[(e >> 1) & 3] = fmax3(mx[(e >> 1) & 3], __uint_as_float(sv[c][e]), __uint_as_float(sv[c][e + 1]));
  return fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]);
}

// Column pairs (of every 8) whose exponentials run on the FMA pipe (exp2_poly2); the
// rest go to the MUFU unit. Three of eight balances the two units for d = 128.
constexpr uint32_t kPolyPairs = 0xA4u;   // pairs 2, 5, 7
__host__ __device__ constexpr bool poly_pair(int j) { return (kPolyPairs >> (j & 7)) & 1u; }

// P for 64 score columns (raw fp32 in sv; masked ones are -inf) as 32 packed bf16 pairs
// in pk. Returns their sum; m is the log2-unit max in use. Scaling and sums run on
// column pairs.
__device__ __forceinline__ float half_probs(const uint32_t (&sv)[2][32], float m, float scale_log2,
                                            uint32_t (&pk)[32]) {
  const float2 sc = make_float2(scale_log2, scale_log2), nm = make_float2(-m, -m);
  float2 acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 2; ++c) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[c][2 * j]), __uint_as_float(sv[c][2 * j + 1])), sc, nm);
      const float2 p = poly_pair(j) ? exp2_poly2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
      acc[j & 3] = __fadd2_rn(acc[j & 3], p);
      pk[16 * c + j] = pack_bf16x2(p.x, p.y);
    }
  }
  const float2 s = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
  return s.x + s.y;
}

// Scratch records are stored column-quad-major: float4 (record, quad q of 4 columns, row r)
// sits at ((record * 32 + q) * 128 + r), so a warp's 32 rows move 512 contiguous bytes.
__device__ __forceinline__ float4* quad_ptr(float* base, size_t record, int q, uint32_t r) {
  return reinterpret_cast<float4*>(base) + ((record * 32 + q) * kRows + r);
}

__device__ __forceinline__ uint4 pack8(const float (&y)[8]) {
  return make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                    pack_bf16x2(y[6], y[7]));
}

// End of a segment: write O (whole query tile), or this segment's partial record and,
// for the CTA completing the tile, the merge of all its records. O_inter (fp32 scratch,
// written by the segment that started the tile) is added by whoever finishes the tile.
// Loads are issued in batches of 16 quads so their latencies overlap. Kept out of line so
// its registers do not compete with the softmax loop. Returns false if a wait gave up.
template <bool kHybrid>
__device__ __noinline__ bool segment_epilogue(const Smem& sm, const QueryArgs& a, const Seg& sg, uint32_t r, int half,
                                              int c0, int ncols, uint32_t tO, float m, float l_row,
                                              uint32_t& gphase, volatile int* merge_flag, const Guard& g) {
  const int d = a.d;
  const int q0 = c0 / 4, nquads = ncols / 4;   // this half's column quads
  const int t_row = sg.qt * kRows + static_cast<int>(r);
  const bool row_ok = t_row < a.T;
  uint16_t* out_row = a.o + ((static_cast<size_t>(sg.b) * a.T + t_row) * a.H + sg.h) * d + c0;
  if (sg.head && sg.tail) {
    const float inv_l = 1.f / l_row;
    // Two passes of 8 column quads (32 columns): O_inter loads first, then O from TMEM.
#pragma unroll
    for (int hp = 0; hp < 2; ++hp) {
      if (32 * hp >= ncols) break;
      float4 oi[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        oi[q] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (kHybrid && 8 * hp + q < nquads) oi[q] = __ldcg(quad_ptr(a.part_oi, sg.Q, q0 + 8 * hp + q, r));
      }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * hp + cc;
        if (16 * c >= ncols) break;
        uint32_t ov[16];
        tmem_ld16(tO + c0 + 16u * c, ov);
        tmem_wait_ld();
        reg_fence16(ov);
        if (row_ok) {
#pragma unroll
          for (int h8 = 0; h8 < 2; ++h8) {
            const float4 i0 = oi[4 * cc + 2 * h8], i1 = oi[4 * cc + 2 * h8 + 1];
            const float y[8] = {__uint_as_float(ov[8 * h8]) * inv_l + i0.x,     __uint_as_float(ov[8 * h8 + 1]) * inv_l + i0.y,
                                __uint_as_float(ov[8 * h8 + 2]) * inv_l + i0.z, __uint_as_float(ov[8 * h8 + 3]) * inv_l + i0.w,
                                __uint_as_float(ov[8 * h8 + 4]) * inv_l + i1.x, __uint_as_float(ov[8 * h8 + 5]) * inv_l + i1.y,
                                __uint_as_float(ov[8 * h8 + 6]) * inv_l + i1.z, __uint_as_float(ov[8 * h8 + 7]) * inv_l + i1.w};
            reinterpret_cast<uint4*>(out_row + 16 * c)[h8] = pack8(y);
          }
        }
      }
    }
    tc_fence_before();
    mbar_arrive(sm.bar(kBarOEmpty));
    return true;
  }
  // Partial record of this segment: O_acc (coalesced quads), m, l.
  const long long first = static_cast<long long>(sg.Q) * a.nkv;
  const int c_first = owner(first, a);
  const int nsegs = owner(first + a.nkv - 1, a) - c_first + 1;
  const size_t slot0 = static_cast<size_t>(sg.Q) * a.max_segs;
  const size_t slot = slot0 + (static_cast<int>(blockIdx.x) - c_first);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    if (16 * c >= ncols) break;
    uint32_t ov[16];
    tmem_ld16(tO + c0 + 16u * c, ov);
    tmem_wait_ld();
    reg_fence16(ov);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      *quad_ptr(a.part_o, slot, q0 + 4 * c + q, r) =
          make_float4(__uint_as_float(ov[4 * q]), __uint_as_float(ov[4 * q + 1]), __uint_as_float(ov[4 * q + 2]),
                      __uint_as_float(ov[4 * q + 3]));
  }
  if (half == 0) {
    a.part_ml[(slot * 2) * kRows + r] = m;
    a.part_ml[(slot * 2 + 1) * kRows + r] = l_row;
  }
  // TMEM is read: the next segment's MMAs may reuse O.
  tc_fence_before();
  mbar_arrive(sm.bar(kBarOEmpty));
  // Publish, then count this segment in; the CTA completing the count merges.
  __threadfence();
  if (!group_sync(sm.bar(kBarGroup), gphase, g)) return false;
  if (half == 0 && r == 0) {
    const int prev = atomicAdd(a.cnt + sg.Q, 1);
    *merge_flag = (prev == nsegs - 1) ? 1 : 0;
  }
  if (!group_sync(sm.bar(kBarGroup), gphase, g)) return false;
  if (!*merge_flag) return true;
  __threadfence();
  float ms[kMaxSegs], ls[kMaxSegs];
  float M = -INFINITY;
#pragma unroll
  for (int s = 0; s < kMaxSegs; ++s) {
    if (s < nsegs) {
      ms[s] = __ldcg(a.part_ml + ((slot0 + s) * 2) * kRows + r);
      ls[s] = __ldcg(a.part_ml + ((slot0 + s) * 2 + 1) * kRows + r);
      M = fmaxf(M, ms[s]);
    }
  }
  float L = 0.f;
#pragma unroll
  for (int s = 0; s < kMaxSegs; ++s)
    if (s < nsegs) L += ex2_approx(ms[s] - M) * ls[s];
  const float inv_L = 1.f / L;
  // Two passes of 8 column quads; each pass issues one segment's 8 loads at a time.
#pragma unroll
  for (int hp = 0; hp < 2; ++hp) {
    if (32 * hp >= ncols) break;
    float4 acc[8], oi[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      oi[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (kHybrid && 8 * hp + q < nquads) oi[q] = __ldcg(quad_ptr(a.part_oi, sg.Q, q0 + 8 * hp + q, r));
    }
#pragma unroll
    for (int s = 0; s < kMaxSegs; ++s) {
      if (s < nsegs) {
        const float w = ex2_approx(ms[s] - M);
        float4 v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          v[q] = (8 * hp + q < nquads) ? __ldcg(quad_ptr(a.part_o, slot0 + s, q0 + 8 * hp + q, r))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          acc[q].x += w * v[q].x;
          acc[q].y += w * v[q].y;
          acc[q].z += w * v[q].z;
          acc[q].w += w * v[q].w;
        }
      }
    }
    if (row_ok) {
#pragma unroll
      for (int h8 = 0; h8 < 4; ++h8) {
        if (32 * hp + 8 * h8 >= ncols) break;
        const float4 a0 = acc[2 * h8], a1 = acc[2 * h8 + 1], i0 = oi[2 * h8], i1 = oi[2 * h8 + 1];
        const float y[8] = {a0.x * inv_L + i0.x, a0.y * inv_L + i0.y, a0.z * inv_L + i0.z, a0.w * inv_L + i0.w,
                            a1.x * inv_L + i1.x, a1.y * inv_L + i1.y, a1.z * inv_L + i1.z, a1.w * inv_L + i1.w};
        reinterpret_cast<uint4*>(out_row + 32 * hp)[h8] = pack8(y);
      }
    }
  }
  if (half == 0 && r == 0) a.cnt[sg.Q] = 0;   // ready for the next launch
  return true;
}

template <bool kHybrid>
__device__ void softmax_role(const Smem& sm, uint8_t* ctl, uint32_t tmem, const QueryArgs& a, int warp, int lane,
                             const Guard& g) {
  const int quarter = warp & 3;
  const int half = (warp - 4) >> 2;                         // 0: columns 0-63, 1: columns 64-127
  const uint32_t r = quarter * 32 + lane;                   // tile row == TMEM lane
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tO = tmem + lane_off + kColO;
  float* xch = reinterpret_cast<float*>(ctl + kCtlX);      // [2 slots][2 halves][128]
  volatile int* merge_flag = reinterpret_cast<volatile int*>(ctl + kCtlMisc + 8);
  const int d = a.d;
  const int c0 = 64 * half;                                 // first column of this thread's half
  const int oc = 64 - c0;                                   // first column of the other half
  const int ncols = max(0, min(64, d - c0));                // output columns of this half
  uint32_t nseg = 0, nhead = 0, tile = 0, gphase = 0;
  // Test hook: a wait that can only run out (the bounded-wait path, without a fault).
  if (a.stall && !mbar_wait_warp(sm.bar(kBarNever), 0, g)) return;
  Sched sch(a, blockIdx.x);
  Seg sg;
  while (sch.next(sg)) {
    const uint32_t t0 = tile, n = sg.ke - sg.kb;
    if (kHybrid && sg.head) {
      // Q' (fp32, O columns) -> bf16 pairs over this half's own O columns: the readout
      // MMA's A operand.
      if (!mbar_wait_warp(sm.bar(kBarQp), nhead & 1, g)) return;
      tc_fence_after();
      {
        uint32_t x0[32], x1[32], pk[32];
        tmem_ld32(tO + c0, x0);
        tmem_ld32(tO + c0 + 32, x1);
        tmem_wait_ld();
        reg_fence(x0);
        reg_fence(x1);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          pk[i] = pack_bf16x2(__uint_as_float(x0[2 * i]), __uint_as_float(x0[2 * i + 1]));
          pk[16 + i] = pack_bf16x2(__uint_as_float(x1[2 * i]), __uint_as_float(x1[2 * i + 1]));
        }
        tmem_st32(tO + c0, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(sm.bar(kBarQpReady));
      // O_inter (fp32, the S buffer of tile t0 + 2) -> this half's quads of the tile's
      // O_inter record in scratch.
      if (!mbar_wait_warp(sm.bar(kBarOIReady), nhead & 1, g)) return;
      tc_fence_after();
      {
        const uint32_t tX = tmem + lane_off + 128u * sbuf(t0 + 2);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (16 * c >= ncols) break;
          uint32_t x[16];
          tmem_ld16(tX + c0 + 16u * c, x);
          tmem_wait_ld();
          reg_fence16(x);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *quad_ptr(a.part_oi, sg.Q, c0 / 4 + 4 * c + q, r) =
                make_float4(__uint_as_float(x[4 * q]), __uint_as_float(x[4 * q + 1]), __uint_as_float(x[4 * q + 2]),
                            __uint_as_float(x[4 * q + 3]));
        }
      }
      tc_fence_before();
      mbar_arrive(sm.bar(kBarOIFree));
      ++nhead;
    }

    float m = -INFINITY, l = 0.f;
    for (uint32_t i = 0; i < n; ++i) {
      const uint32_t t = t0 + i;
      const int sb = sbuf(t);
      if (!mbar_wait_warp(sm.bar(kBarSFull + sb), sphase(t), g)) return;
      tc_fence_after();
      const uint32_t tS = tmem + lane_off + 128u * sb;
      const int valid = a.kv_len - (sg.kb + static_cast<int>(i)) * kRows;   // >= 1
      // This half's scores, then the row max: the two warps holding these rows (one per
      // half) swap their half-row maxima through shared memory, double-buffered by tile
      // parity. Each half reads and writes only its own columns.
      uint32_t sv[2][32];
      tmem_ld32(tS + c0, sv[0]);
      tmem_ld32(tS + c0 + 32, sv[1]);
      tmem_wait_ld();
      reg_fence(sv[0]);
      reg_fence(sv[1]);
      float* xm = xch + (t & 1) * 256;
      xm[half * 128 + r] = half_max(sv, c0, valid);
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.bar(kBarPair + quarter));
      if (!mbar_wait_warp(sm.bar(kBarPair + quarter), t & 1, g)) return;
      const float mt = fmaxf(xm[r], xm[128 + r]) * a.scale_log2;
      float m_new = m;
      bool rescale = false;
      if (i == 0) {
        m_new = mt;
      } else if (mt > m + kRescaleThreshold) {
        m_new = mt;
        rescale = true;
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // O holds the sum up to tile t-1: wait for that P.V MMA, then scale this half-row.
        if (!mbar_wait_warp(sm.bar(kBarPVDone + sbuf(t - 1)), sphase(t - 1), g)) return;
        tc_fence_after();
        const float corr = rescale ? ex2_approx(m - m_new) : 1.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t ov[32];
          tmem_ld32(tO + c0 + 32u * c, ov);
          tmem_wait_ld();
          reg_fence(ov);
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * corr);
          tmem_st32(tO + c0 + 32u * c, ov);
        }
        l *= corr;
      }
      m = m_new;
      uint32_t pk[32];
      l += half_probs(sv, m, a.scale_log2, pk);
      // P overwrites the first 32 of this half's score columns.
      tmem_st32(tS + c0, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(sm.bar(kBarPFull + sb));
    }
    tile += n;

    // ---- end of segment: every MMA of it is done; combine the two half-row sums.
    if (!mbar_wait_warp(sm.bar(kBarOFull), nseg & 1, g)) return;
    tc_fence_after();
    xch[half * 128 + r] = l;
    if (!group_sync(sm.bar(kBarGroup), gphase, g)) return;
    const float l_row = xch[r] + xch[128 + r];
    if (!group_sync(sm.bar(kBarGroup), gphase, g)) return;   // before anyone rewrites xch
    if (!segment_epilogue<kHybrid>(sm, a, sg, r, half, c0, ncols, tO, m, l_row, gphase, merge_flag, g)) return;
    ++nseg;
  }
}

template <bool kHybrid>
__global__ void __launch_bounds__(kThreads, 1)
    arl2_query_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_s, const QueryArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t tiles = smem_u32(smem_raw);
  if (tiles & 1023u) {   // the swizzled tiles need a 1 KiB-aligned base: report, do nothing
    if (threadIdx.x == 0) atomicOr(a.err, kErrLayoutBit);
    return;
  }
  const uint32_t ctl = tiles + kTileRegion;
  uint8_t* ctl_ptr = smem_raw + kTileRegion;
  const Smem sm{ctl, tiles};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl_ptr + kCtlMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl_ptr + kCtlMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Guard g{abort_flag, a.err, a.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(sm.bar(kBarQFull), 1);
    mbar_init(sm.bar(kBarQEmpty), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(sm.bar(kBarKFull + s), 1);
      mbar_init(sm.bar(kBarKEmpty + s), 1);
      mbar_init(sm.bar(kBarVFull + s), 1);
      mbar_init(sm.bar(kBarVEmpty + s), 1);
    }
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(sm.bar(kBarSFull + s), 1);
      mbar_init(sm.bar(kBarPFull + s), kSoftmaxThreads);
      mbar_init(sm.bar(kBarPVDone + s), 1);
    }
    mbar_init(sm.bar(kBarQp), 1);
    mbar_init(sm.bar(kBarQpReady), kSoftmaxThreads);
    mbar_init(sm.bar(kBarOIReady), 1);
    mbar_init(sm.bar(kBarOIFree), kSoftmaxThreads);
    mbar_init(sm.bar(kBarOFull), 1);
    mbar_init(sm.bar(kBarOEmpty), kSoftmaxThreads);
    mbar_init(sm.bar(kBarFinal), 1);
    mbar_init(sm.bar(kBarGroup), kSoftmaxThreads);
    for (int q = 0; q < 4; ++q) mbar_init(sm.bar(kBarPair + q), 2);   // one arrival per warp
    mbar_init(sm.bar(kBarNever), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    if (kHybrid) prefetch_tmap(&tm_w);
  }
  if (warp == 2 && lane == 0) {
    prefetch_tmap(&tm_v);
    if (kHybrid) prefetch_tmap(&tm_s);
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Producers and the MMA issuer run warp-wide (uniform control flow and waits); one
  // elected lane issues each TMA copy, MMA and commit.
  if (warp == 0) {
    producer<kHybrid, true>(sm, &tm_q, &tm_k, &tm_w, a, g, elect_one());
  } else if (warp == 1) {
    const bool lead = elect_one();
    mma_issuer<kHybrid>(sm, tmem, a, g, lead);
    if (lead) mma_commit(sm.bar(kBarFinal));   // arrives once every MMA issued above has finished
    __syncwarp();
  } else if (warp == 2) {
    producer<kHybrid, false>(sm, &tm_q, &tm_v, &tm_s, a, g, elect_one());
  } else if (warp >= 4) {
    softmax_role<kHybrid>(sm, ctl_ptr, tmem, a, warp, lane, g);
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
    arl2_query_kernel<true><<<grid, kThreads, kSmemBytes, stream>>>(tm_q, tm_k, tm_v, tm_w, tm_s, a);
  else
    arl2_query_kernel<false><<<grid, kThreads, kSmemBytes, stream>>>(tm_q, tm_k, tm_v, tm_w, tm_s, a);
  return cudaGetLastError();
}

}  // namespace arl2
