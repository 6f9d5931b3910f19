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
//   - The segment holding key tile 0 of a query tile (its head) finishes the tile. With
//     contiguous ranges it is the last segment of its CTA, and the tile's other segments
//     open the ranges of the following CTAs, so they are normally done by then.
//   - Every other segment writes a partial record (O_acc, running max m, sum l) to
//     scratch; warp 3 then sets the record's flag to the launch's epoch (fence first).
//   - The head waits for those flags (bounded), merges the records with its own O in
//     TMEM in a fixed order and writes O. Epochs differ between launches, so no flag
//     is ever reset.
//   - The head segment also computes the readout O_inter, after its last P.V MMA, into a
//     free S tile in TMEM, and adds it when it writes O.
// Scratch records are column-quad-major, so every scratch access of a warp is coalesced.
//
// Roles (384 threads, one CTA per SM):
//   warp 0      producer: per segment the Q tile, then per key tile its K and V tiles,
//               each into a three-stage ring. When a segment starts a tile, Wq_h follows
//               its key tiles through the K ring and the bf16 state copy S_h through the V
//               ring.
//   warp 1      TMEM owner and score issuer: one lane issues the score MMAs (and Q Wq_h).
//   warp 2      P.V issuer: one lane issues the P.V MMAs (and the readout Q' S_h).
//   warp 3      publisher: raises the flag of each partial record the CTA stores.
//   warps 4-11  two softmax warpgroups. Warps w and w+4 share a TMEM lane quarter (the
//               same SM sub-partition). In the tile loop, w takes the quarter's first 16
//               rows and w+4 the last 16, whole rows of 128 scores through the 16-lane
//               TMEM shapes, four threads a row, so a row's max and sum need only shuffles.
//               For the Q' packing and the epilogue, thread = row = TMEM lane, and warps
//               4-7 own output columns 0-63, warps 8-11 columns 64-127; a row's max and sum
//               reach that layout through shared memory once per segment. These threads
//               also write outputs and partial records. Warp 3 stages the records a merge
//               reads.
// TMEM (512 columns):
//   - cols 0, 128, 256: three S tiles, tile t in buffer t % 3. The score MMA of tile t
//     waits for the P.V MMA of tile t - 3, which read P from the same buffer. P (bf16
//     pairs) overwrites the first 64 columns of its own S tile, keys in order, and feeds
//     the P.V MMA straight from TMEM.
//   - col 384: O.
//   - Readout of a segment holding key tile 0: after its last score MMA, Q' = Q Wq_h goes
//     to the S tile of tile t0 + n (fp32, then packed in place to bf16 like P); after its
//     last P.V MMA, O_inter = Q' S_h goes to the S tile of the segment's last tile. The
//     next segment's score MMAs write the first of these once the readout is done and the
//     second once the epilogue has read O_inter.
// Shared memory: Q | K0 K1 K2 | V0 V1 V2 (32 KiB tiles) from its 1 KiB-aligned base, then a
// small control block (mbarriers, flags, the row-statistics exchange slots).
//
// Online softmax: scores are kept in log2 units. The running max m is raised only when a
// tile's max exceeds it by more than 8 (a factor of 256), so O in TMEM is rescaled rarely.
// Probabilities stay below 2^8. Three column pairs in eight take their exponentials on
// the FMA pipe (exp2_poly2) and the rest on the MUFU unit; scaling, sums and the
// polynomial use the paired fp32 instructions.
#pragma once
#include <algorithm>

#include "arl2_device.cuh"
#include "arl2_kernels.h"

namespace arl2 {
namespace {

constexpr int kStages = 3;      // K and V ring depth
constexpr int kSBufs = 3;       // score tiles in TMEM
constexpr int kThreads = 384;
constexpr int kSoftmaxWarps = 8;   // barriers the softmax threads signal take one arrival per warp
enum : int {
  kBarQFull = 0,      // Q of a segment landed
  kBarQEmpty = 1,     // the segment's MMAs are done with Q
  kBarKFull = 2,      // +stage (3)
  kBarKEmpty = 5,
  kBarVFull = 8,
  kBarVEmpty = 11,
  kBarSFull = 14,     // +S buffer (3): scores of a tile are in TMEM
  kBarPFull = 17,     // +S buffer: P written over them (one arrival per softmax warp)
  kBarPVDone = 20,    // +S buffer: the P.V MMA that read P is done
  kBarQp = 23,        // Q' = Q Wq is in TMEM (a free S buffer), at the end of a head segment
  kBarQpReady = 24,   // Q' is packed to bf16 (per-warp arrivals)
  kBarOFull = 25,     // the segment's MMAs (its readout included) are all done
  kBarOEmpty = 26,    // the segment's O and O_inter were read (per-warp arrivals)
  kBarFinal = 27,     // every MMA done and every softmax warp finished with TMEM (before it is freed)
  kBarGroup = 28,     // bounded rendezvous of the softmax threads (per-warp arrivals)
  kBarPair = 29,      // +row quarter (4): the quarter's two warps stored their rows' max and sum
  kBarNever = 33,     // never signalled: target of the failure-detection test hook
  kBarRec = 34,       // a partial record is stored (per-warp arrivals); warp 3 publishes it
  kBarRecLoad = 35,   // the merge inputs of the CTA's last segment are staged in shared memory
  kBarLastPV = 36,    // the last P.V MMA of a staged merge's segment is done (V stages idle)
  kBarLastQK = 37,    // its last score MMA is done (K stages idle): staging may start
  kNumBars = 38
};
// Tiles at the (1 KiB-aligned) base of dynamic shared memory, then the control block.
constexpr uint32_t kQOff = 0;
constexpr uint32_t kKOff = kTileBytes;
constexpr uint32_t kVOff = kKOff + kStages * kTileBytes;
constexpr uint32_t kTileRegion = kVOff + kStages * kTileBytes;
constexpr uint32_t kCtlBars = 0;
constexpr uint32_t kCtlMisc = 320;           // tmem slot, abort flag, merge flag
// [2 slots][m | l][128] fp32: each row's max and sum at the end of a segment, on their way
// from the tile loop's layout to the epilogue's (slot = exchange parity).
constexpr uint32_t kCtlX = 384;
constexpr uint32_t kCtlBytes = kCtlX + 2 * 2 * 128 * 4;
static_assert(kNumBars * 8 <= kCtlMisc, "barriers must fit their slot");
constexpr uint32_t kSmemBytes = kTileRegion + kCtlBytes;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kMaxSegs = 8;                // the host plan keeps segments per query tile at or below this
constexpr int kHeadWeight = 10;            // key tile 0's extra split weight, quarter units (see QueryPlan)
// Staged merge: a query tile split in two segments is finished by its head segment (the
// CTA's last) from a shared-memory copy of the other record, taken while the head's last
// tiles are still in flight. The readout still reads Q, and Wq_h and S_h in ring stage ws of
// the K and V rings; the other stages are idle:
//   K stage ws+1: record column quads 0-15 (32 KiB)   K stage ws+2: quads 16-31
//   V stage ws+1: the record's m and l rows (1 KiB)   V stage ws+2: the bf16 output tile,
//                                                     stored by TMA (two swizzled panels)
__device__ __forceinline__ bool staged_merge(int nsegs) { return nsegs == 2; }

struct Smem {
  uint32_t ctl, tiles;
  __device__ uint32_t bar(int i) const { return ctl + kCtlBars + 8u * i; }
  __device__ uint32_t q() const { return tiles + kQOff; }
  __device__ uint32_t k(int s) const { return tiles + kKOff + s * kTileBytes; }
  __device__ uint32_t v(int s) const { return tiles + kVOff + s * kTileBytes; }
};

// Rendezvous of the 8 softmax warps with a bounded wait (no hang if a warp aborted).
__device__ __forceinline__ bool group_sync(uint32_t bar, uint32_t& phase, const Guard& g) {
  warp_arrive(bar);
  const bool ok = mbar_wait_warp(bar, phase & 1, g);
  ++phase;
  return ok;
}

// Acquire load of a flag another CTA publishes, and a bounded wait for a given value.
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ bool wait_flag(const int* f, int value, const Guard& g) {
  if (ld_acquire_gpu(f) == value) return true;
  WaitClock clock;
  while (ld_acquire_gpu(f) != value) {
    if (*g.abort) return false;
    if (clock.expired(g.timeout_ns)) {
      raise_timeout(g);
      return false;
    }
  }
  return true;
}

// One segment of a CTA's unit range: key tiles [kb, ke) of query tile Q.
struct Seg {
  int Q, kb, ke;
  int b, h, qt;
  bool head, tail;
  bool last;   // the CTA's last segment
};

// The CTA whose unit range holds unit u.
__device__ __forceinline__ int owner(long long u, const QueryArgs& a) {
  return split_owner(u, a.units, a.nkv, a.head_w, a.num_ctas);
}

// A CTA's walk over its unit range, one segment at a time. The divisions happen once, when
// the walk is set up at kernel start (their latency hides behind the first loads); each
// step then moves to the next query tile by increments, so no segment boundary waits on an
// integer division. The two facts about tiles shared with other CTAs are fixed at set-up
// too: only the range's first segment can lack key tile 0, and only its last can hold key
// tile 0 without the last key tile.
struct Sched {
  long long u, u1;
  int nq, nkv, H;
  int Q, kb, qt, b, h;   // the tile and key tile of unit u
  int first_rec;         // the first segment's record slot within its tile (this CTA - the tile's first CTA)
  int last_nsegs;        // CTAs sharing the last segment's tile (counted from this one)
  __device__ Sched(const QueryArgs& a, int c) : nq(a.nq), nkv(a.nkv), H(a.H) {
    u = split_start(c, a.units, a.nkv, a.head_w, a.num_ctas);
    u1 = split_start(c + 1, a.units, a.nkv, a.head_w, a.num_ctas);
    Q = static_cast<int>(u / nkv);
    kb = static_cast<int>(u % nkv);
    const int bh = Q / nq;
    qt = Q % nq;
    b = bh / H;
    h = bh % H;
    first_rec = c - owner(static_cast<long long>(Q) * nkv, a);
    const long long q_last = (u1 - 1) / nkv;
    last_nsegs = owner(q_last * nkv + nkv - 1, a) - c + 1;
  }
  __device__ bool next(Seg& s) {
    if (u >= u1) return false;
    s.Q = Q;
    s.kb = kb;
    s.qt = qt;
    s.b = b;
    s.h = h;
    const long long left = u1 - u;
    s.ke = left < nkv - kb ? kb + static_cast<int>(left) : nkv;
    u += s.ke - s.kb;
    s.head = s.kb == 0;
    s.tail = s.ke == nkv;
    s.last = u >= u1;
    if (s.tail) {   // on to key tile 0 of the next query tile
      ++Q;
      kb = 0;
      if (++qt == nq) {
        qt = 0;
        if (++h == H) {
          h = 0;
          ++b;
        }
      }
    } else {
      kb = s.ke;   // only when the range ended inside the tile: there is no next segment
    }
    return true;
  }
};


// Ring slot g: stage g % 3, used for the (g / 3)-th time. S buffers cycle the same way.
__device__ __forceinline__ int ring_stage(uint32_t g) { return static_cast<int>(g % kStages); }
__device__ __forceinline__ uint32_t ring_phase(uint32_t g) { return (g / kStages) & 1; }
__device__ __forceinline__ int sbuf(uint32_t t) { return static_cast<int>(t % kSBufs); }
// S buffer that receives O_inter of a head segment (tiles t0 .. t0+n-1). In the CTA's last
// segment: that of tile t0+n-2, whose P.V MMA is not the one just ahead, so the readout
// does not wait for the last P.V to finish reading. Otherwise that of the last tile, which
// the next segment rewrites only with its third score tile, after its O wait.
__device__ __forceinline__ int o_inter_tile(uint32_t t0, uint32_t n, bool last) {
  return sbuf(last ? t0 + n + 1 : t0 + n - 1);
}
__device__ __forceinline__ uint32_t sphase(uint32_t t) { return (t / kSBufs) & 1; }

// Producer (warp 0): per segment its Q tile, then per key tile the K tile and the V tile,
// each through its own three-stage ring; when the segment holds key tile 0 of its query
// tile, the readout operands follow its key tiles (Wq_h through the K ring, the bf16 state
// copy S_h through the V ring).
template <bool kHybrid>
__device__ void producer(const Smem& sm, const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                         const CUtensorMap* tm_w, const CUtensorMap* tm_s, const QueryArgs& a, const Guard& g,
                         bool lead) {
  uint32_t nk[kStages] = {0, 0, 0}, nv[kStages] = {0, 0, 0};   // loads issued per stage
  uint32_t nseg = 0, ring = 0;
  Sched sch(a, static_cast<int>(blockIdx.x) - a.first_cta);
  Seg sg;
  bool ok = true;
  bool waited = false;   // griddepcontrol.wait done before the first state load
  auto slot_wait = [&](int empty0, uint32_t gidx) -> bool {
    return gidx < kStages || mbar_wait_warp(sm.bar(empty0 + ring_stage(gidx)), ring_phase(gidx - kStages), g);
  };
  // q, k and v are this launch's activations: evict-first in L2, so they do not push out
  // what later launches reuse. (A key tile's other readers in this launch still hit L2: the
  // launch's working set is far below its size.)
  const uint64_t stream_policy = l2_evict_first_policy();
  auto load_kv = [&](const CUtensorMap* map, uint32_t dst, int bar, const Seg& s, int j) {
    if (lead) {
      mbar_expect_tx(sm.bar(bar), kTileBytes);
      for (int p = 0; p < 2; ++p)
        tma_load_4d_hint(dst + p * kPanelBytes, map, sm.bar(bar), 64 * p, s.h, j * kRows, s.b, stream_policy);
    }
  };
  auto load_op = [&](const CUtensorMap* map, uint32_t dst, int bar, int c2) {
    if (lead) {
      mbar_expect_tx(sm.bar(bar), kTileBytes);
      for (int p = 0; p < 2; ++p) tma_load_3d(dst + p * kPanelBytes, map, sm.bar(bar), 64 * p, 0, c2);
    }
  };
  while (ok && sch.next(sg)) {
    // The next segment's Q tile goes to L2 now, so that its load (issued only once this
    // segment's MMAs are done with Q) does not wait on HBM.
    if (lead && sch.u < sch.u1)
      for (int p = 0; p < 2; ++p) tma_prefetch_4d(tm_q, 64 * p, sch.h, sch.qt * kRows, sch.b);
    if (nseg > 0 && !mbar_wait_warp(sm.bar(kBarQEmpty), (nseg - 1) & 1, g)) break;
    if (lead) {
      mbar_expect_tx(sm.bar(kBarQFull), kTileBytes);
      for (int p = 0; p < 2; ++p)
        tma_load_4d_hint(sm.q() + p * kPanelBytes, tm_q, sm.bar(kBarQFull), 64 * p, sg.h, sg.qt * kRows, sg.b,
                         stream_policy);
    }
    ++nseg;
    for (int j = sg.kb; j < sg.ke; ++j, ++ring) {
      const int s = ring_stage(ring);
      if (!slot_wait(kBarKEmpty, ring)) {
        ok = false;
        break;
      }
      load_kv(tm_k, sm.k(s), kBarKFull + s, sg, j);
      ++nk[s];
      // Start-up order: the first Q tile and first K tile go out alone (they gate the
      // first score MMA); the rest of both rings fills once that K tile has landed.
      if (ring == 0 && !mbar_wait_warp(sm.bar(kBarKFull), 0, g)) {
        ok = false;
        break;
      }
      if (!slot_wait(kBarVEmpty, ring)) {
        ok = false;
        break;
      }
      load_kv(tm_v, sm.v(s), kBarVFull + s, sg, j);
      ++nv[s];
    }
    if (ok && kHybrid && sg.head) {
      // The readout operands follow the key tiles. S_{N-1} may be the output of the commit
      // right before this launch: when this grid was launched as its programmatic
      // dependent, that commit's writes are visible only after griddepcontrol.wait, which
      // comes once, before the first state load (a no-op for a normal launch, and long past
      // by then behind another query).
      const int s = ring_stage(ring);
      if (!slot_wait(kBarKEmpty, ring)) break;
      load_op(tm_w, sm.k(s), kBarKFull + s, sg.h);
      ++nk[s];
      if (!waited) {
        griddep_wait();
        waited = true;
      }
      if (!slot_wait(kBarVEmpty, ring)) break;
      load_op(tm_s, sm.v(s), kBarVFull + s, a.state_slot * a.B * a.H + sg.b * a.H + sg.h);
      ++nv[s];
      ++ring;
    }
  }
  __syncwarp();
  // Every load issued must land before the CTA may exit (matters only after an abort).
  if (nseg > 0) mbar_wait_drain(sm.bar(kBarQFull), (nseg - 1) & 1);
  for (int s = 0; s < kStages; ++s) {
    if (nk[s]) mbar_wait_drain(sm.bar(kBarKFull + s), (nk[s] - 1) & 1);
    if (nv[s]) mbar_wait_drain(sm.bar(kBarVFull + s), (nv[s] - 1) & 1);
  }
}

// Two MMA issuers, each a warp whose elected lane issues and commits; a tcgen05.mma issue
// blocks until the tensor pipe takes the instruction, so with one issuer the pipe idled
// whenever that thread waited on a barrier between its MMA groups. Here one warp issues
// the score MMAs (and Q' = Q Wq_h), the other the P.V MMAs (and O_inter = Q' S_h): while
// one waits, the other feeds the pipe. A commit tracks only its own thread's MMAs, so every
// reuse of TMEM columns the other issuer's MMA reads is ordered by a barrier:
//   - score tile t overwrites S buffer t % 3 once the P.V MMA of tile t - 3 (which read P
//     from it) is done;
//   - after a head segment (not the CTA's last), the next segment's first score tile goes
//     into the buffer that held Q': it waits until the readout MMA is done (OFull); the
//     buffer holding O_inter is next written once the epilogue has read it (OEmpty);
//   - the P.V MMA of a segment's first tile overwrites O once the epilogue has read it.
// S buffers cycle with the tile count: tile t in buffer t % 3. A segment holding key tile 0
// puts Q' in the buffer of tile t0 + n and O_inter in that of the last tile (t0 + n - 1),
// or, in the CTA's last segment, of tile t0 + n - 2 (see o_inter_tile).
template <bool kHybrid>
__device__ void score_issuer(const Smem& sm, uint32_t tmem, const QueryArgs& a, const Guard& g, bool lead) {
  constexpr uint32_t id_kk = idesc_bf16(128, 128, false, false);   // A, B K-major
  constexpr uint32_t id_kmn = idesc_bf16(128, 128, false, true);   // A K-major, B MN-major
  uint32_t nseg = 0, tile = 0, ring = 0;
  int qp_buf = -1, x_buf = -1;        // buffers still read by the previous segment's readout / epilogue
  uint32_t qp_phase = 0, x_phase = 0;
  Sched sch(a, static_cast<int>(blockIdx.x) - a.first_cta);
  Seg sg;
  // Before an MMA writes the S buffer of tile t: the earlier readers of that buffer are done.
  auto buffer_free = [&](uint32_t t) -> bool {
    const int sb = sbuf(t);
    if (t >= kSBufs && !mbar_wait_warp(sm.bar(kBarPVDone + sb), sphase(t - kSBufs), g)) return false;
    if (sb == qp_buf) {
      if (!mbar_wait_warp(sm.bar(kBarOFull), qp_phase, g)) return false;
      qp_buf = -1;
    }
    if (sb == x_buf) {
      if (!mbar_wait_warp(sm.bar(kBarOEmpty), x_phase, g)) return false;
      x_buf = -1;
    }
    tc_fence_after();
    return true;
  };
  while (sch.next(sg)) {
    const bool rd = kHybrid && sg.head;
    const uint32_t t0 = tile, n = sg.ke - sg.kb;
    const bool staged = sg.head && !sg.tail && staged_merge(sch.last_nsegs);   // the CTA's last segment
    if (!mbar_wait_warp(sm.bar(kBarQFull), nseg & 1, g)) return;
    for (uint32_t i = 0; i < n; ++i) {
      const uint32_t t = t0 + i, r = ring + i;
      const int sb = sbuf(t), ks = ring_stage(r);
      if (!buffer_free(t) || !mbar_wait_warp(sm.bar(kBarKFull + ks), ring_phase(r), g)) return;
      tc_fence_after();
      if (lead) {
        mma8_ss<false, false>(tmem + 128u * sb, desc_kmajor(sm.q(), 0), desc_kmajor(sm.k(ks), 0), id_kk, 0u);
        mma_commit(sm.bar(kBarKEmpty + ks));
        mma_commit(sm.bar(kBarSFull + sb));
      }
    }
    if (lead && staged) mma_commit(sm.bar(kBarLastQK));   // K stages other than the readout's are idle
    if (rd) {
      // Q' = Q Wq_h into the S buffer of tile t0 + n (Wq_h in the K ring after the key tiles).
      const int rs = ring_stage(ring + n);
      if (!buffer_free(t0 + n) || !mbar_wait_warp(sm.bar(kBarKFull + rs), ring_phase(ring + n), g)) return;
      tc_fence_after();
      if (lead) {
        mma8_ss<false, true>(tmem + 128u * sbuf(t0 + n), desc_kmajor(sm.q(), 0), desc_mnmajor(sm.k(rs), 0), id_kmn,
                             0u);
        mma_commit(sm.bar(kBarKEmpty + rs));
        mma_commit(sm.bar(kBarQEmpty));
        mma_commit(sm.bar(kBarQp));
      }
      qp_buf = sbuf(t0 + n);
      qp_phase = nseg & 1;
      x_buf = o_inter_tile(t0, n, sg.last);
      x_phase = nseg & 1;
    } else if (lead) {
      mma_commit(sm.bar(kBarQEmpty));
    }
    tile += n;
    ring += n + (rd ? 1u : 0u);
    ++nseg;
  }
}

template <bool kHybrid>
__device__ void pv_issuer(const Smem& sm, uint32_t tmem, const QueryArgs& a, const Guard& g, bool lead) {
  constexpr uint32_t id_kmn = idesc_bf16(128, 128, false, true);   // A K-major (TMEM), B MN-major
  const uint32_t tO = tmem + kColO;
  // A operands in TMEM, by K step of 16: P packed by the softmax's .16x128b stores (its
  // 64 words in order), and Q' packed in place by column halves (words 0-31 and 64-95).
  const uint32_t kPackedP[8] = {0, 8, 16, 24, 32, 40, 48, 56};
  const uint32_t kPackedQ[8] = {0, 8, 16, 24, 64, 72, 80, 88};
  uint32_t nseg = 0, nhead = 0, tile = 0, ring = 0;
  Sched sch(a, static_cast<int>(blockIdx.x) - a.first_cta);
  Seg sg;
  while (sch.next(sg)) {
    const bool rd = kHybrid && sg.head;
    const uint32_t t0 = tile, n = sg.ke - sg.kb;
    const bool staged = sg.head && !sg.tail && staged_merge(sch.last_nsegs);
    // O (and the previous segment's O_inter) must have been read before O is rewritten.
    if (nseg > 0 && !mbar_wait_warp(sm.bar(kBarOEmpty), (nseg - 1) & 1, g)) return;
    for (uint32_t i = 0; i < n; ++i) {
      const uint32_t t = t0 + i, r = ring + i;
      const int sb = sbuf(t), vs = ring_stage(r);
      if (!mbar_wait_warp(sm.bar(kBarPFull + sb), sphase(t), g)) return;
      if (!mbar_wait_warp(sm.bar(kBarVFull + vs), ring_phase(r), g)) return;
      tc_fence_after();
      if (lead) {
        mma8_ts(tO, tmem + 128u * sb, kPackedP, desc_mnmajor(sm.v(vs), 0), id_kmn, i > 0 ? 1u : 0u);
        mma_commit(sm.bar(kBarPVDone + sb));
        mma_commit(sm.bar(kBarVEmpty + vs));
      }
    }
    if (lead && staged) mma_commit(sm.bar(kBarLastPV));   // V stages other than the readout's are idle
    if (rd) {
      // O_inter = Q' S_{N-1}, with Q' packed to bf16 in place by the softmax threads.
      const uint32_t tY = tmem + 128u * sbuf(t0 + n), tX = tmem + 128u * o_inter_tile(t0, n, sg.last);
      const int rs = ring_stage(ring + n);
      if (!mbar_wait_warp(sm.bar(kBarQpReady), nhead & 1, g)) return;
      if (!mbar_wait_warp(sm.bar(kBarVFull + rs), ring_phase(ring + n), g)) return;
      tc_fence_after();
      if (lead) {
        mma8_ts(tX, tY, kPackedQ, desc_mnmajor(sm.v(rs), 0), id_kmn, 0u);
        mma_commit(sm.bar(kBarVEmpty + rs));
      }
      ++nhead;
    }
    if (lead) mma_commit(sm.bar(kBarOFull));   // every MMA of the segment, the readout included
    tile += n;
    ring += n + (rd ? 1u : 0u);
    ++nseg;
  }
}

// Score layout in the softmax threads: the two warps of a lane quarter split its 32 rows
// (the first takes lanes 0-15, the second 16-31), and each reads whole rows with the
// .16x256b shape. Thread t of a warp holds rows (t / 4) and (t / 4) + 8 of its 16, and in
// every 8-column chunk the two columns 2 (t % 4) and 2 (t % 4) + 1; the four threads of a
// row (consecutive lanes) hold all 128 columns between them. sv[p][4c + 2h + j] is row
// (t / 4) + 8h, column 64p + 8c + 2 (t % 4) + j. Row statistics need only shuffles among
// those four lanes, never another warp.

// Maxima (raw units) of this thread's two rows over its own 32 columns each, with keys at or
// beyond `valid` masked to -inf. The row's other three threads hold the rest of the row.
__device__ __forceinline__ void thread_max2(uint32_t (&sv)[2][32], int g4, int valid, float (&mx)[2]) {
  if (valid < kRows) {
#pragma unroll
    for (int p = 0; p < 2; ++p)
#pragma unroll
      for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (64 * p + 8 * c + 2 * g4 + (e & 1) >= valid) sv[p][4 * c + e] = __float_as_uint(-INFINITY);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float m4[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int p = 0; p < 2; ++p)
#pragma unroll
      for (int c = 0; c < 8; ++c)
        m4[c & 1] = fmax3(m4[c & 1], __uint_as_float(sv[p][4 * c + 2 * h]), __uint_as_float(sv[p][4 * c + 2 * h + 1]));
    mx[h] = fmaxf(m4[0], m4[1]);
  }
}
// The maxima over each row's four threads (consecutive lanes).
__device__ __forceinline__ void row_reduce_max2(float (&mx)[2]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
  }
}

// Column pairs (of every 8) whose exponentials run on the FMA pipe (exp2_poly2); the
// rest go to the MUFU unit. Three of eight balances the two units for d = 128.
constexpr uint32_t kPolyPairs = 0xA4u;   // pairs 2, 5, 7
__host__ __device__ constexpr bool poly_pair(int j) { return (kPolyPairs >> (j & 7)) & 1u; }

// P for this thread's 64 scores (raw fp32 in sv; masked ones are -inf), as 32 packed bf16
// pairs in the .16x128b layout: pk[2 cc + h] is row (t / 4) + 8h, packed column
// 4 cc + (t % 4), which holds keys 8 cc + 2 (t % 4) and the next. Adds this thread's share
// of each row's sum to lsum[h]; m[h] is the log2-unit max in use for row h.
__device__ __forceinline__ void row_probs2(const uint32_t (&sv)[2][32], const float (&m)[2], float scale_log2,
                                           uint32_t (&pk)[32], float (&lsum)[2]) {
  const float2 sc = make_float2(scale_log2, scale_log2);
  float2 acc[2][2];
#pragma unroll
  for (int h = 0; h < 2; ++h) acc[h][0] = acc[h][1] = make_float2(0.f, 0.f);
#pragma unroll
  for (int p = 0; p < 2; ++p) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int cc = 8 * p + c;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[p][4 * c + 2 * h]), __uint_as_float(sv[p][4 * c + 2 * h + 1])),
                                    sc, make_float2(-m[h], -m[h]));
        const float2 pr = poly_pair(cc) ? exp2_poly2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
        acc[h][cc & 1] = __fadd2_rn(acc[h][cc & 1], pr);
        pk[2 * cc + h] = pack_bf16x2(pr.x, pr.y);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float2 s2 = __fadd2_rn(acc[h][0], acc[h][1]);
    lsum[h] += s2.x + s2.y;
  }
}

// Scratch records are stored column-quad-major: float4 (record, quad q of 4 columns, row r)
// sits at ((record * 32 + q) * 128 + r), so a warp's 32 rows move 512 contiguous bytes.
__device__ __forceinline__ float4* quad_ptr(float* base, size_t record, int q, uint32_t r) {
  return reinterpret_cast<float4*>(base) + ((record * 32 + q) * kRows + r);
}

// The merge of a head segment: its own O (TMEM, max m, sum l_row) with the tile's other
// nsegs - 1 records, plus O_inter (TMEM, the layer only), normalised and rounded to bf16.
// kStaged: the single other record is in shared memory (see staged_merge) and the output
// goes to the shared-memory tile otile for a TMA store; otherwise records come from
// scratch and rows go straight to global memory. Two instantiations, so neither path
// carries the other's loads.
template <bool kHybrid, bool kStaged>
__device__ __forceinline__ void merge_rows(const QueryArgs& a, const Seg& sg, uint32_t r, int half, int c0, int ncols,
                                           uint32_t tO, uint32_t tX, float m, float l_row, int nsegs_rt,
                                           size_t slot0, const float* stage, int k1, int k2, uint32_t otile) {
  const int nsegs = kStaged ? 2 : nsegs_rt;
  const int q0 = c0 / 4;
  const float4* st4 = reinterpret_cast<const float4*>(stage);
  // Record s of the tile's other segments: the staged copy (shared memory) or scratch.
  auto rec_m = [&](int s) {
    if constexpr (kStaged) return stage[(kVOff + k1 * kTileBytes) / 4 + r];
    else return __ldcg(a.part_ml + ((slot0 + s) * 2) * kRows + r);
  };
  auto rec_l = [&](int s) {
    if constexpr (kStaged) return stage[(kVOff + k1 * kTileBytes) / 4 + kRows + r];
    else return __ldcg(a.part_ml + ((slot0 + s) * 2 + 1) * kRows + r);
  };
  auto rec_o = [&](int s, int q) {
    if constexpr (kStaged) return st4[(kKOff + (q < 16 ? k1 : k2) * kTileBytes) / 16 + (q & 15) * kRows + r];
    else return __ldcg(quad_ptr(a.part_o, slot0 + s, q, r));
  };
  // Weights of the other records. The staged merge has exactly one; otherwise the loops
  // over records run as loops (not unrolled): this code runs once per query tile, so its
  // size (instruction fetches from L2 on a cold instruction cache) costs more than its
  // arithmetic, and most tiles have no other record at all.
  float M = m;
#pragma unroll 1
  for (int s = 1; s < nsegs; ++s) M = fmaxf(M, rec_m(s));
  const float w_own = ex2_approx(m - M);
  float L = w_own * l_row;
#pragma unroll 1
  for (int s = 1; s < nsegs; ++s) L += ex2_approx(rec_m(s) - M) * rec_l(s);
  const float inv_L = 1.f / L;
  const int t_row = sg.qt * kRows + static_cast<int>(r);
  const bool row_ok = t_row < a.T;
  uint16_t* out_row = a.o + ((static_cast<size_t>(sg.b) * a.T + t_row) * a.H + sg.h) * a.d + c0;
  // Four passes of 16 columns: the other records first, then the TMEM loads (O, and
  // O_inter for the layer) with their wait right behind them. No code sits between a TMEM
  // load and its wait: the load's destination registers are undefined until the wait, and
  // anything in between gives the compiler room to copy them early. The passes run as a
  // loop: this code runs once per tile, on a cold instruction cache, where its size costs
  // more than the loop.
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    if (16 * c >= ncols) break;
    float4 acc[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
    for (int s = 1; s < nsegs; ++s) {
      const float ws = ex2_approx(rec_m(s) - M);
      float4 v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) v[q] = rec_o(s, q0 + 4 * c + q);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[q].x += ws * v[q].x;
        acc[q].y += ws * v[q].y;
        acc[q].z += ws * v[q].z;
        acc[q].w += ws * v[q].w;
      }
    }
    uint32_t ov[16], xv[16];
    if (kHybrid)
      tmem_ld16x2_wait(tO + c0 + 16u * c, ov, tX + c0 + 16u * c, xv);
    else
      tmem_ld16_wait(tO + c0 + 16u * c, ov);
    float y[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      y[4 * q] = (acc[q].x + w_own * __uint_as_float(ov[4 * q])) * inv_L;
      y[4 * q + 1] = (acc[q].y + w_own * __uint_as_float(ov[4 * q + 1])) * inv_L;
      y[4 * q + 2] = (acc[q].z + w_own * __uint_as_float(ov[4 * q + 2])) * inv_L;
      y[4 * q + 3] = (acc[q].w + w_own * __uint_as_float(ov[4 * q + 3])) * inv_L;
    }
    if (kHybrid) {
#pragma unroll
      for (int e = 0; e < 16; ++e) y[e] += __uint_as_float(xv[e]);
    }
    const uint4 w0 = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                                pack_bf16x2(y[6], y[7]));
    const uint4 w1 = make_uint4(pack_bf16x2(y[8], y[9]), pack_bf16x2(y[10], y[11]), pack_bf16x2(y[12], y[13]),
                                pack_bf16x2(y[14], y[15]));
    if constexpr (kStaged) {
      // Columns 16c .. 16c+15 of this half = 16-byte chunks 2c and 2c+1 of panel `half`.
      const uint32_t row = otile + half * kPanelBytes + r * 128u;
      st_shared_v4(row + (((2u * c) ^ (r & 7u)) << 4), w0.x, w0.y, w0.z, w0.w);
      st_shared_v4(row + (((2u * c + 1u) ^ (r & 7u)) << 4), w1.x, w1.y, w1.z, w1.w);
    } else if (row_ok) {
      uint4* dst = reinterpret_cast<uint4*>(out_row + 16 * c);
      dst[0] = w0;
      dst[1] = w1;
    }
    // Rows past T (a ragged last tile) skip the stores: reconverge the warp before the next
    // pass's warp-wide TMEM loads (.sync.aligned), whatever the compiler made of the branch.
    __syncwarp();
  }
}

// End of a segment. The segment holding key tile 0 of a query tile (its head) finishes
// the tile: it combines its own O (TMEM) with the partial records of the tile's other
// segments, adds O_inter and writes O. With contiguous unit ranges the head segment is
// the last segment of its CTA and every other segment of the tile starts another CTA's
// range, so those records are normally published long before. Any other segment stores
// its partial record (O_acc, running max m, sum l) and the publisher warp raises the
// record's flag. Loads are issued in batches so their latencies overlap. Kept out of line
// so its registers do not compete with the softmax loop; the launch arguments it reads stay
// in parameter space (the kernel takes them as a grid constant), not in a per-thread copy
// in local memory; the small structs come by value for the same reason. Returns the number
// of group rendezvous it took (0 or 1), or -1 if a wait gave up.
template <bool kHybrid>
__device__ __noinline__ int segment_epilogue(const Smem sm, const QueryArgs& a, const Seg sg, int first_rec,
                                             int last_nsegs, uint32_t r, int half, int c0, int ncols, uint32_t tO,
                                             uint32_t tX, float m, float l_row, uint32_t gphase,
                                             volatile int* merge_ok, const float* stage, int rs,
                                             const CUtensorMap* tm_o, const Guard g) {
  const uint32_t gphase0 = gphase;
  const int q0 = c0 / 4;   // this half's first column quad
  // First global write of this thread in the launch: a query launched as the programmatic
  // dependent of the previous one waits for it here (shared scratch, maybe the same output).
  griddep_wait();
  const size_t slot0 = static_cast<size_t>(sg.Q) * a.max_segs;
  if (!sg.head) {   // the CTA's first segment
    const size_t slot = slot0 + first_rec;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      if (16 * c >= ncols) break;
      uint32_t ov[16];
      tmem_ld16_wait(tO + c0 + 16u * c, ov);
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
    tc_fence_before();
    warp_arrive(sm.bar(kBarOEmpty));   // TMEM read: the next segment may reuse O
    warp_arrive(sm.bar(kBarRec));      // record stored: the publisher may raise its flag
    return 0;
  }
  // Head segment: the tile's other records (if any), then the merge. Warp 3 stages them
  // in shared memory when they fit; otherwise they are read from scratch here.
  const int nsegs = sg.tail ? 1 : last_nsegs;   // not a tail: the CTA's last segment
  const bool staged = staged_merge(nsegs);
  const int k1 = (rs + 1) % kStages, k2 = (rs + 2) % kStages;   // idle ring stages (see staged_merge)
  if (staged) {
    // At most one staged merge per CTA and launch: the barrier completes once (phase 0).
    if (!mbar_wait_warp(sm.bar(kBarRecLoad), 0, g)) return -1;
  } else if (nsegs > 1) {
    if (half == 0 && r == 0) {
      bool ok = true;
      for (int s = 1; s < nsegs && ok; ++s) ok = wait_flag(a.flags + slot0 + s, a.epoch, g);
      *merge_ok = ok ? 1 : 0;
    }
    if (!group_sync(sm.bar(kBarGroup), gphase, g)) return -1;
    if (!*merge_ok) return -1;
  }
  const uint32_t otile = sm.v(k2);   // staged: the output tile (two 128-byte-swizzled panels)
  if (staged)
    merge_rows<kHybrid, true>(a, sg, r, half, c0, ncols, tO, tX, m, l_row, nsegs, slot0, stage, k1, k2, otile);
  else
    merge_rows<kHybrid, false>(a, sg, r, half, c0, ncols, tO, tX, m, l_row, nsegs, slot0, stage, k1, k2, otile);
  if (staged && 64 * half < a.d) {
    // Each warp stores its own 32 rows x 64 columns by TMA (coalesced; rows past T and
    // columns past d are clipped). A 32-row slice of a swizzled panel starts on a 1 KiB
    // boundary, so it is a swizzled box of its own.
    fence_proxy_async_smem();
    __syncwarp();
    if ((r & 31u) == 0) {
      const uint32_t q32 = r & ~31u;
      tma_store_4d(tm_o, otile + half * kPanelBytes + q32 * 128u, 64 * half, sg.h, sg.qt * kRows + q32, sg.b);
      bulk_commit_group();
      bulk_wait_group_read0();   // the source must stay intact until read (the CTA exits next)
    }
    __syncwarp();
  }
  tc_fence_before();
  warp_arrive(sm.bar(kBarOEmpty));
  return static_cast<int>(gphase - gphase0);
}

// Warp 3. (1) Raises the flag of each partial record this CTA stores, once the softmax
// warps have stored it: their CTA-scope arrival orders those stores before this warp's
// device-scope fence, so a CTA that reads the flag (acquire) sees the whole record.
// (2) For a staged merge (the CTA's last segment): waits for the other record's flag while
// the segment runs, then bulk-copies that record into the idle K stages once the last score
// MMA is done, and its (m, l) rows into an idle V stage once the last P.V MMA is done.
// Every barrier this warp waits on completes at most once per launch, so a parity wait can
// never alias an earlier phase.
template <bool kHybrid>
__device__ void publisher(const Smem& sm, const QueryArgs& a, const Guard& g) {
  const bool lead = (threadIdx.x & 31) == 0;
  uint32_t nrec = 0;   // a CTA stores at most one record (only its first segment can lack key tile 0)
  uint32_t ring = 0;   // ring slots used so far (key tiles, plus one readout operand per head)
  bool staged_issued = false;
  Sched sch(a, static_cast<int>(blockIdx.x) - a.first_cta);
  Seg sg;
  while (sch.next(sg)) {
    const size_t slot0 = static_cast<size_t>(sg.Q) * a.max_segs;
    const uint32_t n = sg.ke - sg.kb;
    const int ws = ring_stage(ring + n);   // the readout operands' stage
    ring += n + ((kHybrid && sg.head) ? 1u : 0u);
    if (!sg.head) {
      if (!mbar_wait_warp(sm.bar(kBarRec), nrec & 1, g)) break;
      ++nrec;
      griddep_wait();   // the previous launch may still poll this flag for its own epoch
      if (lead) {
        __threadfence();
        atomicExch(a.flags + slot0 + sch.first_rec, a.epoch);
      }
      __syncwarp();
    } else if (!sg.tail && staged_merge(sch.last_nsegs)) {
      bool ok = true;
      if (lead) ok = wait_flag(a.flags + slot0 + 1, a.epoch, g);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const int k1 = (ws + 1) % kStages, k2 = (ws + 2) % kStages;
      // The record (d/4 column quads) into K stages k1, k2 once the last score MMA is done,
      // in 4 KiB pieces so that several are in flight; its (m, l) rows into V stage k1
      // once the last P.V MMA is done.
      if (!mbar_wait_warp(sm.bar(kBarLastQK), 0, g)) break;
      const uint32_t rec_bytes = static_cast<uint32_t>(a.d) * kRows * 4;
      const char* rec = reinterpret_cast<const char*>(a.part_o + (slot0 + 1) * kRows * kDP);
      if (lead) {
        fence_proxy_async_global();
        mbar_expect_tx(sm.bar(kBarRecLoad), rec_bytes + 1024u);
      }
      for (uint32_t off = 4096u * (threadIdx.x & 31); off < rec_bytes; off += 4096u * 32) {
        const uint32_t dst = (off < kTileBytes ? sm.k(k1) : sm.k(k2)) + off % kTileBytes;
        bulk_load(dst, rec + off, 4096u, sm.bar(kBarRecLoad));
      }
      staged_issued = true;
      if (!mbar_wait_warp(sm.bar(kBarLastPV), 0, g)) break;
      if (lead) bulk_load(sm.v(k1), a.part_ml + (slot0 + 1) * 2 * kRows, 1024u, sm.bar(kBarRecLoad));
      __syncwarp();
    }
  }
  // Copies into shared memory must land before the CTA exits (matters only after an abort).
  if (staged_issued) mbar_wait_drain(sm.bar(kBarRecLoad), 0);
}

template <bool kHybrid>
__device__ void softmax_role(const Smem& sm, uint8_t* ctl, uint32_t tmem, const QueryArgs& a, int warp,
                             const CUtensorMap* tm_o, const Guard& g) {
  const int quarter = warp & 3;
  // In the epilogue and the Q' packing a thread owns row r (its TMEM lane) and the column
  // half `half`; in the tile loop the same warp owns 16 whole rows of its quarter instead
  // (rows 16 half .. 16 half + 15; see thread_max2).
  const int half = (warp - 4) >> 2;
  const uint32_t r = quarter * 32 + (threadIdx.x & 31);     // tile row == TMEM lane
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t lane16_off = static_cast<uint32_t>(quarter * 32 + 16 * half) << 16;
  const int g4 = static_cast<int>(threadIdx.x & 3);
  const uint32_t row0 = quarter * 32 + 16 * half + ((threadIdx.x & 31) >> 2);   // rows row0, row0 + 8
  const uint32_t tO = tmem + lane_off + kColO;
  float* xch = reinterpret_cast<float*>(ctl + kCtlX);      // [2 slots][m | l][128]
  volatile int* merge_ok = reinterpret_cast<volatile int*>(ctl + kCtlMisc + 8);
  const uint32_t pair_bar = sm.bar(kBarPair + quarter);
  const int d = a.d;
  const int c0 = 64 * half;                                 // first output column of this thread's half
  const int ncols = max(0, min(64, d - c0));                // output columns of this half
  uint32_t nseg = 0, nhead = 0, tile = 0, gphase = 0, nx = 0, ring = 0;
  // Test hook: a wait that can only run out (the bounded-wait path, without a fault).
  if (a.stall && !mbar_wait_warp(sm.bar(kBarNever), 0, g)) return;
  Sched sch(a, static_cast<int>(blockIdx.x) - a.first_cta);
  Seg sg;
  while (sch.next(sg)) {
    const uint32_t t0 = tile, n = sg.ke - sg.kb;
    const int rs = ring_stage(ring + n);   // ring stage of the readout operands (staged merges)
    ring += n + ((kHybrid && sg.head) ? 1u : 0u);
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};   // rows row0, row0 + 8
    for (uint32_t i = 0; i < n; ++i) {
      const uint32_t t = t0 + i;
      const int sb = sbuf(t);
      if (!mbar_wait_warp(sm.bar(kBarSFull + sb), sphase(t), g)) return;
      tc_fence_after();
      const uint32_t tS = tmem + lane16_off + 128u * sb;
      const int valid = a.kv_len - (sg.kb + static_cast<int>(i)) * kRows;   // >= 1
      uint32_t sv[2][32];
      tmem_ld16dp256_x8x2_wait(tS, sv[0], tS + 64u, sv[1]);
      // The running max changes only on a segment's first tile or when a row's max exceeds
      // it by more than the threshold. Each thread first checks its own columns; only if
      // one of the warp's threads sees such a column do the rows' four threads combine
      // their maxima (scaling by the positive scale_log2 commutes with the max, so the
      // rows get exactly the maxima the full reduction gives).
      float mt[2];
      thread_max2(sv, g4, valid, mt);
      float m_new[2] = {m[0], m[1]};
      bool rescale[2] = {false, false};
      bool raise = i == 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        mt[h] *= a.scale_log2;
        raise = raise || mt[h] > m[h] + kRescaleThreshold;
      }
      if (__any_sync(0xffffffffu, raise)) {
        row_reduce_max2(mt);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (i == 0) {
            m_new[h] = mt[h];
          } else if (mt[h] > m[h] + kRescaleThreshold) {
            m_new[h] = mt[h];
            rescale[h] = true;
          }
        }
      }
      if (__any_sync(0xffffffffu, rescale[0] || rescale[1])) {
        // O holds the sum up to tile t-1: wait for that P.V MMA, then scale these rows.
        if (!mbar_wait_warp(sm.bar(kBarPVDone + sbuf(t - 1)), sphase(t - 1), g)) return;
        tc_fence_after();
        const float corr0 = rescale[0] ? ex2_approx(m[0] - m_new[0]) : 1.f;
        const float corr1 = rescale[1] ? ex2_approx(m[1] - m_new[1]) : 1.f;
        const uint32_t tO16 = tmem + lane16_off + kColO;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ov[16];
          tmem_ld16dp256_x4_wait(tO16 + 32u * c, ov);
#pragma unroll
          for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * ((e & 2) ? corr1 : corr0));
          tmem_st16dp256_x4(tO16 + 32u * c, ov);
        }
        l[0] *= corr0;
        l[1] *= corr1;
      }
      m[0] = m_new[0];
      m[1] = m_new[1];
      uint32_t pk[32];
      row_probs2(sv, m, a.scale_log2, pk, l);
      // P (bf16 pairs) overwrites the first 64 columns of the rows' scores.
      tmem_st16dp128_x16(tS, pk);
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(sm.bar(kBarPFull + sb));
    }
    tile += n;

    // ---- end of segment. A segment holding key tile 0 computes the readout here: Q' =
    // Q Wq_h arrives (fp32) in the S buffer of tile t0 + n; each half packs its own 64
    // columns to bf16 pairs in place (the readout MMA's A operand, same layout as P).
    const uint32_t tX = tmem + lane_off + 128u * o_inter_tile(t0, n, sg.last);   // O_inter, when computed
    if (kHybrid && sg.head) {
      const uint32_t tY = tmem + lane_off + 128u * sbuf(t0 + n);
      if (!mbar_wait_warp(sm.bar(kBarQp), nhead & 1, g)) return;
      tc_fence_after();
      // Two rounds of 32 columns; round h packs into columns c0 + 16h .. c0 + 16h + 15,
      // which round h has already read (round 1 writes only what round 0 read).
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t x0[16], x1[16], pk[16];
        tmem_ld16x2_wait(tY + c0 + 32u * h, x0, tY + c0 + 32u * h + 16u, x1);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          pk[i] = pack_bf16x2(__uint_as_float(x0[2 * i]), __uint_as_float(x0[2 * i + 1]));
          pk[8 + i] = pack_bf16x2(__uint_as_float(x1[2 * i]), __uint_as_float(x1[2 * i + 1]));
        }
        tmem_st16(tY + c0 + 16u * h, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(sm.bar(kBarQpReady));
      ++nhead;
    }
    // Every MMA of the segment (the readout included) is done. Each row's max and sum go
    // from the tile-loop layout (16 rows a warp, four threads a row) to the epilogue's
    // (thread = row) through shared memory; the two warps of the quarter meet on their pair
    // barrier. Slots alternate by exchange count, so a slot is rewritten only after the
    // other warp has passed the next exchange, and so has read it.
    if (!mbar_wait_warp(sm.bar(kBarOFull), nseg & 1, g)) return;
    tc_fence_after();
    {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 1);
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 2);
      }
      float* ml = xch + (nx & 1) * 256;
      if (g4 == 0) {
        ml[row0] = m[0];
        ml[row0 + 8] = m[1];
        ml[kRows + row0] = l[0];
        ml[kRows + row0 + 8] = l[1];
      }
      warp_arrive(pair_bar);
      const bool ok = mbar_wait_warp(pair_bar, nx & 1, g);
      ++nx;
      if (!ok) return;
    }
    const float* ml = xch + ((nx - 1) & 1) * 256;
    const int syncs = segment_epilogue<kHybrid>(sm, a, sg, sch.first_rec, sch.last_nsegs, r, half, c0, ncols, tO, tX,
                                                ml[r], ml[kRows + r], gphase, merge_ok,
                                                reinterpret_cast<const float*>(ctl - kTileRegion), rs, tm_o, g);
    if (syncs < 0) return;
    gphase += static_cast<uint32_t>(syncs);
    ++nseg;
  }
}

// One CTA of a query launch (CTA blockIdx.x - a.first_cta of a.num_ctas in the stream-K split). The maps
// and arguments are the launching kernel's __grid_constant__ parameters, passed by reference
// so that every role reads them in parameter space.
template <bool kHybrid>
__device__ __forceinline__ void query_cta(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                          const CUtensorMap& tm_w, const CUtensorMap& tm_s, const CUtensorMap& tm_o,
                                          const QueryArgs& a, uint8_t* smem_raw) {
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
      mbar_init(sm.bar(kBarPFull + s), kSoftmaxWarps);
      mbar_init(sm.bar(kBarPVDone + s), 1);
    }
    mbar_init(sm.bar(kBarQp), 1);
    mbar_init(sm.bar(kBarQpReady), kSoftmaxWarps);
    mbar_init(sm.bar(kBarOFull), 1);
    mbar_init(sm.bar(kBarOEmpty), kSoftmaxWarps);
    mbar_init(sm.bar(kBarFinal), 2 + kSoftmaxWarps);   // a commit per MMA issuer, an arrival per softmax warp
    mbar_init(sm.bar(kBarGroup), kSoftmaxWarps);
    for (int q = 0; q < 4; ++q) mbar_init(sm.bar(kBarPair + q), 2);   // one arrival per warp
    mbar_init(sm.bar(kBarNever), 1);
    mbar_init(sm.bar(kBarRec), kSoftmaxWarps);
    mbar_init(sm.bar(kBarRecLoad), 1);
    mbar_init(sm.bar(kBarLastPV), 1);
    mbar_init(sm.bar(kBarLastQK), 1);
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
  // A kernel launched right behind this one as its programmatic dependent may start its
  // CTAs as SMs free up. A query or commit reads nothing a query writes (the host launches
  // a call whose inputs overlap this grid's output normally). A query waits for the grid
  // before it (this one, or a commit) before its first global write (its scratch and
  // output may be this grid's) and before its first load of the state (a commit's output).
  griddep_launch_dependents();

  // The producer and the MMA issuers run warp-wide (uniform control flow and waits); one
  // elected lane issues each TMA copy, MMA and commit.
  if (warp == 0) {
    producer<kHybrid>(sm, &tm_q, &tm_k, &tm_v, &tm_w, &tm_s, a, g, elect_one());
  } else if (warp == 1 || warp == 2) {
    const bool lead = elect_one();
    if (warp == 1)
      score_issuer<kHybrid>(sm, tmem, a, g, lead);
    else
      pv_issuer<kHybrid>(sm, tmem, a, g, lead);
    if (lead) mma_commit(sm.bar(kBarFinal));   // arrives once every MMA this warp issued has finished
    __syncwarp();
  } else if (warp == 3) {
    publisher<kHybrid>(sm, a, g);
  } else {
    softmax_role<kHybrid>(sm, ctl_ptr, tmem, a, warp, &tm_o, g);
    // Every TMEM access of this warp is done (whichever way the role ended): TMEM may be
    // freed once both MMA issuers and all eight softmax warps have arrived.
    tc_fence_before();
    warp_arrive(sm.bar(kBarFinal));
  }

  // The roles end in per-lane waits (drains), so a warp may arrive here split: reconverge
  // it first, or its parts would count as several arrivals at the CTA barrier.
  __syncwarp();
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
}  // namespace arl2
