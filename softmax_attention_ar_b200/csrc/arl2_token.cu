// Token-level access for the ARL2 hybrid layer: the ablation that the technical summary of
// arXiv 2605.16579 ("Attend Locally, Remember Linearly", §4 Ablations) contrasts with
// frame-level access. Inside a pass the state advances token by token, with the §2.1 update
// rule applied to one token at a time, starting from S_{N-1}; token t reads the state its
// predecessors left:
//     o_inter[t] = q'_t S,    S <- alpha_t S + beta_t k'_t^T (v'_t - k'_t S)
// with q' = q Wq_h, k' = rownorm(k Wk_h), v' = v Wv_h. A query adds o_inter to the intra-frame
// softmax branch (which the query kernel computes without its readout); a commit keeps the
// final state as S_N.
//
// Two kernels:
//  - arl2_token_project_kernel: per (batch, head, 128-token chunk), the projections on the
//    tensor cores (tcgen05, fp32 in TMEM), then one thread per token row writes q', the
//    normalised k' and v' in fp32 to scratch, head-major. The rows of q' and k' are laid out
//    in 8 parts of d/8 values, each followed by 4 padding floats, so that the scan's eight
//    lanes of a column read distinct shared-memory banks; the padding of k' part 0 carries
//    the token's alpha and beta.
//  - arl2_token_scan_kernel: every column of S evolves on its own (column j of the update
//    needs only k'_t, v'_t[j] and the gates), so a CTA takes 16 columns of one head, eight
//    lanes per column (d/8 rows of S each, in registers). Per token the lanes form k'_t S[:, j]
//    and q'_t S[:, j] from their rows and sum them with three butterfly shuffles, then update
//    their rows. The token rows come into shared memory in chunks of 32 through bulk copies
//    (three stages); a query's o_inter goes to shared memory and, per chunk, is added to the
//    intra-branch output it prefetched.
// The scan is sequential in the tokens by definition; this form is exact fp32 on the CUDA
// cores. The chunked (WY) form would move most of it to the tensor cores.
#include <algorithm>

#include "arl2_device.cuh"
#include "arl2_kernels.h"

namespace arl2 {
namespace {

// ------------------------------------------------------------------ projections
constexpr int kThreadsP = 192;
constexpr uint32_t kPWOff = 0;                  // Wq, Wk, Wv tiles
constexpr uint32_t kPXOff = 3 * kTileBytes;     // q, k, v tiles
constexpr uint32_t kPCtlOff = 6 * kTileBytes;
constexpr uint32_t kPSmem = kPCtlOff + 64;
constexpr uint32_t kPSmemAlloc = kPSmem + 1024;
static_assert(kPSmemAlloc <= 232448, "shared memory per CTA");
enum : int { kPBarLoad = 0, kPBarMma = 1, kPBarRead = 3 };   // 16..23 of the control block: TMEM slot, abort flag

__device__ __forceinline__ int part_len(int d) { return d / kTokenParts; }
__device__ __forceinline__ int padded_row(int d) { return d + 4 * kTokenParts; }

__global__ void __launch_bounds__(kThreadsP, 1)
    arl2_token_project_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_wq,
                              const __grid_constant__ CUtensorMap tm_wk, const __grid_constant__ CUtensorMap tm_wv,
                              const __grid_constant__ TokenArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* ctl = smem_raw + (base - raw) + kPCtlOff;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 20);
  const uint32_t bar_load = base + kPCtlOff + 8u * kPBarLoad, bar_mma = base + kPCtlOff + 8u * kPBarMma;
  const uint32_t bar_read = base + kPCtlOff + 8u * kPBarRead;   // the row warps are done reading TMEM
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const bool with_q = a.q_out != nullptr;
  const int ntiles = with_q ? 3 : 2;   // (q,) k, v
  const Guard g{abort_flag, a.err, a.timeout_ns};
  if (threadIdx.x == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_read, 4);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Tiles: slot 0 = q (if any), 1 = k, 2 = v; weights in the same order. TMEM: q' at 0, k' at
  // 128, v' at 256.
  const CUtensorMap* xmap[3] = {&tm_q, &tm_k, &tm_v};
  const CUtensorMap* wmap[3] = {&tm_wq, &tm_wk, &tm_wv};
  if (warp == 0) {
    if (elect_one()) {
      mbar_expect_tx(bar_load, 2u * ntiles * kTileBytes);
#pragma unroll
      for (int i = 0; i < 3; ++i)
        for (int p = 0; p < 2 && (i > 0 || with_q); ++p) {
          tma_load_3d(base + kPWOff + i * kTileBytes + p * kPanelBytes, wmap[i], bar_load, 64 * p, 0, h);
          tma_load_4d(base + kPXOff + i * kTileBytes + p * kPanelBytes, xmap[i], bar_load, 64 * p, h, chunk * kRows,
                      b);
        }
    }
    __syncwarp();
    mbar_wait_drain(bar_load, 0);
  } else if (warp == 1) {
    const bool lead = elect_one();
    if (mbar_wait_warp(bar_load, 0, g)) {
      tc_fence_after();
      constexpr uint32_t id = idesc_bf16(128, 128, false, true);   // A K-major, B MN-major
      if (lead) {
        for (int i = with_q ? 0 : 1; i < 3; ++i)
          mma8_ss<false, true>(tmem + 128u * i, desc_kmajor(base + kPXOff + i * kTileBytes, 0),
                               desc_mnmajor(base + kPWOff + i * kTileBytes, 0), id, 0u);
      }
    }
    if (lead) mma_commit(bar_mma);   // arrives once every MMA issued above has finished
    __syncwarp();
  } else {
    // Warps 2-5: thread = token row = TMEM lane of its quarter.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int t = chunk * kRows + r;
    const size_t bh = static_cast<size_t>(b) * a.H + h;
    const int d = a.d, R = part_len(d), P = padded_row(d);
    const bool ok = mbar_wait_warp(bar_mma, 0, g);
    tc_fence_after();
    if (ok) {
      for (int i = with_q ? 0 : 1; i < 3; ++i) {
        uint32_t x[4][32];
        tmem_ld32x2_wait(tmem + lane_off + 128u * i, x[0], tmem + lane_off + 128u * i + 32u, x[1]);
        tmem_ld32x2_wait(tmem + lane_off + 128u * i + 64u, x[2], tmem + lane_off + 128u * i + 96u, x[3]);
        if (t >= a.T) continue;
        float scale = 1.f;
        if (i == 1) {   // k' = k Wk / max(|k Wk|, 1e-12)
          float ss0 = 0.f, ss1 = 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float u0 = __uint_as_float(x[c][e]), u1 = __uint_as_float(x[c][e + 1]);
              ss0 = fmaf(u0, u0, ss0);
              ss1 = fmaf(u1, u1, ss1);
            }
          scale = 1.f / fmaxf(sqrtf(ss0 + ss1), 1e-12f);
        }
        if (i == 2) {   // v': plain rows of d
          float* dst = a.v_out + (bh * a.T + t) * d;
#pragma unroll
          for (int j = 0; j < kDP; j += 4)
            if (j < d)
              *reinterpret_cast<float4*>(dst + j) =
                  make_float4(__uint_as_float(x[j >> 5][j & 31]), __uint_as_float(x[j >> 5][(j & 31) + 1]),
                              __uint_as_float(x[j >> 5][(j & 31) + 2]), __uint_as_float(x[j >> 5][(j & 31) + 3]));
        } else {        // q', k': 8 parts of R values, each followed by 4 padding floats
          float* dst = (i == 0 ? a.q_out : a.k_out) + (bh * a.T + t) * P;
#pragma unroll
          for (int j = 0; j < kDP; j += 4) {
            if (j >= d) break;
            const int part = j / R, o = part * (R + 4) + (j - part * R);
            *reinterpret_cast<float4*>(dst + o) = make_float4(
                scale * __uint_as_float(x[j >> 5][j & 31]), scale * __uint_as_float(x[j >> 5][(j & 31) + 1]),
                scale * __uint_as_float(x[j >> 5][(j & 31) + 2]), scale * __uint_as_float(x[j >> 5][(j & 31) + 3]));
          }
          if (i == 1) {   // the token's gates ride in the padding of part 0
            const size_t gt = bh * a.T + t;
            *reinterpret_cast<float2*>(dst + R) = make_float2(a.alpha[gt], a.beta[gt]);
          }
        }
      }
    }
  }
  __syncwarp();   // rows past T and the producer's drains split warps: one arrival per warp
  tc_fence_before();
  if (warp >= 2) warp_arrive(bar_read);   // every TMEM read of this warp is done
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    mbar_wait_drain(bar_mma, 0);
    mbar_wait_drain(bar_read, 0);
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ scan
constexpr int kScanThreads = 128;
constexpr int kScanCols = kScanThreads / kTokenParts;   // 16 columns of S per CTA
constexpr int kChunk = 32;                              // tokens per stage
constexpr int kScanStages = 3;
constexpr int kMaxPart = kDP / kTokenParts;             // rows of S per lane, at most (16)
constexpr int kMaxPadded = kDP + 4 * kTokenParts;       // 160 floats per padded row
constexpr uint32_t kStageK = kChunk * kMaxPadded * 4;
constexpr uint32_t kStageV = kChunk * kDP * 4;
constexpr uint32_t kStageBytes = 2 * kStageK + kStageV;   // k', q', v'
constexpr uint32_t kOInterOff = kScanStages * kStageBytes;   // [kChunk][kScanCols] fp32
constexpr uint32_t kScanCtl = kOInterOff + kChunk * kScanCols * 4;
constexpr uint32_t kScanSmem = kScanCtl + 64;
static_assert(kScanSmem <= 232448, "shared memory per CTA");
static_assert(kChunk == 4 * 8, "the o prefetch maps 4 tokens to each of 8 thread rows");

template <int R>
__device__ __forceinline__ void scan_chunk(const TokenArgs& a, const float* ks, const float* qs, const float* vs,
                                           float* oi, int ntok, int col, int lc, int part, bool with_q,
                                           float (&s)[kMaxPart]) {
  const int P = padded_row(a.d);
  for (int tt = 0; tt < ntok; ++tt) {
    const float* kr = ks + tt * P;
    const float4* k4 = reinterpret_cast<const float4*>(kr + part * (R + 4));
    float k[R];
#pragma unroll
    for (int j = 0; j < R / 4; ++j) {
      const float4 x = k4[j];
      k[4 * j] = x.x;
      k[4 * j + 1] = x.y;
      k[4 * j + 2] = x.z;
      k[4 * j + 3] = x.w;
    }
    float kd0 = 0.f, kd1 = 0.f;
#pragma unroll
    for (int i = 0; i < R; i += 2) {
      kd0 = fmaf(k[i], s[i], kd0);
      kd1 = fmaf(k[i + 1], s[i + 1], kd1);
    }
    float kd = kd0 + kd1;
    float qd = 0.f;
    if (with_q) {
      const float4* q4 = reinterpret_cast<const float4*>(qs + tt * P + part * (R + 4));
      float qd0 = 0.f, qd1 = 0.f;
#pragma unroll
      for (int j = 0; j < R / 4; ++j) {
        const float4 x = q4[j];
        qd0 = fmaf(x.x, s[4 * j], qd0);
        qd1 = fmaf(x.y, s[4 * j + 1], qd1);
        qd0 = fmaf(x.z, s[4 * j + 2], qd0);
        qd1 = fmaf(x.w, s[4 * j + 3], qd1);
      }
      qd = qd0 + qd1;
    }
    // Sum over the column's eight lanes (adjacent lanes, butterfly: every lane gets the sum).
#pragma unroll
    for (int m = 1; m < kTokenParts; m <<= 1) {
      kd += __shfl_xor_sync(0xffffffffu, kd, m);
      if (with_q) qd += __shfl_xor_sync(0xffffffffu, qd, m);
    }
    if (with_q && part == 0) oi[tt * kScanCols + lc] = qd;   // read before this token's update
    const float2 ab = *reinterpret_cast<const float2*>(kr + R);   // alpha_t, beta_t
    const float bu = ab.y * (vs[tt * a.d + col] - kd);
#pragma unroll
    for (int i = 0; i < R; ++i) s[i] = fmaf(bu, k[i], ab.x * s[i]);
  }
}

__global__ void __launch_bounds__(kScanThreads, 1) arl2_token_scan_kernel(const __grid_constant__ TokenArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* oi = reinterpret_cast<float*>(smem_raw + kOInterOff);
  uint8_t* ctl = smem_raw + kScanCtl;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 8 * kScanStages);
  const uint32_t bar0 = smem_u32(ctl);
  const int lc = threadIdx.x / kTokenParts;   // column within the CTA
  const int part = threadIdx.x % kTokenParts;
  const int col = blockIdx.x * kScanCols + lc;
  const int h = blockIdx.y, b = blockIdx.z;
  const size_t bh = static_cast<size_t>(b) * a.H + h;
  const int d = a.d, R = part_len(d), P = padded_row(d);
  const bool with_q = a.q_out != nullptr;
  const Guard g{abort_flag, a.err, a.timeout_ns};
  const int nchunks = (a.T + kChunk - 1) / kChunk;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kScanStages; ++i) mbar_init(bar0 + 8 * i, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  auto stage_ptr = [&](int st) { return smem_raw + st * kStageBytes; };
  auto issue = [&](int ci) {   // chunk ci into stage ci % kScanStages (thread 0)
    const int st = ci % kScanStages, t0 = ci * kChunk, n = min(kChunk, a.T - t0);
    const uint32_t bar = bar0 + 8 * st;
    const uint32_t kb = static_cast<uint32_t>(n * P * 4), vb = static_cast<uint32_t>(n * d * 4);
    mbar_expect_tx(bar, kb * (with_q ? 2u : 1u) + vb);
    uint8_t* sp = stage_ptr(st);
    bulk_load(smem_u32(sp), a.k_out + (bh * a.T + t0) * P, kb, bar);
    if (with_q) bulk_load(smem_u32(sp + kStageK), a.q_out + (bh * a.T + t0) * P, kb, bar);
    bulk_load(smem_u32(sp + 2 * kStageK), a.v_out + (bh * a.T + t0) * d, vb, bar);
  };
  if (threadIdx.x == 0)
    for (int ci = 0; ci < min(kScanStages, nchunks); ++ci) issue(ci);

  // This lane's rows of column col of S_{N-1}.
  float s[kMaxPart];
#pragma unroll
  for (int i = 0; i < kMaxPart; ++i) s[i] = i < R ? a.S_old[bh * d * d + static_cast<size_t>(part * R + i) * d + col] : 0.f;

  // The o elements this thread adds o_inter to, per chunk: column lc2, tokens tr + 8j.
  const int lc2 = threadIdx.x % kScanCols, tr = threadIdx.x / kScanCols;
  const int ocol = blockIdx.x * kScanCols + lc2;
  int issued = min(kScanStages, nchunks);
  bool alive = true;
  for (int ci = 0; ci < nchunks && alive; ++ci) {
    const int st = ci % kScanStages, t0 = ci * kChunk, n = min(kChunk, a.T - t0);
    uint16_t ov[4] = {0, 0, 0, 0};
    if (with_q) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int t = t0 + tr + 8 * j;
        if (t < a.T) ov[j] = a.o[((static_cast<size_t>(b) * a.T + t) * a.H + h) * d + ocol];
      }
    }
    // The whole CTA agrees on the outcome, so that every thread takes the same barriers.
    if (!__syncthreads_and(mbar_wait(bar0 + 8 * st, (ci / kScanStages) & 1, g))) {
      alive = false;
      break;
    }
    const uint8_t* sp = stage_ptr(st);
    const float* ks = reinterpret_cast<const float*>(sp);
    const float* qs = reinterpret_cast<const float*>(sp + kStageK);
    const float* vs = reinterpret_cast<const float*>(sp + 2 * kStageK);
    if (R == 16) scan_chunk<16>(a, ks, qs, vs, oi, n, col, lc, part, with_q, s);
    else if (R == 8) scan_chunk<8>(a, ks, qs, vs, oi, n, col, lc, part, with_q, s);
    else scan_chunk<4>(a, ks, qs, vs, oi, n, col, lc, part, with_q, s);
    __syncthreads();   // every lane is done with the stage, and o_inter of the chunk is in oi
    if (issued < nchunks) {   // the stage just freed takes the next chunk
      if (threadIdx.x == 0) issue(issued);
      ++issued;
    }
    if (with_q) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int tt = tr + 8 * j, t = t0 + tt;
        if (t < a.T) {
          const float x = __uint_as_float(static_cast<uint32_t>(ov[j]) << 16) + oi[tt * kScanCols + lc2];
          __nv_bfloat16 y = __float2bfloat16_rn(x);
          a.o[((static_cast<size_t>(b) * a.T + t) * a.H + h) * d + ocol] = *reinterpret_cast<uint16_t*>(&y);
        }
      }
      __syncthreads();   // oi is rewritten by the next chunk
    }
  }
  if (!with_q && alive) {   // the commit: the final state is S_N
#pragma unroll
    for (int i = 0; i < kMaxPart; ++i)
      if (i < R) {
        const size_t o = bh * d * d + static_cast<size_t>(part * R + i) * d + col;
        a.S_new[o] = s[i];
        __nv_bfloat16 y = __float2bfloat16_rn(s[i]);
        a.S_new_bf16[o] = *reinterpret_cast<uint16_t*>(&y);
      }
  }
  // Every copy issued must land before the CTA exits (matters only after an abort). The last
  // kScanStages chunks issued are the latest loads of their stages.
  if (threadIdx.x == 0)
    for (int ci = max(0, issued - kScanStages); ci < issued; ++ci)
      mbar_wait_drain(bar0 + 8 * (ci % kScanStages), (ci / kScanStages) & 1);
}

}  // namespace

size_t token_scratch_floats(int B, int H, int T, int d) {
  return static_cast<size_t>(B) * H * T * (2 * (d + 4 * kTokenParts) + d);
}

cudaError_t token_setup() {
  cudaError_t e = cudaFuncSetAttribute(arl2_token_project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kPSmemAlloc));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(arl2_token_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kScanSmem));
}

cudaError_t launch_token_project(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                 const CUtensorMap& tm_wq, const CUtensorMap& tm_wk, const CUtensorMap& tm_wv,
                                 const TokenArgs& a, cudaStream_t stream) {
  const dim3 grid((a.T + kRows - 1) / kRows, a.H, a.B);
  arl2_token_project_kernel<<<grid, kThreadsP, kPSmemAlloc, stream>>>(tm_q, tm_k, tm_v, tm_wq, tm_wk, tm_wv, a);
  return cudaGetLastError();
}

cudaError_t launch_token_scan(const TokenArgs& a, cudaStream_t stream) {
  if (a.d % (4 * kTokenParts) != 0 || a.d > kDP) return cudaErrorInvalidValue;
  const dim3 grid(a.d / kScanCols, a.H, a.B);
  arl2_token_scan_kernel<<<grid, kScanThreads, kScanSmem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace arl2
