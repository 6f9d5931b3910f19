// Row passes of the commit chain ("Attend Locally, Remember Linearly", technical summary of
// arXiv 2605.16579, §2.1 state update), shared by the commit kernel and the commit CTAs of
// the fused clean pass. The calling thread owns token row r of a 128-token chunk, which is
// TMEM lane r; taddr already carries the lane offset of the warp's lane quarter.
#pragma once

#include "arl2_device.cuh"

namespace arl2 {

constexpr float kCommitNormEps = 1e-12f;

// K' = Kp / max(|Kp|, eps) -> bf16, row r of the swizzled K tile (the K projection of the
// chunk is in TMEM at taddr, 128 fp32 columns). Sums of squares and the scaling run on paired
// fp32 operations with independent accumulators, so the row's dependent chains stay short.
__device__ __forceinline__ void commit_rows_normalise(uint32_t taddr, uint32_t tile, uint32_t r) {
  uint32_t kv[4][32];
  tmem_ld32x2_wait(taddr, kv[0], taddr + 32u, kv[1]);
  tmem_ld32x2_wait(taddr + 64u, kv[2], taddr + 96u, kv[3]);
  float2 ss[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) ss[j] = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const float2 x = make_float2(__uint_as_float(kv[c][e]), __uint_as_float(kv[c][e + 1]));
      ss[(e >> 1) & 3] = __ffma2_rn(x, x, ss[(e >> 1) & 3]);
    }
  const float2 s01 = __fadd2_rn(__fadd2_rn(ss[0], ss[1]), __fadd2_rn(ss[2], ss[3]));
  const float inv = 1.f / fmaxf(sqrtf(s01.x + s01.y), kCommitNormEps);
  const float2 inv2 = make_float2(inv, inv);
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t* x = kv[c] + 8 * q;
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 y = __fmul2_rn(make_float2(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1])), inv2);
        w[e] = pack_bf16x2(y.x, y.y);
      }
      st_shared_v4(tile + swz_chunk(r, 4 * c + q), w[0], w[1], w[2], w[3]);
    }
}

// R = (V' - K'S) * coef -> bf16, row r of the swizzled V tile, with coef = beta_t / T (zero for
// rows past T). The residual is in TMEM at taddr, 128 fp32 columns.
__device__ __forceinline__ void commit_rows_residual(uint32_t taddr, uint32_t tile, uint32_t r, float coef) {
  const float2 cf = make_float2(coef, coef);
  uint32_t vp[2][32];
#pragma unroll
  for (int c2 = 0; c2 < 2; ++c2) {
    tmem_ld32x2_wait(taddr + 64u * c2, vp[0], taddr + 64u * c2 + 32u, vp[1]);
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 y = __fmul2_rn(
              make_float2(__uint_as_float(vp[c][8 * q + 2 * e]), __uint_as_float(vp[c][8 * q + 2 * e + 1])), cf);
          w[e] = pack_bf16x2(y.x, y.y);
        }
        st_shared_v4(tile + swz_chunk(r, 4 * (2 * c2 + c) + q), w[0], w[1], w[2], w[3]);
      }
  }
}

}  // namespace arl2
