// Internal (C++) interface between the C-ABI layer and the kernels. Not part of the
// public boundary, which is include/arl2.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace arl2 {

constexpr unsigned int kErrTimeoutBit = 1u;  // device error word: a bounded wait ran out
constexpr unsigned int kErrLayoutBit = 2u;   // device error word: shared memory not laid out as required

// One query pass (and the growing-KV-cache baseline, which shares the main loop).
struct QueryArgs {
  uint16_t* o;            // [B, T, H, d] bf16 output
  int T;                  // query rows per (batch, head)
  int kv_len;             // keys attended per (batch, head)
  int B, H, d;
  int state_slot;         // which state buffer (0 or 1) the readout uses
  float scale_log2;       // log2(e) / sqrt(d)
  unsigned int* err;      // device error word
  unsigned long long timeout_ns;
  int stall;              // test hook: the softmax threads wait on a barrier nothing signals
  // Persistent stream-K split (see QueryPlan) and its scratch.
  int nq, nkv;            // query tiles and key tiles per (batch, head)
  long long units;        // B * H * nq * nkv (query tile, key tile) pairs
  int num_ctas;           // CTAs of the split
  int first_cta;          // the split's CTAs are blockIdx.x in [first_cta, first_cta + num_ctas)
  int max_segs;           // CTAs sharing one query tile, at most
  int head_w;             // extra weight of a query tile's key tile 0 in the split (quarter units)
  float* part_o;          // [qtiles * max_segs][32 column quads][128 rows] float4: partial O accumulators
  float* part_ml;         // [qtiles * max_segs, 2, 128] running max (log2 units) and sum
  int* flags;             // [qtiles * max_segs] record-published flags, set to the launch's epoch
  int epoch;              // nonzero, different from the previous launch on the same flags
};

// The stream-K split of one query launch. Units are weighted: 4 for a (query tile, key tile)
// pair, 4 + head_w for key tile 0, whose segment also computes the readout and finishes the
// tile; CTA c takes the units whose weighted start lies in [c W / P, (c + 1) W / P), W the
// total weight (see split_start).
struct QueryPlan {
  int nq, nkv, num_ctas, max_segs, head_w;
  long long units, qtiles;
};
// Weighted split of `units` (query tile, key tile) units, nkv per query tile, over P CTAs: the
// first unit of CTA c (c = P gives units), and the CTA that holds unit u. Host and device
// share these two functions, so the plan and the kernels agree on every boundary.
__host__ __device__ inline long long split_start(long long c, long long units, int nkv, int head_w, int P) {
  const long long wt = 4ll * nkv + head_w;   // weight of one query tile
  const long long wc = c * ((units / nkv) * wt) / P;
  const long long k = wc / wt, r = wc - k * wt;
  if (r == 0) return k * nkv;
  const long long j = r > head_w ? (r - head_w + 3) / 4 : 1;   // W(k nkv + j) = k wt + head_w + 4 j >= wc
  return k * nkv + (j > 1 ? j : 1);
}
__host__ __device__ inline int split_owner(long long u, long long units, int nkv, int head_w, int P) {
  const long long wtot = (units / nkv) * (4ll * nkv + head_w);
  const long long w = 4 * u + static_cast<long long>(head_w) * ((u + nkv - 1) / nkv);   // weight before unit u
  return static_cast<int>(((w + 1) * P - 1) / wtot);
}
QueryPlan plan_query(int B, int H, int T, int kv_len, int num_sms);
size_t query_scratch_floats(const QueryPlan& p);   // part_o + part_ml
size_t query_flag_count(const QueryPlan& p);       // flags

// One commit: per (group of 128-token chunks, head, batch) CTA; the groups of a (batch, head)
// form a cluster that reduces U in distributed shared memory.
struct CommitArgs {
  const float* alpha;     // [B, H, T]
  const float* beta;      // [B, H, T]
  int T, B, H, d;
  int chunks_per_group, ngroups;
  int state_slot;         // state buffer read (S_{N-1})
  float inv_T;
  unsigned int* err;
  unsigned long long timeout_ns;
};

// The commit's output side: S_N = abar * S_{N-1} + sum of the groups' U, fp32 plus its
// bf16 copy. Each group writes its U and alpha sum to its own scratch slot; after one
// cluster barrier each CTA sums its block of columns over the groups in a fixed order.
struct ReduceArgs {
  const float* S_old;     // [B*H, d, d]
  float* S_new;           // [B*H, d, d]
  uint16_t* S_new_bf16;   // [B*H, d, d]
  float* part_u;          // [B*H*ngroups][32 column quads][128 rows] float4 partial U
  float* part_alpha;      // [B*H*ngroups] alpha sums
  int d;
  float inv_T;
};

// The fused clean pass (arl2_clean.cu): one launch whose first CTAs run the commit as a
// stream over the B*H*nchunks chunk units, cut into num_ctas contiguous ranges, and whose
// other CTAs run the query's stream-K split (QueryArgs, first_cta = the commit CTAs). A head
// whose chunks span several CTAs is reduced by its last-arriving segment from per-segment
// scratch slots.
struct CommitStreamArgs {
  const float* alpha;     // [B, H, T]
  const float* beta;      // [B, H, T]
  const float* S_old;     // [B*H, d, d] fp32 S_{N-1}
  float* S_new;           // [B*H, d, d] fp32 S_N
  uint16_t* S_new_bf16;   // [B*H, d, d] its bf16 copy
  float* part_u;          // [B*H*max_pieces][32 column quads][128 rows] float4 partial U
  float* part_alpha;      // [B*H*max_pieces] alpha sums of the segments
  unsigned int* counters; // [B*H] segments arrived, wrapping at the head's segment count
  int T, B, H, d;
  int state_slot;         // state buffer read (S_{N-1}), for the bf16 copy's tensor map
  float inv_T;
  int nchunks;            // 128-token chunks per (batch, head)
  long long units;        // B * H * nchunks
  int num_ctas;           // the commit CTAs are blockIdx.x in [0, num_ctas)
  int max_pieces;         // segments of one head, at most (scratch slots per head)
  unsigned int* err;
  unsigned long long timeout_ns;
};
struct CleanPlan {
  QueryPlan q;            // the query CTAs' split
  int commit_ctas;        // commit CTAs
  int nchunks;
  long long cunits;       // chunk units
  int max_pieces;
};
// commit_ctas = 0 picks the split from a cost model; otherwise that many commit CTAs (clamped
// to [1, chunk units] and to leave at least one query CTA).
CleanPlan plan_clean(int B, int H, int T, int num_sms, int commit_ctas);
size_t clean_scratch_floats(const CleanPlan& p);   // part_u, then part_alpha
cudaError_t clean_setup();
cudaError_t launch_clean(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                         const CUtensorMap& tm_wq, const CUtensorMap& tm_s, const CUtensorMap& tm_o,
                         const CUtensorMap& tm_wk, const CUtensorMap& tm_wv, const QueryArgs& qa,
                         const CommitStreamArgs& ca, cudaStream_t stream, bool dependent);

// Token-level access (arl2_token.cu): projections to scratch, then the per-token scan.
constexpr int kTokenParts = 8;   // lanes per column of S in the scan; rows of q', k' come in 8 parts
struct TokenArgs {
  const float* alpha;     // [B, H, T]
  const float* beta;      // [B, H, T]
  float* q_out;           // [B*H, T, d + 32] q' (padded parts); null for a commit
  float* k_out;           // [B*H, T, d + 32] k' normalised (padded parts; part 0's padding holds alpha, beta)
  float* v_out;           // [B*H, T, d] v'
  const float* S_old;     // [B*H, d, d] fp32 S_{N-1}
  float* S_new;           // [B*H, d, d] the final state (commit only)
  uint16_t* S_new_bf16;   // its bf16 copy
  uint16_t* o;            // [B, T, H, d] bf16: holds the intra branch; the scan adds o_inter (query only)
  int T, B, H, d;
  unsigned int* err;
  unsigned long long timeout_ns;
};
size_t token_scratch_floats(int B, int H, int T, int d);
cudaError_t token_setup();
cudaError_t launch_token_project(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                 const CUtensorMap& tm_wq, const CUtensorMap& tm_wk, const CUtensorMap& tm_wv,
                                 const TokenArgs& a, cudaStream_t stream);
cudaError_t launch_token_scan(const TokenArgs& a, cudaStream_t stream);

// Gates produced from the hidden state (arl2_gates.cu): alpha, beta [B, H, T] fp32 from
// x [B, T, D] bf16 and the stacked projections Wg = [Wa; Wb] of 2H rows plus a bias of 2H.
constexpr int kMaxGateCols = 64;   // 2H rounded up to 16 is at most this (H <= 32)
struct GateArgs {
  const float* bias;      // [2H]: ba then bb
  float* alpha;           // [B, H, T]
  float* beta;            // [B, H, T]
  int B, T, H, D;
  int ngates;             // 2H
  int ncols;              // 2H rounded up to 16: the MMA's N and the Wg box rows
  int tmem_cols;          // TMEM columns allocated (a power of two, at least 32)
  unsigned int* err;
  unsigned long long timeout_ns;
};
int gate_split(int D);   // CTAs per cluster (slices of D)
cudaError_t gates_setup();
cudaError_t launch_gates(const CUtensorMap& tm_x, const CUtensorMap& tm_w, const GateArgs& a, cudaStream_t stream);

// Helpers defined in arl2_api.cu: device check and set-up (returns an arl2_status), and
// the bf16 tensor maps every kernel reads through.
int prepare_device(int* dev, int* sms);
bool encode_act_map(CUtensorMap* m, const void* ptr, int B, int L, int H, int d);
bool encode_mat_map(CUtensorMap* m, const void* ptr, int n, int d);

size_t query_smem_bytes();
size_t commit_smem_bytes();
// The commit's work split: 128-token chunks in groups, one CTA per group; the groups of one
// (batch, head) form one cluster (at most 8 CTAs) and no group is empty.
void commit_split(int T, int H, int B, int sms, int* chunks_per_group, int* ngroups);
// Scratch of one commit launch (part_u, then part_alpha), in floats.
size_t commit_scratch_floats(int B, int H, int ngroups);
cudaError_t query_setup();   // per-device function attributes
cudaError_t commit_setup();

// dependent: launch as a programmatic dependent of the preceding kernel in the stream. The
// kernel reads its inputs before that kernel completes, so the caller must know that the
// preceding kernel does not write them.
cudaError_t launch_query(bool hybrid, const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                         const CUtensorMap& tm_w, const CUtensorMap& tm_s, const CUtensorMap& tm_o, const QueryArgs& a,
                         cudaStream_t stream, bool dependent);
cudaError_t launch_commit(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_wk,
                          const CUtensorMap& tm_wv, const CUtensorMap& tm_s, const CommitArgs& a,
                          const ReduceArgs& r, cudaStream_t stream, bool dependent);
// fp32 state -> state buffer (skipped when S is null) + bf16 copy.
cudaError_t launch_state_import(const float* src, float* S, uint16_t* S_bf16, size_t n, cudaStream_t stream);

}  // namespace arl2
