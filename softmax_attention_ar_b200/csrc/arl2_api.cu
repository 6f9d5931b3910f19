// C-ABI layer of the ARL2 library: contexts, argument checks, TMA descriptors, state
// ping-pong and launches. The computation itself lives in arl2_query.cu and arl2_commit.cu.
#include <algorithm>
#include <initializer_list>
#include <utility>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/arl2.h"
#include "arl2_kernels.h"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A bf16 tensor map with 128-byte swizzle and 64-element-wide boxes; out-of-range elements
// read as zero (this is how head dims below 128 and ragged token tails are padded).
bool make_map(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims, const cuuint64_t* strides_bytes,
              const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), dims, strides_bytes, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [B, L, H, d] token-major activations: dims (d, H, L, B), box (64, 1, rows, 1); loads use
// 128-row boxes, the query's output stores 32-row boxes (one per warp).
bool make_act_map(CUtensorMap* m, const void* ptr, int B, int L, int H, int d, int rows = 128) {
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
  const cuuint64_t str[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)L * H * d * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  return make_map(m, ptr, 4, dims, str, box);
}

// [n, d, d] row-major square matrices: dims (d, d, n), box (64, 128, 1).
bool make_mat_map(CUtensorMap* m, const void* ptr, int n, int d) {
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)d, (cuuint64_t)n};
  const cuuint64_t str[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * d * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  return make_map(m, ptr, 3, dims, str, box);
}

// [B, T, D] hidden states: dims (D, T, B), box (64, 128, 1).
bool make_hidden_map(CUtensorMap* m, const void* ptr, int B, int T, int D) {
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)T * D * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  return make_map(m, ptr, 3, dims, str, box);
}

// [rows, D] gate projections: dims (D, rows), box (64, box_rows); rows past `rows` read as zero.
bool make_gate_map(CUtensorMap* m, const void* ptr, int rows, int D, int box_rows) {
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t str[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  return make_map(m, ptr, 2, dims, str, box);
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Small cache of activation maps keyed by base pointer: callers usually reuse buffers.
struct MapCache {
  static constexpr int kSlots = 64;
  explicit MapCache(int box_rows = 128) : rows(box_rows) {}
  int rows;                       // box rows of the maps this cache makes
  const void* ptr[kSlots] = {};
  CUtensorMap map[kSlots];
  int next = 0;
  const CUtensorMap* get(const void* p, int B, int L, int H, int d) {
    for (int i = 0; i < kSlots; ++i)
      if (ptr[i] == p) return &map[i];
    const int i = next;
    next = (next + 1) % kSlots;
    ptr[i] = nullptr;
    if (!make_act_map(&map[i], p, B, L, H, d, rows)) return nullptr;
    ptr[i] = p;
    return &map[i];
  }
};

// Outputs of the most recent query launches, per stream, process-wide. A query or commit may
// run as a programmatic dependent of the previous kernel in its stream only if its inputs do
// not overlap the output of the query launched last on that stream (chained layers).
struct LastOut {
  cudaStream_t stream = nullptr;
  uintptr_t begin = 0, end = 0;
  bool used = false;
};
std::mutex g_lastout_mu;
LastOut g_lastout[16];

// Whether every (pointer, bytes) range is clear of the output of the last query launched on
// stream st.
bool clear_of_last_output(cudaStream_t st, std::initializer_list<std::pair<const void*, size_t>> ranges) {
  std::lock_guard<std::mutex> lk(g_lastout_mu);
  for (const auto& e : g_lastout) {
    if (!e.used || e.stream != st) continue;
    for (const auto& r : ranges) {
      const uintptr_t b = reinterpret_cast<uintptr_t>(r.first), end = b + r.second;
      if (b < e.end && e.begin < end) return false;
    }
  }
  return true;
}

// Record o as the last query output on stream st.
void record_query_output(cudaStream_t st, const void* o, size_t bytes) {
  std::lock_guard<std::mutex> lk(g_lastout_mu);
  LastOut* slot = nullptr;
  for (auto& e : g_lastout)
    if (e.used && e.stream == st) slot = &e;
  for (auto& e : g_lastout)
    if (!slot && !e.used) slot = &e;
  if (!slot) slot = &g_lastout[reinterpret_cast<uintptr_t>(st) % 16];
  slot->used = true;
  slot->stream = st;
  slot->begin = reinterpret_cast<uintptr_t>(o);
  slot->end = slot->begin + bytes;
}

std::mutex g_setup_mu;
bool g_setup_done[64] = {};

cudaError_t device_setup(int dev) {
  std::lock_guard<std::mutex> lk(g_setup_mu);
  if (dev >= 0 && dev < 64 && g_setup_done[dev]) return cudaSuccess;
  cudaError_t e = arl2::query_setup();
  if (e == cudaSuccess) e = arl2::commit_setup();
  if (e == cudaSuccess) e = arl2::clean_setup();
  if (e == cudaSuccess) e = arl2::token_setup();
  if (e == cudaSuccess) e = arl2::gates_setup();
  if (e == cudaSuccess && dev >= 0 && dev < 64) g_setup_done[dev] = true;
  return e;
}

arl2_status check_device(int* dev, int* sms) {
  if (cudaGetDevice(dev) != cudaSuccess) return ARL2_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess ||
      cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess)
    return ARL2_ERR_CUDA;
  if (major != 10 || minor != 0) return ARL2_ERR_UNSUPPORTED;
  if (!encode_fn()) return ARL2_ERR_CUDA;
  if (device_setup(*dev) != cudaSuccess) return ARL2_ERR_CUDA;
  return ARL2_OK;
}

constexpr unsigned long long kDefaultTimeoutNs = 1000000000ull;

}  // namespace

// Entry points for other translation units of the library (the allocation-free commit).
namespace arl2 {
int prepare_device(int* dev, int* sms) { return static_cast<int>(check_device(dev, sms)); }
bool encode_act_map(CUtensorMap* m, const void* ptr, int B, int L, int H, int d) {
  return make_act_map(m, ptr, B, L, H, d);
}
bool encode_mat_map(CUtensorMap* m, const void* ptr, int n, int d) { return make_mat_map(m, ptr, n, d); }
}  // namespace arl2

struct arl2_ctx {
  int B = 0, H = 0, T = 0, d = 0;
  int device = 0, num_sms = 0;
  int chunks_per_group = 1, ngroups = 1;
  uint16_t* W[3] = {};            // phi_q, phi_k, phi_v copies, [H, d, d]
  float* S[2] = {};               // fp32 state buffers, [B, H, d, d]
  uint16_t* S_bf16 = nullptr;     // [2][B, H, d, d] bf16 copies of S[0], S[1]
  unsigned int* err = nullptr;
  // Host-buffer calls: two staging sets, used by turns, so that the copy of one call's inputs
  // (on s_in) overlaps the previous call's kernel (on the caller's stream) and its output
  // copy (on s_out). ev_in[s]: set s's inputs landed; ev_used[s]: the kernel that read set
  // s is done; ev_out[s]: set s's output has been copied out.
  uint16_t* stage_bf16[2][4] = {};   // q, k, v, o
  float* stage_f32[2][2] = {};       // alpha, beta
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev_in[2] = {}, ev_used[2] = {}, ev_out[2] = {};
  unsigned host_turn = 0;
  arl2::QueryPlan qplan{};        // stream-K split of the query kernel
  float* cscratch = nullptr;      // the commit's per-group partial U and alpha sums
  arl2::CleanPlan cplan{};        // split of the fused clean pass
  float* clscratch = nullptr;     // its commit segments' partial U and alpha sums
  size_t clscratch_floats = 0;
  unsigned int* clcounters = nullptr;   // its per-(batch, head) arrival counters
  size_t qscratch_floats = 0;     // query scratch and flags, sized for both query splits
  size_t qflag_count = 0;
  float* tscratch = nullptr;      // token-level access: q', k', v' of one pass (fp32)
  // Gates produced from the hidden state (only when 2H <= kMaxGateCols): Wg = [Wa; Wb] bf16
  // [2H, D], its bias [2H] and the gates of the last gated commit, alpha then beta [B, H, T].
  uint16_t* Wg = nullptr;
  float* bg = nullptr;
  float* gate_buf = nullptr;
  bool gates_set = false;
  CUtensorMap tm_wg;
  float* qscratch = nullptr;      // its partial records
  int* qflags = nullptr;          // their published flags
  int qepoch = 0;                 // epoch of the last query launch
  int cur = 0;                    // buffer holding S_{N-1}
  int frame = 0;
  bool maps_set = false;
  bool stall_next = false;        // failure-detection test hook (next query only)
  bool overlap = false;           // calls may start behind the previous kernel (see the header)
  unsigned long long timeout_ns = kDefaultTimeoutNs;
  CUtensorMap tm_w[3];
  CUtensorMap tm_s;
  MapCache acts;
  MapCache outs{32};              // output maps (32-row store boxes)
  size_t bytes = 0;

  size_t act_elems() const { return (size_t)B * T * H * d; }
  size_t state_elems() const { return (size_t)B * H * d * d; }
};

struct arl2_kvcache {
  int B = 0, H = 0, T = 0, d = 0, max_frames = 0;
  int n = 0;
  int device = 0;
  uint16_t* K = nullptr;   // [B, max_frames*T, H, d]
  uint16_t* V = nullptr;
  unsigned int* err = nullptr;
  CUtensorMap tm_k, tm_v;
  MapCache acts;
  MapCache outs{32};
  size_t bytes = 0;
  unsigned long long timeout_ns = kDefaultTimeoutNs;
  int num_sms = 0;
  float* qscratch = nullptr;      // stream-K partial records, sized for the longest cache
  size_t qscratch_floats = 0;
  int* qflags = nullptr;          // record flags, sized for the longest cache
  size_t qflag_count = 0;
  int qepoch = 0;
};

namespace {

// Gates produced from the hidden state: 2H projection rows, rounded up to 16 for the MMA.
int gate_cols(int H) { return (2 * H + 15) / 16 * 16; }
bool gates_supported(int H, int D) { return gate_cols(H) <= arl2::kMaxGateCols && D % 8 == 0; }

// Launch the gate producer: alpha, beta [B, H, T] from x [B, T, D] (the context's Wg, bg).
arl2_status gates_impl(arl2_ctx* c, const void* x, float* alpha, float* beta, cudaStream_t st);

// Point a query launch at its stream-K plan and scratch.
// Epochs of successive launches on one set of flags: nonzero, never the previous one.
int next_epoch(int* e) {
  *e = (*e == 0x7fffffff) ? 1 : *e + 1;
  return *e;
}

void set_plan(arl2::QueryArgs* a, const arl2::QueryPlan& p, float* scratch, int* flags, int epoch) {
  a->nq = p.nq;
  a->nkv = p.nkv;
  a->units = p.units;
  a->num_ctas = p.num_ctas;
  a->max_segs = p.max_segs;
  a->head_w = p.head_w;
  const size_t slots = static_cast<size_t>(p.qtiles) * p.max_segs;
  a->part_o = scratch;
  a->part_ml = scratch + slots * 128 * 128;
  a->flags = flags;
  a->epoch = epoch;
}

template <typename T>
bool dev_alloc(T** p, size_t count, size_t* total) {
  if (cudaMalloc(reinterpret_cast<void**>(p), count * sizeof(T)) != cudaSuccess) {
    *p = nullptr;
    return false;
  }
  *total += count * sizeof(T);
  return true;
}

void free_ctx(arl2_ctx* c) {
  if (!c) return;
  for (auto& p : c->W) cudaFree(p);
  for (auto& p : c->S) cudaFree(p);
  cudaFree(c->S_bf16);
  cudaFree(c->err);
  for (auto& set : c->stage_bf16)
    for (auto& p : set) cudaFree(p);
  for (auto& set : c->stage_f32)
    for (auto& p : set) cudaFree(p);
  for (int i = 0; i < 2; ++i) {
    if (c->ev_in[i]) cudaEventDestroy(c->ev_in[i]);
    if (c->ev_used[i]) cudaEventDestroy(c->ev_used[i]);
    if (c->ev_out[i]) cudaEventDestroy(c->ev_out[i]);
  }
  if (c->s_in) cudaStreamDestroy(c->s_in);
  if (c->s_out) cudaStreamDestroy(c->s_out);
  cudaFree(c->qscratch);
  cudaFree(c->qflags);
  cudaFree(c->cscratch);
  cudaFree(c->clscratch);
  cudaFree(c->clcounters);
  cudaFree(c->tscratch);
  cudaFree(c->Wg);
  cudaFree(c->bg);
  cudaFree(c->gate_buf);
  delete c;
}

arl2_status query_impl(arl2_ctx* c, const void* q, const void* k, const void* v, void* o, cudaStream_t st,
                       bool may_overlap = true) {
  const CUtensorMap* mq = c->acts.get(q, c->B, c->T, c->H, c->d);
  const CUtensorMap* mk = c->acts.get(k, c->B, c->T, c->H, c->d);
  const CUtensorMap* mv = c->acts.get(v, c->B, c->T, c->H, c->d);
  const CUtensorMap* mo = c->outs.get(o, c->B, c->T, c->H, c->d);
  if (!mq || !mk || !mv || !mo) return ARL2_ERR_CUDA;
  arl2::QueryArgs a{};
  a.o = static_cast<uint16_t*>(o);
  a.T = c->T;
  a.kv_len = c->T;
  a.B = c->B;
  a.H = c->H;
  a.d = c->d;
  a.state_slot = c->cur;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c->d)));
  a.err = c->err;
  a.timeout_ns = c->timeout_ns;
  a.stall = c->stall_next ? 1 : 0;
  c->stall_next = false;
  set_plan(&a, c->qplan, c->qscratch, c->qflags, next_epoch(&c->qepoch));
  const size_t act = c->act_elems() * 2;
  const bool dependent = may_overlap && c->overlap && clear_of_last_output(st, {{q, act}, {k, act}, {v, act}});
  record_query_output(st, o, act);
  return arl2::launch_query(true, *mq, *mk, *mv, c->tm_w[0], c->tm_s, *mo, a, st, dependent) == cudaSuccess
             ? ARL2_OK
             : ARL2_ERR_CUDA;
}

arl2_status commit_impl(arl2_ctx* c, const void* k, const void* v, const float* alpha, const float* beta,
                        cudaStream_t st, bool may_overlap = true) {
  const CUtensorMap* mk = c->acts.get(k, c->B, c->T, c->H, c->d);
  const CUtensorMap* mv = c->acts.get(v, c->B, c->T, c->H, c->d);
  if (!mk || !mv) return ARL2_ERR_CUDA;
  arl2::CommitArgs a{};
  a.alpha = alpha;
  a.beta = beta;
  a.T = c->T;
  a.B = c->B;
  a.H = c->H;
  a.d = c->d;
  a.chunks_per_group = c->chunks_per_group;
  a.ngroups = c->ngroups;
  a.state_slot = c->cur;
  a.inv_T = 1.0f / static_cast<float>(c->T);
  a.err = c->err;
  a.timeout_ns = c->timeout_ns;
  arl2::ReduceArgs r{};
  r.S_old = c->S[c->cur];
  r.S_new = c->S[c->cur ^ 1];
  r.S_new_bf16 = c->S_bf16 + (size_t)(c->cur ^ 1) * c->state_elems();
  r.part_u = c->cscratch;
  r.part_alpha = c->cscratch + arl2::commit_scratch_floats(c->B, c->H, c->ngroups) - (size_t)c->B * c->H * c->ngroups;
  r.d = c->d;
  r.inv_T = a.inv_T;
  const size_t act = c->act_elems() * 2, gate = (size_t)c->B * c->H * c->T * 4;
  const bool dependent = may_overlap && c->overlap &&
                         clear_of_last_output(st, {{k, act}, {v, act}, {alpha, gate}, {beta, gate}});
  if (arl2::launch_commit(*mk, *mv, c->tm_w[1], c->tm_w[2], c->tm_s, a, r, st, dependent) != cudaSuccess)
    return ARL2_ERR_CUDA;
  c->cur ^= 1;
  ++c->frame;
  return ARL2_OK;
}

arl2_status clean_impl(arl2_ctx* c, const void* q, const void* k, const void* v, void* o, const float* alpha,
                       const float* beta, cudaStream_t st) {
  const CUtensorMap* mq = c->acts.get(q, c->B, c->T, c->H, c->d);
  const CUtensorMap* mk = c->acts.get(k, c->B, c->T, c->H, c->d);
  const CUtensorMap* mv = c->acts.get(v, c->B, c->T, c->H, c->d);
  const CUtensorMap* mo = c->outs.get(o, c->B, c->T, c->H, c->d);
  if (!mq || !mk || !mv || !mo) return ARL2_ERR_CUDA;
  arl2::QueryArgs a{};
  a.o = static_cast<uint16_t*>(o);
  a.T = c->T;
  a.kv_len = c->T;
  a.B = c->B;
  a.H = c->H;
  a.d = c->d;
  a.state_slot = c->cur;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c->d)));
  a.err = c->err;
  a.timeout_ns = c->timeout_ns;
  a.stall = c->stall_next ? 1 : 0;
  c->stall_next = false;
  set_plan(&a, c->cplan.q, c->qscratch, c->qflags, next_epoch(&c->qepoch));
  const arl2::CleanPlan& p = c->cplan;
  a.first_cta = p.commit_ctas;   // the commit CTAs come first in the grid
  arl2::CommitStreamArgs m{};
  m.alpha = alpha;
  m.beta = beta;
  m.S_old = c->S[c->cur];
  m.S_new = c->S[c->cur ^ 1];
  m.S_new_bf16 = c->S_bf16 + (size_t)(c->cur ^ 1) * c->state_elems();
  const size_t slots = (size_t)c->B * c->H * p.max_pieces;
  m.part_u = c->clscratch;
  m.part_alpha = c->clscratch + slots * 32 * 128 * 4;
  m.counters = c->clcounters;
  m.T = c->T;
  m.B = c->B;
  m.H = c->H;
  m.d = c->d;
  m.state_slot = c->cur;
  m.inv_T = 1.0f / static_cast<float>(c->T);
  m.nchunks = p.nchunks;
  m.units = p.cunits;
  m.num_ctas = p.commit_ctas;
  m.max_pieces = p.max_pieces;
  m.err = c->err;
  m.timeout_ns = c->timeout_ns;
  const size_t act = c->act_elems() * 2, gate = (size_t)c->B * c->H * c->T * 4;
  const bool dependent = c->overlap && clear_of_last_output(st, {{q, act}, {k, act}, {v, act}, {alpha, gate},
                                                                 {beta, gate}});
  record_query_output(st, o, act);
  if (arl2::launch_clean(*mq, *mk, *mv, c->tm_w[0], c->tm_s, *mo, c->tm_w[1], c->tm_w[2], a, m, st, dependent) !=
      cudaSuccess)
    return ARL2_ERR_CUDA;
  c->cur ^= 1;
  ++c->frame;
  return ARL2_OK;
}

// Token-level access: the projections of the pass to scratch, then the scan. A query first
// writes the intra branch into o (the query kernel without its readout); the scan adds o_inter.
arl2_status token_impl(arl2_ctx* c, const void* q, const void* k, const void* v, void* o, const float* alpha,
                       const float* beta, cudaStream_t st) {
  const bool query = q != nullptr;
  const CUtensorMap* mk = c->acts.get(k, c->B, c->T, c->H, c->d);
  const CUtensorMap* mv = c->acts.get(v, c->B, c->T, c->H, c->d);
  const CUtensorMap* mq = query ? c->acts.get(q, c->B, c->T, c->H, c->d) : mk;
  if (!mk || !mv || !mq) return ARL2_ERR_CUDA;
  if (query) {
    const CUtensorMap* mo = c->outs.get(o, c->B, c->T, c->H, c->d);
    if (!mo) return ARL2_ERR_CUDA;
    arl2::QueryArgs a{};
    a.o = static_cast<uint16_t*>(o);
    a.T = c->T;
    a.kv_len = c->T;
    a.B = c->B;
    a.H = c->H;
    a.d = c->d;
    a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c->d)));
    a.err = c->err;
    a.timeout_ns = c->timeout_ns;
    set_plan(&a, c->qplan, c->qscratch, c->qflags, next_epoch(&c->qepoch));
    if (arl2::launch_query(false, *mq, *mk, *mv, c->tm_w[0], c->tm_s, *mo, a, st, false) != cudaSuccess)
      return ARL2_ERR_CUDA;
  }
  arl2::TokenArgs t{};
  const size_t rows = (size_t)c->B * c->H * c->T;
  const int P = c->d + 4 * arl2::kTokenParts;
  t.alpha = alpha;
  t.beta = beta;
  t.k_out = c->tscratch;
  t.q_out = query ? c->tscratch + rows * P : nullptr;
  t.v_out = c->tscratch + 2 * rows * P;
  t.S_old = c->S[c->cur];
  t.S_new = c->S[c->cur ^ 1];
  t.S_new_bf16 = c->S_bf16 + (size_t)(c->cur ^ 1) * c->state_elems();
  t.o = query ? static_cast<uint16_t*>(o) : nullptr;
  t.T = c->T;
  t.B = c->B;
  t.H = c->H;
  t.d = c->d;
  t.err = c->err;
  t.timeout_ns = c->timeout_ns;
  if (arl2::launch_token_project(*mq, *mk, *mv, c->tm_w[0], c->tm_w[1], c->tm_w[2], t, st) != cudaSuccess ||
      arl2::launch_token_scan(t, st) != cudaSuccess)
    return ARL2_ERR_CUDA;
  if (query) {
    record_query_output(st, o, c->act_elems() * 2);
  } else {
    c->cur ^= 1;
    ++c->frame;
  }
  return ARL2_OK;
}

arl2_status gates_impl(arl2_ctx* c, const void* x, float* alpha, float* beta, cudaStream_t st) {
  CUtensorMap tm_x;
  if (!make_hidden_map(&tm_x, x, c->B, c->T, c->H * c->d)) return ARL2_ERR_CUDA;
  arl2::GateArgs g{};
  g.bias = c->bg;
  g.alpha = alpha;
  g.beta = beta;
  g.B = c->B;
  g.T = c->T;
  g.H = c->H;
  g.D = c->H * c->d;
  g.ngates = 2 * c->H;
  g.ncols = gate_cols(c->H);
  g.tmem_cols = g.ncols <= 32 ? 32 : 64;
  g.err = c->err;
  g.timeout_ns = c->timeout_ns;
  return arl2::launch_gates(tm_x, c->tm_wg, g, st) == cudaSuccess ? ARL2_OK : ARL2_ERR_CUDA;
}

}  // namespace

extern "C" {

arl2_status arl2_set_gate_weights(arl2_ctx* c, const arl2_bf16* Wa, const arl2_bf16* Wb, const float* ba,
                                  const float* bb, arl2_stream stream) {
  if (!c || !Wa || !Wb || !ba || !bb) return ARL2_ERR_INVALID_ARG;
  if (!c->Wg) return ARL2_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t rows = (size_t)c->H * c->H * c->d * 2;   // H rows of D = H d bf16
  if (cudaMemcpyAsync(c->Wg, Wa, rows, cudaMemcpyDefault, st) != cudaSuccess ||
      cudaMemcpyAsync(c->Wg + (size_t)c->H * c->H * c->d, Wb, rows, cudaMemcpyDefault, st) != cudaSuccess ||
      cudaMemcpyAsync(c->bg, ba, (size_t)c->H * 4, cudaMemcpyDefault, st) != cudaSuccess ||
      cudaMemcpyAsync(c->bg + c->H, bb, (size_t)c->H * 4, cudaMemcpyDefault, st) != cudaSuccess)
    return ARL2_ERR_CUDA;
  c->gates_set = true;
  return ARL2_OK;
}

arl2_status arl2_frame_gates(arl2_ctx* c, const arl2_bf16* x, float* alpha, float* beta, arl2_stream stream) {
  if (!c || !aligned16(x) || !aligned4(alpha) || !aligned4(beta)) return ARL2_ERR_INVALID_ARG;
  if (!c->Wg) return ARL2_ERR_UNSUPPORTED;
  if (!c->gates_set) return ARL2_ERR_STATE;
  return gates_impl(c, x, alpha, beta, (cudaStream_t)stream);
}

arl2_status arl2_frame_commit_gated(arl2_ctx* c, const arl2_bf16* x, const arl2_bf16* k, const arl2_bf16* v,
                                    arl2_stream stream) {
  if (!c || !aligned16(x) || !aligned16(k) || !aligned16(v)) return ARL2_ERR_INVALID_ARG;
  if (!c->Wg) return ARL2_ERR_UNSUPPORTED;
  if (!c->gates_set || !c->maps_set) return ARL2_ERR_STATE;
  cudaStream_t st = (cudaStream_t)stream;
  float* alpha = c->gate_buf;
  float* beta = c->gate_buf + (size_t)c->B * c->H * c->T;
  arl2_status r = gates_impl(c, x, alpha, beta, st);
  if (r != ARL2_OK) return r;
  // The commit reads the gates from its first instructions, so it starts after the gate
  // kernel has completed (a normal launch, not a programmatic dependent).
  return commit_impl(c, k, v, alpha, beta, st, false);
}

arl2_status arl2_create(int H, int T, int d_k, int d_v, int B, arl2_ctx** out) {
  if (!out) return ARL2_ERR_INVALID_ARG;
  *out = nullptr;
  if (H < 1 || B < 1 || T < 1 || d_k < 1 || d_v < 1) return ARL2_ERR_INVALID_ARG;
  if (d_k != d_v || (d_k != 32 && d_k != 64 && d_k != 128) || T > 4096 || (long long)B * H > 65535)
    return ARL2_ERR_UNSUPPORTED;
  int dev = 0, sms = 0;
  arl2_status s = check_device(&dev, &sms);
  if (s != ARL2_OK) return s;
  arl2_ctx* c = new (std::nothrow) arl2_ctx();
  if (!c) return ARL2_ERR_OOM;
  c->B = B;
  c->H = H;
  c->T = T;
  c->d = d_k;
  c->device = dev;
  c->num_sms = sms;
  arl2::commit_split(T, H, B, sms, &c->chunks_per_group, &c->ngroups);
  const size_t dd = (size_t)d_k * d_k;
  bool ok = true;
  for (int i = 0; i < 3 && ok; ++i) ok = dev_alloc(&c->W[i], (size_t)H * dd, &c->bytes);
  for (int i = 0; i < 2 && ok; ++i) ok = dev_alloc(&c->S[i], c->state_elems(), &c->bytes);
  ok = ok && dev_alloc(&c->S_bf16, 2 * c->state_elems(), &c->bytes);
  ok = ok && dev_alloc(&c->err, 1, &c->bytes);
  for (int set = 0; set < 2; ++set) {
    for (int i = 0; i < 4 && ok; ++i) ok = dev_alloc(&c->stage_bf16[set][i], c->act_elems(), &c->bytes);
    for (int i = 0; i < 2 && ok; ++i) ok = dev_alloc(&c->stage_f32[set][i], (size_t)B * H * T, &c->bytes);
  }
  c->qplan = arl2::plan_query(B, H, T, T, sms);
  c->cplan = arl2::plan_clean(B, H, T, sms, 0);
  c->qscratch_floats = std::max(arl2::query_scratch_floats(c->qplan), arl2::query_scratch_floats(c->cplan.q));
  c->qflag_count = std::max(arl2::query_flag_count(c->qplan), arl2::query_flag_count(c->cplan.q));
  c->clscratch_floats = arl2::clean_scratch_floats(c->cplan);
  ok = ok && dev_alloc(&c->qscratch, c->qscratch_floats, &c->bytes);
  ok = ok && dev_alloc(&c->qflags, c->qflag_count, &c->bytes);
  ok = ok && dev_alloc(&c->cscratch, arl2::commit_scratch_floats(B, H, c->ngroups), &c->bytes);
  ok = ok && dev_alloc(&c->clscratch, c->clscratch_floats, &c->bytes);
  ok = ok && dev_alloc(&c->clcounters, (size_t)B * H, &c->bytes);
  ok = ok && dev_alloc(&c->tscratch, arl2::token_scratch_floats(B, H, T, d_k), &c->bytes);
  const int D = H * d_k;   // the model width the gate projections read
  if (ok && gates_supported(H, D)) {
    ok = dev_alloc(&c->Wg, (size_t)2 * H * D, &c->bytes) && dev_alloc(&c->bg, (size_t)2 * H, &c->bytes) &&
         dev_alloc(&c->gate_buf, (size_t)2 * B * H * T, &c->bytes);
  }
  if (!ok) {
    free_ctx(c);
    return ARL2_ERR_OOM;
  }
  ok = cudaStreamCreateWithFlags(&c->s_in, cudaStreamNonBlocking) == cudaSuccess &&
       cudaStreamCreateWithFlags(&c->s_out, cudaStreamNonBlocking) == cudaSuccess;
  for (int i = 0; i < 2 && ok; ++i)
    ok = cudaEventCreateWithFlags(&c->ev_in[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&c->ev_used[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&c->ev_out[i], cudaEventDisableTiming) == cudaSuccess;
  ok = ok && cudaMemset(c->S[0], 0, c->state_elems() * 4) == cudaSuccess &&
       cudaMemset(c->S[1], 0, c->state_elems() * 4) == cudaSuccess &&
       cudaMemset(c->S_bf16, 0, 2 * c->state_elems() * 2) == cudaSuccess &&
       cudaMemset(c->qflags, 0, c->qflag_count * sizeof(int)) == cudaSuccess &&
       cudaMemset(c->clcounters, 0, (size_t)B * H * sizeof(unsigned int)) == cudaSuccess &&
       cudaMemset(c->err, 0, sizeof(unsigned int)) == cudaSuccess;
  for (int i = 0; i < 3 && ok; ++i) ok = make_mat_map(&c->tm_w[i], c->W[i], H, d_k);
  ok = ok && make_mat_map(&c->tm_s, c->S_bf16, 2 * B * H, d_k);
  if (ok && c->Wg) ok = make_gate_map(&c->tm_wg, c->Wg, 2 * H, D, gate_cols(H));
  if (ok) ok = cudaDeviceSynchronize() == cudaSuccess;
  if (!ok) {
    free_ctx(c);
    return ARL2_ERR_CUDA;
  }
  *out = c;
  return ARL2_OK;
}

arl2_status arl2_set_feature_maps(arl2_ctx* c, const arl2_bf16* Wq, const arl2_bf16* Wk, const arl2_bf16* Wv,
                                  arl2_stream stream) {
  if (!c || !Wq || !Wk || !Wv) return ARL2_ERR_INVALID_ARG;
  const size_t bytes = (size_t)c->H * c->d * c->d * 2;
  const arl2_bf16* src[3] = {Wq, Wk, Wv};
  for (int i = 0; i < 3; ++i)
    if (cudaMemcpyAsync(c->W[i], src[i], bytes, cudaMemcpyDefault, (cudaStream_t)stream) != cudaSuccess)
      return ARL2_ERR_CUDA;
  c->maps_set = true;
  return ARL2_OK;
}

arl2_status arl2_frame_query(arl2_ctx* c, const arl2_bf16* q, const arl2_bf16* k, const arl2_bf16* v, arl2_bf16* o,
                             arl2_stream stream) {
  if (!c || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ARL2_ERR_INVALID_ARG;
  if (!c->maps_set) return ARL2_ERR_STATE;
  return query_impl(c, q, k, v, o, (cudaStream_t)stream);
}

arl2_status arl2_frame_commit(arl2_ctx* c, const arl2_bf16* k, const arl2_bf16* v, const float* alpha,
                              const float* beta, arl2_stream stream) {
  if (!c || !aligned16(k) || !aligned16(v) || !aligned4(alpha) || !aligned4(beta)) return ARL2_ERR_INVALID_ARG;
  if (!c->maps_set) return ARL2_ERR_STATE;
  return commit_impl(c, k, v, alpha, beta, (cudaStream_t)stream);
}

arl2_status arl2_frame_clean_pass(arl2_ctx* c, const arl2_bf16* q, const arl2_bf16* k, const arl2_bf16* v,
                                  arl2_bf16* o, const float* alpha, const float* beta, arl2_stream stream) {
  if (!c || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(alpha) ||
      !aligned4(beta))
    return ARL2_ERR_INVALID_ARG;
  if (!c->maps_set) return ARL2_ERR_STATE;
  return clean_impl(c, q, k, v, o, alpha, beta, (cudaStream_t)stream);
}

arl2_status arl2_set_clean_split(arl2_ctx* c, int commit_sms) {
  if (!c || commit_sms < 0) return ARL2_ERR_INVALID_ARG;
  const arl2::CleanPlan p = arl2::plan_clean(c->B, c->H, c->T, c->num_sms, commit_sms);
  const size_t qs = std::max(c->qscratch_floats, arl2::query_scratch_floats(p.q));
  const size_t qf = std::max(c->qflag_count, arl2::query_flag_count(p.q));
  const size_t cl = std::max(c->clscratch_floats, arl2::clean_scratch_floats(p));
  if (cudaDeviceSynchronize() != cudaSuccess) return ARL2_ERR_CUDA;   // no launch still uses the scratch
  float *nqs = nullptr, *ncl = nullptr;
  int* nqf = nullptr;
  size_t added = 0;
  bool ok = true;
  if (qs > c->qscratch_floats) ok = dev_alloc(&nqs, qs, &added);
  if (ok && qf > c->qflag_count) ok = dev_alloc(&nqf, qf, &added) && cudaMemset(nqf, 0, qf * sizeof(int)) == cudaSuccess;
  if (ok && cl > c->clscratch_floats) ok = dev_alloc(&ncl, cl, &added);
  if (!ok) {
    cudaFree(nqs);
    cudaFree(nqf);
    cudaFree(ncl);
    return ARL2_ERR_OOM;
  }
  if (nqs) {
    cudaFree(c->qscratch);
    c->bytes -= c->qscratch_floats * sizeof(float);
    c->qscratch = nqs;
    c->qscratch_floats = qs;
  }
  if (nqf) {
    cudaFree(c->qflags);
    c->bytes -= c->qflag_count * sizeof(int);
    c->qflags = nqf;
    c->qflag_count = qf;
  }
  if (ncl) {
    cudaFree(c->clscratch);
    c->bytes -= c->clscratch_floats * sizeof(float);
    c->clscratch = ncl;
    c->clscratch_floats = cl;
  }
  c->bytes += added;
  // Every head's counter restarts at zero for the new segment counts.
  if (cudaMemset(c->clcounters, 0, (size_t)c->B * c->H * sizeof(unsigned int)) != cudaSuccess)
    return ARL2_ERR_CUDA;
  c->cplan = p;
  return ARL2_OK;
}

int arl2_clean_split(const arl2_ctx* c) { return c ? c->cplan.commit_ctas : -1; }

arl2_status arl2_frame_query_token(arl2_ctx* c, const arl2_bf16* q, const arl2_bf16* k, const arl2_bf16* v,
                                   arl2_bf16* o, const float* alpha, const float* beta, arl2_stream stream) {
  if (!c || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(alpha) ||
      !aligned4(beta))
    return ARL2_ERR_INVALID_ARG;
  if (!c->maps_set) return ARL2_ERR_STATE;
  return token_impl(c, q, k, v, o, alpha, beta, (cudaStream_t)stream);
}

arl2_status arl2_frame_commit_token(arl2_ctx* c, const arl2_bf16* k, const arl2_bf16* v, const float* alpha,
                                    const float* beta, arl2_stream stream) {
  if (!c || !aligned16(k) || !aligned16(v) || !aligned4(alpha) || !aligned4(beta)) return ARL2_ERR_INVALID_ARG;
  if (!c->maps_set) return ARL2_ERR_STATE;
  return token_impl(c, nullptr, k, v, nullptr, alpha, beta, (cudaStream_t)stream);
}

arl2_status arl2_frame_query_host(arl2_ctx* c, const arl2_bf16* q, const arl2_bf16* k, const arl2_bf16* v,
                                  arl2_bf16* o, arl2_stream stream) {
  if (!c || !q || !k || !v || !o) return ARL2_ERR_INVALID_ARG;
  if (!c->maps_set) return ARL2_ERR_STATE;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t bytes = c->act_elems() * 2;
  const int s = static_cast<int>(c->host_turn++ & 1u);
  uint16_t* const* buf = c->stage_bf16[s];
  const arl2_bf16* src[3] = {q, k, v};
  // Inputs in, once the kernel that last read this set is done.
  bool ok = cudaStreamWaitEvent(c->s_in, c->ev_used[s], 0) == cudaSuccess;
  for (int i = 0; i < 3 && ok; ++i)
    ok = cudaMemcpyAsync(buf[i], src[i], bytes, cudaMemcpyHostToDevice, c->s_in) == cudaSuccess;
  ok = ok && cudaEventRecord(c->ev_in[s], c->s_in) == cudaSuccess;
  // The kernel, once they landed and this set's previous output has been copied out.
  ok = ok && cudaStreamWaitEvent(st, c->ev_in[s], 0) == cudaSuccess &&
       cudaStreamWaitEvent(st, c->ev_out[s], 0) == cudaSuccess;
  if (!ok) return ARL2_ERR_CUDA;
  arl2_status r = query_impl(c, buf[0], buf[1], buf[2], buf[3], st, false);
  if (r != ARL2_OK) return r;
  // Output out; the call completes on the caller's stream only with its output copied.
  ok = cudaEventRecord(c->ev_used[s], st) == cudaSuccess &&
       cudaStreamWaitEvent(c->s_out, c->ev_used[s], 0) == cudaSuccess &&
       cudaMemcpyAsync(o, buf[3], bytes, cudaMemcpyDeviceToHost, c->s_out) == cudaSuccess &&
       cudaEventRecord(c->ev_out[s], c->s_out) == cudaSuccess &&
       cudaStreamWaitEvent(st, c->ev_out[s], 0) == cudaSuccess;
  return ok ? ARL2_OK : ARL2_ERR_CUDA;
}

arl2_status arl2_frame_commit_host(arl2_ctx* c, const arl2_bf16* k, const arl2_bf16* v, const float* alpha,
                                   const float* beta, arl2_stream stream) {
  if (!c || !k || !v || !alpha || !beta) return ARL2_ERR_INVALID_ARG;
  if (!c->maps_set) return ARL2_ERR_STATE;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t bytes = c->act_elems() * 2, gbytes = (size_t)c->B * c->H * c->T * 4;
  const int s = static_cast<int>(c->host_turn++ & 1u);
  uint16_t* const* buf = c->stage_bf16[s];
  float* const* gbuf = c->stage_f32[s];
  bool ok = cudaStreamWaitEvent(c->s_in, c->ev_used[s], 0) == cudaSuccess &&
            cudaMemcpyAsync(buf[1], k, bytes, cudaMemcpyHostToDevice, c->s_in) == cudaSuccess &&
            cudaMemcpyAsync(buf[2], v, bytes, cudaMemcpyHostToDevice, c->s_in) == cudaSuccess &&
            cudaMemcpyAsync(gbuf[0], alpha, gbytes, cudaMemcpyHostToDevice, c->s_in) == cudaSuccess &&
            cudaMemcpyAsync(gbuf[1], beta, gbytes, cudaMemcpyHostToDevice, c->s_in) == cudaSuccess &&
            cudaEventRecord(c->ev_in[s], c->s_in) == cudaSuccess &&
            cudaStreamWaitEvent(st, c->ev_in[s], 0) == cudaSuccess;
  if (!ok) return ARL2_ERR_CUDA;
  arl2_status r = commit_impl(c, buf[1], buf[2], gbuf[0], gbuf[1], st, false);
  if (r != ARL2_OK) return r;
  return cudaEventRecord(c->ev_used[s], st) == cudaSuccess ? ARL2_OK : ARL2_ERR_CUDA;
}

arl2_status arl2_reset(arl2_ctx* c, arl2_stream stream) {
  if (!c) return ARL2_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemsetAsync(c->S[0], 0, c->state_elems() * 4, st) != cudaSuccess ||
      cudaMemsetAsync(c->S[1], 0, c->state_elems() * 4, st) != cudaSuccess ||
      cudaMemsetAsync(c->S_bf16, 0, 2 * c->state_elems() * 2, st) != cudaSuccess ||
      cudaMemsetAsync(c->clcounters, 0, (size_t)c->B * c->H * sizeof(unsigned int), st) != cudaSuccess)
    return ARL2_ERR_CUDA;
  c->cur = 0;
  c->frame = 0;
  return ARL2_OK;
}

arl2_status arl2_get_state(const arl2_ctx* c, float* dst, arl2_stream stream) {
  if (!c || !dst) return ARL2_ERR_INVALID_ARG;
  return cudaMemcpyAsync(dst, c->S[c->cur], c->state_elems() * 4, cudaMemcpyDefault, (cudaStream_t)stream) ==
                 cudaSuccess
             ? ARL2_OK
             : ARL2_ERR_CUDA;
}

arl2_status arl2_set_state(arl2_ctx* c, const float* src, arl2_stream stream) {
  if (!c || !src) return ARL2_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  const size_t n = c->state_elems();
  // Stage through the other buffer so that host sources work too, then convert in place.
  float* tmp = c->S[c->cur ^ 1];
  if (cudaMemcpyAsync(tmp, src, n * 4, cudaMemcpyDefault, st) != cudaSuccess) return ARL2_ERR_CUDA;
  return arl2::launch_state_import(tmp, c->S[c->cur], c->S_bf16 + (size_t)c->cur * n, n, st) == cudaSuccess
             ? ARL2_OK
             : ARL2_ERR_CUDA;
}

int arl2_frame_index(const arl2_ctx* c) { return c ? c->frame : -1; }

// Synchronise, read and clear the error word. An abandoned query launch may leave record
// flags set to its own epoch; later launches use other epochs, so they need no clearing.
static arl2_status read_status(unsigned int* err) {
  if (cudaDeviceSynchronize() != cudaSuccess) return ARL2_ERR_CUDA;
  unsigned int h = 0;
  if (cudaMemcpy(&h, err, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return ARL2_ERR_CUDA;
  if (h != 0 && cudaMemset(err, 0, sizeof(h)) != cudaSuccess) return ARL2_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return ARL2_ERR_CUDA;
  if (h & arl2::kErrLayoutBit) return ARL2_ERR_CUDA;
  return (h & arl2::kErrTimeoutBit) ? ARL2_ERR_TIMEOUT : ARL2_OK;
}

arl2_status arl2_get_status(arl2_ctx* c) {
  if (!c) return ARL2_ERR_INVALID_ARG;
  return read_status(c->err);
}

arl2_status arl2_set_launch_overlap(arl2_ctx* c, int enable) {
  if (!c) return ARL2_ERR_INVALID_ARG;
  c->overlap = enable != 0;
  return ARL2_OK;
}

arl2_status arl2_set_wait_timeout_ns(arl2_ctx* c, uint64_t timeout_ns) {
  if (!c || timeout_ns == 0) return ARL2_ERR_INVALID_ARG;
  c->timeout_ns = timeout_ns;
  return ARL2_OK;
}

arl2_status arl2_test_stall_next_query(arl2_ctx* c) {
  if (!c) return ARL2_ERR_INVALID_ARG;
  c->stall_next = true;
  return ARL2_OK;
}

size_t arl2_memory_bytes(const arl2_ctx* c) { return c ? c->bytes : 0; }

void arl2_destroy(arl2_ctx* c) { free_ctx(c); }

// ------------------------------------------------------------------ KV-cache baseline
arl2_status arl2_kvcache_create(int H, int T, int d, int B, int max_frames, arl2_kvcache** out) {
  if (!out) return ARL2_ERR_INVALID_ARG;
  *out = nullptr;
  if (H < 1 || B < 1 || T < 1 || d < 1 || max_frames < 1) return ARL2_ERR_INVALID_ARG;
  if ((d != 32 && d != 64 && d != 128) || (long long)B * H > 65535 || (long long)T * max_frames > (1ll << 30))
    return ARL2_ERR_UNSUPPORTED;
  int dev = 0, sms = 0;
  arl2_status s = check_device(&dev, &sms);
  if (s != ARL2_OK) return s;
  arl2_kvcache* c = new (std::nothrow) arl2_kvcache();
  if (!c) return ARL2_ERR_OOM;
  c->B = B;
  c->H = H;
  c->T = T;
  c->d = d;
  c->max_frames = max_frames;
  c->device = dev;
  c->num_sms = sms;
  const size_t elems = (size_t)B * max_frames * T * H * d;
  // Query scratch for the longest cache any frame reaches.
  for (int n = 1; n <= max_frames; ++n) {
    const arl2::QueryPlan p = arl2::plan_query(B, H, T, n * T, sms);
    c->qscratch_floats = std::max(c->qscratch_floats, arl2::query_scratch_floats(p));
    c->qflag_count = std::max(c->qflag_count, arl2::query_flag_count(p));
  }
  bool ok = dev_alloc(&c->K, elems, &c->bytes) && dev_alloc(&c->V, elems, &c->bytes) &&
            dev_alloc(&c->err, 1, &c->bytes) && dev_alloc(&c->qscratch, c->qscratch_floats, &c->bytes) &&
            dev_alloc(&c->qflags, c->qflag_count, &c->bytes);
  if (ok)
    ok = cudaMemset(c->K, 0, elems * 2) == cudaSuccess && cudaMemset(c->V, 0, elems * 2) == cudaSuccess &&
         cudaMemset(c->err, 0, 4) == cudaSuccess &&
         cudaMemset(c->qflags, 0, c->qflag_count * sizeof(int)) == cudaSuccess &&
         make_act_map(&c->tm_k, c->K, B, max_frames * T, H, d) &&
         make_act_map(&c->tm_v, c->V, B, max_frames * T, H, d) && cudaDeviceSynchronize() == cudaSuccess;
  if (!ok) {
    arl2_kvcache_destroy(c);
    return ARL2_ERR_OOM;
  }
  *out = c;
  return ARL2_OK;
}

static arl2_status kv_write_slot(arl2_kvcache* c, const void* k, const void* v, cudaStream_t st) {
  const size_t row = (size_t)c->T * c->H * c->d * 2;          // one frame of one batch entry
  const size_t pitch = (size_t)c->max_frames * row;             // one batch entry of the cache
  const size_t off = (size_t)c->n * c->T * c->H * c->d;
  if (cudaMemcpy2DAsync(c->K + off, pitch, k, row, row, c->B, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
      cudaMemcpy2DAsync(c->V + off, pitch, v, row, row, c->B, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return ARL2_ERR_CUDA;
  return ARL2_OK;
}

arl2_status arl2_kvcache_query(arl2_kvcache* c, const arl2_bf16* q, const arl2_bf16* k, const arl2_bf16* v,
                               arl2_bf16* o, arl2_stream stream) {
  if (!c || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ARL2_ERR_INVALID_ARG;
  if (c->n >= c->max_frames) return ARL2_ERR_STATE;
  cudaStream_t st = (cudaStream_t)stream;
  arl2_status s = kv_write_slot(c, k, v, st);
  if (s != ARL2_OK) return s;
  const CUtensorMap* mq = c->acts.get(q, c->B, c->T, c->H, c->d);
  const CUtensorMap* mo = c->outs.get(o, c->B, c->T, c->H, c->d);
  if (!mq || !mo) return ARL2_ERR_CUDA;
  arl2::QueryArgs a{};
  a.o = o;
  a.T = c->T;
  a.kv_len = (c->n + 1) * c->T;
  a.B = c->B;
  a.H = c->H;
  a.d = c->d;
  a.state_slot = 0;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c->d)));
  a.err = c->err;
  a.timeout_ns = c->timeout_ns;
  set_plan(&a, arl2::plan_query(c->B, c->H, c->T, a.kv_len, c->num_sms), c->qscratch, c->qflags,
           next_epoch(&c->qepoch));
  return arl2::launch_query(false, *mq, c->tm_k, c->tm_v, c->tm_k, c->tm_k, *mo, a, st, false) == cudaSuccess
             ? ARL2_OK
             : ARL2_ERR_CUDA;
}

arl2_status arl2_kvcache_commit(arl2_kvcache* c, const arl2_bf16* k, const arl2_bf16* v, arl2_stream stream) {
  if (!c || !aligned16(k) || !aligned16(v)) return ARL2_ERR_INVALID_ARG;
  if (c->n >= c->max_frames) return ARL2_ERR_STATE;
  arl2_status s = kv_write_slot(c, k, v, (cudaStream_t)stream);
  if (s != ARL2_OK) return s;
  ++c->n;
  return ARL2_OK;
}

arl2_status arl2_kvcache_reset(arl2_kvcache* c) {
  if (!c) return ARL2_ERR_INVALID_ARG;
  c->n = 0;
  return ARL2_OK;
}

int arl2_kvcache_frames(const arl2_kvcache* c) { return c ? c->n : -1; }

arl2_status arl2_kvcache_get_status(arl2_kvcache* c) {
  if (!c) return ARL2_ERR_INVALID_ARG;
  return read_status(c->err);
}

size_t arl2_kvcache_memory_bytes(const arl2_kvcache* c) { return c ? c->bytes : 0; }

void arl2_kvcache_destroy(arl2_kvcache* c) {
  if (!c) return;
  cudaFree(c->K);
  cudaFree(c->V);
  cudaFree(c->err);
  cudaFree(c->qscratch);
  cudaFree(c->qflags);
  delete c;
}

}  // extern "C"
