/*
 * arl2.h - C ABI of the ARL2 hybrid per-frame attention layer on NVIDIA B200 (sm_100a).
 *
 * The layer is the one described in "Attend Locally, Remember Linearly (ARL2)", the
 * technical summary of arXiv 2605.16579 (gist.science, zh/pt/fr pages):
 *   - §2.1: self-attention is split into an intra-frame branch (the original bidirectional
 *     softmax attention among one frame's tokens) and an inter-frame branch. The
 *     inter-frame branch replaces the growing KV cache by a fixed-size recurrent state S.
 *   - §2.1: per-head grouped 1x1 feature maps phi_q, phi_k, phi_v adapt Q, K, V to the
 *     recurrent branch.
 *   - §2.1: the state follows a gated-delta rule, and the branch reads out
 *     O_inter = Q' S_{N-1}.
 *   - §2.2: every token of frame N reads the same S_{N-1} (frame-level access). The
 *     denoising passes only read S. S is written once per frame, after the clean pass
 *     (clean-pass update).
 * Per (batch, head) this library computes
 *     query:   O   = softmax(Q K^T / sqrt(d)) V + (Q Wq_h) S_{N-1}
 *     commit:  S_N = abar S_{N-1} + K'^T diag(beta / T) (V' - K' S_{N-1}),
 *              K'  = rownorm(K Wk_h),  V' = V Wv_h,  abar = mean_t alpha_t.
 * The pages print the update without a transpose. They also do not say how the per-token
 * gates become one factor per frame. Reading K'^T, the mean of alpha and the rate
 * beta_t / T is this library's convention.
 *
 * Conventions for every call:
 *   - Pointers are device pointers unless a name ends in _host. Every call is
 *     asynchronous on the given stream (NULL = the legacy default stream) and returns
 *     after enqueueing the work. Argument checks are synchronous and return a status.
 *     Faults and wait time-outs inside kernels are reported later by arl2_get_status.
 *   - bf16 arrays hold bfloat16 bit patterns (uint16_t). q, k, v and o are [B, T, H, d]
 *     contiguous (token-major, as a linear projection writes them) and 16-byte aligned.
 *     alpha and beta are fp32 [B, H, T]. The state is fp32 [B, H, d_k, d_v].
 *   - The caller owns every buffer it passes. The library owns the two state buffers, its
 *     copies of the feature maps, its scratch and its staging buffers. It allocates all of
 *     them in arl2_create and frees them in arl2_destroy, so no per-frame call allocates
 *     memory (only the tuning call arl2_set_clean_split may).
 *   - Supported shapes: d_k == d_v == d in {32, 64, 128}; 1 <= T <= 4096; B >= 1; H >= 1;
 *     B * H <= 65535. Other shapes return ARL2_ERR_UNSUPPORTED. The device must be sm_100.
 *   - A context is not thread-safe. Calls on one context must be ordered by the caller,
 *     normally by using one stream.
 */
#ifndef ARL2_H
#define ARL2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct arl2_ctx arl2_ctx;        /* opaque; owned by the library */
typedef struct arl2_kvcache arl2_kvcache; /* opaque; the growing-KV-cache baseline */
typedef void* arl2_stream;               /* a cudaStream_t; NULL is the legacy default stream */
typedef uint16_t arl2_bf16;              /* a bfloat16 bit pattern */

typedef enum {
  ARL2_OK = 0,
  ARL2_ERR_INVALID_ARG = 1, /* null or misaligned pointer, bad context */
  ARL2_ERR_UNSUPPORTED = 2, /* shape or device outside the supported set */
  ARL2_ERR_OOM = 3,         /* a device allocation in a create call failed */
  ARL2_ERR_CUDA = 4,        /* a CUDA call failed, or a kernel faulted */
  ARL2_ERR_TIMEOUT = 5,     /* a kernel's bounded wait ran out; the result of that call is invalid */
  ARL2_ERR_STATE = 6        /* call out of order, such as a query before the feature maps are set */
} arl2_status;

/* Create a layer for B independent streams of H heads, T tokens per frame and head
 * dims d_k = d_v. Allocates the fp32 state S (two buffers, which alternate per commit),
 * a bf16 copy of S, the feature-map copies, scratch and staging. S starts at 0 and the
 * frame count at 0. On success *out holds the context; on failure *out is NULL. */
arl2_status arl2_create(int H, int T, int d_k, int d_v, int B, arl2_ctx** out);

/* Copy the per-head feature maps phi_q, phi_k, phi_v into the library (§2.1, the per-head
 * grouped 1x1 maps). Each is bf16 [H, d, d] and applies as x' = x @ W[h]; no bias, no
 * activation. Must be called before the first query or commit; it may be called again.
 * Stream-ordered: the caller's buffers may be reused once the stream has passed the copy. */
arl2_status arl2_set_feature_maps(arl2_ctx* ctx, const arl2_bf16* Wq, const arl2_bf16* Wk,
                                  const arl2_bf16* Wv, arl2_stream stream);

/* One query pass of frame N (a denoising step, or the clean pass): (§2.1, §2.2)
 *   o = softmax(q k^T / sqrt(d)) v  +  (q Wq_h) S_{N-1}    per (batch, head).
 * q, k, v, o: bf16 [B, T, H, d]. Reads S_{N-1} and never writes the state. o must not
 * overlap q, k or v. */
arl2_status arl2_frame_query(arl2_ctx* ctx, const arl2_bf16* q, const arl2_bf16* k,
                             const arl2_bf16* v, arl2_bf16* o, arl2_stream stream);

/* The clean-pass commit of frame N (§2.1 state update, §2.2 clean-pass update):
 *   S_N = abar S_{N-1} + K'^T diag(beta / T) (V' - K' S_{N-1}).
 * k, v: bf16 [B, T, H, d], the clean pass's keys and values. alpha (forget gate, in (0, 1))
 * and beta (rate): fp32 [B, H, T]. Writes S_N into the other state buffer and advances the
 * frame count. Later queries read S_N. Queries enqueued before this commit read S_{N-1},
 * by stream order. */
arl2_status arl2_frame_commit(arl2_ctx* ctx, const arl2_bf16* k, const arl2_bf16* v,
                              const float* alpha, const float* beta, arl2_stream stream);

/* The clean pass of frame N in one launch: the query of arl2_frame_query and the commit of
 * arl2_frame_commit on the same k and v (§2.2 clean-pass update: the final, clean forward
 * pass both reads S_{N-1} for its own output and writes S_N). The result equals calling
 * arl2_frame_query(q, k, v, o) then arl2_frame_commit(k, v, alpha, beta) on the same stream,
 * up to the order of floating-point sums: o reads S_{N-1}, S_N goes into the other state
 * buffer and the frame count advances. Part of the GPU runs the query while the rest runs
 * the commit, so the commit's latency hides behind the query. Arguments as for those two
 * calls; o must not overlap q, k, v, alpha or beta. */
arl2_status arl2_frame_clean_pass(arl2_ctx* ctx, const arl2_bf16* q, const arl2_bf16* k,
                                  const arl2_bf16* v, arl2_bf16* o, const float* alpha,
                                  const float* beta, arl2_stream stream);

/* How many SMs the clean pass gives the commit (the rest run the query). 0 (the default)
 * picks the number from a cost model of the two parts; n > 0 asks for n, clamped to
 * [1, B * H * ceil(T / 128)] and to leave one SM for the query. Synchronises the device, and
 * allocates when the new split needs more scratch (ARL2_ERR_OOM if that fails; the old split
 * then stays). For tuning and tests; results differ between splits only in the order of
 * floating-point sums. */
arl2_status arl2_set_clean_split(arl2_ctx* ctx, int commit_sms);

/* The SMs the clean pass currently gives the commit; -1 for a NULL context. */
int arl2_clean_split(const arl2_ctx* ctx);

/* ---- Token-level access (the ablation of §4, "Ablations") ------------------------------
 * The pages report that letting the state advance token by token inside a frame, instead of
 * every token reading S_{N-1}, degrades quality; they give no form. This library reads it as
 * the §2.1 update applied to one token at a time, in token order, from S_{N-1}: per (batch,
 * head), for t = 0..T-1,
 *   o_inter[t] = q'_t S,    S <- alpha_t S + beta_t k'_t^T (v'_t - k'_t S)
 * with q' = q Wq_h, k' = rownorm(k Wk_h), v' = v Wv_h, and the per-token gates alpha_t (not
 * their mean) and beta_t (not beta_t / T). Layouts and alignment as above.
 *   query:  o = softmax(q k^T / sqrt(d)) v + o_inter, the scan running over this pass's own
 *           k, v and gates; never writes the state.
 *   commit: S_N = the state after the last token of the clean pass; advances the frame count.
 * The scan is sequential in the tokens: these calls run an fp32 scan on the CUDA cores, far
 * slower than the frame-level calls. o must not overlap q, k, v, alpha or beta. */
arl2_status arl2_frame_query_token(arl2_ctx* ctx, const arl2_bf16* q, const arl2_bf16* k,
                                   const arl2_bf16* v, arl2_bf16* o, const float* alpha,
                                   const float* beta, arl2_stream stream);
arl2_status arl2_frame_commit_token(arl2_ctx* ctx, const arl2_bf16* k, const arl2_bf16* v,
                                    const float* alpha, const float* beta, arl2_stream stream);

/* Host-buffer forms of arl2_frame_query and arl2_frame_commit, for callers whose data is in
 * host memory.
 * Each call copies its inputs into library-owned staging, runs the kernel on the stream
 * and (for the query) copies o back. The copies run on two internal streams, and the
 * calls take two staging sets by turns: one call's input copy overlaps the previous
 * call's kernel and output copy. The stream waits for the call's copies, so its
 * completion covers the whole call. With pinned host memory the call returns at once;
 * the caller synchronises the stream before reading o_host or reusing the inputs. With
 * pageable memory the CUDA copies may block. Calls on one context are made from one host
 * thread at a time. */
arl2_status arl2_frame_query_host(arl2_ctx* ctx, const arl2_bf16* q_host, const arl2_bf16* k_host,
                                  const arl2_bf16* v_host, arl2_bf16* o_host, arl2_stream stream);
arl2_status arl2_frame_commit_host(arl2_ctx* ctx, const arl2_bf16* k_host, const arl2_bf16* v_host,
                                   const float* alpha_host, const float* beta_host,
                                   arl2_stream stream);

/* ---- Gates produced from the hidden state ----------------------------------------------
 * §2.1 calls the forget gate alpha and the rate beta per-token learned projections without
 * giving their form. This library reads them as a linear projection of the token's hidden
 * state per head plus a bias, through a sigmoid (both stay in (0, 1)):
 *   alpha[b, h, t] = sigmoid(x[b, t, :] . Wa[h, :] + ba[h])
 *   beta[b, h, t]  = sigmoid(x[b, t, :] . Wb[h, :] + bb[h])
 * x is the layer's hidden state, bf16 [B, T, D] with D = H * d (the model width), 16-byte
 * aligned. Supported when 2H <= 64 (H <= 32); otherwise these calls return
 * ARL2_ERR_UNSUPPORTED and the gates are passed to arl2_frame_commit as before. */

/* Copy the gate projections into the library: Wa, Wb bf16 [H, D] (rows of the model width),
 * ba, bb fp32 [H]; device or host memory, stream-ordered like arl2_set_feature_maps. */
arl2_status arl2_set_gate_weights(arl2_ctx* ctx, const arl2_bf16* Wa, const arl2_bf16* Wb,
                                  const float* ba, const float* bb, arl2_stream stream);

/* The gates alone: alpha, beta fp32 [B, H, T] (device memory, 4-byte aligned) from x.
 * ARL2_ERR_STATE before arl2_set_gate_weights. */
arl2_status arl2_frame_gates(arl2_ctx* ctx, const arl2_bf16* x, float* alpha, float* beta,
                             arl2_stream stream);

/* The clean-pass commit of frame N with its gates produced from x (the clean pass's hidden
 * state): the gate kernel writes alpha and beta into library-owned buffers, then the commit
 * runs as arl2_frame_commit on them. k, v as for arl2_frame_commit. */
arl2_status arl2_frame_commit_gated(arl2_ctx* ctx, const arl2_bf16* x, const arl2_bf16* k,
                                    const arl2_bf16* v, arl2_stream stream);

/* Reset the state to S_0 = 0 and the frame count to 0 (the start of a new video). */
arl2_status arl2_reset(arl2_ctx* ctx, arl2_stream stream);

/* Copy the current state (fp32 [B, H, d_k, d_v]) to dst, which may be device or host
 * memory. Used for checkpointing and tests. */
arl2_status arl2_get_state(const arl2_ctx* ctx, float* dst, arl2_stream stream);

/* Replace the current state with src (fp32 [B, H, d_k, d_v], device or host memory),
 * for resuming from a checkpoint and for tests. The frame count is unchanged. */
arl2_status arl2_set_state(arl2_ctx* ctx, const float* src, arl2_stream stream);

/* Number of commits since creation or the last reset. */
int arl2_frame_index(const arl2_ctx* ctx);

/* Synchronise the device and return, then clear, the context's device error word.
 * Returns ARL2_ERR_TIMEOUT if a kernel's bounded wait ran out since the last call, and
 * ARL2_ERR_CUDA if the device reported an error. Otherwise it returns ARL2_OK. */
arl2_status arl2_get_status(arl2_ctx* ctx);

/* Limit on every wait inside this context's kernels, in nanoseconds (default 1e9). When
 * a wait runs out, the kernel abandons the call and returns; arl2_get_status then reports
 * ARL2_ERR_TIMEOUT. Returns ARL2_ERR_INVALID_ARG for NULL or 0. */
arl2_status arl2_set_wait_timeout_ns(arl2_ctx* ctx, uint64_t timeout_ns);

/* Let this context's queries and commits overlap the kernel before them in their stream
 * (default off). When on, each is launched as a programmatic dependent: its CTAs may start,
 * and read their inputs, while the preceding kernel in the stream is still running. On
 * B200 this hides a call's start-up behind the previous query's last CTAs.
 * - A query waits for that kernel before its first write, so back-to-back queries may
 *   share an output buffer.
 * - A commit writes only the other state buffer and its own scratch.
 * Turn it on only when no kernel that writes a call's inputs can run right before it in
 * the same stream without waiting for completion. Kernels that do not use programmatic
 * launch always complete first, as do copies. As a guard, a call whose inputs overlap the
 * output of the last query launched in the same stream is launched normally. */
arl2_status arl2_set_launch_overlap(arl2_ctx* ctx, int enable);

/* Failure-detection test hook. The next arl2_frame_query (or arl2_frame_query_host)
 * launch makes its softmax threads wait on an mbarrier that nothing signals. That wait
 * runs out after the context's wait limit; every role of the kernel then stops, drains
 * what it issued and frees its tensor memory, and arl2_get_status reports
 * ARL2_ERR_TIMEOUT. The output of that call is undefined. The hook clears itself after
 * that one launch. Returns ARL2_ERR_INVALID_ARG for NULL. */
arl2_status arl2_test_stall_next_query(arl2_ctx* ctx);

/* Bytes of device memory the context holds (everything allocated in arl2_create). */
size_t arl2_memory_bytes(const arl2_ctx* ctx);

/* Free everything the context holds. The caller must make sure none of its work is still
 * in flight. NULL is ignored. */
void arl2_destroy(arl2_ctx* ctx);

/* ---- Allocation-free commit ------------------------------------------------------------
 * This entry point has no counterpart in the paper. It exists for callers that cannot
 * call cudaMalloc. Examples: a serving engine that reserved all device memory for its own
 * pool at start-up; a real-time frame loop that must not take the allocator's locks or
 * its implicit synchronisation; an embedding that only hands the library memory it owns.
 *
 * It computes the same update as arl2_frame_commit without a context:
 *   S_next = abar S_prev + K'^T diag(beta / T) (V' - K' S_prev)
 * The arguments are:
 *   - k, v: bf16 [B, T, H, d].
 *   - alpha, beta: fp32 [B, H, T].
 *   - Wk, Wv: bf16 [H, d, d].
 *   - S_prev, S_next: fp32 [B, H, d, d]. S_next may be S_prev itself (an in-place
 *     update) or must not overlap it.
 *   - status: a device word (4-byte aligned, required), ORed with 1 if a bounded wait in
 *     the kernel ran out. The caller zeroes it before the call and reads it after the
 *     stream has passed the call. Without a context there is nowhere else a time-out could
 *     be reported, so NULL returns ARL2_ERR_INVALID_ARG. After a time-out S_next is
 *     undefined; for an in-place call (S_next == S_prev) that includes S_prev.
 *
 * The call allocates nothing. Its scratch is a fixed device array of
 * ARL2_NOALLOC_SCRATCH_BYTES inside the library. Every GPU that loads the library holds
 * that array until the process exits. Shapes whose scratch would exceed it return
 * ARL2_ERR_UNSUPPORTED before any work is enqueued. The need is about
 * B*H*(d*d*4 + G*64 KiB) bytes: bf16 copies of S_prev and S_next, and the partial update of
 * each of the G <= 8 groups of 128-token chunks a (batch, head) is split into (G = 7 at
 * T = 1560). B=1, H=12, T=1560, d=128 needs about 6.1 MB; at G = 8 the array fits
 * B*H <= 28.
 *
 * The first call on a device looks the array's device address up, with that device
 * current. Make that first call before any stream capture. All calls on a device share
 * the one array and leave their contents in it; each call writes what it reads before
 * reading it, and nothing in it needs to start at zero. Calls that overlap on the GPU,
 * for example on two streams, race on the array.
 * Supported shapes are as for arl2_create. */
#define ARL2_NOALLOC_SCRATCH_BYTES (16u << 20)
arl2_status arl2_frame_commit_noalloc(int B, int H, int T, int d, const arl2_bf16* k, const arl2_bf16* v,
                                      const float* alpha, const float* beta, const arl2_bf16* Wk,
                                      const arl2_bf16* Wv, const float* S_prev, float* S_next,
                                      unsigned int* status, arl2_stream stream);

/* ---- Growing-KV-cache baseline (comparison only; §1 problem statement) -----------------
 * This is full softmax attention of the newest frame over the keys and values of every
 * frame so far, which is what the layer above replaces. Its cache grows by one frame per
 * commit, up to max_frames. The cache is preallocated and zero-filled in create.
 *   query:  writes k, v into the slot of the current frame n (without committing it), then
 *           o = softmax(q K_{1..n+1}^T / sqrt(d)) V_{1..n+1}, over (n+1) T keys.
 *   commit: writes k, v into slot n and advances n.
 * Layouts, alignment and stream rules are as above. */
arl2_status arl2_kvcache_create(int H, int T, int d, int B, int max_frames, arl2_kvcache** out);
arl2_status arl2_kvcache_query(arl2_kvcache* c, const arl2_bf16* q, const arl2_bf16* k,
                               const arl2_bf16* v, arl2_bf16* o, arl2_stream stream);
arl2_status arl2_kvcache_commit(arl2_kvcache* c, const arl2_bf16* k, const arl2_bf16* v,
                                arl2_stream stream);
arl2_status arl2_kvcache_reset(arl2_kvcache* c);
int arl2_kvcache_frames(const arl2_kvcache* c);
arl2_status arl2_kvcache_get_status(arl2_kvcache* c);
size_t arl2_kvcache_memory_bytes(const arl2_kvcache* c);
void arl2_kvcache_destroy(arl2_kvcache* c);

#ifdef __cplusplus
}
#endif

#endif /* ARL2_H */
