/*
 * rm.h -- C ABI of the B200 transformer scorer ("rmscore").
 *
 * Scores batches of variable-length token sequences with a compact
 * transformer scorer and groups queued requests into batches.
 *
 *  - The scorer is a BERT/TinyBERT-style post-LN encoder (SambaNova blog
 *    "Breakthrough efficiency in NLP model deployment", first section; the
 *    transformer served by "TurboTransformers: An Efficient GPU Serving System
 *    For Transformer Models", abstract) or a GPT-style pre-LN causal reward
 *    model with a scalar head ("Learning to summarize from human feedback"
 *    summary, method section: reward model = supervised baseline plus a
 *    scalar head; its reward normalisation is a constant folded into b_r).
 *  - Sequences are packed without padding (TurboTransformers abstract:
 *    variable-length input; proposed-method section: no fixed-length padding).
 *  - Requests are grouped by a dynamic-programming batch scheduler
 *    (TurboTransformers abstract and proposed-method section).
 *
 * Conventions for every function below:
 *  - Return value: RM_OK (0) or a negative RM_E_* code; rm_schedule* return
 *    the number of batches (>= 0) on success.  On error a message is kept in
 *    thread-local storage and returned by rm_last_error().  Nothing aborts,
 *    nothing throws across the ABI, no device trap is ever raised.
 *  - "host" pointers are ordinary CPU memory, "device" pointers are CUDA
 *    global memory on the handle's device.  The caller owns every buffer it
 *    passes; the library owns its device weights and its arena.
 *  - Device work is asynchronous on the caller's stream (a cudaStream_t passed
 *    as void*; NULL = the legacy default stream).  Inputs must stay alive and
 *    unmodified until that stream has finished the call.  One stream at a
 *    time per handle: calls on one handle must be ordered on one stream.
 *    Concurrent scoring uses separate handles.
 */
#ifndef RM_H_
#define RM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define RM_OK        0
#define RM_E_INVAL  -1   /* bad argument (null pointer, bad size or config)        */
#define RM_E_NOMEM  -2   /* device or pinned-host allocation failed                */
#define RM_E_CUDA   -3   /* a CUDA runtime/driver call failed (message has detail) */
#define RM_E_RANGE  -4   /* a size exceeds what the handle was created for         */
#define RM_E_DEVICE -5   /* no usable sm_100 device                                */

/* rm_config.arch */
#define RM_ENC_POSTLN 0  /* encoder, post-LN, bidirectional, head on token 0        */
#define RM_DEC_PRELN  1  /* decoder, pre-LN, causal, final LN, head on last token   */
/* rm_config.weight_dtype */
#define RM_F32  0
#define RM_BF16 1
/* rm_config.gelu */
#define RM_GELU_ERF  0   /* u * Phi(u)                                              */
#define RM_GELU_TANH 1   /* 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3)))         */

/* rm_config.attn_impl: how the attention step runs inside rm_score.
 * FUSED: scores, masked softmax and P.V in one kernel (rm_op_attn_fused);
 * the probabilities stay in registers.  MATERIALIZED: the three kernels
 * rm_op_attn_scores -> rm_op_softmax -> rm_op_attn_context with the score
 * matrix in HBM.  Both compute the same values up to rounding order. */
#define RM_ATTN_FUSED        0
#define RM_ATTN_MATERIALIZED 1

/* rm_config.sched_objective.  THROUGHPUT minimises the total time of the
 * queue's batches.  LATENCY minimises the sum of the queued requests'
 * completion times when the batches run back to back in ascending longest
 * length: a batch that starts at sorted position j delays the n - j requests
 * from j on, so dp[i] = min_j dp[j] + T(i-j, l_i) * (n - j).  The
 * TurboTransformers review's main results report the scheduler's mean
 * latency at its serving rate; this objective targets that figure directly. */
#define RM_SCHED_THROUGHPUT 0
#define RM_SCHED_LATENCY    1

typedef struct rm_handle rm_handle;

typedef struct rm_config {
  int32_t arch;          /* RM_ENC_POSTLN | RM_DEC_PRELN                              */
  int32_t n_layers;      /* >= 1                                                      */
  int32_t hidden;        /* H: multiple of 8, 8..4096                                 */
  int32_t n_heads;       /* h: divides H; head dim d = H/h must be even and <= 128    */
  int32_t ffn;           /* F: multiple of 8                                          */
  int32_t vocab;         /* V >= 1                                                    */
  int32_t max_pos;       /* P >= max_len (learned positions 0..P-1)                   */
  int32_t weight_dtype;  /* RM_F32 | RM_BF16: element type of the weights buffer     */
  int32_t gelu;          /* RM_GELU_ERF | RM_GELU_TANH                                */
  float   ln_eps;        /* LayerNorm epsilon (> 0)                                   */
  /* capacity: sizes the arena once, at create; rm_score never allocates */
  int32_t max_batch_seqs;/* most sequences per rm_score call                          */
  int32_t max_tokens;    /* most packed tokens per rm_score call                      */
  int32_t max_len;       /* longest sequence, 1..1024                                 */
  /* DP scheduler (rm_schedule); cost of a batch of b sequences, longest L */
  int32_t sched_max_batch;       /* Bmax >= 1                                         */
  int64_t sched_c0, sched_c1;    /* default cost T(b,L) = c0 + c1*b*L (both >= 0)     */
  const int64_t* sched_table;    /* optional host table T[b-1][L-1], row-major,       */
  int32_t sched_table_b;         /*   sched_table_b >= Bmax rows, sched_table_l >=    */
  int32_t sched_table_l;         /*   max_len columns, non-decreasing along L; copied */
  int32_t attn_impl;             /* RM_ATTN_FUSED (default) | RM_ATTN_MATERIALIZED    */
  /* latency-aware scheduling (rm_schedule) */
  int32_t sched_objective;       /* RM_SCHED_THROUGHPUT (default) | RM_SCHED_LATENCY  */
  int64_t sched_max_cost;        /* 0 = no cap; else every batch of >= 2 requests     */
                                 /*   costs at most this (single requests always ok) */
} rm_config;

/* Number of bytes the flat weights buffer must hold for cfg.
 * Layout (elements of weight_dtype, in this order; linear weights [out][in]
 * row-major):
 *   E_word[V][H], E_pos[P][H], (encoder: LN_emb gain[H], bias[H]),
 *   per layer: W_qkv[3H][H], b_qkv[3H], W_o[H][H], b_o[H], LN1 gain, bias,
 *              W_1[F][H], b_1[F], W_2[H][F], b_2[H], LN2 gain, bias,
 *   (decoder: LN_f gain[H], bias[H]), w_r[H], b_r[1].
 * W_qkv stacks the Q, K and V projections in that order; head j of each owns
 * rows j*d .. j*d+d-1.  Returns 0 for an invalid cfg. */
size_t rm_weights_bytes(const rm_config* cfg);

/* Create a scorer on the current CUDA device.  weights: host buffer laid out
 * as above, weights_bytes == rm_weights_bytes(cfg); it is copied (to bf16 for
 * matrices and embeddings, fp32 for biases and LN parameters) and may be freed
 * on return.  Reserves the whole arena for the capacity in cfg.  Synchronous.
 * Errors: RM_E_INVAL (cfg/size), RM_E_DEVICE (no sm_100 device), RM_E_NOMEM,
 * RM_E_CUDA.  *out is set only on success. */
int rm_create(const rm_config* cfg, const void* weights, size_t weights_bytes, rm_handle** out);

/* A second handle on the same device that shares base's device weights
 * (no copy) but has its own arena, metadata staging and error words, so that
 * two streams can each keep a batch in flight.  The weights stay alive until
 * the last handle that shares them is destroyed; base may be destroyed first.
 * Errors: RM_E_INVAL (NULL, or the current device is not base's), RM_E_NOMEM,
 * RM_E_CUDA. */
int rm_create_shared(const rm_handle* base, rm_handle** out);

/* Score n_seqs packed sequences.
 *   packed_token_ids: device int32[T], T = seq_offsets[n_seqs]; sequence i is
 *                     ids[seq_offsets[i] .. seq_offsets[i+1]-1].
 *   seq_offsets:      HOST int32[n_seqs+1], seq_offsets[0] = 0, every length
 *                     seq_offsets[i+1]-seq_offsets[i] in 1..max_len.
 *   out_scores:       device float[n_seqs]; out_scores[i] = score of sequence i.
 * Validation happens on the host before anything is enqueued: RM_E_INVAL for
 * null pointers, n_seqs < 1, non-monotone offsets; RM_E_RANGE for n_seqs >
 * max_batch_seqs, T > max_tokens or a length > max_len.  Token ids outside
 * 0..V-1 are clamped on the device and counted (rm_get_device_error).
 * Asynchronous on stream; makes no allocation. */
int rm_score(rm_handle* h, const int32_t* packed_token_ids, const int32_t* seq_offsets,
             int32_t n_seqs, float* out_scores, void* stream);

/* Best-of-N / pairwise scoring of candidates that share a prefix, for the
 * causal decoder (arch RM_DEC_PRELN): the reward model scores each summary
 * of a post as the sequence post + summary, and the best-of-N policy keeps the
 * highest-scoring one ("Learning to summarize from human feedback": reward
 * model and best-of-N sections; the reward model's pairwise loss compares
 * r_1 - r_0).  Because the decoder is causal, the prefix's hidden states do not
 * depend on what follows, so each prefix is computed once and every candidate
 * attends to its keys and values: the result equals rm_score on the N
 * concatenations, with the prefix's work done once instead of N times.
 *   packed_token_ids: device int32, per group g: the prefix (prefix_len[g]
 *                     tokens, may be 0) then its n_cand[g] candidates in order.
 *   prefix_len, n_cand: HOST int32[n_groups]; cand_len: HOST int32[sum n_cand],
 *                     candidates of group 0 first; every prefix_len + cand_len
 *                     in 1..max_len and <= max_pos.
 *   out_scores:       device float[sum n_cand], score of each prefix + candidate.
 *   out_best:         device int32[n_groups] or NULL: index within the group of
 *                     the highest score (the first on ties).
 *   out_logodds:      device float[n_groups] or NULL: r_1 - r_0 of the group's
 *                     first two candidates (the log-odds that candidate 1 is
 *                     preferred), 0 for a single candidate.
 * The prefix and each candidate count as one sequence against max_batch_seqs.
 * RM_E_INVAL for an encoder config, head_dim % 8 != 0, null pointers,
 * n_groups < 1, a negative prefix length or an empty group or candidate;
 * RM_E_RANGE for the limits above.  Asynchronous on stream; no allocation. */
int rm_score_prefix(rm_handle* h, const int32_t* packed_token_ids, const int32_t* prefix_len,
                    const int32_t* n_cand, const int32_t* cand_len, int32_t n_groups,
                    float* out_scores, int32_t* out_best, float* out_logodds, void* stream);

/* A plan: the batch shape (seq_offsets) of repeated rm_score calls, prepared
 * once.  The pages have no counterpart to this entry point; it exists so that
 * a fixed-shape call (batch-1 latency, an ensemble of experts) can be captured
 * into a CUDA graph and replayed without the host launching each kernel.  rm_plan_create validates the offsets as rm_score does, builds the
 * per-call metadata, allocates a small device block for it (the only
 * allocation; synchronous) and fixes the arena placement.  rm_score_plan then
 * enqueues the kernels alone -- no host synchronisation and no copies -- so it
 * may be captured into a CUDA graph and replayed; each replay scores whatever
 * ids are in packed_token_ids at that time.  A plan uses its handle's arena:
 * it must not run concurrently with other calls on the same handle, and it is
 * destroyed before its handle.  Errors as rm_score; RM_E_NOMEM / RM_E_CUDA
 * when the metadata block cannot be made. */
typedef struct rm_plan rm_plan;
int rm_plan_create(rm_handle* h, const int32_t* seq_offsets, int32_t n_seqs, rm_plan** out);
int rm_score_plan(rm_plan* plan, const int32_t* packed_token_ids, float* out_scores, void* stream);
void rm_plan_destroy(rm_plan* plan);

/* As rm_score, but token ids and scores are HOST buffers.  The ids are copied
 * host->device and the scores device->host on stream inside the call's
 * enqueued work; both host buffers should be pinned (cudaHostAlloc /
 * torch pin_memory) for the copies to be asynchronous.  The scores are in
 * host_scores once stream has completed. */
int rm_score_host(rm_handle* h, const int32_t* host_token_ids, const int32_t* seq_offsets,
                  int32_t n_seqs, float* host_scores, void* stream);

/* DP batch scheduling of a queue of n requests with the handle's scheduler
 * settings.  lengths: host int32[n], each in 1..max_len.  out_batches: host
 * int32[n]; out_batches[i] = batch of request i, batches numbered 0..nb-1 in
 * execution order (ascending longest length).  Returns nb >= 0 or an error.
 * Host only; no device work. */
int rm_schedule(const rm_handle* h, const int32_t* lengths, int32_t n, int32_t* out_batches);

/* As rm_schedule, from a config alone (no handle, no device needed).  Only
 * the scheduler fields and max_len of cfg are read. */
int rm_schedule_cfg(const rm_config* cfg, const int32_t* lengths, int32_t n, int32_t* out_batches);

/* Waits for the stream of the last rm_score* call, then reads the device error
 * words: out[0] = token ids clamped since create, out[1] = pipeline waits that
 * gave up (a kernel that timed out wrote this and returned early; its outputs
 * are invalid).  out: host int32[2]. */
int rm_get_device_error(rm_handle* h, int32_t* out);

/* Failure detection without a fault (the pages have no counterpart): runs on
 * the current device one thread that waits, through the same bounded
 * mbarrier wait as the GEMM's producer, MMA and epilogue roles, on a barrier
 * that nothing completes, giving up after limit_ns (1e3 .. 1e10).  Writes
 * *out_timed_out = 1 if the wait gave up (the expected result) and the
 * nanoseconds it waited.  Synchronous; allocates (and frees) 16 bytes of
 * device memory.  The CUDA context stays usable afterwards.  RM_E_INVAL for
 * NULL outputs or a limit out of range, RM_E_CUDA on a CUDA error. */
int rm_selftest_bounded_wait(int64_t limit_ns, int32_t* out_timed_out, int64_t* out_elapsed_ns);

/* Allocation fault injection for tests (the pages have no counterpart): the
 * k-th device or pinned-host allocation that the library makes from now on
 * (counting from 1, in this process, on any handle: rm_create makes five --
 * weights, their upload staging, the arena, the error words, the pinned
 * metadata ring -- rm_create_shared three and rm_plan_create one) fails as if
 * memory were exhausted, without reaching the allocator; k = 0 disarms it.
 * The call that meets the failure releases what it had allocated and returns
 * RM_E_NOMEM; existing handles are untouched and stay usable.  Host only,
 * thread-safe.  RM_E_INVAL for k < 0. */
int rm_debug_fail_alloc(int32_t k);

/* The checked build (the pages have no counterpart): librmscore_checked.so is
 * the same library compiled with RM_CHECKED, in which the kernels test the
 * indices they derive from offsets and other per-call metadata (positions in
 * the position table, sequence and row-block indices, a tile's offsets
 * window, the softmax's row index) before the accesses those indices address,
 * and skip the access and count it when a test fails (no trap, no assert).
 * rm_build_checked() returns 1 in that library and 0 in the product one.
 * rm_bounds_errors: waits for the device, writes the number of failed tests
 * since the last call (all handles and rm_op_* calls of this process on the
 * current device) and clears it; always 0 in the product library.  RM_E_INVAL
 * for NULL out, RM_E_CUDA on a CUDA error. */
int rm_build_checked(void);
int rm_bounds_errors(int64_t* out);

/* Arena figures: out[0] = bytes reserved at create, out[1] = largest plan used
 * by any call so far, out[2] = number of distinct length buckets planned.
 * out: host int64[3]. */
int rm_arena_stats(const rm_handle* h, int64_t* out);

/* ---- measurement ---- */
/* Kernel classes of rm_profile_read. */
#define RM_K_GEMM      0   /* tcgen05 projections (QKV, out, FFN1, FFN2)              */
#define RM_K_SCORES    1   /* attention scores                                       */
#define RM_K_SOFTMAX   2   /* masked row softmax                                     */
#define RM_K_CONTEXT   3   /* attention context                                      */
#define RM_K_LAYERNORM 4   /* residual + LayerNorm                                   */
#define RM_K_EMBED     5   /* embedding gather (+ LN)                                */
#define RM_K_HEAD      6   /* scalar head                                            */
#define RM_K_ATTN_FUSED 7  /* fused attention (scores + softmax + context)           */
#define RM_K_CLASSES   8

/* Opt-in kernel timing.  every >= 1: each every-th rm_score* call from now on
 * records CUDA events around each of its kernel launches on its stream
 * (allocating events on first use); every = 0 switches it off.  Counters
 * restart at every call of rm_profile.  Host only; never synchronizes. */
int rm_profile(rm_handle* h, int32_t every);

/* Waits for the last stream, then for each class k < RM_K_CLASSES:
 * out_ms[k] = summed duration of the timed launches, out_launches[k] = their
 * number, out_flops[k] / out_bytes[k] = their algorithmic work (the FLOPs of
 * the contraction on the unpadded tokens; the HBM bytes the step must read and
 * write).  *out_total_launches = kernels launched by every rm_score* call since
 * create.  Arrays of RM_K_CLASSES entries (host). */
int rm_profile_read(rm_handle* h, double* out_ms, int64_t* out_launches, double* out_flops,
                    double* out_bytes, int64_t* out_total_launches);

/* Free the handle's device memory.  Waits for its last stream.  NULL is a no-op. */
void rm_destroy(rm_handle* h);

/* Message of the last error on this thread ("" if none). */
const char* rm_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* RM_H_ */
