/*
 * rm_ops.h -- one C entry point per step of the scoring hot path.
 *
 * rm_score (rm.h) chains exactly these launchers; they are exported so that
 * each step can be checked on its own against the fp64 oracle.  All pointers
 * are DEVICE pointers unless marked host; all work is asynchronous on stream
 * (a cudaStream_t as void*).  Return RM_OK or a negative RM_E_* code (rm.h);
 * arguments are validated on the host before anything is enqueued.
 *
 * Packed varlen layout shared by the steps (TurboTransformers review,
 * "variable-length input" in the abstract; no padding to a fixed length):
 *   offsets[n+1]  int32 token offsets, sequence i = rows offsets[i]..offsets[i+1]-1,
 *                 L_i = offsets[i+1]-offsets[i] >= 1.
 *   X[T][H]       activations, row-major.
 *   QKV[T][3H]    Q in columns 0..H-1, K in H..2H-1, V in 2H..3H-1; head j
 *                 uses columns j*d .. j*d+d-1 of each.
 *   S             attention scores/probabilities.  With Lp_i = round_up(L_i, 8)
 *                 the entry (sequence i, head j, query r, key c) is at
 *                 S[s_off[i] + (j*L_i + r)*Lp_i + c], s_off[i] = sum_{k<i} h*L_k*Lp_k.
 *                 Only c < L_i (causal: c <= r) is ever read or written.
 *   rb_off[n+1]   prefix sums of ceil(L_i/64): the 64-query row blocks that
 *                 the attention launches distribute over CTAs.
 * dtype arguments: RM_F32 (0) or RM_BF16 (1) from rm.h.
 */
#ifndef RM_OPS_H_
#define RM_OPS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Host helper: rb_off[n+1] and s_off[n+1] for the layout above (host arrays).
 * Returns RM_OK, RM_E_INVAL for a length < 1 or non-monotone offsets. */
int rm_varlen_meta(const int32_t* offsets, int32_t n, int32_t n_heads,
                   int32_t* rb_off, int64_t* s_off);

/* Y[M][N] = act(X[M][K] . W[N][K]^T + bias[N]) -- the QKV, output and FFN
 * projections (the "BLAS routines" of the TurboTransformers abstract; tensor
 * cores per its proposed-method section).  bf16 operands, fp32 accumulation
 * in tensor memory (tcgen05), bias/GELU in the epilogue.
 *   x: bf16 [M][K] row-major; w: bf16 [N][K] row-major (nn.Linear layout);
 *   bias: fp32 [N] or NULL; y: [M][N] row-major of y_dtype (RM_F32|RM_BF16).
 *   act: 0 = none, 1 = GELU (erf), 2 = GELU (tanh).
 * Requires M >= 1, N and K multiples of 8, 16-byte aligned x, w, y. */
int rm_op_gemm(const void* x, const void* w, const float* bias, void* y, int32_t y_dtype,
               int32_t M, int32_t N, int32_t K, int32_t act, void* stream);

/* rm_op_gemm with an explicit output tile (the projections of rm_op_gemm; the
 * tile choice itself has no counterpart in the pages and is exposed for
 * testing every tile and for tuning): cg = 1 (one CTA per 128 x bn tile,
 * bn in {64, 96, 128, 160, 192, 224, 256}) or cg = 2 (a cluster of two CTAs
 * per 256 x bn tile on the pair MMA, bn in {128, 192, 256}); cg = 0 takes the
 * tile rm_gemm_tile picks (what rm_op_gemm does).  Same arguments and
 * requirements as rm_op_gemm; RM_E_INVAL for a tile outside these sets. */
int rm_op_gemm_tiled(const void* x, const void* w, const float* bias, void* y, int32_t y_dtype,
                     int32_t M, int32_t N, int32_t K, int32_t act, int32_t cg, int32_t bn,
                     void* stream);

/* Y[M][N] += X[M][K] . W[N][K]^T + bias[N] with Y in fp32: the pre-LN
 * decoder's output projection and FFN2 added straight into its fp32 residual
 * stream (the residual additions of the layer equations, which the
 * TurboTransformers abstract pairs with the LayerNorm batch reduction; here
 * folded into the GEMM that produces the addend).  The tile is accumulated in
 * fp32 and added to y in L2; each element of y is added to exactly once, with
 * one fp32 rounding, so the result equals a separate fp32 addition of the
 * rm_op_gemm output and does not depend on the order of the tiles.  Same
 * arguments as rm_op_gemm_tiled with y_dtype = RM_F32 and act = 0 (RM_E_INVAL
 * for any other); y must be 16-byte aligned and is read and written. */
int rm_op_gemm_accumulate(const void* x, const void* w, const float* bias, void* y,
                          int32_t y_dtype, int32_t M, int32_t N, int32_t K, int32_t act,
                          int32_t cg, int32_t bn, void* stream);

/* Majority vote of an ensemble of K scorer replicas ("experts"), the SambaNova
 * blog's accuracy section (Figs. 4-5: several TinyBERT instances vote on each
 * input).  scores: device float[K][n], expert k's score of input i at
 * scores[k*n + i].  Expert k answers [score > threshold]; decision[i] = 1 when
 * more than K/2 experts answer 1, 0 when fewer, and on an even split 1 iff the
 * margins sum_k (score - threshold), added in expert order in fp32, are > 0.
 * decision, votes: device int32[n], either may be NULL.  RM_E_INVAL for
 * K < 1, n < 0 or NULL scores.  Asynchronous on stream. */
int rm_op_vote(const float* scores, int32_t K, int32_t n, float threshold, int32_t* decision,
               int32_t* votes, void* stream);

/* Host only (no counterpart in the pages): the output tile the projections
 * without an activation use for an M x N x K product on a device with num_sms
 * SMs (a GELU epilogue may take
 * a single-CTA tile where this returns a pair).  out[0] = cg (1 or 2),
 * out[1] = bn.  RM_E_INVAL for M, N, K or num_sms < 1 or out == NULL. */
int rm_gemm_tile(int32_t M, int32_t N, int32_t K, int32_t num_sms, int32_t* out);

/* X[t] = E_word[clamp(ids[t])] + E_pos[t - offsets[i]] for each token t of
 * sequence i, then (ln_g != NULL) the embedding LayerNorm.  ids out of 0..V-1
 * are clamped and counted with atomicAdd into *err_count (may be NULL).
 * E_word: bf16 [V][H]; E_pos: bf16 [P][H]; ln_g, ln_b: fp32 [H] or NULL;
 * x: [T][H] of x_dtype (RM_BF16, or RM_F32 for the decoder's fp32 residual
 * stream).  Requires every L_i <= P. */
int rm_op_embed(const int32_t* ids, const int32_t* offsets, int32_t n_seqs, int32_t T,
                const void* emb_word, const void* emb_pos, const float* ln_g, const float* ln_b,
                float eps, int32_t V, int32_t P, int32_t H, void* x, int32_t x_dtype,
                int32_t* err_count, void* stream);

/* Attention scores S = (Q K^T)/sqrt(d) per sequence and head, only the valid
 * L_i x L_i block (causal: keys c <= r).  qkv: bf16 [T][3H]; S: bf16.
 * n_row_blocks = rb_off[n] (host value); head_dim even, <= 128. */
int rm_op_attn_scores(const void* qkv, void* S, const int32_t* offsets, const int32_t* rb_off,
                      const int64_t* s_off, int32_t n_seqs, int32_t n_row_blocks,
                      int32_t n_heads, int32_t head_dim, int32_t causal, void* stream);

/* Masked row softmax in place over every row of S: p_c = exp(s_c - max)/sum
 * over keys c < L_i (causal: c <= r) -- the Softmax batch reduction of the
 * TurboTransformers abstract.  fp32 math; s_dtype RM_BF16 or RM_F32.
 * T = offsets[n] and max_len >= every L_i (host values). */
int rm_op_softmax(void* S, int32_t s_dtype, const int32_t* offsets, const int64_t* s_off,
                  int32_t n_seqs, int32_t T, int32_t n_heads, int32_t max_len, int32_t causal,
                  void* stream);

/* The same softmax by row-length class: the rows are first regrouped on the
 * device by the 8-element chunks of their length (<= 1, 2, 4, 8, 16, 32, 64,
 * 96, 128) into scratch, each row recording its sequence, and one persistent
 * kernel then takes each class with lanes per row fitted to it (one lane for
 * rows of up to 8 keys ... 32 lanes holding 4 chunks each for 1024), so that
 * short rows leave no lanes idle when the batch also holds long ones and no
 * lane group searches the offsets.  Same arguments as rm_op_softmax, plus
 * scratch: device memory of rm_softmax_scratch_bytes(n_seqs, T, n_heads) bytes
 * (about 4 bytes per row), 16-byte aligned, overwritten by the call.  The
 * per-row arithmetic is rm_op_softmax's; only the order in which a row's
 * exponentials are summed follows its lanes per row.  RM_E_INVAL for NULL
 * pointers or bad sizes. */
int rm_op_softmax_classes(void* S, int32_t s_dtype, const int32_t* offsets, const int64_t* s_off,
                          int32_t n_seqs, int32_t T, int32_t n_heads, int32_t max_len,
                          int32_t causal, void* scratch, void* stream);
/* Host only: the scratch bytes rm_op_softmax_classes needs (0 for bad sizes). */
size_t rm_softmax_scratch_bytes(int32_t n_seqs, int32_t T, int32_t n_heads);

/* Context C = P V per sequence and head into ctx[T][H] (head j in columns
 * j*d..j*d+d-1).  S holds P (bf16), qkv: bf16 [T][3H], ctx: bf16 [T][H]. */
int rm_op_attn_context(const void* S, const void* qkv, void* ctx, const int32_t* offsets,
                       const int32_t* rb_off, const int64_t* s_off, int32_t n_seqs,
                       int32_t n_row_blocks, int32_t n_heads, int32_t head_dim, int32_t causal,
                       void* stream);

/* The three attention steps above in one kernel: per sequence, head and
 * 64-query block, S = QK^T/sqrt(d) over keys c < L_i (causal: c <= r) with an
 * online (running max and sum) softmax, P rounded to bf16, C = P V written to
 * ctx[T][H].  No score buffer.  qkv: bf16 [T][3H]; ctx: bf16 [T][H]. */
int rm_op_attn_fused(const void* qkv, void* ctx, const int32_t* offsets, const int32_t* rb_off,
                     int32_t n_seqs, int32_t n_row_blocks, int32_t n_heads, int32_t head_dim,
                     int32_t causal, void* stream);

/* The same attention step on tiles of 64 consecutive packed rows: a tile
 * holds whole short sequences and pieces of long ones, and each CTA takes one
 * tile and a group of heads, its K/V rows (the tile's key range) arriving by
 * TMA in 64-row chunks while the previous chunk is multiplied.  A query row
 * admits the keys of its own sequence only (c <= r too when causal); online
 * softmax in fp32, P rounded to bf16 for P V, as in rm_op_attn_fused.
 * head_dim 64 or 128 (H = n_heads * head_dim); qkv: bf16 [T][3H]; ctx: bf16
 * [T][H]; offsets: DEVICE int32[n+1] with offsets[n] = T (host value T);
 * max_len: a host bound on every L_i (it sizes the launch: CTAs take fewer
 * heads each when rows are long).  RM_E_INVAL for other head dims or sizes < 1; waits that give up (none in
 * normal operation) count into an internal error word. */
int rm_op_attn_tiles(const void* qkv, void* ctx, const int32_t* offsets, int32_t n_seqs, int32_t T,
                     int32_t n_heads, int32_t head_dim, int32_t max_len, int32_t causal,
                     void* stream);

/* Tiles of the tensor-core attention (rm_op_attn_tc): a greedy cut of the
 * packed batch into runs of whole sequences of at most 128 rows each.
 * offsets: HOST int32[n_seqs+1] with offsets[0] = 0 and every length in
 * 1..128; tiles: HOST int32[n_seqs+1] (caller-owned), receives tiles[0..k]
 * with tiles[0] = 0 and tiles[k] = n_seqs, tile j holding sequences
 * [tiles[j], tiles[j+1]).  Returns k (>= 1), or RM_E_INVAL / RM_E_RANGE.
 * This cut of the batch has no counterpart in the pages; it is the layout
 * of the kernel below. */
int rm_attn_tc_tiles(const int32_t* offsets, int32_t n_seqs, int32_t* tiles);

/* The attention step of rm_op_attn_tiles on the 5th-generation tensor cores,
 * for head_dim 64 and sequences of at most 128 tokens (the TurboTransformers
 * proposed-method section's batched QK^T, batch softmax and PV, fused): per
 * tile of rm_attn_tc_tiles and head, S = QK^T (tcgen05.mma into tensor
 * memory), the row softmax over the row's own sequence (c <= r too when
 * causal) in fp32 with P rounded to bf16, and C = P V (tcgen05.mma), written
 * to ctx.  qkv: bf16 [T][3H], H = 64 * n_heads; ctx: bf16 [T][H]; offsets:
 * DEVICE int32[n_seqs+1] with offsets[n_seqs] = T (host value T); tiles:
 * DEVICE int32[n_tiles+1] as rm_attn_tc_tiles wrote them for the same
 * offsets.  RM_E_INVAL for NULL pointers or sizes < 1; waits that give up
 * (none in normal operation) count into an internal error word. */
int rm_op_attn_tc(const void* qkv, void* ctx, const int32_t* offsets, const int32_t* tiles,
                  int32_t n_tiles, int32_t n_seqs, int32_t T, int32_t n_heads, int32_t causal,
                  void* stream);

/* Work items of the long-row tensor-core attention (rm_op_attn_tcl): every
 * run of 128 query rows of a sequence, item = (sequence << 2) | tile (tile
 * 0..3 covers rows 128*tile ..), those that read the most 128-key chunks
 * first (causal != 0: a tile reads keys up to its own last row only).
 * offsets: HOST int32[n_seqs+1] with offsets[0] = 0 and every length in
 * 1..512; items: HOST int32[4 * n_seqs] (caller-owned).  Returns the item
 * count (sum over sequences of ceil(L / 128)), or RM_E_INVAL / RM_E_RANGE.
 * This cut has no counterpart in the pages; it is the layout of the kernel
 * below. */
int rm_attn_tcl_items(const int32_t* offsets, int32_t n_seqs, int32_t causal, int32_t* items);

/* rm_op_attn_tc for sequences of up to 512 tokens (head_dim 64): per item of
 * rm_attn_tcl_items and head, S = Q K^T for the item's 128 query rows against
 * every 128-key chunk of its sequence (tcgen05.mma into tensor memory), the
 * row softmax over the row's own sequence (c <= r too when causal) in fp32
 * with P rounded to bf16, and C = P V (tcgen05.mma), written to ctx.  qkv:
 * bf16 [T][3H], H = 64 * n_heads; ctx: bf16 [T][H]; offsets: DEVICE
 * int32[n_seqs+1] with offsets[n_seqs] = T (host value T); items: DEVICE
 * int32[n_items] as rm_attn_tcl_items wrote them for the same offsets and
 * causal flag.  RM_E_INVAL for NULL pointers, sizes < 1 or n_items >
 * 4 * n_seqs; waits that give up (none in normal operation) count into an
 * internal error word. */
int rm_op_attn_tcl(const void* qkv, void* ctx, const int32_t* offsets, const int32_t* items,
                   int32_t n_items, int32_t n_seqs, int32_t T, int32_t n_heads, int32_t causal,
                   void* stream);

/* The materialised attention step (rm_op_attn_scores -> rm_op_softmax ->
 * rm_op_attn_context) without any device allocation: the score matrix and the
 * per-call metadata live in one file-scope device array of 8 MiB of scores
 * plus 65,552 bytes of metadata (8,454,160 bytes) that
 * every device loading this library keeps until the process exits.  The pages
 * have no counterpart to this entry point; it exists for callers that cannot
 * allocate device memory where they run the step (a plugin inside another
 * runtime that owns the device memory pool, or a path where cudaMalloc is not
 * allowed because it may synchronize the device or fail under pressure).
 *   qkv: bf16 [T][3H]; ctx: bf16 [T][H] (written); offsets: HOST int32[n+1].
 * Limits: n_seqs <= 4096, every L_i <= 1024 and sum_i n_heads*L_i*round_up(L_i,8)
 * <= 4 Mi score entries; larger calls return RM_E_RANGE (use the three
 * caller-allocated entry points instead).  The first call in a CUDA context (for most
 * callers, the device's primary context) looks up the array's device address
 * (cudaGetSymbolAddress) and caches it for that context; make that first call
 * before any stream capture.  The call copies its metadata into the
 * array on stream and calls no cudaMalloc or cudaFree.  Every call shares the
 * array and it keeps the last call's contents (nothing in it needs to start at
 * zero: each call writes every entry it reads), so calls that overlap on the
 * GPU -- on different streams, or from different threads without ordering --
 * race and give wrong results. */
int rm_op_attention_noalloc(const void* qkv, void* ctx, const int32_t* offsets, int32_t n_seqs,
                            int32_t n_heads, int32_t head_dim, int32_t causal, void* stream);

/* Residual + LayerNorm over rows of length H (the LayerNorm batch reduction of
 * the TurboTransformers abstract), fp32 math:
 *   mode 0 (post-LN): x = LN(y + x)              (z unused, may be NULL)
 *   mode 1 (pre-LN):  x = y + x;  z = LN(x)      (both written)
 *   mode 2 (plain):   z = LN(x)                  (y unused, may be NULL)
 * LN(u) = g * (u - mean)/sqrt(var + eps) + b with the biased variance.
 * y, x, z: [T][H]; g, b: fp32 [H].  Row types by dtype: RM_F32 or RM_BF16 for
 * all three; RM_ROWS_RESID_F32 for x in fp32 with y and z in bf16;
 * RM_ROWS_F32_IN for y and x in fp32 with z in bf16 (the pre-LN decoder's
 * layout: its residual stream and the sublayer outputs added to it stay fp32,
 * so that each addition is rounded once to fp32 instead of to bf16). */
#define RM_ROWS_RESID_F32 2
#define RM_ROWS_F32_IN 3
int rm_op_res_ln(const void* y, void* x, void* z, const float* g, const float* b, int32_t T,
                 int32_t H, float eps, int32_t dtype, int32_t mode, void* stream);

/* Scalar head ("Learning to summarize from human feedback" summary, method
 * section): out[i] = w_r . u_i + b_r where u_i = x[offsets[i]] (last_token =
 * 0) or x[offsets[i+1]-1] (last_token = 1).  x: bf16 [T][H]; w_r: fp32 [H];
 * out: fp32 [n]. */
int rm_op_head(const void* x, const int32_t* offsets, int32_t n_seqs, const float* w_r,
               float b_r, int32_t H, int32_t last_token, float* out, void* stream);

/* Host only: the arena plan for one call of a handle created with cfg.
 * Fills, for each intermediate buffer k < returned count (<= max_bufs):
 * out_off[k], out_bytes[k] (byte offset/size in the arena), out_first[k],
 * out_last[k] (first and last step that uses it; buffers whose step ranges
 * overlap are live together and never share bytes).  *out_peak = arena bytes
 * the plan needs.  T tokens, n_seqs sequences, s_elems score elements
 * (s_off[n]).  Returns the buffer count or a negative RM_E_* code. */
int rm_arena_plan(const void* cfg, int32_t T, int32_t n_seqs, int64_t s_elems,
                  int64_t* out_off, int64_t* out_bytes, int32_t* out_first, int32_t* out_last,
                  int32_t max_bufs, int64_t* out_peak);

#ifdef __cplusplus
}
#endif
#endif /* RM_OPS_H_ */
