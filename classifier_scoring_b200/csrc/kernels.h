// Internal launchers of the scorer's kernels (host-callable, not exported).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rmk {

// ---- tcgen05 GEMM (gemm_tc.cu) ----
constexpr int kGemmTileCount = 7;
extern const int kGemmTileWidths[kGemmTileCount];   // 64, 96, 128, 160, 192, 224, 256
// Output tile: cg = 1 (one CTA, 128 x bn) or 2 (a CTA pair, 256 x bn, each CTA
// loading bn/2 rows of the weights).
struct GemmTile {
  int cg;
  int bn;
  int b_box() const { return bn / cg; }   // weight rows per TMA box
};
GemmTile gemm_pick(int M, int N, int K, int num_sms, int act = 0);
// One thread waits on an mbarrier that nothing completes, with the GEMM's
// bounded wait and the given limit; writes 1 to *d_timed_out when the wait
// gave up, and the time it took.
cudaError_t bounded_wait_selftest(unsigned long long limit_ns, int* d_timed_out,
                                  unsigned long long* d_elapsed_ns, cudaStream_t st);
inline int gemm_tile_index(int box_rows) { return (box_rows - 64) / 32; }
// a: bf16 [M][K] map with box {64, 128}; b: bf16 [N][K] map with box {64, tile.b_box()};
// y: [>= M][N] output map of make_tmap_store (fp32 when out_f32, else bf16).
// yacc: nullptr to store the tile through y; else (act 0 and out_f32 only)
// the 16-byte aligned row-major fp32 [M][N] tensor that the tile is added to
// in L2 (each sum rounded once to fp32); y is then not used.
// Persistent grid of units of cg CTAs, each walking its share of the tiles.
// With 1-CTA tiles, the tiles of a last partial round (or of a single round
// that fills at most half of the SMs) are cut into gemm_tail_split column
// slices of bn / split columns each; b_split is the weights' map with boxes
// of bn / split rows (b itself when the split is 1).
int gemm_tail_split(GemmTile tile, int M, int N, int num_sms);
cudaError_t gemm_launch(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b_split,
                        const CUtensorMap& y, void* yacc, GemmTile tile, int M, int N, int K,
                        const float* bias, bool out_f32, int act, int* err, int num_sms,
                        cudaStream_t st);

// ---- TMA descriptors (tma.cpp) ----
// 2-D bf16 row-major [rows][cols] tensor, box {64 cols, box_rows}, 128-byte swizzle,
// zero fill outside.  Returns false (message in *why) if the driver refuses it.
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows, const char** why);
// 2-D row-major [rows][cols] output of the GEMM (bf16, or fp32 when f32), box
// {32 cols, 32 rows}, 64-byte (bf16) or 128-byte (fp32) swizzle: the layout of
// the GEMM epilogue's staging boxes.  Stores outside the tensor are clipped.
bool make_tmap_store(CUtensorMap* map, void* base, uint64_t rows, uint64_t cols, bool f32,
                     const char** why);

// Weights of the next GEMMs to pull into L2 while a latency-bound kernel runs
// (the whole model does not stay in L2, so a GEMM would otherwise start on
// cold weights).  Each CTA issues bulk L2 prefetches for its slice.
struct L2Prefetch {
  const void* ptr[2] = {nullptr, nullptr};
  unsigned long long bytes[2] = {0, 0};
};

// ---- row kernels (rowops.cu) ----
cudaError_t embed_launch(const int32_t* ids, const int32_t* offsets, int n_seqs, int T,
                         const void* emb_word, const void* emb_pos, const float* ln_g,
                         const float* ln_b, float eps, int V, int P, int H, void* x,
                         int32_t* err_count, cudaStream_t st, const L2Prefetch& pf = {},
                         const int32_t* pos_base = nullptr, int x_dtype = 1);
// dtype: 0 fp32, 1 bf16, 2 residual x fp32 with y, z bf16, 3 y and x fp32 with
// z bf16; mode 0 post, 1 pre, 2 plain (see rm_ops.h)
cudaError_t res_ln_launch(const void* y, void* x, void* z, const float* g, const float* b, int T,
                          int H, float eps, int dtype, int mode, cudaStream_t st,
                          const L2Prefetch& pf = {});
cudaError_t head_launch(const void* x, const int32_t* offsets, int n_seqs, const float* w_r,
                        float b_r, int H, int last_token, float* out, cudaStream_t st,
                        const int32_t* out_index = nullptr);
// majority vote of K experts' scores [K][n]
cudaError_t vote_launch(const float* scores, int K, int n, float threshold, int32_t* decision,
                        int32_t* votes, cudaStream_t st);
// per group g (candidates group_off[g]..group_off[g+1]-1 of scores): the
// first highest score's index and r_1 - r_0
cudaError_t best_of_n_launch(const float* scores, const int32_t* group_off, int n_groups,
                             int32_t* best, float* logodds, cudaStream_t st);
// weight conversion at create
cudaError_t cvt_to_bf16_launch(const void* src, int src_dtype, void* dst, size_t n,
                               cudaStream_t st);
cudaError_t cvt_to_f32_launch(const void* src, int src_dtype, float* dst, size_t n,
                              cudaStream_t st);

// Bounds counters of the checked build (RM_CHECKED), per translation unit:
// read into *out, cleared when reset.  Always 0 in the product build.
cudaError_t bounds_errors_rowops(int32_t* out, bool reset);
cudaError_t bounds_errors_attention(int32_t* out, bool reset);
cudaError_t bounds_errors_attention_tc(int32_t* out, bool reset);

// ---- attention (attention.cu) ----
cudaError_t attn_scores_launch(const void* qkv, void* S, const int32_t* offsets,
                               const int32_t* rb_off, const int64_t* s_off, int n_seqs,
                               int n_row_blocks, int n_heads, int head_dim, int causal,
                               cudaStream_t st);
// err: device error words (ERR_TIMEOUT counts waits that gave up) or NULL
cudaError_t softmax_launch(void* S, int s_dtype, const int32_t* offsets, const int64_t* s_off,
                           int n_seqs, int T, int n_heads, int max_len, int causal, int* err,
                           cudaStream_t st);
// The masked softmax by row-length class: the rows are regrouped on the device
// by the class of their length into scratch (device,
// softmax_classes_scratch_bytes(n_seqs, T, n_heads) bytes, 16-byte aligned),
// then one persistent kernel takes each class up to that of max_len with lane
// groups sized to it.
size_t softmax_classes_scratch_bytes(int n_seqs, int T, int n_heads);
cudaError_t softmax_classes_launch(void* S, int s_dtype, const int32_t* offsets,
                                   const int64_t* s_off, int n_seqs, int T, int n_heads,
                                   int max_len, int causal, void* scratch, int num_sms,
                                   cudaStream_t st);
// scores + masked softmax + context in one kernel (probabilities stay in registers)
cudaError_t attn_fused_launch(const void* qkv, void* ctx, const int32_t* offsets,
                              const int32_t* rb_off, int n_seqs, int n_row_blocks, int n_heads,
                              int head_dim, int causal, cudaStream_t st,
                              const L2Prefetch& pf = {});
// Packed-row attention (head_dim 64 or 128): tiles of 64 consecutive
// packed rows of any sequences, a group of heads per CTA, TMA-fed K/V chunks
// of each tile's key range; max_len (>= every L_i) sizes the head groups;
// err: device error words (ERR_TIMEOUT).
cudaError_t attn_tile_launch(const void* qkv, void* ctx, const int32_t* offsets, int n_seqs, int T,
                             int n_heads, int head_dim, int max_len, int causal, int* err,
                             int num_sms, cudaStream_t st, const L2Prefetch& pf = {});
// Tensor-core attention (attention_tc.cu): head dim 64, every sequence at
// most 128 tokens.  tiles: DEVICE int32[n_tiles + 1], tile k holds sequences
// [tiles[k], tiles[k+1]) (at most 128 rows), as attn_tc_tiles builds them.
cudaError_t attn_tc_launch(const void* qkv, void* ctx, const int32_t* offsets,
                           const int32_t* tiles, int n_tiles, int n, int T, int nh, int causal,
                           int* err, int num_sms, cudaStream_t st, const L2Prefetch& pf = {});
// Tensor-core attention for sequences of up to 512 tokens, head dim 64: work
// items of 128 query rows of one sequence, item = (sequence << 2) | tile.
// attn_tcl_items writes the items of every sequence (offsets: host, n + 1
// entries, every length 1..512; items: capacity sum of ceil(L / 128) <= 4n),
// those with the most key chunks first, and returns their count.
int32_t attn_tcl_items(const int32_t* offsets, int32_t n, int32_t causal, int32_t* items);
cudaError_t attn_tcl_launch(const void* qkv, void* ctx, const int32_t* offsets,
                            const int32_t* items, int n_items, int n, int T, int nh, int causal,
                            int* err, int num_sms, cudaStream_t st, const L2Prefetch& pf = {});
// Greedy cut of the packed batch into tiles of whole sequences of at most 128
// rows (host; every sequence at most 128 tokens): writes tiles[0..n_tiles],
// returns n_tiles.
int32_t attn_tc_tiles(const int32_t* offsets, int32_t n, int32_t* tiles);
// Causal fused attention over segments that may continue a shared prefix:
// query row r of segment i attends to the pre_len[i] rows starting at packed
// row pre_start[i] (all of them) and to rows 0..r of its own segment.
// head_dim % 8 == 0, <= 128.
cudaError_t attn_fused_prefix_launch(const void* qkv, void* ctx, const int32_t* offsets,
                                     const int32_t* rb_off, const int32_t* pre_start,
                                     const int32_t* pre_len, int n_seqs, int n_row_blocks,
                                     int n_heads, int head_dim, cudaStream_t st,
                                     const L2Prefetch& pf = {});
cudaError_t attn_context_launch(const void* S, const void* qkv, void* ctx, const int32_t* offsets,
                                const int32_t* rb_off, const int64_t* s_off, int n_seqs,
                                int n_row_blocks, int n_heads, int head_dim, int causal,
                                cudaStream_t st);

}  // namespace rmk
