// Row kernels of the scorer: embedding gather (+ embedding LayerNorm),
// residual + LayerNorm, the scalar head, and weight conversion.
//
// LayerNorm is one of the two "batch reduction" hot spots named in the
// TurboTransformers abstract ("TurboTransformers: An Efficient GPU Serving
// System For Transformer Models"); its proposed-method section parallelises
// it with the GPU memory hierarchy and thread-level parallelism in mind.
// Here: one warp per row; each lane holds its 16-byte chunks of the row in
// registers (a row is read from HBM exactly once), mean and biased variance
// are two register passes reduced with warp shuffles, fp32 math throughout.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace rmk {
namespace {

RMK_BOUNDS_UNIT(rowops)

constexpr int kWarps = 4;   // warps (rows) per CTA

template <int MAXC>
__device__ __forceinline__ void row_moments(const float (&v)[MAXC][8], int nch, int lane, int H,
                                            float& mean, float& rstd, float eps) {
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < MAXC; ++c)
    if (lane + 32 * c < nch) {
#pragma unroll
      for (int e = 0; e < 8; ++e) s += v[c][e];
    }
  mean = group_sum<32>(s) / static_cast<float>(H);
  float q = 0.f;
#pragma unroll
  for (int c = 0; c < MAXC; ++c)
    if (lane + 32 * c < nch) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = v[c][e] - mean;
        q += d * d;
      }
    }
  const float var = group_sum<32>(q) / static_cast<float>(H);
  rstd = rsqrtf(var + eps);
}

template <int MAXC>
__device__ __forceinline__ void normalize(float (&v)[MAXC][8], int nch, int lane, float mean,
                                          float rstd, const float* __restrict__ g,
                                          const float* __restrict__ b) {
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int ch = lane + 32 * c;
    if (ch < nch) {
      float gg[8], bb[8];
      load_f32x8(g + ch * 8, gg);
      load_f32x8(b + ch * 8, bb);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[c][e] = (v[c][e] - mean) * rstd * gg[e] + bb[e];
    }
  }
}

template <int MAXC, bool LN, typename TX>
__global__ void __launch_bounds__(kWarps * 32)
    embed_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ offsets, int n_seqs,
                 int T, const bf16* __restrict__ ew, const bf16* __restrict__ ep,
                 const float* __restrict__ g, const float* __restrict__ b, float eps, int V, int H,
                 TX* __restrict__ x, int32_t* __restrict__ err, L2PrefetchArgs pf,
                 const int32_t* __restrict__ pos_base, int P) {
  pdl_launch_dependents();
  l2_prefetch_share(pf);   // static weights: no need to wait for the previous kernel
  pdl_wait();
  const int t = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const int i = upper_index(offsets, n_seqs, t);
  // a segment that continues a shared prefix starts at position pos_base[i]
  const int pos = t - offsets[i] + (pos_base != nullptr ? pos_base[i] : 0);
  if (!in_bounds(pos >= 0 && pos < P)) return;   // checked build: offsets past the position table
  int id = ids[t];
  if (id < 0 || id >= V) {
    if (lane == 0 && err != nullptr) atomicAdd(err, 1);
    id = id < 0 ? 0 : V - 1;
  }
  const int nch = H >> 3;
  const bf16* wr = ew + static_cast<size_t>(id) * H;
  const bf16* pr = ep + static_cast<size_t>(pos) * H;
  float v[MAXC][8];
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int ch = lane + 32 * c;
    if (ch < nch) {
      float a[8], p[8];
      Chunk8<bf16>::load(wr + ch * 8, a);
      Chunk8<bf16>::load(pr + ch * 8, p);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[c][e] = a[e] + p[e];
    }
  }
  if (LN) {
    float mean, rstd;
    row_moments<MAXC>(v, nch, lane, H, mean, rstd, eps);
    normalize<MAXC>(v, nch, lane, mean, rstd, g, b);
  }
  TX* xr = x + static_cast<size_t>(t) * H;
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int ch = lane + 32 * c;
    if (ch < nch) Chunk8<TX>::store(xr + ch * 8, v[c]);
  }
}

// MODE 0: x = LN(y + x); MODE 1: x = y + x, z = LN(x); MODE 2: z = LN(x)
// Row types: TY for y, TX for the residual stream x, TZ for z (the decoder
// keeps x in fp32 and y, z in bf16; every other use has one type).
// Wide rows (H > 1024) are split over WPR warps, so that a lane holds at most
// four chunks: at H = 2048 one warp per row needs ~100 registers, which caps
// an SM at 16 resident warps, too few to keep HBM busy.  The WPR partial sums
// meet in shared memory (two CTA barriers per row pass).
template <typename TY, typename TX, typename TZ, int MAXC, int MODE, int WPR>
__global__ void __launch_bounds__(kWarps * 32)
    res_ln_kernel(const TY* __restrict__ y, TX* __restrict__ x, TZ* __restrict__ z,
                  const float* __restrict__ g, const float* __restrict__ b, int rows, int H,
                  float eps, L2PrefetchArgs pf) {
  pdl_launch_dependents();
  l2_prefetch_share(pf);
  pdl_wait();
  constexpr int LPR = 32 * WPR;                        // lanes per row
  __shared__ float part[kWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * (kWarps / WPR) + warp / WPR;
  const int lr = (warp % WPR) * 32 + lane;             // lane within the row
  const bool live = r < rows;
  if (WPR == 1 && !live) return;
  const int nch = H >> 3;
  const size_t base = static_cast<size_t>(live ? r : 0) * H;
  float v[MAXC][8];
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int ch = lr + LPR * c;
    if (live && ch < nch) {
      Chunk8<TX>::load(x + base + ch * 8, v[c]);
      if (MODE != 2) {
        float u[8];
        Chunk8<TY>::load(y + base + ch * 8, u);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[c][e] += u[e];
      }
    }
  }
  if (MODE == 1) {
    // the residual stream keeps the rounded sum, LN reads the same rounded values
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int ch = lr + LPR * c;
      if (live && ch < nch) {
        Chunk8<TX>::store(x + base + ch * 8, v[c]);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[c][e] = to_f32(from_f32<TX>(v[c][e]));
      }
    }
  }
  float mean, rstd;
  if (WPR == 1) {
    row_moments<MAXC>(v, nch, lr, H, mean, rstd, eps);
  } else {
    // the same two passes, each warp's share reduced across the row's warps
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < MAXC; ++c)
      if (live && lr + LPR * c < nch) {
#pragma unroll
        for (int e = 0; e < 8; ++e) s += v[c][e];
      }
    s = group_sum<32>(s);
    if (lane == 0) part[warp] = s;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < WPR; ++w) tot += part[(warp / WPR) * WPR + w];
    mean = tot / static_cast<float>(H);
    float q = 0.f;
#pragma unroll
    for (int c = 0; c < MAXC; ++c)
      if (live && lr + LPR * c < nch) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float d = v[c][e] - mean;
          q += d * d;
        }
      }
    q = group_sum<32>(q);
    __syncthreads();                                   // every warp has read the sums
    if (lane == 0) part[warp] = q;
    __syncthreads();
    float qt = 0.f;
#pragma unroll
    for (int w = 0; w < WPR; ++w) qt += part[(warp / WPR) * WPR + w];
    rstd = rsqrtf(qt / static_cast<float>(H) + eps);
  }
  if (!live) return;
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int ch = lr + LPR * c;
    if (ch < nch) {
      float gg[8], bb[8];
      load_f32x8(g + ch * 8, gg);
      load_f32x8(b + ch * 8, bb);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[c][e] = (v[c][e] - mean) * rstd * gg[e] + bb[e];
    }
  }
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    const int ch = lr + LPR * c;
    if (ch < nch) {
      if (MODE == 0) Chunk8<TX>::store(x + base + ch * 8, v[c]);
      else Chunk8<TZ>::store(z + base + ch * 8, v[c]);
    }
  }
}

__global__ void __launch_bounds__(kWarps * 32)
    head_kernel(const bf16* __restrict__ x, const int32_t* __restrict__ offsets, int n,
                const float* __restrict__ w, float br, int H, int last, float* __restrict__ out,
                const int32_t* __restrict__ out_index) {
  pdl_launch_dependents();
  pdl_wait();
  const int i = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= n) return;
  // out_index maps segments to output slots; a negative slot is not scored
  const int slot = out_index != nullptr ? out_index[i] : i;
  if (slot < 0) return;
  if (!in_bounds(offsets[i] >= 0 && offsets[i + 1] > offsets[i])) return;
  const int t = last ? offsets[i + 1] - 1 : offsets[i];
  const bf16* xr = x + static_cast<size_t>(t) * H;
  float acc = 0.f;
  for (int ch = lane; ch < (H >> 3); ch += 32) {
    float a[8], ww[8];
    Chunk8<bf16>::load(xr + ch * 8, a);
    load_f32x8(w + ch * 8, ww);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc = fmaf(a[e], ww[e], acc);
  }
  acc = group_sum<32>(acc);
  if (lane == 0) out[slot] = acc + br;
}

// Majority vote of K experts per input i (scores [K][n], expert-major): an
// expert answers [s > threshold]; the ensemble answers 1 with more than half
// of the votes, 0 with fewer, and on an even split the sign of the margins
// summed in expert order decides.
__global__ void __launch_bounds__(128)
    vote_kernel(const float* __restrict__ scores, int K, int n, float thr,
                int32_t* __restrict__ decision, int32_t* __restrict__ votes) {
  pdl_launch_dependents();
  pdl_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  int v = 0;
  float margin = 0.0f;
  for (int k = 0; k < K; ++k) {
    const float s = scores[static_cast<size_t>(k) * n + i];
    v += s > thr ? 1 : 0;
    margin = __fadd_rn(margin, __fsub_rn(s, thr));   // no contraction: the oracle's order and rounding
  }
  if (votes != nullptr) votes[i] = v;
  if (decision != nullptr) decision[i] = 2 * v > K ? 1 : (2 * v < K ? 0 : (margin > 0.0f ? 1 : 0));
}

// Best-of-N selection per group of candidates: best[g] = the index (within
// the group) of the highest score, the first one on ties; logodds[g] =
// r_1 - r_0, the log-odds that candidate 1 is preferred over candidate 0
// under the reward model's pairwise comparison (0 for a single candidate).
__global__ void __launch_bounds__(128)
    best_of_n_kernel(const float* __restrict__ scores, const int32_t* __restrict__ group_off,
                     int n_groups, int32_t* __restrict__ best, float* __restrict__ logodds) {
  pdl_launch_dependents();
  pdl_wait();
  const int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= n_groups) return;
  const int a = group_off[g], e = group_off[g + 1];
  if (!in_bounds(a >= 0 && e > a)) return;
  int arg = 0;
  float top = scores[a];
  for (int k = a + 1; k < e; ++k) {
    const float v = scores[k];
    if (v > top) {
      top = v;
      arg = k - a;
    }
  }
  if (best != nullptr) best[g] = arg;
  if (logodds != nullptr) logodds[g] = e - a >= 2 ? scores[a + 1] - scores[a] : 0.0f;
}

template <typename S>
__global__ void cvt_bf16_kernel(const S* __restrict__ src, bf16* __restrict__ dst, size_t n) {
  for (size_t k = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; k < n;
       k += static_cast<size_t>(gridDim.x) * blockDim.x)
    dst[k] = from_f32<bf16>(to_f32(src[k]));
}
template <typename S>
__global__ void cvt_f32_kernel(const S* __restrict__ src, float* __restrict__ dst, size_t n) {
  for (size_t k = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; k < n;
       k += static_cast<size_t>(gridDim.x) * blockDim.x)
    dst[k] = to_f32(src[k]);
}

L2PrefetchArgs pf_args(const L2Prefetch& pf) {
  L2PrefetchArgs a;
  for (int k = 0; k < 2; ++k) {
    a.ptr[k] = pf.ptr[k];
    a.bytes[k] = pf.bytes[k];
  }
  return a;
}

// Smallest supported chunks-per-lane count >= need (H <= 4096).
int pick_maxc(int H) {
  const int need = (H / 8 + 31) / 32;
  for (int m : {1, 2, 3, 4, 6, 8, 12, 16})
    if (m >= need) return m;
  return -1;
}

template <int MAXC, typename TX>
cudaError_t embed_t(const int32_t* ids, const int32_t* offsets, int n, int T, const void* ew,
                    const void* ep, const float* g, const float* b, float eps, int V, int P, int H,
                    void* x, int32_t* err, cudaStream_t st, const L2Prefetch& pf,
                    const int32_t* pos_base) {
  dim3 grid((T + kWarps - 1) / kWarps);
  if (g != nullptr)
    launch_k(embed_kernel<MAXC, true, TX>, grid, kWarps * 32, 0, st,
        ids, offsets, n, T, static_cast<const bf16*>(ew), static_cast<const bf16*>(ep), g, b, eps,
        V, H, static_cast<TX*>(x), err, pf_args(pf), pos_base, P);
  else
    launch_k(embed_kernel<MAXC, false, TX>, grid, kWarps * 32, 0, st,
        ids, offsets, n, T, static_cast<const bf16*>(ew), static_cast<const bf16*>(ep), g, b, eps,
        V, H, static_cast<TX*>(x), err, pf_args(pf), pos_base, P);
  return cudaGetLastError();
}

template <typename TY, typename TX, typename TZ, int MAXC, int WPR>
cudaError_t res_ln_t(const void* y, void* x, void* z, const float* g, const float* b, int rows,
                     int H, float eps, int mode, cudaStream_t st, const L2Prefetch& pf) {
  dim3 grid((rows + kWarps / WPR - 1) / (kWarps / WPR));
  const TY* yy = static_cast<const TY*>(y);
  TX* xx = static_cast<TX*>(x);
  TZ* zz = static_cast<TZ*>(z);
  if (mode == 0)
    launch_k(res_ln_kernel<TY, TX, TZ, MAXC, 0, WPR>, grid, kWarps * 32, 0, st, yy, xx, zz, g, b,
             rows, H, eps, pf_args(pf));
  else if (mode == 1)
    launch_k(res_ln_kernel<TY, TX, TZ, MAXC, 1, WPR>, grid, kWarps * 32, 0, st, yy, xx, zz, g, b,
             rows, H, eps, pf_args(pf));
  else
    launch_k(res_ln_kernel<TY, TX, TZ, MAXC, 2, WPR>, grid, kWarps * 32, 0, st, yy, xx, zz, g, b,
             rows, H, eps, pf_args(pf));
  return cudaGetLastError();
}

// One warp per row up to H = 1024 (at most 4 chunks a lane); 2 warps per row
// up to 2048 and 4 up to 4096.
template <typename TY, typename TX, typename TZ>
cudaError_t res_ln_dispatch(const void* y, void* x, void* z, const float* g, const float* b,
                            int rows, int H, float eps, int mode, cudaStream_t st,
                            const L2Prefetch& pf) {
  const int chunks = H / 8;
  if (chunks > 256) return res_ln_t<TY, TX, TZ, 4, 4>(y, x, z, g, b, rows, H, eps, mode, st, pf);
  if (chunks > 128) return res_ln_t<TY, TX, TZ, 4, 2>(y, x, z, g, b, rows, H, eps, mode, st, pf);
  if (chunks > 96) return res_ln_t<TY, TX, TZ, 4, 1>(y, x, z, g, b, rows, H, eps, mode, st, pf);
  if (chunks > 64) return res_ln_t<TY, TX, TZ, 3, 1>(y, x, z, g, b, rows, H, eps, mode, st, pf);
  if (chunks > 32) return res_ln_t<TY, TX, TZ, 2, 1>(y, x, z, g, b, rows, H, eps, mode, st, pf);
  return res_ln_t<TY, TX, TZ, 1, 1>(y, x, z, g, b, rows, H, eps, mode, st, pf);
}

}  // namespace

#define RMK_MAXC_SWITCH(maxc, CALL)      \
  switch (maxc) {                        \
    case 1: { constexpr int M_ = 1; return CALL; }  \
    case 2: { constexpr int M_ = 2; return CALL; }  \
    case 3: { constexpr int M_ = 3; return CALL; }  \
    case 4: { constexpr int M_ = 4; return CALL; }  \
    case 6: { constexpr int M_ = 6; return CALL; }  \
    case 8: { constexpr int M_ = 8; return CALL; }  \
    case 12: { constexpr int M_ = 12; return CALL; } \
    case 16: { constexpr int M_ = 16; return CALL; } \
    default: return cudaErrorInvalidValue;            \
  }

cudaError_t embed_launch(const int32_t* ids, const int32_t* offsets, int n_seqs, int T,
                         const void* emb_word, const void* emb_pos, const float* ln_g,
                         const float* ln_b, float eps, int V, int P, int H, void* x,
                         int32_t* err_count, cudaStream_t st, const L2Prefetch& pf,
                         const int32_t* pos_base, int x_dtype) {
  if (T == 0) return cudaSuccess;
  const int maxc = pick_maxc(H);
  if (x_dtype == 0)
    RMK_MAXC_SWITCH(maxc, (embed_t<M_, float>(ids, offsets, n_seqs, T, emb_word, emb_pos, ln_g,
                                              ln_b, eps, V, P, H, x, err_count, st, pf, pos_base)))
  RMK_MAXC_SWITCH(maxc, (embed_t<M_, bf16>(ids, offsets, n_seqs, T, emb_word, emb_pos, ln_g, ln_b,
                                           eps, V, P, H, x, err_count, st, pf, pos_base)))
}

cudaError_t res_ln_launch(const void* y, void* x, void* z, const float* g, const float* b, int T,
                          int H, float eps, int dtype, int mode, cudaStream_t st,
                          const L2Prefetch& pf) {
  if (T == 0) return cudaSuccess;
  if (H % 8 != 0 || H > 4096) return cudaErrorInvalidValue;
  if (dtype == 0) return res_ln_dispatch<float, float, float>(y, x, z, g, b, T, H, eps, mode, st, pf);
  if (dtype == 2) return res_ln_dispatch<bf16, float, bf16>(y, x, z, g, b, T, H, eps, mode, st, pf);
  if (dtype == 3) return res_ln_dispatch<float, float, bf16>(y, x, z, g, b, T, H, eps, mode, st, pf);
  return res_ln_dispatch<bf16, bf16, bf16>(y, x, z, g, b, T, H, eps, mode, st, pf);
}

cudaError_t bounds_errors_rowops(int32_t* out, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_bounds_rowops, sizeof(int32_t));
  if (e == cudaSuccess && reset) {
    const int32_t zero = 0;
    e = cudaMemcpyToSymbol(g_bounds_rowops, &zero, sizeof(int32_t));
  }
  return e;
}

cudaError_t head_launch(const void* x, const int32_t* offsets, int n_seqs, const float* w_r,
                        float b_r, int H, int last_token, float* out, cudaStream_t st,
                        const int32_t* out_index) {
  if (n_seqs == 0) return cudaSuccess;
  dim3 grid((n_seqs + kWarps - 1) / kWarps);
  launch_k(head_kernel, grid, kWarps * 32, 0, st, static_cast<const bf16*>(x), offsets, n_seqs, w_r,
           b_r, H, last_token, out, out_index);
  return cudaGetLastError();
}

cudaError_t vote_launch(const float* scores, int K, int n, float threshold, int32_t* decision,
                        int32_t* votes, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  launch_k(vote_kernel, dim3((n + 127) / 128), dim3(128), 0, st, scores, K, n, threshold, decision,
           votes);
  return cudaGetLastError();
}

cudaError_t best_of_n_launch(const float* scores, const int32_t* group_off, int n_groups,
                             int32_t* best, float* logodds, cudaStream_t st) {
  if (n_groups == 0) return cudaSuccess;
  launch_k(best_of_n_kernel, dim3((n_groups + 127) / 128), dim3(128), 0, st, scores, group_off,
           n_groups, best, logodds);
  return cudaGetLastError();
}

cudaError_t cvt_to_bf16_launch(const void* src, int src_dtype, void* dst, size_t n,
                               cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<size_t>((n + 255) / 256, 148 * 16));
  if (src_dtype == 0)
    launch_k(cvt_bf16_kernel<float>, blocks, 256, 0, st, static_cast<const float*>(src),
                                                   static_cast<bf16*>(dst), n);
  else
    launch_k(cvt_bf16_kernel<bf16>, blocks, 256, 0, st, static_cast<const bf16*>(src),
                                                  static_cast<bf16*>(dst), n);
  return cudaGetLastError();
}

cudaError_t cvt_to_f32_launch(const void* src, int src_dtype, float* dst, size_t n,
                              cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<size_t>((n + 255) / 256, 148 * 16));
  if (src_dtype == 0)
    launch_k(cvt_f32_kernel<float>, blocks, 256, 0, st, static_cast<const float*>(src), dst, n);
  else
    launch_k(cvt_f32_kernel<bf16>, blocks, 256, 0, st, static_cast<const bf16*>(src), dst, n);
  return cudaGetLastError();
}

}  // namespace rmk
