// Varlen multi-head attention in three kernels over the packed layout:
//   scores   S = Q K^T / sqrt(d) for each sequence and head, only the valid
//            L x L block (causal: the lower triangle);
//   softmax  masked row softmax in place on S -- the Softmax batch reduction
//            of the TurboTransformers abstract ("TurboTransformers: An
//            Efficient GPU Serving System For Transformer Models");
//   context  C = P V into the packed [T][H] context.
// No token of one sequence ever meets a token of another: every CTA works
// inside one sequence, located from the per-sequence offsets.
//
// The two small per-sequence contractions (L <= 1024, d <= 128) use warp-level
// mma.sync m16n8k16 bf16 tiles with fp32 accumulation; together they are a few
// percent of the scorer's FLOPs.
#include <math.h>

#include <algorithm>
#include <climits>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rmk {
namespace {

RMK_BOUNDS_UNIT(attention)

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct BlockSeq {
  int t0, L, Lp, row0;
  long long sbase;
};

// CTA blockIdx.x -> (sequence, 64-row query block).
__device__ __forceinline__ BlockSeq locate_block(const int32_t* offsets, const int32_t* rb_off,
                                                 const int64_t* s_off, int n, int b) {
  BlockSeq q;
  const int i = upper_index(rb_off, n, b);
  q.t0 = offsets[i];
  q.L = offsets[i + 1] - q.t0;
  q.Lp = (q.L + 7) & ~7;
  q.row0 = (b - rb_off[i]) * 64;
  q.sbase = s_off[i];
  return q;
}

// 4 warps x 16 query rows; keys in blocks of 64 staged in shared memory.
template <int DP>
__global__ void __launch_bounds__(128)
    attn_scores_kernel(const bf16* __restrict__ qkv, bf16* __restrict__ S,
                       const int32_t* __restrict__ offsets, const int32_t* __restrict__ rb_off,
                       const int64_t* __restrict__ s_off, int n, int H, int d, float scale,
                       int causal) {
  __shared__ __align__(16) bf16 ks[64][DP + 8];
  pdl_launch_dependents();
  pdl_wait();
  const BlockSeq q = locate_block(offsets, rb_off, s_off, n, blockIdx.x);
  if (!in_bounds(q.L >= 1 && q.row0 < q.L)) return;   // checked build: inconsistent row blocks
  const int hd = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const size_t H3 = 3 * static_cast<size_t>(H);
  const bf16* qb = qkv + static_cast<size_t>(q.t0) * H3 + hd * d;
  const bf16* kbp = qkv + static_cast<size_t>(q.t0) * H3 + H + hd * d;
  bf16* sb = S + q.sbase + static_cast<size_t>(hd) * q.L * q.Lp;
  const int ra = q.row0 + warp * 16 + g, rb = ra + 8;

  auto ld_pair = [&](const bf16* base, int r, int c) -> uint32_t {
    return (r < q.L && c < d) ? *reinterpret_cast<const uint32_t*>(base + r * H3 + c) : 0u;
  };
  uint32_t qa[DP / 16][4];
#pragma unroll
  for (int s = 0; s < DP / 16; ++s) {
    const int c0 = s * 16 + 2 * tq;
    qa[s][0] = ld_pair(qb, ra, c0);
    qa[s][1] = ld_pair(qb, rb, c0);
    qa[s][2] = ld_pair(qb, ra, c0 + 8);
    qa[s][3] = ld_pair(qb, rb, c0 + 8);
  }
  const int row_end = min(q.L, q.row0 + 64);
  const int kend = causal ? row_end : q.L;
  const int wrow0 = q.row0 + warp * 16;
  const int wrow_last = min(wrow0 + 15, q.L - 1);
  for (int kb = 0; kb < kend; kb += 64) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < 64 * (DP / 2); idx += 128) {
      const int r = idx / (DP / 2), cp = (idx % (DP / 2)) * 2;
      *reinterpret_cast<uint32_t*>(&ks[r][cp]) = ld_pair(kbp, kb + r, cp);
    }
    __syncthreads();
    if (wrow0 >= q.L) continue;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int key0 = kb + nt * 8;
      if (key0 >= kend || (causal && key0 > wrow_last)) break;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < DP / 16; ++s) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&ks[nt * 8 + g][s * 16 + 2 * tq]);
        const uint32_t b1 =
            *reinterpret_cast<const uint32_t*>(&ks[nt * 8 + g][s * 16 + 8 + 2 * tq]);
        mma_bf16_16816(acc, qa[s], b0, b1);
      }
      const int c = key0 + 2 * tq;
      // the pair (c, c+1) stays inside the row's Lp (c even, Lp a multiple of 8)
      if (ra < q.L && c < (causal ? ra + 1 : q.L))
        *reinterpret_cast<uint32_t*>(sb + static_cast<size_t>(ra) * q.Lp + c) =
            pack_bf16x2(acc[0] * scale, acc[1] * scale);
      if (rb < q.L && c < (causal ? rb + 1 : q.L))
        *reinterpret_cast<uint32_t*>(sb + static_cast<size_t>(rb) * q.Lp + c) =
            pack_bf16x2(acc[2] * scale, acc[3] * scale);
    }
  }
}

// One lane group's softmax over its U rows (row[u] of valid length len[u];
// len 0 = no row): each lane holds MAXC 8-element chunks of each row in
// registers, all loads issued before the first reduction so that short rows
// still keep enough bytes in flight.  Every lane of the warp calls it (the
// group reductions are warp shuffles).
template <typename T, int G, int MAXC, int U>
__device__ __forceinline__ void softmax_group(T* const (&row)[U], const int (&len)[U], int sub) {
  float v[U][MAXC][8];
#pragma unroll
  for (int u = 0; u < U; ++u)
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int col = (c * G + sub) * 8;
      if (col < len[u]) Chunk8<T>::load(row[u] + col, v[u][c]);
    }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    float m = -INFINITY;
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int col = (c * G + sub) * 8;
      if (col < len[u]) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (col + e >= len[u]) v[u][c][e] = -INFINITY;
          m = fmaxf(m, v[u][c][e]);
        }
      }
    }
    m = group_max<G>(m);
    float sum = 0.f;
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int col = (c * G + sub) * 8;
      if (col < len[u]) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float p = (col + e < len[u]) ? __expf(v[u][c][e] - m) : 0.f;
          v[u][c][e] = p;
          sum += p;
        }
      }
    }
    sum = group_sum<G>(sum);
    const float inv = 1.0f / sum;
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int col = (c * G + sub) * 8;
      if (col < len[u]) {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[u][c][e] *= inv;
        Chunk8<T>::store(row[u] + col, v[u][c]);
      }
    }
  }
}

// Masked softmax.  A group of G lanes owns U consecutive rows; each lane
// holds MAXC 8-element chunks of each of them in registers.  All U*MAXC loads
// of a lane are issued before the first reduction, so short rows still keep
// enough bytes in flight to cover HBM latency.  The group finds the sequence
// of its first row by binary search over the offsets and walks forward from
// there (consecutive rows belong to the same sequence or the next ones).
template <typename T, int G, int MAXC, int U>
__global__ void __launch_bounds__(256)
    softmax_kernel(T* __restrict__ S, const int32_t* __restrict__ offsets,
                   const int64_t* __restrict__ s_off, int n, long long rows, int nh, int causal) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31, sub = lane % G;
  const long long R0 =
      ((static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * (32 / G) + lane / G) * U;
  int len[U];
  T* row[U];
  if (R0 < rows) {
    int lo = 0, hi = n - 1;   // largest i with nh * offsets[i] <= R0
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (static_cast<long long>(nh) * offsets[mid] <= R0) lo = mid; else hi = mid - 1;
    }
    int i = lo;
    long long seq_row0 = static_cast<long long>(nh) * offsets[i];
    long long seq_row1 = static_cast<long long>(nh) * offsets[i + 1];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long R = R0 + u;
      len[u] = 0;
      row[u] = S;
      if (R < rows) {
        while (R >= seq_row1 && in_bounds(i + 1 < n)) {
          ++i;
          seq_row0 = seq_row1;
          seq_row1 = static_cast<long long>(nh) * offsets[i + 1];
        }
        const int L = offsets[i + 1] - offsets[i];
        if (!in_bounds(R < seq_row1 && L >= 1)) continue;   // rows past offsets[n]
        const long long rr = R - seq_row0;
        len[u] = causal ? static_cast<int>(rr % L) + 1 : L;
        row[u] = S + s_off[i] + rr * ((L + 7) & ~7);
      }
    }
  } else {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      len[u] = 0;
      row[u] = S;
    }
  }
  softmax_group<T, G, MAXC, U>(row, len, sub);
}

// softmax_group for bf16 rows, written for instruction count and registers
// (the class kernel below is bound by the latency of its loads, so it keeps
// the next rows' loads in flight while it computes): the row maximum over
// packed bf16 pairs (exact in any precision), the masking of a row's last
// partial chunk at 16-bit granularity (-inf), and the exponent's argument
// and the sum in packed fp32 pairs; exp2 of -inf gives the masked entries
// exactly 0.  A row's exponentials are held (two per 64-bit register) from
// the sum to the output, which is one packed multiply per pair.
template <int G, int MAXC, int U>
__device__ __forceinline__ void softmax_load_bf16(bf16* const (&row)[U], const int (&len)[U], int sub,
                                                  uint32_t (&w)[U][MAXC][4]) {
#pragma unroll
  for (int u = 0; u < U; ++u)
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int col = (c * G + sub) * 8;
      if (col < len[u]) {
        const uint4 q = *reinterpret_cast<const uint4*>(row[u] + col);
        w[u][c][0] = q.x;
        w[u][c][1] = q.y;
        w[u][c][2] = q.z;
        w[u][c][3] = q.w;
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) w[u][c][j] = 0xff80ff80u;   // -inf pairs
      }
    }
}

template <int G, int MAXC, int U>
__device__ __forceinline__ void softmax_compute_bf16(bf16* const (&row)[U], const int (&len)[U],
                                                     int sub, uint32_t (&w)[U][MAXC][4]) {
  constexpr float kLog2e = 1.4426950408889634f;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    // entries past the row inside its last chunk read as -inf
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int nv = len[u] - (c * G + sub) * 8;
      if (nv > 0 && nv < 8) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (2 * j >= nv) w[u][c][j] = 0xff80ff80u;
          else if (2 * j + 1 >= nv) w[u][c][j] = (w[u][c][j] & 0x0000ffffu) | 0xff800000u;
        }
      }
    }
    __nv_bfloat162 mx = *reinterpret_cast<const __nv_bfloat162*>(&w[u][0][0]);
#pragma unroll
    for (int c = 0; c < MAXC; ++c)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        mx = __hmax2(mx, *reinterpret_cast<const __nv_bfloat162*>(&w[u][c][j]));
    float m = fmaxf(__low2float(mx), __high2float(mx));
    m = group_max<G>(m);
    // a row with no entry (len 0) keeps m = -inf: shift by 0 then
    const uint64_t shift = f32x2_splat(m == -INFINITY ? 0.f : -m * kLog2e);
    const uint64_t l2e = f32x2_splat(kLog2e);
    uint64_t acc = 0;                                         // +0.0 in both lanes
    uint64_t e2[MAXC][4];                                     // the exponentials, two per register
#pragma unroll
    for (int c = 0; c < MAXC; ++c)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float x0, x1;
        f32x2_unpack(f32x2_fma(f32x2_pack(bf16_lo(w[u][c][j]), bf16_hi(w[u][c][j])), l2e, shift), x0, x1);
        e2[c][j] = f32x2_pack(ex2_approx_ftz(x0), ex2_approx_ftz(x1));
        acc = f32x2_add(acc, e2[c][j]);
      }
    float a0, a1;
    f32x2_unpack(acc, a0, a1);
    const uint64_t inv2 = f32x2_splat(1.0f / group_sum<G>(a0 + a1));
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int col = (c * G + sub) * 8;
      if (col < len[u]) {
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float y0, y1;
          f32x2_unpack(f32x2_mul(e2[c][j], inv2), y0, y1);
          o[j] = pack_bf16x2(y0, y1);
        }
        *reinterpret_cast<uint4*>(row[u] + col) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Masked softmax by row-length class.  The batch-wide kernel above sizes its
// lane groups for the longest row and finds each group's sequence by a binary
// search over the offsets: with many short rows most lanes idle and the
// search's dependent loads cost more than the rows.  Here the rows are first
// regrouped, on the device, by the class of their length (8-element chunks
// <= 1, 2, 4, 8, 16, 32, 64, 96, 128):
//   softmax_count_kernel: rows per class (n_heads * L_i per sequence);
//   softmax_index_kernel: each sequence reserves a stretch of its class's
//     segment of a class-ordered row space and writes, for every row of the
//     stretch, its sequence (row_seq) and the stretch's start (seq_base);
//   softmax_class_kernel: one persistent pass per class, lane groups sized
//     to the class, each group finding its sequence with one load.
// The order of sequences inside a class (reservation order) does not matter:
// every row is computed on its own, with the same arithmetic whatever its
// position.
// ---------------------------------------------------------------------------
constexpr int kSmClasses = 13;

// 8-element chunks of a row: <= 1, 2, 4, 6, 8, 12, 16, 24, 32, 48, 64, 96, 128
__host__ __device__ constexpr int softmax_class_of(int L) {
  return (L + 7) / 8 <= 1 ? 0 : (L + 7) / 8 <= 2 ? 1 : (L + 7) / 8 <= 4 ? 2 : (L + 7) / 8 <= 6 ? 3
       : (L + 7) / 8 <= 8 ? 4 : (L + 7) / 8 <= 12 ? 5 : (L + 7) / 8 <= 16 ? 6
       : (L + 7) / 8 <= 24 ? 7 : (L + 7) / 8 <= 32 ? 8 : (L + 7) / 8 <= 48 ? 9
       : (L + 7) / 8 <= 64 ? 10 : (L + 7) / 8 <= 96 ? 11 : 12;
}

// Largest chunk count of class k.
__host__ __device__ constexpr int softmax_class_hi(int k) {
  return k == 0 ? 1 : k == 1 ? 2 : k == 2 ? 4 : k == 3 ? 6 : k == 4 ? 8 : k == 5 ? 12 : k == 6 ? 16
       : k == 7 ? 24 : k == 8 ? 32 : k == 9 ? 48 : k == 10 ? 64 : k == 11 ? 96 : 128;
}
// The rows of a sequence of length L that class k takes, per head: every
// row when not causal (when k is L's class); when causal, the rows r whose
// own length r + 1 falls in the class: [r_lo, r_lo + run).
struct ClassRun {
  int r_lo, run;
};
__host__ __device__ inline ClassRun softmax_class_run(int L, int k, int causal) {
  if (!causal) return ClassRun{0, softmax_class_of(L) == k ? L : 0};
  const int lo = k == 0 ? 0 : 8 * softmax_class_hi(k - 1);       // first row of the class
  const int hi = 8 * softmax_class_hi(k) < L ? 8 * softmax_class_hi(k) : L;   // one past its last
  return ClassRun{lo, hi > lo ? hi - lo : 0};
}

// scratch: counters int64[2 * kSmClasses] (rows per class, reservation
// cursors) | seq_base int64[n][kSmClasses] (the start of each sequence's
// stretch in each class) | row_seq int32[n_heads * T]
struct SoftmaxIndexLayout {
  size_t base, rows, bytes;
  SoftmaxIndexLayout(long long n, long long rows_total) {
    base = 16 * kSmClasses;
    rows = base + 8 * static_cast<size_t>(n) * kSmClasses;
    bytes = rows + 4 * static_cast<size_t>(rows_total);
  }
};

__global__ void __launch_bounds__(256)
    softmax_count_kernel(const int32_t* __restrict__ offsets, int n, int nh, int causal,
                         unsigned long long* __restrict__ ctr) {
  __shared__ unsigned long long part[kSmClasses];
  if (threadIdx.x < kSmClasses) part[threadIdx.x] = 0;
  pdl_launch_dependents();
  pdl_wait();
  __syncthreads();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int L = offsets[i + 1] - offsets[i];
    if (!causal) {
      atomicAdd(&part[softmax_class_of(L)], static_cast<unsigned long long>(nh) * L);
    } else {
      for (int k = 0; k <= softmax_class_of(L); ++k) {
        const ClassRun cr = softmax_class_run(L, k, 1);
        if (cr.run > 0) atomicAdd(&part[k], static_cast<unsigned long long>(nh) * cr.run);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x < kSmClasses && part[threadIdx.x] != 0) atomicAdd(&ctr[threadIdx.x], part[threadIdx.x]);
}

__global__ void __launch_bounds__(256)
    softmax_index_kernel(const int32_t* __restrict__ offsets, int n, int nh, int causal,
                         unsigned long long* __restrict__ ctr, long long* __restrict__ seq_base,
                         int32_t* __restrict__ row_seq) {
  __shared__ long long seg[kSmClasses];
  pdl_launch_dependents();
  pdl_wait();
  if (threadIdx.x == 0) {
    long long a = 0;
    for (int k = 0; k < kSmClasses; ++k) {
      seg[k] = a;
      a += static_cast<long long>(ctr[k]);
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  for (int i = blockIdx.x * 8 + (threadIdx.x >> 5); i < n; i += gridDim.x * 8) {
    const int L = offsets[i + 1] - offsets[i];
    // one stretch per class the sequence's rows fall in: its own class, or
    // when causal every class of a row length 1..L
    for (int k = causal ? 0 : softmax_class_of(L); k <= softmax_class_of(L); ++k) {
      const ClassRun cr = softmax_class_run(L, k, causal);
      if (cr.run == 0) continue;
      const long long cnt = static_cast<long long>(nh) * cr.run;
      long long base = 0;
      if (lane == 0)
        base = seg[k] + static_cast<long long>(atomicAdd(&ctr[kSmClasses + k], static_cast<unsigned long long>(cnt)));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (lane == 0) seq_base[static_cast<long long>(i) * kSmClasses + k] = base;
      for (long long r = lane; r < cnt; r += 32) row_seq[base + r] = i;
    }
  }
}

// The sequence a lane's rows belong to: the start of its stretch in the
// class-ordered row space, the stretch's rows per head (run, from row r_lo
// of each head block), its length and score offset.  Kept across
// iterations so that a lane walking consecutive rows looks a sequence up
// only when it crosses into the next one.
struct SeqCache {
  long long b = 0;             // stretch [b, b + rows)
  int rows = 0, L = 0, r_lo = 0, run = 1;
  float inv_run = 1.f;
  long long soff = 0;
};

// Rows [R0, R0 + U) of class k's row space (those below Re): their addresses
// and lengths (length 0 for none).  A stretch row rr is row r_lo + rr % run
// of head rr / run (the quotient from a float reciprocal, corrected: exact
// for rr < 2^24).
template <typename T, int U>
__device__ __forceinline__ void class_rows_at(T* S, const int32_t* __restrict__ offsets,
                                              const int64_t* __restrict__ s_off,
                                              const long long* __restrict__ seq_base,
                                              const int32_t* __restrict__ row_seq, long long R0,
                                              long long Re, int n, int nh, int causal, int k,
                                              SeqCache& sc, T* (&row)[U], int (&len)[U]) {
#pragma unroll
  for (int u = 0; u < U; ++u) {
    len[u] = 0;
    row[u] = S;
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const long long R = R0 + u;
    if (R < Re) {
      if (R < sc.b || R - sc.b >= sc.rows) {                 // another sequence's stretch
        // the index is rewritten by every call's index kernel: read it from L2
        const int i = __ldcg(row_seq + R);
        if (!in_bounds(i >= 0 && i < n)) return;
        sc.b = __ldcg(seq_base + static_cast<long long>(i) * kSmClasses + k);
        sc.L = offsets[i + 1] - offsets[i];
        const ClassRun cr = softmax_class_run(sc.L, k, causal);
        sc.r_lo = cr.r_lo;
        sc.run = cr.run > 0 ? cr.run : 1;
        sc.inv_run = 1.0f / static_cast<float>(sc.run);
        sc.rows = nh * cr.run;
        sc.soff = s_off[i];
      }
      const int rr = static_cast<int>(R - sc.b);             // row inside the stretch
      if (!in_bounds(sc.L >= 1 && rr >= 0 && rr < sc.rows)) return;
      if (!causal) {
        len[u] = sc.L;
        row[u] = S + sc.soff + static_cast<long long>(rr) * ((sc.L + 7) & ~7);
      } else {
        int h = __float2int_rz(static_cast<float>(rr) * sc.inv_run);
        int r = rr - h * sc.run;
        if (r < 0) {
          --h;
          r += sc.run;
        } else if (r >= sc.run) {
          ++h;
          r -= sc.run;
        }
        r += sc.r_lo;
        len[u] = r + 1;
        row[u] = S + sc.soff + static_cast<long long>(h * sc.L + r) * ((sc.L + 7) & ~7);
      }
    }
  }
}

// The bf16 class kernel stages its rows through shared memory with cp.async:
// per warp a ring of kSmStages iterations, each up to kSmChunks 16-byte chunks
// per lane (chunk-major, so a warp's accesses to one chunk are contiguous).
// The loads in flight are then not bounded by registers: about 8 KB per warp.
constexpr int kSmStages = 4;
constexpr int kSmChunks = 4;
constexpr int kSmRingWarpBytes = kSmStages * kSmChunks * 32 * 16;
constexpr int kSmClassThreads = 256;

__device__ __forceinline__ void sm_cp16(uint32_t saddr, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void sm_cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void sm_cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One class: lane groups of G lanes, U consecutive rows (of the class-ordered
// row space) each; a warp-iteration takes 32 / G * U consecutive rows.  The
// warp runs iterations [it, it_end) of the class: consecutive iterations of
// a lane group stay inside one sequence's rows, so its address arithmetic
// needs no lookup (the class-ordered row space keeps a sequence's rows
// together).  The loop bound is uniform across a warp (groups past the end
// get empty rows): the group reductions are warp shuffles.  bf16 rows are
// loaded kSmStages - 1 iterations ahead into the warp's shared-memory ring.
template <int G, int U>
__host__ __device__ constexpr long long class_rows_per_iter() {
  return static_cast<long long>(32 / G) * U;
}
template <typename T, int G, int MAXC, int U>
__device__ __forceinline__ void softmax_class_pass(T* S, const int32_t* __restrict__ offsets,
                                                   const int64_t* __restrict__ s_off,
                                                   const long long* __restrict__ seq_base,
                                                   const int32_t* __restrict__ row_seq,
                                                   long long Rb, long long Re, long long it,
                                                   long long it_end, int n, int nh, int causal,
                                                   int k, uint32_t ring) {
  if (it >= it_end) return;                                  // uniform across the warp
  const int lane = threadIdx.x & 31, sub = lane % G;
  constexpr long long GU = class_rows_per_iter<G, U>();      // rows per warp-iteration
  const long long lane_off = static_cast<long long>(lane / G) * U;
  SeqCache sc;
  int len[U];
  T* row[U];
  if constexpr (std::is_same<T, bf16>::value) {
    constexpr int D = kSmStages;
    static_assert(U * MAXC <= kSmChunks, "a lane's chunks fit its ring slot");
    // this lane's chunk k of stage st
    auto slot = [&](int st, int k) { return ring + static_cast<uint32_t>((st * kSmChunks + k) * 512); };
    SeqCache sci;                                            // the issuing side's sequence
    // With one row per lane group the issuing side's row address and length
    // are kept for the computing side, D iterations deep (a register queue
    // shifted once per iteration); with more rows per group they are
    // recomputed (the queue would cost 3 * D * U registers).
    T* qrow[D];
    int qlen[D];
    auto issue = [&](long long t, int q) {
      int il[U];
      T* ir[U];
      class_rows_at<T, U>(S, offsets, s_off, seq_base, row_seq, Rb + t * GU + lane_off, Re, n, nh,
                          causal, k, sci, ir, il);
      const int st = static_cast<int>(t & (D - 1));
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int c = 0; c < MAXC; ++c) {
          const int col = (c * G + sub) * 8;
          if (col < il[u]) sm_cp16(slot(st, u * MAXC + c), ir[u] + col);
        }
      if (U == 1) {
        qrow[q] = ir[0];
        qlen[q] = il[0];
      }
    };
#pragma unroll
    for (int q = 0; q < D - 1; ++q) {
      qrow[q] = S;
      qlen[q] = 0;
      if (it + q < it_end) issue(it + q, q);
      sm_cp_commit();
    }
    for (; it < it_end; ++it) {
      qrow[D - 1] = S;
      qlen[D - 1] = 0;
      if (it + D - 1 < it_end) issue(it + D - 1, D - 1);
      sm_cp_commit();
      sm_cp_wait<D - 1>();                                   // iteration it has landed
      if (U == 1) {
        row[0] = qrow[0];
        len[0] = qlen[0];
#pragma unroll
        for (int q = 0; q < D - 1; ++q) {
          qrow[q] = qrow[q + 1];
          qlen[q] = qlen[q + 1];
        }
      } else {
        class_rows_at<T, U>(S, offsets, s_off, seq_base, row_seq, Rb + it * GU + lane_off, Re, n,
                            nh, causal, k, sc, row, len);
      }
      const int st = static_cast<int>(it & (D - 1));
      uint32_t w4[U][MAXC][4];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int c = 0; c < MAXC; ++c) {
          const int col = (c * G + sub) * 8;
          if (col < len[u]) {
            uint32_t q0, q1, q2, q3;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(q0), "=r"(q1), "=r"(q2), "=r"(q3)
                         : "r"(slot(st, u * MAXC + c)));
            w4[u][c][0] = q0;
            w4[u][c][1] = q1;
            w4[u][c][2] = q2;
            w4[u][c][3] = q3;
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) w4[u][c][j] = 0xff80ff80u;   // -inf pairs
          }
        }
      softmax_compute_bf16<G, MAXC, U>(row, len, sub, w4);
    }
    sm_cp_wait<0>();
  } else {
    class_rows_at<T, U>(S, offsets, s_off, seq_base, row_seq, Rb + it * GU + lane_off, Re, n, nh,
                        causal, k, sc, row, len);
    for (;;) {
      softmax_group<T, G, MAXC, U>(row, len, sub);
      if (++it >= it_end) break;
      class_rows_at<T, U>(S, offsets, s_off, seq_base, row_seq, Rb + it * GU + lane_off, Re, n, nh,
                          causal, k, sc, row, len);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kSmClassThreads, 3)
    softmax_class_kernel(T* __restrict__ S, const int32_t* __restrict__ offsets,
                         const int64_t* __restrict__ s_off, const unsigned long long* __restrict__ ctr,
                         const long long* __restrict__ seq_base, const int32_t* __restrict__ row_seq,
                         int k_max, int n, int nh, int causal) {
  extern __shared__ __align__(16) uint8_t sm_ring_raw[];
  // this warp's ring (bf16 rows), offset by the lane's 16 bytes
  const uint32_t ring = smem_u32(sm_ring_raw) + (threadIdx.x >> 5) * kSmRingWarpBytes + (threadIdx.x & 31) * 16;
  pdl_launch_dependents();
  pdl_wait();
  long long seg[kSmClasses + 1];
  seg[0] = 0;
#pragma unroll
  for (int k = 0; k < kSmClasses; ++k) seg[k + 1] = seg[k] + static_cast<long long>(ctr[k]);
  // lanes per row G and chunks per lane MAXC with G * MAXC covering the
  // class's chunks and MAXC three or four: a lane holds up to four chunks of
  // one row, so the per-row work (addresses, masks, reductions) is spread
  // over up to 32 entries; rows of one or two chunks take four or two rows
  // per lane.  Each class's warp-iterations are split evenly over all warps,
  // one contiguous share each (laying the classes end to end and cutting
  // that sequence into equal shares measured slower on B200: 2..100 scores
  // 67% -> 28% of HBM, causal 50% -> 24%).
  constexpr long long kRpi[kSmClasses] = {
      class_rows_per_iter<1, 4>(),  class_rows_per_iter<1, 2>(),  class_rows_per_iter<1, 1>(),
      class_rows_per_iter<2, 1>(),  class_rows_per_iter<2, 1>(),  class_rows_per_iter<4, 1>(),
      class_rows_per_iter<4, 1>(),  class_rows_per_iter<8, 1>(),  class_rows_per_iter<8, 1>(),
      class_rows_per_iter<16, 1>(), class_rows_per_iter<16, 1>(), class_rows_per_iter<32, 1>(),
      class_rows_per_iter<32, 1>()};
  long long ibase[kSmClasses + 1];
  ibase[0] = 0;
#pragma unroll
  for (int k = 0; k < kSmClasses; ++k)
    ibase[k + 1] = ibase[k] + (k <= k_max ? (seg[k + 1] - seg[k] + kRpi[k] - 1) / kRpi[k] : 0);
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long w = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
#define RM_SM_PASS(k, G, MAXC, U)                                                                \
  if (k_max >= k) {                                                                             \
    const long long nit = ibase[k + 1] - ibase[k];                                              \
    const long long pk = (nit + warps - 1) / warps;                                             \
    softmax_class_pass<T, G, MAXC, U>(S, offsets, s_off, seq_base, row_seq, seg[k], seg[k + 1],  \
                                      w * pk < nit ? w * pk : nit, (w + 1) * pk < nit ? (w + 1) * pk : nit, \
                                      n, nh, causal, k, ring);                                  \
  }
  RM_SM_PASS(0, 1, 1, 4);
  RM_SM_PASS(1, 1, 2, 2);
  RM_SM_PASS(2, 1, 4, 1);
  RM_SM_PASS(3, 2, 3, 1);
  RM_SM_PASS(4, 2, 4, 1);
  RM_SM_PASS(5, 4, 3, 1);
  RM_SM_PASS(6, 4, 4, 1);
  RM_SM_PASS(7, 8, 3, 1);
  RM_SM_PASS(8, 8, 4, 1);
  RM_SM_PASS(9, 16, 3, 1);
  RM_SM_PASS(10, 16, 4, 1);
  RM_SM_PASS(11, 32, 3, 1);
  RM_SM_PASS(12, 32, 4, 1);
#undef RM_SM_PASS
}

template <int DP>
__global__ void __launch_bounds__(128)
    attn_context_kernel(const bf16* __restrict__ S, const bf16* __restrict__ qkv,
                        bf16* __restrict__ ctx, const int32_t* __restrict__ offsets,
                        const int32_t* __restrict__ rb_off, const int64_t* __restrict__ s_off,
                        int n, int H, int d, int causal) {
  __shared__ __align__(16) bf16 vt[DP][64 + 8];   // V block transposed: [dim][key]
  pdl_launch_dependents();
  pdl_wait();
  const BlockSeq q = locate_block(offsets, rb_off, s_off, n, blockIdx.x);
  if (!in_bounds(q.L >= 1 && q.row0 < q.L)) return;   // checked build: inconsistent row blocks
  const int hd = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const size_t H3 = 3 * static_cast<size_t>(H);
  const bf16* vb = qkv + static_cast<size_t>(q.t0) * H3 + 2 * H + hd * d;
  const bf16* pb = S + q.sbase + static_cast<size_t>(hd) * q.L * q.Lp;
  const int ra = q.row0 + warp * 16 + g, rb = ra + 8;
  const int lim_a = causal ? ra + 1 : q.L, lim_b = causal ? rb + 1 : q.L;

  auto ld_p = [&](int r, int lim, int c) -> uint32_t {
    if (r >= q.L || c >= lim) return 0u;
    uint32_t v = *reinterpret_cast<const uint32_t*>(pb + static_cast<size_t>(r) * q.Lp + c);
    return (c + 1 < lim) ? v : (v & 0xffffu);
  };
  float acc[DP / 8][4];
#pragma unroll
  for (int t = 0; t < DP / 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

  const int row_end = min(q.L, q.row0 + 64);
  const int kend = causal ? row_end : q.L;
  const int wrow0 = q.row0 + warp * 16;
  const int wrow_last = min(wrow0 + 15, q.L - 1);
  for (int kb = 0; kb < kend; kb += 64) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < 64 * (DP / 2); idx += 128) {
      const int r = idx & 63, cp = (idx >> 6) * 2;
      uint32_t v = 0u;
      if (kb + r < q.L && cp < d) v = *reinterpret_cast<const uint32_t*>(vb + (kb + r) * H3 + cp);
      *reinterpret_cast<uint16_t*>(&vt[cp][r]) = static_cast<uint16_t>(v & 0xffffu);
      *reinterpret_cast<uint16_t*>(&vt[cp + 1][r]) = static_cast<uint16_t>(v >> 16);
    }
    __syncthreads();
    if (wrow0 >= q.L) continue;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int key0 = kb + s * 16;
      if (key0 >= kend || (causal && key0 > wrow_last)) break;
      uint32_t a[4];
      a[0] = ld_p(ra, lim_a, key0 + 2 * tq);
      a[1] = ld_p(rb, lim_b, key0 + 2 * tq);
      a[2] = ld_p(ra, lim_a, key0 + 8 + 2 * tq);
      a[3] = ld_p(rb, lim_b, key0 + 8 + 2 * tq);
#pragma unroll
      for (int t = 0; t < DP / 8; ++t) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&vt[t * 8 + g][s * 16 + 2 * tq]);
        const uint32_t b1 =
            *reinterpret_cast<const uint32_t*>(&vt[t * 8 + g][s * 16 + 8 + 2 * tq]);
        mma_bf16_16816(acc[t], a, b0, b1);
      }
    }
  }
  if (wrow0 >= q.L) return;
  bf16* cb = ctx + static_cast<size_t>(q.t0) * H + hd * d;
#pragma unroll
  for (int t = 0; t < DP / 8; ++t) {
    const int col = t * 8 + 2 * tq;
    if (col < d) {
      if (ra < q.L)
        *reinterpret_cast<uint32_t*>(cb + static_cast<size_t>(ra) * H + col) =
            pack_bf16x2(acc[t][0], acc[t][1]);
      if (rb < q.L)
        *reinterpret_cast<uint32_t*>(cb + static_cast<size_t>(rb) * H + col) =
            pack_bf16x2(acc[t][2], acc[t][3]);
    }
  }
}

// ---------------------------------------------------------------------------
// Fused attention: scores, masked online softmax and P.V in one pass, the
// probabilities never leave registers.  Same work decomposition as above: a
// CTA per (sequence, 64-query block, head), 4 warps x 16 query rows, keys in
// blocks of 64 staged in shared memory.  The running row maximum m and sum l
// are rescaled per key block (the online softmax); P is rounded to bf16 for
// the P.V tile exactly as the materialised path stores it.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

template <int DP>
__global__ void __launch_bounds__(128)
    attn_fused_kernel(const bf16* __restrict__ qkv, bf16* __restrict__ ctx,
                      const int32_t* __restrict__ offsets, const int32_t* __restrict__ rb_off,
                      int n, int H, int d, float scale_log2, int causal) {
  __shared__ __align__(16) bf16 ks[64][DP + 8];
  __shared__ __align__(16) bf16 vs[64][DP + 8];
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.x, hd = blockIdx.y;
  const int i = upper_index(rb_off, n, b);
  const int t0 = offsets[i];
  const int L = offsets[i + 1] - t0;
  const int row0 = (b - rb_off[i]) * 64;
  if (!in_bounds(L >= 1 && row0 < L)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const size_t H3 = 3 * static_cast<size_t>(H);
  const bf16* qb = qkv + static_cast<size_t>(t0) * H3 + hd * d;
  const bf16* kb_ = qkv + static_cast<size_t>(t0) * H3 + H + hd * d;
  const bf16* vb = qkv + static_cast<size_t>(t0) * H3 + 2 * H + hd * d;
  const int ra = row0 + warp * 16 + g, rb = ra + 8;

  auto ld_pair = [&](const bf16* base, int r, int c) -> uint32_t {
    return (r < L && c < d) ? *reinterpret_cast<const uint32_t*>(base + r * H3 + c) : 0u;
  };
  uint32_t qa[DP / 16][4];
#pragma unroll
  for (int s = 0; s < DP / 16; ++s) {
    const int c0 = s * 16 + 2 * tq;
    qa[s][0] = ld_pair(qb, ra, c0);
    qa[s][1] = ld_pair(qb, rb, c0);
    qa[s][2] = ld_pair(qb, ra, c0 + 8);
    qa[s][3] = ld_pair(qb, rb, c0 + 8);
  }
  float o[DP / 8][4];
#pragma unroll
  for (int t = 0; t < DP / 8; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  const int row_end = min(L, row0 + 64);
  const int kend = causal ? row_end : L;
  const int wrow0 = row0 + warp * 16;
  const int wrow_last = min(wrow0 + 15, L - 1);
  const uint32_t vs_base = static_cast<uint32_t>(__cvta_generic_to_shared(&vs[0][0]));
  for (int kb = 0; kb < kend; kb += 64) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < 64 * (DP / 2); idx += 128) {
      const int r = idx / (DP / 2), cp = (idx % (DP / 2)) * 2;
      *reinterpret_cast<uint32_t*>(&ks[r][cp]) = ld_pair(kb_, kb + r, cp);
      *reinterpret_cast<uint32_t*>(&vs[r][cp]) = ld_pair(vb, kb + r, cp);
    }
    __syncthreads();
    if (wrow0 >= L || (causal && kb > wrow_last)) continue;
    // S = Q K^T for this warp's 16 rows and 64 keys (8 tiles of 8 keys)
    float sc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int s = 0; s < DP / 16; ++s) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&ks[nt * 8 + g][s * 16 + 2 * tq]);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(&ks[nt * 8 + g][s * 16 + 8 + 2 * tq]);
        mma_bf16_16816(sc[nt], qa[s], b0, b1);
      }
    }
    // mask, scale (log2 domain), row maxima over this block
    const int lim_a = causal ? min(ra + 1, L) : L, lim_b = causal ? min(rb + 1, L) : L;
    float bm_a = -INFINITY, bm_b = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const int c = kb + nt * 8 + 2 * tq;
      sc[nt][0] = (c < lim_a) ? sc[nt][0] * scale_log2 : -INFINITY;
      sc[nt][1] = (c + 1 < lim_a) ? sc[nt][1] * scale_log2 : -INFINITY;
      sc[nt][2] = (c < lim_b) ? sc[nt][2] * scale_log2 : -INFINITY;
      sc[nt][3] = (c + 1 < lim_b) ? sc[nt][3] * scale_log2 : -INFINITY;
      bm_a = fmaxf(bm_a, fmaxf(sc[nt][0], sc[nt][1]));
      bm_b = fmaxf(bm_b, fmaxf(sc[nt][2], sc[nt][3]));
    }
    bm_a = fmaxf(bm_a, __shfl_xor_sync(0xffffffffu, bm_a, 1));
    bm_a = fmaxf(bm_a, __shfl_xor_sync(0xffffffffu, bm_a, 2));
    bm_b = fmaxf(bm_b, __shfl_xor_sync(0xffffffffu, bm_b, 1));
    bm_b = fmaxf(bm_b, __shfl_xor_sync(0xffffffffu, bm_b, 2));
    const float mn_a = fmaxf(m_a, bm_a), mn_b = fmaxf(m_b, bm_b);
    // rows whose keys are all masked so far keep m = -inf; use 0 as the shift then
    const float sh_a = mn_a == -INFINITY ? 0.f : mn_a, sh_b = mn_b == -INFINITY ? 0.f : mn_b;
    const float al_a = ex2_approx_ftz(m_a - sh_a), al_b = ex2_approx_ftz(m_b - sh_b);
    m_a = mn_a;
    m_b = mn_b;
    float ps_a = 0.f, ps_b = 0.f;
    uint32_t pa[4][4];   // P as the A operand of four k=16 steps
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = ex2_approx_ftz(sc[nt][0] - sh_a), p1 = ex2_approx_ftz(sc[nt][1] - sh_a);
      const float p2 = ex2_approx_ftz(sc[nt][2] - sh_b), p3 = ex2_approx_ftz(sc[nt][3] - sh_b);
      ps_a += p0 + p1;
      ps_b += p2 + p3;
      pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16x2(p0, p1);
      pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16x2(p2, p3);
    }
    l_a = l_a * al_a + ps_a;
    l_b = l_b * al_b + ps_b;
#pragma unroll
    for (int t = 0; t < DP / 8; ++t) {
      o[t][0] *= al_a;
      o[t][1] *= al_a;
      o[t][2] *= al_b;
      o[t][3] *= al_b;
    }
    // O += P V: B operand (keys x dims) from row-major V via ldmatrix.trans;
    // one x4 load gives the fragments of two 8-dim tiles for 16 keys
#pragma unroll
    for (int s = 0; s < 4; ++s) {
#pragma unroll
      for (int t = 0; t < DP / 8; t += 2) {
        uint32_t bv[4];
        const int key = s * 16 + (lane & 15);
        const int dim = t * 8 + (lane >> 4) * 8;
        ldmatrix_x4_trans(bv, vs_base + static_cast<uint32_t>((key * (DP + 8) + dim) * 2));
        mma_bf16_16816(o[t], pa[s], bv[0], bv[1]);
        mma_bf16_16816(o[t + 1], pa[s], bv[2], bv[3]);
      }
    }
  }
  if (wrow0 >= L) return;
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  const float inv_a = 1.0f / l_a, inv_b = 1.0f / l_b;
  bf16* cb = ctx + static_cast<size_t>(t0) * H + hd * d;
#pragma unroll
  for (int t = 0; t < DP / 8; ++t) {
    const int col = t * 8 + 2 * tq;
    if (col < d) {
      if (ra < L)
        *reinterpret_cast<uint32_t*>(cb + static_cast<size_t>(ra) * H + col) =
            pack_bf16x2(o[t][0] * inv_a, o[t][1] * inv_a);
      if (rb < L)
        *reinterpret_cast<uint32_t*>(cb + static_cast<size_t>(rb) * H + col) =
            pack_bf16x2(o[t][2] * inv_b, o[t][3] * inv_b);
    }
  }
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// 16-byte asynchronous copy global -> shared; src_size 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* gptr, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr), "l"(gptr),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// The same fused attention for head dims that are a multiple of 8: Q, K and V
// tiles arrive by 16-byte cp.async (zero-filled outside the sequence), Q, K0
// and V0 all in flight at once, and K/V are double-buffered so the next key
// block loads while the current one is multiplied.  Q fragments come from
// shared memory through ldmatrix.
template <int DP>
struct FusedSmem {
  static constexpr int kPitch = DP + 8;          // elements; 16-byte aligned rows
  static constexpr int kTile = 64 * kPitch;      // elements per 64-row tile
  static constexpr int kBytes = 5 * kTile * 2;   // Q, K x2, V x2
};

//
// With PFX, segment i continues a shared prefix: its keys are the pre_len[i]
// rows that start at packed row pre_start[i] (all visible), followed by its
// own rows (causal), so query row r sees virtual keys 0 .. pre_len[i] + r.
// Head dims up to 64 are held to 128 registers so that four CTAs share an SM
// (137 registers allowed only three; 16 bytes of spill cost less than the
// occupancy bought: 45.7 -> 42.0 us per BERT-base launch of 13k tokens).
template <int DP, bool PFX>
__global__ void __launch_bounds__(128, (DP <= 64 ? 4 : 1))
    attn_fused_async_kernel(const bf16* __restrict__ qkv, bf16* __restrict__ ctx,
                            const int32_t* __restrict__ offsets, const int32_t* __restrict__ rb_off,
                            int n, int H, int d, float scale_log2, int causal, L2PrefetchArgs pf,
                            const int32_t* __restrict__ pre_start,
                            const int32_t* __restrict__ pre_len) {
  using FS = FusedSmem<DP>;
  constexpr int P = FS::kPitch;
  extern __shared__ __align__(16) uint8_t fsm_raw[];
  bf16* qs = reinterpret_cast<bf16*>(fsm_raw);
  bf16* kbuf = qs + FS::kTile;
  bf16* vbuf = kbuf + 2 * FS::kTile;
  pdl_launch_dependents();
  l2_prefetch_share(pf);
  pdl_wait();
  const int b = blockIdx.x, hd = blockIdx.y;
  const int i = upper_index(rb_off, n, b);
  const int t0 = offsets[i];
  const int L = offsets[i + 1] - t0;
  const int P0 = PFX ? pre_len[i] : 0;                 // shared-prefix keys before the own rows
  const int ps = PFX ? pre_start[i] : 0;
  const int Lk = P0 + L;                               // keys of the segment
  const int row0 = (b - rb_off[i]) * 64;
  if (!in_bounds(L >= 1 && row0 < L && P0 >= 0)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const size_t H3 = 3 * static_cast<size_t>(H);
  const bf16* qb = qkv + static_cast<size_t>(t0) * H3 + hd * d;
  const bf16* colb = qkv + hd * d;                     // head column base of row 0
  const int ra = row0 + warp * 16 + g, rb = ra + 8;
  const int row_end = min(L, row0 + 64);
  const int kend = causal ? P0 + row_end : Lk;
  const int nkb = (kend + 63) / 64;
  const int wrow0 = row0 + warp * 16;
  const int wrow_last = min(wrow0 + 15, L - 1);

  auto issue = [&](bf16* dst, const bf16* src, int rbase) {
#pragma unroll
    for (int k = 0; k < (64 * (DP / 8)) / 128; ++k) {
      const int idx = threadIdx.x + k * 128;
      const int r = idx / (DP / 8), c = (idx % (DP / 8)) * 8;
      const bool ok = (rbase + r < L) && (c < d);
      const bf16* gsrc = ok ? src + static_cast<size_t>(rbase + r) * H3 + c : src;
      cp_async16(static_cast<uint32_t>(__cvta_generic_to_shared(dst + r * P + c)), gsrc, ok);
    }
  };
  // key/value rows kbase.. of the segment's key sequence (prefix rows first)
  auto issue_kv = [&](bf16* dst, int coff, int kbase) {
#pragma unroll
    for (int k = 0; k < (64 * (DP / 8)) / 128; ++k) {
      const int idx = threadIdx.x + k * 128;
      const int r = idx / (DP / 8), c = (idx % (DP / 8)) * 8;
      const int vr = kbase + r;
      const bool ok = (vr < Lk) && (c < d);
      const int grow = vr < P0 ? ps + vr : t0 + vr - P0;
      const bf16* gsrc = ok ? colb + static_cast<size_t>(grow) * H3 + coff + c : colb;
      cp_async16(static_cast<uint32_t>(__cvta_generic_to_shared(dst + r * P + c)), gsrc, ok);
    }
  };
  issue(qs, qb, row0);
  issue_kv(kbuf, H, 0);
  issue_kv(vbuf, 2 * H, 0);
  cp_async_commit();                                   // group 0: Q, K0, V0
  if (nkb > 1) {
    issue_kv(kbuf + FS::kTile, H, 64);
    issue_kv(vbuf + FS::kTile, 2 * H, 64);
  }
  cp_async_commit();                                   // group 1: K1, V1 (may be empty)
  cp_async_wait_1();
  __syncthreads();

  uint32_t qa[DP / 16][4];
  {
    const uint32_t qs_base = static_cast<uint32_t>(__cvta_generic_to_shared(qs));
#pragma unroll
    for (int s = 0; s < DP / 16; ++s) {
      const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int c = s * 16 + (lane >> 4) * 8;
      ldmatrix_x4(qa[s], qs_base + static_cast<uint32_t>((r * P + c) * 2));
    }
  }
  float o[DP / 8][4];
#pragma unroll
  for (int t = 0; t < DP / 8; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

  for (int j = 0; j < nkb; ++j) {
    const int kb = j * 64;
    const int buf = j & 1;
    if (j > 0) {
      cp_async_wait_1();                               // group j (K_j, V_j) has landed
      __syncthreads();
    }
    const bf16* ks = kbuf + buf * FS::kTile;
    const uint32_t vs_base = static_cast<uint32_t>(__cvta_generic_to_shared(vbuf + buf * FS::kTile));
    if (!(wrow0 >= L || (causal && kb > P0 + wrow_last))) {
      float sc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int s = 0; s < DP / 16; ++s) {
          const uint32_t b0 = *reinterpret_cast<const uint32_t*>(ks + (nt * 8 + g) * P + s * 16 + 2 * tq);
          const uint32_t b1 = *reinterpret_cast<const uint32_t*>(ks + (nt * 8 + g) * P + s * 16 + 8 + 2 * tq);
          mma_bf16_16816(sc[nt], qa[s], b0, b1);
        }
      }
      const int lim_a = causal ? min(P0 + ra + 1, Lk) : Lk, lim_b = causal ? min(P0 + rb + 1, Lk) : Lk;
      float bm_a = -INFINITY, bm_b = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int c = kb + nt * 8 + 2 * tq;
        sc[nt][0] = (c < lim_a) ? sc[nt][0] * scale_log2 : -INFINITY;
        sc[nt][1] = (c + 1 < lim_a) ? sc[nt][1] * scale_log2 : -INFINITY;
        sc[nt][2] = (c < lim_b) ? sc[nt][2] * scale_log2 : -INFINITY;
        sc[nt][3] = (c + 1 < lim_b) ? sc[nt][3] * scale_log2 : -INFINITY;
        bm_a = fmaxf(bm_a, fmaxf(sc[nt][0], sc[nt][1]));
        bm_b = fmaxf(bm_b, fmaxf(sc[nt][2], sc[nt][3]));
      }
      bm_a = fmaxf(bm_a, __shfl_xor_sync(0xffffffffu, bm_a, 1));
      bm_a = fmaxf(bm_a, __shfl_xor_sync(0xffffffffu, bm_a, 2));
      bm_b = fmaxf(bm_b, __shfl_xor_sync(0xffffffffu, bm_b, 1));
      bm_b = fmaxf(bm_b, __shfl_xor_sync(0xffffffffu, bm_b, 2));
      const float mn_a = fmaxf(m_a, bm_a), mn_b = fmaxf(m_b, bm_b);
      const float sh_a = mn_a == -INFINITY ? 0.f : mn_a, sh_b = mn_b == -INFINITY ? 0.f : mn_b;
      const float al_a = ex2_approx_ftz(m_a - sh_a), al_b = ex2_approx_ftz(m_b - sh_b);
      m_a = mn_a;
      m_b = mn_b;
      float ps_a = 0.f, ps_b = 0.f;
      uint32_t pa[4][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = ex2_approx_ftz(sc[nt][0] - sh_a), p1 = ex2_approx_ftz(sc[nt][1] - sh_a);
        const float p2 = ex2_approx_ftz(sc[nt][2] - sh_b), p3 = ex2_approx_ftz(sc[nt][3] - sh_b);
        ps_a += p0 + p1;
        ps_b += p2 + p3;
        pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16x2(p0, p1);
        pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16x2(p2, p3);
      }
      l_a = l_a * al_a + ps_a;
      l_b = l_b * al_b + ps_b;
#pragma unroll
      for (int t = 0; t < DP / 8; ++t) {
        o[t][0] *= al_a;
        o[t][1] *= al_a;
        o[t][2] *= al_b;
        o[t][3] *= al_b;
      }
#pragma unroll
      for (int s = 0; s < 4; ++s) {
#pragma unroll
        for (int t = 0; t < DP / 8; t += 2) {
          uint32_t bv[4];
          const int key = s * 16 + (lane & 15);
          const int dim = t * 8 + (lane >> 4) * 8;
          ldmatrix_x4_trans(bv, vs_base + static_cast<uint32_t>((key * P + dim) * 2));
          mma_bf16_16816(o[t], pa[s], bv[0], bv[1]);
          mma_bf16_16816(o[t + 1], pa[s], bv[2], bv[3]);
        }
      }
    }
    __syncthreads();                                   // every warp is done with buffer buf
    if (j + 2 < nkb) {
      issue_kv(kbuf + buf * FS::kTile, H, kb + 128);
      issue_kv(vbuf + buf * FS::kTile, 2 * H, kb + 128);
    }
    cp_async_commit();                                 // group j+2 (may be empty)
  }
  if (wrow0 >= L) return;
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
  l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
  l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
  const float inv_a = 1.0f / l_a, inv_b = 1.0f / l_b;
  bf16* cb = ctx + static_cast<size_t>(t0) * H + hd * d;
#pragma unroll
  for (int t = 0; t < DP / 8; ++t) {
    const int col = t * 8 + 2 * tq;
    if (col < d) {
      if (ra < L)
        *reinterpret_cast<uint32_t*>(cb + static_cast<size_t>(ra) * H + col) =
            pack_bf16x2(o[t][0] * inv_a, o[t][1] * inv_a);
      if (rb < L)
        *reinterpret_cast<uint32_t*>(cb + static_cast<size_t>(rb) * H + col) =
            pack_bf16x2(o[t][2] * inv_b, o[t][3] * inv_b);
    }
  }
}

// ---------------------------------------------------------------------------
// Packed-row attention (head dims 64 and 128).  The batch is cut into tiles of
// 64 consecutive packed rows, whatever sequences they belong to: short
// sequences share a tile, long ones span several, and no warp holds only
// padding (the one-CTA-per-sequence-block layout above leaves most warps of a
// short sequence's block idle).  A CTA takes one tile and a group of heads:
//   warp 4, one lane : TMA producer -- per head the tile's 64 query rows,
//                      then the K and V rows of the tile's key range
//                      [first key of its first sequence, last key of its last
//                      sequence) in chunks of 64 rows, into a ring of stages
//                      that runs on across the heads (128-byte swizzle; rows
//                      past the batch read as zeros);
//   warps 0..3       : 16 query rows each; per chunk S = QK^T (mma.sync
//                      m16n8k16, fragments by ldmatrix), a key admitted only
//                      inside the row's own sequence (and c <= r when causal),
//                      online softmax (running max and sum in fp32; P rounded
//                      to bf16 for P.V as the materialised path stores it),
//                      O += P V; chunks outside the warp's own key range are
//                      skipped.  The heads pipeline: head j+1's rows are in
//                      flight while head j is multiplied.
// A consumer releases a buffer only after a proxy fence: its ldmatrix reads
// are generic-proxy accesses and the TMA refill an async-proxy write (without
// the fence a refill could overtake the reads; seen as an occasional wrong
// (tile, head) block when the ring ran several heads ahead).
// Every mbarrier wait is bounded; a wait that gives up counts into
// err[ERR_TIMEOUT], the role stops, and the producer waits (bounded) for its
// copies before the CTA exits.
// ---------------------------------------------------------------------------
template <int DP>
struct TileSmem {
  static constexpr int kBox = 64 * 64 * 2;                  // TMA box: 64 rows x 128 bytes
  static constexpr int kNB = DP / 64;                       // boxes across a row of DP
  static constexpr int kQ = kNB * kBox;                     // 64 query rows
  static constexpr int kKV = 2 * kNB * kBox;                // 64 key rows of K and of V
  static constexpr int kStages = DP == 64 ? 3 : 2;
  static constexpr int kKVOff = 2 * kQ;                     // after two query buffers
  static constexpr int kBarOff = kKVOff + kStages * kKV;
  static constexpr int kBars = 4 + 2 * kStages;             // qfull[2] qempty[2] kvfull[S] kvempty[S]
  static constexpr int kSeqOff = kBarOff + kBars * 8;       // the tile's offsets window
  static constexpr int kMaxSeqs = 66;                       // 64 rows: at most 64 sequences + 2
  static constexpr int kBytes = kSeqOff + kMaxSeqs * 4 + 1024;   // + 1024-byte alignment slack
  static constexpr int kCtasPerSm = DP == 64 ? 3 : 2;
};

// Byte offset of the 16-byte chunk `ch` (8 bf16 along the row) of row `r` in
// a tile of 128-byte-swizzled boxes.
__device__ __forceinline__ uint32_t sw128_off(int r, int ch) {
  return static_cast<uint32_t>((ch >> 3) * (64 * 128) + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

template <int DP>
__global__ void __launch_bounds__(160)
    attn_tile_kernel(const __grid_constant__ CUtensorMap tm, bf16* __restrict__ ctx,
                     const int32_t* __restrict__ offsets, int n, int T, int H, int nh, int hpc,
                     float scale_log2, int causal, int* __restrict__ err, L2PrefetchArgs pf) {
  using SL = TileSmem<DP>;
  constexpr int S = SL::kStages;
  extern __shared__ uint8_t tsm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tsm_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(sm);
  const uint32_t qfull0 = smem_u32(sm + SL::kBarOff), qempty0 = qfull0 + 16, kvfull0 = qfull0 + 32,
                 kvempty0 = kvfull0 + 8 * S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(qfull0 + 8 * b, 1);
      mbar_init(qempty0 + 8 * b, 4);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(kvfull0 + 8 * s, 1);
      mbar_init(kvempty0 + 8 * s, 4);
    }
    mbar_init_fence();
  }
  __syncthreads();
  pdl_launch_dependents();
  l2_prefetch_share(pf);
  pdl_wait();

  const int r0 = blockIdx.x * 64;
  const int h0 = blockIdx.y * hpc;
  const int nhl = min(hpc, nh - h0);
  const int rlast = min(r0 + 64, T) - 1;
  // the tile's first and last sequence: one search each, shared
  __shared__ int s_edge[2];
  if (threadIdx.x == 0) s_edge[0] = upper_index(offsets, n, r0);
  if (threadIdx.x == 32) s_edge[1] = upper_index(offsets, n, rlast);
  __syncthreads();
  const int s_first = s_edge[0], s_last = s_edge[1];
  const int Klo = offsets[s_first];
  const int Khi = causal ? rlast + 1 : offsets[s_last + 1];
  const int nch = (Khi - Klo + 63) / 64;
  // checked build: the tile's sequences must fit the offsets window, and its
  // key range must hold its rows (the same test in every thread of the CTA)
  if (!in_bounds(s_last - s_first + 2 <= SL::kMaxSeqs && Klo >= 0 && Klo <= r0 && Khi > rlast &&
                 Khi <= T))
    return;

  if (warp == 4) {
    // ---- TMA producer ----
    if (lane == 0) {
      int it = 0, nq = 0;
      bool ok = true;
      for (int j = 0; j < nhl && ok; ++j) {
        const int h = h0 + j, qb = j & 1;
        if (j >= 2 && !mbar_wait(qempty0 + 8 * qb, ((j >> 1) - 1) & 1)) {
          atomicAdd(err + ERR_TIMEOUT, 1);
          break;
        }
        mbar_arrive_expect_tx(qfull0 + 8 * qb, SL::kQ);
#pragma unroll
        for (int b = 0; b < SL::kNB; ++b)
          tma_load_2d(sbase + qb * SL::kQ + b * SL::kBox, &tm, h * DP + 64 * b, r0, qfull0 + 8 * qb);
        ++nq;
        for (int c = 0; c < nch; ++c, ++it) {
          const int s = it % S;
          if (it >= S && !mbar_wait(kvempty0 + 8 * s, ((it / S) - 1) & 1)) {
            atomicAdd(err + ERR_TIMEOUT, 1);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(kvfull0 + 8 * s, SL::kKV);
          const uint32_t dk = sbase + SL::kKVOff + s * SL::kKV, dv = dk + SL::kNB * SL::kBox;
#pragma unroll
          for (int b = 0; b < SL::kNB; ++b) {
            tma_load_2d(dk + b * SL::kBox, &tm, H + h * DP + 64 * b, Klo + 64 * c, kvfull0 + 8 * s);
            tma_load_2d(dv + b * SL::kBox, &tm, 2 * H + h * DP + 64 * b, Klo + 64 * c, kvfull0 + 8 * s);
          }
        }
      }
      // no copy into this CTA's shared memory may be in flight when it exits
      bool drained = true;
      for (int j = it - 1; drained && j >= 0 && j >= it - S; --j)
        drained = mbar_wait(kvfull0 + 8 * (j % S), (j / S) & 1);
      for (int j = nq - 1; drained && j >= 0 && j >= nq - 2; --j)
        drained = mbar_wait(qfull0 + 8 * (j & 1), (j >> 1) & 1);
    }
    return;
  }

  // ---- consumers: 16 query rows per warp ----
  // the offsets of the tile's sequences (s_first .. s_last + 1) go to shared
  // memory once, so that each row finds its sequence there
  int32_t* soff = reinterpret_cast<int32_t*>(sm + SL::kSeqOff);
  const int nseq = s_last - s_first + 2;
  if (threadIdx.x < nseq) soff[threadIdx.x] = offsets[s_first + threadIdx.x];
  asm volatile("bar.sync 1, 128;" ::: "memory");              // the four consumer warps
  const int g = lane >> 2, tq = lane & 3;
  const int ra = r0 + warp * 16 + g, rb = ra + 8;
  // keys a row admits: its own sequence's rows [lo, lo + len) (up to r when
  // causal); rows past the batch admit none
  auto key_range = [&](int r, int& lo, int& len) {
    if (r >= T) {
      lo = 0;
      len = 0;
      return;
    }
    int a = 0, b2 = nseq - 2;                                   // largest i with soff[i] <= r
    while (a < b2) {
      const int mid = (a + b2 + 1) >> 1;
      if (soff[mid] <= r) a = mid; else b2 = mid - 1;
    }
    lo = soff[a];
    len = (causal ? r + 1 : soff[a + 1]) - lo;
  };
  int lo_a, len_a, lo_b, len_b;
  key_range(ra, lo_a, len_a);
  key_range(rb, lo_b, len_b);
  // the warp's key range: chunks outside it are skipped
  const int wlo = __reduce_min_sync(0xffffffffu, min(len_a > 0 ? lo_a : INT_MAX, len_b > 0 ? lo_b : INT_MAX));
  const int whi = __reduce_max_sync(0xffffffffu, max(lo_a + len_a, lo_b + len_b));

  int it = 0;
  for (int j = 0; j < nhl; ++j) {
    const int h = h0 + j, qb = j & 1;
    if (!mbar_wait(qfull0 + 8 * qb, (j >> 1) & 1)) {
      if (lane == 0) atomicAdd(err + ERR_TIMEOUT, 1);
      return;
    }
    uint32_t qa[DP / 16][4];
    {
      const int qr = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int ks = 0; ks < DP / 16; ++ks)
        ldmatrix_x4(qa[ks], sbase + qb * SL::kQ + sw128_off(qr, 2 * ks + (lane >> 4)));
    }
    // Q is in registers: the buffer may refill.  The reads are generic-proxy,
    // the refill an async-proxy (TMA) write: fence the two before the release.
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(qempty0 + 8 * qb);

    float o[DP / 8][4];
#pragma unroll
    for (int t = 0; t < DP / 8; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

    for (int c = 0; c < nch; ++c, ++it) {
      const int s = it % S;
      if (!mbar_wait(kvfull0 + 8 * s, (it / S) & 1)) {
        if (lane == 0) atomicAdd(err + ERR_TIMEOUT, 1);
        return;
      }
      const int c0 = Klo + 64 * c;
      if (c0 < whi && c0 + 64 > wlo) {
        const uint32_t kb = sbase + SL::kKVOff + s * SL::kKV, vb = kb + SL::kNB * SL::kBox;
        float sc[8][4];
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          sc[2 * np][0] = sc[2 * np][1] = sc[2 * np][2] = sc[2 * np][3] = 0.f;
          sc[2 * np + 1][0] = sc[2 * np + 1][1] = sc[2 * np + 1][2] = sc[2 * np + 1][3] = 0.f;
          if (c0 + 16 * np < whi && c0 + 16 * np + 16 > wlo) {
            const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
            for (int ks = 0; ks < DP / 16; ++ks) {
              uint32_t kf[4];
              ldmatrix_x4(kf, kb + sw128_off(key, 2 * ks + ((lane >> 3) & 1)));
              mma_bf16_16816(sc[2 * np], qa[ks], kf[0], kf[1]);
              mma_bf16_16816(sc[2 * np + 1], qa[ks], kf[2], kf[3]);
            }
          }
        }
        // mask to the row's own keys; block maxima of the raw scores (the
        // log2-domain scale is positive and folds into the exponent below)
        float bm_a = -INFINITY, bm_b = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const int cc = c0 + nt * 8 + 2 * tq;
          const unsigned ua = static_cast<unsigned>(cc - lo_a), ub = static_cast<unsigned>(cc - lo_b);
          sc[nt][0] = ua < static_cast<unsigned>(len_a) ? sc[nt][0] : -INFINITY;
          sc[nt][1] = ua + 1u < static_cast<unsigned>(len_a) ? sc[nt][1] : -INFINITY;
          sc[nt][2] = ub < static_cast<unsigned>(len_b) ? sc[nt][2] : -INFINITY;
          sc[nt][3] = ub + 1u < static_cast<unsigned>(len_b) ? sc[nt][3] : -INFINITY;
          bm_a = fmaxf(bm_a, fmaxf(sc[nt][0], sc[nt][1]));
          bm_b = fmaxf(bm_b, fmaxf(sc[nt][2], sc[nt][3]));
        }
        bm_a = fmaxf(bm_a, __shfl_xor_sync(0xffffffffu, bm_a, 1));
        bm_a = fmaxf(bm_a, __shfl_xor_sync(0xffffffffu, bm_a, 2));
        bm_b = fmaxf(bm_b, __shfl_xor_sync(0xffffffffu, bm_b, 1));
        bm_b = fmaxf(bm_b, __shfl_xor_sync(0xffffffffu, bm_b, 2));
        const float mn_a = fmaxf(m_a, bm_a), mn_b = fmaxf(m_b, bm_b);
        // shift in the log2 domain; a row with no admitted key so far keeps
        // m = -inf and shifts by 0
        const float sh_a = mn_a == -INFINITY ? 0.f : mn_a * scale_log2;
        const float sh_b = mn_b == -INFINITY ? 0.f : mn_b * scale_log2;
        const float al_a = ex2_approx_ftz(fmaf(m_a, scale_log2, -sh_a));
        const float al_b = ex2_approx_ftz(fmaf(m_b, scale_log2, -sh_b));
        m_a = mn_a;
        m_b = mn_b;
        float ps_a = 0.f, ps_b = 0.f;
        uint32_t pa[4][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const float p0 = ex2_approx_ftz(fmaf(sc[nt][0], scale_log2, -sh_a));
          const float p1 = ex2_approx_ftz(fmaf(sc[nt][1], scale_log2, -sh_a));
          const float p2 = ex2_approx_ftz(fmaf(sc[nt][2], scale_log2, -sh_b));
          const float p3 = ex2_approx_ftz(fmaf(sc[nt][3], scale_log2, -sh_b));
          ps_a += p0 + p1;
          ps_b += p2 + p3;
          pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16x2(p0, p1);
          pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16x2(p2, p3);
        }
        l_a = l_a * al_a + ps_a;
        l_b = l_b * al_b + ps_b;
#pragma unroll
        for (int t = 0; t < DP / 8; ++t) {
          o[t][0] *= al_a;
          o[t][1] *= al_a;
          o[t][2] *= al_b;
          o[t][3] *= al_b;
        }
        // O += P V: V fragments by ldmatrix.trans from the key-major rows
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          if (c0 + 16 * ks < whi && c0 + 16 * ks + 16 > wlo) {
            const int key = ks * 16 + (lane & 15);
#pragma unroll
            for (int t = 0; t < DP / 8; t += 2) {
              uint32_t bv[4];
              ldmatrix_x4_trans(bv, vb + sw128_off(key, t + (lane >> 4)));
              mma_bf16_16816(o[t], pa[ks], bv[0], bv[1]);
              mma_bf16_16816(o[t + 1], pa[ks], bv[2], bv[3]);
            }
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(kvempty0 + 8 * s);
    }
    // normalise and store this head's rows
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    const float inv_a = ra < T ? 1.0f / l_a : 0.f, inv_b = rb < T ? 1.0f / l_b : 0.f;
    bf16* cb = ctx + h * DP;
#pragma unroll
    for (int t = 0; t < DP / 8; ++t) {
      const int col = t * 8 + 2 * tq;
      if (ra < T)
        *reinterpret_cast<uint32_t*>(cb + static_cast<size_t>(ra) * H + col) =
            pack_bf16x2(o[t][0] * inv_a, o[t][1] * inv_a);
      if (rb < T)
        *reinterpret_cast<uint32_t*>(cb + static_cast<size_t>(rb) * H + col) =
            pack_bf16x2(o[t][2] * inv_b, o[t][3] * inv_b);
    }
  }
}

template <int DP>
cudaError_t launch_tile(const void* qkv, void* ctx, const int32_t* offsets, int n, int T, int nh,
                        int max_len, int causal, int* err, int num_sms, cudaStream_t st,
                        const L2Prefetch& pf) {
  using SL = TileSmem<DP>;
  const int H = nh * DP;
  CUtensorMap tm;
  const char* why = "";
  // exactly T rows: key rows past the batch read as zeros
  if (!make_tmap_bf16(&tm, qkv, static_cast<uint64_t>(T), static_cast<uint64_t>(3 * H), 64, &why))
    return cudaErrorInvalidValue;
  static const cudaError_t attr_err = cudaFuncSetAttribute(
      attn_tile_kernel<DP>, cudaFuncAttributeMaxDynamicSharedMemorySize, SL::kBytes);
  if (attr_err != cudaSuccess) return attr_err;
  const int tiles = (T + 63) / 64;
  // heads per CTA: enough CTAs for a few rounds of the resident ones, and as
  // many heads per CTA as that leaves (their loads pipeline across heads).
  // Short rows give a tile one or two key chunks per head, so fewer, longer
  // CTAs keep the ring busy; long rows pipeline within a head and balance
  // better over more CTAs (measured on B200: lengths 2..100 best at 4
  // rounds, lengths 5..500 and the causal 1.3B shape at 8).
  const int rounds = max_len <= 128 ? 4 : 8;
  const int target = rounds * num_sms * SL::kCtasPerSm;
  const int groups = std::min(nh, std::max(1, (target + tiles - 1) / tiles));
  const int hpc = (nh + groups - 1) / groups;
  dim3 grid(tiles, (nh + hpc - 1) / hpc);
  L2PrefetchArgs pa;
  for (int k = 0; k < 2; ++k) {
    pa.ptr[k] = pf.ptr[k];
    pa.bytes[k] = pf.bytes[k];
  }
  const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(DP));
  launch_k(attn_tile_kernel<DP>, grid, dim3(160), SL::kBytes, st, tm, static_cast<bf16*>(ctx),
           offsets, n, T, H, nh, hpc, scale_log2, causal, err, pa);
  return cudaGetLastError();
}

int pad_head_dim(int d) { return d <= 32 ? 32 : (d <= 64 ? 64 : (d <= 128 ? 128 : -1)); }

template <int DP, bool PFX>
cudaError_t launch_fused_async(dim3 grid, cudaStream_t st, const bf16* q, bf16* c,
                               const int32_t* offsets, const int32_t* rb_off, int n, int H, int d,
                               float scale_log2, int causal, const L2Prefetch& pf,
                               const int32_t* pre_start = nullptr, const int32_t* pre_len = nullptr) {
  L2PrefetchArgs pa;
  for (int k = 0; k < 2; ++k) {
    pa.ptr[k] = pf.ptr[k];
    pa.bytes[k] = pf.bytes[k];
  }
  // the attribute is per function: set once (thread-safe static initialisation)
  static const cudaError_t attr_err = cudaFuncSetAttribute(
      attn_fused_async_kernel<DP, PFX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
      FusedSmem<DP>::kBytes);
  if (attr_err != cudaSuccess) return attr_err;
  launch_k(attn_fused_async_kernel<DP, PFX>, grid, dim3(128), FusedSmem<DP>::kBytes, st, q, c,
           offsets, rb_off, n, H, d, scale_log2, causal, pa, pre_start, pre_len);
  return cudaGetLastError();
}

template <typename T, int G, int MAXC, int U>
cudaError_t softmax_t(void* S, const int32_t* offsets, const int64_t* s_off, int n, long long rows,
                      int nh, int causal, cudaStream_t st) {
  const long long rows_per_cta = 8LL * (32 / G) * U;
  const long long blocks = (rows + rows_per_cta - 1) / rows_per_cta;
  launch_k(softmax_kernel<T, G, MAXC, U>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st,
           static_cast<T*>(S), offsets, s_off, n, rows, nh, causal);
  return cudaGetLastError();
}

// Lanes per row G = the smallest power of two covering the longest row's
// 8-element chunks (at most 32), and U rows per lane group so that a lane has
// four chunks in flight.
template <typename T>
cudaError_t softmax_dispatch(void* S, const int32_t* offsets, const int64_t* s_off, int n,
                             long long rows, int nh, int max_len, int causal, cudaStream_t st) {
  const int chunks = ((max_len + 7) & ~7) / 8;
  if (chunks <= 4) return softmax_t<T, 4, 1, 4>(S, offsets, s_off, n, rows, nh, causal, st);
  if (chunks <= 8) return softmax_t<T, 8, 1, 4>(S, offsets, s_off, n, rows, nh, causal, st);
  if (chunks <= 16) return softmax_t<T, 16, 1, 4>(S, offsets, s_off, n, rows, nh, causal, st);
  if (chunks <= 32) return softmax_t<T, 32, 1, 4>(S, offsets, s_off, n, rows, nh, causal, st);
  if (chunks <= 64) return softmax_t<T, 32, 2, 2>(S, offsets, s_off, n, rows, nh, causal, st);
  if (chunks <= 96) return softmax_t<T, 32, 3, 1>(S, offsets, s_off, n, rows, nh, causal, st);
  if (chunks <= 128) return softmax_t<T, 32, 4, 1>(S, offsets, s_off, n, rows, nh, causal, st);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t bounds_errors_attention(int32_t* out, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_bounds_attention, sizeof(int32_t));
  if (e == cudaSuccess && reset) {
    const int32_t zero = 0;
    e = cudaMemcpyToSymbol(g_bounds_attention, &zero, sizeof(int32_t));
  }
  return e;
}

cudaError_t attn_scores_launch(const void* qkv, void* S, const int32_t* offsets,
                               const int32_t* rb_off, const int64_t* s_off, int n_seqs,
                               int n_row_blocks, int n_heads, int head_dim, int causal,
                               cudaStream_t st) {
  if (n_row_blocks == 0) return cudaSuccess;
  const int H = n_heads * head_dim;
  const float scale = 1.0f / sqrtf(static_cast<float>(head_dim));
  dim3 grid(n_row_blocks, n_heads);
  const bf16* q = static_cast<const bf16*>(qkv);
  bf16* s = static_cast<bf16*>(S);
  switch (pad_head_dim(head_dim)) {
    case 32: launch_k(attn_scores_kernel<32>, grid, 128, 0, st, q, s, offsets, rb_off, s_off, n_seqs, H, head_dim, scale, causal); break;
    case 64: launch_k(attn_scores_kernel<64>, grid, 128, 0, st, q, s, offsets, rb_off, s_off, n_seqs, H, head_dim, scale, causal); break;
    case 128: launch_k(attn_scores_kernel<128>, grid, 128, 0, st, q, s, offsets, rb_off, s_off, n_seqs, H, head_dim, scale, causal); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

size_t softmax_classes_scratch_bytes(int n_seqs, int T, int n_heads) {
  return SoftmaxIndexLayout(n_seqs, static_cast<long long>(n_heads) * T).bytes;
}

cudaError_t softmax_classes_launch(void* S, int s_dtype, const int32_t* offsets,
                                   const int64_t* s_off, int n_seqs, int T, int n_heads,
                                   int max_len, int causal, void* scratch, int num_sms,
                                   cudaStream_t st) {
  if (n_seqs == 0 || T == 0) return cudaSuccess;
  if (max_len < 1 || max_len > 1024) return cudaErrorInvalidValue;
  const SoftmaxIndexLayout lay(n_seqs, static_cast<long long>(n_heads) * T);
  // The count, index and class kernels run in plain stream order (no
  // programmatic dependent launch), each after the previous kernel has
  // completed.  With all three launched programmatically after the scores
  // kernel, rm_score on B200 gave rows of P that had not been normalised
  // (decoder, materialised attention, wrong in some calls and not in others);
  // with either the class kernel or the two index kernels in plain order the
  // scores matched the oracle in every call.  Every kernel of the chain waits
  // (griddepcontrol.wait) before it touches global memory; the cause was not
  // isolated.
  PdlScope plain(false);
  uint8_t* base = static_cast<uint8_t*>(scratch);
  unsigned long long* ctr = reinterpret_cast<unsigned long long*>(base);
  long long* seq_base = reinterpret_cast<long long*>(base + lay.base);
  int32_t* row_seq = reinterpret_cast<int32_t*>(base + lay.rows);
  cudaError_t e = cudaMemsetAsync(ctr, 0, 16 * kSmClasses, st);
  if (e != cudaSuccess) return e;
  const int seq_blocks = std::max(1, std::min((n_seqs + 255) / 256, num_sms * 4));
  launch_k(softmax_count_kernel, dim3(seq_blocks), dim3(256), 0, st, offsets, n_seqs, n_heads, causal,
           ctr);
  const int idx_blocks = std::max(1, std::min((n_seqs + 7) / 8, num_sms * 8));
  launch_k(softmax_index_kernel, dim3(idx_blocks), dim3(256), 0, st, offsets, n_seqs, n_heads, causal,
           ctr, seq_base, row_seq);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int k_max = softmax_class_of(max_len);
  // three CTAs of 256 threads per SM, each warp walking one stretch of each
  // class; bf16 rows through the warps' shared-memory rings (64 KB per CTA)
  if (s_dtype == 0) {
    launch_k(softmax_class_kernel<float>, dim3(num_sms * 3), dim3(kSmClassThreads), 0, st,
             static_cast<float*>(S), offsets, s_off, ctr, seq_base, row_seq, k_max, n_seqs, n_heads,
             causal);
  } else {
    constexpr int kRing = (kSmClassThreads / 32) * kSmRingWarpBytes;
    static const cudaError_t attr_err = cudaFuncSetAttribute(
        softmax_class_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize, kRing);
    if (attr_err != cudaSuccess) return attr_err;
    launch_k(softmax_class_kernel<bf16>, dim3(num_sms * 3), dim3(kSmClassThreads), kRing, st,
             static_cast<bf16*>(S), offsets, s_off, ctr, seq_base, row_seq, k_max, n_seqs, n_heads,
             causal);
  }
  return cudaGetLastError();
}

cudaError_t softmax_launch(void* S, int s_dtype, const int32_t* offsets, const int64_t* s_off,
                           int n_seqs, int T, int n_heads, int max_len, int causal, int* err,
                           cudaStream_t st) {
  const long long rows = static_cast<long long>(n_heads) * T;
  if (rows == 0) return cudaSuccess;
  (void)err;   // the row kernel has no waits that could give up
  if (s_dtype == 0)
    return softmax_dispatch<float>(S, offsets, s_off, n_seqs, rows, n_heads, max_len, causal, st);
  return softmax_dispatch<bf16>(S, offsets, s_off, n_seqs, rows, n_heads, max_len, causal, st);
}

cudaError_t attn_fused_launch(const void* qkv, void* ctx, const int32_t* offsets,
                              const int32_t* rb_off, int n_seqs, int n_row_blocks, int n_heads,
                              int head_dim, int causal, cudaStream_t st, const L2Prefetch& pf) {
  if (n_row_blocks == 0) return cudaSuccess;
  const int H = n_heads * head_dim;
  const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(head_dim));
  dim3 grid(n_row_blocks, n_heads);
  const bf16* q = static_cast<const bf16*>(qkv);
  bf16* c = static_cast<bf16*>(ctx);
  if (head_dim % 8 == 0) {
    switch (pad_head_dim(head_dim)) {
      case 32: return launch_fused_async<32, false>(grid, st, q, c, offsets, rb_off, n_seqs, H, head_dim, scale_log2, causal, pf);
      case 64: return launch_fused_async<64, false>(grid, st, q, c, offsets, rb_off, n_seqs, H, head_dim, scale_log2, causal, pf);
      case 128: return launch_fused_async<128, false>(grid, st, q, c, offsets, rb_off, n_seqs, H, head_dim, scale_log2, causal, pf);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (pad_head_dim(head_dim)) {
    case 32: launch_k(attn_fused_kernel<32>, grid, 128, 0, st, q, c, offsets, rb_off, n_seqs, H, head_dim, scale_log2, causal); break;
    case 64: launch_k(attn_fused_kernel<64>, grid, 128, 0, st, q, c, offsets, rb_off, n_seqs, H, head_dim, scale_log2, causal); break;
    case 128: launch_k(attn_fused_kernel<128>, grid, 128, 0, st, q, c, offsets, rb_off, n_seqs, H, head_dim, scale_log2, causal); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t attn_tile_launch(const void* qkv, void* ctx, const int32_t* offsets, int n_seqs, int T,
                             int n_heads, int head_dim, int max_len, int causal, int* err,
                             int num_sms, cudaStream_t st, const L2Prefetch& pf) {
  if (T == 0) return cudaSuccess;
  if (head_dim == 64)
    return launch_tile<64>(qkv, ctx, offsets, n_seqs, T, n_heads, max_len, causal, err, num_sms, st,
                           pf);
  if (head_dim == 128)
    return launch_tile<128>(qkv, ctx, offsets, n_seqs, T, n_heads, max_len, causal, err, num_sms,
                            st, pf);
  return cudaErrorInvalidValue;
}

cudaError_t attn_fused_prefix_launch(const void* qkv, void* ctx, const int32_t* offsets,
                                     const int32_t* rb_off, const int32_t* pre_start,
                                     const int32_t* pre_len, int n_seqs, int n_row_blocks,
                                     int n_heads, int head_dim, cudaStream_t st,
                                     const L2Prefetch& pf) {
  if (n_row_blocks == 0) return cudaSuccess;
  if (head_dim % 8 != 0) return cudaErrorInvalidValue;
  const int H = n_heads * head_dim;
  const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(head_dim));
  dim3 grid(n_row_blocks, n_heads);
  const bf16* q = static_cast<const bf16*>(qkv);
  bf16* c = static_cast<bf16*>(ctx);
  switch (pad_head_dim(head_dim)) {
    case 32: return launch_fused_async<32, true>(grid, st, q, c, offsets, rb_off, n_seqs, H, head_dim, scale_log2, 1, pf, pre_start, pre_len);
    case 64: return launch_fused_async<64, true>(grid, st, q, c, offsets, rb_off, n_seqs, H, head_dim, scale_log2, 1, pf, pre_start, pre_len);
    case 128: return launch_fused_async<128, true>(grid, st, q, c, offsets, rb_off, n_seqs, H, head_dim, scale_log2, 1, pf, pre_start, pre_len);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t attn_context_launch(const void* S, const void* qkv, void* ctx, const int32_t* offsets,
                                const int32_t* rb_off, const int64_t* s_off, int n_seqs,
                                int n_row_blocks, int n_heads, int head_dim, int causal,
                                cudaStream_t st) {
  if (n_row_blocks == 0) return cudaSuccess;
  const int H = n_heads * head_dim;
  dim3 grid(n_row_blocks, n_heads);
  const bf16* s = static_cast<const bf16*>(S);
  const bf16* q = static_cast<const bf16*>(qkv);
  bf16* c = static_cast<bf16*>(ctx);
  switch (pad_head_dim(head_dim)) {
    case 32: launch_k(attn_context_kernel<32>, grid, 128, 0, st, s, q, c, offsets, rb_off, s_off, n_seqs, H, head_dim, causal); break;
    case 64: launch_k(attn_context_kernel<64>, grid, 128, 0, st, s, q, c, offsets, rb_off, s_off, n_seqs, H, head_dim, causal); break;
    case 128: launch_k(attn_context_kernel<128>, grid, 128, 0, st, s, q, c, offsets, rb_off, s_off, n_seqs, H, head_dim, causal); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace rmk
