// Packed-row attention on the 5th-generation tensor cores: head dim 64, every
// sequence at most 128 tokens (BERT-base and the other encoders of this size
// scoring short texts).  The math is the scorer's attention sublayer as in
// attention.cu (TurboTransformers, proposed-method section: batch GEMMs with
// a batch softmax in between): per head, S = Q K^T scaled by 1/sqrt(64), a
// row softmax over the row's own sequence (keys c <= r when causal), O = P V.
//
// Work decomposition.  The host cuts the batch into tiles of whole
// sequences, at most 128 packed rows each (a greedy pass over the offsets,
// attn_tc_tiles), so that a tile's keys are exactly its own rows.  A CTA (one
// per SM) takes one tile and a group of heads and runs them through a
// pipeline:
//   warp 0, one lane : TMA producer -- per head the 128-row boxes of Q, K and V
//                      (128-byte swizzle; rows past the batch read as zeros)
//                      into a ring of four head slots; Q and K are released
//                      when S is computed, V after P V, and V loads trail the
//                      Q and K loads by one head;
//   warp 1, one lane : tcgen05.mma -- S = Q K^T (M = N = 128, K = 64) into the
//                      head's 128-column TMEM region; once the softmax has
//                      written P there, O = P V (M = 128, N = 64, K = the
//                      tile's rows in steps of 16; A = P read from TMEM, B = V
//                      in its natural [key][dim] layout through an MN-major
//                      descriptor) into the region's upper 64 columns;
//                      whichever of the two is ready first;
//   warps 2..17      : four softmax groups of four warps, group w taking heads
//                      w, w+4, ... in TMEM region w.  A thread owns one tile
//                      row (its TMEM lane): it reads the row's scores one
//                      32-column group at a time (only the groups its warp's
//                      rows admit), takes the maximum and the sum over the keys
//                      of its own sequence in fp32 (the scale folded into the
//                      exponent's FMA in the log2 domain), writes P rounded to
//                      bf16 over the scores it has read (two keys per TMEM
//                      column), then reads O, divides by the sum and stores
//                      the row's 64 context values.
// No warp-level reduction is needed: a row's maximum and sum stay in one
// thread.  Every mbarrier wait is bounded; a wait that gives up counts into
// err[ERR_TIMEOUT], the role stops, and the producer and the MMA issuer wait
// (bounded) for their copies and MMAs before the CTA frees its TMEM and exits.
#include <cuda.h>

#include <algorithm>
#include <climits>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rmk {
namespace {

RMK_BOUNDS_UNIT(attention_tc)

constexpr int kTcRows = 128;   // rows of a tile, and keys of a tile
constexpr int kTcDim = 64;     // head dim

struct TcSmem {
  static constexpr int kBox = kTcRows * kTcDim * 2;   // 16 KB: 128 rows x 128 B, 128-byte swizzle
  static constexpr int kSlots = 4;                     // Q, K and V of four heads in flight
  static constexpr int kSlot = 3 * kBox;
  static constexpr int kBarOff = kSlots * kSlot;
  // qk_full[4] v_full[4] qk_free[4] v_free[4] s_full[4] o_full[4] p_full[4] tmem_free[4]
  static constexpr int kBars = 32;
  static constexpr int kTmemSlotOff = kBarOff + kBars * 8;
  static constexpr int kSeqOff = kTmemSlotOff + 16;    // offsets of the tile's sequences
  static constexpr int kMaxSeqs = kTcRows + 1;
  static constexpr int kBytes = kSeqOff + kMaxSeqs * 4 + 1024;   // + 1024-byte alignment slack
  static_assert(kBytes <= 232448, "fits one CTA's shared memory");
};
constexpr int kTcGroups = 4;                           // softmax groups = TMEM regions
constexpr int kTcThreads = 64 + kTcGroups * 128;

// One tcgen05.mma (kind::f16, one CTA) with both operands in shared memory.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                            bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

// Bits [0, x) of a 32-bit word, for x clamped to 0..32.
__device__ __forceinline__ uint32_t low_bits(int x) {
  return x <= 0 ? 0u : (x >= 32 ? 0xffffffffu : ((1u << x) - 1u));
}

// Named barrier 1 over the 512 softmax threads that also ANDs a flag across
// them: every thread leaves with the same answer, so a bounded wait that gave
// up in one thread ends the loop in all of them together (none is left at a
// barrier that the others will not reach).
__device__ __forceinline__ bool softmax_bar_and(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 512, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"(ok ? 1u : 0u)
      : "memory");
  return r != 0;
}

// The same with A read from tensor memory (M = 128 lanes, two 16-bit
// elements of a row per 32-bit column).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                            bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

// Shared-memory descriptor of an MN-major operand written by TMA with the
// 128-byte swizzle: rows of 128 B along K (here: keys), each holding 64
// elements of the MN dimension (here: the head dim), 8-row swizzle atoms of
// 1024 B.  The stride between 8-row groups along K (stride byte offset) is
// 1024 B; with 64 MN elements there is one atom across MN, so the leading
// byte offset is not used (set to the same 1024 B).
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (64ull << 16) | (64ull << 32) |
         (1ull << 46) | (2ull << 61);
}

__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm, bf16* __restrict__ ctx,
                   const int32_t* __restrict__ offsets, const int32_t* __restrict__ tiles,
                   int n, int T, int H, int nh, int hpc, float scale_log2, int causal,
                   int* __restrict__ err, L2PrefetchArgs pf) {
  using SL = TcSmem;
  constexpr int NS = SL::kSlots;
  extern __shared__ uint8_t tc_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(sm);
  const uint32_t bar0 = sbase + SL::kBarOff;
  auto qk_full = [&](int s) { return bar0 + 8u * s; };
  auto v_full = [&](int s) { return bar0 + 8u * (4 + s); };
  auto qk_free = [&](int s) { return bar0 + 8u * (8 + s); };
  auto v_free = [&](int s) { return bar0 + 8u * (12 + s); };
  auto s_full = [&](int t) { return bar0 + 8u * (16 + t); };
  auto o_full = [&](int t) { return bar0 + 8u * (20 + t); };
  auto p_full = [&](int t) { return bar0 + 8u * (24 + t); };
  auto tmem_free = [&](int t) { return bar0 + 8u * (28 + t); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SL::kTmemSlotOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int k = 0; k < 4; ++k) {
      mbar_init(qk_full(k), 1);
      mbar_init(v_full(k), 1);
      mbar_init(qk_free(k), 1);
      mbar_init(v_free(k), 1);
      mbar_init(s_full(k), 1);
      mbar_init(o_full(k), 1);
      mbar_init(p_full(k), 4);      // the four warps of a softmax group
      mbar_init(tmem_free(k), 4);
    }
    mbar_init_fence();
  }
  if (warp == 1) {
    // four 128-column regions: all 512 columns of this SM's TMEM (one CTA per SM)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();
  l2_prefetch_share(pf);
  pdl_wait();

  const int h0 = blockIdx.y * hpc;
  const int s_first = tiles[blockIdx.x], s_end = tiles[blockIdx.x + 1];
  const int r0 = offsets[s_first], r1 = offsets[s_end];
  const int nrows = r1 - r0;
  // checked build: the tile holds whole sequences and at most 128 rows (the
  // same test in every thread); a failed tile does no work
  const bool tile_ok = in_bounds(s_first >= 0 && s_end > s_first && s_end <= n &&
                                 s_end - s_first + 1 <= SL::kMaxSeqs && r0 >= 0 && nrows >= 1 &&
                                 nrows <= kTcRows && r1 <= T);
  const int nhl = tile_ok ? min(hpc, nh - h0) : 0;

  if (warp == 0) {
    // ---- TMA producer ----
    // Q and K of head j, then V of head j-1: Q and K are free again once S is
    // computed, V only after P V, so V trails by one head and a wait for a V
    // slot never holds up the next head's Q and K.
    if (lane == 0) {
      int nqk = 0, nv = 0;
      bool ok = true;
      for (int j = 0; j <= nhl && ok; ++j) {
        if (j < nhl) {
          const int s = j % NS;
          if (j >= NS && !mbar_wait(qk_free(s), ((j / NS) - 1) & 1)) {
            atomicAdd(err + ERR_TIMEOUT, 1);
            break;
          }
          const int col = (h0 + j) * kTcDim;
          const uint32_t dst = sbase + s * SL::kSlot;
          mbar_arrive_expect_tx(qk_full(s), 2 * SL::kBox);
          tma_load_2d(dst, &tm, col, r0, qk_full(s));
          tma_load_2d(dst + SL::kBox, &tm, H + col, r0, qk_full(s));
          ++nqk;
        }
        if (j >= 1) {
          const int jv = j - 1, s = jv % NS;
          if (jv >= NS && !mbar_wait(v_free(s), ((jv / NS) - 1) & 1)) {
            atomicAdd(err + ERR_TIMEOUT, 1);
            break;
          }
          mbar_arrive_expect_tx(v_full(s), SL::kBox);
          tma_load_2d(sbase + s * SL::kSlot + 2 * SL::kBox, &tm, 2 * H + (h0 + jv) * kTcDim, r0,
                      v_full(s));
          ++nv;
        }
      }
      // no copy into this CTA's shared memory may be in flight when it exits
      bool drained = true;
      for (int j = nqk - 1; drained && j >= 0 && j >= nqk - NS; --j)
        drained = mbar_wait(qk_full(j % NS), (j / NS) & 1);
      for (int j = nv - 1; drained && j >= 0 && j >= nv - NS; --j)
        drained = mbar_wait(v_full(j % NS), (j / NS) & 1);
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    // Issues S of the next head and P V of the oldest head whose P is
    // written, whichever is ready first (each in head order).
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTcRows, kTcRows);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kTcRows, kTcDim) | (1u << 16);   // B MN-major
      // 16-key steps of P V that hold a tile key (at most the tile's 8)
      const int nk16 = min((nrows + 15) / 16, kTcRows / 16);
      int js = 0, jp = 0;                    // next S, next P V
      unsigned long long idle_since = globaltimer_ns();
      while (jp < nhl) {
        bool progressed = false;
        if (js < nhl) {
          const int s = js % NS, t = js & 3;
          if (mbar_test_wait(qk_full(s), (js / NS) & 1) &&
              (js < 4 || mbar_test_wait(tmem_free(t), ((js >> 2) - 1) & 1))) {
            tc_fence_after();
            const uint32_t q = sbase + s * SL::kSlot;
            const uint64_t qd = smem_desc_k_sw128(q), kd = smem_desc_k_sw128(q + SL::kBox);
            const uint32_t d = tmem + static_cast<uint32_t>(t * 128);
#pragma unroll
            for (int ks = 0; ks < kTcDim / 16; ++ks)   // 16 dims = 32 bytes along the swizzled row
              mma_bf16_ss(d, qd + 2ull * ks, kd + 2ull * ks, idesc_s, ks > 0);
            tc_commit<1>(s_full(t));
            tc_commit<1>(qk_free(s));
            ++js;
            progressed = true;
          }
        }
        if (jp < js) {
          const int s = jp % NS, t = jp & 3;
          if (mbar_test_wait(p_full(t), (jp >> 2) & 1) && mbar_test_wait(v_full(s), (jp / NS) & 1)) {
            tc_fence_after();
            const uint32_t v = sbase + s * SL::kSlot + 2 * SL::kBox;
            const uint32_t reg = tmem + static_cast<uint32_t>(t * 128);
            for (int kb = 0; kb < nk16; ++kb)   // P: 8 columns per 16 keys; V: 16 key rows
              mma_bf16_ts(reg + 64, reg + kb * 8, smem_desc_mn_sw128(v + kb * 16 * 128), idesc_o,
                          kb > 0);
            tc_commit<1>(o_full(t));
            tc_commit<1>(v_free(s));
            ++jp;
            progressed = true;
          }
        }
        if (progressed) {
          idle_since = globaltimer_ns();
        } else if (globaltimer_ns() - idle_since > kWaitLimitNs) {
          atomicAdd(err + ERR_TIMEOUT, 1);
          break;
        }
      }
      // TMEM is freed after the last MMAs have completed (bounded waits)
      bool drained = true;
      if (js > 0) drained = mbar_wait(s_full((js - 1) & 3), ((js - 1) >> 2) & 1);
      if (drained && jp > 0) mbar_wait(o_full((jp - 1) & 3), ((jp - 1) >> 2) & 1);
    }
  } else {
    // ---- softmax groups: one tile row per thread ----
    const int w = (warp - 2) >> 2;            // group = TMEM region
    const int qtr = warp & 3;                 // TMEM lane quarter of this warp
    const int i = qtr * 32 + lane;            // tile row = TMEM lane
    const int r = r0 + i;
    int32_t* soff = reinterpret_cast<int32_t*>(sm + SL::kSeqOff);
    const int nseq = min(s_end - s_first, SL::kMaxSeqs - 1);   // <= 128 for tiles of whole sequences
    for (int k = threadIdx.x - 64; k <= nseq && nhl > 0; k += kTcGroups * 128)
      soff[k] = offsets[s_first + k];
    asm volatile("bar.sync 1, %0;" ::"n"(kTcGroups * 128) : "memory");   // the softmax warps
    // the keys this row admits, as tile columns [lo, lo + len)
    int lo = 0, len = 0;
    if (i < nrows && nhl > 0) {
      int a = 0, b = nseq - 1;                // largest a with soff[a] <= r
      while (a < b) {
        const int mid = (a + b + 1) >> 1;
        if (soff[mid] <= r) a = mid; else b = mid - 1;
      }
      lo = soff[a] - r0;
      len = causal ? r - soff[a] + 1 : soff[a + 1] - soff[a];
    }
    // 32-column groups that some row of this warp admits
    const int wlo = __reduce_min_sync(0xffffffffu, len > 0 ? lo : INT_MAX);
    const int whi = __reduce_max_sync(0xffffffffu, len > 0 ? lo + len : 0);
    bool need[4];
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) need[gi] = gi * 32 < whi && gi * 32 + 32 > wlo;
    const uint32_t treg = tmem + (static_cast<uint32_t>(qtr * 32) << 16) + w * 128;

    for (int j = w; j < nhl; j += kTcGroups) {
      const int use = j >> 2;
      // the row's key range, re-read per head through an opaque move: the
      // per-column tests below (bits of vm) would otherwise be hoisted out of
      // this loop as 128 loop-invariant booleans, one register each
      int lo_h, len_h;
      asm volatile("mov.b32 %0, %1;" : "=r"(lo_h) : "r"(lo));
      asm volatile("mov.b32 %0, %1;" : "=r"(len_h) : "r"(len));
      if (!mbar_wait(s_full(w), use & 1)) {
        if (lane == 0) atomicAdd(err + ERR_TIMEOUT, 1);
        break;
      }
      tc_fence_after();
      // the row's maximum over its own keys
      // columns 32gi + c the row admits, as bit c of vm[gi]
      uint32_t vm[4];
#pragma unroll
      for (int gi = 0; gi < 4; ++gi)
        vm[gi] = low_bits(lo_h + len_h - 32 * gi) & ~low_bits(lo_h - 32 * gi);
      float m = -INFINITY;
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) {
        if (!need[gi]) continue;
        uint32_t sv[32];
        tmem_ld_32cols(treg + gi * 32, sv);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (vm[gi] & (1u << c)) m = fmaxf(m, __uint_as_float(sv[c]));
      }
      const float msc = len_h > 0 ? m * scale_log2 : 0.f;
      // P = exp2(s * scale_log2 - m * scale_log2) on the row's keys, 0 elsewhere,
      // written over the scores as bf16 pairs: keys 32gi.. go to columns
      // 16gi.., which hold scores of group gi/2 <= gi, already read.  The sum
      // is taken in fp32 before P is rounded to bf16.
      // Two columns per packed fp32x2 FMA and add; the exponential is the
      // hardware's ex2.approx with subnormal results flushed to zero (terms
      // below 2^-126 of the row maximum's term, far under one bf16 ulp of P).
      const uint64_t sc2 = f32x2_splat(scale_log2), nm2 = f32x2_splat(-msc);
      uint64_t l2 = 0ull;                     // two running partial sums
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) {
        uint32_t pk[16];
        if (need[gi]) {
          uint32_t sv[32];
          tmem_ld_32cols(treg + gi * 32, sv);
          tmem_wait_ld();
#pragma unroll
          for (int c2 = 0; c2 < 16; ++c2) {
            const bool in0 = (vm[gi] >> (2 * c2)) & 1u, in1 = (vm[gi] >> (2 * c2 + 1)) & 1u;
            float x0, x1;
            f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(sv[2 * c2]), __uint_as_float(sv[2 * c2 + 1])),
                                   sc2, nm2),
                         x0, x1);
            const float p0 = in0 ? ex2_approx_ftz(x0) : 0.f;
            const float p1 = in1 ? ex2_approx_ftz(x1) : 0.f;
            l2 = f32x2_add(l2, f32x2_pack(p0, p1));
            pk[c2] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int c2 = 0; c2 < 16; ++c2) pk[c2] = 0u;
        }
        tmem_st_16cols(treg + gi * 16, pk);
      }
      float l0, l1;
      f32x2_unpack(l2, l0, l1);
      const float l = l0 + l1;
      // P's stores complete before the MMA reads them
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full(w));

      if (!mbar_wait(o_full(w), use & 1)) {
        if (lane == 0) atomicAdd(err + ERR_TIMEOUT, 1);
        break;
      }
      tc_fence_after();
      uint32_t ov[2][32];
      tmem_ld_32cols(treg + 64, ov[0]);
      tmem_ld_32cols(treg + 96, ov[1]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_free(w));   // the region may take the next head's S
      if (len > 0) {
        const float inv = 1.0f / l;
        uint4* dst = reinterpret_cast<uint4*>(ctx + static_cast<size_t>(r) * H + (h0 + j) * kTcDim);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint32_t wv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            wv[e] = pack_bf16x2(__uint_as_float(ov[u >> 2][(u & 3) * 8 + 2 * e]) * inv,
                                __uint_as_float(ov[u >> 2][(u & 3) * 8 + 2 * e + 1]) * inv);
          dst[u] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ---------------------------------------------------------------------------
// Longer rows: head dim 64, sequences of up to 512 tokens.  A CTA takes a
// work item -- 128 consecutive query rows of one sequence -- and a group of
// heads, one head at a time:
//   warp 0, one lane : TMA producer -- Q (the item's 128 rows) and the K
//                      chunks of the sequence (128 key rows each, at most 4)
//                      once the previous head's S is computed; the V chunks
//                      once the previous head's P V is done;
//   warp 1, one lane : tcgen05.mma -- S_c = Q K_c^T for every chunk c into
//                      TMEM columns 128c.., then, chunk by chunk as the
//                      softmax releases P_c, O += P_c V_c (A = P_c from TMEM,
//                      B = V_c through the MN-major descriptor) into columns
//                      64..127, which chunk 0's scores no longer need by then;
//   warps 2..17      : four softmax groups, group g owning key chunk g of
//                      every row (one thread per row and group).  Each group
//                      takes its chunk's maximum; the four maxima meet in
//                      shared memory, so the row's exponentials use the
//                      row's own maximum (the exact softmax, no rescaling);
//                      P_c goes over the scores as bf16, the four partial sums
//                      meet the same way, and group g writes context dims
//                      16g..16g+15 of the row.
// The whole of TMEM (512 columns) holds one head's scores, so heads do not
// overlap in TMEM; the next head's loads overlap this head's softmax.
constexpr int kTclChunks = 4;                          // key chunks: up to 512 keys
constexpr int kTclThreads = 64 + 4 * 128;

struct TclSmem {
  static constexpr int kBox = kTcRows * kTcDim * 2;    // 16 KB
  static constexpr int kQ = 0;
  static constexpr int kK = kBox;                      // K chunk c at kK + c * kBox
  static constexpr int kV = kK + kTclChunks * kBox;    // V chunk c at kV + c * kBox
  static constexpr int kRed = kV + kTclChunks * kBox;  // float [2][4][128]: partial max, sum
  // qk_full v_full s_full o_full p_full[4] tmem_free
  static constexpr int kBarOff = kRed + 2 * 4 * 128 * 4;
  static constexpr int kBars = 9;
  static constexpr int kTmemSlotOff = kBarOff + kBars * 8;
  static constexpr int kBytes = kTmemSlotOff + 16 + 1024;   // + 1024-byte alignment slack
  static_assert(kBytes <= 232448, "fits one CTA's shared memory");
};

__global__ void __launch_bounds__(kTclThreads, 1)
    attn_tcl_kernel(const __grid_constant__ CUtensorMap tm, bf16* __restrict__ ctx,
                    const int32_t* __restrict__ offsets, const int32_t* __restrict__ items,
                    int n, int T, int H, int nh, int hpc, float scale_log2, int causal,
                    int* __restrict__ err, L2PrefetchArgs pf) {
  using SL = TclSmem;
  extern __shared__ uint8_t tc_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(sm);
  const uint32_t bar0 = sbase + SL::kBarOff;
  const uint32_t qk_full = bar0, v_full = bar0 + 8, s_full = bar0 + 16, o_full = bar0 + 24;
  auto p_full = [&](int c) { return bar0 + 32u + 8u * c; };
  const uint32_t tmem_free = bar0 + 64;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SL::kTmemSlotOff);
  float* red_max = reinterpret_cast<float*>(sm + SL::kRed);   // [4][128]
  float* red_sum = red_max + 4 * 128;                          // [4][128]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(qk_full, 1);
    mbar_init(v_full, 1);
    mbar_init(s_full, 1);
    mbar_init(o_full, 1);
    for (int c = 0; c < kTclChunks; ++c) mbar_init(p_full(c), 4);   // the group's four warps
    mbar_init(tmem_free, 16);                                      // every softmax warp
    mbar_init_fence();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();
  l2_prefetch_share(pf);
  pdl_wait();

  // work item: sequence s, query rows [q0, q0 + 128) of it
  const int it = items[blockIdx.x];
  const int s = it >> 2, qt = it & 3;
  const int h0 = blockIdx.y * hpc;
  const bool seq_ok = in_bounds(s >= 0 && s < n);
  const int r0 = seq_ok ? offsets[s] : 0;
  const int L = seq_ok ? offsets[s + 1] - r0 : 0;
  const int q0 = qt * kTcRows;
  // checked build: whole sequences of 1..512 tokens inside the batch, a query
  // tile inside its sequence; a failed item does no work
  const bool item_ok = in_bounds(seq_ok && L >= 1 && L <= kTclChunks * kTcRows && r0 >= 0 &&
                                 r0 + L <= T && q0 < L);
  const int nhl = item_ok ? min(hpc, nh - h0) : 0;
  const int nc = (L + kTcRows - 1) / kTcRows;                // key chunks of this sequence
  // causal: a query tile sees keys up to its last row only
  const int kend_tile = causal ? min(L, q0 + kTcRows) : L;
  const int nc_used = (kend_tile + kTcRows - 1) / kTcRows;

  if (warp == 0) {
    // ---- TMA producer ----
    if (lane == 0) {
      int nqk = 0, nv = 0;
      for (int j = 0; j < nhl; ++j) {
        const int col = (h0 + j) * kTcDim;
        if (j > 0 && !mbar_wait(s_full, (j - 1) & 1)) {        // Q and K of head j-1 consumed
          atomicAdd(err + ERR_TIMEOUT, 1);
          break;
        }
        mbar_arrive_expect_tx(qk_full, (1 + nc_used) * SL::kBox);
        tma_load_2d(sbase + SL::kQ, &tm, col, r0 + q0, qk_full);
        for (int c = 0; c < nc_used; ++c)
          tma_load_2d(sbase + SL::kK + c * SL::kBox, &tm, H + col, r0 + c * kTcRows, qk_full);
        ++nqk;
        if (j > 0 && !mbar_wait(o_full, (j - 1) & 1)) {        // V of head j-1 consumed
          atomicAdd(err + ERR_TIMEOUT, 1);
          break;
        }
        mbar_arrive_expect_tx(v_full, nc_used * SL::kBox);
        for (int c = 0; c < nc_used; ++c)
          tma_load_2d(sbase + SL::kV + c * SL::kBox, &tm, 2 * H + col, r0 + c * kTcRows, v_full);
        ++nv;
      }
      // no copy into this CTA's shared memory may be in flight when it exits
      bool drained = true;
      if (nqk > 0) drained = mbar_wait(qk_full, (nqk - 1) & 1);
      if (drained && nv > 0) mbar_wait(v_full, (nv - 1) & 1);
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTcRows, kTcRows);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kTcRows, kTcDim) | (1u << 16);   // B MN-major
      int js = 0, jo = 0;
      for (int j = 0; j < nhl; ++j) {
        if (!mbar_wait(qk_full, j & 1) || (j > 0 && !mbar_wait(tmem_free, (j - 1) & 1))) {
          atomicAdd(err + ERR_TIMEOUT, 1);
          break;
        }
        tc_fence_after();
        const uint64_t qd = smem_desc_k_sw128(sbase + SL::kQ);
        for (int c = 0; c < nc_used; ++c) {
          const uint64_t kd = smem_desc_k_sw128(sbase + SL::kK + c * SL::kBox);
          const uint32_t d = tmem + static_cast<uint32_t>(c * kTcRows);
#pragma unroll
          for (int ks = 0; ks < kTcDim / 16; ++ks)
            mma_bf16_ss(d, qd + 2ull * ks, kd + 2ull * ks, idesc_s, ks > 0);
        }
        tc_commit<1>(s_full);
        ++js;
        bool ok = mbar_wait(v_full, j & 1);
        for (int c = 0; c < nc_used && ok; ++c) {
          if (!mbar_wait(p_full(c), j & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // 16-key steps holding a key some row of the tile admits
          const int nk16 = min((kend_tile - c * kTcRows + 15) / 16, kTcRows / 16);
          const uint32_t v = sbase + SL::kV + c * SL::kBox;
          const uint32_t pc = tmem + static_cast<uint32_t>(c * kTcRows);
          for (int kb = 0; kb < nk16; ++kb)
            mma_bf16_ts(tmem + kTcDim, pc + kb * 8, smem_desc_mn_sw128(v + kb * 16 * 128), idesc_o,
                        c > 0 || kb > 0);
        }
        if (!ok) {
          atomicAdd(err + ERR_TIMEOUT, 1);
          break;
        }
        tc_commit<1>(o_full);
        ++jo;
      }
      // TMEM is freed after the last MMAs have completed (bounded waits)
      bool drained = true;
      if (js > 0) drained = mbar_wait(s_full, (js - 1) & 1);
      if (drained && jo > 0) mbar_wait(o_full, (jo - 1) & 1);
    }
  } else {
    // ---- softmax groups: group g = key chunk g, one tile row per thread ----
    const int g = (warp - 2) >> 2;
    const int qtr = warp & 3;                   // TMEM lane quarter of this warp
    const int i = qtr * 32 + lane;              // tile row = TMEM lane
    const bool row_ok = q0 + i < L;
    // keys [0, kend) of the sequence; those of chunk g as chunk columns [0, klen)
    const int kend = !row_ok ? 0 : (causal ? q0 + i + 1 : L);
    const int klen = max(0, min(kend - g * kTcRows, kTcRows));
    // 32-column groups of chunk g that some row of this warp admits
    const int wlen = __reduce_max_sync(0xffffffffu, klen);
    bool need[4];
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) need[gi] = gi * 32 < wlen;
    const bool active = g < nc_used;
    const uint32_t treg = tmem + (static_cast<uint32_t>(qtr * 32) << 16) + g * kTcRows;
    const int r = r0 + q0 + i;

    for (int j = 0; j < nhl; ++j) {
      int klen_h;
      asm volatile("mov.b32 %0, %1;" : "=r"(klen_h) : "r"(klen));
      const bool s_ok = mbar_wait(s_full, j & 1);
      if (!s_ok && lane == 0) atomicAdd(err + ERR_TIMEOUT, 1);
      tc_fence_after();
      uint32_t vm[4];
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) vm[gi] = low_bits(klen_h - 32 * gi);
      float m = -INFINITY;
      // groups that every row of the warp admits in full (most of a long
      // sequence) take no per-column mask
      bool full[4];
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) full[gi] = __all_sync(0xffffffffu, vm[gi] == 0xffffffffu);
      if (active && s_ok) {
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) {
          if (!need[gi]) continue;
          uint32_t sv[32];
          tmem_ld_32cols(treg + gi * 32, sv);
          tmem_wait_ld();
          if (full[gi]) {
#pragma unroll
            for (int c = 0; c < 32; ++c) m = fmaxf(m, __uint_as_float(sv[c]));
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (vm[gi] & (1u << c)) m = fmaxf(m, __uint_as_float(sv[c]));
          }
        }
      }
      red_max[g * 128 + i] = m;
      if (!softmax_bar_and(s_ok)) break;          // the softmax warps, all or none
      float mrow = red_max[i];
#pragma unroll
      for (int gg = 1; gg < kTclChunks; ++gg) mrow = fmaxf(mrow, red_max[gg * 128 + i]);
      const float msc = kend > 0 ? mrow * scale_log2 : 0.f;
      // P = exp2(s * scale_log2 - max * scale_log2) on the row's keys of
      // this chunk, 0 elsewhere, written over the scores as bf16 pairs (keys
      // 32gi.. to columns 16gi.., already read); the sum in fp32 before P is
      // rounded to bf16
      const uint64_t sc2 = f32x2_splat(scale_log2), nm2 = f32x2_splat(-msc);
      uint64_t l2 = 0ull;
      if (active) {
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) {
          uint32_t pk[16];
          if (need[gi]) {
            uint32_t sv[32];
            tmem_ld_32cols(treg + gi * 32, sv);
            tmem_wait_ld();
            if (full[gi]) {
#pragma unroll
              for (int c2 = 0; c2 < 16; ++c2) {
                float x0, x1;
                f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(sv[2 * c2]),
                                                  __uint_as_float(sv[2 * c2 + 1])),
                                       sc2, nm2),
                             x0, x1);
                const float p0 = ex2_approx_ftz(x0), p1 = ex2_approx_ftz(x1);
                l2 = f32x2_add(l2, f32x2_pack(p0, p1));
                pk[c2] = pack_bf16x2(p0, p1);
              }
            } else {
#pragma unroll
              for (int c2 = 0; c2 < 16; ++c2) {
                const bool in0 = (vm[gi] >> (2 * c2)) & 1u, in1 = (vm[gi] >> (2 * c2 + 1)) & 1u;
                float x0, x1;
                f32x2_unpack(f32x2_fma(f32x2_pack(__uint_as_float(sv[2 * c2]),
                                                  __uint_as_float(sv[2 * c2 + 1])),
                                       sc2, nm2),
                             x0, x1);
                const float p0 = in0 ? ex2_approx_ftz(x0) : 0.f;
                const float p1 = in1 ? ex2_approx_ftz(x1) : 0.f;
                l2 = f32x2_add(l2, f32x2_pack(p0, p1));
                pk[c2] = pack_bf16x2(p0, p1);
              }
            }
          } else {
#pragma unroll
            for (int c2 = 0; c2 < 16; ++c2) pk[c2] = 0u;
          }
          tmem_st_16cols(treg + gi * 16, pk);
        }
        // P's stores complete before the MMA reads them
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(g));
      }
      float l0, l1;
      f32x2_unpack(l2, l0, l1);
      red_sum[g * 128 + i] = l0 + l1;
      const bool o_ok = mbar_wait(o_full, j & 1);
      if (!o_ok && lane == 0) atomicAdd(err + ERR_TIMEOUT, 1);
      if (!softmax_bar_and(o_ok)) break;
      tc_fence_after();
      float l = red_sum[i];
#pragma unroll
      for (int gg = 1; gg < kTclChunks; ++gg) l += red_sum[gg * 128 + i];
      // context dims 16g..16g+15 of the row: O columns 64 + 16g..
      uint32_t ov[16];
      tmem_ld_16cols(tmem + (static_cast<uint32_t>(qtr * 32) << 16) + kTcDim + 16 * g, ov);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_free);   // TMEM may take the next head's S
      if (kend > 0) {
        const float inv = 1.0f / l;
        uint4* dst = reinterpret_cast<uint4*>(ctx + static_cast<size_t>(r) * H + (h0 + j) * kTcDim +
                                              16 * g);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          uint32_t wv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            wv[e] = pack_bf16x2(__uint_as_float(ov[8 * u + 2 * e]) * inv,
                                __uint_as_float(ov[8 * u + 2 * e + 1]) * inv);
          dst[u] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

}  // namespace

int32_t attn_tc_tiles(const int32_t* offsets, int32_t n, int32_t* tiles) {
  int32_t nt = 0;
  tiles[0] = 0;
  int32_t start = offsets[0];
  for (int32_t i = 0; i < n; ++i) {
    if (offsets[i + 1] - start > kTcRows) {   // sequence i opens a new tile
      tiles[++nt] = i;
      start = offsets[i];
    }
  }
  tiles[++nt] = n;
  return nt;
}

cudaError_t attn_tc_launch(const void* qkv, void* ctx, const int32_t* offsets,
                           const int32_t* tiles, int n_tiles, int n, int T, int nh, int causal,
                           int* err, int num_sms, cudaStream_t st, const L2Prefetch& pf) {
  using SL = TcSmem;
  if (n_tiles < 1 || T < 1) return cudaSuccess;
  const int H = nh * kTcDim;
  CUtensorMap tm;
  const char* why = "";
  // exactly T rows: rows past the batch read as zeros
  if (!make_tmap_bf16(&tm, qkv, static_cast<uint64_t>(T), static_cast<uint64_t>(3 * H), kTcRows,
                      &why))
    return cudaErrorInvalidValue;
  static const cudaError_t attr_err =
      cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SL::kBytes);
  if (attr_err != cudaSuccess) return attr_err;
  // one CTA per SM: all heads of a tile in one CTA (their loads and MMAs
  // pipeline across heads) unless that leaves SMs without a tile
  const int groups = std::min(nh, std::max(1, (num_sms + n_tiles - 1) / n_tiles));
  const int hpc = (nh + groups - 1) / groups;
  dim3 grid(n_tiles, (nh + hpc - 1) / hpc);
  L2PrefetchArgs pa;
  for (int k = 0; k < 2; ++k) {
    pa.ptr[k] = pf.ptr[k];
    pa.bytes[k] = pf.bytes[k];
  }
  const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(kTcDim));
  launch_k(attn_tc_kernel, grid, dim3(kTcThreads), SL::kBytes, st, tm, static_cast<bf16*>(ctx), offsets,
           tiles, n, T, H, nh, hpc, scale_log2, causal, err, pa);
  return cudaGetLastError();
}

int32_t attn_tcl_items(const int32_t* offsets, int32_t n, int32_t causal, int32_t* items) {
  // (sequence, query tile) pairs, those with the most key chunks first so that
  // the grid's last CTAs are short ones
  int32_t count[kTclChunks + 1] = {0};
  auto chunks = [&](int32_t i, int32_t q) {
    const int32_t L = offsets[i + 1] - offsets[i];
    const int32_t kend = causal ? std::min(L, (q + 1) * kTcRows) : L;
    return (kend + kTcRows - 1) / kTcRows;
  };
  for (int32_t i = 0; i < n; ++i)
    for (int32_t q = 0; q * kTcRows < offsets[i + 1] - offsets[i]; ++q) ++count[chunks(i, q)];
  int32_t start[kTclChunks + 1];
  int32_t k = 0;
  for (int32_t c = kTclChunks; c >= 1; --c) {
    start[c] = k;
    k += count[c];
  }
  for (int32_t i = 0; i < n; ++i)
    for (int32_t q = 0; q * kTcRows < offsets[i + 1] - offsets[i]; ++q)
      items[start[chunks(i, q)]++] = (i << 2) | q;
  return k;
}

cudaError_t attn_tcl_launch(const void* qkv, void* ctx, const int32_t* offsets,
                            const int32_t* items, int n_items, int n, int T, int nh, int causal,
                            int* err, int num_sms, cudaStream_t st, const L2Prefetch& pf) {
  using SL = TclSmem;
  if (n_items < 1 || T < 1) return cudaSuccess;
  const int H = nh * kTcDim;
  CUtensorMap tm;
  const char* why = "";
  // exactly T rows: rows past the batch read as zeros
  if (!make_tmap_bf16(&tm, qkv, static_cast<uint64_t>(T), static_cast<uint64_t>(3 * H), kTcRows,
                      &why))
    return cudaErrorInvalidValue;
  static const cudaError_t attr_err =
      cudaFuncSetAttribute(attn_tcl_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SL::kBytes);
  if (attr_err != cudaSuccess) return attr_err;
  // one CTA per SM: all heads of an item in one CTA unless that leaves SMs idle
  const int groups = std::min(nh, std::max(1, (num_sms + n_items - 1) / n_items));
  const int hpc = (nh + groups - 1) / groups;
  dim3 grid(n_items, (nh + hpc - 1) / hpc);
  L2PrefetchArgs pa;
  for (int k = 0; k < 2; ++k) {
    pa.ptr[k] = pf.ptr[k];
    pa.bytes[k] = pf.bytes[k];
  }
  const float scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(kTcDim));
  launch_k(attn_tcl_kernel, grid, dim3(kTclThreads), SL::kBytes, st, tm, static_cast<bf16*>(ctx),
           offsets, items, n, T, H, nh, hpc, scale_log2, causal, err, pa);
  return cudaGetLastError();
}

cudaError_t bounds_errors_attention_tc(int32_t* out, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_bounds_attention_tc, sizeof(int32_t));
  if (e == cudaSuccess && reset) {
    const int32_t zero = 0;
    e = cudaMemcpyToSymbol(g_bounds_attention_tc, &zero, sizeof(int32_t));
  }
  return e;
}

}  // namespace rmk
