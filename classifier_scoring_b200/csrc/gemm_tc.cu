// Y[M][N] = act(X[M][K] . W[N][K]^T + bias) on the 5th-generation tensor
// cores: the QKV, attention-output and FFN projections of the scorer (the
// "BLAS routines" of the TurboTransformers abstract, on tensor cores as its
// proposed-method section does; here bf16 in, fp32 accumulation).  With an
// fp32 accumulation target the tile is added to Y instead (Y += X.W^T + bias),
// which folds a residual add into the projection that produces its addend.
//
// Persistent, warp-specialised kernel: one CTA per SM (CG = 1) or one CTA pair
// per two SMs (CG = 2) walks the (128*CG) x BN output tiles t = unit,
// unit + units, ...  Tiles run N fastest when the activations (A) are at least
// as large as the weights (B): the CTAs of one wave then share a few A row
// panels, so each panel leaves DRAM once while B stays in L2; otherwise M
// fastest.  With CG = 2 the pair is a cluster of two CTAs and the MMA is
// tcgen05.mma.cta_group::2 (M = 256): each CTA loads its own 128 rows of A and
// half of the BN rows of B, the leader CTA issues the MMAs for both, and each
// CTA's TMEM receives its own 128 rows of the accumulator.  Per SM this moves
// half of B through shared memory.  No load uses multicast.  Warps:
//   warp 0, one lane : TMA producer -- K-major 128x64 (A) and BNx64 (B) bf16
//                      boxes, 128-byte swizzle, into a STAGES-deep smem ring
//                      that runs on across tile boundaries;
//   warp 1, one lane : issues tcgen05.mma (M=128*CG, N=BN, K=16) into one of
//                      two TMEM accumulators, tcgen05.commit frees each stage
//                      and marks the accumulator full;
//   warps 2..        : epilogue (four warps, or sixteen when the epilogue applies
//                      GELU) -- tcgen05.ld (warp w reads TMEM lanes
//                      32*(w%4)..+31 = tile rows), + bias, optional GELU, into
//                      swizzled 32 x 32 boxes in shared memory that one lane
//                      writes out with bulk tensor stores (TMA), or, when
//                      accumulating into fp32, row-contiguous boxes that every
//                      lane adds to its row of Y with a bulk reduction; then release
//                      the accumulator.  The epilogue of tile i overlaps the
//                      mainloop of tile i+1.
// Every mbarrier wait is bounded (about 2 s of %globaltimer); a wait that
// gives up counts into err[ERR_TIMEOUT] and the role leaves its loop; the CTA
// then waits (bounded) for its own copies, frees its TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace rmk {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;                      // 64 bf16 = one 128-byte swizzle row

// Epilogue warps: eight (two per TMEM lane quarter, taking the column rounds
// in turn) for a plain epilogue, sixteen when it applies GELU, whose
// arithmetic otherwise outlasts a short mainloop (B200, 27.8k tokens: the
// QKV projection in a power-capped loop 97.9 us with eight against 104.3 us
// with four; FFN1 with L2 flushed 122.9 us with sixteen against 128.9 us with
// eight).
constexpr int epi_warps(int act) { return act != 0 ? 16 : 8; }
constexpr int gemm_threads(int act) { return 64 + 32 * epi_warps(act); }
// Time per column of a CTA-pair tile relative to a single-CTA tile, and the
// smallest products for which pairs are considered (measured on B200 with
// N-fastest tile order: pairs won by 12-16% on the M = 26112 projections and
// by up to 3.5% at M = 13556 with N >= 2304, and lost at M <= 10048 or
// N = 768).
constexpr double kPairColumnCost = 0.8;
constexpr int kPairMinM = 12288;
constexpr int kPairMinN = 2048;

__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y,
                                                 uint32_t leader_bar) {
  // both CTAs of the pair complete their bytes on the leader's barrier
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(leader_bar)
      : "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar)
               : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
constexpr uint32_t tmem_cols_for(int bn) {
  // two accumulators of bn fp32 columns, rounded up to a power of two >= 32
  return 2 * bn <= 32 ? 32 : (2 * bn <= 64 ? 64 : (2 * bn <= 128 ? 128 : (2 * bn <= 256 ? 256 : 512)));
}

template <int BN, int CG, int EW, int ESZ>
struct GemmSmem {
  static constexpr int kA = BM * BK * 2;
  static constexpr int kB = (BN / CG) * BK * 2;   // this CTA's share of the B tile
  static constexpr int kStage = kA + kB;          // multiple of 1024 for BN/CG % 8 == 0
  // epilogue: per warp, kEpiBufs staging boxes of 32 rows x 32 output columns
  // (64-byte rows of bf16 or 128-byte rows of fp32) in the swizzled layout of
  // the output tensor map, written out by bulk tensor stores
  static constexpr int kRowBytes = 32 * ESZ;
  static constexpr int kBoxBytes = 32 * kRowBytes;
  // barriers (full[S], empty[S], accf[2], acce[2], S <= 8), TMEM slot, and
  // the slack that aligns the dynamic shared memory to 1024 bytes
  static constexpr int kTail = (2 * 8 + 4) * 8 + 16 + 1024;
  // as many 64-deep K stages as fit beside the rest (227 KB per CTA), at most
  // 8; two staging boxes per warp unless that costs a stage
  static constexpr int stages_with(int bufs) {
    return (232448 - EW * bufs * kBoxBytes - kTail) / kStage < 8
               ? (232448 - EW * bufs * kBoxBytes - kTail) / kStage
               : 8;
  }
  static constexpr int kEpiBufs = stages_with(2) >= stages_with(1) ? 2 : 1;
  static constexpr int kStages = stages_with(kEpiBufs);
  static constexpr int kEpiOff = kStages * kStage;   // 1024-byte aligned: the boxes are too
  static constexpr int kBarOff = kEpiOff + EW * kEpiBufs * kBoxBytes;
  static constexpr int kSlotOff = kBarOff + (2 * kStages + 4) * 8;
  static constexpr int kBytes = kSlotOff + 16 + 1024;   // + alignment slack
  static_assert(kStages >= 3, "at least three stages");
  static_assert(kBytes <= 232448, "fits one CTA's shared memory");
};

template <int BN, int CG, int ACT, bool OUT_F32>
__global__ void __launch_bounds__(gemm_threads(ACT), 1)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmB2,
                        const __grid_constant__ CUtensorMap tmY, int M, int N, int K,
                        const float* __restrict__ bias, int* __restrict__ err, int n_fastest,
                        void* __restrict__ yacc, int full, int split) {
  constexpr int EW = epi_warps(ACT);
  using L = GemmSmem<BN, CG, EW, OUT_F32 ? 4 : 2>;
  constexpr int S = L::kStages;
  constexpr uint32_t kTmemCols = tmem_cols_for(BN);
  static_assert(L::kStage % 1024 == 0, "stage size keeps the 1024-byte swizzle alignment");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_rank() : 0u;   // 0 = leader of the pair
  const int unit = blockIdx.x / CG, units = gridDim.x / CG;
  const int tiles_m = (M + BM * CG - 1) / (BM * CG);
  const int tiles_n = (N + BN - 1) / BN;
  const int tiles = tiles_m * tiles_n;
  // tile t -> (row block, column block).  N fastest: the CTAs running at the
  // same time share a few A row panels and sweep all of B, so each A panel
  // leaves DRAM once (the activations outgrow L2 well before the weights do);
  // M fastest: they share a few B column panels.
  auto m_blk = [&](int t) { return n_fastest ? t / tiles_n : t % tiles_m; };
  auto n_blk = [&](int t) { return n_fastest ? t % tiles_n : t / tiles_m; };
  // Work items: tiles 0..full-1 whole, then each remaining tile (the last,
  // partial round of the persistent grid) as `split` slices of BN/split
  // columns, so that SMs that would idle in that round take a slice each
  // (1-CTA tiles only; a slice loads its own narrower box of B, tmB2).  Not
  // with the tanh GELU, whose epilogue has no registers to spare.
  if (ACT == 2) {
    split = 1;
    full = tiles;
  }
  const int cols_split = BN / split;
  const int works = full + (tiles - full) * split;
  auto work_tile = [&](int w, int& t, int& c0) {
    if (w < full) {
      t = w;
      c0 = 0;
      return BN;
    }
    t = full + (w - full) / split;
    c0 = ((w - full) % split) * cols_split;
    return cols_split;
  };
  const int nk = (K + BK - 1) / BK;
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + S),
                 accf0 = smem_u32(bars + 2 * S), acce0 = smem_u32(bars + 2 * S + 2);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf0 + 8 * a, 1);
      mbar_init(acce0 + 8 * a, EW * CG);   // one arrival per epilogue warp of the pair
    }
    mbar_init_fence();
  }
  if (warp == 0) {
    if (CG == 1) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(kTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(kTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
  }
  tc_fence_before();
  if (CG == 2) cluster_sync_all();   // both CTAs' barriers exist before any remote signal
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the prologue above overlaps the previous kernel; global memory waits for it
  pdl_launch_dependents();
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      // ---- TMA producer ----
      int it = 0;
      bool ok = true;
      for (int w = unit; w < works && ok; w += units) {
        int t, c0;
        const int cols = work_tile(w, t, c0);
        const int m0 = m_blk(t) * BM * CG + static_cast<int>(rank) * BM;
        const int nb0 = n_blk(t) * BN + c0 + static_cast<int>(rank) * (BN / CG);
        const bool whole = cols == BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (it >= S && !mbar_wait(empty0 + 8 * s, ph ^ 1)) {
            atomicAdd(err + ERR_TIMEOUT, 1);
            ok = false;
            break;
          }
          const uint32_t dA = smem_u32(smem + s * L::kStage), dB = dA + L::kA;
          if (CG == 1) {
            mbar_arrive_expect_tx(full0 + 8 * s, whole ? L::kStage : L::kA + cols * BK * 2);
            tma_load_2d(dA, &tmA, kb * BK, m0, full0 + 8 * s);
            tma_load_2d(dB, whole ? &tmB : &tmB2, kb * BK, nb0, full0 + 8 * s);
          } else {
            // the leader expects the bytes of both CTAs on its own barrier
            if (rank == 0) mbar_arrive_expect_tx(full0 + 8 * s, 2 * L::kStage);
            const uint32_t lbar = map_to_rank(full0 + 8 * s, 0);
            tma_load_2d_pair(dA, &tmA, kb * BK, m0, lbar);
            tma_load_2d_pair(dB, &tmB, kb * BK, nb0, lbar);
          }
        }
      }
      // Before shared memory is released: the copies in flight have landed
      // (the leader's full barriers count both CTAs' bytes) and the MMA
      // completions that arrive on this CTA's empty barriers (from the
      // leader, with a pair) have arrived.  Bounded; gives up at the first
      // wait that runs out.
      bool drained = true;
      if (rank == 0)
        for (int j = it - 1; drained && j >= 0 && j >= it - S; --j)
          drained = mbar_wait(full0 + 8 * (j % S), (j / S) & 1);
      if (ok)
        for (int j = it - 1; drained && j >= 0 && j >= it - S; --j)
          drained = mbar_wait(empty0 + 8 * (j % S), (j / S) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---- MMA issuer (the leader issues for the pair) ----
      constexpr uint32_t idesc_whole = idesc_bf16_f32(BM * CG, BN);
      const uint32_t idesc_slice = idesc_bf16_f32(BM * CG, cols_split);
      int it = 0, local = 0;
      bool ok = true;
      for (int w = unit; w < works && ok; w += units, ++local) {
        int t, c0;
        const uint32_t idesc = work_tile(w, t, c0) == BN ? idesc_whole : idesc_slice;
        const int acc = local & 1, use = local >> 1;
        if (use > 0 && !mbar_wait(acce0 + 8 * acc, (use - 1) & 1)) {
          atomicAdd(err + ERR_TIMEOUT, 1);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(acc) * (kTmemCols / 2);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!mbar_wait(full0 + 8 * s, ph)) {
            atomicAdd(err + ERR_TIMEOUT, 1);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = smem_desc_k_sw128(smem_u32(smem + s * L::kStage));
          const uint64_t bd = smem_desc_k_sw128(smem_u32(smem + s * L::kStage + L::kA));
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // advance 16 elements = 32 bytes along K inside the swizzle atom
            const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
            if (CG == 1)
              asm volatile(
                  "{\n\t.reg .pred p;\n\t"
                  "setp.ne.b32 p, %4, 0;\n\t"
                  "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
                  "l"(ad + 2ull * k), "l"(bd + 2ull * k), "r"(idesc), "r"(accum)
                  : "memory");
            else
              asm volatile(
                  "{\n\t.reg .pred p;\n\t"
                  "setp.ne.b32 p, %4, 0;\n\t"
                  "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
                  "l"(ad + 2ull * k), "l"(bd + 2ull * k), "r"(idesc), "r"(accum)
                  : "memory");
          }
          // frees the stage (in both CTAs of a pair) once these MMAs are done
          tc_commit<CG>(empty0 + 8 * s);
          if (CG == 2) tc_commit<CG>(map_to_rank(empty0 + 8 * s, 1));
        }
        tc_commit<CG>(accf0 + 8 * acc);    // the accumulator is complete
        if (CG == 2) tc_commit<CG>(map_to_rank(accf0 + 8 * acc, 1));
      }
    }
  } else {
    // ---- epilogue: TMEM -> registers -> bias/GELU -> swizzled smem box -> TMA store ----
    // Each thread owns one tile row (its TMEM lane).  A round takes 32
    // columns of that row, adds the bias (and GELU), writes the warp's 32 x 32
    // box into one of its staging buffers and lane 0 stores the box with one
    // bulk tensor copy; rows and columns outside Y are clipped by the copy.
    // With more than four warps the warps of a lane quarter take the rounds
    // in turn.
    constexpr int NB = L::kEpiBufs;
    constexpr int NH = EW / 4;                   // warps per TMEM lane quarter
    const int ew = warp - 2;
    const int q = warp & 3;                      // TMEM lane quarter of this warp
    const int h0 = ew >> 2;                      // this warp's first round
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    uint8_t* stg0 = smem + L::kEpiOff + ew * NB * L::kBoxBytes;
    int nst = 0;                                 // boxes this warp has stored
    int local = 0;
    for (int w = unit; w < works; w += units, ++local) {
      int t, c0;
      const int cols = work_tile(w, t, c0);
      const int acc = local & 1, use = local >> 1;
      const bool ready = mbar_wait(accf0 + 8 * acc, use & 1);
      if (!__all_sync(0xffffffffu, ready)) {
        if (lane == 0) atomicAdd(err + ERR_TIMEOUT, 1);
        break;
      }
      tc_fence_after();
      const int m0 = m_blk(t) * BM * CG + static_cast<int>(rank) * BM;
      const int n0 = n_blk(t) * BN + c0;
      const int row0 = m0 + q * 32;
      const uint32_t base = tmem + lane_base + static_cast<uint32_t>(acc) * (kTmemCols / 2);
      if (row0 < M) {                            // uniform across the warp
        // TMEM loads run one round ahead: round c+1's columns are in flight
        // while round c's values go through the bias, GELU and the store
        int c = h0 * 32;
        bool have = c < cols && n0 + c < N;      // uniform across the warp
        uint32_t r[32];
        if (have) tmem_ld_32cols(base + c, r);
        while (have) {
          // the bias of these columns: the same address in every lane (L1)
          float4 b4[8];
#pragma unroll
          for (int g = 0; g < 8; ++g)
            b4[g] = (bias != nullptr && n0 + c + 4 * g < N)
                        ? __ldg(reinterpret_cast<const float4*>(bias + n0 + c + 4 * g))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
          tmem_wait_ld();
          uint64_t p2[16];                       // bias added, two columns per register
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            p2[2 * g] = f32x2_add(f32x2_pack(__uint_as_float(r[4 * g]), __uint_as_float(r[4 * g + 1])),
                                  f32x2_pack(b4[g].x, b4[g].y));
            p2[2 * g + 1] = f32x2_add(
                f32x2_pack(__uint_as_float(r[4 * g + 2]), __uint_as_float(r[4 * g + 3])),
                f32x2_pack(b4[g].z, b4[g].w));
          }
          const int cn = c + NH * 32;
          const bool next = cn < cols && n0 + cn < N;
          if (next) tmem_ld_32cols(base + cn, r);
          float v[32];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            if (ACT == 1) p2[k] = gelu_erf_fast_x2(p2[k]);
            f32x2_unpack(p2[k], v[2 * k], v[2 * k + 1]);
            if (ACT == 2) {
              v[2 * k] = gelu_tanh(v[2 * k]);
              v[2 * k + 1] = gelu_tanh(v[2 * k + 1]);
            }
          }
          // this buffer's previous box has been read out by its store
          const int buf = NB == 1 ? 0 : (nst & 1);
          if (nst >= NB) {
            bulk_wait_group_read<NB - 1>();      // no-op in lanes without copies in flight
            __syncwarp();
          }
          uint8_t* box = stg0 + buf * L::kBoxBytes;
          if (ACT == 0 && OUT_F32 && yacc != nullptr) {
            // Y += the tile: each lane adds its own row's 32 columns with one
            // bulk reduction in L2 (fp32 adds: the sum is rounded once, as a
            // separate addition would round it), so the row stays contiguous
            // (no swizzle).  The
            // lane writes its 16-byte chunks in an order rotated by its
            // position, which spreads each quarter warp over all banks.
            constexpr int NCH = 8;
            uint4 ch[NCH];
#pragma unroll
            for (int j = 0; j < NCH; ++j)
              ch[j] = make_uint4(__float_as_uint(v[4 * j]), __float_as_uint(v[4 * j + 1]),
                                 __float_as_uint(v[4 * j + 2]), __float_as_uint(v[4 * j + 3]));
            const int key = lane & 7;
            // rotate left by key (register indices stay compile-time)
#pragma unroll
            for (int bit = 1; bit < NCH; bit <<= 1) {
              const bool rot = (key & bit) != 0;
              uint4 t[NCH];
#pragma unroll
              for (int j = 0; j < NCH; ++j) t[j] = rot ? ch[(j + bit) % NCH] : ch[j];
#pragma unroll
              for (int j = 0; j < NCH; ++j) ch[j] = t[j];
            }
            uint8_t* row = box + lane * (NCH * 16);
#pragma unroll
            for (int j = 0; j < NCH; ++j)
              *reinterpret_cast<uint4*>(row + (((j + key) % NCH) << 4)) = ch[j];
            fence_proxy_async_smem();
            const int grow = row0 + lane, gcol = n0 + c;
            if (grow < M) {
              const int cols = N - gcol < 32 ? N - gcol : 32;   // a multiple of 8
              float* dst = static_cast<float*>(yacc) + static_cast<size_t>(grow) * N + gcol;
              bulk_reduce_add_f32(dst, smem_u32(row), cols * 4);
            }
            bulk_commit_group();
          } else {
            if (OUT_F32) {
              // 128-byte rows, 128-byte swizzle: 16-byte chunk j of row r at j ^ (r % 8)
#pragma unroll
              for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4*>(box + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                    make_uint4(__float_as_uint(v[4 * j]), __float_as_uint(v[4 * j + 1]),
                               __float_as_uint(v[4 * j + 2]), __float_as_uint(v[4 * j + 3]));
            } else {
              // 64-byte rows, 64-byte swizzle: 16-byte chunk j of row r at j ^ ((r / 2) % 4)
#pragma unroll
              for (int j = 0; j < 4; ++j)
                *reinterpret_cast<uint4*>(box + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
                    make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]),
                               pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                               pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                               pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
            }
            // the box's generic-proxy writes before the async-proxy store reads them
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmY, smem_u32(box), n0 + c, row0);
              bulk_commit_group();
            }
          }
          ++nst;
          c = cn;
          have = next;
        }
      }
      tc_fence_before();
      __syncwarp();
      // accumulator free for tile local+2 (the leader's barrier counts both CTAs)
      if (lane == 0) {
        if (CG == 1 || rank == 0) mbar_arrive(acce0 + 8 * acc);
        else mbar_arrive_cluster(map_to_rank(acce0 + 8 * acc, 0));
      }
    }
    // every store of this warp has finished before the CTA's shared memory goes
    bulk_wait_group<0>();
  }
  __syncwarp();
  tc_fence_before();
  if (CG == 2) cluster_sync_all();   // no remote signal or copy can outlive either CTA
  else __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    if (CG == 1)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(kTmemCols)
                   : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                   "r"(kTmemCols)
                   : "memory");
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <int BN, int CG, int ACT, bool OUT_F32>
cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b_split,
                       const CUtensorMap& y, void* yacc, int M, int N, int K, const float* bias,
                       int* err, int num_sms, cudaStream_t st) {
  using L = GemmSmem<BN, CG, epi_warps(ACT), OUT_F32 ? 4 : 2>;
  auto kern = gemm_bf16_tc_kernel<BN, CG, ACT, OUT_F32>;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(gemm_threads(ACT));
  cfg.dynamicSmemBytes = L::kBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (CG == 2) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 2;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  // Once per instantiation (thread-safe static initialisation): the shared
  // memory attribute, per function, and for pairs the number of clusters
  // that fit at once, per device model; one device model per process.
  struct Setup {
    cudaError_t err;
    int resident_units;
  };
  static const Setup setup = [&]() {
    Setup r{cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes), 0};
    if (r.err == cudaSuccess && CG == 2) {
      // pairs must sit on the two SMs of one cluster slot: ask how many fit at once
      cudaLaunchConfig_t q = cfg;
      q.gridDim = dim3(2 * (num_sms / 2));
      q.attrs = attr;
      q.numAttrs = na;
      r.err = cudaOccupancyMaxActiveClusters(&r.resident_units, kern, &q);
    }
    return r;
  }();
  if (setup.err != cudaSuccess) return setup.err;
  const int tiles = ((M + BM * CG - 1) / (BM * CG)) * ((N + BN - 1) / BN);
  int max_units = num_sms / CG;
  if (CG == 2 && setup.resident_units > 0 && setup.resident_units < max_units)
    max_units = setup.resident_units;
  // the last partial round's tiles as column slices (1-CTA tiles, not with
  // the tanh GELU)
  const int split = CG == 1 && ACT != 2 ? gemm_tail_split(GemmTile{CG, BN}, M, N, num_sms) : 1;
  const int rem = tiles >= max_units ? tiles % max_units : tiles;
  const int full = split > 1 ? tiles - rem : tiles;
  const int works = full + (tiles - full) * split;
  cfg.gridDim = dim3(CG * (works < max_units ? works : max_units));
  if (g_pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  // the activations (A, M rows) are at least as large as the weights (B, N rows)
  const int n_fastest = M >= N ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, a, b, b_split, y, M, N, K, bias, err, n_fastest, yacc,
                            full, split);
}

template <int BN, int CG>
cudaError_t launch_act(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& bs,
                       const CUtensorMap& y, void* yacc, int M, int N, int K, const float* bias,
                       bool out_f32, int act, int* err, int num_sms, cudaStream_t st) {
  if (out_f32) {
    if (act == 1) return launch_one<BN, CG, 1, true>(a, b, bs, y, yacc, M, N, K, bias, err, num_sms, st);
    if (act == 2) return launch_one<BN, CG, 2, true>(a, b, bs, y, yacc, M, N, K, bias, err, num_sms, st);
    return launch_one<BN, CG, 0, true>(a, b, bs, y, yacc, M, N, K, bias, err, num_sms, st);
  }
  if (act == 1) return launch_one<BN, CG, 1, false>(a, b, bs, y, yacc, M, N, K, bias, err, num_sms, st);
  if (act == 2) return launch_one<BN, CG, 2, false>(a, b, bs, y, yacc, M, N, K, bias, err, num_sms, st);
  return launch_one<BN, CG, 0, false>(a, b, bs, y, yacc, M, N, K, bias, err, num_sms, st);
}

}  // namespace

const int kGemmTileWidths[kGemmTileCount] = {64, 96, 128, 160, 192, 224, 256};

GemmTile gemm_pick(int M, int N, int K, int num_sms, int act) {
  // Makespan of the persistent grid: rounds of tiles times the per-SM time of
  // one tile, modelled as proportional to BN plus a fixed part worth about 160
  // columns (pipeline fill, epilogue tail, and the A panel each tile reads
  // whatever its width; fitted to B200 sweeps of the BERT projections).  A CTA pair moves
  // half of the weight tile per SM, so its mainloop runs faster per column,
  // but on B200 it only paid off on large products (M >= kPairMinM rows and
  // N >= kPairMinN columns): on smaller or narrower projections a pair ran
  // slower than one CTA of the same width.
  GemmTile best{1, 256};
  double best_cost = -1;
  auto consider = [&](int cg, int bn, double per_col) {
    const long long tm = (M + 128LL * cg - 1) / (128LL * cg);
    const long long tiles = tm * ((N + bn - 1) / bn);
    const long long units = num_sms / cg;
    const long long rounds = (tiles + units - 1) / units;
    const double cost = static_cast<double>(rounds) * (bn * per_col + 160.0);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = GemmTile{cg, bn};
    }
  };
  for (int i = kGemmTileCount - 1; i >= 0; --i) consider(1, kGemmTileWidths[i], 1.0);
  // With a GELU epilogue and a short K the epilogue, not the mainloop, sets
  // the pace, and single-CTA tiles measured 5-6% faster than pairs there.
  const bool pair_ok = act == 0 || K >= 2048;
  if (num_sms >= 2 && M >= kPairMinM && N >= kPairMinN && pair_ok)
    for (int bn : {256, 192, 128}) consider(2, bn, kPairColumnCost);
  return best;
}

int gemm_tail_split(GemmTile tile, int M, int N, int num_sms) {
  if (tile.cg != 1 || num_sms < 1) return 1;
  const long long tiles = ((M + 127LL) / 128) * ((N + tile.bn - 1LL) / tile.bn);
  const long long rem = tiles >= num_sms ? tiles % num_sms : tiles;
  if (rem == 0) return 1;
  for (int f : {4, 2}) {
    if (tile.bn % f != 0 || rem * f > num_sms) continue;
    for (int i = 0; i < kGemmTileCount; ++i)
      if (kGemmTileWidths[i] == tile.bn / f) return f;
  }
  return 1;
}

cudaError_t gemm_launch(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b_split,
                        const CUtensorMap& y, void* yacc, GemmTile tile, int M, int N, int K,
                        const float* bias, bool out_f32, int act, int* err, int num_sms,
                        cudaStream_t st) {
#define RM_GEMM_TILE(cg, bn)                                                                  \
  case bn:                                                                                    \
    return launch_act<bn, cg>(a, b, b_split, y, yacc, M, N, K, bias, out_f32, act, err, num_sms, \
                              st)
  if (tile.cg == 2) {
    switch (tile.bn) {
      RM_GEMM_TILE(2, 128);
      RM_GEMM_TILE(2, 192);
      RM_GEMM_TILE(2, 256);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (tile.bn) {
    RM_GEMM_TILE(1, 64);
    RM_GEMM_TILE(1, 96);
    RM_GEMM_TILE(1, 128);
    RM_GEMM_TILE(1, 160);
    RM_GEMM_TILE(1, 192);
    RM_GEMM_TILE(1, 224);
    RM_GEMM_TILE(1, 256);
    default: return cudaErrorInvalidValue;
  }
#undef RM_GEMM_TILE
}

// Failure detection without a fault: one thread waits on an mbarrier that
// nothing completes, through the same bounded wait the GEMM's roles use, and
// records whether the wait gave up and how long it took.
__global__ void bounded_wait_selftest_kernel(unsigned long long limit_ns, int* timed_out,
                                             unsigned long long* elapsed_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  const unsigned long long t0 = globaltimer_ns();
  const bool ok = mbar_wait_for(b, 0, limit_ns);   // phase 0 never completes: no arrival
  *elapsed_ns = globaltimer_ns() - t0;
  *timed_out = ok ? 0 : 1;
}

cudaError_t bounded_wait_selftest(unsigned long long limit_ns, int* d_timed_out,
                                  unsigned long long* d_elapsed_ns, cudaStream_t st) {
  bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(limit_ns, d_timed_out, d_elapsed_ns);
  return cudaGetLastError();
}

}  // namespace rmk
