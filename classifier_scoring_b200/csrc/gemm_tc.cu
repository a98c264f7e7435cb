// Y[M][N] = act(X[M][K] . W[N][K]^T + bias) on the 5th-generation tensor
// cores: the QKV, attention-output and FFN projections of the scorer (the
// "BLAS routines" of the TurboTransformers abstract, on tensor cores as its
// proposed-method section does; here bf16 in, fp32 accumulation).
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
//                      32*(w%4)..+31 = tile rows), + bias, optional GELU,
//                      staged through shared memory into whole row segments of
//                      bf16 or fp32, then release the accumulator.  The
//                      epilogue of tile i overlaps the mainloop of tile i+1.
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

// Epilogue warps: four (one per TMEM lane quarter) for a plain epilogue;
// sixteen (four per quarter, taking the column rounds in turn) when the
// epilogue applies GELU, whose arithmetic otherwise outlasts a short mainloop
// (B200, FFN1 of 27.8k tokens: 128.9 us with eight, 122.9 us with sixteen).
constexpr int epi_warps(int act) { return act != 0 ? 16 : 4; }
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
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
template <int CG>
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  if (CG == 1)
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
  else
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile written by TMA
// with the 128-byte swizzle: rows of 128 B, 8-row (1024 B) swizzle atoms.
// Fields: start address >> 4 (bits 0..13), leading byte offset >> 4 = 1
// (unused for swizzled K-major), stride byte offset >> 4 = 1024 >> 4 (bits
// 32..45), descriptor version 1 (bit 46), layout 2 = 128-byte swizzle (61..63).
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) |
         (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16: D fp32 (bits 4..5 = 1), A and B bf16
// (bits 7..9 = 1, 10..12 = 1), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

__device__ __forceinline__ void tmem_ld_32cols(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
      " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_16cols(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

constexpr uint32_t tmem_cols_for(int bn) {
  // two accumulators of bn fp32 columns, rounded up to a power of two >= 32
  return 2 * bn <= 32 ? 32 : (2 * bn <= 64 ? 64 : (2 * bn <= 128 ? 128 : (2 * bn <= 256 ? 256 : 512)));
}

template <int BN, int CG, int EW>
struct GemmSmem {
  static constexpr int kA = BM * BK * 2;
  static constexpr int kB = (BN / CG) * BK * 2;   // this CTA's share of the B tile
  static constexpr int kStage = kA + kB;          // multiple of 1024 for BN/CG % 8 == 0
  // epilogue staging: per epilogue warp 32 rows x one round of output (128 B
  // with four epilogue warps, 64 B with more), row pitch padded by 16 B so
  // that both the row-wise writes and the segment-wise reads spread over the
  // bank groups
  static constexpr int kRoundBytes = EW == 4 ? 128 : 64;
  static constexpr int kStagePitch = kRoundBytes + 16;
  static constexpr int kStageWarpBytes = 32 * kStagePitch;
  // bias of the tile per epilogue warp (no cross-warp barrier): two buffers
  // (one per accumulator) with four warps, one with more
  static constexpr int kBiasFloatsPerWarp = EW == 4 ? 2 * BN : BN;
  static constexpr int kBiasBytes = EW * kBiasFloatsPerWarp * 4;
  // as many 64-deep K stages as fit beside the rest (227 KB per CTA), at most 8
  static constexpr int kFixed = EW * kStageWarpBytes + kBiasBytes + 20 * 8 + 16 + 1024;
  static constexpr int kStagesFit = (232448 - kFixed) / kStage;
  static constexpr int kStages = kStagesFit < 8 ? kStagesFit : 8;
  static constexpr int kEpiOff = kStages * kStage;
  static constexpr int kBiasOff = kEpiOff + EW * kStageWarpBytes;
  static constexpr int kBarOff = kBiasOff + kBiasBytes;   // full[S], empty[S], accf[2], acce[2]
  static constexpr int kSlotOff = kBarOff + (2 * kStages + 4) * 8;
  static constexpr int kBytes = kSlotOff + 16 + 1024;   // + alignment slack
  static_assert(kStages >= 3, "at least three stages");
  static_assert(kBytes <= 232448, "fits one CTA's shared memory");
};

template <int ACT>
__device__ __forceinline__ float epilogue_act(float t) {
  if (ACT == 1) return gelu_erf_fast(t);
  if (ACT == 2) return gelu_tanh(t);
  return t;
}

template <int BN, int CG, int ACT, bool OUT_F32>
__global__ void __launch_bounds__(gemm_threads(ACT), 1)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, int M, int N, int K,
                        const float* __restrict__ bias, void* __restrict__ y,
                        int* __restrict__ err, int n_fastest) {
  constexpr int EW = epi_warps(ACT);
  using L = GemmSmem<BN, CG, EW>;
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
      for (int t = unit; t < tiles && ok; t += units) {
        const int m0 = m_blk(t) * BM * CG + static_cast<int>(rank) * BM;
        const int nb0 = n_blk(t) * BN + static_cast<int>(rank) * (BN / CG);
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
            mbar_arrive_expect_tx(full0 + 8 * s, L::kStage);
            tma_load_2d(dA, &tmA, kb * BK, m0, full0 + 8 * s);
            tma_load_2d(dB, &tmB, kb * BK, nb0, full0 + 8 * s);
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
      constexpr uint32_t idesc = idesc_bf16_f32(BM * CG, BN);
      int it = 0, local = 0;
      bool ok = true;
      for (int t = unit; t < tiles && ok; t += units, ++local) {
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
    // ---- epilogue: TMEM -> registers -> bias/GELU -> smem staging -> global ----
    // Each thread owns one tile row (its TMEM lane).  A round takes
    // kRoundBytes of that row, writes it to the warp's staging rows, then the
    // warp stores whole row segments.  With more than four warps the warps of
    // a lane quarter take the rounds in turn.
    constexpr int ESZ = OUT_F32 ? 4 : 2;
    constexpr int RB = L::kRoundBytes;
    constexpr int CPR = RB / ESZ;                // columns per round
    constexpr int NH = EW / 4;                   // warps per TMEM lane quarter
    const int ew = warp - 2;
    const int q = warp & 3;                      // TMEM lane quarter of this warp
    const int h0 = ew >> 2;                      // this warp's first round
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    uint8_t* stg = smem + L::kEpiOff + ew * L::kStageWarpBytes;
    float* sbias_warp = reinterpret_cast<float*>(smem + L::kBiasOff) + ew * L::kBiasFloatsPerWarp;
    int local = 0;
    for (int t = unit; t < tiles; t += units, ++local) {
      const int acc = local & 1, use = local >> 1;
      // stage this tile's bias while the mainloop still runs (with two
      // buffers, the one for this accumulator was last read two tiles ago;
      // with one, this warp's reads of the previous tile ended before its
      // arrival below)
      float* sbias = sbias_warp + (EW == 4 ? acc * BN : 0);
      {
        const int nb0 = n_blk(t) * BN;
        for (int j = lane; j < BN; j += 32)
          sbias[j] = (bias != nullptr && nb0 + j < N) ? __ldg(bias + nb0 + j) : 0.0f;
        __syncwarp();
      }
      const bool ready = mbar_wait(accf0 + 8 * acc, use & 1);
      if (!__all_sync(0xffffffffu, ready)) {
        if (lane == 0) atomicAdd(err + ERR_TIMEOUT, 1);
        break;
      }
      tc_fence_after();
      const int m0 = m_blk(t) * BM * CG + static_cast<int>(rank) * BM;
      const int n0 = n_blk(t) * BN;
      const int row0 = m0 + q * 32;
      const uint32_t base = tmem + lane_base + static_cast<uint32_t>(acc) * (kTmemCols / 2);
#pragma unroll 1
      for (int c = h0 * CPR; c < BN; c += NH * CPR) {
        if (n0 + c >= N) break;                  // uniform across the warp
        float v[CPR];
        if (CPR >= 32) {
          uint32_t r[32];
#pragma unroll
          for (int h = 0; h < CPR / 32; ++h) {
            tmem_ld_32cols(base + c + 32 * h, r);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[32 * h + j] = __uint_as_float(r[j]);
          }
        } else {
          uint32_t r[16];
          tmem_ld_16cols(base + c, r);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
        }
#pragma unroll
        for (int g = 0; g < CPR / 4; ++g) {
          // c + 4g < BN except in a partial last round, whose columns are not stored
          const float4 b4 = (c + 4 * g < BN) ? *reinterpret_cast<const float4*>(sbias + c + 4 * g)
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
          if (ACT == 1) {
            // bias and GELU two columns per packed instruction
            uint64_t lo = f32x2_add(f32x2_pack(v[4 * g + 0], v[4 * g + 1]), f32x2_pack(b4.x, b4.y));
            uint64_t hi = f32x2_add(f32x2_pack(v[4 * g + 2], v[4 * g + 3]), f32x2_pack(b4.z, b4.w));
            lo = gelu_erf_fast_x2(lo);
            hi = gelu_erf_fast_x2(hi);
            f32x2_unpack(lo, v[4 * g + 0], v[4 * g + 1]);
            f32x2_unpack(hi, v[4 * g + 2], v[4 * g + 3]);
          } else {
            v[4 * g + 0] = epilogue_act<ACT>(v[4 * g + 0] + b4.x);
            v[4 * g + 1] = epilogue_act<ACT>(v[4 * g + 1] + b4.y);
            v[4 * g + 2] = epilogue_act<ACT>(v[4 * g + 2] + b4.z);
            v[4 * g + 3] = epilogue_act<ACT>(v[4 * g + 3] + b4.w);
          }
        }
        __syncwarp();                            // the previous round's reads are done
        uint8_t* my_row = stg + lane * L::kStagePitch;
#pragma unroll
        for (int j = 0; j < RB / 16; ++j) {
          uint4 u;
          if (OUT_F32) {
            u = make_uint4(__float_as_uint(v[4 * j]), __float_as_uint(v[4 * j + 1]),
                           __float_as_uint(v[4 * j + 2]), __float_as_uint(v[4 * j + 3]));
          } else {
            u = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                           pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
          }
          *reinterpret_cast<uint4*>(my_row + 16 * j) = u;
        }
        __syncwarp();
        // RB/16 16-byte chunks per row; a store instruction covers 32/(RB/16)
        // rows (128-byte rows: 4, lanes along the row; 64-byte rows: 8, lanes
        // down the rows, which keeps the 80-byte pitch free of bank conflicts)
        constexpr int CH = RB / 16;
        constexpr int RPI = 32 / CH;
        const int ch = RB == 128 ? (lane & 7) : (lane >> 3);
        const int rsub = RB == 128 ? (lane >> 3) : (lane & 7);
        const int tcol = c + ch * (16 / ESZ);    // column inside the tile
        const int gcol = n0 + tcol;
        // a round can run past the tile (BN not a multiple of the round width):
        // those columns belong to the next tile and are not stored
        const bool col_ok = tcol < BN && gcol < N;
#pragma unroll
        for (int it = 0; it < 32 / RPI; ++it) {
          const int rr = it * RPI + rsub;
          const int grow = row0 + rr;
          if (grow < M && col_ok) {
            const uint4 u = *reinterpret_cast<const uint4*>(stg + rr * L::kStagePitch + ch * 16);
            *reinterpret_cast<uint4*>(static_cast<uint8_t*>(y) +
                                      (static_cast<size_t>(grow) * N + gcol) * ESZ) = u;
          }
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
cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b, int M, int N, int K,
                       const float* bias, void* y, int* err, int num_sms, cudaStream_t st) {
  using L = GemmSmem<BN, CG, epi_warps(ACT)>;
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
  cfg.gridDim = dim3(CG * (tiles < max_units ? tiles : max_units));
  if (g_pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  // the activations (A, M rows) are at least as large as the weights (B, N rows)
  const int n_fastest = M >= N ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, a, b, M, N, K, bias, y, err, n_fastest);
}

template <int BN, int CG>
cudaError_t launch_act(const CUtensorMap& a, const CUtensorMap& b, int M, int N, int K,
                       const float* bias, void* y, bool out_f32, int act, int* err, int num_sms,
                       cudaStream_t st) {
  if (out_f32) {
    if (act == 1) return launch_one<BN, CG, 1, true>(a, b, M, N, K, bias, y, err, num_sms, st);
    if (act == 2) return launch_one<BN, CG, 2, true>(a, b, M, N, K, bias, y, err, num_sms, st);
    return launch_one<BN, CG, 0, true>(a, b, M, N, K, bias, y, err, num_sms, st);
  }
  if (act == 1) return launch_one<BN, CG, 1, false>(a, b, M, N, K, bias, y, err, num_sms, st);
  if (act == 2) return launch_one<BN, CG, 2, false>(a, b, M, N, K, bias, y, err, num_sms, st);
  return launch_one<BN, CG, 0, false>(a, b, M, N, K, bias, y, err, num_sms, st);
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

cudaError_t gemm_launch(const CUtensorMap& a, const CUtensorMap& b, GemmTile tile, int M, int N,
                        int K, const float* bias, void* y, bool out_f32, int act, int* err,
                        int num_sms, cudaStream_t st) {
  if (tile.cg == 2) {
    switch (tile.bn) {
      case 128: return launch_act<128, 2>(a, b, M, N, K, bias, y, out_f32, act, err, num_sms, st);
      case 192: return launch_act<192, 2>(a, b, M, N, K, bias, y, out_f32, act, err, num_sms, st);
      case 256: return launch_act<256, 2>(a, b, M, N, K, bias, y, out_f32, act, err, num_sms, st);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (tile.bn) {
    case 64: return launch_act<64, 1>(a, b, M, N, K, bias, y, out_f32, act, err, num_sms, st);
    case 96: return launch_act<96, 1>(a, b, M, N, K, bias, y, out_f32, act, err, num_sms, st);
    case 128: return launch_act<128, 1>(a, b, M, N, K, bias, y, out_f32, act, err, num_sms, st);
    case 160: return launch_act<160, 1>(a, b, M, N, K, bias, y, out_f32, act, err, num_sms, st);
    case 192: return launch_act<192, 1>(a, b, M, N, K, bias, y, out_f32, act, err, num_sms, st);
    case 224: return launch_act<224, 1>(a, b, M, N, K, bias, y, out_f32, act, err, num_sms, st);
    case 256: return launch_act<256, 1>(a, b, M, N, K, bias, y, out_f32, act, err, num_sms, st);
    default: return cudaErrorInvalidValue;
  }
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
