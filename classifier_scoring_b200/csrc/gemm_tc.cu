// Y[M][N] = act(X[M][K] . W[N][K]^T + bias) on the 5th-generation tensor
// cores: the QKV, attention-output and FFN projections of the scorer (the
// "BLAS routines" of the TurboTransformers abstract, on tensor cores as its
// proposed-method section does; here bf16 in, fp32 accumulation).
//
// One CTA computes one 128 x BN output tile.  Four warps:
//   warp 0, one lane : TMA producer -- K-major 128x64 (A) and BNx64 (B) bf16
//                      boxes, 128-byte swizzle, into a STAGES-deep smem ring;
//   warp 1, one lane : issues tcgen05.mma (M=128, N=BN, K=16) into a TMEM
//                      accumulator, and tcgen05.commit to free each stage;
//   all four warps   : epilogue -- tcgen05.ld 32 columns at a time (warp w
//                      owns TMEM lanes 32w..32w+31 = tile rows), + bias,
//                      optional GELU, store bf16 or fp32.
// Every mbarrier wait is bounded (about 2 s of %globaltimer); a wait that
// gives up counts into err[ERR_TIMEOUT], the CTA skips its stores, frees its
// TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

namespace rmk {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;                      // 64 bf16 = one 128-byte swizzle row
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase of the given parity to complete.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
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
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr int kA = BM * BK * 2;
  static constexpr int kB = BN * BK * 2;
  static constexpr int kStage = kA + kB;
  static constexpr int kBarOff = STAGES * kStage;                 // full[S], empty[S], done
  static constexpr int kSlotOff = kBarOff + (2 * STAGES + 1) * 8;
  static constexpr int kBiasOff = (kSlotOff + 16 + 15) & ~15;
  static constexpr int kBytes = kBiasOff + BN * 4 + 1024;          // + alignment slack
};

template <int BN, int STAGES, int ACT, bool OUT_F32>
__global__ void __launch_bounds__(128, 1)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, int M, int N, int K,
                        const float* __restrict__ bias, void* __restrict__ y,
                        int* __restrict__ err) {
  using L = GemmSmem<BN, STAGES>;
  constexpr uint32_t kTmemCols = BN;   // BN in {64, 128, 256}: a power of two >= 32
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);
  float* sbias = reinterpret_cast<float*>(smem + L::kBiasOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM;
  const int nk = (K + BK - 1) / BK;
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES),
                 done = smem_u32(bars + 2 * STAGES);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  for (int c = threadIdx.x; c < BN; c += blockDim.x)
    sbias[c] = (bias != nullptr && n0 + c < N) ? bias[n0 + c] : 0.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---- TMA producer ----
    int issued = 0;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1;
      if (kb >= STAGES && !mbar_wait(empty0 + 8 * s, ph ^ 1)) {
        atomicAdd(err + ERR_TIMEOUT, 1);
        break;
      }
      mbar_arrive_expect_tx(full0 + 8 * s, L::kStage);
      tma_load_2d(smem_u32(smem + s * L::kStage), &tmA, kb * BK, m0, full0 + 8 * s);
      tma_load_2d(smem_u32(smem + s * L::kStage + L::kA), &tmB, kb * BK, n0, full0 + 8 * s);
      ++issued;
    }
    // Copies still in flight land before this CTA's shared memory is released:
    // wait (bounded) for the last min(issued, STAGES) stages to fill.
    for (int kb = issued - 1; kb >= 0 && kb >= issued - STAGES; --kb)
      mbar_wait(full0 + 8 * (kb % STAGES), (kb / STAGES) & 1);
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer ----
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1;
      if (!mbar_wait(full0 + 8 * s, ph)) {
        atomicAdd(err + ERR_TIMEOUT, 1);
        break;
      }
      tc_fence_after();
      const uint64_t ad = smem_desc_k_sw128(smem_u32(smem + s * L::kStage));
      const uint64_t bd = smem_desc_k_sw128(smem_u32(smem + s * L::kStage + L::kA));
#pragma unroll
      for (int k = 0; k < BK / 16; ++k) {
        // advance 16 elements = 32 bytes along K inside the swizzle atom
        const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
            "l"(ad + 2ull * k), "l"(bd + 2ull * k), "r"(idesc), "r"(acc)
            : "memory");
      }
      asm volatile(
          "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
              empty0 + 8 * s)
          : "memory");
    }
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(done)
        : "memory");
  }
  __syncwarp();

  // ---- epilogue: TMEM -> registers -> bias/GELU -> global ----
  const bool ready = mbar_wait(done, 0);
  tc_fence_after();
  if (!ready && lane == 0) atomicAdd(err + ERR_TIMEOUT, 1);
  const int row = m0 + warp * 32 + lane;
  if (__all_sync(0xffffffffu, ready)) {
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t r[32];
      tmem_ld_32cols(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c, r);
      if (row < M && n0 + c < N) {
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float t = __uint_as_float(r[j]) + sbias[c + j];
          if (ACT == 1) t = gelu_erf(t);
          if (ACT == 2) t = gelu_tanh(t);
          v[j] = t;
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int col = n0 + c + 8 * g;
          if (col < N) {
            if (OUT_F32) {
              float* dst = static_cast<float*>(y) + static_cast<size_t>(row) * N + col;
              Chunk8<float>::store(dst, v + 8 * g);
            } else {
              bf16* dst = static_cast<bf16*>(y) + static_cast<size_t>(row) * N + col;
              Chunk8<bf16>::store(dst, v + 8 * g);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <int BN, int STAGES, int ACT, bool OUT_F32>
cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b, int M, int N, int K,
                       const float* bias, void* y, int* err, cudaStream_t st) {
  using L = GemmSmem<BN, STAGES>;
  auto kern = gemm_bf16_tc_kernel<BN, STAGES, ACT, OUT_F32>;
  static bool configured = false;   // per instantiation; attribute is per device function
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  kern<<<grid, 128, L::kBytes, st>>>(a, b, M, N, K, bias, y, err);
  return cudaGetLastError();
}

template <int BN, int STAGES>
cudaError_t launch_act(const CUtensorMap& a, const CUtensorMap& b, int M, int N, int K,
                       const float* bias, void* y, bool out_f32, int act, int* err,
                       cudaStream_t st) {
  if (out_f32) {
    if (act == 1) return launch_one<BN, STAGES, 1, true>(a, b, M, N, K, bias, y, err, st);
    if (act == 2) return launch_one<BN, STAGES, 2, true>(a, b, M, N, K, bias, y, err, st);
    return launch_one<BN, STAGES, 0, true>(a, b, M, N, K, bias, y, err, st);
  }
  if (act == 1) return launch_one<BN, STAGES, 1, false>(a, b, M, N, K, bias, y, err, st);
  if (act == 2) return launch_one<BN, STAGES, 2, false>(a, b, M, N, K, bias, y, err, st);
  return launch_one<BN, STAGES, 0, false>(a, b, M, N, K, bias, y, err, st);
}

}  // namespace

int gemm_pick_bn(int M, int N, int num_sms) {
  // Fewest waves first, then the larger tile (less B re-read, longer mainloop).
  const int tm = (M + BM - 1) / BM;
  int best = 256;
  long long best_cost = -1;
  for (int bn : {256, 128}) {
    const long long tiles = static_cast<long long>(tm) * ((N + bn - 1) / bn);
    const long long waves = (tiles + num_sms - 1) / num_sms;
    const long long cost = waves * (bn + 64);   // per-tile time ~ bn, plus fixed overhead
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

cudaError_t gemm_launch(const CUtensorMap& a, const CUtensorMap& b, int bn, int M, int N, int K,
                        const float* bias, void* y, bool out_f32, int act, int* err,
                        cudaStream_t st) {
  if (bn == 256) return launch_act<256, 4>(a, b, M, N, K, bias, y, out_f32, act, err, st);
  return launch_act<128, 6>(a, b, M, N, K, bias, y, out_f32, act, err, st);
}

}  // namespace rmk
