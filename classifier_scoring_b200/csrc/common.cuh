// Shared device/host helpers of the scorer's kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rmk {

using bf16 = __nv_bfloat16;

// ---------------------------------------------------------------------------
// Element conversion.  fp32 -> bf16 rounds to nearest even (the intrinsic).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(float v) { return v; }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);   // .x = lo (low half), .y = hi
  return *reinterpret_cast<uint32_t*>(&p);
}
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Eight consecutive elements ("a chunk"): 16 bytes of bf16 or 32 bytes of fp32.
template <typename T> struct Chunk8;
template <> struct Chunk8<bf16> {
  static __device__ __forceinline__ void load(const bf16* p, float* f) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
  }
  static __device__ __forceinline__ void store(bf16* p, const float* f) {
    uint4 v;
    v.x = pack_bf16x2(f[0], f[1]); v.y = pack_bf16x2(f[2], f[3]);
    v.z = pack_bf16x2(f[4], f[5]); v.w = pack_bf16x2(f[6], f[7]);
    *reinterpret_cast<uint4*>(p) = v;
  }
};
template <> struct Chunk8<float> {
  static __device__ __forceinline__ void load(const float* p, float* f) {
    float4 a = reinterpret_cast<const float4*>(p)[0];
    float4 b = reinterpret_cast<const float4*>(p)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float* f) {
    reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
  }
};

__device__ __forceinline__ void load_f32x8(const float* p, float* f) { Chunk8<float>::load(p, f); }

// Reductions over aligned groups of G lanes (G a power of two <= 32).
template <int G> __device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
template <int G> __device__ __forceinline__ float group_max(float v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Largest i in [0, n) with a[i] <= key, for a non-decreasing a with a[0] <= key.
template <typename I>
__device__ __forceinline__ int upper_index(const I* a, int n, long long key) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if ((long long)a[mid] <= key) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// GELU: u * Phi(u) (erf form) or the tanh approximation (CUDA's tanhf).
// gelu_erf calls CUDA's erff; gelu_erf_fast evaluates erf with approximation
// 7.1.28 of Abramowitz & Stegun, "Handbook of Mathematical Functions"
// (|error| <= 3e-7 for x >= 0, odd extension for x < 0):
//   erf(x) = 1 - (1 + a1 x + a2 x^2 + a3 x^3 + a4 x^4 + a5 x^5 + a6 x^6)^-16.
// It is the GEMM epilogue's GELU: one reciprocal (the only special-function
// unit operation) and eleven multiply-adds, where 7.1.26 needs an exp and a
// reciprocal; the epilogue of the FFN1 projection is bound by exactly these
// operations.  The 16th power is formed before the reciprocal so that the
// reciprocal's rounding is not raised to the 16th power.
__device__ __forceinline__ float gelu_erf(float u) { return 0.5f * u * (1.0f + erff(u * 0.70710678118654752f)); }
__device__ __forceinline__ float erf_as7128(float x) {
  const float ax = fabsf(x);
  float p = fmaf(0.0000430638f, ax, 0.0002765672f);
  p = fmaf(p, ax, 0.0001520143f);
  p = fmaf(p, ax, 0.0092705272f);
  p = fmaf(p, ax, 0.0422820123f);
  p = fmaf(p, ax, 0.0705230784f);
  p = fmaf(p, ax, 1.0f);
  p = p * p;
  p = p * p;
  p = p * p;
  p = p * p;                                   // p^16 (overflows to inf for large x: erf = 1)
  const float y = 1.0f - __fdividef(1.0f, p);
  return copysignf(y, x);
}
__device__ __forceinline__ float gelu_erf_fast(float u) {
  return 0.5f * u * (1.0f + erf_as7128(u * 0.70710678118654752f));
}

// 2^x by the hardware approximation (PTX ex2.approx.ftz.f32): one
// special-function-unit instruction; subnormal inputs and results flush to
// zero (for the softmax kernels: terms below 2^-126 of the row maximum's
// term, far under one bf16 ulp of the largest probability).
__device__ __forceinline__ float ex2_approx_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 lanes in one 64-bit register, for sm_100's packed arithmetic
// (add/sub/mul/fma .rn.f32x2: one instruction, two IEEE fp32 operations, each
// rounded as its scalar form would be).
__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ uint64_t f32x2_splat(float v) { return f32x2_pack(v, v); }
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// gelu_erf_fast on two values at once: the same A&S 7.1.28 polynomial and
// 16th power in packed fp32 (identical roundings lane by lane), the two
// reciprocals scalar; the last step forms h + h*erf with h = u/2 (one fused
// rounding where the scalar form rounds 1 + erf and the product).
__device__ __forceinline__ uint64_t gelu_erf_fast_x2(uint64_t u) {
  const uint64_t x = f32x2_mul(u, f32x2_splat(0.70710678118654752f));
  const uint64_t ax = x & 0x7fffffff7fffffffull;
  uint64_t p = f32x2_fma(f32x2_splat(0.0000430638f), ax, f32x2_splat(0.0002765672f));
  p = f32x2_fma(p, ax, f32x2_splat(0.0001520143f));
  p = f32x2_fma(p, ax, f32x2_splat(0.0092705272f));
  p = f32x2_fma(p, ax, f32x2_splat(0.0422820123f));
  p = f32x2_fma(p, ax, f32x2_splat(0.0705230784f));
  p = f32x2_fma(p, ax, f32x2_splat(1.0f));
  p = f32x2_mul(p, p);
  p = f32x2_mul(p, p);
  p = f32x2_mul(p, p);
  p = f32x2_mul(p, p);                        // p^16 (inf for large |x|: erf = +-1)
  float p0, p1;
  f32x2_unpack(p, p0, p1);
  // 1 - 1/p is in [0, 1): its sign bit is clear, so the sign of x is OR-ed in
  const uint64_t y = f32x2_sub(f32x2_splat(1.0f), f32x2_pack(__fdividef(1.0f, p0), __fdividef(1.0f, p1)));
  const uint64_t erf = y | (x & 0x8000000080000000ull);
  const uint64_t h = f32x2_mul(u, f32x2_splat(0.5f));
  return f32x2_fma(erf, h, h);
}
__device__ __forceinline__ float gelu_tanh(float u) {
  return 0.5f * u * (1.0f + tanhf(0.79788456080286536f * (u + 0.044715f * u * u * u)));
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel on its stream finishes;
// pdl_wait() blocks until that kernel has completed and its writes are
// visible, and pdl_launch_dependents() lets the next kernel start launching.
// Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// This CTA's share of up to two byte ranges, pulled into L2 with bulk
// prefetches (16-byte granules; no shared memory, no completion to wait for).
struct L2PrefetchArgs {
  const void* ptr[2];
  unsigned long long bytes[2];
};
__device__ __forceinline__ void l2_prefetch_share(const L2PrefetchArgs& pf) {
  if (threadIdx.x != 0) return;
  for (int k = 0; k < 2; ++k) {
    if (pf.ptr[k] == nullptr || pf.bytes[k] == 0) continue;
    const unsigned long long granules = pf.bytes[k] / 16;
    const unsigned long long per = (granules + gridDim.x - 1) / gridDim.x;
    const unsigned long long g0 = per * blockIdx.x;
    if (g0 >= granules) continue;
    unsigned long long left = (granules - g0 < per ? granules - g0 : per) * 16;
    const char* a = static_cast<const char*>(pf.ptr[k]) + g0 * 16;
    while (left > 0) {
      const unsigned int sz = left > 65536ull ? 65536u : static_cast<unsigned int>(left);
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"(sz) : "memory");
      a += sz;
      left -= sz;
    }
  }
}

// Device error words (rm_get_device_error): [0] clamped token ids, [1] waits
// that gave up.
enum { ERR_CLAMPED = 0, ERR_TIMEOUT = 1, ERR_WORDS = 2 };

// The checked build (-DRM_CHECKED, librmscore_checked.so): kernels test the
// indices they derive from offsets and other metadata before the accesses
// those indices address; a failed test adds one to the translation unit's
// bounds counter (rm_bounds_errors sums and clears them) and the access is
// skipped.  No trap, no assert.  In the product build in_bounds() is
// constant true and the tests compile away.
#ifdef RM_CHECKED
#define RMK_CHECKED 1
#else
#define RMK_CHECKED 0
#endif
#define RMK_BOUNDS_UNIT(unit)                                                      \
  __device__ int32_t g_bounds_##unit = 0;                                          \
  __device__ __forceinline__ bool in_bounds(bool ok) {                             \
    if (RMK_CHECKED && !ok) atomicAdd(&g_bounds_##unit, 1);                        \
    return !RMK_CHECKED || ok;                                                     \
  }

}  // namespace rmk

namespace rmk {

// Launches with programmatic stream serialization while a PdlScope is alive
// on this thread (rm_score's launch sequence); plain stream order otherwise.
inline thread_local bool g_pdl = false;
struct PdlScope {
  bool saved;
  explicit PdlScope(bool on) : saved(g_pdl) { g_pdl = on; }
  ~PdlScope() { g_pdl = saved; }
};

template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace rmk
