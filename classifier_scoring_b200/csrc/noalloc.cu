// Attention step (scores -> masked softmax -> context) whose score matrix and
// per-call metadata live in a fixed, file-scope device array instead of
// memory the caller or the library allocates per call.  For callers that
// cannot allocate device memory at the point where they run the step: a
// plugin executing inside another runtime that owns the device memory pool,
// or code on a path where cudaMalloc is not allowed because it can
// synchronize the device or fail under memory pressure.
//
// The array is a static __device__ object: every device that loads this
// library holds it until the process exits.  Host code never passes the
// array's name to a kernel (in host code that name is only a host-side
// stand-in); it passes the device address obtained with cudaGetSymbolAddress
// once per CUDA context.
#include <cudaTypedefs.h>

#include <map>
#include <mutex>

#include "../../include/rm.h"
#include "../../include/rm_ops.h"
#include "host.h"
#include "kernels.h"

namespace rmk {
namespace {

constexpr int64_t kNoallocMaxScoreElems = 4 * 1024 * 1024;   // bf16 score entries (8 MiB)
constexpr int32_t kNoallocMaxSeqs = 4096;
constexpr int64_t kMetaBytes = 16 * (kNoallocMaxSeqs + 1);     // offsets, rb_off (int32), s_off (int64)
constexpr int64_t kScratchBytes = kMetaBytes + 2 * kNoallocMaxScoreElems;

__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the scratch array per CUDA context.  The library's module
// (and so the array) is loaded once per context: a caller that runs in a
// context of its own (cuCtxCreate, or a host runtime that owns its context)
// sees a different array than the device's primary context.  The address is
// resolved on the first call made with that context current.
std::mutex g_setup_mu;
std::map<CUcontext, void*> g_scratch_ptr;

// Host staging of the metadata, copied into the device scratch before each
// launch.  These are pageable host arrays: for a pageable host-to-device
// cudaMemcpyAsync the runtime documents (API synchronization behavior) that
// the call returns once the source has been copied to staging memory for the
// DMA, so the arrays may be refilled by the next call after it returns.
std::mutex g_meta_mu;
int32_t g_meta_off[kNoallocMaxSeqs + 1];
int32_t g_meta_rb[kNoallocMaxSeqs + 1];
int64_t g_meta_so[kNoallocMaxSeqs + 1];

PFN_cuCtxGetCurrent_v4000 ctx_get_current() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  return fn;
}

int scratch_for_current_context(unsigned char** out) {
  auto get = ctx_get_current();
  if (get == nullptr) return set_error(RM_E_CUDA, "cuCtxGetCurrent is not available from the driver");
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return set_error(RM_E_CUDA, "cuCtxGetCurrent failed");
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (ctx != nullptr) {
    auto it = g_scratch_ptr.find(ctx);
    if (it != g_scratch_ptr.end()) {
      *out = static_cast<unsigned char*>(it->second);
      return RM_OK;
    }
  }
  // first call in this context: with no context current, the lookup binds the
  // device's primary context, which the launches of this call then use
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr)
    return set_error(RM_E_CUDA, "cudaGetSymbolAddress of the scratch array: %s", cudaGetErrorString(e));
  if (ctx == nullptr && (get(&ctx) != CUDA_SUCCESS || ctx == nullptr))
    return set_error(RM_E_CUDA, "no current CUDA context after the scratch lookup");
  g_scratch_ptr[ctx] = p;
  *out = static_cast<unsigned char*>(p);
  return RM_OK;
}

}  // namespace
}  // namespace rmk

using namespace rmk;

extern "C" int rm_op_attention_noalloc(const void* qkv, void* ctx, const int32_t* offsets,
                                       int32_t n_seqs, int32_t n_heads, int32_t head_dim,
                                       int32_t causal, void* stream) {
  if (qkv == nullptr || ctx == nullptr || offsets == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  if (n_seqs < 1 || n_heads < 1 || head_dim < 2 || head_dim % 2 || head_dim > 128)
    return set_error(RM_E_INVAL, "bad sizes");
  if (n_seqs > kNoallocMaxSeqs)
    return set_error(RM_E_RANGE, "%d sequences exceed the scratch limit of %d", n_seqs,
                     kNoallocMaxSeqs);
  if (offsets[0] != 0) return set_error(RM_E_INVAL, "offsets[0] must be 0");
  int32_t max_len = 0;
  int64_t elems = 0;
  for (int32_t i = 0; i < n_seqs; ++i) {
    const int64_t L = static_cast<int64_t>(offsets[i + 1]) - offsets[i];
    if (L < 1) return set_error(RM_E_INVAL, "sequence %d has length %lld (< 1)", i, (long long)L);
    if (L > 1024) return set_error(RM_E_RANGE, "sequence %d is longer than 1024 tokens", i);
    if (L > max_len) max_len = static_cast<int32_t>(L);
    elems += static_cast<int64_t>(n_heads) * L * ((L + 7) / 8 * 8);
  }
  if (elems > kNoallocMaxScoreElems)
    return set_error(RM_E_RANGE,
                     "the score matrix needs %lld entries; the scratch array holds %lld "
                     "(use rm_op_attn_scores/softmax/context with caller-allocated memory)",
                     (long long)elems, (long long)kNoallocMaxScoreElems);
  unsigned char* scratch = nullptr;
  int rc = scratch_for_current_context(&scratch);
  if (rc != RM_OK) return rc;
  int32_t* d_off = reinterpret_cast<int32_t*>(scratch);
  int32_t* d_rb = reinterpret_cast<int32_t*>(scratch + 4 * (kNoallocMaxSeqs + 1));
  int64_t* d_so = reinterpret_cast<int64_t*>(scratch + 8 * (kNoallocMaxSeqs + 1));
  void* d_s = scratch + kMetaBytes;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t nb = static_cast<size_t>(n_seqs) + 1;
  int32_t n_row_blocks = 0;
  {
    std::lock_guard<std::mutex> lock(g_meta_mu);
    for (size_t k = 0; k < nb; ++k) g_meta_off[k] = offsets[k];
    rc = rm_varlen_meta(g_meta_off, n_seqs, n_heads, g_meta_rb, g_meta_so);
    if (rc != RM_OK) return rc;
    n_row_blocks = g_meta_rb[n_seqs];
    cudaError_t e = cudaMemcpyAsync(d_off, g_meta_off, 4 * nb, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(d_rb, g_meta_rb, 4 * nb, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(d_so, g_meta_so, 8 * nb, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return set_error(RM_E_CUDA, "metadata copy: %s", cudaGetErrorString(e));
  }
  // every score entry that a later kernel reads is written by the scores
  // kernel of the same call, so nothing in the array needs clearing
  cudaError_t e = attn_scores_launch(qkv, d_s, d_off, d_rb, d_so, n_seqs, n_row_blocks, n_heads,
                                     head_dim, causal != 0, st);
  if (e == cudaSuccess)
    e = softmax_launch(d_s, RM_BF16, d_off, d_so, n_seqs, offsets[n_seqs], n_heads, max_len,
                       causal != 0, nullptr, st);
  if (e == cudaSuccess)
    e = attn_context_launch(d_s, qkv, ctx, d_off, d_rb, d_so, n_seqs, n_row_blocks, n_heads,
                            head_dim, causal != 0, st);
  if (e != cudaSuccess) return set_error(RM_E_CUDA, "attention launch: %s", cudaGetErrorString(e));
  return RM_OK;
}
