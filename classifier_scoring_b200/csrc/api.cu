// C ABI of the scorer (include/rm.h, include/rm_ops.h): validation, weight
// upload, the arena, per-call metadata and the forward launch sequence.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <memory>
#include <string>
#include <utility>
#include <vector>

#include "../../include/rm.h"
#include "../../include/rm_ops.h"
#include "common.cuh"
#include "host.h"
#include "kernels.h"

namespace rmk {

namespace {
thread_local char g_msg[512] = "";
__device__ int32_t g_err_sink[ERR_WORDS];   // error words for handle-less rm_op_* calls

// Test hook (rm_debug_fail_alloc): the k-th allocation from now on fails as if
// memory were exhausted, without reaching the allocator.
std::atomic<int32_t> g_fail_alloc{0};

bool injected_alloc_failure() {
  int32_t k = g_fail_alloc.load();
  while (k > 0)
    if (g_fail_alloc.compare_exchange_weak(k, k - 1)) return k == 1;
  return false;
}

cudaError_t dev_malloc(void** p, size_t bytes) {
  if (injected_alloc_failure()) {
    *p = nullptr;
    return cudaErrorMemoryAllocation;
  }
  return cudaMalloc(p, bytes);
}

cudaError_t pinned_malloc(void** p, size_t bytes) {
  if (injected_alloc_failure()) {
    *p = nullptr;
    return cudaErrorMemoryAllocation;
  }
  return cudaHostAlloc(p, bytes, cudaHostAllocDefault);
}
}  // namespace

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof g_msg, fmt, ap);
  va_end(ap);
  return code;
}

#define RM_CUDA(call)                                                                  \
  do {                                                                                 \
    cudaError_t e_ = (call);                                                           \
    if (e_ != cudaSuccess)                                                             \
      return set_error(e_ == cudaErrorMemoryAllocation ? RM_E_NOMEM : RM_E_CUDA,       \
                       "%s: %s (%s:%d)", #call, cudaGetErrorString(e_), __FILE__, __LINE__); \
  } while (0)

int validate_config(const rm_config* c, bool sched_only, const char** why) {
  auto bad = [&](const char* m) { *why = m; return RM_E_INVAL; };
  if (c == nullptr) return bad("config is NULL");
  if (c->max_len < 1 || c->max_len > 1024) return bad("max_len must be in 1..1024");
  if (c->sched_max_batch < 1) return bad("sched_max_batch must be >= 1");
  if (c->sched_c0 < 0 || c->sched_c1 < 0 || c->sched_c0 > (1LL << 40) || c->sched_c1 > (1LL << 40))
    return bad("sched_c0 and sched_c1 must be in 0..2^40");
  if (c->sched_objective != RM_SCHED_THROUGHPUT && c->sched_objective != RM_SCHED_LATENCY)
    return bad("sched_objective must be 0 or 1");
  if (c->sched_max_cost < 0) return bad("sched_max_cost must be >= 0");
  if (c->sched_table != nullptr) {
    if (c->sched_table_b < c->sched_max_batch || c->sched_table_l < c->max_len)
      return bad("sched_table must have >= sched_max_batch rows and >= max_len columns");
    for (int32_t b = 0; b < c->sched_table_b; ++b)
      for (int32_t l = 0; l < c->sched_table_l; ++l) {
        const int64_t v = c->sched_table[static_cast<size_t>(b) * c->sched_table_l + l];
        if (v < 0 || v > (1LL << 56)) return bad("sched_table entries must be in 0..2^56");
        if (l > 0 && v < c->sched_table[static_cast<size_t>(b) * c->sched_table_l + l - 1])
          return bad("sched_table must be non-decreasing along L");
      }
  }
  if (sched_only) return RM_OK;
  if (c->arch != RM_ENC_POSTLN && c->arch != RM_DEC_PRELN) return bad("arch must be 0 or 1");
  if (c->n_layers < 1) return bad("n_layers must be >= 1");
  if (c->hidden < 8 || c->hidden > 4096 || c->hidden % 8 != 0)
    return bad("hidden must be a multiple of 8 in 8..4096");
  if (c->n_heads < 1 || c->hidden % c->n_heads != 0) return bad("n_heads must divide hidden");
  const int d = c->hidden / c->n_heads;
  if (d % 2 != 0 || d > 128) return bad("head dim hidden/n_heads must be even and <= 128");
  if (c->ffn < 8 || c->ffn % 8 != 0 || c->ffn > 65536) return bad("ffn must be a multiple of 8");
  if (c->vocab < 1) return bad("vocab must be >= 1");
  if (c->max_pos < c->max_len) return bad("max_pos must be >= max_len");
  if (c->weight_dtype != RM_F32 && c->weight_dtype != RM_BF16) return bad("weight_dtype must be 0 or 1");
  if (c->gelu != RM_GELU_ERF && c->gelu != RM_GELU_TANH) return bad("gelu must be 0 or 1");
  if (!(c->ln_eps > 0.0f) || !std::isfinite(c->ln_eps)) return bad("ln_eps must be > 0");
  if (c->max_batch_seqs < 1) return bad("max_batch_seqs must be >= 1");
  if (c->max_tokens < 1 || c->max_tokens > (1 << 24)) return bad("max_tokens must be in 1..2^24");
  if (c->attn_impl != RM_ATTN_FUSED && c->attn_impl != RM_ATTN_MATERIALIZED)
    return bad("attn_impl must be 0 or 1");
  return RM_OK;
}

SchedCost sched_cost_from(const rm_config* c) {
  SchedCost s;
  s.bmax = c->sched_max_batch;
  s.objective = c->sched_objective;
  s.max_cost = c->sched_max_cost;
  s.c0 = c->sched_c0;
  s.c1 = c->sched_c1;
  if (c->sched_table != nullptr) {
    s.tb = c->sched_table_b;
    s.tl = c->sched_table_l;
    s.table.assign(c->sched_table, c->sched_table + static_cast<size_t>(s.tb) * s.tl);
  }
  return s;
}

namespace {

// ---- weight layout ----
struct Segment {
  const char* name;
  int64_t elems;
  bool matrix;       // stored bf16 on device (GEMM operand or embedding table)
};

std::vector<Segment> segments(const rm_config* c) {
  const int64_t H = c->hidden, F = c->ffn;
  std::vector<Segment> s;
  s.push_back({"emb_word", static_cast<int64_t>(c->vocab) * H, true});
  s.push_back({"emb_pos", static_cast<int64_t>(c->max_pos) * H, true});
  if (c->arch == RM_ENC_POSTLN) {
    s.push_back({"ln_emb_g", H, false});
    s.push_back({"ln_emb_b", H, false});
  }
  for (int l = 0; l < c->n_layers; ++l) {
    s.push_back({"w_qkv", 3 * H * H, true});
    s.push_back({"b_qkv", 3 * H, false});
    s.push_back({"w_o", H * H, true});
    s.push_back({"b_o", H, false});
    s.push_back({"ln1_g", H, false});
    s.push_back({"ln1_b", H, false});
    s.push_back({"w_1", F * H, true});
    s.push_back({"b_1", F, false});
    s.push_back({"w_2", H * F, true});
    s.push_back({"b_2", H, false});
    s.push_back({"ln2_g", H, false});
    s.push_back({"ln2_b", H, false});
  }
  if (c->arch == RM_DEC_PRELN) {
    s.push_back({"lnf_g", H, false});
    s.push_back({"lnf_b", H, false});
  }
  s.push_back({"w_r", H, false});
  s.push_back({"b_r", 1, false});
  return s;
}

int64_t align_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

struct LayerW {
  bf16 *w_qkv, *w_o, *w_1, *w_2;
  float *b_qkv, *b_o, *ln1_g, *ln1_b, *b_1, *b_2, *ln2_g, *ln2_b;
  CUtensorMap tm[4][kGemmTileCount];   // [qkv, o, 1, 2][box rows of each tile width]
};

struct Bucket {
  ArenaPlan plan;
  CUtensorMap a_in, a_ctx, a_f;      // A operands: x (encoder) or z (decoder), ctx, f
  CUtensorMap y_qkv, y_o, y_f, y_2;  // outputs: qkv, y1, f, y2 (the bucket's rows)
};

constexpr int kSlots = 4;

}  // namespace
}  // namespace rmk

using namespace rmk;

struct rm_handle {
  rm_config cfg;
  SchedCost sched;
  int device = 0, num_sms = 148;
  void* wbuf = nullptr;
  std::shared_ptr<void> weights_owner;   // shared by handles made with rm_create_shared
  bf16 *emb_word = nullptr, *emb_pos = nullptr;
  float *ln_emb_g = nullptr, *ln_emb_b = nullptr, *lnf_g = nullptr, *lnf_b = nullptr,
        *w_r = nullptr;
  float b_r = 0.f;
  std::vector<LayerW> layers;
  uint8_t* arena = nullptr;
  int64_t arena_bytes = 0, fixed_bytes = 0, meta_bytes = 0;
  int32_t* d_ids = nullptr;
  float* d_scores = nullptr;
  void* d_sm_scratch = nullptr;   // row index of the materialised softmax
  uint8_t* d_meta = nullptr;
  uint8_t* planned = nullptr;
  int32_t* d_err = nullptr;
  uint8_t* pinned = nullptr;
  cudaEvent_t ev[kSlots] = {};
  int slot = 0;
  std::map<std::pair<int64_t, int64_t>, Bucket> buckets;
  int64_t max_peak = 0;
  cudaStream_t last_stream = nullptr;
  // measurement
  int64_t launches = 0, calls = 0;
  int32_t prof_every = 0;
  struct ProfRec { int cls; double flops, bytes; cudaEvent_t a, b; };
  std::vector<ProfRec> prof;
  std::vector<cudaEvent_t> ev_pool;
  // host scratch of rm_score_prefix's segment list (reused across calls)
  std::vector<int32_t> px_off, px_start, px_len, px_out, px_goff;
};

namespace {

// Metadata of one call in a staging slot / the device meta region:
// offsets int32[n+1] | rb_off int32[n+1] | s_off int64[n+1] | tiles int32[n+1]
// (16-byte aligned parts; tiles: the tensor-core attention's sequence tiles),
// then for shared-prefix calls pre_start int32[n] | pre_len int32[n] |
// out_index int32[n] | group_off int32[n+1].  `base` bytes are copied for a
// plain call, `bytes` for a shared-prefix call.
struct MetaLayout {
  int64_t rb, so, tl, base, pst, pln, oix, gof, bytes;
  explicit MetaLayout(int64_t n) {
    rb = align_up(4 * (n + 1), 16);
    so = rb + align_up(4 * (n + 1), 16);
    tl = so + align_up(8 * (n + 1), 16);
    base = tl + align_up(4 * (4 * n + 1), 16);   // tiles (n + 1) or long-row items (<= 4n)
    pst = base;
    pln = pst + align_up(4 * n, 16);
    oix = pln + align_up(4 * n, 16);
    gof = oix + align_up(4 * n, 16);
    bytes = gof + align_up(4 * (n + 1), 16);
  }
};

// Segments of a shared-prefix call (rm_score_prefix), host arrays.
struct PrefixSpec {
  const int32_t* pre_start;   // [n] packed row of the prefix a segment continues
  const int32_t* pre_len;     // [n] its length (0 for a prefix or a plain segment)
  const int32_t* out_index;   // [n] output slot of the segment's score, -1 for none
  const int32_t* group_off;   // [n_groups + 1] candidate slots of each group
  int32_t n_groups;
  int32_t* d_best;            // device [n_groups] or NULL
  float* d_logodds;           // device [n_groups] or NULL
};

int host_varlen_meta(const int32_t* off, int32_t n, int32_t nh, int32_t* rb, int64_t* so,
                     int32_t* max_len) {
  if (off[0] != 0) return set_error(RM_E_INVAL, "seq_offsets[0] must be 0");
  rb[0] = 0;
  so[0] = 0;
  int32_t ml = 0;
  for (int32_t i = 0; i < n; ++i) {
    const int64_t L = static_cast<int64_t>(off[i + 1]) - off[i];
    if (L < 1) return set_error(RM_E_INVAL, "sequence %d has length %lld (< 1)", i, (long long)L);
    ml = std::max<int32_t>(ml, static_cast<int32_t>(L));
    rb[i + 1] = rb[i] + static_cast<int32_t>((L + 63) / 64);
    so[i + 1] = so[i] + static_cast<int64_t>(nh) * L * align_up(L, 8);
  }
  if (max_len) *max_len = ml;
  return RM_OK;
}

int upload_weights(rm_handle* h, const void* weights) {
  const rm_config* c = &h->cfg;
  const auto seg = segments(c);
  const int esz = c->weight_dtype == RM_F32 ? 4 : 2;
  int64_t nbf = 0, nf = 0, total = 0;
  for (const auto& s : seg) {
    if (s.matrix) nbf += align_up(s.elems, 128);
    else nf += align_up(s.elems, 64);
    total += s.elems;
  }
  const size_t wbytes = static_cast<size_t>(nbf) * 2 + static_cast<size_t>(nf) * 4;
  RM_CUDA(dev_malloc(&h->wbuf, wbytes));
  void* staging = nullptr;
  RM_CUDA(dev_malloc(&staging, static_cast<size_t>(total) * esz));
  cudaError_t e = cudaMemcpy(staging, weights, static_cast<size_t>(total) * esz, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(staging);
    return set_error(RM_E_CUDA, "weight upload: %s", cudaGetErrorString(e));
  }
  bf16* pb = static_cast<bf16*>(h->wbuf);
  float* pf = reinterpret_cast<float*>(static_cast<uint8_t*>(h->wbuf) + nbf * 2);
  int64_t src = 0;
  int layer = -1;
  for (const auto& s : seg) {
    const void* from = static_cast<const uint8_t*>(staging) + src * esz;
    void* dst;
    if (s.matrix) {
      dst = pb;
      e = cvt_to_bf16_launch(from, c->weight_dtype, pb, static_cast<size_t>(s.elems), 0);
      pb += align_up(s.elems, 128);
    } else {
      dst = pf;
      e = cvt_to_f32_launch(from, c->weight_dtype, pf, static_cast<size_t>(s.elems), 0);
      pf += align_up(s.elems, 64);
    }
    if (e != cudaSuccess) break;
    const std::string nm = s.name;
    if (nm == "w_qkv") { h->layers.emplace_back(); ++layer; }
    LayerW* L = layer >= 0 ? &h->layers[layer] : nullptr;
    if (nm == "emb_word") h->emb_word = static_cast<bf16*>(dst);
    else if (nm == "emb_pos") h->emb_pos = static_cast<bf16*>(dst);
    else if (nm == "ln_emb_g") h->ln_emb_g = static_cast<float*>(dst);
    else if (nm == "ln_emb_b") h->ln_emb_b = static_cast<float*>(dst);
    else if (nm == "lnf_g") h->lnf_g = static_cast<float*>(dst);
    else if (nm == "lnf_b") h->lnf_b = static_cast<float*>(dst);
    else if (nm == "w_r") h->w_r = static_cast<float*>(dst);
    else if (nm == "b_r") {
      // the head bias is also a kernel argument: read it on the host
      if (c->weight_dtype == RM_F32) {
        std::memcpy(&h->b_r, static_cast<const uint8_t*>(weights) + src * 4, 4);
      } else {
        uint16_t bits;
        std::memcpy(&bits, static_cast<const uint8_t*>(weights) + src * 2, 2);
        const uint32_t u = static_cast<uint32_t>(bits) << 16;
        std::memcpy(&h->b_r, &u, 4);
      }
    } else if (L) {
      if (nm == "w_qkv") L->w_qkv = static_cast<bf16*>(dst);
      else if (nm == "b_qkv") L->b_qkv = static_cast<float*>(dst);
      else if (nm == "w_o") L->w_o = static_cast<bf16*>(dst);
      else if (nm == "b_o") L->b_o = static_cast<float*>(dst);
      else if (nm == "ln1_g") L->ln1_g = static_cast<float*>(dst);
      else if (nm == "ln1_b") L->ln1_b = static_cast<float*>(dst);
      else if (nm == "w_1") L->w_1 = static_cast<bf16*>(dst);
      else if (nm == "b_1") L->b_1 = static_cast<float*>(dst);
      else if (nm == "w_2") L->w_2 = static_cast<bf16*>(dst);
      else if (nm == "b_2") L->b_2 = static_cast<float*>(dst);
      else if (nm == "ln2_g") L->ln2_g = static_cast<float*>(dst);
      else if (nm == "ln2_b") L->ln2_b = static_cast<float*>(dst);
    }
    src += s.elems;
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  cudaFree(staging);
  if (e != cudaSuccess) return set_error(RM_E_CUDA, "weight conversion: %s", cudaGetErrorString(e));
  // TMA maps of every weight matrix, for both column-tile widths
  const int64_t H = c->hidden, F = c->ffn;
  for (auto& L : h->layers) {
    const bf16* mats[4] = {L.w_qkv, L.w_o, L.w_1, L.w_2};
    const int64_t rows[4] = {3 * H, H, F, H}, cols[4] = {H, H, H, F};
    for (int m = 0; m < 4; ++m)
      for (int b = 0; b < kGemmTileCount; ++b) {
        const char* why = "";
        if (!make_tmap_bf16(&L.tm[m][b], mats[m], rows[m], cols[m], kGemmTileWidths[b], &why))
          return set_error(RM_E_CUDA, "weight tensor map: %s", why);
      }
  }
  return RM_OK;
}

int get_bucket(rm_handle* h, int64_t T, int64_t S, Bucket** out) {
  // length buckets: tokens rounded up to 128, score elements to 64 Ki; the
  // fused attention keeps no score matrix, so its buckets are keyed on tokens alone
  const int64_t Tb = align_up(T, 128);
  const int64_t Sb =
      h->cfg.attn_impl == RM_ATTN_FUSED ? 0 : align_up(std::max<int64_t>(S, 1), 65536);
  auto key = std::make_pair(Tb, Sb);
  auto it = h->buckets.find(key);
  if (it != h->buckets.end()) {
    *out = &it->second;
    return RM_OK;
  }
  const rm_config* c = &h->cfg;
  Bucket b;
  b.plan = plan_arena(c->arch, c->hidden, c->ffn, Tb, Sb);
  if (h->fixed_bytes + b.plan.peak > h->arena_bytes)
    return set_error(RM_E_RANGE, "arena plan (%lld bytes) exceeds the reservation",
                     (long long)b.plan.peak);
  uint8_t* base = h->planned;
  const void* a_in = base + (c->arch == RM_DEC_PRELN ? b.plan.off[B_Z] : b.plan.off[B_X]);
  const char* why = "";
  if (!make_tmap_bf16(&b.a_in, a_in, Tb, c->hidden, 128, &why) ||
      !make_tmap_bf16(&b.a_ctx, base + b.plan.off[B_CTX], Tb, c->hidden, 128, &why) ||
      !make_tmap_bf16(&b.a_f, base + b.plan.off[B_F], Tb, c->ffn, 128, &why))
    return set_error(RM_E_CUDA, "activation tensor map: %s", why);
  // output maps cover the bucket's Tb rows (the buffers' extent): the rows of
  // a call's last 128-row tile past its T tokens land in their own buffer's
  // padding rows, which no later step reads
  // (y1, y2: the encoder's sublayer outputs; the decoder adds its sublayer
  // outputs straight into its fp32 residual stream and has neither, so its
  // maps stand in for them unused)
  const bool dec = c->arch == RM_DEC_PRELN;
  const int64_t y1 = dec ? b.plan.off[B_F] : b.plan.off[B_Y1];
  const int64_t y2 = dec ? b.plan.off[B_F] : b.plan.off[B_Y2];
  if (!make_tmap_store(&b.y_qkv, base + b.plan.off[B_QKV], Tb, 3 * c->hidden, false, &why) ||
      !make_tmap_store(&b.y_o, base + y1, Tb, c->hidden, false, &why) ||
      !make_tmap_store(&b.y_f, base + b.plan.off[B_F], Tb, c->ffn, false, &why) ||
      !make_tmap_store(&b.y_2, base + y2, Tb, c->hidden, false, &why))
    return set_error(RM_E_CUDA, "output tensor map: %s", why);
  h->max_peak = std::max(h->max_peak, b.plan.peak);
  auto res = h->buckets.emplace(key, b);
  *out = &res.first->second;
  return RM_OK;
}

// y: the output map; yacc (when not null, act 0 and out_f32 only): the fp32
// [M][N] tensor the product is added to instead (y then unused)
int gemm(rm_handle* h, const CUtensorMap& a, const CUtensorMap (&b)[kGemmTileCount], int M, int N,
         int K, const float* bias, const CUtensorMap& y, int act, cudaStream_t st,
         bool out_f32 = false, void* yacc = nullptr) {
  const GemmTile tile = gemm_pick(M, N, K, h->num_sms, act);
  const int split = gemm_tail_split(tile, M, N, h->num_sms);
  cudaError_t e = gemm_launch(a, b[gemm_tile_index(tile.b_box())],
                              b[gemm_tile_index(tile.b_box() / split)], y, yacc, tile, M, N, K,
                              bias, out_f32, act, h->d_err, h->num_sms, st);
  if (e != cudaSuccess) return set_error(RM_E_CUDA, "gemm launch: %s", cudaGetErrorString(e));
  return RM_OK;
}

#define RM_LAUNCH(call)                                                                   \
  do {                                                                                    \
    cudaError_t e_ = (call);                                                              \
    if (e_ != cudaSuccess)                                                                \
      return set_error(RM_E_CUDA, "%s: %s", #call, cudaGetErrorString(e_));              \
  } while (0)
#define RM_TRY(call)          \
  do {                        \
    int r_ = (call);          \
    if (r_ != RM_OK) return r_; \
  } while (0)

// Events around one launch when this call is profiled.
struct ProfScope {
  rm_handle* h;
  bool on;
  cudaEvent_t a = nullptr, b = nullptr;
  cudaStream_t st;
  ProfScope(rm_handle* hh, bool enabled, cudaStream_t s) : h(hh), on(enabled), st(s) {
    if (!on) return;
    a = take();
    b = take();
    if (a == nullptr || b == nullptr || cudaEventRecord(a, st) != cudaSuccess) on = false;
  }
  cudaEvent_t take() {
    if (!h->ev_pool.empty()) {
      cudaEvent_t e = h->ev_pool.back();
      h->ev_pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    return cudaEventCreate(&e) == cudaSuccess ? e : nullptr;
  }
  void done(int cls, double flops, double bytes) {
    ++h->launches;
    if (on && cudaEventRecord(b, st) == cudaSuccess) {
      h->prof.push_back({cls, flops, bytes, a, b});
      a = b = nullptr;
    }
  }
  ~ProfScope() {
    if (a) h->ev_pool.push_back(a);
    if (b) h->ev_pool.push_back(b);
  }
};

#define RM_KERNEL(cls, flops, bytes, call)          \
  do {                                               \
    ProfScope ps_(h, prof_on, st);                   \
    RM_LAUNCH(call);                                 \
    ps_.done(cls, flops, bytes);                     \
  } while (0)
#define RM_GEMM(flops, bytes, call)                  \
  do {                                               \
    ProfScope ps_(h, prof_on, st);                   \
    RM_TRY(call);                                    \
    ps_.done(RM_K_GEMM, flops, bytes);               \
  } while (0)

// What the launch sequence of one call needs to know on the host.
struct CallInfo {
  int32_t n = 0, T = 0, nrb = 0, Lmax = 0;
  int32_t ntc = 0;                   // tensor-core attention tiles (0: that kernel does not apply)
  int32_t ntcl = 0;                  // or its long-row work items (0: does not apply)
  const int32_t* d_tl = nullptr;     // the tiles or the items
  int64_t S = 0;
  double att = 0;   // attention entries the mask admits, summed over heads
  const int32_t* d_off = nullptr;
  const int32_t* d_rb = nullptr;
  const int64_t* d_so = nullptr;
  const int32_t *d_pst = nullptr, *d_pln = nullptr, *d_oix = nullptr, *d_gof = nullptr;
  const PrefixSpec* px = nullptr;
};

// Attention entries the mask admits: L*L per head, L*(L+1)/2 when causal,
// plus L*P for a segment that continues a shared prefix of P tokens.
double attention_entries(const rm_config* c, const int32_t* offsets, int32_t n,
                         const PrefixSpec* px) {
  const bool dec = c->arch == RM_DEC_PRELN;
  double att = 0;
  for (int32_t i = 0; i < n; ++i) {
    const double L = static_cast<double>(offsets[i + 1] - offsets[i]);
    const double P0 = px ? px->pre_len[i] : 0;
    att += dec ? L * P0 + L * (L + 1) / 2 : L * L;
  }
  return att * c->n_heads;
}

int enqueue_forward(rm_handle* h, const CallInfo& ci, const int32_t* d_ids, float* d_out,
                    cudaStream_t st);

// The tensor-core attention takes a plain call of the fused attention when
// the head dim is 64 and no sequence is longer than its 128-row tiles.
bool tc_attention_applies(const rm_config* c, int32_t max_len, bool prefix) {
  return !prefix && c->attn_impl == RM_ATTN_FUSED && c->hidden / c->n_heads == 64 && max_len <= 128;
}
// Its long-row form takes the other plain encoder calls with head dim 64 and
// sequences of up to 512 tokens (causal calls measured faster on the
// packed-row tiles, which skip the keys past each row in 16-key steps).
bool tcl_attention_applies(const rm_config* c, int32_t max_len, bool prefix) {
  return !prefix && c->attn_impl == RM_ATTN_FUSED && c->hidden / c->n_heads == 64 &&
         c->arch != RM_DEC_PRELN && max_len > 128 && max_len <= 512;
}

// host_ids != NULL: copy the ids host->device (into the arena) once the call
// has been validated, and the scores back into host_out at the end.
int score_impl(rm_handle* h, const int32_t* d_ids, const int32_t* host_ids, const int32_t* offsets,
               int32_t n, float* d_out, float* host_out, cudaStream_t st,
               const PrefixSpec* px = nullptr) {
  const rm_config* c = &h->cfg;
  if (n < 1) return set_error(RM_E_INVAL, "n_seqs must be >= 1");
  if (n > c->max_batch_seqs)
    return set_error(RM_E_RANGE, "n_seqs %d exceeds max_batch_seqs %d", n, c->max_batch_seqs);
  // metadata into the next pinned slot
  const int slot = h->slot;
  h->slot = (h->slot + 1) % kSlots;
  RM_CUDA(cudaEventSynchronize(h->ev[slot]));
  uint8_t* ps = h->pinned + static_cast<size_t>(slot) * h->meta_bytes;
  const MetaLayout ml(n);
  int32_t* p_off = reinterpret_cast<int32_t*>(ps);
  int32_t* p_rb = reinterpret_cast<int32_t*>(ps + ml.rb);
  int64_t* p_so = reinterpret_cast<int64_t*>(ps + ml.so);
  if (offsets[0] != 0) return set_error(RM_E_INVAL, "seq_offsets[0] must be 0");
  for (int32_t i = 0; i < n; ++i) {
    const int64_t L = static_cast<int64_t>(offsets[i + 1]) - offsets[i] + (px ? px->pre_len[i] : 0);
    if (L < 1) return set_error(RM_E_INVAL, "sequence %d has length %lld (< 1)", i, (long long)L);
    if (L > c->max_len)
      return set_error(RM_E_RANGE, "sequence %d has length %lld > max_len %d", i, (long long)L,
                       c->max_len);
  }
  const int32_t T = offsets[n];
  if (T > c->max_tokens)
    return set_error(RM_E_RANGE, "%d tokens exceed max_tokens %d", T, c->max_tokens);
  std::memcpy(p_off, offsets, 4 * static_cast<size_t>(n + 1));
  int32_t Lmax = 0;
  RM_TRY(host_varlen_meta(offsets, n, c->n_heads, p_rb, p_so, &Lmax));
  const int32_t nrb = p_rb[n];
  const int64_t S = p_so[n];
  const bool dec_c = c->arch == RM_DEC_PRELN;
  const int32_t ntc =
      tc_attention_applies(c, Lmax, px != nullptr) ? attn_tc_tiles(offsets, n, reinterpret_cast<int32_t*>(ps + ml.tl)) : 0;
  const int32_t ntcl = tcl_attention_applies(c, Lmax, px != nullptr)
                           ? attn_tcl_items(offsets, n, dec_c ? 1 : 0, reinterpret_cast<int32_t*>(ps + ml.tl))
                           : 0;
  if (host_ids != nullptr) {
    RM_CUDA(cudaMemcpyAsync(h->d_ids, host_ids, 4 * static_cast<size_t>(T), cudaMemcpyHostToDevice, st));
    d_ids = h->d_ids;
    d_out = h->d_scores;
  }
  if (px != nullptr) {
    std::memcpy(ps + ml.pst, px->pre_start, 4 * static_cast<size_t>(n));
    std::memcpy(ps + ml.pln, px->pre_len, 4 * static_cast<size_t>(n));
    std::memcpy(ps + ml.oix, px->out_index, 4 * static_cast<size_t>(n));
    std::memcpy(ps + ml.gof, px->group_off, 4 * static_cast<size_t>(px->n_groups + 1));
  }
  RM_CUDA(cudaMemcpyAsync(h->d_meta, ps, px != nullptr ? ml.bytes : ml.base, cudaMemcpyHostToDevice, st));
  RM_CUDA(cudaEventRecord(h->ev[slot], st));
  const int32_t* d_off = reinterpret_cast<const int32_t*>(h->d_meta);
  const int32_t* d_rb = reinterpret_cast<const int32_t*>(h->d_meta + ml.rb);
  const int64_t* d_so = reinterpret_cast<const int64_t*>(h->d_meta + ml.so);
  const int32_t* d_pst = px ? reinterpret_cast<const int32_t*>(h->d_meta + ml.pst) : nullptr;
  const int32_t* d_pln = px ? reinterpret_cast<const int32_t*>(h->d_meta + ml.pln) : nullptr;
  const int32_t* d_oix = px ? reinterpret_cast<const int32_t*>(h->d_meta + ml.oix) : nullptr;
  const int32_t* d_gof = px ? reinterpret_cast<const int32_t*>(h->d_meta + ml.gof) : nullptr;
  CallInfo ci;
  ci.n = n;
  ci.T = T;
  ci.nrb = nrb;
  ci.Lmax = Lmax;
  ci.ntc = ntc;
  ci.ntcl = ntcl;
  ci.d_tl = reinterpret_cast<const int32_t*>(h->d_meta + ml.tl);
  ci.S = S;
  ci.att = attention_entries(c, offsets, n, px);
  ci.d_off = d_off;
  ci.d_rb = d_rb;
  ci.d_so = d_so;
  ci.d_pst = d_pst;
  ci.d_pln = d_pln;
  ci.d_oix = d_oix;
  ci.d_gof = d_gof;
  ci.px = px;
  RM_TRY(enqueue_forward(h, ci, d_ids, d_out, st));
  if (host_out != nullptr)
    RM_CUDA(cudaMemcpyAsync(host_out, d_out, 4 * static_cast<size_t>(n), cudaMemcpyDeviceToHost, st));
  return RM_OK;
}

// The launch sequence of one call whose metadata is already on the device:
// kernels only (no host synchronisation, no copies), so a caller may capture
// it into a CUDA graph (rm_score_plan).
int enqueue_forward(rm_handle* h, const CallInfo& ci, const int32_t* d_ids, float* d_out,
                    cudaStream_t st) {
  const rm_config* c = &h->cfg;
  const int32_t n = ci.n, T = ci.T, nrb = ci.nrb, Lmax = ci.Lmax;
  const int64_t S = ci.S;
  const int32_t *d_off = ci.d_off, *d_rb = ci.d_rb, *d_pst = ci.d_pst, *d_pln = ci.d_pln,
                *d_oix = ci.d_oix, *d_gof = ci.d_gof;
  const int64_t* d_so = ci.d_so;
  const PrefixSpec* px = ci.px;
  Bucket* bk = nullptr;
  RM_TRY(get_bucket(h, T, S, &bk));
  uint8_t* base = h->planned;
  bf16* x = reinterpret_cast<bf16*>(base + bk->plan.off[B_X]);
  bf16* z = reinterpret_cast<bf16*>(base + bk->plan.off[B_Z]);
  bf16* qkv = reinterpret_cast<bf16*>(base + bk->plan.off[B_QKV]);
  bf16* s = reinterpret_cast<bf16*>(base + bk->plan.off[B_S]);
  bf16* ctx = reinterpret_cast<bf16*>(base + bk->plan.off[B_CTX]);
  bf16* y1 = reinterpret_cast<bf16*>(base + bk->plan.off[B_Y1]);   // encoder only
  bf16* f = reinterpret_cast<bf16*>(base + bk->plan.off[B_F]);
  bf16* y2 = reinterpret_cast<bf16*>(base + bk->plan.off[B_Y2]);   // encoder only
  const int H = c->hidden, F = c->ffn, nh = c->n_heads, d = H / nh;
  const int act = c->gelu == RM_GELU_TANH ? 2 : 1;
  const bool dec = c->arch == RM_DEC_PRELN;
  const float eps = c->ln_eps;
  const bool prof_on = h->prof_every > 0 && (h->calls % h->prof_every) == 0;
  ++h->calls;
  // the launch sequence below overlaps each kernel's launch with its predecessor
  PdlScope pdl(true);

  // algorithmic work of each launch (unpadded tokens; attention entries that
  // the mask admits: L*L per head, or L*(L+1)/2 when causal)
  const double att = ci.att;
  const double Td = T, Hd = H, Fd = F;
  auto gemm_flops = [&](double N, double K) { return 2.0 * Td * N * K; };
  auto gemm_bytes = [&](double N, double K, double out_bytes = 2.0) {
    return 2.0 * (Td * K + N * K) + out_bytes * Td * N;
  };
  const double att_flops = 2.0 * att * d;            // one of the two contractions
  const double sm_bytes = 4.0 * att;                 // bf16 read + write per admitted entry
  const double ctx_bytes = 2.0 * att + 2.0 * Td * Hd * 2;   // P, V, ctx

  // weights of the next GEMMs to pull into L2 during the latency-bound kernels
  // before them (skipped when they would crowd out the activations)
  const unsigned long long pf_cap = 32ull << 20;
  auto pf_of = [&](const void* a, unsigned long long na, const void* b, unsigned long long nb) {
    L2Prefetch p;
    if (na + nb > pf_cap) return p;
    p.ptr[0] = a;
    p.bytes[0] = na;
    p.ptr[1] = b;
    p.bytes[1] = nb;
    return p;
  };
  const unsigned long long w_qkv_b = 2ull * 3 * H * H, w_o_b = 2ull * H * H, w_1_b = 2ull * F * H,
                           w_2_b = 2ull * H * F;
  const L2Prefetch pf_qkv0 = pf_of(h->layers[0].w_qkv, w_qkv_b, nullptr, 0);
  // the decoder keeps its residual stream x and the sublayer outputs y in
  // fp32 (LayerNorm row dtype 3: y and x fp32, z bf16); the encoder's x is
  // the bf16 LayerNorm output
  const int ln_dtype = dec ? 3 : 1;
  RM_KERNEL(RM_K_EMBED, 0, (dec ? 8.0 : 6.0) * Td * Hd + 4.0 * Td,
            embed_launch(d_ids, d_off, n, T, h->emb_word, h->emb_pos, dec ? nullptr : h->ln_emb_g,
                         dec ? nullptr : h->ln_emb_b, eps, c->vocab, c->max_pos, H, x,
                         h->d_err + ERR_CLAMPED, st, dec ? L2Prefetch{} : pf_qkv0, d_pln,
                         dec ? 0 : 1));
  if (dec)
    RM_KERNEL(RM_K_LAYERNORM, 0, 6.0 * Td * Hd,
              res_ln_launch(nullptr, x, z, h->layers[0].ln1_g, h->layers[0].ln1_b, T, H, eps,
                            ln_dtype, 2, st, pf_qkv0));
  // algorithmic bytes per token: post-LN reads y, x and writes x (bf16); the
  // decoder reads x (fp32, the sublayer output already added) and writes z (bf16)
  const double ln_bytes = 6.0 * Td * Hd;
  for (int l = 0; l < c->n_layers; ++l) {
    const LayerW& L = h->layers[l];
    const L2Prefetch pf_o = pf_of(L.w_o, w_o_b, nullptr, 0);
    const L2Prefetch pf_ffn = pf_of(L.w_1, w_1_b, L.w_2, w_2_b);
    const L2Prefetch pf_next =
        l + 1 < c->n_layers ? pf_of(h->layers[l + 1].w_qkv, w_qkv_b, nullptr, 0) : L2Prefetch{};
    RM_GEMM(gemm_flops(3 * Hd, Hd), gemm_bytes(3 * Hd, Hd),
            gemm(h, bk->a_in, L.tm[0], T, 3 * H, H, L.b_qkv, bk->y_qkv, 0, st));
    if (px != nullptr) {
      RM_KERNEL(RM_K_ATTN_FUSED, 2.0 * att_flops, 2.0 * Td * 3 * Hd + 2.0 * Td * Hd,
                attn_fused_prefix_launch(qkv, ctx, d_off, d_rb, d_pst, d_pln, n, nrb, nh, d, st, pf_o));
    } else if (ci.ntc > 0) {
      // tensor-core attention on tiles of whole sequences (head dim 64, L <= 128)
      RM_KERNEL(RM_K_ATTN_FUSED, 2.0 * att_flops, 2.0 * Td * 3 * Hd + 2.0 * Td * Hd,
                attn_tc_launch(qkv, ctx, d_off, ci.d_tl, ci.ntc, n, T, nh, dec, h->d_err,
                               h->num_sms, st, pf_o));
    } else if (ci.ntcl > 0) {
      // its long-row form: 128-row query tiles of one sequence (head dim 64, L <= 512)
      RM_KERNEL(RM_K_ATTN_FUSED, 2.0 * att_flops, 2.0 * Td * 3 * Hd + 2.0 * Td * Hd,
                attn_tcl_launch(qkv, ctx, d_off, ci.d_tl, ci.ntcl, n, T, nh, dec, h->d_err,
                                h->num_sms, st, pf_o));
    } else if (c->attn_impl == RM_ATTN_FUSED && (d == 64 || d == 128)) {
      // packed-row tiles (head dims 64 and 128); other head dims below
      RM_KERNEL(RM_K_ATTN_FUSED, 2.0 * att_flops, 2.0 * Td * 3 * Hd + 2.0 * Td * Hd,
                attn_tile_launch(qkv, ctx, d_off, n, T, nh, d, Lmax, dec, h->d_err, h->num_sms,
                                 st, pf_o));
    } else if (c->attn_impl == RM_ATTN_FUSED) {
      RM_KERNEL(RM_K_ATTN_FUSED, 2.0 * att_flops, 2.0 * Td * 3 * Hd + 2.0 * Td * Hd,
                attn_fused_launch(qkv, ctx, d_off, d_rb, n, nrb, nh, d, dec, st, pf_o));
    } else {
      RM_KERNEL(RM_K_SCORES, att_flops, 2.0 * Td * Hd * 2 + 2.0 * att,
                attn_scores_launch(qkv, s, d_off, d_rb, d_so, n, nrb, nh, d, dec, st));
      RM_KERNEL(RM_K_SOFTMAX, 0, sm_bytes,
                softmax_classes_launch(s, 1, d_off, d_so, n, T, nh, Lmax, dec, h->d_sm_scratch,
                                       h->num_sms, st));
      RM_KERNEL(RM_K_CONTEXT, att_flops, ctx_bytes,
                attn_context_launch(s, qkv, ctx, d_off, d_rb, d_so, n, nrb, nh, d, dec, st));
    }
    if (!dec) {
      RM_GEMM(gemm_flops(Hd, Hd), gemm_bytes(Hd, Hd),
              gemm(h, bk->a_ctx, L.tm[1], T, H, H, L.b_o, bk->y_o, 0, st));
      RM_KERNEL(RM_K_LAYERNORM, 0, ln_bytes,
                res_ln_launch(y1, x, nullptr, L.ln1_g, L.ln1_b, T, H, eps, ln_dtype, 0, st, pf_ffn));
      RM_GEMM(gemm_flops(Fd, Hd), gemm_bytes(Fd, Hd),
              gemm(h, bk->a_in, L.tm[2], T, F, H, L.b_1, bk->y_f, act, st));
      RM_GEMM(gemm_flops(Hd, Fd), gemm_bytes(Hd, Fd),
              gemm(h, bk->a_f, L.tm[3], T, H, F, L.b_2, bk->y_2, 0, st));
      RM_KERNEL(RM_K_LAYERNORM, 0, ln_bytes,
                res_ln_launch(y2, x, nullptr, L.ln2_g, L.ln2_b, T, H, eps, ln_dtype, 0, st, pf_next));
    } else {
      // The output projection and FFN2 add their outputs straight into the
      // fp32 residual stream x (in L2, each sum rounded once to fp32, as the
      // separate addition would round it); the LayerNorm after each reads x.
      RM_GEMM(gemm_flops(Hd, Hd), gemm_bytes(Hd, Hd, 8.0),
              gemm(h, bk->a_ctx, L.tm[1], T, H, H, L.b_o, bk->y_o, 0, st, true, x));
      RM_KERNEL(RM_K_LAYERNORM, 0, ln_bytes,
                res_ln_launch(nullptr, x, z, L.ln2_g, L.ln2_b, T, H, eps, ln_dtype, 2, st, pf_ffn));
      RM_GEMM(gemm_flops(Fd, Hd), gemm_bytes(Fd, Hd),
              gemm(h, bk->a_in, L.tm[2], T, F, H, L.b_1, bk->y_f, act, st));
      RM_GEMM(gemm_flops(Hd, Fd), gemm_bytes(Hd, Fd, 8.0),
              gemm(h, bk->a_f, L.tm[3], T, H, F, L.b_2, bk->y_2, 0, st, true, x));
      const bool last = l + 1 == c->n_layers;
      const float* g = last ? h->lnf_g : h->layers[l + 1].ln1_g;
      const float* b = last ? h->lnf_b : h->layers[l + 1].ln1_b;
      RM_KERNEL(RM_K_LAYERNORM, 0, ln_bytes,
                res_ln_launch(nullptr, x, z, g, b, T, H, eps, ln_dtype, 2, st, pf_next));
    }
  }
  RM_KERNEL(RM_K_HEAD, 2.0 * n * Hd, 2.0 * n * Hd + 4.0 * n,
            head_launch(dec ? z : x, d_off, n, h->w_r, h->b_r, H, dec ? 1 : 0, d_out, st, d_oix));
  if (px != nullptr && (px->d_best != nullptr || px->d_logodds != nullptr))
    RM_KERNEL(RM_K_HEAD, 0, 4.0 * px->group_off[px->n_groups] + 8.0 * px->n_groups,
              best_of_n_launch(d_out, d_gof, px->n_groups, px->d_best, px->d_logodds, st));
  h->last_stream = st;
  return RM_OK;
}

// Arena, error words, pinned metadata ring and its events of one handle.
int alloc_runtime(rm_handle* h) {
  const rm_config* cfg = &h->cfg;
  const int64_t T = cfg->max_tokens;
  const int64_t Lp = align_up(cfg->max_len, 8);
  const int64_t Smax = static_cast<int64_t>(cfg->n_heads) * T * Lp;
  const MetaLayout ml(cfg->max_batch_seqs);
  h->meta_bytes = align_up(ml.bytes, 256);
  // fixed part: metadata | ids (rm_score_host) | scores (rm_score_host) |
  // the materialised softmax's row index (none with the fused attention)
  const int64_t sm_scratch =
      cfg->attn_impl == RM_ATTN_FUSED
          ? 0
          : align_up(static_cast<int64_t>(softmax_classes_scratch_bytes(cfg->max_batch_seqs,
                                                                        static_cast<int>(T),
                                                                        cfg->n_heads)), 256);
  h->fixed_bytes = h->meta_bytes + align_up(4 * T, 256) + align_up(4 * cfg->max_batch_seqs, 256) +
                   sm_scratch;
  const int64_t Sres =
      cfg->attn_impl == RM_ATTN_FUSED ? 0 : align_up(std::max<int64_t>(Smax, 1), 65536);
  h->arena_bytes =
      h->fixed_bytes + arena_bound(cfg->arch, cfg->hidden, cfg->ffn, align_up(T, 128), Sres);
  cudaError_t e = dev_malloc(reinterpret_cast<void**>(&h->arena), h->arena_bytes);
  if (e == cudaSuccess) e = dev_malloc(reinterpret_cast<void**>(&h->d_err), ERR_WORDS * sizeof(int32_t));
  if (e == cudaSuccess) e = cudaMemset(h->d_err, 0, ERR_WORDS * sizeof(int32_t));
  if (e == cudaSuccess)
    e = pinned_malloc(reinterpret_cast<void**>(&h->pinned), static_cast<size_t>(kSlots) * h->meta_bytes);
  for (int k = 0; k < kSlots && e == cudaSuccess; ++k)
    e = cudaEventCreateWithFlags(&h->ev[k], cudaEventDisableTiming);
  if (e != cudaSuccess)
    return set_error(e == cudaErrorMemoryAllocation ? RM_E_NOMEM : RM_E_CUDA, "create: %s",
                     cudaGetErrorString(e));
  h->d_meta = h->arena;
  h->d_ids = reinterpret_cast<int32_t*>(h->arena + h->meta_bytes);
  h->d_scores = reinterpret_cast<float*>(h->arena + h->meta_bytes + align_up(4 * T, 256));
  h->d_sm_scratch = h->arena + h->meta_bytes + align_up(4 * T, 256) +
                    align_up(4 * cfg->max_batch_seqs, 256);
  h->planned = h->arena + h->fixed_bytes;
  return RM_OK;
}

}  // namespace

extern "C" {

const char* rm_last_error(void) { return g_msg; }

int rm_debug_fail_alloc(int32_t k) {
  if (k < 0) return set_error(RM_E_INVAL, "k must be >= 0");
  g_fail_alloc.store(k);
  return RM_OK;
}

size_t rm_weights_bytes(const rm_config* cfg) {
  const char* why = "";
  if (validate_config(cfg, false, &why) != RM_OK) return 0;
  int64_t total = 0;
  for (const auto& s : segments(cfg)) total += s.elems;
  return static_cast<size_t>(total) * (cfg->weight_dtype == RM_F32 ? 4 : 2);
}

int rm_create(const rm_config* cfg, const void* weights, size_t weights_bytes, rm_handle** out) {
  g_msg[0] = '\0';
  const char* why = "";
  if (out == nullptr || weights == nullptr) return set_error(RM_E_INVAL, "NULL argument");
  if (validate_config(cfg, false, &why) != RM_OK) return set_error(RM_E_INVAL, "%s", why);
  const size_t need = rm_weights_bytes(cfg);
  if (weights_bytes != need)
    return set_error(RM_E_INVAL, "weights_bytes is %zu, the layout needs %zu", weights_bytes, need);
  int dev = 0, ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0)
    return set_error(RM_E_DEVICE, "no CUDA device");
  RM_CUDA(cudaGetDevice(&dev));
  cudaDeviceProp prop;
  RM_CUDA(cudaGetDeviceProperties(&prop, dev));
  if (prop.major != 10)
    return set_error(RM_E_DEVICE, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                     prop.major, prop.minor);
  rm_handle* h = new rm_handle();
  h->cfg = *cfg;
  h->cfg.sched_table = nullptr;   // the handle keeps its own copy in sched
  h->sched = sched_cost_from(cfg);
  h->device = dev;
  h->num_sms = prop.multiProcessorCount;
  int rc = upload_weights(h, weights);
  if (h->wbuf != nullptr) h->weights_owner = std::shared_ptr<void>(h->wbuf, [](void* p) { cudaFree(p); });
  if (rc == RM_OK) rc = alloc_runtime(h);
  if (rc != RM_OK) {
    rm_destroy(h);
    return rc;
  }
  *out = h;
  return RM_OK;
}

int rm_create_shared(const rm_handle* base, rm_handle** out) {
  g_msg[0] = '\0';
  if (base == nullptr || out == nullptr) return set_error(RM_E_INVAL, "NULL argument");
  int dev = 0;
  RM_CUDA(cudaGetDevice(&dev));
  if (dev != base->device)
    return set_error(RM_E_INVAL, "the current device (%d) is not the base handle's (%d)", dev,
                     base->device);
  rm_handle* h = new rm_handle();
  h->cfg = base->cfg;
  h->sched = base->sched;
  h->device = base->device;
  h->num_sms = base->num_sms;
  h->wbuf = base->wbuf;
  h->weights_owner = base->weights_owner;
  h->emb_word = base->emb_word;
  h->emb_pos = base->emb_pos;
  h->ln_emb_g = base->ln_emb_g;
  h->ln_emb_b = base->ln_emb_b;
  h->lnf_g = base->lnf_g;
  h->lnf_b = base->lnf_b;
  h->w_r = base->w_r;
  h->b_r = base->b_r;
  h->layers = base->layers;      // tensor maps of the same (shared) weight matrices
  const int rc = alloc_runtime(h);
  if (rc != RM_OK) {
    rm_destroy(h);
    return rc;
  }
  *out = h;
  return RM_OK;
}

int rm_score(rm_handle* h, const int32_t* packed_token_ids, const int32_t* seq_offsets,
             int32_t n_seqs, float* out_scores, void* stream) {
  if (h == nullptr || packed_token_ids == nullptr || seq_offsets == nullptr || out_scores == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  return score_impl(h, packed_token_ids, nullptr, seq_offsets, n_seqs, out_scores, nullptr,
                    static_cast<cudaStream_t>(stream));
}

int rm_score_prefix(rm_handle* h, const int32_t* packed_token_ids, const int32_t* prefix_len,
                    const int32_t* n_cand, const int32_t* cand_len, int32_t n_groups,
                    float* out_scores, int32_t* out_best, float* out_logodds, void* stream) {
  if (h == nullptr || packed_token_ids == nullptr || prefix_len == nullptr || n_cand == nullptr ||
      cand_len == nullptr || out_scores == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  const rm_config* c = &h->cfg;
  if (c->arch != RM_DEC_PRELN)
    return set_error(RM_E_INVAL, "prefix sharing needs the causal decoder: an encoder's prefix "
                                 "tokens attend to the candidate");
  if ((c->hidden / c->n_heads) % 8 != 0)
    return set_error(RM_E_INVAL, "prefix sharing needs head_dim %% 8 == 0");
  if (n_groups < 1) return set_error(RM_E_INVAL, "n_groups must be >= 1");
  h->px_off.assign(1, 0);
  h->px_start.clear();
  h->px_len.clear();
  h->px_out.clear();
  h->px_goff.assign(1, 0);
  int64_t tok = 0;
  int32_t slot = 0, k = 0;
  for (int32_t g = 0; g < n_groups; ++g) {
    const int32_t P = prefix_len[g];
    if (P < 0 || n_cand[g] < 1)
      return set_error(RM_E_INVAL, "group %d: prefix length %d, %d candidates", g, P, n_cand[g]);
    const int64_t pstart = tok;
    if (P > 0) {   // the prefix itself: one causal segment, not scored
      tok += P;
      h->px_off.push_back(static_cast<int32_t>(std::min<int64_t>(tok, INT32_MAX)));
      h->px_start.push_back(0);
      h->px_len.push_back(0);
      h->px_out.push_back(-1);
    }
    for (int32_t j = 0; j < n_cand[g]; ++j, ++k) {
      const int32_t l = cand_len[k];
      if (l < 1) return set_error(RM_E_INVAL, "candidate %d of group %d has length %d", j, g, l);
      if (static_cast<int64_t>(P) + l > c->max_pos)
        return set_error(RM_E_RANGE, "group %d candidate %d: %lld positions exceed max_pos %d", g,
                         j, (long long)P + l, c->max_pos);
      tok += l;
      h->px_off.push_back(static_cast<int32_t>(std::min<int64_t>(tok, INT32_MAX)));
      h->px_start.push_back(static_cast<int32_t>(pstart));
      h->px_len.push_back(P);
      h->px_out.push_back(slot++);
    }
    h->px_goff.push_back(slot);
    if (tok > c->max_tokens) return set_error(RM_E_RANGE, "%lld tokens exceed max_tokens %d",
                                              (long long)tok, c->max_tokens);
  }
  const int32_t n = static_cast<int32_t>(h->px_start.size());
  PrefixSpec px{h->px_start.data(), h->px_len.data(), h->px_out.data(), h->px_goff.data(),
                n_groups, out_best, out_logodds};
  return score_impl(h, packed_token_ids, nullptr, h->px_off.data(), n, out_scores, nullptr,
                    static_cast<cudaStream_t>(stream), &px);
}

struct rm_plan {
  rm_handle* h = nullptr;
  CallInfo ci;
  uint8_t* d_meta = nullptr;
};

int rm_plan_create(rm_handle* h, const int32_t* seq_offsets, int32_t n_seqs, rm_plan** out) {
  if (h == nullptr || seq_offsets == nullptr || out == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  const rm_config* c = &h->cfg;
  const int32_t n = n_seqs;
  if (n < 1) return set_error(RM_E_INVAL, "n_seqs must be >= 1");
  if (n > c->max_batch_seqs)
    return set_error(RM_E_RANGE, "n_seqs %d exceeds max_batch_seqs %d", n, c->max_batch_seqs);
  if (seq_offsets[0] != 0) return set_error(RM_E_INVAL, "seq_offsets[0] must be 0");
  for (int32_t i = 0; i < n; ++i) {
    const int64_t L = static_cast<int64_t>(seq_offsets[i + 1]) - seq_offsets[i];
    if (L < 1) return set_error(RM_E_INVAL, "sequence %d has length %lld (< 1)", i, (long long)L);
    if (L > c->max_len)
      return set_error(RM_E_RANGE, "sequence %d has length %lld > max_len %d", i, (long long)L,
                       c->max_len);
  }
  const int32_t T = seq_offsets[n];
  if (T > c->max_tokens)
    return set_error(RM_E_RANGE, "%d tokens exceed max_tokens %d", T, c->max_tokens);
  const MetaLayout ml(n);
  std::vector<uint8_t> meta(static_cast<size_t>(ml.base));
  int32_t* p_off = reinterpret_cast<int32_t*>(meta.data());
  int32_t* p_rb = reinterpret_cast<int32_t*>(meta.data() + ml.rb);
  int64_t* p_so = reinterpret_cast<int64_t*>(meta.data() + ml.so);
  std::memcpy(p_off, seq_offsets, 4 * static_cast<size_t>(n + 1));
  int32_t Lmax = 0;
  RM_TRY(host_varlen_meta(seq_offsets, n, c->n_heads, p_rb, p_so, &Lmax));
  const int32_t ntc = tc_attention_applies(c, Lmax, false)
                          ? attn_tc_tiles(seq_offsets, n, reinterpret_cast<int32_t*>(meta.data() + ml.tl))
                          : 0;
  const int32_t ntcl = tcl_attention_applies(c, Lmax, false)
                           ? attn_tcl_items(seq_offsets, n, c->arch == RM_DEC_PRELN ? 1 : 0,
                                            reinterpret_cast<int32_t*>(meta.data() + ml.tl))
                           : 0;
  Bucket* bk = nullptr;
  RM_TRY(get_bucket(h, T, p_so[n], &bk));   // the arena placement and tensor maps, made now
  rm_plan* p = new rm_plan();
  p->h = h;
  cudaError_t e = dev_malloc(reinterpret_cast<void**>(&p->d_meta), ml.base);
  if (e == cudaSuccess) e = cudaMemcpy(p->d_meta, meta.data(), ml.base, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(p->d_meta);
    delete p;
    return set_error(e == cudaErrorMemoryAllocation ? RM_E_NOMEM : RM_E_CUDA, "plan: %s",
                     cudaGetErrorString(e));
  }
  CallInfo& ci = p->ci;
  ci.n = n;
  ci.T = T;
  ci.nrb = p_rb[n];
  ci.Lmax = Lmax;
  ci.ntc = ntc;
  ci.ntcl = ntcl;
  ci.d_tl = reinterpret_cast<const int32_t*>(p->d_meta + ml.tl);
  ci.S = p_so[n];
  ci.att = attention_entries(c, seq_offsets, n, nullptr);
  ci.d_off = reinterpret_cast<const int32_t*>(p->d_meta);
  ci.d_rb = reinterpret_cast<const int32_t*>(p->d_meta + ml.rb);
  ci.d_so = reinterpret_cast<const int64_t*>(p->d_meta + ml.so);
  *out = p;
  return RM_OK;
}

int rm_score_plan(rm_plan* p, const int32_t* packed_token_ids, float* out_scores, void* stream) {
  if (p == nullptr || packed_token_ids == nullptr || out_scores == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  return enqueue_forward(p->h, p->ci, packed_token_ids, out_scores, static_cast<cudaStream_t>(stream));
}

void rm_plan_destroy(rm_plan* p) {
  if (p == nullptr) return;
  cudaFree(p->d_meta);
  delete p;
}

int rm_score_host(rm_handle* h, const int32_t* host_token_ids, const int32_t* seq_offsets,
                  int32_t n_seqs, float* host_scores, void* stream) {
  if (h == nullptr || host_token_ids == nullptr || seq_offsets == nullptr || host_scores == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  return score_impl(h, nullptr, host_token_ids, seq_offsets, n_seqs, nullptr, host_scores,
                    static_cast<cudaStream_t>(stream));
}

int rm_schedule_cfg(const rm_config* cfg, const int32_t* lengths, int32_t n, int32_t* out_batches) {
  const char* why = "";
  if (validate_config(cfg, true, &why) != RM_OK) return set_error(RM_E_INVAL, "%s", why);
  if (n < 0) return set_error(RM_E_INVAL, "n must be >= 0");
  if (n > 0 && (lengths == nullptr || out_batches == nullptr))
    return set_error(RM_E_INVAL, "NULL argument");
  for (int32_t i = 0; i < n; ++i)
    if (lengths[i] < 1 || lengths[i] > cfg->max_len)
      return set_error(RM_E_RANGE, "length %d of request %d outside 1..max_len", lengths[i], i);
  if (n == 0) return 0;
  return schedule_dp(sched_cost_from(cfg), lengths, n, out_batches);
}

int rm_schedule(const rm_handle* h, const int32_t* lengths, int32_t n, int32_t* out_batches) {
  if (h == nullptr) return set_error(RM_E_INVAL, "NULL handle");
  if (n < 0) return set_error(RM_E_INVAL, "n must be >= 0");
  if (n > 0 && (lengths == nullptr || out_batches == nullptr))
    return set_error(RM_E_INVAL, "NULL argument");
  for (int32_t i = 0; i < n; ++i)
    if (lengths[i] < 1 || lengths[i] > h->cfg.max_len)
      return set_error(RM_E_RANGE, "length %d of request %d outside 1..max_len", lengths[i], i);
  if (n == 0) return 0;
  return schedule_dp(h->sched, lengths, n, out_batches);
}

int rm_get_device_error(rm_handle* h, int32_t* out) {
  if (h == nullptr || out == nullptr) return set_error(RM_E_INVAL, "NULL argument");
  RM_CUDA(cudaStreamSynchronize(h->last_stream));
  RM_CUDA(cudaMemcpy(out, h->d_err, ERR_WORDS * sizeof(int32_t), cudaMemcpyDeviceToHost));
  return RM_OK;
}

int rm_build_checked(void) { return RMK_CHECKED; }

int rm_bounds_errors(int64_t* out) {
  if (out == nullptr) return set_error(RM_E_INVAL, "NULL argument");
  int32_t a = 0, b = 0, c = 0;
  RM_CUDA(cudaDeviceSynchronize());
  RM_CUDA(bounds_errors_rowops(&a, true));
  RM_CUDA(bounds_errors_attention(&b, true));
  RM_CUDA(bounds_errors_attention_tc(&c, true));
  *out = static_cast<int64_t>(a) + b + c;
  return RM_OK;
}

int rm_profile(rm_handle* h, int32_t every) {
  if (h == nullptr || every < 0) return set_error(RM_E_INVAL, "bad argument");
  for (auto& r : h->prof) {
    h->ev_pool.push_back(r.a);
    h->ev_pool.push_back(r.b);
  }
  h->prof.clear();
  h->prof_every = every;
  h->calls = 0;
  return RM_OK;
}

int rm_profile_read(rm_handle* h, double* out_ms, int64_t* out_launches, double* out_flops,
                    double* out_bytes, int64_t* out_total_launches) {
  if (h == nullptr || out_ms == nullptr || out_launches == nullptr || out_flops == nullptr ||
      out_bytes == nullptr || out_total_launches == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  RM_CUDA(cudaStreamSynchronize(h->last_stream));
  for (int k = 0; k < RM_K_CLASSES; ++k) {
    out_ms[k] = 0;
    out_launches[k] = 0;
    out_flops[k] = 0;
    out_bytes[k] = 0;
  }
  for (const auto& r : h->prof) {
    float ms = 0;
    RM_CUDA(cudaEventElapsedTime(&ms, r.a, r.b));
    out_ms[r.cls] += ms;
    out_launches[r.cls] += 1;
    out_flops[r.cls] += r.flops;
    out_bytes[r.cls] += r.bytes;
  }
  *out_total_launches = h->launches;
  return RM_OK;
}

int rm_selftest_bounded_wait(int64_t limit_ns, int32_t* out_timed_out, int64_t* out_elapsed_ns) {
  if (out_timed_out == nullptr || out_elapsed_ns == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  if (limit_ns < 1000 || limit_ns > 10000000000LL)
    return set_error(RM_E_INVAL, "limit_ns must be in 1e3 .. 1e10");
  void* d = nullptr;
  RM_CUDA(cudaMalloc(&d, 16));
  int* d_flag = static_cast<int*>(d);
  unsigned long long* d_ns = reinterpret_cast<unsigned long long*>(static_cast<char*>(d) + 8);
  cudaError_t e = cudaMemset(d, 0, 16);
  if (e == cudaSuccess)
    e = bounded_wait_selftest(static_cast<unsigned long long>(limit_ns), d_flag, d_ns, nullptr);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  int flag = 0;
  unsigned long long ns = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&flag, d_flag, sizeof flag, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(&ns, d_ns, sizeof ns, cudaMemcpyDeviceToHost);
  cudaFree(d);
  if (e != cudaSuccess) return set_error(RM_E_CUDA, "self-test: %s", cudaGetErrorString(e));
  *out_timed_out = flag;
  *out_elapsed_ns = static_cast<int64_t>(ns);
  return RM_OK;
}

int rm_arena_stats(const rm_handle* h, int64_t* out) {
  if (h == nullptr || out == nullptr) return set_error(RM_E_INVAL, "NULL argument");
  out[0] = h->arena_bytes;
  out[1] = h->fixed_bytes + h->max_peak;
  out[2] = static_cast<int64_t>(h->buckets.size());
  return RM_OK;
}

void rm_destroy(rm_handle* h) {
  if (h == nullptr) return;
  if (h->last_stream != nullptr || h->arena != nullptr) cudaStreamSynchronize(h->last_stream);
  for (int k = 0; k < kSlots; ++k)
    if (h->ev[k]) cudaEventDestroy(h->ev[k]);
  for (auto& r : h->prof) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (auto e : h->ev_pool) cudaEventDestroy(e);
  if (h->pinned) cudaFreeHost(h->pinned);
  if (h->d_err) cudaFree(h->d_err);
  if (h->arena) cudaFree(h->arena);
  if (h->wbuf && !h->weights_owner) cudaFree(h->wbuf);   // upload failed before ownership
  delete h;                                                // drops this handle's weight reference
}

// ---------------------------------------------------------------------------
// rm_ops.h
// ---------------------------------------------------------------------------

int rm_varlen_meta(const int32_t* offsets, int32_t n, int32_t n_heads, int32_t* rb_off,
                   int64_t* s_off) {
  if (offsets == nullptr || rb_off == nullptr || s_off == nullptr || n < 0 || n_heads < 1)
    return set_error(RM_E_INVAL, "bad argument");
  return host_varlen_meta(offsets, n, n_heads, rb_off, s_off, nullptr);
}

int rm_op_gemm(const void* x, const void* w, const float* bias, void* y, int32_t y_dtype,
               int32_t M, int32_t N, int32_t K, int32_t act, void* stream) {
  return rm_op_gemm_tiled(x, w, bias, y, y_dtype, M, N, K, act, 0, 0, stream);
}

namespace {
// rm_op_gemm_tiled and rm_op_gemm_accumulate: store the product into y, or
// add it to y
int op_gemm(const void* x, const void* w, const float* bias, void* y, int32_t y_dtype, int32_t M,
            int32_t N, int32_t K, int32_t act, int32_t cg, int32_t bn, bool accumulate,
            void* stream) {
  if (x == nullptr || w == nullptr || y == nullptr) return set_error(RM_E_INVAL, "NULL argument");
  if (M < 1 || N < 8 || K < 8 || N % 8 != 0 || K % 8 != 0)
    return set_error(RM_E_INVAL, "need M >= 1 and N, K positive multiples of 8");
  if (act < 0 || act > 2 || (y_dtype != RM_F32 && y_dtype != RM_BF16) ||
      (accumulate && (act != 0 || y_dtype != RM_F32)))
    return set_error(RM_E_INVAL, "bad act or y_dtype");
  if ((reinterpret_cast<uintptr_t>(y) & 15) != 0 || (reinterpret_cast<uintptr_t>(bias) & 15) != 0)
    return set_error(RM_E_INVAL, "y and bias must be 16-byte aligned");
  if (cg != 0) {
    bool known = false;
    if (cg == 1)
      for (int i = 0; i < kGemmTileCount; ++i) known = known || kGemmTileWidths[i] == bn;
    if (cg == 2) known = bn == 128 || bn == 192 || bn == 256;
    if (!known) return set_error(RM_E_INVAL, "no %d-CTA tile of width %d", cg, bn);
  }
  int dev = 0, sms = 148;
  RM_CUDA(cudaGetDevice(&dev));
  RM_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const GemmTile tile = cg != 0 ? GemmTile{cg, bn} : gemm_pick(M, N, K, sms, act);
  const int split = gemm_tail_split(tile, M, N, sms);
  CUtensorMap ta, tb, tbs, ty;
  const char* why = "";
  if (!make_tmap_bf16(&ta, x, M, K, 128, &why) || !make_tmap_bf16(&tb, w, N, K, tile.b_box(), &why) ||
      !make_tmap_bf16(&tbs, w, N, K, tile.b_box() / split, &why) ||
      !make_tmap_store(&ty, y, M, N, y_dtype == RM_F32, &why))
    return set_error(RM_E_INVAL, "tensor map: %s", why);
  int32_t* err = nullptr;
  RM_CUDA(cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_err_sink));
  RM_LAUNCH(gemm_launch(ta, tb, tbs, ty, accumulate ? y : nullptr, tile, M, N, K, bias,
                        y_dtype == RM_F32, act, err, sms, static_cast<cudaStream_t>(stream)));
  return RM_OK;
}
}  // namespace

int rm_op_gemm_tiled(const void* x, const void* w, const float* bias, void* y, int32_t y_dtype,
                     int32_t M, int32_t N, int32_t K, int32_t act, int32_t cg, int32_t bn,
                     void* stream) {
  return op_gemm(x, w, bias, y, y_dtype, M, N, K, act, cg, bn, false, stream);
}

int rm_op_gemm_accumulate(const void* x, const void* w, const float* bias, void* y,
                          int32_t y_dtype, int32_t M, int32_t N, int32_t K, int32_t act,
                          int32_t cg, int32_t bn, void* stream) {
  return op_gemm(x, w, bias, y, y_dtype, M, N, K, act, cg, bn, true, stream);
}

int rm_op_vote(const float* scores, int32_t K, int32_t n, float threshold, int32_t* decision,
               int32_t* votes, void* stream) {
  if (scores == nullptr || K < 1 || n < 0) return set_error(RM_E_INVAL, "bad arguments");
  RM_LAUNCH(vote_launch(scores, K, n, threshold, decision, votes, static_cast<cudaStream_t>(stream)));
  return RM_OK;
}

int rm_gemm_tile(int32_t M, int32_t N, int32_t K, int32_t num_sms, int32_t* out) {
  if (out == nullptr || M < 1 || N < 1 || K < 1 || num_sms < 1)
    return set_error(RM_E_INVAL, "bad arguments");
  const GemmTile t = gemm_pick(M, N, K, num_sms);
  out[0] = t.cg;
  out[1] = t.bn;
  return RM_OK;
}

int rm_op_embed(const int32_t* ids, const int32_t* offsets, int32_t n_seqs, int32_t T,
                const void* emb_word, const void* emb_pos, const float* ln_g, const float* ln_b,
                float eps, int32_t V, int32_t P, int32_t H, void* x, int32_t x_dtype,
                int32_t* err_count, void* stream) {
  if (ids == nullptr || offsets == nullptr || emb_word == nullptr || emb_pos == nullptr || x == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  if (n_seqs < 1 || T < 0 || V < 1 || P < 1 || H < 8 || H % 8 != 0 || H > 4096)
    return set_error(RM_E_INVAL, "bad sizes");
  if (x_dtype != RM_F32 && x_dtype != RM_BF16) return set_error(RM_E_INVAL, "bad x_dtype");
  if ((ln_g == nullptr) != (ln_b == nullptr)) return set_error(RM_E_INVAL, "ln_g and ln_b go together");
  RM_LAUNCH(embed_launch(ids, offsets, n_seqs, T, emb_word, emb_pos, ln_g, ln_b, eps, V, P, H, x,
                         err_count, static_cast<cudaStream_t>(stream), L2Prefetch{}, nullptr,
                         x_dtype));
  return RM_OK;
}

int rm_op_attn_scores(const void* qkv, void* S, const int32_t* offsets, const int32_t* rb_off,
                      const int64_t* s_off, int32_t n_seqs, int32_t n_row_blocks,
                      int32_t n_heads, int32_t head_dim, int32_t causal, void* stream) {
  if (qkv == nullptr || S == nullptr || offsets == nullptr || rb_off == nullptr || s_off == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  if (n_seqs < 1 || n_row_blocks < 0 || n_heads < 1 || head_dim < 2 || head_dim % 2 || head_dim > 128)
    return set_error(RM_E_INVAL, "bad sizes");
  RM_LAUNCH(attn_scores_launch(qkv, S, offsets, rb_off, s_off, n_seqs, n_row_blocks, n_heads,
                               head_dim, causal != 0, static_cast<cudaStream_t>(stream)));
  return RM_OK;
}

int rm_op_softmax(void* S, int32_t s_dtype, const int32_t* offsets, const int64_t* s_off,
                  int32_t n_seqs, int32_t T, int32_t n_heads, int32_t max_len, int32_t causal,
                  void* stream) {
  if (S == nullptr || offsets == nullptr || s_off == nullptr) return set_error(RM_E_INVAL, "NULL argument");
  if (n_seqs < 1 || T < 0 || n_heads < 1 || max_len < 1 || max_len > 1024 ||
      (s_dtype != RM_F32 && s_dtype != RM_BF16))
    return set_error(RM_E_INVAL, "bad sizes");
  RM_LAUNCH(softmax_launch(S, s_dtype, offsets, s_off, n_seqs, T, n_heads, max_len, causal != 0,
                           nullptr, static_cast<cudaStream_t>(stream)));
  return RM_OK;
}

int rm_op_attn_context(const void* S, const void* qkv, void* ctx, const int32_t* offsets,
                       const int32_t* rb_off, const int64_t* s_off, int32_t n_seqs,
                       int32_t n_row_blocks, int32_t n_heads, int32_t head_dim, int32_t causal,
                       void* stream) {
  if (S == nullptr || qkv == nullptr || ctx == nullptr || offsets == nullptr || rb_off == nullptr ||
      s_off == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  if (n_seqs < 1 || n_row_blocks < 0 || n_heads < 1 || head_dim < 2 || head_dim % 2 || head_dim > 128)
    return set_error(RM_E_INVAL, "bad sizes");
  RM_LAUNCH(attn_context_launch(S, qkv, ctx, offsets, rb_off, s_off, n_seqs, n_row_blocks, n_heads,
                                head_dim, causal != 0, static_cast<cudaStream_t>(stream)));
  return RM_OK;
}

int rm_op_attn_fused(const void* qkv, void* ctx, const int32_t* offsets, const int32_t* rb_off,
                     int32_t n_seqs, int32_t n_row_blocks, int32_t n_heads, int32_t head_dim,
                     int32_t causal, void* stream) {
  if (qkv == nullptr || ctx == nullptr || offsets == nullptr || rb_off == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  if (n_seqs < 1 || n_row_blocks < 0 || n_heads < 1 || head_dim < 2 || head_dim % 2 || head_dim > 128)
    return set_error(RM_E_INVAL, "bad sizes");
  RM_LAUNCH(attn_fused_launch(qkv, ctx, offsets, rb_off, n_seqs, n_row_blocks, n_heads, head_dim,
                              causal != 0, static_cast<cudaStream_t>(stream)));
  return RM_OK;
}

size_t rm_softmax_scratch_bytes(int32_t n_seqs, int32_t T, int32_t n_heads) {
  if (n_seqs < 0 || T < 0 || n_heads < 1) return 0;
  return softmax_classes_scratch_bytes(n_seqs, T, n_heads);
}

int rm_op_softmax_classes(void* S, int32_t s_dtype, const int32_t* offsets, const int64_t* s_off,
                          int32_t n_seqs, int32_t T, int32_t n_heads, int32_t max_len,
                          int32_t causal, void* scratch, void* stream) {
  if (S == nullptr || offsets == nullptr || s_off == nullptr || scratch == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  if (n_seqs < 1 || T < 1 || n_heads < 1 || max_len < 1 || max_len > 1024 ||
      (s_dtype != RM_F32 && s_dtype != RM_BF16))
    return set_error(RM_E_INVAL, "bad sizes");
  if ((reinterpret_cast<uintptr_t>(scratch) & 15) != 0)
    return set_error(RM_E_INVAL, "scratch must be 16-byte aligned");
  int dev = 0, sms = 0;
  RM_CUDA(cudaGetDevice(&dev));
  RM_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  RM_LAUNCH(softmax_classes_launch(S, s_dtype, offsets, s_off, n_seqs, T, n_heads, max_len,
                                   causal != 0, scratch, sms, static_cast<cudaStream_t>(stream)));
  return RM_OK;
}

int rm_op_attn_tiles(const void* qkv, void* ctx, const int32_t* offsets, int32_t n_seqs, int32_t T,
                     int32_t n_heads, int32_t head_dim, int32_t max_len, int32_t causal,
                     void* stream) {
  if (qkv == nullptr || ctx == nullptr || offsets == nullptr) return set_error(RM_E_INVAL, "NULL argument");
  if (n_seqs < 1 || T < 1 || n_heads < 1 || max_len < 1 || (head_dim != 64 && head_dim != 128))
    return set_error(RM_E_INVAL, "bad sizes (head_dim must be 64 or 128)");
  int dev = 0, sms = 0;
  RM_CUDA(cudaGetDevice(&dev));
  RM_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  int32_t* err = nullptr;
  RM_CUDA(cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_err_sink));
  RM_LAUNCH(attn_tile_launch(qkv, ctx, offsets, n_seqs, T, n_heads, head_dim, max_len, causal, err,
                             sms, static_cast<cudaStream_t>(stream)));
  return RM_OK;
}

int rm_attn_tc_tiles(const int32_t* offsets, int32_t n_seqs, int32_t* tiles) {
  if (offsets == nullptr || tiles == nullptr || n_seqs < 1) return set_error(RM_E_INVAL, "bad arguments");
  if (offsets[0] != 0) return set_error(RM_E_INVAL, "seq_offsets[0] must be 0");
  for (int32_t i = 0; i < n_seqs; ++i) {
    const int64_t L = static_cast<int64_t>(offsets[i + 1]) - offsets[i];
    if (L < 1 || L > 128)
      return set_error(RM_E_RANGE, "sequence %d has length %lld (tiles need 1..128)", i, (long long)L);
  }
  return attn_tc_tiles(offsets, n_seqs, tiles);
}

int rm_op_attn_tc(const void* qkv, void* ctx, const int32_t* offsets, const int32_t* tiles,
                  int32_t n_tiles, int32_t n_seqs, int32_t T, int32_t n_heads, int32_t causal,
                  void* stream) {
  if (qkv == nullptr || ctx == nullptr || offsets == nullptr || tiles == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  if (n_seqs < 1 || T < 1 || n_heads < 1 || n_tiles < 1 || n_tiles > n_seqs)
    return set_error(RM_E_INVAL, "bad sizes");
  int dev = 0, sms = 0;
  RM_CUDA(cudaGetDevice(&dev));
  RM_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  int32_t* err = nullptr;
  RM_CUDA(cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_err_sink));
  RM_LAUNCH(attn_tc_launch(qkv, ctx, offsets, tiles, n_tiles, n_seqs, T, n_heads, causal, err, sms,
                           static_cast<cudaStream_t>(stream)));
  return RM_OK;
}

int rm_attn_tcl_items(const int32_t* offsets, int32_t n_seqs, int32_t causal, int32_t* items) {
  if (offsets == nullptr || items == nullptr || n_seqs < 1) return set_error(RM_E_INVAL, "bad arguments");
  if (offsets[0] != 0) return set_error(RM_E_INVAL, "seq_offsets[0] must be 0");
  for (int32_t i = 0; i < n_seqs; ++i) {
    const int64_t L = static_cast<int64_t>(offsets[i + 1]) - offsets[i];
    if (L < 1 || L > 512)
      return set_error(RM_E_RANGE, "sequence %d has length %lld (items need 1..512)", i, (long long)L);
  }
  return attn_tcl_items(offsets, n_seqs, causal != 0 ? 1 : 0, items);
}

int rm_op_attn_tcl(const void* qkv, void* ctx, const int32_t* offsets, const int32_t* items,
                   int32_t n_items, int32_t n_seqs, int32_t T, int32_t n_heads, int32_t causal,
                   void* stream) {
  if (qkv == nullptr || ctx == nullptr || offsets == nullptr || items == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  if (n_seqs < 1 || T < 1 || n_heads < 1 || n_items < 1 || n_items > 4 * n_seqs)
    return set_error(RM_E_INVAL, "bad sizes");
  int dev = 0, sms = 0;
  RM_CUDA(cudaGetDevice(&dev));
  RM_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  int32_t* err = nullptr;
  RM_CUDA(cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_err_sink));
  RM_LAUNCH(attn_tcl_launch(qkv, ctx, offsets, items, n_items, n_seqs, T, n_heads, causal, err, sms,
                            static_cast<cudaStream_t>(stream)));
  return RM_OK;
}

int rm_op_res_ln(const void* y, void* x, void* z, const float* g, const float* b, int32_t T,
                 int32_t H, float eps, int32_t dtype, int32_t mode, void* stream) {
  if (x == nullptr || g == nullptr || b == nullptr) return set_error(RM_E_INVAL, "NULL argument");
  if (mode < 0 || mode > 2 || (mode != 2 && y == nullptr) || (mode != 0 && z == nullptr))
    return set_error(RM_E_INVAL, "bad mode or missing y/z");
  if (T < 0 || H < 8 || H % 8 != 0 || H > 4096 ||
      (dtype != RM_F32 && dtype != RM_BF16 && dtype != RM_ROWS_RESID_F32 &&
       dtype != RM_ROWS_F32_IN))
    return set_error(RM_E_INVAL, "bad sizes");
  RM_LAUNCH(res_ln_launch(y, x, z, g, b, T, H, eps, dtype, mode, static_cast<cudaStream_t>(stream)));
  return RM_OK;
}

int rm_op_head(const void* x, const int32_t* offsets, int32_t n_seqs, const float* w_r, float b_r,
               int32_t H, int32_t last_token, float* out, void* stream) {
  if (x == nullptr || offsets == nullptr || w_r == nullptr || out == nullptr)
    return set_error(RM_E_INVAL, "NULL argument");
  if (n_seqs < 0 || H < 8 || H % 8 != 0) return set_error(RM_E_INVAL, "bad sizes");
  RM_LAUNCH(head_launch(x, offsets, n_seqs, w_r, b_r, H, last_token != 0, out,
                        static_cast<cudaStream_t>(stream)));
  return RM_OK;
}

int rm_arena_plan(const void* cfgp, int32_t T, int32_t n_seqs, int64_t s_elems, int64_t* out_off,
                  int64_t* out_bytes, int32_t* out_first, int32_t* out_last, int32_t max_bufs,
                  int64_t* out_peak) {
  (void)n_seqs;
  const rm_config* cfg = static_cast<const rm_config*>(cfgp);
  const char* why = "";
  if (validate_config(cfg, false, &why) != RM_OK) return set_error(RM_E_INVAL, "%s", why);
  if (T < 0 || s_elems < 0 || out_off == nullptr || out_bytes == nullptr || out_first == nullptr ||
      out_last == nullptr || out_peak == nullptr)
    return set_error(RM_E_INVAL, "bad argument");
  const ArenaPlan p = plan_arena(cfg->arch, cfg->hidden, cfg->ffn, T, s_elems);
  const int nb = std::min<int>(B_COUNT, max_bufs);
  for (int k = 0; k < nb; ++k) {
    out_off[k] = p.off[k];
    out_bytes[k] = p.bytes[k];
    out_first[k] = p.first[k];
    out_last[k] = p.last[k];
  }
  *out_peak = p.peak;
  return B_COUNT;
}

}  // extern "C"
