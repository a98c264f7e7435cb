// Host-side structures of the scorer runtime (not exported).
#pragma once

#include <stdint.h>

#include <vector>

#include "../../include/rm.h"

namespace rmk {

// ---- DP scheduler cost model ----
struct SchedCost {
  int32_t bmax = 1;
  int32_t objective = 0;        // RM_SCHED_THROUGHPUT | RM_SCHED_LATENCY
  int64_t max_cost = 0;         // 0 = no cap on a batch of >= 2 requests
  int64_t c0 = 0, c1 = 0;
  std::vector<int64_t> table;   // [tb][tl] row-major, empty = linear model
  int32_t tb = 0, tl = 0;
  int64_t eval(int32_t b, int32_t L) const {
    if (!table.empty()) return table[static_cast<size_t>(b - 1) * tl + (L - 1)];
    return c0 + c1 * static_cast<int64_t>(b) * L;
  }
};
// Fills out[i] with the batch of request i; returns the batch count.
int schedule_dp(const SchedCost& cost, const int32_t* lengths, int32_t n, int32_t* out);

// ---- arena plan ----
// Intermediate buffers of one rm_score call.  Steps inside a layer:
//   0 LN1 (decoder)  1 QKV GEMM  2 scores  3 softmax  4 context  5 out-proj GEMM
//   6 residual+LN   7 FFN1 GEMM  8 FFN2 GEMM  9 residual+LN
// x (and z for the decoder) live through every step; the rest are planned.
// The decoder's out-proj and FFN2 add into x, so its y1 and y2 take no bytes.
enum Buf { B_X = 0, B_Z, B_QKV, B_S, B_CTX, B_Y1, B_F, B_Y2, B_COUNT };
struct ArenaPlan {
  int64_t off[B_COUNT] = {0};
  int64_t bytes[B_COUNT] = {0};
  int32_t first[B_COUNT] = {0};
  int32_t last[B_COUNT] = {0};
  int64_t peak = 0;
};
constexpr int64_t kArenaAlign = 256;
// Plan for T tokens and s_elems score elements (decoder adds z).
ArenaPlan plan_arena(int arch, int H, int F, int64_t T, int64_t s_elems);
// Upper bound of any plan with T <= T_max, s_elems <= S_max.
int64_t arena_bound(int arch, int H, int F, int64_t T_max, int64_t S_max);

// Validates cfg (all fields, or scheduler fields only); message in *why.
int validate_config(const rm_config* cfg, bool sched_only, const char** why);
SchedCost sched_cost_from(const rm_config* cfg);

// thread-local error message
int set_error(int code, const char* fmt, ...);

}  // namespace rmk
