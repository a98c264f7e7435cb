// Length-bucketed intermediate-tensor arena.
//
// "TurboTransformers: An Efficient GPU Serving System For Transformer Models"
// (abstract; proposed-method section; main results) designs a
// sequence-length-aware allocator for variable-length input that balances
// memory footprint against allocation speed and does not bloat after long or
// large batches.  Reading used here: the scorer's intermediates have fixed
// lifetimes inside a layer, so a call's sizes (T tokens, S score elements)
// determine one placement in which buffers that are never live together share
// bytes.  Placements are computed per length bucket and cached; the device
// memory behind them is reserved once, at create, for the largest bucket the
// handle admits, and never returned or grown while scoring.
#include <algorithm>

#include "host.h"

namespace rmk {
namespace {

int64_t align_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

bool overlap_steps(const ArenaPlan& p, int a, int b) {
  return p.first[a] <= p.last[b] && p.first[b] <= p.last[a];
}

void sizes(int arch, int H, int F, int64_t T, int64_t s_elems, ArenaPlan& p) {
  const int64_t row = 2;   // bf16 bytes
  // the decoder's residual stream is kept in fp32 (its rounding to bf16,
  // repeated over every layer's two additions, dominated the score error)
  p.bytes[B_X] = align_up(T * H * (arch == RM_DEC_PRELN ? 4 : row), kArenaAlign);
  p.bytes[B_Z] = arch == RM_DEC_PRELN ? align_up(T * H * row, kArenaAlign) : 0;
  p.bytes[B_QKV] = align_up(T * 3 * H * row, kArenaAlign);
  p.bytes[B_S] = align_up(s_elems * row, kArenaAlign);
  p.bytes[B_CTX] = align_up(T * H * row, kArenaAlign);
  // the decoder's output projection and FFN2 add into its fp32 x: no buffer
  // for their outputs
  const int64_t yrow = arch == RM_DEC_PRELN ? 0 : row;
  p.bytes[B_Y1] = align_up(T * H * yrow, kArenaAlign);
  p.bytes[B_F] = align_up(T * F * row, kArenaAlign);
  p.bytes[B_Y2] = align_up(T * H * yrow, kArenaAlign);
  static const int32_t first[B_COUNT] = {0, 0, 1, 2, 4, 5, 7, 8};
  static const int32_t last[B_COUNT] = {9, 9, 4, 4, 5, 6, 8, 9};
  for (int k = 0; k < B_COUNT; ++k) {
    p.first[k] = first[k];
    p.last[k] = last[k];
  }
}

}  // namespace

ArenaPlan plan_arena(int arch, int H, int F, int64_t T, int64_t s_elems) {
  ArenaPlan p;
  sizes(arch, H, F, T, s_elems, p);
  // Greedy offset assignment: largest buffer first, each at the lowest offset
  // that clears every already placed buffer it is live together with.
  int order[B_COUNT];
  for (int k = 0; k < B_COUNT; ++k) order[k] = k;
  std::stable_sort(order, order + B_COUNT, [&](int a, int b) { return p.bytes[a] > p.bytes[b]; });
  bool placed[B_COUNT] = {false};
  for (int oi = 0; oi < B_COUNT; ++oi) {
    const int k = order[oi];
    if (p.bytes[k] == 0) {
      p.off[k] = 0;
      placed[k] = true;
      continue;
    }
    // candidate offsets: 0 and the end of every conflicting placed buffer
    std::vector<int64_t> cand{0};
    for (int j = 0; j < B_COUNT; ++j)
      if (placed[j] && p.bytes[j] > 0 && overlap_steps(p, j, k)) cand.push_back(p.off[j] + p.bytes[j]);
    std::sort(cand.begin(), cand.end());
    for (int64_t c : cand) {
      bool ok = true;
      for (int j = 0; j < B_COUNT && ok; ++j)
        if (placed[j] && p.bytes[j] > 0 && overlap_steps(p, j, k) &&
            c < p.off[j] + p.bytes[j] && p.off[j] < c + p.bytes[k])
          ok = false;
      if (ok) {
        p.off[k] = c;
        break;
      }
    }
    placed[k] = true;
  }
  p.peak = 0;
  for (int k = 0; k < B_COUNT; ++k) p.peak = std::max(p.peak, p.off[k] + p.bytes[k]);
  return p;
}

int64_t arena_bound(int arch, int H, int F, int64_t T_max, int64_t S_max) {
  // no plan can exceed the sum of its buffers, and every size is monotone in
  // T and S, so the sum at the maxima bounds every bucket's placement
  ArenaPlan p;
  sizes(arch, H, F, T_max, S_max, p);
  int64_t s = 0;
  for (int k = 0; k < B_COUNT; ++k) s += p.bytes[k];
  return s;
}

}  // namespace rmk
