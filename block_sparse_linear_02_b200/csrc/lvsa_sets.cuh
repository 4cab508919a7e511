// lvsa_sets.cuh -- the LVSA attention set A(t) = G_s u W(t) of one query frame,
// compiled for both the host (slr_lvsa_attention_sets) and the device (the set
// builder kernel of slr_frame_mask_attn), so both run the same routine.
//
// Source: rainbus digest of LVSA (arXiv 2605.31057), sections "核心方法" and
// "方法步骤详情":
//   T_per = ceil(T / (C - (2W+1)))                 global period
//   G_s   = {(s mod T_per + i*T_per) mod T}, i < ceil(T/T_per)
//   w_lo  = max(0, min(t - W, T - 1 - 2W)), w_hi = w_lo + 2W
//   expand toward the side with more room until the window holds
//   min(2W+1, T - |G|) frames that are not global.
// Reading for the expansion tie: equal room on both sides grows the right side.
#pragma once

#include <stdint.h>

namespace slr {

struct LvsaGlobals {
  int T, period, count, offset;
};

__host__ __device__ inline LvsaGlobals lvsa_globals(int T, int C, int W, int step) {
  LvsaGlobals g;
  g.T = T;
  const int span = C - (2 * W + 1);
  g.period = (T + span - 1) / span;
  g.count = (T + g.period - 1) / g.period;
  g.offset = step % g.period;
  return g;
}

// Frame f is global iff f = (offset + i*period) mod T for some i < count.
__host__ __device__ inline bool lvsa_is_global(const LvsaGlobals& g, int f) {
  const int a = f - g.offset;
  if (a >= 0 && a % g.period == 0 && a / g.period < g.count) return true;
  const int b = f + g.T - g.offset;             // a member that wrapped past T
  return b % g.period == 0 && b / g.period < g.count;
}

// Writes A(t) ascending into out[0..cap) and returns its size, or -1 if cap is too small.
__host__ __device__ inline int lvsa_attention_set(int T, int C, int W, int step, int t, int32_t* out, int cap) {
  const LvsaGlobals g = lvsa_globals(T, C, W, step);
  int lo = t - W;
  if (lo > T - 1 - 2 * W) lo = T - 1 - 2 * W;
  if (lo < 0) lo = 0;
  int hi = lo + 2 * W;
  if (hi > T - 1) hi = T - 1;
  const int target = (2 * W + 1 < T - g.count) ? 2 * W + 1 : T - g.count;
  int non_global = 0;
  for (int f = lo; f <= hi; ++f) non_global += lvsa_is_global(g, f) ? 0 : 1;
  while (non_global < target) {
    const int room_lo = lo, room_hi = T - 1 - hi;
    if (room_hi >= room_lo && room_hi > 0) {
      ++hi;
      non_global += lvsa_is_global(g, hi) ? 0 : 1;
    } else if (room_lo > 0) {
      --lo;
      non_global += lvsa_is_global(g, lo) ? 0 : 1;
    } else {
      break;
    }
  }
  int n = 0;
  for (int f = 0; f < T; ++f) {
    if ((f >= lo && f <= hi) || lvsa_is_global(g, f)) {
      if (n >= cap) return -1;
      out[n++] = f;
    }
  }
  return n;
}

}  // namespace slr
