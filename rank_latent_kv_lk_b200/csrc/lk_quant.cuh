// Warp-cooperative latent quantiser shared by the stand-alone quantiser and
// the projection's quantise-and-append epilogue.
#pragma once

#include "lk_common.cuh"

// One row of r <= 64 latent values; lane l holds v0 = row[l] and
// v1 = row[l + 32] (ignored past r).  Returns each element's code and the
// scale of the group it belongs to.
struct LkQRow {
  int c0, c1;
  float s0, s1;
};

LK_DEVICE LkQRow lk_quantize_row_warp(float v0, float v1, int r, int kind, int group) {
  const int lane = threadIdx.x & 31;
  const bool h0 = lane < r, h1 = lane + 32 < r;
  LkQRow q;
  if (kind == 0) {
    float a = fmaxf(h0 ? fabsf(v0) : 0.0f, h1 ? fabsf(v1) : 0.0f);
    a = lk_warp_max(a);
    const float s = lk_q8_scale(a);
    q.c0 = h0 ? lk_q8_code(v0, s) : 0;
    q.c1 = h1 ? lk_q8_code(v1, s) : 0;
    q.s0 = q.s1 = s;
  } else {
    const int g = min(group, r);
    const int ng = (r + g - 1) / g;
    const int gi0 = lane / g, gi1 = (lane + 32) / g;
    float s0 = 0.0f, s1 = 0.0f;
    for (int gi = 0; gi < ng; ++gi) {
      float a = fmaxf((h0 && gi0 == gi) ? fabsf(v0) : 0.0f, (h1 && gi1 == gi) ? fabsf(v1) : 0.0f);
      a = lk_warp_max(a);
      const float s = lk_q4_scale(a);
      if (gi == gi0) s0 = s;
      if (gi == gi1) s1 = s;
    }
    q.c0 = h0 ? lk_q4_code(v0, s0) : 0;
    q.c1 = h1 ? lk_q4_code(v1, s1) : 0;
    q.s0 = s0;
    q.s1 = s1;
  }
  return q;
}
