// Warp-cooperative latent quantiser shared by the stand-alone quantiser and
// the projection's quantise-and-append epilogue.
#pragma once

#include "lk_common.cuh"

// S2 of one head's latent (WSVD page §2C: an orthogonal rotation of the
// latent before RTN smooths outlier dims): block diagonal, each block the
// normalised Walsh-Hadamard matrix of order n = the largest power of two
// dividing r (at most 64).  Lane l holds v0 = dim l and v1 = dim l + 32;
// in place, y_j = sum_i v_i (-1)^popcount(i & j) / sqrt(n) over each block
// (butterflies across lanes by shuffles; the order-64 stage combines v0 and
// v1 of the same lane).
LK_DEVICE void lk_rotate_latent_warp(float& v0, float& v1, int r) {
  const int lane = threadIdx.x & 31;
  int n = 1;
  while (r % (2 * n) == 0 && 2 * n <= 64) n *= 2;
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
    if (h < n) {
      const float p0 = __shfl_xor_sync(0xffffffffu, v0, h);
      const float p1 = __shfl_xor_sync(0xffffffffu, v1, h);
      v0 = (lane & h) ? __fsub_rn(p0, v0) : __fadd_rn(v0, p0);
      v1 = (lane & h) ? __fsub_rn(p1, v1) : __fadd_rn(v1, p1);
    }
  }
  if (n == 64) {
    const float a = v0, b = v1;
    v0 = __fadd_rn(a, b);
    v1 = __fsub_rn(a, b);
  }
  const float c = __double2float_rn(1.0 / sqrt((double)n));  // fl32(1 / sqrt(n))
  v0 = __fmul_rn(v0, c);
  v1 = __fmul_rn(v1, c);
}

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
