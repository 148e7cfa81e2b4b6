// The two comparison points of the latent decode (sm_100a):
//
// 1. dense_decode_kernel: flash-decoding over materialised bf16 K and V, the
//    baseline the pages measure their decode speed-ups against (WSVD page,
//    technical summary §4; LASER page, results).  For every (b, h):
//    softmax(q K^T * scale) V over positions [0, seq_len[b]).
// 2. reconstruct_kernel: the naive low-rank path the WSVD page contrasts
//    with its fused kernel (technical summary §1): K = dequant(C_K) B_K and
//    V = dequant(C_V) B_V are rebuilt into memory (bf16), then attended by
//    (1) -- twice the dense bytes of traffic on top of the latent reads.
//
// Dense kernel work split: a (b, h) unit's tokens are cut into 128-token
// stages; the (unit, stage) items are dealt out in equal contiguous ranges to
// a fixed grid (as the latent kernel does); a unit cut by range boundaries
// leaves one partial (m, l, o[H]) per piece and the last piece to arrive
// (atomic ticket) merges them.  Inside a CTA each of the 8 warps takes 16
// tokens of a stage: lanes 0..15 hold one token's row (16-byte chunks of the
// head dim), lanes 16..31 the next one, so a warp-wide 16-byte load reads
// two full rows; the dot products are reduced over the 16 lanes of a half,
// the running softmax state is per warp, and the warps merge at the end of
// a piece.  HBM-bound: every K and V byte is read once with 16-byte loads,
// 16 loads per lane in flight per 8 tokens.
#include <cstdio>

#include "lk_common.cuh"
#include "lk_internal.h"

namespace {

constexpr int kDThreads = 256;
constexpr int kDWarps = kDThreads / 32;
constexpr int kDStage = 128;          // tokens per item (16 per warp)
constexpr int kDMaxH = LK_MAX_HEAD_DIM;
constexpr int kDAutoCtaBound = 1024;

struct DenseParams {
  const uint16_t* q;
  const uint16_t* K;
  const uint16_t* V;
  const int32_t* seq_len;
  void* out;
  float* partials;
  int32_t* counters;
  int n_heads, H, capacity, max_len;
  int S, W, G;
  int part_stride;
  int out_bf16;
  float qscale;  // softmax_scale * log2(e)
};

LK_DEVICE int d_cta_first(const DenseParams& p, int c) { return (int)((int64_t)c * p.W / p.G); }
LK_DEVICE int d_cta_of(const DenseParams& p, int i) { return (int)(((int64_t)(i + 1) * p.G - 1) / p.W); }

// 8 bf16 values of a 16-byte chunk as fp32.
LK_DEVICE void bf16x8(const uint4& v, float* f) {
  f[0] = lk_bf16lo(v.x); f[1] = lk_bf16hi(v.x); f[2] = lk_bf16lo(v.y); f[3] = lk_bf16hi(v.y);
  f[4] = lk_bf16lo(v.z); f[5] = lk_bf16hi(v.z); f[6] = lk_bf16lo(v.w); f[7] = lk_bf16hi(v.w);
}

// Per-warp state of the current unit: running max and sum (in log2 units)
// and the partial output, lane (half, c) holding dims 8 c .. 8 c + 7 (for
// head dims over 128, chunks c and c + 16 ...) summed over the half's tokens.
template <int NCH>
struct WarpState {
  float m, l;
  float o[NCH][8];
};

// One unit's stages [s0, s1) for this warp (16 tokens of each stage).
template <int NCH>
LK_DEVICE void dense_run(const DenseParams& p, int64_t bh, int len, int s0, int s1, WarpState<NCH>& st,
                         const float (&qf)[NCH][8]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = lane >> 4, c = lane & 15;
  const int H = p.H;
  const uint16_t* Kb = p.K + bh * p.capacity * H;
  const uint16_t* Vb = p.V + bh * p.capacity * H;
  for (int s = s0; s < s1; ++s) {
    const int t0 = s * kDStage + warp * 16;
    if (t0 >= len) break;
    // 8 pairs of tokens: this lane's token of pair i is t0 + 2 i + half
    uint4 kv[8][NCH], vv[8][NCH];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int t = t0 + 2 * i + half;
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        const int col = 8 * (c + 16 * j);
        const bool live = t < len && col < H;
        kv[i][j] = live ? __ldg(reinterpret_cast<const uint4*>(Kb + (int64_t)t * H + col)) : make_uint4(0, 0, 0, 0);
        vv[i][j] = live ? __ldg(reinterpret_cast<const uint4*>(Vb + (int64_t)t * H + col)) : make_uint4(0, 0, 0, 0);
      }
    }
    float sc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float a = 0.0f;
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        float kf[8];
        bf16x8(kv[i][j], kf);
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaf(qf[j][e], kf[e], a);
      }
      // sum over the 16 lanes of this half
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      a += __shfl_xor_sync(0xffffffffu, a, 2);
      a += __shfl_xor_sync(0xffffffffu, a, 4);
      a += __shfl_xor_sync(0xffffffffu, a, 8);
      const int t = t0 + 2 * i + half;
      sc[i] = t < len ? a * p.qscale : -INFINITY;
    }
    // the warp's running max over both halves' tokens
    float mx = sc[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) mx = fmaxf(mx, sc[i]);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    const float m_new = fmaxf(st.m, mx);
    if (m_new == -INFINITY) continue;  // no valid token yet
    const float alpha = st.m == -INFINITY ? 0.0f : exp2f(st.m - m_new);
    st.m = m_new;
    float lsum = 0.0f;
#pragma unroll
    for (int j = 0; j < NCH; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) st.o[j][e] *= alpha;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float pw = exp2f(sc[i] - m_new);  // 0 for masked tokens
      lsum += pw;
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        float vf[8];
        bf16x8(vv[i][j], vf);
#pragma unroll
        for (int e = 0; e < 8; ++e) st.o[j][e] = fmaf(pw, vf[e], st.o[j][e]);
      }
    }
    // lsum counts this half's tokens once per lane of the half
    st.l = st.l * alpha + lsum + __shfl_xor_sync(0xffffffffu, lsum, 16);
  }
}

template <int NCH>
LK_DEVICE void dense_write(const DenseParams& p, int64_t bh, const float* cta) {
  const int H = p.H;
  const float inv = (cta[0] == -INFINITY || cta[1] == 0.0f) ? 0.0f : 1.0f / cta[1];
  for (int d = threadIdx.x; d < H; d += kDThreads) {
    const float o = cta[2 + d] * inv;
    if (p.out_bf16) reinterpret_cast<uint16_t*>(p.out)[bh * H + d] = lk_f32_to_bf16(o);
    else reinterpret_cast<float*>(p.out)[bh * H + d] = o;
  }
}

template <int NCH>
__global__ void __launch_bounds__(kDThreads) dense_decode_kernel(const __grid_constant__ DenseParams p) {
  __shared__ float wst[kDWarps][2 + kDMaxH];
  __shared__ float cta[2 + kDMaxH];
  __shared__ int ticket;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = lane >> 4, cidx = lane & 15;
  const int c = blockIdx.x;
  const int i0 = d_cta_first(p, c), i1 = d_cta_first(p, c + 1);
  const int H = p.H;
  int it = i0;
  while (it < i1) {
    const int u = it / p.S, s = it - u * p.S;
    const int s_end = min(p.S, s + (i1 - it));
    const int seg_first = it, seg_end = it + (s_end - s);
    const int b = u / p.n_heads;
    const int64_t bh = u;  // units are (b, h) in order
    const int len = max(0, min(p.seq_len[b], p.max_len));
    float qf[NCH][8];
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
      const int col = 8 * (cidx + 16 * j);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (col < H) v = __ldg(reinterpret_cast<const uint4*>(p.q + bh * H + col));
      bf16x8(v, qf[j]);
    }
    WarpState<NCH> st;
    st.m = -INFINITY;
    st.l = 0.0f;
#pragma unroll
    for (int j = 0; j < NCH; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) st.o[j][e] = 0.0f;
    dense_run<NCH>(p, bh, len, s, s_end, st, qf);
    // the two halves' outputs, then the warps' states in shared memory
#pragma unroll
    for (int j = 0; j < NCH; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) st.o[j][e] += __shfl_xor_sync(0xffffffffu, st.o[j][e], 16);
    if (lane == 0) {
      wst[warp][0] = st.m;
      wst[warp][1] = st.l;
    }
    if (half == 0) {
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        const int col = 8 * (cidx + 16 * j);
        if (col < H)
#pragma unroll
          for (int e = 0; e < 8; ++e) wst[warp][2 + col + e] = st.o[j][e];
      }
    }
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDWarps; ++w) M = fmaxf(M, wst[w][0]);
    for (int d = threadIdx.x; d < 2 + H; d += kDThreads) {
      float acc = d == 0 ? M : 0.0f;
      if (d > 0 && M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kDWarps; ++w) {
          const float mw = wst[w][0];
          if (mw != -INFINITY) acc += wst[w][d] * exp2f(mw - M);
        }
      }
      cta[d] = acc;
    }
    __syncthreads();
    const int u0 = u * p.S, u1 = u0 + p.S;
    if (seg_first == u0 && seg_end == u1) {
      dense_write<NCH>(p, bh, cta);
    } else {
      const int slot = seg_first == i0 ? 0 : 1;
      float* part = p.partials + ((int64_t)c * 2 + slot) * p.part_stride;
      for (int d = threadIdx.x; d < 2 + H; d += kDThreads) part[d] = cta[d];
      __threadfence();
      __syncthreads();
      const int c0 = d_cta_of(p, u0), c1 = d_cta_of(p, u1 - 1);
      if (threadIdx.x == 0) ticket = atomicAdd(&p.counters[u], 1) == c1 - c0;
      __syncthreads();
      if (ticket) {
        __threadfence();
        const int slot0 = d_cta_first(p, c0) >= u0 ? 0 : 1;
        auto piece = [&](int cc) {
          return p.partials + ((int64_t)cc * 2 + (cc == c0 ? slot0 : 0)) * p.part_stride;
        };
        float Mg = -INFINITY;
        for (int cc = c0; cc <= c1; ++cc) Mg = fmaxf(Mg, __ldcg(piece(cc)));
        __syncthreads();  // every thread has read cta[] before it is overwritten
        for (int d = threadIdx.x; d < 2 + H; d += kDThreads) {
          float acc = d == 0 ? Mg : 0.0f;
          if (d > 0 && Mg != -INFINITY)
            for (int cc = c0; cc <= c1; ++cc) {
              const float* pc = piece(cc);
              const float mc = __ldcg(pc);
              if (mc != -INFINITY) acc = fmaf(exp2f(mc - Mg), __ldcg(pc + d), acc);
            }
          cta[d] = acc;
        }
        if (threadIdx.x == 0) p.counters[u] = 0;  // ready for the next call
        __syncthreads();
        dense_write<NCH>(p, bh, cta);
      }
    }
    __syncthreads();  // wst, cta and ticket are free for the next unit
    it = seg_end;
  }
}

// ---------------------------------------------------------------- naive reconstruction
// K[b, h, t, :] = dequant(c_K[t]) B_K^h for t < seq_len[b] (and V likewise),
// stored bf16 [B, n_heads, capacity, H], on the tensor cores: a CTA takes
// kRTok tokens of one (b, h, K-or-V).  The codes of those tokens (one
// contiguous byte range of the cache plane in either layout) are expanded to
// bf16 rows [token][dim] in shared memory (exact: |code| <= 127), B^h is
// staged as bf16 [dim][H]; each warp takes 16-token tiles and, per pair of
// 8-dim output columns, runs m16n8k16 products over the latent dims (int4
// with several scale groups: m16n8k8 products, one accumulator per group,
// each group's sum scaled by the token's group scale), then scales by the
// token's scale, rounds to bf16 once and stores.  The code and factor
// products are exact; the only rounding besides the fp32 sums is the final
// one to bf16.
struct ReconParams {
  const uint8_t* codes[2];
  const uint8_t* scales[2];
  const uint16_t* Bf[2];
  uint16_t* dst[2];
  const int32_t* seq_len;
  int kind, n_heads, H, capacity, max_len;
  int tot_rb[2], tot_ng[2];
  uint8_t rank[2][LK_MAX_HEADS], group[2][LK_MAX_HEADS];
  uint16_t pref_rb[2][LK_MAX_HEADS], pref_ng[2][LK_MAX_HEADS], pref_r[2][LK_MAX_HEADS];
};

constexpr int kRTok = 256;      // tokens per CTA
constexpr int kRWarps = 8;

// Shared-memory strides (bf16 elements): rows padded by 8 so that the eight
// 16-byte rows an ldmatrix reads fall in distinct banks.
LK_DEVICE int recon_cstride(int r16) { return r16 + 8; }

__global__ void __launch_bounds__(kRWarps * 32) reconstruct_kernel(const __grid_constant__ ReconParams p) {
  extern __shared__ __align__(16) uint8_t rsm[];
  const int which = blockIdx.z;  // 0: K, 1: V
  const int bh = blockIdx.y;
  const int b = bh / p.n_heads, h = bh - b * p.n_heads;
  const int t0 = blockIdx.x * kRTok;
  const int len = max(0, min(p.seq_len[b], p.max_len));
  if (t0 >= len) return;
  const int r = p.rank[which][h], H = p.H;
  const int r16 = (r + 15) & ~15;
  const int rb = p.kind == 0 ? r : r / 2;
  const int g = p.group[which][h], ng = (r + g - 1) / g;
  const int cst = recon_cstride(r16), bst = H + 8;
  uint16_t* Cs = reinterpret_cast<uint16_t*>(rsm);              // [kRTok][cst]
  uint16_t* Bs = Cs + kRTok * cst;                              // [r16][bst]
  float* Ss = reinterpret_cast<float*>(Bs + r16 * bst);         // [kRTok][ng]
  const int ntok = min(kRTok, len - t0);
  const int ntok16 = (ntok + 15) & ~15;                         // whole 16-token blocks (the cache holds them)
  // B^h rows, zero rows up to r16
  const uint16_t* Bg = p.Bf[which] + (int64_t)p.pref_r[which][h] * H;
  for (int i = threadIdx.x; i < r16 * (H / 8); i += blockDim.x) {
    const int d = i / (H / 8), c8 = i - d * (H / 8);
    const uint4 v = d < r ? *reinterpret_cast<const uint4*>(Bg + (int64_t)d * H + 8 * c8) : make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(Bs + d * bst + 8 * c8) = v;
  }
  // code dims r .. r16 - 1 are zero
  for (int i = threadIdx.x; i < ntok16 * (r16 - r); i += blockDim.x) {
    const int t = i / (r16 - r), d = r + i - t * (r16 - r);
    Cs[t * cst + d] = 0;
  }
  // codes: the plane's bytes of tokens t0 .. t0 + ntok16, read as words
  const uint8_t* plane = p.codes[which] + ((int64_t)b * p.tot_rb[which] + p.pref_rb[which][h]) * p.capacity;
  const uint32_t* src = reinterpret_cast<const uint32_t*>(plane + (int64_t)t0 * rb);
  const int nwords = ntok16 * rb / 4;
  const int cs = lk_chunk_bytes(rb);
  for (int i = threadIdx.x; i < nwords; i += blockDim.x) {
    const uint32_t w = __ldg(src + i);
    const int o = 4 * i;
    const int blk = o / (16 * rb), rem = o - blk * 16 * rb;
    if (which == 0) {  // token-major chunks: the word is consecutive bytes of one token
      const int ch = rem / (16 * cs), rem2 = rem - ch * 16 * cs;
      const int t = blk * 16 + rem2 / cs, byte0 = ch * cs + rem2 % cs;
      uint16_t* row = Cs + t * cst;
      if (p.kind == 0) {
#pragma unroll
        for (int k = 0; k < 4; ++k) row[byte0 + k] = __bfloat16_as_ushort(__int2bfloat16_rn((int)(int8_t)(w >> (8 * k))));
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int nib = (int)((w >> (4 * k)) & 0xF);
          row[2 * byte0 + k] = __bfloat16_as_ushort(__int2bfloat16_rn(nib >= 8 ? nib - 16 : nib));
        }
      }
    } else if (p.kind == 0) {  // dimension-major: the word is 4 consecutive tokens of one dim
      const int d = rem / 16, tt = rem % 16;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        Cs[(blk * 16 + tt + k) * cst + d] = __bfloat16_as_ushort(__int2bfloat16_rn((int)(int8_t)(w >> (8 * k))));
    } else {                   // int4 dimension-major: 8 consecutive tokens of one dim
      const int d = rem / 8, tt = 2 * (rem % 8);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int nib = (int)((w >> (4 * k)) & 0xF);
        Cs[(blk * 16 + tt + k) * cst + d] = __bfloat16_as_ushort(__int2bfloat16_rn(nib >= 8 ? nib - 16 : nib));
      }
    }
  }
  // scales as fp32 [token][group]
  if (p.kind == 0) {
    const float* sp = reinterpret_cast<const float*>(p.scales[which]) + ((int64_t)b * p.n_heads + h) * p.capacity + t0;
    for (int i = threadIdx.x; i < ntok16; i += blockDim.x) Ss[i] = sp[i];
  } else {
    const uint16_t* sp = reinterpret_cast<const uint16_t*>(p.scales[which]) +
                         ((int64_t)b * p.tot_ng[which] + p.pref_ng[which][h]) * p.capacity + (int64_t)t0 * ng;
    for (int i = threadIdx.x; i < ntok16 * ng; i += blockDim.x) Ss[i] = lk_f16_to_f32(sp[i]);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int nks = r16 / 16;
  const bool grouped = ng > 1;  // int4 with several groups (groups are multiples of 8 dims)
  uint16_t* out = p.dst[which] + (int64_t)bh * p.capacity * H;
  // a warp takes two 16-token tiles at a time, so that each B fragment read
  // from shared memory feeds both
  for (int tb0 = 32 * warp; tb0 < ntok16; tb0 += 32 * kRWarps) {
    const int nmt = tb0 + 16 < ntok16 ? 2 : 1;
    // A fragments of each tile and k step: matrices (rows 0-7, k 0-7),
    // (rows 8-15, k 0-7), (rows 0-7, k 8-15), (rows 8-15, k 8-15)
    uint32_t af[2][4][4];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        if (m < nmt && ks < nks) {
          const int row = tb0 + 16 * m + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int col = 16 * ks + (lane >> 4) * 8;
          lk_ldmatrix_x4(af[m][ks], Cs + row * cst + col);
        } else {
          af[m][ks][0] = af[m][ks][1] = af[m][ks][2] = af[m][ks][3] = 0u;
        }
      }
    }
    for (int n0 = 0; n0 < H; n0 += 16) {
      // [tile][column octet][fragment]
      float acc[2][2][4], o[2][2][4];
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[m][n][e] = o[m][n][e] = 0.0f;
      int cur = 0;  // scale group of the open accumulators
      auto fold = [&](int gi) {
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const int tl = tb0 + 16 * m + gid;
          const float sl = Ss[tl * ng + gi], sh = Ss[(tl + 8) * ng + gi];
#pragma unroll
          for (int n = 0; n < 2; ++n) {
            o[m][n][0] = fmaf(sl, acc[m][n][0], o[m][n][0]);
            o[m][n][1] = fmaf(sl, acc[m][n][1], o[m][n][1]);
            o[m][n][2] = fmaf(sh, acc[m][n][2], o[m][n][2]);
            o[m][n][3] = fmaf(sh, acc[m][n][3], o[m][n][3]);
            acc[m][n][0] = acc[m][n][1] = acc[m][n][2] = acc[m][n][3] = 0.0f;
          }
        }
      };
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        if (ks < nks) {
          // B fragments for columns n0 .. n0 + 15: matrices (k 0-7, n 0-7),
          // (k 8-15, n 0-7), (k 0-7, n 8-15), (k 8-15, n 8-15), transposed
          uint32_t bfr[4];
          const int krow = 16 * ks + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int ncol = n0 + (lane >> 4) * 8;
          lk_ldmatrix_x4_trans(bfr, Bs + krow * bst + ncol);
          if (!grouped) {
#pragma unroll
            for (int m = 0; m < 2; ++m) {
              lk_mma_bf16_16816(acc[m][0], af[m][ks][0], af[m][ks][1], af[m][ks][2], af[m][ks][3], bfr[0], bfr[1]);
              lk_mma_bf16_16816(acc[m][1], af[m][ks][0], af[m][ks][1], af[m][ks][2], af[m][ks][3], bfr[2], bfr[3]);
            }
          } else {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const int d0 = 16 * ks + 8 * hf;
              if (d0 < r) {
                const int gi = d0 / g;
                if (gi != cur) {  // the previous group is complete
                  fold(cur);
                  cur = gi;
                }
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                  lk_mma_bf16_1688(acc[m][0], af[m][ks][2 * hf], af[m][ks][2 * hf + 1], bfr[hf]);
                  lk_mma_bf16_1688(acc[m][1], af[m][ks][2 * hf], af[m][ks][2 * hf + 1], bfr[2 + hf]);
                }
              }
            }
          }
        }
      }
      fold(cur);  // (one group: o = sigma * acc)
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int t_lo = t0 + tb0 + 16 * m + gid, t_hi = t_lo + 8;
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          const int col = n0 + 8 * n + 2 * tig;
          if (m < nmt && t_lo < len)
            *reinterpret_cast<uint32_t*>(out + (int64_t)t_lo * H + col) = lk_pack_bf16x2(o[m][n][0], o[m][n][1]);
          if (m < nmt && t_hi < len)
            *reinterpret_cast<uint32_t*>(out + (int64_t)t_hi * H + col) = lk_pack_bf16x2(o[m][n][2], o[m][n][3]);
        }
      }
    }
  }
}

int d_round_up(int x, int m) { return (x + m - 1) / m * m; }

int64_t dense_ctas(int units, int max_len, int num_sms) {
  const int64_t W = (int64_t)units * std::max(1, (max_len + kDStage - 1) / kDStage);
  const int64_t cap = std::min<int64_t>((int64_t)2 * num_sms, kDAutoCtaBound);  // 2 CTAs of 8 warps per SM (registers)
  if (2 * (int64_t)units > cap) return std::min(W, cap);
  return std::min(W, (int64_t)units * (cap / units));
}

}  // namespace

namespace lk {

size_t dense_workspace_bytes(int units, int head_dim, int max_len, int num_sms) {
  const size_t counters = (size_t)d_round_up(units * 4, 256);
  const int64_t G = dense_ctas(units, max_len, num_sms);
  return counters + (size_t)G * 2 * d_round_up(2 + head_dim, 4) * 4;
}

cudaError_t launch_dense_decode(const DenseLaunch& a, cudaStream_t stream) {
  DenseParams p{};
  p.q = static_cast<const uint16_t*>(a.q);
  p.K = static_cast<const uint16_t*>(a.K);
  p.V = static_cast<const uint16_t*>(a.V);
  p.seq_len = a.seq_len;
  p.out = a.out;
  p.n_heads = a.n_heads;
  p.H = a.head_dim;
  p.capacity = a.capacity;
  p.max_len = a.max_len;
  p.out_bf16 = a.out_bf16;
  p.qscale = a.softmax_scale * 1.4426950408889634f;
  const int units = a.batch * a.n_heads;
  p.S = std::max(1, (a.max_len + kDStage - 1) / kDStage);
  const int64_t W = (int64_t)units * p.S;
  const int64_t G = dense_ctas(units, a.max_len, a.num_sms);
  if (W > INT32_MAX || G < 1) return cudaErrorInvalidValue;
  p.W = (int)W;
  p.G = (int)G;
  p.part_stride = d_round_up(2 + a.head_dim, 4);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  p.counters = reinterpret_cast<int32_t*>(ws);
  p.partials = reinterpret_cast<float*>(ws + d_round_up(units * 4, 256));
  const dim3 grid((unsigned)G);
  if (a.head_dim <= 128) dense_decode_kernel<1><<<grid, kDThreads, 0, stream>>>(p);
  else dense_decode_kernel<2><<<grid, kDThreads, 0, stream>>>(p);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_reconstruct_kv(const ReconLaunch& a, cudaStream_t stream) {
  ReconParams p{};
  p.kind = a.kind;
  p.n_heads = a.n_heads;
  p.H = a.head_dim;
  p.capacity = a.capacity;
  if (!a.b_bf16) return cudaErrorInvalidValue;  // the factors are bf16 tensor-core operands
  p.max_len = a.max_len;
  p.seq_len = a.seq_len;
  int r_max = 0;
  for (int c = 0; c < 2; ++c) {
    p.codes[c] = static_cast<const uint8_t*>(a.codes[c]);
    p.scales[c] = static_cast<const uint8_t*>(a.scales[c]);
    p.Bf[c] = static_cast<const uint16_t*>(a.B[c]);
    p.dst[c] = static_cast<uint16_t*>(a.out[c]);
    int prb = 0, png = 0, pr = 0;
    for (int h = 0; h < a.n_heads; ++h) {
      const int r = a.ranks[c][h];
      const int g = a.kind == 0 ? r : std::min(a.group[c], r);
      p.rank[c][h] = (uint8_t)r;
      p.group[c][h] = (uint8_t)g;
      p.pref_rb[c][h] = (uint16_t)prb;
      p.pref_ng[c][h] = (uint16_t)png;
      p.pref_r[c][h] = (uint16_t)pr;
      prb += a.kind == 0 ? r : r / 2;
      png += a.kind == 0 ? 1 : (r + g - 1) / g;
      pr += r;
      r_max = std::max(r_max, r);
    }
    p.tot_rb[c] = prb;
    p.tot_ng[c] = png;
  }
  int ng_max = 1;
  for (int c = 0; c < 2; ++c)
    for (int h = 0; h < a.n_heads; ++h) ng_max = std::max(ng_max, (a.ranks[c][h] + p.group[c][h] - 1) / p.group[c][h]);
  const int r16 = (r_max + 15) & ~15;
  const int smem = (kRTok * (r16 + 8) + r16 * (a.head_dim + 8)) * 2 + kRTok * ng_max * 4;
  cudaError_t e = cudaFuncSetAttribute(reconstruct_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((a.max_len + kRTok - 1) / kRTok), (unsigned)(a.batch * a.n_heads), 2);
  if (grid.x == 0) return cudaSuccess;
  reconstruct_kernel<<<grid, kRWarps * 32, smem, stream>>>(p);
  count_launch();
  return cudaGetLastError();
}

}  // namespace lk
