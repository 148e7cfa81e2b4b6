// Latent decode attention, split-K over the sequence (sm_100a).
//
// Per (batch row b, head h, split s) one CTA of 256 threads:
//   1. absorbs q into latent space, q~ = B_K^h q * softmax_scale * log2(e)
//      (WSVD page §2C: the fused kernel works from the per-head latents;
//      without positional rotation (q B_K^T) C^T equals q K^T), and writes
//      q~ as a three-term int8 expansion q~ = a (t0 + t1/254 + t2/254^2)
//      (error <= 6e-8 of max|q~|, i.e. float32 level);
//   2. streams its slice of the latent cache (K codes, V codes and their
//      scales) HBM -> shared memory with bulk copies on the TMA engine,
//      2 or 3 stages deep, one mbarrier per stage;
//   3. per stage of 256 tokens (three block barriers):
//      a. one token per thread: s_t = sigma_K (c_K . q~) with exact int32
//         dp4a dot products against the expansion;
//      b. a CTA-uniform running max, p_t = 2^(s_t - max), running sum;
//      c. u += p_t sigma_V c_V: the stage's weights w_t = p_t sigma_V[t] are
//         written as a three-term int8 expansion relative to
//         W = max_t p_t * max_t sigma_V[t] >= every w_t (both maxima come out
//         of the score reduction; error <= 6e-8 W per weight), and each
//         lane takes exact int32 dp4a sums over 4 (int8) or 8 (int4) tokens
//         of one latent dim at a time from the dimension-major V layout; one
//         float fold per stage;
//   4. reduces (max, sum, u) over the CTA into a partial in latent space; the
//      last CTA of the (b, h) to arrive (atomic ticket, no waiting) merges
//      all partials and applies out = (u / sum) B_V^h.
// K and V are never formed; the per-token traffic is the latent codes and
// their scales.
#include "lk_common.cuh"
#include "lk_internal.h"

#include <cooperative_groups.h>
namespace cg = cooperative_groups;

namespace {

constexpr int kCW = 8;                          // consumer warps
constexpr int kConsumerThreads = kCW * 32;
constexpr int kWTerms = 4;                      // int8 terms of the weight expansion
constexpr int kThreads = kConsumerThreads + 32;  // + one producer warp
constexpr int kStageT = 256;   // tokens per pipeline stage: one per thread in the score phase
constexpr int kMaxStages = 8;  // pipeline depth chosen at launch (2 .. 8)
constexpr int kMaxR = LK_MAX_RANK;
constexpr int kMaxWords = kMaxR / 4;  // 32-bit words of q~ terms (int8 per dim)
constexpr int kMaxGroups = 8;
constexpr int kMaxSplit = 256;

struct DecodeParams {
  const uint8_t* codes_k;
  const uint8_t* codes_v;
  const uint8_t* scales_k;
  const uint8_t* scales_v;
  const void* q;
  const void* BK;
  const void* BV;
  const int32_t* seq_len;
  void* out;
  float* partials;    // [B * n_heads][n_split][part_stride]
  int32_t* counters;  // [B * n_heads]
  int batch, n_heads, head_dim, capacity;
  int group_k, group_v;  // int4 requested group size (effective min(g, r))
  int q_bf16, b_bf16, out_bf16;
  int n_split, stages_per_split, part_stride, max_len;
  float qscale;  // softmax_scale * log2(e)
  // bytes of the shared-memory regions (max over heads), multiples of 128
  int st_kc, st_vc, st_ks, st_vs;
  int st_q, st_bk, st_bv, st_tw;
  int nstages;
  int q_size, b_size;  // element sizes of q and of the factors
  int cluster_merge;   // the n_split CTAs of a head form one thread-block cluster
  uint8_t rk[LK_MAX_HEADS];
  uint8_t rv[LK_MAX_HEADS];
};

struct HeadGeom {
  int rk, rv;      // ranks
  int rbk, rbv;    // code bytes per token
  int ngk, ngv;    // scale groups per token (1 for int8)
  int gk, gv;      // effective group size (int4)
  int64_t kc_off;  // byte offset of this (b, h) K code plane
  int64_t vc_off;
  int64_t ks_off;  // element offset of this (b, h) K scale plane
  int64_t vs_off;
  int64_t bk_off;  // element offset of B_K^h
  int64_t bv_off;
};

template <int KIND>
LK_DEVICE int row_bytes(int r) { return KIND == 0 ? r : r / 2; }
template <int KIND>
LK_DEVICE int n_groups(int r, int g) { return KIND == 0 ? 1 : (r + g - 1) / g; }

// Prefix sums over heads, computed by each warp with strided lanes + shuffles.
template <int KIND>
LK_DEVICE HeadGeom head_geometry(const DecodeParams& p, int b, int h) {
  int lane = threadIdx.x & 31;
  int pk = 0, pv = 0, tk = 0, tv = 0, pgk = 0, pgv = 0, tgk = 0, tgv = 0, prk = 0, prv = 0;
  for (int i = lane; i < p.n_heads; i += 32) {
    int rk = p.rk[i], rv = p.rv[i];
    int bk = row_bytes<KIND>(rk), bv = row_bytes<KIND>(rv);
    int gk = n_groups<KIND>(rk, min(p.group_k, rk)), gv = n_groups<KIND>(rv, min(p.group_v, rv));
    tk += bk; tv += bv; tgk += gk; tgv += gv;
    if (i < h) { pk += bk; pv += bv; pgk += gk; pgv += gv; prk += rk; prv += rv; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    pk += __shfl_xor_sync(0xffffffffu, pk, o);
    pv += __shfl_xor_sync(0xffffffffu, pv, o);
    tk += __shfl_xor_sync(0xffffffffu, tk, o);
    tv += __shfl_xor_sync(0xffffffffu, tv, o);
    pgk += __shfl_xor_sync(0xffffffffu, pgk, o);
    pgv += __shfl_xor_sync(0xffffffffu, pgv, o);
    tgk += __shfl_xor_sync(0xffffffffu, tgk, o);
    tgv += __shfl_xor_sync(0xffffffffu, tgv, o);
    prk += __shfl_xor_sync(0xffffffffu, prk, o);
    prv += __shfl_xor_sync(0xffffffffu, prv, o);
  }
  HeadGeom g;
  g.rk = p.rk[h];
  g.rv = p.rv[h];
  g.rbk = row_bytes<KIND>(g.rk);
  g.rbv = row_bytes<KIND>(g.rv);
  g.gk = KIND == 0 ? g.rk : min(p.group_k, g.rk);
  g.gv = KIND == 0 ? g.rv : min(p.group_v, g.rv);
  g.ngk = n_groups<KIND>(g.rk, g.gk);
  g.ngv = n_groups<KIND>(g.rv, g.gv);
  const int64_t cap = p.capacity;
  g.kc_off = ((int64_t)b * tk + pk) * cap;
  g.vc_off = ((int64_t)b * tv + pv) * cap;
  g.ks_off = ((int64_t)b * tgk + pgk) * cap;
  g.vs_off = ((int64_t)b * tgv + pgv) * cap;
  g.bk_off = (int64_t)prk * p.head_dim;
  g.bv_off = (int64_t)prv * p.head_dim;
  return g;
}

// Loads the code chunk `c` (CS bytes) of local token `tl` from a staged
// region laid out in 16-token blocks (chunk-major inside a block).
template <int CS>
struct Chunk;
template <>
struct Chunk<16> {
  uint32_t w[4];
  LK_DEVICE void load(const uint8_t* base, int rb, int tl, int c) {
    const uint4 v = *reinterpret_cast<const uint4*>(base + (tl >> 4) * 16 * rb + c * 256 + (tl & 15) * 16);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  }
};
template <>
struct Chunk<8> {
  uint32_t w[2];
  LK_DEVICE void load(const uint8_t* base, int rb, int tl, int c) {
    const uint2 v = *reinterpret_cast<const uint2*>(base + (tl >> 4) * 16 * rb + c * 128 + (tl & 15) * 8);
    w[0] = v.x; w[1] = v.y;
  }
};
template <>
struct Chunk<4> {
  uint32_t w[1];
  LK_DEVICE void load(const uint8_t* base, int rb, int tl, int c) {
    w[0] = *reinterpret_cast<const uint32_t*>(base + (tl >> 4) * 16 * rb + c * 64 + (tl & 15) * 4);
  }
};

LK_DEVICE float load_scale(const uint8_t* base, int i, int kind) {
  return kind == 0 ? reinterpret_cast<const float*>(base)[i]
                   : lk_f16_to_f32(reinterpret_cast<const uint16_t*>(base)[i]);
}

LK_DEVICE float ld_f(const uint8_t* base, int i, int is_bf16) {
  return is_bf16 ? lk_bf16_to_f32(reinterpret_cast<const uint16_t*>(base)[i])
                 : reinterpret_cast<const float*>(base)[i];
}

// Expands code word `wd` into fp32 values: 4 signed bytes (int8) or 8 signed
// nibbles (int4, low nibble = even dim).  Exact integers.
template <int KIND>
LK_DEVICE void expand_word(uint32_t wd, float* f) {
  if (KIND == 0) {
    const uint32_t x = wd ^ 0x80808080u;
#pragma unroll
    for (int k = 0; k < 4; ++k) f[k] = lk_s8_from_xored(x, k);
  } else {
    const uint32_t x = wd ^ 0x88888888u;        // each nibble n -> c + 8
    const uint32_t ev = x & 0x0F0F0F0Fu;         // dims 0, 2, 4, 6
    const uint32_t od = (x >> 4) & 0x0F0F0F0Fu;  // dims 1, 3, 5, 7
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = __uint_as_float(__byte_perm(ev, 0x4B000000u, 0x7540u | k)) - 8388616.0f;
      f[2 * k + 1] = __uint_as_float(__byte_perm(od, 0x4B000000u, 0x7540u | k)) - 8388616.0f;
    }
  }
}

// Signed int4 nibbles of a word as signed int8 bytes: `ev` gets the low
// nibbles (elements 0, 2, 4, 6), `od` the high ones (1, 3, 5, 7).  Setting
// the upper half of a byte whose bit 3 is set is one multiply: 0x08 * 0x1E =
// 0xF0 stays inside its byte.
LK_DEVICE void nibbles_to_s8(uint32_t x, int& ev, int& od) {
  const uint32_t e = x & 0x0F0F0F0Fu, o = (x >> 4) & 0x0F0F0F0Fu;
  ev = (int)(e | ((e & 0x08080808u) * 0x1Eu));
  od = (int)(o | ((o & 0x08080808u) * 0x1Eu));
}

constexpr float kInv254 = 1.0f / 254.0f;
constexpr float kInv254sq = 1.0f / (254.0f * 254.0f);

// Score of one token in log2 units: sum over groups g of
//   sigma_g * a * (D0 + D1/254 + D2/254^2),  D_i = c . t_i  (exact dp4a sums)
// (int8 keys: one group and one scale per token).
template <int KIND, int CS>
LK_DEVICE float token_score(const uint8_t* kc, const uint8_t* ks, const HeadGeom& g, int tl,
                            const uint32_t (&qw)[3][kMaxWords], float qa) {
  constexpr int WPC = CS / 4;  // words per chunk
  constexpr int MAXCH = (KIND == 0 ? kMaxR : kMaxR / 2) / CS;
  const int nch = g.rbk / CS;
  if (KIND == 0) {
    int d0 = 0, d1 = 0, d2 = 0;
#pragma unroll
    for (int c = 0; c < MAXCH; ++c) {
      if (c < nch) {
        Chunk<CS> ch;
        ch.load(kc, g.rbk, tl, c);
#pragma unroll
        for (int wi = 0; wi < WPC; ++wi) {
          const int w = c * WPC + wi;
          d0 = __dp4a((int)ch.w[wi], (int)qw[0][w], d0);
          d1 = __dp4a((int)ch.w[wi], (int)qw[1][w], d1);
          d2 = __dp4a((int)ch.w[wi], (int)qw[2][w], d2);
        }
      }
    }
    const float x = fmaf((float)d2, kInv254sq, fmaf((float)d1, kInv254, (float)d0));
    return reinterpret_cast<const float*>(ks)[tl] * (qa * x);
  } else {
    float s = 0.0f;
    int d0 = 0, d1 = 0, d2 = 0;
    int cur_g = 0;
    // code word w holds dims 8w .. 8w+7; groups are multiples of 8 dims
#pragma unroll
    for (int c = 0; c < MAXCH; ++c) {
      if (c < nch) {
        Chunk<CS> ch;
        ch.load(kc, g.rbk, tl, c);
#pragma unroll
        for (int wi = 0; wi < WPC; ++wi) {
          const int w = c * WPC + wi;
          const int gw = (8 * w) / g.gk;
          if (gw != cur_g) {  // flush the finished group (uniform branch)
            const float x = fmaf((float)d2, kInv254sq, fmaf((float)d1, kInv254, (float)d0));
            s = fmaf(load_scale(ks, tl * g.ngk + cur_g, 1), qa * x, s);
            d0 = d1 = d2 = 0;
            cur_g = gw;
          }
          int ev, od;
          nibbles_to_s8(ch.w[wi], ev, od);
          d0 = __dp4a(od, (int)qw[0][2 * w + 1], __dp4a(ev, (int)qw[0][2 * w], d0));
          d1 = __dp4a(od, (int)qw[1][2 * w + 1], __dp4a(ev, (int)qw[1][2 * w], d1));
          d2 = __dp4a(od, (int)qw[2][2 * w + 1], __dp4a(ev, (int)qw[2][2 * w], d2));
        }
      }
    }
    const float x = fmaf((float)d2, kInv254sq, fmaf((float)d1, kInv254, (float)d0));
    return fmaf(load_scale(ks, tl * g.ngk + cur_g, 1), qa * x, s);
  }
}

struct SmemLayout {
  int stage_bytes;
  int off_kc, off_vc, off_ks, off_vs;  // within a stage
  int off_q, off_bk, off_bv;           // q^h, B_K^h, B_V^h staged once per CTA
  int off_tw;                          // per consumer warp: weight expansion bytes [ngv][3][32]
  int off_qt;                          // q~ [kMaxR] floats
  int off_qterm;                       // q~ expansion bytes [3][kMaxR]
  int off_wst;                         // per consumer warp: (m, l, u[kMaxR])
  int off_cta;                         // CTA partial [2 + kMaxR]
  int off_mw;                          // merge weights [kMaxSplit]
  int off_bar;                         // full[kMaxStages], empty[kMaxStages], factor barrier
  int off_misc;
  int total;
};

constexpr int kSmemFixed = kMaxR * 4 + 3 * kMaxR + kCW * (2 + kMaxR) * 4 + (2 + kMaxR) * 4 + kMaxSplit * 4 +
                           (2 * kMaxStages + 1) * 8 + 16;

LK_DEVICE SmemLayout smem_layout(const DecodeParams& p) {
  SmemLayout L;
  L.off_kc = 0;
  L.off_vc = p.st_kc;
  L.off_ks = p.st_kc + p.st_vc;
  L.off_vs = p.st_kc + p.st_vc + p.st_ks;
  L.stage_bytes = p.st_kc + p.st_vc + p.st_ks + p.st_vs;
  L.off_q = p.nstages * L.stage_bytes;
  L.off_bk = L.off_q + p.st_q;
  L.off_bv = L.off_bk + p.st_bk;
  L.off_tw = L.off_bv + p.st_bv;
  L.off_qt = L.off_tw + p.st_tw;
  L.off_qterm = L.off_qt + kMaxR * 4;
  L.off_wst = L.off_qterm + 3 * kMaxR;
  L.off_cta = L.off_wst + kCW * (2 + kMaxR) * 4;
  L.off_mw = L.off_cta + (2 + kMaxR) * 4;
  L.off_bar = L.off_mw + kMaxSplit * 4;
  L.off_misc = L.off_bar + (2 * kMaxStages + 1) * 8;
  L.total = L.off_misc + 16;
  return L;
}

inline int smem_bytes_for(const DecodeParams& p) {
  const int stage = p.st_kc + p.st_vc + p.st_ks + p.st_vs;
  return p.nstages * stage + p.st_q + p.st_bk + p.st_bv + p.st_tw + kSmemFixed;
}

template <int KIND, int CSK, int CSV>
LK_DEVICE void decode_body(const DecodeParams& p, const HeadGeom& g, uint8_t* smem, const SmemLayout& L,
                           int b, int h, int split, int len, int first_stage, int n_my) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.head_dim;
  const int NS = p.nstages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.off_bar);
  uint64_t* empty = full + kMaxStages;
  uint64_t* fbar = full + 2 * kMaxStages;
  float* qt_s = reinterpret_cast<float*>(smem + L.off_qt);
  int8_t* qterm = reinterpret_cast<int8_t*>(smem + L.off_qterm);
  float* wst = reinterpret_cast<float*>(smem + L.off_wst);
  float* cta = reinterpret_cast<float*>(smem + L.off_cta);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.off_misc);
  int* flag = reinterpret_cast<int*>(smem + L.off_misc) + 1;
  float* qa_s = reinterpret_cast<float*>(smem + L.off_misc) + 2;
  const int ssz = KIND == 0 ? 4 : 2;
  const int64_t bh = (int64_t)b * p.n_heads + h;

  auto issue = [&](int j) {  // stage j of this split -> buffer j % NS
    const int buf = j % NS;
    const int64_t t0 = (int64_t)(first_stage + j) * kStageT;
    const int64_t end = min((int64_t)((len + 15) & ~15), (int64_t)p.capacity);
    const int ntok = (int)min((int64_t)kStageT, end - t0);
    uint8_t* st = smem + buf * L.stage_bytes;
    const uint32_t bkc = ntok * g.rbk, bvc = ntok * g.rbv;
    const uint32_t bks = ntok * g.ngk * ssz, bvs = ntok * g.ngv * ssz;
    lk_mbar_arrive_expect_tx(&full[buf], bkc + bvc + bks + bvs);
    lk_bulk_g2s(st + L.off_kc, p.codes_k + g.kc_off + t0 * g.rbk, bkc, &full[buf]);
    lk_bulk_g2s(st + L.off_vc, p.codes_v + g.vc_off + t0 * g.rbv, bvc, &full[buf]);
    lk_bulk_g2s(st + L.off_ks, p.scales_k + (g.ks_off + t0 * g.ngk) * ssz, bks, &full[buf]);
    lk_bulk_g2s(st + L.off_vs, p.scales_v + (g.vs_off + t0 * g.ngv) * ssz, bvs, &full[buf]);
  };
  // the producer starts the copies at once: B_V^h, then the first stages (the
  // buffers are free), so they stream in while q is absorbed
  if (tid == kConsumerThreads) {
    const uint32_t qb = H * p.q_size, bkb = g.rk * H * p.b_size, bvb = g.rv * H * p.b_size;
    lk_mbar_arrive_expect_tx(fbar, qb + bkb + bvb);
    lk_bulk_g2s(smem + L.off_q, static_cast<const uint8_t*>(p.q) + bh * H * p.q_size, qb, fbar);
    lk_bulk_g2s(smem + L.off_bk, static_cast<const uint8_t*>(p.BK) + g.bk_off * p.b_size, bkb, fbar);
    lk_bulk_g2s(smem + L.off_bv, static_cast<const uint8_t*>(p.BV) + g.bv_off * p.b_size, bvb, fbar);
    for (int j = 0; j < min(NS, n_my); ++j) issue(j);
  }

  // ---- absorb q (consumer warps): q~[i] = qscale * sum_d B_K[i][d] q[d] from the
  //      staged copies of q^h and B_K^h
  if (warp < kCW) {
    if (!lk_mbar_wait_bounded(fbar, 0, LK_WAIT_LIMIT_NS)) *abort_flag = 1;
    const uint8_t* qs = smem + L.off_q;
    const uint8_t* bks = smem + L.off_bk;
    if (!*abort_flag) {
      for (int i = warp; i < g.rk; i += kCW) {
        float acc = 0.0f;
        for (int d = lane; d < H; d += 32) acc = fmaf(ld_f(qs, d, p.q_bf16), ld_f(bks, i * H + d, p.b_bf16), acc);
        acc = lk_warp_sum(acc);
        if (lane == 0) qt_s[i] = acc * p.qscale;
      }
    }
  }
  __syncthreads();
  // ---- three-term int8 expansion of q~ (warp 0): q~ = a (t0 + t1/254 + t2/254^2)
  if (warp == 0) {
    const float v0 = lane < g.rk ? qt_s[lane] : 0.0f;
    const float v1 = lane + 32 < g.rk ? qt_s[lane + 32] : 0.0f;
    const float amax = lk_warp_max(fmaxf(fabsf(v0), fabsf(v1)));
    const float a = amax / 127.0f;
    const float inva = amax > 0.0f ? 127.0f / amax : 0.0f;
#pragma unroll
    for (int q2 = 0; q2 < 2; ++q2) {
      const float x = (q2 == 0 ? v0 : v1) * inva;
      const float t0 = rintf(x);
      const float x1 = (x - t0) * 254.0f;
      const float t1 = rintf(x1);
      const float t2 = fminf(fmaxf(rintf((x1 - t1) * 254.0f), -127.0f), 127.0f);
      const int d = lane + 32 * q2;
      // int4 keys meet even dims and odd dims in separate words
      const int pos = KIND == 0 ? d : ((d >> 3) << 3) + ((d & 1) ? 4 : 0) + ((d & 7) >> 1);
      const bool live = d < g.rk;
      qterm[0 * kMaxR + pos] = (int8_t)(live ? (int)t0 : 0);
      qterm[1 * kMaxR + pos] = (int8_t)(live ? (int)t1 : 0);
      qterm[2 * kMaxR + pos] = (int8_t)(live ? (int)t2 : 0);
    }
    if (lane == 0) *qa_s = a;
  }
  __syncthreads();

  if (warp == kCW) {
    // ================= producer warp: bulk copies, gated by the empty barriers
    if (lane == 0) {
      int issued = min(NS, n_my);
      for (int j = issued; j < n_my; ++j) {
        if (*abort_flag) break;
        if (j >= NS) {  // the consumers released this buffer's previous stage
          if (!lk_mbar_wait_bounded(&empty[j % NS], (uint32_t)(((j / NS) - 1) & 1), LK_WAIT_LIMIT_NS)) {
            *abort_flag = 1;
            break;
          }
        }
        issue(j);
        issued = j + 1;
      }
      // before the CTA may finish, every copy this CTA started has landed
      for (int j = max(0, issued - NS); j < issued; ++j) {
        if (!lk_mbar_wait_bounded(&full[j % NS], (uint32_t)((j / NS) & 1), LK_WAIT_LIMIT_NS)) {
          lk_dev_fail(LK_DEV_TIMEOUT_DRAIN);
          *abort_flag = 1;
        }
      }
      if (!lk_mbar_wait_bounded(fbar, 0, LK_WAIT_LIMIT_NS)) {
        lk_dev_fail(LK_DEV_TIMEOUT_DRAIN);
        *abort_flag = 1;
      }
    }
  } else {
    // ================= consumer warp: tokens 32 * warp .. 32 * warp + 31 of every stage
    const float qa = *qa_s;
    uint32_t qw[3][kMaxWords];
#pragma unroll
    for (int i = 0; i < 3; ++i)
#pragma unroll
      for (int w = 0; w < kMaxWords; ++w) qw[i][w] = reinterpret_cast<const uint32_t*>(qterm + i * kMaxR)[w];
    // weight-expansion bytes of this warp: [group][term][32 tokens]
    int8_t* tw = reinterpret_cast<int8_t*>(smem + L.off_tw) + warp * (p.st_tw / kCW);
    const int tl = 32 * warp + lane;  // this lane's token within a stage
    // int4 values: even and odd tokens of an octet live in separate words
    const int tpos = KIND == 0 ? lane : (lane & ~7) + ((lane & 1) ? 4 : 0) + ((lane & 7) >> 1);
    // V: this lane owns latent dims lane and lane + 32; exact int32 sums of
    // (expanded weight term) x code, folded into float only when the running
    // max or the reference scale changes
    int A[2][kWTerms];
    float u[2] = {0.0f, 0.0f};
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int i = 0; i < kWTerms; ++i) A[k][i] = 0;
    float m_run = -INFINITY, l_run = 0.0f;
    float wref = 0.0f;  // every weight of the open accumulation is <= wref
    auto fold = [&](float alpha) {
      const float sc = wref * (1.0f / 127.0f);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        float x = (float)A[k][kWTerms - 1];
#pragma unroll
        for (int i = kWTerms - 2; i >= 0; --i) x = fmaf(x, kInv254, (float)A[k][i]);
        u[k] = (u[k] + sc * x) * alpha;
#pragma unroll
        for (int i = 0; i < kWTerms; ++i) A[k][i] = 0;
      }
    };

    for (int j = 0; j < n_my; ++j) {
      const int buf = j % NS;
      if (!lk_mbar_wait_bounded(&full[buf], (uint32_t)((j / NS) & 1), LK_WAIT_LIMIT_NS)) *abort_flag = 1;
      if (*abort_flag) break;
      const uint8_t* st = smem + buf * L.stage_bytes;
      const uint8_t* vs = st + L.off_vs;
      const bool valid = (first_stage + j) * kStageT + tl < len;
      // a. score; a new running max (warp vote) folds the open sums
      float s = -INFINITY;
      if (valid) s = token_score<KIND, CSK>(st + L.off_kc, st + L.off_ks, g, tl, qw, qa);
      if (__any_sync(0xffffffffu, s > m_run)) {
        const float m_new = fmaxf(m_run, lk_warp_max(s));
        const float alpha = (m_run == -INFINITY) ? 0.0f : exp2f(m_run - m_new);
        fold(alpha);
        l_run *= alpha;
        m_run = m_new;
      }
      const float pr = valid ? exp2f(s - m_run) : 0.0f;
      l_run += pr;
      // b. reference scale: a larger V scale (warp vote) folds, then raises wref
      float smax_t = 0.0f;
      for (int gi = 0; gi < g.ngv; ++gi) smax_t = fmaxf(smax_t, valid ? load_scale(vs, tl * g.ngv + gi, KIND) : 0.0f);
      if (__any_sync(0xffffffffu, smax_t > wref)) {
        fold(1.0f);
        wref = fmaxf(wref, lk_warp_max(smax_t));
      }
      //    weights w = p sigma_V as a four-term int8 expansion of w * 127 / wref
      const float inv = wref > 0.0f ? 127.0f / wref : 0.0f;
      for (int gi = 0; gi < g.ngv; ++gi) {
        const float sg = valid ? load_scale(vs, tl * g.ngv + gi, KIND) : 0.0f;
        float x = fminf(pr * sg * inv, 127.0f);
        int8_t* tg = tw + gi * (kWTerms * 32);
#pragma unroll
        for (int i = 0; i < kWTerms; ++i) {
          const float t = fminf(fmaxf(rintf(x), -127.0f), 127.0f);
          tg[32 * i + tpos] = (int8_t)(int)t;
          x = (x - t) * 254.0f;
        }
      }
      __syncwarp();
      // c. A[d][i] += sum over the warp's 32 tokens of term_i(t) * c_{t,d}
      const uint8_t* vc = st + L.off_vc;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int d = lane + 32 * k;
        if (d < g.rv) {
          const int gi = KIND == 0 ? 0 : d / g.gv;
          const uint32_t* T = reinterpret_cast<const uint32_t*>(tw + gi * (kWTerms * 32));
#pragma unroll
          for (int blk = 0; blk < 2; ++blk) {  // the warp's two 16-token blocks
            const int b16 = 2 * warp + blk;
            if (KIND == 0) {
              const uint4 v = *reinterpret_cast<const uint4*>(vc + b16 * 16 * g.rbv + d * 16);
              const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int qd = 0; qd < 4; ++qd)
#pragma unroll
                for (int i = 0; i < kWTerms; ++i) A[k][i] = __dp4a((int)vw[qd], (int)T[8 * i + 4 * blk + qd], A[k][i]);
            } else {
              const uint2 v = *reinterpret_cast<const uint2*>(vc + b16 * 16 * g.rbv + d * 8);
              const uint32_t vw[2] = {v.x, v.y};
#pragma unroll
              for (int oc = 0; oc < 2; ++oc) {
                int ev, od;
                nibbles_to_s8(vw[oc], ev, od);
                const int o = 2 * blk + oc;  // octet of the warp's tokens
#pragma unroll
                for (int i = 0; i < kWTerms; ++i)
                  A[k][i] = __dp4a(od, (int)T[8 * i + 2 * o + 1], __dp4a(ev, (int)T[8 * i + 2 * o], A[k][i]));
              }
            }
          }
        }
      }
      __syncwarp();  // this warp is done with the stage buffer and its weight bytes
      if (lane == 0) lk_mbar_arrive(&empty[buf]);
    }
    fold(1.0f);
    // per-warp state (m, l, u)
    const float lw = lk_warp_sum(l_run);
    float* ws = wst + warp * (2 + kMaxR);
    if (lane == 0) {
      ws[0] = m_run;
      ws[1] = lw;
    }
    if (lane < g.rv) ws[2 + lane] = u[0];
    if (lane + 32 < g.rv) ws[2 + lane + 32] = u[1];
  }
  __syncthreads();
  const bool aborted = *abort_flag != 0;
  if (aborted && tid == 0) lk_dev_fail(LK_DEV_TIMEOUT_PIPE);

  // ---- merge the consumer warps' states into the CTA partial
  {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kCW; ++w) M = fmaxf(M, wst[w * (2 + kMaxR)]);
    const int idx = (tid < g.rv) ? 2 + tid : (tid == kMaxR ? 1 : -1);
    float acc = 0.0f;
    if (idx >= 0 && M != -INFINITY && !aborted) {
#pragma unroll
      for (int w = 0; w < kCW; ++w) {
        const float mw = wst[w * (2 + kMaxR)];
        if (mw != -INFINITY) acc += wst[w * (2 + kMaxR) + idx] * exp2f(mw - M);
      }
    }
    if (idx >= 0) cta[idx] = acc;
    if (tid == 0) cta[0] = aborted ? -INFINITY : M;
  }
  __syncthreads();

  const int idx = (tid < g.rv) ? 2 + tid : (tid == kMaxR ? 1 : -1);
  if (p.cluster_merge) {
    // the head's splits form one cluster: rank 0 merges the partials straight
    // from the other CTAs' shared memory
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const unsigned nrank = cluster.num_blocks();
    const bool lead = cluster.block_rank() == 0;
    float acc = 0.0f, Mg = -INFINITY;
    if (lead) {
      for (unsigned q = 0; q < nrank; ++q) Mg = fmaxf(Mg, cluster.map_shared_rank(cta, q)[0]);
      if (idx >= 0 && Mg != -INFINITY) {
        for (unsigned q = 0; q < nrank; ++q) {
          const float* pq = cluster.map_shared_rank(cta, q);
          const float mq = pq[0];
          if (mq != -INFINITY) acc += pq[idx] * exp2f(mq - Mg);
        }
      }
    }
    cluster.sync();  // every rank's partial has been read
    if (!lead) return;
    if (idx >= 0) cta[idx] = acc;
    if (tid == 0) cta[0] = Mg;
    __syncthreads();
  } else if (p.n_split > 1) {
    float* part = p.partials + (bh * p.n_split + split) * p.part_stride;
    for (int i = tid; i < 2 + g.rv; i += kThreads) part[i] = cta[i];
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const int ticket = atomicAdd(&p.counters[bh], 1);
      *flag = (ticket == p.n_split - 1);
    }
    __syncthreads();
    if (!*flag) return;
    __threadfence();
    // last arriver: merge every split's partial (all visible in L2), all
    // splits' loads in flight at once
    float* mw = reinterpret_cast<float*>(smem + L.off_mw);
    const float* P0 = p.partials + bh * p.n_split * p.part_stride;
    for (int s2 = tid; s2 < p.n_split; s2 += kThreads) mw[s2] = __ldcg(P0 + (int64_t)s2 * p.part_stride);
    __syncthreads();
    float Mg = -INFINITY;
    for (int s2 = 0; s2 < p.n_split; ++s2) Mg = fmaxf(Mg, mw[s2]);
    __syncthreads();
    for (int s2 = tid; s2 < p.n_split; s2 += kThreads)
      mw[s2] = (mw[s2] == -INFINITY || Mg == -INFINITY) ? 0.0f : exp2f(mw[s2] - Mg);
    __syncthreads();
    float acc = 0.0f;
    if (idx >= 0) {
      int s2 = 0;
      for (; s2 + 4 <= p.n_split; s2 += 4) {
        const float v0 = __ldcg(P0 + (int64_t)(s2 + 0) * p.part_stride + idx);
        const float v1 = __ldcg(P0 + (int64_t)(s2 + 1) * p.part_stride + idx);
        const float v2 = __ldcg(P0 + (int64_t)(s2 + 2) * p.part_stride + idx);
        const float v3 = __ldcg(P0 + (int64_t)(s2 + 3) * p.part_stride + idx);
        acc += v0 * mw[s2] + v1 * mw[s2 + 1] + v2 * mw[s2 + 2] + v3 * mw[s2 + 3];
      }
      for (; s2 < p.n_split; ++s2) acc += __ldcg(P0 + (int64_t)s2 * p.part_stride + idx) * mw[s2];
    }
    __syncthreads();
    if (idx >= 0) cta[idx] = acc;
    if (tid == 0) {
      cta[0] = Mg;
      p.counters[bh] = 0;  // ready for the next call
    }
    __syncthreads();
  }

  // ---- out = (u / l) B_V^h, B_V^h from shared memory
  const float lsum = cta[1];
  const float inv = (cta[0] == -INFINITY || lsum == 0.0f || aborted) ? 0.0f : 1.0f / lsum;
  const uint8_t* bvs = smem + L.off_bv;
  const int64_t ooff = bh * H;
  for (int d = tid; d < H; d += kThreads) {
    float o = 0.0f;
    for (int j = 0; j < g.rv; ++j) o = fmaf(cta[2 + j], ld_f(bvs, j * H + d, p.b_bf16), o);
    o *= inv;
    if (p.out_bf16) reinterpret_cast<uint16_t*>(p.out)[ooff + d] = lk_f32_to_bf16(o);
    else reinterpret_cast<float*>(p.out)[ooff + d] = o;
  }
}

template <int KIND>
__global__ void __launch_bounds__(kThreads, 2) decode_attn_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const SmemLayout L = smem_layout(p);
  const HeadGeom g = head_geometry<KIND>(p, b, h);
  int len = p.seq_len[b];
  len = max(0, min(len, p.max_len));

  const int total_stages = (len + kStageT - 1) / kStageT;
  const int first_stage = split * p.stages_per_split;
  const int n_my = max(0, min(p.stages_per_split, total_stages - first_stage));

  if (threadIdx.x == 0) {
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.off_bar);
    for (int i = 0; i < kMaxStages; ++i) lk_mbar_init(&bars[i], 1);                       // full
    for (int i = kMaxStages; i < 2 * kMaxStages; ++i) lk_mbar_init(&bars[i], kCW);       // empty
    lk_mbar_init(&bars[2 * kMaxStages], 1);                                              // factor
    lk_fence_mbar_init();
    *reinterpret_cast<int*>(smem + L.off_misc) = 0;
  }
  __syncthreads();

  const int csk = lk_chunk_bytes(g.rbk), csv = lk_chunk_bytes(g.rbv);
#define LK_BODY(A, B_) decode_body<KIND, A, B_>(p, g, smem, L, b, h, split, len, first_stage, n_my)
  if (csk == 16) {
    if (csv == 16) LK_BODY(16, 16); else if (csv == 8) LK_BODY(16, 8); else LK_BODY(16, 4);
  } else if (csk == 8) {
    if (csv == 16) LK_BODY(8, 16); else if (csv == 8) LK_BODY(8, 8); else LK_BODY(8, 4);
  } else {
    if (csv == 16) LK_BODY(4, 16); else if (csv == 8) LK_BODY(4, 8); else LK_BODY(4, 4);
  }
#undef LK_BODY
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

}  // namespace

LK_DEFINE_STATUS_ACCESSOR(lk_decode_status_word)

namespace lk {

int decode_pick_split(int units, int max_len, int num_sms) {
  const int stages = (max_len + kStageT - 1) / kStageT;
  if (stages <= 1) return 1;
  // splitting only pays while the (batch, head) units leave SMs idle: with
  // two resident CTAs per SM, aim for about one full wave
  if (units >= num_sms) return 1;
  const int target = num_sms * 2;
  int s = (target + units - 1) / units;
  s = std::max(1, std::min(std::min(s, stages), 8));  // <= 8: the splits merge inside one cluster
  return s;
}

size_t decode_workspace_bytes(int batch, int n_heads, int rv_max, int n_split) {
  const size_t counters = (size_t)round_up(batch * n_heads * 4, 256);
  const size_t stride = (size_t)round_up(2 + rv_max, 4);
  return counters + (size_t)batch * n_heads * n_split * stride * 4;
}

cudaError_t launch_decode_attn(const DecodeLaunch& a, cudaStream_t stream) {
  DecodeParams p{};
  p.codes_k = static_cast<const uint8_t*>(a.codes_k);
  p.codes_v = static_cast<const uint8_t*>(a.codes_v);
  p.scales_k = static_cast<const uint8_t*>(a.scales_k);
  p.scales_v = static_cast<const uint8_t*>(a.scales_v);
  p.q = a.q;
  p.BK = a.BK;
  p.BV = a.BV;
  p.seq_len = a.seq_len;
  p.out = a.out;
  p.batch = a.batch;
  p.n_heads = a.n_heads;
  p.head_dim = a.head_dim;
  p.capacity = a.capacity;
  p.group_k = a.group_k;
  p.group_v = a.group_v;
  p.q_bf16 = a.q_bf16;
  p.b_bf16 = a.b_bf16;
  p.out_bf16 = a.out_bf16;
  p.max_len = a.max_len;
  p.qscale = a.softmax_scale * 1.4426950408889634f;
  int rk_max = 0, rv_max = 0, ngk_max = 1, ngv_max = 1;
  for (int h = 0; h < a.n_heads; ++h) {
    p.rk[h] = (uint8_t)a.ranks_k[h];
    p.rv[h] = (uint8_t)a.ranks_v[h];
    rk_max = std::max(rk_max, a.ranks_k[h]);
    rv_max = std::max(rv_max, a.ranks_v[h]);
    if (a.kind == 1) {
      const int gk = std::min(a.group_k, a.ranks_k[h]), gv = std::min(a.group_v, a.ranks_v[h]);
      ngk_max = std::max(ngk_max, (a.ranks_k[h] + gk - 1) / gk);
      ngv_max = std::max(ngv_max, (a.ranks_v[h] + gv - 1) / gv);
    }
  }
  const int rbk_max = a.kind == 0 ? rk_max : rk_max / 2;
  const int rbv_max = a.kind == 0 ? rv_max : rv_max / 2;
  const int ssz = a.kind == 0 ? 4 : 2;
  p.st_kc = round_up(kStageT * rbk_max, 128);
  p.st_vc = round_up(kStageT * rbv_max, 128);
  p.st_ks = round_up(kStageT * ngk_max * ssz, 128);
  p.st_vs = round_up(kStageT * ngv_max * ssz, 128);
  p.q_size = a.q_bf16 ? 2 : 4;
  p.b_size = a.b_bf16 ? 2 : 4;
  p.st_q = round_up(a.head_dim * p.q_size, 128);
  p.st_bk = round_up(rk_max * a.head_dim * p.b_size, 128);
  p.st_bv = round_up(rv_max * a.head_dim * p.b_size, 128);
  p.st_tw = kCW * round_up(ngv_max * kWTerms * 32, 16);
  // as many stages as fit while two CTAs share an SM (about 64 KB of copies
  // in flight per SM keeps HBM busy), between 2 and kMaxStages
  {
    p.nstages = 0;
    const int stage = p.st_kc + p.st_vc + p.st_ks + p.st_vs;
    const int room = 110 * 1024 - (smem_bytes_for(p));  // smem_bytes_for counts 0 stages here
    p.nstages = std::max(2, std::min(kMaxStages, room / std::max(stage, 1)));
  }
  const int stages = std::max(1, (a.max_len + kStageT - 1) / kStageT);
  int n_split = a.n_split;
  if (n_split <= 0) n_split = decode_pick_split(a.batch * a.n_heads, a.max_len, a.num_sms);
  n_split = std::max(1, std::min(std::min(n_split, stages), kMaxSplit));
  p.stages_per_split = (stages + n_split - 1) / n_split;
  n_split = (stages + p.stages_per_split - 1) / p.stages_per_split;
  p.n_split = n_split;
  p.part_stride = round_up(2 + rv_max, 4);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  p.counters = reinterpret_cast<int32_t*>(ws);
  p.partials = reinterpret_cast<float*>(ws + round_up(a.batch * a.n_heads * 4, 256));

  // up to eight splits of a head merge inside a cluster (portable cluster size)
  p.cluster_merge = (n_split > 1 && n_split <= 8) ? 1 : 0;
  const int smem = smem_bytes_for(p);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_split, a.n_heads, a.batch);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.cluster_merge ? n_split : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (a.kind == 0) {
    e = cudaFuncSetAttribute(decode_attn_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, decode_attn_kernel<0>, p);
  } else {
    e = cudaFuncSetAttribute(decode_attn_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, decode_attn_kernel<1>, p);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace lk

// ---------------------------------------------------------------- allocation-free variant
// Split-K scratch for lk_latent_decode_attn_noalloc: a file-scope device
// array (zero at load), so callers that cannot allocate need no workspace.
// Host code must not hand its name to a kernel (in host code it is only a
// stand-in); the device address is looked up once per device below.
#include <cstdio>
#include <mutex>

namespace lk {
lk_status set_error(lk_status s, const char* msg);
}

static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[LK_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoallocMaxDevices] = {};
}  // namespace

extern "C" lk_status lk_latent_decode_attn_noalloc(const lk_latent_cache* k, const lk_latent_cache* v,
                                                   const void* q, lk_dtype q_dtype, const void* B_K,
                                                   const void* B_V, lk_dtype b_dtype, int32_t head_dim,
                                                   const int32_t* seq_len, int32_t max_seq_len,
                                                   float softmax_scale, void* out, lk_dtype out_dtype,
                                                   int32_t n_split, lk_stream_t stream) {
  char msg[256];
  // enough of the arguments to size the scratch; lk_latent_decode_attn checks the rest
  if (!k || !v || !k->ranks || !v->ranks) return lk::set_error(LK_ERR_INVALID_ARG, "null cache descriptor or ranks");
  if (k->batch < 1 || k->n_heads < 1 || k->n_heads > LK_MAX_HEADS || v->n_heads != k->n_heads ||
      v->batch != k->batch || max_seq_len < 0 || n_split < 0)
    return lk::set_error(LK_ERR_SHAPE, "bad batch, heads, max_seq_len or n_split");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) {
    snprintf(msg, sizeof(msg), "lk_latent_decode_attn_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
    return lk::set_error(LK_ERR_CUDA, msg);
  }
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
      // once per device, with that device current
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_decode_noalloc_scratch);
      if (e != cudaSuccess || !p) {
        snprintf(msg, sizeof(msg), "lk_latent_decode_attn_noalloc: cudaGetSymbolAddress: %s",
                 cudaGetErrorString(e));
        return lk::set_error(LK_ERR_CUDA, msg);
      }
      g_noalloc_ptr[dev] = p;
    }
    scratch = g_noalloc_ptr[dev];
  }
  int rv_max = 0;
  for (int h = 0; h < v->n_heads; ++h) rv_max = std::max(rv_max, (int)v->ranks[h]);
  int num_sms = 0;
  if (cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || num_sms <= 0)
    num_sms = 148;
  const int stages = std::max(1, (max_seq_len + kStageT - 1) / kStageT);
  int n_eff = n_split > 0 ? std::min(n_split, stages) : lk::decode_pick_split(k->batch * k->n_heads, max_seq_len, num_sms);
  n_eff = std::max(1, std::min(std::min(n_eff, stages), kMaxSplit));
  const size_t need = lk::decode_workspace_bytes(k->batch, k->n_heads, rv_max, n_eff);
  if (need > LK_DECODE_NOALLOC_SCRATCH_BYTES) {
    snprintf(msg, sizeof(msg),
             "lk_latent_decode_attn_noalloc: needs %zu bytes of scratch, the static array holds %u; "
             "lower n_split or use lk_latent_decode_attn with a workspace",
             need, (unsigned)LK_DECODE_NOALLOC_SCRATCH_BYTES);
    return lk::set_error(LK_ERR_WORKSPACE, msg);
  }
  const lk_status st = lk_latent_decode_attn(k, v, q, q_dtype, B_K, B_V, b_dtype, head_dim, seq_len, max_seq_len,
                                             softmax_scale, out, out_dtype, n_eff, scratch,
                                             LK_DECODE_NOALLOC_SCRATCH_BYTES, stream);
  if (st != LK_OK) return st;
  // leave the arrival counters zero for the next call (the kernel already does;
  // this also covers a call cut short)
  const size_t counters = (size_t)((k->batch * k->n_heads * 4 + 255) / 256 * 256);
  e = cudaMemsetAsync(scratch, 0, counters, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "lk_latent_decode_attn_noalloc: clearing counters: %s", cudaGetErrorString(e));
    return lk::set_error(LK_ERR_CUDA, msg);
  }
  return LK_OK;
}
