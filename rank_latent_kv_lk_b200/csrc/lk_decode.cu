// Latent decode attention on B200 (sm_100a): a persistent, stream-K
// flash-decode over the per-head latent cache.
//
// What it computes (WSVD page, technical summary §2A and §2C): for every batch
// row b and head h, softmax(q K^T / sqrt(H)) V with K = dequant(C_K) B_K and
// V = dequant(C_V) B_V, without forming K or V.  Without positional rotation
// q K^T = (B_K q)^T dequant(C_K)^T, so q is absorbed once per head
// (q~ = B_K q) and scores are taken against the latent codes; the
// probability-weighted latent sum u = sum_t p_t dequant(c_V[t]) is up-projected
// once, out = (u / sum_t p_t) B_V.
//
// Work split.  A (b, h) pair is a unit; a unit's tokens are cut into stages
// of 224.  The (unit, stage) items, in unit order, are dealt out in equal
// contiguous ranges to a fixed grid of CTAs (two per SM by default), so every
// SM streams the same number of bytes and each CTA pays its start-up once.  A
// CTA walks its range: at a unit boundary it absorbs the next q (its q and B_K
// copies were prefetched while the previous unit streamed), then streams the
// unit's stages through an NS-deep ring of shared-memory buffers filled with
// bulk copies (TMA engine) by a producer warp.  A unit that lies inside one
// CTA is finished there; a unit cut by range boundaries leaves one partial
// (m, l, u) per piece, and the piece that arrives last (atomic ticket, no
// waiting) merges them and writes the output.
//
// Per stage, each of 7 consumer warps takes 32 tokens:
//   a. score, one token per lane: s_t = sigma_K[t] (c_K[t] . q~), exact int32
//      dp4a sums against a three-term int8 expansion of q~
//      (q~ = a (t0 + t1/254 + t2/254^2), error <= 6e-8 max|q~|);
//   b. running max by warp vote, p_t = 2^(s_t - m);
//   c. w_t = p_t sigma_V[t] as four int8 terms relative to a reference scale,
//      then u_d += sum_t w_t c_V[t][d] as exact int8 tensor-core products
//      [4 terms x 32 tokens] x [32 tokens x 8 dims] (mma.sync m16n8k32),
//      folded into float only when the max or the reference changes.
// Every wait on a shared-memory barrier is bounded (2 s); an expired wait
// sets the library status word, stops the math and lets the CTA finish its
// protocol steps, so no other CTA waits on it.
#include <atomic>
#include <map>
#include <mutex>
#include <tuple>

#include "lk_common.cuh"
#include "lk_internal.h"

namespace {

// 7 consumer warps + 1 producer warp: two CTAs of 8 warps fill an SM with 4
// warps per scheduler and leave each thread 128 registers (a ninth warp would
// put 5 warps on one scheduler and cap every thread at 96)
constexpr int kCW = 7;                           // consumer warps
constexpr int kConsumerThreads = kCW * 32;
constexpr int kThreads = kConsumerThreads + 32;  // + one producer warp
// tokens per stage: TG groups of 32 per consumer warp (TG = 2 when two stages
// of the widest head fit beside each other in ~110 KB, else 1)
constexpr int kStageMin = 32 * kCW;  // 224 (TG = 1); 448 with TG = 2
constexpr int kMaxStages = 8;                    // ring depth chosen at launch (2 .. 8)
constexpr int kMaxR = LK_MAX_RANK;
constexpr int kAutoCtaBound = 1024;              // grid bound of the automatic split (sizes the workspace)

// Per-head geometry, computed on the host (prefix sums over the heads of a
// batch row).
struct HeadInfo {
  uint8_t rk, rv;     // ranks
  uint8_t ngk, ngv;   // scale groups per token (1 for int8)
  uint8_t gk, gv;     // effective group sizes (int4; = rank for int8)
  uint16_t pk, pv;    // code bytes of the heads before this one (one batch row)
  uint16_t pgk, pgv;  // scale groups of the heads before this one
  uint16_t prk, prv;  // ranks of the heads before this one (offset of B_K^h / B_V^h rows)
};

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
  float* partials;    // [G][2][part_stride]: a CTA's first and last unit pieces
  int32_t* counters;  // [units] arrival tickets, zero at entry, left zero
  int n_heads, head_dim, capacity;
  int tk, tv, tgk, tgv;  // code bytes / scale groups of one batch row (all heads)
  int q_bf16, b_bf16, out_bf16;
  int early_inputs;  // q, B_K, B_V are read before waiting for the previous kernel on the stream
  int stable_len;    // with early_inputs: cache positions below it are final before the kernel starts
  uint64_t wait_ns;  // limit of the pipeline waits (draining copies after an error always allows 2 s)
  int stall_item;    // test hook: the producer stops before this (unit, stage) item (-1: never)
  int max_len;
  int ST;  // tokens per stage: 32 * TG * kCW
  int S;   // stages per unit: ceil(max_len / ST)
  int W;   // items: units * S
  int G;   // CTAs
  int part_stride;
  float qscale;  // softmax_scale * log2(e)
  // bytes of the shared-memory regions (max over heads), multiples of 128
  int st_kc, st_vc, st_ks, st_vs, st_q, st_bk, st_bv, st_fr;
  int nstages;
  int q_size, b_size;  // element sizes of q and of the factors
  HeadInfo head[LK_MAX_HEADS];
};

struct HeadGeom {
  int rk, rv;      // ranks
  int rbk, rbv;    // code bytes per token
  int ngk, ngv;    // scale groups per token
  int gk, gv;      // effective group sizes
  int64_t kc_off;  // byte offset of this (b, h) K code plane
  int64_t vc_off;
  int64_t ks_off;  // element offset of this (b, h) K scale plane
  int64_t vs_off;
  int64_t bk_off;  // element offset of B_K^h
  int64_t bv_off;
};

template <int KIND>
LK_DEVICE HeadGeom unit_geometry(const DecodeParams& p, int b, int h) {
  const HeadInfo& hi = p.head[h];
  HeadGeom g;
  g.rk = hi.rk;
  g.rv = hi.rv;
  g.rbk = KIND == 0 ? g.rk : g.rk / 2;
  g.rbv = KIND == 0 ? g.rv : g.rv / 2;
  g.ngk = hi.ngk;
  g.ngv = hi.ngv;
  g.gk = hi.gk;
  g.gv = hi.gv;
  const int64_t cap = p.capacity;
  g.kc_off = ((int64_t)b * p.tk + hi.pk) * cap;
  g.vc_off = ((int64_t)b * p.tv + hi.pv) * cap;
  g.ks_off = ((int64_t)b * p.tgk + hi.pgk) * cap;
  g.vs_off = ((int64_t)b * p.tgv + hi.pgv) * cap;
  g.bk_off = (int64_t)hi.prk * p.head_dim;
  g.bv_off = (int64_t)hi.prv * p.head_dim;
  return g;
}

LK_DEVICE int unit_len(const DecodeParams& p, int b) { return max(0, min(p.seq_len[b], p.max_len)); }

// First item of CTA c, and the CTA that holds item i.
LK_DEVICE int cta_first(const DecodeParams& p, int c) { return (int)((int64_t)c * p.W / p.G); }
LK_DEVICE int cta_of(const DecodeParams& p, int i) { return (int)(((int64_t)(i + 1) * p.G - 1) / p.W); }

// Barrier over the consumer warps only (the producer warp never joins).
LK_DEVICE void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory"); }
// The same barrier, returning whether any consumer thread passed `pred`.
LK_DEVICE bool consumer_sync_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "n"(kConsumerThreads)
      : "memory");
  return r != 0;
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

// A non-negative finite fp16 value as fp32, exactly, without a conversion
// instruction: its bits shifted into fp32 position read as the value times
// 2^-112 (normal or subnormal alike), so one multiply by 2^112 restores it.
LK_DEVICE float f16_nonneg_to_f32(uint32_t h) { return __uint_as_float(h << 13) * 0x1p112f; }

LK_DEVICE float load_scale(const uint8_t* base, int i, int kind) {
  return kind == 0 ? reinterpret_cast<const float*>(base)[i]
                   : f16_nonneg_to_f32(reinterpret_cast<const uint16_t*>(base)[i]);
}

// Exact int -> float for |a| < 2^22 on the integer and FMA pipes: a added to
// the bit pattern of 1.5 * 2^23 is that float plus a, so one subtraction
// leaves a.  (The conversion instruction shares the pipe with exp2.)
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
constexpr int kMagicBits = 0x4B400000;
LK_DEVICE float i2f_small(int a) { return __fsub_rn(__int_as_float(a + kMagicBits), kMagic); }

LK_DEVICE float ld_f(const uint8_t* base, int i, int is_bf16) {
  return is_bf16 ? lk_bf16_to_f32(reinterpret_cast<const uint16_t*>(base)[i])
                 : reinterpret_cast<const float*>(base)[i];
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

constexpr float kInv254cu = 1.0f / (254.0f * 254.0f * 254.0f);

// Four int8 terms t_i of x in [0, 127]: x = t0 + t1/254 + t2/254^2 + t3/254^3
// up to 127/254^4 (each remainder lies in [-1/2, 1/2], so |t_i| <= 127),
// packed little-endian into one word (byte i = t_i).
// Each rounding is x + 1.5 * 2^23 (round half to even, |x| < 2^22): the sum's
// low byte is already the two's-complement int8 of the rounded value, and
// subtracting the constant again gives it as a float.  No conversion
// instruction is needed (those share a pipe with exp2).
// (Explicitly rounded operations: a product contracted into the rounding
// add would round the exact product instead of the stored one.)
// WT = 3 stops after t2 (t3 = 0): x is then kept to 1/(2 * 254^2), a
// relative 6e-8 of the largest weight (the bf16-output path).
template <int WT>
LK_DEVICE uint32_t expand_weight(float x) {
  x = fminf(x, 127.0f);
  const float m0 = __fadd_rn(x, kMagic);
  x = __fmul_rn(__fsub_rn(x, __fsub_rn(m0, kMagic)), 254.0f);
  const float m1 = __fadd_rn(x, kMagic);
  x = __fmul_rn(__fsub_rn(x, __fsub_rn(m1, kMagic)), 254.0f);
  const float m2 = __fadd_rn(x, kMagic);
  uint32_t m3 = 0u;
  if constexpr (WT == 4) {
    x = __fmul_rn(__fsub_rn(x, __fsub_rn(m2, kMagic)), 254.0f);
    m3 = __float_as_uint(__fadd_rn(x, kMagic));
  }
  const uint32_t lo = __byte_perm(__float_as_uint(m0), __float_as_uint(m1), 0x0040u);
  const uint32_t hi = __byte_perm(__float_as_uint(m2), m3, 0x0040u);
  return __byte_perm(lo, hi, 0x5410u);
}

// Lane L holds the four terms of k position L (byte i = term i).  Returns the
// A fragments of an m16n8k32 int8 product whose row i (< 4) is term i over
// the 32 positions: a0 = row gid, positions 4 tig .. 4 tig + 3; a2 = the same
// row, positions 16 + 4 tig ..; rows 4..15 are zero.  A 4 x 4 byte transpose
// inside each quad of lanes (two exchanges) puts term c of positions
// 4q .. 4q + 3 in lane 4q + c; two shuffles fetch the fragments.
LK_DEVICE void weight_frags(uint32_t w, uint32_t sel1, uint32_t sel2, int gid, int tig, uint32_t& a0,
                            uint32_t& a2) {
  w = __byte_perm(w, __shfl_xor_sync(0xffffffffu, w, 1), sel1);
  w = __byte_perm(w, __shfl_xor_sync(0xffffffffu, w, 2), sel2);
  a0 = __shfl_sync(0xffffffffu, w, (4 * tig + gid) & 31);
  a2 = __shfl_sync(0xffffffffu, w, (16 + 4 * tig + gid) & 31);
  if (gid >= 4) a0 = a2 = 0u;
}

// D = A B + C for a 16 x 32 int8 A (rows gid + 8 zero: a1 = a3 = 0) and a
// 32 x 8 int8 B; exact int32.  Only the rows < 8 of C/D are carried.
LK_DEVICE void mma_s8_rows8(uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1, int& c0, int& c1) {
  int d2, d3;
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %11, %12, %13};"
      : "=r"(c0), "=r"(c1), "=r"(d2), "=r"(d3)
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "r"(c0), "r"(c1), "r"(0), "r"(0));
  (void)d2;
  (void)d3;
}

// B fragment word of the V product: the codes of latent dim d for the four
// k positions 4 tig .. 4 tig + 3 of one 16-token block (dimension-major
// block layout).  int4: positions 4 tig + m are tokens 8 (tig / 2) + 2 m +
// (tig % 2), i.e. the low (even tokens) or high (odd tokens) nibbles of one
// word, sign-extended to bytes.
template <int KIND>
LK_DEVICE uint32_t v_frag(const uint8_t* blk, int d, int tig) {
  if (KIND == 0) return *reinterpret_cast<const uint32_t*>(blk + d * 16 + tig * 4);
  const uint32_t w = *reinterpret_cast<const uint32_t*>(blk + d * 8 + (tig >> 1) * 4);
  const uint32_t x = (w >> ((tig & 1) * 4)) & 0x0F0F0F0Fu;
  return x | ((x & 0x08080808u) * 0x1Eu);
}

// Loads N consecutive 32-bit words from shared memory (16-byte aligned for
// N >= 4, 8-byte for N = 2).
template <int N>
LK_DEVICE void lds_words(const void* p, uint32_t (&w)[N]) {
  if constexpr (N == 1) {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  } else if constexpr (N == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x; w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const uint4 v = reinterpret_cast<const uint4*>(p)[i];
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  }
}

// Scores of two tokens (tl and tl + 32) in log2 units: sum over groups g of
//   sigma_g * a * (D0 + D1/254 + D2/254^2),  D_i = c . t_i  (exact dp4a sums)
// with the q~ terms t_i read from shared memory once for both tokens (the
// same words for every lane: broadcast loads).  int8 keys: one group and one
// scale per token.  The two tokens' chains are independent (instruction-level
// parallelism for the warp).
template <int KIND, int CS, int TG>
LK_DEVICE void token_score2(const uint8_t* kc, const uint8_t* ks, const HeadGeom& g, int tl, const int8_t* qterm,
                            float qa, float& sa, float& sb) {
  constexpr int WPC = CS / 4;  // words per chunk
  constexpr int MAXCH = (KIND == 0 ? kMaxR : kMaxR / 2) / CS;
  const int nch = g.rbk / CS;
  const int tb = tl + 32;
  if (KIND == 0) {
    int a0 = 0, a1 = 0, a2 = 0, b0 = 0, b1 = 0, b2 = 0;
#pragma unroll
    for (int c = 0; c < MAXCH; ++c) {
      if (c >= nch) break;  // (uniform; the chunks left hold no codes)
      {
        Chunk<CS> ca, cb;
        ca.load(kc, g.rbk, tl, c);
        if constexpr (TG == 2) cb.load(kc, g.rbk, tb, c);
        uint32_t t0[WPC], t1[WPC], t2[WPC];
        lds_words<WPC>(qterm + 0 * kMaxR + c * CS, t0);
        lds_words<WPC>(qterm + 1 * kMaxR + c * CS, t1);
        lds_words<WPC>(qterm + 2 * kMaxR + c * CS, t2);
#pragma unroll
        for (int wi = 0; wi < WPC; ++wi) {
          a0 = __dp4a((int)ca.w[wi], (int)t0[wi], a0);
          if constexpr (TG == 2) b0 = __dp4a((int)cb.w[wi], (int)t0[wi], b0);
          a1 = __dp4a((int)ca.w[wi], (int)t1[wi], a1);
          if constexpr (TG == 2) b1 = __dp4a((int)cb.w[wi], (int)t1[wi], b1);
          a2 = __dp4a((int)ca.w[wi], (int)t2[wi], a2);
          if constexpr (TG == 2) b2 = __dp4a((int)cb.w[wi], (int)t2[wi], b2);
        }
      }
    }
    // |a_i| <= 64 * 127 * 127 < 2^22
    const float xa = fmaf(i2f_small(a2), kInv254sq, fmaf(i2f_small(a1), kInv254, i2f_small(a0)));
    const float xb = fmaf(i2f_small(b2), kInv254sq, fmaf(i2f_small(b1), kInv254, i2f_small(b0)));
    sa = reinterpret_cast<const float*>(ks)[tl] * (qa * xa);
    if constexpr (TG == 2) sb = reinterpret_cast<const float*>(ks)[tb] * (qa * xb);
  } else {
    float s_a = 0.0f, s_b = 0.0f;
    int a0 = 0, a1 = 0, a2 = 0, b0 = 0, b1 = 0, b2 = 0;
    int cur_g = 0;
    const int wpg = g.gk >> 3;  // code words per scale group
    int wleft = wpg;            // words left in the current group
    // code word w holds dims 8w .. 8w+7 (q~ bytes 8w .. 8w+7: even dims, then
    // odd dims); groups are multiples of 8 dims
#pragma unroll
    for (int c = 0; c < MAXCH; ++c) {
      if (c >= nch) break;  // (uniform; the chunks left hold no codes)
      {
        Chunk<CS> ca, cb;
        ca.load(kc, g.rbk, tl, c);
        if constexpr (TG == 2) cb.load(kc, g.rbk, tb, c);
        uint32_t t0[2 * WPC], t1[2 * WPC], t2[2 * WPC];
        lds_words<2 * WPC>(qterm + 0 * kMaxR + c * 2 * CS, t0);
        lds_words<2 * WPC>(qterm + 1 * kMaxR + c * 2 * CS, t1);
        lds_words<2 * WPC>(qterm + 2 * kMaxR + c * 2 * CS, t2);
#pragma unroll
        for (int wi = 0; wi < WPC; ++wi) {
          if (wleft == 0) {  // flush the finished group (uniform branch)
            const float sg_a = load_scale(ks, tl * g.ngk + cur_g, 1);
            s_a = fmaf(sg_a, qa * fmaf(i2f_small(a2), kInv254sq, fmaf(i2f_small(a1), kInv254, i2f_small(a0))), s_a);
            if constexpr (TG == 2) {
              const float sg_b = load_scale(ks, tb * g.ngk + cur_g, 1);
              s_b = fmaf(sg_b, qa * fmaf(i2f_small(b2), kInv254sq, fmaf(i2f_small(b1), kInv254, i2f_small(b0))), s_b);
            }
            a0 = a1 = a2 = b0 = b1 = b2 = 0;
            ++cur_g;
            wleft = wpg;
          }
          --wleft;
          int eva, oda, evb = 0, odb = 0;
          nibbles_to_s8(ca.w[wi], eva, oda);
          if constexpr (TG == 2) nibbles_to_s8(cb.w[wi], evb, odb);
          a0 = __dp4a(oda, (int)t0[2 * wi + 1], __dp4a(eva, (int)t0[2 * wi], a0));
          if constexpr (TG == 2) b0 = __dp4a(odb, (int)t0[2 * wi + 1], __dp4a(evb, (int)t0[2 * wi], b0));
          a1 = __dp4a(oda, (int)t1[2 * wi + 1], __dp4a(eva, (int)t1[2 * wi], a1));
          if constexpr (TG == 2) b1 = __dp4a(odb, (int)t1[2 * wi + 1], __dp4a(evb, (int)t1[2 * wi], b1));
          a2 = __dp4a(oda, (int)t2[2 * wi + 1], __dp4a(eva, (int)t2[2 * wi], a2));
          if constexpr (TG == 2) b2 = __dp4a(odb, (int)t2[2 * wi + 1], __dp4a(evb, (int)t2[2 * wi], b2));
        }
      }
    }
    // per group |a_i| <= 64 * 7 * 127 < 2^22
    sa = fmaf(load_scale(ks, tl * g.ngk + cur_g, 1),
              qa * fmaf(i2f_small(a2), kInv254sq, fmaf(i2f_small(a1), kInv254, i2f_small(a0))), s_a);
    if constexpr (TG == 2)
      sb = fmaf(load_scale(ks, tb * g.ngk + cur_g, 1),
                qa * fmaf(i2f_small(b2), kInv254sq, fmaf(i2f_small(b1), kInv254, i2f_small(b0))), s_b);
  }
}

struct SmemLayout {
  int stage_bytes;
  int off_kc, off_vc, off_ks, off_vs;  // within a stage
  int off_q, off_bk;                   // factor slot: q^h and B_K^h of the current or next unit
  int off_bv;                          // B_V^h of the current unit
  int off_fr;                          // per consumer warp: V weight fragments [ngv][32 lanes] (several groups)
  int off_qt;                          // q~ [kMaxR] floats
  int off_qterm;                       // q~ expansion bytes [3][kMaxR]
  int off_wst;                         // per consumer warp: (m, l, u[kMaxR])
  int off_cta;                         // CTA state of the unit [2 + kMaxR]
  int off_bar;                         // full[kMaxStages], empty[kMaxStages], factor full, factor empty, B_V full
  int off_misc;                        // abort flag, ticket flag, q~ expansion scale
};

constexpr int kSmemFixed = kMaxR * 4 + 3 * kMaxR + kCW * (2 + kMaxR) * 4 + (2 + kMaxR) * 4 +
                           (2 * kMaxStages + 4) * 8 + 32;

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
  L.off_fr = L.off_bv + p.st_bv;
  L.off_qt = L.off_fr + p.st_fr;
  L.off_qterm = L.off_qt + kMaxR * 4;
  L.off_wst = L.off_qterm + 3 * kMaxR;
  L.off_cta = L.off_wst + kCW * (2 + kMaxR) * 4;
  L.off_bar = L.off_cta + (2 + kMaxR) * 4;
  L.off_misc = L.off_bar + (2 * kMaxStages + 4) * 8;
  return L;
}

inline int smem_bytes_for(const DecodeParams& p) {
  const int stage = p.st_kc + p.st_vc + p.st_ks + p.st_vs;
  return p.nstages * stage + p.st_q + p.st_bk + p.st_bv + p.st_fr + kSmemFixed;
}

struct Bars {
  uint64_t* full;
  uint64_t* empty;
  uint64_t* fbar;    // factor slot filled
  uint64_t* fempty;  // factor slot released by every consumer warp
  uint64_t* vbar;    // B_V slot filled
  volatile int* abort_flag;
  int* ticket_flag;
  float* qa;
  int* bv_issued;  // this unit's B_V copy was started (it must land before the CTA may end)
};

LK_DEVICE Bars bars_of(uint8_t* smem, const SmemLayout& L) {
  Bars B;
  B.full = reinterpret_cast<uint64_t*>(smem + L.off_bar);
  B.empty = B.full + kMaxStages;
  B.fbar = B.full + 2 * kMaxStages;
  B.fempty = B.fbar + 1;
  B.vbar = B.fbar + 2;
  B.abort_flag = reinterpret_cast<volatile int*>(smem + L.off_misc);
  B.ticket_flag = reinterpret_cast<int*>(smem + L.off_misc) + 1;
  B.qa = reinterpret_cast<float*>(smem + L.off_misc) + 2;
  B.bv_issued = reinterpret_cast<int*>(smem + L.off_misc) + 3;
  return B;
}

// ------------------------------------------------------------------ producer
// One thread: for every unit of the CTA's range, the factor copies (q^h,
// B_K^h) once the consumers released the slot, then each non-empty stage once
// its ring buffer is free.
template <int KIND>
LK_DEVICE void produce(const DecodeParams& p, uint8_t* smem, const SmemLayout& L, int i0, int i1) {
  const Bars B = bars_of(smem, L);
  const int NS = p.nstages;
  const int H = p.head_dim;
  const int ssz = KIND == 0 ? 4 : 2;
  int u = i0 / p.S, s = i0 - u * p.S;
  int it = i0, k = 0, nunit = 0, nf = 0;  // stages issued, units begun, factor copies issued
  bool ok = true;
  bool waited = !p.early_inputs;  // the previous kernel on the stream has completed
  while (it < i1) {
    const int s_end = min(p.S, s + (i1 - it));
    const int b = u / p.n_heads, h = u - b * p.n_heads;
    const HeadGeom g = unit_geometry<KIND>(p, b, h);
    if (ok && nunit > 0 && !lk_mbar_wait_bounded(B.fempty, (uint32_t)((nunit - 1) & 1), p.wait_ns)) {
      *B.abort_flag = 1;
      ok = false;
    }
    if (ok) {
      const uint32_t qb = H * p.q_size, bkb = g.rk * H * p.b_size;
      lk_mbar_arrive_expect_tx(B.fbar, qb + bkb);
      lk_bulk_g2s(smem + L.off_q, static_cast<const uint8_t*>(p.q) + (int64_t)(b * p.n_heads + h) * H * p.q_size, qb,
                  B.fbar);
      lk_bulk_g2s(smem + L.off_bk, static_cast<const uint8_t*>(p.BK) + g.bk_off * p.b_size, bkb, B.fbar);
      ++nf;
    }
    ++nunit;
    // until the wait, only stages below the stable prefix are read: they are
    // full (every row is at least stable_len long) and final
    int len = waited ? unit_len(p, b) : p.stable_len;
    int64_t end = min((int64_t)((len + 15) & ~15), (int64_t)p.capacity);
    for (int ss = s; ss < s_end && ok; ++ss) {
      const int64_t t0 = (int64_t)ss * p.ST;
      if (!waited && t0 + p.ST > p.stable_len) {  // the stage may hold what the append writes
        lk_grid_dep_wait();
        waited = true;
        len = unit_len(p, b);
        end = min((int64_t)((len + 15) & ~15), (int64_t)p.capacity);
      }
      if (t0 >= len) break;  // this and the unit's later stages hold no tokens
      if (*B.abort_flag || u * p.S + ss == p.stall_item) {  // (the test hook stops here, copies unissued)
        ok = false;
        break;
      }
      const int buf = k % NS;
      if (k >= NS && !lk_mbar_wait_bounded(&B.empty[buf], (uint32_t)(((k / NS) - 1) & 1), p.wait_ns)) {
        *B.abort_flag = 1;
        ok = false;
        break;
      }
      const int ntok = (int)min((int64_t)p.ST, end - t0);
      uint8_t* st = smem + buf * L.stage_bytes;
      const uint32_t bkc = ntok * g.rbk, bvc = ntok * g.rbv;
      const uint32_t bks = ntok * g.ngk * ssz, bvs = ntok * g.ngv * ssz;
      lk_mbar_arrive_expect_tx(&B.full[buf], bkc + bvc + bks + bvs);
      lk_bulk_g2s(st + L.off_kc, p.codes_k + g.kc_off + t0 * g.rbk, bkc, &B.full[buf]);
      lk_bulk_g2s(st + L.off_vc, p.codes_v + g.vc_off + t0 * g.rbv, bvc, &B.full[buf]);
      lk_bulk_g2s(st + L.off_ks, p.scales_k + (g.ks_off + t0 * g.ngk) * ssz, bks, &B.full[buf]);
      lk_bulk_g2s(st + L.off_vs, p.scales_v + (g.vs_off + t0 * g.ngv) * ssz, bvs, &B.full[buf]);
      ++k;
    }
    it += s_end - s;
    ++u;
    s = 0;
  }
  if (!waited) lk_grid_dep_wait();  // this grid never completes before the previous one
  // before the CTA may finish, every copy this CTA started has landed
  for (int j = max(0, k - NS); j < k; ++j)
    if (!lk_mbar_wait_bounded(&B.full[j % NS], (uint32_t)((j / NS) & 1), LK_WAIT_LIMIT_NS))
      lk_dev_fail(LK_DEV_TIMEOUT_DRAIN);
  if (nf > 0 && !lk_mbar_wait_bounded(B.fbar, (uint32_t)((nf - 1) & 1), LK_WAIT_LIMIT_NS))
    lk_dev_fail(LK_DEV_TIMEOUT_DRAIN);
}

// ------------------------------------------------------------------ consumers
// q~ of unit (b, h) from the staged q^h and B_K^h, then its three-term int8
// expansion (warp 0).  `n` counts the units this CTA has begun.
template <int KIND>
LK_DEVICE void absorb_q(const DecodeParams& p, uint8_t* smem, const SmemLayout& L, const HeadGeom& g, int n) {
  const Bars B = bars_of(smem, L);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int H = p.head_dim;
  float* qt_s = reinterpret_cast<float*>(smem + L.off_qt);
  int8_t* qterm = reinterpret_cast<int8_t*>(smem + L.off_qterm);
  if (threadIdx.x == 0) {
    // B_V^h is read when the unit ends; the previous unit's output is done
    // (the slot is free) and its copy was waited for
    *B.bv_issued = !*B.abort_flag;
    if (*B.bv_issued) {
      const uint32_t bvb = g.rv * H * p.b_size;
      lk_mbar_arrive_expect_tx(B.vbar, bvb);
      lk_bulk_g2s(smem + L.off_bv, static_cast<const uint8_t*>(p.BV) + g.bv_off * p.b_size, bvb, B.vbar);
    }
  }
  if (!*B.abort_flag && !lk_mbar_wait_bounded(B.fbar, (uint32_t)(n & 1), p.wait_ns)) *B.abort_flag = 1;
  if (!*B.abort_flag) {
    const uint8_t* qs = smem + L.off_q;
    const uint8_t* bks = smem + L.off_bk;
    for (int i = warp; i < g.rk; i += kCW) {
      float acc = 0.0f;
      for (int d = lane; d < H; d += 32) acc = fmaf(ld_f(qs, d, p.q_bf16), ld_f(bks, i * H + d, p.b_bf16), acc);
      acc = lk_warp_sum(acc);
      if (lane == 0) qt_s[i] = acc * p.qscale;
    }
  }
  __syncwarp();
  if (lane == 0) lk_mbar_arrive(B.fempty);  // this warp is done with the factor slot
  consumer_sync();
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
    if (lane == 0) *B.qa = a;
  }
  consumer_sync();
}

// The stages [s0, s1) of one unit (tokens below len), then this warp's state
// (m, l, u) in shared memory.  buf / phase: ring position and parity of the
// CTA's next stage, carried across units.  NM = ceil(r_V / 8) V products per
// stage, fixed at compile time (runtime bounds on these loops cost more
// instructions than the products themselves).
template <int KIND, int CSK, int NM, bool VG1, int TG, int WT>
LK_DEVICE void run_unit(const DecodeParams& p, uint8_t* smem, const SmemLayout& L, const HeadGeom& g, int b,
                        int len, int s0, int s1, int& buf, uint32_t& phase, bool& waited) {
  const Bars B = bars_of(smem, L);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int NS = p.nstages;
  const int8_t* qterm = reinterpret_cast<const int8_t*>(smem + L.off_qterm);
  float* wst = reinterpret_cast<float*>(smem + L.off_wst);
  const float qa = *B.qa;
  const int gid = lane >> 2, tig = lane & 3;
  // Score phase: lane L takes token tok(L) of the warp's 32 (int4: the even
  // tokens of each octet before the odd ones), so that lane order is the k
  // order of the V products.
  const int tok = KIND == 0 ? lane : (lane & 16) | (((lane >> 3) & 1) << 3) | ((lane & 3) << 1) | ((lane >> 2) & 1);
  // two independent groups of 32 tokens per warp and stage: tokens tl and tl + 32
  constexpr int ST = 32 * TG * kCW;
  const int tl = 32 * TG * warp + tok;  // this lane's first token within a stage
  const uint32_t sel1 = (lane & 1) ? 0x3715u : 0x6240u;
  const uint32_t sel2 = (lane & 2) ? 0x3276u : 0x5410u;
  const float fterm = gid == 0 ? 1.0f : gid == 1 ? kInv254 : gid == 2 ? kInv254sq : gid == 3 ? kInv254cu : 0.0f;
  uint2* fr = reinterpret_cast<uint2*>(smem + L.off_fr) + warp * (p.st_fr / (kCW * 8));
  int acc[NM][2];
#pragma unroll
  for (int j = 0; j < NM; ++j) acc[j][0] = acc[j][1] = 0;
  float u[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};  // lanes < 16: MMAs j = gid and gid + 4
  float m_run = -INFINITY, l_run = 0.0f;
  float wref = 0.0f;  // every weight of the open accumulation is <= wref
  float inv = 0.0f;   // 127 / wref
  auto fold = [&](float alpha) {
    const float sc = wref * (1.0f / 127.0f);
#pragma unroll
    for (int j = 0; j < NM; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float x = (float)acc[j][e] * fterm;
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        x += __shfl_xor_sync(0xffffffffu, x, 8);
        acc[j][e] = 0;
        if ((j & 3) == gid) u[j >> 2][e] = (u[j >> 2][e] + sc * x) * alpha;
      }
    }
  };

  int tl_end = len - s0 * ST - tl;  // token (s0 + j) * ST + tl is valid iff j * ST < tl_end
  // after an expired wait (error path) later units skip their stages; within
  // a unit the flag is consulted only when a wait expires
  const int nst = *B.abort_flag ? 0 : s1 - s0;
  for (int j = 0; j < nst; ++j) {
    if (!waited && (s0 + j + 1) * ST > p.stable_len) {  // past the stable prefix: the append's output
      lk_grid_dep_wait();
      waited = true;
      len = unit_len(p, b);
      tl_end = len - s0 * ST - tl;
    }
    if ((s0 + j) * ST >= len) break;  // no copies were issued for the unit's later stages
    if (!lk_mbar_wait_bounded(&B.full[buf], phase, p.wait_ns)) {
      *B.abort_flag = 1;
      break;
    }
    const uint8_t* st = smem + buf * L.stage_bytes;
    const uint8_t* vs = st + L.off_vs;
    const bool va = j * ST < tl_end, vb = TG == 2 && j * ST + 32 < tl_end;
    // a. scores of the token groups; a new running max (warp vote) folds the open sums
    float sa, sb = -INFINITY;
    token_score2<KIND, CSK, TG>(st + L.off_kc, st + L.off_ks, g, tl, qterm, qa, sa, sb);
    sa = va ? sa : -INFINITY;
    sb = vb ? sb : -INFINITY;
    const float smx = fmaxf(sa, sb);
    if (__any_sync(0xffffffffu, smx > m_run)) {
      const float m_new = fmaxf(m_run, lk_warp_max(smx));
      const float alpha = (m_run == -INFINITY) ? 0.0f : exp2f(m_run - m_new);
      fold(alpha);
      l_run *= alpha;
      m_run = m_new;
    }
    const float pa = va ? exp2f(sa - m_run) : 0.0f;
    const float pb = vb ? exp2f(sb - m_run) : 0.0f;
    l_run += pa + pb;
    // b. V scales: a larger one (warp vote) folds, then raises wref; the
    //    weights w = p sigma_V become four int8 terms of w * 127 / wref
    const uint8_t* vca = st + L.off_vc + 2 * TG * warp * 16 * g.rbv;  // the warp's 16-token blocks
    const uint8_t* vca1 = vca + 16 * g.rbv;
    const uint8_t* vcb = vca + 32 * g.rbv;
    const uint8_t* vcb1 = vca + 48 * g.rbv;
    if (VG1) {
      const float ga = va ? load_scale(vs, tl, KIND) : 0.0f;
      const float gb = TG == 2 && vb ? load_scale(vs, tl + 32, KIND) : 0.0f;
      if (__any_sync(0xffffffffu, fmaxf(ga, gb) > wref)) {  // then some scale > 0, so wref > 0 below
        fold(1.0f);
        wref = fmaxf(wref, lk_warp_max(fmaxf(ga, gb)));
        inv = 127.0f / wref;
      }
      uint32_t a0a, a2a, a0b = 0u, a2b = 0u;
      weight_frags(expand_weight<WT>(pa * ga * inv), sel1, sel2, gid, tig, a0a, a2a);
      if constexpr (TG == 2) weight_frags(expand_weight<WT>(pb * gb * inv), sel1, sel2, gid, tig, a0b, a2b);
      // c. acc[jm] += terms x codes of dims 8 jm .. 8 jm + 7, each group
      //    (dims >= r_V only in the last product, when r_V % 8 != 0)
#pragma unroll
      for (int jm = 0; jm < NM; ++jm) {
        const int d = 8 * jm + gid;
        const bool live = jm < NM - 1 || d < g.rv;
        const uint32_t b0 = live ? v_frag<KIND>(vca, d, tig) : 0u;
        const uint32_t b1 = live ? v_frag<KIND>(vca1, d, tig) : 0u;
        mma_s8_rows8(a0a, a2a, b0, b1, acc[jm][0], acc[jm][1]);
        if constexpr (TG == 2) {
          const uint32_t b2 = live ? v_frag<KIND>(vcb, d, tig) : 0u;
          const uint32_t b3 = live ? v_frag<KIND>(vcb1, d, tig) : 0u;
          mma_s8_rows8(a0b, a2b, b2, b3, acc[jm][0], acc[jm][1]);
        }
      }
    } else {
      float smax_t = 0.0f;
      for (int gi = 0; gi < g.ngv; ++gi) {
        smax_t = fmaxf(smax_t, va ? load_scale(vs, tl * g.ngv + gi, KIND) : 0.0f);
        if (TG == 2) smax_t = fmaxf(smax_t, vb ? load_scale(vs, (tl + 32) * g.ngv + gi, KIND) : 0.0f);
      }
      if (__any_sync(0xffffffffu, smax_t > wref)) {
        fold(1.0f);
        wref = fmaxf(wref, lk_warp_max(smax_t));
        inv = 127.0f / wref;
      }
      for (int gi = 0; gi < g.ngv; ++gi) {
        const float ga = va ? load_scale(vs, tl * g.ngv + gi, KIND) : 0.0f;
        uint32_t a0a, a2a;
        weight_frags(expand_weight<WT>(pa * ga * inv), sel1, sel2, gid, tig, a0a, a2a);
        fr[(gi * 2 + 0) * 32 + lane] = make_uint2(a0a, a2a);
        if constexpr (TG == 2) {
          const float gb = vb ? load_scale(vs, (tl + 32) * g.ngv + gi, KIND) : 0.0f;
          uint32_t a0b, a2b;
          weight_frags(expand_weight<WT>(pb * gb * inv), sel1, sel2, gid, tig, a0b, a2b);
          fr[(gi * 2 + 1) * 32 + lane] = make_uint2(a0b, a2b);
        }
      }
      __syncwarp();
#pragma unroll
      for (int jm = 0; jm < NM; ++jm) {
        const int gi = (8 * jm) / g.gv;
        const uint2 fa = fr[(gi * 2 + 0) * 32 + lane];
        const int d = 8 * jm + gid;
        const bool live = jm < NM - 1 || d < g.rv;
        const uint32_t b0 = live ? v_frag<KIND>(vca, d, tig) : 0u;
        const uint32_t b1 = live ? v_frag<KIND>(vca1, d, tig) : 0u;
        mma_s8_rows8(fa.x, fa.y, b0, b1, acc[jm][0], acc[jm][1]);
        if constexpr (TG == 2) {
          const uint2 fb = fr[(gi * 2 + 1) * 32 + lane];
          const uint32_t b2 = live ? v_frag<KIND>(vcb, d, tig) : 0u;
          const uint32_t b3 = live ? v_frag<KIND>(vcb1, d, tig) : 0u;
          mma_s8_rows8(fb.x, fb.y, b2, b3, acc[jm][0], acc[jm][1]);
        }
      }
    }
    __syncwarp();  // this warp is done with the stage buffer (and its fragment store)
    if (lane == 0) lk_mbar_arrive(&B.empty[buf]);
    if (++buf == NS) {
      buf = 0;
      phase ^= 1u;
    }
    if ((j & 255) == 255) fold(1.0f);  // int32 sums stay far from overflow
  }
  fold(1.0f);
  const float lw = lk_warp_sum(l_run);
  float* ws = wst + warp * (2 + kMaxR);
  if (lane == 0) {
    ws[0] = m_run;
    ws[1] = lw;
  }
  if (gid < 4) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int jm = gid + 4 * k;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int d = 8 * jm + 2 * tig + e;
        if (jm < NM && d < g.rv) ws[2 + d] = u[k][e];
      }
    }
  }
}

template <int KIND, int CSK, bool VG1, int TG, int WT>
LK_DEVICE void run_unit_nm(const DecodeParams& p, uint8_t* smem, const SmemLayout& L, const HeadGeom& g, int b,
                           int len, int s0, int s1, int& buf, uint32_t& phase, bool& waited) {
#define LK_RUN(NMV) run_unit<KIND, CSK, NMV, VG1, TG, WT>(p, smem, L, g, b, len, s0, s1, buf, phase, waited)
  switch ((g.rv + 7) >> 3) {
    case 1: LK_RUN(1); break;
    case 2: LK_RUN(2); break;
    case 3: LK_RUN(3); break;
    case 4: LK_RUN(4); break;
    case 5: LK_RUN(5); break;
    case 6: LK_RUN(6); break;
    case 7: LK_RUN(7); break;
    default: LK_RUN(8); break;
  }
#undef LK_RUN
}

// Block-wide max over the consumer threads (red: kCW floats of shared memory).
LK_DEVICE float consumer_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = lk_warp_max(v);
  if (lane == 0) red[warp] = v;
  consumer_sync();
  float m = red[0];
#pragma unroll
  for (int w = 1; w < kCW; ++w) m = fmaxf(m, red[w]);
  consumer_sync();  // red is free again
  return m;
}

// out^h = (u / l) B_V^h from the CTA state, B_V^h staged in shared memory.
LK_DEVICE void write_output(const DecodeParams& p, const uint8_t* bvs, const float* cta, const HeadGeom& g,
                            int64_t bh, bool aborted) {
  const int H = p.head_dim;
  const float lsum = cta[1];
  const float inv = (cta[0] == -INFINITY || lsum == 0.0f || aborted) ? 0.0f : 1.0f / lsum;
  for (int d = threadIdx.x; d < H; d += kConsumerThreads) {
    float o = 0.0f;
    for (int j = 0; j < g.rv; ++j) o = fmaf(cta[2 + j], ld_f(bvs, j * H + d, p.b_bf16), o);
    o *= inv;
    if (p.out_bf16) reinterpret_cast<uint16_t*>(p.out)[bh * H + d] = lk_f32_to_bf16(o);
    else reinterpret_cast<float*>(p.out)[bh * H + d] = o;
  }
}

// Merges the warps' states into the unit's CTA state; then writes the output
// (unit whole inside this CTA) or this piece's partial, and the last piece of
// the unit to arrive merges every piece and writes the output.
template <int KIND>
LK_DEVICE void finish_unit(const DecodeParams& p, uint8_t* smem, const SmemLayout& L, const HeadGeom& g, int b,
                           int h, int u, int seg_first, int seg_end, int i0, int c, int n) {
  const Bars B = bars_of(smem, L);
  const int tid = threadIdx.x;
  float* wst = reinterpret_cast<float*>(smem + L.off_wst);
  float* cta = reinterpret_cast<float*>(smem + L.off_cta);
  // this unit's B_V copy has landed long ago; waiting here also keeps the next
  // unit's copy from starting while this one is in flight, and a copy that
  // was started is waited for even after an error (it must land before the
  // CTA may end)
  if (*B.bv_issued) {
    const bool was_aborted = *B.abort_flag != 0;
    if (!lk_mbar_wait_bounded(B.vbar, (uint32_t)(n & 1), was_aborted ? LK_WAIT_LIMIT_NS : p.wait_ns)) {
      *B.abort_flag = 1;
      if (was_aborted) lk_dev_fail(LK_DEV_TIMEOUT_DRAIN);
    }
  }
  const bool aborted = consumer_sync_or(*B.abort_flag != 0);  // every warp's state is written
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kCW; ++w) M = fmaxf(M, wst[w * (2 + kMaxR)]);
  if (tid < 2 + g.rv) {
    float acc = M;
    if (tid > 0) {
      acc = 0.0f;
      if (M != -INFINITY && !aborted) {
#pragma unroll
        for (int w = 0; w < kCW; ++w) {
          const float mw = wst[w * (2 + kMaxR)];
          if (mw != -INFINITY) acc += wst[w * (2 + kMaxR) + tid] * exp2f(mw - M);
        }
      }
    } else if (aborted) {
      acc = -INFINITY;
    }
    cta[tid] = acc;
  }
  consumer_sync();  // cta[] is written; wst is free for the merge below
  const int64_t bh = (int64_t)b * p.n_heads + h;
  const int u0 = u * p.S, u1 = u0 + p.S;
  if (seg_first == u0 && seg_end == u1) {  // the whole unit ran here
    write_output(p, smem + L.off_bv, cta, g, bh, aborted);
    consumer_sync();  // cta[] and the B_V slot are free for the next unit
    return;
  }
  const int slot = seg_first == i0 ? 0 : 1;
  float* part = p.partials + ((int64_t)c * 2 + slot) * p.part_stride;
  if (tid < 2 + g.rv) part[tid] = cta[tid];
  __threadfence();
  consumer_sync();
  const int c0 = cta_of(p, u0), c1 = cta_of(p, u1 - 1);
  if (tid == 0) *B.ticket_flag = atomicAdd(&p.counters[u], 1) == c1 - c0;
  consumer_sync();
  const bool last = *B.ticket_flag != 0;
  consumer_sync();  // every thread read the flag before the next unit may set it
  if (!last) return;
  __threadfence();
  // last piece: merge every piece of the unit (partials visible in L2).  The
  // pieces are CTAs c0 .. c1; only c0 may hold the unit in its second slot.
  const int slot0 = cta_first(p, c0) >= u0 ? 0 : 1;
  auto piece = [&](int cc) {
    return p.partials + ((int64_t)cc * 2 + (cc == c0 ? slot0 : 0)) * p.part_stride;
  };
  float mloc = -INFINITY;
  for (int cc = c0 + tid; cc <= c1; cc += kConsumerThreads) mloc = fmaxf(mloc, __ldcg(piece(cc)));
  const float Mg = consumer_max(mloc, wst);
  // warp w sums pieces w, w + kCW, ... (lanes over the state), then the warps'
  // sums meet in shared memory
  {
    const int lane = tid & 31, warp = tid >> 5;
    float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f;
    if (Mg != -INFINITY) {
      for (int cc = c0 + warp; cc <= c1; cc += kCW) {
        const float* pc = piece(cc);
        const float mc = __ldcg(pc);
        const float v0 = lane < 2 + g.rv ? __ldcg(pc + lane) : 0.0f;
        const float v1 = lane + 32 < 2 + g.rv ? __ldcg(pc + lane + 32) : 0.0f;
        const float v2 = lane + 64 < 2 + g.rv ? __ldcg(pc + lane + 64) : 0.0f;
        const float w = mc == -INFINITY ? 0.0f : exp2f(mc - Mg);
        a0 = fmaf(w, v0, a0);
        a1 = fmaf(w, v1, a1);
        a2 = fmaf(w, v2, a2);
      }
    }
    float* ws = wst + warp * (2 + kMaxR);
    if (lane < 2 + g.rv) ws[lane] = a0;
    if (lane + 32 < 2 + g.rv) ws[lane + 32] = a1;
    if (lane + 64 < 2 + g.rv) ws[lane + 64] = a2;
  }
  consumer_sync();
  if (tid == 0) {
    cta[0] = Mg;
    p.counters[u] = 0;  // ready for the next call (and for a replay of this launch)
  } else if (tid < 2 + g.rv) {
    float acc = 0.0f;
#pragma unroll
    for (int w = 0; w < kCW; ++w) acc += wst[w * (2 + kMaxR) + tid];
    cta[tid] = acc;
  }
  consumer_sync();
  write_output(p, smem + L.off_bv, cta, g, bh, aborted);
  consumer_sync();
}

template <int KIND, int TG, int WT>
LK_DEVICE void consume(const DecodeParams& p, uint8_t* smem, const SmemLayout& L, int i0, int i1, int c) {
  int u = i0 / p.S, s = i0 - u * p.S;
  int it = i0, n = 0, buf = 0;
  uint32_t phase = 0u;
  bool waited = !p.early_inputs;  // this thread waited for the previous kernel on the stream
  while (it < i1) {
    const int s_end = min(p.S, s + (i1 - it));
    const int seg_end = it + (s_end - s);
    const int b = u / p.n_heads, h = u - b * p.n_heads;
    const HeadGeom g = unit_geometry<KIND>(p, b, h);
    absorb_q<KIND>(p, smem, L, g, n);
    // before the wait, the stable prefix is the length every row has
    const int len = waited ? unit_len(p, b) : p.stable_len;
    const int csk = lk_chunk_bytes(g.rbk);
    if (KIND == 0 || g.ngv == 1) {
      if (csk == 16) run_unit_nm<KIND, 16, true, TG, WT>(p, smem, L, g, b, len, s, s_end, buf, phase, waited);
      else if (csk == 8) run_unit_nm<KIND, 8, true, TG, WT>(p, smem, L, g, b, len, s, s_end, buf, phase, waited);
      else run_unit_nm<KIND, 4, true, TG, WT>(p, smem, L, g, b, len, s, s_end, buf, phase, waited);
    } else if constexpr (KIND == 1) {
      if (csk == 16) run_unit_nm<KIND, 16, false, TG, WT>(p, smem, L, g, b, len, s, s_end, buf, phase, waited);
      else if (csk == 8) run_unit_nm<KIND, 8, false, TG, WT>(p, smem, L, g, b, len, s, s_end, buf, phase, waited);
      else run_unit_nm<KIND, 4, false, TG, WT>(p, smem, L, g, b, len, s, s_end, buf, phase, waited);
    }
    finish_unit<KIND>(p, smem, L, g, b, h, u, it, seg_end, i0, c, n);
    it = seg_end;
    ++u;
    ++n;
    s = 0;
  }
  if (!waited) lk_grid_dep_wait();  // this grid never completes before the previous one
}

// WT: int8 terms of the value weights (4 for fp32 outputs, 3 for bf16 outputs)
template <int KIND, int TG, int WT>
__global__ void __launch_bounds__(kThreads, 2) decode_attn_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const SmemLayout L = smem_layout(p);
  const int c = blockIdx.x;
  const int i0 = cta_first(p, c), i1 = cta_first(p, c + 1);
  if (threadIdx.x == 0) {
    const Bars B = bars_of(smem, L);
    for (int i = 0; i < kMaxStages; ++i) {
      lk_mbar_init(&B.full[i], 1);
      lk_mbar_init(&B.empty[i], kCW);
    }
    lk_mbar_init(B.fbar, 1);
    lk_mbar_init(B.fempty, kCW);
    lk_mbar_init(B.vbar, 1);
    lk_fence_mbar_init();
    *B.abort_flag = 0;
  }
  __syncthreads();
  // launched with programmatic stream serialisation, this CTA may run while
  // the previous kernel on the stream (e.g. the latent append) finishes.
  // Nothing before this point reads global memory; with early_inputs the
  // first unit's q, B_K and B_V are fetched before the wait (in produce and
  // absorb_q), everything else after it.
  if (!p.early_inputs) lk_grid_dep_wait();
  if (i0 >= i1) return;
  if (threadIdx.x >= kConsumerThreads) {
    if (threadIdx.x == kConsumerThreads) produce<KIND>(p, smem, L, i0, i1);
    return;
  }
  consume<KIND, TG, WT>(p, smem, L, i0, i1, c);
  if (threadIdx.x == 0 && *bars_of(smem, L).abort_flag) lk_dev_fail(LK_DEV_TIMEOUT_PIPE);
}

}  // namespace

LK_DEFINE_STATUS_ACCESSOR(lk_decode_status_word)

namespace lk {

namespace {
int round_up(int x, int m) { return (x + m - 1) / m * m; }

using DecodeKernel = void (*)(DecodeParams);
DecodeKernel decode_kernel(int kind, int tg, int wt) {
  if (wt == 3) {
    if (kind == 0) return tg == 2 ? decode_attn_kernel<0, 2, 3> : decode_attn_kernel<0, 1, 3>;
    return tg == 2 ? decode_attn_kernel<1, 2, 3> : decode_attn_kernel<1, 1, 3>;
  }
  if (kind == 0) return tg == 2 ? decode_attn_kernel<0, 2, 4> : decode_attn_kernel<0, 1, 4>;
  return tg == 2 ? decode_attn_kernel<1, 2, 4> : decode_attn_kernel<1, 1, 4>;
}

// Resident CTAs per SM of the decode kernel for `smem` bytes of shared memory
// (cached per device, kernel and size; the query costs a few microseconds).
int decode_occupancy(int kind, int tg, int wt, int smem) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  const auto key = std::make_tuple(dev, kind * 16 + wt * 4 + tg, smem);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int occ = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_kernel(kind, tg, wt), kThreads, smem);
  if (e != cudaSuccess || occ < 1) occ = 1;
  cache[key] = occ;
  return occ;
}
int decode_stages(int max_len, int st = kStageMin) { return std::max(1, (max_len + st - 1) / st); }
// CTAs of the split (never more than items).  n_split > 0 asks for about
// n_split pieces per (b, h) unit.  Automatic (n_split = 0), `cap` = CTAs that
// fit on the GPU at once: with fewer units than that, each unit is cut into
// the same number k = cap / units of pieces, so that no CTA straddles two
// units (a straddling CTA pays a second q absorption and its pieces a merge);
// with more units, `cap` CTAs share all items evenly (stream-K).
int64_t decode_ctas(int units, int max_len, int n_split, int64_t cap, int st = kStageMin) {
  const int64_t W = (int64_t)units * decode_stages(max_len, st);
  if (n_split > 0) return std::min(W, (int64_t)units * n_split);
  if (units >= cap) return std::min(W, cap);
  return std::min(W, (int64_t)units * (cap / units));
}
}  // namespace

size_t decode_workspace_bytes(int units, int rv_max, int max_len, int n_split) {
  const size_t counters = (size_t)round_up(units * 4, 256);
  const size_t stride = (size_t)round_up(2 + rv_max, 4);
  // the automatic grid never exceeds min(items, kAutoCtaBound)
  const int64_t G = n_split > 0 ? decode_ctas(units, max_len, n_split, kAutoCtaBound)
                                 : std::min((int64_t)units * decode_stages(max_len), (int64_t)kAutoCtaBound);
  return counters + (size_t)G * 2 * stride * 4;
}

cudaError_t launch_decode_attn(const DecodeLaunch& a, cudaStream_t stream) {
  DecodeParams p{};
  p.wait_ns = a.wait_ns ? a.wait_ns : LK_WAIT_LIMIT_NS;
  p.stall_item = a.stall_item;
  p.codes_k = static_cast<const uint8_t*>(a.codes_k);
  p.codes_v = static_cast<const uint8_t*>(a.codes_v);
  p.scales_k = static_cast<const uint8_t*>(a.scales_k);
  p.scales_v = static_cast<const uint8_t*>(a.scales_v);
  p.q = a.q;
  p.BK = a.BK;
  p.BV = a.BV;
  p.seq_len = a.seq_len;
  p.out = a.out;
  p.n_heads = a.n_heads;
  p.head_dim = a.head_dim;
  p.capacity = a.capacity;
  p.q_bf16 = a.q_bf16;
  p.b_bf16 = a.b_bf16;
  p.out_bf16 = a.out_bf16;
  p.early_inputs = a.early_inputs;
  p.stable_len = a.early_inputs ? std::max(0, std::min(a.stable_len, a.max_len)) : 0;
  p.max_len = a.max_len;
  p.qscale = a.softmax_scale * 1.4426950408889634f;
  int rk_max = 0, rv_max = 0, ngk_max = 1, ngv_max = 1;
  int pk = 0, pv = 0, pgk = 0, pgv = 0, prk = 0, prv = 0;

  for (int h = 0; h < a.n_heads; ++h) {
    const int rk = a.ranks_k[h], rv = a.ranks_v[h];
    const int gk = a.kind == 0 ? rk : std::min(a.group_k, rk);
    const int gv = a.kind == 0 ? rv : std::min(a.group_v, rv);
    const int ngk = (rk + gk - 1) / gk, ngv = (rv + gv - 1) / gv;
    HeadInfo& hi = p.head[h];
    hi.rk = (uint8_t)rk;
    hi.rv = (uint8_t)rv;
    hi.ngk = (uint8_t)ngk;
    hi.ngv = (uint8_t)ngv;
    hi.gk = (uint8_t)gk;
    hi.gv = (uint8_t)gv;
    hi.pk = (uint16_t)pk;
    hi.pv = (uint16_t)pv;
    hi.pgk = (uint16_t)pgk;
    hi.pgv = (uint16_t)pgv;
    hi.prk = (uint16_t)prk;
    hi.prv = (uint16_t)prv;

    pk += a.kind == 0 ? rk : rk / 2;
    pv += a.kind == 0 ? rv : rv / 2;
    pgk += ngk;
    pgv += ngv;
    prk += rk;
    prv += rv;
    rk_max = std::max(rk_max, rk);
    rv_max = std::max(rv_max, rv);
    ngk_max = std::max(ngk_max, ngk);
    ngv_max = std::max(ngv_max, ngv);
  }
  p.tk = pk;
  p.tv = pv;
  p.tgk = pgk;
  p.tgv = pgv;
  const int rbk_max = a.kind == 0 ? rk_max : rk_max / 2;
  const int rbv_max = a.kind == 0 ? rv_max : rv_max / 2;
  const int ssz = a.kind == 0 ? 4 : 2;
  p.q_size = a.q_bf16 ? 2 : 4;
  p.b_size = a.b_bf16 ? 2 : 4;
  p.st_q = round_up(a.head_dim * p.q_size, 128);
  p.st_bk = round_up(rk_max * a.head_dim * p.b_size, 128);
  p.st_bv = round_up(rv_max * a.head_dim * p.b_size, 128);
  // two token groups per warp (448-token stages: more independent work per
  // warp) when two such stages of the widest head fit in ~110 KB beside the
  // fixed regions, so that two CTAs still share an SM; else one (224 tokens)
  int tg = 2;
  for (;; tg = 1) {
    p.ST = 32 * tg * kCW;
    p.st_kc = round_up(p.ST * rbk_max, 128);
    p.st_vc = round_up(p.ST * rbv_max, 128);
    p.st_ks = round_up(p.ST * ngk_max * ssz, 128);
    p.st_vs = round_up(p.ST * ngv_max * ssz, 128);
    p.st_fr = ngv_max > 1 ? kCW * ngv_max * 2 * 32 * 8 : 0;  // per-warp V fragments: scale group x token group
    p.nstages = 0;
    const int stage = p.st_kc + p.st_vc + p.st_ks + p.st_vs;
    const int room = 110 * 1024 - smem_bytes_for(p);  // smem_bytes_for counts 0 stages here
    if (tg == 1 || room >= 2 * stage) {
      // as many stages as fit (about 64 KB of copies in flight per SM keeps
      // HBM busy), between 2 and kMaxStages
      p.nstages = std::max(2, std::min(kMaxStages, room / std::max(stage, 1)));
      break;
    }
  }
  const int units = a.batch * a.n_heads;
  p.S = decode_stages(a.max_len, p.ST);
  const int64_t W = (int64_t)units * p.S;
  // a ring deeper than the stages a CTA streams only costs shared memory (and
  // keeps the kernel off SMs the previous kernel still occupies): size it for
  // the grid a full GPU would take
  {
    const int64_t g_full = decode_ctas(units, a.max_len, a.n_split, std::min(2 * a.num_sms, kAutoCtaBound), p.ST);
    const int64_t per_cta = (W + g_full - 1) / std::max<int64_t>(1, g_full) + 1;
    p.nstages = (int)std::max<int64_t>(2, std::min<int64_t>(p.nstages, per_cta));
  }
  const int smem = smem_bytes_for(p);
  // bf16 outputs (bound 1e-2 RMS) take three value-weight terms, fp32 four
  const int wt = a.out_bf16 ? 3 : 4;
  const DecodeKernel kernel = decode_kernel(a.kind, tg, wt);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int resident = decode_occupancy(a.kind, tg, wt, smem) * a.num_sms;
  int64_t cap = std::min(resident, kAutoCtaBound);
  // In a decode step this launch overlaps the projection kernel, whose CTAs
  // hold part of every SM's registers until it ends: only one attention CTA
  // per SM runs beside them, and a second wave would start only after the
  // projection.  With few units (at least 4 pieces each), one CTA per SM
  // then finishes first (measured, 32 heads: B = 1, 23.6 us per step against
  // 25.6 us for two per SM; at B = 2 two per SM stay faster, 25.7 against 26.6).
  if (a.early_inputs && a.n_split == 0 && (int64_t)units * 4 <= a.num_sms) cap = std::min(cap, (int64_t)a.num_sms);
  const int64_t G = decode_ctas(units, a.max_len, a.n_split, cap, p.ST);
  if (W > INT32_MAX || G < 1) return cudaErrorInvalidValue;
  p.W = (int)W;
  p.G = (int)G;
  p.part_stride = round_up(2 + rv_max, 4);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  p.counters = reinterpret_cast<int32_t*>(ws);
  p.partials = reinterpret_cast<float*>(ws + round_up(units * 4, 256));

  // programmatic stream serialisation: the launch and the barrier set-up
  // overlap the tail of the previous kernel (the kernel waits for it before
  // its first global read)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)G, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, p);
  if (e != cudaSuccess) return e;
  count_launch();
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
int g_noalloc_units[kNoallocMaxDevices] = {};  // B * n_heads of the device's last call (0: none)
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
  int rv_max = 0;
  for (int h = 0; h < v->n_heads; ++h) rv_max = std::max(rv_max, (int)v->ranks[h]);
  const int units = k->batch * k->n_heads;
  const size_t need = lk::decode_workspace_bytes(units, rv_max, max_seq_len, n_split);
  if (need > LK_DECODE_NOALLOC_SCRATCH_BYTES) {
    // rejected before any state changes: the next call sees the array as the
    // last accepted call left it
    snprintf(msg, sizeof(msg),
             "lk_latent_decode_attn_noalloc: needs %zu bytes of scratch, the static array holds %u; "
             "lower n_split or use lk_latent_decode_attn with a workspace",
             need, (unsigned)LK_DECODE_NOALLOC_SCRATCH_BYTES);
    return lk::set_error(LK_ERR_WORKSPACE, msg);
  }
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(cs, &capture);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "lk_latent_decode_attn_noalloc: cudaStreamIsCapturing: %s", cudaGetErrorString(e));
    return lk::set_error(LK_ERR_CUDA, msg);
  }
  // One lock over the whole call: the recorded shape must describe what the
  // stream will find in the array, so no other host thread may interleave.
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    // once per device, with that device current
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      snprintf(msg, sizeof(msg), "lk_latent_decode_attn_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
      return lk::set_error(LK_ERR_CUDA, msg);
    }
    g_noalloc_ptr[dev] = p;
  }
  void* scratch = g_noalloc_ptr[dev];
  // The partials of a call with another B * n_heads may cover this call's
  // arrival counters: clear them first (every completed call leaves its own
  // counters zero).  While the stream is being captured the clear is always
  // recorded, because a replay may follow direct calls of any shape.
  const bool clear = g_noalloc_units[dev] != units || capture != cudaStreamCaptureStatusNone;
  g_noalloc_units[dev] = 0;  // unknown until this call has been enqueued
  if (clear) {
    e = cudaMemsetAsync(scratch, 0, (size_t)(units * 4 + 255) / 256 * 256, cs);
    if (e != cudaSuccess) {
      snprintf(msg, sizeof(msg), "lk_latent_decode_attn_noalloc: clearing counters: %s", cudaGetErrorString(e));
      return lk::set_error(LK_ERR_CUDA, msg);
    }
  }
  const lk_status st = lk_latent_decode_attn(k, v, q, q_dtype, B_K, B_V, b_dtype, head_dim, seq_len, max_seq_len,
                                             softmax_scale, out, out_dtype, n_split, scratch,
                                             LK_DECODE_NOALLOC_SCRATCH_BYTES, stream);
  if (st != LK_OK) return st;  // the recorded shape stays 0: the next call clears
  g_noalloc_units[dev] = units;
  return LK_OK;
}
