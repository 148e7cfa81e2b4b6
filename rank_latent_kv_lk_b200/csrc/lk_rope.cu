// Latent decode attention with rotary positions (sm_100a).
//
// Neither page uses a positional encoding; this is the extension for models
// that rotate keys and queries.  Under a rotation that depends on the key's
// position, q can no longer be folded into B_K, so each key is rebuilt on
// chip from its latent code -- the form of the WSVD page's fused kernel,
// which rebuilds K_h on chip and runs the flash-decoding QK^T / softmax / PV
// over it (technical summary §2C).  For batch row b, head h, positions
// t < len = seq_len[b]:
//   K_t = sigma_K[t] (c_K[t] B_K^h)            (per scale group for int4)
//   s_t = <rot(K_t, t), rot(q, len - 1)> * softmax_scale
//   u = sum_t softmax(s)_t sigma_V[t] c_V[t];  out = u B_V^h   (V not rotated)
// rot turns the pairs (i, i + H/2) by t * base^(-2 i / H), with cos / sin
// from a table the library builds once (lk_rope_table): per 16-token block
// one table row, and for the positions inside the block the angle-sum
// identities with the table's rows 0..15.
//
// Work split: each (b, h) unit's positions are cut into pieces of a fixed
// number of 128-token tiles; a CTA of 8 warps takes one piece.  Per tile the
// K codes are expanded to bf16 rows in shared memory (exact); each warp
// rebuilds the keys of 16 tokens with m16n8k16 tensor-core products against
// B_K^h (bf16, staged once per CTA), for the column tiles of dims i and of
// dims i + H/2 together, so that a thread holds both members of its rotation
// pairs; it scales, rotates and dots them with the rotated query in
// registers, reduces each token's score over the four lanes that share it,
// updates its running max and sum, and adds p_t sigma_V[t] c_V[t] to its
// latent value sum (lane = latent dim).  At the end the warps' states merge
// in shared memory, each piece leaves a partial (m, l, u) and the last piece
// of the unit to arrive (atomic ticket, no waiting) merges them and writes
// out = (u / l) B_V^h.
#include <cmath>

#include "lk_common.cuh"
#include "lk_internal.h"

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTile = 16 * kWarps;  // tokens per tile
constexpr int kMaxR = LK_MAX_RANK;
constexpr int kMaxPieces = 4096;

struct RopeParams {
  const uint8_t* codes_k;
  const uint8_t* codes_v;
  const uint8_t* scales_k;
  const uint8_t* scales_v;
  const void* q;
  const uint16_t* BK;
  const uint16_t* BV;
  const float* table;  // [positions][H / 2][2] (cos, sin)
  const int32_t* seq_len;
  void* out;
  float* partials;     // [units][pieces][part_stride]
  int32_t* counters;   // [units], zero at entry, left zero
  int kind, n_heads, H, capacity, max_len, q_bf16, out_bf16;
  int piece_tiles, pieces, part_stride;
  int tk, tv, tgk, tgv;  // code bytes / scale groups of one batch row (all heads)
  float qscale;          // softmax_scale * log2(e)
  uint8_t rk[LK_MAX_HEADS], rv[LK_MAX_HEADS], gk[LK_MAX_HEADS], gv[LK_MAX_HEADS];
  uint16_t pk[LK_MAX_HEADS], pv[LK_MAX_HEADS], pgk[LK_MAX_HEADS], pgv[LK_MAX_HEADS];
  uint16_t prk[LK_MAX_HEADS], prv[LK_MAX_HEADS];
};

struct Smem {
  int off_kc, off_raw, raw_bytes, r_vc, r_ks, r_vs, r_ang, off_bk, off_q, off_wst, off_cta, off_to, total;
};

// Shared-memory plan (bytes): bf16 key codes [kTile][rk16 + 8] (converted
// per tile); two raw staging slots, each holding one tile's key codes, value
// codes, both scale planes and the table rows of its 16-token blocks (filled
// by cp.async one tile ahead); bf16 B_K [rk16][H + 8]; the rotated query;
// per-warp states; the table rows of positions 0..15.
Smem smem_plan(int rk16, int rbk_max, int rvb_max, int ngk, int ngv, int ssz, int H) {
  auto up = [](int x) { return (x + 15) & ~15; };
  Smem s;
  s.off_kc = 0;
  s.off_raw = up(kTile * (rk16 + 8) * 2);
  s.r_vc = up(kTile * rbk_max);
  s.r_ks = s.r_vc + up(kTile * rvb_max);
  s.r_vs = s.r_ks + up(kTile * ngk * ssz);
  s.r_ang = s.r_vs + up(kTile * ngv * ssz);
  s.raw_bytes = s.r_ang + up((kTile / 16) * (H / 2) * 8);
  s.off_bk = s.off_raw + 2 * s.raw_bytes;
  s.off_q = s.off_bk + up(rk16 * (H + 8) * 2);
  s.off_wst = s.off_q + up(H * 4);
  s.off_cta = s.off_wst + up(kWarps * (2 + kMaxR) * 4);
  s.off_to = s.off_cta + up((2 + kMaxR) * 4 + 16);
  s.total = s.off_to + up(16 * (H / 2) * 8);
  return s;
}

LK_DEVICE float ld_qv(const void* p, int64_t i, int bf16) {
  return bf16 ? lk_bf16_to_f32(static_cast<const uint16_t*>(p)[i]) : static_cast<const float*>(p)[i];
}

LK_DEVICE float scale_at(const uint8_t* base, int64_t i, int kind) {
  return kind == 0 ? reinterpret_cast<const float*>(base)[i]
                   : lk_f16_to_f32(reinterpret_cast<const uint16_t*>(base)[i]);
}

__global__ void __launch_bounds__(kThreads, 2) rope_decode_kernel(const __grid_constant__ RopeParams p,
                                                                   const __grid_constant__ Smem L) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int u = blockIdx.y, piece = blockIdx.x;
  const int b = u / p.n_heads, h = u - b * p.n_heads;
  const int H = p.H, half = H / 2;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int len = max(0, min(p.seq_len[b], p.max_len));
  const int t_begin = piece * p.piece_tiles * kTile;
  const int t_end = min(len, t_begin + p.piece_tiles * kTile);
  const int rk = p.rk[h], rv = p.rv[h];
  const int rk16 = (rk + 15) & ~15;
  const int rbk = p.kind == 0 ? rk : rk / 2, rbv = p.kind == 0 ? rv : rv / 2;
  const int gk = p.gk[h], gv = p.gv[h];
  const int ngk = (rk + gk - 1) / gk, ngv = (rv + gv - 1) / gv;
  const int cst = rk16 + 8, bst = H + 8;
  uint16_t* Kc = reinterpret_cast<uint16_t*>(sm + L.off_kc);
  uint16_t* Bs = reinterpret_cast<uint16_t*>(sm + L.off_bk);
  float* qr = reinterpret_cast<float*>(sm + L.off_q);
  float* wst = reinterpret_cast<float*>(sm + L.off_wst);
  float* cta = reinterpret_cast<float*>(sm + L.off_cta);
  int* ticket = reinterpret_cast<int*>(cta + 2 + kMaxR);
  float2* ang_off = reinterpret_cast<float2*>(sm + L.off_to);  // [j < 16][half]: (cos, sin) of position j

  float m_run = -INFINITY, l_run = 0.0f;
  float u0 = 0.0f, u1 = 0.0f;  // latent value sums of dims lane and lane + 32
  if (t_begin < t_end) {
    // rotated query at position len - 1, scaled into log2 units
    for (int i = threadIdx.x; i < half; i += kThreads) {
      const float2 cs = reinterpret_cast<const float2*>(p.table)[(int64_t)(len - 1) * half + i];
      const int64_t qo = (int64_t)u * H;
      const float x1 = ld_qv(p.q, qo + i, p.q_bf16), x2 = ld_qv(p.q, qo + i + half, p.q_bf16);
      qr[i] = (x1 * cs.x - x2 * cs.y) * p.qscale;
      qr[i + half] = (x2 * cs.x + x1 * cs.y) * p.qscale;
    }
    // B_K^h as bf16 rows, zero rows up to rk16
    const uint16_t* Bg = p.BK + (int64_t)p.prk[h] * H;
    for (int i = threadIdx.x; i < rk16 * (H / 8); i += kThreads) {
      const int d = i / (H / 8), c8 = i - d * (H / 8);
      const uint4 v = d < rk ? *reinterpret_cast<const uint4*>(Bg + (int64_t)d * H + 8 * c8) : make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(Bs + d * bst + 8 * c8) = v;
    }
    for (int i = threadIdx.x; i < 16 * half; i += kThreads) ang_off[i] = reinterpret_cast<const float2*>(p.table)[i];
    // key code dims rk .. rk16 stay zero for every tile
    for (int i = threadIdx.x; i < kTile * (rk16 - rk); i += kThreads) {
      const int t = i / (rk16 - rk);
      Kc[t * cst + rk + (i - t * (rk16 - rk))] = 0;
    }
  }
  const uint8_t* kplane = p.codes_k + ((int64_t)b * p.tk + p.pk[h]) * p.capacity;
  const uint8_t* vplane = p.codes_v + ((int64_t)b * p.tv + p.pv[h]) * p.capacity;
  const int64_t ks_base = p.kind == 0 ? (int64_t)u * p.capacity : ((int64_t)b * p.tgk + p.pgk[h]) * p.capacity;
  const int64_t vs_base = p.kind == 0 ? (int64_t)u * p.capacity : ((int64_t)b * p.tgv + p.pgv[h]) * p.capacity;
  const int csk = lk_chunk_bytes(rbk);
  const int nks = rk16 / 16;

  const int ssz = p.kind == 0 ? 4 : 2;
  const int ntiles = t_begin < t_end ? (t_end - t_begin + kTile - 1) / kTile : 0;
  // raw copies of tile ti into staging slot `slot` (16-byte cp.async chunks;
  // every region is a whole number of chunks: tiles are whole 16-token blocks)
  auto issue = [&](int ti, int slot) {
    const int t0 = t_begin + ti * kTile;
    const int n16 = (min(kTile, t_end - t0) + 15) & ~15;
    uint8_t* r = sm + L.off_raw + slot * L.raw_bytes;
    const uint8_t* srcs[4] = {kplane + (int64_t)t0 * rbk, vplane + (int64_t)t0 * rbv,
                              p.scales_k + (ks_base + (int64_t)t0 * ngk) * ssz,
                              p.scales_v + (vs_base + (int64_t)t0 * ngv) * ssz};
    const int offs[4] = {0, L.r_vc, L.r_ks, L.r_vs};
    const int bytes[4] = {n16 * rbk, n16 * rbv, n16 * ngk * ssz, n16 * ngv * ssz};
#pragma unroll
    for (int q = 0; q < 4; ++q)
      for (int i = threadIdx.x; i < bytes[q] / 16; i += kThreads) lk_cp_async16(r + offs[q] + 16 * i, srcs[q] + 16 * i);
    const int rowc = half / 2;  // 16-byte chunks of one table row
    for (int i = threadIdx.x; i < (n16 / 16) * rowc; i += kThreads) {
      const int blk = i / rowc, c = i - blk * rowc;
      lk_cp_async16(r + L.r_ang + (blk * rowc + c) * 16,
                    reinterpret_cast<const uint8_t*>(p.table) + ((int64_t)(t0 + 16 * blk) * half * 2) * 4 + 16 * c);
    }
  };
  if (ntiles > 0) issue(0, 0);
  lk_cp_async_commit();

  for (int ti = 0; ti < ntiles; ++ti) {
    const int t0 = t_begin + ti * kTile;
    const int ntok = min(kTile, t_end - t0);
    const int ntok16 = (ntok + 15) & ~15;  // whole 16-token blocks (inside the capacity)
    if (ti + 1 < ntiles) issue(ti + 1, (ti + 1) & 1);  // the next tile streams in while this one is computed
    lk_cp_async_commit();
    lk_cp_async_wait<1>();  // this tile's copies (issued by this thread) have landed
    __syncthreads();        // ... and every thread's
    const uint8_t* raw = sm + L.off_raw + (ti & 1) * L.raw_bytes;
    const uint8_t* Vc = raw + L.r_vc;
    const uint8_t* Ks = raw + L.r_ks;
    const uint8_t* Vs = raw + L.r_vs;
    const float2* ang_blk = reinterpret_cast<const float2*>(raw + L.r_ang);  // [block][half]: its first position
    // key codes -> bf16 rows (token-major chunks: each word is 4 bytes of one token)
    {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(raw);
      for (int i = threadIdx.x; i < ntok16 * rbk / 4; i += kThreads) {
        const uint32_t w = src[i];
        const int o = 4 * i;
        const int blk = o / (16 * rbk), rem = o - blk * 16 * rbk;
        const int ch = rem / (16 * csk), rem2 = rem - ch * 16 * csk;
        const int t = blk * 16 + rem2 / csk, byte0 = ch * csk + rem2 % csk;
        uint16_t* row = Kc + t * cst;
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
      }
    }
    __syncthreads();

    const int tb = 16 * warp;  // this warp's tokens within the tile
    if (tb < ntok16) {
      // ---- keys: rebuild, rotate, dot with the rotated query
      uint32_t af[4][4];
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        if (ks < nks) {
          const int row = tb + (lane & 7) + ((lane >> 3) & 1) * 8;
          lk_ldmatrix_x4(af[ks], Kc + row * cst + 16 * ks + (lane >> 4) * 8);
        } else {
          af[ks][0] = af[ks][1] = af[ks][2] = af[ks][3] = 0u;
        }
      }
      const int tl_lo = tb + gid, tl_hi = tl_lo + 8;            // tile rows of this thread's two tokens
      const int64_t pos_lo = t0 + tl_lo, pos_hi = t0 + tl_hi;
      float s_lo = 0.0f, s_hi = 0.0f;
      for (int n0 = 0; n0 < half; n0 += 16) {
        // [half: dims n0.. or n0 + H/2..][column octet][fragment]
        float acc[2][2][4], kv[2][2][4];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[a][n][e] = kv[a][n][e] = 0.0f;
        int cur = 0;
        auto fold = [&](int gi) {
          const float sl = scale_at(Ks, tl_lo * ngk + gi, p.kind), sh = scale_at(Ks, tl_hi * ngk + gi, p.kind);
#pragma unroll
          for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int n = 0; n < 2; ++n) {
              kv[a][n][0] = fmaf(sl, acc[a][n][0], kv[a][n][0]);
              kv[a][n][1] = fmaf(sl, acc[a][n][1], kv[a][n][1]);
              kv[a][n][2] = fmaf(sh, acc[a][n][2], kv[a][n][2]);
              kv[a][n][3] = fmaf(sh, acc[a][n][3], kv[a][n][3]);
              acc[a][n][0] = acc[a][n][1] = acc[a][n][2] = acc[a][n][3] = 0.0f;
            }
        };
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          if (ks < nks) {
            uint32_t bfr[2][4];
            const int krow = 16 * ks + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int a = 0; a < 2; ++a)
              lk_ldmatrix_x4_trans(bfr[a], Bs + krow * bst + n0 + a * half + (lane >> 4) * 8);
            if (ngk == 1) {
#pragma unroll
              for (int a = 0; a < 2; ++a) {
                lk_mma_bf16_16816(acc[a][0], af[ks][0], af[ks][1], af[ks][2], af[ks][3], bfr[a][0], bfr[a][1]);
                lk_mma_bf16_16816(acc[a][1], af[ks][0], af[ks][1], af[ks][2], af[ks][3], bfr[a][2], bfr[a][3]);
              }
            } else {
#pragma unroll
              for (int hf = 0; hf < 2; ++hf) {
                const int d0 = 16 * ks + 8 * hf;
                if (d0 < rk) {
                  const int gi = d0 / gk;
                  if (gi != cur) {
                    fold(cur);
                    cur = gi;
                  }
#pragma unroll
                  for (int a = 0; a < 2; ++a) {
                    lk_mma_bf16_1688(acc[a][0], af[ks][2 * hf], af[ks][2 * hf + 1], bfr[a][hf]);
                    lk_mma_bf16_1688(acc[a][1], af[ks][2 * hf], af[ks][2 * hf + 1], bfr[a][2 + hf]);
                  }
                }
              }
            }
          }
        }
        fold(cur);
        // rotate and dot: dims d (first half) and d + H/2, d = n0 + 8 n + 2 tig + e
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          const int d = n0 + 8 * n + 2 * tig;
          const float q1a = qr[d], q1b = qr[d + 1], q2a = qr[d + half], q2b = qr[d + half + 1];
#pragma unroll
          for (int row = 0; row < 2; ++row) {
            const int tl = row == 0 ? tl_lo : tl_hi;
            // angle of position t0 + tl: its block's first position plus tl % 16
            const float4 cb = *reinterpret_cast<const float4*>(ang_blk + (tl >> 4) * half + d);
            const float4 co = *reinterpret_cast<const float4*>(ang_off + (tl & 15) * half + d);
            float4 cs;
            cs.x = cb.x * co.x - cb.y * co.y;
            cs.y = cb.y * co.x + cb.x * co.y;
            cs.z = cb.z * co.z - cb.w * co.w;
            cs.w = cb.w * co.z + cb.z * co.w;
            const float k1a = kv[0][n][2 * row], k1b = kv[0][n][2 * row + 1];
            const float k2a = kv[1][n][2 * row], k2b = kv[1][n][2 * row + 1];
            float s = fmaf(q1a, k1a * cs.x - k2a * cs.y, q2a * (k2a * cs.x + k1a * cs.y));
            s = fmaf(q1b, k1b * cs.z - k2b * cs.w, s + q2b * (k2b * cs.z + k1b * cs.w));
            if (row == 0) s_lo += s;
            else s_hi += s;
          }
        }
      }
      s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 1);
      s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 2);
      s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 1);
      s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 2);
      if (pos_lo >= t_end) s_lo = -INFINITY;
      if (pos_hi >= t_end) s_hi = -INFINITY;
      // ---- running softmax over the warp's 16 tokens
      const float m_tile = lk_warp_max(fmaxf(s_lo, s_hi));
      if (m_tile != -INFINITY) {
        const float m_new = fmaxf(m_run, m_tile);
        const float alpha = m_run == -INFINITY ? 0.0f : exp2f(m_run - m_new);
        const float p_lo = pos_lo < t_end ? exp2f(s_lo - m_new) : 0.0f;
        const float p_hi = pos_hi < t_end ? exp2f(s_hi - m_new) : 0.0f;
        l_run = l_run * alpha + lk_warp_sum(tig == 0 ? p_lo + p_hi : 0.0f);
        m_run = m_new;
        u0 *= alpha;
        u1 *= alpha;
        // ---- values: u_d += sum_j p_j sigma_V[j] c_V[j][d]; token j's weight sits in lane 4 (j % 8)
        const uint8_t* vblk = Vc + (tb / 16) * 16 * rbv;
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          const int d = lane + 32 * q2;
          float acc = 0.0f;
          int codes[16];
          if (d < rv) {
            if (p.kind == 0) {
              const uint4 w = *reinterpret_cast<const uint4*>(vblk + d * 16);
              const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int j = 0; j < 16; ++j) codes[j] = (int)(int8_t)(ww[j >> 2] >> (8 * (j & 3)));
            } else {
              const uint2 w = *reinterpret_cast<const uint2*>(vblk + d * 8);
              const uint32_t ww[2] = {w.x, w.y};
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int nib = (int)((ww[j >> 3] >> (4 * (j & 7))) & 0xF);
                codes[j] = nib >= 8 ? nib - 16 : nib;
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) codes[j] = 0;
          }
          const int gi = d < rv ? d / gv : 0;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float pj = __shfl_sync(0xffffffffu, j < 8 ? p_lo : p_hi, 4 * (j & 7));
            // (positions past the row's length carry p = 0 and whatever the cache holds)
            const float wj = pj == 0.0f ? 0.0f : pj * scale_at(Vs, (tb + j) * ngv + gi, p.kind);
            acc = fmaf(wj, (float)codes[j], acc);
          }
          if (q2 == 0) u0 += acc;
          else u1 += acc;
        }
      }
    }
    __syncthreads();  // the slot and the key rows are free for the tile after next / the next conversion
  }
  // ---- merge the warps, then the pieces of the unit
  __syncthreads();
  float* ws = wst + warp * (2 + kMaxR);
  if (lane == 0) {
    ws[0] = m_run;
    ws[1] = l_run;
  }
  if (lane < rv) ws[2 + lane] = u0;
  if (lane + 32 < rv) ws[2 + lane + 32] = u1;
  __syncthreads();
  if (threadIdx.x < 2 + rv) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wst[w * (2 + kMaxR)]);
    float acc = threadIdx.x == 0 ? M : 0.0f;
    if (threadIdx.x > 0 && M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float mw = wst[w * (2 + kMaxR)];
        if (mw != -INFINITY) acc = fmaf(wst[w * (2 + kMaxR) + threadIdx.x], exp2f(mw - M), acc);
      }
    }
    cta[threadIdx.x] = acc;
  }
  __syncthreads();
  float* part = p.partials + ((int64_t)u * p.pieces + piece) * p.part_stride;
  if (threadIdx.x < 2 + rv) part[threadIdx.x] = cta[threadIdx.x];
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) *ticket = atomicAdd(&p.counters[u], 1) == p.pieces - 1;
  __syncthreads();
  if (!*ticket) return;
  __threadfence();
  const float* pu = p.partials + (int64_t)u * p.pieces * p.part_stride;
  float Mg = -INFINITY;
  for (int c = 0; c < p.pieces; ++c) Mg = fmaxf(Mg, __ldcg(pu + (int64_t)c * p.part_stride));
  __syncthreads();
  if (threadIdx.x < 2 + rv) {
    float acc = threadIdx.x == 0 ? Mg : 0.0f;
    if (threadIdx.x > 0 && Mg != -INFINITY) {
      for (int c = 0; c < p.pieces; ++c) {
        const float mc = __ldcg(pu + (int64_t)c * p.part_stride);
        if (mc != -INFINITY) acc = fmaf(__ldcg(pu + (int64_t)c * p.part_stride + threadIdx.x), exp2f(mc - Mg), acc);
      }
    }
    cta[threadIdx.x] = acc;
  }
  if (threadIdx.x == 0) p.counters[u] = 0;  // ready for the next call
  __syncthreads();
  const float inv = (cta[0] == -INFINITY || cta[1] == 0.0f) ? 0.0f : 1.0f / cta[1];
  const uint16_t* Bv = p.BV + (int64_t)p.prv[h] * H;
  for (int d = threadIdx.x; d < H; d += kThreads) {
    float o = 0.0f;
    for (int j = 0; j < rv; ++j) o = fmaf(cta[2 + j], lk_bf16_to_f32(Bv[(int64_t)j * H + d]), o);
    o *= inv;
    if (p.out_bf16) static_cast<uint16_t*>(p.out)[(int64_t)u * H + d] = lk_f32_to_bf16(o);
    else static_cast<float*>(p.out)[(int64_t)u * H + d] = o;
  }
}

// cos / sin of t * base^(-2 i / H) in float64, stored float32.
__global__ void rope_table_kernel(float* table, int H, int max_pos, double base) {
  const int half = H / 2;
  const int64_t n = (int64_t)max_pos * half;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = idx / half;
    const int i = (int)(idx - t * half);
    const double a = (double)t * pow(base, -2.0 * i / H);
    table[2 * idx] = (float)cos(a);
    table[2 * idx + 1] = (float)sin(a);
  }
}

int pieces_for(int units, int max_len, int num_sms, int* piece_tiles) {
  const int tiles = std::max(1, (max_len + kTile - 1) / kTile);
  // about two CTAs per SM in total, whole tiles per piece
  const int64_t want = std::max<int64_t>(1, (int64_t)2 * num_sms / std::max(1, units));
  int pt = (int)std::max<int64_t>(1, (tiles + want - 1) / want);
  int np = (tiles + pt - 1) / pt;
  if (np > kMaxPieces) {
    pt = (tiles + kMaxPieces - 1) / kMaxPieces;
    np = (tiles + pt - 1) / pt;
  }
  if (piece_tiles) *piece_tiles = pt;
  return np;
}

}  // namespace

namespace lk {

size_t rope_workspace_bytes(int units, int rv_max, int max_len, int num_sms) {
  const int np = pieces_for(units, max_len, num_sms, nullptr);
  const size_t counters = ((size_t)units * 4 + 255) / 256 * 256;
  const size_t stride = (size_t)((2 + rv_max + 3) / 4 * 4);
  return counters + (size_t)units * np * stride * 4;
}

cudaError_t launch_rope_table(float* table, int head_dim, int max_pos, double base, cudaStream_t stream) {
  if (max_pos == 0) return cudaSuccess;
  const int64_t n = (int64_t)max_pos * (head_dim / 2);
  const int grid = (int)std::min<int64_t>((n + 255) / 256, 4096);
  rope_table_kernel<<<grid, 256, 0, stream>>>(table, head_dim, max_pos, base);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_rope_decode(const RopeLaunch& a, cudaStream_t stream) {
  RopeParams p{};
  p.codes_k = static_cast<const uint8_t*>(a.codes_k);
  p.codes_v = static_cast<const uint8_t*>(a.codes_v);
  p.scales_k = static_cast<const uint8_t*>(a.scales_k);
  p.scales_v = static_cast<const uint8_t*>(a.scales_v);
  p.q = a.q;
  p.BK = static_cast<const uint16_t*>(a.BK);
  p.BV = static_cast<const uint16_t*>(a.BV);
  p.table = a.table;
  p.seq_len = a.seq_len;
  p.out = a.out;
  p.kind = a.kind;
  p.n_heads = a.n_heads;
  p.H = a.head_dim;
  p.capacity = a.capacity;
  p.max_len = a.max_len;
  p.q_bf16 = a.q_bf16;
  p.out_bf16 = a.out_bf16;
  p.qscale = a.softmax_scale * 1.4426950408889634f;
  int pk = 0, pv = 0, pgk = 0, pgv = 0, prk = 0, prv = 0;
  int rk_max = 0, rvb_max = 0, rv_max = 0, ngk_max = 1, ngv_max = 1;
  for (int h = 0; h < a.n_heads; ++h) {
    const int rk = a.ranks_k[h], rv = a.ranks_v[h];
    const int gk = a.kind == 0 ? rk : std::min(a.group_k, rk);
    const int gv = a.kind == 0 ? rv : std::min(a.group_v, rv);
    p.rk[h] = (uint8_t)rk;
    p.rv[h] = (uint8_t)rv;
    p.gk[h] = (uint8_t)gk;
    p.gv[h] = (uint8_t)gv;
    p.pk[h] = (uint16_t)pk;
    p.pv[h] = (uint16_t)pv;
    p.pgk[h] = (uint16_t)pgk;
    p.pgv[h] = (uint16_t)pgv;
    p.prk[h] = (uint16_t)prk;
    p.prv[h] = (uint16_t)prv;
    pk += a.kind == 0 ? rk : rk / 2;
    pv += a.kind == 0 ? rv : rv / 2;
    pgk += (rk + gk - 1) / gk;
    pgv += (rv + gv - 1) / gv;
    prk += rk;
    prv += rv;
    rk_max = std::max(rk_max, rk);
    rv_max = std::max(rv_max, rv);
    rvb_max = std::max(rvb_max, a.kind == 0 ? rv : rv / 2);
    ngk_max = std::max(ngk_max, (rk + gk - 1) / gk);
    ngv_max = std::max(ngv_max, (rv + gv - 1) / gv);
  }
  p.tk = pk;
  p.tv = pv;
  p.tgk = pgk;
  p.tgv = pgv;
  const int units = a.batch * a.n_heads;
  p.pieces = pieces_for(units, a.max_len, a.num_sms, &p.piece_tiles);
  p.part_stride = (2 + rv_max + 3) / 4 * 4;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  p.counters = reinterpret_cast<int32_t*>(ws);
  p.partials = reinterpret_cast<float*>(ws + ((size_t)units * 4 + 255) / 256 * 256);
  const int rbk_max = a.kind == 0 ? rk_max : rk_max / 2;
  const Smem s = smem_plan((rk_max + 15) & ~15, rbk_max, rvb_max, ngk_max, ngv_max, a.kind == 0 ? 4 : 2,
                           a.head_dim);
  cudaError_t e = cudaFuncSetAttribute(rope_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, s.total);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)p.pieces, (unsigned)units);
  rope_decode_kernel<<<grid, kThreads, s.total, stream>>>(p, s);
  count_launch();
  return cudaGetLastError();
}

}  // namespace lk
