// Latent projection + quantisation + append (WSVD page §2A: every head stores
// only its latent x A^h; §2C: stored in 8 or 4 bits; LASER page §4: the
// projection, latent generation and quantisation are fused).
//
// Two phases per call:
//   1. v = x A^T for all heads at once (A is [N_tot, E], K heads then V
//      heads), partial sums to the workspace.
//   2. One warp per (token, head): sum the partials in a fixed order, apply
//      the int8 dequantisation scales when the inputs are int8, quantise the
//      r_h values (absmax, RNE) and write codes + scale at position
//      seq_len[b] + t in the token-tiled cache layout.
// Decode (at most kGemvMaxRows = 8 token rows) runs both phases in ONE
// launch: a cluster of CTAs per head splits E, and the cluster's rank 0 sums
// the partials over distributed shared memory and appends; the last head to
// finish advances seq_len.  More rows (prefill, or a decode batch above 8)
// run the tensor-core GEMM, then the quantise-and-append launch.
#include "lk_common.cuh"
#include "lk_internal.h"
#include "lk_quant.cuh"

#include <cooperative_groups.h>
namespace cg = cooperative_groups;

namespace lk {
cudaError_t launch_gemm_f(const void* A, int lda, const void* B, int ldb, float* C, int ldc, int M,
                          int N, int K, bool bf16, cudaStream_t stream);
}

namespace {

constexpr int kGemvThreads = 256;
constexpr int kGemvMaxRows = 8;  // more rows: the tensor-core GEMM, then the quantise-and-append pass

template <int XT> struct XTraits;
template <> struct XTraits<lk::X_F32> { using T = float; static constexpr int VE = 4; };
template <> struct XTraits<lk::X_BF16> { using T = uint16_t; static constexpr int VE = 8; };
template <> struct XTraits<lk::X_I8> { using T = int8_t; static constexpr int VE = 16; };

// Expands a 16-byte chunk into fp32 values.
template <int XT>
LK_DEVICE void expand16(const uint4& v, float* f) {
  if (XT == lk::X_F32) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  } else {
    f[0] = lk_bf16lo(v.x); f[1] = lk_bf16hi(v.x); f[2] = lk_bf16lo(v.y); f[3] = lk_bf16hi(v.y);
    f[4] = lk_bf16lo(v.z); f[5] = lk_bf16hi(v.z); f[6] = lk_bf16lo(v.w); f[7] = lk_bf16hi(v.w);
  }
}

// Per-head tables for the epilogue.
struct FinalizeParams {
  uint32_t* ws;      // [n_ksplit][rows][n_tot] partials (fp32 bits or int32)
  int n_ksplit;
  int ws_rows;       // rows in the workspace slab (partials index local rows)
  int row0;          // global row of local row 0
  int rows;          // rows this launch finalises
  int n_tot;
  int n_new;
  int int_inputs;
  const float* x_scale;
  const uint16_t* a_scale;
  int32_t* seq_len;
  int32_t* counter;
  int do_update;
  int batch;
  lk::CacheView k, v;
  int tot_rb_k, tot_rb_v, tot_ng_k, tot_ng_v;
  uint8_t rank[2 * LK_MAX_HEADS];      // K heads then V heads
  int16_t col[2 * LK_MAX_HEADS];       // first latent column
  int16_t pref_rb[2 * LK_MAX_HEADS];   // prefix of row bytes within its cache
  int16_t pref_ng[2 * LK_MAX_HEADS];   // prefix of scale groups within its cache
};

LK_DEVICE void append_values(const FinalizeParams& p, int grow, int j, float v0, float v1);

// Sums the partials of head j for local row lrow, quantises them and writes
// the codes and scale of token seq_len[b] + t into the cache (one warp).
LK_DEVICE void append_head(const FinalizeParams& p, int lrow, int grow, int j) {
  const int lane = threadIdx.x & 31;
  const int r = p.rank[j];
  const int col0 = p.col[j];
  float vals[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int d = lane + 32 * q;
    float val = 0.0f;
    if (d < r) {
      const int n = col0 + d;
      // all slices' partials in flight at once, then summed in slice order
      const uint32_t* src = p.ws + (int64_t)lrow * p.n_tot + n;
      const int64_t stride = (int64_t)p.ws_rows * p.n_tot;
      if (p.int_inputs) {
        int acc = 0;
        int s = 0;
        for (; s + 8 <= p.n_ksplit; s += 8) {
          uint32_t v[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] = __ldcg(src + (s + k) * stride);
#pragma unroll
          for (int k = 0; k < 8; ++k) acc += (int)v[k];
        }
        for (; s < p.n_ksplit; ++s) acc += (int)__ldcg(src + s * stride);
        val = __fmul_rn(__fmul_rn((float)acc, p.x_scale[grow]), lk_f16_to_f32(p.a_scale[n]));
      } else {
        int s = 0;
        for (; s + 8 <= p.n_ksplit; s += 8) {
          uint32_t v[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] = __ldcg(src + (s + k) * stride);
#pragma unroll
          for (int k = 0; k < 8; ++k) val += __uint_as_float(v[k]);
        }
        for (; s < p.n_ksplit; ++s) val += __uint_as_float(__ldcg(src + s * stride));
      }
    }
    vals[q] = val;
  }
  append_values(p, grow, j, vals[0], vals[1]);
}

// Quantises one head's latent row (lane l holds dims l and l + 32) and writes
// the codes and scale of token seq_len[b] + t into the cache (one warp).
LK_DEVICE void append_values(const FinalizeParams& p, int grow, int j, float v0, float v1) {
  const int lane = threadIdx.x & 31;
  const int b = grow / p.n_new, t = grow % p.n_new;
  const bool is_k = j < p.k.n_heads;
  const lk::CacheView& cv = is_k ? p.k : p.v;
  const int hh = is_k ? j : j - p.k.n_heads;
  const int r = p.rank[j];
  if (cv.rotation) lk_rotate_latent_warp(v0, v1, r);
  const LkQRow qr = lk_quantize_row_warp(v0, v1, r, cv.kind, cv.group);
  const int64_t pos = (int64_t)p.seq_len[b] + t;
  const int cap = cv.capacity;
  // the host checked the capacity against its copy of seq_len; never write past
  // it even if the device copy disagrees
  if (pos < 0 || pos >= cap) return;
  const int tot_rb = is_k ? p.tot_rb_k : p.tot_rb_v;
  const int tot_ng = is_k ? p.tot_ng_k : p.tot_ng_v;
  if (cv.kind == 0) {
    int8_t* plane = static_cast<int8_t*>(cv.codes) + ((int64_t)b * tot_rb + p.pref_rb[j]) * cap;
    if (is_k) {  // token-major chunks
      const int cs = lk_chunk_bytes(r);
      if (lane < r) plane[lk_code_offset(pos, lane, r, cs)] = (int8_t)qr.c0;
      if (lane + 32 < r) plane[lk_code_offset(pos, lane + 32, r, cs)] = (int8_t)qr.c1;
    } else {     // dimension-major: dim d of token t at (t/16)*16*r + d*16 + t%16
      const int64_t base = (pos >> 4) * 16 * r + (pos & 15);
      if (lane < r) plane[base + lane * 16] = (int8_t)qr.c0;
      if (lane + 32 < r) plane[base + (lane + 32) * 16] = (int8_t)qr.c1;
    }
    if (lane == 0) static_cast<float*>(cv.scales)[((int64_t)b * cv.n_heads + hh) * cap + pos] = qr.s0;
  } else {
    const int rb = r / 2;
    uint8_t* plane = static_cast<uint8_t*>(cv.codes) + ((int64_t)b * tot_rb + p.pref_rb[j]) * cap;
    if (is_k) {  // token-major chunks, two dims per byte
      const int cs = lk_chunk_bytes(rb);
      const int n0 = __shfl_down_sync(0xffffffffu, qr.c0, 1);
      const int n1 = __shfl_down_sync(0xffffffffu, qr.c1, 1);
      if ((lane & 1) == 0) {
        if (lane < r) plane[lk_code_offset(pos, lane / 2, rb, cs)] = (uint8_t)((qr.c0 & 0xF) | ((n0 & 0xF) << 4));
        if (lane + 32 < r)
          plane[lk_code_offset(pos, (lane + 32) / 2, rb, cs)] = (uint8_t)((qr.c1 & 0xF) | ((n1 & 0xF) << 4));
      }
    } else {     // dimension-major, two tokens per byte: write this token's nibble only
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        const int d = lane + 32 * q2;
        if (d < r) {
          const int64_t off = (pos >> 4) * 16 * rb + d * 8 + ((pos & 15) >> 1);
          unsigned int* word = reinterpret_cast<unsigned int*>(plane + (off & ~(int64_t)3));
          const unsigned int shift = (unsigned int)((off & 3) * 8 + (pos & 1) * 4);
          const unsigned int code = (unsigned int)((q2 == 0 ? qr.c0 : qr.c1) & 0xF);
          atomicAnd(word, ~(0xFu << shift));  // the neighbour token's nibble may be written concurrently
          atomicOr(word, code << shift);
        }
      }
    }
    const int g = min(cv.group, r), ng = (r + g - 1) / g;
    uint16_t* sp = static_cast<uint16_t*>(cv.scales) + ((int64_t)b * tot_ng + p.pref_ng[j]) * cap + pos * ng;
    if (lane < r && lane % g == 0) sp[lane / g] = lk_f32_to_f16_bits(qr.s0);
    if (lane + 32 < r && (lane + 32) % g == 0) sp[(lane + 32) / g] = lk_f32_to_f16_bits(qr.s1);
  }
}

// Prefill epilogue: a warp per (row, head) item, the warps striding over all
// items (a grid of a few CTAs per SM, so that the closing ticket below is a
// few thousand atomics on one word, not one per 4 items); the last CTA
// advances seq_len.
__global__ void __launch_bounds__(128) proj_finalize_kernel(const __grid_constant__ FinalizeParams p) {
  lk_grid_dep_launch();  // a decode launched next may start its set-up now
  const int n_heads_tot = p.k.n_heads + p.v.n_heads;
  const int64_t items = (int64_t)p.rows * n_heads_tot;
  for (int64_t item = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5); item < items; item += (int64_t)gridDim.x * 4) {
    const int lrow = (int)(item / n_heads_tot);
    append_head(p, lrow, p.row0 + lrow, (int)(item % n_heads_tot));
  }
  if (!p.do_update) return;
  // last CTA to arrive advances the sequence lengths (every CTA has read them)
  __shared__ int last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = (atomicAdd(p.counter, 1) == (int)gridDim.x - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int b = threadIdx.x; b < p.batch; b += blockDim.x) p.seq_len[b] += p.n_new;
  if (threadIdx.x == 0) *p.counter = 0;
}

// ---------------------------------------------------------------- decode: one cluster per head
// A thread-block cluster of CE CTAs owns one head: CTA q reduces the q-th
// slice of E for every latent column of the head and every row; the
// cluster's rank 0 sums the CE partials over distributed shared memory,
// quantises and appends.  No partials leave the SMs and nobody waits on a
// global counter; the last head to finish advances seq_len (atomic ticket).
//
// Inside a CTA the head's columns are cut into tiles of 8; a warp takes one
// tile over a contiguous range of the slice (the 8 warps spread over the
// tiles, several warps per tile when the head has fewer than 8 tiles).
// Lane 4 c + k takes column c of the tile and every fourth 16-byte chunk of
// the range starting at k: the four lanes of a column read 64 consecutive
// bytes of its weight row per load, each weight is read once from memory,
// and the rows of x (converted once to fp32 in shared memory) are broadcast
// loads.  The four lanes' sums meet by two shuffles, the warps of a tile in
// shared memory in a fixed order (the result does not depend on timing).
// CTAs per head: 8 (the portable cluster size) for 3..8 token rows; 4 for one
// or two rows, whose CTAs finish sooner and leave more of the GPU to an
// attention launch that overlaps them (decode step)
constexpr int kClusterMax = 8;
int cluster_for_rows(int rows) { return rows <= 2 ? 4 : 8; }
constexpr int kProjWarps = kGemvThreads / 32;

struct ClusterProjParams {
  FinalizeParams f;
  const void* x;
  const void* A;
  int M, E, slice;
  int32_t* done_cnt;
  int off_x, off_red;  // shared-memory offsets: x slice (fp32, or int8 for int8 inputs), warp partials
};

template <int XT, int MT, int CE>
__global__ void __launch_bounds__(kGemvThreads) proj_cluster_kernel(const __grid_constant__ ClusterProjParams p) {
  lk_grid_dep_launch();  // a decode launched next may start its set-up now
  using T = typename XTraits<XT>::T;
  constexpr int VE = XTraits<XT>::VE;
  constexpr bool INT = XT == lk::X_I8;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const FinalizeParams& f = p.f;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int j = blockIdx.y;
  const int r = f.rank[j], col0 = f.col[j];
  const int M = p.M;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int e0 = rank * p.slice;
  const int elen = max(0, min(p.slice, p.E - e0));
  const int chunks = elen / VE;
  // every CTA's partials go straight into rank 0's shared memory:
  // part[q][n][m] for slice q, latent column n, row m
  uint32_t* part = reinterpret_cast<uint32_t*>(smem_raw);
  uint32_t* mine = cluster.map_shared_rank(part, 0) + (size_t)rank * LK_MAX_RANK * M;
  // a peer's shared memory may be written only once that CTA runs: arrive now,
  // wait just before the first remote write
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  const T* x = static_cast<const T*>(p.x);
  const T* A = static_cast<const T*>(p.A);
  // x slice into shared memory: fp32 for float inputs, the int8 codes as they are
  float* xf = reinterpret_cast<float*>(smem_raw + p.off_x);
  int8_t* xi = reinterpret_cast<int8_t*>(smem_raw + p.off_x);
  for (int i = threadIdx.x; i < M * chunks; i += kGemvThreads) {
    const int m = i / chunks, cc = i - m * chunks;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + (int64_t)m * p.E + e0 + cc * VE));
    if constexpr (INT) {
      *reinterpret_cast<uint4*>(xi + (size_t)m * p.slice + cc * VE) = v;
    } else {
      float vf[VE];
      expand16<XT>(v, vf);
      float4* dst = reinterpret_cast<float4*>(xf + (size_t)m * p.slice + cc * VE);
#pragma unroll
      for (int k = 0; k < VE / 4; ++k) dst[k] = make_float4(vf[4 * k], vf[4 * k + 1], vf[4 * k + 2], vf[4 * k + 3]);
    }
  }
  __syncthreads();
  // warps -> (column tile, range of the slice)
  const int ntiles = (r + 7) / 8;
  const int wpt = ntiles >= kProjWarps ? 1 : kProjWarps / ntiles;  // warps per tile
  const int tile = warp / wpt, sub = warp - tile * wpt;
  const int c = lane >> 2, kp = lane & 3;
  const int n = 8 * tile + c;  // column of this lane
  const bool live = tile < ntiles && n < r;
  float facc[MT];
  int iacc[MT];
#pragma unroll
  for (int i = 0; i < MT; ++i) { facc[i] = 0.0f; iacc[i] = 0; }
  if (tile < ntiles) {
    const int per = (chunks + wpt - 1) / wpt;
    const int k0 = sub * per, k1 = min(chunks, k0 + per);
    const T* arow = A + (int64_t)(col0 + (live ? n : 0)) * p.E + e0;
    constexpr int U = 8;  // loads in flight per lane
    for (int kc0 = k0 + kp; kc0 < k1; kc0 += 4 * U) {
      uint4 wv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int kc = kc0 + 4 * u;
        wv[u] = (live && kc < k1) ? __ldg(reinterpret_cast<const uint4*>(arow + kc * VE)) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int kc = kc0 + 4 * u;
        if (kc < k1) {
          if constexpr (INT) {
#pragma unroll
            for (int i = 0; i < MT; ++i) {
              if (i < M) {
                const uint4 xv = *reinterpret_cast<const uint4*>(xi + (size_t)i * p.slice + kc * VE);
                int a2 = iacc[i];
                a2 = __dp4a((int)xv.x, (int)wv[u].x, a2);
                a2 = __dp4a((int)xv.y, (int)wv[u].y, a2);
                a2 = __dp4a((int)xv.z, (int)wv[u].z, a2);
                a2 = __dp4a((int)xv.w, (int)wv[u].w, a2);
                iacc[i] = a2;
              }
            }
          } else {
            float wf[VE];
            expand16<XT>(wv[u], wf);
#pragma unroll
            for (int i = 0; i < MT; ++i) {
              if (i < M) {
                const float4* xr = reinterpret_cast<const float4*>(xf + (size_t)i * p.slice + kc * VE);
                float a2 = facc[i];
#pragma unroll
                for (int k = 0; k < VE / 4; ++k) {
                  const float4 xv = xr[k];
                  a2 = fmaf(xv.x, wf[4 * k], a2);
                  a2 = fmaf(xv.y, wf[4 * k + 1], a2);
                  a2 = fmaf(xv.z, wf[4 * k + 2], a2);
                  a2 = fmaf(xv.w, wf[4 * k + 3], a2);
                }
                facc[i] = a2;
              }
            }
          }
        }
      }
    }
  }
  // the four lanes of a column (k phases 0..3), then the warps of a tile
  uint32_t* red = reinterpret_cast<uint32_t*>(smem_raw + p.off_red);  // [warp][8 columns][MT]
#pragma unroll
  for (int i = 0; i < MT; ++i) {
    uint32_t val;
    if (INT) {
      int a2 = iacc[i];
      a2 += __shfl_xor_sync(0xffffffffu, a2, 1);
      a2 += __shfl_xor_sync(0xffffffffu, a2, 2);
      val = (uint32_t)a2;
    } else {
      float a2 = facc[i];
      a2 += __shfl_xor_sync(0xffffffffu, a2, 1);
      a2 += __shfl_xor_sync(0xffffffffu, a2, 2);
      val = __float_as_uint(a2);
    }
    if (kp == 0) red[(warp * 8 + c) * MT + i] = val;
  }
  __syncthreads();
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");  // every peer runs: its shared memory may be written
  for (int idx = threadIdx.x; idx < r * M; idx += kGemvThreads) {
    const int nn = idx / M, m = idx - nn * M;
    const int t = nn / 8, cc = nn - 8 * t;
    uint32_t val;
    if (INT) {
      int a2 = 0;
      for (int s2 = 0; s2 < wpt; ++s2) a2 += (int)red[((t * wpt + s2) * 8 + cc) * MT + m];
      val = (uint32_t)a2;
    } else {
      float a2 = 0.0f;
      for (int s2 = 0; s2 < wpt; ++s2) a2 += __uint_as_float(red[((t * wpt + s2) * 8 + cc) * MT + m]);
      val = __float_as_uint(a2);
    }
    mine[nn * M + m] = val;
  }
  cluster.sync();  // every CTA's partials are in rank 0's shared memory
  if (rank != 0) return;
  {
    for (int m = warp; m < M; m += kGemvThreads / 32) {
      float vals[2];
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        const int d = lane + 32 * q2;
        float val = 0.0f;
        if (d < r) {
          const int nn = col0 + d;
          if (INT) {
            int acc = 0;
#pragma unroll
            for (int q = 0; q < CE; ++q) acc += (int)part[((size_t)q * LK_MAX_RANK + d) * M + m];
            val = __fmul_rn(__fmul_rn((float)acc, f.x_scale[m]), lk_f16_to_f32(f.a_scale[nn]));
          } else {
#pragma unroll
            for (int q = 0; q < CE; ++q) val += __uint_as_float(part[((size_t)q * LK_MAX_RANK + d) * M + m]);
          }
        }
        vals[q2] = val;
      }
      append_values(f, m, j, vals[0], vals[1]);
    }
  }
  __syncthreads();  // every append of this head is written
  if (threadIdx.x == 0) {
    __threadfence();
    const int n_heads_tot = f.k.n_heads + f.v.n_heads;
    if (atomicAdd(p.done_cnt, 1) == n_heads_tot - 1) {  // every head appended: advance the rows
      __threadfence();
      for (int b = 0; b < f.batch; ++b) f.seq_len[b] += f.n_new;
      *p.done_cnt = 0;
    }
  }
}

// ---------------------------------------------------------------- decode, bf16: tensor-core GEMV
// v^T = A x^T for up to 32 token rows of bf16 inputs, one launch.  A CTA owns
// 16 latent columns (one m16 tile) over all of E; its 8 warps split E.  Per
// 64-element k block a lane loads 16 consecutive k of two weight rows (gid,
// gid + 8) and of its token rows (gid, gid + 8, ...), and the block's four
// m16n8k16 products take their k slots from those registers: product s uses
// k = 16 tig + 4 s + {0, 1} for the slots 2 tig, 2 tig + 1 and 16 tig + 4 s +
// {2, 3} for 2 tig + 8, 2 tig + 9, for A and x alike, so every k of the block
// meets its own x once and the sum is the plain dot product.  Each weight is
// read once (16-byte loads, L1 bypassed); the tensor cores only keep the
// instruction count per byte low, the launch is bound by HBM.  The warps'
// sums meet in shared memory in a fixed order, go to the workspace, and the
// CTA that completes a head's last column block (ticket per head) quantises
// and appends that head for every row; the last head advances seq_len.
constexpr int kMmaWarps = 8;
constexpr int kMmaMaxRows = 32;

struct MmaProjParams {
  FinalizeParams f;
  const uint16_t* x;
  const uint16_t* A;
  int M, E;
  int32_t* done_cnt;
  int32_t* head_cnt;  // [heads] column blocks of the head done in this launch
};

LK_DEVICE uint4 ldg_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

LK_DEVICE uint32_t word_of(const uint4 (&v)[2], int w) {
  const uint4& q = v[w >> 2];
  return (w & 3) == 0 ? q.x : (w & 3) == 1 ? q.y : (w & 3) == 2 ? q.z : q.w;
}

template <int NT>  // n8 tiles of token rows: M <= 8 NT
__global__ void __launch_bounds__(kMmaWarps * 32) proj_mma_kernel(const __grid_constant__ MmaProjParams p) {
  lk_grid_dep_launch();  // a decode launched next may start its set-up now
  constexpr int BR = NT == 1 ? 4 : (NT == 2 ? 2 : 1);  // k blocks whose loads are in flight together
  __shared__ float red[kMmaWarps][16][8 * NT + 1];
  __shared__ int fin[16];  // heads whose last column block this CTA completed
  __shared__ int nfin;
  const FinalizeParams& f = p.f;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int col0 = blockIdx.x * 16;
  const int M = p.M, E = p.E;
  const int nb = (E + 63) / 64;
  const int kb0 = warp * nb / kMmaWarps, kb1 = (warp + 1) * nb / kMmaWarps;
  // columns past n_tot (last tile) repeat the last row: computed, never stored
  const uint16_t* A0 = p.A + (int64_t)min(col0 + gid, f.n_tot - 1) * E;
  const uint16_t* A1 = p.A + (int64_t)min(col0 + gid + 8, f.n_tot - 1) * E;
  if (threadIdx.x == 0) nfin = 0;
  float c[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) c[t][0] = c[t][1] = c[t][2] = c[t][3] = 0.0f;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (int kb = kb0; kb < kb1; kb += BR) {
    uint4 wa[BR][2], wb[BR][2], xv[BR][NT][2];
#pragma unroll
    for (int u = 0; u < BR; ++u) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int k = (kb + u) * 64 + 16 * tig + 8 * h;
        const bool ok = kb + u < kb1 && k < E;  // E is a multiple of 8
        wa[u][h] = ok ? ldg_stream16(A0 + k) : z;
        wb[u][h] = ok ? ldg_stream16(A1 + k) : z;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const int m = 8 * t + gid;
          // (volatile like the weight loads, so that all of a round's loads are
          // issued before the first product waits on one)
          xv[u][t][h] = ok && m < M ? ldg_stream16(p.x + (int64_t)m * E + k) : z;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < BR; ++u) {
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint32_t a0 = word_of(wa[u], 2 * s), a2 = word_of(wa[u], 2 * s + 1);
        const uint32_t a1 = word_of(wb[u], 2 * s), a3 = word_of(wb[u], 2 * s + 1);
#pragma unroll
        for (int t = 0; t < NT; ++t)
          lk_mma_bf16_16816(c[t], a0, a1, a2, a3, word_of(xv[u][t], 2 * s), word_of(xv[u][t], 2 * s + 1));
      }
    }
  }
  // D fragment: c0, c1 = (column gid, rows 2 tig, 2 tig + 1), c2, c3 = column gid + 8
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    red[warp][gid][8 * t + 2 * tig] = c[t][0];
    red[warp][gid][8 * t + 2 * tig + 1] = c[t][1];
    red[warp][gid + 8][8 * t + 2 * tig] = c[t][2];
    red[warp][gid + 8][8 * t + 2 * tig + 1] = c[t][3];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < 16 * M; idx += kMmaWarps * 32) {
    const int cc = idx / M, m = idx - cc * M;
    const int n = col0 + cc;
    if (n < f.n_tot) {
      float s = 0.0f;
#pragma unroll
      for (int w = 0; w < kMmaWarps; ++w) s += red[w][cc][m];
      f.ws[(int64_t)m * f.n_tot + n] = __float_as_uint(s);
    }
  }
  __threadfence();
  __syncthreads();
  const int nh = f.k.n_heads + f.v.n_heads;
  for (int j = threadIdx.x; j < nh; j += kMmaWarps * 32) {
    const int h0 = f.col[j], h1 = h0 + f.rank[j];
    if (h0 < col0 + 16 && h1 > col0) {
      const int nblk = (h1 - 1) / 16 - h0 / 16 + 1;
      if (atomicAdd(&p.head_cnt[j], 1) == nblk - 1) fin[atomicAdd(&nfin, 1)] = j;
    }
  }
  __syncthreads();
  const int nf = nfin;
  if (nf == 0) return;
  __threadfence();  // the other blocks' columns of these heads are visible
  for (int it = warp; it < nf * M; it += kMmaWarps) {
    const int j = fin[it / M], m = it - (it / M) * M;
    append_head(f, m, m, j);
  }
  __syncthreads();  // every append of these heads is written
  if (threadIdx.x == 0) {
    for (int i = 0; i < nf; ++i) p.head_cnt[fin[i]] = 0;  // ready for the next call
    __threadfence();
    if (atomicAdd(p.done_cnt, nf) == nh - nf) {  // every head appended: advance the rows
      __threadfence();
      for (int b = 0; b < f.batch; ++b) f.seq_len[b] += f.n_new;
      *p.done_cnt = 0;
    }
  }
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

// E-slice of each cluster CTA for the decode kernel (16-byte multiple).
int cluster_slice(int E, int xtype, int ce) {
  const int ve = xtype == lk::X_F32 ? 4 : (xtype == lk::X_BF16 ? 8 : 16);
  return round_up((E + ce - 1) / ce, ve);
}

int x_size(int xtype) { return xtype == lk::X_F32 ? 4 : (xtype == lk::X_BF16 ? 2 : 1); }

constexpr int kPrefillRowChunk = 8192;
constexpr size_t kWsHeader = 2048;  // done counter at 0, per-head counters from byte 256 on
constexpr int kHeadCntOffset = 256;

}  // namespace

LK_DEFINE_STATUS_ACCESSOR(lk_project_status_word)

namespace lk {

size_t project_workspace_bytes(int rows, int n_tot, int embed_dim, int xtype, int num_sms) {
  (void)num_sms;
  size_t body;
  if (xtype == X_BF16 && rows <= kMmaMaxRows) {
    body = (size_t)rows * n_tot * 4;  // the column sums, read back by each head's finishing CTA
  } else if (rows <= kGemvMaxRows) {
    body = 0;  // partials stay in the cluster's shared memory
  } else {
    body = (size_t)std::min(rows, kPrefillRowChunk) * n_tot * 4;
  }
  return kWsHeader + body;
}

cudaError_t launch_project_append(const ProjectLaunch& a, cudaStream_t stream) {
  const int rows = a.batch * a.n_new;
  if (rows == 0) return cudaSuccess;
  FinalizeParams f{};
  f.n_tot = a.n_tot;
  f.n_new = a.n_new;
  f.int_inputs = a.xtype == X_I8;
  f.x_scale = a.x_scale;
  f.a_scale = a.a_scale;
  f.seq_len = a.seq_len;
  f.counter = static_cast<int32_t*>(a.workspace);
  f.batch = a.batch;
  f.k = a.k;
  f.v = a.v;
  f.ws = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(a.workspace) + kWsHeader);
  int col = 0;
  for (int c = 0; c < 2; ++c) {
    const CacheView& cv = c == 0 ? a.k : a.v;
    const int32_t* ranks = c == 0 ? a.ranks_k : a.ranks_v;
    int prb = 0, png = 0;
    for (int h = 0; h < cv.n_heads; ++h) {
      const int j = c * a.k.n_heads + h;
      const int r = ranks[h];
      f.rank[j] = (uint8_t)r;
      f.col[j] = (int16_t)col;
      f.pref_rb[j] = (int16_t)prb;
      f.pref_ng[j] = (int16_t)png;
      col += r;
      prb += cv.kind == 0 ? r : r / 2;
      const int g = std::min(cv.group, r);
      png += cv.kind == 0 ? 1 : (r + g - 1) / g;
    }
    if (c == 0) { f.tot_rb_k = prb; f.tot_ng_k = png; }
    else { f.tot_rb_v = prb; f.tot_ng_v = png; }
  }
  const int heads_tot = a.k.n_heads + a.v.n_heads;
  cudaError_t e;

  if (a.xtype == X_BF16 && rows <= kMmaMaxRows) {
    MmaProjParams d{};
    f.n_ksplit = 1;
    f.ws_rows = rows;
    f.row0 = 0;
    f.rows = rows;
    f.do_update = 1;
    d.f = f;
    d.x = static_cast<const uint16_t*>(a.x);
    d.A = static_cast<const uint16_t*>(a.A);
    d.M = rows;
    d.E = a.embed_dim;
    d.done_cnt = static_cast<int32_t*>(a.workspace);
    d.head_cnt = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(a.workspace) + kHeadCntOffset);
    const unsigned grid = (unsigned)((a.n_tot + 15) / 16);
    if (rows <= 8) proj_mma_kernel<1><<<grid, kMmaWarps * 32, 0, stream>>>(d);
    else if (rows <= 16) proj_mma_kernel<2><<<grid, kMmaWarps * 32, 0, stream>>>(d);
    else proj_mma_kernel<4><<<grid, kMmaWarps * 32, 0, stream>>>(d);
    count_launch();
    return cudaGetLastError();
  }

  if (rows <= kGemvMaxRows) {
    ClusterProjParams d{};
    f.n_ksplit = 1;
    f.ws_rows = rows;
    f.row0 = 0;
    f.rows = rows;
    f.do_update = 1;
    d.f = f;
    d.x = a.x;
    d.A = a.A;
    d.M = rows;
    d.E = a.embed_dim;
    d.done_cnt = static_cast<int32_t*>(a.workspace);
    const size_t xelem = a.xtype == X_I8 ? 1 : 4;  // x slice in shared memory: int8 or fp32
    const int ce = cluster_for_rows(rows);
    d.slice = cluster_slice(a.embed_dim, a.xtype, ce);
    d.off_x = round_up(kClusterMax * LK_MAX_RANK * rows * 4, 128);
    d.off_red = d.off_x + round_up((int)(rows * d.slice * xelem), 128);
    const int mt = rows <= 1 ? 1 : (rows <= 2 ? 2 : (rows <= 4 ? 4 : 8));
    const size_t smem = (size_t)d.off_red + (size_t)kProjWarps * 8 * mt * 4;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ce, heads_tot, 1);
    cfg.blockDim = dim3(kGemvThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ce;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
#define LK_PROJ_LAUNCH3(XTV, MTV, CEV)                                                                      \
  do {                                                                                                     \
    e = cudaFuncSetAttribute(proj_cluster_kernel<XTV, MTV, CEV>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             (int)smem);                                                                  \
    if (e != cudaSuccess) return e;                                                                        \
    e = cudaLaunchKernelEx(&cfg, proj_cluster_kernel<XTV, MTV, CEV>, d);                                  \
    if (e == cudaSuccess) count_launch();                                                                  \
  } while (0)
#define LK_PROJ_LAUNCH(XTV, MTV)                 \
  do {                                           \
    if (ce == 4) LK_PROJ_LAUNCH3(XTV, MTV, 4);   \
    else LK_PROJ_LAUNCH3(XTV, MTV, 8);           \
  } while (0)
#define LK_PROJ_MT(XTV)                          \
  do {                                           \
    if (mt == 1) LK_PROJ_LAUNCH(XTV, 1);         \
    else if (mt == 2) LK_PROJ_LAUNCH(XTV, 2);    \
    else if (mt == 4) LK_PROJ_LAUNCH(XTV, 4);    \
    else LK_PROJ_LAUNCH(XTV, 8);                 \
  } while (0)
    if (a.xtype == X_F32) LK_PROJ_MT(X_F32);
    else if (a.xtype == X_BF16) LK_PROJ_MT(X_BF16);
    else LK_PROJ_MT(X_I8);
#undef LK_PROJ_MT
#undef LK_PROJ_LAUNCH
#undef LK_PROJ_LAUNCH3
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }

  // prefill: row chunks through the tiled GEMM
  const int chunk = std::min(rows, kPrefillRowChunk);
  const int xs = x_size(a.xtype);
  for (int r0 = 0; r0 < rows; r0 += chunk) {
    const int nr = std::min(chunk, rows - r0);
    const uint8_t* xr = static_cast<const uint8_t*>(a.x) + (size_t)r0 * a.embed_dim * xs;
    if (a.xtype == X_I8) {
      e = launch_gemm_i8(reinterpret_cast<const int8_t*>(xr), a.embed_dim,
                         static_cast<const int8_t*>(a.A), a.embed_dim,
                         reinterpret_cast<int32_t*>(f.ws), a.n_tot, nr, a.n_tot, a.embed_dim, stream);
    } else if (a.xtype == X_BF16) {
      // a dense bf16 contraction: tcgen05 with TMEM accumulators
      if (!gemm_bf16_tc_supported(xr, a.embed_dim, a.A, a.embed_dim, a.embed_dim)) return cudaErrorInvalidValue;
      e = launch_gemm_bf16_tc(xr, a.embed_dim, a.A, a.embed_dim, reinterpret_cast<float*>(f.ws), a.n_tot, nr,
                              a.n_tot, a.embed_dim, stream);
    } else {
      e = launch_gemm_f(xr, a.embed_dim, a.A, a.embed_dim, reinterpret_cast<float*>(f.ws), a.n_tot, nr,
                        a.n_tot, a.embed_dim, false, stream);
    }
    if (e != cudaSuccess) return e;
    f.n_ksplit = 1;
    f.ws_rows = nr;
    f.row0 = r0;
    f.rows = nr;
    f.do_update = (r0 + nr == rows);
    const int64_t items = (int64_t)nr * heads_tot;
    const int64_t grid = std::min<int64_t>((items + 3) / 4, (int64_t)std::max(1, a.num_sms) * 16);
    proj_finalize_kernel<<<(unsigned)grid, 128, 0, stream>>>(f);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace lk
