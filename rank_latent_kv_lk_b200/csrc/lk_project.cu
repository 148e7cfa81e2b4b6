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
// Decode (<= 32 rows) runs both phases in ONE launch: a split-E GEMV with
// every weight chunk loaded up front, then per-head arrival tickets (no
// waiting) so the CTA that completes a head appends it, and the CTA that
// completes the last head advances seq_len.  Prefill runs the tiled GEMM per
// row chunk, then an epilogue launch.
#include "lk_common.cuh"
#include "lk_internal.h"
#include "lk_quant.cuh"

namespace lk {
cudaError_t launch_gemm_f(const void* A, int lda, const void* B, int ldb, float* C, int ldc, int M,
                          int N, int K, bool bf16, cudaStream_t stream);
}

namespace {

constexpr int kGemvThreads = 256;
constexpr int kColsPerWarp = 4;
constexpr int kColsPerCta = kColsPerWarp * (kGemvThreads / 32);  // 32
constexpr int kMT = 8;  // rows per pass
constexpr int kGemvMaxRows = 32;

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

// Sums the partials of head j for local row lrow, quantises them and writes
// the codes and scale of token seq_len[b] + t into the cache (one warp).
LK_DEVICE void append_head(const FinalizeParams& p, int lrow, int grow, int j) {
  const int lane = threadIdx.x & 31;
  const int b = grow / p.n_new, t = grow % p.n_new;
  const bool is_k = j < p.k.n_heads;
  const lk::CacheView& cv = is_k ? p.k : p.v;
  const int hh = is_k ? j : j - p.k.n_heads;
  const int r = p.rank[j];
  const int col0 = p.col[j];
  float vals[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int d = lane + 32 * q;
    float val = 0.0f;
    if (d < r) {
      const int n = col0 + d;
      if (p.int_inputs) {
        int acc = 0;
        for (int s = 0; s < p.n_ksplit; ++s) acc += (int)__ldcg(p.ws + ((int64_t)s * p.ws_rows + lrow) * p.n_tot + n);
        val = __fmul_rn(__fmul_rn((float)acc, p.x_scale[grow]), lk_f16_to_f32(p.a_scale[n]));
      } else {
        for (int s = 0; s < p.n_ksplit; ++s)
          val += __uint_as_float(__ldcg(p.ws + ((int64_t)s * p.ws_rows + lrow) * p.n_tot + n));
      }
    }
    vals[q] = val;
  }
  const LkQRow qr = lk_quantize_row_warp(vals[0], vals[1], r, cv.kind, cv.group);
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

// Prefill epilogue: one warp per (row, head); the last CTA advances seq_len.
__global__ void __launch_bounds__(128) proj_finalize_kernel(const __grid_constant__ FinalizeParams p) {
  const int n_heads_tot = p.k.n_heads + p.v.n_heads;
  const int64_t item = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  if (item < (int64_t)p.rows * n_heads_tot) {
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

// ---------------------------------------------------------------- decode: one fused launch
constexpr int kDecU = 2;  // 16-byte chunks per lane per column in one E-slice

struct DecodeProjParams {
  FinalizeParams f;
  const void* x;
  const void* A;
  int M, E, slice;
  int32_t* head_cnt;            // [n_heads_tot] arrival counters
  int32_t* done_cnt;            // heads appended so far
  int16_t expect[2 * LK_MAX_HEADS];  // arrivals that complete head j
};

// Split-E GEMV over 32 latent columns per CTA (4 per warp) with every weight
// chunk of the slice loaded up front, then per-head tickets: the CTA whose
// arrival completes a head quantises and appends it; the CTA completing the
// last head advances seq_len.
template <int XT>
__global__ void __launch_bounds__(kGemvThreads) proj_decode_kernel(const __grid_constant__ DecodeProjParams p) {
  using T = typename XTraits<XT>::T;
  constexpr int VE = XTraits<XT>::VE;
  constexpr bool INT = XT == lk::X_I8;
  extern __shared__ __align__(16) uint8_t xs_raw[];  // [M][slice] of T
  __shared__ int ready[2 * LK_MAX_HEADS];
  __shared__ int n_ready;
  const FinalizeParams& f = p.f;
  const T* x = static_cast<const T*>(p.x);
  const T* A = static_cast<const T*>(p.A);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ks = blockIdx.y;
  const int e0 = ks * p.slice;
  const int elen = min(p.slice, p.E - e0);
  const int chunks = elen / VE;
  const int n0 = blockIdx.x * kColsPerCta;
  const int nbase = n0 + warp * kColsPerWarp;
  const int N = f.n_tot, M = p.M;
  T* xs = reinterpret_cast<T*>(xs_raw);

  // all weight loads of this lane in flight before any use
  uint4 wv[kColsPerWarp][kDecU];
#pragma unroll
  for (int j = 0; j < kColsPerWarp; ++j)
#pragma unroll
    for (int u = 0; u < kDecU; ++u) {
      const int cc = lane + 32 * u, n = nbase + j;
      wv[j][u] = (cc < chunks && n < N)
                     ? __ldg(reinterpret_cast<const uint4*>(A + (int64_t)n * p.E + e0 + cc * VE))
                     : make_uint4(0, 0, 0, 0);
    }
  for (int c = threadIdx.x; c < M * chunks; c += kGemvThreads) {
    const int mm = c / chunks, cc = c % chunks;
    *reinterpret_cast<uint4*>(xs + mm * p.slice + cc * VE) =
        *reinterpret_cast<const uint4*>(x + (int64_t)mm * p.E + e0 + cc * VE);
  }
  if (threadIdx.x == 0) n_ready = 0;
  __syncthreads();

  for (int m0 = 0; m0 < M; m0 += kMT) {
    const int mt = min(kMT, M - m0);
    float facc[kColsPerWarp][kMT];
    int iacc[kColsPerWarp][kMT];
#pragma unroll
    for (int j = 0; j < kColsPerWarp; ++j)
#pragma unroll
      for (int i = 0; i < kMT; ++i) { facc[j][i] = 0.0f; iacc[j][i] = 0; }
#pragma unroll
    for (int u = 0; u < kDecU; ++u) {
      const int cc = lane + 32 * u;
      if (cc < chunks) {
#pragma unroll
        for (int i = 0; i < kMT; ++i) {
          if (i < mt) {
            const uint4 xv4 = *reinterpret_cast<const uint4*>(xs + (m0 + i) * p.slice + cc * VE);
            if (INT) {
#pragma unroll
              for (int j = 0; j < kColsPerWarp; ++j) {
                int a = iacc[j][i];
                a = __dp4a((int)xv4.x, (int)wv[j][u].x, a);
                a = __dp4a((int)xv4.y, (int)wv[j][u].y, a);
                a = __dp4a((int)xv4.z, (int)wv[j][u].z, a);
                a = __dp4a((int)xv4.w, (int)wv[j][u].w, a);
                iacc[j][i] = a;
              }
            } else {
              float xf[VE];
              expand16<XT>(xv4, xf);
#pragma unroll
              for (int j = 0; j < kColsPerWarp; ++j) {
                float wf[VE];
                expand16<XT>(wv[j][u], wf);
                float a = facc[j][i];
#pragma unroll
                for (int k = 0; k < VE; ++k) a = fmaf(xf[k], wf[k], a);
                facc[j][i] = a;
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kColsPerWarp; ++j) {
#pragma unroll
      for (int i = 0; i < kMT; ++i) {
        uint32_t val;
        if (INT) {
          int a = iacc[j][i];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
          val = (uint32_t)a;
        } else {
          val = __float_as_uint(lk_warp_sum(facc[j][i]));
        }
        const int n = nbase + j;
        if (lane == j * kMT + i && i < mt && n < N) f.ws[((int64_t)ks * M + m0 + i) * N + n] = val;
      }
    }
  }

  // arrivals: this CTA's 32 columns of slice ks are written
  __threadfence();
  __syncthreads();
  const int n_heads_tot = f.k.n_heads + f.v.n_heads;
  if (threadIdx.x == 0) {
    int nr = 0;
    for (int j = 0; j < n_heads_tot; ++j) {
      const int c0 = f.col[j], c1 = f.col[j] + f.rank[j];
      if (c0 < n0 + kColsPerCta && c1 > n0) {
        if (atomicAdd(&p.head_cnt[j], 1) + 1 == p.expect[j]) ready[nr++] = j;
      }
    }
    n_ready = nr;
  }
  __syncthreads();
  const int nr = n_ready;
  if (nr == 0) return;
  __threadfence();
  for (int it = warp; it < nr * M; it += kGemvThreads / 32) {
    const int j = ready[it / M], m = it % M;
    append_head(f, m, m, j);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 0; i < nr; ++i) p.head_cnt[ready[i]] = 0;
    __threadfence();
    if (atomicAdd(p.done_cnt, nr) + nr == n_heads_tot) {
      for (int b = 0; b < f.batch; ++b) f.seq_len[b] += f.n_new;
      *p.done_cnt = 0;
    }
  }
}

int round_up(int x, int m) { return (x + m - 1) / m * m; }

// E-slice per CTA for the decode kernel: kDecU chunks of 16 bytes per lane.
int decode_slice(int xtype) {
  const int ve = xtype == lk::X_F32 ? 4 : (xtype == lk::X_BF16 ? 8 : 16);
  return 32 * ve * kDecU;
}

int x_ve(int xtype) { return xtype == lk::X_F32 ? 4 : (xtype == lk::X_BF16 ? 8 : 16); }
int x_size(int xtype) { return xtype == lk::X_F32 ? 4 : (xtype == lk::X_BF16 ? 2 : 1); }

constexpr int kPrefillRowChunk = 8192;
constexpr size_t kWsHeader = 2048;  // done counter at 0, head counters at 256

}  // namespace

LK_DEFINE_STATUS_ACCESSOR(lk_project_status_word)

namespace lk {

size_t project_workspace_bytes(int rows, int n_tot, int embed_dim, int xtype, int num_sms) {
  (void)num_sms;
  size_t body;
  if (rows <= kGemvMaxRows) {
    const int slice = decode_slice(xtype);
    const int nks = (embed_dim + slice - 1) / slice;
    body = (size_t)nks * rows * n_tot * 4;
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

  if (rows <= kGemvMaxRows) {
    DecodeProjParams d{};
    const int slice = decode_slice(a.xtype);
    const int nks = (a.embed_dim + slice - 1) / slice;
    f.n_ksplit = nks;
    f.ws_rows = rows;
    f.row0 = 0;
    f.rows = rows;
    f.do_update = 1;
    d.f = f;
    d.x = a.x;
    d.A = a.A;
    d.M = rows;
    d.E = a.embed_dim;
    d.slice = slice;
    d.done_cnt = static_cast<int32_t*>(a.workspace);
    d.head_cnt = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(a.workspace) + 256);
    for (int j = 0; j < heads_tot; ++j) {
      const int c0 = f.col[j], c1 = f.col[j] + f.rank[j] - 1;
      d.expect[j] = (int16_t)((c1 / kColsPerCta - c0 / kColsPerCta + 1) * nks);
    }
    const size_t smem = (size_t)rows * slice * x_size(a.xtype);
    dim3 grid((a.n_tot + kColsPerCta - 1) / kColsPerCta, nks);
    if (a.xtype == X_F32) {
      e = cudaFuncSetAttribute(proj_decode_kernel<X_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      proj_decode_kernel<X_F32><<<grid, kGemvThreads, smem, stream>>>(d);
    } else if (a.xtype == X_BF16) {
      e = cudaFuncSetAttribute(proj_decode_kernel<X_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      proj_decode_kernel<X_BF16><<<grid, kGemvThreads, smem, stream>>>(d);
    } else {
      e = cudaFuncSetAttribute(proj_decode_kernel<X_I8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      proj_decode_kernel<X_I8><<<grid, kGemvThreads, smem, stream>>>(d);
    }
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
    } else {
      e = launch_gemm_f(xr, a.embed_dim, a.A, a.embed_dim, reinterpret_cast<float*>(f.ws), a.n_tot, nr,
                        a.n_tot, a.embed_dim, a.xtype == X_BF16, stream);
    }
    if (e != cudaSuccess) return e;
    f.n_ksplit = 1;
    f.ws_rows = nr;
    f.row0 = r0;
    f.rows = nr;
    f.do_update = (r0 + nr == rows);
    const int64_t items = (int64_t)nr * heads_tot;
    proj_finalize_kernel<<<(unsigned)((items + 3) / 4), 128, 0, stream>>>(f);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace lk
