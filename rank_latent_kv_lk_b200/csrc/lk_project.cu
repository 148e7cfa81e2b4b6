// Latent projection + quantisation + append (WSVD page §2A: every head stores
// only its latent x A^h; §2C: stored in 8 or 4 bits; LASER page §4: the
// projection, latent generation and quantisation are fused).
//
// Two phases per call:
//   1. v = x A^T for all heads at once (A is [N_tot, E], K heads then V
//      heads).  Small batches (decode) use a split-E GEMV that streams A once
//      with 16-byte loads; large batches (prefill) use the tiled GEMM.
//      Partial sums go to the workspace.
//   2. One warp per (token, head): sum the partials in a fixed order, apply
//      the int8 dequantisation scales when the inputs are int8, quantise the
//      r_h values (absmax, RNE) and write codes + scale at position
//      seq_len[b] + t in the token-tiled cache layout.  The last CTA to
//      finish (atomic ticket) bumps seq_len.
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

// Split-E GEMV: ws[ks][m][n] = sum_{e in slice ks} x[m][e] * A[n][e].
// Each warp owns kColsPerWarp columns; lanes sweep the slice in 16-byte chunks.
template <int XT>
__global__ void __launch_bounds__(kGemvThreads) proj_gemv_kernel(const void* __restrict__ xv,
                                                                const void* __restrict__ Av, int M, int N,
                                                                int E, int slice, uint32_t* __restrict__ ws) {
  using T = typename XTraits<XT>::T;
  constexpr int VE = XTraits<XT>::VE;
  constexpr bool INT = XT == lk::X_I8;
  extern __shared__ __align__(16) uint8_t xs_raw[];  // [kMT][slice] of T
  const T* x = static_cast<const T*>(xv);
  const T* A = static_cast<const T*>(Av);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ks = blockIdx.y;
  const int e0 = ks * slice;
  const int elen = min(slice, E - e0);
  const int nbase = blockIdx.x * kColsPerCta + warp * kColsPerWarp;
  T* xs = reinterpret_cast<T*>(xs_raw);

  for (int m0 = 0; m0 < M; m0 += kMT) {
    const int mt = min(kMT, M - m0);
    __syncthreads();
    // stage x[m0 .. m0+mt)[e0 .. e0+elen) (16-byte chunks)
    const int chunks_per_row = elen / VE;
    for (int c = threadIdx.x; c < mt * chunks_per_row; c += kGemvThreads) {
      const int mm = c / chunks_per_row, cc = c % chunks_per_row;
      *reinterpret_cast<uint4*>(xs + mm * slice + cc * VE) =
          *reinterpret_cast<const uint4*>(x + (int64_t)(m0 + mm) * E + e0 + cc * VE);
    }
    __syncthreads();

    float facc[kColsPerWarp][kMT];
    int iacc[kColsPerWarp][kMT];
#pragma unroll
    for (int j = 0; j < kColsPerWarp; ++j)
#pragma unroll
      for (int i = 0; i < kMT; ++i) { facc[j][i] = 0.0f; iacc[j][i] = 0; }

    for (int cc = lane; cc < chunks_per_row; cc += 32) {
      uint4 wv[kColsPerWarp];
#pragma unroll
      for (int j = 0; j < kColsPerWarp; ++j) {
        const int n = nbase + j;
        wv[j] = n < N ? __ldg(reinterpret_cast<const uint4*>(A + (int64_t)n * E + e0 + cc * VE))
                      : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < kMT; ++i) {
        if (i < mt) {
          const uint4 xv4 = *reinterpret_cast<const uint4*>(xs + i * slice + cc * VE);
          if (INT) {
#pragma unroll
            for (int j = 0; j < kColsPerWarp; ++j) {
              int a = iacc[j][i];
              a = __dp4a((int)xv4.x, (int)wv[j].x, a);
              a = __dp4a((int)xv4.y, (int)wv[j].y, a);
              a = __dp4a((int)xv4.z, (int)wv[j].z, a);
              a = __dp4a((int)xv4.w, (int)wv[j].w, a);
              iacc[j][i] = a;
            }
          } else {
            float xf[VE];
            expand16<XT>(xv4, xf);
#pragma unroll
            for (int j = 0; j < kColsPerWarp; ++j) {
              float wf[VE];
              expand16<XT>(wv[j], wf);
              float a = facc[j][i];
#pragma unroll
              for (int k = 0; k < VE; ++k) a = fmaf(xf[k], wf[k], a);
              facc[j][i] = a;
            }
          }
        }
      }
    }
    // reduce over lanes and store
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
        if (lane == j * kMT + i && i < mt && n < N)
          ws[((int64_t)ks * M + m0 + i) * N + n] = val;
      }
    }
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

__global__ void __launch_bounds__(128) proj_finalize_kernel(const __grid_constant__ FinalizeParams p) {
  const int lane = threadIdx.x & 31;
  const int n_heads_tot = p.k.n_heads + p.v.n_heads;
  const int64_t item = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  if (item < (int64_t)p.rows * n_heads_tot) {
    const int lrow = (int)(item / n_heads_tot);
    const int j = (int)(item % n_heads_tot);
    const int grow = p.row0 + lrow;
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
          for (int s = 0; s < p.n_ksplit; ++s)
            acc += (int)p.ws[((int64_t)s * p.ws_rows + lrow) * p.n_tot + n];
          val = __fmul_rn(__fmul_rn((float)acc, p.x_scale[grow]), lk_f16_to_f32(p.a_scale[n]));
        } else {
          for (int s = 0; s < p.n_ksplit; ++s)
            val += __uint_as_float(p.ws[((int64_t)s * p.ws_rows + lrow) * p.n_tot + n]);
        }
      }
      vals[q] = val;
    }
    const LkQRow qr = lk_quantize_row_warp(vals[0], vals[1], r, cv.kind, cv.group);
    const int64_t pos = (int64_t)p.seq_len[b] + t;
    const int cap = cv.capacity;
    // the host checked the capacity against its copy of seq_len; never write past it
    // even if the device copy disagrees
    if (pos < 0 || pos >= cap) goto done;
    const int tot_rb = is_k ? p.tot_rb_k : p.tot_rb_v;
    const int tot_ng = is_k ? p.tot_ng_k : p.tot_ng_v;
    if (cv.kind == 0) {
      int8_t* plane = static_cast<int8_t*>(cv.codes) + ((int64_t)b * tot_rb + p.pref_rb[j]) * cap;
      const int cs = lk_chunk_bytes(r);
      if (lane < r) plane[lk_code_offset(pos, lane, r, cs)] = (int8_t)qr.c0;
      if (lane + 32 < r) plane[lk_code_offset(pos, lane + 32, r, cs)] = (int8_t)qr.c1;
      if (lane == 0) static_cast<float*>(cv.scales)[((int64_t)b * cv.n_heads + hh) * cap + pos] = qr.s0;
    } else {
      const int rb = r / 2;
      uint8_t* plane = static_cast<uint8_t*>(cv.codes) + ((int64_t)b * tot_rb + p.pref_rb[j]) * cap;
      const int cs = lk_chunk_bytes(rb);
      const int n0 = __shfl_down_sync(0xffffffffu, qr.c0, 1);
      const int n1 = __shfl_down_sync(0xffffffffu, qr.c1, 1);
      if ((lane & 1) == 0) {
        if (lane < r)
          plane[lk_code_offset(pos, lane / 2, rb, cs)] = (uint8_t)((qr.c0 & 0xF) | ((n0 & 0xF) << 4));
        if (lane + 32 < r)
          plane[lk_code_offset(pos, (lane + 32) / 2, rb, cs)] = (uint8_t)((qr.c1 & 0xF) | ((n1 & 0xF) << 4));
      }
      const int g = min(cv.group, r), ng = (r + g - 1) / g;
      uint16_t* sp = static_cast<uint16_t*>(cv.scales) + ((int64_t)b * tot_ng + p.pref_ng[j]) * cap + pos * ng;
      if (lane < r && lane % g == 0) sp[lane / g] = lk_f32_to_f16_bits(qr.s0);
      if (lane + 32 < r && (lane + 32) % g == 0) sp[(lane + 32) / g] = lk_f32_to_f16_bits(qr.s1);
    }
  }
done:
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

int round_up(int x, int m) { return (x + m - 1) / m * m; }

int gemv_ksplit(int n_tot, int E, int ve, int num_sms) {
  const int col_blocks = (n_tot + kColsPerCta - 1) / kColsPerCta;
  const int sweep = 32 * ve;
  const int max_split = std::max(1, E / sweep);
  int s = (2 * num_sms + col_blocks - 1) / col_blocks;
  return std::max(1, std::min(s, max_split));
}

int x_ve(int xtype) { return xtype == lk::X_F32 ? 4 : (xtype == lk::X_BF16 ? 8 : 16); }
int x_size(int xtype) { return xtype == lk::X_F32 ? 4 : (xtype == lk::X_BF16 ? 2 : 1); }

constexpr int kPrefillRowChunk = 8192;

}  // namespace

LK_DEFINE_STATUS_ACCESSOR(lk_project_status_word)

namespace lk {

size_t project_workspace_bytes(int rows, int n_tot, int embed_dim, int xtype, int num_sms) {
  size_t body;
  if (rows <= kGemvMaxRows) {
    const int ks = gemv_ksplit(n_tot, embed_dim, x_ve(xtype), num_sms);
    body = (size_t)ks * rows * n_tot * 4;
  } else {
    body = (size_t)std::min(rows, kPrefillRowChunk) * n_tot * 4;
  }
  return 256 + body;
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
  f.ws = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(a.workspace) + 256);
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
    const int ve = x_ve(a.xtype);
    const int ks = gemv_ksplit(a.n_tot, a.embed_dim, ve, a.num_sms);
    int slice = (a.embed_dim + ks - 1) / ks;
    slice = round_up(slice, ve);
    const int nks = (a.embed_dim + slice - 1) / slice;
    const size_t smem = (size_t)kMT * slice * x_size(a.xtype);
    dim3 grid((a.n_tot + kColsPerCta - 1) / kColsPerCta, nks);
    if (a.xtype == X_F32) {
      e = cudaFuncSetAttribute(proj_gemv_kernel<X_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      proj_gemv_kernel<X_F32><<<grid, kGemvThreads, smem, stream>>>(a.x, a.A, rows, a.n_tot, a.embed_dim, slice, f.ws);
    } else if (a.xtype == X_BF16) {
      e = cudaFuncSetAttribute(proj_gemv_kernel<X_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      proj_gemv_kernel<X_BF16><<<grid, kGemvThreads, smem, stream>>>(a.x, a.A, rows, a.n_tot, a.embed_dim, slice, f.ws);
    } else {
      e = cudaFuncSetAttribute(proj_gemv_kernel<X_I8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      proj_gemv_kernel<X_I8><<<grid, kGemvThreads, smem, stream>>>(a.x, a.A, rows, a.n_tot, a.embed_dim, slice, f.ws);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    f.n_ksplit = nks;
    f.ws_rows = rows;
    f.row0 = 0;
    f.rows = rows;
    f.do_update = 1;
    const int64_t items = (int64_t)rows * heads_tot;
    proj_finalize_kernel<<<(unsigned)((items + 3) / 4), 128, 0, stream>>>(f);
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
