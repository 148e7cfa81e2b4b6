// LASER hybrid FFN input side, split on OUTPUT (hidden) channels, W8A8
// (LASER page, technical summary §3: the selected hidden channels keep dense
// weights, the rest go through the SVD factors; §4: the input projections,
// the latent activation and the SwiGLU are fused).  For token rows x_q
// (int8, per-token scale s_x) and hidden channel j:
//   j dense:     g_j = fl32(fl32(acc * s_x) * s_D[j]),  acc = x_q . W_D[j]   (exact int32)
//   j low-rank:  g_j = fl32(fl32(acc * s_t) * s_V[j]),  acc = t_q . V[j]
//                with t = fl32(fl32(fl32(x_q U^T) * s_x) * s_U) requantised per token (t_q, s_t)
//   u likewise with the up weights (the same channel split), out_j = silu(g_j) * u_j (fp32).
// Launches: the two latent products x_q U^T (tcgen05 int8 GEMM), one
// requantisation of both latents, then ONE launch for gate + up + SwiGLU:
// a CTA owns 16 hidden channels of one branch (dense or low-rank) for both
// gate and up, its 8 warps split the contraction, and each 128-byte k block
// of a lane (two weight rows per projection, its token rows) feeds four
// m16n8k32 int8 products whose k slots are taken from the lane's registers
// (the same permuted k order for weights and tokens, so the int32 sums are
// the plain dot products, exactly).  The warps' int32 sums meet in shared
// memory; the epilogue scales, applies SwiGLU and writes each channel at its
// place in the hidden vector.
#include "lk_common.cuh"
#include "lk_internal.h"

namespace {

constexpr int kFW = 8;  // warps per CTA

struct FfnParams {
  const int8_t* x_q;
  const float* x_scale;
  const int8_t* tq_g;
  const int8_t* tq_u;
  const float* st_g;
  const float* st_u;
  const int8_t* WDg;
  const int8_t* WDu;
  const uint16_t* sDg;
  const uint16_t* sDu;
  const int8_t* Vg;
  const int8_t* Vu;
  const uint16_t* sVg;
  const uint16_t* sVu;
  const int32_t* dense_out;
  const int32_t* lr_out;
  float* out;
  int m, k_in, n_out, n_dense, rank, dense_tiles;
};

LK_DEVICE uint32_t word8(const uint4 (&v)[2], int w) {
  const uint4& q = v[w >> 2];
  return (w & 3) == 0 ? q.x : (w & 3) == 1 ? q.y : (w & 3) == 2 ? q.z : q.w;
}

LK_DEVICE void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                            uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

LK_DEVICE uint4 ldg16(const int8_t* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

template <int NT>  // n8 tiles of token rows per CTA: 8 NT rows (grid.y covers the rest)
__global__ void __launch_bounds__(kFW * 32) ffn_gate_up_kernel(const __grid_constant__ FfnParams p) {
  __shared__ int red[2][kFW][16][8 * NT + 1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int tile = blockIdx.x;
  const int m0 = blockIdx.y * 8 * NT;
  const bool dense = tile < p.dense_tiles;
  const int r0 = (dense ? tile : tile - p.dense_tiles) * 16;  // first row of the tile within its branch
  const int nrows = dense ? p.n_dense : p.n_out - p.n_dense;
  const int K = dense ? p.k_in : p.rank;
  const int8_t* Ag = dense ? p.WDg : p.Vg;
  const int8_t* Au = dense ? p.WDu : p.Vu;
  const int8_t* Xg = dense ? p.x_q : p.tq_g;
  const int8_t* Xu = dense ? p.x_q : p.tq_u;
  // rows past the branch (last tile) repeat its last row: computed, never stored
  const int64_t ra = (int64_t)min(r0 + gid, nrows - 1) * K, rb = (int64_t)min(r0 + gid + 8, nrows - 1) * K;
  int cg[NT][4], cu[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) cg[t][e] = cu[t][e] = 0;
  const int nb = (K + 127) / 128;
  const int kb0 = warp * nb / kFW, kb1 = (warp + 1) * nb / kFW;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (int kb = kb0; kb < kb1; ++kb) {
    uint4 wag[2], wbg[2], wau[2], wbu[2], xg[NT][2], xu[NT][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int k = kb * 128 + 32 * tig + 16 * h;
      const bool ok = k < K;  // K is a multiple of 16
      wag[h] = ok ? ldg16(Ag + ra + k) : z;
      wbg[h] = ok ? ldg16(Ag + rb + k) : z;
      wau[h] = ok ? ldg16(Au + ra + k) : z;
      wbu[h] = ok ? ldg16(Au + rb + k) : z;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const int m = m0 + 8 * t + gid;
        const bool okx = ok && m < p.m;
        xg[t][h] = okx ? ldg16(Xg + (int64_t)m * K + k) : z;
        xu[t][h] = dense ? xg[t][h] : (okx ? ldg16(Xu + (int64_t)m * K + k) : z);
      }
    }
    // product s takes k = 32 tig + 8 s + {0..3} for the slots 4 tig .. 4 tig + 3
    // and 32 tig + 8 s + {4..7} for 16 + 4 tig .., for weights and tokens alike
#pragma unroll
    for (int s = 0; s < 4; ++s) {
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        mma_s8_16832(cg[t], word8(wag, 2 * s), word8(wbg, 2 * s), word8(wag, 2 * s + 1), word8(wbg, 2 * s + 1),
                     word8(xg[t], 2 * s), word8(xg[t], 2 * s + 1));
        mma_s8_16832(cu[t], word8(wau, 2 * s), word8(wbu, 2 * s), word8(wau, 2 * s + 1), word8(wbu, 2 * s + 1),
                     word8(xu[t], 2 * s), word8(xu[t], 2 * s + 1));
      }
    }
  }
  // D fragment: (channel gid, tokens 2 tig, 2 tig + 1) and channel gid + 8
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    red[0][warp][gid][8 * t + 2 * tig] = cg[t][0];
    red[0][warp][gid][8 * t + 2 * tig + 1] = cg[t][1];
    red[0][warp][gid + 8][8 * t + 2 * tig] = cg[t][2];
    red[0][warp][gid + 8][8 * t + 2 * tig + 1] = cg[t][3];
    red[1][warp][gid][8 * t + 2 * tig] = cu[t][0];
    red[1][warp][gid][8 * t + 2 * tig + 1] = cu[t][1];
    red[1][warp][gid + 8][8 * t + 2 * tig] = cu[t][2];
    red[1][warp][gid + 8][8 * t + 2 * tig + 1] = cu[t][3];
  }
  __syncthreads();
  const int mt = min(8 * NT, p.m - m0);
  for (int idx = threadIdx.x; idx < 16 * mt; idx += kFW * 32) {
    const int ch = idx / mt, tk = idx - ch * mt;
    const int r = r0 + ch;
    if (r >= nrows) continue;
    int ag = 0, au = 0;  // exact int32 sums in a fixed order
#pragma unroll
    for (int w = 0; w < kFW; ++w) {
      ag += red[0][w][ch][tk];
      au += red[1][w][ch][tk];
    }
    const int m = m0 + tk;
    float g, u;
    int j;
    if (dense) {
      const float sx = p.x_scale[m];
      g = __fmul_rn(__fmul_rn((float)ag, sx), lk_f16_to_f32(p.sDg[r]));
      u = __fmul_rn(__fmul_rn((float)au, sx), lk_f16_to_f32(p.sDu[r]));
      j = p.dense_out[r];
    } else {
      g = __fmul_rn(__fmul_rn((float)ag, p.st_g[m]), lk_f16_to_f32(p.sVg[r]));
      u = __fmul_rn(__fmul_rn((float)au, p.st_u[m]), lk_f16_to_f32(p.sVu[r]));
      j = p.lr_out[r];
    }
    p.out[(int64_t)m * p.n_out + j] = g / (1.0f + expf(-g)) * u;
  }
}

// t = fl32(fl32(acc * s_x) * s_U) of row blockIdx.x, latent blockIdx.y (0: gate,
// 1: up), requantised with the int8 absmax rule.
__global__ void __launch_bounds__(256) requant2_kernel(const int32_t* __restrict__ acc_g,
                                                      const int32_t* __restrict__ acc_u, int rank,
                                                      const float* __restrict__ x_scale,
                                                      const uint16_t* __restrict__ sUg,
                                                      const uint16_t* __restrict__ sUu, int8_t* __restrict__ tq_g,
                                                      int8_t* __restrict__ tq_u, float* __restrict__ st_g,
                                                      float* __restrict__ st_u) {
  __shared__ float red[8];
  __shared__ float s_shared;
  const int64_t m = blockIdx.x;
  const bool up = blockIdx.y == 1;
  const int32_t* acc = (up ? acc_u : acc_g) + m * rank;
  const uint16_t* sU = up ? sUu : sUg;
  const float sx = x_scale[m];
  float a = 0.0f;
  for (int k = threadIdx.x; k < rank; k += blockDim.x)
    a = fmaxf(a, fabsf(__fmul_rn(__fmul_rn((float)acc[k], sx), lk_f16_to_f32(sU[k]))));
  a = lk_warp_max(a);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    float mx = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, red[w]);
    s_shared = lk_q8_scale(mx);
    (up ? st_u : st_g)[m] = s_shared;
  }
  __syncthreads();
  const float s = s_shared;
  int8_t* tq = (up ? tq_u : tq_g) + m * rank;
  for (int k = threadIdx.x; k < rank; k += blockDim.x)
    tq[k] = (int8_t)lk_q8_code(__fmul_rn(__fmul_rn((float)acc[k], sx), lk_f16_to_f32(sU[k])), s);
}

size_t al256(size_t x) { return (x + 255) / 256 * 256; }

struct FfnWs {
  size_t acc_g, acc_u, tq_g, tq_u, st_g, st_u, total;
};

FfnWs ffn_ws(int m, int rank) {
  FfnWs L{};
  size_t off = 0;
  L.acc_g = off; off += al256((size_t)m * rank * 4);
  L.acc_u = off; off += al256((size_t)m * rank * 4);
  L.tq_g = off; off += al256((size_t)m * rank);
  L.tq_u = off; off += al256((size_t)m * rank);
  L.st_g = off; off += al256((size_t)m * 4);
  L.st_u = off; off += al256((size_t)m * 4);
  L.total = std::max<size_t>(off, 256);
  return L;
}

}  // namespace

namespace lk {

size_t ffn_workspace_bytes(int m, int rank) { return ffn_ws(m, rank).total; }

cudaError_t launch_ffn_gate_up(const FfnLaunch& a, cudaStream_t stream) {
  if (a.m == 0) return cudaSuccess;
  const FfnWs L = ffn_ws(a.m, a.rank);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  FfnParams p{};
  p.x_q = a.x_q;
  p.x_scale = a.x_scale;
  p.WDg = a.gate.W_D;
  p.WDu = a.up.W_D;
  p.sDg = a.gate.s_D;
  p.sDu = a.up.s_D;
  p.Vg = a.gate.V;
  p.Vu = a.up.V;
  p.sVg = a.gate.s_V;
  p.sVu = a.up.s_V;
  p.dense_out = a.dense_out;
  p.lr_out = a.lr_out;
  p.out = a.out;
  p.m = a.m;
  p.k_in = a.k_in;
  p.n_out = a.n_out;
  p.n_dense = a.n_dense;
  p.rank = a.rank;
  p.dense_tiles = (a.n_dense + 15) / 16;
  cudaError_t e;
  if (a.n_dense < a.n_out) {  // the low-rank latents of gate and up
    int32_t* acc_g = reinterpret_cast<int32_t*>(ws + L.acc_g);
    int32_t* acc_u = reinterpret_cast<int32_t*>(ws + L.acc_u);
    e = launch_gemm_i8(a.x_q, a.k_in, a.gate.U, a.k_in, acc_g, a.rank, a.m, a.rank, a.k_in, stream);
    if (e != cudaSuccess) return e;
    e = launch_gemm_i8(a.x_q, a.k_in, a.up.U, a.k_in, acc_u, a.rank, a.m, a.rank, a.k_in, stream);
    if (e != cudaSuccess) return e;
    p.tq_g = reinterpret_cast<int8_t*>(ws + L.tq_g);
    p.tq_u = reinterpret_cast<int8_t*>(ws + L.tq_u);
    p.st_g = reinterpret_cast<float*>(ws + L.st_g);
    p.st_u = reinterpret_cast<float*>(ws + L.st_u);
    requant2_kernel<<<dim3((unsigned)a.m, 2), 256, 0, stream>>>(acc_g, acc_u, a.rank, a.x_scale, a.gate.s_U,
                                                               a.up.s_U, const_cast<int8_t*>(p.tq_g),
                                                               const_cast<int8_t*>(p.tq_u),
                                                               const_cast<float*>(p.st_g), const_cast<float*>(p.st_u));
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const int tiles = p.dense_tiles + (a.n_out - a.n_dense + 15) / 16;
  const int nt = a.m <= 8 ? 1 : (a.m <= 16 ? 2 : 4);
  const dim3 grid((unsigned)tiles, (unsigned)((a.m + 8 * nt - 1) / (8 * nt)));
  if (nt == 1) ffn_gate_up_kernel<1><<<grid, kFW * 32, 0, stream>>>(p);
  else if (nt == 2) ffn_gate_up_kernel<2><<<grid, kFW * 32, 0, stream>>>(p);
  else ffn_gate_up_kernel<4><<<grid, kFW * 32, 0, stream>>>(p);
  count_launch();
  return cudaGetLastError();
}

}  // namespace lk
