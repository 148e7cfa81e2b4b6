// LASER hybrid dense + low-rank linear, W8A8 (LASER page, technical summary
// §3: selected input channels go through the SVD factors, the remaining
// channels stay dense, and both branches are round-to-nearest quantised).
//
//   acc_D = x_q[:, D] W_D^T                       exact int32
//   t     = fl32(fl32(fl32(x_q[:, not D] U^T) * s_x) * s_U)
//   t_q, s_t = per-token int8 absmax of t         (bit-exact rule)
//   acc_V = t_q V^T                               exact int32
//   y     = acc_D * s_x * s_D + acc_V * s_t * s_V (+ residual)
#include "lk_common.cuh"
#include "lk_internal.h"

namespace {

// xg[m][i] = x[m][idx[i]] for i < n; rows padded to `ld` bytes (zeros).
__global__ void gather_cols_kernel(const int8_t* __restrict__ x, int k_in, const int32_t* __restrict__ idx,
                                   int n, int ld, int8_t* __restrict__ out) {
  const int m = blockIdx.y;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < ld; i += gridDim.x * blockDim.x)
    out[(int64_t)m * ld + i] = i < n ? x[(int64_t)m * k_in + idx[i]] : (int8_t)0;
}

// One CTA per token row: t = fl32(fl32(acc * s_x) * s_U), then int8 absmax.
__global__ void __launch_bounds__(256) requant_kernel(const int32_t* __restrict__ acc, int rank,
                                                     const float* __restrict__ x_scale,
                                                     const uint16_t* __restrict__ s_U, int8_t* __restrict__ t_q,
                                                     int ld_tq, float* __restrict__ s_t) {
  __shared__ float red[8];
  __shared__ float s_shared;
  const int64_t m = blockIdx.x;
  const float sx = x_scale[m];
  float a = 0.0f;
  for (int k = threadIdx.x; k < rank; k += blockDim.x) {
    const float t = __fmul_rn(__fmul_rn((float)acc[m * rank + k], sx), lk_f16_to_f32(s_U[k]));
    a = fmaxf(a, fabsf(t));
  }
  a = lk_warp_max(a);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    float mx = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, red[w]);
    s_shared = lk_q8_scale(mx);
    s_t[m] = s_shared;
  }
  __syncthreads();
  const float s = s_shared;
  for (int k = threadIdx.x; k < ld_tq; k += blockDim.x) {
    int c = 0;
    if (k < rank) {
      const float t = __fmul_rn(__fmul_rn((float)acc[m * rank + k], sx), lk_f16_to_f32(s_U[k]));
      c = lk_q8_code(t, s);
    }
    t_q[m * ld_tq + k] = (int8_t)c;
  }
}

// One CTA row per token row (blockIdx.y), columns strided over x.
__global__ void lowrank_epilogue_kernel(const int32_t* __restrict__ accD, const int32_t* __restrict__ accV,
                                        const float* __restrict__ x_scale, const float* __restrict__ s_t,
                                        const uint16_t* __restrict__ s_D, const uint16_t* __restrict__ s_V,
                                        const uint16_t* __restrict__ residual, int m, int n, void* y,
                                        int y_bf16) {
  const int64_t row = blockIdx.y;
  const float sx = accD ? x_scale[row] : 0.0f;
  const float st = accV ? s_t[row] : 0.0f;
  for (int col = blockIdx.x * blockDim.x + threadIdx.x; col < n; col += gridDim.x * blockDim.x) {
    const int64_t i = row * n + col;
    float out = 0.0f;
    if (accD) out = __fmul_rn(__fmul_rn((float)accD[i], sx), lk_f16_to_f32(s_D[col]));
    if (accV) out += __fmul_rn(__fmul_rn((float)accV[i], st), lk_f16_to_f32(s_V[col]));
    if (residual) out += lk_bf16_to_f32(residual[i]);
    if (y_bf16) static_cast<uint16_t*>(y)[i] = lk_f32_to_bf16(out);
    else static_cast<float*>(y)[i] = out;
  }
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }
int pad16(int x) { return (x + 15) / 16 * 16; }

struct WsLayout {
  size_t xg, xd, accU, tq, st, accD, accV, total;
};

WsLayout ws_layout(int k_in, int n_out, int rank, int n_dense, int m) {
  const int n_lr = k_in - n_dense;
  WsLayout L{};
  size_t off = 0;
  L.xg = off; off += align256((size_t)m * pad16(n_lr));
  L.xd = off; off += align256((size_t)m * pad16(n_dense));
  L.accU = off; off += align256((size_t)m * rank * 4);
  L.tq = off; off += align256((size_t)m * pad16(rank));
  L.st = off; off += align256((size_t)m * 4);
  L.accD = off; off += align256((size_t)m * n_out * 4);
  L.accV = off; off += align256((size_t)m * n_out * 4);
  L.total = off;
  return L;
}

}  // namespace

LK_DEFINE_STATUS_ACCESSOR(lk_lowrank_status_word)

namespace lk {

size_t lowrank_workspace_bytes(int k_in, int n_out, int rank, int n_dense, int m) {
  return ws_layout(k_in, n_out, rank, n_dense, m).total;
}

cudaError_t launch_lowrank_linear(const LowrankLaunch& a, cudaStream_t stream) {
  if (a.m == 0) return cudaSuccess;
  const WsLayout L = ws_layout(a.k_in, a.n_out, a.rank, a.n_dense, a.m);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  const int n_lr = a.k_in - a.n_dense;
  cudaError_t e;
  int32_t* accD = nullptr;
  int32_t* accV = nullptr;
  float* s_t = a.t_scale_out ? a.t_scale_out : reinterpret_cast<float*>(ws + L.st);
  // rank is a multiple of 16, so the requantised latent rows are already aligned
  int8_t* t_q = a.t_q_out ? a.t_q_out : reinterpret_cast<int8_t*>(ws + L.tq);
  const int ld_tq = a.rank;
  if (a.n_dense > 0) {
    int8_t* xd = reinterpret_cast<int8_t*>(ws + L.xd);
    const int ld = pad16(a.n_dense);
    gather_cols_kernel<<<dim3((ld + 255) / 256, a.m), 256, 0, stream>>>(a.x_q, a.k_in, a.dense_idx, a.n_dense, ld, xd);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    accD = reinterpret_cast<int32_t*>(ws + L.accD);
    e = launch_gemm_i8(xd, ld, a.W_D, a.n_dense, accD, a.n_out, a.m, a.n_out, a.n_dense, stream);
    if (e != cudaSuccess) return e;
  }
  if (a.rank > 0) {
    int8_t* xg = reinterpret_cast<int8_t*>(ws + L.xg);
    const int ld = pad16(n_lr);
    gather_cols_kernel<<<dim3((ld + 255) / 256, a.m), 256, 0, stream>>>(a.x_q, a.k_in, a.lr_idx, n_lr, ld, xg);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    int32_t* accU = reinterpret_cast<int32_t*>(ws + L.accU);
    e = launch_gemm_i8(xg, ld, a.U, n_lr, accU, a.rank, a.m, a.rank, n_lr, stream);
    if (e != cudaSuccess) return e;
    requant_kernel<<<a.m, 256, 0, stream>>>(accU, a.rank, a.x_scale, a.s_U, t_q, ld_tq, s_t);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    accV = reinterpret_cast<int32_t*>(ws + L.accV);
    e = launch_gemm_i8(t_q, ld_tq, a.V, a.rank, accV, a.n_out, a.m, a.n_out, a.rank, stream);
    if (e != cudaSuccess) return e;
  }
  const dim3 egrid((unsigned)std::min((a.n_out + 255) / 256, 64), (unsigned)a.m);
  lowrank_epilogue_kernel<<<egrid, 256, 0, stream>>>(accD, accV, a.x_scale, s_t, a.s_D, a.s_V, a.residual, a.m,
                                                     a.n_out, a.y, a.y_bf16);
  count_launch();
  return cudaGetLastError();
}

}  // namespace lk
