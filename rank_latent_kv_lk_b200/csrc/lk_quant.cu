// Stand-alone quantisers and the row-wise activation kernels:
//  - latent quantiser (int8 absmax / int4 grouped absmax, stated packing)
//  - per-row int8 quantisation of activations, optionally after RMSNorm or
//    after SwiGLU (LASER page §4 fuses SwiGLU and quantisation into the FFN).
#include "lk_common.cuh"
#include "lk_internal.h"
#include "lk_quant.cuh"

namespace {

// One warp per row of r <= 64 values; codes in plain row layout.
__global__ void quantize_latent_kernel(const float* __restrict__ v, int m, int r, int kind,
                                       int group, uint8_t* __restrict__ codes,
                                       uint8_t* __restrict__ scales) {
  const int warps = blockDim.x / 32;
  const int row = blockIdx.x * warps + (threadIdx.x >> 5);
  if (row >= m) return;
  const int lane = threadIdx.x & 31;
  const float* vr = v + (int64_t)row * r;
  const float v0 = lane < r ? vr[lane] : 0.0f;
  const float v1 = lane + 32 < r ? vr[lane + 32] : 0.0f;
  const LkQRow q = lk_quantize_row_warp(v0, v1, r, kind, group);
  if (kind == 0) {
    int8_t* cr = reinterpret_cast<int8_t*>(codes) + (int64_t)row * r;
    if (lane < r) cr[lane] = (int8_t)q.c0;
    if (lane + 32 < r) cr[lane + 32] = (int8_t)q.c1;
    if (lane == 0) reinterpret_cast<float*>(scales)[row] = q.s0;
  } else {
    const int g = min(group, r), ng = (r + g - 1) / g;
    uint8_t* cr = codes + (int64_t)row * (r / 2);
    const int n0 = __shfl_down_sync(0xffffffffu, q.c0, 1);
    const int n1 = __shfl_down_sync(0xffffffffu, q.c1, 1);
    if ((lane & 1) == 0) {
      if (lane < r) cr[lane / 2] = (uint8_t)((q.c0 & 0xF) | ((n0 & 0xF) << 4));
      if (lane + 32 < r) cr[(lane + 32) / 2] = (uint8_t)((q.c1 & 0xF) | ((n1 & 0xF) << 4));
    }
    uint16_t* sr = reinterpret_cast<uint16_t*>(scales) + (int64_t)row * ng;
    if (lane < r && lane % g == 0) sr[lane / g] = lk_f32_to_f16_bits(q.s0);
    if (lane + 32 < r && (lane + 32) % g == 0) sr[(lane + 32) / g] = lk_f32_to_f16_bits(q.s1);
  }
}

constexpr int kRowThreads = 256;

LK_DEVICE float block_reduce(float v, float* scratch, bool is_max) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = is_max ? lk_warp_max(v) : lk_warp_sum(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  float r = is_max ? 0.0f : 0.0f;
  if (threadIdx.x < 32) {
    r = threadIdx.x < kRowThreads / 32 ? scratch[threadIdx.x] : 0.0f;
    r = is_max ? lk_warp_max(r) : lk_warp_sum(r);
    if (threadIdx.x == 0) scratch[32] = r;
  }
  __syncthreads();
  return scratch[32];
}

// One CTA per row: y = f(x) kept in shared memory, then int8 absmax codes.
// mode 0: y = x; 1: y = x / sqrt(mean(x^2) + eps); 2: y = silu(x) * x2;
// 3: mode 1, then the normalised Walsh-Hadamard transform of the row.
template <bool BF16>
__global__ void __launch_bounds__(kRowThreads) rowquant_kernel(int mode, const void* __restrict__ x,
                                                              const void* __restrict__ x2, int k, float eps,
                                                              int8_t* __restrict__ x_q,
                                                              float* __restrict__ x_scale) {
  extern __shared__ float ys[];
  __shared__ float scratch[33];
  const int64_t row = blockIdx.x;
  using T = typename std::conditional<BF16, uint16_t, float>::type;
  const T* xr = reinterpret_cast<const T*>(x) + row * k;
  const T* x2r = reinterpret_cast<const T*>(x2) + row * k;
  float ss = 0.0f;
  auto f = [&](float a, float b) { return mode == 2 ? __fmul_rn(__fdiv_rn(a, 1.0f + expf(-a)), b) : a; };
  constexpr int VE = BF16 ? 8 : 4;  // elements per 16-byte vector
  const bool vec = (k % VE) == 0 && ((reinterpret_cast<uintptr_t>(xr) | reinterpret_cast<uintptr_t>(x2r)) & 15) == 0;
  if (vec) {
    // 16-byte loads, several in flight per thread
    const int nv = k / VE;
#pragma unroll 4
    for (int v = threadIdx.x; v < nv; v += kRowThreads) {
      const uint4 xv = reinterpret_cast<const uint4*>(xr)[v];
      uint4 yv = make_uint4(0, 0, 0, 0);
      if (mode == 2) yv = reinterpret_cast<const uint4*>(x2r)[v];
      float xa[VE], xb[VE];
      if constexpr (BF16) {
        const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w}, u[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          xa[2 * j] = lk_bf16lo(w[j]); xa[2 * j + 1] = lk_bf16hi(w[j]);
          xb[2 * j] = lk_bf16lo(u[j]); xb[2 * j + 1] = lk_bf16hi(u[j]);
        }
      } else {
        xa[0] = __uint_as_float(xv.x); xa[1] = __uint_as_float(xv.y);
        xa[2] = __uint_as_float(xv.z); xa[3] = __uint_as_float(xv.w);
        xb[0] = __uint_as_float(yv.x); xb[1] = __uint_as_float(yv.y);
        xb[2] = __uint_as_float(yv.z); xb[3] = __uint_as_float(yv.w);
      }
#pragma unroll
      for (int j = 0; j < VE; ++j) {
        const float a = f(xa[j], xb[j]);
        ys[v * VE + j] = a;
        ss = fmaf(a, a, ss);
      }
    }
  } else {
    for (int i = threadIdx.x; i < k; i += kRowThreads) {
      const float a = f(lk_load_f<T>(xr, i), mode == 2 ? lk_load_f<T>(x2r, i) : 0.0f);
      ys[i] = a;
      ss = fmaf(a, a, ss);
    }
  }
  if (mode == 1 || mode == 3) {
    const float tot = block_reduce(ss, scratch, false);
    const float denom = sqrtf(__fdiv_rn(tot, (float)k) + eps);
    for (int i = threadIdx.x; i < k; i += kRowThreads) ys[i] = __fdiv_rn(ys[i], denom);
  }
  if (mode == 3) {
    // S1 (WSVD page §2C): the normalised Walsh-Hadamard transform of the
    // row (k a power of two), butterflies in shared memory
    for (int h = 1; h < k; h <<= 1) {
      __syncthreads();
      for (int i = threadIdx.x; i < k / 2; i += kRowThreads) {
        const int i0 = (i / h) * 2 * h + (i % h), i1 = i0 + h;
        const float a = ys[i0], b = ys[i1];
        ys[i0] = __fadd_rn(a, b);
        ys[i1] = __fsub_rn(a, b);
      }
    }
    __syncthreads();
    const float c = __double2float_rn(1.0 / sqrt((double)k));  // fl32(1 / sqrt(k))
    for (int i = threadIdx.x; i < k; i += kRowThreads) ys[i] = __fmul_rn(ys[i], c);
  }
  __syncthreads();
  float a = 0.0f;
  for (int i = threadIdx.x; i < k; i += kRowThreads) a = fmaxf(a, fabsf(ys[i]));
  a = block_reduce(a, scratch, true);
  const float s = lk_q8_scale(a);
  for (int i = threadIdx.x; i < k; i += kRowThreads) x_q[row * k + i] = (int8_t)lk_q8_code(ys[i], s);
  if (threadIdx.x == 0) x_scale[row] = s;
}

}  // namespace

LK_DEFINE_STATUS_ACCESSOR(lk_quant_status_word)

namespace lk {

cudaError_t launch_quantize_latent(const float* v, int m, int r, int kind, int group, void* codes,
                                   void* scales, cudaStream_t stream) {
  if (m == 0) return cudaSuccess;
  const int warps = 4;
  count_launch();
  quantize_latent_kernel<<<(m + warps - 1) / warps, warps * 32, 0, stream>>>(
      v, m, r, kind, group, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales));
  return cudaGetLastError();
}

cudaError_t launch_rowquant(int mode, const void* x, const void* x2, int x_bf16, int m, int k,
                            float eps, int8_t* x_q, float* x_scale, cudaStream_t stream) {
  if (m == 0) return cudaSuccess;
  const size_t smem = (size_t)k * sizeof(float);
  cudaError_t e;
  if (x_bf16) {
    e = cudaFuncSetAttribute(rowquant_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    rowquant_kernel<true><<<m, kRowThreads, smem, stream>>>(mode, x, x2, k, eps, x_q, x_scale);
  } else {
    e = cudaFuncSetAttribute(rowquant_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    rowquant_kernel<false><<<m, kRowThreads, smem, stream>>>(mode, x, x2, k, eps, x_q, x_scale);
  }
  return cudaGetLastError();
}

}  // namespace lk
