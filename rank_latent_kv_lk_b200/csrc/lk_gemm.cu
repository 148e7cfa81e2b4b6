// C[m][n] = sum_k A[m][k] * B[n][k] with both operands K-contiguous.  fp32
// operands (the fp32 prefill projection): a tiled CUDA-core GEMM with fp32
// accumulation.  int8 operands (the W8A8 linears and the int8 prefill
// projection): the tcgen05 kernels of lk_gemm_tc.cu, exact int32.
#include "lk_common.cuh"
#include "lk_internal.h"

namespace {

constexpr int kBM = 64, kBN = 64;
constexpr int kThreads = 256;  // 16 x 16 threads, 4 x 4 outputs each

// ---- fp32 / bf16 operands, fp32 accumulate: K tile of 16 elements
template <bool BF16>
__global__ void __launch_bounds__(kThreads) gemm_f_kernel(const void* __restrict__ Av, int lda,
                                                         const void* __restrict__ Bv, int ldb,
                                                         float* __restrict__ C, int ldc, int M, int N, int K) {
  __shared__ float As[16][kBM + 4];
  __shared__ float Bs[16][kBN + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * kBN;
  const int lrow = tid >> 2, lq = tid & 3;  // loader: row 0..63, 4 elements at k = lq*4
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    const int kk = k0 + lq * 4;
    float a4[4] = {0, 0, 0, 0}, b4[4] = {0, 0, 0, 0};
    if (BF16) {
      const uint16_t* A = static_cast<const uint16_t*>(Av);
      const uint16_t* B = static_cast<const uint16_t*>(Bv);
      if (m0 + lrow < M && kk < K) {
        const uint2 v = *reinterpret_cast<const uint2*>(A + (int64_t)(m0 + lrow) * lda + kk);
        a4[0] = lk_bf16lo(v.x); a4[1] = lk_bf16hi(v.x); a4[2] = lk_bf16lo(v.y); a4[3] = lk_bf16hi(v.y);
      }
      if (n0 + lrow < N && kk < K) {
        const uint2 v = *reinterpret_cast<const uint2*>(B + (int64_t)(n0 + lrow) * ldb + kk);
        b4[0] = lk_bf16lo(v.x); b4[1] = lk_bf16hi(v.x); b4[2] = lk_bf16lo(v.y); b4[3] = lk_bf16hi(v.y);
      }
    } else {
      const float* A = static_cast<const float*>(Av);
      const float* B = static_cast<const float*>(Bv);
      if (m0 + lrow < M && kk < K) {
        const float4 v = *reinterpret_cast<const float4*>(A + (int64_t)(m0 + lrow) * lda + kk);
        a4[0] = v.x; a4[1] = v.y; a4[2] = v.z; a4[3] = v.w;
      }
      if (n0 + lrow < N && kk < K) {
        const float4 v = *reinterpret_cast<const float4*>(B + (int64_t)(n0 + lrow) * ldb + kk);
        b4[0] = v.x; b4[1] = v.y; b4[2] = v.z; b4[3] = v.w;
      }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      As[lq * 4 + i][lrow] = a4[i];
      Bs[lq * 4 + i][lrow] = b4[i];
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < N) C[(int64_t)m * ldc + n] = acc[i][j];
    }
  }
}

}  // namespace

namespace lk {

// int8 products run on the tensor cores (lk_gemm_tc.cu); they need 16-byte
// aligned operands with lda, ldb multiples of 16.
cudaError_t launch_gemm_i8(const int8_t* A, int lda, const int8_t* B, int ldb, int32_t* C, int ldc,
                           int M, int N, int K, cudaStream_t stream) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (!gemm_i8_tc_supported(A, lda, B, ldb, K)) return cudaErrorInvalidValue;
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      sms = 148;
  }
  return launch_gemm_i8_tc(A, lda, B, ldb, C, ldc, M, N, K, sms, stream);
}

// Requires K % 4 == 0 (fp32) / K % 4 == 0 (bf16) with 16 / 8-byte aligned rows.
cudaError_t launch_gemm_f(const void* A, int lda, const void* B, int ldb, float* C, int ldc, int M,
                          int N, int K, bool bf16, cudaStream_t stream) {
  if (M == 0 || N == 0) return cudaSuccess;
  dim3 grid((N + kBN - 1) / kBN, (M + kBM - 1) / kBM);
  if (bf16) gemm_f_kernel<true><<<grid, kThreads, 0, stream>>>(A, lda, B, ldb, C, ldc, M, N, K);
  else gemm_f_kernel<false><<<grid, kThreads, 0, stream>>>(A, lda, B, ldb, C, ldc, M, N, K);
  count_launch();
  return cudaGetLastError();
}

}  // namespace lk
