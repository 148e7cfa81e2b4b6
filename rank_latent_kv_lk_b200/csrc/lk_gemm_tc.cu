// Dense bf16 GEMM on the fifth-generation tensor cores (tcgen05, sm_100a):
//   C[m][n] = sum_k A[m][k] * B[n][k]      A [M, K], B [N, K] bf16 (K contiguous), C fp32
// Used for the prefill latent projection v = x A^T (WSVD page, technical
// summary §2A: the latent of every context token; LASER page §4: latent
// generation fused with the projection), where the work is a dense
// contraction.
//
// One CTA per 128 x 128 tile of C, K in blocks of 64 (128 bytes of bf16 per
// row, the width of the 128-byte swizzle):
//   warp 0, one thread : TMA tensor loads of the A and B tiles into a
//                        4-stage shared-memory ring (no multicast);
//   warp 1             : allocates 128 TMEM columns; one thread issues
//                        tcgen05.mma (M=128, N=128, K=16) x 4 per block with
//                        the fp32 accumulator in TMEM and releases each ring
//                        slot with tcgen05.commit;
//   warps 2..5         : epilogue, tcgen05.ld of the accumulator (each warp
//                        reads its 32-lane quarter of TMEM) and fp32 stores.
// Every mbarrier wait is bounded; an expired wait sets the library status
// word, and the CTA still drains its copies and frees its TMEM.
#include <cuda.h>

#include "lk_common.cuh"
#include "lk_internal.h"

namespace {

constexpr int kBM = 128, kBN = 128, kBK = 64;
constexpr int kStages = 4;    // int8 kernel ring depth
// bf16 kernel: 3 stages (≈100 KB) so that two CTAs share an SM and one's
// epilogue (TMEM -> global) overlaps the other's MMAs
constexpr int kStagesBf = 3;
constexpr int kTileBytes = kBM * kBK * 2;  // 16 KB; the B tile has the same size (kBN == kBM)
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 128;  // fp32 accumulator: 128 lanes x 128 columns
constexpr int kSmemBytes = 2 * kStagesBf * kTileBytes + 1024 /* barriers */ + 1024 /* alignment */;

// Shared-memory matrix descriptor of a K-major tile with the 128-byte swizzle
// (rows of 128 bytes, 8-row groups 1024 bytes apart): start address >> 4,
// leading byte offset 16 B (unused by this layout), stride byte offset
// 1024 B, descriptor version 1, layout type 2 (128-byte swizzle).
LK_DEVICE uint64_t sw128_desc(uint32_t smem_addr) {
  return (uint64_t)((smem_addr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: fp32 accumulator, bf16 A and B, both K-major,
// N = 128, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                            ((uint32_t)(kBM >> 4) << 24);

LK_DEVICE void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          lk_smem_addr(dst)),
      "l"(map), "r"(lk_smem_addr(bar)), "r"(x), "r"(y)
      : "memory");
}

LK_DEVICE void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

LK_DEVICE void umma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

LK_DEVICE void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   lk_smem_addr(bar))
               : "memory");
}

LK_DEVICE void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
LK_DEVICE void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
LK_DEVICE void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__global__ void __launch_bounds__(kThreads, 2)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                        float* __restrict__ C, int ldc, int M, int N, int K) {
  extern __shared__ uint8_t smem_raw[];
  // the 128-byte swizzle repeats every 1024 bytes: tiles start 1024-aligned
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* tiles_a = smem;
  uint8_t* tiles_b = smem + kStagesBf * kTileBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + 2 * kStagesBf * kTileBytes);
  uint64_t* empty = full + kStagesBf;
  uint64_t* done = empty + kStagesBf;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * kBN;
  const int nk = (K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesBf; ++s) {
      lk_mbar_init(&full[s], 1);
      lk_mbar_init(&empty[s], 1);
    }
    lk_mbar_init(done, 1);
    lk_fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(lk_smem_addr(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ================= producer: TMA loads of the A and B tiles
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kStagesBf;
        if (kb >= kStagesBf &&
            !lk_mbar_wait_bounded(&empty[s], (uint32_t)(((kb / kStagesBf) - 1) & 1), LK_WAIT_LIMIT_NS)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        lk_mbar_arrive_expect_tx(&full[s], 2 * kTileBytes);
        tma_load_2d(tiles_a + s * kTileBytes, &map_a, kb * kBK, m0, &full[s]);
        tma_load_2d(tiles_b + s * kTileBytes, &map_b, kb * kBK, n0, &full[s]);
        issued = kb + 1;
      }
      // every load this CTA started has landed before it may finish
      for (int kb = max(0, issued - kStagesBf); kb < issued; ++kb)
        if (!lk_mbar_wait_bounded(&full[kb % kStagesBf], (uint32_t)((kb / kStagesBf) & 1), LK_WAIT_LIMIT_NS))
          lk_dev_fail(LK_DEV_TIMEOUT_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ================= MMA issue: the accumulator lives in TMEM
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kStagesBf;
        if (!lk_mbar_wait_bounded(&full[s], (uint32_t)((kb / kStagesBf) & 1), LK_WAIT_LIMIT_NS)) *abort_flag = 1;
        if (*abort_flag) break;
        tc_fence_after();
        const uint64_t adesc = sw128_desc(lk_smem_addr(tiles_a + s * kTileBytes));
        const uint64_t bdesc = sw128_desc(lk_smem_addr(tiles_b + s * kTileBytes));
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k)  // 16 bf16 = 32 bytes further along K per step
          umma_bf16(tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), (kb | k) != 0 ? 1u : 0u);
        umma_commit(&empty[s]);  // the slot is free once these products have read it
      }
      umma_commit(done);  // every product issued so far has completed
    }
  } else {
    // ================= epilogue: TMEM -> registers -> C
    // one verdict per warp: the TMEM loads below are warp-collective
    const bool ok = __all_sync(0xffffffffu, lk_mbar_wait_bounded(done, 0, LK_WAIT_LIMIT_NS));
    if (!ok && lane == 0) lk_dev_fail(LK_DEV_TIMEOUT_PIPE);
    tc_fence_after();
    const int q = warp & 3;  // this warp's TMEM lane quarter
    const int row = m0 + 32 * q + lane;
    if (ok && !*abort_flag) {
#pragma unroll 1
      for (int c0 = 0; c0 < kBN; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
        if (row < M) {
          float* crow = C + (int64_t)row * ldc + n0 + c0;
          if (n0 + c0 + 32 <= N && (ldc & 3) == 0) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<float4*>(crow + j) = make_float4(
                  __uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
          } else {
            for (int j = 0; j < 32; ++j)
              if (n0 + c0 + j < N) crow[j] = __uint_as_float(v[j]);
          }
        }
      }
    }
  }
  if (*abort_flag && threadIdx.x == 0) lk_dev_fail(LK_DEV_TIMEOUT_PIPE);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

// ---------------------------------------------------------------- int8 (W8A8 linears)
// C[m][n] (+)= sum_k X[m][k] * W[n][k], exact int32, for the W8A8 linears
// (LASER page, technical summary §3: both branches of the hybrid linear are
// int8 products).  The weights are the MMA's M side (128 output channels per
// CTA) and the NT tokens its N side, so a decode batch of 32 tokens fills an
// N=32 product while the weights stream through at full width.  The K range
// is split over gridDim.z CTAs; with more than one split the partial sums are
// added into C (zeroed by the caller) with integer atomics, exact and
// order-free.
constexpr int kI8BK = 128;  // bytes of K per block (the 128-byte swizzle)

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_i8_tc_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                      int32_t* __restrict__ C, int ldc, int M, int N, int K, int kblocks_per_split) {
  constexpr int kWBytes = 128 * kI8BK;   // 16 KB
  constexpr int kXBytes = NT * kI8BK;    // NT rows of 128 bytes
  constexpr uint32_t kCols = NT < 32 ? 32 : NT;
  constexpr uint32_t kIdescI8 = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NT >> 3) << 17) |
                                ((uint32_t)(128 >> 4) << 24);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* tiles_w = smem;
  uint8_t* tiles_x = smem + kStages * kWBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * (kWBytes + kXBytes));
  uint64_t* empty = full + kStages;
  uint64_t* done = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * 128, m0 = blockIdx.y * NT;
  const int nkb = (K + kI8BK - 1) / kI8BK;
  const int kb0 = blockIdx.z * kblocks_per_split;
  const int kb1 = min(nkb, kb0 + kblocks_per_split);
  const int nk = max(0, kb1 - kb0);
  const bool split = gridDim.z > 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      lk_mbar_init(&full[s], 1);
      lk_mbar_init(&empty[s], 1);
    }
    lk_mbar_init(done, 1);
    lk_fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(lk_smem_addr(tmem_slot)),
                 "r"(kCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < nk; ++j) {
        const int s = j % kStages;
        if (j >= kStages && !lk_mbar_wait_bounded(&empty[s], (uint32_t)(((j / kStages) - 1) & 1), LK_WAIT_LIMIT_NS)) {
          *abort_flag = 1;
          break;
        }
        if (*abort_flag) break;
        lk_mbar_arrive_expect_tx(&full[s], kWBytes + kXBytes);
        tma_load_2d(tiles_w + s * kWBytes, &map_w, (kb0 + j) * kI8BK, n0, &full[s]);
        tma_load_2d(tiles_x + s * kXBytes, &map_x, (kb0 + j) * kI8BK, m0, &full[s]);
        issued = j + 1;
      }
      for (int j = max(0, issued - kStages); j < issued; ++j)
        if (!lk_mbar_wait_bounded(&full[j % kStages], (uint32_t)((j / kStages) & 1), LK_WAIT_LIMIT_NS))
          lk_dev_fail(LK_DEV_TIMEOUT_DRAIN);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      for (int j = 0; j < nk; ++j) {
        const int s = j % kStages;
        if (!lk_mbar_wait_bounded(&full[s], (uint32_t)((j / kStages) & 1), LK_WAIT_LIMIT_NS)) *abort_flag = 1;
        if (*abort_flag) break;
        tc_fence_after();
        const uint64_t wdesc = sw128_desc(lk_smem_addr(tiles_w + s * kWBytes));
        const uint64_t xdesc = sw128_desc(lk_smem_addr(tiles_x + s * kXBytes));
#pragma unroll
        for (int k = 0; k < kI8BK / 32; ++k)  // 32 int8 = 32 bytes further along K per step
          umma_i8(tmem, wdesc + (uint64_t)(2 * k), xdesc + (uint64_t)(2 * k), kIdescI8, (j | k) != 0 ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      umma_commit(done);
    }
  } else {
    // epilogue: TMEM lane = output channel n, column = token m
    const bool ok = __all_sync(0xffffffffu, lk_mbar_wait_bounded(done, 0, LK_WAIT_LIMIT_NS));
    if (!ok && lane == 0) lk_dev_fail(LK_DEV_TIMEOUT_PIPE);
    tc_fence_after();
    const int q = warp & 3;
    const int n = n0 + 32 * q + lane;
    if (ok && !*abort_flag && nk > 0) {
#pragma unroll 1
      for (int c0 = 0; c0 < NT; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
        if (n < N) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int m = m0 + c0 + j;
            if (j < NT && m < M) {
              int32_t* dst = C + (int64_t)m * ldc + n;
              if (split) atomicAdd(dst, (int)v[j]);
              else *dst = (int)v[j];
            }
          }
        }
      }
    }
  }
  if (*abort_flag && threadIdx.x == 0) lk_dev_fail(LK_DEV_TIMEOUT_PIPE);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols));
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// [rows, K] elements of `esize` bytes, row stride ld elements; boxes of
// box_rows rows x 128 bytes, 128-byte swizzle, zero fill outside.
bool make_map(CUtensorMap* map, const void* base, int rows, int K, int ld, int esize, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * esize};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / esize), (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

LK_DEFINE_STATUS_ACCESSOR(lk_gemm_tc_status_word)

namespace lk {

bool gemm_bf16_tc_supported(const void* A, int lda, const void* B, int ldb, int K) {
  return K >= 1 && lda % 8 == 0 && ldb % 8 == 0 && (reinterpret_cast<uintptr_t>(A) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(B) & 15) == 0 && encode_fn() != nullptr;
}

cudaError_t launch_gemm_bf16_tc(const void* A, int lda, const void* B, int ldb, float* C, int ldc, int M, int N,
                                int K, cudaStream_t stream) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  CUtensorMap map_a, map_b;
  if (!make_map(&map_a, A, M, K, lda, 2, kBM) || !make_map(&map_b, B, N, K, ldb, 2, kBN)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gemm_bf16_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((N + kBN - 1) / kBN), (unsigned)((M + kBM - 1) / kBM));
  gemm_bf16_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(map_a, map_b, C, ldc, M, N, K);
  count_launch();
  return cudaGetLastError();
}

template <int NT>
cudaError_t launch_i8_nt(const CUtensorMap& mw, const CUtensorMap& mx, int32_t* C, int ldc, int M, int N, int K,
                         int kbps, int splits, cudaStream_t stream) {
  constexpr int smem = kStages * (128 * kI8BK + NT * kI8BK) + 1024 + 1024;
  cudaError_t e = cudaFuncSetAttribute(gemm_i8_tc_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((N + 127) / 128), (unsigned)((M + NT - 1) / NT), (unsigned)splits);
  gemm_i8_tc_kernel<NT><<<grid, kThreads, smem, stream>>>(mw, mx, C, ldc, M, N, K, kbps);
  count_launch();
  return cudaGetLastError();
}

bool gemm_i8_tc_supported(const void* A, int lda, const void* B, int ldb, int K) {
  return K >= 1 && lda % 16 == 0 && ldb % 16 == 0 && (reinterpret_cast<uintptr_t>(A) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(B) & 15) == 0 && encode_fn() != nullptr;
}

cudaError_t launch_gemm_i8_tc(const int8_t* A, int lda, const int8_t* B, int ldb, int32_t* C, int ldc, int M, int N,
                              int K, int num_sms, cudaStream_t stream) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  const int NT = M <= 32 ? 32 : (M <= 64 ? 64 : (M <= 128 ? 128 : 256));
  CUtensorMap mw, mx;
  if (!make_map(&mw, B, N, K, ldb, 1, 128) || !make_map(&mx, A, M, K, lda, 1, NT)) return cudaErrorInvalidValue;
  // split K until about two CTAs per SM are busy, at least two K blocks each
  const int nkb = (K + kI8BK - 1) / kI8BK;
  const int64_t tiles = (int64_t)((N + 127) / 128) * ((M + NT - 1) / NT);
  int splits = (int)std::min<int64_t>(std::max<int64_t>(1, (2 * num_sms + tiles - 1) / tiles), std::max(1, nkb / 2));
  const int kbps = (nkb + splits - 1) / splits;
  splits = (nkb + kbps - 1) / kbps;
  if (splits > 1) {
    cudaError_t e = cudaMemsetAsync(C, 0, ((size_t)(M - 1) * ldc + N) * sizeof(int32_t), stream);
    if (e != cudaSuccess) return e;
  }
  switch (NT) {
    case 32: return launch_i8_nt<32>(mw, mx, C, ldc, M, N, K, kbps, splits, stream);
    case 64: return launch_i8_nt<64>(mw, mx, C, ldc, M, N, K, kbps, splits, stream);
    case 128: return launch_i8_nt<128>(mw, mx, C, ldc, M, N, K, kbps, splits, stream);
    default: return launch_i8_nt<256>(mw, mx, C, ldc, M, N, K, kbps, splits, stream);
  }
}

}  // namespace lk
