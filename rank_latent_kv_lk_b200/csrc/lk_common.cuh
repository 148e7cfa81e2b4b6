// Device-side helpers shared by the latent-KV kernels (sm_100a).
//
// - 16-bit float storage helpers (bf16 / fp16 bit patterns <-> fp32)
// - the latent quantiser rule (absmax, round half to even, stated packing)
// - bulk-copy (TMA engine, non-tensor) + mbarrier wrappers with bounded waits
// - a per-translation-unit device status word set when a bounded wait expires
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

#include "lk.h"

#define LK_DEVICE __device__ __forceinline__

// Status word of this translation unit; kernels OR an error code into it
// instead of trapping, and the host reads it through lk_device_status().
static __device__ unsigned int lk_dev_status_word;

enum : unsigned int {
  LK_DEV_TIMEOUT_PIPE = 1u,   // a shared-memory pipeline wait expired
  LK_DEV_TIMEOUT_DRAIN = 2u,  // draining in-flight copies after an error expired
};

LK_DEVICE void lk_dev_fail(unsigned int code) { atomicOr(&lk_dev_status_word, code); }

// Host accessor for this translation unit's status word.
#define LK_DEFINE_STATUS_ACCESSOR(NAME)                                              \
  cudaError_t NAME(unsigned int* value, int reset) {                                 \
    cudaError_t e = cudaMemcpyFromSymbol(value, lk_dev_status_word, sizeof(unsigned int)); \
    if (e != cudaSuccess) return e;                                                  \
    if (reset && *value) {                                                           \
      unsigned int zero = 0;                                                         \
      e = cudaMemcpyToSymbol(lk_dev_status_word, &zero, sizeof(unsigned int));       \
    }                                                                                \
    return e;                                                                        \
  }

// ---------------------------------------------------------------- conversions

LK_DEVICE float lk_bf16_to_f32(uint16_t bits) { return __uint_as_float(((uint32_t)bits) << 16); }
LK_DEVICE float lk_bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
LK_DEVICE float lk_bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
LK_DEVICE uint16_t lk_f32_to_bf16(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}
LK_DEVICE float lk_f16_to_f32(uint16_t bits) {
  __half h = *reinterpret_cast<__half*>(&bits);
  return __half2float(h);
}

template <typename T> LK_DEVICE float lk_load_f(const T* p, int64_t i);
template <> LK_DEVICE float lk_load_f<float>(const float* p, int64_t i) { return p[i]; }
template <> LK_DEVICE float lk_load_f<uint16_t>(const uint16_t* p, int64_t i) {
  return lk_bf16_to_f32(p[i]);
}

// Signed byte k of a 32-bit word as fp32.  Built from the float bit pattern
// 2^23 + (c + 128): the byte (offset by 128) is spliced into the mantissa of
// 2^23 with one byte-permute and the offset removed with one exact subtract.
// `wx` must be the word XOR 0x80808080.
LK_DEVICE float lk_s8_from_xored(uint32_t wx, int k) {
  const uint32_t sel = 0x7540u | (uint32_t)k;
  return __uint_as_float(__byte_perm(wx, 0x4B000000u, sel)) - 8388736.0f;
}

// ---------------------------------------------------------------- quantiser
// Latent / activation quantiser (RTN): absmax scale, true division, round
// half to even, clamp.  Bit-exact with the CPU rule; requires IEEE fp32 (the
// library is built without fast-math and without flush-to-zero).

LK_DEVICE float lk_q8_scale(float absmax) { return __fdiv_rn(absmax, 127.0f); }

LK_DEVICE int lk_q8_code(float v, float scale) {
  if (scale == 0.0f) return 0;
  float c = rintf(__fdiv_rn(v, scale));
  c = fminf(fmaxf(c, -127.0f), 127.0f);
  return (int)c;
}

// Returns the fp16 scale (as fp32, exactly representable in fp16).
LK_DEVICE float lk_q4_scale(float absmax) {
  float s = __half2float(__float2half_rn(__fdiv_rn(absmax, 7.0f)));
  return fminf(s, 65504.0f);  // an infinite fp16 scale saturates to the largest finite
}

LK_DEVICE int lk_q4_code(float v, float scale) {
  if (scale == 0.0f) return 0;
  float c = rintf(__fdiv_rn(v, scale));
  c = fminf(fmaxf(c, -7.0f), 7.0f);
  return (int)c;
}

LK_DEVICE uint16_t lk_f32_to_f16_bits(float f) {
  __half h = __float2half_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

// ---------------------------------------------------------------- reductions

LK_DEVICE float lk_warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
LK_DEVICE float lk_warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- cache layout
// Byte offset of code byte k of token t inside one (b, h) plane whose code
// rows are rb bytes (tokens in blocks of 16, chunk-major inside a block).
LK_DEVICE int lk_chunk_bytes(int rb) { return (rb % 16 == 0) ? 16 : ((rb % 8 == 0) ? 8 : 4); }
LK_DEVICE int64_t lk_code_offset(int64_t t, int k, int rb, int cs) {
  return (t >> 4) * 16 * rb + (int64_t)(k / cs) * 16 * cs + (t & 15) * cs + (k % cs);
}

// ---------------------------------------------------------------- bulk copy / mbarrier

LK_DEVICE uint32_t lk_smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

LK_DEVICE void lk_mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(lk_smem_addr(bar)), "r"(count)
               : "memory");
}

LK_DEVICE void lk_fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

LK_DEVICE void lk_mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(lk_smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

LK_DEVICE void lk_mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(lk_smem_addr(bar)) : "memory");
}

LK_DEVICE bool lk_mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(lk_smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

LK_DEVICE uint64_t lk_globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Waits for the mbarrier phase with the given parity to complete; gives up
// after `limit_ns` nanoseconds and returns false.  Each try_wait (no time
// hint) suspends the thread in hardware until the phase completes or a
// system-dependent limit passes, so the loop costs few issue slots.  (A
// try_wait with a suspend-time hint measured late wake-ups, about 2-3 us
// after the phase completed, and is not used.)
LK_DEVICE bool lk_mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (lk_mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = lk_globaltimer_ns();
  for (uint32_t i = 0;; ++i) {
    if (lk_mbar_try_wait(bar, parity)) return true;
    if ((i & 7u) == 7u && lk_globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// One bulk global -> shared copy completing on `bar` (TMA engine, no tensor
// map, no multicast).  dst, src 16-byte aligned; bytes a multiple of 16.
LK_DEVICE void lk_bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          lk_smem_addr(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(lk_smem_addr(bar))
      : "memory");
}

static constexpr uint64_t LK_WAIT_LIMIT_NS = 2000000000ull;  // 2 s

// ---------------------------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialisation may start while
// the previous kernel on its stream still runs; it must call lk_grid_dep_wait
// before touching anything that kernel writes (the wait returns once the
// previous grid has completed and its memory is visible; without the launch
// attribute it returns at once).  lk_grid_dep_launch lets such a dependent
// kernel be scheduled early.
LK_DEVICE void lk_grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
LK_DEVICE void lk_grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// ---------------------------------------------------------------- warp-level bf16 tensor-core products
// D = A B + D for a 16 x 16 (m16n8k16) or 16 x 8 (m16n8k8) bf16 A and a
// 16 x 8 / 8 x 8 bf16 B, fp32 accumulators.  Fragments (gid = lane / 4,
// tig = lane % 4): a0 = (row gid, k 2 tig, 2 tig + 1), a1 = row gid + 8,
// a2 / a3 = the same rows at k + 8; b0 = (k 2 tig, 2 tig + 1, column gid),
// b1 = k + 8; c0, c1 = (row gid, columns 2 tig, 2 tig + 1), c2, c3 = row
// gid + 8.  The k8 form takes a0, a1 and b0 only.
LK_DEVICE void lk_mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                 uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
LK_DEVICE void lk_mma_bf16_1688(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(b0));
}
// Four 8 x 8 b16 matrices from shared memory: lanes 8 i .. 8 i + 7 give the
// row addresses of matrix i (16 bytes each); lane l receives, of matrix i,
// row l / 4, elements 2 (l % 4) and 2 (l % 4) + 1 (.trans: the transpose).
LK_DEVICE void lk_ldmatrix_x4(uint32_t (&r)[4], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(lk_smem_addr(row_addr)));
}
LK_DEVICE void lk_ldmatrix_x4_trans(uint32_t (&r)[4], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(lk_smem_addr(row_addr)));
}
// Two values as packed bf16 (first in the low half), round to nearest even.
LK_DEVICE uint32_t lk_pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------- cp.async (16 bytes, L1 bypassed)
// Copies 16 bytes from global to shared memory asynchronously (both 16-byte
// aligned).  lk_cp_async_commit closes a group; lk_cp_async_wait<N> waits
// until at most N of this thread's groups are pending.
LK_DEVICE void lk_cp_async16(void* dst_smem, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(lk_smem_addr(dst_smem)), "l"(src) : "memory");
}
LK_DEVICE void lk_cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
LK_DEVICE void lk_cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
