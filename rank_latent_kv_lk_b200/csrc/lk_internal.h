// Internal launch interfaces between the C-ABI layer (lk_api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

#include <algorithm>

#include "lk.h"

namespace lk {

// Kernels this library has launched in the process (every launch site calls
// count_launch once per kernel it enqueues; read through lk_kernel_launches).
void count_launch(unsigned n = 1);

// ---------------------------------------------------------------- decode
struct DecodeLaunch {
  const void* codes_k;
  const void* codes_v;
  const void* scales_k;
  const void* scales_v;
  const void* q;
  const void* BK;
  const void* BV;
  const int32_t* seq_len;
  void* out;
  void* workspace;
  const int32_t* ranks_k;  // host
  const int32_t* ranks_v;  // host
  int kind;                // 0 = int8, 1 = int4
  int batch, n_heads, head_dim, capacity;
  int group_k, group_v;
  int q_bf16, b_bf16, out_bf16;
  int max_len, n_split, num_sms;
  int early_inputs;  // read q, B_K, B_V before waiting for the previous kernel (decode step entry point)
  int stable_len;    // with early_inputs: positions below it are final before the kernel starts
  float softmax_scale;
  uint64_t wait_ns = 0;  // bound of the pipeline waits (0: the library's default)
  int stall_item = -1;   // test hook: the copy producer stops before this item
};
// Workspace of a decode call: arrival counters for the units plus two partial
// slots per CTA; n_split > 0 asks for about n_split pieces per unit, 0 for a
// grid that fills the GPU (at most 1024 CTAs).
size_t decode_workspace_bytes(int units, int rv_max, int max_len, int n_split);
cudaError_t launch_decode_attn(const DecodeLaunch& a, cudaStream_t stream);


// ---------------------------------------------------------------- FFN input side split on output channels
struct OutsplitWeights {
  const int8_t* W_D;    // [n_dense][k_in]
  const uint16_t* s_D;  // fp16 [n_dense]
  const int8_t* U;      // [rank][k_in]
  const uint16_t* s_U;  // fp16 [rank]
  const int8_t* V;      // [n_out - n_dense][rank]
  const uint16_t* s_V;  // fp16 [n_out - n_dense]
};
struct FfnLaunch {
  OutsplitWeights gate, up;
  const int32_t* dense_out;  // device [n_dense]
  const int32_t* lr_out;     // device [n_out - n_dense]
  const int8_t* x_q;
  const float* x_scale;
  float* out;
  void* workspace;
  int m, k_in, n_out, n_dense, rank;
};
size_t ffn_workspace_bytes(int m, int rank);
cudaError_t launch_ffn_gate_up(const FfnLaunch& a, cudaStream_t stream);

// ---------------------------------------------------------------- rotary-position decode
struct RopeLaunch {
  const void* codes_k;
  const void* codes_v;
  const void* scales_k;
  const void* scales_v;
  const void* q;
  const void* BK;  // bf16
  const void* BV;  // bf16
  const float* table;
  const int32_t* seq_len;
  void* out;
  void* workspace;
  const int32_t* ranks_k;  // host
  const int32_t* ranks_v;  // host
  int kind, batch, n_heads, head_dim, capacity, group_k, group_v;
  int q_bf16, out_bf16, max_len, num_sms;
  float softmax_scale;
};
size_t rope_workspace_bytes(int units, int rv_max, int max_len, int num_sms);
cudaError_t launch_rope_decode(const RopeLaunch& a, cudaStream_t stream);
cudaError_t launch_rope_table(float* table, int head_dim, int max_pos, double base, cudaStream_t stream);

// ---------------------------------------------------------------- dense comparison points
struct DenseLaunch {
  const void* q;  // bf16 [B, n_heads, H]
  const void* K;  // bf16 [B, n_heads, capacity, H]
  const void* V;
  const int32_t* seq_len;
  void* out;
  void* workspace;
  int batch, n_heads, head_dim, capacity, max_len, out_bf16, num_sms;
  float softmax_scale;
};
size_t dense_workspace_bytes(int units, int head_dim, int max_len, int num_sms);
cudaError_t launch_dense_decode(const DenseLaunch& a, cudaStream_t stream);

struct ReconLaunch {
  const void* codes[2];      // K cache, V cache
  const void* scales[2];
  const void* B[2];          // B_K, B_V packed per head
  void* out[2];              // bf16 [B, n_heads, capacity, H]
  const int32_t* ranks[2];   // host
  int group[2];
  const int32_t* seq_len;
  int kind, batch, n_heads, head_dim, capacity, max_len, b_bf16;
};
cudaError_t launch_reconstruct_kv(const ReconLaunch& a, cudaStream_t stream);

// ---------------------------------------------------------------- projection
enum XType { X_F32 = 0, X_BF16 = 1, X_I8 = 2 };

// Heads of one cache as seen by the quantise-and-append epilogue.
struct CacheView {
  void* codes;
  void* scales;
  int kind;      // 0 = int8, 1 = int4
  int group;
  int n_heads;
  int capacity;
  int rotation;  // 1: each head's latent is rotated by its S2 before quantisation
};

struct ProjectLaunch {
  CacheView k, v;
  const int32_t* ranks_k;  // host
  const int32_t* ranks_v;  // host
  const void* x;
  const float* x_scale;
  const void* A;
  const uint16_t* a_scale;
  int xtype;
  int batch, n_new, embed_dim, n_tot;
  int32_t* seq_len;
  void* workspace;
  size_t workspace_bytes;
  int num_sms;
};
size_t project_workspace_bytes(int rows, int n_tot, int embed_dim, int xtype, int num_sms);
cudaError_t launch_project_append(const ProjectLaunch& a, cudaStream_t stream);

// ---------------------------------------------------------------- low-rank linear
struct LowrankLaunch {
  int k_in, n_out, rank, n_dense, m;
  const int32_t* dense_idx;
  const int32_t* lr_idx;
  const int8_t* W_D;
  const uint16_t* s_D;
  const int8_t* U;
  const uint16_t* s_U;
  const int8_t* V;
  const uint16_t* s_V;
  const int8_t* x_q;
  const float* x_scale;
  const uint16_t* residual;
  void* y;
  int y_bf16;
  int8_t* t_q_out;
  float* t_scale_out;
  void* workspace;
  int num_sms;
};
size_t lowrank_workspace_bytes(int k_in, int n_out, int rank, int n_dense, int m);
cudaError_t launch_lowrank_linear(const LowrankLaunch& a, cudaStream_t stream);

// ---------------------------------------------------------------- quantisers / elementwise
cudaError_t launch_quantize_latent(const float* v, int m, int r, int kind, int group, void* codes,
                                   void* scales, cudaStream_t stream);
// mode 0: quantise x; 1: RMSNorm then quantise; 2: SwiGLU(x, x2) then quantise;
// 3: RMSNorm, then the normalised Walsh-Hadamard transform (k a power of two), then quantise
cudaError_t launch_rowquant(int mode, const void* x, const void* x2, int x_bf16, int m, int k,
                            float eps, int8_t* x_q, float* x_scale, cudaStream_t stream);

// ---------------------------------------------------------------- generic int8 GEMM
// C[m][n] = sum_k A[m][k] * B[n][k]  (int32), A, B row-major with given row strides (bytes)
// tcgen05 bf16 GEMM with TMEM accumulators (lk_gemm_tc.cu): same contract as
// launch_gemm_f with bf16 operands; needs lda, ldb multiples of 8 and
// 16-byte aligned operands.
bool gemm_bf16_tc_supported(const void* A, int lda, const void* B, int ldb, int K);
cudaError_t launch_gemm_bf16_tc(const void* A, int lda, const void* B, int ldb, float* C, int ldc, int M, int N,
                                int K, cudaStream_t stream);
// tcgen05 int8 GEMM (exact int32), K split over CTAs with integer atomics;
// needs lda, ldb multiples of 16 and 16-byte aligned operands.
bool gemm_i8_tc_supported(const void* A, int lda, const void* B, int ldb, int K);
cudaError_t launch_gemm_i8_tc(const int8_t* A, int lda, const int8_t* B, int ldb, int32_t* C, int ldc, int M, int N,
                              int K, int num_sms, cudaStream_t stream);
cudaError_t launch_gemm_i8(const int8_t* A, int lda, const int8_t* B, int ldb, int32_t* C, int ldc,
                           int M, int N, int K, cudaStream_t stream);

}  // namespace lk

// Per-translation-unit device status words (see lk_common.cuh).
cudaError_t lk_decode_status_word(unsigned int* value, int reset);
