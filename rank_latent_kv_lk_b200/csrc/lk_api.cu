// C ABI: host-side validation and dispatch for every entry point in lk.h.
// Nothing is launched and nothing is written unless every check passes.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include <atomic>

#include "lk_internal.h"

namespace lk {
namespace {
std::atomic<unsigned long long> g_launches{0};
}
void count_launch(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
unsigned long long launches_value() { return g_launches.load(std::memory_order_relaxed); }
}  // namespace lk

cudaError_t lk_quant_status_word(unsigned int* value, int reset);
cudaError_t lk_project_status_word(unsigned int* value, int reset);
cudaError_t lk_lowrank_status_word(unsigned int* value, int reset);
cudaError_t lk_gemm_tc_status_word(unsigned int* value, int reset);

namespace {

thread_local char g_last_error[512] = "";

lk_status fail(lk_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

lk_status cuda_fail(cudaError_t e, const char* where) {
  return fail(LK_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

int row_bytes(const lk_latent_cache* c, int r) { return c->code_dtype == LK_I8 ? r : r / 2; }
int n_groups(const lk_latent_cache* c, int r) {
  if (c->code_dtype == LK_I8) return 1;
  const int g = std::min(c->group, r);
  return (r + g - 1) / g;
}

lk_status check_cache(const lk_latent_cache* c, const char* name, bool need_buffers) {
  if (!c) return fail(LK_ERR_INVALID_ARG, "%s: null cache descriptor", name);
  if (c->batch < 1) return fail(LK_ERR_SHAPE, "%s: batch %d < 1", name, c->batch);
  if (c->n_heads < 1 || c->n_heads > LK_MAX_HEADS)
    return fail(LK_ERR_SHAPE, "%s: n_heads %d outside [1, %d]", name, c->n_heads, LK_MAX_HEADS);
  if (c->capacity < 16 || c->capacity % 16 != 0)
    return fail(LK_ERR_SHAPE, "%s: capacity %d is not a positive multiple of 16", name, c->capacity);
  if (c->code_dtype != LK_I8 && c->code_dtype != LK_I4)
    return fail(LK_ERR_DTYPE, "%s: code dtype must be LK_I8 or LK_I4", name);
  if (c->code_dtype == LK_I4 && (c->group < 8 || c->group % 8 != 0))
    return fail(LK_ERR_SHAPE, "%s: int4 group %d must be a positive multiple of 8", name, c->group);
  if (!c->ranks) return fail(LK_ERR_INVALID_ARG, "%s: null ranks", name);
  if (c->rotation != 0 && c->rotation != 1) return fail(LK_ERR_INVALID_ARG, "%s: rotation must be 0 or 1", name);
  const int mult = c->code_dtype == LK_I8 ? 4 : 8;
  for (int h = 0; h < c->n_heads; ++h) {
    const int r = c->ranks[h];
    if (r < 4 || r > LK_MAX_RANK || r % mult != 0)
      return fail(LK_ERR_SHAPE, "%s: rank[%d] = %d must be in [4, %d] and a multiple of %d", name, h, r,
                  LK_MAX_RANK, mult);
  }
  if (need_buffers) {
    if (!c->codes || !c->scales) return fail(LK_ERR_INVALID_ARG, "%s: null codes or scales", name);
    if (!aligned(c->codes, 256) || !aligned(c->scales, 256))
      return fail(LK_ERR_ALIGN, "%s: codes and scales must be 256-byte aligned", name);
  }
  return LK_OK;
}

size_t decode_ws_bytes(const lk_latent_cache* k, const lk_latent_cache* v, int max_seq_len, int n_split) {
  int rv_max = 0;
  for (int h = 0; h < v->n_heads; ++h) rv_max = std::max(rv_max, v->ranks[h]);
  return lk::decode_workspace_bytes(k->batch * k->n_heads, rv_max, max_seq_len, n_split);
}

}  // namespace

namespace lk {
// Records an error for lk_last_error() from another translation unit.
lk_status set_error(lk_status s, const char* msg) {
  snprintf(g_last_error, sizeof(g_last_error), "%s", msg);
  return s;
}
}  // namespace lk

extern "C" {

int32_t lk_version(void) { return 1; }

uint64_t lk_kernel_launches(void) { return lk::launches_value(); }

const char* lk_last_error(void) { return g_last_error; }

const char* lk_status_string(lk_status s) {
  switch (s) {
    case LK_OK: return "ok";
    case LK_ERR_INVALID_ARG: return "invalid argument";
    case LK_ERR_SHAPE: return "bad shape";
    case LK_ERR_DTYPE: return "unsupported dtype";
    case LK_ERR_ALIGN: return "misaligned pointer or size";
    case LK_ERR_CAPACITY: return "cache capacity exceeded";
    case LK_ERR_UNSUPPORTED: return "unsupported";
    case LK_ERR_WORKSPACE: return "workspace too small";
    case LK_ERR_CUDA: return "CUDA error";
    case LK_ERR_DEVICE: return "device-side bounded wait expired";
  }
  return "unknown status";
}

lk_status lk_latent_cache_bytes(const lk_latent_cache* cache, size_t* codes_bytes, size_t* scales_bytes) {
  lk_status s = check_cache(cache, "cache", false);
  if (s != LK_OK) return s;
  if (!codes_bytes || !scales_bytes) return fail(LK_ERR_INVALID_ARG, "null output pointer");
  size_t rb = 0, ng = 0;
  for (int h = 0; h < cache->n_heads; ++h) {
    rb += row_bytes(cache, cache->ranks[h]);
    ng += n_groups(cache, cache->ranks[h]);
  }
  *codes_bytes = (size_t)cache->batch * rb * cache->capacity;
  *scales_bytes = (size_t)cache->batch * ng * cache->capacity * (cache->code_dtype == LK_I8 ? 4 : 2);
  return LK_OK;
}

size_t lk_latent_project_workspace_bytes(const lk_latent_cache* k, const lk_latent_cache* v, int32_t embed_dim,
                                         int32_t n_new, lk_dtype x_dtype) {
  if (check_cache(k, "k_cache", false) != LK_OK || check_cache(v, "v_cache", false) != LK_OK) return 0;
  if (embed_dim < 1 || n_new < 1) return 0;
  int n_tot = 0;
  for (int h = 0; h < k->n_heads; ++h) n_tot += k->ranks[h];
  for (int h = 0; h < v->n_heads; ++h) n_tot += v->ranks[h];
  const int xt = x_dtype == LK_F32 ? lk::X_F32 : (x_dtype == LK_BF16 ? lk::X_BF16 : lk::X_I8);
  return lk::project_workspace_bytes(k->batch * n_new, n_tot, embed_dim, xt, num_sms());
}

lk_status lk_latent_project_append(const lk_latent_cache* k, const lk_latent_cache* v, const void* x,
                                   lk_dtype x_dtype, const float* x_scale, const void* A, lk_dtype a_dtype,
                                   const uint16_t* a_scale, int32_t embed_dim, int32_t n_new, int32_t* seq_len,
                                   const int32_t* seq_len_host, void* workspace, size_t workspace_bytes,
                                   lk_stream_t stream) {
  lk_status s;
  if ((s = check_cache(k, "k_cache", true)) != LK_OK) return s;
  if ((s = check_cache(v, "v_cache", true)) != LK_OK) return s;
  if (k->batch != v->batch) return fail(LK_ERR_SHAPE, "k and v caches differ in batch");
  if (!x || !A) return fail(LK_ERR_INVALID_ARG, "null x or A");
  if (x_dtype != LK_F32 && x_dtype != LK_BF16 && x_dtype != LK_I8)
    return fail(LK_ERR_DTYPE, "x dtype must be LK_F32, LK_BF16 or LK_I8");
  if (a_dtype != x_dtype) return fail(LK_ERR_DTYPE, "A dtype must equal x dtype");
  if (x_dtype == LK_I8 && (!x_scale || !a_scale))
    return fail(LK_ERR_INVALID_ARG, "int8 inputs need x_scale and a_scale");
  if (embed_dim < 1) return fail(LK_ERR_SHAPE, "embed_dim %d < 1", embed_dim);
  const int xsz = x_dtype == LK_F32 ? 4 : (x_dtype == LK_BF16 ? 2 : 1);
  if (((size_t)embed_dim * xsz) % 16 != 0)
    return fail(LK_ERR_ALIGN, "embed_dim * element size must be a multiple of 16 bytes");
  if (!aligned(x, 16) || !aligned(A, 16)) return fail(LK_ERR_ALIGN, "x and A must be 16-byte aligned");
  if (n_new < 1) return fail(LK_ERR_SHAPE, "n_new %d < 1", n_new);
  if (!seq_len || !seq_len_host) return fail(LK_ERR_INVALID_ARG, "null seq_len or seq_len_host");
  for (int b = 0; b < k->batch; ++b) {
    const int64_t L = seq_len_host[b];
    if (L < 0) return fail(LK_ERR_SHAPE, "seq_len_host[%d] = %lld < 0", b, (long long)L);
    if (L + n_new > k->capacity || L + n_new > v->capacity)
      return fail(LK_ERR_CAPACITY, "row %d: %lld + %d tokens exceed capacity", b, (long long)L, n_new);
  }
  const int64_t rows = (int64_t)k->batch * n_new;
  if (rows > (int64_t)1 << 30) return fail(LK_ERR_SHAPE, "too many rows");
  const size_t need = lk_latent_project_workspace_bytes(k, v, embed_dim, n_new, x_dtype);
  if (!workspace || workspace_bytes < need)
    return fail(LK_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need, workspace_bytes);
  if (!aligned(workspace, 256)) return fail(LK_ERR_ALIGN, "workspace must be 256-byte aligned");

  lk::ProjectLaunch a{};
  a.k = {k->codes, k->scales, k->code_dtype == LK_I8 ? 0 : 1, k->group, k->n_heads, k->capacity, k->rotation};
  a.v = {v->codes, v->scales, v->code_dtype == LK_I8 ? 0 : 1, v->group, v->n_heads, v->capacity, v->rotation};
  a.ranks_k = k->ranks;
  a.ranks_v = v->ranks;
  a.x = x;
  a.x_scale = x_scale;
  a.A = A;
  a.a_scale = a_scale;
  a.xtype = x_dtype == LK_F32 ? lk::X_F32 : (x_dtype == LK_BF16 ? lk::X_BF16 : lk::X_I8);
  a.batch = k->batch;
  a.n_new = n_new;
  a.embed_dim = embed_dim;
  int n_tot = 0;
  for (int h = 0; h < k->n_heads; ++h) n_tot += k->ranks[h];
  for (int h = 0; h < v->n_heads; ++h) n_tot += v->ranks[h];
  a.n_tot = n_tot;
  a.seq_len = seq_len;
  a.workspace = workspace;
  a.workspace_bytes = workspace_bytes;
  a.num_sms = num_sms();
  cudaError_t e = lk::launch_project_append(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lk_latent_project_append");
  return LK_OK;
}

size_t lk_latent_decode_workspace_bytes(const lk_latent_cache* k, const lk_latent_cache* v, int32_t max_seq_len,
                                        int32_t n_split) {
  if (check_cache(k, "k_cache", false) != LK_OK || check_cache(v, "v_cache", false) != LK_OK) return 0;
  if (max_seq_len < 0 || n_split < 0) return 0;
  return decode_ws_bytes(k, v, max_seq_len, n_split);
}

namespace {
// Validates a decode call and, if `launch`, launches it.  early_inputs: the
// kernel may read q, B_K and B_V before the previous kernel on the stream
// has finished (only the decode step entry point, which itself launches that
// previous kernel, sets it).
lk_status decode_attn_impl(const lk_latent_cache* k, const lk_latent_cache* v, const void* q, lk_dtype q_dtype,
                           const void* B_K, const void* B_V, lk_dtype b_dtype, int32_t head_dim,
                           const int32_t* seq_len, int32_t max_seq_len, float softmax_scale, void* out,
                           lk_dtype out_dtype, int32_t n_split, void* workspace, size_t workspace_bytes,
                           lk_stream_t stream, bool launch, int early_inputs, int stable_len,
                           int stall_item = -1, uint64_t wait_ns = 0) {
  lk_status s;
  if ((s = check_cache(k, "k_cache", true)) != LK_OK) return s;
  if ((s = check_cache(v, "v_cache", true)) != LK_OK) return s;
  if (k->batch != v->batch || k->n_heads != v->n_heads)
    return fail(LK_ERR_SHAPE, "k and v caches differ in batch or heads");
  if (k->capacity != v->capacity) return fail(LK_ERR_SHAPE, "k and v caches differ in capacity");
  if (k->code_dtype != v->code_dtype) return fail(LK_ERR_UNSUPPORTED, "k and v caches differ in code dtype");
  if (!q || !B_K || !B_V || !out || !seq_len) return fail(LK_ERR_INVALID_ARG, "null q, B_K, B_V, out or seq_len");
  if (q_dtype != LK_F32 && q_dtype != LK_BF16) return fail(LK_ERR_DTYPE, "q dtype must be LK_F32 or LK_BF16");
  if (b_dtype != LK_F32 && b_dtype != LK_BF16) return fail(LK_ERR_DTYPE, "B dtype must be LK_F32 or LK_BF16");
  if (out_dtype != LK_F32 && out_dtype != LK_BF16) return fail(LK_ERR_DTYPE, "out dtype must be LK_F32 or LK_BF16");
  if (head_dim < 8 || head_dim > LK_MAX_HEAD_DIM || head_dim % 8 != 0)
    return fail(LK_ERR_SHAPE, "head_dim %d must be a multiple of 8 in [8, %d]", head_dim, LK_MAX_HEAD_DIM);
  if (!aligned(q, 16) || !aligned(B_K, 16) || !aligned(B_V, 16))
    return fail(LK_ERR_ALIGN, "q, B_K and B_V must be 16-byte aligned");
  if (max_seq_len < 0 || max_seq_len > k->capacity)
    return fail(LK_ERR_SHAPE, "max_seq_len %d outside [0, capacity]", max_seq_len);
  if (n_split < 0) return fail(LK_ERR_SHAPE, "n_split %d < 0", n_split);
  if (!(softmax_scale == softmax_scale)) return fail(LK_ERR_INVALID_ARG, "softmax_scale is NaN");
  const size_t need = decode_ws_bytes(k, v, max_seq_len, n_split);
  if (!workspace || workspace_bytes < need)
    return fail(LK_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need, workspace_bytes);
  if (!aligned(workspace, 256)) return fail(LK_ERR_ALIGN, "workspace must be 256-byte aligned");

  lk::DecodeLaunch a{};
  a.codes_k = k->codes;
  a.codes_v = v->codes;
  a.scales_k = k->scales;
  a.scales_v = v->scales;
  a.q = q;
  a.BK = B_K;
  a.BV = B_V;
  a.seq_len = seq_len;
  a.out = out;
  a.workspace = workspace;
  a.ranks_k = k->ranks;
  a.ranks_v = v->ranks;
  a.kind = k->code_dtype == LK_I8 ? 0 : 1;
  a.batch = k->batch;
  a.n_heads = k->n_heads;
  a.head_dim = head_dim;
  a.capacity = k->capacity;
  a.group_k = k->group;
  a.group_v = v->group;
  a.q_bf16 = q_dtype == LK_BF16;
  a.b_bf16 = b_dtype == LK_BF16;
  a.out_bf16 = out_dtype == LK_BF16;
  a.max_len = max_seq_len;
  a.n_split = n_split;
  a.num_sms = num_sms();
  a.softmax_scale = softmax_scale;
  a.early_inputs = early_inputs;
  a.stable_len = stable_len;
  a.stall_item = stall_item;
  a.wait_ns = wait_ns;
  if (!launch) return LK_OK;
  cudaError_t e = lk::launch_decode_attn(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lk_latent_decode_attn");
  return LK_OK;
}
}  // namespace

lk_status lk_latent_decode_attn(const lk_latent_cache* k, const lk_latent_cache* v, const void* q,
                                lk_dtype q_dtype, const void* B_K, const void* B_V, lk_dtype b_dtype,
                                int32_t head_dim, const int32_t* seq_len, int32_t max_seq_len,
                                float softmax_scale, void* out, lk_dtype out_dtype, int32_t n_split,
                                void* workspace, size_t workspace_bytes, lk_stream_t stream) {
  return decode_attn_impl(k, v, q, q_dtype, B_K, B_V, b_dtype, head_dim, seq_len, max_seq_len, softmax_scale, out,
                          out_dtype, n_split, workspace, workspace_bytes, stream, true, 0, 0);
}

lk_status lk_debug_decode_attn_stall(const lk_latent_cache* k, const lk_latent_cache* v, const void* q,
                                     lk_dtype q_dtype, const void* B_K, const void* B_V, lk_dtype b_dtype,
                                     int32_t head_dim, const int32_t* seq_len, int32_t max_seq_len,
                                     float softmax_scale, void* out, lk_dtype out_dtype, int32_t n_split,
                                     void* workspace, size_t workspace_bytes, int32_t stall_item, uint32_t wait_us,
                                     lk_stream_t stream) {
  if (stall_item < 0 || wait_us == 0) return fail(LK_ERR_INVALID_ARG, "stall_item must be >= 0 and wait_us > 0");
  return decode_attn_impl(k, v, q, q_dtype, B_K, B_V, b_dtype, head_dim, seq_len, max_seq_len, softmax_scale, out,
                          out_dtype, n_split, workspace, workspace_bytes, stream, true, 0, 0, stall_item,
                          (uint64_t)wait_us * 1000u);
}

lk_status lk_latent_decode_step(const lk_latent_cache* k, const lk_latent_cache* v, const void* x, lk_dtype x_dtype,
                                const float* x_scale, const void* A, lk_dtype a_dtype, const uint16_t* a_scale,
                                int32_t embed_dim, int32_t* seq_len, const int32_t* seq_len_host, const void* q,
                                lk_dtype q_dtype, const void* B_K, const void* B_V, lk_dtype b_dtype,
                                int32_t head_dim, float softmax_scale, void* out, lk_dtype out_dtype,
                                int32_t n_split, void* project_workspace, size_t project_workspace_bytes,
                                void* decode_workspace, size_t decode_workspace_bytes, lk_stream_t stream) {
  if (!k || !seq_len_host) return fail(LK_ERR_INVALID_ARG, "null k_cache or seq_len_host");
  if (k->batch < 1) return fail(LK_ERR_SHAPE, "batch %d < 1", k->batch);
  int max_len = 0, stable_len = INT32_MAX;
  for (int b = 0; b < k->batch; ++b) {
    max_len = std::max(max_len, (int)seq_len_host[b] + 1);
    stable_len = std::min(stable_len, (int)seq_len_host[b]);  // the append writes at or past it
  }
  // the attention is validated first, so a rejected call launches nothing
  lk_status s = decode_attn_impl(k, v, q, q_dtype, B_K, B_V, b_dtype, head_dim, seq_len, max_len, softmax_scale,
                                 out, out_dtype, n_split, decode_workspace, decode_workspace_bytes, stream, false, 1,
                                 stable_len);
  if (s != LK_OK) return s;
  s = lk_latent_project_append(k, v, x, x_dtype, x_scale, A, a_dtype, a_scale, embed_dim, 1, seq_len, seq_len_host,
                               project_workspace, project_workspace_bytes, stream);
  if (s != LK_OK) return s;
  return decode_attn_impl(k, v, q, q_dtype, B_K, B_V, b_dtype, head_dim, seq_len, max_len, softmax_scale, out,
                          out_dtype, n_split, decode_workspace, decode_workspace_bytes, stream, true, 1, stable_len);
}

size_t lk_dense_decode_workspace_bytes(int32_t batch, int32_t n_heads, int32_t head_dim, int32_t max_seq_len) {
  if (batch < 1 || n_heads < 1 || head_dim < 8 || max_seq_len < 0) return 0;
  return lk::dense_workspace_bytes(batch * n_heads, head_dim, max_seq_len, num_sms());
}

lk_status lk_dense_decode_attn(const void* q, const void* K, const void* V, int32_t batch, int32_t n_heads,
                               int32_t head_dim, int32_t capacity, const int32_t* seq_len, int32_t max_seq_len,
                               float softmax_scale, void* out, lk_dtype out_dtype, void* workspace,
                               size_t workspace_bytes, lk_stream_t stream) {
  if (!q || !K || !V || !seq_len || !out) return fail(LK_ERR_INVALID_ARG, "null q, K, V, seq_len or out");
  if (batch < 1 || n_heads < 1 || capacity < 1) return fail(LK_ERR_SHAPE, "batch, n_heads and capacity must be >= 1");
  if (head_dim < 8 || head_dim > LK_MAX_HEAD_DIM || head_dim % 8 != 0)
    return fail(LK_ERR_SHAPE, "head_dim %d must be a multiple of 8 in [8, %d]", head_dim, LK_MAX_HEAD_DIM);
  if (max_seq_len < 0 || max_seq_len > capacity)
    return fail(LK_ERR_SHAPE, "max_seq_len %d outside [0, capacity]", max_seq_len);
  if (out_dtype != LK_F32 && out_dtype != LK_BF16) return fail(LK_ERR_DTYPE, "out dtype must be LK_F32 or LK_BF16");
  if (!aligned(q, 16) || !aligned(K, 16) || !aligned(V, 16)) return fail(LK_ERR_ALIGN, "q, K and V must be 16-byte aligned");
  if (!(softmax_scale == softmax_scale)) return fail(LK_ERR_INVALID_ARG, "softmax_scale is NaN");
  const size_t need = lk_dense_decode_workspace_bytes(batch, n_heads, head_dim, max_seq_len);
  if (!workspace || workspace_bytes < need)
    return fail(LK_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need, workspace_bytes);
  if (!aligned(workspace, 256)) return fail(LK_ERR_ALIGN, "workspace must be 256-byte aligned");
  lk::DenseLaunch a{};
  a.q = q;
  a.K = K;
  a.V = V;
  a.seq_len = seq_len;
  a.out = out;
  a.workspace = workspace;
  a.batch = batch;
  a.n_heads = n_heads;
  a.head_dim = head_dim;
  a.capacity = capacity;
  a.max_len = max_seq_len;
  a.out_bf16 = out_dtype == LK_BF16;
  a.num_sms = num_sms();
  a.softmax_scale = softmax_scale;
  if (max_seq_len == 0 && batch * n_heads == 0) return LK_OK;
  cudaError_t e = lk::launch_dense_decode(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lk_dense_decode_attn");
  return LK_OK;
}

size_t lk_ffn_gate_up_swiglu_workspace_bytes(int32_t rank, int32_t m) {
  if (rank < 0 || m < 0) return 0;
  return lk::ffn_workspace_bytes(m, rank);
}

lk_status lk_ffn_gate_up_swiglu(const lk_outsplit_weight* gate, const lk_outsplit_weight* up, int32_t k_in,
                                int32_t n_out, int32_t n_dense, int32_t rank, const int32_t* dense_out,
                                const int32_t* lr_out, const int8_t* x_q, const float* x_scale, int32_t m,
                                float* out, void* workspace, size_t workspace_bytes, lk_stream_t stream) {
  if (!gate || !up) return fail(LK_ERR_INVALID_ARG, "null weight descriptor");
  if (k_in < 16 || k_in % 16 || n_out < 1 || n_dense < 0 || n_dense > n_out || rank < 0 || rank % 16)
    return fail(LK_ERR_SHAPE, "bad k_in %d / n_out %d / n_dense %d / rank %d", k_in, n_out, n_dense, rank);
  if ((n_dense < n_out) != (rank > 0))
    return fail(LK_ERR_SHAPE, "rank %d must be > 0 exactly when some channels are low-rank", rank);
  if (m < 0 || m > 65535) return fail(LK_ERR_SHAPE, "m %d outside [0, 65535]", m);
  if (m > 0 && (!x_q || !x_scale || !out)) return fail(LK_ERR_INVALID_ARG, "null x_q, x_scale or out");
  for (const lk_outsplit_weight* w : {gate, up}) {
    if (n_dense > 0 && (!w->W_D || !w->s_D || !dense_out))
      return fail(LK_ERR_INVALID_ARG, "null dense weights, scales or channel list");
    if (n_dense < n_out && (!w->U || !w->s_U || !w->V || !w->s_V || !lr_out))
      return fail(LK_ERR_INVALID_ARG, "null low-rank weights, scales or channel list");
    if (!aligned(w->W_D, 16) || !aligned(w->U, 16) || !aligned(w->V, 16))
      return fail(LK_ERR_ALIGN, "weights must be 16-byte aligned");
  }
  if (!aligned(x_q, 16)) return fail(LK_ERR_ALIGN, "x_q must be 16-byte aligned");
  const size_t need = lk::ffn_workspace_bytes(m, rank);
  if (!workspace || workspace_bytes < need)
    return fail(LK_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need, workspace_bytes);
  if (!aligned(workspace, 256)) return fail(LK_ERR_ALIGN, "workspace must be 256-byte aligned");
  lk::FfnLaunch a{};
  a.gate = {gate->W_D, gate->s_D, gate->U, gate->s_U, gate->V, gate->s_V};
  a.up = {up->W_D, up->s_D, up->U, up->s_U, up->V, up->s_V};
  a.dense_out = dense_out;
  a.lr_out = lr_out;
  a.x_q = x_q;
  a.x_scale = x_scale;
  a.out = out;
  a.workspace = workspace;
  a.m = m;
  a.k_in = k_in;
  a.n_out = n_out;
  a.n_dense = n_dense;
  a.rank = rank;
  cudaError_t e = lk::launch_ffn_gate_up(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lk_ffn_gate_up_swiglu");
  return LK_OK;
}

lk_status lk_rope_table(int32_t head_dim, int32_t max_pos, float base, float* table, lk_stream_t stream) {
  if (head_dim < 2 || head_dim > LK_MAX_HEAD_DIM || head_dim % 2 != 0)
    return fail(LK_ERR_SHAPE, "head_dim %d must be even in [2, %d]", head_dim, LK_MAX_HEAD_DIM);
  if (max_pos < 0) return fail(LK_ERR_SHAPE, "max_pos %d < 0", max_pos);
  if (!(base > 1.0f) || !std::isfinite(base)) return fail(LK_ERR_INVALID_ARG, "base must be finite and > 1");
  if (max_pos > 0 && !table) return fail(LK_ERR_INVALID_ARG, "null table");
  cudaError_t e = lk::launch_rope_table(table, head_dim, max_pos, (double)base, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lk_rope_table");
  return LK_OK;
}

namespace {
lk_status rope_check(const lk_latent_cache* k, const lk_latent_cache* v, int32_t head_dim, int32_t max_seq_len) {
  lk_status s;
  if ((s = check_cache(k, "k_cache", true)) != LK_OK) return s;
  if ((s = check_cache(v, "v_cache", true)) != LK_OK) return s;
  if (k->batch != v->batch || k->n_heads != v->n_heads || k->capacity != v->capacity)
    return fail(LK_ERR_SHAPE, "k and v caches differ in batch, heads or capacity");
  if (k->code_dtype != v->code_dtype) return fail(LK_ERR_UNSUPPORTED, "k and v caches differ in code dtype");
  if (head_dim < 32 || head_dim > LK_MAX_HEAD_DIM || head_dim % 32 != 0)
    return fail(LK_ERR_SHAPE, "head_dim %d must be a multiple of 32 in [32, %d]", head_dim, LK_MAX_HEAD_DIM);
  if (max_seq_len < 0 || max_seq_len > k->capacity)
    return fail(LK_ERR_SHAPE, "max_seq_len %d outside [0, capacity]", max_seq_len);
  return LK_OK;
}
int rv_max_of(const lk_latent_cache* v) {
  int m = 0;
  for (int h = 0; h < v->n_heads; ++h) m = std::max(m, (int)v->ranks[h]);
  return m;
}
}  // namespace

size_t lk_latent_decode_rope_workspace_bytes(const lk_latent_cache* k, const lk_latent_cache* v, int32_t head_dim,
                                             int32_t max_seq_len) {
  if (rope_check(k, v, head_dim, max_seq_len) != LK_OK) return 0;
  return lk::rope_workspace_bytes(k->batch * k->n_heads, rv_max_of(v), max_seq_len, num_sms());
}

lk_status lk_latent_decode_attn_rope(const lk_latent_cache* k, const lk_latent_cache* v, const void* q,
                                     lk_dtype q_dtype, const void* B_K, const void* B_V, lk_dtype b_dtype,
                                     int32_t head_dim, const int32_t* seq_len, int32_t max_seq_len,
                                     const float* rope_table, float softmax_scale, void* out, lk_dtype out_dtype,
                                     void* workspace, size_t workspace_bytes, lk_stream_t stream) {
  lk_status s;
  if ((s = rope_check(k, v, head_dim, max_seq_len)) != LK_OK) return s;
  if (!q || !B_K || !B_V || !out || !seq_len || !rope_table)
    return fail(LK_ERR_INVALID_ARG, "null q, B_K, B_V, out, seq_len or rope_table");
  if (q_dtype != LK_F32 && q_dtype != LK_BF16) return fail(LK_ERR_DTYPE, "q dtype must be LK_F32 or LK_BF16");
  if (b_dtype != LK_BF16) return fail(LK_ERR_DTYPE, "B dtype must be LK_BF16");
  if (out_dtype != LK_F32 && out_dtype != LK_BF16) return fail(LK_ERR_DTYPE, "out dtype must be LK_F32 or LK_BF16");
  if (!aligned(q, 16) || !aligned(B_K, 16) || !aligned(B_V, 16) || !aligned(rope_table, 16))
    return fail(LK_ERR_ALIGN, "q, B_K, B_V and rope_table must be 16-byte aligned");
  if (!(softmax_scale == softmax_scale)) return fail(LK_ERR_INVALID_ARG, "softmax_scale is NaN");
  const size_t need = lk_latent_decode_rope_workspace_bytes(k, v, head_dim, max_seq_len);
  if (!workspace || workspace_bytes < need)
    return fail(LK_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need, workspace_bytes);
  if (!aligned(workspace, 256)) return fail(LK_ERR_ALIGN, "workspace must be 256-byte aligned");
  lk::RopeLaunch a{};
  a.codes_k = k->codes;
  a.codes_v = v->codes;
  a.scales_k = k->scales;
  a.scales_v = v->scales;
  a.q = q;
  a.BK = B_K;
  a.BV = B_V;
  a.table = rope_table;
  a.seq_len = seq_len;
  a.out = out;
  a.workspace = workspace;
  a.ranks_k = k->ranks;
  a.ranks_v = v->ranks;
  a.kind = k->code_dtype == LK_I8 ? 0 : 1;
  a.batch = k->batch;
  a.n_heads = k->n_heads;
  a.head_dim = head_dim;
  a.capacity = k->capacity;
  a.group_k = k->group;
  a.group_v = v->group;
  a.q_bf16 = q_dtype == LK_BF16;
  a.out_bf16 = out_dtype == LK_BF16;
  a.max_len = max_seq_len;
  a.num_sms = num_sms();
  a.softmax_scale = softmax_scale;
  if (max_seq_len == 0) {
    // nothing to attend: every output is zero
    const size_t ob = (size_t)k->batch * k->n_heads * head_dim * (out_dtype == LK_BF16 ? 2 : 4);
    cudaError_t e = cudaMemsetAsync(out, 0, ob, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "lk_latent_decode_attn_rope");
    return LK_OK;
  }
  cudaError_t e = lk::launch_rope_decode(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lk_latent_decode_attn_rope");
  return LK_OK;
}

lk_status lk_latent_reconstruct_kv(const lk_latent_cache* k, const lk_latent_cache* v, const void* B_K,
                                   const void* B_V, lk_dtype b_dtype, int32_t head_dim, const int32_t* seq_len,
                                   int32_t max_seq_len, void* K_out, void* V_out, lk_stream_t stream) {
  lk_status s;
  if ((s = check_cache(k, "k_cache", true)) != LK_OK) return s;
  if ((s = check_cache(v, "v_cache", true)) != LK_OK) return s;
  if (k->batch != v->batch || k->n_heads != v->n_heads || k->capacity != v->capacity)
    return fail(LK_ERR_SHAPE, "k and v caches differ in batch, heads or capacity");
  if (k->code_dtype != v->code_dtype) return fail(LK_ERR_UNSUPPORTED, "k and v caches differ in code dtype");
  if (!B_K || !B_V || !seq_len || !K_out || !V_out) return fail(LK_ERR_INVALID_ARG, "null B_K, B_V, seq_len or outputs");
  if (b_dtype != LK_BF16) return fail(LK_ERR_DTYPE, "B dtype must be LK_BF16");
  if (head_dim < 16 || head_dim > LK_MAX_HEAD_DIM || head_dim % 16 != 0)
    return fail(LK_ERR_SHAPE, "head_dim %d must be a multiple of 16 in [16, %d]", head_dim, LK_MAX_HEAD_DIM);
  if (max_seq_len < 0 || max_seq_len > k->capacity)
    return fail(LK_ERR_SHAPE, "max_seq_len %d outside [0, capacity]", max_seq_len);
  if (!aligned(K_out, 16) || !aligned(V_out, 16)) return fail(LK_ERR_ALIGN, "K_out and V_out must be 16-byte aligned");
  if (!aligned(B_K, 16) || !aligned(B_V, 16)) return fail(LK_ERR_ALIGN, "B_K and B_V must be 16-byte aligned");
  lk::ReconLaunch a{};
  a.codes[0] = k->codes;
  a.codes[1] = v->codes;
  a.scales[0] = k->scales;
  a.scales[1] = v->scales;
  a.B[0] = B_K;
  a.B[1] = B_V;
  a.out[0] = K_out;
  a.out[1] = V_out;
  a.ranks[0] = k->ranks;
  a.ranks[1] = v->ranks;
  a.group[0] = k->group;
  a.group[1] = v->group;
  a.seq_len = seq_len;
  a.kind = k->code_dtype == LK_I8 ? 0 : 1;
  a.batch = k->batch;
  a.n_heads = k->n_heads;
  a.head_dim = head_dim;
  a.capacity = k->capacity;
  a.max_len = max_seq_len;
  a.b_bf16 = b_dtype == LK_BF16;
  cudaError_t e = lk::launch_reconstruct_kv(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lk_latent_reconstruct_kv");
  return LK_OK;
}

size_t lk_lowrank_workspace_bytes(const lk_lowrank_weight* w, int32_t m) {
  if (!w || m < 0) return 0;
  return lk::lowrank_workspace_bytes(w->k_in, w->n_out, w->rank, w->n_dense, m);
}

lk_status lk_lowrank_linear(const lk_lowrank_weight* w, const int8_t* x_q, const float* x_scale, int32_t m,
                            const uint16_t* residual, void* y, lk_dtype y_dtype, int8_t* t_q_out,
                            float* t_scale_out, void* workspace, size_t workspace_bytes, lk_stream_t stream) {
  if (!w) return fail(LK_ERR_INVALID_ARG, "null weight descriptor");
  if (w->k_in < 1 || w->n_out < 1 || w->rank < 0 || w->n_dense < 0 || w->n_dense > w->k_in)
    return fail(LK_ERR_SHAPE, "bad k_in %d / n_out %d / rank %d / n_dense %d", w->k_in, w->n_out, w->rank,
                w->n_dense);
  const int n_lr = w->k_in - w->n_dense;
  if ((n_lr > 0) != (w->rank > 0))
    return fail(LK_ERR_SHAPE, "a low-rank branch needs both channels (%d) and rank (%d)", n_lr, w->rank);
  if (w->n_dense % 16 || n_lr % 16 || w->rank % 16)
    return fail(LK_ERR_ALIGN, "n_dense, k_in - n_dense and rank must be multiples of 16");
  if (m < 0 || m > 65535) return fail(LK_ERR_SHAPE, "m %d outside [0, 65535]", m);
  if (!x_q || !x_scale || !y) return fail(LK_ERR_INVALID_ARG, "null x_q, x_scale or y");
  if (y_dtype != LK_BF16 && y_dtype != LK_F32) return fail(LK_ERR_DTYPE, "y dtype must be LK_BF16 or LK_F32");
  if (w->n_dense > 0 && (!w->dense_idx || !w->W_D || !w->s_D))
    return fail(LK_ERR_INVALID_ARG, "dense branch needs dense_idx, W_D and s_D");
  if (w->rank > 0 && (!w->lr_idx || !w->U || !w->s_U || !w->V || !w->s_V))
    return fail(LK_ERR_INVALID_ARG, "low-rank branch needs lr_idx, U, s_U, V and s_V");
  if ((w->W_D && !aligned(w->W_D, 16)) || (w->U && !aligned(w->U, 16)) || (w->V && !aligned(w->V, 16)) ||
      (t_q_out && !aligned(t_q_out, 16)))
    return fail(LK_ERR_ALIGN, "int8 weight matrices must be 16-byte aligned");
  if ((t_q_out || t_scale_out) && w->rank == 0)
    return fail(LK_ERR_INVALID_ARG, "t_q_out / t_scale_out need a low-rank branch");
  const size_t need = lk::lowrank_workspace_bytes(w->k_in, w->n_out, w->rank, w->n_dense, m);
  if (!workspace || workspace_bytes < need)
    return fail(LK_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need, workspace_bytes);
  if (!aligned(workspace, 256)) return fail(LK_ERR_ALIGN, "workspace must be 256-byte aligned");
  lk::LowrankLaunch a{};
  a.k_in = w->k_in;
  a.n_out = w->n_out;
  a.rank = w->rank;
  a.n_dense = w->n_dense;
  a.m = m;
  a.dense_idx = w->dense_idx;
  a.lr_idx = w->lr_idx;
  a.W_D = w->W_D;
  a.s_D = w->s_D;
  a.U = w->U;
  a.s_U = w->s_U;
  a.V = w->V;
  a.s_V = w->s_V;
  a.x_q = x_q;
  a.x_scale = x_scale;
  a.residual = residual;
  a.y = y;
  a.y_bf16 = y_dtype == LK_BF16;
  a.t_q_out = t_q_out;
  a.t_scale_out = t_scale_out;
  a.workspace = workspace;
  a.num_sms = num_sms();
  cudaError_t e = lk::launch_lowrank_linear(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lk_lowrank_linear");
  return LK_OK;
}

lk_status lk_quantize_latent(const float* v, int32_t m, int32_t r, lk_dtype code_dtype, int32_t group, void* codes,
                             void* scales, lk_stream_t stream) {
  if (m < 0 || r < 1 || r > LK_MAX_RANK) return fail(LK_ERR_SHAPE, "m %d / r %d outside range", m, r);
  if (code_dtype != LK_I8 && code_dtype != LK_I4) return fail(LK_ERR_DTYPE, "code dtype must be LK_I8 or LK_I4");
  if (code_dtype == LK_I4 && (r % 2 != 0 || group < 1))
    return fail(LK_ERR_SHAPE, "int4 needs an even r and group >= 1");
  if (m > 0 && (!v || !codes || !scales)) return fail(LK_ERR_INVALID_ARG, "null v, codes or scales");
  cudaError_t e = lk::launch_quantize_latent(v, m, r, code_dtype == LK_I8 ? 0 : 1, group, codes, scales,
                                             reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lk_quantize_latent");
  return LK_OK;
}

static lk_status rowquant(int mode, const void* x, const void* x2, lk_dtype dtype, int32_t m, int32_t k, float eps,
                          int8_t* x_q, float* x_scale, lk_stream_t stream, const char* name) {
  if (m < 0 || k < 1 || k > 32768) return fail(LK_ERR_SHAPE, "%s: m %d / k %d outside range", name, m, k);
  if (dtype != LK_F32 && dtype != LK_BF16) return fail(LK_ERR_DTYPE, "%s: dtype must be LK_F32 or LK_BF16", name);
  if (m > 0 && (!x || !x_q || !x_scale || (mode == 2 && !x2)))
    return fail(LK_ERR_INVALID_ARG, "%s: null pointer", name);
  cudaError_t e = lk::launch_rowquant(mode, x, x2, dtype == LK_BF16, m, k, eps, x_q, x_scale,
                                      reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, name);
  return LK_OK;
}

lk_status lk_quantize_rows_i8(const void* x, lk_dtype x_dtype, int32_t m, int32_t k, int8_t* x_q, float* x_scale,
                              lk_stream_t stream) {
  return rowquant(0, x, nullptr, x_dtype, m, k, 0.0f, x_q, x_scale, stream, "lk_quantize_rows_i8");
}

lk_status lk_rmsnorm_quant_i8(const void* x, lk_dtype x_dtype, int32_t m, int32_t k, float eps, int8_t* x_q,
                              float* x_scale, lk_stream_t stream) {
  if (!(eps >= 0.0f)) return fail(LK_ERR_INVALID_ARG, "eps must be >= 0");
  return rowquant(1, x, nullptr, x_dtype, m, k, eps, x_q, x_scale, stream, "lk_rmsnorm_quant_i8");
}

lk_status lk_rmsnorm_hadamard_quant_i8(const void* x, lk_dtype x_dtype, int32_t m, int32_t k, float eps,
                                       int8_t* x_q, float* x_scale, lk_stream_t stream) {
  if (!(eps >= 0.0f)) return fail(LK_ERR_INVALID_ARG, "eps must be >= 0");
  if (k < 1 || (k & (k - 1)) != 0) return fail(LK_ERR_SHAPE, "lk_rmsnorm_hadamard_quant_i8: k %d not a power of two", k);
  return rowquant(3, x, nullptr, x_dtype, m, k, eps, x_q, x_scale, stream, "lk_rmsnorm_hadamard_quant_i8");
}

lk_status lk_swiglu_quant_i8(const void* gate, const void* up, lk_dtype dtype, int32_t m, int32_t n, int8_t* h_q,
                             float* h_scale, lk_stream_t stream) {
  return rowquant(2, gate, up, dtype, m, n, 0.0f, h_q, h_scale, stream, "lk_swiglu_quant_i8");
}

lk_status lk_device_status(int32_t reset) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "lk_device_status");
  cudaError_t (*fns[])(unsigned int*, int) = {lk_decode_status_word, lk_quant_status_word,
                                               lk_project_status_word, lk_lowrank_status_word,
                                               lk_gemm_tc_status_word};
  constexpr int kWords = (int)(sizeof(fns) / sizeof(fns[0]));
  unsigned int words[kWords] = {};
  unsigned int any = 0;
  for (int i = 0; i < kWords; ++i) {
    e = fns[i](&words[i], reset);
    if (e != cudaSuccess) return cuda_fail(e, "lk_device_status");
    any |= words[i];
  }
  if (any) return fail(LK_ERR_DEVICE, "device status word 0x%x (a bounded wait expired)", any);
  return LK_OK;
}

}  // extern "C"
