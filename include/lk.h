/*
 * lk.h — C ABI of the per-head latent-KV decode library (sm_100a).
 *
 * What it computes.  A transformer whose K and V projections are factored per
 * head, W_K^h ~ A_K^h B_K^h and W_V^h ~ A_V^h B_V^h with rank r_h << head dim
 * H, caches only the quantised latents c^h = quant(x A^h) ("WSVD: Weighted
 * Low-Rank Approximation for Fast and Efficient Execution of Low-Precision
 * Vision-Language Models", technical summary §2A per-head SVD and §2C W8A8 /
 * W8A4 and the fused decode kernel; "LASER: Loss-Aware Singular-value
 * Decomposition and Rank Allocation ...", technical summary §2 non-uniform
 * per-head ranks).  A decode step computes softmax(q K^T / sqrt(H)) V with
 * K = dequant(C_K) B_K and V = dequant(C_V) B_V without ever writing K or V
 * to memory: q is absorbed into latent space (q~ = B_K q), scores are taken
 * against the latent codes, and the probability-weighted latent sum is
 * up-projected by B_V once per head.  The LASER hybrid FFN linear
 * (technical summary §3) y = x[:,D] W_D + (x[:,not D] U) V is provided in
 * W8A8 form.
 *
 * Conventions for every entry point.
 *  - All tensor pointers are DEVICE pointers owned by the caller unless the
 *    argument says "host".  The library never allocates, frees or
 *    synchronises device memory; scratch space is passed in as `workspace`.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).
 *  - Every call validates its arguments on the host first and returns an
 *    error status WITHOUT launching anything or writing any output if a check
 *    fails.  lk_last_error() then holds a one-line explanation (per host
 *    thread).  A CUDA launch error is reported as LK_ERR_CUDA.
 *  - Device pointers must be 16-byte aligned unless stated otherwise; the
 *    latent cache planes and workspaces must be 256-byte aligned.
 *  - Weight matrices are stored [out_features, in_features], row-major
 *    (each output's weights contiguous), like torch.nn.Linear.weight.
 *  - fp16 / bf16 values are passed as 16-bit storage (uint16_t bit patterns).
 */
#ifndef LK_H_
#define LK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so callers need no CUDA header. */
typedef struct CUstream_st* lk_stream_t;

typedef enum {
  LK_OK = 0,
  LK_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad enum          */
  LK_ERR_SHAPE = 2,       /* sizes inconsistent or outside supported range  */
  LK_ERR_DTYPE = 3,       /* dtype not supported for this argument          */
  LK_ERR_ALIGN = 4,       /* pointer or size not aligned as required        */
  LK_ERR_CAPACITY = 5,    /* append would overrun the cache capacity        */
  LK_ERR_UNSUPPORTED = 6, /* valid request the library does not implement   */
  LK_ERR_WORKSPACE = 7,   /* workspace null or smaller than required        */
  LK_ERR_CUDA = 8,        /* a CUDA call failed (text in lk_last_error)     */
  LK_ERR_DEVICE = 9       /* a kernel reported a bounded wait that expired  */
} lk_status;

typedef enum {
  LK_F32 = 0,
  LK_BF16 = 1,
  LK_F16 = 2,
  LK_I8 = 3, /* int8 codes: r codes per (token, head), one fp32 scale        */
  LK_I4 = 4  /* int4 codes: two per byte (low nibble = even dim), one fp16
                scale per group of g consecutive dims                         */
} lk_dtype;

#define LK_MAX_HEADS 128 /* heads per layer                                   */
#define LK_MAX_RANK 64   /* latent rank per head for attention               */
#define LK_MAX_HEAD_DIM 256

/*
 * Latent cache of one layer, for K or for V (caller-owned device memory).
 *
 * Ranks: ranks[h] = r_h (HOST array, read during the call only).  int8 caches
 * need r_h % 4 == 0, int4 caches r_h % 8 == 0, 4 <= r_h <= LK_MAX_RANK.  The K
 * and V caches of a layer may have different ranks (LASER allocates them
 * independently).
 *
 * Row bytes of head h: rb_h = r_h (int8) or r_h / 2 (int4).  Scale groups:
 * ng_h = 1 (int8) or ceil(r_h / min(group, r_h)) (int4).
 *
 * codes: for batch row b and head h, one contiguous plane of capacity * rb_h
 *   bytes at byte offset (b * sum_h rb_h + sum_{h' < h} rb_h') * capacity.
 *   Inside a plane, tokens are kept in blocks of 16 (16 * rb bytes each);
 *   the order inside a block depends on the cache's role:
 *   K caches (token-major chunks): with chunk size cs = 16 if rb % 16 == 0,
 *     else 8 if rb % 8 == 0, else 4, byte k of token t's code row sits at
 *       (t / 16) * 16 * rb + (k / cs) * 16 * cs + (t % 16) * cs + (k % cs)
 *     (a reader with one thread per token touches consecutive words);
 *   V caches (dimension-major): int8: the code of dim d of token t sits at
 *       (t / 16) * 16 * rb + d * 16 + (t % 16);
 *     int4: byte (t / 16) * 16 * rb + d * 8 + (t % 16) / 2 holds dim d of
 *     tokens 2i (low nibble) and 2i + 1 (high nibble)
 *     (one 32-bit word then holds 4 or 8 consecutive tokens of one dim).
 * scales: int8: fp32 [capacity] per (b, h) at element offset
 *   (b * n_heads + h) * capacity.  int4: fp16 [capacity][ng_h] per (b, h)
 *   at element offset (b * sum_h ng_h + sum_{h' < h} ng_h') * capacity.
 * capacity must be a multiple of 16.
 */
typedef struct {
  int32_t batch;        /* B                                                */
  int32_t n_heads;      /* n_h <= LK_MAX_HEADS                              */
  int32_t capacity;     /* T_max, multiple of 16                            */
  lk_dtype code_dtype;  /* LK_I8 or LK_I4                                   */
  int32_t group;        /* int4 group size along r (effective min(g, r_h))  */
  const int32_t* ranks; /* HOST [n_heads]                                   */
  void* codes;          /* device, 256-byte aligned                        */
  void* scales;         /* device, 256-byte aligned                        */
  int32_t rotation;     /* 0 or 1; see below                                */
} lk_latent_cache;

/*
 * rotation = 1 (WSVD §2C: an orthogonal S2 applied to the latent smooths its
 * outlier channels before round-to-nearest): lk_latent_project_append
 * multiplies each head's fp32 latent v^h by S2_h before quantising it, where
 * S2_h is block diagonal with normalised Walsh-Hadamard blocks of order n =
 * the largest power of two dividing r_h, capped at 64 (S2_h = S2_h^T =
 * S2_h^-1).  The cache then holds codes of v^h S2_h; since
 * (v S2)(S2 B) = v B, the decode entry points stay unchanged when they are
 * given the counter-rotated factors S2_h B_K^h and S2_h B_V^h.  Folding S2
 * into A offline (A^h S2_h) gives the same cache without this flag.  Only
 * the append reads the flag; 0 is the plain cache.
 */

/* Bytes the caller must allocate for a cache's code and scale planes. */
lk_status lk_latent_cache_bytes(const lk_latent_cache* cache, size_t* codes_bytes,
                                size_t* scales_bytes);

/*
 * Latent projection + quantisation + append (WSVD §2A: the per-head latent
 * x A^h is what is cached; §2C: it is stored in 8 or 4 bits; LASER §4 fuses
 * projection, latent generation and quantisation).
 *
 * x: [B * n_new, embed_dim] row-major, row b * n_new + t is batch row b's
 *   t-th new token.  x_dtype LK_F32, LK_BF16 or LK_I8 (then x_scale, fp32
 *   [B * n_new], is the per-token dequantisation scale; else NULL).
 * A: [N_tot, embed_dim] (K-major), N_tot = sum r_K + sum r_V: rows are the
 *   K heads' latent dims in head order, then the V heads'.  a_dtype must
 *   equal x_dtype; for LK_I8, a_scale is fp16 [N_tot] (per latent dim).
 * For every new token and head the latent v^h (fp32) is quantised with the
 *   cache's rule (see lk_quantize_latent) and written at position
 *   seq_len[b] + t.  Float inputs: v is the fp32 dot product.  LK_I8 inputs:
 *   v = fl32(fl32(fl32(sum x_q A_q) * x_scale) * a_scale), exact int32 sum.
 * seq_len: device int32 [B], read as the write offset, then increased by
 *   n_new once every token is written.  seq_len_host: HOST copy of the same
 *   values, used for the capacity check seq_len + n_new <= capacity.
 * workspace: lk_latent_project_workspace_bytes(...) bytes, 256-B aligned;
 *   its first 2048 bytes are arrival counters that must be zero before the
 *   first call and that every completed call leaves zero.
 */
lk_status lk_latent_project_append(const lk_latent_cache* k_cache, const lk_latent_cache* v_cache,
                                   const void* x, lk_dtype x_dtype, const float* x_scale,
                                   const void* A, lk_dtype a_dtype, const uint16_t* a_scale,
                                   int32_t embed_dim, int32_t n_new, int32_t* seq_len,
                                   const int32_t* seq_len_host, void* workspace,
                                   size_t workspace_bytes, lk_stream_t stream);
size_t lk_latent_project_workspace_bytes(const lk_latent_cache* k_cache,
                                         const lk_latent_cache* v_cache, int32_t embed_dim,
                                         int32_t n_new, lk_dtype x_dtype);

/*
 * Latent decode attention (WSVD §2C fused kernel; absorption form).
 *
 * For each batch row b and head h, over positions t in [0, seq_len[b]):
 *   q~ = B_K^h q^h                                  (absorb q, r_K values)
 *   s_t = softmax_scale * sigma_K[t] . (c_K[t] . q~)   (per group for int4)
 *   p = softmax(s);  u = sum_t p_t * sigma_V[t] * c_V[t]   (r_V values)
 *   out^h = u B_V^h                                  ([H])
 * computed split-K over t (flash-decoding): the (b, h, stage) items
 * (448-token stages, or 224 where two 448-token stages of the widest head
 * do not fit in shared memory) are dealt out in equal ranges to a fixed
 * grid of CTAs; a (b, h) cut by a range boundary leaves partials (max, sum,
 * u) that are merged in latent space by the last piece to finish.  K and V
 * are never formed.
 *
 * q: [B, n_heads, head_dim], q_dtype LK_F32 or LK_BF16; head_dim a multiple
 *   of 8 (<= LK_MAX_HEAD_DIM); q, B_K and B_V 16-byte aligned (they are
 *   staged into shared memory with bulk copies).
 * B_K, B_V: per-head factors [r_h, head_dim] row-major, packed head after
 *   head (head h starts at element sum_{h'<h} r_h' * head_dim); b_dtype
 *   LK_F32 or LK_BF16.
 * seq_len: device [B] (values may differ per row); max_seq_len: HOST upper
 *   bound on those values (<= capacity); positions past it are not read.
 *   A row with seq_len 0 gets a zero output.
 * out: [B, n_heads, head_dim], LK_F32 or LK_BF16.
 * n_split: about how many pieces each (b, h) is cut into (grid = B * n_heads
 *   * n_split CTAs, at most one per stage); 0 picks a grid that
 *   fills the GPU.  The result does not depend on it beyond float rounding.
 * workspace: lk_latent_decode_workspace_bytes(...) bytes, 256-B aligned.
 *   Its first round_up(4 * B * n_heads, 256) bytes are per-(b, h) arrival
 *   counters that must read zero at entry (a fresh zeroed buffer); every
 *   completed call leaves them zero, so a replayed launch (CUDA graph) also
 *   starts clean.  The partials that follow may cover the counters of a call
 *   with another B * n_heads: clear that region before reusing a workspace
 *   for another shape.  Calls sharing a workspace must not overlap on the GPU.
 */
lk_status lk_latent_decode_attn(const lk_latent_cache* k_cache, const lk_latent_cache* v_cache,
                                const void* q, lk_dtype q_dtype, const void* B_K,
                                const void* B_V, lk_dtype b_dtype, int32_t head_dim,
                                const int32_t* seq_len, int32_t max_seq_len,
                                float softmax_scale, void* out, lk_dtype out_dtype,
                                int32_t n_split, void* workspace, size_t workspace_bytes,
                                lk_stream_t stream);
size_t lk_latent_decode_workspace_bytes(const lk_latent_cache* k_cache,
                                        const lk_latent_cache* v_cache, int32_t max_seq_len,
                                        int32_t n_split);

/*
 * Latent decode attention for callers that cannot allocate device memory
 * (no counterpart in the paper).  Some callers cannot call cudaMalloc or
 * hand out scratch buffers -- for example code running under an allocator
 * that forbids new device allocations, or a host runtime that only passes
 * tensors it already owns.  This variant takes the same arguments as
 * lk_latent_decode_attn minus the workspace and keeps its split-K scratch
 * (arrival counters + per-split partials) in a static device array of
 * LK_DECODE_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that
 * loads the library holds until the process exits.  It allocates nothing
 * and calls no allocating routine; inputs and outputs are still the
 * caller's.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - A request whose scratch would exceed LK_DECODE_NOALLOC_SCRATCH_BYTES is
 *    rejected with LK_ERR_WORKSPACE (lk_last_error says how much it needs);
 *    lower n_split or use lk_latent_decode_attn with a workspace.
 *  - All calls share the one array: calls that overlap on the GPU (other
 *    streams, other host threads) race on it.  Serialise them.
 *  - The arrival counters in the array start at zero when the library loads
 *    and every completed call leaves them zero.  A call first clears them on
 *    `stream` when its B * n_heads differs from the device's last accepted
 *    call, when the last call failed, and always while `stream` is being
 *    captured (a replay may follow direct calls of any shape).  A rejected
 *    call launches nothing and leaves the array as it was.
 */
#define LK_DECODE_NOALLOC_SCRATCH_BYTES (4u << 20)
lk_status lk_latent_decode_attn_noalloc(const lk_latent_cache* k_cache, const lk_latent_cache* v_cache,
                                        const void* q, lk_dtype q_dtype, const void* B_K,
                                        const void* B_V, lk_dtype b_dtype, int32_t head_dim,
                                        const int32_t* seq_len, int32_t max_seq_len,
                                        float softmax_scale, void* out, lk_dtype out_dtype,
                                        int32_t n_split, lk_stream_t stream);

/*
 * One decode step of the latent-KV attention: lk_latent_project_append of
 * one new token per batch row (x: [B, embed_dim]), then
 * lk_latent_decode_attn over positions [0, seq_len_host[b] + 1) (the new
 * token included; max_seq_len = max_b seq_len_host[b] + 1).  The arguments
 * mean what they mean for those two calls.
 * The attention kernel is launched so that it may start while the append
 * still runs: it fetches q, B_K and B_V (and absorbs q) before it waits for
 * the append, and reads the cache and seq_len only after.  q, B_K and B_V
 * must therefore be complete before this call's first kernel starts (they
 * are never written by the append).  All arguments are validated before
 * anything is launched.
 */
lk_status lk_latent_decode_step(const lk_latent_cache* k_cache, const lk_latent_cache* v_cache,
                                const void* x, lk_dtype x_dtype, const float* x_scale,
                                const void* A, lk_dtype a_dtype, const uint16_t* a_scale,
                                int32_t embed_dim, int32_t* seq_len, const int32_t* seq_len_host,
                                const void* q, lk_dtype q_dtype, const void* B_K, const void* B_V,
                                lk_dtype b_dtype, int32_t head_dim, float softmax_scale, void* out,
                                lk_dtype out_dtype, int32_t n_split, void* project_workspace,
                                size_t project_workspace_bytes, void* decode_workspace,
                                size_t decode_workspace_bytes, lk_stream_t stream);

/*
 * Dense bf16 flash-decoding over materialised K and V: the baseline the
 * pages measure their decode speed-ups against (WSVD technical summary §4:
 * speed-up over flash decoding; LASER results).  For every batch row b and
 * head h, out = softmax(q K^T * softmax_scale) V over positions
 * [0, seq_len[b]), split over the tokens like lk_latent_decode_attn.
 * q: bf16 [B, n_heads, head_dim]; K, V: bf16 [B, n_heads, capacity,
 * head_dim] (one row per position); head_dim a multiple of 8 up to 256;
 * q, K, V 16-byte aligned.  out: [B, n_heads, head_dim] LK_F32 or LK_BF16.
 * workspace: lk_dense_decode_workspace_bytes(...) bytes, 256-B aligned, its
 * first round_up(4 * B * n_heads, 256) bytes zero at entry (left zero).
 */
lk_status lk_dense_decode_attn(const void* q, const void* K, const void* V, int32_t batch, int32_t n_heads,
                               int32_t head_dim, int32_t capacity, const int32_t* seq_len,
                               int32_t max_seq_len, float softmax_scale, void* out, lk_dtype out_dtype,
                               void* workspace, size_t workspace_bytes, lk_stream_t stream);
size_t lk_dense_decode_workspace_bytes(int32_t batch, int32_t n_heads, int32_t head_dim, int32_t max_seq_len);

/*
 * Rotary positions (an extension: neither page uses a positional encoding).
 *
 * lk_rope_table: table[t][i] = (cos a, sin a), a = t * base^(-2 i / head_dim),
 * for t < max_pos and i < head_dim / 2, computed in float64 and stored fp32
 * ([max_pos][head_dim / 2][2], device, written on `stream`).  base > 1.
 *
 * lk_latent_decode_attn_rope: latent decode attention for a model that
 * rotates keys and queries (rotate-half pairs (i, i + H/2)).  The rotation
 * of a key depends on its position, so q cannot be absorbed into B_K: each
 * key is rebuilt from its latent code on chip (the WSVD page's fused kernel
 * rebuilds K_h on chip, technical summary §2C).  For batch row b, head h,
 * positions t < len = min(seq_len[b], max_seq_len):
 *   K_t = dequant(c_K[t]) B_K^h, rotated by the table row t;
 *   q rotated by the table row len - 1 (the newest cached position);
 *   s_t = (rot q) . (rot K_t) * softmax_scale;  p = softmax(s);
 *   out = (sum_t p_t dequant(c_V[t])) B_V^h   (values are not rotated).
 * Caches and their layouts as for lk_latent_decode_attn (the rotation flag
 * of a cache is not read here).  q: [B, n_heads, head_dim] LK_F32 or
 * LK_BF16; B_K, B_V: bf16 (b_dtype LK_BF16), packed per head as for
 * lk_latent_decode_attn; head_dim a multiple of 32 (<= LK_MAX_HEAD_DIM);
 * rope_table: an lk_rope_table table of the same head_dim with at least
 * max(max_seq_len, 16) rows (the kernel takes the angles of positions inside
 * a 16-token block from the block's row and rows 0..15 by the angle-sum
 * identities, in fp32); q, B_K, B_V, rope_table 16-byte aligned.  out:
 * [B, n_heads, head_dim] LK_F32 or LK_BF16; rows with len = 0 are zero.
 * workspace: lk_latent_decode_rope_workspace_bytes(...) bytes, 256-byte
 * aligned, its first round_up(4 * B * n_heads, 256) bytes zero at entry
 * (left zero by every completed call).  The keys are rebuilt with exact
 * bf16 products summed in fp32; everything after is fp32.
 */
lk_status lk_rope_table(int32_t head_dim, int32_t max_pos, float base, float* table, lk_stream_t stream);
lk_status lk_latent_decode_attn_rope(const lk_latent_cache* k_cache, const lk_latent_cache* v_cache,
                                     const void* q, lk_dtype q_dtype, const void* B_K, const void* B_V,
                                     lk_dtype b_dtype, int32_t head_dim, const int32_t* seq_len,
                                     int32_t max_seq_len, const float* rope_table, float softmax_scale,
                                     void* out, lk_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                     lk_stream_t stream);
size_t lk_latent_decode_rope_workspace_bytes(const lk_latent_cache* k_cache, const lk_latent_cache* v_cache,
                                             int32_t head_dim, int32_t max_seq_len);

/*
 * The naive low-rank path the WSVD page contrasts with its fused kernel
 * (technical summary §1: rebuilding K and V from the factors through
 * memory costs more than it saves): for positions [0, seq_len[b]),
 *   K_out[b, h, t, :] = dequant(c_K[b, h, t]) B_K^h,  V_out likewise,
 * stored bf16 [B, n_heads, capacity, head_dim] (rows past seq_len[b] are not
 * written).  Caches and their layouts as for lk_latent_decode_attn; B_K and
 * B_V bf16 (b_dtype LK_BF16, else LK_ERR_DTYPE), 16-byte aligned; head_dim a
 * multiple of 16.  Each value is the fp32 sum of exact code x factor
 * products (per scale group, times the group's scale), rounded once to bf16.
 * Attending the result with lk_dense_decode_attn gives the same output as
 * lk_latent_decode_attn up to the bf16 rounding of K and V.
 */
lk_status lk_latent_reconstruct_kv(const lk_latent_cache* k_cache, const lk_latent_cache* v_cache,
                                   const void* B_K, const void* B_V, lk_dtype b_dtype, int32_t head_dim,
                                   const int32_t* seq_len, int32_t max_seq_len, void* K_out, void* V_out,
                                   lk_stream_t stream);

/*
 * LASER hybrid dense + low-rank linear, W8A8 (LASER technical summary §3:
 * selected input channels go through SVD factors, the rest stay dense; both
 * branches RTN-quantised).
 *
 *   acc_D = x_q[:, dense_idx] W_D^T            (exact int32)
 *   t     = fl32(fl32(fl32(x_q[:, lr_idx] U^T) * x_scale) * s_U)
 *   (t_q, s_t) = per-token int8 absmax quantisation of t
 *   acc_V = t_q V^T                            (exact int32)
 *   y     = acc_D * x_scale * s_D + acc_V * s_t * s_V (+ residual), fp32,
 *           stored as y_dtype.
 * rank == 0 with n_dense == k_in is a plain W8A8 linear.
 */
typedef struct {
  int32_t k_in;              /* input channels                                 */
  int32_t n_out;             /* output channels                                */
  int32_t rank;              /* low-rank width R (0 = no low-rank branch)      */
  int32_t n_dense;           /* |D|                                            */
  const int32_t* dense_idx;  /* device [n_dense], sorted, disjoint from lr_idx */
  const int32_t* lr_idx;     /* device [k_in - n_dense], sorted                */
  const int8_t* W_D;         /* [n_out, n_dense]                               */
  const uint16_t* s_D;       /* fp16 [n_out]                                   */
  const int8_t* U;           /* [rank, k_in - n_dense]                         */
  const uint16_t* s_U;       /* fp16 [rank]                                    */
  const int8_t* V;           /* [n_out, rank]                                  */
  const uint16_t* s_V;       /* fp16 [n_out]                                   */
} lk_lowrank_weight;

/* x_q: int8 [m, k_in]; x_scale fp32 [m]; residual: bf16 [m, n_out] or NULL;
 * y: [m, n_out] LK_BF16 or LK_F32; t_q_out / t_scale_out: optional
 * ([m, rank] int8, [m] fp32) copies of the requantised latent;
 * workspace: lk_lowrank_workspace_bytes(w, m) bytes. */
lk_status lk_lowrank_linear(const lk_lowrank_weight* w, const int8_t* x_q, const float* x_scale,
                            int32_t m, const uint16_t* residual, void* y, lk_dtype y_dtype,
                            int8_t* t_q_out, float* t_scale_out, void* workspace,
                            size_t workspace_bytes, lk_stream_t stream);
size_t lk_lowrank_workspace_bytes(const lk_lowrank_weight* w, int32_t m);

/*
 * The FFN input side with the hybrid split on OUTPUT (hidden) channels
 * (LASER technical summary §3: the selected hidden channels keep dense
 * weights, the rest come from the SVD factors; §4: the input projections,
 * the latent activation and SwiGLU fused), W8A8.  Gate and up keep the same
 * hidden channels dense: dense_out (device int32 [n_dense]) lists them, in
 * the order of the W_D rows, and lr_out (device int32 [n_out - n_dense]) the
 * others, in the order of the V rows; together they cover [0, n_out) once.
 * For each token row m and projection P in {gate, up}:
 *   channel dense_out[i]: P = fl32(fl32(acc * s_x[m]) * s_D[i]),
 *                         acc = x_q[m] . W_D[i]                (exact int32)
 *   latent:   t = fl32(fl32(fl32(x_q[m] . U[k]) * s_x[m]) * s_U[k]), k < rank,
 *             requantised per token with the int8 absmax rule -> (t_q, s_t)
 *   channel lr_out[i]:    P = fl32(fl32(acc * s_t[m]) * s_V[i]), acc = t_q . V[i]
 *   out[m][j] = silu(gate_j) * up_j = gate_j / (1 + exp(-gate_j)) * up_j  (fp32)
 * Launches: the two latent products (tcgen05 int8 GEMM), one requantisation
 * of both, then one launch for gate, up and SwiGLU together.
 * Weights (per projection): W_D int8 [n_dense][k_in], U int8 [rank][k_in],
 * V int8 [n_out - n_dense][rank] (rows contiguous along the contraction),
 * fp16 scales; all 16-byte aligned.  k_in and rank multiples of 16; rank > 0
 * exactly when n_dense < n_out.  x_q int8 [m][k_in] (16-byte aligned),
 * x_scale fp32 [m]; out fp32 [m][n_out].  workspace:
 * lk_ffn_gate_up_swiglu_workspace_bytes(...) bytes, 256-byte aligned.
 */
typedef struct {
  const int8_t* W_D;
  const uint16_t* s_D;
  const int8_t* U;
  const uint16_t* s_U;
  const int8_t* V;
  const uint16_t* s_V;
} lk_outsplit_weight;

lk_status lk_ffn_gate_up_swiglu(const lk_outsplit_weight* gate, const lk_outsplit_weight* up, int32_t k_in,
                                int32_t n_out, int32_t n_dense, int32_t rank, const int32_t* dense_out,
                                const int32_t* lr_out, const int8_t* x_q, const float* x_scale, int32_t m,
                                float* out, void* workspace, size_t workspace_bytes, lk_stream_t stream);
size_t lk_ffn_gate_up_swiglu_workspace_bytes(int32_t rank, int32_t m);

/*
 * Stand-alone latent quantiser (the rule lk_latent_project_append applies),
 * exposed for bit-exact testing.  v: fp32 [m, r].
 *  LK_I8: scale = fl32(absmax / 127); code = clamp(rint(fl32(v / scale)),
 *    -127, 127) (round half to even); scale 0 gives zero codes.
 *    codes int8 [m, r]; scales fp32 [m].
 *  LK_I4: per group of g = min(group, r) dims: scale16 = fp16_rn(fl32(absmax /
 *    7)) saturated to 65504; code = clamp(rint(fl32(v / scale)), -7, 7);
 *    codes packed [m, r / 2] (low nibble = even dim); scales fp16
 *    [m, ceil(r / g)].  r must be even.
 */
lk_status lk_quantize_latent(const float* v, int32_t m, int32_t r, lk_dtype code_dtype,
                             int32_t group, void* codes, void* scales, lk_stream_t stream);

/* Per-row int8 absmax quantisation of activations (same rule as LK_I8
 * above).  x: [m, k] LK_F32 or LK_BF16; x_q int8 [m, k]; x_scale fp32 [m]. */
lk_status lk_quantize_rows_i8(const void* x, lk_dtype x_dtype, int32_t m, int32_t k,
                              int8_t* x_q, float* x_scale, lk_stream_t stream);

/* RMSNorm with unit weight, y = x / sqrt(mean(x^2) + eps), then per-row int8
 * quantisation of y (fp32).  x: [m, k] LK_F32 or LK_BF16. */
lk_status lk_rmsnorm_quant_i8(const void* x, lk_dtype x_dtype, int32_t m, int32_t k, float eps,
                              int8_t* x_q, float* x_scale, lk_stream_t stream);

/* S1 on the input of the latent projection (WSVD §2C: S1 is a Hadamard
 * matrix applied to the input to smooth its outlier channels):
 * y = RMSNorm(x) H_k with H_k the normalised Walsh-Hadamard matrix of order
 * k (k a power of two, <= 32768), then per-row int8 quantisation of y as in
 * lk_quantize_rows_i8.  The projection weight must then be H_k A (H_k is
 * symmetric and orthogonal), so y (H_k A) = RMSNorm(x) A.  The transform is
 * fp32 butterflies (log2 k adds per element, then one multiply by
 * fl32(1 / sqrt(k))).  x: [m, k] LK_F32 or LK_BF16; x_q int8 [m, k];
 * x_scale fp32 [m].  LK_ERR_SHAPE when k is not a power of two. */
lk_status lk_rmsnorm_hadamard_quant_i8(const void* x, lk_dtype x_dtype, int32_t m, int32_t k, float eps,
                              int8_t* x_q, float* x_scale, lk_stream_t stream);

/* SwiGLU h = silu(gate) * up in fp32 (LASER §4 fuses it into the FFN), then
 * per-row int8 quantisation of h.  gate, up: [m, n] LK_F32 or LK_BF16. */
lk_status lk_swiglu_quant_i8(const void* gate, const void* up, lk_dtype dtype, int32_t m,
                             int32_t n, int8_t* h_q, float* h_scale, lk_stream_t stream);

/*
 * Test hook for the failure path (no counterpart on the pages): the decode
 * attention of lk_latent_decode_attn (same arguments and validation), with its
 * copy producer told to stop before work item `stall_item` (>= 0; items are
 * (b, h) units times stages of 224 or 448 tokens) as if that copy never
 * arrived, and every pipeline wait bounded by `wait_us` microseconds instead
 * of the default 2 s.  The waits behind the missing copy expire, the kernel
 * lets every copy it did start land (allowing 2 s for each) and returns;
 * `out` then holds no meaningful values, the workspace counters are left
 * zero, and lk_device_status() reports LK_ERR_DEVICE.  No other entry point
 * reaches this path.
 */
lk_status lk_debug_decode_attn_stall(const lk_latent_cache* k_cache, const lk_latent_cache* v_cache,
                                     const void* q, lk_dtype q_dtype, const void* B_K, const void* B_V,
                                     lk_dtype b_dtype, int32_t head_dim, const int32_t* seq_len,
                                     int32_t max_seq_len, float softmax_scale, void* out, lk_dtype out_dtype,
                                     int32_t n_split, void* workspace, size_t workspace_bytes,
                                     int32_t stall_item, uint32_t wait_us, lk_stream_t stream);

/* Synchronises the device, then reports (and with reset != 0 clears) the
 * error word kernels set when a bounded wait expires: LK_OK or LK_ERR_DEVICE. */
lk_status lk_device_status(int32_t reset);

const char* lk_status_string(lk_status status);
const char* lk_last_error(void);
int32_t lk_version(void);

/* Number of kernels this library has enqueued in this process so far, over
 * all devices, streams and host threads (memsets not counted).  The
 * difference across a region of calls is how many of the library's kernels
 * that region launched (no counterpart on the pages: instrumentation). */
uint64_t lk_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* LK_H_ */
