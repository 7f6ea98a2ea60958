/*
 * mla.h -- C ABI of the B200 (sm_100a) library for absorbed Multi-head Latent
 * Attention decode over a paged latent cache ("libmla_b200.so").
 *
 * What the library computes (one decode step of one attention layer, per
 * sequence b with a new token at position pos_b):
 *
 *   mla_cache_append   c = RMSNorm(W_DKV h), k_R = RoPE_pos(W_KR h); writes the
 *                      row [c ; k_R] into the paged cache.
 *   mla_absorb_q       c_Q = W_DQ h (optional), q_C = W_UQ c_Q,
 *                      q_R = RoPE_pos(W_QR c_Q), q_lat_i = [W_UK,i^T q_C,i ; q_R,i].
 *   mla_decode_attn    z_i = sum_s softmax_s(scale * q_lat_i . row_s) c_s over all
 *                      rows of the sequence (its own new row included).
 *   mla_unabsorb_out   o_i = W_UV,i z_i, optionally u = W_O concat_i o_i.
 *
 * Sources (web pages on the method, by title and section):
 *   "解耦 RoPE（MLA 下）" (Decoupled RoPE, MLA part 2): §三 the split score
 *     content + position, §3.3 one k_R shared by all heads, §3.4 k_R cached
 *     already rotated, §五 the five inference steps, §六 576 values per token.
 *   "从零理解 MLA": 低秩联合压缩 (c = W^DKV h), 矩阵吸收 (absorption on both
 *     sides), 查询压缩 (c_Q = W^DQ h, q^C = W^UQ c_Q), 解耦 RoPE (q^R, k^R, the
 *     sqrt(d_head + d_r) scale, absorbed_step with a [c ; k_R] cache row),
 *     实际配置 (DeepSeek-V2 sizes and the extra RMSNorm on the latent).
 *   "Hands-on DeepSeek MLA": the RMSNorm (mean of squares, eps 1e-6).
 *
 * Conventions shared by every call
 *   - `dims` and `cache` point to HOST structs read during the call; every
 *     other pointer (including the ones inside `cache`) is a DEVICE pointer.
 *     The caller owns every buffer; the library never
 *     allocates, frees or synchronises inside the compute calls.  All work is
 *     enqueued on `stream` and is asynchronous.
 *   - Element types: `dims->dtype` selects bf16 (MLA_BF16) or fp32 (MLA_FP32)
 *     for every "void*" tensor (weights, activations, cache, outputs).  `lse`
 *     is always fp32; positions, block tables and lengths are int32.
 *   - Weights use the [out, in] row-major layout of a linear layer.  W_UK is
 *     [n_heads * d_nope, d_c] and W_UV is [n_heads * d_v, d_c], read per head as
 *     [n_heads][d_nope | d_v][d_c].
 *   - Host-side checks run before anything is launched and return a non-OK
 *     status with no side effect: null pointers, sizes, 16-byte alignment of
 *     every tensor, workspace size, supported shapes.
 *   - Device-side checks (page-table entries outside [0, num_pages), seq_len <= 0,
 *     positions outside the sequence's pages) skip the offending sequence (its
 *     outputs are zeroed, nothing is written out of bounds) and set the error
 *     word in the workspace; read it with mla_get_device_error().
 *   - Supported shapes: MLA_FP32 accepts any n_heads <= 256, d_c <= 1024 (a
 *     multiple of 4), d_rope <= 128 (even), d_nope, d_v <= 256, page_size >= 1.  MLA_BF16
 *     requires the DeepSeek-V2 attention sizes n_heads = 128, d_c = 512,
 *     d_rope = 64, d_nope = d_v = 128, page_size = 64, and d_model, d_q
 *     multiples of 64; other shapes return MLA_ERR_UNSUPPORTED.
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *mla_stream_t;  /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, bad enum      */
  MLA_ERR_UNSUPPORTED = 2,   /* shape outside the supported set (see above)    */
  MLA_ERR_ALIGNMENT = 3,     /* a tensor pointer is not 16-byte aligned        */
  MLA_ERR_WORKSPACE = 4,     /* workspace null or smaller than required        */
  MLA_ERR_CUDA = 5,          /* a CUDA runtime call failed (launch, copy ...)  */
  MLA_ERR_DEVICE_RANGE = 6,  /* device check: bad page entry, length, position */
  MLA_ERR_TIMEOUT = 7        /* device check: a bounded wait gave up           */
} mla_status;

enum { MLA_BF16 = 0, MLA_FP32 = 1 };
enum { MLA_ROPE_INTERLEAVED = 0, MLA_ROPE_HALF = 1 };

/* Cache row formats.
 *   MLA_CACHE_NATIVE: a row is [c ; k_R] in dims->dtype (d_c + d_rope values).
 *   MLA_CACHE_INT8 (MLA_BF16 only): the KV cache stored at lower precision
 *     ("DeepSeek-V3多头潜在注意力(MLA)架构", 多头潜在注意力与KV缓存优化: INT8 or
 *     INT4 keys and values).  A row is MLA_INT8_ROW_BYTES = 656 bytes:
 *       bytes [0, 512)    c as int8 codes q_j in [-127, 127],
 *       bytes [512, 640)  k_R as 64 bf16 values (not quantised),
 *       bytes [640, 644)  the row's scale s = 2^e as an fp32 value,
 *       bytes [644, 656)  zero.
 *     The row holds c_j = q_j * s with e the smallest integer such that
 *     max_j |c_j| <= 127 * 2^e, q_j = round-half-even(c_j / s).  Because s is a
 *     power of two, q_j * s is exactly representable in bf16: decode attention
 *     over an int8 cache computes exactly what it computes over the bf16 rows
 *     [q * s ; k_R]. */
enum { MLA_CACHE_NATIVE = 0, MLA_CACHE_INT8 = 1 };
enum { MLA_INT8_ROW_BYTES = 656 };

/* Sizes of one MLA layer.
 *   n_heads, d_nope (per-head content query/key width), d_v (per-head value
 *   width), d_c (latent width), d_rope (decoupled RoPE width, shared key).
 *   page_size: rows per cache page.
 *   rope_layout: MLA_ROPE_INTERLEAVED pairs (0,1),(2,3),... ("解耦 RoPE（MLA 下）"
 *   §七 rope); MLA_ROPE_HALF pairs (i, i + d_rope/2) ("从零理解 MLA", 解耦 RoPE
 *   apply_rope).  Frequencies theta_i = rope_base^(-2i/d_rope).
 *   rms_eps: RMSNorm epsilon (1e-6 on the pages).
 *   softmax_scale: 0 selects 1/sqrt(d_nope + d_rope) ("从零理解 MLA", 解耦 RoPE). */
typedef struct {
  int n_heads, d_c, d_rope, d_nope, d_v, page_size;
  int dtype;        /* MLA_BF16 | MLA_FP32 */
  int rope_layout;  /* MLA_ROPE_INTERLEAVED | MLA_ROPE_HALF */
  double rope_base, rms_eps, softmax_scale;
  int cache_format; /* MLA_CACHE_NATIVE (0) | MLA_CACHE_INT8 */
} mla_dims;

/* The paged latent cache (device memory, caller-owned).
 *   pool: [num_pages][page_size][d_c + d_rope] elements of dims->dtype; a row is
 *         [c (d_c) ; k_R (d_rope)] ("从零理解 MLA", 解耦 RoPE absorbed_step caches
 *         cat([c_kv, k_r])); with MLA_CACHE_INT8 a row is the 656-byte int8 row
 *         described above, [num_pages][page_size][656] bytes.  Row s of sequence b lives at page
 *         block_table[b * max_pages_per_seq + s / page_size], slot s % page_size.
 *   seq_lens[b]: rows of sequence b that decode attention reads (rows
 *         0 .. seq_lens[b]-1).  mla_cache_append does not change it. */
typedef struct {
  void *pool;
  int num_pages;
  const int32_t *block_table;
  int max_pages_per_seq;
  const int32_t *seq_lens;
} mla_paged_cache;

/* Bytes of workspace the calls need for `batch` sequences (d_model: hidden
 * width; d_q: query latent width, 0 without query compression; num_splits as
 * passed to mla_decode_attn, 0 = automatic).  One workspace serves all four
 * calls on one stream; calls that overlap on different streams need separate
 * workspaces. */
size_t mla_workspace_size(const mla_dims *dims, int batch, int d_model, int d_q, int num_splits);

/* Zeroes the workspace's error word and counters (enqueued on `stream`).
 * Call once after allocating a workspace. */
mla_status mla_workspace_init(void *ws, size_t ws_bytes, mla_stream_t stream);

/* Cache append ("解耦 RoPE（MLA 下）" §五 steps 2-3; "从零理解 MLA", 解耦 RoPE
 * k_t^R = RoPE(W^KR h_t); "构建DeepSeek-V3：多头潜在注意力(MLA)架构" step 1,
 * c_KV = RMSNorm(W_dkv x)).  For each b:
 *   x = W_DKV h_b (fp32 accumulation);  c = gamma * x / sqrt(mean(x^2) + rms_eps);
 *   k_R = RoPE_{positions[b]}(W_KR h_b);  the row [c ; k_R] is rounded once to
 *   dtype (round to nearest even) and written to slot positions[b] of sequence b.
 * h: [batch][d_model]; W_DKV: [d_c][d_model]; W_KR: [d_rope][d_model];
 * gamma: [d_c]; positions: [batch] int32 (device).  Only the one row per
 * sequence is written; seq_lens is not read or changed (set seq_lens[b] =
 * positions[b] + 1 before attending so the new token sees itself). */
mla_status mla_cache_append(const mla_dims *dims, const mla_paged_cache *cache, int batch,
                            int d_model, const void *h, const void *W_DKV, const void *W_KR,
                            const void *gamma, const int32_t *positions, void *ws,
                            size_t ws_bytes, mla_stream_t stream);

/* Absorbed query ("从零理解 MLA", 矩阵吸收 / 查询压缩 / 解耦 RoPE;
 * "解耦 RoPE（MLA 下）" §五 step 4).  For each b and head i:
 *   c_Q = W_DQ x_b if W_DQ != NULL (d_q rows), else c_Q = x_b (then d_q must equal d_in);
 *   q_C,i = W_UQ,i c_Q;  q_R,i = RoPE_{positions[b]}(W_QR,i c_Q);
 *   q_lat[b][i] = [W_UK,i^T q_C,i ; q_R,i]   (d_c + d_rope values).
 * x: [batch][d_in]; W_DQ: [d_q][d_in] or NULL; W_UQ: [n_heads*d_nope][d_q];
 * W_QR: [n_heads*d_rope][d_q]; W_UK: [n_heads*d_nope][d_c];
 * q_lat: [batch][n_heads][d_c + d_rope] (output).  Intermediates live in the
 * workspace: with MLA_BF16, c_Q and q_C are stored as bf16 (as a bf16 model
 * stores activations) and q_R stays fp32 until it is rotated and rounded once
 * into q_lat; with MLA_FP32 all of them are fp32. */
mla_status mla_absorb_q(const mla_dims *dims, int batch, int d_in, const void *x,
                        const void *W_DQ, int d_q, const void *W_UQ, const void *W_QR,
                        const void *W_UK, const int32_t *positions, void *q_lat, void *ws,
                        size_t ws_bytes, mla_stream_t stream);

/* Latent decode attention ("从零理解 MLA", 解耦 RoPE absorbed_step: scores
 * s_c + s_r against the cached rows, softmax, z = attn . c; "解耦 RoPE（MLA 下）"
 * §五 steps 4-5).  For each b and head i over rows s = 0 .. seq_lens[b]-1:
 *   z[b][i] = sum_s softmax_s(scale * q_lat[b][i] . row_s) * c_s,
 *   lse[b][i] = log sum_s exp(scale * q_lat[b][i] . row_s)   (natural log).
 * q_lat: [batch][n_heads][d_c + d_rope]; z: [batch][n_heads][d_c] (output);
 * lse: [batch][n_heads] fp32 or NULL.
 * num_splits: the number of equal-work partitions the batch's rows are cut
 * into (each sequence is split only where a partition boundary falls inside
 * it; split sequences are merged by a combine pass); 0 = automatic.
 * A sequence with seq_len <= 0 gets z = 0, lse = -inf and sets the error word. */
mla_status mla_decode_attn(const mla_dims *dims, const mla_paged_cache *cache, int batch,
                           const void *q_lat, void *z, float *lse, int num_splits, void *ws,
                           size_t ws_bytes, mla_stream_t stream);

/* Partial softmax of decode attention, for a sequence whose cached rows are
 * split across devices (each device holds some of its pages and attends over
 * them; the partials are then gathered and merged with mla_merge_partials).
 * Same arguments and rows as mla_decode_attn, but instead of z / lse it writes,
 * for each b and head i over the rows this cache holds:
 *   m[b][i] = max_s logit_s (natural log units),  l[b][i] = sum_s e^(logit_s - m),
 *   O[b][i] = sum_s e^(logit_s - m) c_s            (fp32, not normalised),
 * with logit_s = scale * q_lat[b][i] . row_s.  z_i = O_i / l_i over these rows
 * alone; several shares merge as in mla_merge_partials.  This is the standard
 * rewriting of one softmax as a weighted merge of partial softmaxes; the pages
 * describe no split.  O: [batch][n_heads][d_c] (16-byte aligned); m, l:
 * [batch][n_heads].  A sequence with seq_lens[b] == 0 (no rows on this device)
 * is an empty share: O = 0, m = -inf, l = 0, and no error is recorded. */
mla_status mla_decode_attn_partial(const mla_dims *dims, const mla_paged_cache *cache, int batch,
                                   const void *q_lat, float *O, float *m, float *l, int num_splits,
                                   void *ws, size_t ws_bytes, mla_stream_t stream);

/* Merges n_parts partial softmaxes (e.g. one per device, gathered):
 *   M = max_j m_j,  w_j = e^(m_j - M),  z = sum_j w_j O_j / sum_j w_j l_j,
 *   lse = M + log(sum_j w_j l_j)   (parts summed in increasing j).
 * O: [n_parts][batch][n_heads][d_c] fp32; m, l: [n_parts][batch][n_heads];
 * z: [batch][n_heads][d_c] of dims->dtype; lse: [batch][n_heads] or NULL.
 * A row whose parts are all empty (m = -inf) gets z = 0, lse = -inf. */
mla_status mla_merge_partials(const mla_dims *dims, int batch, int n_parts, const float *O,
                              const float *m, const float *l, void *z, float *lse,
                              mla_stream_t stream);

/* Value up-projection after latent aggregation ("从零理解 MLA", 矩阵吸收: value
 * side, o_{t,i} = W_i^UV z_{t,i}; absorbed_step: o, then w_o).  For each b:
 *   o[b][i] = W_UV,i z[b][i];  if W_O != NULL: out[b] = W_O concat_i(o[b][i]).
 * z: [batch][n_heads][d_c]; W_UV: [n_heads*d_v][d_c]; W_O: [d_model][n_heads*d_v]
 * or NULL; out: [batch][d_model] when W_O is given, else [batch][n_heads*d_v]. */
mla_status mla_unabsorb_out(const mla_dims *dims, int batch, const void *z, const void *W_UV,
                            const void *W_O, int d_model, void *out, void *ws, size_t ws_bytes,
                            mla_stream_t stream);

/* Decode attention without a caller-provided workspace.  The pages describe no
 * such variant: it exists for callers that cannot allocate device memory, e.g.
 * code whose device memory belongs entirely to another allocator (a
 * framework's caching pool or an arena reserved at start-up) or a plugin
 * interface that hands over only the operation's tensors and allows no
 * allocation while it runs.
 * Computes exactly what mla_decode_attn computes, with the same arguments
 * minus the workspace.  Its scratch (plan, split-KV partials, error word) is a
 * fixed 16 MiB array inside the library, present on every device that loads
 * the library until the process exits.  num_splits = 0 picks the most
 * partitions that fit (at most one per pair of SMs); a batch or num_splits
 * whose scratch would exceed 16 MiB returns MLA_ERR_WORKSPACE before any work
 * is enqueued (for the bf16 sizes: at most 30 partitions, i.e. 60 of the SMs).
 * The first call on a device looks up the array's device address for that
 * device; make it before any stream capture.  Calls share the array: calls
 * whose work overlaps on the GPU race and must be serialised by the caller.
 * Device-side range errors zero the affected sequence (z = 0, lse = -inf) as in
 * mla_decode_attn.  The array's error word is cleared at the start of each call
 * and read with mla_noalloc_get_device_error; after MLA_ERR_TIMEOUT (a bounded
 * wait inside the kernels gave up) z and lse of that call are not valid. */
mla_status mla_decode_attn_noalloc(const mla_dims *dims, const mla_paged_cache *cache, int batch,
                                   const void *q_lat, void *z, float *lse, int num_splits,
                                   mla_stream_t stream);

/* The device status of the most recent mla_decode_attn_noalloc call on the
 * current device: waits for `stream` (the stream of that call), then reads and
 * clears the error word of the library's fixed scratch array.  Returns MLA_OK,
 * MLA_ERR_DEVICE_RANGE or MLA_ERR_TIMEOUT (MLA_ERR_CUDA if the stream failed).
 * Like the call it reports on, it allocates nothing and synchronises only. */
mla_status mla_noalloc_get_device_error(mla_stream_t stream);

/* Waits for `stream`, then reads and clears the workspace's device error word.
 * Returns MLA_OK, MLA_ERR_DEVICE_RANGE or MLA_ERR_TIMEOUT (or MLA_ERR_CUDA if
 * the stream itself failed).  This is the only call that synchronises. */
mla_status mla_get_device_error(void *ws, mla_stream_t stream);

/* Test hook, not for production use: exercises the bounded waits.  With
 * enable != 0, every later mla_absorb_q (MLA_BF16) call bounds each of its
 * kernel's internal waits by wait_limit_us microseconds (instead of 2 s) and
 * makes one epilogue warp of the per-head absorption kernel withhold its arrive
 * on the barrier that hands the q_C tile to the W_UK products; that wait then
 * runs out, the kernel records MLA_ERR_TIMEOUT in the workspace error word,
 * drains the loads and MMAs it issued and exits (q_lat is not valid).
 * enable = 0 restores normal operation.  Process-wide; not thread-safe with
 * concurrent mla_absorb_q calls.  No page describes this; it exists for tests. */
mla_status mla_debug_absorb_timeout(int enable, unsigned wait_limit_us);

/* Static, NUL-terminated description of a status code. */
const char *mla_status_string(mla_status status);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H */
