/*
 * qkv.h -- C ABI of the B200 (sm_100a) decode hot path for long-context
 * serving over a paged, 4-bit ("F4") K/V cache with YaRN partial rotary.
 *
 * The operations follow these sources (page title, section):
 *   [YARN]  mistral.rs PR "YaRN rope scaling, 4-bit F4 packed KV cache, and
 *           hybrid paged attention for Qwen3.5-Next long-context serving",
 *           section 1: YaRN for a partial rotary, llama.cpp-style corr_dims
 *           ramp from beta_fast/beta_slow, table scale 1 + 0.1 ln(factor).
 *   [AUTO]  ignis docs "context-and-speculation", --model-rope-scaling: auto
 *           factor max_context / 262,144; the attention factor applies to
 *           queries and keys alike.
 *   [F4]    same PR, section 2: packed 4-bit cache written by a
 *           reshape-and-cache kernel through a slot mapping, values
 *           (nibble - 8) * scale, 32 values per 16-byte cell.
 *   [PAGED] same PR section 2 (v1/v2 paged attention dequantising cells
 *           inline) and ignis "context-and-speculation" (the KV pool in
 *           64-token pages, lanes sharing one pool).
 *   [FOLD]  FreeToken issue #568 "Serving ...'s 1M-token window on one 24 GB
 *           card", proposed solution item 2: partial results folded by
 *           log2-sum-exp.
 *
 * Conventions for every call:
 *   - Array arguments are DEVICE pointers owned by the caller, except where a
 *     comment says "host". The library allocates no memory.
 *   - bf16 and fp16 values travel as uint16_t bit patterns.
 *   - Every call is asynchronous on `stream` (NULL = legacy default stream);
 *     the library never synchronises the host.
 *   - Return value: QKV_OK, or an error code below when an argument is
 *     invalid (nothing is launched) or a launch fails.
 *   - Data-dependent problems found on the device (a page id outside the
 *     pool, a slot outside the pool, a position outside the table, a length
 *     past the page table) never trap: the kernel skips the offending item
 *     and ORs a QKV_DEV_* flag into `*device_status` when that pointer is not
 *     NULL. The caller zeroes the word and reads it when convenient.
 *   - Kernels contain no waits on other blocks. The waits on their own copy
 *     barriers are bounded; one that runs out sets QKV_DEV_TIMEOUT and the
 *     block returns.
 */
#ifndef QKV_H_
#define QKV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QKV_API __attribute__((visibility("default")))
#else
#define QKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* qkv_stream_t;

/* Return codes. */
#define QKV_OK 0
#define QKV_EINVAL 1       /* invalid argument (null pointer, bad size or alignment) */
#define QKV_EUNSUPPORTED 2 /* valid, but outside the compiled shapes */
#define QKV_ECUDA 3        /* a CUDA launch or driver call failed */

/* Device status flags (ORed into *device_status). */
#define QKV_DEV_BAD_POSITION 0x1 /* rope position outside the table: token left unrotated */
#define QKV_DEV_BAD_SLOT 0x2     /* write slot >= num_pages * block_size: token skipped */
#define QKV_DEV_BAD_PAGE 0x4     /* page id < 0 or >= num_pages: page skipped */
#define QKV_DEV_BAD_SEQLEN 0x8   /* seq_len < 0 or > max_pages_per_seq * block_size: clamped */
#define QKV_DEV_TIMEOUT 0x10     /* a bounded wait on a copy barrier ran out */

/* Rotary configuration [YARN], [AUTO].
 *   rope_base    frequency base (1e7 for the workloads here).
 *   rot_dim      rotated dims per head (the first rot_dim of head_dim);
 *                even, 2..512.
 *   factor       YaRN scale s >= 1; 1 = no scaling (textbook RoPE table).
 *   orig_max_pos trained context length the ramp is measured against.
 *   beta_fast, beta_slow  ramp bounds in turns over orig_max_pos (32, 1).
 *   ext_factor   ramp weight; < 0 selects 1 when factor > 1, else 0.
 *   attn_factor  table scale; <= 0 selects 1 + 0.1 ln(factor) when
 *                factor > 1, else 1.
 * Pair j < rot_dim/2 has omega_j = rope_base^(-2j/rot_dim) and angle step
 *   theta_j = (omega_j / s) (1 - r_j e) + omega_j r_j e,
 * r_j = 1 - clamp((j - low) / max(0.001, high - low), 0, 1), where low =
 * max(0, floor(c(beta_fast))), high = min(rot_dim - 1, ceil(c(beta_slow))),
 * c(b) = rot_dim ln(orig_max_pos / (2 pi b)) / (2 ln rope_base). */
typedef struct {
  double rope_base;
  int32_t rot_dim;
  int32_t reserved; /* set to 0 */
  double factor;
  int64_t orig_max_pos;
  double beta_fast;
  double beta_slow;
  double ext_factor;
  double attn_factor;
} qkv_yarn_params;

/* [AUTO] Host-only helper: the YaRN factor the auto rule picks for a
 * maximum context. Returns 0 when no scaling is needed (max_context <=
 * orig_max_pos), -1 when the context is refused (factor above 64 or a
 * non-positive argument), else max_context / orig_max_pos. */
QKV_API double qkv_yarn_auto_factor(int64_t max_context, int64_t orig_max_pos);

/* a1 [YARN] YaRN rotary table.
 *   params   HOST pointer.
 *   cos_out, sin_out  float [n_pos][rot_dim/2]; row i is position
 *            pos_start + i; each value is mscale * cos|sin(p * theta_j) with
 *            the angle formed and evaluated in double, stored as float.
 * EINVAL: null pointer, n_pos < 0, pos_start < 0, rot_dim odd or out of
 * range, factor < 1, rope_base <= 1, orig_max_pos <= 0. */
QKV_API int qkv_yarn_rope_table(const qkv_yarn_params* params, int64_t pos_start, int64_t n_pos,
                        float* cos_out, float* sin_out, qkv_stream_t stream);

/* a2 [YARN], [AUTO] Partial NEOX rotary on q or k rows.
 *   x_in, x_out  bf16 [n_tok][n_heads][head_dim]; x_out may equal x_in
 *                (in place); otherwise the ranges must not overlap.
 *   positions    int64 [n_tok], position of each token.
 *   cos_tab, sin_tab  a table from qkv_yarn_rope_table covering positions
 *                table_pos_start .. table_pos_start + table_len - 1.
 * For j < rot_dim/2: (x_j, x_{j+rot/2}) -> (x_j c - x_{j+rot/2} s,
 * x_{j+rot/2} c + x_j s) in float, rounded to bf16 (nearest even); dims >=
 * rot_dim are copied. A position outside the table copies the token
 * unrotated and sets QKV_DEV_BAD_POSITION.
 * n_tok == 0 or n_heads == 0 returns QKV_OK without touching any pointer.
 * EINVAL: null pointer, n_tok/n_heads < 0, rot_dim odd or > head_dim,
 * head_dim odd, table_len < 0, distinct x_in/x_out that overlap. */
QKV_API int qkv_rope_apply(const uint16_t* x_in, uint16_t* x_out, const int64_t* positions, int32_t n_tok,
                   int32_t n_heads, int32_t head_dim, int32_t rot_dim, const float* cos_tab,
                   const float* sin_tab, int64_t table_pos_start, int64_t table_len,
                   int32_t* device_status, qkv_stream_t stream);

/* a3 [F4] Quantise and write new K/V rows into the paged F4 cache.
 *   k, v          bf16 [n_tok][kv_heads][head_dim].
 *   slot_mapping  int64 [n_tok]: page * block_size + offset; < 0 skips the
 *                 token; >= num_pages * block_size skips it and sets
 *                 QKV_DEV_BAD_SLOT.
 *   k_data, v_data    u8  [num_pages][kv_heads][block_size][head_dim/2]
 *   k_scale, v_scale  fp16 [num_pages][kv_heads][block_size][head_dim/32]
 * Per 32-value cell: scale = fp16(amax / 7), round to nearest even,
 * saturating at 65504; code = clamp(rint(x / scale), -8, 7) + 8 (all 8 when
 * scale is 0); byte b holds element 2b in bits 0-3 and 2b+1 in bits 4-7.
 * The result is bit-identical to evaluating both divisions exactly.
 * n_tok == 0 returns QKV_OK without touching any pointer.
 * EINVAL: null pointer, n_tok < 0, head_dim not a multiple of 32 or > 256,
 * kv_heads < 1, block_size < 1, num_pages < 1, k/v not 16-byte aligned. */
QKV_API int qkv_kv_write_f4(const uint16_t* k, const uint16_t* v, const int64_t* slot_mapping,
                    int32_t n_tok, uint8_t* k_data, uint16_t* k_scale, uint8_t* v_data,
                    uint16_t* v_scale, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                    int64_t num_pages, int32_t* device_status, qkv_stream_t stream);

/* a3 with the V scale layout as a parameter. The mistral.rs PR's own F4
 * cache keeps "one scale per 32-value K cell and one scale per token per V
 * head"; qkv_kv_write_f4 gives V the K layout.
 *   v_group   values of a V row sharing one scale: 32 (v_scale as in
 *             qkv_kv_write_f4) or head_dim (v_scale fp16
 *             [num_pages][kv_heads][block_size][1], one scale per token and
 *             head: fp16(amax of the row / 7), same rounding and codes).
 * K is always quantised per 32-value cell. Other arguments, results and
 * errors as in qkv_kv_write_f4; EINVAL also for any other v_group. */
QKV_API int qkv_kv_write_f4_v(const uint16_t* k, const uint16_t* v, const int64_t* slot_mapping,
                              int32_t n_tok, uint8_t* k_data, uint16_t* k_scale, uint8_t* v_data,
                              uint16_t* v_scale, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                              int64_t num_pages, int32_t v_group, int32_t* device_status,
                              qkv_stream_t stream);

/* a2 + a3 in one launch: the partial rotary of q and of the new k, and the
 * F4 write of the rotated k and of v through the slot mapping.
 *   q_in, q_out  bf16 [n_tok][q_heads][head_dim] (q_out may equal q_in).
 *   k_in, v_in   bf16 [n_tok][kv_heads][head_dim], not modified.
 *   k_out        bf16 [n_tok][kv_heads][head_dim] receives the rotated k, or
 *                NULL.
 * Other arguments as in qkv_rope_apply and qkv_kv_write_f4; the results are
 * bit-identical to qkv_rope_apply on q and on k followed by
 * qkv_kv_write_f4 of the rotated k and v. rot_dim must be a multiple of 16.
 * n_tok == 0 returns QKV_OK without touching any pointer. */
QKV_API int qkv_rope_kv_write_f4(const uint16_t* q_in, uint16_t* q_out, const uint16_t* k_in,
                                 const uint16_t* v_in, uint16_t* k_out, const int64_t* positions,
                                 const int64_t* slot_mapping, int32_t n_tok, int32_t q_heads,
                                 int32_t kv_heads, int32_t head_dim, int32_t rot_dim,
                                 const float* cos_tab, const float* sin_tab, int64_t table_pos_start,
                                 int64_t table_len, uint8_t* k_data, uint16_t* k_scale,
                                 uint8_t* v_data, uint16_t* v_scale, int32_t block_size,
                                 int64_t num_pages, int32_t* device_status, qkv_stream_t stream);

/* qkv_rope_kv_write_f4 with the V scale layout of qkv_kv_write_f4_v. */
QKV_API int qkv_rope_kv_write_f4_v(const uint16_t* q_in, uint16_t* q_out, const uint16_t* k_in,
                                   const uint16_t* v_in, uint16_t* k_out, const int64_t* positions,
                                   const int64_t* slot_mapping, int32_t n_tok, int32_t q_heads,
                                   int32_t kv_heads, int32_t head_dim, int32_t rot_dim,
                                   const float* cos_tab, const float* sin_tab, int64_t table_pos_start,
                                   int64_t table_len, uint8_t* k_data, uint16_t* k_scale,
                                   uint8_t* v_data, uint16_t* v_scale, int32_t block_size,
                                   int64_t num_pages, int32_t v_group, int32_t* device_status,
                                   qkv_stream_t stream);

/* Number of splits per sequence the automatic plan aims for on the current
 * device (resident split blocks / kv_heads); a workspace sized with this as
 * max_splits never limits the automatic plan. Host-only; returns 0 when no
 * CUDA device is present. */
QKV_API int32_t qkv_paged_decode_auto_splits(int32_t kv_heads, int32_t block_size);

/* Bytes of workspace qkv_paged_decode_attn_f4 needs: max_splits *
 * n_seq * q_heads * head_dim floats (o_parts) and max_splits * n_seq *
 * q_heads floats (lse2_parts), each rounded up to 256 bytes. */
QKV_API size_t qkv_paged_decode_workspace_bytes(int32_t n_seq, int32_t q_heads, int32_t head_dim,
                                        int32_t max_splits);

/* a4 [PAGED], [FOLD] Split pass of paged GQA decode attention.
 *   q         bf16 [n_seq][q_heads][head_dim] (already rotated).
 *   k_data, k_scale, v_data, v_scale  the F4 cache (layout as in
 *             qkv_kv_write_f4).
 *   page_table  int32 [n_seq][max_pages_per_seq]; token i of sequence s is
 *             in page page_table[s][i / block_size] at offset i % block_size.
 *   seq_lens  int32 [n_seq], context tokens of each sequence.
 *   softmax_scale  0 selects 1/sqrt(head_dim).
 *   num_splits  > 0: every sequence is cut into exactly num_splits splits
 *             (EINVAL when num_splits > max_splits: the count is never cut
 *             to fit); 0: the plan balances pages over the device (splits of
 *             about sum(pages) / auto_splits pages each, at most max_splits
 *             per sequence). Split i of a sequence with n pages covers pages
 *             [b(i), b(i+1)): b(i) = i*n/S, except that with S >= 8 the
 *             first m = ceil(S/7) splits are d pages shorter each (d: 400
 *             tokens at head_dim 256, 800 at 128, at most a quarter split),
 *             the others sharing those pages; the grid places the first
 *             splits last, and the last CTAs placed start late.
 *   o_parts   float [max_splits][n_seq * q_heads][head_dim]: partial output
 *             of split i for row (s, h) at [i][s * q_heads + h], normalised
 *             by its own softmax sum.
 *   lse2_parts float [max_splits][n_seq * q_heads]: log2 of the split's
 *             softmax normaliser, log2 sum_t 2^(score_t log2 e); -inf for an
 *             empty or unused split (its o_parts row is then unspecified).
 * Shapes compiled: head_dim 256 and 128, q_heads / kv_heads in {1, 2, 4, 8},
 * block_size in {16, 32, 64}; others return QKV_EUNSUPPORTED. Cache and q
 * pointers must be 16-byte aligned (EINVAL otherwise). */
QKV_API int qkv_paged_decode_split_f4(float* o_parts, float* lse2_parts, int32_t max_splits,
                              const uint16_t* q, const uint8_t* k_data, const uint16_t* k_scale,
                              const uint8_t* v_data, const uint16_t* v_scale,
                              const int32_t* page_table, const int32_t* seq_lens, int32_t n_seq,
                              int32_t q_heads, int32_t kv_heads, int32_t head_dim,
                              int32_t block_size, int32_t max_pages_per_seq, int64_t num_pages,
                              float softmax_scale, int32_t num_splits, int32_t* device_status,
                              qkv_stream_t stream);

/* qkv_paged_decode_split_f4 over a cache written with qkv_kv_write_f4_v:
 * v_group 32 (V scale per cell) or head_dim (one V scale per token; the P V
 * product then takes one scale per token for all of the row). EINVAL for
 * any other v_group; other arguments as in qkv_paged_decode_split_f4. */
QKV_API int qkv_paged_decode_split_f4_v(float* o_parts, float* lse2_parts, int32_t max_splits,
                                        const uint16_t* q, const uint8_t* k_data,
                                        const uint16_t* k_scale, const uint8_t* v_data,
                                        const uint16_t* v_scale, const int32_t* page_table,
                                        const int32_t* seq_lens, int32_t n_seq, int32_t q_heads,
                                        int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                        int32_t max_pages_per_seq, int64_t num_pages,
                                        float softmax_scale, int32_t num_splits, int32_t v_group,
                                        int32_t* device_status, qkv_stream_t stream);

/* a5 [FOLD] log2-sum-exp merge of partial attention results.
 *   o_parts   float [n_parts][rows][head_dim], lse2_parts float [n_parts][rows].
 *   out       bf16 [rows][head_dim] (nearest even); lse2_out float [rows] or NULL.
 * Per row: M = max_i lse2_i; w_i = 2^(lse2_i - M); out = sum_i w_i o_i /
 * sum_i w_i; lse2 = M + log2 sum_i w_i. Parts with lse2 = -inf carry no
 * weight: their o rows may be read but never enter the result (they may
 * hold anything, NaN included); a row without any weighted part gives
 * out = 0 and lse2 = -inf.
 * EINVAL: null pointer, n_parts < 1, rows < 0, head_dim not a multiple of 4
 * or > 1024. EUNSUPPORTED: n_parts <= 8 and rows * ceil(head_dim / 64) above
 * 2^31 - 1 (that case runs one warp per row and 64 dims). */
QKV_API int qkv_lse_merge(const float* o_parts, const float* lse2_parts, int32_t n_parts, int32_t rows,
                  int32_t head_dim, uint16_t* out, float* lse2_out, qkv_stream_t stream);

/* a4 + a5: the decode attention of one layer. Runs the split pass into
 * `workspace` (see qkv_paged_decode_workspace_bytes) and merges it into
 * `out` (bf16 [n_seq][q_heads][head_dim]) and `lse2_out` (float
 * [n_seq][q_heads] or NULL). Arguments and errors as in the two calls;
 * EINVAL also when workspace_bytes is too small or workspace is not
 * 256-byte aligned. After the call the workspace holds the split pass's
 * o_parts (float [max_splits][n_seq * q_heads][head_dim], from offset 0)
 * and lse2_parts (float [max_splits][n_seq * q_heads], from the next
 * 256-byte boundary); it needs no initialisation.
 * Programmatic dependent launch: the split launch may start while the
 * kernel ahead of it in the stream still runs (when that kernel allows
 * it), and reads the page table, the sequence lengths and the cache pages
 * before that kernel completes; q is read after. A kernel that lets its
 * successor start early must therefore not write those (this library's
 * cache writers never let their successor start early). */
QKV_API int qkv_paged_decode_attn_f4(uint16_t* out, float* lse2_out, const uint16_t* q,
                             const uint8_t* k_data, const uint16_t* k_scale,
                             const uint8_t* v_data, const uint16_t* v_scale,
                             const int32_t* page_table, const int32_t* seq_lens, int32_t n_seq,
                             int32_t q_heads, int32_t kv_heads, int32_t head_dim,
                             int32_t block_size, int32_t max_pages_per_seq, int64_t num_pages,
                             float softmax_scale, int32_t num_splits, int32_t max_splits,
                             void* workspace, size_t workspace_bytes, int32_t* device_status,
                             qkv_stream_t stream);

/* One decode step of a layer in two launches: a2 + a3 + a4 in the split
 * pass, then a5. The split kernel rotates each sequence's q itself (NEOX on
 * the first rot_dim dims, rounded to bf16 as qkv_rope_apply rounds), and the
 * CTA whose split holds a sequence's last page first writes the step's new
 * k (rotated) and v into the cache at slot_mapping[s] (F4, as
 * qkv_kv_write_f4(_v)), so out, lse2_out and the cache bytes equal those of
 * qkv_rope_kv_write_f4 followed by qkv_paged_decode_attn_f4(_v).
 *   q            bf16 [n_seq][q_heads][head_dim], NOT rotated (read only).
 *   k_new, v_new bf16 [n_seq][kv_heads][head_dim]: the step's new token, the
 *                last of each sequence's seq_lens[s] tokens (16-byte aligned).
 *   positions    int64 [n_seq]: rotary position of each step token.
 *   slot_mapping int64 [n_seq]: cache slot of token seq_lens[s] - 1 (< 0:
 *                not written).
 *   cos_tab, sin_tab, table_pos_start, table_len, rot_dim: as in
 *                qkv_rope_apply (a position outside the table leaves q and k
 *                unrotated and sets QKV_DEV_BAD_POSITION).
 *   the rest as in qkv_paged_decode_attn_f4_v (v_group 32 or head_dim).
 * A slot past the pool sets QKV_DEV_BAD_SLOT and skips the write.
 * Besides what qkv_paged_decode_attn_f4 reads early, positions,
 * slot_mapping and the cos/sin tables are read before the kernel ahead in
 * the stream completes (q, k_new and v_new after): the step's metadata must
 * not be written by a kernel that lets its successor start early (the
 * library's table kernel never does). */
QKV_API int qkv_decode_step_f4(uint16_t* out, float* lse2_out, const uint16_t* q, const uint16_t* k_new,
                               const uint16_t* v_new, const int64_t* positions, const int64_t* slot_mapping,
                               const float* cos_tab, const float* sin_tab, int64_t table_pos_start,
                               int64_t table_len, int32_t rot_dim, uint8_t* k_data, uint16_t* k_scale,
                               uint8_t* v_data, uint16_t* v_scale, const int32_t* page_table,
                               const int32_t* seq_lens, int32_t n_seq, int32_t q_heads, int32_t kv_heads,
                               int32_t head_dim, int32_t block_size, int32_t max_pages_per_seq,
                               int64_t num_pages, float softmax_scale, int32_t num_splits, int32_t max_splits,
                               int32_t v_group, void* workspace, size_t workspace_bytes, int32_t* device_status,
                               qkv_stream_t stream);

/* The split pass of qkv_decode_step_f4 alone (a2 + a3 + a4 in one launch):
 * rotates q, writes the step's new token into the cache and writes the
 * partials like qkv_paged_decode_split_f4_v, for a caller that merges them
 * itself (qkv_lse_merge). Arguments as in qkv_decode_step_f4, with o_parts /
 * lse2_parts / max_splits as in qkv_paged_decode_split_f4. */
QKV_API int qkv_decode_step_split_f4(float* o_parts, float* lse2_parts, int32_t max_splits, const uint16_t* q,
                                     const uint16_t* k_new, const uint16_t* v_new, const int64_t* positions,
                                     const int64_t* slot_mapping, const float* cos_tab, const float* sin_tab,
                                     int64_t table_pos_start, int64_t table_len, int32_t rot_dim,
                                     uint8_t* k_data, uint16_t* k_scale, uint8_t* v_data, uint16_t* v_scale,
                                     const int32_t* page_table, const int32_t* seq_lens, int32_t n_seq,
                                     int32_t q_heads, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                     int32_t max_pages_per_seq, int64_t num_pages, float softmax_scale,
                                     int32_t num_splits, int32_t v_group, int32_t* device_status,
                                     qkv_stream_t stream);

/* qkv_paged_decode_attn_f4 over a cache written with qkv_kv_write_f4_v
 * (v_group 32 or head_dim). */
QKV_API int qkv_paged_decode_attn_f4_v(uint16_t* out, float* lse2_out, const uint16_t* q,
                                       const uint8_t* k_data, const uint16_t* k_scale,
                                       const uint8_t* v_data, const uint16_t* v_scale,
                                       const int32_t* page_table, const int32_t* seq_lens,
                                       int32_t n_seq, int32_t q_heads, int32_t kv_heads,
                                       int32_t head_dim, int32_t block_size,
                                       int32_t max_pages_per_seq, int64_t num_pages,
                                       float softmax_scale, int32_t num_splits, int32_t max_splits,
                                       int32_t v_group, void* workspace, size_t workspace_bytes,
                                       int32_t* device_status, qkv_stream_t stream);

/* Paged -> contiguous gather of the F4 cache ([F4] section 2: gather_kv_cache
 * with an F4 path, the cache read back for attention outside the paged
 * kernels).
 *   k_out, v_out  bf16 [n_out][kv_heads][head_dim]: row out_start[s] + t holds
 *                 token t of sequence s, t < seq_lens[s], each element
 *                 bf16((code - 8) * scale) rounded to nearest even (the
 *                 product is exact). Other rows are not written. 16-byte
 *                 aligned.
 *   out_start     int64 [n_seq], the first output row of each sequence.
 *   page_table, seq_lens, cache and v_group as in qkv_paged_decode_split_f4_v
 *                 (head_dim a multiple of 32 up to 256, any block_size).
 * A page id outside [0, num_pages) gives zero rows and QKV_DEV_BAD_PAGE; a
 * seq_len outside [0, max_pages_per_seq * block_size] is clamped and an
 * output row outside [0, n_out) skipped, each with QKV_DEV_BAD_SEQLEN.
 * One thread per 32-value cell; bound by HBM (144 bytes read and 512
 * written per token, KV head and K or V). */
QKV_API int qkv_gather_kv_f4(uint16_t* k_out, uint16_t* v_out, int64_t n_out, const uint8_t* k_data,
                             const uint16_t* k_scale, const uint8_t* v_data, const uint16_t* v_scale,
                             const int32_t* page_table, const int32_t* seq_lens, const int64_t* out_start,
                             int32_t n_seq, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                             int32_t max_pages_per_seq, int64_t num_pages, int32_t v_group,
                             int32_t* device_status, qkv_stream_t stream);

/* Chunked causal prefill attention over the paged F4 cache ([F4] section 5:
 * paged prefill in chunks of 2048 tokens). A chunk of n_q queries of one
 * sequence occupies cache tokens prefix_len .. prefix_len + n_q - 1, already
 * written with qkv_kv_write_f4(_v); query i attends the cached tokens
 * 0 .. prefix_len + i:
 *   out[i][h] = sum_t softmax_t(softmax_scale * q[i][h] . k^_t) v^_t
 * with query head h reading KV head h / (q_heads / kv_heads).
 *   out        bf16 [n_q][q_heads][head_dim]; lse2_out float [n_q][q_heads]
 *              (log2 sum_t exp(score_t)) or NULL.
 *   q          bf16 [n_q][q_heads][head_dim], rotary already applied.
 *   page_table int32 [max_pages_per_seq]: the sequence's row; token t is on
 *              page page_table[t / block_size]. prefix_len + n_q must not
 *              exceed max_pages_per_seq * block_size (else QKV_EINVAL).
 *   cache, v_group, softmax_scale as in qkv_paged_decode_split_f4_v.
 *   num_splits parts of each query block's context (each part's partials go
 *              to the workspace and a log2-sum-exp merge folds them): 1 for
 *              none (workspace may be NULL), 0 for automatic (the fewest
 *              parts, up to 8, that fill the GPU's waves of CTA pairs, within
 *              the workspace given; 1 without one). QKV_EINVAL when a part
 *              would have no 64-token stage or the workspace is too small.
 *   workspace  device buffer (256-byte aligned) of at least
 *              qkv_paged_prefill_workspace_bytes(n_q, q_heads, head_dim,
 *              num_splits) bytes, owned by the caller.
 * Compiled shapes: head_dim 256 and 128, q_heads / kv_heads in {1, 2, 4,
 * 8}, a power-of-two block_size (else QKV_EUNSUPPORTED). Runs on the tensor cores
 * (tcgen05 on clusters of two CTAs, fp16 operands, fp32 accumulators in
 * tensor memory): K (as exact hi + lo halves) and V are dequantised to fp16
 * in shared memory, q scaled by a power of two per row; outputs match
 * exact attention within 2e-3. A page id outside the pool reads as zero
 * rows and sets QKV_DEV_BAD_PAGE. */
QKV_API int qkv_paged_prefill_attn_f4(uint16_t* out, float* lse2_out, const uint16_t* q, const uint8_t* k_data,
                                      const uint16_t* k_scale, const uint8_t* v_data, const uint16_t* v_scale,
                                      const int32_t* page_table, int32_t n_q, int32_t prefix_len,
                                      int32_t q_heads, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                      int32_t max_pages_per_seq, int64_t num_pages, float softmax_scale,
                                      int32_t v_group, int32_t num_splits, void* workspace,
                                      size_t workspace_bytes, int32_t* device_status, qkv_stream_t stream);

/* Workspace bytes of qkv_paged_prefill_attn_f4 for num_splits parts (0 for
 * one part; the automatic choice never needs more than 8 parts' worth).
 * Host-only. */
QKV_API size_t qkv_paged_prefill_workspace_bytes(int32_t n_q, int32_t q_heads, int32_t head_dim,
                                                 int32_t num_splits);

/* The part count qkv_paged_prefill_attn_f4 chooses with num_splits 0 and a
 * workspace of workspace_bytes (1: one launch, no merge; k > 1: k parts and
 * the merge, two launches). 0 for shapes the prefill does not compile.
 * Host-only; asks the current device for its SM count. */
QKV_API int32_t qkv_paged_prefill_auto_splits(int32_t n_q, int32_t prefix_len, int32_t q_heads,
                                              int32_t kv_heads, int32_t head_dim, size_t workspace_bytes);

/* Size of the partials array compiled into the library for
 * qkv_paged_decode_attn_f4_static (16 MiB per GPU that loads the library). */
#define QKV_STATIC_SCRATCH_BYTES (16u << 20)

/* Decode attention (a4 + a5) without caller-provided scratch. The paper has
 * no counterpart to this call; it exists for callers that cannot call
 * cudaMalloc: plugins inside a host engine that owns all device memory, and
 * runtimes that forbid allocation after start-up (cudaMalloc can
 * synchronise the device and fragments a pre-planned budget).
 * Same arguments and results as qkv_paged_decode_attn_f4, minus the
 * workspace: the partials live in a QKV_STATIC_SCRATCH_BYTES array compiled
 * into the library. The call allocates nothing. Splits per sequence: num_splits
 * when > 0, else qkv_paged_decode_auto_splits(kv_heads, block_size).
 *   - EINVAL when qkv_paged_decode_workspace_bytes(n_seq, q_heads, head_dim,
 *     splits) exceeds QKV_STATIC_SCRATCH_BYTES (16 query heads of dimension
 *     256 at a B200's automatic 37 splits: up to 27 sequences).
 *   - The first call on a device resolves the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture. The address is cached with the identity of
 *     the device's CUDA context: after cudaDeviceReset (or any new context
 *     on the device) the next call resolves it again, so make that call
 *     outside capture as well; a call whose launch fails drops the cached
 *     address.
 *   - Every call on a device shares the one array and it keeps the last
 *     call's contents (nothing in it needs to start at zero). Calls whose
 *     kernels overlap on the GPU -- on different streams, or from different
 *     host threads -- race on it: order them on one stream. */
QKV_API int qkv_paged_decode_attn_f4_static(uint16_t* out, float* lse2_out, const uint16_t* q,
                                            const uint8_t* k_data, const uint16_t* k_scale,
                                            const uint8_t* v_data, const uint16_t* v_scale,
                                            const int32_t* page_table, const int32_t* seq_lens,
                                            int32_t n_seq, int32_t q_heads, int32_t kv_heads,
                                            int32_t head_dim, int32_t block_size,
                                            int32_t max_pages_per_seq, int64_t num_pages,
                                            float softmax_scale, int32_t num_splits,
                                            int32_t* device_status, qkv_stream_t stream);

/* [TIER] Copy pages of one F4 pool into consecutive pages of another: the
 * host tier's pages into a device window. FreeToken issue #568, proposed
 * solution item 2 (host-placed K/V: the K/V of a long context kept in host
 * RAM and read over the host link; a prefill stages its pages into a device
 * window).
 *   dst_*       destination pool (layout as in qkv_kv_write_f4_v) of
 *               dst_num_pages pages; pages dst_page0 .. dst_page0 + n_pages - 1
 *               are overwritten. Device memory, 16-byte aligned.
 *   src_*       source pool of src_num_pages pages with the same kv_heads,
 *               block_size, head_dim and v_group: pinned host memory mapped
 *               into the device's address space (cudaHostAlloc, or
 *               cudaHostRegister with the mapped flag) or device memory,
 *               16-byte aligned. The kernel reads it in place, each byte
 *               once, with 16-byte loads.
 *   src_pages   int32 [n_pages], device or mapped pinned host memory: the
 *               source page of destination page dst_page0 + i.
 * The bytes are copied unchanged. A source page id outside [0,
 * src_num_pages) zero-fills its destination page and sets QKV_DEV_BAD_PAGE.
 * EINVAL: a null or misaligned pointer; a source pointer that is pageable
 * host memory (the call asks the driver what each pointer is); n_pages < 0;
 * a destination range outside the pool; head_dim not a multiple of 32 up to
 * 256; v_group not 32 or head_dim; a per-page scale slab that is not a
 * multiple of 16 bytes (kv_heads * block_size * head_dim / v_group * 2). */
QKV_API int qkv_stage_pages_f4(uint8_t* dst_k_data, uint16_t* dst_k_scale, uint8_t* dst_v_data,
                               uint16_t* dst_v_scale, int64_t dst_num_pages, int64_t dst_page0,
                               const uint8_t* src_k_data, const uint16_t* src_k_scale,
                               const uint8_t* src_v_data, const uint16_t* src_v_scale,
                               int64_t src_num_pages, const int32_t* src_pages, int32_t n_pages,
                               int32_t kv_heads, int32_t head_dim, int32_t block_size, int32_t v_group,
                               int32_t* device_status, qkv_stream_t stream);

/* Workspace bytes of qkv_paged_decode_attn_f4_tiered: the window (window_pages
 * pages of the F4 layout), its page table, and the partials of one sequence,
 * (ceil(max_host_pages_per_seq / window_pages) + 1) * max_splits parts of
 * q_heads * (head_dim + 1) floats; each region 256-byte aligned. 0 for
 * invalid sizes. Host-only. */
QKV_API size_t qkv_paged_decode_tiered_workspace_bytes(int32_t q_heads, int32_t kv_heads, int32_t head_dim,
                                                       int32_t block_size, int32_t v_group,
                                                       int32_t max_host_pages_per_seq, int32_t window_pages,
                                                       int32_t max_splits);

/* [TIER] + a4 + a5: decode attention of one layer whose context sits partly in
 * a host-placed tier. FreeToken issue #568, proposed solution item 2: the
 * host K/V read over the host link, the parts folded by log2-sum-exp.
 * Context of sequence s, in order: host_lens[s] tokens in the host pool
 * (token i in page host_page_table[s][i / block_size]), then seq_lens[s]
 * tokens in the device pool (token i in page page_table[s][i / block_size]).
 *   q, out, lse2_out, the device pool, page_table, seq_lens, softmax_scale,
 *               v_group: as in qkv_paged_decode_attn_f4_v.
 *   host_*      the host pool (host_num_pages pages, same shape), pinned and
 *               mapped as for qkv_stage_pages_f4.
 *   host_page_table  int32 [n_seq][max_host_pages_per_seq], device or
 *               mapped pinned host memory.
 *   host_lens   int32 [n_seq] in HOST memory, read by this call on the CPU to
 *               plan the windows: multiples of block_size, at most
 *               max_host_pages_per_seq * block_size (EINVAL otherwise).
 *   window_pages  device pages per window; workspace as sized by
 *               qkv_paged_decode_tiered_workspace_bytes, 256-byte aligned.
 *   max_splits  split slots per window and for the device part
 *               (qkv_paged_decode_auto_splits fills the device).
 * Per sequence, per window of its host pages: qkv_stage_pages_f4 into the
 * window, then the split pass over the window; then the split pass over the
 * device pages and qkv_lse_merge of all the parts. Launch count per sequence:
 * 2 * ceil(host pages / window_pages) + 2. The host tier's bytes cross the
 * link once per call. Data-dependent errors as in the two kernels. */
QKV_API int qkv_paged_decode_attn_f4_tiered(
    uint16_t* out, float* lse2_out, const uint16_t* q, const uint8_t* k_data, const uint16_t* k_scale,
    const uint8_t* v_data, const uint16_t* v_scale, const int32_t* page_table, const int32_t* seq_lens,
    int32_t max_pages_per_seq, int64_t num_pages, const uint8_t* host_k_data, const uint16_t* host_k_scale,
    const uint8_t* host_v_data, const uint16_t* host_v_scale, int64_t host_num_pages,
    const int32_t* host_page_table, int32_t max_host_pages_per_seq, const int32_t* host_lens, int32_t n_seq,
    int32_t q_heads, int32_t kv_heads, int32_t head_dim, int32_t block_size, int32_t v_group,
    float softmax_scale, int32_t window_pages, int32_t max_splits, void* workspace, size_t workspace_bytes,
    int32_t* device_status, qkv_stream_t stream);

/* Workspace bytes of qkv_paged_prefill_attn_f4_tiered: the window and its
 * page table, then fp32 partials for (ceil(max_host_pages / window_pages) +
 * 1) * parts_per_launch parts of n_q * q_heads * (head_dim + 1) floats; each
 * region 256-byte aligned. 0 for invalid sizes. Host-only. */
QKV_API size_t qkv_paged_prefill_tiered_workspace_bytes(int32_t n_q, int32_t q_heads, int32_t kv_heads,
                                                        int32_t head_dim, int32_t block_size, int32_t v_group,
                                                        int32_t max_host_pages, int32_t window_pages,
                                                        int32_t parts_per_launch);

/* [TIER] + [CHUNK]: causal attention of a chunk of queries of one sequence
 * whose oldest tokens sit in a host-placed tier. FreeToken issue #568,
 * proposed solution item 2: a prefill stages the host pages into a device
 * window, attends it there, and the parts are folded by log2-sum-exp.
 * The sequence's context, in order: host_len tokens in the host pool (token
 * i in page host_page_table[i / block_size]), then the device tokens of
 * page_table (the row, as in qkv_paged_prefill_attn_f4). The chunk's queries
 * sit at device tokens prefix_len .. prefix_len + n_q - 1 (already written):
 * query i attends all host_len host tokens and device tokens 0 ..
 * prefix_len + i.
 *   out, lse2_out, q, the device pool, page_table, n_q, prefix_len,
 *               softmax_scale, v_group: as in qkv_paged_prefill_attn_f4
 *               (head_dim 256 or 128, power-of-two block_size).
 *   host_*      the host pool (host_num_pages pages, same shape), pinned and
 *               mapped as for qkv_stage_pages_f4; host_page_table int32
 *               [host_len / block_size], device or mapped pinned memory.
 *   host_len    whole pages (EINVAL otherwise).
 *   window_pages  device pages per window.
 *   parts_per_launch  upper bound of the context split of each prefill
 *               launch (the automatic count fills the device's waves).
 *   workspace   qkv_paged_prefill_tiered_workspace_bytes(n_q, ..., host_len
 *               / block_size, window_pages, parts_per_launch) bytes or more,
 *               256-byte aligned.
 * Per window: qkv_stage_pages_f4 of its host pages, then the prefill kernel
 * over the window with every query seeing every token; then the causal
 * prefill over the device pages; qkv_lse_merge of all the fp32 parts. The
 * staging of a window and the attention run one after the other on
 * `stream` (the staging is bound by the host link, the attention by the
 * tensor cores; they are not overlapped). */
QKV_API int qkv_paged_prefill_attn_f4_tiered(
    uint16_t* out, float* lse2_out, const uint16_t* q, const uint8_t* k_data, const uint16_t* k_scale,
    const uint8_t* v_data, const uint16_t* v_scale, const int32_t* page_table, int32_t n_q, int32_t prefix_len,
    int32_t max_pages_per_seq, int64_t num_pages, const uint8_t* host_k_data, const uint16_t* host_k_scale,
    const uint8_t* host_v_data, const uint16_t* host_v_scale, int64_t host_num_pages,
    const int32_t* host_page_table, int32_t host_len, int32_t q_heads, int32_t kv_heads, int32_t head_dim,
    int32_t block_size, int32_t v_group, float softmax_scale, int32_t window_pages, int32_t parts_per_launch,
    void* workspace, size_t workspace_bytes, int32_t* device_status, qkv_stream_t stream);

/* Static text for a return code. */
QKV_API const char* qkv_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* QKV_H_ */
