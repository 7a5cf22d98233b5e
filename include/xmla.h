/*
 * xmla.h — C ABI of libxmla: Multi-head Latent Attention (MLA) decode over a
 * paged latent KV cache with YaRN RoPE, for NVIDIA B200 (sm_100a).
 *
 * Sources (web pages, cited by title and section):
 *   [P1] "256K 长上下文真能本地用：Xing4.0 原生长上下文的工程代价拆解"
 *        (lpnh.cn/news/2764750), section 一 "256K的规格真相" (config.json:
 *        rope_scaling yarn, factor 64, original_max_position_embeddings 4096,
 *        beta_fast 32, beta_slow 1, mscale 1.0, mscale_all_dim 1.0,
 *        kv_lora_rank 512, v_head_dim 128, attention_bias false) and section
 *        二 "KV Cache 显存账本" (32 heads, qk_nope 128 + qk_rope 64).
 *   [P5] "mHC+MLA+MTP 是什么？拆开给 Agent 用的百亿 MoE"
 *        (hotelren.com/news/5507480), section "MLA：256K 上下文的'内存革命'"
 *        (kv_a_proj_with_mqa -> latent 512 + rope 64 is what is cached;
 *        kv_b_proj: 512 -> 32 x (128 + 128) expands K and V from it;
 *        yarn_get_mscale corrects the attention scale).
 *
 * Shapes fixed by the model: H = 32 heads, D_NOPE = 128, D_ROPE = 64,
 * D_LATENT = 512, D_V = 128.  One cache row per token and layer is
 * [c_kv (512) | k_pe rotated (64)] bf16 = 1152 bytes; the cache is paged in
 * blocks of 64 tokens.  All tensors are row-major and contiguous.  bf16 is
 * IEEE bfloat16 stored as 16-bit words.
 *
 * Conventions for every call:
 *   - Ownership: the caller owns every buffer.  The library never allocates,
 *     frees or synchronises.  Device pointers must point to memory of the
 *     current CUDA device.
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy
 *     default stream).  Work is enqueued asynchronously on it.
 *   - Errors: argument and shape errors are detected on the host and return
 *     at once with nothing launched.  A failed launch returns XMLA_ERR_CUDA.
 *     Errors the device detects (a block id outside the pool, a sequence
 *     length outside [q_len, max_seqlen], a bounded wait that ran out) are
 *     written to *status_dev when it is not NULL (the first error wins via an
 *     atomic compare-and-swap on XMLA_OK); the caller reads it after
 *     synchronising.  No kernel traps or faults on bad data: out-of-range
 *     block ids are skipped (append) or read as zeros (decode).
 */
#ifndef XMLA_H
#define XMLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  XMLA_OK = 0,
  XMLA_ERR_INVALID_ARG = 1, /* null pointer, misaligned pointer, bad scalar */
  XMLA_ERR_SHAPE = 2,       /* sizes out of the supported range */
  XMLA_ERR_WORKSPACE = 3,   /* workspace smaller than xmla_decode_workspace_size */
  XMLA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
  XMLA_ERR_DEVICE_OOB = 5,  /* device: block id or sequence length out of range */
  XMLA_ERR_TIMEOUT = 6,     /* device: a bounded wait inside a kernel ran out */
  XMLA_ERR_UNSUPPORTED = 7  /* device lacks sm_100a features */
} xmla_status;

/* YaRN rope_scaling parameters, [P1] section 一.  rope_theta is not printed on
 * the pages; xmla_yarn_default sets it to 10000. */
typedef struct {
  double rope_theta;                        /* RoPE base */
  double factor;                            /* 64 */
  int64_t original_max_position_embeddings; /* 4096 */
  double beta_fast;                         /* 32 */
  double beta_slow;                         /* 1 */
  double mscale;                            /* 1.0 */
  double mscale_all_dim;                    /* 1.0 */
  int32_t rotary_dim;                       /* 64 (only 64 is supported) */
} xmla_yarn_cfg;

/* Fill *cfg with the Xing4.0-29B-A4B rope_scaling of [P1] section 一 and
 * rope_theta = 10000.  A NULL cfg is ignored. */
void xmla_yarn_default(xmla_yarn_cfg* cfg);

/* The YaRN inverse-frequency table, computed on the host in float64
 * (NTK-by-parts interpolation of the YaRN paper, section 3.2; [P1] section 一
 * gives the parameters).  inv_freq_out: host array of rotary_dim/2 doubles.
 * Errors: XMLA_ERR_INVALID_ARG for NULL pointers or non-positive
 * theta/factor/lengths, XMLA_ERR_SHAPE if rotary_dim != 64. */
xmla_status xmla_yarn_inv_freq(const xmla_yarn_cfg* cfg, double* inv_freq_out);

/* Softmax (logit) scale qk_head_dim^-1/2 * yarn_get_mscale(factor,
 * mscale_all_dim)^2 ([P5] MLA section: yarn_get_mscale corrects the attention
 * scale; [P1] section 一: the YaRN alignment includes attention-logit
 * scaling).  0.14467962580268923 for the default config and qk_head_dim 192.
 * Returns 0.0 for a NULL cfg or qk_head_dim <= 0. */
double xmla_softmax_scale(const xmla_yarn_cfg* cfg, int32_t qk_head_dim);

/* In-place YaRN RoPE on bf16 vectors ([P5] MLA section: the 64-dim rope part
 * of q and k carries the YaRN rotary embedding).
 *   x: device bf16; vector (r, h) starts at element
 *      r*row_stride_elems + h*head_stride_elems + rope_offset_elems and is
 *      rotary_dim (64) wide.  Dimension i is paired with i + 32 and rotated by
 *      angle positions[r] * inv_freq[i] (angle formed in float64 from the
 *      exact int64 position), scaled by mscale(factor, mscale) /
 *      mscale(factor, mscale_all_dim).
 *   positions: device int64 [rows], each in [0, 2^31).
 * Examples: q [B, q_len, 32, 192] -> rows = B*q_len, n_heads = 32,
 * head_stride 192, row_stride 6144, rope_offset 128; k_pe [T, 64] -> rows = T,
 * n_heads = 1, head_stride 64, row_stride 64, rope_offset 0.
 * rows == 0 is a no-op.  Errors: XMLA_ERR_INVALID_ARG (NULL cfg/x/positions
 * with rows > 0, odd element offsets), XMLA_ERR_SHAPE (rotary_dim != 64,
 * n_heads < 1, rows < 0), XMLA_ERR_CUDA. */
xmla_status xmla_rope_yarn(const xmla_yarn_cfg* cfg, void* x, int64_t rows, int32_t n_heads,
                           int64_t head_stride_elems, int64_t row_stride_elems,
                           int32_t rope_offset_elems, const int64_t* positions, void* stream);

/* Append token rows to the paged latent cache ([P1] section 二 and [P5] MLA
 * section: per token and layer the cache holds the latent and the rope key).
 * For i < T:  pool[block_table[seq_ids[i]*max_blocks + positions[i]/64]]
 *                 [positions[i] % 64] = [c_kv[i] (512) | k_rot[i] (64)]
 * where k_rot[i] = k_pe[i] when rope_cfg is NULL (an exact bit copy of rows
 * rotated beforehand, e.g. by xmla_rope_yarn), and otherwise the YaRN RoPE of
 * k_pe[i] at positions[i] with rope_cfg, computed as xmla_rope_yarn does
 * (float64 angle, one bf16 rounding).  c_kv is always copied bit-exactly.
 *   pool: device bf16 [num_blocks, 64, 576] (written);
 *   block_table: device int32 [batch, max_blocks];
 *   seq_ids: device int32 [T] in [0, batch); positions: device int64 [T];
 *   c_kv: device bf16 [T, 512]; k_pe: device bf16 [T, 64];
 *   rope_cfg: host pointer or NULL (see above).
 * A row whose seq id, position or block id falls outside its range is skipped
 * and XMLA_ERR_DEVICE_OOB is recorded in *status_dev (if not NULL).
 * T == 0 is a no-op.  Errors: XMLA_ERR_INVALID_ARG, XMLA_ERR_SHAPE, XMLA_ERR_CUDA. */
xmla_status xmla_cache_append(void* pool, int64_t num_blocks, const int32_t* block_table,
                              int32_t max_blocks, int32_t batch, const int32_t* seq_ids,
                              const int64_t* positions, const void* c_kv, const void* k_pe,
                              const xmla_yarn_cfg* rope_cfg, int64_t T, int32_t* status_dev,
                              void* stream);

/* Produce and append the cache rows of T tokens from their hidden states
 * ([P5] MLA section: kv_a_proj_with_mqa = Linear(hidden_size, 512 + 64)
 * compresses a token into the cached latent and rope key; hidden size 3584 from
 * the model summary page "Xing4.0", architecture paragraph; [P1] section 一:
 * attention_bias false).  For i < T:
 *   y = hidden[i] . W_kva^T (+ bias), each of the 576 outputs rounded to bf16;
 *   c_kv = y[0:512], k_raw = y[512:576];
 *   pool[block_table[seq_ids[i]*max_blocks + positions[i]/64]][positions[i] % 64]
 *       = [c_kv | k_rot]
 * where k_rot is the YaRN RoPE of k_raw at positions[i] with rope_cfg (float64
 * angle, one bf16 rounding, as xmla_rope_yarn), or k_raw when rope_cfg is NULL.
 * Accumulation in fp32.
 *   hidden: device bf16 [T, 3584], 16-byte aligned;
 *   W_kva: device bf16 [576, 3584] (Linear weight layout), 16-byte aligned;
 *   bias: device bf16 [576] or NULL (no bias);
 *   pool, block_table, max_blocks, batch, seq_ids, positions, status_dev: as in
 *   xmla_cache_append (rows out of range are skipped and reported).
 * T == 0 is a no-op.  Errors: XMLA_ERR_INVALID_ARG, XMLA_ERR_SHAPE, XMLA_ERR_CUDA. */
xmla_status xmla_kv_produce(const void* hidden, const void* W_kva, const void* bias, int64_t T,
                            const xmla_yarn_cfg* rope_cfg, void* pool, int64_t num_blocks,
                            const int32_t* block_table, int32_t max_blocks, int32_t batch,
                            const int32_t* seq_ids, const int64_t* positions,
                            int32_t* status_dev, void* stream);

/* Bytes of device workspace xmla_decode needs for these sizes on a device with
 * num_sms SMs (num_splits = 0 picks the split count automatically, > 0 forces
 * it).  Returns 0 for unsupported sizes. */
size_t xmla_decode_workspace_size(int32_t batch, int32_t q_len, int64_t max_seqlen,
                                  int32_t num_sms, int32_t num_splits);

/* Number of KV splits xmla_decode uses for these sizes (0 for unsupported sizes). */
int32_t xmla_decode_num_splits(int32_t batch, int32_t q_len, int64_t max_seqlen, int32_t num_sms,
                               int32_t num_splits);

/* MLA decode in the weight-absorbed form ([P5] MLA section; W_UK and W_UV are
 * the per-head K_nope and V blocks of kv_b_proj, without bias as
 * attention_bias is false in [P1] section 一):
 *   pos[b,j]      = seqlens[b] - q_len + j  (the q_len new tokens are the last
 *                   q_len cache entries of sequence b)
 *   q_lat[b,j,h]  = W_UK[h]^T q_nope[b,j,h]                      (512)
 *   q_rot[b,j,h]  = YaRN RoPE of q_pe[b,j,h] at pos[b,j] (as xmla_rope_yarn,
 *                   without an intermediate bf16 rounding)
 *   S[b,j,h,t]    = softmax_scale * (q_lat . c_kv[t] + q_rot . k_pe_rot[t])
 *   P             = softmax over t <= seqlens[b] - q_len + j     (causal among
 *                   the q_len newest tokens, which are in the cache already)
 *   out[b,j,h]    = W_UV[h]^T (sum_t P c_kv[t])                  (128)
 * Tokens are read in logical order through block_table (token t of sequence b
 * is row t % 64 of block block_table[b*max_blocks + t/64]).
 *   cfg: YaRN parameters used to rotate q_pe (host pointer);
 *   q: device bf16 [batch, q_len, 32, 192] = [q_nope 128 | q_pe 64], q_pe NOT
 *      rotated (the call rotates it).  This deliberately differs from
 *      rotating q_pe with xmla_rope_yarn before the call: a q_pe already
 *      rotated would be rotated a second time, so pass the raw query.  q and
 *      out may also be pinned host memory mapped into the device (unified
 *      addressing) when q_len <= 8: they are read and written with ordinary
 *      loads and stores; a prompt chunk (q_len > 8) reads q by TMA and needs
 *      it in device memory;
 *   W_UK: device bf16 [32, 128, 512]; W_UV: device bf16 [32, 512, 128];
 *   pool: device bf16 [num_blocks, 64, 576], 16-byte aligned;
 *   block_table: device int32 [batch, max_blocks];
 *   seqlens: device int32 [batch], each in [q_len, max_seqlen] (includes the
 *      q_len new tokens);
 *   max_seqlen: host upper bound of seqlens, <= max_blocks*64;
 *   softmax_scale: usually xmla_softmax_scale(cfg, 192);
 *   num_splits: 0 = automatic, > 0 forces the KV split count;
 *   workspace: device scratch of >= xmla_decode_workspace_size(...) bytes,
 *      256-byte aligned; its contents on entry do not matter;
 *   status_dev: device int32 or NULL (see conventions);
 *   out: device bf16 [batch, q_len, 32, 128].
 * Supported: 1 <= batch, 1 <= q_len <= 65536, q_len <= max_seqlen <= 2^31 - 64,
 * num_blocks*64 < 2^31.  A q_len of a few tokens is a decode step (speculative
 * verification above 1); a long q_len is a chunk of a prompt (chunked
 * prefill), attended causally: each query sees the cache up to its own
 * position.  Up to 63 new tokens per sequence the chunk runs in the same
 * absorbed form as a decode step; from 64 on, in the non-absorbed form of the
 * MLA module ([P5] MLA section: kv_b_proj expands K_nope and V per head from
 * the cached latent): K_nope and V of every cached token are expanded per
 * head into the workspace, then attention runs per head over [K_nope |
 * rotated k_pe] and V with fp16 tensor-core operands.  The workspace then
 * holds, per sequence, max_seqlen (rounded up to 128) tokens x 32 heads x 256
 * fp16 values.  Errors: XMLA_ERR_INVALID_ARG, XMLA_ERR_SHAPE,
 * XMLA_ERR_WORKSPACE, XMLA_ERR_CUDA, XMLA_ERR_UNSUPPORTED (not an sm_100
 * device); device errors via status_dev. */
xmla_status xmla_decode(const xmla_yarn_cfg* cfg, const void* q, const void* W_UK,
                        const void* W_UV, const void* pool, int64_t num_blocks,
                        const int32_t* block_table, int32_t max_blocks, const int32_t* seqlens,
                        int32_t batch, int32_t q_len, int64_t max_seqlen,
                        float softmax_scale, int32_t num_splits, void* workspace,
                        size_t workspace_bytes, int32_t* status_dev, void* out, void* stream);

/* xmla_decode that also records two CUDA events (cudaEvent_t passed as void*,
 * either may be NULL) on `stream` immediately before and after the split-K
 * attention kernel, so a caller can time that kernel alone.  Inside a stream
 * capture the records become event-record graph nodes.  Same arguments,
 * results and errors as xmla_decode otherwise. */
xmla_status xmla_decode_profiled(const xmla_yarn_cfg* cfg, const void* q, const void* W_UK,
                                 const void* W_UV, const void* pool, int64_t num_blocks,
                                 const int32_t* block_table,
                                 int32_t max_blocks, const int32_t* seqlens, int32_t batch,
                                 int32_t q_len, int64_t max_seqlen, float softmax_scale,
                                 int32_t num_splits, void* workspace, size_t workspace_bytes,
                                 int32_t* status_dev, void* out, void* stream, void* attn_start,
                                 void* attn_stop);

/* ---- 8-bit latent cache ([P1] section 三, 方案 A: a q8_0 KV cache halves
 * the bytes of the bf16 one at a small precision cost; the page names 8-bit
 * codes with one scale per block of 32 values).
 *
 * Row layout (608 bytes per token, 16-byte aligned rows): bytes [0, 576) are
 * int8 codes of [c_kv 512 | rotated k_pe 64]; bytes [576, 594) the int8
 * exponents e of blocks 0..17 (block k = values [32k, 32k+32)); bytes
 * [594, 608) zero.  Value = code * 2^e.  Quantisation of a bf16 row: e = the
 * smallest integer with 127 * 2^e >= max |x| over the block, clamped to
 * [-14, 8]; code = x / 2^e rounded to nearest (ties to even), clamped to
 * [-127, 127].  The power-of-two scale keeps every value exact in f16.  A
 * pool is [num_blocks, 64, 608] bytes, addressed through the block table as
 * the bf16 pool. */

/* Quantise and append T token rows: row i = [c_kv[i] | k_rot[i]] goes to
 * block block_table[seq_ids[i]*max_blocks + positions[i]/64], row
 * positions[i] % 64, of pool_q8, where k_rot is the YaRN RoPE of k_pe[i] at
 * positions[i] rounded to bf16 (float64 angle, as xmla_rope_yarn), or k_pe[i]
 * itself when rope_cfg is NULL.
 *   pool_q8: device [num_blocks, 64, 608] bytes, 16-byte aligned;
 *   c_kv: device bf16 [T, 512]; k_pe: device bf16 [T, 64], both 16-byte aligned;
 *   other arguments as xmla_cache_append (rows out of range are skipped and
 *   reported through status_dev).
 * T == 0 is a no-op.  Errors: XMLA_ERR_INVALID_ARG, XMLA_ERR_SHAPE, XMLA_ERR_CUDA. */
xmla_status xmla_cache_append_q8(void* pool_q8, int64_t num_blocks, const int32_t* block_table,
                                 int32_t max_blocks, int32_t batch, const int32_t* seq_ids,
                                 const int64_t* positions, const void* c_kv, const void* k_pe,
                                 const xmla_yarn_cfg* rope_cfg, int64_t T, int32_t* status_dev,
                                 void* stream);

/* Workspace bytes and split count of xmla_decode_q8 (0 for unsupported sizes). */
size_t xmla_decode_q8_workspace_size(int32_t batch, int32_t q_len, int64_t max_seqlen,
                                     int32_t num_sms, int32_t num_splits);
int32_t xmla_decode_q8_num_splits(int32_t batch, int32_t q_len, int64_t max_seqlen,
                                  int32_t num_sms, int32_t num_splits);

/* xmla_decode over an 8-bit pool: the same attention with c_kv and k_pe_rot
 * the dequantised values code * 2^e of each cached row.  The products run on
 * the tensor cores in f16 (the absorbed query rounded once to f16, the
 * probabilities to f16, fp32 accumulation).  Arguments as xmla_decode except
 * pool_q8 (device [num_blocks, 64, 608] bytes, 16-byte aligned) and the
 * workspace size (xmla_decode_q8_workspace_size).  Supported: 1 <= q_len <= 8,
 * other limits as xmla_decode.  Errors as xmla_decode. */
xmla_status xmla_decode_q8(const xmla_yarn_cfg* cfg, const void* q, const void* W_UK,
                           const void* W_UV, const void* pool_q8, int64_t num_blocks,
                           const int32_t* block_table, int32_t max_blocks, const int32_t* seqlens,
                           int32_t batch, int32_t q_len, int64_t max_seqlen, float softmax_scale,
                           int32_t num_splits, void* workspace, size_t workspace_bytes,
                           int32_t* status_dev, void* out, void* stream);

/* xmla_decode_q8 with CUDA events around its attention kernel, as
 * xmla_decode_profiled. */
xmla_status xmla_decode_q8_profiled(const xmla_yarn_cfg* cfg, const void* q, const void* W_UK,
                                    const void* W_UV, const void* pool_q8, int64_t num_blocks,
                                    const int32_t* block_table, int32_t max_blocks,
                                    const int32_t* seqlens, int32_t batch, int32_t q_len,
                                    int64_t max_seqlen, float softmax_scale, int32_t num_splits,
                                    void* workspace, size_t workspace_bytes, int32_t* status_dev,
                                    void* out, void* stream, void* attn_start, void* attn_stop);

/* One decode step ([P5] MLA section; [P1] sections 一 and 二): append the
 * step's T new token rows to the cache, then attend.  The result is that of
 *   xmla_cache_append(pool, num_blocks, block_table, max_blocks, batch, seq_ids,
 *                     positions, c_kv, k_pe, cfg, T, status_dev, stream);
 *   xmla_decode_profiled(cfg, q, ..., attn_start, attn_stop);
 * (k_pe is raw and is rotated with cfg at positions[i]), but the append runs
 * inside the first kernel of the decode chain, beside the query absorb, which
 * saves one kernel boundary.  Arguments as in those two calls; T >= 0 (T == 0
 * appends nothing); c_kv and k_pe 16-byte aligned.  A new row must not share
 * its cache slot with another row of the same call.  Errors: the union of
 * theirs. */
xmla_status xmla_decode_step(const xmla_yarn_cfg* cfg, const void* q, const void* W_UK,
                             const void* W_UV, void* pool, int64_t num_blocks,
                             const int32_t* block_table, int32_t max_blocks,
                             const int32_t* seqlens, int32_t batch, int32_t q_len,
                             int64_t max_seqlen, const int32_t* seq_ids, const int64_t* positions,
                             const void* c_kv, const void* k_pe, int64_t T, float softmax_scale,
                             int32_t num_splits, void* workspace, size_t workspace_bytes,
                             int32_t* status_dev, void* out, void* stream, void* attn_start,
                             void* attn_stop);

/* One decode step from the new tokens' hidden states: xmla_kv_produce (the
 * kv_a_proj_with_mqa projection, RoPE of the rope key with cfg, append) and then
 * xmla_decode_profiled, with the producer's blocks inside the first kernel of
 * the decode chain beside the query absorb.  Arguments as in those two calls
 * (hidden [T, 3584], W_kva [576, 3584], bias [576] or NULL); T >= 0.  A new row
 * must not share its cache slot with another row of the same call.  Errors:
 * the union of theirs. */
xmla_status xmla_decode_step_from_hidden(const xmla_yarn_cfg* cfg, const void* q,
                                         const void* W_UK, const void* W_UV, const void* hidden,
                                         const void* W_kva, const void* bias, void* pool,
                                         int64_t num_blocks, const int32_t* block_table,
                                         int32_t max_blocks, const int32_t* seqlens,
                                         int32_t batch, int32_t q_len, int64_t max_seqlen,
                                         const int32_t* seq_ids, const int64_t* positions,
                                         int64_t T, float softmax_scale, int32_t num_splits,
                                         void* workspace, size_t workspace_bytes,
                                         int32_t* status_dev, void* out, void* stream,
                                         void* attn_start, void* attn_stop);

/* ---- Sequence-parallel decode: one sequence's pages spread over G GPUs.
 * ([P5] MLA section: the absorbed attention is a softmax-weighted sum of the
 * cached latent rows, so it splits over any partition of a sequence's tokens
 * and the parts merge exactly by their log-sum-exp.  [P1] "256K 长上下文真能
 * 本地用：Xing4.0 原生长上下文的工程代价拆解", introduction: contexts of this
 * size are usually run on several data-centre GPUs; [P3] "别把上下文开满：3.0
 * Flash 256K 最稳背后的设置避坑" (another model), hardware paragraph: its
 * longest contexts need a second GPU.)
 *
 * Rank g of G holds logical pages [page_lo, page_hi) of every sequence in its
 * own pool (block_table is indexed by the logical page; entries outside the
 * rank's range are not read).  Each rank calls xmla_decode_shard, the ranks
 * all-gather their partials (rank order, one after another), and every rank
 * (or one) calls xmla_combine_shards on the gathered buffer. */

/* Floats of one rank's partial: batch * q_len * 32 * 514 (0 for bad sizes).
 * Layout, with R = batch * q_len * 32 and row index (b * q_len + j) * 32 + h:
 *   [R][512]  O, unnormalised, relative to M
 *   [R][2]    (M, L): running maximum (log2 units, scale folded in) and sum
 * A row that saw no token has M = -inf, L = 0, O = 0. */
size_t xmla_shard_partial_floats(int32_t batch, int32_t q_len);

/* Workspace bytes of xmla_decode_shard for a rank's page range; the split
 * count is sized for page_hi - page_lo pages.  0 for unsupported sizes. */
size_t xmla_decode_shard_workspace_size(int32_t batch, int32_t q_len, int64_t max_seqlen,
                                        int64_t page_lo, int64_t page_hi, int32_t num_sms,
                                        int32_t num_splits);

/* One rank's part of a sequence-parallel decode: the query absorb, the
 * split-K attention over the logical pages [page_lo, page_hi) of each
 * sequence (clipped to the sequence; causal masking and the last-page
 * handling use the global positions), and the merge of its splits into
 * shard_partial (device, xmla_shard_partial_floats floats, 16-byte aligned,
 * caller-owned, overwritten).  Other arguments as in xmla_decode; seqlens
 * are the global sequence lengths.  Errors: those of xmla_decode;
 * XMLA_ERR_SHAPE if page_lo < 0 or page_hi < page_lo. */
xmla_status xmla_decode_shard(const xmla_yarn_cfg* cfg, const void* q, const void* W_UK,
                              const void* pool, int64_t num_blocks, const int32_t* block_table,
                              int32_t max_blocks, const int32_t* seqlens, int32_t batch,
                              int32_t q_len, int64_t max_seqlen, float softmax_scale,
                              int64_t page_lo, int64_t page_hi, int32_t num_splits,
                              void* workspace, size_t workspace_bytes, int32_t* status_dev,
                              float* shard_partial, void* stream);

/* Merge of num_shards gathered partials (device, num_shards *
 * xmla_shard_partial_floats floats, rank-major, 16-byte aligned) and the
 * W_UV product: out[b, j, h, :] (bf16, [batch, q_len, 32, 128]) as
 * xmla_decode writes it.  Errors: XMLA_ERR_INVALID_ARG (null or misaligned),
 * XMLA_ERR_SHAPE (sizes, num_shards outside [1, 1024]), XMLA_ERR_UNSUPPORTED,
 * XMLA_ERR_CUDA. */
xmla_status xmla_combine_shards(const float* partials, int32_t num_shards, const void* W_UV,
                                int32_t batch, int32_t q_len, void* out, void* stream);

/* Size in bytes of the fixed device scratch used by xmla_decode_noalloc. */
#define XMLA_NOALLOC_SCRATCH_BYTES (32u << 20)

/* xmla_decode for callers that must not allocate device memory.  (The source
 * pages describe the model, not a library; this entry point has no
 * counterpart there.)
 *
 * Some callers cannot provide or allocate scratch: a plugin or backend inside
 * an inference server whose host process owns every device allocation, code
 * that runs on a latency-critical path where cudaMalloc's implicit device
 * synchronisation and allocator locks are not acceptable, or a program whose
 * memory is pre-carved into a fixed arena.  This entry point takes the same
 * inputs and output as xmla_decode but no workspace: its scratch is a fixed
 * XMLA_NOALLOC_SCRATCH_BYTES array compiled into the library, which every GPU
 * that loads the library keeps until the process exits.  It calls no
 * cudaMalloc, cudaFree or allocating routine.
 *
 * Limits and behaviour:
 *   - Sizes whose workspace (xmla_decode_workspace_size) exceeds
 *     XMLA_NOALLOC_SCRATCH_BYTES are rejected with XMLA_ERR_WORKSPACE before
 *     anything is launched.
 *   - The first call in a CUDA context looks up the scratch array's device
 *     address in that context (cudaGetSymbolAddress) and caches it for that
 *     context only (a context created anew, e.g. after cudaDeviceReset, gets
 *     a fresh lookup); make that first call before any stream capture on
 *     the device.
 *   - All calls share the one array and it keeps the previous call's
 *     contents.  Nothing in it has to start at zero: every value a call reads
 *     was written earlier by the same call.  Calls whose work may overlap on
 *     the GPU (concurrent streams, or several host threads) race on the array
 *     and give wrong results; serialise them.
 * Results equal xmla_decode's for the same arguments and split count. */
xmla_status xmla_decode_noalloc(const xmla_yarn_cfg* cfg, const void* q, const void* W_UK,
                                const void* W_UV, const void* pool, int64_t num_blocks,
                                const int32_t* block_table, int32_t max_blocks,
                                const int32_t* seqlens, int32_t batch, int32_t q_len,
                                int64_t max_seqlen, float softmax_scale, int32_t num_splits,
                                int32_t* status_dev, void* out, void* stream);

/* Self-test of the kernels' bounded wait: launches one CTA that waits on a
 * shared-memory barrier nothing ever arrives on, with the given limit in
 * nanoseconds, and records XMLA_ERR_TIMEOUT in *status_dev when the wait gives
 * up (the kernel then returns normally; the context stays usable). */
xmla_status xmla_selftest_wait_timeout(int32_t* status_dev, uint64_t timeout_ns, void* stream);

/* Static description of a status code. */
const char* xmla_status_string(xmla_status s);

#ifdef __cplusplus
}
#endif

#endif /* XMLA_H */
