/*
 * pa.h -- C ABI of the B200 paged-KV-cache decode library (libpa369.so).
 *
 * The operation, as the pages state it:
 *   - the KV cache is cut into fixed blocks of 16 tokens that sit anywhere in a
 *     physical block pool; each sequence owns a block table mapping its logical
 *     blocks to physical ones ("Transformer 推理优化：KV Cache、PagedAttention 与
 *     vLLM", §3.2-§3.3; "KV Cache 与 PageAttention深度实战", §3.1-§3.2);
 *   - a decode step computes, for the single new query row of each sequence,
 *     Attention(Q_t, [K_prefix, K_t], [V_prefix, V_t]) =
 *     softmax(Q_t K^T / sqrt(d_k)) V, reading K and V through the block table
 *     ("KV Cache 与 PageAttention深度实战", §1.2 and §3.2-§3.3);
 *   - the new token's K/V row is appended into its (block, offset) slot; a new
 *     block is opened every 16 tokens ("vLLM推理引擎深度解析：PagedAttention与
 *     连续批处理", §2.2-§2.3);
 *   - the cache may hold 8-bit codes in place of 16-bit values: FP8 E4M3
 *     (range +-448), FP8 E5M2 or INT8
 *     ("大语言模型推理引擎深度剖析：从 KV Cache 内存管理到 PagedAttention、投机
 *     解码与量化加速的完全工程指南", §4.2-§4.3).
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument is DEVICE memory owned by the caller, unless the
 *     comment says otherwise.  The library allocates nothing, keeps no state
 *     between calls and never synchronises: work is enqueued on `stream`
 *     (a cudaStream_t; NULL = the legacy default stream) and the call returns.
 *   - Layouts are dense, row-major, C order:
 *       q, out            [num_seqs, num_q_heads, head_dim]
 *       k_new, v_new      [num_tokens, num_kv_heads, head_dim]
 *       k_cache, v_cache  [num_blocks, num_kv_heads, block_size, head_dim]
 *       block_tables      int32 [num_seqs, max_blocks_per_seq]
 *       seq_lens          int32 [num_seqs]   (tokens in the cache, the one
 *                                             written this step included)
 *       slot_mapping      int64 [num_tokens] (slot = block * block_size + offset;
 *                                             a negative slot is padding)
 *   - GQA: query head h reads KV head h / (num_q_heads / num_kv_heads).
 *   - q, out, the caches and k_new / v_new must be 16-byte aligned.
 *   - Host-side argument checks run before any launch and return
 *     PA_ERR_INVALID_ARG or PA_ERR_UNSUPPORTED without touching the GPU; a
 *     failed launch returns PA_ERR_CUDA.
 *   - `dev_err` (nullable, device int32) receives the first device-side error
 *     of the call (PA_ERR_DEVICE_BOUNDS for a block-table entry, slot, sequence
 *     index or length outside its range; PA_ERR_DEVICE_TIMEOUT for an
 *     asynchronous copy that did not complete in time).  The kernels check every
 *     such index before using it and skip the access, so a corrupt table never
 *     makes them read or write outside the buffers; the affected outputs are
 *     still written (finite).  The caller zeroes *dev_err and reads it after
 *     synchronising.
 */
#ifndef PA369_H
#define PA369_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,    /* null pointer, bad size, misaligned buffer, ... */
    PA_ERR_UNSUPPORTED = 2,    /* valid but not implemented (head_dim, dtype pair, ...) */
    PA_ERR_CUDA = 3,           /* a CUDA launch or query failed */
    PA_ERR_DEVICE_BOUNDS = 4,  /* written to *dev_err by a kernel */
    PA_ERR_DEVICE_TIMEOUT = 5  /* written to *dev_err by a kernel */
} pa_status;

typedef enum pa_dtype {
    PA_F16 = 0,       /* IEEE binary16 */
    PA_BF16 = 1,      /* bfloat16 */
    PA_FP8_E4M3 = 2,  /* OCP E4M3 (FN): bias 7, max 448, no infinities */
    PA_FP8_E5M2 = 3,  /* OCP E5M2: bias 15, max 57344 (infinities and NaNs exist) */
    PA_INT8 = 4       /* symmetric signed 8-bit integer code, -127 .. 127 */
} pa_dtype;

/*
 * 8-bit caches (PA_FP8_E4M3, PA_FP8_E5M2, PA_INT8; the openeuler page's §2.3
 * lists FP8 E5M2 / E4M3 and INT8 KV caches, "大语言模型推理引擎深度剖析"
 * §4.2-§4.3 the FP8 formats and their ranges) store code(x / scale) with one
 * fp32 scale per tensor (K and V separately) and read value = code * scale:
 *   E4M3 / E5M2: x / scale in fp32 (IEEE division), round to nearest even
 *                onto the format, finite overflow and infinity saturating to
 *                +-448 / +-57344, NaN -> NaN;
 *   INT8:        round half to even to an integer, clamped to [-127, 127],
 *                NaN -> 0.
 * The scale is the caller's (e.g. amax / 448, amax / 57344, amax / 127).
 */

/* Human-readable name of a status code (host only, static string). */
const char *pa_status_string(pa_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH (host only). */
int pa_version(void);

/*
 * pa_slot_mapping -- slot of each token to be written (block-table lookup).
 *
 * Source: "Transformer 推理优化：KV Cache、PagedAttention 与 vLLM", §3.3: logical
 * block pos / block_size of sequence s lives in physical block
 * block_tables[s][pos / block_size]; the token sits at offset pos % block_size.
 *
 *   slot_mapping[t] = block_tables[s][pos / B] * B + pos % B,
 *     s   = token_seq ? token_seq[t] : t         (s < 0: padding, slot = -1)
 *     pos = token_pos ? token_pos[t] : seq_lens[s] - 1   (decode: last token)
 *
 * seq_lens may be NULL when token_pos is given.  A sequence index >= num_seqs,
 * a position outside [0, max_blocks_per_seq * B) or a table entry outside
 * [0, num_blocks) gives slot -1 and PA_ERR_DEVICE_BOUNDS in *dev_err.
 */
pa_status pa_slot_mapping(int64_t *slot_mapping, const int32_t *block_tables,
                          int max_blocks_per_seq, const int32_t *seq_lens,
                          const int32_t *token_seq, const int32_t *token_pos, int num_tokens,
                          int num_seqs, int block_size, int num_blocks, int *dev_err,
                          void *stream);

/*
 * pa_cache_write -- append each token's K/V rows into its cache slot.
 *
 * Source: "vLLM推理引擎深度解析：PagedAttention与连续批处理", §2.2 (one new block
 * every 16 generated tokens; the token goes to its slot) and, for FP8, "大语言
 * 模型推理引擎深度剖析", §4.3 (KV stored as E4M3, dequantised for attention).
 *
 *   k_cache[slot / B][h][slot % B][:] = k_new[t][h][:]   (likewise V)
 *
 * act_dtype (of k_new / v_new) is PA_F16 or PA_BF16.  kv_dtype is act_dtype
 * (a bit-exact copy) or an 8-bit format, in which case each value is stored
 * as code(x / scale) as described under pa_dtype (E4M3: rounded to
 * nearest even onto the E4M3 grid and saturated to +-448); k_scale / v_scale
 * must then be finite and > 0.
 * Negative slots are skipped; a slot >= num_blocks * B is skipped with
 * PA_ERR_DEVICE_BOUNDS.  Tokens must map to distinct slots.
 */
pa_status pa_cache_write(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                         const int64_t *slot_mapping, int num_tokens, int num_blocks,
                         int num_kv_heads, int head_dim, int block_size, pa_dtype act_dtype,
                         pa_dtype kv_dtype, float k_scale, float v_scale, int *dev_err,
                         void *stream);

/*
 * pa_decode -- paged decode attention, one pass per (sequence, KV head).
 *
 * Source: "KV Cache 与 PageAttention深度实战", §1.2 (softmax(Q K^T / sqrt(d_k)) V
 * with one new query row per step), §3.2 (reading K/V through the block table
 * gathers them implicitly) and §3.3 (paged block addressing, coalesced loads,
 * the block table kept on chip).
 *
 * For every sequence s, query head h, with g = num_q_heads / num_kv_heads and
 * L = seq_lens[s]:
 *   out[s][h] = sum_t p_t * V_t,  p = softmax_t(softmax_scale * q[s][h] . K_t),
 *   t < L, K_t / V_t rows of KV head h / g read at block_tables[s][t / B],
 *   offset t % B (B = block_size).  For an 8-bit cache, K_t = code * k_scale, V_t = code * v_scale.
 * L = 0 gives a zero row.  Slots at t >= L (the tail of the last block) and
 * unused table entries are never read into the result.
 *
 * Supported: block_size 16 or 32 (the fifth page's §2.2: blocks of 16-32
 * tokens), head_dim 64 or 128, num_q_heads a multiple of
 * num_kv_heads, q_dtype (= out dtype) PA_F16 / PA_BF16, kv_dtype = q_dtype or
 * an 8-bit format (PA_FP8_E4M3, PA_FP8_E5M2, PA_INT8).  Arithmetic is fp32
 * (8-bit codes are widened exactly); out is rounded to nearest even once.
 */
pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_tables, int max_blocks_per_seq, const int32_t *seq_lens,
                    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                    int block_size, int num_blocks, float softmax_scale, pa_dtype q_dtype,
                    pa_dtype kv_dtype, float k_scale, float v_scale, int *dev_err,
                    void *stream);

/*
 * pa_decode_append -- one whole decode step: store every sequence's new token,
 * then attend (slot mapping + cache write + decode [+ split-KV reduce]).
 *
 * Source: the decode form of the pages' step, "KV Cache 与 PageAttention深度
 * 实战", §1.2: Output_t = Attention(Q_t, [K_prefix, K_t], [V_prefix, V_t]) --
 * the new K_t / V_t join the cache ("vLLM推理引擎深度解析：PagedAttention与
 * 连续批处理", §2.2) and take part in the same step's attention.
 *
 * For every sequence s with L = seq_lens[s] > 0 (L counts the new token), the
 * rows k_new[s] / v_new[s] ([num_seqs, num_kv_heads, head_dim], q dtype) are
 * stored at position L - 1, i.e. slot block_tables[s][(L-1)/16]*16 + (L-1)%16,
 * exactly as pa_slot_mapping + pa_cache_write store them (same 8-bit
 * quantisation, same bits); then out is computed as by pa_decode
 * (partition_size == 0: single pass, workspace unused and may be NULL) or by
 * pa_decode_split_reduce (partition_size > 0: a positive multiple of 16,
 * workspace as documented there).  The tensor-core kernel stores the new
 * token from inside the attention launch, so the step is one launch (single
 * pass) or two (split).  The pools are written: k_cache / v_cache are not
 * const here.  Errors as for pa_decode_split_reduce; a new token whose table
 * entry is out of range is not stored (PA_ERR_DEVICE_BOUNDS).
 */
pa_status pa_decode_append(void *out, const void *q, const void *k_new, const void *v_new,
                           void *k_cache, void *v_cache, const int32_t *block_tables,
                           int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs,
                           int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                           int num_blocks, float softmax_scale, pa_dtype q_dtype,
                           pa_dtype kv_dtype, float k_scale, float v_scale, int partition_size,
                           int max_seq_len, void *workspace, size_t workspace_bytes, int *dev_err,
                           void *stream);

/*
 * Workspace bytes pa_decode_split_reduce needs: with
 * NP = ceil(max_seq_len / partition_size) partitions,
 *   lse [num_seqs, num_q_heads, NP] fp32, then o [num_seqs, num_q_heads, NP, head_dim] fp32,
 * each section starting on a 256-byte boundary.  Returns 0 on invalid input.
 * Host only.
 */
size_t pa_split_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, int max_seq_len,
                                int partition_size);

/*
 * pa_decode_split_reduce -- split-KV decode: partition kernel + reduce kernel.
 *
 * Same result as pa_decode (up to fp32 rounding order), computed in two
 * launches for long or uneven contexts.  The pages do not describe this split;
 * it is the standard log-sum-exp decomposition of the same softmax.
 *   1. Partition: for every (s, KV head, p) the tokens
 *      [p * P, min((p + 1) * P, L)) of sequence s give, per query head,
 *        lse[s][h][p] = ln sum_t exp(softmax_scale * q . K_t)   (-inf if empty)
 *        o[s][h][p][:] = sum_t softmax-weight_t V_t over the partition (0 if empty)
 *   2. Reduce: M = max_p lse, w_p = exp(lse_p - M),
 *        out[s][h] = sum_p w_p o_p / sum_p w_p      (0 if every partition is empty)
 * partition_size P is a positive multiple of 16, at most 2^30 (a partition
 * may end inside a 32-token block); max_seq_len, at most 2^30, bounds
 * every seq_lens[s] (a longer one is truncated and flags PA_ERR_DEVICE_BOUNDS).
 * workspace (device, caller-owned, >= pa_split_workspace_bytes(...) bytes,
 * 256-byte aligned) holds the partials in the layout above after the call;
 * it needs no initialisation.
 */
pa_status pa_decode_split_reduce(void *out, const void *q, const void *k_cache,
                                 const void *v_cache, const int32_t *block_tables,
                                 int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs,
                                 int num_q_heads, int num_kv_heads, int head_dim,
                                 int block_size, int num_blocks, float softmax_scale,
                                 pa_dtype q_dtype, pa_dtype kv_dtype, float k_scale,
                                 float v_scale, int partition_size, int max_seq_len,
                                 void *workspace, size_t workspace_bytes, int *dev_err,
                                 void *stream);

/*
 * pa_prefill -- chunked-prefill attention: several new query tokens per
 * sequence, causal, over the paged cache.
 *
 * Source: "openeuler.csdn.net 推理优化篇", §4.5 (Chunked Prefill: a long prompt
 * is cut into chunks, e.g. 512 tokens, processed one after another and mixed
 * with decode steps) and "vLLM推理引擎深度解析：PagedAttention与连续批处理",
 * §3.3; the attention itself is the pages' softmax(Q K^T / sqrt(d_k)) V with
 * K / V read through the block table ("KV Cache 与 PageAttention深度实战",
 * §1.2, §3.2).
 *
 * Sequence s has L = seq_lens[s] tokens in the cache, the chunk included; its
 * chunk is the last n = query_start[s+1] - query_start[s] of them (its K/V
 * rows are already stored, e.g. by pa_slot_mapping with token positions +
 * pa_cache_write).  Its query token j is row query_start[s] + j of q and out
 * ([num_tokens, num_q_heads, head_dim]) and sits at position L - n + j:
 *   out[row][h] = sum_t p_t V_t,  p = softmax_t(softmax_scale * q[row][h] . K_t),
 *   t = 0 .. L - n + j   (causal), KV head h / (num_q_heads / num_kv_heads).
 * A chunk of one token is a decode step.  query_start ([num_seqs + 1], device
 * int32) is non-decreasing with query_start[num_seqs] <= num_tokens; rows no
 * sequence covers are not written.  max_query_len bounds every n.
 *
 * Supported: block_size 16 or 32, head_dim 64 or 128, q_dtype (= out dtype)
 * PA_F16 or PA_BF16, kv_dtype = q_dtype or, with head_dim 128, an 8-bit
 * format read as code * k_scale / code * v_scale (per-tensor scales, finite
 * and > 0; ignored for 16-bit caches; the codes are widened to f16 exactly
 * in shared memory and the MMAs then run in f16, q scaled by a power of two
 * into f16 range), GQA
 * groups up to 128, num_seqs and num_kv_heads up to 65535, softmax_scale
 * finite and > 0 (else PA_ERR_INVALID_ARG).  Arithmetic is
 * fp32 with the probabilities kept to ~16 bits (bf16 hi + lo) or f16; out is
 * rounded to nearest even once.  Errors as for pa_decode: a chunk longer
 * than its sequence or than max_query_len, a length past the table, or a
 * table entry outside the pool flags PA_ERR_DEVICE_BOUNDS (that sequence's
 * rows are then not written, or the bad block reads as zeros).
 *
 * The launch is persistent (one CTA per SM taking work items from a device
 * counter inside the library).  The library keeps 64 such counters and gives
 * each launch the next one in turn, so at most 64 pa_prefill or
 * pa_decode_shared_prefix launches may be in flight at the same time (on
 * different streams); a launch resets its counter when it finishes.
 */
pa_status pa_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                     const int32_t *block_tables, int max_blocks_per_seq, const int32_t *seq_lens,
                     const int32_t *query_start, int num_seqs, int num_tokens, int max_query_len,
                     int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                     int num_blocks, float softmax_scale, pa_dtype q_dtype, pa_dtype kv_dtype,
                     float k_scale, float v_scale, int *dev_err, void *stream);

/*
 * pa_copy_blocks -- copy whole KV blocks inside the pools (copy-on-write).
 *
 * Source: "Transformer 推理优化：KV Cache、PagedAttention 与 vLLM", §3.5 (beam
 * search: candidates share their common blocks; only the block where they
 * diverge is new) and "大语言模型推理引擎深度剖析", §2.3 (before a request
 * writes into a block it shares, the engine copies the block; refcounts
 * track the sharing).  The engine decides which blocks to copy and repoints
 * its block tables; this call moves the bytes.
 *
 *   for every i < num_pairs, with (src, dst) = (block_pairs[2i], block_pairs[2i+1]):
 *     k_cache[dst][:][:][:] = k_cache[src][:][:][:]   and likewise v_cache
 *   (a block is num_kv_heads x block_size x head_dim elements of kv_dtype).
 *
 * block_pairs: device int32 [num_pairs][2].  The pairs are copied
 * concurrently: no dst may appear twice or also be a src in the same call
 * (then the result equals copying the pairs in order); src == dst is a
 * no-op.  A pair with an id outside [0, num_blocks) is skipped and flags
 * PA_ERR_DEVICE_BOUNDS in *dev_err.  k_cache / v_cache 16-byte aligned;
 * kv_dtype any pa_dtype (only its size matters).
 */
pa_status pa_copy_blocks(void *k_cache, void *v_cache, const int32_t *block_pairs, int num_pairs,
                         int num_blocks, int num_kv_heads, int head_dim, int block_size,
                         pa_dtype kv_dtype, int *dev_err, void *stream);

/*
 * Per-channel scales for 8-bit caches.
 *
 * Source: "大语言模型推理引擎深度剖析：从 KV Cache 内存管理到 PagedAttention、投机
 * 解码与量化加速的完全工程指南", §4.3 (per-channel FP8/E4M3: each channel of K /
 * V quantised on its own, stored as FP8, widened for attention).
 *
 * k_scales / v_scales: device fp32 [num_kv_heads, head_dim], finite and > 0,
 * 16-byte aligned for the cache write.  Channel i of KV head h stores
 * code(x / scales[h][i]) (rounding as under pa_dtype) and reads
 * code * scales[h][i].  kv_dtype must be an 8-bit format.
 *
 * pa_cache_write_per_channel: pa_cache_write with those scales in place of
 * the per-tensor ones (same slots, same errors).
 *
 * pa_decode_per_channel: decode over such a cache; partition_size 0 runs the
 * single-pass kernel (workspace unused, may be NULL), a positive multiple of
 * 16 runs split-KV with the workspace of pa_decode_split_reduce.  The K
 * scales are folded into q (q . (code * s) = (q * s) . code) and the V scales
 * applied to each output channel, so the inner loop is the per-tensor one.
 * Results, supported shapes and errors as for pa_decode /
 * pa_decode_split_reduce.
 */
pa_status pa_cache_write_per_channel(const void *k_new, const void *v_new, void *k_cache,
                                     void *v_cache, const int64_t *slot_mapping, int num_tokens,
                                     int num_blocks, int num_kv_heads, int head_dim,
                                     int block_size, pa_dtype act_dtype, pa_dtype kv_dtype,
                                     const float *k_scales, const float *v_scales, int *dev_err,
                                     void *stream);

pa_status pa_decode_per_channel(void *out, const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *block_tables, int max_blocks_per_seq,
                                const int32_t *seq_lens, int num_seqs, int num_q_heads,
                                int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                float softmax_scale, pa_dtype q_dtype, pa_dtype kv_dtype,
                                const float *k_scales, const float *v_scales, int partition_size,
                                int max_seq_len, void *workspace, size_t workspace_bytes,
                                int *dev_err, void *stream);

/*
 * pa_decode_shared_prefix -- decode for a batch whose sequences all begin with
 * the same cached prefix (the same physical blocks), computing the prefix once.
 *
 * Source: "大语言模型推理引擎深度剖析", §2.3 (requests sharing a system prompt /
 * prompt prefix share the same KV cache blocks) and "Transformer 推理优化：KV
 * Cache、PagedAttention 与 vLLM", §3.5; the result is pa_decode's, split by
 * the log-sum-exp decomposition described at pa_decode_split_reduce.
 *
 * Requirements: the first prefix_len / block_size entries of every row of
 * block_tables are the same blocks (row 0 is read for them; the caller's
 * allocator guarantees the sharing), prefix_len is a positive multiple of
 * block_size, every seq_lens[s] >= prefix_len (a shorter one flags
 * PA_ERR_DEVICE_BOUNDS), kv_dtype = q_dtype or an 8-bit format with
 * head_dim 128 (per-tensor k_scale / v_scale as for pa_decode),
 * softmax_scale > 0, GQA groups up to 128.  Three launches on `stream`:
 *   1. the prefix: for each KV head, the queries of all sequences against the
 *      prefix keys as one dense tensor-core pass (the prefix K/V is read once,
 *      not once per sequence).  The prefix's keys are cut into Z contiguous
 *      ranges (Z = min(8, ceil(prefix_len / 256)), fewer if a range would be
 *      empty) that run side by side; each gives every (sequence, head) a
 *      partial (lse, o) in workspace slot z;
 *   2. the tails (positions prefix_len .. L - 1) in partitions of
 *      partition_size tokens (a positive multiple of 16): slots Z ..;
 *   3. the merge of all slots into out.
 * workspace: >= pa_shared_prefix_workspace_bytes(num_seqs, num_q_heads,
 * head_dim, max_seq_len, prefix_len, partition_size) bytes, 256-byte aligned:
 * lse [S, Hq, NP] fp32, then o [S, Hq, NP, d] fp32, NP = Z +
 * ceil((max_seq_len - prefix_len) / partition_size), each section on a
 * 256-byte boundary.  Other arguments and errors as for
 * pa_decode_split_reduce.
 */
size_t pa_shared_prefix_workspace_bytes(int num_seqs, int num_q_heads, int head_dim,
                                        int max_seq_len, int prefix_len, int partition_size);

pa_status pa_decode_shared_prefix(void *out, const void *q, const void *k_cache,
                                  const void *v_cache, const int32_t *block_tables,
                                  int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs,
                                  int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                  int num_blocks, float softmax_scale, pa_dtype q_dtype,
                                  pa_dtype kv_dtype, float k_scale, float v_scale, int prefix_len,
                                  int partition_size, int max_seq_len, void *workspace,
                                  size_t workspace_bytes, int *dev_err, void *stream);

/* Bytes of scratch built into the library for
 * pa_decode_split_reduce_static_scratch (32 MiB). */
#define PA_STATIC_SCRATCH_BYTES (32u * 1024u * 1024u)

/*
 * pa_decode_split_reduce_static_scratch -- pa_decode_split_reduce for callers
 * that cannot allocate device memory.
 *
 * No counterpart in the paper: this is a deployment convenience, not part of
 * the method.  Some callers have no allocator to draw a workspace from: a
 * plugin or custom-op host that passes tensors but no allocator, a serving
 * engine that has already reserved all free HBM for its KV block pool, or a
 * latency-critical loop that must not pay cudaMalloc's implicit device
 * synchronisation.  This entry point takes no workspace: the per-partition
 * partials go to a __device__ array of PA_STATIC_SCRATCH_BYTES bytes inside
 * the library, which a GPU that loads this code may hold until the process
 * exits.  The caller still provides every input and the output; the call
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 *
 * Arguments and result are those of pa_decode_split_reduce without
 * `workspace` / `workspace_bytes`.
 *   - Argument errors are those of pa_decode_split_reduce and are returned
 *     before the GPU is touched; so is PA_ERR_INVALID_ARG when the partials
 *     for these sizes, pa_split_workspace_bytes(num_seqs, num_q_heads,
 *     head_dim, max_seq_len, partition_size), exceed PA_STATIC_SCRATCH_BYTES.
 *   - The first call in a CUDA context looks up the array's device address
 *     on the current device; make that first call before any stream capture.
 *     The address is remembered per device with the context's id, so a call
 *     in another context of the device (e.g. after cudaDeviceReset, which
 *     discards the array and its contents) looks it up again.  PA_ERR_CUDA
 *     if the lookup fails.
 *   - Every call, on every stream, shares the one array per device, and the
 *     array keeps the last call's partials: nothing in it has to start at zero
 *     (each partial is written before it is read), but calls that overlap on
 *     the GPU race with each other.  Serialise them (one stream, or events).
 */
pa_status pa_decode_split_reduce_static_scratch(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs,
    int num_q_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
    float softmax_scale, pa_dtype q_dtype, pa_dtype kv_dtype, float k_scale, float v_scale,
    int partition_size, int max_seq_len, int *dev_err, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PA369_H */
