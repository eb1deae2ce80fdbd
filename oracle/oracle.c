/*
 * CPU oracle for paged-KV-cache decode attention.  fp64, plain loops.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may use this file:
 * only the tests, the smoke check and the benchmark's CPU-baseline leg call it.
 * It shares no code, header, table or helper with the CUDA kernels.
 *
 * What it computes, and where the pages state it:
 *   - slot addressing through a per-sequence block table: "Transformer 推理优化：
 *     KV Cache、PagedAttention 与 vLLM", §3.2-§3.3 (Block Table 机制), and
 *     "KV Cache 与 PageAttention深度实战", §3.2 (block table indirection);
 *   - block growth, one new 16-token block every 16 tokens: "vLLM推理引擎深度
 *     解析：PagedAttention与连续批处理", §2.2 (内存分配器设计);
 *   - the KV-size formula 2 x layers x kv_heads x d x bytes: first page §2.5;
 *   - attention softmax(q K^T / sqrt(d_k)) V with the decode form
 *     Attention(Q_t, [K_prefix, K_t], [V_prefix, V_t]):
 *     "KV Cache 与 PageAttention深度实战", §1.2;
 *   - fp8 E4M3 KV values (max 448): "大语言模型推理引擎深度剖析：从 KV Cache
 *     内存管理到 PagedAttention、投机解码与量化加速的完全工程指南", §4.2-§4.3;
 *   - chunked prefill: a long prompt is cut into chunks (e.g. 512 tokens)
 *     processed one after another, each chunk's queries attending causally
 *     over the cache: openeuler page §4.5 and the second page §3.3;
 *   - per-channel scales for 8-bit caches: the fifth page's §4.3 quantises
 *     each channel of K / V separately (one scale per (KV head, element of
 *     head_dim));
 *   - copy-on-write of a shared block: first page §3.5 (a beam-search
 *     candidate that diverges gets a new block for the diverging part only)
 *     and the fifth page §2.3 (a request about to write into a shared block
 *     copies it first, refcounts track the sharing).
 *
 * Paging changes only where K and V rows live, so the oracle gathers every
 * sequence's rows into contiguous fp64 arrays and then runs textbook two-pass
 * softmax attention on them.  Readings where the pages are silent:
 *   - GQA: query head h reads KV head h / (Hq / Hk);
 *   - pool layout [num_blocks, num_kv_heads, block_size, head_dim], row-major;
 *   - slot = physical_block * block_size + offset; a negative slot is padding;
 *   - seq_len counts the token written in this step; seq_len 0 gives zeros;
 *   - fp8: y = x / scale in fp32 (IEEE), then round to nearest even onto the
 *     E4M3 grid, saturating to +-448; NaN encodes to 0x7F.  E5M2 alike,
 *     saturating to +-57344 (the fifth page's §4.2 range), NaN to 0x7F;
 *   - INT8 (openeuler page §2.3 lists it beside FP8): symmetric, code =
 *     round-half-even(x / scale) clamped to [-127, 127], value = code * scale;
 *   - split-KV: partition p covers tokens [p*P, min((p+1)*P, L)), summarised by
 *     its log-sum-exp and normalised output, merged by log-sum-exp weighting.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F16 0
#define ORC_BF16 1
#define ORC_E4M3 2
#define ORC_E5M2 3
#define ORC_INT8 4

/* the 8-bit cache formats: each stores code(x / scale) and reads code * scale */
static int orc_is_8bit(int dtype) { return dtype == ORC_E4M3 || dtype == ORC_E5M2 || dtype == ORC_INT8; }

/* ------------------------------------------------------------------------- */
/* element formats                                                            */
/* ------------------------------------------------------------------------- */

/* IEEE 754 binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double orc_f16_decode(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

/* bfloat16: 1 sign, 8 exponent (bias 127), 7 fraction bits. */
double orc_bf16_decode(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 7) & 0xFF;
    int m = h & 0x7F;
    double v;
    if (e == 0)
        v = ldexp((double)m, -133);
    else if (e == 255)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + m), e - 134);
    return sign ? -v : v;
}

/* OCP 8-bit floating point, E4M3 ("FN"): 1 sign, 4 exponent (bias 7),
 * 3 fraction bits; no infinities; S.1111.111 is NaN; largest value 448. */
double orc_e4m3_decode(uint8_t c) {
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 0xF;
    int m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp((double)(8 + m), e - 10);
    return sign ? -v : v;
}

/* Round half to even of a non-negative double to an integer value. */
static double orc_rne(double q) {
    double f = floor(q);
    double r = q - f;
    if (r > 0.5) return f + 1.0;
    if (r < 0.5) return f;
    return fmod(f, 2.0) == 0.0 ? f : f + 1.0;
}

/* fp32 -> E4M3, round to nearest even, saturate finite overflow and infinity
 * to +-448, NaN -> 0x7F. */
uint8_t orc_e4m3_encode(float y) {
    if (isnan(y)) return 0x7F;
    uint8_t sign = signbit(y) ? 0x80 : 0x00;
    double a = fabs((double)y);
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: multiples of 2^-9; 8 * 2^-9 is the smallest normal,
         * whose code (exponent 1, fraction 0) is also 8 */
        double n = orc_rne(a * 512.0);
        return sign | (uint8_t)n;
    }
    int e;
    frexp(a, &e); /* a = f * 2^e, f in [0.5, 1) */
    e -= 1;       /* a in [2^e, 2^(e+1)) */
    double n = orc_rne(ldexp(a, 3 - e)); /* in [8, 16] */
    if (n == 16.0) {
        n = 8.0;
        e += 1;
    }
    /* a < 448 rounds to at most 448 (exponent 15, fraction 6) */
    return sign | (uint8_t)(((e + 7) << 3) | ((int)n - 8));
}

/* OCP 8-bit floating point, E5M2: 1 sign, 5 exponent (bias 15), 2 fraction
 * bits; exponent 31 holds infinities (fraction 0) and NaNs; largest finite
 * value 57344. */
double orc_e5m2_decode(uint8_t c) {
    int sign = (c >> 7) & 1;
    int e = (c >> 2) & 0x1F;
    int m = c & 3;
    double v;
    if (e == 31)
        v = m ? NAN : INFINITY;
    else if (e == 0)
        v = ldexp((double)m, -16);
    else
        v = ldexp((double)(4 + m), e - 17);
    return sign ? -v : v;
}

/* fp32 -> E5M2, round to nearest even, saturating finite overflow and
 * infinity to +-57344, NaN -> 0x7F. */
uint8_t orc_e5m2_encode(float y) {
    if (isnan(y)) return 0x7F;
    uint8_t sign = signbit(y) ? 0x80 : 0x00;
    double a = fabs((double)y);
    if (a >= 57344.0) return sign | 0x7B;
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: multiples of 2^-16; 4 * 2^-16 is the smallest
         * normal, whose code (exponent 1, fraction 0) is also 4 */
        double n = orc_rne(a * 65536.0);
        return sign | (uint8_t)n;
    }
    int e;
    frexp(a, &e);
    e -= 1; /* a in [2^e, 2^(e+1)) */
    double n = orc_rne(ldexp(a, 2 - e)); /* in [4, 8] */
    if (n == 8.0) {
        n = 4.0;
        e += 1;
    }
    /* a < 57344 rounds to at most 57344 (exponent 30, fraction 3) */
    return sign | (uint8_t)(((e + 15) << 2) | ((int)n - 4));
}

/* symmetric INT8: the code is the integer itself */
double orc_int8_decode(uint8_t c) { return (double)(int8_t)c; }

/* fp32 -> INT8: round half to even, clamp to [-127, 127]; NaN -> 0. */
uint8_t orc_int8_encode(float y) {
    if (isnan(y)) return 0;
    double n = orc_rne(fabs((double)y));
    if (n > 127.0) n = 127.0;
    int v = signbit(y) ? -(int)n : (int)n;
    return (uint8_t)(int8_t)v;
}

double orc_elem(int dtype, const void *base, int64_t i) {
    if (dtype == ORC_F16) return orc_f16_decode(((const uint16_t *)base)[i]);
    if (dtype == ORC_BF16) return orc_bf16_decode(((const uint16_t *)base)[i]);
    if (dtype == ORC_E5M2) return orc_e5m2_decode(((const uint8_t *)base)[i]);
    if (dtype == ORC_INT8) return orc_int8_decode(((const uint8_t *)base)[i]);
    return orc_e4m3_decode(((const uint8_t *)base)[i]);
}

static uint8_t orc_encode8(int dtype, float y) {
    if (dtype == ORC_E5M2) return orc_e5m2_encode(y);
    if (dtype == ORC_INT8) return orc_int8_encode(y);
    return orc_e4m3_encode(y);
}

/* ------------------------------------------------------------------------- */
/* block table arithmetic                                                     */
/* ------------------------------------------------------------------------- */

/* Blocks a sequence of `len` tokens occupies: only the last one may be partly
 * filled (first page §3.2 / §3.4). */
int64_t orc_blocks_for_len(int64_t len, int block_size) {
    return (len + block_size - 1) / block_size;
}

/* Per-token KV bytes: 2 (K and V) x layers x kv_heads x head_dim x bytes
 * (first page §2.5). */
int64_t orc_kv_bytes_per_token(int layers, int kv_heads, int head_dim, int bytes_per_elem) {
    return (int64_t)2 * layers * kv_heads * head_dim * bytes_per_elem;
}

/* Slot of logical position `pos`: the block table maps logical block
 * pos / B to a physical block; the token sits at offset pos % B in it
 * (first page §3.3). */
int64_t orc_slot(const int32_t *block_table_row, int64_t pos, int block_size) {
    int64_t phys = block_table_row[pos / block_size];
    return phys * block_size + pos % block_size;
}

/* Slots for a list of (sequence, position) tokens.  token_seq NULL means
 * token t belongs to sequence t; token_pos NULL means the last position,
 * seq_lens[s] - 1.  A negative sequence index gives slot -1 (padding). */
void orc_slot_mapping(int64_t *slots, const int32_t *block_tables, int max_blocks_per_seq,
                      const int32_t *seq_lens, const int32_t *token_seq, const int32_t *token_pos,
                      int num_tokens, int block_size) {
    for (int t = 0; t < num_tokens; ++t) {
        int s = token_seq ? token_seq[t] : t;
        if (s < 0) {
            slots[t] = -1;
            continue;
        }
        int64_t pos = token_pos ? token_pos[t] : (int64_t)seq_lens[s] - 1;
        slots[t] = orc_slot(block_tables + (int64_t)s * max_blocks_per_seq, pos, block_size);
    }
}

/* ------------------------------------------------------------------------- */
/* cache write                                                                */
/* ------------------------------------------------------------------------- */

/* Store each token's per-head K/V rows at its slot in the pools
 * [num_blocks, Hk, B, d].  16-bit caches hold the activation bits unchanged;
 * an E4M3 cache holds encode((float)x / scale).  Returns -1 on an
 * unsupported dtype pair, else the number of out-of-range slots (skipped). */
int orc_cache_write(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                    const int64_t *slots, int num_tokens, int num_blocks, int num_kv_heads,
                    int head_dim, int block_size, int act_dtype, int kv_dtype, float k_scale,
                    float v_scale) {
    if (orc_is_8bit(act_dtype)) return -1;
    if (!orc_is_8bit(kv_dtype) && kv_dtype != act_dtype) return -1;
    int bad = 0;
    for (int t = 0; t < num_tokens; ++t) {
        int64_t slot = slots[t];
        if (slot < 0) continue;
        if (slot >= (int64_t)num_blocks * block_size) {
            ++bad;
            continue;
        }
        int64_t blk = slot / block_size, off = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim;
            int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim;
            for (int i = 0; i < head_dim; ++i) {
                if (orc_is_8bit(kv_dtype)) {
                    float xk = (float)orc_elem(act_dtype, k_new, src + i);
                    float xv = (float)orc_elem(act_dtype, v_new, src + i);
                    float yk = xk / k_scale;
                    float yv = xv / v_scale;
                    ((uint8_t *)k_cache)[dst + i] = orc_encode8(kv_dtype, yk);
                    ((uint8_t *)v_cache)[dst + i] = orc_encode8(kv_dtype, yv);
                } else {
                    ((uint16_t *)k_cache)[dst + i] = ((const uint16_t *)k_new)[src + i];
                    ((uint16_t *)v_cache)[dst + i] = ((const uint16_t *)v_new)[src + i];
                }
            }
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------- */
/* gather + attention                                                         */
/* ------------------------------------------------------------------------- */

/* Contiguous fp64 rows [len][d] of KV head `kvh` of one sequence, read through
 * its block table; 8-bit values are decode(code) * scale, with the scale of
 * channel i taken from chan_scales[i] when that row of per-channel scales
 * is given (else the per-tensor `scale`). */
static void orc_gather_scaled(double *rows, const void *cache, int kv_dtype, double scale,
                              const float *chan_scales, const int32_t *block_table_row, int len,
                              int num_kv_heads, int kvh, int head_dim, int block_size) {
    for (int t = 0; t < len; ++t) {
        int64_t phys = block_table_row[t / block_size];
        int64_t off = t % block_size;
        int64_t base = ((phys * num_kv_heads + kvh) * block_size + off) * head_dim;
        for (int i = 0; i < head_dim; ++i) {
            double v = orc_elem(kv_dtype, cache, base + i);
            double sc = chan_scales ? (double)chan_scales[i] : scale;
            rows[(int64_t)t * head_dim + i] = orc_is_8bit(kv_dtype) ? v * sc : v;
        }
    }
}

void orc_gather(double *rows, const void *cache, int kv_dtype, double scale,
                const int32_t *block_table_row, int len, int num_kv_heads, int kvh, int head_dim,
                int block_size) {
    orc_gather_scaled(rows, cache, kv_dtype, scale, NULL, block_table_row, len, num_kv_heads, kvh,
                      head_dim, block_size);
}

/* Textbook attention of one query row over contiguous K, V [len][d]:
 *   s_t = scale * q.k_t;  p = exp(s - max s) / sum exp(s - max s);  o = sum p_t v_t.
 * Also returns lse = max s + log(sum exp(s - max s)).  len 0 gives o = 0 and
 * lse = -inf. */
void orc_attention(double *out, double *lse, const double *q, const double *K, const double *V,
                   int len, int head_dim, double softmax_scale) {
    for (int i = 0; i < head_dim; ++i) out[i] = 0.0;
    if (len <= 0) {
        if (lse) *lse = -INFINITY;
        return;
    }
    double *s = (double *)malloc(sizeof(double) * (size_t)len);
    double mx = -INFINITY;
    for (int t = 0; t < len; ++t) {
        double dot = 0.0;
        for (int i = 0; i < head_dim; ++i) dot += q[i] * K[(int64_t)t * head_dim + i];
        s[t] = softmax_scale * dot;
        if (s[t] > mx) mx = s[t];
    }
    double z = 0.0;
    for (int t = 0; t < len; ++t) {
        s[t] = exp(s[t] - mx);
        z += s[t];
    }
    for (int t = 0; t < len; ++t) {
        double p = s[t] / z;
        for (int i = 0; i < head_dim; ++i) out[i] += p * V[(int64_t)t * head_dim + i];
    }
    if (lse) *lse = mx + log(z);
    free(s);
}

/* Decode attention for a list of (sequence, q head) pairs, or all of them
 * when pairs == NULL (then out is [S][Hq][d]; else out is [npairs][d]).
 * Split-KV partials for the same pairs come from orc_split_partials. */
int orc_decode(double *out, const void *q, int q_dtype, const void *k_cache, const void *v_cache,
               int kv_dtype, double k_scale, double v_scale, const int32_t *block_tables,
               int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs, int num_q_heads,
               int num_kv_heads, int head_dim, int block_size, double softmax_scale,
               const int32_t *pairs, int npairs) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads) return -1;
    int g = num_q_heads / num_kv_heads;
    int n = pairs ? npairs : num_seqs * num_q_heads;
    double *qrow = (double *)malloc(sizeof(double) * (size_t)head_dim);
    for (int w = 0; w < n; ++w) {
        int s = pairs ? pairs[2 * w] : w / num_q_heads;
        int h = pairs ? pairs[2 * w + 1] : w % num_q_heads;
        int len = seq_lens[s];
        int kvh = h / g;
        const int32_t *bt = block_tables + (int64_t)s * max_blocks_per_seq;
        double *K = (double *)malloc(sizeof(double) * ((size_t)len * head_dim + 1));
        double *V = (double *)malloc(sizeof(double) * ((size_t)len * head_dim + 1));
        orc_gather(K, k_cache, kv_dtype, k_scale, bt, len, num_kv_heads, kvh, head_dim, block_size);
        orc_gather(V, v_cache, kv_dtype, v_scale, bt, len, num_kv_heads, kvh, head_dim, block_size);
        int64_t qb = ((int64_t)s * num_q_heads + h) * head_dim;
        for (int i = 0; i < head_dim; ++i) qrow[i] = orc_elem(q_dtype, q, qb + i);
        orc_attention(out + (int64_t)w * head_dim, NULL, qrow, K, V, len, head_dim, softmax_scale);
        free(K);
        free(V);
    }
    free(qrow);
    return 0;
}

/* Split-KV partials: for every listed (s, h) and partition p < num_partitions,
 * attention restricted to tokens [p*P, min((p+1)*P, L)):
 *   lse[w][p]    = log-sum-exp of the partition's scaled logits (-inf if empty)
 *   o[w][p][d]   = the partition's normalised output (0 if empty). */
int orc_split_partials(double *lse, double *o, const void *q, int q_dtype, const void *k_cache,
                       const void *v_cache, int kv_dtype, double k_scale, double v_scale,
                       const int32_t *block_tables, int max_blocks_per_seq,
                       const int32_t *seq_lens, int num_q_heads, int num_kv_heads, int head_dim,
                       int block_size, double softmax_scale, int partition_size,
                       int num_partitions, const int32_t *pairs, int npairs) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads || partition_size <= 0) return -1;
    int g = num_q_heads / num_kv_heads;
    double *qrow = (double *)malloc(sizeof(double) * (size_t)head_dim);
    for (int w = 0; w < npairs; ++w) {
        int s = pairs[2 * w], h = pairs[2 * w + 1];
        int len = seq_lens[s];
        int kvh = h / g;
        const int32_t *bt = block_tables + (int64_t)s * max_blocks_per_seq;
        double *K = (double *)malloc(sizeof(double) * ((size_t)len * head_dim + 1));
        double *V = (double *)malloc(sizeof(double) * ((size_t)len * head_dim + 1));
        orc_gather(K, k_cache, kv_dtype, k_scale, bt, len, num_kv_heads, kvh, head_dim, block_size);
        orc_gather(V, v_cache, kv_dtype, v_scale, bt, len, num_kv_heads, kvh, head_dim, block_size);
        int64_t qb = ((int64_t)s * num_q_heads + h) * head_dim;
        for (int i = 0; i < head_dim; ++i) qrow[i] = orc_elem(q_dtype, q, qb + i);
        for (int p = 0; p < num_partitions; ++p) {
            int64_t lo = (int64_t)p * partition_size;
            int64_t hi = lo + partition_size < len ? lo + partition_size : len;
            int n = hi > lo ? (int)(hi - lo) : 0;
            double *op = o + ((int64_t)w * num_partitions + p) * head_dim;
            orc_attention(op, lse + (int64_t)w * num_partitions + p, qrow,
                          K + lo * head_dim * (n > 0), V + lo * head_dim * (n > 0), n, head_dim,
                          softmax_scale);
        }
        free(K);
        free(V);
    }
    free(qrow);
    return 0;
}

/* Log-sum-exp merge of partition partials into one output row:
 *   M = max_p lse_p;  w_p = exp(lse_p - M);  out = sum_p w_p o_p / sum_p w_p.
 * All partitions empty gives 0. */
void orc_split_merge(double *out, const double *lse, const double *o, int num_partitions,
                     int head_dim) {
    double M = -INFINITY;
    for (int p = 0; p < num_partitions; ++p)
        if (lse[p] > M) M = lse[p];
    for (int i = 0; i < head_dim; ++i) out[i] = 0.0;
    if (M == -INFINITY) return;
    double den = 0.0;
    for (int p = 0; p < num_partitions; ++p) {
        if (lse[p] == -INFINITY) continue;
        double w = exp(lse[p] - M);
        den += w;
        for (int i = 0; i < head_dim; ++i) out[i] += w * o[(int64_t)p * head_dim + i];
    }
    for (int i = 0; i < head_dim; ++i) out[i] /= den;
}

/* ------------------------------------------------------------------------- */
/* copy-on-write block copy                                                   */
/* ------------------------------------------------------------------------- */

/* Copy whole physical blocks inside both pools [num_blocks, Hk, B, d]: for
 * each pair i, in order, block pairs[2i+1] of k_cache and of v_cache becomes
 * a byte copy of block pairs[2i].  This is the copy step of copy-on-write
 * (first page §3.5; fifth page §2.3): before a sequence writes into a block
 * it shares with others, the block is duplicated into a free one and the
 * sequence's table is pointed at the duplicate.  A pair with an id outside
 * [0, num_blocks) is skipped and counted; the count is returned. */
int orc_copy_blocks(void *k_cache, void *v_cache, const int32_t *pairs, int num_pairs,
                    int num_blocks, int num_kv_heads, int head_dim, int block_size,
                    int elem_bytes) {
    int64_t block_bytes = (int64_t)num_kv_heads * block_size * head_dim * elem_bytes;
    int bad = 0;
    for (int i = 0; i < num_pairs; ++i) {
        int32_t src = pairs[2 * i], dst = pairs[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            ++bad;
            continue;
        }
        for (int pool = 0; pool < 2; ++pool) {
            uint8_t *base = (uint8_t *)(pool == 0 ? k_cache : v_cache);
            for (int64_t b = 0; b < block_bytes; ++b)
                base[(int64_t)dst * block_bytes + b] = base[(int64_t)src * block_bytes + b];
        }
    }
    return bad;
}

/* ------------------------------------------------------------------------- */
/* chunked prefill: several query tokens per sequence, causal mask            */
/* ------------------------------------------------------------------------- */

/* Attention of one chunk of query tokens per sequence over the paged cache,
 * causally masked (openeuler page §4.5; second page §3.3).  Sequence s holds
 * L = seq_lens[s] tokens in the cache; the last n = query_start[s+1] -
 * query_start[s] of them are this chunk.  Its query token j, row
 * query_start[s] + j of q and out ([T][Hq][d]), sits at position
 * L - n + j and attends to the keys at positions 0 .. L - n + j.  A decode
 * step is the case n = 1.  Rows of out that no sequence covers are left as
 * they are.  Returns -1 on a bad head configuration or a chunk longer than
 * its sequence. */
int orc_prefill(double *out, const void *q, int q_dtype, const void *k_cache, const void *v_cache,
                int kv_dtype, double k_scale, double v_scale, const int32_t *block_tables,
                int max_blocks_per_seq, const int32_t *seq_lens, const int32_t *query_start,
                int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                double softmax_scale) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads) return -1;
    int g = num_q_heads / num_kv_heads;
    double *qrow = (double *)malloc(sizeof(double) * (size_t)head_dim);
    for (int s = 0; s < num_seqs; ++s) {
        int len = seq_lens[s];
        int n = query_start[s + 1] - query_start[s];
        if (n < 0 || n > len) {
            free(qrow);
            return -1;
        }
        if (n == 0) continue;
        const int32_t *bt = block_tables + (int64_t)s * max_blocks_per_seq;
        double *K = (double *)malloc(sizeof(double) * ((size_t)len * head_dim + 1));
        double *V = (double *)malloc(sizeof(double) * ((size_t)len * head_dim + 1));
        for (int kvh = 0; kvh < num_kv_heads; ++kvh) {
            orc_gather(K, k_cache, kv_dtype, k_scale, bt, len, num_kv_heads, kvh, head_dim, block_size);
            orc_gather(V, v_cache, kv_dtype, v_scale, bt, len, num_kv_heads, kvh, head_dim, block_size);
            for (int j = 0; j < n; ++j) {
                int pos = len - n + j;
                int64_t row_tok = (int64_t)query_start[s] + j;
                for (int hh = 0; hh < g; ++hh) {
                    int h = kvh * g + hh;
                    int64_t row = row_tok * num_q_heads + h;
                    for (int i = 0; i < head_dim; ++i) qrow[i] = orc_elem(q_dtype, q, row * head_dim + i);
                    orc_attention(out + row * head_dim, NULL, qrow, K, V, pos + 1, head_dim,
                                  softmax_scale);
                }
            }
        }
        free(K);
        free(V);
    }
    free(qrow);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* per-channel scales for 8-bit caches                                        */
/* ------------------------------------------------------------------------- */

/* Cache write with one scale per (KV head, channel) (the fifth page's §4.3:
 * each channel of K / V quantised separately): channel i of head h stores
 * code(x / k_scales[h * head_dim + i]), x / s in fp32 with IEEE division.
 * kv_dtype must be an 8-bit format.  Returns -1 on an unsupported dtype
 * pair, else the number of out-of-range slots (skipped). */
int orc_cache_write_channel(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                            const int64_t *slots, int num_tokens, int num_blocks, int num_kv_heads,
                            int head_dim, int block_size, int act_dtype, int kv_dtype,
                            const float *k_scales, const float *v_scales) {
    if (orc_is_8bit(act_dtype) || !orc_is_8bit(kv_dtype)) return -1;
    int bad = 0;
    for (int t = 0; t < num_tokens; ++t) {
        int64_t slot = slots[t];
        if (slot < 0) continue;
        if (slot >= (int64_t)num_blocks * block_size) {
            ++bad;
            continue;
        }
        int64_t blk = slot / block_size, off = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim;
            int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim;
            for (int i = 0; i < head_dim; ++i) {
                float xk = (float)orc_elem(act_dtype, k_new, src + i);
                float xv = (float)orc_elem(act_dtype, v_new, src + i);
                float yk = xk / k_scales[(int64_t)h * head_dim + i];
                float yv = xv / v_scales[(int64_t)h * head_dim + i];
                ((uint8_t *)k_cache)[dst + i] = orc_encode8(kv_dtype, yk);
                ((uint8_t *)v_cache)[dst + i] = orc_encode8(kv_dtype, yv);
            }
        }
    }
    return bad;
}

/* Decode attention (as orc_decode) over an 8-bit cache with per-channel
 * scales k_scales / v_scales [num_kv_heads][head_dim]: K_t[i] =
 * code * k_scales[kvh][i], V_t[i] = code * v_scales[kvh][i]. */
int orc_decode_channel(double *out, const void *q, int q_dtype, const void *k_cache,
                       const void *v_cache, int kv_dtype, const float *k_scales,
                       const float *v_scales, const int32_t *block_tables, int max_blocks_per_seq,
                       const int32_t *seq_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                       int head_dim, int block_size, double softmax_scale, const int32_t *pairs,
                       int npairs) {
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads || !orc_is_8bit(kv_dtype)) return -1;
    int g = num_q_heads / num_kv_heads;
    int n = pairs ? npairs : num_seqs * num_q_heads;
    double *qrow = (double *)malloc(sizeof(double) * (size_t)head_dim);
    for (int w = 0; w < n; ++w) {
        int s = pairs ? pairs[2 * w] : w / num_q_heads;
        int h = pairs ? pairs[2 * w + 1] : w % num_q_heads;
        int len = seq_lens[s];
        int kvh = h / g;
        const int32_t *bt = block_tables + (int64_t)s * max_blocks_per_seq;
        double *K = (double *)malloc(sizeof(double) * ((size_t)len * head_dim + 1));
        double *V = (double *)malloc(sizeof(double) * ((size_t)len * head_dim + 1));
        orc_gather_scaled(K, k_cache, kv_dtype, 1.0, k_scales + (int64_t)kvh * head_dim, bt, len,
                          num_kv_heads, kvh, head_dim, block_size);
        orc_gather_scaled(V, v_cache, kv_dtype, 1.0, v_scales + (int64_t)kvh * head_dim, bt, len,
                          num_kv_heads, kvh, head_dim, block_size);
        int64_t qb = ((int64_t)s * num_q_heads + h) * head_dim;
        for (int i = 0; i < head_dim; ++i) qrow[i] = orc_elem(q_dtype, q, qb + i);
        orc_attention(out + (int64_t)w * head_dim, NULL, qrow, K, V, len, head_dim, softmax_scale);
        free(K);
        free(V);
    }
    free(qrow);
    return 0;
}
