// C ABI of libpa369.so (declared in include/pa.h): host-side argument checks,
// launch configuration and dispatch to the kernel launchers.  No entry point
// allocates memory, synchronises, or touches the GPU before its checks pass.
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "../../include/pa.h"
#include "pa_internal.h"
#include "pa_shared_prefix.h"

namespace {

constexpr int kVersion = 10000;  // 1.0.0

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_act(pa_dtype t) { return t == PA_F16 || t == PA_BF16; }

// the 8-bit cache formats: codes of x / scale, values code * scale
bool is_8bit(pa_dtype t) { return t == PA_FP8_E4M3 || t == PA_FP8_E5M2 || t == PA_INT8; }

pa::DType to_internal(pa_dtype t) { return static_cast<pa::DType>(static_cast<int>(t)); }

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }
// ceil(a / b) for a >= 0, b > 0, without int overflow
int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }
// largest partition and max_seq_len the split entry points take: then every
// token count the kernels form (partitions x partition size) stays in int
constexpr int kMaxPartitionSize = 1 << 30;
constexpr int kMaxSeqLen = 1 << 30;

// Template group size (1, 2, 4 or 8) used for a GQA group of g query heads;
// groups larger than 8 run as ceil(g / 8) CTAs per KV head.
int template_group(int g) {
    if (g >= 8) return 8;
    int t = 1;
    while (t < g) t <<= 1;
    return t;
}

pa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? PA_OK : PA_ERR_CUDA; }

// Decode kernel choice: the tensor-core kernel wherever it supports the shape;
// the CUDA-core kernel otherwise, or everywhere when the environment variable
// PA369_DECODE_KERNEL is "simt" (kept for A/B measurement and tests).
bool use_mma(pa_dtype kv, int head_dim, int num_blocks, int num_kv_heads, int block_size) {
    const char *env = getenv("PA369_DECODE_KERNEL");
    if (env && strcmp(env, "simt") == 0) return false;
    return pa::mma_decode_supported(static_cast<pa::DType>(static_cast<int>(kv)), head_dim,
                                    num_blocks, num_kv_heads, block_size);
}

// Launch whichever decode kernel applies, with its own head grouping.  With
// p.append set, the tensor-core kernel stores the new tokens itself; the
// CUDA-core route runs the fused append kernel first.
cudaError_t launch_any_decode(pa::DecodeParams &p, pa_dtype q, pa_dtype kv, int head_dim,
                              cudaStream_t stream) {
    const int g = p.group;
    const bool mma = use_mma(kv, head_dim, p.num_blocks, p.num_kv_heads, p.block_size);
    if (p.append && !mma) {
        pa::AppendParams a = {};
        a.k_new = p.k_new;
        a.v_new = p.v_new;
        a.k_cache = p.k_pool_w;
        a.v_cache = p.v_pool_w;
        a.block_tables = p.block_tables;
        a.seq_lens = p.seq_lens;
        a.err = p.err;
        a.max_blocks_per_seq = p.max_blocks_per_seq;
        a.num_seqs = p.num_seqs;
        a.num_kv_heads = p.num_kv_heads;
        a.head_dim = head_dim;
        a.num_blocks = p.num_blocks;
        a.block_size = p.block_size;
        a.k_scale = p.k_scale_w;
        a.v_scale = p.v_scale_w;
        const cudaError_t e = pa::launch_append(a, to_internal(q), to_internal(kv), stream);
        if (e != cudaSuccess) return e;
        p.append = 0;
    }
    if (mma) {
        const int rows = g <= 8 ? 8 : 16;
        p.head_groups = (g + rows - 1) / rows;
        return pa::launch_decode_mma(p, to_internal(q), to_internal(kv), head_dim, rows, stream);
    }
    const int tg = template_group(g);
    p.head_groups = (g + tg - 1) / tg;
    return pa::launch_decode(p, to_internal(q), to_internal(kv), head_dim, tg, stream);
}

struct DecodeArgs {
    void *out;
    const void *q;
    const void *k_cache;
    const void *v_cache;
    const int32_t *block_tables;
    int max_blocks_per_seq;
    const int32_t *seq_lens;
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int head_dim;
    int block_size;
    int num_blocks;
    float softmax_scale;
    pa_dtype q_dtype;
    pa_dtype kv_dtype;
    float k_scale;
    float v_scale;
};

pa_status check_decode(const DecodeArgs &a) {
    if (a.num_seqs < 0 || a.num_q_heads <= 0 || a.num_kv_heads <= 0 || a.head_dim <= 0 ||
        a.block_size <= 0)
        return PA_ERR_INVALID_ARG;
    if (a.num_q_heads % a.num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if (!is_act(a.q_dtype)) return PA_ERR_UNSUPPORTED;
    if (a.kv_dtype != a.q_dtype && !is_8bit(a.kv_dtype)) return PA_ERR_UNSUPPORTED;
    if (a.head_dim != 64 && a.head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (a.block_size != 16 && a.block_size != 32) return PA_ERR_UNSUPPORTED;
    if (!isfinite(a.softmax_scale)) return PA_ERR_INVALID_ARG;
    if (is_8bit(a.kv_dtype) &&
        !(isfinite(a.k_scale) && a.k_scale > 0.f && isfinite(a.v_scale) && a.v_scale > 0.f))
        return PA_ERR_INVALID_ARG;
    if (a.num_seqs == 0) return PA_OK;
    if (!a.out || !a.q || !a.k_cache || !a.v_cache || !a.block_tables || !a.seq_lens)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(a.out) || !aligned16(a.q) || !aligned16(a.k_cache) || !aligned16(a.v_cache))
        return PA_ERR_INVALID_ARG;
    if (a.max_blocks_per_seq <= 0 || a.num_blocks <= 0) return PA_ERR_INVALID_ARG;
    if ((int64_t)a.max_blocks_per_seq * a.block_size >= (int64_t(1) << 30)) return PA_ERR_UNSUPPORTED;
    const int g = a.num_q_heads / a.num_kv_heads;
    const int tg = template_group(g);
    const int64_t ycta = (int64_t)a.num_kv_heads * ((g + tg - 1) / tg);
    if (ycta > 65535) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

pa::DecodeParams make_decode_params(const DecodeArgs &a, int *dev_err) {
    pa::DecodeParams p = {};
    const bool fp8 = is_8bit(a.kv_dtype);
    const int g = a.num_q_heads / a.num_kv_heads;
    const int tg = template_group(g);
    p.out = a.out;
    p.q = a.q;
    p.k_cache = static_cast<const uint8_t *>(a.k_cache);
    p.v_cache = static_cast<const uint8_t *>(a.v_cache);
    p.block_tables = a.block_tables;
    p.seq_lens = a.seq_lens;
    p.err = dev_err;
    p.max_blocks_per_seq = a.max_blocks_per_seq;
    p.num_seqs = a.num_seqs;
    p.num_q_heads = a.num_q_heads;
    p.num_kv_heads = a.num_kv_heads;
    p.num_blocks = a.num_blocks;
    p.block_size = a.block_size;
    p.tile_shift = a.block_size == 32 ? 1 : 0;
    p.group = g;
    p.head_groups = (g + tg - 1) / tg;
    const double log2e = 1.4426950408889634074;
    p.qk_scale_log2 = (float)((double)a.softmax_scale * (fp8 ? (double)a.k_scale : 1.0) * log2e);
    p.v_scale = fp8 ? a.v_scale : 1.0f;
    // failure-detection test hook: PA369_TEST_DECODE_STALL_NS=<ns> makes every
    // decode warp's first copy wait run out after <ns> nanoseconds (see
    // DecodeParams); unset in normal use
    if (const char *env = getenv("PA369_TEST_DECODE_STALL_NS")) {
        const long long ns = atoll(env);
        if (ns > 0) {
            p.wait_limit_ns = (uint64_t)ns;
            p.hold_first_tile = 1;
        }
    }
    return p;
}

}  // namespace

extern "C" {

const char *pa_status_string(pa_status status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG: invalid argument";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: configuration not supported";
        case PA_ERR_CUDA: return "PA_ERR_CUDA: a CUDA launch or query failed";
        case PA_ERR_DEVICE_BOUNDS: return "PA_ERR_DEVICE_BOUNDS: index or length out of range on the device";
        case PA_ERR_DEVICE_TIMEOUT: return "PA_ERR_DEVICE_TIMEOUT: a device wait timed out";
    }
    return "unknown pa_status";
}

int pa_version(void) { return kVersion; }

pa_status pa_slot_mapping(int64_t *slot_mapping, const int32_t *block_tables,
                          int max_blocks_per_seq, const int32_t *seq_lens,
                          const int32_t *token_seq, const int32_t *token_pos, int num_tokens,
                          int num_seqs, int block_size, int num_blocks, int *dev_err,
                          void *stream) {
    if (num_tokens < 0 || num_seqs < 0 || block_size <= 0 || num_blocks < 0)
        return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    if (!slot_mapping || !block_tables || max_blocks_per_seq <= 0) return PA_ERR_INVALID_ARG;
    if (!token_pos && !seq_lens) return PA_ERR_INVALID_ARG;
    if (!token_seq && num_tokens > num_seqs) return PA_ERR_INVALID_ARG;  // token t is sequence t
    pa::SlotParams p = {};
    p.slot_mapping = slot_mapping;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.token_seq = token_seq;
    p.token_pos = token_pos;
    p.err = dev_err;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_tokens = num_tokens;
    p.num_seqs = num_seqs;
    p.block_size = block_size;
    p.num_blocks = num_blocks;
    return from_cuda(pa::launch_slot_mapping(p, static_cast<cudaStream_t>(stream)));
}

pa_status pa_cache_write(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                         const int64_t *slot_mapping, int num_tokens, int num_blocks,
                         int num_kv_heads, int head_dim, int block_size, pa_dtype act_dtype,
                         pa_dtype kv_dtype, float k_scale, float v_scale, int *dev_err,
                         void *stream) {
    if (num_tokens < 0 || num_blocks < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
        return PA_ERR_INVALID_ARG;
    if (!is_act(act_dtype)) return PA_ERR_UNSUPPORTED;
    if (kv_dtype != act_dtype && !is_8bit(kv_dtype)) return PA_ERR_UNSUPPORTED;
    if (head_dim % 8 != 0) return PA_ERR_UNSUPPORTED;
    if (is_8bit(kv_dtype) &&
        !(isfinite(k_scale) && k_scale > 0.f && isfinite(v_scale) && v_scale > 0.f))
        return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
        return PA_ERR_INVALID_ARG;
    pa::CacheWriteParams p = {};
    p.k_new = k_new;
    p.v_new = v_new;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.slot_mapping = slot_mapping;
    p.err = dev_err;
    p.num_tokens = num_tokens;
    p.num_blocks = num_blocks;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.block_size = block_size;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    return from_cuda(pa::launch_cache_write(p, to_internal(act_dtype), to_internal(kv_dtype),
                                            static_cast<cudaStream_t>(stream)));
}

pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_tables, int max_blocks_per_seq, const int32_t *seq_lens,
                    int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                    int block_size, int num_blocks, float softmax_scale, pa_dtype q_dtype,
                    pa_dtype kv_dtype, float k_scale, float v_scale, int *dev_err,
                    void *stream) {
    const DecodeArgs a = {out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                          num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                          softmax_scale, q_dtype, kv_dtype, k_scale, v_scale};
    const pa_status st = check_decode(a);
    if (st != PA_OK || num_seqs == 0) return st;
    pa::DecodeParams p = make_decode_params(a, dev_err);
    p.partition_blocks = max_blocks_per_seq << p.tile_shift;  // every 16-token tile
    p.num_partitions = 1;
    p.split = 0;
    return from_cuda(launch_any_decode(p, q_dtype, kv_dtype, head_dim, static_cast<cudaStream_t>(stream)));
}

pa_status pa_decode_append(void *out, const void *q, const void *k_new, const void *v_new,
                           void *k_cache, void *v_cache, const int32_t *block_tables,
                           int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs,
                           int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                           int num_blocks, float softmax_scale, pa_dtype q_dtype,
                           pa_dtype kv_dtype, float k_scale, float v_scale, int partition_size,
                           int max_seq_len, void *workspace, size_t workspace_bytes, int *dev_err,
                           void *stream) {
    const DecodeArgs a = {out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                          num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                          softmax_scale, q_dtype, kv_dtype, k_scale, v_scale};
    pa_status st = check_decode(a);
    if (st != PA_OK) return st;
    if (partition_size < 0 || partition_size > kMaxPartitionSize || partition_size % pa::kBlockSize != 0 ||
        max_seq_len < 0 || max_seq_len > kMaxSeqLen)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return PA_ERR_INVALID_ARG;
    const bool split = partition_size > 0;
    int np = 1;
    if (split) {
        const size_t need = pa_split_workspace_bytes(num_seqs, num_q_heads, head_dim, max_seq_len,
                                                     partition_size);
        if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
            return PA_ERR_INVALID_ARG;
        np = max_seq_len > 0 ? (int)ceil_div64(max_seq_len, partition_size) : 1;
        if ((int64_t)num_seqs * np > 0x7FFFFFFF) return PA_ERR_UNSUPPORTED;
    }
    pa::DecodeParams p = make_decode_params(a, dev_err);
    p.append = 1;
    p.k_new = k_new;
    p.v_new = v_new;
    p.k_pool_w = static_cast<uint8_t *>(k_cache);
    p.v_pool_w = static_cast<uint8_t *>(v_cache);
    p.k_scale_w = is_8bit(kv_dtype) ? k_scale : 1.0f;
    p.v_scale_w = is_8bit(kv_dtype) ? v_scale : 1.0f;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!split) {
        p.partition_blocks = max_blocks_per_seq << p.tile_shift;  // every 16-token tile
        p.num_partitions = 1;
        p.split = 0;
        return from_cuda(launch_any_decode(p, q_dtype, kv_dtype, head_dim, s));
    }
    const size_t rows = (size_t)num_seqs * num_q_heads * np;
    p.ws_lse = static_cast<float *>(workspace);
    p.ws_o = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + align256(rows * sizeof(float)));
    p.partition_blocks = partition_size / pa::kBlockSize;
    p.num_partitions = np;
    p.split = 1;
    if (launch_any_decode(p, q_dtype, kv_dtype, head_dim, s) != cudaSuccess) return PA_ERR_CUDA;
    pa::ReduceParams r = {};
    r.out = out;
    r.ws_lse = p.ws_lse;
    r.ws_o = p.ws_o;
    r.seq_lens = seq_lens;
    r.num_seqs = num_seqs;
    r.num_q_heads = num_q_heads;
    r.num_partitions = np;
    r.partition_size = partition_size;
    return from_cuda(pa::launch_reduce(r, to_internal(q_dtype), head_dim, s));
}

pa_status pa_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                     const int32_t *block_tables, int max_blocks_per_seq, const int32_t *seq_lens,
                     const int32_t *query_start, int num_seqs, int num_tokens, int max_query_len,
                     int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                     int num_blocks, float softmax_scale, pa_dtype q_dtype, pa_dtype kv_dtype,
                     float k_scale, float v_scale, int *dev_err, void *stream) {
    if (num_seqs < 0 || num_tokens < 0 || max_query_len < 0 || num_q_heads <= 0 ||
        num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
        return PA_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if (!is_act(q_dtype)) return PA_ERR_UNSUPPORTED;
    if (kv_dtype != q_dtype && !is_8bit(kv_dtype)) return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (is_8bit(kv_dtype) && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (is_8bit(kv_dtype) &&
        !(isfinite(k_scale) && k_scale > 0.f && isfinite(v_scale) && v_scale > 0.f))
        return PA_ERR_INVALID_ARG;
    if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
    const int g = num_q_heads / num_kv_heads;
    if (g > 128) return PA_ERR_UNSUPPORTED;
    if (!isfinite(softmax_scale) || !(softmax_scale > 0.f)) return PA_ERR_INVALID_ARG;
    if (num_seqs == 0 || num_tokens == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || !query_start)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
        return PA_ERR_INVALID_ARG;
    if (max_blocks_per_seq <= 0 || num_blocks <= 0 || max_query_len <= 0) return PA_ERR_INVALID_ARG;
    if (num_seqs > 65535 || num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;
    const int64_t rows = (int64_t)num_blocks * num_kv_heads * block_size;
    if (rows + block_size >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
    if (!pa::prefill_supported()) return PA_ERR_CUDA;
    pa::PrefillParams p = {};
    p.out = out;
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.query_start = query_start;
    p.err = dev_err;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_seqs = num_seqs;
    p.num_tokens = num_tokens;
    p.max_query_len = max_query_len;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.num_blocks = num_blocks;
    p.block_size = block_size;
    p.tile_shift = block_size == 32 ? 1 : 0;
    p.group = g;
    p.tok_per_tile = 128 / g;
    p.oob_row = (int)rows;
    const bool kv8 = is_8bit(kv_dtype);
    p.qk_scale_log2 =
        (float)((double)softmax_scale * (kv8 ? (double)k_scale : 1.0) * 1.4426950408889634074);
    p.v_scale = kv8 ? v_scale : 1.0f;
    return from_cuda(pa::launch_prefill(p, to_internal(q_dtype), to_internal(kv_dtype), head_dim,
                                        static_cast<cudaStream_t>(stream)));
}

pa_status pa_copy_blocks(void *k_cache, void *v_cache, const int32_t *block_pairs, int num_pairs,
                         int num_blocks, int num_kv_heads, int head_dim, int block_size,
                         pa_dtype kv_dtype, int *dev_err, void *stream) {
    if (num_pairs < 0 || num_blocks <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
        return PA_ERR_INVALID_ARG;
    if (!is_act(kv_dtype) && !is_8bit(kv_dtype)) return PA_ERR_UNSUPPORTED;
    const int64_t elem = is_8bit(kv_dtype) ? 1 : 2;
    const int64_t block_bytes = (int64_t)num_kv_heads * block_size * head_dim * elem;
    if (block_bytes % 16 != 0) return PA_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !block_pairs) return PA_ERR_INVALID_ARG;
    if (!aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
    pa::CopyBlocksParams p = {};
    p.k_cache = static_cast<uint8_t *>(k_cache);
    p.v_cache = static_cast<uint8_t *>(v_cache);
    p.pairs = block_pairs;
    p.err = dev_err;
    p.num_pairs = num_pairs;
    p.num_blocks = num_blocks;
    p.block_bytes = block_bytes;
    return from_cuda(pa::launch_copy_blocks(p, static_cast<cudaStream_t>(stream)));
}

pa_status pa_cache_write_per_channel(const void *k_new, const void *v_new, void *k_cache,
                                     void *v_cache, const int64_t *slot_mapping, int num_tokens,
                                     int num_blocks, int num_kv_heads, int head_dim,
                                     int block_size, pa_dtype act_dtype, pa_dtype kv_dtype,
                                     const float *k_scales, const float *v_scales, int *dev_err,
                                     void *stream) {
    if (num_tokens < 0 || num_blocks < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
        return PA_ERR_INVALID_ARG;
    if (!is_act(act_dtype) || !is_8bit(kv_dtype)) return PA_ERR_UNSUPPORTED;
    if (head_dim % 8 != 0) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping || !k_scales || !v_scales)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned16(k_scales) || !aligned16(v_scales))
        return PA_ERR_INVALID_ARG;
    pa::CacheWriteParams p = {};
    p.k_new = k_new;
    p.v_new = v_new;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.slot_mapping = slot_mapping;
    p.err = dev_err;
    p.num_tokens = num_tokens;
    p.num_blocks = num_blocks;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.block_size = block_size;
    p.k_scale = 1.0f;
    p.v_scale = 1.0f;
    p.k_chan = k_scales;
    p.v_chan = v_scales;
    return from_cuda(pa::launch_cache_write(p, to_internal(act_dtype), to_internal(kv_dtype),
                                            static_cast<cudaStream_t>(stream)));
}

pa_status pa_decode_per_channel(void *out, const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *block_tables, int max_blocks_per_seq,
                                const int32_t *seq_lens, int num_seqs, int num_q_heads,
                                int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                float softmax_scale, pa_dtype q_dtype, pa_dtype kv_dtype,
                                const float *k_scales, const float *v_scales, int partition_size,
                                int max_seq_len, void *workspace, size_t workspace_bytes,
                                int *dev_err, void *stream) {
    const DecodeArgs a = {out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                          num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                          softmax_scale, q_dtype, kv_dtype, 1.0f, 1.0f};
    if (!is_8bit(kv_dtype)) return PA_ERR_UNSUPPORTED;
    const pa_status st = check_decode(a);
    if (st != PA_OK) return st;
    if (partition_size < 0 || partition_size > kMaxPartitionSize || partition_size % pa::kBlockSize != 0 ||
        max_seq_len < 0 || max_seq_len > kMaxSeqLen)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    if (!k_scales || !v_scales || (reinterpret_cast<uintptr_t>(k_scales) & 3u) ||
        (reinterpret_cast<uintptr_t>(v_scales) & 3u))
        return PA_ERR_INVALID_ARG;
    pa::DecodeParams p = make_decode_params(a, dev_err);
    p.k_chan = k_scales;
    p.v_chan = v_scales;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (partition_size == 0) {
        p.partition_blocks = max_blocks_per_seq << p.tile_shift;  // every 16-token tile
        p.num_partitions = 1;
        p.split = 0;
        return from_cuda(launch_any_decode(p, q_dtype, kv_dtype, head_dim, s));
    }
    const size_t need = pa_split_workspace_bytes(num_seqs, num_q_heads, head_dim, max_seq_len,
                                                 partition_size);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return PA_ERR_INVALID_ARG;
    const int np = max_seq_len > 0 ? (int)ceil_div64(max_seq_len, partition_size) : 1;
    if ((int64_t)num_seqs * np > 0x7FFFFFFF) return PA_ERR_UNSUPPORTED;
    const size_t rows = (size_t)num_seqs * num_q_heads * np;
    p.ws_lse = static_cast<float *>(workspace);
    p.ws_o = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + align256(rows * sizeof(float)));
    p.partition_blocks = partition_size / pa::kBlockSize;
    p.num_partitions = np;
    p.split = 1;
    if (launch_any_decode(p, q_dtype, kv_dtype, head_dim, s) != cudaSuccess) return PA_ERR_CUDA;
    pa::ReduceParams r = {};
    r.out = out;
    r.ws_lse = p.ws_lse;
    r.ws_o = p.ws_o;
    r.seq_lens = seq_lens;
    r.num_seqs = num_seqs;
    r.num_q_heads = num_q_heads;
    r.num_partitions = np;
    r.partition_size = partition_size;
    return from_cuda(pa::launch_reduce(r, to_internal(q_dtype), head_dim, s));
}

size_t pa_shared_prefix_workspace_bytes(int num_seqs, int num_q_heads, int head_dim,
                                        int max_seq_len, int prefix_len, int partition_size) {
    if (num_seqs < 0 || num_q_heads <= 0 || head_dim <= 0 || max_seq_len < 0 || prefix_len < 0 ||
        partition_size <= 0)
        return 0;
    const int tail = max_seq_len > prefix_len ? max_seq_len - prefix_len : 0;
    const size_t np = (size_t)pa::prefix_splits(prefix_len) + (size_t)ceil_div64(tail, partition_size);
    const size_t rows = (size_t)num_seqs * (size_t)num_q_heads * np;
    return align256(rows * sizeof(float)) + align256(rows * (size_t)head_dim * sizeof(float));
}

pa_status pa_decode_shared_prefix(void *out, const void *q, const void *k_cache,
                                  const void *v_cache, const int32_t *block_tables,
                                  int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs,
                                  int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                  int num_blocks, float softmax_scale, pa_dtype q_dtype,
                                  pa_dtype kv_dtype, float k_scale, float v_scale, int prefix_len,
                                  int partition_size, int max_seq_len, void *workspace,
                                  size_t workspace_bytes, int *dev_err, void *stream) {
    const DecodeArgs a = {out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                          num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                          softmax_scale, q_dtype, kv_dtype, k_scale, v_scale};
    pa_status st = check_decode(a);
    if (st != PA_OK) return st;
    const bool kv8 = is_8bit(kv_dtype);
    if (kv8 && head_dim != 128) return PA_ERR_UNSUPPORTED;  // the prefix pass: 8-bit needs d 128
    const int g = num_q_heads / num_kv_heads;
    if (g > 128) return PA_ERR_UNSUPPORTED;
    if (!(softmax_scale > 0.f)) return PA_ERR_INVALID_ARG;
    if (partition_size <= 0 || partition_size > kMaxPartitionSize || partition_size % pa::kBlockSize != 0 ||
        max_seq_len < 0 || max_seq_len > kMaxSeqLen)
        return PA_ERR_INVALID_ARG;
    if (prefix_len <= 0 || prefix_len % block_size != 0 || prefix_len > max_seq_len ||
        prefix_len > max_blocks_per_seq * block_size)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    if (num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;
    const int64_t pool_rows = (int64_t)num_blocks * num_kv_heads * block_size;
    if (pool_rows + block_size >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
    const size_t need = pa_shared_prefix_workspace_bytes(num_seqs, num_q_heads, head_dim,
                                                         max_seq_len, prefix_len, partition_size);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return PA_ERR_INVALID_ARG;
    if (!pa::prefill_supported()) return PA_ERR_CUDA;  // no tensor-map encoder in the driver
    const int np_tail = (int)ceil_div64((int64_t)max_seq_len - prefix_len, partition_size);
    const int nz = pa::prefix_splits(prefix_len);  // prefix key ranges: slots 0 .. nz - 1
    const int np = nz + np_tail;
    if ((int64_t)num_seqs * (np_tail > 0 ? np_tail : 1) > 0x7FFFFFFF) return PA_ERR_UNSUPPORTED;
    const size_t rows = (size_t)num_seqs * num_q_heads * np;
    float *ws_lse = static_cast<float *>(workspace);
    float *ws_o = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + align256(rows * sizeof(float)));
    const cudaStream_t s = static_cast<cudaStream_t>(stream);

    // 1. the prefix, once for every sequence: workspace slots 0 .. nz - 1
    pa::PrefillParams f = {};
    f.q = q;
    f.k_cache = k_cache;
    f.v_cache = v_cache;
    f.block_tables = block_tables;  // row 0 names the shared blocks
    f.err = dev_err;
    f.max_blocks_per_seq = max_blocks_per_seq;
    f.num_seqs = 1;
    f.num_tokens = num_seqs;        // one query row per decoding sequence
    f.max_query_len = num_seqs;
    f.num_q_heads = num_q_heads;
    f.num_kv_heads = num_kv_heads;
    f.num_blocks = num_blocks;
    f.block_size = block_size;
    f.tile_shift = block_size == 32 ? 1 : 0;
    f.group = g;
    f.tok_per_tile = 128 / g;
    f.oob_row = (int)pool_rows;
    f.qk_scale_log2 =
        (float)((double)softmax_scale * (kv8 ? (double)k_scale : 1.0) * 1.4426950408889634074);
    f.v_scale = kv8 ? v_scale : 1.0f;
    f.shared_len = prefix_len;
    f.ws_o = ws_o;
    f.ws_lse = ws_lse;
    f.ws_np = np;
    if (pa::launch_prefill(f, to_internal(q_dtype), to_internal(kv_dtype), head_dim, s) != cudaSuccess)
        return PA_ERR_CUDA;

    // 2. every sequence's tail, split into partitions: slots nz .. np - 1
    if (np_tail > 0) {
        pa::DecodeParams p = make_decode_params(a, dev_err);
        p.ws_lse = ws_lse;
        p.ws_o = ws_o;
        p.partition_blocks = partition_size / pa::kBlockSize;
        p.num_partitions = np_tail;
        p.split = 1;
        p.tile_begin = prefix_len / pa::kBlockSize;
        p.ws_offset = nz;
        p.ws_np = np;
        if (launch_any_decode(p, q_dtype, kv_dtype, head_dim, s) != cudaSuccess) return PA_ERR_CUDA;
    }

    // 3. merge the prefix partials with the tail partitions
    pa::ReduceParams r = {};
    r.out = out;
    r.ws_lse = ws_lse;
    r.ws_o = ws_o;
    r.seq_lens = seq_lens;
    r.num_seqs = num_seqs;
    r.num_q_heads = num_q_heads;
    r.num_partitions = np;
    r.partition_size = partition_size;
    r.extra = nz;
    r.token_begin = prefix_len;
    return from_cuda(pa::launch_reduce(r, to_internal(q_dtype), head_dim, s));
}

size_t pa_split_workspace_bytes(int num_seqs, int num_q_heads, int head_dim, int max_seq_len,
                                int partition_size) {
    if (num_seqs < 0 || num_q_heads <= 0 || head_dim <= 0 || max_seq_len < 0 ||
        partition_size <= 0)
        return 0;
    const size_t np = max_seq_len > 0 ? (size_t)ceil_div64(max_seq_len, partition_size) : 1;
    const size_t rows = (size_t)num_seqs * (size_t)num_q_heads * np;
    return align256(rows * sizeof(float)) + align256(rows * (size_t)head_dim * sizeof(float));
}

}  // extern "C"

namespace pa {

// The host-side checks of pa_decode_split_reduce, workspace aside (no GPU
// access): PA_OK or the status the call returns before any launch.
int check_split_reduce_args(const void *out, const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *block_tables,
                            int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs,
                            int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                            int num_blocks, float softmax_scale, int q_dtype, int kv_dtype,
                            float k_scale, float v_scale, int partition_size, int max_seq_len) {
    // the checks only test out for null and alignment
    const DecodeArgs a = {const_cast<void *>(out), q, k_cache, v_cache, block_tables,
                          max_blocks_per_seq, seq_lens,
                          num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                          softmax_scale, static_cast<pa_dtype>(q_dtype),
                          static_cast<pa_dtype>(kv_dtype), k_scale, v_scale};
    const pa_status st = check_decode(a);
    if (st != PA_OK) return st;
    if (partition_size <= 0 || partition_size > kMaxPartitionSize || partition_size % kBlockSize != 0 ||
        max_seq_len < 0 || max_seq_len > kMaxSeqLen)
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    const int64_t np = max_seq_len > 0 ? ceil_div64(max_seq_len, partition_size) : 1;
    if ((int64_t)num_seqs * np > 0x7FFFFFFF) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

}  // namespace pa

extern "C" {

pa_status pa_decode_split_reduce(void *out, const void *q, const void *k_cache,
                                 const void *v_cache, const int32_t *block_tables,
                                 int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs,
                                 int num_q_heads, int num_kv_heads, int head_dim,
                                 int block_size, int num_blocks, float softmax_scale,
                                 pa_dtype q_dtype, pa_dtype kv_dtype, float k_scale,
                                 float v_scale, int partition_size, int max_seq_len,
                                 void *workspace, size_t workspace_bytes, int *dev_err,
                                 void *stream) {
    const pa_status st = static_cast<pa_status>(pa::check_split_reduce_args(
        out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
        num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, softmax_scale, q_dtype,
        kv_dtype, k_scale, v_scale, partition_size, max_seq_len));
    if (st != PA_OK || num_seqs == 0) return st;
    const DecodeArgs a = {out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                          num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                          softmax_scale, q_dtype, kv_dtype, k_scale, v_scale};
    const size_t need = pa_split_workspace_bytes(num_seqs, num_q_heads, head_dim, max_seq_len,
                                                 partition_size);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return PA_ERR_INVALID_ARG;
    const int np = max_seq_len > 0 ? (int)ceil_div64(max_seq_len, partition_size) : 1;

    pa::DecodeParams p = make_decode_params(a, dev_err);
    const size_t rows = (size_t)num_seqs * num_q_heads * np;
    p.ws_lse = static_cast<float *>(workspace);
    p.ws_o = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + align256(rows * sizeof(float)));
    p.partition_blocks = partition_size / pa::kBlockSize;
    p.num_partitions = np;
    p.split = 1;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_any_decode(p, q_dtype, kv_dtype, head_dim, s);
    if (e != cudaSuccess) return PA_ERR_CUDA;
    pa::ReduceParams r = {};
    r.out = out;
    r.ws_lse = p.ws_lse;
    r.ws_o = p.ws_o;
    r.seq_lens = seq_lens;
    r.num_seqs = num_seqs;
    r.num_q_heads = num_q_heads;
    r.num_partitions = np;
    r.partition_size = partition_size;
    return from_cuda(pa::launch_reduce(r, to_internal(q_dtype), head_dim, s));
}

}  // extern "C"
