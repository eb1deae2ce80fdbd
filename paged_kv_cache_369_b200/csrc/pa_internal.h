// Internal interface between the C-ABI shim (pa_capi.cu) and the kernel
// translation units.  Not installed; the public ABI is include/pa.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace pa {

// Kernels work in tiles of 16 tokens (one TMA box, one MMA n-tile).  A pool
// block holds block_size = 16 or 32 tokens, i.e. 1 or 2 tiles: tile u of a
// sequence lives in its block u >> tile_shift, at row (u & (tiles per block
// - 1)) * 16 of that block.
constexpr int kBlockSize = 16;        // tokens per tile
constexpr int kMaxBlockSize = 32;     // largest supported pool block
constexpr int kDecodeWarps = 4;       // consumer warps per decode CTA
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s bound on any device wait
constexpr int kErrBounds = 4;         // = PA_ERR_DEVICE_BOUNDS
constexpr int kErrTimeout = 5;        // = PA_ERR_DEVICE_TIMEOUT

enum class DType : int { F16 = 0, BF16 = 1, E4M3 = 2, E5M2 = 3, I8 = 4 };

inline bool is_8bit(DType t) { return t == DType::E4M3 || t == DType::E5M2 || t == DType::I8; }

struct SlotParams {
    int64_t *slot_mapping;
    const int32_t *block_tables;
    const int32_t *seq_lens;
    const int32_t *token_seq;
    const int32_t *token_pos;
    int *err;
    int max_blocks_per_seq;
    int num_tokens;
    int num_seqs;
    int block_size;
    int num_blocks;
};

struct CacheWriteParams {
    const void *k_new;
    const void *v_new;
    void *k_cache;
    void *v_cache;
    const int64_t *slot_mapping;
    int *err;
    int num_tokens;
    int num_blocks;
    int num_kv_heads;
    int head_dim;
    int block_size;
    float k_scale;
    float v_scale;
    const float *k_chan;        // per-channel scales [Hk, D] (8-bit caches) or null
    const float *v_chan;
};

struct DecodeParams {
    void *out;                  // [S, Hq, D] q dtype (single pass)
    const void *q;              // [S, Hq, D]
    const uint8_t *k_cache;     // [NB, Hk, 16, D] kv dtype, as bytes
    const uint8_t *v_cache;
    const int32_t *block_tables;
    const int32_t *seq_lens;
    float *ws_lse;              // split: [S, Hq, NP]
    float *ws_o;                // split: [S, Hq, NP, D]
    int *err;
    int max_blocks_per_seq;
    int num_seqs;
    int num_q_heads;
    int num_kv_heads;
    int num_blocks;
    int block_size;             // tokens per pool block: 16 or 32
    int tile_shift;             // log2(block_size / 16)
    int group;                  // Hq / Hk
    int head_groups;            // CTAs per KV head (ceil(group / G))
    int partition_blocks;       // 16-token tiles per partition
    int num_partitions;         // NP (1 in single-pass mode)
    int split;                  // 1: write partials to the workspace
    // shared-prefix decode: the tail of every sequence starts at tile
    // tile_begin (0 otherwise); partition p is written to workspace slot
    // ws_offset + p of ws_np slots per row (ws_np 0: num_partitions)
    int tile_begin;
    int ws_offset;
    int ws_np;
    // split mode, tensor-core kernel: 0, or each warp attends `chain`
    // consecutive partitions on its own, one after another (its copies run
    // ahead across their boundaries), writing each one's partial from its
    // registers; set by the launcher for long contexts
    int chain;
    float qk_scale_log2;        // softmax_scale * k_scale * log2(e)
    float v_scale;              // applied to the output (1 for 16-bit caches)
    // per-channel scales of an 8-bit cache, [Hk, D] fp32, or null: K's are
    // folded into q (k_scale then 1), V's applied to the output per channel
    const float *k_chan;
    const float *v_chan;
    // append (pa_decode_append): this step's new token of every sequence,
    // stored at position seq_len - 1 before it is attended
    int append;
    const void *k_new;          // [S, Hk, D] activation dtype
    const void *v_new;
    uint8_t *k_pool_w;          // the pools again, writable
    uint8_t *v_pool_w;
    float k_scale_w;            // E4M3 quantisation scales (1 for 16-bit caches)
    float v_scale_w;
    // failure-detection test hook, never set through the public ABI (the C
    // shim reads it from the environment variable PA369_TEST_DECODE_STALL_NS):
    // the main loop's copy waits give up after wait_limit_ns (0: kWaitLimitNs),
    // and with hold_first_tile every warp leaves its first tile's copies
    // unissued, so that the first wait can only run out.  The drain of the
    // copies that were issued keeps its own bound.
    uint64_t wait_limit_ns;
    int hold_first_tile;
};

struct AppendParams {  // decode-form slot mapping + cache write in one kernel
    const void *k_new;
    const void *v_new;
    void *k_cache;
    void *v_cache;
    const int32_t *block_tables;
    const int32_t *seq_lens;
    int *err;
    int max_blocks_per_seq;
    int num_seqs;
    int num_kv_heads;
    int head_dim;
    int num_blocks;
    int block_size;
    float k_scale;
    float v_scale;
};

struct CopyBlocksParams {  // copy-on-write: whole blocks inside both pools
    uint8_t *k_cache;
    uint8_t *v_cache;
    const int32_t *pairs;  // [num_pairs][2] = (src, dst)
    int *err;
    int num_pairs;
    int num_blocks;
    int64_t block_bytes;   // num_kv_heads * block_size * head_dim * elem bytes
};

struct PrefillParams {  // chunked prefill (pa_prefill)
    void *out;                  // [T, Hq, D] q dtype
    const void *q;              // [T, Hq, D]
    const void *k_cache;        // [NB, Hk, 16, D]
    const void *v_cache;
    const int32_t *block_tables;
    const int32_t *seq_lens;    // [S] cached tokens, the chunk included
    const int32_t *query_start; // [S + 1] chunk rows of each sequence
    int *err;
    int max_blocks_per_seq;
    int num_seqs;
    int num_tokens;             // T
    int max_query_len;          // bounds every chunk length
    int num_q_heads;
    int num_kv_heads;
    int num_blocks;
    int block_size;             // tokens per pool block: 16 or 32
    int tile_shift;             // log2(block_size / 16)
    int group;                  // Hq / Hk
    int tok_per_tile;           // floor(128 / group) chunk tokens per query tile
    int oob_row;                // a pool row index past the end (zero-filled loads)
    float qk_scale_log2;        // softmax_scale * k_scale * log2(e)
    float v_scale;              // applied to the output (1 for 16-bit caches)
    // shared-prefix mode (shared_len > 0): one "sequence" = the first
    // shared_len tokens of block table row 0; the T query rows (one per
    // decoding sequence) all see every one of them (no causal mask).  The
    // keys are cut into items_z ranges; range z writes each row's partial
    // (lse, o / l) to workspace slot z of ws_np per row
    int shared_len;
    float *ws_o;
    float *ws_lse;
    int ws_np;
    // set by the launch: the work items are items_x (query tile pairs) x
    // num_kv_heads x items_z (sequences, or prefix key ranges), and
    // work_slot names the launch's work counter
    int items_x;
    int items_z;
    int work_slot;
    // failure-detection test hook, never set through the public ABI (the
    // launch reads it from the environment variable PA369_TEST_PREFILL_STALL_NS):
    // every device wait gives up after wait_limit_ns (0: kWaitLimitNs), and
    // with hold_first_tile each CTA leaves its first K/V stage's copies
    // unissued, so that the first wait on it can only run out
    uint64_t wait_limit_ns;
    int hold_first_tile;
};

struct ReduceParams {
    void *out;
    const float *ws_lse;
    const float *ws_o;
    const int32_t *seq_lens;
    int num_seqs;
    int num_q_heads;
    int num_partitions;         // workspace slots per row
    int partition_size;
    // shared-prefix decode: `extra` leading slots hold the prefix partials and
    // the partitions cover tokens from token_begin (0 / 0 otherwise)
    int extra;
    int token_begin;
};

// Host-side argument checks of pa_decode_split_reduce, the workspace aside;
// touches no GPU.  Returns PA_OK (0) or the pa_status the call would return
// before any launch.  q_dtype / kv_dtype are pa_dtype values.
int check_split_reduce_args(const void *out, const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *block_tables,
                            int max_blocks_per_seq, const int32_t *seq_lens, int num_seqs,
                            int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                            int num_blocks, float softmax_scale, int q_dtype, int kv_dtype,
                            float k_scale, float v_scale, int partition_size, int max_seq_len);

// Launchers: return cudaSuccess or the launch error.
cudaError_t launch_slot_mapping(const SlotParams &p, cudaStream_t stream);
cudaError_t launch_append(const AppendParams &p, DType act, DType kv, cudaStream_t stream);
cudaError_t launch_cache_write(const CacheWriteParams &p, DType act, DType kv, cudaStream_t stream);
cudaError_t launch_decode(const DecodeParams &p, DType q, DType kv, int head_dim, int tpl_group,
                          cudaStream_t stream);
cudaError_t launch_reduce(const ReduceParams &p, DType q, int head_dim, cudaStream_t stream);
cudaError_t launch_copy_blocks(const CopyBlocksParams &p, cudaStream_t stream);

// Chunked prefill on tcgen05 tensor cores (pa_prefill.cu): 16-bit caches
// (head_dim 64 / 128) or 8-bit ones (head_dim 128), GQA groups up to 128.
bool prefill_supported();
cudaError_t launch_prefill(const PrefillParams &p, DType q, DType kv, int head_dim, cudaStream_t stream);

// Tensor-core decode (pa_decode_mma.cu): rows of the MMA used for the GQA
// group (8 or 16); supported for head_dim 64/128 16-bit caches and head_dim
// 128 8-bit caches whose pool has fewer than 2^31 token rows.
bool mma_decode_supported(DType kv, int head_dim, int num_blocks, int num_kv_heads, int block_size);
cudaError_t launch_decode_mma(const DecodeParams &p, DType q, DType kv, int head_dim, int mma_rows,
                              cudaStream_t stream);

}  // namespace pa
