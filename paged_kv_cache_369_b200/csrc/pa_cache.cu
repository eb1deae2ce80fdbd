// Slot mapping and cache write: the append side of the paged KV cache.
//
// Slot of a token: its sequence's block table maps logical block pos / 16 to
// a physical block; the token sits at offset pos % 16 ("Transformer 推理优化：
// KV Cache、PagedAttention 与 vLLM", §3.3).  The cache write stores each
// token's per-head K/V rows there, one new block being opened every 16 tokens
// ("vLLM推理引擎深度解析：PagedAttention与连续批处理", §2.2), optionally as
// 8-bit codes: FP8 E4M3 ("大语言模型推理引擎深度剖析", §4.3), FP8 E5M2 or INT8
// (the openeuler page's §2.3 table of KV cache formats).
//
// Both kernels are HBM-trivial next to attention (a few MB per step); they are
// written for full 16-byte vector traffic and a grid of whole waves.
//
// Copy-on-write: before a sequence writes into a block it shares with other
// sequences (a beam-search fork, a shared prompt prefix), the engine copies
// that block into a free one and repoints the sequence's table entry
// ("Transformer 推理优化：KV Cache、PagedAttention 与 vLLM", §3.5; "大语言模型推理
// 引擎深度剖析", §2.3).  copy_blocks_kernel does the copy for a batch of
// (src, dst) pairs, K and V pools alike.
#include "pa_device.cuh"

namespace pa {

// ---------------------------------------------------------------------------
// slot mapping: one thread per token
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(256) slot_mapping_kernel(const SlotParams p) {
    const int64_t B = p.block_size;
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < p.num_tokens;
         t += gridDim.x * blockDim.x) {
        const int s = p.token_seq ? p.token_seq[t] : t;
        int64_t slot = -1;
        if (s >= 0) {
            bool ok = s < p.num_seqs;
            int64_t pos = -1;
            if (ok) pos = p.token_pos ? (int64_t)p.token_pos[t] : (int64_t)p.seq_lens[s] - 1;
            ok = ok && pos >= 0 && pos < (int64_t)p.max_blocks_per_seq * B;
            if (ok) {
                const int64_t phys = p.block_tables[(int64_t)s * p.max_blocks_per_seq + pos / B];
                ok = phys >= 0 && phys < p.num_blocks;
                if (ok) slot = phys * B + pos % B;
            }
            if (!ok) flag_error(p.err, kErrBounds);
        }
        p.slot_mapping[t] = slot;
    }
}

cudaError_t launch_slot_mapping(const SlotParams &p, cudaStream_t stream) {
    if (p.num_tokens <= 0) return cudaSuccess;
    const int threads = 256;
    int blocks = (p.num_tokens + threads - 1) / threads;
    if (blocks > 65536) blocks = 65536;
    slot_mapping_kernel<<<blocks, threads, 0, stream>>>(p);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// cache write: one thread per 8-element vector of one (token, head) row,
// handling the K and the V vector at the same position
// ---------------------------------------------------------------------------

template <typename ACT, typename KVT>
__global__ void __launch_bounds__(256) cache_write_kernel(const CacheWriteParams p) {
    constexpr bool FP8 = Elem<KVT>::kBytes == 1;  // any 8-bit code
    const int vecs_per_row = p.head_dim / 8;
    const int64_t per_token = (int64_t)p.num_kv_heads * vecs_per_row;
    const int64_t total = (int64_t)p.num_tokens * per_token;
    const int64_t nslots = (int64_t)p.num_blocks * p.block_size;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total;
         g += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = g / per_token;
        const int64_t rem = g - t * per_token;
        const int64_t h = rem / vecs_per_row;
        const int64_t c = rem - h * vecs_per_row;
        const int64_t slot = p.slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= nslots) {
            if (h == 0 && c == 0) flag_error(p.err, kErrBounds);
            continue;
        }
        const int64_t blk = slot / p.block_size, off = slot - blk * p.block_size;
        const int64_t src = ((t * p.num_kv_heads + h) * p.head_dim + c * 8);
        const int64_t dst = (((blk * p.num_kv_heads + h) * p.block_size + off) * p.head_dim + c * 8);
        const uint4 kin = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.k_new) + src);
        const uint4 vin = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.v_new) + src);
        if constexpr (FP8) {
            uint2 kq, vq;
            if (p.k_chan) {  // per-channel scales of this head's 8 elements
                const float4 *ks = reinterpret_cast<const float4 *>(p.k_chan + h * p.head_dim + c * 8);
                const float4 *vs = reinterpret_cast<const float4 *>(p.v_chan + h * p.head_dim + c * 8);
                const float4 k0 = ks[0], k1 = ks[1], v0 = vs[0], v1 = vs[1];
                const float kk[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
                const float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                kq = quantise8_chan<ACT, KVT>(kin, kk);
                vq = quantise8_chan<ACT, KVT>(vin, vv);
            } else {
                kq = quantise8<ACT, KVT>(kin, p.k_scale);
                vq = quantise8<ACT, KVT>(vin, p.v_scale);
            }
            *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(p.k_cache) + dst) = kq;
            *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(p.v_cache) + dst) = vq;
        } else {
            *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.k_cache) + dst) = kin;
            *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.v_cache) + dst) = vin;
        }
    }
}

// Launch kernel template K<ACT, KVT> for an (activation, cache) dtype pair.
template <template <typename, typename> class K, typename P>
static cudaError_t launch_by_dtypes(const P &p, DType act, DType kv, unsigned blocks, cudaStream_t stream) {
    auto go = [&](auto act_tag, auto kv_tag) {
        using A = decltype(act_tag);
        using KV = decltype(kv_tag);
        K<A, KV>::launch(p, blocks, stream);
        return cudaGetLastError();
    };
    const bool f16 = act == DType::F16;
    switch (kv) {
        case DType::E4M3: return f16 ? go(f16_t{}, e4m3_t{}) : go(bf16_t{}, e4m3_t{});
        case DType::E5M2: return f16 ? go(f16_t{}, e5m2_t{}) : go(bf16_t{}, e5m2_t{});
        case DType::I8: return f16 ? go(f16_t{}, i8_t{}) : go(bf16_t{}, i8_t{});
        default: return f16 ? go(f16_t{}, f16_t{}) : go(bf16_t{}, bf16_t{});
    }
}

template <typename ACT, typename KVT> struct CacheWriteLaunch {
    static void launch(const CacheWriteParams &p, unsigned blocks, cudaStream_t stream) {
        cache_write_kernel<ACT, KVT><<<blocks, 256, 0, stream>>>(p);
    }
};

cudaError_t launch_cache_write(const CacheWriteParams &p, DType act, DType kv, cudaStream_t stream) {
    const int64_t total = (int64_t)p.num_tokens * p.num_kv_heads * (p.head_dim / 8);
    if (total <= 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    if (blocks > (1 << 20)) blocks = 1 << 20;
    return launch_by_dtypes<CacheWriteLaunch>(p, act, kv, (unsigned)blocks, stream);
}

// ---------------------------------------------------------------------------
// append: the decode form of slot mapping + cache write in one kernel.  The
// new token of sequence s sits at position seq_lens[s] - 1; its slot is
// computed inline (no slot array).  Used where the decode kernel does not
// patch the new token itself.
// ---------------------------------------------------------------------------

template <typename ACT, typename KVT>
__global__ void __launch_bounds__(256) append_kernel(const AppendParams p) {
    constexpr bool FP8 = Elem<KVT>::kBytes == 1;  // any 8-bit code
    const int vecs_per_row = p.head_dim / 8;
    const int64_t per_seq = (int64_t)p.num_kv_heads * vecs_per_row;
    const int64_t total = (int64_t)p.num_seqs * per_seq;
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total;
         g += (int64_t)gridDim.x * blockDim.x) {
        const int64_t s = g / per_seq;
        const int64_t rem = g - s * per_seq;
        const int64_t h = rem / vecs_per_row;
        const int64_t c = rem - h * vecs_per_row;
        const int L = p.seq_lens[s];
        if (L <= 0) continue;  // an empty sequence has no new token
        const bool first = h == 0 && c == 0;
        const int64_t pos = L - 1;
        if (pos >= (int64_t)p.max_blocks_per_seq * p.block_size) {
            if (first) flag_error(p.err, kErrBounds);
            continue;
        }
        const int64_t phys = p.block_tables[s * p.max_blocks_per_seq + pos / p.block_size];
        if (phys < 0 || phys >= p.num_blocks) {
            if (first) flag_error(p.err, kErrBounds);
            continue;
        }
        const int64_t src = ((s * p.num_kv_heads + h) * p.head_dim + c * 8);
        const int64_t dst = (((phys * p.num_kv_heads + h) * p.block_size + pos % p.block_size) * p.head_dim + c * 8);
        const uint4 kin = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.k_new) + src);
        const uint4 vin = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.v_new) + src);
        if constexpr (FP8) {
            *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(p.k_cache) + dst) = quantise8<ACT, KVT>(kin, p.k_scale);
            *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(p.v_cache) + dst) = quantise8<ACT, KVT>(vin, p.v_scale);
        } else {
            *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.k_cache) + dst) = kin;
            *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.v_cache) + dst) = vin;
        }
    }
}

template <typename ACT, typename KVT> struct AppendLaunch {
    static void launch(const AppendParams &p, unsigned blocks, cudaStream_t stream) {
        append_kernel<ACT, KVT><<<blocks, 256, 0, stream>>>(p);
    }
};

cudaError_t launch_append(const AppendParams &p, DType act, DType kv, cudaStream_t stream) {
    const int64_t total = (int64_t)p.num_seqs * p.num_kv_heads * (p.head_dim / 8);
    if (total <= 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    if (blocks > (1 << 20)) blocks = 1 << 20;
    return launch_by_dtypes<AppendLaunch>(p, act, kv, (unsigned)blocks, stream);
}

// ---------------------------------------------------------------------------
// copy-on-write block copy: grid (pair, stripe, pool); a block is one
// contiguous span of block_bytes in each pool, copied with 16-byte vectors,
// kCopyUnroll loads in flight per thread before the stores
// ---------------------------------------------------------------------------

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(kCopyThreads) copy_blocks_kernel(const CopyBlocksParams p) {
    const int64_t pair = blockIdx.x;
    const int src = p.pairs[2 * pair], dst = p.pairs[2 * pair + 1];
    if ((unsigned)src >= (unsigned)p.num_blocks || (unsigned)dst >= (unsigned)p.num_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) flag_error(p.err, kErrBounds);
        return;
    }
    if (src == dst) return;
    uint8_t *pool = blockIdx.z ? p.v_cache : p.k_cache;
    const uint4 *from = reinterpret_cast<const uint4 *>(pool + (int64_t)src * p.block_bytes);
    uint4 *to = reinterpret_cast<uint4 *>(pool + (int64_t)dst * p.block_bytes);
    const int64_t nv = p.block_bytes / 16;
    const int64_t step = (int64_t)gridDim.y * kCopyThreads * kCopyUnroll;
    for (int64_t base = (int64_t)blockIdx.y * kCopyThreads * kCopyUnroll + threadIdx.x; base < nv;
         base += step) {
        uint4 r[kCopyUnroll];
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t i = base + (int64_t)u * kCopyThreads;
            if (i < nv) r[u] = from[i];
        }
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t i = base + (int64_t)u * kCopyThreads;
            if (i < nv) to[i] = r[u];
        }
    }
}

cudaError_t launch_copy_blocks(const CopyBlocksParams &p, cudaStream_t stream) {
    if (p.num_pairs <= 0 || p.block_bytes <= 0) return cudaSuccess;
    const int64_t per_cta = (int64_t)kCopyThreads * kCopyUnroll * 16;
    int64_t stripes = (p.block_bytes + per_cta - 1) / per_cta;
    if (stripes > 65535) stripes = 65535;
    copy_blocks_kernel<<<dim3((unsigned)p.num_pairs, (unsigned)stripes, 2), kCopyThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace pa
