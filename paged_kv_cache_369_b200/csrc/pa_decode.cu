// Paged decode attention for sm_100a.
//
// What is computed ("KV Cache 与 PageAttention深度实战", §1.2 and §3.2-§3.3):
// for the one new query row of every sequence and every query head,
// softmax(q K^T / sqrt(d)) V over the sequence's cached tokens, whose K/V rows
// live in 16-token blocks found through the sequence's block table.
//
// Design (B200): decode is HBM-bound ("openeuler.csdn.net 推理优化篇", §2.1:
// decode reads the whole cache for one token), so the kernel is built to
// stream every K/V byte exactly once at full bandwidth:
//   - one CTA per (sequence, partition of KV blocks, KV head [, head group])
//     serves all G query heads that share the KV head, so each KV byte is read
//     once per step (GQA);
//   - a (block, KV head) tile of K (or V) is one contiguous 16 x d span
//     (4 KiB for bf16 / d128) in the pool [blocks, heads, 16, d]; each warp
//     fetches its own tiles with 1-D TMA bulk copies (cp.async.bulk, no
//     multicast) into a private ring of shared-memory stages completed by
//     mbarriers, so many KiB per SM are in flight without register cost;
//   - the warp's block-table entries sit in its lanes' registers and are
//     shuffled out when a tile is issued (the table is read once, coalesced);
//   - q.K: 8 lanes per token row, 4 rows per pass, 16-byte shared loads
//     (every 8-lane phase reads 128 contiguous bytes: no bank conflicts); the
//     G partial dot products are reduce-scattered over the 8 lanes (7G/8
//     shuffles per 4 tokens instead of 3G);
//   - online softmax in the log2 domain (the softmax scale, the fp8 K scale and
//     log2(e) are folded into q); masked slots (t >= L) are excluded by select,
//     never by multiplication, so poisoned tails cannot leak in;
//   - P.V: 32 lanes across the row, p broadcast from shared memory;
//   - the warps' (m, l, acc) are merged through shared memory at the end and
//     written as the output row (single pass) or as the partition's
//     (lse, normalised o) for the split-KV reduce.
// Every wait on an mbarrier is bounded in time; every block-table entry and
// length is range-checked before use and reported through *err.
#include <math_constants.h>

#include "pa_device.cuh"

namespace pa {

template <typename QT, typename KVT, int D, int G> struct DecodeCfg {
    static constexpr int NW = kDecodeWarps;
    static constexpr int EB = Elem<KVT>::kBytes;
    static constexpr int ROW_BYTES = D * EB;            // one token row of a tile
    static constexpr int TILE_BYTES = kBlockSize * ROW_BYTES;
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;  // K tile + V tile
    static constexpr int NST = (16384 / STAGE_BYTES) < 2 ? 2 : (16384 / STAGE_BYTES);
    // q.K lane layout: 8 lanes per row
    static constexpr int LANE_BYTES = ROW_BYTES / 8;
    static constexpr int CHUNK_BYTES = LANE_BYTES < 16 ? LANE_BYTES : 16;
    static constexpr int NCHUNK = LANE_BYTES / CHUNK_BYTES;
    static constexpr int EPC = CHUNK_BYTES / EB;  // elements per chunk
    static constexpr int EPL = D / 8;             // elements per lane
    static constexpr int KWORDS = LANE_BYTES / 4 > 0 ? LANE_BYTES / 4 : 1;
    // P.V lane layout: 32 lanes per row
    static constexpr int V_LANE_BYTES = ROW_BYTES / 32;
    static constexpr int EPLV = D / 32;
    // shared memory carve-up (bytes)
    static constexpr int OFF_STAGES = 0;
    static constexpr int SZ_STAGES = NW * NST * STAGE_BYTES;
    static constexpr int OFF_P = OFF_STAGES + SZ_STAGES;
    static constexpr int P_FLOATS = kBlockSize * G + G;  // p[16][G] then alpha[G]
    static constexpr int SZ_P = NW * P_FLOATS * 4;
    static constexpr int OFF_BAR = (OFF_P + SZ_P + 7) / 8 * 8;
    static constexpr int SMEM = OFF_BAR + NW * NST * 8;
    static constexpr int MERGE_BYTES = NW * (G * D + 2 * G) * 4;
    static_assert(MERGE_BYTES <= SZ_STAGES, "merge area must fit in the stage buffers");
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "G in {1,2,4,8}");
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static_assert(TILE_BYTES % 16 == 0, "bulk copies move multiples of 16 bytes");
};

constexpr unsigned kFull = 0xFFFFFFFFu;

// Reduce-scatter step over lanes `lane ^ mask`: each lane keeps half of its N
// values (the upper half if `upper`), summed with the partner's copy.
template <int N> struct RsStep {
    static __device__ __forceinline__ void run(float *v, int mask, bool upper) {
        if constexpr (N >= 2) {
#pragma unroll
            for (int i = 0; i < N / 2; ++i) {
                const float keep = upper ? v[i + N / 2] : v[i];
                const float send = upper ? v[i] : v[i + N / 2];
                v[i] = keep + __shfl_xor_sync(kFull, send, mask);
            }
        } else {
            v[0] += __shfl_xor_sync(kFull, v[0], mask);
        }
    }
};

// After this, lane dp (0..7 inside its group of 8) holds in v[0] the sum over
// the 8 lanes of head (dp * G) / 8.
template <int G> __device__ __forceinline__ void reduce_scatter8(float *v, int dp) {
    RsStep<G>::run(v, 4, (dp & 4) != 0);
    RsStep<(G / 2 > 1 ? G / 2 : 1)>::run(v, 2, (dp & 2) != 0);
    RsStep<(G / 4 > 1 ? G / 4 : 1)>::run(v, 1, (dp & 1) != 0);
}

template <typename QT, typename KVT, int D, int G>
__global__ void __launch_bounds__(kDecodeWarps * 32)
    decode_kernel(const DecodeParams p) {
    using C = DecodeCfg<QT, KVT, D, G>;
    constexpr int NW = C::NW, NST = C::NST;
    extern __shared__ __align__(128) uint8_t smem[];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tr = lane >> 3, dp = lane & 7;  // q.K: token-in-row, lane-in-row
    const int NP = p.num_partitions;
    const int s = blockIdx.x / NP, part = blockIdx.x - s * NP;
    const int kvh = blockIdx.y / p.head_groups, hg = blockIdx.y - kvh * p.head_groups;

    const uint32_t bar0 = smem_addr(smem + C::OFF_BAR) + warp * NST * 8;
    const uint32_t stage0 = smem_addr(smem + C::OFF_STAGES) + warp * NST * C::STAGE_BYTES;
    const uint8_t *stage0_ptr = smem + C::OFF_STAGES + warp * NST * C::STAGE_BYTES;
    float *p_s = reinterpret_cast<float *>(smem + C::OFF_P) + warp * C::P_FLOATS;
    float *alpha_s = p_s + kBlockSize * G;

    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < NST; ++i) mbar_init(bar0 + 8 * i, 1);
        mbar_init_fence();
    }
    __syncwarp();

    // everything below reads memory the previous kernel may have written
    pdl_wait();

    // ---- sequence length and this CTA's block range ----------------------
    const int max_tokens = p.max_blocks_per_seq * p.block_size;
    int L = p.seq_lens[s];
    if (L < 0 || L > max_tokens) {
        if (threadIdx.x == 0) flag_error(p.err, kErrBounds);
        L = L < 0 ? 0 : max_tokens;
    }
    if (p.split) {
        const int cap = (p.tile_begin + NP * p.partition_blocks) * kBlockSize;
        if (L > cap) {
            if (threadIdx.x == 0 && part == 0) flag_error(p.err, kErrBounds);
            L = cap;
        }
    }
    const int nblk_seq = (L + kBlockSize - 1) / kBlockSize;
    if (L < p.tile_begin * kBlockSize) {  // shared-prefix decode: shorter than the prefix
        if (threadIdx.x == 0 && part == 0) flag_error(p.err, kErrBounds);
        L = p.tile_begin * kBlockSize;
    }
    const int blk_begin = p.tile_begin + part * p.partition_blocks;
    int blk_end = blk_begin + p.partition_blocks;
    if (blk_end > nblk_seq) blk_end = nblk_seq;
    if (p.split && blk_begin >= blk_end) return;  // empty partition: nothing to write
    const int nblk = blk_end > blk_begin ? blk_end - blk_begin : 0;
    const int nk = nblk > warp ? (nblk - warp + NW - 1) / NW : 0;  // this warp's blocks

    // ---- q rows of the G heads, scaled into the log2 domain ---------------
    const int group_base = hg * G;  // first head of this CTA inside the KV group
    float qf[G][C::EPL];
    {
        const QT *q = static_cast<const QT *>(p.q);
#pragma unroll
        for (int i = 0; i < G; ++i) {
            const bool hv = group_base + i < p.group;
            const int64_t hq = (int64_t)kvh * p.group + group_base + i;
            const uint16_t *qrow =
                reinterpret_cast<const uint16_t *>(q) + ((int64_t)s * p.num_q_heads + hq) * D;
#pragma unroll
            for (int c = 0; c < C::NCHUNK; ++c) {
                const int e0 = (c * 8 * C::CHUNK_BYTES + dp * C::CHUNK_BYTES) / C::EB;
#pragma unroll
                for (int v8 = 0; v8 < C::EPC; v8 += 8) {
                    uint4 w = make_uint4(0, 0, 0, 0);
                    if (hv) w = *reinterpret_cast<const uint4 *>(qrow + e0 + v8);
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                    float f[8];
                    Unpack<QT, 8>::run(ww, f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        // per-channel K scales: q.(code * s) = (q * s).code
                        const float ks = p.k_chan ? p.k_chan[(int64_t)kvh * D + e0 + v8 + e] : 1.f;
                        qf[i][c * C::EPC + v8 + e] = f[e] * ks * p.qk_scale_log2;
                    }
                }
            }
        }
    }

    // ---- this warp's block-table entries: lane i holds the entry of the
    //      warp's block 32 * batch + i ----------------------------------------
    const int32_t *bt_row = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
    auto load_batch = [&](int batch) -> int {  // the block holding each of the warp's tiles
        const int k = batch * 32 + lane;
        return k < nk ? bt_row[(blk_begin + warp + NW * k) >> p.tile_shift] : 0;
    };
    int cur_batch = 0;
    int bt_cur = load_batch(0);
    int bt_nxt = nk > 32 ? load_batch(1) : 0;
    auto bt_of = [&](int k) -> int {
        const int a = __shfl_sync(kFull, bt_cur, k & 31);
        const int b = __shfl_sync(kFull, bt_nxt, k & 31);
        return (k >> 5) == cur_batch ? a : b;
    };

    const uint8_t *kc = p.k_cache, *vc = p.v_cache;
    const int tiles_per_block = 1 << p.tile_shift;
    const int64_t head_off = (int64_t)kvh * tiles_per_block * C::TILE_BYTES;
    const int64_t blk_stride = (int64_t)p.num_kv_heads * tiles_per_block * C::TILE_BYTES;
    auto issue = [&](int k) {  // called by the whole warp
        int phys = bt_of(k);
        if (lane == 0) {
            if ((unsigned)phys >= (unsigned)p.num_blocks) {
                flag_error(p.err, kErrBounds);
                phys = 0;  // fetch a valid block; all its tokens are masked
            }
            const int st = k % NST;
            const uint32_t bar = bar0 + 8 * st;
            const uint32_t dst = stage0 + st * C::STAGE_BYTES;
            const int sub = (blk_begin + warp + NW * k) & (tiles_per_block - 1);  // tile in block
            const int64_t off = (int64_t)phys * blk_stride + head_off + (int64_t)sub * C::TILE_BYTES;
            mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
            bulk_g2s(dst, kc + off, C::TILE_BYTES, bar);
            bulk_g2s(dst + C::TILE_BYTES, vc + off, C::TILE_BYTES, bar);
        }
    };

    const int npre = nk < NST ? nk : NST;
    const int first_issued = p.hold_first_tile ? 1 : 0;  // test hook: tile 0 never issued
    for (int k = first_issued; k < npre; ++k) issue(k);
    const uint64_t wait_limit = p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs;

    // ---- main loop over this warp's blocks --------------------------------
    float m_run = -CUDART_INF_F, l_run = 0.f;
    float acc[G][C::EPLV];
#pragma unroll
    for (int i = 0; i < G; ++i)
#pragma unroll
        for (int e = 0; e < C::EPLV; ++e) acc[i][e] = 0.f;
    const int my_head = (dp * G) >> 3;
    const bool owner = ((dp * G) & 7) == 0;
    bool timed_out = false;
    int k = 0;

    for (; k < nk; ++k) {
        if (k > 0 && (k & 31) == 0) {
            bt_cur = bt_nxt;
            ++cur_batch;
            bt_nxt = nk > (cur_batch + 1) * 32 ? load_batch(cur_batch + 1) : 0;
        }
        const int st = k % NST;
        const bool ok = __all_sync(kFull, mbar_wait_bounded(bar0 + 8 * st, (k / NST) & 1, wait_limit));
        if (!ok) {
            if (lane == 0) flag_error(p.err, kErrTimeout);
            timed_out = true;
            break;
        }
        const int j = blk_begin + warp + NW * k;
        const bool valid = (unsigned)bt_of(k) < (unsigned)p.num_blocks;
        int nvalid = L - j * kBlockSize;
        nvalid = valid ? (nvalid < kBlockSize ? nvalid : kBlockSize) : 0;

        const uint8_t *ks = stage0_ptr + st * C::STAGE_BYTES;
        const uint8_t *vs = ks + C::TILE_BYTES;

        // q.K for the 16 tokens: 4 rows x (4 tokens, 8 lanes each)
        float sv[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int t = 4 * r + tr;
            uint32_t kw[C::KWORDS];
#pragma unroll
            for (int c = 0; c < C::NCHUNK; ++c) {
                const uint8_t *src = ks + t * C::ROW_BYTES + c * 8 * C::CHUNK_BYTES + dp * C::CHUNK_BYTES;
                if constexpr (C::CHUNK_BYTES == 16) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(src);
                    kw[4 * c] = w.x; kw[4 * c + 1] = w.y; kw[4 * c + 2] = w.z; kw[4 * c + 3] = w.w;
                } else {
                    const uint2 w = *reinterpret_cast<const uint2 *>(src);
                    kw[2 * c] = w.x; kw[2 * c + 1] = w.y;
                }
            }
            float kf[C::EPL];
            Unpack<KVT, C::EPL>::run(kw, kf);
            float part_dot[G];
#pragma unroll
            for (int i = 0; i < G; ++i) {
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < C::EPL; ++e) a = fmaf(qf[i][e], kf[e], a);
                part_dot[i] = a;
            }
            reduce_scatter8<G>(part_dot, dp);
            sv[r] = t < nvalid ? part_dot[0] : -CUDART_INF_F;
        }

        // online softmax for head my_head over this block
        float bm = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
        bm = fmaxf(bm, __shfl_xor_sync(kFull, bm, 8));
        bm = fmaxf(bm, __shfl_xor_sync(kFull, bm, 16));
        const float m_new = fmaxf(m_run, bm);
        float alpha = 1.f, pr[4] = {0.f, 0.f, 0.f, 0.f};
        if (m_new != -CUDART_INF_F) {
            alpha = exp2f(m_run - m_new);
#pragma unroll
            for (int r = 0; r < 4; ++r) pr[r] = exp2f(sv[r] - m_new);
        }
        l_run = l_run * alpha + ((pr[0] + pr[1]) + (pr[2] + pr[3]));
        m_run = m_new;
        if (owner) {
#pragma unroll
            for (int r = 0; r < 4; ++r) p_s[(4 * r + tr) * G + my_head] = pr[r];
            if (tr == 0) alpha_s[my_head] = alpha;
        }
        __syncwarp();

        // P.V: rescale, then accumulate the valid tokens
        {
            float al[G];
#pragma unroll
            for (int i = 0; i < G; ++i) al[i] = alpha_s[i];
#pragma unroll
            for (int i = 0; i < G; ++i)
#pragma unroll
                for (int e = 0; e < C::EPLV; ++e) acc[i][e] *= al[i];
        }
        auto pv_token = [&](int t) {
            uint32_t vw[C::V_LANE_BYTES >= 4 ? C::V_LANE_BYTES / 4 : 1];
            const uint8_t *src = vs + t * C::ROW_BYTES + lane * C::V_LANE_BYTES;
            if constexpr (C::V_LANE_BYTES == 8) {
                const uint2 w = *reinterpret_cast<const uint2 *>(src);
                vw[0] = w.x; vw[1] = w.y;
            } else if constexpr (C::V_LANE_BYTES == 4) {
                vw[0] = *reinterpret_cast<const uint32_t *>(src);
            } else {
                vw[0] = *reinterpret_cast<const uint16_t *>(src);
            }
            float vf[C::EPLV];
            Unpack<KVT, C::EPLV>::run(vw, vf);
            float pt[G];
#pragma unroll
            for (int i = 0; i < G; ++i) pt[i] = p_s[t * G + i];
#pragma unroll
            for (int i = 0; i < G; ++i)
#pragma unroll
                for (int e = 0; e < C::EPLV; ++e) acc[i][e] = fmaf(pt[i], vf[e], acc[i][e]);
        };
        if (nvalid == kBlockSize) {
#pragma unroll
            for (int t = 0; t < kBlockSize; ++t) pv_token(t);
        } else {
#pragma unroll 1
            for (int t = 0; t < nvalid; ++t) pv_token(t);
        }
        __syncwarp();
        if (k + NST < nk) issue(k + NST);
    }

    if (timed_out) {
        // let copies still in flight land before the buffers are reused
        if (lane == 0) {
            for (int kk = k > first_issued ? k : first_issued; kk < nk && kk < k + NST; ++kk)
                (void)mbar_wait_bounded(bar0 + 8 * (kk % NST), (kk / NST) & 1, kWaitLimitNs / 16);
        }
        __syncwarp();
    }

    pdl_launch_dependents();

    // ---- merge the warps' partial softmax states ---------------------------
    l_run += __shfl_xor_sync(kFull, l_run, 8);
    l_run += __shfl_xor_sync(kFull, l_run, 16);
    __syncthreads();  // every warp is done with its stage buffers
    float *ms = reinterpret_cast<float *>(smem);
    float *ls = ms + NW * G;
    float *accs = ls + NW * G;
    if (owner && tr == 0) {
        ms[warp * G + my_head] = m_run;
        ls[warp * G + my_head] = l_run;
    }
#pragma unroll
    for (int i = 0; i < G; ++i)
#pragma unroll
        for (int e = 0; e < C::EPLV; ++e) accs[(warp * G + i) * D + lane * C::EPLV + e] = acc[i][e];
    __syncthreads();

    for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
        const int i = idx / D, d = idx - i * D;
        if (group_base + i >= p.group) continue;
        const int64_t hq = (int64_t)kvh * p.group + group_base + i;
        float M = -CUDART_INF_F;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, ms[w * G + i]);
        float O = 0.f, Ls = 0.f;
        if (M != -CUDART_INF_F) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float f = exp2f(ms[w * G + i] - M);
                Ls = fmaf(f, ls[w * G + i], Ls);
                O = fmaf(f, accs[(w * G + i) * D + d], O);
            }
        }
        const float vs = p.v_chan ? p.v_chan[(int64_t)kvh * D + d] : p.v_scale;
        const float o = Ls > 0.f ? (O / Ls) * vs : 0.f;
        const int64_t row = (int64_t)s * p.num_q_heads + hq;
        if (!p.split) {
            reinterpret_cast<uint16_t *>(p.out)[row * D + d] = from_float(QT{}, o);
        } else {
            const int ws_np = p.ws_np > 0 ? p.ws_np : NP, slot = p.ws_offset + part;
            p.ws_o[(row * ws_np + slot) * D + d] = o;
            if (d == 0)
                p.ws_lse[row * ws_np + slot] =
                    Ls > 0.f ? (M + log2f(Ls)) * 0.69314718055994530942f : -CUDART_INF_F;
        }
    }
}

// ---------------------------------------------------------------------------
// split-KV reduce: one CTA of kReduceWarps warps per (sequence, query head).
// Each lane owns D / 32 consecutive elements (one vector load per partition);
// the warps take interleaved partitions, keeping kReduceUnroll partitions'
// loads in flight per lane, and their sums meet in shared memory.  The
// partition weights exp(lse_p - m) come from lse values every lane of the
// warp reads at the same address (one broadcast load), against a running
// maximum m per warp.
// ---------------------------------------------------------------------------

constexpr int kReduceWarps = 4;
constexpr int kReduceUnroll = 8;

template <int V> struct VecF;
template <> struct VecF<4> {
    using T = float4;
    __device__ static void add(float *acc, float w, const T &v) {
        acc[0] = fmaf(w, v.x, acc[0]); acc[1] = fmaf(w, v.y, acc[1]);
        acc[2] = fmaf(w, v.z, acc[2]); acc[3] = fmaf(w, v.w, acc[3]);
    }
};
template <> struct VecF<2> {
    using T = float2;
    __device__ static void add(float *acc, float w, const T &v) {
        acc[0] = fmaf(w, v.x, acc[0]); acc[1] = fmaf(w, v.y, acc[1]);
    }
};

template <typename QT, int D>
__global__ void __launch_bounds__(kReduceWarps * 32) reduce_kernel(const ReduceParams p) {
    constexpr int V = D / 32;  // elements per lane
    using VF = VecF<V>;
    using VT = typename VF::T;
    __shared__ float red[kReduceWarps];
    __shared__ float part_num[kReduceWarps][D];
    __shared__ float part_den[kReduceWarps];
    pdl_wait();
    const int64_t row = blockIdx.x;
    const int s = (int)(row / p.num_q_heads);
    const int NP = p.num_partitions;
    // tokens past token_begin, split into partitions after `extra` leading slots
    int L = p.seq_lens[s] - p.token_begin;
    const int cap = (NP - p.extra) * p.partition_size;
    L = L < 0 ? 0 : (L > cap ? cap : L);
    const int np = p.extra + (L + p.partition_size - 1) / p.partition_size;
    const float *lse = p.ws_lse + row * NP;
    const VT *o = reinterpret_cast<const VT *>(p.ws_o + row * NP * D);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;

    // One pass: each warp keeps a running (m, den, acc) over its partitions,
    // rescaled when a batch brings a larger lse (no separate pass for the
    // maximum); the warps' states meet in shared memory.
    float m = -CUDART_INF_F, den = 0.f;
    float acc[V];
#pragma unroll
    for (int j = 0; j < V; ++j) acc[j] = 0.f;
    auto absorb = [&](float lv, const VT &v) {  // one partition, m already >= lv
        const float w = lv == -CUDART_INF_F ? 0.f : expf(lv - m);
        den += w;
        VF::add(acc, w, v);
    };
    auto rescale_to = [&](float mb) {  // raise m to mb (> m)
        const float sc = m == -CUDART_INF_F ? 0.f : expf(m - mb);
        den *= sc;
#pragma unroll
        for (int j = 0; j < V; ++j) acc[j] *= sc;
        m = mb;
    };
    {
        constexpr int STRIDE = kReduceWarps * kReduceUnroll;
        int i0 = wid;
        for (; i0 + (kReduceUnroll - 1) * kReduceWarps < np; i0 += STRIDE) {
            VT v[kReduceUnroll];
            float lv[kReduceUnroll];
#pragma unroll
            for (int u = 0; u < kReduceUnroll; ++u) {
                const int i = i0 + u * kReduceWarps;
                v[u] = o[(int64_t)i * (D / V) + lane];
                lv[u] = lse[i];
            }
            float mb = lv[0];
#pragma unroll
            for (int u = 1; u < kReduceUnroll; ++u) mb = fmaxf(mb, lv[u]);
            if (mb > m) rescale_to(mb);
#pragma unroll
            for (int u = 0; u < kReduceUnroll; ++u) absorb(lv[u], v[u]);
        }
        for (int i = i0; i < np; i += kReduceWarps) {
            const float lv = lse[i];
            const VT v = o[(int64_t)i * (D / V) + lane];
            if (lv > m) rescale_to(lv);
            absorb(lv, v);
        }
    }
    if (lane == 0) red[wid] = m;
    __syncthreads();
    float M = red[0];
#pragma unroll
    for (int w = 1; w < kReduceWarps; ++w) M = fmaxf(M, red[w]);
    const float sc = m == -CUDART_INF_F ? 0.f : expf(m - M);  // this warp's share at M
#pragma unroll
    for (int j = 0; j < V; ++j) part_num[wid][lane * V + j] = acc[j] * sc;
    if (lane == 0) part_den[wid] = den * sc;
    __syncthreads();
    for (int d = threadIdx.x; d < D; d += kReduceWarps * 32) {
        float num = 0.f, dsum = 0.f;
#pragma unroll
        for (int w = 0; w < kReduceWarps; ++w) {
            num += part_num[w][d];
            dsum += part_den[w];
        }
        const float r = dsum > 0.f ? num / dsum : 0.f;
        reinterpret_cast<uint16_t *>(p.out)[row * D + d] = from_float(QT{}, r);
    }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

template <typename F, typename P>
static cudaError_t launch_pdl(F kern, dim3 grid, dim3 block, int smem, cudaStream_t stream,
                              const P &params) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, params);
}

template <typename QT, typename KVT, int D, int G>
static cudaError_t launch_decode_t(const DecodeParams &p, cudaStream_t stream) {
    using C = DecodeCfg<QT, KVT, D, G>;
    auto kern = decode_kernel<QT, KVT, D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)(p.num_seqs * p.num_partitions), (unsigned)(p.num_kv_heads * p.head_groups));
    return launch_pdl(kern, grid, dim3(C::NW * 32), C::SMEM, stream, p);
}

template <typename QT, typename KVT, int D>
static cudaError_t decode_by_group(const DecodeParams &p, int g, cudaStream_t stream) {
    switch (g) {
        case 1: return launch_decode_t<QT, KVT, D, 1>(p, stream);
        case 2: return launch_decode_t<QT, KVT, D, 2>(p, stream);
        case 4: return launch_decode_t<QT, KVT, D, 4>(p, stream);
        case 8: return launch_decode_t<QT, KVT, D, 8>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <typename QT, typename KVT>
static cudaError_t decode_by_dim(const DecodeParams &p, int d, int g, cudaStream_t stream) {
    if (d == 64) return decode_by_group<QT, KVT, 64>(p, g, stream);
    if (d == 128) return decode_by_group<QT, KVT, 128>(p, g, stream);
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const DecodeParams &p, DType q, DType kv, int head_dim, int tpl_group,
                          cudaStream_t stream) {
    if (p.num_seqs <= 0) return cudaSuccess;
    const bool f16 = q == DType::F16;
    switch (kv) {
        case DType::E4M3:
            return f16 ? decode_by_dim<f16_t, e4m3_t>(p, head_dim, tpl_group, stream)
                       : decode_by_dim<bf16_t, e4m3_t>(p, head_dim, tpl_group, stream);
        case DType::E5M2:
            return f16 ? decode_by_dim<f16_t, e5m2_t>(p, head_dim, tpl_group, stream)
                       : decode_by_dim<bf16_t, e5m2_t>(p, head_dim, tpl_group, stream);
        case DType::I8:
            return f16 ? decode_by_dim<f16_t, i8_t>(p, head_dim, tpl_group, stream)
                       : decode_by_dim<bf16_t, i8_t>(p, head_dim, tpl_group, stream);
        default:
            return f16 ? decode_by_dim<f16_t, f16_t>(p, head_dim, tpl_group, stream)
                       : decode_by_dim<bf16_t, bf16_t>(p, head_dim, tpl_group, stream);
    }
}

cudaError_t launch_reduce(const ReduceParams &p, DType q, int head_dim, cudaStream_t stream) {
    if (p.num_seqs <= 0) return cudaSuccess;
    const dim3 grid((unsigned)((int64_t)p.num_seqs * p.num_q_heads));
    const dim3 block(kReduceWarps * 32);
    if (q == DType::F16) {
        if (head_dim == 64) return launch_pdl(reduce_kernel<f16_t, 64>, grid, block, 0, stream, p);
        return launch_pdl(reduce_kernel<f16_t, 128>, grid, block, 0, stream, p);
    }
    if (head_dim == 64) return launch_pdl(reduce_kernel<bf16_t, 64>, grid, block, 0, stream, p);
    return launch_pdl(reduce_kernel<bf16_t, 128>, grid, block, 0, stream, p);
}

}  // namespace pa
