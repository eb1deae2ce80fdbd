// Paged decode attention on tensor cores (mma.sync m16n8k16, fp32 accumulate)
// with TMA tensor copies of the K/V tiles into 128-byte-swizzled shared memory.
//
// Same operation as pa_decode.cu ("KV Cache 与 PageAttention深度实战", §1.2,
// §3.2-§3.3): per sequence and query head, softmax(q K^T / sqrt(d)) V over the
// 16-token blocks the block table lists.  What changes is where the
// arithmetic runs: the q.K and P.V contractions of a (sequence, KV head)
// group are dense tiles -- [G query heads x 16 tokens x d] -- so they go to the
// tensor cores, leaving the CUDA cores only the softmax.  The per-block cost
// drops from ~1000 warp instructions (CUDA-core dot products, GQA 4) to ~170,
// which keeps the kernel on the HBM roofline up to GQA 16 and for FP8 caches.
//
// Layout of the work:
//   - one CTA per (sequence, partition, KV head, head group of <= 16); 4 warps
//     (2 for long split contexts), each owning every 4th (2nd) 16-token tile of
//     the partition with a private ring of shared-memory stages filled by TMA
//     (cp.async.bulk.tensor.2d, no multicast); for long split contexts with
//     at least as many partitions as resident warps, each warp instead takes
//     whole partitions alone, one after another (CHAINED), and writes each
//     one's partial from its registers;
//   - a tile row is 128 bytes per TMA box (d = 64 16-bit, or half of d = 128
//     16-bit, or d = 128 E4M3) and the box lands 128B-swizzled, so ldmatrix of
//     8 token rows at one 16-byte column touches 8 distinct bank groups;
//   - q.K: S[16 x 16] = Q[16 x d] K^T, M = query heads (zero rows beyond the
//     group), N = the block's tokens, ldmatrix.x4 feeding B;
//   - online softmax on the accumulator fragments (row = head); masked tokens
//     are set to -inf by select;
//   - P.V: O[16 x d] += P[16 x 16] V, P taken straight from the S fragments;
//     ldmatrix.x4.trans feeds V.  For a bf16 cache P is split into bf16 hi + lo
//     (two MMAs), keeping P to ~16 bits; for f16 and E4M3 caches P is f16;
//   - 8-bit tiles (E4M3, E5M2, INT8) are converted to f16 (exact) in
//     registers, two codes per instruction pair; the contraction index d is
//     permuted consistently in q and K so that one ldmatrix word yields both B
//     registers of a k-step.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <cstdlib>
#include <type_traits>

#include "pa_device.cuh"
#include "pa_tmap.h"

namespace pa {

namespace mma_detail {

constexpr unsigned kFull = 0xFFFFFFFFu;

template <typename KVT> struct MmaType;  // element type the tensor cores see
template <> struct MmaType<bf16_t> {
    using T = bf16_t;
};
template <> struct MmaType<f16_t> {
    using T = f16_t;
};
template <> struct MmaType<e4m3_t> {
    using T = f16_t;
};
template <> struct MmaType<e5m2_t> {
    using T = f16_t;
};
template <> struct MmaType<i8_t> {
    using T = f16_t;
};

__device__ __forceinline__ void mma16816(float *c, const uint32_t *a, uint32_t b0, uint32_t b1,
                                         bf16_t) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma16816(float *c, const uint32_t *a, uint32_t b0, uint32_t b1,
                                         f16_t) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// m16n8k32 with A and B in the 8-bit cache format (fp32 accumulate; INT8:
// s32 accumulate, exact)
__device__ __forceinline__ void mma_k32(float *c, const uint32_t *a, uint32_t b0, uint32_t b1,
                                        e4m3_t) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_k32(float *c, const uint32_t *a, uint32_t b0, uint32_t b1,
                                        e5m2_t) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e5m2.e5m2.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_k32(int *c, const uint32_t *a, uint32_t b0, uint32_t b1, i8_t) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t *r, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t *r, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}


template <typename KVT> __device__ __forceinline__ uint32_t cvt8x2_f16x2(uint32_t two) {
    return ::pa::cvt8x2_f16x2(two, KVT{});
}

__device__ __forceinline__ uint32_t prmt2(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}
__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Four 8-bit codes of one word -> two f16x2 (exact).  SEL_LO / SEL_HI name
// the byte pairs: 0x10 / 0x32 for bytes (0,1) / (2,3), 0x20 / 0x31 for the
// interleaved pairs (0,2) / (1,3).
template <typename KVT, uint32_t SEL_LO, uint32_t SEL_HI>
__device__ __forceinline__ void cvt8x4_f16x2(uint32_t w, uint32_t &lo, uint32_t &hi) {
    if constexpr (std::is_same<KVT, i8_t>::value) {
        // the biased byte b ^ 0x80 goes under the f16 exponent byte 0x64
        // (value 1024 + 128 + b); subtracting 1152 leaves b
        const uint32_t x = w ^ 0x80808080u;
        constexpr uint32_t kLo = 0x5040u | ((SEL_LO & 0xFu) | ((SEL_LO >> 4) << 8));
        constexpr uint32_t kHi = 0x5040u | ((SEL_HI & 0xFu) | ((SEL_HI >> 4) << 8));
        lo = hsub2(prmt2(x, 0x6464u, kLo), 0x64806480u);
        hi = hsub2(prmt2(x, 0x6464u, kHi), 0x64806480u);
    } else {
        const uint32_t a = (SEL_LO == 0x10u) ? w : prmt2(w, 0u, 0x3120u);
        cvt8x4_halves(a, lo, hi, KVT{});
    }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi, f16_t) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi, bf16_t) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// 2^x on the MUFU unit (-inf -> +0; results below 2^-126 flush to 0, which
// only drops weights too small to matter next to the row maximum's 1)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(a), "r"(sel));
    return r;
}

// a tensor-map tile copy with an L2 eviction-priority policy (createpolicy):
// the K/V stream is read once, so it goes first when L2 needs room, and the
// split partials the reduce reads back stay resident
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
        : "memory");
}

}  // namespace mma_detail

template <typename QT, typename KVT, int D, int GT, int NW_ = kDecodeWarps> struct MmaCfg {
    using ET = typename mma_detail::MmaType<KVT>::T;
    static constexpr bool FP8 = Elem<KVT>::kBytes == 1;
    static constexpr bool HILO = (Elem<KVT>::kBytes == 2) && sizeof(ET) == 2 &&
                                 std::is_same<KVT, bf16_t>::value;
    static constexpr int NW = NW_;  // warps per CTA
    static constexpr int EB = Elem<KVT>::kBytes;
    static constexpr int ROW_BYTES = D * EB;
    static constexpr int NBOX = ROW_BYTES / 128;  // 128-byte TMA boxes per row
    static constexpr int BOX_ELEMS = 128 / EB;
    static constexpr int BOX_BYTES = kBlockSize * 128;  // 2 KiB
    static constexpr int TILE_BYTES = NBOX * BOX_BYTES;
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
    // Residency.  8-bit tiles (4 KiB a stage) with 8 MMA rows: 3 stages a warp
    // and 16 warps an SM at 128 registers a thread -- the 8-bit path is
    // latency-bound, and 16 warps beat 12 warps with 4 stages (long-context
    // E4M3: 129.7 -> 120.3 us; 10 two-warp CTAs with 2 stages, 126.4 us).
    // Otherwise 16 KiB of stages a warp and 12 warps an SM (16-bit tiles:
    // shared memory bound; 16 MMA rows: their accumulators need the registers).
    static constexpr bool WIDE = FP8 && GT == 8;
    static constexpr int NST = WIDE ? 3 : ((16384 / STAGE_BYTES) < 2 ? 2 : (16384 / STAGE_BYTES));
    static constexpr int MIN_CTAS = (WIDE ? 16 : 12) / NW_;
    static constexpr int KS = D / 16;   // k-steps of q.K (16-bit: m16n8k16; 8-bit: pairs of them
                                        // make one m16n8k32 step)
    // 8-bit caches: q.K runs in the cache's format with q split into QT8
    // terms (term t scaled by 2^(QSH t)); the largest |q| is put at 2^QB
    static constexpr bool INT8 = std::is_same<KVT, i8_t>::value;
    static constexpr bool E5M2 = std::is_same<KVT, e5m2_t>::value;
    static constexpr int QT8 = INT8 ? 2 : ((E5M2 || std::is_same<QT, f16_t>::value) ? 3 : 2);
    static constexpr int QSH = INT8 ? 7 : (E5M2 ? 3 : 4);
    static constexpr int QB = INT8 ? 5 : (E5M2 ? 14 : 7);
    // with 8 MMA rows for 8 heads, A rows 8-15 carry the next q term (rows
    // 0-7 term 2m, rows 8-15 term 2m+1 of MMA m), so the rows the GQA group
    // leaves empty do useful work; 16 heads need one MMA per term
    static constexpr bool PACK8 = GT == 8;
    // the 8-bit q.K path for INT8 caches with groups of up to 8 heads (two
    // terms, packed into one MMA): its widening costs five instructions per
    // four codes, and the integer MMA measured faster (long-context INT8:
    // 117.6 -> 112.4 us).  E4M3 keeps widening K to f16: its two-instruction
    // widening beat the E4M3 MMA (110.1 vs 114.8 us); E5M2, f16-q and 16-row
    // cases would need three terms and run out of registers.
    static constexpr bool K8MMA = INT8 && PACK8;
    static constexpr int NA8 = PACK8 ? (QT8 + 1) / 2 : QT8;  // A-operand sets (MMAs per k32 step)
    static constexpr int MT = D / 16;   // m-tiles (16 rows of d) of O^T = V^T P^T
    static constexpr int NH = GT / 8;   // n-tiles (8 heads) of O^T
    static constexpr int SZ_STAGES = NW * NST * STAGE_BYTES;
    static constexpr int OFF_BAR = SZ_STAGES;
    static constexpr int SMEM = 1024 /* alignment slack */ + OFF_BAR + NW * NST * 8;
    static constexpr int MERGE_BYTES = NW * (GT * D + 2 * GT) * 4;
    static_assert(NBOX >= 1 && ROW_BYTES % 128 == 0, "rows must be whole 128-byte boxes");
    static_assert(MERGE_BYTES <= SZ_STAGES, "merge area must fit in the stage buffers");
    static_assert(GT == 8 || GT == 16, "MMA rows used: 8 or 16");
};

// Byte offset of logical 16-byte chunk `c` of token row `r` inside a tile made
// of 128B-swizzled TMA boxes (box = 16 rows x 128 bytes, 1 KiB aligned).
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return (uint32_t)((c >> 3) * (kBlockSize * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// CHAN: per-channel scales (8-bit caches only), a separate instantiation so
// that the per-tensor kernels compile exactly as without them.  CHAINED: each
// warp attends p.chain consecutive partitions alone (long split contexts).
template <typename QT, typename KVT, int D, int GT, bool CHAN, int NWARPS, bool CHAINED>
__global__ void __launch_bounds__(NWARPS * 32, MmaCfg<QT, KVT, D, GT, NWARPS>::MIN_CTAS)
    decode_mma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_v) {
    using C = MmaCfg<QT, KVT, D, GT, NWARPS>;
    using ET = typename C::ET;
    using namespace mma_detail;
    constexpr int NW = C::NW, NST = C::NST;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base_addr - raw_addr);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, kq = lane & 3;  // MMA fragment coordinates
    const int NP = p.num_partitions;
    // chained (long split contexts): each warp attends p.chain consecutive
    // partitions alone; otherwise the CTA's warps share one partition
    constexpr bool chain = CHAINED;
    const int cps = chain ? (NP + NW * p.chain - 1) / (NW * p.chain) : NP;  // CTAs per sequence
    const int s = blockIdx.x / cps, cta = blockIdx.x - s * cps;
    const int part = chain ? (cta * NW + warp) * p.chain : cta;  // the (first) partition
    const int kvh = blockIdx.y / p.head_groups, hg = blockIdx.y - kvh * p.head_groups;

    const uint32_t bar0 = base_addr + C::OFF_BAR + warp * NST * 8;
    const uint32_t stage0 = base_addr + warp * NST * C::STAGE_BYTES;

    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < NST; ++i) mbar_init(bar0 + 8 * i, 1);
        mbar_init_fence();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_v)) : "memory");
    }
    __syncwarp();

    pdl_wait();

    // ---- the block-table entries of this warp's first 32 tiles, one per lane,
    // read before the sequence length is known (any index inside the table
    // row is readable), so the two loads are in flight together
    const int32_t *bt_row = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
    const int blk_begin = p.tile_begin + part * p.partition_blocks;
    auto tile_of = [&](int k) -> int {  // the warp's k-th 16-token tile
        return chain ? blk_begin + k : blk_begin + warp + NW * k;
    };
    auto table_at = [&](int k) -> int {  // the block holding the warp's tile k
        const int idx = tile_of(k) >> p.tile_shift;
        return (unsigned)idx < (unsigned)p.max_blocks_per_seq ? bt_row[idx] : 0;
    };
    const int bt_first = table_at(lane);

    // ---- sequence length and this CTA's block range -----------------------
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
    const bool len_ok = L == p.seq_lens[s];  // not clamped: the new token's slot is known
    const int nblk_seq = (L + kBlockSize - 1) / kBlockSize;
    if (L < p.tile_begin * kBlockSize) {  // shared-prefix decode: shorter than the prefix
        if (threadIdx.x == 0 && part == 0) flag_error(p.err, kErrBounds);
        L = p.tile_begin * kBlockSize;
    }
    int span = p.partition_blocks;
    if (chain) span *= NP - part < p.chain ? (NP - part > 0 ? NP - part : 0) : p.chain;
    int blk_end = blk_begin + span;
    if (blk_end > nblk_seq) blk_end = nblk_seq;
    if (p.split && blk_begin >= blk_end) return;  // (chained: no CTA barrier follows)
    const int nblk = blk_end > blk_begin ? blk_end - blk_begin : 0;
    const int nk = chain ? nblk : (nblk > warp ? (nblk - warp + NW - 1) / NW : 0);

    // ---- block table entries of this warp, one per lane --------------------
    auto load_batch = [&](int batch) -> int {  // the block holding each of the warp's tiles
        const int k = batch * 32 + lane;
        return k < nk ? table_at(k) : 0;
    };
    const int tile_mask = (1 << p.tile_shift) - 1;
    const uint64_t kv_policy = policy_evict_first();
    int cur_batch = 0;
    int bt_cur = lane < nk ? bt_first : 0;
    int bt_nxt = nk > 32 ? load_batch(1) : 0;
    auto bt_of = [&](int k) -> int {
        const int a = __shfl_sync(kFull, bt_cur, k & 31);
        const int b = __shfl_sync(kFull, bt_nxt, k & 31);
        return (k >> 5) == cur_batch ? a : b;
    };
    auto issue = [&](int k, int st) {  // whole warp calls; lane 0 issues the copies; st = k % NST
        int phys = bt_of(k);
        if (lane == 0) {
            if ((unsigned)phys >= (unsigned)p.num_blocks) {
                flag_error(p.err, kErrBounds);
                phys = 0;  // a valid block whose tokens are all masked
            }
            const uint32_t bar = bar0 + 8 * st;
            const uint32_t dst = stage0 + st * C::STAGE_BYTES;
            const int sub = tile_of(k) & tile_mask;  // tile within the block
            const int y = (phys * p.num_kv_heads + kvh) * p.block_size + sub * kBlockSize;
            mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
#pragma unroll
            for (int b = 0; b < C::NBOX; ++b) {
                tma_load_2d(dst + b * C::BOX_BYTES, &tmap_k, b * C::BOX_ELEMS, y, bar, kv_policy);
                tma_load_2d(dst + C::TILE_BYTES + b * C::BOX_BYTES, &tmap_v, b * C::BOX_ELEMS, y, bar,
                            kv_policy);
            }
        }
    };
    const int npre = nk < NST ? nk : NST;
    const int first_issued = p.hold_first_tile ? 1 : 0;  // test hook: tile 0 never issued
    for (int k = first_issued; k < npre; ++k) issue(k, k);
    const uint64_t wait_limit = p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs;

    // ---- q as MMA A fragments (rows = heads of this group) ----------------
    // 16-bit caches, k-step ks: qa[ks][0]: row g, [1]: row g+8, [2]: row g (k+8),
    // [3]: row g+8 (k+8).  8-bit caches, k32-step jj, term t: q8[t][jj][0]: row g
    // codes k 4kq..4kq+3, [1]: row g+8, [2] / [3]: the same at k + 16.
    uint32_t qa[C::K8MMA ? 1 : C::KS][4];
    uint32_t q8[C::K8MMA ? C::NA8 : 1][C::K8MMA ? C::KS / 2 : 1][4];
    float qscale = p.qk_scale_log2;
    {
        const int group_base = hg * GT;
        const uint16_t *q16 = static_cast<const uint16_t *>(p.q);
        float qv[2][C::KS][4];  // [row half][ks][4 values]
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int row = g + 8 * hh;
            const bool hv = (GT == 16 || hh == 0) && row < GT && group_base + row < p.group;
            const int64_t hq = (int64_t)kvh * p.group + group_base + row;
            const uint16_t *qrow = q16 + ((int64_t)s * p.num_q_heads + (hv ? hq : 0)) * D;
#pragma unroll
            for (int ks = 0; ks < C::KS; ++ks) {
                // physical d of the four values this lane feeds in k-step ks
                int d0, d1, d2, d3;
                if constexpr (C::FP8) {
                    d0 = 16 * ks + 4 * kq; d1 = d0 + 1; d2 = d0 + 2; d3 = d0 + 3;
                } else {
                    d0 = 16 * ks + 2 * kq; d1 = d0 + 1; d2 = d0 + 8; d3 = d0 + 9;
                }
                float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
                if (hv) {
                    const uint32_t w01 = *reinterpret_cast<const uint32_t *>(qrow + d0);
                    const uint32_t w23 = *reinterpret_cast<const uint32_t *>(qrow + d2);
                    unpack2(QT{}, w01, v0, v1);
                    unpack2(QT{}, w23, v2, v3);
                    if constexpr (CHAN) {  // per-channel K scales: q.(code * s) = (q * s).code
                        const float *kc = p.k_chan + (int64_t)kvh * D;
                        v0 *= kc[d0]; v1 *= kc[d1]; v2 *= kc[d2]; v3 *= kc[d3];
                    }
                }
                qv[hh][ks][0] = v0; qv[hh][ks][1] = v1; qv[hh][ks][2] = v2; qv[hh][ks][3] = v3;
            }
        }
        if constexpr (C::FP8 || CHAN) {
            // 8-bit caches (and q times per-channel scales): scale q by a power
            // of two so its largest element sits at 2^QB (8-bit q.K: then split
            // into terms of the cache's format) or at 2^14 (converted to f16),
            // and fold the inverse power into the logit scale (exact).
            float amax = 0.f;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int ks = 0; ks < C::KS; ++ks)
#pragma unroll
                    for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fabsf(qv[hh][ks][i]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
            int e = 0;
            if (amax > 0.f) {
                const int ex = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;  // floor(log2)
                e = (C::K8MMA ? C::QB : 14) - ex;
                if (e > 100) e = 100;
                if (e < -100) e = -100;
            }
            const float up = __uint_as_float((uint32_t)(127 + e) << 23);   // 2^e, exact
            qscale = p.qk_scale_log2 * __uint_as_float((uint32_t)(127 - e) << 23);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int ks = 0; ks < C::KS; ++ks)
#pragma unroll
                    for (int i = 0; i < 4; ++i) qv[hh][ks][i] *= up;
        }
        if constexpr (C::K8MMA) {
            // term t: the codes of the remainder left by the terms before it,
            // times 2^(QSH t): q 2^e = sum_t code_t 2^(-QSH t).  Two terms hold a
            // bf16 q exactly against E4M3 (4 + 4 significant bits) or INT8
            // (integer part + 7 bits); three hold an f16 q, or q against E5M2
            // (3 bits a term).  Elements below 2^(QB - 20) of the largest may
            // lose low bits, an error far below the logits' fp32 rounding.
            constexpr float kUp = (float)(1 << C::QSH);
#pragma unroll
            for (int a = 0; a < C::NA8; ++a)
#pragma unroll
                for (int jj = 0; jj < C::KS / 2; ++jj)
#pragma unroll
                    for (int r = 0; r < 4; ++r) q8[a][jj][r] = 0u;
#pragma unroll
            for (int t = 0; t < C::QT8; ++t) {
#pragma unroll
                for (int jj = 0; jj < C::KS / 2; ++jj) {
#pragma unroll
                    for (int r = 0; r < (C::PACK8 ? 4 : 4); ++r) {
                        // PACK8: rows g only (hh 0), term t in MMA t / 2, rows
                        // g (t even) or g + 8 (t odd); else row g + 8 * hh
                        if (C::PACK8 && (r & 1)) continue;
                        const int hh = r & 1, ks = 2 * jj + (r >> 1);
                        float *v = qv[hh][ks];
                        const uint16_t c01 = code8x2(v[0], v[1], KVT{});
                        const uint16_t c23 = code8x2(v[2], v[3], KVT{});
                        const uint32_t word = (uint32_t)c01 | ((uint32_t)c23 << 16);
                        if constexpr (C::PACK8)
                            q8[t >> 1][jj][r + (t & 1)] = word;
                        else
                            q8[t][jj][r] = word;
                        if (t + 1 < C::QT8) {
                            float d0, d1, d2, d3;
                            unpack2_8<KVT>(c01, d0, d1);
                            unpack2_8<KVT>(c23, d2, d3);
                            v[0] = (v[0] - d0) * kUp;
                            v[1] = (v[1] - d1) * kUp;
                            v[2] = (v[2] - d2) * kUp;
                            v[3] = (v[3] - d3) * kUp;
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int ks = 0; ks < (C::K8MMA ? 0 : C::KS); ++ks) {
            qa[ks][0] = pack2(qv[0][ks][0], qv[0][ks][1], ET{});
            qa[ks][1] = pack2(qv[1][ks][0], qv[1][ks][1], ET{});
            qa[ks][2] = pack2(qv[0][ks][2], qv[0][ks][3], ET{});
            qa[ks][3] = pack2(qv[1][ks][2], qv[1][ks][3], ET{});
        }
    }

    // ---- main loop ------------------------------------------------------------
    constexpr int NR = GT / 8;  // accumulator rows a lane owns: g (and g+8)
    float m_run[NR], l_run[NR];
    // O^T accumulators: o[mt][nh] = rows (d) of m-tile mt x heads 8nh..8nh+7;
    // c0, c1: d-row g, heads 2kq, 2kq+1; c2, c3: d-row g+8, same heads
    float o[C::MT][C::NH][4];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        m_run[r] = -CUDART_INF_F;
        l_run[r] = 0.f;
    }
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
        for (int nh = 0; nh < C::NH; ++nh)
#pragma unroll
            for (int i = 0; i < 4; ++i) o[mt][nh][i] = 0.f;

    // per-lane ldmatrix row / chunk selectors
    const int lrow_b = (lane & 7) + 8 * (lane >> 4);   // q.K: tokens 0-7 | 8-15
    const int lsel_b = (lane >> 3) & 1;                 // q.K: chunk +0 | +1
    const int lrow_v = (lane & 7) + 8 * ((lane >> 3) & 1);  // P.V: tokens 0-7 | 8-15
    const int lsel_v = lane >> 4;                       // P.V: chunk +0 | +1
    // chained: partition pp's partial (lse, o / l) straight from the
    // registers, then a fresh softmax state for the next partition
    auto flush = [&](int pp) {
        const int ws_np = p.ws_np > 0 ? p.ws_np : NP, slot = p.ws_offset + pp;
        const int group_base = hg * GT;
        const int64_t row0 = (int64_t)s * p.num_q_heads + (int64_t)kvh * p.group + group_base;
        float lq[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            lq[r] = l_run[r] + __shfl_xor_sync(kFull, l_run[r], 1);
            lq[r] += __shfl_xor_sync(kFull, lq[r], 2);
        }
        if (kq == 0) {
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                const int head = g + 8 * r;
                if (group_base + head < p.group)
                    p.ws_lse[(row0 + head) * ws_np + slot] =
                        lq[r] > 0.f ? (m_run[r] + log2f(lq[r])) * 0.69314718055994530942f : -CUDART_INF_F;
            }
        }
#pragma unroll
        for (int nh = 0; nh < C::NH; ++nh) {
            // the O^T columns of this lane: heads ha = 8 nh + 2 kq and ha + 1,
            // whose sums sit in the lanes with that softmax row
            const int ha = 8 * nh + 2 * kq;
            const float la = __shfl_sync(kFull, lq[nh], (2 * kq) * 4);
            const float lb = __shfl_sync(kFull, lq[nh], (2 * kq + 1) * 4);
            const float ia = la > 0.f ? 1.f / la : 0.f, ib = lb > 0.f ? 1.f / lb : 0.f;
            const bool va = group_base + ha < p.group, vb = group_base + ha + 1 < p.group;
            float *oa = p.ws_o + ((row0 + ha) * ws_np + slot) * D;
            float *ob = oa + (int64_t)ws_np * D;
#pragma unroll
            for (int mt = 0; mt < C::MT; ++mt) {
                if constexpr (C::FP8) {  // d-rows 2g, 2g + 1 of m-tile mt
                    const int d0 = 16 * mt + 2 * g;
                    float s0 = p.v_scale, s1 = p.v_scale;
                    if constexpr (CHAN) {
                        s0 = p.v_chan[(int64_t)kvh * D + d0];
                        s1 = p.v_chan[(int64_t)kvh * D + d0 + 1];
                    }
                    if (va) *reinterpret_cast<float2 *>(oa + d0) = make_float2(o[mt][nh][0] * ia * s0, o[mt][nh][2] * ia * s1);
                    if (vb) *reinterpret_cast<float2 *>(ob + d0) = make_float2(o[mt][nh][1] * ib * s0, o[mt][nh][3] * ib * s1);
                } else {  // d-rows g, g + 8
                    const int d0 = 16 * mt + g;
                    if (va) {
                        oa[d0] = o[mt][nh][0] * ia * p.v_scale;
                        oa[d0 + 8] = o[mt][nh][2] * ia * p.v_scale;
                    }
                    if (vb) {
                        ob[d0] = o[mt][nh][1] * ib * p.v_scale;
                        ob[d0 + 8] = o[mt][nh][3] * ib * p.v_scale;
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            m_run[r] = -CUDART_INF_F;
            l_run[r] = 0.f;
        }
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
            for (int nh = 0; nh < C::NH; ++nh)
#pragma unroll
                for (int i = 0; i < 4; ++i) o[mt][nh][i] = 0.f;
    };

    bool timed_out = false;
    int k = 0;
    int st = 0;          // k % NST
    uint32_t phase = 0;  // (k / NST) & 1

    for (; k < nk; ++k) {
        if (k > 0 && (k & 31) == 0) {
            bt_cur = bt_nxt;
            ++cur_batch;
            bt_nxt = nk > (cur_batch + 1) * 32 ? load_batch(cur_batch + 1) : 0;
        }
        const bool ok = __all_sync(kFull, mbar_wait_bounded(bar0 + 8 * st, phase, wait_limit));
        if (!ok) {
            if (lane == 0) flag_error(p.err, kErrTimeout);
            timed_out = true;
            break;
        }
        const int j = tile_of(k);
        const bool valid = (unsigned)bt_of(k) < (unsigned)p.num_blocks;
        int nvalid = L - j * kBlockSize;
        nvalid = valid ? (nvalid < kBlockSize ? nvalid : kBlockSize) : 0;
        const uint32_t kt = stage0 + st * C::STAGE_BYTES;
        const uint32_t vt = kt + C::TILE_BYTES;

        // append: the warp holding the sequence's last block writes this step's
        // new token (position L - 1) into its landed tile and, once per KV head,
        // into the pool -- the slot mapping and cache write of the step fused
        // here.  8-bit codes come from the same quantiser as pa_cache_write.
        if (p.append && len_ok && valid && j == (L - 1) / kBlockSize) {
            const int r = (L - 1) & (kBlockSize - 1);
            const int64_t phys = bt_of(k);
            constexpr int CPR = C::ROW_BYTES / 16;        // 16-byte chunks per tile row
            constexpr int SRC_ELEMS = C::FP8 ? 16 : 8;    // activations per chunk
            const int64_t src_row = ((int64_t)s * p.num_kv_heads + kvh) * D;
            const int64_t dst_row =
                ((phys * p.num_kv_heads + kvh) * p.block_size + (L - 1) % p.block_size) * C::ROW_BYTES;
            for (int c = lane; c < 2 * CPR; c += 32) {
                const bool isv = c >= CPR;
                const int cc = isv ? c - CPR : c;
                const uint16_t *src =
                    static_cast<const uint16_t *>(isv ? p.v_new : p.k_new) + src_row + cc * SRC_ELEMS;
                uint4 val;
                if constexpr (C::FP8) {
                    const float sc = isv ? p.v_scale_w : p.k_scale_w;
                    const uint2 lo = quantise8<QT, KVT>(*reinterpret_cast<const uint4 *>(src), sc);
                    const uint2 hi = quantise8<QT, KVT>(*reinterpret_cast<const uint4 *>(src + 8), sc);
                    val = make_uint4(lo.x, lo.y, hi.x, hi.y);
                } else {
                    val = *reinterpret_cast<const uint4 *>(src);
                }
                const uint32_t dst = (isv ? vt : kt) + swz(r, cc);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(val.x),
                             "r"(val.y), "r"(val.z), "r"(val.w)
                             : "memory");
                if (hg == 0)
                    *reinterpret_cast<uint4 *>((isv ? p.v_pool_w : p.k_pool_w) + dst_row + cc * 16) = val;
            }
            // these generic writes precede the next TMA write into this stage
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
        }

        // S = Q K^T for the block's 16 tokens (two n-tiles of 8)
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        if constexpr (!C::FP8) {
#pragma unroll
            for (int ks = 0; ks < C::KS; ++ks) {
                uint32_t b[4];
                ldsm_x4(b, kt + swz(lrow_b, 2 * ks + lsel_b));
                mma16816(sc[0], qa[ks], b[0], b[1], ET{});
                mma16816(sc[1], qa[ks], b[2], b[3], ET{});
            }
        } else if constexpr (!C::K8MMA) {
            // 8-bit codes widened to f16 (exact), d permuted consistently in q
#pragma unroll
            for (int jj = 0; jj < C::KS / 2; ++jj) {
                uint32_t w[4];  // (nt0, ks=2jj), (nt0, 2jj+1), (nt1, 2jj), (nt1, 2jj+1)
                ldsm_x4(w, kt + swz(lrow_b, 2 * jj + lsel_b));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int ks = 2 * jj + h;
                    uint32_t b0, b1, b2, b3;
                    cvt8x4_f16x2<KVT, 0x10u, 0x32u>(w[h], b0, b1);
                    cvt8x4_f16x2<KVT, 0x10u, 0x32u>(w[2 + h], b2, b3);
                    mma16816(sc[0], qa[ks], b0, b1, ET{});
                    mma16816(sc[1], qa[ks], b2, b3, ET{});
                }
            }
        } else {
            // the K codes feed the 8-bit MMA as they landed: an ldmatrix row is
            // 16 codes of one token, so each lane's word holds the 4 codes of
            // k 4kq..4kq+3 that the m16n8k32 B fragment wants
            using AccT = typename std::conditional<C::INT8, int, float>::type;
            AccT acc[C::NA8][2][4];
#pragma unroll
            for (int a = 0; a < C::NA8; ++a)
#pragma unroll
                for (int n = 0; n < 2; ++n)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[a][n][i] = 0;
#pragma unroll
            for (int jj = 0; jj < C::KS / 2; ++jj) {
                uint32_t w[4];  // (tokens 0-7, k 0-15), (0-7, k 16-31), (8-15, k 0-15), (8-15, k 16-31)
                ldsm_x4(w, kt + swz(lrow_b, 2 * jj + lsel_b));
#pragma unroll
                for (int a = 0; a < C::NA8; ++a) {
                    mma_k32(acc[a][0], q8[a][jj], w[0], w[1], KVT{});
                    mma_k32(acc[a][1], q8[a][jj], w[2], w[3], KVT{});
                }
            }
            // S = sum_t 2^(-QSH t) (term t . K); term t of row i sits in
            // acc[t / 2][n][i + 2 (t & 1)] (PACK8) or acc[t][n][i]
            constexpr float kDown = 1.f / (float)(1 << C::QSH);
            auto term = [&](int t, int n, int i) -> float {
                return C::PACK8 ? (float)acc[t >> 1][n][i + 2 * (t & 1)] : (float)acc[t][n][i];
            };
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int i = 0; i < (C::PACK8 ? 2 : 4); ++i) {
                    float v = term(C::QT8 - 1, n, i);
#pragma unroll
                    for (int t = C::QT8 - 2; t >= 0; --t) v = fmaf(v, kDown, term(t, n, i));
                    sc[n][i] = v;
                }
        }

        // online softmax; lane holds S[row g (+8)][tokens 2kq, 2kq+1, 8+2kq, 9+2kq]
        const int t0 = 2 * kq;
        float alpha[NR];
        float pr[NR][4];
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            float sv[4];
            sv[0] = t0 < nvalid ? sc[0][2 * r] * qscale : -CUDART_INF_F;
            sv[1] = t0 + 1 < nvalid ? sc[0][2 * r + 1] * qscale : -CUDART_INF_F;
            sv[2] = t0 + 8 < nvalid ? sc[1][2 * r] * qscale : -CUDART_INF_F;
            sv[3] = t0 + 9 < nvalid ? sc[1][2 * r + 1] * qscale : -CUDART_INF_F;
            float bm = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
            bm = fmaxf(bm, __shfl_xor_sync(kFull, bm, 1));
            bm = fmaxf(bm, __shfl_xor_sync(kFull, bm, 2));
            const float m_new = fmaxf(m_run[r], bm);
            alpha[r] = 1.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) pr[r][i] = 0.f;
            if (m_new != -CUDART_INF_F) {
                alpha[r] = ex2(m_run[r] - m_new);
#pragma unroll
                for (int i = 0; i < 4; ++i) pr[r][i] = ex2(sv[i] - m_new);
            }
            l_run[r] = l_run[r] * alpha[r] + ((pr[r][0] + pr[r][1]) + (pr[r][2] + pr[r][3]));
            m_run[r] = m_new;
        }
        // the O^T columns this lane holds are heads 8nh + 2kq (+1); their
        // rescale factors live in the lanes whose softmax row is that head
#pragma unroll
        for (int nh = 0; nh < C::NH; ++nh) {
            const float a0 = __shfl_sync(kFull, alpha[nh], (2 * kq) * 4);
            const float a1 = __shfl_sync(kFull, alpha[nh], (2 * kq + 1) * 4);
#pragma unroll
            for (int mt = 0; mt < C::MT; ++mt) {
                o[mt][nh][0] *= a0;
                o[mt][nh][1] *= a1;
                o[mt][nh][2] *= a0;
                o[mt][nh][3] *= a1;
            }
        }

        // P as B fragments of O^T = V^T P^T (k = tokens, n = heads): the S
        // accumulators already sit in that layout -- b0 = tokens 2kq, 2kq+1,
        // b1 = tokens 8+2kq, 9+2kq of head (8nh + g).  bf16 caches get a hi
        // and a lo part.
        uint32_t pb_hi[C::NH][2], pb_lo[C::NH][2];
#pragma unroll
        for (int nh = 0; nh < C::NH; ++nh) {
            pb_hi[nh][0] = pack2(pr[nh][0], pr[nh][1], ET{});
            pb_hi[nh][1] = pack2(pr[nh][2], pr[nh][3], ET{});
            if constexpr (C::HILO) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const float h0 = __uint_as_float(pb_hi[nh][i] << 16);
                    const float h1 = __uint_as_float(pb_hi[nh][i] & 0xFFFF0000u);
                    pb_lo[nh][i] = pack2(pr[nh][2 * i] - h0, pr[nh][2 * i + 1] - h1, ET{});
                }
            }
        }

        // O^T += V^T P^T; tokens past nvalid have p = 0 but their V rows may
        // hold NaN poison (0 * NaN = NaN): zero those V fragments first.
        // A fragment of V^T: a0 = (d-row g, tokens 2kq, 2kq+1), a1 = (d-row g+8,
        // same tokens), a2 / a3 = the same d-rows, tokens 8+2kq, 9+2kq.
        const bool full = nvalid == kBlockSize;
        const bool tv0 = t0 < nvalid, tv1 = t0 + 1 < nvalid, tv8 = t0 + 8 < nvalid, tv9 = t0 + 9 < nvalid;
        const uint32_t m0 = (tv0 ? 0x0000FFFFu : 0u) | (tv1 ? 0xFFFF0000u : 0u);
        const uint32_t m8 = (tv8 ? 0x0000FFFFu : 0u) | (tv9 ? 0xFFFF0000u : 0u);
        if constexpr (!C::FP8) {
            // m-tile mt = d rows 16mt..16mt+15: ldmatrix.x4.trans of tokens
            // 0-7 / 8-15 at chunks 2mt (d-rows 0-7) and 2mt+1 (d-rows 8-15)
#pragma unroll
            for (int mt = 0; mt < C::MT; ++mt) {
                uint32_t a[4];  // r0: tok 0-7 chunk 2mt, r1: tok 0-7 chunk 2mt+1, r2/r3: tok 8-15
                ldsm_x4_t(a, vt + swz(lrow_b, 2 * mt + lsel_b));
                uint32_t av[4] = {a[0], a[1], a[2], a[3]};
                if (!full) {
                    av[0] &= m0; av[1] &= m0; av[2] &= m8; av[3] &= m8;
                }
#pragma unroll
                for (int nh = 0; nh < C::NH; ++nh) {
                    mma16816(o[mt][nh], av, pb_hi[nh][0], pb_hi[nh][1], ET{});
                    if constexpr (C::HILO) mma16816(o[mt][nh], av, pb_lo[nh][0], pb_lo[nh][1], ET{});
                }
            }
        } else {
            // m-tile mt = the 16 d of chunk mt: rows g / g+8 hold d = 16mt+2g
            // and 16mt+2g+1 (byte regroup after the transposing load)
#pragma unroll
            for (int cp = 0; cp < C::MT / 2; ++cp) {
                uint32_t w[4];  // chunk 2cp: tok 0-7, tok 8-15; chunk 2cp+1: tok 0-7, tok 8-15
                ldsm_x4_t(w, vt + swz(lrow_v, 2 * cp + lsel_v));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    // regroup bytes: (tok 2kq, 2kq+1) at even d, then at odd d
                    uint32_t av[4];
                    cvt8x4_f16x2<KVT, 0x20u, 0x31u>(w[2 * h], av[0], av[1]);      // tokens 0-7
                    cvt8x4_f16x2<KVT, 0x20u, 0x31u>(w[2 * h + 1], av[2], av[3]);  // tokens 8-15
                    if (!full) {
                        av[0] &= m0; av[1] &= m0; av[2] &= m8; av[3] &= m8;
                    }
                    const int mt = 2 * cp + h;
#pragma unroll
                    for (int nh = 0; nh < C::NH; ++nh) mma16816(o[mt][nh], av, pb_hi[nh][0], pb_hi[nh][1], ET{});
                }
            }
        }
        __syncwarp();
        if (k + NST < nk) issue(k + NST, st);
        if (++st == NST) {
            st = 0;
            phase ^= 1u;
        }
        if constexpr (CHAINED) {
            if ((k + 1) % p.partition_blocks == 0 || k + 1 == nk) flush(part + k / p.partition_blocks);
        }
    }

    if (timed_out) {
        if (lane == 0) {
            for (int kk = k > first_issued ? k : first_issued; kk < nk && kk < k + NST; ++kk)
                (void)mbar_wait_bounded(bar0 + 8 * (kk % NST), (kk / NST) & 1, kWaitLimitNs / 16);
        }
        __syncwarp();
    }

    pdl_launch_dependents();
    if constexpr (CHAINED) return;  // every partition's partial is written

    // ---- merge the warps' partial states ---------------------------------------
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        l_run[r] += __shfl_xor_sync(kFull, l_run[r], 1);
        l_run[r] += __shfl_xor_sync(kFull, l_run[r], 2);
    }
    __syncthreads();
    float *ms = reinterpret_cast<float *>(smem);
    float *ls = ms + NW * GT;
    float *accs = ls + NW * GT;
    if (kq == 0) {
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            ms[warp * GT + g + 8 * r] = m_run[r];
            ls[warp * GT + g + 8 * r] = l_run[r];
        }
    }
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) {
#pragma unroll
        for (int nh = 0; nh < C::NH; ++nh) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int head = 8 * nh + 2 * kq + (i & 1);
                const int hi_row = i >> 1;  // 0: d-row g, 1: d-row g+8
                int d;
                if constexpr (C::FP8) {
                    d = 16 * mt + 2 * g + hi_row;
                } else {
                    d = 16 * mt + 8 * hi_row + g;
                }
                accs[(warp * GT + head) * D + d] = o[mt][nh][i];
            }
        }
    }
    __syncthreads();

    const int group_base = hg * GT;
    for (int idx = threadIdx.x; idx < GT * D; idx += NW * 32) {
        const int i = idx / D, d = idx - i * D;
        if (group_base + i >= p.group) continue;
        const int64_t hq = (int64_t)kvh * p.group + group_base + i;
        float M = -CUDART_INF_F;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, ms[w * GT + i]);
        float O = 0.f, Ls = 0.f;
        if (M != -CUDART_INF_F) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float f = exp2f(ms[w * GT + i] - M);
                Ls = fmaf(f, ls[w * GT + i], Ls);
                O = fmaf(f, accs[(w * GT + i) * D + d], O);
            }
        }
        float vs = p.v_scale;
        if constexpr (CHAN) vs = p.v_chan[(int64_t)kvh * D + d];
        const float ov = Ls > 0.f ? (O / Ls) * vs : 0.f;
        const int64_t row = (int64_t)s * p.num_q_heads + hq;
        if (!p.split) {
            reinterpret_cast<uint16_t *>(p.out)[row * D + d] = from_float(QT{}, ov);
        } else {
            const int ws_np = p.ws_np > 0 ? p.ws_np : NP, slot = p.ws_offset + part;
            p.ws_o[(row * ws_np + slot) * D + d] = ov;
            if (d == 0)
                p.ws_lse[row * ws_np + slot] =
                    Ls > 0.f ? (M + log2f(Ls)) * 0.69314718055994530942f : -CUDART_INF_F;
        }
    }
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launch
// ---------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    // looked up once; a function-local static is initialised exactly once
    // even when several host threads make their first call together
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        return nullptr;
    }();
    return fn;
}

// 2-D view of a pool [NB, Hk, 16, d]: rows = NB * Hk * 16 tokens, d columns;
// boxes of 16 rows x 128 bytes, 128-byte swizzle.
bool encode_pool_map(CUtensorMap *m, const void *base, int elem_bytes, int d, int64_t rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)d * (cuuint64_t)elem_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)(128 / elem_bytes), (cuuint32_t)kBlockSize};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16,
                          2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {

template <typename QT, typename KVT, int D, int GT, bool CHAN, int NWARPS, bool CHAINED>
cudaError_t launch_mma_t(const DecodeParams &p, cudaStream_t stream) {
    using C = MmaCfg<QT, KVT, D, GT, NWARPS>;
    const int64_t rows = (int64_t)p.num_blocks * p.num_kv_heads * p.block_size;
    CUtensorMap mk, mv;
    if (!encode_pool_map(&mk, p.k_cache, C::EB, D, rows) ||
        !encode_pool_map(&mv, p.v_cache, C::EB, D, rows))
        return cudaErrorInvalidValue;
    auto kern = decode_mma_kernel<QT, KVT, D, GT, CHAN, NWARPS, CHAINED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    if (CHAINED != (p.chain > 0)) return cudaErrorInvalidValue;
    const int cps = CHAINED ? (p.num_partitions + C::NW * p.chain - 1) / (C::NW * p.chain) : p.num_partitions;
    cfg.gridDim = dim3((unsigned)(p.num_seqs * cps), (unsigned)(p.num_kv_heads * p.head_groups));
    cfg.blockDim = dim3(C::NW * 32);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p, mk, mv);
}

// Warps per CTA.  Four warps share a partition's tiles and merge their
// softmax states; with many partitions per sequence (long contexts) two warps
// per CTA do better: half the per-CTA q preparation and merge work for the
// same warps per SM (long-context E4M3 shape, 512-token partitions, 12 warps
// an SM: 146.6 -> 130.1 us), while for shorter, uneven sequences the smaller
// work units of four warps balance better over the SMs (Qwen3-8B shape: 105.2
// vs 111.9 us).
constexpr int kLongSplitPartitions = 16;

// Long split contexts: with at least as many partitions as the device holds
// resident warps, each warp attends floor(partitions / resident warps) (at
// most 4) consecutive partitions alone (DecodeParams::chain): no merge of
// warps' states within a CTA, and the partials written straight from
// registers (long-context E4M3 shape, 4096 partitions of 512 tokens over
// 2368 resident warps: 109.8 us with two warps sharing each partition, 100.4
// with one warp a partition, 108.4 with two partitions a warp).  With fewer
// partitions (0 here) a CTA's two warps share each one, so that every
// resident warp has work.  The environment variable PA369_DECODE_CHAIN (a
// count, 1 .. 64) overrides the choice; it is kept for A/B measurement and
// tests.
template <typename C> int chain_length(const DecodeParams &p) {
    if (const char *env = getenv("PA369_DECODE_CHAIN")) {
        const int r = atoi(env);
        if (r > 0) return r < 64 ? r : 64;
    }
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = 148;
    const int64_t slots = (int64_t)sms * C::MIN_CTAS * C::NW;  // resident warps
    const int64_t parts = (int64_t)p.num_seqs * p.num_partitions * p.num_kv_heads * p.head_groups;
    const int64_t r = parts / slots;
    return (int)(r > 4 ? 4 : r);
}

template <typename QT, typename KVT, int D, bool CHAN>
cudaError_t mma_by_warps(const DecodeParams &p, int gt, cudaStream_t stream) {
    if (p.split && p.num_partitions >= kLongSplitPartitions) {
        DecodeParams q = p;
        if (gt == 16) {
            q.chain = chain_length<MmaCfg<QT, KVT, D, 16, 2>>(p);
            return q.chain > 0 ? launch_mma_t<QT, KVT, D, 16, CHAN, 2, true>(q, stream)
                               : launch_mma_t<QT, KVT, D, 16, CHAN, 2, false>(q, stream);
        }
        q.chain = chain_length<MmaCfg<QT, KVT, D, 8, 2>>(p);
        return q.chain > 0 ? launch_mma_t<QT, KVT, D, 8, CHAN, 2, true>(q, stream)
                           : launch_mma_t<QT, KVT, D, 8, CHAN, 2, false>(q, stream);
    }
    DecodeParams q = p;
    q.chain = 0;
    return gt == 16 ? launch_mma_t<QT, KVT, D, 16, CHAN, kDecodeWarps, false>(q, stream)
                    : launch_mma_t<QT, KVT, D, 8, CHAN, kDecodeWarps, false>(q, stream);
}

template <typename QT, typename KVT, int D>
cudaError_t mma_by_rows(const DecodeParams &p, int gt, cudaStream_t stream) {
    if constexpr (Elem<KVT>::kBytes == 1) {
        if (p.k_chan) return mma_by_warps<QT, KVT, D, true>(p, gt, stream);
    }
    return mma_by_warps<QT, KVT, D, false>(p, gt, stream);
}

}  // namespace

bool mma_decode_supported(DType kv, int head_dim, int num_blocks, int num_kv_heads, int block_size) {
    if (!encode_fn()) return false;
    const int64_t rows = (int64_t)num_blocks * num_kv_heads * block_size;
    if (rows >= (int64_t(1) << 31)) return false;  // TMA row coordinate is a signed 32-bit int
    if (is_8bit(kv)) return head_dim == 128;
    return head_dim == 64 || head_dim == 128;
}

cudaError_t launch_decode_mma(const DecodeParams &p, DType q, DType kv, int head_dim, int mma_rows,
                              cudaStream_t stream) {
    if (p.num_seqs <= 0) return cudaSuccess;
    if (is_8bit(kv)) {
        if (head_dim != 128) return cudaErrorInvalidValue;
        const bool f16 = q == DType::F16;
        if (kv == DType::E4M3)
            return f16 ? mma_by_rows<f16_t, e4m3_t, 128>(p, mma_rows, stream)
                       : mma_by_rows<bf16_t, e4m3_t, 128>(p, mma_rows, stream);
        if (kv == DType::E5M2)
            return f16 ? mma_by_rows<f16_t, e5m2_t, 128>(p, mma_rows, stream)
                       : mma_by_rows<bf16_t, e5m2_t, 128>(p, mma_rows, stream);
        return f16 ? mma_by_rows<f16_t, i8_t, 128>(p, mma_rows, stream)
                   : mma_by_rows<bf16_t, i8_t, 128>(p, mma_rows, stream);
    }
    if (q == DType::F16)
        return head_dim == 64 ? mma_by_rows<f16_t, f16_t, 64>(p, mma_rows, stream)
                              : mma_by_rows<f16_t, f16_t, 128>(p, mma_rows, stream);
    return head_dim == 64 ? mma_by_rows<bf16_t, bf16_t, 64>(p, mma_rows, stream)
                          : mma_by_rows<bf16_t, bf16_t, 128>(p, mma_rows, stream);
}

}  // namespace pa
