// Chunked-prefill attention over the paged KV cache on the fifth-generation
// tensor cores: tcgen05.mma with accumulators in tensor memory (TMEM),
// operands staged in shared memory by TMA.
//
// What it computes ("openeuler.csdn.net 推理优化篇", §4.5 Chunked Prefill;
// "vLLM推理引擎深度解析：PagedAttention与连续批处理", §3.3): a long prompt is cut
// into chunks (the pages' example: 512 tokens); each chunk's K/V rows are
// appended to the cache (pa_slot_mapping + pa_cache_write) and its query
// tokens then attend causally over everything cached so far,
//   out[j][h] = softmax_t(scale * q[j][h] . K_t) V_t,   t <= L - n + j,
// K_t / V_t read through the sequence's block table ("Transformer 推理优化：
// KV Cache、PagedAttention 与 vLLM", §3.3).  A decode step is the one-token
// chunk.
//
// Work decomposition: a work item is (pair of query tiles, KV head,
// sequence).  A query tile is 128 rows = floor(128 / g) chunk tokens x the g
// query heads of the KV head (row r: token r / g, head r % g), so the whole
// GQA group shares each K/V tile it reads; the item's two tiles (A, B:
// consecutive token ranges) share them too.  Keys come in tiles of 64 = 4
// blocks of 16 tokens.  The launch is persistent: one CTA an SM takes items
// from a device counter until none are left, and every role below runs the
// items in the same order with its barrier phases continuing from item to
// item, so one item's first loads and MMAs overlap the previous one's last.
//   - warp 8, TMA producer: takes the items and passes them on; per item both
//     Q tiles through a 3-D tensor map over q [T, Hq, d], and per key tile the
//     4 K and 4 V blocks named by the block table through the pool's 2-D map
//     (16-row x 128-byte boxes, 128B swizzle; one copy per lane) into a
//     4-stage ring.  Blocks past the sequence's end are fetched from past the
//     end of the map, which the copy fills with zeros.
//   - warps 9 (tile A) and 10 (tile B; 12 for 8-bit caches), MMA issuers, one
//     lane each: S_t = Q_t K_j^T (M 128, N 64, K d) into one of tile t's two
//     TMEM score buffers; O_t += P_t V_j with A = P read from TMEM and B = V
//     from shared memory (MN-major).  Issue order per key tile j: PV_t(j),
//     QK_t(j+2) -- the tile's next scores are ready before its softmax
//     finishes, and while one issuer waits for its softmax the other keeps the
//     tensor core busy; tcgen05 operations of one thread run in issue order,
//     which makes reusing a score buffer's columns for P and then for the
//     scores two tiles later safe.
//   - warps 0-3 (tile A) and 4-7 (tile B), one thread per row: S from TMEM,
//     causal mask by select on the diagonal tile only, the scale folded into
//     one FFMA before ex2, online softmax with a lazy rescale (O and l are
//     rescaled only when the row max grows by more than 8 in log2 units;
//     otherwise p is taken against the old max, at most 2^8), P written back
//     over S (bf16 as hi + lo halves so P keeps ~16 bits; f16 as one half),
//     O / l at the end.
//   - 8-bit caches (E4M3 / E5M2 / INT8, per-tensor scales, d = 128): the
//     copies land in a staging ring; warp 10 widens Q (bf16 to f16 times a
//     power of two) and each K tile, warp 11 each V tile, to f16 in the
//     operand layout, so the MMAs run f16 x f16 (each code is exact in f16).
// Shared-prefix mode (pa_decode_shared_prefix): the rows are the decoding
// sequences' queries, every one of them sees all prefix keys (no mask), and
// the prefix's key tiles are cut into items_z ranges, each writing its own
// partial (lse, o) workspace slot for the reduce to merge.
// V rows past the sequence's last token (the tail of its last block) are
// cleared in shared memory before P.V: p = 0 there, but 0 x NaN poison = NaN.
// Every wait is bounded; a timeout reports PA_ERR_DEVICE_TIMEOUT, makes the
// other roles give up, drains the copies and MMAs in flight and frees TMEM.
#include <cuda.h>
#include <math_constants.h>

#include <atomic>
#include <cstdlib>
#include <cstdint>
#include <type_traits>

#include "pa_device.cuh"
#include "pa_shared_prefix.h"
#include "pa_tmap.h"

namespace pa {

namespace tc {

constexpr unsigned kFull = 0xFFFFFFFFu;

// Shared-memory matrix descriptor (sm_100 form): start, leading / stride
// byte offsets (16-byte units), version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// D[tmem] (+)= A[smem] B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

// D[tmem] (+)= A[tmem] B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
        "r"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

// arrive on `bar` once every tcgen05 operation this thread issued is done
__device__ __forceinline__ void commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

__device__ __forceinline__ void fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void alloc(uint32_t slot_addr, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_addr),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// 32 consecutive 32-bit columns of this thread's TMEM lane
__device__ __forceinline__ void ld32(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
// Wait for this thread's TMEM loads; the empty asm per register makes every
// later use of the loaded values come after the wait.
template <int N> __device__ __forceinline__ void wait_ld(uint32_t *r) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

__device__ __forceinline__ void st16(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void st32(uint32_t taddr, const uint32_t *r) {
    st16(taddr, r);
    st16(taddr + 16, r + 16);
}
__device__ __forceinline__ void wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
        "{%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            int z, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
        "{%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

// Four 8-bit codes of one word -> two f16x2 (codes 0,1 in lo; 2,3 in hi), exact.
template <typename KT>
__device__ __forceinline__ void widen4(uint32_t w, uint32_t &lo, uint32_t &hi, KT) {
    cvt8x4_halves(w, lo, hi, KT{});
}
// INT8, a word at a time: one bias flip (b ^ 0x80 = b + 128) for the four
// bytes, each pair under the f16 exponent byte 0x64 (value 1024 + 128 + b),
// then 1152 subtracted from both halves.
__device__ __forceinline__ void widen4(uint32_t w, uint32_t &lo, uint32_t &hi, i8_t) {
    const uint32_t x = w ^ 0x80808080u;
    uint32_t a, b;
    asm("prmt.b32 %0, %1, %2, 0x5140;" : "=r"(a) : "r"(x), "r"(0x6464u));
    asm("prmt.b32 %0, %1, %2, 0x5342;" : "=r"(b) : "r"(x), "r"(0x6464u));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(lo) : "r"(a), "r"(0x64806480u));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(hi) : "r"(b), "r"(0x64806480u));
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Bounded wait on an mbarrier phase that also gives up when another role of
// the CTA has already given up (abort flag); the thread that runs out of
// time raises the flag and reports the timeout.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                           int *err, uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            flag_error(err, kErrTimeout);
            return false;
        }
    }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi, bf16_t) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi, f16_t) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ void unpack2(uint32_t w, float &lo, float &hi, bf16_t) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
}

}  // namespace tc

// Work items are taken longest first where that is cheap to know: with up to
// kOrderSeqs sequences the TMA warp ranks them by cached context (the chunks
// of one launch are alike) and hands out, per sequence in that order, its
// query tile pairs last first (they see the most keys); the item index it
// publishes is the natural one below.
constexpr int kOrderSeqs = 128;

// T: q / out dtype; KVT: cache dtype (T, or an 8-bit code for which two
// converter warps widen each landed K and V tile to f16 in shared memory).
template <typename T, int D, typename KVT = T> struct PfCfg {
    static constexpr bool KV8 = Elem<KVT>::kBytes == 1;
    static constexpr int BM = 128;  // query rows per tile (TMEM lanes); two tiles per CTA
    static constexpr int BN = 64;   // keys per tile = 4 blocks
    // K/V operand ring stages (16-bit): the MMA issuer reads tile j + 2's
    // stage while PV(j) still holds tile j's, so at least 3
    static constexpr int ST = KV8 ? 3 : 4;
    static constexpr int SST = KV8 ? 4 : 0;  // 8-bit staging ring stages
    static constexpr int ATOMS = D / 64;  // 128-byte swizzle atoms across d (16-bit)
    static constexpr int Q_BYTES = ATOMS * BM * 128;  // one query tile
    static constexpr int KV_BYTES = ATOMS * BN * 128;
    static constexpr int KV8_BYTES = BN * D;          // one 8-bit tile (d = 128: 128-byte rows)
    static constexpr int OFF_Q = 0;                   // tile A, then tile B
    static constexpr int OFF_KV = 2 * Q_BYTES;        // stage st: K, then V
    static constexpr int OFF_STG = OFF_KV + ST * 2 * KV_BYTES;  // 8-bit stage: K, then V
    static constexpr int OFF_BAR = OFF_STG + SST * 2 * KV8_BYTES;
    // q_full, kv_full[ST], kv_empty[ST], then per (tile, score buffer):
    // s_full, p_full, pv_done; drain; q_ready, stg_full[SST], stg_empty[SST];
    // drain of the second MMA issuer; tail cleared; q_empty; o_free[2];
    // item_full[2], item_empty[2]
    static constexpr int NBAR = 1 + 2 * ST + 4 + 4 + 4 + 1 + 1 + 2 * SST + 2 + 7;
    static constexpr int OFF_SLOT = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ABORT = OFF_SLOT + 4;
    static constexpr int OFF_QEXP = OFF_ABORT + 4;    // log2 of the q scaling, per item parity (8-bit caches)
    static constexpr int OFF_TAIL = OFF_QEXP + 8;     // tails of V claimed for clearing so far
    static constexpr int OFF_ITEM = OFF_TAIL + 4;     // the item ring's two slots
    static constexpr int OFF_ORDER = OFF_ITEM + 8;    // sequences by context length, then their contexts
    // 16-bit caches: each softmax warp's output rows pass through 4 KiB of
    // shared memory (32 rows x 128 bytes, one 64-column half at a time), so the
    // epilogue's global stores cover whole 128-byte row segments (8-bit caches
    // have no room left for it)
    static constexpr bool OSTAGE = !KV8;
    static constexpr int OFF_OSTG = (OFF_ORDER + 8 * kOrderSeqs + 127) / 128 * 128;
    static constexpr int USED = OSTAGE ? OFF_OSTG + 8 * 4096 : OFF_ORDER + 8 * kOrderSeqs;
    // at least 120 KiB so that one CTA holds an SM (and its 512 TMEM columns)
    static constexpr int SMEM = 1024 + (USED < 120 * 1024 ? 120 * 1024 : USED);
    // MMA operand type: T, or f16 for 8-bit caches (codes widen to f16 exactly)
    static constexpr bool OP_BF16 = std::is_same<T, bf16_t>::value && !KV8;
    static constexpr bool HILO = OP_BF16;
    static constexpr uint32_t TMEM_COLS = 512;
    // score buffer b of tile t at column 64 (2 t + b) (P written over it), O
    // of tile t at 256 + 128 t
    static constexpr uint32_t COL_S = 0, COL_O = 256;
    static constexpr uint32_t FMT = OP_BF16 ? 1u : 0u;  // kind::f16 operand format: f16 0, bf16 1
    // instruction descriptors: fp32 accumulate, A/B format, majors, N >> 3, M >> 4
    static constexpr uint32_t IDESC_QK = (1u << 4) | (FMT << 7) | (FMT << 10) |
                                         ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
    static constexpr uint32_t IDESC_PV = (1u << 4) | (FMT << 7) | (FMT << 10) | (1u << 16) |
                                         ((uint32_t)(D >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
    // 8 softmax warps, a TMA warp, an MMA warp per query tile (9 for A and
    // MMA_B for B), + two converter warps (K and V) for 8-bit caches
    static constexpr int CONVERTERS = KV8 ? 2 : 0;
    static constexpr int MMA_B = 10 + CONVERTERS;
    static constexpr int THREADS = 352 + 32 * CONVERTERS;
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static_assert(!KV8 || D == 128, "8-bit caches: head_dim 128");
    static_assert(ST >= 3, "two key tiles of look-ahead plus the one in PV");
    static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ float ex2(float x) {  // 2^x; -inf -> +0
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Work-item counters of the persistent launch: [next item, CTAs finished] per
// slot.  The host gives each launch the next of kWorkSlots slots in turn; the
// last CTA of a launch to finish resets its slot to zero.
constexpr int kWorkSlots = 64;
__device__ unsigned int g_prefill_work[kWorkSlots][2];

// One work item: a (pair of query tiles, KV head, sequence or prefix key range).
struct PfItem {
    int kvh, s, split, L, q0, tok0, ntok, ctx, nt, j0, nblk;
    int state;  // 0: attend; 1: nothing to do; 2: an empty key range (write an empty partial)
};

template <int BN>
__device__ __forceinline__ PfItem decode_item(const PrefillParams &p, int item, bool flag_errors) {
    PfItem w{};
    const int x = item % p.items_x, rest = item / p.items_x;
    w.kvh = rest % p.num_kv_heads;
    const int z = rest / p.num_kv_heads;
    const bool causal = p.shared_len == 0;
    w.s = causal ? z : 0;
    w.split = causal ? 0 : z;
    w.L = causal ? p.seq_lens[w.s] : p.shared_len;
    w.q0 = causal ? p.query_start[w.s] : 0;
    const int n = causal ? p.query_start[w.s + 1] - w.q0 : p.num_tokens;
    w.state = 1;
    if (w.L < 0 || w.L > p.max_blocks_per_seq * p.block_size || n < 0 || (causal && n > w.L) || w.q0 < 0 ||
        w.q0 + n > p.num_tokens || n > p.max_query_len) {
        if (flag_errors && x == 0 && w.kvh == 0) flag_error(p.err, kErrBounds);
        return w;
    }
    w.tok0 = x * 2 * p.tok_per_tile;  // query tile A: tok0 .., tile B: tok0 + tpt ..
    if (w.tok0 >= n) return w;
    w.ntok = min(2 * p.tok_per_tile, n - w.tok0);
    w.ctx = w.L - n;
    // key tiles up to the last row's position (all of the prefix without the
    // mask); shared mode: tiles j0 .. j0 + nt - 1 of the prefix, range z
    w.nt = causal ? (w.ctx + w.tok0 + w.ntok - 1) / BN + 1 : (w.L + BN - 1) / BN;
    if (!causal) {
        const int per = (w.nt + p.items_z - 1) / p.items_z;
        w.j0 = w.split * per;
        w.nt = min(per, w.nt - w.j0);
        if (w.nt <= 0) {  // an empty range (the host never makes one)
            w.state = 2;
            return w;
        }
    }
    if (w.nt <= 0) return w;  // an empty prefix
    w.nblk = (w.L + kBlockSize - 1) / kBlockSize;  // 16-token tiles
    w.state = 0;
    return w;
}

// Persistent: gridDim.x CTAs (one an SM) take work items from the launch's
// counter until they run out.  The TMA warp takes each item and passes it to
// the other roles through a two-slot ring in shared memory; every role then
// runs the item with its barrier phases continuing from the previous one, so
// one item's loads and first MMAs overlap the previous item's last tiles.
template <typename T, int D, typename KVT>
__global__ void __launch_bounds__(PfCfg<T, D, KVT>::THREADS, 1)
    prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmap_q,
                   const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v) {
    using C = PfCfg<T, D, KVT>;
    using OpT = typename std::conditional<C::OP_BF16, bf16_t, f16_t>::type;  // MMA operand type
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = p.group, tpt = p.tok_per_tile;
    const bool causal = p.shared_len == 0;
    const int n_items = p.items_x * p.num_kv_heads * p.items_z;
    const uint64_t wl = p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs;  // bound on every wait
    const int tile_mask = (1 << p.tile_shift) - 1;

    const uint32_t bars = base + C::OFF_BAR;
    const uint32_t bar_q = bars;
    auto bar_kv_full = [&](int st) { return bars + 8u * (1 + st); };
    auto bar_kv_empty = [&](int st) { return bars + 8u * (1 + C::ST + st); };
    // one barrier per (tile, score buffer): a buffer's next phase needs the
    // other roles to have used the last one, so no wait can see a phase twice
    auto bar_s_full = [&](int t, int b) { return bars + 8u * (1 + 2 * C::ST + 2 * t + b); };
    auto bar_p_full = [&](int t, int b) { return bars + 8u * (5 + 2 * C::ST + 2 * t + b); };
    auto bar_pv = [&](int t, int b) { return bars + 8u * (9 + 2 * C::ST + 2 * t + b); };
    const uint32_t bar_drain = bars + 8u * (13 + 2 * C::ST);
    // 8-bit caches: Q converted to f16 (q_ready); staging ring of 8-bit tiles
    const uint32_t bar_q_ready = bars + 8u * (14 + 2 * C::ST);
    auto bar_stg_full = [&](int st) { return bars + 8u * (15 + 2 * C::ST + st); };
    auto bar_stg_empty = [&](int st) { return bars + 8u * (15 + 2 * C::ST + C::SST + st); };
    const uint32_t bar_drain_b = bars + 8u * (15 + 2 * C::ST + 2 * C::SST);
    const uint32_t bar_tail = bars + 8u * (16 + 2 * C::ST + 2 * C::SST);
    // both issuers' last Q.K^T of an item done (Q may be reloaded); tile t's
    // O read out by its softmax warps (the next item's P.V may overwrite it);
    // the item ring: slot written / read by every consumer warp
    const uint32_t bar_q_empty = bars + 8u * (17 + 2 * C::ST + 2 * C::SST);
    auto bar_o_free = [&](int t) { return bars + 8u * (18 + 2 * C::ST + 2 * C::SST + t); };
    auto bar_item_full = [&](int b) { return bars + 8u * (20 + 2 * C::ST + 2 * C::SST + b); };
    auto bar_item_empty = [&](int b) { return bars + 8u * (22 + 2 * C::ST + 2 * C::SST + b); };
    volatile int *item_slot = reinterpret_cast<volatile int *>(smem + C::OFF_ITEM);
    volatile int *qexp = reinterpret_cast<volatile int *>(smem + C::OFF_QEXP);  // per item parity
    auto s_col = [&](int t, int b) { return C::COL_S + 64u * (2 * t + b); };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_ABORT);
    uint32_t *slot = reinterpret_cast<uint32_t *>(smem + C::OFF_SLOT);
    constexpr int CONSUMERS = 8 + 2 + C::CONVERTERS;  // warps that read the item ring

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
#pragma unroll
        for (int st = 0; st < C::ST; ++st) {
            mbar_init(bar_kv_full(st), C::KV8 ? C::CONVERTERS : 1);  // TMA, or the converters
            mbar_init(bar_kv_empty(st), 2);  // both MMA issuers
        }
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                mbar_init(bar_s_full(t, b), 1);
                mbar_init(bar_p_full(t, b), 128);
                mbar_init(bar_pv(t, b), 1);
            }
        mbar_init(bar_drain, 1);
        mbar_init(bar_drain_b, 1);
        mbar_init(bar_tail, 1);
        *reinterpret_cast<volatile int *>(smem + C::OFF_TAIL) = 0;
        mbar_init(bar_q_ready, 1);
#pragma unroll
        for (int st = 0; st < C::SST; ++st) {
            mbar_init(bar_stg_full(st), 1);
            mbar_init(bar_stg_empty(st), C::CONVERTERS);
        }
        mbar_init(bar_q_empty, 2);
        mbar_init(bar_o_free(0), 128);
        mbar_init(bar_o_free(1), 128);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_item_full(b), 1);
            mbar_init(bar_item_empty(b), CONSUMERS);
        }
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 0) tc::alloc(smem_addr(slot), C::TMEM_COLS);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *slot;

    auto q_smem = [&](int t) { return base + C::OFF_Q + (uint32_t)(t * C::Q_BYTES); };
    auto k_smem = [&](int st) { return base + C::OFF_KV + (uint32_t)(st * 2 * C::KV_BYTES); };
    auto v_smem = [&](int st) { return k_smem(st) + (uint32_t)C::KV_BYTES; };
    auto stg_k = [&](int st) { return base + C::OFF_STG + (uint32_t)(st * 2 * C::KV8_BYTES); };
    auto stg_v = [&](int st) { return stg_k(st) + (uint32_t)C::KV8_BYTES; };
    // a consumer warp's next item (-1: none left); k counts the items taken
    auto next_item = [&](int k) -> int {
        const bool ok = __all_sync(tc::kFull, tc::wait_phase(bar_item_full(k & 1), (k >> 1) & 1, abort_flag, p.err, wl));
        const int item = ok ? item_slot[k & 1] : -1;
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar_item_empty(k & 1));
        return item;
    };

    if (warp == 8) {
        // ================= TMA producer ===========================================
        // Takes the items.  Lane 0 issues the copies.  The whole warp holds the
        // pool rows of an item's 16-token tiles: lane i the row of tile 32 b + i
        // of the current batch b and of the next one, read a batch ahead, so no
        // copy waits on a block-table load.
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_q)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_v)) : "memory");
        }
        constexpr int TPK = C::BN / kBlockSize;  // 16-token tiles per key tile
        static_assert(32 % TPK == 0, "a batch of 32 tiles holds whole key tiles");
        constexpr int RING = C::KV8 ? C::SST : C::ST;  // the ring the copies land in
        auto full_bar = [&](int st) { return C::KV8 ? bar_stg_full(st) : bar_kv_full(st); };
        auto empty_bar = [&](int st) { return C::KV8 ? bar_stg_empty(st) : bar_kv_empty(st); };
        int U = 0, kq = 0;  // key tiles issued, items with work (Q loads)
        bool ok = true;
        // the order items are handed out in (see kOrderSeqs)
        int *order = reinterpret_cast<int *>(smem + C::OFF_ORDER);
        const bool ordered = causal && p.num_seqs <= kOrderSeqs;
        if (ordered) {
            volatile int *ctxs = order + kOrderSeqs;
            for (int q = lane; q < p.num_seqs; q += 32)
                ctxs[q] = p.seq_lens[q] - (p.query_start[q + 1] - p.query_start[q]);
            __syncwarp();
            for (int q = lane; q < p.num_seqs; q += 32) {
                const int cq = ctxs[q];
                int rank = 0;
                for (int o = 0; o < p.num_seqs; ++o) {
                    const int co = ctxs[o];
                    rank += (co > cq) || (co == cq && o < q);
                }
                order[rank] = q;
            }
            __syncwarp();
        }
        auto natural_item = [&](int c) -> int {  // c-th item handed out -> its natural index
            if (!ordered) return c;
            const int per_seq = p.items_x * p.num_kv_heads;
            const int r = c / per_seq, rem = c - r * per_seq;
            const int x = p.items_x - 1 - rem / p.num_kv_heads, kvh = rem % p.num_kv_heads;
            return (order[r] * p.num_kv_heads + kvh) * p.items_x + x;
        };
        for (int k = 0; ok; ++k) {
            // take an item and publish it to the ring (slot k & 1)
            int item = -1;
            if (lane == 0) {
                item = (int)atomicAdd(&g_prefill_work[p.work_slot][0], 1u);
                item = item < n_items ? natural_item(item) : -1;
                if (k >= 2) ok = tc::wait_phase(bar_item_empty(k & 1), ((k >> 1) - 1) & 1, abort_flag, p.err, wl);
                item_slot[k & 1] = ok ? item : -1;
                tc::mbar_arrive(bar_item_full(k & 1));
            }
            ok = __shfl_sync(tc::kFull, (int)ok, 0) != 0;
            item = __shfl_sync(tc::kFull, item, 0);
            if (!ok || item < 0) break;
            const PfItem w = decode_item<C::BN>(p, item, true);
            if (w.state != 0) continue;
            // Q of both tiles, once both issuers are done with the previous item's
            if (lane == 0) {
                if (kq > 0) ok = tc::wait_phase(bar_q_empty, (kq - 1) & 1, abort_flag, p.err, wl);
                if (ok) {
                    mbar_arrive_expect_tx(bar_q, (uint32_t)(2 * C::ATOMS * tpt * g * 128));
#pragma unroll
                    for (int t = 0; t < 2; ++t)
#pragma unroll
                        for (int a = 0; a < C::ATOMS; ++a)
                            tc::tma_load_3d(q_smem(t) + a * C::BM * 128, &tmap_q, a * 64, w.kvh * g,
                                            w.q0 + w.tok0 + t * tpt, bar_q);
                }
            }
            ok = __shfl_sync(tc::kFull, (int)ok, 0) != 0;
            if (!ok) break;
            ++kq;
            const int32_t *bt = p.block_tables + (int64_t)w.s * p.max_blocks_per_seq;
            const int tile0 = w.j0 * TPK, ntiles = w.nt * TPK;
            auto rows_of_batch = [&](int batch) -> int {  // pool row of this lane's tile (past the pool: zeros)
                const int i = batch * 32 + lane, lb = tile0 + i;
                int y = p.oob_row;
                if (i < ntiles && lb < w.nblk) {
                    const int phys = bt[lb >> p.tile_shift];
                    if ((unsigned)phys < (unsigned)p.num_blocks)
                        y = (phys * p.num_kv_heads + w.kvh) * p.block_size + (lb & tile_mask) * kBlockSize;
                    else
                        flag_error(p.err, kErrBounds);
                }
                return y;
            };
            int rows_cur = rows_of_batch(0), rows_nxt = ntiles > 32 ? rows_of_batch(1) : p.oob_row;
            int cur_batch = 0;
            for (int j = 0; j < w.nt; ++j, ++U) {
                const int st = U % RING;
                if (U >= RING) {
                    int r = lane == 0 ? (int)tc::wait_phase(empty_bar(st), ((U / RING) - 1) & 1, abort_flag, p.err, wl) : 0;
                    if (!__shfl_sync(tc::kFull, r, 0)) {
                        ok = false;
                        break;
                    }
                }
                if ((j * TPK) >> 5 != cur_batch) {  // uniform: the next batch becomes current
                    rows_cur = rows_nxt;
                    ++cur_batch;
                    rows_nxt = (cur_batch + 1) * 32 < ntiles ? rows_of_batch(cur_batch + 1) : p.oob_row;
                }
                // one copy per lane: lane l takes block l % TPK of the key tile, then
                // (16-bit caches) atom l / TPK % ATOMS, K for l < NCOPY / 2 and V after
                const int y = __shfl_sync(tc::kFull, rows_cur, (j * TPK + lane % TPK) & 31);
                if (lane == 0)
                    mbar_arrive_expect_tx(full_bar(st), C::KV8 ? 2u * C::KV8_BYTES : 2u * C::KV_BYTES);
                __syncwarp();
                constexpr int NCOPY = 2 * TPK * (C::KV8 ? 1 : C::ATOMS);
                static_assert(NCOPY <= 32, "one copy per lane");
                if (lane < NCOPY && !(p.hold_first_tile && U == 0)) {
                    const int b = lane % TPK, is_v = lane >= NCOPY / 2;
                    if constexpr (C::KV8) {  // 16 rows x 128 codes, 128B swizzle
                        const uint32_t dst = (is_v ? stg_v(st) : stg_k(st)) + b * kBlockSize * 128;
                        tc::tma_load_2d(dst, is_v ? &tmap_v : &tmap_k, 0, y, full_bar(st));
                    } else {
                        const int a = (lane / TPK) % C::ATOMS;
                        const uint32_t dst = (is_v ? v_smem(st) : k_smem(st)) + a * C::BN * 128 + b * kBlockSize * 128;
                        tc::tma_load_2d(dst, is_v ? &tmap_v : &tmap_k, a * 64, y, full_bar(st));
                    }
                }
            }
        }
        // nothing may still be landing in shared memory when the CTA exits
        if (lane == 0) {
            if (kq > 0) (void)mbar_wait_bounded(bar_q, (kq - 1) & 1, wl);
            for (int u = U - RING < 0 ? 0 : U - RING; u < U; ++u)
                (void)mbar_wait_bounded(full_bar(u % RING), (u / RING) & 1, wl);
        }
        __syncwarp();
    } else if (warp == 9 || warp == C::MMA_B) {
        // ================= MMA issuers ============================================
        // One per query tile (warp 9: A, warp MMA_B: B), so that while one waits
        // for its softmax the other keeps the tensor core fed; one lane of each
        // does all of it, and the shared-memory descriptors are formed once
        // and stepped by constant offsets.  Order per key tile j: PV_t(j),
        // QK_t(j+2) -- the tile's scores are computed two key tiles ahead into
        // its other S buffer; tcgen05 operations of one thread run in issue
        // order, which makes reusing a score buffer's columns for P and then
        // for the scores two tiles later safe.  A K/V stage is free once both
        // issuers' P.V of it is done (kv_empty counts two commits).
        const int t = warp == 9 ? 0 : 1;
        const uint64_t qd = tc::sdesc(q_smem(t), 16, 1024);
        const uint64_t kdesc = tc::sdesc(k_smem(0), 16, 1024);
        const uint64_t vdesc = tc::sdesc(v_smem(0), C::BN * 128, 1024);
        const uint32_t ocol = tmem + C::COL_O + 128u * t;
        int J = 0, kq = 0, ntail = 0;  // key tiles done (all items), items with work, tails cleared
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int item = next_item(k);
            if (item < 0) break;
            const PfItem w = decode_item<C::BN>(p, item, false);
            if (w.state != 0) continue;
            if (lane == 0) {
                const int nt = w.nt;
                // key tile j of this item: stage (J + j) % ST, score buffer (J + j) & 1
                auto issue_qk = [&](int j) {
                    const int jj = J + j;
                    const uint64_t kd = kdesc + (uint64_t)(((jj % C::ST) * 2 * C::KV_BYTES) >> 4);
                    const uint32_t d = tmem + s_col(t, jj & 1);
                    tc::fence_after();
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t in_atom = (ks & 3) * 32;
                        tc::mma_ss(d, qd + (uint64_t)(((ks >> 2) * (C::BM * 128) + in_atom) >> 4),
                                   kd + (uint64_t)(((ks >> 2) * (C::BN * 128) + in_atom) >> 4), C::IDESC_QK, ks > 0);
                    }
                    tc::commit(bar_s_full(t, jj & 1));
                    if (j == nt - 1) tc::commit(bar_q_empty);  // this issuer's last read of Q
                };
                auto issue_pv = [&](int j) {
                    const int jj = J + j;
                    const uint64_t vd = vdesc + (uint64_t)(((jj % C::ST) * 2 * C::KV_BYTES) >> 4);
                    const uint32_t pcol = tmem + s_col(t, jj & 1);
                    tc::fence_after();
#pragma unroll
                    for (int ks = 0; ks < C::BN / 16; ++ks) {
                        const uint64_t bd = vd + (uint64_t)((ks * 2048) >> 4);
                        if constexpr (C::HILO) {  // hi of keys 16 ks .. in column 32 (ks / 2) + 8 (ks % 2), lo 16 after
                            const uint32_t pc = pcol + (ks >> 1) * 32 + (ks & 1) * 8;
                            tc::mma_ts(ocol, pc, bd, C::IDESC_PV, (j > 0 || ks > 0));
                            tc::mma_ts(ocol, pc + 16, bd, C::IDESC_PV, 1);
                        } else {
                            tc::mma_ts(ocol, pcol + ks * 8, bd, C::IDESC_PV, (j > 0 || ks > 0));
                        }
                    }
                    tc::commit(bar_pv(t, jj & 1));
                    tc::commit(bar_kv_empty(jj % C::ST));  // this issuer's last read of the stage
                };
                auto wait1 = [&](uint32_t bar, uint32_t parity) {
                    return tc::wait_phase(bar, parity, abort_flag, p.err, wl);
                };
                auto kv_ready = [&](int j) {
                    const int jj = J + j;
                    return wait1(bar_kv_full(jj % C::ST), (jj / C::ST) & 1);
                };
                const int j_tail = (w.L & (kBlockSize - 1)) ? (w.nblk - 1) / (C::BN / kBlockSize) - w.j0 : -1;
                // the tail tile's unused rows: [r0, r1) of its key tile
                const int tail_r0 = w.L - (w.j0 + j_tail) * C::BN, tail_r1 = w.nblk * kBlockSize - (w.j0 + j_tail) * C::BN;
                // Before P.V of the key tile holding the sequence's last block: the
                // V rows of its unused slots (positions >= L) are cleared (p = 0
                // there, but 0 x NaN poison = NaN).  The first issuer to get there
                // clears them (its Q.K^T of the tile came after the copies landed),
                // the other waits until it is done.
                auto tail_ready = [&](int j) {
                    if (j != j_tail) return true;
                    if (atomicCAS(reinterpret_cast<int *>(smem + C::OFF_TAIL), ntail, ntail + 1) == ntail) {
                        const int st = (J + j) % C::ST;
                        const int chunks = (tail_r1 - tail_r0) * C::ATOMS * 8;
                        for (int c = 0; c < chunks; ++c) {
                            const int row = tail_r0 + c / (C::ATOMS * 8), rem = c % (C::ATOMS * 8);
                            const uint32_t addr = v_smem(st) + (rem >> 3) * C::BN * 128 + row * 128 + (rem & 7) * 16;
                            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
                        }
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                        tc::mbar_arrive(bar_tail);
                    }
                    return wait1(bar_tail, (ntail++) & 1);
                };
                ok = wait1(C::KV8 ? bar_q_ready : bar_q, kq & 1);  // 8-bit caches: q converted
                for (int j = 0; ok && j < 2 && j < nt; ++j) {
                    ok = kv_ready(j);
                    if (!ok) break;
                    issue_qk(j);
                }
                // the previous item's O has been read out of tile t's accumulator
                if (ok && kq > 0) {
                    ok = wait1(bar_o_free(t), (kq - 1) & 1);
                    tc::fence_after();
                }
                for (int j = 0; ok && j < nt; ++j) {
                    const int jj = J + j;
                    ok = wait1(bar_p_full(t, jj & 1), (jj >> 1) & 1) && tail_ready(j);
                    if (!ok) break;
                    issue_pv(j);
                    if (j + 2 < nt) {
                        ok = kv_ready(j + 2);
                        if (!ok) break;
                        issue_qk(j + 2);
                    }
                }
            }
            ok = __shfl_sync(tc::kFull, (int)ok, 0) != 0;
            J += w.nt;
            ++kq;
        }
        // every MMA of this thread must be complete before TMEM is freed
        if (lane == 0) {
            const uint32_t drain = t == 0 ? bar_drain : bar_drain_b;
            tc::commit(drain);
            (void)mbar_wait_bounded(drain, 0, wl);
        }
        __syncwarp();
    } else if (warp >= 10 && warp < 10 + C::CONVERTERS) {
        // ================= converters (8-bit caches only) ===========================
        // warp 10 widens q (bf16 -> f16, scaled by a power of two so its
        // largest magnitude sits near 2^14; the inverse folds into the logit
        // scale) and every landed 8-bit K tile, warp 11 every V tile, to f16
        // in the swizzled operand layout the MMAs read; each code's value is
        // exact in f16
        if constexpr (C::KV8) {
            const int kv = warp - 10;  // 0: K, 1: V
            int U = 0, kq = 0;          // key tiles converted (all items), items with work
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int item = next_item(k);
                if (item < 0) break;
                const PfItem w = decode_item<C::BN>(p, item, false);
                if (w.state != 0) continue;
                if (kv == 0) {
                    ok = __all_sync(tc::kFull, tc::wait_phase(bar_q, kq & 1, abort_flag, p.err, wl));
                    int e = 0;
                    if (ok && std::is_same<T, bf16_t>::value) {
                        const int rows = tpt * g;  // rows the copy wrote in each tile
                        float amax = 0.f;
                        for (int t = 0; t < 2; ++t)
                            for (int a = 0; a < C::ATOMS; ++a)
                                for (int idx = lane; idx < rows * 8; idx += 32) {
                                    uint32_t wv[4];
                                    lds<16>(wv, q_smem(t) + a * C::BM * 128 + (idx >> 3) * 128 + (idx & 7) * 16);
                                    float f[8];
                                    Unpack<bf16_t, 8>::run(wv, f);
#pragma unroll
                                    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
                                }
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(tc::kFull, amax, o));
                        if (amax > 0.f && amax <= 3.0e38f) {
                            e = 14 - ((int)((__float_as_uint(amax) >> 23) & 0xFF) - 127);
                            e = e > 100 ? 100 : (e < -100 ? -100 : e);
                        }
                        const float up = __uint_as_float((uint32_t)(127 + e) << 23);  // 2^e, exact
                        for (int t = 0; t < 2; ++t)
                            for (int a = 0; a < C::ATOMS; ++a)
                                for (int idx = lane; idx < rows * 8; idx += 32) {
                                    const uint32_t addr = q_smem(t) + a * C::BM * 128 + (idx >> 3) * 128 + (idx & 7) * 16;
                                    uint32_t wv[4];
                                    lds<16>(wv, addr);
                                    float f[8];
                                    Unpack<bf16_t, 8>::run(wv, f);
                                    uint32_t h[4];
#pragma unroll
                                    for (int i = 0; i < 4; ++i) h[i] = tc::pack2(f[2 * i] * up, f[2 * i + 1] * up, f16_t{});
                                    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(h[0]),
                                                 "r"(h[1]), "r"(h[2]), "r"(h[3])
                                                 : "memory");
                                }
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    }
                    if (lane == 0) qexp[kq & 1] = e;
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar_q_ready);
                }
                for (int j = 0; ok && j < w.nt; ++j) {
                    const int uu = U + j;
                    const int sst = uu % C::SST, st = uu % C::ST;
                    ok = __all_sync(tc::kFull, tc::wait_phase(bar_stg_full(sst), (uu / C::SST) & 1, abort_flag, p.err, wl));
                    if (!ok) break;
                    if (uu >= C::ST) {  // the MMAs are done with this operand stage
                        ok = __all_sync(tc::kFull,
                                        tc::wait_phase(bar_kv_empty(st), ((uu / C::ST) - 1) & 1, abort_flag, p.err, wl));
                        if (!ok) break;
                    }
                    {
                        const uint32_t src = kv ? stg_v(sst) : stg_k(sst);
                        const uint32_t dst = kv ? v_smem(st) : k_smem(st);
                        // BN * 8 chunks of 16 codes, batches of 4 a lane: the loads of
                        // a batch go out together, then its conversions and stores
                        constexpr int NB = 4, PER = C::BN * 8 / 32;
                        static_assert(PER % NB == 0, "batches");
#pragma unroll
                        for (int i0 = 0; i0 < PER; i0 += NB) {
                            uint32_t wv[NB][4];
#pragma unroll
                            for (int b = 0; b < NB; ++b) {
                                const int idx = lane + 32 * (i0 + b), r = idx >> 3, c8 = idx & 7;
                                lds<16>(wv[b], src + r * 128 + ((c8 ^ (r & 7)) << 4));
                            }
#pragma unroll
                            for (int b = 0; b < NB; ++b) {
                                const int idx = lane + 32 * (i0 + b);
                                const int r = idx >> 3, c8 = idx & 7;  // row, chunk of 16 codes
                                uint32_t h[8];
#pragma unroll
                                for (int i = 0; i < 4; ++i) tc::widen4(wv[b][i], h[2 * i], h[2 * i + 1], KVT{});
                                // codes 16 c8 .. +15 = f16 chunks 2 (c8 % 4) and +1 of atom c8 / 4
                                const uint32_t rowb = dst + (c8 >> 2) * C::BN * 128 + r * 128;
                                const int cf = (c8 & 3) * 2;
                                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(rowb + ((cf ^ (r & 7)) << 4)),
                                             "r"(h[0]), "r"(h[1]), "r"(h[2]), "r"(h[3])
                                             : "memory");
                                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(rowb + (((cf + 1) ^ (r & 7)) << 4)),
                                             "r"(h[4]), "r"(h[5]), "r"(h[6]), "r"(h[7])
                                             : "memory");
                            }
                        }
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) {
                        tc::mbar_arrive(bar_stg_empty(sst));
                        tc::mbar_arrive(bar_kv_full(st));
                    }
                }
                U += w.nt;
                ++kq;
            }
        }
    } else {
        // ================= softmax: one thread per query row =======================
        const int t = warp >> 2;                  // query tile (0: A, 1: B)
        const int r = (warp & 3) * 32 + lane;     // row = TMEM lane
        const uint32_t lane_bits = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t ocol = tmem + lane_bits + C::COL_O + 128u * t;
        int J = 0, kq = 0;  // key tiles done (all items), items with work
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int item = next_item(k);
            if (item < 0) break;
            const PfItem w = decode_item<C::BN>(p, item, false);
            if (w.state == 2) {
                // an empty key range: an empty partial (lse = -inf, o = 0) for this
                // warp's rows
                const int rtok = t * tpt + r / g;
                if (r < tpt * g && rtok < w.ntok) {
                    const int64_t row = (int64_t)(w.q0 + w.tok0 + rtok) * p.num_q_heads + (int64_t)w.kvh * g + r % g;
                    p.ws_lse[row * p.ws_np + w.split] = -CUDART_INF_F;
                    for (int d = 0; d < D; ++d) p.ws_o[(row * p.ws_np + w.split) * D + d] = 0.f;
                }
                continue;
            }
            if (w.state != 0) continue;
            const int nt = w.nt;
            const int rtok = t * tpt + r / g;  // token within the item's range
            const bool row_ok = r < tpt * g && rtok < w.ntok;
            // the row's last visible key, counted from the item's first key tile
            const int pos0 = (causal ? w.ctx + w.tok0 + rtok : w.L - 1) - w.j0 * C::BN;
            const int64_t row = ((int64_t)(w.q0 + w.tok0 + rtok) * p.num_q_heads + (int64_t)w.kvh * g + r % g);
            const int split = w.split;
            float sl2 = p.qk_scale_log2;  // > 0
            if constexpr (C::KV8) {  // q was scaled by 2^e on its way to f16
                if (!__all_sync(tc::kFull, tc::wait_phase(bar_q_ready, kq & 1, abort_flag, p.err, wl))) {
                    ok = false;
                    break;
                }
                const int e = qexp[kq & 1];
                sl2 *= __uint_as_float((uint32_t)(127 - e) << 23);
            }
            float m_ref = -CUDART_INF_F, l = 0.f;
            for (int j = 0; j < nt; ++j) {
                const int jj = J + j;
                ok = __all_sync(tc::kFull, tc::wait_phase(bar_s_full(t, jj & 1), (jj >> 1) & 1, abort_flag, p.err, wl));
                if (!ok) break;
                tc::fence_after();
                const uint32_t scol = tmem + lane_bits + s_col(t, jj & 1);
                uint32_t sv[C::BN];
#pragma unroll
                for (int c = 0; c < C::BN; c += 32) tc::ld32(scol + c, sv + c);
                tc::wait_ld<C::BN>(sv);
                // keys of this tile the row may see: all, a prefix (diagonal tile), none
                const int lim = row_ok ? pos0 - j * C::BN + 1 : 0;
                if (lim < C::BN) {
#pragma unroll
                    for (int c = 0; c < C::BN; ++c)
                        if (c >= lim) sv[c] = __float_as_uint(-CUDART_INF_F);
                }
                float m4[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
                for (int c = 0; c < C::BN; ++c) m4[c & 3] = fmaxf(m4[c & 3], __uint_as_float(sv[c]));
                const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
                // lazy rescale: move the reference max only when it grows by > 8
                float alpha = 1.f;
                const bool grow = mx > m_ref + 8.f;
                if (grow) {
                    alpha = m_ref == -CUDART_INF_F ? 0.f : ex2(m_ref - mx);
                    m_ref = mx;
                }
                const float nmb = m_ref == -CUDART_INF_F ? 0.f : -m_ref;
                l *= alpha;
                float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c0 = 0; c0 < C::BN; c0 += 32) {
                    uint32_t hl[32];  // hi pairs, then lo pairs (bf16 caches)
                    uint32_t *hi = hl, *lo = hl + 16;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float p0 = ex2(fmaf(__uint_as_float(sv[c0 + 2 * i]), sl2, nmb));
                        const float p1 = ex2(fmaf(__uint_as_float(sv[c0 + 2 * i + 1]), sl2, nmb));
                        ps[i & 3] += p0 + p1;
                        hi[i] = tc::pack2(p0, p1, OpT{});
                        if constexpr (C::HILO) {
                            float h0, h1;
                            tc::unpack2(hi[i], h0, h1, bf16_t{});
                            lo[i] = tc::pack2(p0 - h0, p1 - h1, OpT{});
                        }
                    }
                    // bf16 caches: one store of the chunk's 16 hi and 16 lo columns
                    // (columns c0 .. c0 + 31); f16: its 16 columns at c0 / 2
                    if constexpr (C::HILO) tc::st32(scol + c0, hl);
                    else tc::st16(scol + c0 / 2, hi);
                }
                l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
                if (j > 0 && __any_sync(tc::kFull, grow)) {
                    // O may be rescaled only once the previous P.V of this tile is
                    // complete (the earlier ones completed before it)
                    ok = __all_sync(tc::kFull, tc::wait_phase(bar_pv(t, (jj - 1) & 1), ((jj - 1) >> 1) & 1,
                                                             abort_flag, p.err, wl));
                    if (!ok) break;
                    tc::fence_after();
#pragma unroll
                    for (int c = 0; c < D; c += 32) {
                        uint32_t o[32];
                        tc::ld32(ocol + c, o);
                        tc::wait_ld<32>(o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tc::st32(ocol + c, o);
                    }
                }
                tc::wait_st();
                tc::fence_before();
                tc::mbar_arrive(bar_p_full(t, jj & 1));
            }
            if (ok) {
                const int jl = J + nt - 1;
                ok = __all_sync(tc::kFull, tc::wait_phase(bar_pv(t, jl & 1), (jl >> 1) & 1, abort_flag, p.err, wl));
            }
            if (!ok) break;
            // ---- epilogue: out = O / l, rounded once to the q dtype ----------------
            // (shared-prefix mode: the partial o / l and its log-sum-exp, fp32).
            // Once O is out of TMEM, tile t's accumulator is handed to the next
            // item's P.V (o_free).
            tc::fence_after();
            const float inv = l > 0.f ? p.v_scale / l : 0.f;  // v_scale: 1 for 16-bit caches
            if (causal && C::OSTAGE) {
                // per 64-column half: the warp's 32 rows x 128 bytes into its
                // shared-memory slab (16-byte chunk c of row r at chunk
                // c ^ (r & 7): conflict-free), then read back four rows at a
                // time, each lane one 16-byte chunk, and stored as 128-byte
                // row segments
                const uint32_t slab = base + C::OFF_OSTG + (uint32_t)warp * 4096u;
                uint4 *out16 = reinterpret_cast<uint4 *>(p.out);
                const int64_t row16 = row * (D / 8);  // 16-byte units
#pragma unroll
                for (int a = 0; a < C::ATOMS; ++a) {
                    uint32_t wv[32];
#pragma unroll
                    for (int c = 0; c < 64; c += 32) {
                        uint32_t o[32];
                        tc::ld32(ocol + a * 64 + c, o);
                        tc::wait_ld<32>(o);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            wv[c / 2 + i] =
                                tc::pack2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv, T{});
                    }
                    if (a == C::ATOMS - 1) {  // O is out of TMEM
                        tc::fence_before();
                        tc::mbar_arrive(bar_o_free(t));
                    }
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(slab + lane * 128 + ((c ^ (lane & 7)) << 4)),
                                     "r"(wv[4 * c]), "r"(wv[4 * c + 1]), "r"(wv[4 * c + 2]), "r"(wv[4 * c + 3])
                                     : "memory");
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int rr = 4 * i + (lane >> 3), c = lane & 7;  // the warp's row, its chunk
                        const int ok_r = __shfl_sync(tc::kFull, (int)row_ok, rr);
                        const int64_t dst = (int64_t)__shfl_sync(tc::kFull, (long long)row16, rr) + a * 8 + c;
                        uint32_t v[4];
                        lds<16>(v, slab + rr * 128 + ((c ^ (rr & 7)) << 4));
                        if (ok_r) out16[dst] = make_uint4(v[0], v[1], v[2], v[3]);
                    }
                    __syncwarp();
                }
            } else if (causal) {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.out) + row * D);
#pragma unroll
                for (int c = 0; c < D; c += 32) {
                    uint32_t o[32];
                    tc::ld32(ocol + c, o);
                    tc::wait_ld<32>(o);
                    uint32_t wv[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        wv[i] = tc::pack2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv, T{});
                    if (row_ok) {
#pragma unroll
                        for (int v = 0; v < 4; ++v) dst[c / 8 + v] = make_uint4(wv[4 * v], wv[4 * v + 1], wv[4 * v + 2], wv[4 * v + 3]);
                    }
                }
                tc::fence_before();
                tc::mbar_arrive(bar_o_free(t));
            } else {
                float4 *wo = reinterpret_cast<float4 *>(p.ws_o + (row * p.ws_np + split) * D);
                if (row_ok)
                    p.ws_lse[row * p.ws_np + split] =
                        l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994530942f : -CUDART_INF_F;
#pragma unroll
                for (int c = 0; c < D; c += 32) {
                    uint32_t o[32];
                    tc::ld32(ocol + c, o);
                    tc::wait_ld<32>(o);
                    if (row_ok) {
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            wo[c / 4 + v] = make_float4(__uint_as_float(o[4 * v]) * inv, __uint_as_float(o[4 * v + 1]) * inv,
                                                        __uint_as_float(o[4 * v + 2]) * inv, __uint_as_float(o[4 * v + 3]) * inv);
                    }
                }
                tc::fence_before();
                tc::mbar_arrive(bar_o_free(t));
            }
            J += nt;
            ++kq;
        }
    }

    // ---- teardown: every role is done with TMEM --------------------------------
    tc::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after();
        tc::dealloc(tmem, C::TMEM_COLS);
    }
    // the launch's last CTA to finish resets its work counter for the next launch
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&g_prefill_work[p.work_slot][1], 1u) == gridDim.x - 1) {
            atomicExch(&g_prefill_work[p.work_slot][0], 0u);
            atomicExch(&g_prefill_work[p.work_slot][1], 0u);
        }
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

namespace {

// q [T, Hq, d] as a 3-D map (d, Hq, T); a box is 64 elements (128 bytes) x g
// heads x tpt tokens, 128-byte swizzle, so a box lands as tpt * g rows of
// 128 bytes in row order (token, head).
bool encode_q_map(CUtensorMap *m, const void *q, int d, int hq, int64_t tokens, int g, int tpt) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)hq, (cuuint64_t)tokens};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)hq * d * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)g, (cuuint32_t)tpt};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void *>(q), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int D, typename KVT>
cudaError_t launch_prefill_t(const PrefillParams &p, cudaStream_t stream) {
    using C = PfCfg<T, D, KVT>;
    const int64_t rows = (int64_t)p.num_blocks * p.num_kv_heads * p.block_size;
    constexpr int EB = Elem<KVT>::kBytes;
    CUtensorMap mq, mk, mv;
    if (!encode_q_map(&mq, p.q, D, p.num_q_heads, p.num_tokens, p.group, p.tok_per_tile) ||
        !encode_pool_map(&mk, p.k_cache, EB, D, rows) || !encode_pool_map(&mv, p.v_cache, EB, D, rows))
        return cudaErrorInvalidValue;
    auto kern = prefill_kernel<T, D, KVT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const int per_cta = 2 * p.tok_per_tile;  // two query tiles
    static_assert(C::BN == kPrefixKeyTile, "shared-prefix key ranges are counted in key tiles");
    PrefillParams q = p;
    q.items_x = (p.max_query_len + per_cta - 1) / per_cta;
    q.items_z = p.shared_len > 0 ? prefix_splits(p.shared_len) : p.num_seqs;
    const int64_t items = (int64_t)q.items_x * p.num_kv_heads * q.items_z;
    if (items <= 0) return cudaSuccess;
    if (items > INT32_MAX) return cudaErrorInvalidValue;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    // failure-detection test hook (see PrefillParams); unset in normal use
    if (const char *env = getenv("PA369_TEST_PREFILL_STALL_NS")) {
        const long long ns = atoll(env);
        if (ns > 0) {
            q.wait_limit_ns = (uint64_t)ns;
            q.hold_first_tile = 1;
        }
    }
    static std::atomic<unsigned> next_slot{0};
    q.work_slot = (int)(next_slot.fetch_add(1u) % (unsigned)kWorkSlots);
    const unsigned grid = (unsigned)(items < sms ? items : sms);  // one CTA an SM, persistent
    kern<<<grid, C::THREADS, C::SMEM, stream>>>(q, mq, mk, mv);
    return cudaGetLastError();
}

}  // namespace

bool prefill_supported() { return encode_fn() != nullptr; }

template <typename T>
static cudaError_t prefill_by_kv(const PrefillParams &p, DType kv, int head_dim, cudaStream_t stream) {
    switch (kv) {
        case DType::E4M3: return launch_prefill_t<T, 128, e4m3_t>(p, stream);
        case DType::E5M2: return launch_prefill_t<T, 128, e5m2_t>(p, stream);
        case DType::I8: return launch_prefill_t<T, 128, i8_t>(p, stream);
        default:
            return head_dim == 64 ? launch_prefill_t<T, 64, T>(p, stream) : launch_prefill_t<T, 128, T>(p, stream);
    }
}

cudaError_t launch_prefill(const PrefillParams &p, DType q, DType kv, int head_dim, cudaStream_t stream) {
    if (p.num_seqs <= 0 || p.num_tokens <= 0 || p.max_query_len <= 0) return cudaSuccess;
    if (is_8bit(kv) && head_dim != 128) return cudaErrorInvalidValue;
    return q == DType::F16 ? prefill_by_kv<f16_t>(p, kv, head_dim, stream)
                           : prefill_by_kv<bf16_t>(p, kv, head_dim, stream);
}

}  // namespace pa
