// Device helpers for the sm_100a paged-KV kernels: element conversions,
// mbarrier + bulk-copy (TMA, non-tensor, no multicast) primitives, bounded
// waits and device-side error reporting.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "pa_internal.h"

namespace pa {

// ---------------------------------------------------------------------------
// element types
// ---------------------------------------------------------------------------

struct f16_t {
    uint16_t bits;
};
struct bf16_t {
    uint16_t bits;
};
struct e4m3_t {
    uint8_t bits;
};
struct e5m2_t {
    uint8_t bits;
};
struct i8_t {  // symmetric INT8 code
    uint8_t bits;
};

template <typename T> struct Elem;
template <> struct Elem<f16_t> {
    static constexpr int kBytes = 2;
};
template <> struct Elem<bf16_t> {
    static constexpr int kBytes = 2;
};
template <> struct Elem<e4m3_t> {
    static constexpr int kBytes = 1;
};
template <> struct Elem<e5m2_t> {
    static constexpr int kBytes = 1;
};
template <> struct Elem<i8_t> {
    static constexpr int kBytes = 1;
};

// ---------------------------------------------------------------------------
// two 8-bit cache codes (low byte first) -> f16x2, exact for every format:
// E4M3 and E5M2 values are f16 values, and so are the integers -127..127
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t cvt8x2_f16x2(uint32_t two, e4m3_t) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)two));
    return h2;
}
__device__ __forceinline__ uint32_t cvt8x2_f16x2(uint32_t two, e5m2_t) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)two));
    return h2;
}
// Four codes of one word (low byte first) -> two f16x2: codes 0, 1 in lo and
// 2, 3 in hi.  The word is split into its two 16-bit halves inside the asm, so
// no shift is needed to reach the high pair.
__device__ __forceinline__ void cvt8x4_halves(uint32_t w, uint32_t &lo, uint32_t &hi, e4m3_t) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}
__device__ __forceinline__ void cvt8x4_halves(uint32_t w, uint32_t &lo, uint32_t &hi, e5m2_t) {
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e5m2x2 %0, l;\n\tcvt.rn.f16x2.e5m2x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}
// INT8: the biased byte b ^ 0x80 = b + 128 becomes the low mantissa byte of an
// f16 with exponent byte 0x64 (the value 1024 + b + 128, exact); subtracting
// 1152 leaves b.
__device__ __forceinline__ uint32_t cvt8x2_f16x2(uint32_t two, i8_t) {
    uint32_t h2;
    asm("prmt.b32 %0, %1, %2, 0x5140;" : "=r"(h2) : "r"((two ^ 0x8080u) & 0xFFFFu), "r"(0x6464u));
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h2), "r"(0x64806480u));
    return r;
}

// Two packed 16-bit values -> two floats (exact).
__device__ __forceinline__ void unpack2(f16_t, uint32_t w, float &lo, float &hi) {
    __half2 h = *reinterpret_cast<__half2 *>(&w);
    float2 f = __half22float2(h);
    lo = f.x;
    hi = f.y;
}
__device__ __forceinline__ void unpack2(bf16_t, uint32_t w, float &lo, float &hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
}

// Two packed E4M3 codes (low byte first) -> two floats (exact: every E4M3
// value is an f16 value).
__device__ __forceinline__ void unpack2_e4m3(uint16_t w, float &lo, float &hi) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(w));
    __half2 h = *reinterpret_cast<__half2 *>(&h2);
    float2 f = __half22float2(h);
    lo = f.x;
    hi = f.y;
}

// Two packed 8-bit codes (low byte first) -> two floats (exact).
template <typename T> __device__ __forceinline__ void unpack2_8(uint32_t two, float &lo, float &hi) {
    const uint32_t h2 = cvt8x2_f16x2(two, T{});
    __half2 h = *reinterpret_cast<const __half2 *>(&h2);
    float2 f = __half22float2(h);
    lo = f.x;
    hi = f.y;
}

// N consecutive elements held in registers (raw words) -> N floats.
template <typename T, int N> struct Unpack;
template <int N> struct Unpack<f16_t, N> {
    static __device__ __forceinline__ void run(const uint32_t *w, float *f) {
#pragma unroll
        for (int i = 0; i < N / 2; ++i) unpack2(f16_t{}, w[i], f[2 * i], f[2 * i + 1]);
    }
};
template <int N> struct Unpack<bf16_t, N> {
    static __device__ __forceinline__ void run(const uint32_t *w, float *f) {
#pragma unroll
        for (int i = 0; i < N / 2; ++i) unpack2(bf16_t{}, w[i], f[2 * i], f[2 * i + 1]);
    }
};
template <int N> struct Unpack<e4m3_t, N> {
    static __device__ __forceinline__ void run(const uint32_t *w, float *f) {
#pragma unroll
        for (int i = 0; i < N / 4; ++i) {
            unpack2_e4m3((uint16_t)(w[i] & 0xFFFFu), f[4 * i], f[4 * i + 1]);
            unpack2_e4m3((uint16_t)(w[i] >> 16), f[4 * i + 2], f[4 * i + 3]);
        }
        if constexpr (N % 4 == 2) unpack2_e4m3((uint16_t)(w[N / 4] & 0xFFFFu), f[N - 2], f[N - 1]);
    }
};
template <typename T8, int N> struct Unpack8 {
    static __device__ __forceinline__ void run(const uint32_t *w, float *f) {
#pragma unroll
        for (int i = 0; i < N / 4; ++i) {
            unpack2_8<T8>(w[i] & 0xFFFFu, f[4 * i], f[4 * i + 1]);
            unpack2_8<T8>(w[i] >> 16, f[4 * i + 2], f[4 * i + 3]);
        }
        if constexpr (N % 4 == 2) unpack2_8<T8>(w[N / 4] & 0xFFFFu, f[N - 2], f[N - 1]);
    }
};
template <int N> struct Unpack<e5m2_t, N> : Unpack8<e5m2_t, N> {};
template <int N> struct Unpack<i8_t, N> : Unpack8<i8_t, N> {};

__device__ __forceinline__ float to_float(f16_t, uint16_t b) {
    return __half2float(__ushort_as_half(b));
}
__device__ __forceinline__ float to_float(bf16_t, uint16_t b) {
    return __uint_as_float((uint32_t)b << 16);
}
__device__ __forceinline__ uint16_t from_float(f16_t, float x) {
    return __half_as_ushort(__float2half_rn(x));
}
__device__ __forceinline__ uint16_t from_float(bf16_t, float x) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// ---------------------------------------------------------------------------
// quantisation of the cache write (shared by every path that stores 8-bit
// codes, so they agree bit for bit): y = x / scale in fp32 with IEEE
// division, then
//   E4M3 / E5M2: round to nearest even onto the format, saturating to the
//                largest finite value (+-448 / +-57344), NaN -> NaN;
//   INT8:        round half to even to an integer, clamped to [-127, 127].
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint16_t code8x2(float first, float second, e4m3_t) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(second), "f"(first));
    return r;
}
__device__ __forceinline__ uint16_t code8x2(float first, float second, e5m2_t) {
    uint16_t r;
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(second), "f"(first));
    return r;
}
__device__ __forceinline__ uint32_t int8_code(float y) {
    int v = __float2int_rn(y);  // NaN -> 0
    v = v > 127 ? 127 : (v < -127 ? -127 : v);
    return (uint32_t)v & 0xFFu;
}
__device__ __forceinline__ uint16_t code8x2(float first, float second, i8_t) {
    return (uint16_t)(int8_code(first) | (int8_code(second) << 8));
}

__device__ __forceinline__ uint16_t e4m3x2_rn_sat(float first, float second) {
    return code8x2(first, second, e4m3_t{});
}

// eight 16-bit activations -> eight 8-bit codes, one scale per element
// (per-channel scales)
template <typename ACT, typename KV>
__device__ __forceinline__ uint2 quantise8_chan(const uint4 &in, const float *scales) {
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
    float f[8];
    Unpack<ACT, 8>::run(w, f);
    uint16_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        c[i] = code8x2(__fdiv_rn(f[2 * i], scales[2 * i]), __fdiv_rn(f[2 * i + 1], scales[2 * i + 1]),
                       KV{});
    return make_uint2((uint32_t)c[0] | ((uint32_t)c[1] << 16), (uint32_t)c[2] | ((uint32_t)c[3] << 16));
}

// eight 16-bit activations (one uint4) -> eight 8-bit codes (one uint2)
template <typename ACT, typename KV = e4m3_t>
__device__ __forceinline__ uint2 quantise8(const uint4 &in, float scale) {
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
    float f[8];
    Unpack<ACT, 8>::run(w, f);
    uint16_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        c[i] = code8x2(__fdiv_rn(f[2 * i], scale), __fdiv_rn(f[2 * i + 1], scale), KV{});
    return make_uint2((uint32_t)c[0] | ((uint32_t)c[1] << 16), (uint32_t)c[2] | ((uint32_t)c[3] << 16));
}

// ---------------------------------------------------------------------------
// shared-memory loads of 2 / 4 / 8 / 16 bytes into 32-bit words
// ---------------------------------------------------------------------------

template <int BYTES> __device__ __forceinline__ void lds(uint32_t *w, uint32_t addr) {
    if constexpr (BYTES == 16) {
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                     : "r"(addr));
    } else if constexpr (BYTES == 8) {
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(addr));
    } else if constexpr (BYTES == 4) {
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[0]) : "r"(addr));
    } else {
        static_assert(BYTES == 2, "unsupported load width");
        uint16_t h;
        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h) : "r"(addr));
        w[0] = h;
    }
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier + bulk async copy
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred P1;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, P1;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of an mbarrier, giving up after `limit_ns`
// nanoseconds of wall time.  Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

// One bulk (non-tensor) global -> shared copy completing on `bar`.
// dst / src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Same, with an L2 eviction-priority policy (createpolicy) attached.
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void *src, uint32_t bytes,
                                              uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// ---------------------------------------------------------------------------
// programmatic dependent launch
// ---------------------------------------------------------------------------

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// device-side errors: the first one wins
// ---------------------------------------------------------------------------

__device__ __forceinline__ void flag_error(int *err, int code) {
    if (err) atomicCAS(err, 0, code);
}

}  // namespace pa
