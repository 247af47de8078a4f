// rfx_device.cuh -- sm_100a device primitives: mbarrier / bulk-copy (TMA)
// wrappers with bounded waits, legacy tensor-core mma.sync, and the exact
// in-register dequantisation of packed ROCmFPX-style codes into m16n8k16 A
// fragments.
//
// Dequantisation (format of [TZ] taozi.news, "DeepSeek V4 Flash 在 128GB 锐龙
// AI MAX+ 上跑到 32 tok/s", section "ROCmFPX：把 284B 权重压进 128 GB", with this
// library's level reading level = c - (2^b - 1)/2): a b-bit code c sitting at
// mantissa bits [s, s+b) of a 16-bit float whose other mantissa bits are zero
// and whose exponent is that of M (128 for bf16, 1024 for fp16) has the value
// v = M + c*2^s.  One packed FMA v * 2^-s - (M*2^-s + (2^b-1)/2) gives the
// level exactly, because the level is representable and both constants are
// (s >= 1 keeps M*2^-s + off within 8 / 11 significant bits).  The block
// scale is applied afterwards in fp32, so the tensor-core products level * x
// are exact and the only rounding is fp32 accumulation.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace rfx {

// ------------------------------------------------------------------ misc ---

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

// Round a double to bf16 bits, nearest-even, in one step (no intermediate
// float rounding): sign, 8-bit exponent with bias 127, 7 explicit mantissa
// bits; values below 2^-126 become bf16 subnormals, values beyond the largest
// finite bf16 become infinity.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double v) {
    const unsigned long long d = (unsigned long long)__double_as_longlong(v);
    const uint32_t sign = (uint32_t)(d >> 48) & 0x8000u;
    const int e = (int)((d >> 52) & 0x7FF);
    const unsigned long long m = d & ((1ull << 52) - 1ull);
    if (e == 0x7FF) return (uint16_t)(sign | 0x7F80u | (m ? 0x40u : 0u));   // inf / nan
    if (e == 0) return (uint16_t)sign;                                       // zero (and fp64 subnormals)
    const int E = e - 1023;                                                  // unbiased exponent
    const unsigned long long sig = (1ull << 52) | m;                         // 53-bit significand
    int shift;                                                               // significand bits dropped
    int be;                                                                  // bf16 biased exponent before rounding
    if (E >= -126) {
        shift = 45;
        be = E + 127;
    } else {
        shift = 45 + (-126 - E);                                             // subnormal: fixed exponent 2^-126
        be = 0;
        if (shift > 54) return (uint16_t)sign;                               // rounds to zero
    }
    unsigned long long q = sig >> shift;
    const unsigned long long rem = sig & ((1ull << shift) - 1ull), half = 1ull << (shift - 1);
    if (rem > half || (rem == half && (q & 1ull))) ++q;
    // q holds the implicit bit (normal) at bit 7; a carry out of it bumps the exponent
    uint32_t bits;
    if (be > 0) {
        if (q >> 8) { q >>= 1; ++be; }
        if (be >= 255) return (uint16_t)(sign | 0x7F80u);
        bits = ((uint32_t)be << 7) | (uint32_t)(q & 0x7Fu);
    } else {
        bits = (uint32_t)q;   // subnormal; q == 0x80 is the smallest normal, which has the same bits
    }
    return (uint16_t)(sign | bits);
}

// silu(g) * u for g < -64, where sigmoid(g) equals exp(g) to fp32 precision.
// exp(g) is taken as exp(g + 64 ln 2) * 2^-64 so that the products stay in
// fp32's normal range while h itself is still representable (a plain
// g / (1 + exp(-g)) gives 0 below g = -88.7, where the true value is ~1e-37).
__device__ __forceinline__ float silu_mul_tail(float g, float u) {
    return (g * __expf(g + 44.3614195558365f) * u) * 0x1.0p-64f;
}

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue now, and wait until the previous kernel has finished and its
// writes are visible (a no-op when the launch had no such dependency).
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------- mbarrier ---

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking test of the phase with the given parity (try_wait may suspend
// the thread for a while; test_wait never does).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes or about `ns` nanoseconds pass, instead of re-issuing the
// test (a spinning warp takes issue slots from the warps doing the math).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Bounded wait on the phase with the given parity.  Returns false after about
// `limit_cycles` SM clocks without completion (the caller records an error and
// unwinds instead of hanging).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long limit_cycles) {
    if (mbar_try_wait(bar, parity)) return true;
    long long t0 = clock64();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, 1000000u)) return true;
        if (clock64() - t0 > limit_cycles) return false;
    }
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// L2 policy: weights are streamed once per pass; let them go first.
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

// 1-D bulk copy global -> shared (TMA unit, no tensor map, no multicast).
// dst/src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// ------------------------------------------------------- global atomics ---

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

__device__ __forceinline__ uint32_t atom_add_release_gpu(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Fire-and-forget add with release semantics (no return trip).
__device__ __forceinline__ void red_add_release_gpu(uint32_t* p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// 64-bit counters of the grid barriers (they only grow, so they never wrap in practice).
__device__ __forceinline__ unsigned long long atom_add_release_gpu_u64(unsigned long long* p, unsigned long long v) {
    unsigned long long old;
    asm volatile("atom.add.release.gpu.global.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
    return old;
}

__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// ------------------------------------------------------------------- mma ---

// D = A(16x16) * B(16x8) + C, fp32 accumulate; A/B bf16 (F16 = false) or fp16.
template <bool F16>
__device__ __forceinline__ void mma16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1, const float c[4]) {
    if constexpr (F16) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%10,%11,%12,%13};"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
              "f"(c[3]));
    } else {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%10,%11,%12,%13};"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
              "f"(c[3]));
    }
}

// -------------------------------------------------------- dequantisation ---

// Bits of an exactly representable value in a 16-bit float with `mb` mantissa
// bits and exponent bias `bias` (bf16: 7/127, fp16: 10/15).  Evaluated at
// compile time only; the static_asserts below check the constants used.
constexpr uint32_t f16like_bits(double v, int mb, int bias) {
    uint32_t s = v < 0 ? 1u : 0u;
    double a = v < 0 ? -v : v;
    int e = 0;
    while (a >= 2.0) { a /= 2.0; ++e; }
    while (a < 1.0) { a *= 2.0; --e; }
    double m = (a - 1.0) * (double)(1 << mb);
    return (s << 15) | ((uint32_t)(e + bias) << mb) | (uint32_t)m;
}
constexpr bool f16like_exact(double v, int mb) {
    double a = v < 0 ? -v : v;
    while (a >= 2.0) a /= 2.0;
    while (a < 1.0) a *= 2.0;
    double m = (a - 1.0) * (double)(1 << mb);
    return m == (double)(uint32_t)m;
}
constexpr uint32_t pair(uint32_t h) { return h | (h << 16); }

template <bool F16> struct Op {
    static constexpr int MB = F16 ? 10 : 7;
    static constexpr int BIAS = F16 ? 15 : 127;
    static constexpr double M = F16 ? 1024.0 : 128.0;
    static constexpr uint32_t MAGIC = pair(F16 ? 0x6400u : 0x4300u);
};

template <int B, int S, bool F16> struct Field {
    static constexpr double off = ((1 << B) - 1) / 2.0;
    static constexpr double mul = 1.0 / (double)(1 << S);
    static constexpr double add = -(Op<F16>::M / (double)(1 << S) + off);
    static_assert(S >= 1 && S + B <= Op<F16>::MB, "field must sit inside the mantissa, above bit 0");
    static_assert(f16like_exact(add, Op<F16>::MB), "offset constant must be exact");
    static constexpr uint32_t MASK = pair(((1u << B) - 1u) << S);
    static constexpr uint32_t MUL = pair(f16like_bits(mul, Op<F16>::MB, Op<F16>::BIAS));
    static constexpr uint32_t ADD = pair(f16like_bits(add, Op<F16>::MB, Op<F16>::BIAS));
};
static_assert(f16like_bits(1.0, 7, 127) == 0x3F80u, "bf16 1.0");
static_assert(f16like_bits(-65.5, 7, 127) == 0xC283u, "bf16 -65.5");
static_assert(f16like_bits(1.0, 10, 15) == 0x3C00u, "fp16 1.0");
static_assert(f16like_bits(-513.5, 10, 15) == 0xE003u, "fp16 -513.5");

template <bool F16>
__device__ __forceinline__ uint32_t fma2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    if constexpr (F16) asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    else asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Two codes at bits [S, S+B) of each half of u -> the two levels, exactly.
template <int B, int S, bool F16>
__device__ __forceinline__ uint32_t lv(uint32_t u) {
    using Fd = Field<B, S, F16>;
    return fma2<F16>((u & Fd::MASK) | Op<F16>::MAGIC, Fd::MUL, Fd::ADD);
}

// FP2: one word per tile, register r at bits 2r / 16+2r.
template <bool F16>
__device__ __forceinline__ void unpack_fp2(uint32_t w, uint32_t a[8]) {
    if constexpr (F16) {
        const uint32_t u0 = w << 1, u1 = w >> 7;
        a[0] = lv<2, 1, F16>(u0); a[1] = lv<2, 3, F16>(u0); a[2] = lv<2, 5, F16>(u0); a[3] = lv<2, 7, F16>(u0);
        a[4] = lv<2, 1, F16>(u1); a[5] = lv<2, 3, F16>(u1); a[6] = lv<2, 5, F16>(u1); a[7] = lv<2, 7, F16>(u1);
    } else {
        const uint32_t u0 = w << 1, u1 = w >> 5, u2 = w >> 11;
        a[0] = lv<2, 1, F16>(u0); a[1] = lv<2, 3, F16>(u0); a[2] = lv<2, 5, F16>(u0);
        a[3] = lv<2, 1, F16>(u1); a[4] = lv<2, 3, F16>(u1); a[5] = lv<2, 5, F16>(u1);
        a[6] = lv<2, 1, F16>(u2); a[7] = lv<2, 3, F16>(u2);
    }
}

// FP4: word m holds registers 4m..4m+3, field j at bits 4j / 16+4j.
template <bool F16>
__device__ __forceinline__ void unpack_fp4_word(uint32_t w, uint32_t a[4]) {
    if constexpr (F16) {
        const uint32_t u0 = w << 1, u1 = w >> 7;
        a[0] = lv<4, 1, F16>(u0); a[1] = lv<4, 5, F16>(u0);
        a[2] = lv<4, 1, F16>(u1); a[3] = lv<4, 5, F16>(u1);
    } else {
        a[0] = lv<4, 1, F16>(w << 1); a[1] = lv<4, 3, F16>(w >> 1);
        a[2] = lv<4, 3, F16>(w >> 5); a[3] = lv<4, 3, F16>(w >> 9);
    }
}

// FP3 tile pair: 3 words, register R < 15 at word R/5 field R%5 (bits 3p /
// 16+3p); register 15 spread over bit 15 / 31 of the three words.
template <bool F16>
__device__ __forceinline__ void unpack_fp3_word(uint32_t w, uint32_t a[5]) {
    if constexpr (F16) {
        const uint32_t u0 = w << 1, u1 = w >> 8;
        a[0] = lv<3, 1, F16>(u0); a[1] = lv<3, 4, F16>(u0); a[2] = lv<3, 7, F16>(u0);
        a[3] = lv<3, 1, F16>(u1); a[4] = lv<3, 4, F16>(u1);
    } else {
        const uint32_t u0 = w << 1, u1 = w >> 5, u2 = w >> 11;
        a[0] = lv<3, 1, F16>(u0); a[1] = lv<3, 4, F16>(u0);
        a[2] = lv<3, 1, F16>(u1); a[3] = lv<3, 4, F16>(u1);
        a[4] = lv<3, 1, F16>(u2);
    }
}

template <bool F16>
__device__ __forceinline__ uint32_t unpack_fp3_r15(uint32_t w0, uint32_t w1, uint32_t w2) {
    const uint32_t u = ((w0 >> 14) & 0x00020002u) | ((w1 >> 13) & 0x00040004u) | ((w2 >> 12) & 0x00080008u);
    return lv<3, 1, F16>(u);
}

template <bool F16>
__device__ __forceinline__ void unpack_fp3_pair(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t a[16]) {
    unpack_fp3_word<F16>(w0, a);
    unpack_fp3_word<F16>(w1, a + 5);
    unpack_fp3_word<F16>(w2, a + 10);
    a[15] = unpack_fp3_r15<F16>(w0, w1, w2);
}

// Lone FP3 tile: 48-bit stream, code 2r+e at bits 3(2r+e).
template <bool F16>
__device__ __forceinline__ void unpack_fp3_lone(uint64_t s, uint32_t a[8]) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        uint32_t lo = (uint32_t)(s >> (6 * r)) & 7u, hi = (uint32_t)(s >> (6 * r + 3)) & 7u;
        a[r] = lv<3, 1, F16>((lo << 1) | (hi << 17));
    }
}

// Scales -> fp32.  binary16 pair (rows g, g+8) in one word.
__device__ __forceinline__ float2 scale_f16x2(uint32_t w) {
    __half2 h = *reinterpret_cast<__half2*>(&w);
    return __half22float2(h);
}
// E8M0 byte -> 2^(e-127) as fp32 (e = 0 -> 2^-127, a subnormal).
__device__ __forceinline__ float scale_e8m0(uint32_t e) {
    return __uint_as_float(e ? (e << 23) : 0x00400000u);
}

}  // namespace rfx
