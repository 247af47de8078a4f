// tc.cuh -- sm_100a fifth-generation tensor-core (tcgen05) and tensor-map TMA
// wrappers used by the prefill grouped GEMM: tensor-memory allocation, the
// shared-memory matrix descriptor and instruction descriptor of a
// bf16 x bf16 -> fp32 MMA with both operands K-major in the 128-byte swizzled
// layout, MMA issue / commit, tensor-memory loads, and 2-D tiled TMA loads
// (no multicast).
#pragma once
#include <stdint.h>

#include "rfx_device.cuh"

namespace rfx {

// ------------------------------------------------------ tensor memory ---

// Allocate `ncols` (a power of two >= 32) tensor-memory columns for this CTA;
// the base address is written to *dst (shared memory).  Whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// --------------------------------------------------------- descriptors ---

// Shared-memory matrix descriptor of a K-major operand tile stored in the
// 128-byte swizzled layout: rows of 64 bf16 (128 B), 8-row atoms of 1024 B
// placed back to back (stride between atoms 1024 B), the 16-byte chunk c of
// row r stored at chunk position c ^ (r % 8).  Fields: start address >> 4 in
// bits [0,14), leading byte offset >> 4 in [16,30) (1: unused by swizzled
// K-major layouts), stride byte offset >> 4 in [32,46), descriptor version 1
// in [46,48), base offset 0 (atoms 1024-byte aligned), layout type 2
// (128-byte swizzle) in [61,64).  Advancing K by 16 elements within the atom
// adds 32 B to the start address.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// Instruction descriptor of kind::f16 with bf16 A and B, fp32 accumulator,
// both operands K-major, M = 128 and the given N (a multiple of 16, 16..256):
// accumulator format bits [4,6) = 1, A format [7,10) = 1 (bf16), B format
// [10,13) = 1, N >> 3 in [17,23), M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t idesc_bf16_m128(uint32_t n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}
static_assert(idesc_bf16_m128(256) == 0x08400490u, "instruction descriptor bit layout");

// D[tmem] (+)= A[smem] * B[smem]^T, one 128 x N x 16 step; issued by one thread.
__device__ __forceinline__ void tc_mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 lanes x 16 columns of 32-bit tensor memory: thread i of the warp gets
// lane (taddr.lane + i), columns taddr.col .. +15.  The warp may only touch
// the 32-lane quarter (warp id % 4).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t v[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ TMA ---

// 2-D tiled load of the tensor map's box at (c0 = inner element, c1 = row)
// into shared memory; completion counted on `bar` in bytes.  No multicast.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int c0, int c1, uint64_t* bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// Bring the tensor map's box at (c0, c1) into L2 (no shared memory, no completion).
__device__ __forceinline__ void tma_prefetch_l2_2d(const void* tmap, int c0, int c1) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(reinterpret_cast<uint64_t>(tmap)),
                 "r"(c0), "r"(c1)
                 : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// ------------------------------------------------- exact bf16 dequant ---

// Two codes at mantissa bits [S, S+b) of each half of `v`, with the fp16
// exponent of 2^(10-S) or-ed in, are the fp16 values 2^(10-S) + c.  With
// C = -(2^(10-S) + off) * s in fp32, the mixed-precision FMA
// v_half * s_half + C yields (c - off) * s exactly (the product of two fp16
// numbers and the sum are exact in fp32 because (c - off) * s needs at most
// 15 significant bits and C at most 23), and one round-to-nearest-even
// conversion gives bf16(level * scale) for both elements.  HS selects the
// scale half (row g or row g+8) of the packed fp16 scale pair.
template <int HS>
__device__ __forceinline__ uint32_t deq_pair_f16scale(uint32_t v, uint32_t sc, float C) {
    uint32_t out;
    asm("{\n\t.reg .f16 a0, a1, s0, s1;\n\t.reg .f32 f0, f1;\n\t"
        "mov.b32 {a0, a1}, %1;\n\t"
        "mov.b32 {s0, s1}, %2;\n\t"
        "fma.rn.f32.f16 f0, a0, s%4, %3;\n\t"
        "fma.rn.f32.f16 f1, a1, s%4, %3;\n\t"
        "cvt.rn.bf16x2.f32 %0, f1, f0;\n\t}"
        : "=r"(out)
        : "r"(v), "r"(sc), "f"(C), "n"(HS));
    return out;
}

// The same for a power-of-two fp32 scale s: (v_half * 1 + K) is the level,
// exact; times s is exact unless it leaves the fp32 range (as the bf16 value
// would).
__device__ __forceinline__ uint32_t deq_pair_pow2scale(uint32_t v, float K, float s) {
    uint32_t out;
    asm("{\n\t.reg .f16 a0, a1, one;\n\t.reg .f32 f0, f1;\n\t"
        "mov.b32 {a0, a1}, %1;\n\t"
        "mov.b16 one, 0x3C00;\n\t"
        "fma.rn.f32.f16 f0, a0, one, %2;\n\t"
        "fma.rn.f32.f16 f1, a1, one, %2;\n\t"
        "mul.rn.f32 f0, f0, %3;\n\t"
        "mul.rn.f32 f1, f1, %3;\n\t"
        "cvt.rn.bf16x2.f32 %0, f1, f0;\n\t}"
        : "=r"(out)
        : "r"(v), "f"(K), "f"(s));
    return out;
}

// The exact values of deq_pair_f16scale / deq_pair_pow2scale as bf16 pairs
// hi + lo: hi = bf16(w), lo = bf16(w - hi).  w - hi is exact in fp32, and
// since w = level * scale has at most 15 significant bits (11 of a binary16
// scale, 4 of a level), lo holds it exactly.
__device__ __forceinline__ void bf16_hilo(float f0, float f1, uint32_t& hi, uint32_t& lo) {
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(hi) : "f"(f1), "f"(f0));
    const float r0 = f0 - __uint_as_float(hi << 16), r1 = f1 - __uint_as_float(hi & 0xffff0000u);
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(lo) : "f"(r1), "f"(r0));
}
template <int HS>
__device__ __forceinline__ void deq_pair_f16scale_hilo(uint32_t v, uint32_t sc, float C, uint32_t& hi, uint32_t& lo) {
    float f0, f1;
    asm("{\n\t.reg .f16 a0, a1, s0, s1;\n\t"
        "mov.b32 {a0, a1}, %2;\n\t"
        "mov.b32 {s0, s1}, %3;\n\t"
        "fma.rn.f32.f16 %0, a0, s%5, %4;\n\t"
        "fma.rn.f32.f16 %1, a1, s%5, %4;\n\t}"
        : "=f"(f0), "=f"(f1)
        : "r"(v), "r"(sc), "f"(C), "n"(HS));
    bf16_hilo(f0, f1, hi, lo);
}
__device__ __forceinline__ void deq_pair_pow2scale_hilo(uint32_t v, float K, float s, uint32_t& hi, uint32_t& lo) {
    float f0, f1;
    asm("{\n\t.reg .f16 a0, a1, one;\n\t"
        "mov.b32 {a0, a1}, %2;\n\t"
        "mov.b16 one, 0x3C00;\n\t"
        "fma.rn.f32.f16 %0, a0, one, %3;\n\t"
        "fma.rn.f32.f16 %1, a1, one, %3;\n\t}"
        : "=f"(f0), "=f"(f1)
        : "r"(v), "f"(K));
    bf16_hilo(f0 * s, f1 * s, hi, lo);
}

// 16-byte asynchronous copy global -> shared through the load/store unit
// (completion tracked per thread: commit a group, then wait for it).
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* src, uint64_t policy) {
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(saddr), "l"(src), "l"(policy)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void sts32(uint32_t saddr, uint32_t v) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(saddr), "r"(v) : "memory");
}

}  // namespace rfx
