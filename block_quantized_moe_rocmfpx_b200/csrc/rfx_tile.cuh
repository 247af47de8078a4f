// rfx_tile.cuh -- per-chunk tensor-core work on packed ROCmFPX-style codes.
//
// A "chunk" is up to 8 tiles (16 rows x one 32-weight block each) of one
// row-group (layout in include/rfx.h).  Every packed block is decoded once in
// registers and multiplied against the B fragments of all the token columns at
// once (decode once, apply to every verify column: ainomam.com, "APU 实现 token
// 自由…", section "Lucebox 的优化三板斧").
//
// Full chunks (8 tiles) use the plane layout: the 8 A-registers of tile b sit
// at one bit offset s_b in 8 different words, so a single AND turns each into
// two fp16 subnormals of value code * 2^(s_b - 24).  The tensor core computes
// sum_k code_k * B_k exactly; with level = code - off, the block dot product is
//     sum_k level_k B_k = sum_k code_k B_k - off * sum_k B_k,
// so each lane also accumulates scale * (block sum of B) and subtracts off times
// it at the end.  The 2^(s_b - 24) factor is removed either by pre-scaling the
// B operand by 2^-s_b (gate/up: x is staged that way) or by keeping one
// accumulator per distinct s_b (down: h is used as it is).  Partial chunks use
// the per-tile layout and an exact magic-exponent decode of the levels.
#pragma once
#include "rfx_device.cuh"
#include "rfx_layout.h"

namespace rfx {

__device__ __forceinline__ uint2 lds64(const uint8_t* p) { return *reinterpret_cast<const uint2*>(p); }
__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ uint32_t lds32(const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); }
__device__ __forceinline__ uint32_t lds16(const uint8_t* p) { return *reinterpret_cast<const uint16_t*>(p); }
__device__ __forceinline__ float4 ldsf4(const uint8_t* p) { return *reinterpret_cast<const float4*>(p); }

// B-operand source: 4 fp16 values (k = 2t, 2t+1, 2t+8, 2t+9 of a k16 step)
// per lane at base + step * stride; lanes whose column is empty read zero.
struct BSrc {
    const uint8_t* base;
    int stride;
    bool valid;
    __device__ __forceinline__ uint2 get(int step) const {
        uint2 v = make_uint2(0u, 0u);
        if (valid) v = lds64(base + step * stride);
        return v;
    }
};

// B-operand source with a compile-time step stride (STRIDE > 0) or a run-time
// one (STRIDE == 0), and no predicate: a lane whose column is empty points at
// a real column, whose products only reach output columns that are dropped.
template <int STRIDE>
struct BSrcK {
    const uint8_t* base;
    int stride;
    __device__ __forceinline__ uint2 get(int step) const {
        return lds64(base + step * (STRIDE > 0 ? STRIDE : stride));
    }
};

// --------------------------------------------------------- plane layout ---

// Shift exponent s_b of tile b of a full chunk (bit offset of its fields after
// the optional pre-shift), and the number of distinct values.
template <int FMT> struct Plane {
    static constexpr int NW = 4 * FMT;           // code words per lane
    static constexpr int NSW = FMT == 4 ? 4 : 8;  // scale words per g
    static constexpr int CODE_BYTES = 8 * 16 * FMT * 4;
    static constexpr float OFF = ((1 << FMT) - 1) * 0.5f;
    static constexpr int NCLS = FMT == 2 ? 5 : (FMT == 3 ? 3 : 2);
    __host__ __device__ static constexpr int s_of(int b) {
        return FMT == 2 ? (b < 5 ? 2 * b : 2 * b - 10)
                        : (FMT == 3 ? (b == 0 || b == 3 || b == 5 ? 0 : (b == 2 || b == 7 ? 6 : 3)) : 4 * (b & 1));
    }
    __host__ __device__ static constexpr int cls_of(int b) { return s_of(b) / (FMT == 2 ? 2 : (FMT == 3 ? 3 : 4)); }
    __host__ __device__ static constexpr int s_of_cls(int c) { return c * (FMT == 2 ? 2 : (FMT == 3 ? 3 : 4)); }
};

template <int BITS, int S>
__device__ __forceinline__ uint32_t fld(uint32_t w) {
    constexpr uint32_t m = ((1u << BITS) - 1u) << S;
    return w & (m | (m << 16));
}

// The 8 A registers of tile B of a full chunk; W = lane words, Wsh = W >> (10,
// 9, 8 for FP2, FP3, FP4).
template <int FMT, int B>
__device__ __forceinline__ void plane_regs(const uint32_t* W, const uint32_t* Wsh, uint32_t a[8]) {
    constexpr int S = Plane<FMT>::s_of(B);
    if constexpr (FMT == 2) {
#pragma unroll
        for (int r = 0; r < 8; ++r) a[r] = fld<2, S>(B < 5 ? W[r] : Wsh[r]);
    } else if constexpr (FMT == 4) {
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int wi = (B < 4 ? 0 : 8) + r;
            a[r] = fld<4, S>((B & 2) ? Wsh[wi] : W[wi]);
        }
    } else {
        if constexpr (B < 3) {
#pragma unroll
            for (int r = 0; r < 8; ++r) a[r] = fld<3, S>(W[r]);
        } else if constexpr (B < 5) {
#pragma unroll
            for (int r = 0; r < 8; ++r) a[r] = fld<3, S>(Wsh[r]);
        } else if constexpr (B < 7) {
#pragma unroll
            for (int r = 0; r < 4; ++r) a[r] = fld<3, S>(W[8 + r]);
#pragma unroll
            for (int r = 0; r < 4; ++r) a[4 + r] = fld<3, S>(Wsh[8 + r]);
        } else {
#pragma unroll
            for (int r = 0; r < 4; ++r) a[r] = fld<3, 6>(W[8 + r]);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t w0 = W[3 * j], w1 = W[3 * j + 1], w2 = W[3 * j + 2];
                a[4 + j] = ((w0 >> 9) & 0x00400040u) | ((w1 >> 8) & 0x00800080u) | ((w2 >> 7) & 0x01000100u);
            }
        }
    }
}

template <int FMT>
__device__ __forceinline__ void plane_shift(const uint32_t* W, uint32_t* Wsh) {
    constexpr int SH = FMT == 2 ? 10 : (FMT == 3 ? 9 : 8);
#pragma unroll
    for (int i = 0; i < Plane<FMT>::NW; ++i) Wsh[i] = W[i] >> SH;
}

// Lane words and scale words of a full chunk.
template <int FMT>
struct FullChunk {
    uint32_t wd[Plane<FMT>::NW];
    uint32_t sh[Plane<FMT>::NW];
    uint32_t sc[Plane<FMT>::NSW];
    // slab-major chunk (rfx_layout.h): every 128-bit load of the warp reads
    // 512 contiguous code bytes or 128 contiguous scale bytes
    __device__ __forceinline__ void load(const uint8_t* st, int lane, int g) {
        constexpr int NW = Plane<FMT>::NW, NSW = Plane<FMT>::NSW;
#pragma unroll
        for (int i = 0; i < NW / 4; ++i) {
            uint4 v = lds128(st + (i * 32 + lane) * 16);
            wd[4 * i] = v.x; wd[4 * i + 1] = v.y; wd[4 * i + 2] = v.z; wd[4 * i + 3] = v.w;
        }
#pragma unroll
        for (int i = 0; i < NSW / 4; ++i) {
            uint4 v = lds128(st + Plane<FMT>::CODE_BYTES + (i * 8 + g) * 16);
            sc[4 * i] = v.x; sc[4 * i + 1] = v.y; sc[4 * i + 2] = v.z; sc[4 * i + 3] = v.w;
        }
        plane_shift<FMT>(wd, sh);
    }
    __device__ __forceinline__ void scales(int b, float& s0, float& s1) const {
        if constexpr (FMT == 4) {
            uint32_t w = sc[b >> 1] >> (16 * (b & 1));
            s0 = scale_e8m0(w & 0xFFu);
            s1 = scale_e8m0((w >> 8) & 0xFFu);
        } else {
            float2 f = scale_f16x2(sc[b]);
            s0 = f.x; s1 = f.y;
        }
    }
};

// acc[i] (i = 0..3: rows g,g,g+8,g+8 x cols 2t,2t+1,2t,2t+1) and the matching
// offset-correction sums.
struct AccA {
    float acc[4];
    float corr[4];
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < 4; ++i) { acc[i] = 0.f; corr[i] = 0.f; }
    }
};

__device__ __forceinline__ void mma_tile(float c[4], const uint32_t a[8], uint2 blo, uint2 bhi) {
    const float z[4] = {0.f, 0.f, 0.f, 0.f};
    mma16816<true>(c, a, blo.x, blo.y, z);
    mma16816<true>(c, a + 4, bhi.x, bhi.y, c);
}

// One full gate/up chunk pair sharing the x fragments (x pre-scaled by
// 2^-s_b): all tiles accumulate in units of 2^-24.  S[b] / S1[b] are the
// block sums of the lane's two columns; TWO = the second column can be live.
// FC: the format whose bit offsets s'_b the x fragments were pre-scaled for.
// When FC != FMT, 2^(s'_b - s_b) goes on the products' scales (a power of
// two: exact); the block sums, which do not depend on the offsets, keep the
// raw scale.
template <int FMT, int FC, bool TWO, class SRC>
__device__ __forceinline__ void chunkA_full(const uint8_t* st0, const uint8_t* st1, int lane, int g, const SRC& bs,
                                            int step0, const float* S0, const float* S1, AccA& ag, AccA& au) {
    constexpr bool COMP = FC != FMT;
    FullChunk<FMT> f0, f1;
    f0.load(st0, lane, g);
    f1.load(st1, lane, g);
#pragma unroll
    for (int b = 0; b < 8; ++b) {
        const uint2 blo = bs.get(step0 + 2 * b), bhi = bs.get(step0 + 2 * b + 1);
        uint32_t a[8];
        float c[4], s0, s1;
        switch (b) {
            case 0: plane_regs<FMT, 0>(f0.wd, f0.sh, a); break;
            case 1: plane_regs<FMT, 1>(f0.wd, f0.sh, a); break;
            case 2: plane_regs<FMT, 2>(f0.wd, f0.sh, a); break;
            case 3: plane_regs<FMT, 3>(f0.wd, f0.sh, a); break;
            case 4: plane_regs<FMT, 4>(f0.wd, f0.sh, a); break;
            case 5: plane_regs<FMT, 5>(f0.wd, f0.sh, a); break;
            case 6: plane_regs<FMT, 6>(f0.wd, f0.sh, a); break;
            default: plane_regs<FMT, 7>(f0.wd, f0.sh, a); break;
        }
        mma_tile(c, a, blo, bhi);
        f0.scales(b, s0, s1);
        const float cmb = __int_as_float((127 + Plane<FC>::s_of(b) - Plane<FMT>::s_of(b)) << 23);
        float p0 = s0, p1 = s1;
        if (COMP) { p0 *= cmb; p1 *= cmb; }
        ag.acc[0] = fmaf(p0, c[0], ag.acc[0]);
        ag.acc[2] = fmaf(p1, c[2], ag.acc[2]);
        ag.corr[0] = fmaf(s0, S0[b], ag.corr[0]);
        ag.corr[2] = fmaf(s1, S0[b], ag.corr[2]);
        if (TWO) {
            ag.acc[1] = fmaf(p0, c[1], ag.acc[1]);
            ag.acc[3] = fmaf(p1, c[3], ag.acc[3]);
            ag.corr[1] = fmaf(s0, S1[b], ag.corr[1]);
            ag.corr[3] = fmaf(s1, S1[b], ag.corr[3]);
        }
        switch (b) {
            case 0: plane_regs<FMT, 0>(f1.wd, f1.sh, a); break;
            case 1: plane_regs<FMT, 1>(f1.wd, f1.sh, a); break;
            case 2: plane_regs<FMT, 2>(f1.wd, f1.sh, a); break;
            case 3: plane_regs<FMT, 3>(f1.wd, f1.sh, a); break;
            case 4: plane_regs<FMT, 4>(f1.wd, f1.sh, a); break;
            case 5: plane_regs<FMT, 5>(f1.wd, f1.sh, a); break;
            case 6: plane_regs<FMT, 6>(f1.wd, f1.sh, a); break;
            default: plane_regs<FMT, 7>(f1.wd, f1.sh, a); break;
        }
        mma_tile(c, a, blo, bhi);
        f1.scales(b, s0, s1);
        p0 = s0; p1 = s1;
        if (COMP) { p0 *= cmb; p1 *= cmb; }
        au.acc[0] = fmaf(p0, c[0], au.acc[0]);
        au.acc[2] = fmaf(p1, c[2], au.acc[2]);
        au.corr[0] = fmaf(s0, S0[b], au.corr[0]);
        au.corr[2] = fmaf(s1, S0[b], au.corr[2]);
        if (TWO) {
            au.acc[1] = fmaf(p0, c[1], au.acc[1]);
            au.acc[3] = fmaf(p1, c[3], au.acc[3]);
            au.corr[1] = fmaf(s0, S1[b], au.corr[1]);
            au.corr[3] = fmaf(s1, S1[b], au.corr[3]);
        }
    }
}

// Down projection accumulators: one per distinct bit offset (class) and per
// n-block of virtual columns (hi / lo halves of h), plus the per-row
// correction sums of the lane's real column.
template <int NB>
struct AccB {
    float acc[5][NB][4];
    float corr[NB][2];
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int c = 0; c < 5; ++c)
#pragma unroll
            for (int n = 0; n < NB; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[c][n][i] = 0.f;
#pragma unroll
        for (int n = 0; n < NB; ++n) { corr[n][0] = 0.f; corr[n][1] = 0.f; }
    }
};

// One full down chunk (B operands: hi/lo fp16 pairs of h * 2^n, n a
// power-of-two exponent per column and 32-block).  Sb[n][b] = block sum of
// the staged h for the lane's real column of n-block n; Hs[n][b] = 2^-n of
// that column and block, folded into the weight scale of the tile (exact).
template <int FMT, int NB, class SRC>
__device__ __forceinline__ void chunkB_full(const uint8_t* st, int lane, int g, const SRC* bs, int step0,
                                            const float (*Sb)[8], const float (*Hs)[8], AccB<NB>& ab) {
    FullChunk<FMT> f;
    f.load(st, lane, g);
#pragma unroll
    for (int b = 0; b < 8; ++b) {
        uint32_t a[8];
        switch (b) {
            case 0: plane_regs<FMT, 0>(f.wd, f.sh, a); break;
            case 1: plane_regs<FMT, 1>(f.wd, f.sh, a); break;
            case 2: plane_regs<FMT, 2>(f.wd, f.sh, a); break;
            case 3: plane_regs<FMT, 3>(f.wd, f.sh, a); break;
            case 4: plane_regs<FMT, 4>(f.wd, f.sh, a); break;
            case 5: plane_regs<FMT, 5>(f.wd, f.sh, a); break;
            case 6: plane_regs<FMT, 6>(f.wd, f.sh, a); break;
            default: plane_regs<FMT, 7>(f.wd, f.sh, a); break;
        }
        float s0, s1;
        f.scales(b, s0, s1);
        const int cls = Plane<FMT>::cls_of(b);
#pragma unroll
        for (int n = 0; n < NB; ++n) {
            float c[4];
            mma_tile(c, a, bs[n].get(step0 + 2 * b), bs[n].get(step0 + 2 * b + 1));
            const float s0n = s0 * Hs[n][b], s1n = s1 * Hs[n][b];
            ab.acc[cls][n][0] = fmaf(s0n, c[0], ab.acc[cls][n][0]);
            ab.acc[cls][n][1] = fmaf(s0n, c[1], ab.acc[cls][n][1]);
            ab.acc[cls][n][2] = fmaf(s1n, c[2], ab.acc[cls][n][2]);
            ab.acc[cls][n][3] = fmaf(s1n, c[3], ab.acc[cls][n][3]);
            ab.corr[n][0] = fmaf(s0n, Sb[n][b], ab.corr[n][0]);
            ab.corr[n][1] = fmaf(s1n, Sb[n][b], ab.corr[n][1]);
        }
    }
}

// ------------------------------------------------------- partial chunks ---

// Registers (exact levels, fp16) and scales of tile b of a partial chunk
// (nt < 8 tiles, per-tile layout).
template <int FMT>
__device__ __forceinline__ void partial_tile(const uint8_t* st, int nt, int lane, int g, int b, uint32_t a[8],
                                             float& s0, float& s1) {
    const int code_bytes = nt * 16 * FMT * 4;
    if constexpr (FMT == 2) {
        unpack_fp2<true>(lds32(st + lane * 4 * nt + 4 * b), a);
        float2 f = scale_f16x2(lds32(st + code_bytes + (g * nt + b) * 4));
        s0 = f.x; s1 = f.y;
    } else if constexpr (FMT == 4) {
        const uint8_t* p = st + lane * 8 * nt + 8 * b;
        unpack_fp4_word<true>(lds32(p), a);
        unpack_fp4_word<true>(lds32(p + 4), a + 4);
        uint32_t e = lds16(st + code_bytes + (g * nt + b) * 2);
        s0 = scale_e8m0(e & 0xFFu);
        s1 = scale_e8m0(e >> 8);
    } else {
        const uint8_t* lp = st + lane * 6 * nt;       // 2-byte aligned
        const int pair = b >> 1;
        const bool lone = (b == nt - 1) && (nt & 1);
        const uint8_t* p = lp + 12 * pair;
        if (lone) {
            uint64_t s = (uint64_t)lds16(p) | ((uint64_t)lds16(p + 2) << 16) | ((uint64_t)lds16(p + 4) << 32);
            unpack_fp3_lone<true>(s, a);
        } else {
            uint32_t w0 = lds16(p) | (lds16(p + 2) << 16);
            uint32_t w1 = lds16(p + 4) | (lds16(p + 6) << 16);
            uint32_t w2 = lds16(p + 8) | (lds16(p + 10) << 16);
            uint32_t r[16];
            unpack_fp3_pair<true>(w0, w1, w2, r);
#pragma unroll
            for (int i = 0; i < 8; ++i) a[i] = (b & 1) ? r[8 + i] : r[i];
        }
        float2 f = scale_f16x2(lds32(st + code_bytes + (g * nt + b) * 4));
        s0 = f.x; s1 = f.y;
    }
}

// A partial chunk adds s * (exact level dot product) in units of 2^-24 so that
// it shares the full chunks' accumulator (no offset correction: levels exact).
// The 2^-24 goes on the dot product, not on the scale: an E8M0 scale of 2^-127
// times 2^-24 would fall below fp32's smallest subnormal.
template <int FMT, bool TWO, class SRC>
__device__ __forceinline__ void chunkA_partial(const uint8_t* st0, const uint8_t* st1, int nt, int lane, int g,
                                               const SRC& bs, int step0, AccA& ag, AccA& au) {
    for (int b = 0; b < nt; ++b) {
        const uint2 blo = bs.get(step0 + 2 * b), bhi = bs.get(step0 + 2 * b + 1);
        uint32_t a[8];
        float c[4], s0, s1;
        partial_tile<FMT>(st0, nt, lane, g, b, a, s0, s1);
        mma_tile(c, a, blo, bhi);
        ag.acc[0] = fmaf(s0, c[0] * 0x1.0p-24f, ag.acc[0]); ag.acc[1] = fmaf(s0, c[1] * 0x1.0p-24f, ag.acc[1]);
        ag.acc[2] = fmaf(s1, c[2] * 0x1.0p-24f, ag.acc[2]); ag.acc[3] = fmaf(s1, c[3] * 0x1.0p-24f, ag.acc[3]);
        partial_tile<FMT>(st1, nt, lane, g, b, a, s0, s1);
        mma_tile(c, a, blo, bhi);
        au.acc[0] = fmaf(s0, c[0] * 0x1.0p-24f, au.acc[0]); au.acc[1] = fmaf(s0, c[1] * 0x1.0p-24f, au.acc[1]);
        au.acc[2] = fmaf(s1, c[2] * 0x1.0p-24f, au.acc[2]); au.acc[3] = fmaf(s1, c[3] * 0x1.0p-24f, au.acc[3]);
    }
}

template <int FMT, int NB, class SRC>
__device__ __forceinline__ void chunkB_partial(const uint8_t* st, int nt, int lane, int g, const SRC* bs, int step0,
                                               const float (*Hs)[8], AccB<NB>& ab) {
    for (int b = 0; b < nt; ++b) {
        uint32_t a[8];
        float s0, s1;
        partial_tile<FMT>(st, nt, lane, g, b, a, s0, s1);
#pragma unroll
        for (int n = 0; n < NB; ++n) {
            float c[4];
            mma_tile(c, a, bs[n].get(step0 + 2 * b), bs[n].get(step0 + 2 * b + 1));
            const float s0n = s0 * Hs[n][b], s1n = s1 * Hs[n][b];
            // class 0 is scaled by 2^24 at the end
            ab.acc[0][n][0] = fmaf(s0n, c[0] * 0x1.0p-24f, ab.acc[0][n][0]);
            ab.acc[0][n][1] = fmaf(s0n, c[1] * 0x1.0p-24f, ab.acc[0][n][1]);
            ab.acc[0][n][2] = fmaf(s1n, c[2] * 0x1.0p-24f, ab.acc[0][n][2]);
            ab.acc[0][n][3] = fmaf(s1n, c[3] * 0x1.0p-24f, ab.acc[0][n][3]);
        }
    }
}

// Final per-lane values.  A: 2^24 * acc - off * corr (x16 units).
template <int FMT>
__device__ __forceinline__ void finishA(const AccA& a, float v[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = fmaf(-Plane<FMT>::OFF, a.corr[i], a.acc[i] * 0x1.0p24f);
}

// B: sum_cls 2^(24 - s_cls) acc[cls] - off * corr, the correction folded into
// the hi virtual column (v[n][0], v[n][2]).
template <int FMT, int NB>
__device__ __forceinline__ void finishB(const AccB<NB>& a, float v[NB][4]) {
#pragma unroll
    for (int n = 0; n < NB; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float s = 0.f;
#pragma unroll
            for (int c = Plane<FMT>::NCLS - 1; c >= 0; --c)
                s = fmaf(a.acc[c][n][i], __int_as_float((127 + 24 - Plane<FMT>::s_of_cls(c)) << 23), s);
            v[n][i] = s;
        }
#pragma unroll
    for (int n = 0; n < NB; ++n) {
        v[n][0] = fmaf(-Plane<FMT>::OFF, a.corr[n][0], v[n][0]);
        v[n][2] = fmaf(-Plane<FMT>::OFF, a.corr[n][1], v[n][2]);
    }
}

}  // namespace rfx
