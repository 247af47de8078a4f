// rfx_tile.cuh -- per-chunk tensor-core work on packed ROCmFPX-style codes.
//
// A "chunk" is up to 8 tiles (16 rows x 32-weight block each) of one
// row-group, laid out as in include/rfx.h.  Every packed block is decoded once
// in registers and multiplied against the B fragments of all the token columns
// at once (decode once, apply to every verify column: ainomam.com,
// "APU 实现 token 自由…", section "Lucebox 的优化三板斧").  Per tile:
//   C = A_lo(16x16) B(step 2b) + A_hi(16x16) B(step 2b+1)      (mma.sync, fp32)
//   acc[row][col] += scale[row] * C[row][col]                   (fp32 FFMA)
// so each block is accumulated exactly and scaled once, in fp32.
#pragma once
#include "rfx_device.cuh"
#include "rfx_layout.h"

namespace rfx {

__device__ __forceinline__ uint2 lds64(const uint8_t* p) { return *reinterpret_cast<const uint2*>(p); }
__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ uint32_t lds32(const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); }
__device__ __forceinline__ uint32_t lds16(const uint8_t* p) { return *reinterpret_cast<const uint16_t*>(p); }

// B-operand source: 4 16-bit values (k = 2t, 2t+1, 2t+8, 2t+9 of a k16 step)
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

template <int NB>
struct Acc {
    float v[NB][4];
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int n = 0; n < NB; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) v[n][i] = 0.f;
    }
};

// One tile: a[0..3] = k 0..15, a[4..7] = k 16..31; s0/s1 scales of rows g/g+8.
template <bool F16, int NB>
__device__ __forceinline__ void tile_mma(const uint32_t a[8], const uint2 blo[NB], const uint2 bhi[NB], float s0,
                                         float s1, Acc<NB>& acc) {
    const float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int n = 0; n < NB; ++n) {
        float c[4];
        mma16816<F16>(c, a, blo[n].x, blo[n].y, z);
        mma16816<F16>(c, a + 4, bhi[n].x, bhi[n].y, c);
        acc.v[n][0] = fmaf(s0, c[0], acc.v[n][0]);
        acc.v[n][1] = fmaf(s0, c[1], acc.v[n][1]);
        acc.v[n][2] = fmaf(s1, c[2], acc.v[n][2]);
        acc.v[n][3] = fmaf(s1, c[3], acc.v[n][3]);
    }
}

// Lane words of a full chunk (8 tiles) and its scale words.
template <int FMT>
struct FullChunk {
    static constexpr int NW = FMT * 4;           // 8, 12, 16 words of codes per lane
    static constexpr int NS = FMT == 4 ? 4 : 8;  // scale words per g
    static constexpr int CODE_BYTES = 8 * 16 * FMT * 4;
    uint32_t wd[NW];
    uint32_t sc[NS];
    __device__ __forceinline__ void load(const uint8_t* st, int lane, int g) {
#pragma unroll
        for (int i = 0; i < NW / 4; ++i) {
            uint4 v = lds128(st + lane * (NW * 4) + 16 * i);
            wd[4 * i] = v.x; wd[4 * i + 1] = v.y; wd[4 * i + 2] = v.z; wd[4 * i + 3] = v.w;
        }
#pragma unroll
        for (int i = 0; i < NS / 4; ++i) {
            uint4 v = lds128(st + CODE_BYTES + g * (NS * 4) + 16 * i);
            sc[4 * i] = v.x; sc[4 * i + 1] = v.y; sc[4 * i + 2] = v.z; sc[4 * i + 3] = v.w;
        }
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

// Decode the registers of tiles [b, b + TPG) (TPG = 2 for FP3 pairs, else 1).
template <int FMT> struct Grp { static constexpr int TPG = FMT == 3 ? 2 : 1; };

template <int FMT, bool F16>
__device__ __forceinline__ void unpack_group(const uint32_t* wd, int grp, uint32_t a[16]) {
    if constexpr (FMT == 2) {
        unpack_fp2<F16>(wd[grp], a);
    } else if constexpr (FMT == 4) {
        unpack_fp4_word<F16>(wd[2 * grp], a);
        unpack_fp4_word<F16>(wd[2 * grp + 1], a + 4);
    } else {
        unpack_fp3_pair<F16>(wd[3 * grp], wd[3 * grp + 1], wd[3 * grp + 2], a);
    }
}

// Full chunk of one matrix: accumulate into acc.  step0 = k16 step of tile 0.
template <int FMT, bool F16, int NB>
__device__ __forceinline__ void chunk_full(const uint8_t* st, int lane, int g, const BSrc* bs, int step0,
                                           Acc<NB>& acc) {
    FullChunk<FMT> fc;
    fc.load(st, lane, g);
    constexpr int TPG = Grp<FMT>::TPG;
#pragma unroll
    for (int grp = 0; grp < 8 / TPG; ++grp) {
        uint32_t a[16];
        unpack_group<FMT, F16>(fc.wd, grp, a);
#pragma unroll
        for (int u = 0; u < TPG; ++u) {
            const int b = grp * TPG + u;
            uint2 blo[NB], bhi[NB];
#pragma unroll
            for (int n = 0; n < NB; ++n) {
                blo[n] = bs[n].get(step0 + 2 * b);
                bhi[n] = bs[n].get(step0 + 2 * b + 1);
            }
            float s0, s1;
            fc.scales(b, s0, s1);
            tile_mma<F16, NB>(a + 8 * u, blo, bhi, s0, s1, acc);
        }
    }
}

// Two matrices (gate, up) sharing the B fragments, full chunks.
template <int FMT, bool F16, int NB>
__device__ __forceinline__ void chunk_full2(const uint8_t* st0, const uint8_t* st1, int lane, int g, const BSrc* bs,
                                            int step0, Acc<NB>& acc0, Acc<NB>& acc1) {
    FullChunk<FMT> f0, f1;
    f0.load(st0, lane, g);
    f1.load(st1, lane, g);
    constexpr int TPG = Grp<FMT>::TPG;
#pragma unroll
    for (int grp = 0; grp < 8 / TPG; ++grp) {
        uint32_t a0[16], a1[16];
        unpack_group<FMT, F16>(f0.wd, grp, a0);
        unpack_group<FMT, F16>(f1.wd, grp, a1);
#pragma unroll
        for (int u = 0; u < TPG; ++u) {
            const int b = grp * TPG + u;
            uint2 blo[NB], bhi[NB];
#pragma unroll
            for (int n = 0; n < NB; ++n) {
                blo[n] = bs[n].get(step0 + 2 * b);
                bhi[n] = bs[n].get(step0 + 2 * b + 1);
            }
            float s0, s1;
            f0.scales(b, s0, s1);
            tile_mma<F16, NB>(a0 + 8 * u, blo, bhi, s0, s1, acc0);
            f1.scales(b, s0, s1);
            tile_mma<F16, NB>(a1 + 8 * u, blo, bhi, s0, s1, acc1);
        }
    }
}

// Registers and scales of tile b of a partial chunk (nt < 8 tiles).
template <int FMT, bool F16>
__device__ __forceinline__ void partial_tile(const uint8_t* st, int nt, int lane, int g, int b, uint32_t a[8],
                                             float& s0, float& s1) {
    const int code_bytes = nt * 16 * FMT * 4;
    if constexpr (FMT == 2) {
        unpack_fp2<F16>(lds32(st + lane * 4 * nt + 4 * b), a);
        float2 f = scale_f16x2(lds32(st + code_bytes + (g * nt + b) * 4));
        s0 = f.x; s1 = f.y;
    } else if constexpr (FMT == 4) {
        const uint8_t* p = st + lane * 8 * nt + 8 * b;
        unpack_fp4_word<F16>(lds32(p), a);
        unpack_fp4_word<F16>(lds32(p + 4), a + 4);
        uint32_t e = lds16(st + code_bytes + (g * nt + b) * 2);
        s0 = scale_e8m0(e & 0xFFu);
        s1 = scale_e8m0(e >> 8);
    } else {
        const uint8_t* lp = st + lane * 6 * nt;       // 2-byte aligned
        const int pair = b >> 1;
        const bool lone = (b == nt - 1) && (nt & 1);
        if (lone) {
            const uint8_t* p = lp + 12 * pair;
            uint64_t s = (uint64_t)lds16(p) | ((uint64_t)lds16(p + 2) << 16) | ((uint64_t)lds16(p + 4) << 32);
            unpack_fp3_lone<F16>(s, a);
        } else {
            const uint8_t* p = lp + 12 * pair;
            uint32_t w0 = lds16(p) | (lds16(p + 2) << 16);
            uint32_t w1 = lds16(p + 4) | (lds16(p + 6) << 16);
            uint32_t w2 = lds16(p + 8) | (lds16(p + 10) << 16);
            uint32_t r[16];
            unpack_fp3_pair<F16>(w0, w1, w2, r);
#pragma unroll
            for (int i = 0; i < 8; ++i) a[i] = (b & 1) ? r[8 + i] : r[i];
        }
        float2 f = scale_f16x2(lds32(st + code_bytes + (g * nt + b) * 4));
        s0 = f.x; s1 = f.y;
    }
}

template <int FMT, bool F16, int NB>
__device__ __noinline__ void chunk_partial(const uint8_t* st, int nt, int lane, int g, const BSrc* bs, int step0,
                                           Acc<NB>& acc) {
    for (int b = 0; b < nt; ++b) {
        uint32_t a[8];
        float s0, s1;
        partial_tile<FMT, F16>(st, nt, lane, g, b, a, s0, s1);
        uint2 blo[NB], bhi[NB];
#pragma unroll
        for (int n = 0; n < NB; ++n) {
            blo[n] = bs[n].get(step0 + 2 * b);
            bhi[n] = bs[n].get(step0 + 2 * b + 1);
        }
        tile_mma<F16, NB>(a, blo, bhi, s0, s1, acc);
    }
}

// Dispatch one chunk of nt tiles of one matrix.
template <int FMT, bool F16, int NB>
__device__ __forceinline__ void chunk_any(const uint8_t* st, int nt, int lane, int g, const BSrc* bs, int step0,
                                          Acc<NB>& acc) {
    if (nt == 8) chunk_full<FMT, F16, NB>(st, lane, g, bs, step0, acc);
    else chunk_partial<FMT, F16, NB>(st, nt, lane, g, bs, step0, acc);
}

template <int FMT, bool F16, int NB>
__device__ __forceinline__ void chunk_any2(const uint8_t* st0, const uint8_t* st1, int nt, int lane, int g,
                                           const BSrc* bs, int step0, Acc<NB>& acc0, Acc<NB>& acc1) {
    if (nt == 8) {
        chunk_full2<FMT, F16, NB>(st0, st1, lane, g, bs, step0, acc0, acc1);
    } else {
        chunk_partial<FMT, F16, NB>(st0, nt, lane, g, bs, step0, acc0);
        chunk_partial<FMT, F16, NB>(st1, nt, lane, g, bs, step0, acc1);
    }
}

}  // namespace rfx
