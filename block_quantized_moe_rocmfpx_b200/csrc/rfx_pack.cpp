// rfx_pack.cpp -- host packer/unpacker of the ROCmFPX-style block format and
// the thread-local error text of the C ABI.
//
// Block format: [TZ] taozi.news, "DeepSeek V4 Flash 在 128GB 锐龙 AI MAX+ 上跑到
// 32 tok/s", section "ROCmFPX：把 284B 权重压进 128 GB" (32 weights per block,
// codes plus scale; 10 / 14 / 17 bytes per block for FP2 / FP3 / FP4 in this
// library's reading).  The lane-major layout is described in include/rfx.h.
#include <cstdint>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/rfx.h"
#include "rfx_layout.h"

static thread_local std::string g_last_error;

extern "C" const char* rfx_last_error(void) { return g_last_error.c_str(); }

int rfx_fail(int code, const std::string& msg) {
    g_last_error = msg;
    return code;
}

static bool fmt_ok(int f) { return f == 2 || f == 3 || f == 4; }

extern "C" size_t rfx_packed_bytes(rfx_format f, int64_t rows, int64_t cols) {
    if (!fmt_ok(f) || rows < 0 || cols < 0 || cols % 32 != 0) return 0;
    return (size_t)rfx_matrix_bytes(f, rows, cols);
}

namespace {

// Codes of register r (low, high element) of a tile for lane (g, t).
struct TileView {
    const uint8_t* codes;  // [rows][cols]
    int64_t rows, cols;
    int64_t row0;          // first row of the row-group
    int64_t k0;            // first column of the tile's block
    int code(int row_in_group, int k_in_block) const {
        int64_t r = row0 + row_in_group;
        if (r >= rows) return 0;
        return codes[r * cols + k0 + k_in_block];
    }
};

inline void reg_coords(int g, int t, int r, int& row, int& k) {
    int m = r >> 2, j = r & 3;
    row = g + 8 * (j & 1);
    k = 16 * m + 2 * t + 8 * (j >> 1);
}

// ---- full chunks (8 tiles): "plane" layout ----
// Register r of tile b sits at the same bit offset for every r, in a
// different word per r, so one AND yields an fp16 subnormal code * 2^(s-24).
//   FP2: word r, field b (bits 2b | 16+2b).                         8 words
//   FP4: word r (tiles 0..3) or 8+r (tiles 4..7), field b&3 (4f | 16+4f).  16 words
//   FP3: tiles 0..4: word r, field b (bits 3b | 16+3b).
//        tiles 5, 6: r<4 -> word 8+r, field b-5; r>=4 -> word 8+r-4, field b-2.
//        tile 7:     r<4 -> word 8+r, field 2;   r>=4 -> bit i of the low code at
//        bit 15, of the high code at bit 31, of word 3(r-4)+i.          12 words
struct FieldRef { int word, shift, spare; };
static FieldRef full_field(int fmt, int b, int r) {
    if (fmt == 2) return {r, 2 * b, 0};
    if (fmt == 4) return {(b < 4 ? r : 8 + r), 4 * (b & 3), 0};
    if (b < 5) return {r, 3 * b, 0};
    if (b < 7) return r < 4 ? FieldRef{8 + r, 3 * (b - 5), 0} : FieldRef{8 + r - 4, 3 * (b - 2), 0};
    if (r < 4) return {8 + r, 6, 0};
    return {3 * (r - 4), 0, 1};
}

void pack_lane_full(int fmt, const TileView* tv, int g, int t, uint8_t* out) {
    uint32_t w[16] = {0};
    const uint32_t m = (1u << fmt) - 1u;
    for (int b = 0; b < 8; ++b)
        for (int r = 0; r < 8; ++r) {
            int row, k;
            reg_coords(g, t, r, row, k);
            const uint32_t lo = (uint32_t)tv[b].code(row, k) & m, hi = (uint32_t)tv[b].code(row, k + 1) & m;
            const FieldRef f = full_field(fmt, b, r);
            if (!f.spare) {
                w[f.word] |= lo << f.shift;
                w[f.word] |= hi << (16 + f.shift);
            } else {
                for (int i = 0; i < 3; ++i) {
                    w[f.word + i] |= ((lo >> i) & 1u) << 15;
                    w[f.word + i] |= ((hi >> i) & 1u) << 31;
                }
            }
        }
    // slab-major: word i of lane L at rfx_full_word_off(L, i) from the chunk start
    const int L = 4 * g + t;
    for (int i = 0; i < 4 * fmt; ++i) std::memcpy(out + rfx_full_word_off(L, i), &w[i], 4);
}

void unpack_lane_full(int fmt, const struct TileOut* to, int g, int t, const uint8_t* in);

// ---- partial chunks (< 8 tiles): per-tile layout ----
// Write the lane's codes of one tile (FP2 / FP4) or tile pair / lone tile (FP3).
void pack_lane_fp2(const TileView& tv, int g, int t, uint8_t* out) {
    uint32_t w = 0;
    for (int r = 0; r < 8; ++r) {
        int row, k;
        reg_coords(g, t, r, row, k);
        w |= (uint32_t)(tv.code(row, k) & 3) << (2 * r);
        w |= (uint32_t)(tv.code(row, k + 1) & 3) << (16 + 2 * r);
    }
    std::memcpy(out, &w, 4);
}

void pack_lane_fp4(const TileView& tv, int g, int t, uint8_t* out) {
    uint32_t w[2] = {0, 0};
    for (int r = 0; r < 8; ++r) {
        int row, k;
        reg_coords(g, t, r, row, k);
        int j = r & 3;
        w[r >> 2] |= (uint32_t)(tv.code(row, k) & 15) << (4 * j);
        w[r >> 2] |= (uint32_t)(tv.code(row, k + 1) & 15) << (16 + 4 * j);
    }
    std::memcpy(out, w, 8);
}

void pack_lane_fp3_pair(const TileView& a, const TileView& b, int g, int t, uint8_t* out) {
    uint32_t w[3] = {0, 0, 0};
    for (int R = 0; R < 16; ++R) {
        const TileView& tv = R < 8 ? a : b;
        int row, k;
        reg_coords(g, t, R & 7, row, k);
        uint32_t lo = (uint32_t)(tv.code(row, k) & 7), hi = (uint32_t)(tv.code(row, k + 1) & 7);
        if (R < 15) {
            int i = R / 5, p = R % 5;
            w[i] |= lo << (3 * p);
            w[i] |= hi << (16 + 3 * p);
        } else {
            for (int i = 0; i < 3; ++i) {
                w[i] |= ((lo >> i) & 1u) << 15;
                w[i] |= ((hi >> i) & 1u) << 31;
            }
        }
    }
    std::memcpy(out, w, 12);
}

void pack_lane_fp3_lone(const TileView& tv, int g, int t, uint8_t* out) {
    uint64_t s = 0;
    for (int r = 0; r < 8; ++r) {
        int row, k;
        reg_coords(g, t, r, row, k);
        s |= (uint64_t)(tv.code(row, k) & 7) << (3 * (2 * r));
        s |= (uint64_t)(tv.code(row, k + 1) & 7) << (3 * (2 * r + 1));
    }
    for (int i = 0; i < 6; ++i) out[i] = (uint8_t)(s >> (8 * i));
}

// ---- inverse ----
struct TileOut {
    uint8_t* codes;
    int64_t rows, cols, row0, k0;
    void set(int row_in_group, int k_in_block, int v) const {
        int64_t r = row0 + row_in_group;
        if (r < rows) codes[r * cols + k0 + k_in_block] = (uint8_t)v;
    }
};

void unpack_lane_fp2(const TileOut& to, int g, int t, const uint8_t* in) {
    uint32_t w;
    std::memcpy(&w, in, 4);
    for (int r = 0; r < 8; ++r) {
        int row, k;
        reg_coords(g, t, r, row, k);
        to.set(row, k, (w >> (2 * r)) & 3);
        to.set(row, k + 1, (w >> (16 + 2 * r)) & 3);
    }
}

void unpack_lane_fp4(const TileOut& to, int g, int t, const uint8_t* in) {
    uint32_t w[2];
    std::memcpy(w, in, 8);
    for (int r = 0; r < 8; ++r) {
        int row, k;
        reg_coords(g, t, r, row, k);
        int j = r & 3;
        to.set(row, k, (w[r >> 2] >> (4 * j)) & 15);
        to.set(row, k + 1, (w[r >> 2] >> (16 + 4 * j)) & 15);
    }
}

void unpack_lane_fp3_pair(const TileOut& a, const TileOut& b, int g, int t, const uint8_t* in) {
    uint32_t w[3];
    std::memcpy(w, in, 12);
    for (int R = 0; R < 16; ++R) {
        const TileOut& to = R < 8 ? a : b;
        int row, k;
        reg_coords(g, t, R & 7, row, k);
        int lo = 0, hi = 0;
        if (R < 15) {
            int i = R / 5, p = R % 5;
            lo = (w[i] >> (3 * p)) & 7;
            hi = (w[i] >> (16 + 3 * p)) & 7;
        } else {
            for (int i = 0; i < 3; ++i) {
                lo |= (int)((w[i] >> 15) & 1u) << i;
                hi |= (int)((w[i] >> 31) & 1u) << i;
            }
        }
        to.set(row, k, lo);
        to.set(row, k + 1, hi);
    }
}

void unpack_lane_full(int fmt, const TileOut* to, int g, int t, const uint8_t* in) {
    uint32_t w[16];
    const int L = 4 * g + t;
    for (int i = 0; i < 4 * fmt; ++i) std::memcpy(&w[i], in + rfx_full_word_off(L, i), 4);
    const uint32_t m = (1u << fmt) - 1u;
    for (int b = 0; b < 8; ++b)
        for (int r = 0; r < 8; ++r) {
            int row, k;
            reg_coords(g, t, r, row, k);
            const FieldRef f = full_field(fmt, b, r);
            uint32_t lo = 0, hi = 0;
            if (!f.spare) {
                lo = (w[f.word] >> f.shift) & m;
                hi = (w[f.word] >> (16 + f.shift)) & m;
            } else {
                for (int i = 0; i < 3; ++i) {
                    lo |= ((w[f.word + i] >> 15) & 1u) << i;
                    hi |= ((w[f.word + i] >> 31) & 1u) << i;
                }
            }
            to[b].set(row, k, (int)lo);
            to[b].set(row, k + 1, (int)hi);
        }
}

void unpack_lane_fp3_lone(const TileOut& to, int g, int t, const uint8_t* in) {
    uint64_t s = 0;
    for (int i = 0; i < 6; ++i) s |= (uint64_t)in[i] << (8 * i);
    for (int r = 0; r < 8; ++r) {
        int row, k;
        reg_coords(g, t, r, row, k);
        to.set(row, k, (int)((s >> (3 * (2 * r))) & 7));
        to.set(row, k + 1, (int)((s >> (3 * (2 * r + 1))) & 7));
    }
}

}  // namespace

extern "C" int rfx_pack(rfx_format f, const uint8_t* codes, const void* scales, int64_t rows, int64_t cols,
                        void* dst, size_t dst_bytes) {
    if (!fmt_ok(f)) return rfx_fail(RFX_EINVAL, "rfx_pack: format must be RFX_FP2, RFX_FP3 or RFX_FP4");
    if (rows < 0 || cols <= 0 || cols % 32 != 0) return rfx_fail(RFX_EINVAL, "rfx_pack: rows >= 0 and cols a positive multiple of 32 required");
    if ((!codes || !scales || !dst) && rows > 0) return rfx_fail(RFX_EINVAL, "rfx_pack: null pointer");
    const size_t need = (size_t)rfx_matrix_bytes(f, rows, cols);
    if (dst_bytes < need) return rfx_fail(RFX_EINVAL, "rfx_pack: dst_bytes smaller than rfx_packed_bytes");
    const int64_t nb = cols / 32;
    // validate values first
    const int cmax = 1 << f;
    for (int64_t i = 0; i < rows * cols; ++i)
        if (codes[i] >= cmax) return rfx_fail(RFX_EINVAL, "rfx_pack: code out of range for the format");
    for (int64_t i = 0; i < rows * nb; ++i) {
        if (f == RFX_FP4) {
            if (((const uint8_t*)scales)[i] == 0xFF) return rfx_fail(RFX_EINVAL, "rfx_pack: E8M0 scale 0xFF is not a number");
        } else {
            if ((((const uint16_t*)scales)[i] & 0x7C00u) == 0x7C00u)
                return rfx_fail(RFX_EINVAL, "rfx_pack: binary16 scale must be finite");
        }
    }
    uint8_t* out = (uint8_t*)dst;
    const int64_t ngroups = rfx_padded_rows(rows) / 16;
    const int64_t rg_bytes = rfx_rowgroup_bytes(f, cols);
    const int nch = rfx_num_chunks(cols);
    const int ltb = rfx_lane_tile_bytes(f);
    const int sb = rfx_scale_bytes(f);
#pragma omp parallel for schedule(static)
    for (int64_t rg = 0; rg < ngroups; ++rg) {
        uint8_t* base = out + rg * rg_bytes;
        for (int j = 0; j < nch; ++j) {
            const int nt = rfx_chunk_tiles(cols, j);
            uint8_t* chunk = base + (int64_t)j * rfx_chunk_bytes(f, 8);
            uint8_t* sc = chunk + (int64_t)nt * 16 * rfx_code_bytes(f);
            for (int L = 0; L < 32; ++L) {
                const int g = L >> 2, t = L & 3;
                uint8_t* lane = chunk + (int64_t)L * nt * ltb;
                if (nt == 8) {
                    TileView tv[8];
                    for (int b = 0; b < 8; ++b) tv[b] = TileView{codes, rows, cols, rg * 16, (int64_t)(8 * j + b) * 32};
                    pack_lane_full(f, tv, g, t, chunk);
                } else if (f == RFX_FP3) {
                    int b = 0;
                    for (; b + 1 < nt; b += 2) {
                        TileView A{codes, rows, cols, rg * 16, (int64_t)(8 * j + b) * 32};
                        TileView B{codes, rows, cols, rg * 16, (int64_t)(8 * j + b + 1) * 32};
                        pack_lane_fp3_pair(A, B, g, t, lane + 6 * b);
                    }
                    if (b < nt) {
                        TileView A{codes, rows, cols, rg * 16, (int64_t)(8 * j + b) * 32};
                        pack_lane_fp3_lone(A, g, t, lane + 6 * b);
                    }
                } else {
                    for (int b = 0; b < nt; ++b) {
                        TileView tv{codes, rows, cols, rg * 16, (int64_t)(8 * j + b) * 32};
                        if (f == RFX_FP2) pack_lane_fp2(tv, g, t, lane + 4 * b);
                        else pack_lane_fp4(tv, g, t, lane + 8 * b);
                    }
                }
            }
            for (int g = 0; g < 8; ++g)
                for (int b = 0; b < nt; ++b)
                    for (int h = 0; h < 2; ++h) {
                        int64_t r = rg * 16 + g + 8 * h;
                        int64_t bi = r * nb + 8 * j + b;
                        uint8_t* d = nt == 8 ? sc + rfx_full_scale_off(f, g, b, h) : sc + ((int64_t)(g * nt + b) * 2 + h) * sb;
                        if (r >= rows) { std::memset(d, 0, sb); continue; }
                        std::memcpy(d, (const uint8_t*)scales + bi * sb, sb);
                    }
        }
    }
    return RFX_OK;
}

extern "C" int rfx_unpack(rfx_format f, const void* src, int64_t rows, int64_t cols, uint8_t* codes, void* scales) {
    if (!fmt_ok(f)) return rfx_fail(RFX_EINVAL, "rfx_unpack: bad format");
    if (rows < 0 || cols <= 0 || cols % 32 != 0) return rfx_fail(RFX_EINVAL, "rfx_unpack: bad shape");
    if ((!src || !codes || !scales) && rows > 0) return rfx_fail(RFX_EINVAL, "rfx_unpack: null pointer");
    const uint8_t* in = (const uint8_t*)src;
    const int64_t nb = cols / 32;
    const int64_t ngroups = rfx_padded_rows(rows) / 16;
    const int64_t rg_bytes = rfx_rowgroup_bytes(f, cols);
    const int nch = rfx_num_chunks(cols);
    const int ltb = rfx_lane_tile_bytes(f);
    const int sb = rfx_scale_bytes(f);
#pragma omp parallel for schedule(static)
    for (int64_t rg = 0; rg < ngroups; ++rg) {
        const uint8_t* base = in + rg * rg_bytes;
        for (int j = 0; j < nch; ++j) {
            const int nt = rfx_chunk_tiles(cols, j);
            const uint8_t* chunk = base + (int64_t)j * rfx_chunk_bytes(f, 8);
            const uint8_t* sc = chunk + (int64_t)nt * 16 * rfx_code_bytes(f);
            for (int L = 0; L < 32; ++L) {
                const int g = L >> 2, t = L & 3;
                const uint8_t* lane = chunk + (int64_t)L * nt * ltb;
                if (nt == 8) {
                    TileOut to[8];
                    for (int b = 0; b < 8; ++b) to[b] = TileOut{codes, rows, cols, rg * 16, (int64_t)(8 * j + b) * 32};
                    unpack_lane_full(f, to, g, t, chunk);
                } else if (f == RFX_FP3) {
                    int b = 0;
                    for (; b + 1 < nt; b += 2) {
                        TileOut A{codes, rows, cols, rg * 16, (int64_t)(8 * j + b) * 32};
                        TileOut B{codes, rows, cols, rg * 16, (int64_t)(8 * j + b + 1) * 32};
                        unpack_lane_fp3_pair(A, B, g, t, lane + 6 * b);
                    }
                    if (b < nt) {
                        TileOut A{codes, rows, cols, rg * 16, (int64_t)(8 * j + b) * 32};
                        unpack_lane_fp3_lone(A, g, t, lane + 6 * b);
                    }
                } else {
                    for (int b = 0; b < nt; ++b) {
                        TileOut to{codes, rows, cols, rg * 16, (int64_t)(8 * j + b) * 32};
                        if (f == RFX_FP2) unpack_lane_fp2(to, g, t, lane + 4 * b);
                        else unpack_lane_fp4(to, g, t, lane + 8 * b);
                    }
                }
            }
            for (int g = 0; g < 8; ++g)
                for (int b = 0; b < nt; ++b)
                    for (int h = 0; h < 2; ++h) {
                        int64_t r = rg * 16 + g + 8 * h;
                        if (r >= rows) continue;
                        int64_t bi = r * nb + 8 * j + b;
                        const uint8_t* d = nt == 8 ? sc + rfx_full_scale_off(f, g, b, h) : sc + ((int64_t)(g * nt + b) * 2 + h) * sb;
                        std::memcpy((uint8_t*)scales + bi * sb, d, sb);
                    }
        }
    }
    return RFX_OK;
}
