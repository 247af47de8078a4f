// rfx_layout.h -- the packed ROCmFPX-style weight layout used by this library.
//
// A matrix W[N][K] (K % 32 == 0) is stored as row-groups of 16 rows (N is
// padded up to a multiple of 16 with zero rows).  Each row-group is one
// contiguous stream of chunks; a chunk holds up to 8 "tiles", a tile being the
// 16 rows x one 32-weight block of the row-group.  The bytes per block are
// those of the format (10 / 14 / 17 for FP2 / FP3 / FP4), so the packed size
// is exactly ceil(N/16)*16 * K/32 * bytes_per_block.
//
// Inside a chunk of nt tiles: first the codes (nt*16*codes_per_block bytes),
// then the scales (nt*16*scale_bytes).  Codes are lane-major for the m16n8k16
// tensor-core A fragment: lane L = 4*g + t owns 2*b bytes per tile (4, 6 or
// 8) at offset L * nt * 2*b and holds, per tile, the 16 codes of rows g and
// g+8 at k offsets {2t, 2t+1, 2t+8, 2t+9} and 16 + those.  Scales of a chunk
// are [g][tile][row g, row g+8].  The exact word layouts are in rfx.h.
//
// The bit position of each code inside a lane's words is chosen so that one
// LOP3 (mask + magic exponent) and one packed FMA turn two codes into the two
// 16-bit halves of an A-fragment register exactly (see rfx_dequant.cuh).
#pragma once
#include <stdint.h>
#include <stddef.h>

#define RFX_BLOCK 32
#define RFX_ROWS_PER_GROUP 16
#define RFX_TILES_PER_CHUNK 8

#ifdef __CUDACC__
#define RFX_HD __host__ __device__ __forceinline__
#else
#define RFX_HD static inline
#endif

// bytes of codes of one 32-weight block, of its scale, and of the block
RFX_HD int rfx_code_bytes(int fmt) { return fmt * 4; }          // 32 * b / 8
RFX_HD int rfx_scale_bytes(int fmt) { return fmt == 4 ? 1 : 2; }
RFX_HD int rfx_block_bytes(int fmt) { return fmt * 4 + (fmt == 4 ? 1 : 2); }
// per-lane code bytes of one tile (16 rows x 32 codes / 32 lanes)
RFX_HD int rfx_lane_tile_bytes(int fmt) { return fmt * 2; }
// bytes of a chunk of nt tiles
RFX_HD int64_t rfx_chunk_bytes(int fmt, int nt) { return (int64_t)nt * 16 * rfx_block_bytes(fmt); }
// bytes of one row-group stream for K columns
RFX_HD int64_t rfx_rowgroup_bytes(int fmt, int64_t K) { return (K / 32) * 16 * (int64_t)rfx_block_bytes(fmt); }
RFX_HD int64_t rfx_padded_rows(int64_t N) { return (N + 15) / 16 * 16; }
RFX_HD int64_t rfx_matrix_bytes(int fmt, int64_t N, int64_t K) {
    return rfx_padded_rows(N) / 16 * rfx_rowgroup_bytes(fmt, K);
}
// Full chunks (8 tiles) are stored slab-major so that each 128-bit shared
// memory load of a warp reads 512 contiguous bytes: code word w (0 .. 4*fmt-1)
// of lane L sits at byte ((w/4)*32 + L)*16 + (w%4)*4 of the chunk's codes, and
// the scale of (row g + 8h, tile b) at byte ((b/4)*8 + g)*16 + (b%4)*4 + 2h of
// its scales (binary16; E8M0 scales are [g][b][h] bytes, already 16 bytes per
// g).
RFX_HD int rfx_full_word_off(int lane, int w) { return (((w >> 2) * 32 + lane) << 4) + ((w & 3) << 2); }
RFX_HD int rfx_full_scale_off(int fmt, int g, int b, int h) {
    return fmt == 4 ? (g * 8 + b) * 2 + h : (((b >> 2) * 8 + g) << 4) + ((b & 3) << 2) + 2 * h;
}

// number of chunks of a row-group and tiles in chunk j
RFX_HD int rfx_num_chunks(int64_t K) { return (int)((K / 32 + 7) / 8); }
RFX_HD int rfx_chunk_tiles(int64_t K, int j) {
    int nb = (int)(K / 32);
    int rest = nb - 8 * j;
    return rest >= 8 ? 8 : rest;
}
