// prefill.h -- launch parameters and workspace layout of the prefill MoE FFN
// (prefill.cu): per-expert grouping of the routed tokens, then a grouped GEMM
// on the tcgen05 tensor cores with the packed weights dequantised to bf16 in
// shared memory.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe_decode.h"

// workspace control words (uint32 index).  Word 2 is the device error flag,
// at the same place as in the decode workspace so that one status call reads
// both.
#define PF_CTRL_ERR 2
#define PF_CTRL_NTILES 8     // token tiles (written by the grouping)
#define PF_CTRL_ROWS 9       // routed rows (sum of the per-expert counts)
#define PF_CTRL_NEXT0 10     // next unit to hand out, gate/up GEMM (reset by the grouping)
#define PF_CTRL_NEXT1 11     // next unit to hand out, down GEMM
#define PF_CTRL_WORDS 64

#define PF_TILE_N 256        // most tokens per token tile (the MMA's largest N)
#define PF_BM 128            // weight rows per tile (the MMA's M)
#define PF_BK 64             // reduction step per pipeline stage (one 128-byte swizzle atom of bf16)
#define PF_SLICE 1024        // routed entries per grouping CTA

namespace rfx {

struct PfParams {
    int H, I, E, k, T;
    int fA, fB, fsA, fsB;   // routed gate/up, routed down, shared gate/up, shared down formats
    const uint8_t* gate;
    const uint8_t* up;
    const uint8_t* down;
    long long sg, su, sd;   // routed expert strides (bytes)
    const MoeMixEntry* mix; // device [E], or null: every routed expert at e * stride in fA / fB
    int has_shared;
    const uint8_t* shg;
    const uint8_t* shu;
    const uint8_t* shd;
    const uint16_t* x;      // bf16 [T][H]
    const int32_t* idx;     // [T][k]
    const float* wts;       // [T][k]
    float* y;               // [T][H]
    // workspace
    uint32_t* ctrl;
    int32_t* cnt;           // [E] tokens per routed expert
    int32_t* cnt_part;      // [slices][E] tokens per routed expert in each slice of PF_SLICE entries
    int32_t* off;           // [E] first grouped row of each routed expert
    int32_t* perm_tok;      // [T*k] token of each routed row (rows grouped by expert, stable)
    float* perm_w;          // [T*k] combine weight of each routed row
    int4* tiles;            // token tiles {row0, n, expert (-1 = shared), 0}
    uint16_t* xp;           // bf16 [T*k][H] routed rows of x, grouped
    uint16_t* hp;           // bf16 [T*k + T][I] SwiGLU output rows (routed rows, then the shared expert's);
                            // exact precision: then as many rows of h - bf16(h)
    int exact;              // 1: weights as bf16 hi + lo pairs and h as h1 + h2 (exact-precision prefill)
    int max_tiles;
    long long wait_limit;   // SM clocks before a bounded wait gives up
    int fault;              // tests of the error path only: 3 = the down GEMM waits for a stage nothing loads
};

struct PfWs {
    size_t ctrl, cnt, cnt_part, off, perm_tok, perm_w, tiles, xp, hp, total;
    int max_tiles;
};

inline PfWs pf_ws_layout(int T, int k, int E, int H, int I, int hparts = 1) {
    auto up = [](size_t n) { return (n + 255) / 256 * 256; };
    PfWs L;
    const size_t R = (size_t)T * k;
    L.max_tiles = (int)((R + PF_TILE_N - 1) / PF_TILE_N + (size_t)(E < (int)R ? E : (int)R) +
                        ((size_t)T + PF_TILE_N - 1) / PF_TILE_N + 1);
    L.ctrl = 0;
    L.cnt = up(PF_CTRL_WORDS * 4);
    const size_t slices = (R + PF_SLICE - 1) / PF_SLICE;
    L.cnt_part = L.cnt + up((size_t)E * 4);
    L.off = L.cnt_part + up(slices * E * 4);
    L.perm_tok = L.off + up((size_t)E * 4);
    L.perm_w = L.perm_tok + up(R * 4);
    L.tiles = L.perm_w + up(R * 4);
    L.xp = L.tiles + up((size_t)L.max_tiles * 16);
    L.hp = L.xp + up(R * H * 2);
    L.total = L.hp + up((size_t)hparts * (R + T) * I * 2);
    return L;
}

size_t pf_gemm_smem_bytes(int mode, bool exact);
// Launch the whole prefill step on `stream`: grouping, gather, gate/up GEMM
// with SwiGLU, down GEMM with the weighted combine into y.  `sms` = SM count.
long long pf_default_wait_limit();
cudaError_t pf_launch(const PfParams& p, int sms, cudaStream_t stream);

}  // namespace rfx
