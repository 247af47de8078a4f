// moe_decode.h -- launch parameters and workspace layout of the MoE decode /
// verify kernel (moe_decode.cu).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#define MOE_MAXT 8            // token columns per call (decode / verify)
#define MOE_MAXK 8            // routed experts per token
#define MOE_MAXS (MOE_MAXT * MOE_MAXK + 1)
#define MOE_MAX_STAGES 8
#define MOE_MAX_RED 6          // reduction buffers (a multiple of the 3 epilogue warps)
#define MOE_CHUNKS_PER_STAGE 8
#define MOE_HALF_BYTES 17408   // 8 full FP4 chunks of one matrix
#define MOE_STAGE_BYTES 34816  // two halves: gate + up, or two down row-groups

// Workspace control block (uint32 words).  Every word is zero before a call
// and the kernel returns it to zero at its end (the grid-barrier counter
// excepted: it only grows).
#define MOE_CTRL_QUEUE 0          // work items handed out beyond each CTA's first
#define MOE_CTRL_ERR 2            // device error bits
#define MOE_CTRL_BAR 4            // u64: final grid barrier (only grows)
#define MOE_CTRL_SLOT_DONE 64     // [MOE_MAXS] gate/up units (32 rows of I) whose h image is written
#define MOE_CTRL_WORDS 256

// device error bits
#define MOE_ERR_EXPERT 1u
#define MOE_ERR_TIMEOUT 4u
#define MOE_ERR_RANGE 8u

namespace rfx {

// ROCmFPX MIX: the packed matrices of routed expert e are at gate + og,
// up + ou, down + od, gate and up in format fa, down in format fb.
struct MoeMixEntry {
    long long og, ou, od;
    int fa, fb;
};
static_assert(sizeof(MoeMixEntry) == 32, "one 32-byte entry per expert");

struct MoeParams {
    int H, I, E, k, T;
    int fA, fB, fsA, fsB;  // routed gate/up, routed down, shared gate/up, shared down formats
    const uint8_t* gate;
    const uint8_t* up;
    const uint8_t* down;
    long long sg, su, sd;  // routed expert strides (bytes)
    const MoeMixEntry* mix;  // device [E], or null: every routed expert at e * stride in fA / fB
    int nxc;               // copies of the staged x (gate/up formats with their own copy)
    int xf[2];             // format of each copy; a slot of another format reads copy 0 with compensated scales
    int other;             // some routed expert's gate/up format has no copy (the kernel with those variants)
    int has_shared;
    const uint8_t* shg;
    const uint8_t* shu;
    const uint8_t* shd;
    const uint16_t* x;     // bf16 [T][H]
    const float* xc;       // or, chained from a previous layer: fp32 [T][H], x = bf16(xc / rms(xc)) per column
    const int32_t* idx;    // [T][k]
    const float* wts;      // [T][k]
    float* y;              // [T][H]
    uint32_t* ctrl;
    uint8_t* hfrag;        // [slots] x hslot_bytes: the down projection's B operand (moe_h_image_bytes)
    float* dpart;          // [slots][T][H] per-slot down outputs
    long long hslot_bytes; // bytes per slot in hfrag
    int ns;                // stages in the ring
    int nred;              // reduction buffers
    int x_stride;          // bytes per x column in shared memory
    int x_bytes;           // bytes of the staged x (gate/up phase)
    int xh_bytes;          // bytes of the x / h region
    int hoff0, hoff1;      // offsets of the two h buffers inside that region
    long long wait_limit;  // bounded waits give up after this many SM clocks
    int fault;             // tests of the error path only: 1 = the final grid barrier expects one CTA more than
                           // the grid has; 2 = no slot ever counts as ready for the down projection
};

// Per-column tables read with 16-byte loads by lanes of different columns:
// rows of 8k + 4 floats, so that column c starts c * 16 bytes further into
// the 128-byte bank window (up to 8 columns, one 16-byte load each, without
// bank conflicts) and every row stays 16-byte aligned.
inline __host__ __device__ int moe_col_stride(int n) { return ((n + 7) & ~7) + 4; }

// Floats per column of the h block-sum table: one per 16-row group of I.
inline __host__ __device__ int moe_sstr(int I) { return moe_col_stride(I / 16); }

// Floats per column of the x block-sum table: one per 32-block of H.
inline __host__ __device__ int moe_sxs(int H) { return moe_col_stride(H / 32); }

// Floats per column of the h block-scale table: one per 32-block of I (a
// chunk's 8 blocks are read as two 16-byte loads).
inline __host__ __device__ int moe_sbs(int I) { return moe_col_stride(I / 32); }

// Bytes of a slot's h image for ncols columns: the fp16 hi/lo fragments of
// h * 2^n (4 bytes per value), the 16-row block sums, the 2^-n factors.
inline __host__ __device__ int moe_h_image_bytes(int ncols, int I) {
    return 4 * ncols * I + 4 * ncols * moe_sstr(I) + 4 * ncols * moe_sbs(I);
}

// Reduction-buffer bytes per row-group for a column class (1: T = 1, 2: T <= 4,
// 3: T <= 8); a buffer holds two row-groups.
inline __host__ __device__ int moe_red_bytes(int qc) { return qc == 1 ? 8 * 128 : (qc == 2 ? 8 * 512 : 8 * 1024); }
inline __host__ __device__ int moe_qclass(int T) { return T == 1 ? 1 : (T <= 4 ? 2 : 3); }

// Workspace layout for (T, k, H, I).
struct MoeWs {
    size_t ctrl_off, hf_off, d_off, total;
    size_t hslot;
};

inline MoeWs moe_ws_layout(int T, int k, int H, int I) {
    auto up = [](size_t n) { return (n + 255) / 256 * 256; };
    MoeWs L;
    const size_t ns = (size_t)T * k + 1;
    L.hslot = up((size_t)moe_h_image_bytes(T, I));
    L.ctrl_off = 0;
    L.hf_off = MOE_CTRL_WORDS * 4;
    L.d_off = L.hf_off + ns * L.hslot;
    L.total = L.d_off + up(ns * T * (size_t)H * 4);
    return L;
}

size_t moe_decode_smem_bytes(int ns, int nred, int xh_bytes, int qc);
cudaError_t moe_decode_launch(const MoeParams& p, int grid, cudaStream_t stream);

}  // namespace rfx
