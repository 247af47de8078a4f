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
#define MOE_MAX_RED 8          // reduction buffers
#define MOE_CHUNKS_PER_STAGE 8
#define MOE_HALF_BYTES 17408   // 8 full FP4 chunks of one matrix
#define MOE_STAGE_BYTES 34816  // two halves: gate + up, or two down row-groups

// workspace control words (uint32 index); the grid-barrier counters are
// 64-bit and only grow
#define MOE_CTRL_TASK_A 0      // next gate/up row-group to hand out (reset after the first barrier)
#define MOE_CTRL_ERR 2
#define MOE_CTRL_BAR_H 4       // u64: gate/up phase done (h complete)
#define MOE_CTRL_BAR_D 6       // u64: down phase done (partials complete)
#define MOE_CTRL_WORDS 64

// device error bits
#define MOE_ERR_EXPERT 1u
#define MOE_ERR_DUP 2u
#define MOE_ERR_TIMEOUT 4u
#define MOE_ERR_RANGE 8u

namespace rfx {

struct MoeParams {
    int H, I, E, k, T;
    int fA, fB, fsA, fsB;  // routed gate/up, routed down, shared gate/up, shared down formats
    const uint8_t* gate;
    const uint8_t* up;
    const uint8_t* down;
    long long sg, su, sd;  // routed expert strides (bytes)
    int has_shared;
    const uint8_t* shg;
    const uint8_t* shu;
    const uint8_t* shd;
    const uint16_t* x;     // bf16 [T][H]
    const int32_t* idx;    // [T][k]
    const float* wts;      // [T][k]
    float* y;              // [T][H]
    uint32_t* ctrl;
    uint16_t* hbuf;        // per slot: fp16 h fragments [2*T*I] then fp32 block sums [T][sstr]
    float* dpart;          // fp32 [MAXS_T][T][H]
    int ns;                // stages in the ring
    int nred;              // reduction buffers
    int x_stride;          // bytes per x column in shared memory
    int xh_bytes;          // bytes of the x / h region
};

// Floats per column of the h block-sum table: one per 16-row group of I,
// padded to a multiple of 4 (16 bytes).
inline __host__ __device__ int moe_sstr(int I) { return ((I / 16) + 3) & ~3; }

// Floats per column of the x block-sum table (H/32 padded to 16-byte rows).
inline __host__ __device__ int moe_sxs(int H) { return ((H / 32) + 3) & ~3; }

// Workspace layout for (T, k, H, I).
struct MoeWs {
    size_t ctrl_off, h_off, d_off, total;
};

inline MoeWs moe_ws_layout(int T, int k, int H, int I) {
    MoeWs L;
    const size_t ns = (size_t)T * k + 1;
    L.ctrl_off = 0;
    L.h_off = (MOE_CTRL_WORDS * 4 + 255) / 256 * 256;
    L.d_off = L.h_off + (ns * 4 * T * (size_t)(I + moe_sstr(I)) + 255) / 256 * 256;
    L.total = L.d_off + (ns * T * H * 4 + 255) / 256 * 256;
    return L;
}

size_t moe_decode_smem_bytes(int ns, int nred, int xh_bytes);
cudaError_t moe_decode_launch(const MoeParams& p, int grid, cudaStream_t stream);

}  // namespace rfx
