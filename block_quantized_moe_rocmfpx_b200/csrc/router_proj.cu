// router_proj.cu -- the router projection ahead of the top-k:
//     logits[t][e] = sum_h W[e][h] x[t][h] + b[e]
// with bf16 W [E][H] and x [T][H], fp32 accumulation and an optional fp32
// bias [E].  The projection is the MoE gate that decides the routing and is
// kept at high precision (FP8 in the bit allocation of ai-manual.ru, "DeepSeek
// V4 Flash на AMD Ryzen AI MAX+ 395…", section "Технические детали ROCmFPX";
// sensitive projections at FP4 or above in taozi.news, "DeepSeek V4 Flash 在
// 128GB 锐龙 AI MAX+ 上跑到 32 tok/s", section "ROCmFPX：把 284B 权重压进 128
// GB"); this library reads that as bf16 weights.
//
// B200 design: a GEMV over E rows (2 MB for 256 x 4096), HBM-bound, spread over
// all SMs.  A CTA owns two rows and up to 8 columns; each of its 8 warps takes a
// quarter of H for one row (16-byte loads of 8 bf16 of W and of x, fp32 FMAs in
// index order per lane, then a butterfly over the lanes); the four quarters
// are added in a fixed tree, so a logit's bits depend neither on T nor on the
// launch.  W is a constant input: each warp asks L2 for its slice before the
// kernel waits for the previous one (programmatic dependent launch); x may come
// from that kernel and is read after the wait.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gemv.h"
#include "rfx_device.cuh"

namespace rfx {

constexpr int RP_ROWS = 2;     // router rows per CTA
constexpr int RP_SPLIT = 4;    // warps per row (quarters of H)
constexpr int RP_COLS = 8;     // token columns per CTA
constexpr int RP_THREADS = 32 * RP_ROWS * RP_SPLIT;

__device__ __forceinline__ void bf16x8(uint4 v, float f[8]) {
    f[0] = __uint_as_float(v.x << 16); f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16); f[3] = __uint_as_float(v.y & 0xffff0000u);
    f[4] = __uint_as_float(v.z << 16); f[5] = __uint_as_float(v.z & 0xffff0000u);
    f[6] = __uint_as_float(v.w << 16); f[7] = __uint_as_float(v.w & 0xffff0000u);
}

__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__global__ void __launch_bounds__(RP_THREADS) router_logits_kernel(const uint16_t* __restrict__ W,
                                                                  const float* __restrict__ bias,
                                                                  const uint16_t* __restrict__ x, int T, int H, int E,
                                                                  float* __restrict__ logits) {
    grid_dep_launch();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = warp / RP_SPLIT, part = warp - r * RP_SPLIT;
    const int row = blockIdx.x * RP_ROWS + r;
    const int c0 = blockIdx.y * RP_COLS;
    const int nc = min(RP_COLS, T - c0);
    const int kp = H / RP_SPLIT;   // a multiple of 8 (H % 32 == 0)
    const uint16_t* wp = W + (size_t)row * H + (size_t)part * kp;
    if (row < E && lane == 0) bulk_prefetch_l2(wp, (uint32_t)kp * 2u);
    grid_dep_wait();
    float acc[RP_COLS];
#pragma unroll
    for (int c = 0; c < RP_COLS; ++c) acc[c] = 0.f;
    if (row < E) {
        const uint4* w4 = reinterpret_cast<const uint4*>(wp);
        for (int ch = lane; ch < kp / 8; ch += 32) {
            float wf[8];
            bf16x8(__ldg(w4 + ch), wf);
#pragma unroll
            for (int c = 0; c < RP_COLS; ++c) {
                if (c >= nc) break;
                const uint4* x4 = reinterpret_cast<const uint4*>(x + (size_t)(c0 + c) * H + (size_t)part * kp);
                float xf[8];
                bf16x8(__ldg(x4 + ch), xf);
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[c] = fmaf(wf[i], xf[i], acc[c]);
            }
        }
    }
#pragma unroll
    for (int c = 0; c < RP_COLS; ++c)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], o);
    __shared__ float ps[RP_ROWS * RP_SPLIT][RP_COLS];
    if (lane == 0)
#pragma unroll
        for (int c = 0; c < RP_COLS; ++c) ps[warp][c] = acc[c];
    __syncthreads();
    if (threadIdx.x < RP_ROWS * RP_COLS) {
        const int rr = threadIdx.x / RP_COLS, c = threadIdx.x - rr * RP_COLS;
        const int e = blockIdx.x * RP_ROWS + rr;
        if (e < E && c < nc) {
            const float* q = &ps[rr * RP_SPLIT][0];
            float v = (q[0 * RP_COLS + c] + q[1 * RP_COLS + c]) + (q[2 * RP_COLS + c] + q[3 * RP_COLS + c]);
            if (bias) v += __ldg(bias + e);
            logits[(size_t)(c0 + c) * E + e] = v;
        }
    }
}

cudaError_t router_logits_launch(const uint16_t* W, const float* bias, const uint16_t* x, int T, int H, int E,
                                 float* logits, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((E + RP_ROWS - 1) / RP_ROWS), (unsigned)((T + RP_COLS - 1) / RP_COLS));
    cfg.blockDim = dim3(RP_THREADS);
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, router_logits_kernel, W, bias, x, T, H, E, logits);
}

}  // namespace rfx
