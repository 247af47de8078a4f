// stack.cu -- chaining of MoE layers: each layer's fp32 output, normalised to
// unit RMS and rounded to bf16, is the next layer's input (the 43-layer stack
// of m.mzlw.cn, "Lucebox专攻DeepSeek V4…", section "MoE 专家并行"; the
// unit-RMS, bf16 chaining rule is this library's stack workload).
#include <cuda_runtime.h>
#include <stdint.h>

#include "rfx_device.cuh"
#include "stack.h"

namespace rfx {

// One CTA per column: fp64 sum of squares, then x = bf16(y / sqrt(mean)).
__global__ void __launch_bounds__(256) rms_bf16_kernel(const float* __restrict__ y, int H, uint16_t* __restrict__ x) {
    const float* yc = y + (long long)blockIdx.x * H;
    uint16_t* xc = x + (long long)blockIdx.x * H;
    double ss = 0.0;
    for (int i = threadIdx.x; i < H; i += blockDim.x) {
        const double v = (double)yc[i];
        ss = fma(v, v, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    __shared__ double part[8];
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        double t = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (threadIdx.x == 0) part[0] = t;
    }
    __syncthreads();
    const double r = sqrt(part[0] / (double)H);
    for (int i = threadIdx.x; i < H; i += blockDim.x) xc[i] = f64_to_bf16_rne((double)yc[i] / r);
}

cudaError_t rms_bf16_launch(const float* y, int T, int H, uint16_t* x, cudaStream_t stream) {
    (void)cudaGetLastError();   // an earlier call's launch error is not this launch's
    rms_bf16_kernel<<<T, 256, 0, stream>>>(y, H, x);
    return cudaGetLastError();
}

}  // namespace rfx
