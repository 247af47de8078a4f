// stack.cu -- chaining of MoE layers: each layer's fp32 output, normalised to
// unit RMS and rounded to bf16, is the next layer's input (the 43-layer stack
// of m.mzlw.cn, "Lucebox专攻DeepSeek V4…", section "MoE 专家并行"; the
// unit-RMS, bf16 chaining rule is this library's stack workload).
#include <cuda_runtime.h>
#include <stdint.h>

#include "stack.h"

namespace rfx {

// Round a double to bf16 bits, nearest-even, in one step (no intermediate
// float rounding): sign, 8-bit exponent with bias 127, 7 explicit mantissa
// bits; values below 2^-126 become bf16 subnormals, values beyond the largest
// finite bf16 become infinity.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double v) {
    const unsigned long long d = (unsigned long long)__double_as_longlong(v);
    const uint32_t sign = (uint32_t)(d >> 48) & 0x8000u;
    const int e = (int)((d >> 52) & 0x7FF);
    const unsigned long long m = d & ((1ull << 52) - 1ull);
    if (e == 0x7FF) return (uint16_t)(sign | 0x7F80u | (m ? 0x40u : 0u));   // inf / nan
    if (e == 0) return (uint16_t)sign;                                       // zero (and fp64 subnormals)
    const int E = e - 1023;                                                  // unbiased exponent
    const unsigned long long sig = (1ull << 52) | m;                         // 53-bit significand
    int shift;                                                               // significand bits dropped
    int be;                                                                  // bf16 biased exponent before rounding
    if (E >= -126) {
        shift = 45;
        be = E + 127;
    } else {
        shift = 45 + (-126 - E);                                             // subnormal: fixed exponent 2^-126
        be = 0;
        if (shift > 54) return (uint16_t)sign;                               // rounds to zero
    }
    unsigned long long q = sig >> shift;
    const unsigned long long rem = sig & ((1ull << shift) - 1ull), half = 1ull << (shift - 1);
    if (rem > half || (rem == half && (q & 1ull))) ++q;
    // q holds the implicit bit (normal) at bit 7; a carry out of it bumps the exponent
    uint32_t bits;
    if (be > 0) {
        if (q >> 8) { q >>= 1; ++be; }
        if (be >= 255) return (uint16_t)(sign | 0x7F80u);
        bits = ((uint32_t)be << 7) | (uint32_t)(q & 0x7Fu);
    } else {
        bits = (uint32_t)q;   // subnormal; q == 0x80 is the smallest normal, which has the same bits
    }
    return (uint16_t)(sign | bits);
}

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
    rms_bf16_kernel<<<T, 256, 0, stream>>>(y, H, x);
    return cudaGetLastError();
}

}  // namespace rfx
