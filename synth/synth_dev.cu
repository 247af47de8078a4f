// synth_dev.cu -- device twin of synth.c for large synthetic layers.
//
// Same SplitMix64 counter-based definition (Steele, Lea, Flood 2014) and the
// same block-scale table (computed once on the host by synth.c and uploaded),
// so every code and scale equals the host generator's bit for bit.  Input
// generation only: no dequantisation, packing or any other step of the method.
#include <cuda_runtime.h>
#include <stdint.h>

#define SYNTH_GAMMA 0x9e3779b97f4a7c15ULL

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}
__device__ __forceinline__ uint64_t draw(uint64_t key, uint64_t n) { return mix64(key + (n + 1) * SYNTH_GAMMA); }

// one thread per 32-code block; out row-major [nrows][cols]
__global__ void codes_kernel(uint64_t key, int bits, int64_t row0, int64_t nrows, int64_t cols, uint8_t* out) {
    const int64_t nb = cols / 32;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nrows * nb) return;
    const int64_t r = i / nb, b = i % nb;
    const uint64_t beta = (uint64_t)((row0 + r) * nb + b);
    uint8_t c[32];
    if (bits == 2) {
        uint64_t d = draw(key, beta);
        for (int j = 0; j < 32; ++j) c[j] = (uint8_t)((d >> (2 * j)) & 3u);
    } else {
        uint64_t d0 = draw(key, 2 * beta), d1 = draw(key, 2 * beta + 1);
        const int s = bits == 3 ? 3 : 4;
        const unsigned m = (1u << s) - 1u;
        for (int j = 0; j < 16; ++j) c[j] = (uint8_t)((d0 >> (s * j)) & m);
        for (int j = 0; j < 16; ++j) c[16 + j] = (uint8_t)((d1 >> (s * j)) & m);
    }
    uint4* o = (uint4*)(out + r * cols + b * 32);
    o[0] = *(uint4*)&c[0];
    o[1] = *(uint4*)&c[16];
}

__global__ void scales_kernel(uint64_t key, int bits, int64_t row0, int64_t nrows, int64_t cols, void* out,
                              const uint16_t* tf16, const uint8_t* te8) {
    const int64_t nb = cols / 32;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= nrows * nb) return;
    const int64_t r = i / nb, b = i % nb;
    const unsigned idx = (unsigned)(draw(key, (uint64_t)((row0 + r) * nb + b)) >> 48);
    if (bits == 4) ((uint8_t*)out)[i] = te8[idx];
    else ((uint16_t*)out)[i] = tf16[idx];
}

extern "C" int synth_codes_dev(uint64_t key, int bits, int64_t row0, int64_t nrows, int64_t cols, uint8_t* out,
                               void* stream) {
    if (cols % 32 || (bits < 2 || bits > 4) || nrows < 0 || ((uintptr_t)out & 15)) return -1;
    const int64_t n = nrows * (cols / 32);
    if (n == 0) return 0;
    codes_kernel<<<(unsigned)((n + 255) / 256), 256, 0, (cudaStream_t)stream>>>(key, bits, row0, nrows, cols, out);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

extern "C" int synth_scales_dev(uint64_t key, int bits, int64_t row0, int64_t nrows, int64_t cols, void* out,
                                const uint16_t* tf16, const uint8_t* te8, void* stream) {
    if (cols % 32 || (bits < 2 || bits > 4) || nrows < 0) return -1;
    const int64_t n = nrows * (cols / 32);
    if (n == 0) return 0;
    scales_kernel<<<(unsigned)((n + 255) / 256), 256, 0, (cudaStream_t)stream>>>(key, bits, row0, nrows, cols, out,
                                                                                 tf16, te8);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}
