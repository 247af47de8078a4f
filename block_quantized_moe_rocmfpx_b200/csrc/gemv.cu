// gemv.cu -- standalone quantised mat-vec y[q][N] = W x over packed blocks.
//
// The mat-vec with in-kernel block dequantisation (taozi.news, "DeepSeek V4
// Flash 在 128GB 锐龙 AI MAX+ 上跑到 32 tok/s", section "ROCmFPX：把 284B 权重压进
// 128 GB"), each block decoded once for all q columns (ainomam.com, "APU 实现
// token 自由…", section "Lucebox 的优化三板斧").  A CTA owns 32 output rows
// (2 row-groups) and its 8 warps split K in quarters; packed chunks are read
// straight from global memory with 128-bit loads, x is staged once per CTA in
// shared memory in B-fragment order (bf16, or an exact-to-2^-22 fp16 hi/lo
// split of fp32 x), and the K-quarter partials are summed in a fixed order.
#include <cuda_runtime.h>

#include "gemv.h"
#include "rfx_tile.cuh"

namespace rfx {

constexpr int GEMV_WARPS = 8;

template <int FMT, bool F16, int NB>
__global__ void __launch_bounds__(GEMV_WARPS * 32) gemv_kernel(GemvParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    float* red = (float*)smem;                              // [8][32][8]
    uint8_t* xs = smem + GEMV_WARPS * 32 * 8 * sizeof(float);
    const int nsteps = (int)(p.K / 16);
    // stage x in B-fragment order
    if constexpr (!F16) {
        // bf16 [q][K] -> [c][step][t][4], column stride nsteps*32 + 32
        const int cs = nsteps * 32 + 32;
        const uint32_t* x32 = (const uint32_t*)p.x;
        const long long npairs = (long long)p.q * p.K / 2;
        for (long long i = threadIdx.x; i < npairs; i += blockDim.x) {
            const int c = (int)((2 * i) / p.K), k = (int)((2 * i) % p.K);
            const int step = k >> 4, r = k & 15;
            *(uint32_t*)(xs + c * cs + ((step * 4 + ((r & 7) >> 1)) * 8) + (r >> 3) * 4) = x32[i];
        }
    } else {
        // fp32 [q][K] -> virtual columns v = 2c (hi) / 2c+1 (lo): [step][v][t][4] fp16
        const float* xf = (const float*)p.x;
        const long long n = (long long)p.q * p.K;
        for (long long i = threadIdx.x; i < n; i += blockDim.x) {
            const int c = (int)(i / p.K), k = (int)(i % p.K);
            const int step = k >> 4, r = k & 15;
            const float v = xf[i];
            const __half hi = __float2half_rn(v);
            const __half lo = __float2half_rn(v - __half2float(hi));
            const int tt = (r & 7) >> 1, pos = (r >> 3) * 2 + (r & 1);
            uint16_t* base = (uint16_t*)xs + ((long long)(step * 2 * p.q) * 4 + tt) * 4 + pos;
            base[(2 * c) * 16] = __half_as_ushort(hi);
            base[(2 * c + 1) * 16] = __half_as_ushort(lo);
        }
    }
    __syncthreads();
    BSrc bs[2];
    if constexpr (!F16) {
        const int cs = nsteps * 32 + 32;
        bs[0] = {xs + (g < p.q ? g : 0) * cs + t * 8, 32, g < p.q};
        bs[1] = bs[0];
    } else {
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
            const int v = 8 * nb + g;
            bs[nb] = {xs + (v * 4 + t) * 8, 64 * p.q, v < 2 * p.q};
        }
    }
    const int rg = 2 * blockIdx.x + (w & 1);
    const int nch = rfx_num_chunks(p.K);
    const int kq = w >> 1;
    const int c0 = kq * nch / 4, c1 = (kq + 1) * nch / 4;
    const uint8_t* Wrg = p.W + (long long)rg * rfx_rowgroup_bytes(FMT, p.K);
    const int fullb = (int)rfx_chunk_bytes(FMT, 8);
    Acc<NB> acc;
    acc.zero();
    const bool live = (long long)rg * 16 < p.N;
    if (live) {
        for (int c = c0; c < c1; ++c)
            chunk_any<FMT, F16, NB>(Wrg + (long long)c * fullb, rfx_chunk_tiles(p.K, c), lane, g, bs, 16 * c, acc);
    }
    float* my = red + (w * 32 + lane) * 8;
#pragma unroll
    for (int n = 0; n < NB; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) my[4 * n + i] = acc.v[n][i];
    __syncthreads();
    if (w >= 2 || !live) return;
    float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
        const float* r = red + ((2 * q4 + w) * 32 + lane) * 8;
#pragma unroll
        for (int i = 0; i < 4 * NB; ++i) s[i] += r[i];
    }
    const long long row0 = (long long)rg * 16 + g, row1 = row0 + 8;
#pragma unroll
    for (int n = 0; n < NB; ++n) {
        if constexpr (!F16) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int col = 2 * t + (i & 1);
                const long long row = (i >> 1) ? row1 : row0;
                if (col < p.q && row < p.N) p.y[(long long)col * p.N + row] = s[4 * n + i];
            }
        } else {
            const int col = 4 * n + t;
            if (col < p.q) {
                if (row0 < p.N) p.y[(long long)col * p.N + row0] = s[4 * n + 0] + s[4 * n + 1];
                if (row1 < p.N) p.y[(long long)col * p.N + row1] = s[4 * n + 2] + s[4 * n + 3];
            }
        }
    }
}

size_t gemv_smem_bytes(int q, long long K, bool x_fp32) {
    const size_t red = GEMV_WARPS * 32 * 8 * sizeof(float);
    const size_t xs = x_fp32 ? (size_t)K / 16 * 64 * q : (size_t)q * ((size_t)K / 16 * 32 + 32);
    return red + xs;
}

template <int FMT, bool F16, int NB>
static cudaError_t launch_t(const GemvParams& p, size_t smem, cudaStream_t stream) {
    auto kern = gemv_kernel<FMT, F16, NB>;
    static int set_bytes[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && set_bytes[dev] < (int)smem) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        set_bytes[dev] = (int)smem;
    }
    const long long ngroups = (p.N + 15) / 16;
    const int grid = (int)((ngroups + 1) / 2);
    kern<<<grid, GEMV_WARPS * 32, smem, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t gemv_launch(const GemvParams& p, int fmt, bool x_fp32, cudaStream_t stream) {
    const size_t smem = gemv_smem_bytes(p.q, p.K, x_fp32);
    if (!x_fp32) {
        switch (fmt) {
            case 2: return launch_t<2, false, 1>(p, smem, stream);
            case 3: return launch_t<3, false, 1>(p, smem, stream);
            default: return launch_t<4, false, 1>(p, smem, stream);
        }
    }
    const bool two = p.q > 4;
    switch (fmt) {
        case 2: return two ? launch_t<2, true, 2>(p, smem, stream) : launch_t<2, true, 1>(p, smem, stream);
        case 3: return two ? launch_t<3, true, 2>(p, smem, stream) : launch_t<3, true, 1>(p, smem, stream);
        default: return two ? launch_t<4, true, 2>(p, smem, stream) : launch_t<4, true, 1>(p, smem, stream);
    }
}

}  // namespace rfx
