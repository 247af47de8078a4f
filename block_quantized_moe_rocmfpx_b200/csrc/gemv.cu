// gemv.cu -- standalone quantised mat-vec y[q][N] = W x over packed blocks.
//
// The mat-vec with in-kernel block dequantisation (taozi.news, "DeepSeek V4
// Flash 在 128GB 锐龙 AI MAX+ 上跑到 32 tok/s", section "ROCmFPX：把 284B 权重压进
// 128 GB"), each block decoded once for all q columns (ainomam.com, "APU 实现
// token 自由…", section "Lucebox 的优化三板斧").  A persistent CTA takes 32
// output rows (2 row-groups) at a time and its 8 warps split K in quarters;
// packed chunks are read straight from global memory with 128-bit loads.  x
// is staged once per CTA
// in shared memory as fp16 in B-fragment order: each column scaled by a power
// of two that puts max|x| in [2^13, 2^14) and each tile by 2^-s_b for the
// format's bit offsets (see rfx_tile.cuh); fp32 x becomes an exact-to-2^-22
// hi/lo pair of virtual columns.  K-quarter partials are summed in a fixed
// order.
#include <cuda_runtime.h>

#include <algorithm>

#include "gemv.h"
#include "launch_util.h"
#include "rfx_tile.cuh"

namespace rfx {

constexpr int GEMV_WARPS = 8;

__device__ __forceinline__ int gemv_s_pos(int fmt, int k, long long K) {
    const int blk = k >> 5;
    if ((blk >> 3) == (int)(K >> 8) && (K & 255)) return 0;
    const int b = blk & 7;
    return fmt == 2 ? Plane<2>::s_of(b) : (fmt == 3 ? Plane<3>::s_of(b) : Plane<4>::s_of(b));
}

template <int FMT, bool F32X, int NB>
__global__ void __launch_bounds__(GEMV_WARPS * 32) gemv_kernel(GemvParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ unsigned xmax[8];
    __shared__ int xn[8];
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int K = (int)p.K;
    const int nv = F32X ? 2 * p.q : p.q;             // virtual B columns
    float* red = (float*)smem;                        // [8][32][8]
    const int kbs = ((K / 32) + 3) & ~3;              // block-sum row stride (16-byte rows)
    float* sx = red + GEMV_WARPS * 32 * 8;            // [nv][kbs] block sums
    uint8_t* xs = (uint8_t*)(sx + nv * kbs);          // [step][v][t][4] fp16, 16-byte aligned
    const int vstride = 32 * nv;                      // bytes per k16 step
    if (threadIdx.x < 8) xmax[threadIdx.x] = 0u;
    __syncthreads();
    const long long n = (long long)p.q * K;
    // max |x| per column: K is a multiple of 32, so a warp's 32 consecutive
    // elements lie in one column (one shared atomic per warp and step)
    for (long long i0 = threadIdx.x - lane; i0 < n; i0 += blockDim.x) {
        const long long i = i0 + lane;
        const int c = (int)(i0 / K);
        float v;
        if constexpr (F32X) v = ((const float*)p.x)[i];
        else v = __uint_as_float((uint32_t)((const uint16_t*)p.x)[i] << 16);
        const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(v)));
        if (lane == 0 && m) atomicMax(&xmax[c], m);
    }
    __syncthreads();
    if (threadIdx.x < p.q) {
        const uint32_t m = xmax[threadIdx.x];
        const int e = m ? 13 - ((int)((m >> 23) & 255u) - 127) : 0;
        xn[threadIdx.x] = max(-100, min(100, e));
    }
    __syncthreads();
    // stage: each thread one k of one column (both virtual halves for fp32)
    for (long long i = threadIdx.x; i < n; i += blockDim.x) {
        const int c = (int)(i / K), k = (int)(i % K);
        const int s = gemv_s_pos(FMT, k, p.K);
        float v;
        if constexpr (F32X) v = ((const float*)p.x)[i];
        else v = __uint_as_float((uint32_t)((const uint16_t*)p.x)[i] << 16);
        const float sc = __int_as_float((127 + xn[c] - s) << 23);
        const float vs = v * __int_as_float((127 + xn[c]) << 23);
        const int step = k >> 4, r = k & 15;
        const int tt = (r & 7) >> 1, pos = (r >> 3) * 2 + (r & 1);
        uint16_t* base = (uint16_t*)xs + ((long long)(step * nv) * 4 + tt) * 4 + pos;
        if constexpr (F32X) {
            const __half hi = __float2half_rn(vs * __int_as_float((127 - s) << 23));
            const __half lo = __float2half_rn((vs - __half2float(__float2half_rn(vs))) * __int_as_float((127 - s) << 23));
            base[(2 * c) * 16] = __half_as_ushort(hi);
            base[(2 * c + 1) * 16] = __half_as_ushort(lo);
        } else {
            base[c * 16] = __half_as_ushort(__float2half_rn(v * sc));
        }
    }
    __syncthreads();
    // block sums of the staged values (times 2^s_b), per virtual column
    for (int i = threadIdx.x; i < nv * (K / 32); i += blockDim.x) {
        const int v = i / (K / 32), kb = i % (K / 32);
        float sum = 0.f;
        for (int kk = 0; kk < 32; ++kk) {
            const int k = kb * 32 + kk;
            const int step = k >> 4, r = k & 15;
            const int tt = (r & 7) >> 1, pos = (r >> 3) * 2 + (r & 1);
            const uint16_t hv = ((const uint16_t*)xs)[((long long)(step * nv + v) * 4 + tt) * 4 + pos];
            sum += __half2float(__ushort_as_half(hv));
        }
        sx[v * kbs + kb] = sum * __int_as_float((127 + gemv_s_pos(FMT, kb * 32, p.K)) << 23);
    }
    __syncthreads();
    BSrc bs[2];
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
        const int v = 8 * nb + g;
        bs[nb] = {xs + (v * 4 + t) * 8, vstride, v < nv};
    }
    const int nch = rfx_num_chunks(p.K);
    const int kq = w >> 1;
    const int c0 = kq * nch / 4, c1 = (kq + 1) * nch / 4;
    const int fullb = (int)rfx_chunk_bytes(FMT, 8);
    const long long rgb = rfx_rowgroup_bytes(FMT, p.K);
    const long long npairs = ((p.N + 15) / 16 + 1) / 2;
    // persistent: x is staged once per CTA, then the CTA takes row-group pairs
    // blockIdx.x, blockIdx.x + gridDim.x, ...
    for (long long pr = blockIdx.x; pr < npairs; pr += gridDim.x) {
        const long long rg = 2 * pr + (w & 1);
        const uint8_t* Wrg = p.W + rg * rgb;
        float acc[NB][4], corr[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int i = 0; i < 4; ++i) { acc[nb][i] = 0.f; corr[nb][i] = 0.f; }
        const bool live = rg * 16 < p.N;
        // block-sum rows of the lane's two virtual columns per n-block (for fp32 x
        // the hi and lo halves each carry their own sum; the corrections add up)
        const float* srow[NB][2];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int v = 8 * nb + 2 * t + j;
                srow[nb][j] = v < nv ? sx + v * kbs : nullptr;
            }
        if (live) {
            for (int c = c0; c < c1; ++c) {
                const uint8_t* st = Wrg + (long long)c * fullb;
                const int nt = rfx_chunk_tiles(p.K, c);
                const int step0 = 16 * c;
                if (nt == 8) {
                    FullChunk<FMT> f;
                    f.load(st, lane, g);
#pragma unroll
                    for (int b = 0; b < 8; ++b) {
                        uint32_t a[8];
                        switch (b) {
                            case 0: plane_regs<FMT, 0>(f.wd, f.sh, a); break;
                            case 1: plane_regs<FMT, 1>(f.wd, f.sh, a); break;
                            case 2: plane_regs<FMT, 2>(f.wd, f.sh, a); break;
                            case 3: plane_regs<FMT, 3>(f.wd, f.sh, a); break;
                            case 4: plane_regs<FMT, 4>(f.wd, f.sh, a); break;
                            case 5: plane_regs<FMT, 5>(f.wd, f.sh, a); break;
                            case 6: plane_regs<FMT, 6>(f.wd, f.sh, a); break;
                            default: plane_regs<FMT, 7>(f.wd, f.sh, a); break;
                        }
                        float s0, s1;
                        f.scales(b, s0, s1);
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb) {
                            float cc[4];
                            mma_tile(cc, a, bs[nb].get(step0 + 2 * b), bs[nb].get(step0 + 2 * b + 1));
                            acc[nb][0] = fmaf(s0, cc[0], acc[nb][0]);
                            acc[nb][1] = fmaf(s0, cc[1], acc[nb][1]);
                            acc[nb][2] = fmaf(s1, cc[2], acc[nb][2]);
                            acc[nb][3] = fmaf(s1, cc[3], acc[nb][3]);
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                if (srow[nb][j]) {
                                    const float sb = srow[nb][j][8 * c + b];
                                    corr[nb][j] = fmaf(s0, sb, corr[nb][j]);
                                    corr[nb][2 + j] = fmaf(s1, sb, corr[nb][2 + j]);
                                }
                            }
                        }
                    }
                } else {
                    for (int b = 0; b < nt; ++b) {
                        uint32_t a[8];
                        float s0, s1;
                        partial_tile<FMT>(st, nt, lane, g, b, a, s0, s1);
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb) {
                            float cc[4];
                            mma_tile(cc, a, bs[nb].get(step0 + 2 * b), bs[nb].get(step0 + 2 * b + 1));
                            // the exact level dot product in units of 2^-24 (scale untouched: it may be 2^-127)
                            acc[nb][0] = fmaf(s0, cc[0] * 0x1.0p-24f, acc[nb][0]);
                            acc[nb][1] = fmaf(s0, cc[1] * 0x1.0p-24f, acc[nb][1]);
                            acc[nb][2] = fmaf(s1, cc[2] * 0x1.0p-24f, acc[nb][2]);
                            acc[nb][3] = fmaf(s1, cc[3] * 0x1.0p-24f, acc[nb][3]);
                        }
                    }
                }
            }
        }
        float* my = red + (w * 32 + lane) * 8;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int i = 0; i < 4; ++i) my[4 * nb + i] = fmaf(-Plane<FMT>::OFF, corr[nb][i], acc[nb][i] * 0x1.0p24f);
        __syncthreads();
        if (w < 2 && live) {
            float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const float* r = red + ((2 * q4 + w) * 32 + lane) * 8;
#pragma unroll
                for (int i = 0; i < 4 * NB; ++i) s[i] += r[i];
            }
            const long long row0 = rg * 16 + g, row1 = row0 + 8;
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                if constexpr (!F32X) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int col = 8 * nb + 2 * t + (i & 1);
                        const long long row = (i >> 1) ? row1 : row0;
                        if (col < p.q && row < p.N)
                            p.y[(long long)col * p.N + row] = s[4 * nb + i] * __int_as_float((127 - xn[col]) << 23);
                    }
                } else {
                    const int col = 4 * nb + t;
                    if (col < p.q) {
                        const float sc = __int_as_float((127 - xn[col]) << 23);
                        if (row0 < p.N) p.y[(long long)col * p.N + row0] = (s[4 * nb + 0] + s[4 * nb + 1]) * sc;
                        if (row1 < p.N) p.y[(long long)col * p.N + row1] = (s[4 * nb + 2] + s[4 * nb + 3]) * sc;
                    }
                }
            }
        }
        __syncthreads();   // the reduction buffer is reused by the next pair
    }
}

size_t gemv_smem_bytes(int q, long long K, bool x_fp32) {
    const int nv = x_fp32 ? 2 * q : q;
    const size_t red = GEMV_WARPS * 32 * 8 * sizeof(float);
    const size_t sx = (size_t)nv * (((K / 32) + 3) & ~3) * sizeof(float);
    const size_t xs = (size_t)K / 16 * 32 * nv;
    return red + sx + xs;
}

template <int FMT, bool F32X, int NB>
static cudaError_t launch_t(const GemvParams& p, size_t smem, cudaStream_t stream) {
    auto kern = gemv_kernel<FMT, F32X, NB>;
    static SmemLimit limit;   // one per instantiation
    cudaError_t e = limit.ensure((const void*)kern, (int)smem);
    if (e != cudaSuccess) return e;
    // persistent grid: as many CTAs as are resident at once (x is staged once
    // per CTA), never more than there are row-group pairs
    int dev = 0, sms = 0, per_sm = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, GEMV_WARPS * 32, smem);
    if (e != cudaSuccess) return e;
    const long long npairs = ((p.N + 15) / 16 + 1) / 2;
    const int grid = (int)std::min<long long>(npairs, (long long)sms * std::max(per_sm, 1));
    (void)cudaGetLastError();   // an earlier call's launch error is not this launch's
    kern<<<grid, GEMV_WARPS * 32, smem, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t gemv_launch(const GemvParams& p, int fmt, bool x_fp32, cudaStream_t stream) {
    const size_t smem = gemv_smem_bytes(p.q, p.K, x_fp32);
    const bool two = (x_fp32 ? 2 * p.q : p.q) > 8;
    if (!x_fp32) {
        switch (fmt) {
            case 2: return launch_t<2, false, 1>(p, smem, stream);
            case 3: return launch_t<3, false, 1>(p, smem, stream);
            default: return launch_t<4, false, 1>(p, smem, stream);
        }
    }
    switch (fmt) {
        case 2: return two ? launch_t<2, true, 2>(p, smem, stream) : launch_t<2, true, 1>(p, smem, stream);
        case 3: return two ? launch_t<3, true, 2>(p, smem, stream) : launch_t<3, true, 1>(p, smem, stream);
        default: return two ? launch_t<4, true, 2>(p, smem, stream) : launch_t<4, true, 1>(p, smem, stream);
    }
}

}  // namespace rfx
