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
// B200 design, T <= 8 (decode / verify): a GEMV over E rows (2 MB for 256 x
// 4096), HBM-bound, spread over all SMs.  A CTA owns two rows and up to 8
// columns; each of its 8 warps takes a quarter of H for one row (16-byte loads of 8 bf16 of W and of x, fp32 FMAs in
// index order per lane, then a butterfly over the lanes); the four quarters
// are added in a fixed tree, so a logit's bits depend neither on T nor on the
// launch.  W is a constant input: each warp asks L2 for its slice before the
// kernel waits for the previous one (programmatic dependent launch); x may come
// from that kernel and is read after the wait.
//
// T > 8 (prefill): a tcgen05 GEMM, logits^T = W x^T, bf16 operands with fp32
// accumulation in tensor memory (every product is exact; the sums are fp32
// in the tensor core's fixed order per element, so a column's logits do not
// depend on the other columns).  Operands by TMA, one MMA thread, 4 epilogue
// warps (below).
#include <cuda_runtime.h>
#include <stdint.h>

#include <cooperative_groups.h>

#include "gemv.h"
#include "launch_util.h"
#include "rfx_device.cuh"
#include "router_dev.cuh"
#include "tc.cuh"
#include "tmap.h"

namespace rfx {

namespace cg = cooperative_groups;

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

// The projection of the CTA's RP_ROWS rows for up to RP_COLS columns.
__device__ __forceinline__ void project_rows(const uint16_t* __restrict__ W, const float* __restrict__ bias,
                                             const uint16_t* __restrict__ x, int T, int H, int E,
                                             float* __restrict__ logits) {
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
        const int nch = kp / 8;   // 16-byte chunks of the warp's quarter
        // four chunks per lane in flight at once (H = 4096: all of them)
        for (int ch0 = lane; ch0 < nch; ch0 += 4 * 32) {
            uint4 wv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int ch = ch0 + 32 * u;
                wv[u] = ch < nch ? __ldg(w4 + ch) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int ch = ch0 + 32 * u;
                if (ch >= nch) break;
                float wf[8];
                bf16x8(wv[u], wf);
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

__global__ void __launch_bounds__(RP_THREADS) router_logits_kernel(const uint16_t* __restrict__ W,
                                                                  const float* __restrict__ bias,
                                                                  const uint16_t* __restrict__ x, int T, int H, int E,
                                                                  float* __restrict__ logits) {
    grid_dep_launch();
    project_rows(W, bias, x, T, H, E, logits);
}

// T <= 8 with the top-k in the same launch (cooperative: every CTA is
// resident): after a grid-wide barrier that orders the logit stores, warp t of
// CTA 0 runs the router's warp top-k on column t.
template <int PER_LANE>
__global__ void __launch_bounds__(RP_THREADS) router_project_topk_kernel(const uint16_t* __restrict__ W,
                                                                        const float* __restrict__ bias,
                                                                        const uint16_t* __restrict__ x, int T, int H,
                                                                        int E, int k, float* __restrict__ logits,
                                                                        int32_t* __restrict__ idx,
                                                                        float* __restrict__ w) {
    grid_dep_launch();
    project_rows(W, bias, x, T, H, E, logits);
    cg::this_grid().sync();
    const int warp = threadIdx.x >> 5;
    if (blockIdx.x == 0 && warp < T)
        router_warp<PER_LANE, true>(logits + (size_t)warp * E, E, k, idx + (size_t)warp * k, w + (size_t)warp * k);
}

// ------------------------------------------------------------- T > 8 ---
//
// A CTA computes 128 experts x 128 tokens: K in steps of 64 through a 6-stage
// ring of TMA boxes (128 rows of W, 128 rows of x, 128-byte swizzle; rows and
// columns beyond the tensors read as zero); one thread issues the
// 128 x 128 x 16 MMAs into a 128-column fp32 accumulator in tensor memory; 4
// warps (one tensor-memory lane quarter each) add the bias and store the
// logits.  Every wait is bounded; a CTA that gives up stores nothing (the
// test of the call is its parity check).
constexpr int RT_BM = 128, RT_BN = 128, RT_BK = 64, RT_NS = 6;
constexpr int RT_TILE_A = RT_BM * RT_BK * 2, RT_TILE_B = RT_BN * RT_BK * 2, RT_STAGE = RT_TILE_A + RT_TILE_B;
static_assert(RT_TILE_A % 1024 == 0 && RT_TILE_B % 1024 == 0, "swizzle atoms must stay 1024-byte aligned");
constexpr int RT_THREADS = 256;   // warp 0: TMA; warp 1: tensor memory + MMA; warps 4..7: epilogue
constexpr size_t RT_SMEM = 1024 + (size_t)RT_NS * RT_STAGE;
constexpr long long RT_WAIT = 1000000000LL;   // SM clocks before a wait gives up

struct RtShared {
    uint64_t full[RT_NS], empty[RT_NS], acc;
    uint32_t tmem;
    volatile int abort;
};

__global__ void __launch_bounds__(RT_THREADS, 1)
    router_logits_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                            const float* __restrict__ bias, int T, int H, int E, float* __restrict__ logits) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    RtShared& sh = *reinterpret_cast<RtShared*>(smem_raw);
    const uint32_t off = ((smem_u32(smem_raw) + (uint32_t)sizeof(RtShared) + 1023u) & ~1023u) - smem_u32(smem_raw);
    if (off > 1024u) return;   // the ring would overrun the allocation
    uint8_t* ring = smem_raw + off;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e0 = blockIdx.x * RT_BM, t0 = blockIdx.y * RT_BN;
    const int nk = (H + RT_BK - 1) / RT_BK;
    grid_dep_launch();
    if (threadIdx.x == 0) {
        for (int s = 0; s < RT_NS; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], 1);
        }
        mbar_init(&sh.acc, 1);
        sh.abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        __syncwarp();
        tmem_alloc(&sh.tmem, RT_BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem;
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
        const uint64_t pol = policy_evict_last();
        grid_dep_wait();   // x may be the previous kernel's output
        int ks = 0;
        for (; ks < nk; ++ks) {
            const int s = ks % RT_NS;
            if (!mbar_wait(&sh.empty[s], ((uint32_t)(ks / RT_NS) & 1u) ^ 1u, RT_WAIT)) {
                sh.abort = 1;
                break;
            }
            uint8_t* a = ring + (size_t)s * RT_STAGE;
            mbar_arrive_expect_tx(&sh.full[s], RT_STAGE);
            tma_load_2d(a, &tmW, ks * RT_BK, e0, &sh.full[s], pol);
            tma_load_2d(a + RT_TILE_A, &tmX, ks * RT_BK, t0, &sh.full[s], pol);
        }
        // no copy may land after the CTA exits
        for (int i = 1; i <= RT_NS && ks - i >= 0; ++i) {
            const int g = ks - i;
            (void)mbar_wait(&sh.full[g % RT_NS], (uint32_t)(g / RT_NS) & 1u, RT_WAIT);
        }
    } else if (warp == 1 && lane == 0) {
        const uint32_t idesc = idesc_bf16_m128(RT_BN);
        for (int ks = 0; ks < nk; ++ks) {
            const int s = ks % RT_NS;
            if (!mbar_wait(&sh.full[s], (uint32_t)(ks / RT_NS) & 1u, RT_WAIT) || sh.abort) {
                sh.abort = 1;
                break;
            }
            tc_fence_after();
            const uint32_t a = smem_u32(ring + (size_t)s * RT_STAGE), b = a + RT_TILE_A;
#pragma unroll
            for (int kk = 0; kk < RT_BK / 16; ++kk)
                tc_mma_bf16(tmem, sw128_desc(a + kk * 32), sw128_desc(b + kk * 32), idesc, (ks | kk) != 0);
            tc_commit(&sh.empty[s]);
        }
        tc_commit(&sh.acc);
        // every MMA is done before tensor memory is released
        if (!mbar_wait(&sh.acc, 0u, RT_WAIT)) sh.abort = 1;
    } else if (warp >= 4) {
        const int q = warp & 3;   // the tensor-memory lane quarter this warp may read
        const bool ok = mbar_wait(&sh.acc, 0u, RT_WAIT);
        tc_fence_after();
        if (__all_sync(0xffffffffu, ok) && !sh.abort) {
            const int e = e0 + 32 * q + lane;
            const float bv = (bias && e < E) ? __ldg(bias + e) : 0.f;
            for (int c0 = 0; c0 < RT_BN && t0 + c0 < T; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int t = t0 + c0 + j;
                    if (e < E && t < T) logits[(size_t)t * E + e] = __uint_as_float(v[j]) + bv;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, RT_BN);
    }
}

cudaError_t router_logits_launch(const uint16_t* W, const float* bias, const uint16_t* x, int T, int H, int E,
                                 float* logits, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    if (T > RP_COLS) {
        static SmemLimit limit;
        cudaError_t e = limit.ensure((const void*)router_logits_tc_kernel, (int)RT_SMEM);
        if (e != cudaSuccess) return e;
        CUtensorMap tmW, tmX;
        if (!make_tmap_bf16(&tmW, W, E, H, RT_BM) || !make_tmap_bf16(&tmX, x, T, H, RT_BN))
            return cudaErrorInvalidValue;
        cfg.gridDim = dim3((unsigned)((E + RT_BM - 1) / RT_BM), (unsigned)((T + RT_BN - 1) / RT_BN));
        cfg.blockDim = dim3(RT_THREADS);
        cfg.dynamicSmemBytes = RT_SMEM;
        cfg.stream = stream;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, router_logits_tc_kernel, tmW, tmX, bias, T, H, E, logits);
    }
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

template <int PER_LANE>
static cudaError_t launch_fused(const uint16_t* W, const float* bias, const uint16_t* x, int T, int H, int E, int k,
                                float* logits, int32_t* idx, float* w, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((E + RP_ROWS - 1) / RP_ROWS));
    cfg.blockDim = dim3(RP_THREADS);
    cfg.stream = stream;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, router_project_topk_kernel<PER_LANE>, W, bias, x, T, H, E, k, logits, idx, w);
}

// The fused launch when every CTA fits on the device at once, else the two
// launches (cudaErrorNotSupported tells the caller to use them).
template <int PER_LANE>
static bool fused_fits(int E) {
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, router_project_topk_kernel<PER_LANE>, RP_THREADS, 0) !=
        cudaSuccess)
        return false;
    return (long long)per_sm * sms >= (E + RP_ROWS - 1) / RP_ROWS;
}

cudaError_t router_project_topk_launch(const uint16_t* W, const float* bias, const uint16_t* x, int T, int H, int E,
                                       int k, float* logits, int32_t* idx, float* w, cudaStream_t stream) {
    const int per = (E + 31) / 32;
    const bool fits = per <= 1 ? fused_fits<1>(E) : per <= 2 ? fused_fits<2>(E) : per <= 4 ? fused_fits<4>(E)
                      : per <= 8 ? fused_fits<8>(E) : per <= 16 ? fused_fits<16>(E) : fused_fits<32>(E);
    if (!fits) return cudaErrorNotSupported;
    if (per <= 1) return launch_fused<1>(W, bias, x, T, H, E, k, logits, idx, w, stream);
    if (per <= 2) return launch_fused<2>(W, bias, x, T, H, E, k, logits, idx, w, stream);
    if (per <= 4) return launch_fused<4>(W, bias, x, T, H, E, k, logits, idx, w, stream);
    if (per <= 8) return launch_fused<8>(W, bias, x, T, H, E, k, logits, idx, w, stream);
    if (per <= 16) return launch_fused<16>(W, bias, x, T, H, E, k, logits, idx, w, stream);
    return launch_fused<32>(W, bias, x, T, H, E, k, logits, idx, w, stream);
}

}  // namespace rfx
