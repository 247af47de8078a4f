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
// 4096), HBM-bound, spread over all SMs.  A CTA owns two rows and up to 8 columns; each of its 8 warps takes a
// quarter of H for one row (16-byte loads of 8 bf16 of W and of x, fp32 FMAs in
// index order per lane, then a butterfly over the lanes); the four quarters
// are added in a fixed tree, so a logit's bits depend neither on T nor on the
// launch.  W is a constant input: each warp asks L2 for its slice before the
// kernel waits for the previous one (programmatic dependent launch); x may come
// from that kernel and is read after the wait.
//
// T > 8 (prefill): a tensor-core GEMM, logits^T = W x^T, bf16 operands with
// fp32 accumulation (mma.sync m16n8k16: every product is exact, the sums are
// fp32 in a fixed order per element).  A CTA computes 64 experts x 32 tokens
// (256 CTAs at E = 256, T = 2048); K runs in chunks of 64 staged by cp.async
// through a 4-deep shared-memory ring (padded rows: conflict-free ldmatrix);
// 4 warps of 32 x 16.
#include <cuda_runtime.h>
#include <stdint.h>

#include <cooperative_groups.h>

#include "gemv.h"
#include "launch_util.h"
#include "rfx_device.cuh"
#include "router_dev.cuh"

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

constexpr int RM_BM = 64, RM_BN = 32, RM_BK = 64, RM_STAGES = 4;
constexpr int RM_LD = RM_BK + 8;   // padded row (144 bytes): ldmatrix rows hit distinct banks
constexpr int RM_THREADS = 128;
constexpr int RM_STAGE_ELEMS = (RM_BM + RM_BN) * RM_LD;
constexpr size_t RM_SMEM = (size_t)RM_STAGES * RM_STAGE_ELEMS * 2;

__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, bool valid) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(valid ? 16 : 0) : "memory");
}

__device__ __forceinline__ void ldsm_x4(const void* p, uint32_t r[4]) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(a));
}

__global__ void __launch_bounds__(RM_THREADS) router_logits_mma_kernel(const uint16_t* __restrict__ W,
                                                                      const float* __restrict__ bias,
                                                                      const uint16_t* __restrict__ x, int T, int H,
                                                                      int E, float* __restrict__ logits) {
    extern __shared__ __align__(16) uint16_t rm_smem[];   // [stage][A rows 64 | B rows 32][RM_LD]
    grid_dep_launch();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int e0 = blockIdx.x * RM_BM, t0 = blockIdx.y * RM_BN;
    const int wm = (warp >> 1) * 32, wn = (warp & 1) * 16;
    const int nk = (H + RM_BK - 1) / RM_BK;
    // stage tiles: A 64 rows x 8 pieces of 16 bytes (4 per thread), B 32 x 8 (2 per thread);
    // a K tail shorter than 64 (H % 64 == 32) is zero-filled
    auto load = [&](int kc) {
        uint16_t* sa = rm_smem + (kc % RM_STAGES) * RM_STAGE_ELEMS;
        uint16_t* sb = sa + RM_BM * RM_LD;
        const int pc = tid & 7, k = kc * RM_BK + pc * 8;
        const bool kv = k < H;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const int r = (tid >> 3) + 16 * h;
            const bool v = kv && e0 + r < E;
            cp_async16_zfill(sa + r * RM_LD + pc * 8, W + (size_t)(v ? e0 + r : 0) * H + (kv ? k : 0), v);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = (tid >> 3) + 16 * h;
            const bool v = kv && t0 + r < T;
            cp_async16_zfill(sb + r * RM_LD + pc * 8, x + (size_t)(v ? t0 + r : 0) * H + (kv ? k : 0), v);
        }
    };
    grid_dep_wait();   // x may be the previous kernel's output
    float acc[2][2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[i][j][c] = 0.f;
#pragma unroll
    for (int s = 0; s < RM_STAGES - 1; ++s) {
        if (s < nk) load(s);
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    for (int kc = 0; kc < nk; ++kc) {
        asm volatile("cp.async.wait_group %0;" ::"n"(RM_STAGES - 2) : "memory");
        __syncthreads();   // stage kc landed for all threads; stage kc - 1 is free again
        if (kc + RM_STAGES - 1 < nk) load(kc + RM_STAGES - 1);
        asm volatile("cp.async.commit_group;" ::: "memory");
        const uint16_t* sa = rm_smem + (kc % RM_STAGES) * RM_STAGE_ELEMS;
        const uint16_t* sb = sa + RM_BM * RM_LD;
#pragma unroll
        for (int ks = 0; ks < RM_BK; ks += 16) {
            uint32_t a[2][4], b[4];
#pragma unroll
            for (int i = 0; i < 2; ++i) ldsm_x4(sa + (wm + 16 * i + (lane & 15)) * RM_LD + ks + (lane >> 4) * 8, a[i]);
            // B is stored [token][k]: matrices (n 0-7, k 0-7), (n 0-7, k 8-15), (n 8-15, k 0-7), (n 8-15, k 8-15)
            ldsm_x4(sb + (wn + (lane & 7) + ((lane >> 4) << 3)) * RM_LD + ks + ((lane >> 3) & 1) * 8, b);
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) mma16816<false>(acc[i][j], a[i], b[2 * j], b[2 * j + 1], acc[i][j]);
        }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    // acc[i][j]: rows (experts) wm + 16 i + g (+8), columns (tokens) wn + 8 j + 2 t (+1)
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int e = e0 + wm + 16 * i + g + 8 * hr;
            if (e >= E) continue;
            const float bv = bias ? __ldg(bias + e) : 0.f;
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int tok = t0 + wn + 8 * j + 2 * t + cc;
                    if (tok < T) logits[(size_t)tok * E + e] = acc[i][j][2 * hr + cc] + bv;
                }
        }
}

cudaError_t router_logits_launch(const uint16_t* W, const float* bias, const uint16_t* x, int T, int H, int E,
                                 float* logits, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    if (T > RP_COLS) {
        static SmemLimit limit;
        cudaError_t e = limit.ensure((const void*)router_logits_mma_kernel, (int)RM_SMEM);
        if (e != cudaSuccess) return e;
        cfg.gridDim = dim3((unsigned)((E + RM_BM - 1) / RM_BM), (unsigned)((T + RM_BN - 1) / RM_BN));
        cfg.blockDim = dim3(RM_THREADS);
        cfg.dynamicSmemBytes = RM_SMEM;
        cfg.stream = stream;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, router_logits_mma_kernel, W, bias, x, T, H, E, logits);
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
