// router.cu -- router top-k + softmax over the selected logits.
//
// ainomam.com, "APU 实现 token 自由…", section "Lucebox 的优化三板斧" (tuned
// TOP-K / ARGSORT routing kernels; 6 of 256 experts active) and m.mzlw.cn,
// "Lucebox专攻DeepSeek V4…", section "MoE 专家并行" (top-6 of 256).  One warp
// per token: every lane keeps its strided share of the logits in registers,
// and k rounds of a warp-shuffle arg-max pick the winners in descending order
// (equal values: lower expert index first).  No sort and no shared memory.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

namespace rfx {

constexpr int ROUTER_WARPS = 8;

template <int PER_LANE>
__global__ void __launch_bounds__(ROUTER_WARPS * 32) router_topk_kernel(const float* __restrict__ logits, int T, int E,
                                                                       int k, int32_t* __restrict__ idx,
                                                                       float* __restrict__ w) {
    const int lane = threadIdx.x & 31;
    const int tok = blockIdx.x * ROUTER_WARPS + (threadIdx.x >> 5);
    if (tok >= T) return;
    const float* l = logits + (long long)tok * E;
    float v[PER_LANE];
    uint32_t live = 0;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? __ldg(l + e) : 0.f;
        if (e < E) live |= 1u << i;
    }
    float sel_v = 0.f, v0 = 0.f;
    int sel_e = 0;
    for (int j = 0; j < k; ++j) {
        // local best among live entries: larger value, then lower index
        float bv = -INFINITY;
        int be = 0x7fffffff, bi = -1;
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i) {
            if (!(live >> i & 1u)) continue;
            const int e = lane + 32 * i;
            if (bi < 0 || v[i] > bv) { bv = v[i]; be = e; bi = i; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (oe != 0x7fffffff && (be == 0x7fffffff || ov > bv || (ov == bv && oe < be))) { bv = ov; be = oe; }
        }
        if ((be & 31) == lane) live &= ~(1u << (be >> 5));
        if (j == 0) v0 = bv;
        if (lane == j) { sel_v = bv; sel_e = be; }
    }
    // softmax over the k selected values, summed in routing order
    float z = 0.f;
    for (int j = 0; j < k; ++j) {
        const float vj = __shfl_sync(0xffffffffu, sel_v, j);
        z += expf(vj - v0);
    }
    if (lane < k) {
        idx[(long long)tok * k + lane] = sel_e;
        w[(long long)tok * k + lane] = expf(sel_v - v0) / z;
    }
}

cudaError_t router_topk_launch(const float* logits, int T, int E, int k, int32_t* idx, float* w,
                               cudaStream_t stream) {
    const int grid = (T + ROUTER_WARPS - 1) / ROUTER_WARPS;
    const int per = (E + 31) / 32;
    if (per <= 1) router_topk_kernel<1><<<grid, ROUTER_WARPS * 32, 0, stream>>>(logits, T, E, k, idx, w);
    else if (per <= 2) router_topk_kernel<2><<<grid, ROUTER_WARPS * 32, 0, stream>>>(logits, T, E, k, idx, w);
    else if (per <= 4) router_topk_kernel<4><<<grid, ROUTER_WARPS * 32, 0, stream>>>(logits, T, E, k, idx, w);
    else if (per <= 8) router_topk_kernel<8><<<grid, ROUTER_WARPS * 32, 0, stream>>>(logits, T, E, k, idx, w);
    else if (per <= 16) router_topk_kernel<16><<<grid, ROUTER_WARPS * 32, 0, stream>>>(logits, T, E, k, idx, w);
    else router_topk_kernel<32><<<grid, ROUTER_WARPS * 32, 0, stream>>>(logits, T, E, k, idx, w);
    return cudaGetLastError();
}

}  // namespace rfx
