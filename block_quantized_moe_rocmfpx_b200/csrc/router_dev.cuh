// router_dev.cuh -- one warp's router top-k + softmax for one token.
//
// ainomam.com, "APU 实现 token 自由…", section "Lucebox 的优化三板斧" (tuned
// TOP-K / ARGSORT routing kernels; 6 of 256 experts active) and m.mzlw.cn,
// "Lucebox专攻DeepSeek V4…", section "MoE 专家并行" (top-6 of 256).  Every
// lane keeps its strided share of the logits in registers, and k rounds of a
// warp-shuffle arg-max pick the winners in descending order (equal values:
// lower expert index first); the weights are the softmax over the k selected
// logits, summed in routing order.  No sort and no shared memory.
#pragma once
#include <math.h>
#include <stdint.h>

namespace rfx {

// Lane j < k writes idx_out[j] and w_out[j].  E <= 32 * PER_LANE.  COHERENT:
// the logits were written earlier in the same kernel by other CTAs (read
// through L2, not the read-only path).
template <int PER_LANE, bool COHERENT = false>
__device__ __forceinline__ void router_warp(const float* __restrict__ l, int E, int k, int32_t* idx_out,
                                            float* w_out) {
    const int lane = threadIdx.x & 31;
    float v[PER_LANE];
    uint32_t live = 0;
#pragma unroll
    for (int i = 0; i < PER_LANE; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? (COHERENT ? __ldcg(l + e) : __ldg(l + e)) : 0.f;
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
    float z = 0.f;
    for (int j = 0; j < k; ++j) {
        const float vj = __shfl_sync(0xffffffffu, sel_v, j);
        z += expf(vj - v0);
    }
    if (lane < k) {
        idx_out[lane] = sel_e;
        w_out[lane] = expf(sel_v - v0) / z;
    }
}

}  // namespace rfx
