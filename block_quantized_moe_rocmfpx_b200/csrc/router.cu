// router.cu -- router top-k + softmax over the selected logits, one warp per
// token (the warp's work is router_warp in router_dev.cuh).
#include <cuda_runtime.h>
#include <stdint.h>

#include "router_dev.cuh"

namespace rfx {

constexpr int ROUTER_WARPS = 8;

template <int PER_LANE>
__global__ void __launch_bounds__(ROUTER_WARPS * 32) router_topk_kernel(const float* __restrict__ logits, int T, int E,
                                                                       int k, int32_t* __restrict__ idx,
                                                                       float* __restrict__ w) {
    const int tok = blockIdx.x * ROUTER_WARPS + (threadIdx.x >> 5);
    if (tok >= T) return;
    router_warp<PER_LANE>(logits + (long long)tok * E, E, k, idx + (long long)tok * k, w + (long long)tok * k);
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
