// router.cu -- router top-k + softmax over the selected logits, one warp per
// token (the warp's work is router_warp in router_dev.cuh).  Launched as a
// programmatic dependent of the kernel before it: the launch overlaps that
// kernel's tail, and every load waits until it has finished (the logits may be
// its output, and idx / w may still be its input); the next kernel may launch
// at once.
#include <cuda_runtime.h>
#include <stdint.h>

#include "rfx_device.cuh"
#include "router_dev.cuh"

namespace rfx {

constexpr int ROUTER_WARPS = 8;

template <int PER_LANE>
__global__ void __launch_bounds__(ROUTER_WARPS * 32) router_topk_kernel(const float* __restrict__ logits, int T, int E,
                                                                       int k, int32_t* __restrict__ idx,
                                                                       float* __restrict__ w) {
    grid_dep_launch();
    grid_dep_wait();
    const int tok = blockIdx.x * ROUTER_WARPS + (threadIdx.x >> 5);
    if (tok >= T) return;
    router_warp<PER_LANE>(logits + (long long)tok * E, E, k, idx + (long long)tok * k, w + (long long)tok * k);
}

template <int PER_LANE>
cudaError_t launch(const float* logits, int T, int E, int k, int32_t* idx, float* w, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((T + ROUTER_WARPS - 1) / ROUTER_WARPS);
    cfg.blockDim = dim3(ROUTER_WARPS * 32);
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, router_topk_kernel<PER_LANE>, logits, T, E, k, idx, w);
}

cudaError_t router_topk_launch(const float* logits, int T, int E, int k, int32_t* idx, float* w,
                               cudaStream_t stream) {
    const int per = (E + 31) / 32;
    if (per <= 1) return launch<1>(logits, T, E, k, idx, w, stream);
    if (per <= 2) return launch<2>(logits, T, E, k, idx, w, stream);
    if (per <= 4) return launch<4>(logits, T, E, k, idx, w, stream);
    if (per <= 8) return launch<8>(logits, T, E, k, idx, w, stream);
    if (per <= 16) return launch<16>(logits, T, E, k, idx, w, stream);
    return launch<32>(logits, T, E, k, idx, w, stream);
}

}  // namespace rfx
