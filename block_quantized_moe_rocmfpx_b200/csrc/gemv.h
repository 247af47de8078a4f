// gemv.h -- launch parameters of the standalone quantised mat-vec (gemv.cu).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace rfx {

struct GemvParams {
    const uint8_t* W;   // packed [N][K]
    long long N, K;
    const void* x;      // [q][K] bf16 bits or fp32
    int q;
    float* y;           // [q][N]
};

size_t gemv_smem_bytes(int q, long long K, bool x_fp32);
cudaError_t gemv_launch(const GemvParams& p, int fmt, bool x_fp32, cudaStream_t stream);
cudaError_t router_topk_launch(const float* logits, int T, int E, int k, int32_t* idx, float* w, cudaStream_t stream);
cudaError_t router_logits_launch(const uint16_t* W, const float* bias, const uint16_t* x, int T, int H, int E,
                                 float* logits, cudaStream_t stream);
// T <= 8: the projection and the top-k in one cooperative launch.
cudaError_t router_project_topk_launch(const uint16_t* W, const float* bias, const uint16_t* x, int T, int H, int E,
                                       int k, float* logits, int32_t* idx, float* w, cudaStream_t stream);
cudaError_t pack_device_launch(int fmt, const uint8_t* codes, const void* scales, long long rows, long long cols,
                               uint8_t* dst, cudaStream_t stream);

}  // namespace rfx
