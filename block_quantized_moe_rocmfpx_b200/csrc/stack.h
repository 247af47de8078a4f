// stack.h -- layer chaining kernel (stack.cu).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace rfx {

// x[t] = bf16(y[t] / sqrt(mean(y[t]^2))) for each of T columns of H values.
cudaError_t rms_bf16_launch(const float* y, int T, int H, uint16_t* x, cudaStream_t stream);

}  // namespace rfx
