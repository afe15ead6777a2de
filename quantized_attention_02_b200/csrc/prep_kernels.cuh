// prep_kernels.cuh -- launchers for the K-smoothing and INT8 quantization kernels.
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace sage {

// km[bh, c] = mean over N tokens of k[bh, :, c]; k fp16 [BH, N, D], km fp32 [BH, D].
cudaError_t launch_smooth_k(const __half* k, float* km, int BH, int N, int D, cudaStream_t st);

// Quantize x fp16 [BH, N, D] in groups of `group` tokens (1, 64 or 128) to int8 q and fp32
// scales s [BH, N/group].  km (fp32 [BH, D]) is subtracted first when not null.
cudaError_t launch_quant(const __half* x, const float* km, int8_t* q, float* s, int BH, int N, int D, int group,
                         cudaStream_t st);

}  // namespace sage
