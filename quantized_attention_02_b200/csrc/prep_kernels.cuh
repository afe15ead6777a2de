// prep_kernels.cuh -- launchers for the K-smoothing and INT8 quantization kernels.
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace sage {

// km[bh, c] = mean over N tokens of k[bh, :, c]; k fp16 [BH, N, D], km fp32 [BH, D].
cudaError_t launch_smooth_k(const __half* k, float* km, int BH, int N, int D, cudaStream_t st);
// K mean, K codes and Q codes in one launch (one cluster per head, one pass over its tokens);
// same results as launch_smooth_k followed by launch_quant_qk with the mean.
cudaError_t launch_prep_fused(const __half* q, const __half* k, float* km, int8_t* q8, int8_t* k8, float* sq,
                              float* sk, int BH, int N, int D, bool per_token, cudaStream_t st);
// V to E4M3 with per-(head, channel) scales sv; vm: channel means (V smoothed) or nullptr (not smoothed).
cudaError_t launch_quant_v_fp8(const __half* v, uint8_t* v8, float* sv, float* vm, int BH, int N, int D,
                               cudaStream_t st);

// Quantize q and k fp16 [BH, N, D] to int8 q8 / k8 with fp32 scales sq / sk (one launch per
// tensor): per token (per_token), else in groups of 128 Q tokens and 64 K tokens.  km (fp32 [BH, D])
// is subtracted from k first when not null.
cudaError_t launch_quant_qk(const __half* q, const __half* k, const float* km, int8_t* q8, int8_t* k8, float* sq,
                            float* sk, int BH, int N, int D, bool per_token, cudaStream_t st);

// Microscaling FP4 variant (head dimension D = 64 or 128).  Q and K (minus km when not null) to
// E2M1 codes [BH][N][D/2 bytes] and tile scales [BH][ceil(N/128)]; scale atoms of Q
// [BH][ceil(N/128)][D/64][512], of K [BH][ceil(N/64)][D/64][512] (64 tokens per atom).
cudaError_t launch_quant_qk_fp4(const __half* q, const __half* k, const float* km, uint8_t* q4, uint8_t* sfq,
                                float* gq, uint8_t* k4, uint8_t* sfk, float* gk, int BH, int N, int D,
                                cudaStream_t st);
// V to E2M1 along the tokens: transposed codes [BH][D][ceil(N/128) * 64 bytes], scale atoms
// [BH][ceil(N/128)][2][512] (the channels as rows), channel scales gv [BH][D], channel means vm
// (V smoothed; nullptr: not smoothed), rv [BH][D] scratch (the inverse channel scales).
cudaError_t launch_quant_v_fp4(const __half* v, uint8_t* v4t, uint8_t* sfv, float* gv, float* vm, float* rv, int BH,
                               int N, int D, cudaStream_t st);

}  // namespace sage
