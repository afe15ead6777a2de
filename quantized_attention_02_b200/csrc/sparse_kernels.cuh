// sparse_kernels.cuh -- the first stage (predicted block map) of the block-sparse variant.
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace sage {

constexpr int kSparseBQ = 256;             // query block: the fused kernel's pair of 128-row query tiles
constexpr int kSparseBK = 128;             // key block: the fused kernel's key tile
constexpr int kSparseMaxKeyBlocks = 512;   // N <= 65536

// Bytes of device workspace launch_sparse_predict needs (block means and similarities).
size_t sparse_predict_workspace(int BH, int N, int D);

// q, k: fp16 [BH][N][D]; kv_count: int [BH][ceil(N/256)]; kv_index: int16 [BH][ceil(N/256)][ceil(N/128)]
// (entries past the count are left as they were).
cudaError_t launch_sparse_predict(const __half* q, const __half* k, void* workspace, int BH, int N, int D, int causal,
                                  float sm_scale, float tau, float theta, int* kv_count, int16_t* kv_index,
                                  cudaStream_t st);

}  // namespace sage
