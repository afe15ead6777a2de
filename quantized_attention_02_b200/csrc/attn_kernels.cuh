// attn_kernels.cuh -- launchers for the fused attention kernel and the INT32 Q.K^T debug kernel.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace sage {

struct AttnArgs {
  const CUtensorMap* tm_q;  // int8 [BH][N][D] (3-D), box {D, 128, 1}, 128 B (D=128) / 64 B (D=64) swizzle
  const CUtensorMap* tm_k;  // int8 [BH][N][D] (3-D), same boxes
  const CUtensorMap* tm_v;  // fp16 [BH][N][D] (3-D), box {64, 128, 1}, 128 B swizzle
  const CUtensorMap* tm_o;  // fp16 [BH][N][D] (3-D), box {64, 128, 1}, no swizzle (TMA store of O, D = 128)
  const float* sq;          // [BH, N] per token or [BH, ceil(N/128)] per block
  const float* sk;          // [BH, N] per token or [BH, ceil(N/64)] per block
  __half* o;                // fp16 [BH, N, D]
  int BH, N, D;
  bool causal, per_token;
  float sm_scale_log2;      // sm_scale * log2(e)
  long long* trace = nullptr;  // non-null: traced build, stamps of the first trace_ctas CTAs
  int trace_ctas = 0;
  // FP8 P.V variant (D = 128): tm_v maps E4M3 codes [BH][N][128] (box {128, 128, 1}, 128 B
  // swizzle); sv: per-(head, channel) scales [BH][128]; vm: channel means [BH][128] or null
  bool fp8 = false;
  const float* sv = nullptr;
  const float* vm = nullptr;
  // block-sparse variant (D = 128, fp16 P.V): per CTA (head, pair of query tiles) the number of
  // kept key tiles and their ascending list ([BH][ceil(N/256)][ceil(N/128)] int16); the stage-2
  // threshold in log2 units (+inf: no stage 2)
  const int* kv_count = nullptr;
  const int16_t* kv_index = nullptr;
  float skip_lambda = 0.f;
};

cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st);

// Microscaling FP4 variant (head dimension D = 64 or 128): E2M1 codes, UE4M3 scale atoms and fp32
// tile / channel scales as written by launch_quant_qk_fp4 / launch_quant_v_fp4.
struct Fp4Args {
  const CUtensorMap* tm_q;  // uint8 [BH][N][D/2] (3-D), box {D/2, 128, 1}, 64 B (D=128) / 32 B (D=64) swizzle
  const CUtensorMap* tm_k;  // uint8 [BH][N][D/2], box {D/2, 64, 1} (64 keys), same swizzle
  const CUtensorMap* tm_v;  // uint8 [BH][D][ceil(N/128) * 64] (V transposed), box {32, D, 1}, 32 B swizzle
  const uint8_t* sfq;       // [BH][ceil(N/128)][D/64][512] scale atoms of Q
  const uint8_t* sfk;       // [BH][ceil(N/64)][D/64][512] of K (64 tokens per atom)
  const uint8_t* sfv;       // [BH][ceil(N/128)][2][512] of V (channels as rows)
  const float* gq;          // [BH][ceil(N/128)] tile scales of Q and K
  const float* gk;
  const float* gv;          // [BH][D] channel scales of V
  const float* vm;          // [BH][D] channel means of V, or null
  __half* o;                // fp16 [BH][N][D]
  int BH, N, D;
  bool causal;
  float sm_scale_log2;      // sm_scale * log2(e)
};
cudaError_t launch_attn_fp4(const Fp4Args& a, cudaStream_t st);
cudaError_t launch_qk_debug(const CUtensorMap& tq, const CUtensorMap& tk, int32_t* s, int BH, int N, int D,
                            cudaStream_t st);
// One warp waits on an mbarrier that nothing arrives on, with the pipelines' bounded wait.
cudaError_t launch_wait_timeout(int* out, cudaStream_t st);
// Synchronizes st, returns the device status word (and clears it); -1 if a CUDA call failed.
int read_and_clear_device_error(cudaStream_t st, cudaError_t* err);

}  // namespace sage
