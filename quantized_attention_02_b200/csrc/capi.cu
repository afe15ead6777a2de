// capi.cu -- the C ABI declared in include/sage_attn.h: argument validation, TMA tensor
// maps, stream-ordered workspace and the launches of the three steps of the method
// (smooth K -> quantize Q and K -> fused INT8/FP16 attention).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <nvtx3/nvToolsExt.h>  // header-only NVTX3: ranges cost a pointer check unless a profiler is attached

#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn_kernels.cuh"
#include "prep_kernels.cuh"
#include "sage_attn.h"
#include "sparse_kernels.cuh"
#include "workspace.cuh"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled comes from the driver through the runtime's entry-point query, so
// the library links no libcuda and loads on machines without a GPU driver.
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major view [rows, D] with a box of {box_cols, 128} rows.
bool make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes, long long rows, int D,
              int box_cols, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * elem_bytes};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), 128u};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [BH, N, D] as a 3-D tensor (D innermost, then the N tokens of a head, then heads), box
// [box_cols x 128 tokens x 1 head]: a box never reaches into the next head; token rows past N
// read as zeros and are not written by stores.
bool make_map3(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes, int N, int BH, int D,
               int box_cols, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * elem_bytes,
                                 static_cast<cuuint64_t>(N) * D * elem_bytes};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), 128u, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_qk_map3(CUtensorMap* map, const int8_t* base, int N, int BH, int D) {
  return make_map3(map, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, BH, D, D,
                   D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

bool make_v_map3(CUtensorMap* map, const void* base, int N, int BH, int D) {
  return make_map3(map, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, BH, D, 64, CU_TENSOR_MAP_SWIZZLE_128B);
}

// E4M3 V codes of the FP8 P.V variant: [BH][N][128] bytes, one box of 128 columns x 128 tokens.
bool make_v8_map3(CUtensorMap* map, const void* base, int N, int BH, int D) {
  return make_map3(map, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, N, BH, D, D, CU_TENSOR_MAP_SWIZZLE_128B);
}

// O written by TMA stores of [128 rows x 64 columns] fp16 boxes from unswizzled shared memory.
bool make_o_map3(CUtensorMap* map, const void* base, int N, int BH, int D) {
  return make_map3(map, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, N, BH, D, 64, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// FP4 codes: [BH][rows][cols] bytes (Q and K: rows = N tokens, cols = d / 2; V transposed: rows =
// d channels, cols = tiles * 64), boxes of box_cols bytes x box_rows rows (a box never reaches
// into the next head), swizzle matching the box width (64 bytes: 64-byte, 32 bytes: 32-byte).
bool make_fp4_map3(CUtensorMap* map, const void* base, int rows, int BH, int cols, int box_cols, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows) * cols};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_qk_map(CUtensorMap* map, const int8_t* base, long long rows, int D) {
  return make_map(map, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, D, D,
                  D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by every entry point.
int check_shape(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return SAGE_ERR_INVALID;
  if (d != 64 && d != 128) return SAGE_ERR_UNSUPPORTED;
  const long long elems = static_cast<long long>(B) * H * N * d;
  if (elems >= (1ll << 31)) return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

int check_scale(float sm_scale) {
  return (std::isfinite(sm_scale) && sm_scale > 0.f) ? SAGE_OK : SAGE_ERR_INVALID;
}

int check_gran(int g) { return (g == SAGE_PER_TOKEN || g == SAGE_PER_BLOCK) ? SAGE_OK : SAGE_ERR_INVALID; }

// The block-sparse variant: at most 512 key tiles (N <= 65536), either head dimension.
int check_sparse(int N) {
  return (N + 127) / 128 <= sage::kSparseMaxKeyBlocks ? SAGE_OK : SAGE_ERR_UNSUPPORTED;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA; }

// v: fp16 V, or (fp8_sv != nullptr) the E4M3 codes of the FP8 P.V variant with their
// per-channel scales fp8_sv and means fp8_vm (may be null).
int attn_quantized_impl(const int8_t* q8, const int8_t* k8, const float* sq, const float* sk, const void* v, void* o,
                        int B, int H, int N, int d, int causal, float sm_scale, int granularity,
                        cudaStream_t st, long long* trace = nullptr, int trace_ctas = 0,
                        const float* fp8_sv = nullptr, const float* fp8_vm = nullptr,
                        const int* kv_count = nullptr, const int16_t* kv_index = nullptr, float skip_lambda = 0.f) {
  const int BH = B * H;
  CUtensorMap tq, tk, tv, to;
  const bool vmap_ok = fp8_sv ? make_v8_map3(&tv, v, N, BH, d) : make_v_map3(&tv, v, N, BH, d);
  if (!make_qk_map3(&tq, q8, N, BH, d) || !make_qk_map3(&tk, k8, N, BH, d) || !vmap_ok ||
      !make_o_map3(&to, o, N, BH, d))
    return SAGE_ERR_CUDA;
  sage::AttnArgs a{};
  a.tm_q = &tq;
  a.tm_k = &tk;
  a.tm_v = &tv;
  a.tm_o = &to;
  a.sq = sq;
  a.sk = sk;
  a.o = static_cast<__half*>(o);
  a.BH = BH;
  a.N = N;
  a.D = d;
  a.causal = causal != 0;
  a.per_token = granularity == SAGE_PER_TOKEN;
  a.sm_scale_log2 = sm_scale * 1.4426950408889634f;
  a.trace = trace;
  a.trace_ctas = trace_ctas;
  a.fp8 = fp8_sv != nullptr;
  a.sv = fp8_sv;
  a.vm = fp8_vm;
  a.kv_count = kv_count;
  a.kv_index = kv_index;
  a.skip_lambda = skip_lambda;
  const cudaError_t e = sage::launch_attn(a, st);
  return e == cudaErrorNotSupported ? SAGE_ERR_UNSUPPORTED : cuda_status(e);
}

}  // namespace

namespace sage {

cudaError_t workspace_alloc(void** p, size_t bytes, cudaStream_t st) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static cudaMemPool_t pools[kMaxDevices] = {};
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaMemPool_t pool = nullptr;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!pools[dev]) {
      cudaMemPoolProps props{};
      props.allocType = cudaMemAllocationTypePinned;
      props.handleTypes = cudaMemHandleTypeNone;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      cudaMemPool_t created = nullptr;
      if ((e = cudaMemPoolCreate(&created, &props)) != cudaSuccess) return e;
      unsigned long long keep = ~0ull;  // never hand freed memory back at synchronizations
      if ((e = cudaMemPoolSetAttribute(created, cudaMemPoolAttrReleaseThreshold, &keep)) != cudaSuccess) {
        cudaMemPoolDestroy(created);
        return e;
      }
      pools[dev] = created;
    }
    pool = pools[dev];
  }
  return cudaMallocFromPoolAsync(p, bytes, pool, st);
}

}  // namespace sage

extern "C" {

const char* sage_status_string(int status) {
  switch (status) {
    case SAGE_OK: return "ok";
    case SAGE_ERR_INVALID: return "invalid argument";
    case SAGE_ERR_UNSUPPORTED: return "unsupported size (d must be 64 or 128; the INT32 debug entry also needs N a multiple of 128)";
    case SAGE_ERR_CUDA: return "CUDA runtime error";
    case SAGE_ERR_TIMEOUT: return "a kernel wait timed out";
    case SAGE_ERR_NOMEM: return "workspace allocation failed";
    case SAGE_ERR_TOO_LARGE: return "problem needs more than the no-alloc scratch (SAGE_NOALLOC_SCRATCH_BYTES)";
    default: return "unknown status";
  }
}

size_t sage_scale_count(int N, int granularity, int is_q) {
  if (N <= 0) return 0;
  if (granularity == SAGE_PER_TOKEN) return static_cast<size_t>(N);
  if (granularity == SAGE_PER_BLOCK) {
    const int g = is_q ? 128 : 64;
    return static_cast<size_t>((N + g - 1) / g);
  }
  return 0;
}

int sage_smooth_k(const void* k, float* km, int B, int H, int N, int d, void* stream) {
  if (!k || !km) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if (!aligned16(k)) return SAGE_ERR_INVALID;
  return cuda_status(sage::launch_smooth_k(static_cast<const __half*>(k), km, B * H, N, d,
                                           static_cast<cudaStream_t>(stream)));
}

int sage_quant_qk(const void* q, const void* k, const float* km, int8_t* q8, int8_t* k8, float* sq, float* sk,
                  int B, int H, int N, int d, int granularity, void* stream) {
  if (!q || !k || !q8 || !k8 || !sq || !sk) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if ((rc = check_gran(granularity))) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q8) || !aligned16(k8)) return SAGE_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_status(sage::launch_quant_qk(static_cast<const __half*>(q), static_cast<const __half*>(k), km, q8, k8,
                                           sq, sk, B * H, N, d, granularity == SAGE_PER_TOKEN, st));
}

int sage_attn_fwd_quantized(const int8_t* q8, const int8_t* k8, const float* sq, const float* sk, const void* v,
                            void* o, int B, int H, int N, int d, int causal, float sm_scale, int granularity,
                            void* stream) {
  if (!q8 || !k8 || !sq || !sk || !v || !o) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if ((rc = check_scale(sm_scale)) || (rc = check_gran(granularity))) return rc;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v) || !aligned16(o) || !aligned16(sk)) return SAGE_ERR_INVALID;
  return attn_quantized_impl(q8, k8, sq, sk, v, o, B, H, N, d, causal, sm_scale, granularity,
                             static_cast<cudaStream_t>(stream));
}

int sage_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d, int causal,
                  float sm_scale, int granularity, void* stream) {
  if (!q || !k || !v || !o) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if ((rc = check_scale(sm_scale)) || (rc = check_gran(granularity))) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SAGE_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  const size_t elems = static_cast<size_t>(BH) * N * d;
  const size_t nsq = static_cast<size_t>(BH) * sage_scale_count(N, granularity, 1);
  const size_t nsk = static_cast<size_t>(BH) * sage_scale_count(N, granularity, 0);
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t off_k8 = up(elems);
  const size_t off_sq = off_k8 + up(elems);
  const size_t off_sk = off_sq + up(nsq * 4);
  const size_t off_km = off_sk + up(nsk * 4);
  const size_t total = off_km + up(static_cast<size_t>(BH) * d * 4);
  void* ws = nullptr;
  if (sage::workspace_alloc(&ws, total, st) != cudaSuccess) {
    cudaGetLastError();
    return SAGE_ERR_NOMEM;
  }
  uint8_t* w = static_cast<uint8_t*>(ws);
  int8_t* q8 = reinterpret_cast<int8_t*>(w);
  int8_t* k8 = reinterpret_cast<int8_t*>(w + off_k8);
  float* sq = reinterpret_cast<float*>(w + off_sq);
  float* sk = reinterpret_cast<float*>(w + off_sk);
  float* km = reinterpret_cast<float*>(w + off_km);
  // NVTX ranges mark the host-side enqueue of each step in a profiler's timeline
  nvtxRangePushA("sage_smooth_k");
  rc = cuda_status(sage::launch_smooth_k(static_cast<const __half*>(k), km, BH, N, d, st));
  nvtxRangePop();
  nvtxRangePushA("sage_quant_qk");
  if (!rc) rc = sage_quant_qk(q, k, km, q8, k8, sq, sk, B, H, N, d, granularity, stream);
  nvtxRangePop();
  nvtxRangePushA("sage_attn_fused");
  if (!rc) rc = attn_quantized_impl(q8, k8, sq, sk, v, o, B, H, N, d, causal, sm_scale, granularity, st);
  nvtxRangePop();
  const cudaError_t fe = cudaFreeAsync(ws, st);
  if (!rc && fe != cudaSuccess) rc = SAGE_ERR_CUDA;
  return rc;
}

int sage_prep_qk(const void* q, const void* k, float* km, int8_t* q8, int8_t* k8, float* sq, float* sk, int B, int H,
                 int N, int d, int granularity, void* stream) {
  if (!q || !k || !km || !q8 || !k8 || !sq || !sk) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if ((rc = check_gran(granularity))) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q8) || !aligned16(k8)) return SAGE_ERR_INVALID;
  return cuda_status(sage::launch_prep_fused(static_cast<const __half*>(q), static_cast<const __half*>(k), km, q8, k8,
                                             sq, sk, B * H, N, d, granularity == SAGE_PER_TOKEN,
                                             static_cast<cudaStream_t>(stream)));
}

int sage_quant_v_fp8(const void* v, uint8_t* v8, float* sv, float* vm, int B, int H, int N, int d, void* stream) {
  if (!v || !v8 || !sv) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if (!aligned16(v) || !aligned16(v8)) return SAGE_ERR_INVALID;
  return cuda_status(sage::launch_quant_v_fp8(static_cast<const __half*>(v), v8, sv, vm, B * H, N, d,
                                              static_cast<cudaStream_t>(stream)));
}

int sage_attn_fwd_fp8pv_quantized(const int8_t* q8, const int8_t* k8, const float* sq, const float* sk,
                                  const uint8_t* v8, const float* sv, const float* vm, void* o, int B, int H, int N,
                                  int d, int causal, float sm_scale, int granularity, void* stream) {
  if (!q8 || !k8 || !sq || !sk || !v8 || !sv || !o) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if (d != 128) return SAGE_ERR_UNSUPPORTED;
  if ((rc = check_scale(sm_scale)) || (rc = check_gran(granularity))) return rc;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o) || !aligned16(sk)) return SAGE_ERR_INVALID;
  return attn_quantized_impl(q8, k8, sq, sk, v8, o, B, H, N, d, causal, sm_scale, granularity,
                             static_cast<cudaStream_t>(stream), nullptr, 0, sv, vm);
}

int sage_attn_fwd_fp8pv(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d, int causal,
                        float sm_scale, int granularity, void* stream) {
  if (!q || !k || !v || !o) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if (d != 128) return SAGE_ERR_UNSUPPORTED;
  if ((rc = check_scale(sm_scale)) || (rc = check_gran(granularity))) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SAGE_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  const size_t elems = static_cast<size_t>(BH) * N * d;
  const size_t nsq = static_cast<size_t>(BH) * sage_scale_count(N, granularity, 1);
  const size_t nsk = static_cast<size_t>(BH) * sage_scale_count(N, granularity, 0);
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t chan = up(static_cast<size_t>(BH) * d * 4);
  const size_t off_k8 = up(elems);
  const size_t off_v8 = off_k8 + up(elems);
  const size_t off_sq = off_v8 + up(elems);
  const size_t off_sk = off_sq + up(nsq * 4);
  const size_t off_km = off_sk + up(nsk * 4);
  const size_t off_sv = off_km + chan;
  const size_t off_vm = off_sv + chan;
  const size_t total = off_vm + chan;
  void* ws = nullptr;
  if (sage::workspace_alloc(&ws, total, st) != cudaSuccess) {
    cudaGetLastError();
    return SAGE_ERR_NOMEM;
  }
  uint8_t* w = static_cast<uint8_t*>(ws);
  int8_t* q8 = reinterpret_cast<int8_t*>(w);
  int8_t* k8 = reinterpret_cast<int8_t*>(w + off_k8);
  uint8_t* v8 = w + off_v8;
  float* sq = reinterpret_cast<float*>(w + off_sq);
  float* sk = reinterpret_cast<float*>(w + off_sk);
  float* km = reinterpret_cast<float*>(w + off_km);
  float* sv = reinterpret_cast<float*>(w + off_sv);
  float* vm = reinterpret_cast<float*>(w + off_vm);
  nvtxRangePushA("sage_fp8pv_prep");
  rc = cuda_status(sage::launch_smooth_k(static_cast<const __half*>(k), km, BH, N, d, st));
  if (!rc) rc = sage_quant_qk(q, k, km, q8, k8, sq, sk, B, H, N, d, granularity, stream);
  if (!rc) rc = cuda_status(sage::launch_quant_v_fp8(static_cast<const __half*>(v), v8, sv, vm, BH, N, d, st));
  nvtxRangePop();
  nvtxRangePushA("sage_fp8pv_fused");
  if (!rc) rc = attn_quantized_impl(q8, k8, sq, sk, v8, o, B, H, N, d, causal, sm_scale, granularity, st, nullptr, 0,
                                    sv, vm);
  nvtxRangePop();
  const cudaError_t fe = cudaFreeAsync(ws, st);
  if (!rc && fe != cudaSuccess) rc = SAGE_ERR_CUDA;
  return rc;
}

int sage_sparse_predict(const void* q, const void* k, int B, int H, int N, int d, int causal, float sm_scale, float tau,
                        float theta, int* kv_count, int16_t* kv_index, void* stream) {
  if (!q || !k || !kv_count || !kv_index) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if ((rc = check_sparse(N))) return rc;
  if ((rc = check_scale(sm_scale))) return rc;
  if (!(tau > 0.f && tau <= 1.f) || !std::isfinite(theta)) return SAGE_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k)) return SAGE_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  void* ws = nullptr;
  if (sage::workspace_alloc(&ws, sage::sparse_predict_workspace(BH, N, d), st) != cudaSuccess) {
    cudaGetLastError();
    return SAGE_ERR_NOMEM;
  }
  rc = cuda_status(sage::launch_sparse_predict(static_cast<const __half*>(q), static_cast<const __half*>(k), ws, BH, N,
                                               d, causal != 0, sm_scale, tau, theta, kv_count, kv_index, st));
  const cudaError_t fe = cudaFreeAsync(ws, st);
  if (!rc && fe != cudaSuccess) rc = SAGE_ERR_CUDA;
  return rc;
}

int sage_attn_fwd_sparse_quantized(const int8_t* q8, const int8_t* k8, const float* sq, const float* sk, const void* v,
                                   void* o, int B, int H, int N, int d, int causal, float sm_scale, int granularity,
                                   const int* kv_count, const int16_t* kv_index, float skip_lambda, void* stream) {
  if (!q8 || !k8 || !sq || !sk || !v || !o || !kv_count || !kv_index) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if ((rc = check_sparse(N))) return rc;
  if ((rc = check_scale(sm_scale)) || (rc = check_gran(granularity))) return rc;
  if (!(skip_lambda > 0.f)) return SAGE_ERR_INVALID;  // +inf: no second stage; NaN rejected
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v) || !aligned16(o) || !aligned16(sk)) return SAGE_ERR_INVALID;
  return attn_quantized_impl(q8, k8, sq, sk, v, o, B, H, N, d, causal, sm_scale, granularity,
                             static_cast<cudaStream_t>(stream), nullptr, 0, nullptr, nullptr, kv_count, kv_index,
                             skip_lambda);
}

int sage_attn_fwd_sparse(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d, int causal,
                         float sm_scale, int granularity, float tau, float theta, float skip_lambda, void* stream) {
  if (!q || !k || !v || !o) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if ((rc = check_sparse(N))) return rc;
  if ((rc = check_scale(sm_scale)) || (rc = check_gran(granularity))) return rc;
  if (!(tau > 0.f && tau <= 1.f) || !std::isfinite(theta) || !(skip_lambda > 0.f)) return SAGE_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SAGE_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  const size_t elems = static_cast<size_t>(BH) * N * d;
  const size_t nsq = static_cast<size_t>(BH) * sage_scale_count(N, granularity, 1);
  const size_t nsk = static_cast<size_t>(BH) * sage_scale_count(N, granularity, 0);
  const size_t nqb = static_cast<size_t>((N + 255) / 256), nkb = static_cast<size_t>((N + 127) / 128);
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t off_k8 = up(elems);
  const size_t off_sq = off_k8 + up(elems);
  const size_t off_sk = off_sq + up(nsq * 4);
  const size_t off_km = off_sk + up(nsk * 4);
  const size_t off_cnt = off_km + up(static_cast<size_t>(BH) * d * 4);
  const size_t off_idx = off_cnt + up(static_cast<size_t>(BH) * nqb * 4);
  const size_t off_pred = off_idx + up(static_cast<size_t>(BH) * nqb * nkb * 2);
  const size_t total = off_pred + up(sage::sparse_predict_workspace(BH, N, d));
  void* ws = nullptr;
  if (sage::workspace_alloc(&ws, total, st) != cudaSuccess) {
    cudaGetLastError();
    return SAGE_ERR_NOMEM;
  }
  uint8_t* w = static_cast<uint8_t*>(ws);
  int8_t* q8 = reinterpret_cast<int8_t*>(w);
  int8_t* k8 = reinterpret_cast<int8_t*>(w + off_k8);
  float* sq = reinterpret_cast<float*>(w + off_sq);
  float* sk = reinterpret_cast<float*>(w + off_sk);
  float* km = reinterpret_cast<float*>(w + off_km);
  int* cnt = reinterpret_cast<int*>(w + off_cnt);
  int16_t* idx = reinterpret_cast<int16_t*>(w + off_idx);
  nvtxRangePushA("sage_sparse_prep");
  rc = cuda_status(sage::launch_sparse_predict(static_cast<const __half*>(q), static_cast<const __half*>(k),
                                               w + off_pred, BH, N, d, causal != 0, sm_scale, tau, theta, cnt, idx, st));
  if (!rc) rc = cuda_status(sage::launch_smooth_k(static_cast<const __half*>(k), km, BH, N, d, st));
  if (!rc) rc = sage_quant_qk(q, k, km, q8, k8, sq, sk, B, H, N, d, granularity, stream);
  nvtxRangePop();
  nvtxRangePushA("sage_sparse_fused");
  if (!rc) rc = attn_quantized_impl(q8, k8, sq, sk, v, o, B, H, N, d, causal, sm_scale, granularity, st, nullptr, 0,
                                    nullptr, nullptr, cnt, idx, skip_lambda);
  nvtxRangePop();
  const cudaError_t fe = cudaFreeAsync(ws, st);
  if (!rc && fe != cudaSuccess) rc = SAGE_ERR_CUDA;
  return rc;
}

int sage_debug_qk_int32(const int8_t* q8, const int8_t* k8, int32_t* s, int B, int H, int N, int d, void* stream) {
  if (!q8 || !k8 || !s) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if (N % 128 != 0) return SAGE_ERR_UNSUPPORTED;  // whole 128 x 128 tiles only
  if (static_cast<long long>(B) * H * N * N >= (1ll << 31)) return SAGE_ERR_UNSUPPORTED;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(s)) return SAGE_ERR_INVALID;
  const long long rows = static_cast<long long>(B) * H * N;
  CUtensorMap tq, tk;
  if (!make_qk_map(&tq, q8, rows, d) || !make_qk_map(&tk, k8, rows, d)) return SAGE_ERR_CUDA;
  return cuda_status(sage::launch_qk_debug(tq, tk, s, B * H, N, d, static_cast<cudaStream_t>(stream)));
}

int sage_debug_attn_trace(const int8_t* q8, const int8_t* k8, const float* sq, const float* sk, const void* v,
                          void* o, int B, int H, int N, int d, int causal, float sm_scale, int granularity,
                          long long* trace, int trace_ctas, void* stream) {
  if (!trace || trace_ctas <= 0) return SAGE_ERR_INVALID;
  if (granularity != SAGE_PER_BLOCK) return SAGE_ERR_UNSUPPORTED;
  if (!q8 || !k8 || !sq || !sk || !v || !o) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if ((rc = check_scale(sm_scale))) return rc;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v) || !aligned16(o)) return SAGE_ERR_INVALID;
  return attn_quantized_impl(q8, k8, sq, sk, v, o, B, H, N, d, causal, sm_scale, granularity,
                             static_cast<cudaStream_t>(stream), trace, trace_ctas);
}

int sage_debug_wait_timeout(int* gave_up, void* stream) {
  if (!gave_up) return SAGE_ERR_INVALID;
  return cuda_status(sage::launch_wait_timeout(gave_up, static_cast<cudaStream_t>(stream)));
}

int sage_last_device_error(void* stream) {
  cudaError_t e;
  const int code = sage::read_and_clear_device_error(static_cast<cudaStream_t>(stream), &e);
  return code < 0 ? SAGE_ERR_CUDA : code;
}


// ---------------------------------------------------------------- microscaling FP4 variant
int sage_quant_qk_fp4(const void* q, const void* k, const float* km, uint8_t* q4, uint8_t* sfq, float* gq,
                      uint8_t* k4, uint8_t* sfk, float* gk, int B, int H, int N, int d, void* stream) {
  if (!q || !k || !q4 || !sfq || !gq || !k4 || !sfk || !gk) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q4) || !aligned16(k4) || !aligned16(sfq) || !aligned16(sfk))
    return SAGE_ERR_INVALID;
  return cuda_status(sage::launch_quant_qk_fp4(static_cast<const __half*>(q), static_cast<const __half*>(k), km, q4,
                                               sfq, gq, k4, sfk, gk, B * H, N, d, static_cast<cudaStream_t>(stream)));
}

int sage_quant_v_fp4(const void* v, uint8_t* v4t, uint8_t* sfv, float* gv, float* vm, int B, int H, int N, int d,
                     void* stream) {
  if (!v || !v4t || !sfv || !gv) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if (!aligned16(v) || !aligned16(v4t) || !aligned16(sfv)) return SAGE_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  void* ws = nullptr;
  if (sage::workspace_alloc(&ws, static_cast<size_t>(BH) * d * 4, st) != cudaSuccess) {
    cudaGetLastError();
    return SAGE_ERR_NOMEM;
  }
  rc = cuda_status(sage::launch_quant_v_fp4(static_cast<const __half*>(v), v4t, sfv, gv, vm, static_cast<float*>(ws),
                                            BH, N, d, st));
  const cudaError_t fe = cudaFreeAsync(ws, st);
  if (!rc && fe != cudaSuccess) rc = SAGE_ERR_CUDA;
  return rc;
}

int sage_attn_fwd_fp4_quantized(const uint8_t* q4, const uint8_t* sfq, const float* gq, const uint8_t* k4,
                                const uint8_t* sfk, const float* gk, const uint8_t* v4t, const uint8_t* sfv,
                                const float* gv, const float* vm, void* o, int B, int H, int N, int d, int causal,
                                float sm_scale, void* stream) {
  if (!q4 || !sfq || !gq || !k4 || !sfk || !gk || !v4t || !sfv || !gv || !o) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if ((rc = check_scale(sm_scale))) return rc;
  if (!aligned16(q4) || !aligned16(k4) || !aligned16(v4t) || !aligned16(sfq) || !aligned16(sfk) || !aligned16(sfv) ||
      !aligned16(o))
    return SAGE_ERR_INVALID;
  const int BH = B * H, tiles = (N + 127) / 128;
  CUtensorMap tq, tk, tv;
  // Q: 128-token boxes; K: 64-key boxes; V^T: 64 keys (32 bytes) of all d channels
  if (!make_fp4_map3(&tq, q4, N, BH, d / 2, d / 2, 128) || !make_fp4_map3(&tk, k4, N, BH, d / 2, d / 2, 64) ||
      !make_fp4_map3(&tv, v4t, d, BH, tiles * 64, 32, d))
    return SAGE_ERR_CUDA;
  sage::Fp4Args a{};
  a.tm_q = &tq;
  a.tm_k = &tk;
  a.tm_v = &tv;
  a.sfq = sfq;
  a.sfk = sfk;
  a.sfv = sfv;
  a.gq = gq;
  a.gk = gk;
  a.gv = gv;
  a.vm = vm;
  a.o = static_cast<__half*>(o);
  a.BH = BH;
  a.N = N;
  a.D = d;
  a.causal = causal != 0;
  a.sm_scale_log2 = sm_scale * 1.4426950408889634f;
  return cuda_status(sage::launch_attn_fp4(a, static_cast<cudaStream_t>(stream)));
}

int sage_attn_fwd_fp4(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d, int causal,
                      float sm_scale, void* stream) {
  if (!q || !k || !v || !o) return SAGE_ERR_INVALID;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if ((rc = check_scale(sm_scale))) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SAGE_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  const size_t tiles = static_cast<size_t>((N + 127) / 128);
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  // atoms: the largest of sfq (tiles x d/64), sfk (2 tiles x d/64) and sfv (tiles x 2) atoms of 512 bytes
  const size_t codes = up(static_cast<size_t>(BH) * N * (d / 2)), atoms = up(static_cast<size_t>(BH) * tiles * 4 * 512);
  const size_t tscales = up(static_cast<size_t>(BH) * tiles * 4), chan = up(static_cast<size_t>(BH) * d * 4);
  const size_t off_k4 = codes;
  const size_t off_v4 = off_k4 + codes;
  const size_t off_sfq = off_v4 + up(static_cast<size_t>(BH) * d * tiles * 64);
  const size_t off_sfk = off_sfq + atoms;
  const size_t off_sfv = off_sfk + atoms;
  const size_t off_gq = off_sfv + atoms;
  const size_t off_gk = off_gq + tscales;
  const size_t off_km = off_gk + tscales;
  const size_t off_gv = off_km + chan;
  const size_t off_vm = off_gv + chan;
  const size_t off_rv = off_vm + chan;
  const size_t total = off_rv + chan;
  void* ws = nullptr;
  if (sage::workspace_alloc(&ws, total, st) != cudaSuccess) {
    cudaGetLastError();
    return SAGE_ERR_NOMEM;
  }
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* km = reinterpret_cast<float*>(w + off_km);
  float* gv = reinterpret_cast<float*>(w + off_gv);
  float* vm = reinterpret_cast<float*>(w + off_vm);
  nvtxRangePushA("sage_fp4_prep");
  rc = cuda_status(sage::launch_smooth_k(static_cast<const __half*>(k), km, BH, N, d, st));
  if (!rc)
    rc = cuda_status(sage::launch_quant_qk_fp4(static_cast<const __half*>(q), static_cast<const __half*>(k), km, w,
                                               w + off_sfq, reinterpret_cast<float*>(w + off_gq), w + off_k4,
                                               w + off_sfk, reinterpret_cast<float*>(w + off_gk), BH, N, d, st));
  if (!rc)
    rc = cuda_status(sage::launch_quant_v_fp4(static_cast<const __half*>(v), w + off_v4, w + off_sfv, gv, vm,
                                              reinterpret_cast<float*>(w + off_rv), BH, N, d, st));
  nvtxRangePop();
  nvtxRangePushA("sage_fp4_fused");
  if (!rc)
    rc = sage_attn_fwd_fp4_quantized(w, w + off_sfq, reinterpret_cast<float*>(w + off_gq), w + off_k4, w + off_sfk,
                                     reinterpret_cast<float*>(w + off_gk), w + off_v4, w + off_sfv, gv, vm, o, B, H, N,
                                     d, causal, sm_scale, stream);
  nvtxRangePop();
  const cudaError_t fe = cudaFreeAsync(ws, st);
  if (!rc && fe != cudaSuccess) rc = SAGE_ERR_CUDA;
  return rc;
}

}  // extern "C"
