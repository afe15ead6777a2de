// noalloc.cu -- sage_attn_fwd_noalloc: the whole forward pass without any allocation.
//
// sage_attn_fwd needs a workspace for the INT8 copies of Q and K, their scales and the K
// mean, and gets it with a stream-ordered allocation.  Some callers cannot allocate device memory at
// call time: embedded or real-time hosts whose memory budget is fixed after start-up, and
// plugins of frameworks that own every allocation themselves and do not let a library call
// the CUDA allocator.  For them this entry point uses a
// fixed scratch area that lives in the library itself: a file-scope __device__ array that
// every GPU which loads the library holds (kScratchBytes) until the process exits.
//
// Host code cannot use the array's name as a device address (on the host it names a
// stand-in object), so the first call on each device asks the runtime for the device
// address with cudaGetSymbolAddress, with that device current, and caches it.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "sage_attn.h"

namespace {

constexpr size_t kScratchBytes = size_t(64) << 20;  // SAGE_NOALLOC_SCRATCH_BYTES
static_assert(kScratchBytes == SAGE_NOALLOC_SCRATCH_BYTES, "header and library disagree on the scratch size");

static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on first use).
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SAGE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return SAGE_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SAGE_OK;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" {

size_t sage_noalloc_scratch_bytes(int B, int H, int N, int d, int granularity) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return 0;
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t elems = BH * N * d;
  const size_t nsq = BH * sage_scale_count(N, granularity, 1);
  const size_t nsk = BH * sage_scale_count(N, granularity, 0);
  if (nsq == 0 || nsk == 0) return 0;
  return up256(elems) * 2 + up256(nsq * 4) + up256(nsk * 4) + up256(BH * d * 4);
}

int sage_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                          int causal, float sm_scale, int granularity, void* stream) {
  // the checks of sage_attn_fwd, in its order (same status for the same arguments)
  if (!q || !k || !v || !o) return SAGE_ERR_INVALID;
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return SAGE_ERR_INVALID;
  if (d != 64 && d != 128) return SAGE_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * N * d >= (1ll << 31)) return SAGE_ERR_UNSUPPORTED;
  if (!std::isfinite(sm_scale) || !(sm_scale > 0.f)) return SAGE_ERR_INVALID;
  if (granularity != SAGE_PER_TOKEN && granularity != SAGE_PER_BLOCK) return SAGE_ERR_INVALID;
  for (const void* p : {q, k, static_cast<const void*>(v), static_cast<const void*>(o)})
    if (reinterpret_cast<uintptr_t>(p) & 15u) return SAGE_ERR_INVALID;
  const size_t need = sage_noalloc_scratch_bytes(B, H, N, d, granularity);
  if (need > kScratchBytes) return SAGE_ERR_TOO_LARGE;
  void* base = nullptr;
  int rc = scratch_address(&base);
  if (rc) return rc;
  const size_t BH = static_cast<size_t>(B) * H;
  const size_t elems = BH * N * d;
  const size_t nsq = BH * sage_scale_count(N, granularity, 1);
  const size_t nsk = BH * sage_scale_count(N, granularity, 0);
  uint8_t* w = static_cast<uint8_t*>(base);
  int8_t* q8 = reinterpret_cast<int8_t*>(w);
  int8_t* k8 = reinterpret_cast<int8_t*>(w + up256(elems));
  float* sq = reinterpret_cast<float*>(w + 2 * up256(elems));
  float* sk = reinterpret_cast<float*>(w + 2 * up256(elems) + up256(nsq * 4));
  float* km = reinterpret_cast<float*>(w + 2 * up256(elems) + up256(nsq * 4) + up256(nsk * 4));
  // Every scratch value is fully rewritten before it is read (K mean, codes, scales), so
  // nothing has to be cleared between calls.  The public entry points below validate the
  // remaining arguments (d, N, sm_scale, alignment) before they enqueue anything.
  rc = sage_smooth_k(k, km, B, H, N, d, stream);
  if (!rc) rc = sage_quant_qk(q, k, km, q8, k8, sq, sk, B, H, N, d, granularity, stream);
  if (!rc) rc = sage_attn_fwd_quantized(q8, k8, sq, sk, v, o, B, H, N, d, causal, sm_scale, granularity, stream);
  return rc;
}

}  // extern "C"
