// host_pipeline.cu -- sage_attn_fwd_host(_variant): the whole forward pass (the method, or its
// FP8 P.V or FP4 variant) for Q, K, V and O in host memory, with the host<->device copies
// overlapped with the compute.
//
// Heads are independent problems (the K mean, the scales and the attention of a (b,h) use
// that head's tokens only), so the B*H heads are cut into chunks of consecutive heads, each a
// contiguous byte range of every [B][H][N][d] tensor.  Chunk c is copied in on one stream,
// computed (smooth K, quantize, fused kernel) on the caller's stream and copied out on a third
// stream, so that the input copy of chunk c+1 and the output copy of chunk c-1 run while chunk
// c is computed.  Two sets of device buffers alternate between chunks; events order every
// reuse.  With pinned host buffers the copy engines run both directions at once and a call
// costs about max(input copies, compute, output copies) plus one chunk of pipeline fill.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "sage_attn.h"
#include "workspace.cuh"

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
cudaStream_t g_in_stream[kMaxDevices] = {};
cudaStream_t g_out_stream[kMaxDevices] = {};

// The two copy streams of the current device, created on first use (non-blocking, so that
// they never synchronize with the legacy default stream) and kept for the process lifetime.
int copy_streams(cudaStream_t* in, cudaStream_t* out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SAGE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_in_stream[dev]) {
    cudaStream_t a = nullptr, b = nullptr;
    if (cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking) != cudaSuccess) {
      cudaGetLastError();
      return SAGE_ERR_CUDA;
    }
    if (cudaStreamCreateWithFlags(&b, cudaStreamNonBlocking) != cudaSuccess) {
      cudaStreamDestroy(a);
      cudaGetLastError();
      return SAGE_ERR_CUDA;
    }
    g_in_stream[dev] = a;
    g_out_stream[dev] = b;
  }
  *in = g_in_stream[dev];
  *out = g_out_stream[dev];
  return SAGE_OK;
}

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Device buffers of one chunk slot (all 256-byte aligned inside one allocation).
struct Slot {
  uint8_t *q, *k, *v, *o;     // fp16 [hc][N][d]
  int8_t *q8, *k8;            // int8 [hc][N][d]
  float *sq, *sk, *km;        // scales and K mean
};

size_t slot_bytes(int hc, int N, int d, int granularity) {
  const size_t e = static_cast<size_t>(hc) * N * d;
  return 4 * up256(2 * e) + 2 * up256(e) + up256(4 * hc * sage_scale_count(N, granularity, 1)) +
         up256(4 * hc * sage_scale_count(N, granularity, 0)) + up256(4 * static_cast<size_t>(hc) * d);
}

Slot carve(uint8_t* base, int hc, int N, int d, int granularity) {
  const size_t e = static_cast<size_t>(hc) * N * d;
  Slot s{};
  uint8_t* p = base;
  s.q = p; p += up256(2 * e);
  s.k = p; p += up256(2 * e);
  s.v = p; p += up256(2 * e);
  s.o = p; p += up256(2 * e);
  s.q8 = reinterpret_cast<int8_t*>(p); p += up256(e);
  s.k8 = reinterpret_cast<int8_t*>(p); p += up256(e);
  s.sq = reinterpret_cast<float*>(p); p += up256(4 * hc * sage_scale_count(N, granularity, 1));
  s.sk = reinterpret_cast<float*>(p); p += up256(4 * hc * sage_scale_count(N, granularity, 0));
  s.km = reinterpret_cast<float*>(p);
  return s;
}

}  // namespace

extern "C" {

int sage_attn_fwd_host_variant(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                               int causal, float sm_scale, int granularity, int heads_per_chunk, int variant,
                               void* stream) {
  if (!q || !k || !v || !o) return SAGE_ERR_INVALID;
  if (variant != SAGE_VARIANT_FP16PV && variant != SAGE_VARIANT_FP8PV && variant != SAGE_VARIANT_FP4)
    return SAGE_ERR_INVALID;
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return SAGE_ERR_INVALID;
  if (granularity != SAGE_PER_TOKEN && granularity != SAGE_PER_BLOCK) return SAGE_ERR_INVALID;
  if (!(sm_scale > 0.f) || sm_scale > 3.4e38f) return SAGE_ERR_INVALID;  // also rejects NaN and inf
  if (heads_per_chunk < 0) return SAGE_ERR_INVALID;
  if (d != 64 && d != 128) return SAGE_ERR_UNSUPPORTED;
  if (variant == SAGE_VARIANT_FP8PV && d != 128) return SAGE_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * N * d >= (1ll << 31)) return SAGE_ERR_UNSUPPORTED;
  const int BH = B * H;
  // default: sixteen chunks, at least one head each (measured at B*H = 64, N = 16384, d = 128:
  // 16 chunks 16.6 ms, 8 chunks 17.8 ms, 32 chunks 17.3 ms, one chunk (no overlap) 29.2 ms)
  const int hc = heads_per_chunk > 0 ? (heads_per_chunk < BH ? heads_per_chunk : BH) : (BH + 15) / 16;
  const int n_chunks = (BH + hc - 1) / hc;
  const int n_slots = n_chunks > 1 ? 2 : 1;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStream_t s_in = nullptr, s_out = nullptr;
  int rc = copy_streams(&s_in, &s_out);
  if (rc) return rc;

  const size_t per_slot = slot_bytes(hc, N, d, granularity);
  void* ws = nullptr;
  if (sage::workspace_alloc(&ws, per_slot * n_slots, st) != cudaSuccess) {
    cudaGetLastError();
    return SAGE_ERR_NOMEM;
  }
  Slot slot[2];
  for (int i = 0; i < n_slots; ++i) slot[i] = carve(static_cast<uint8_t*>(ws) + i * per_slot, hc, N, d, granularity);

  // events: entry (work already on the caller's stream, including the allocation), and per
  // slot the last chunk's "inputs copied", "computed" and "output copied"
  cudaEvent_t ev_entry = nullptr, ev_in[2] = {}, ev_done[2] = {}, ev_out[2] = {};
  bool ok = cudaEventCreateWithFlags(&ev_entry, cudaEventDisableTiming) == cudaSuccess;
  for (int i = 0; i < 2 && ok; ++i)
    ok = cudaEventCreateWithFlags(&ev_in[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&ev_done[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&ev_out[i], cudaEventDisableTiming) == cudaSuccess;
  ok = ok && cudaEventRecord(ev_entry, st) == cudaSuccess && cudaStreamWaitEvent(s_in, ev_entry, 0) == cudaSuccess &&
       cudaStreamWaitEvent(s_out, ev_entry, 0) == cudaSuccess;
  if (!ok) rc = SAGE_ERR_CUDA;

  const size_t head_bytes = static_cast<size_t>(N) * d * 2;
  const uint8_t* hq = static_cast<const uint8_t*>(q);
  const uint8_t* hk = static_cast<const uint8_t*>(k);
  const uint8_t* hv = static_cast<const uint8_t*>(v);
  uint8_t* ho = static_cast<uint8_t*>(o);
  for (int c = 0; c < n_chunks && !rc; ++c) {
    const int i = c % n_slots;
    const int h0 = c * hc;
    const int hn = (BH - h0) < hc ? (BH - h0) : hc;
    const size_t off = static_cast<size_t>(h0) * head_bytes, bytes = static_cast<size_t>(hn) * head_bytes;
    const Slot& s = slot[i];
    // inputs of chunk c into slot i once chunk c-2 has left it (its output copy waited for
    // its compute, which consumed the inputs)
    if (c >= n_slots && cudaStreamWaitEvent(s_in, ev_out[i], 0) != cudaSuccess) { rc = SAGE_ERR_CUDA; break; }
    if (cudaMemcpyAsync(s.q, hq + off, bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaMemcpyAsync(s.k, hk + off, bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaMemcpyAsync(s.v, hv + off, bytes, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaEventRecord(ev_in[i], s_in) != cudaSuccess || cudaStreamWaitEvent(st, ev_in[i], 0) != cudaSuccess) {
      rc = SAGE_ERR_CUDA;
      break;
    }
    // the slot's output buffer must have been copied out before this chunk's kernels write it
    if (c >= n_slots && cudaStreamWaitEvent(st, ev_out[i], 0) != cudaSuccess) { rc = SAGE_ERR_CUDA; break; }
    if (variant == SAGE_VARIANT_FP4) {
      rc = sage_attn_fwd_fp4(s.q, s.k, s.v, s.o, 1, hn, N, d, causal, sm_scale, st);
    } else if (variant == SAGE_VARIANT_FP8PV) {
      rc = sage_attn_fwd_fp8pv(s.q, s.k, s.v, s.o, 1, hn, N, d, causal, sm_scale, granularity, st);
    } else {
      rc = sage_smooth_k(s.k, s.km, 1, hn, N, d, st);
      if (!rc) rc = sage_quant_qk(s.q, s.k, s.km, s.q8, s.k8, s.sq, s.sk, 1, hn, N, d, granularity, st);
      if (!rc) rc = sage_attn_fwd_quantized(s.q8, s.k8, s.sq, s.sk, s.v, s.o, 1, hn, N, d, causal, sm_scale, granularity, st);
    }
    if (rc) break;
    if (cudaEventRecord(ev_done[i], st) != cudaSuccess || cudaStreamWaitEvent(s_out, ev_done[i], 0) != cudaSuccess ||
        cudaMemcpyAsync(ho + off, s.o, bytes, cudaMemcpyDeviceToHost, s_out) != cudaSuccess ||
        cudaEventRecord(ev_out[i], s_out) != cudaSuccess) {
      rc = SAGE_ERR_CUDA;
      break;
    }
  }
  // the caller's stream continues after every output copy (and after every input copy, so
  // that freeing the workspace is ordered after all uses of it)
  if (ok) {
    cudaEvent_t tail_in = nullptr, tail_out = nullptr;
    if (cudaEventCreateWithFlags(&tail_in, cudaEventDisableTiming) == cudaSuccess &&
        cudaEventCreateWithFlags(&tail_out, cudaEventDisableTiming) == cudaSuccess &&
        cudaEventRecord(tail_in, s_in) == cudaSuccess && cudaEventRecord(tail_out, s_out) == cudaSuccess &&
        cudaStreamWaitEvent(st, tail_in, 0) == cudaSuccess && cudaStreamWaitEvent(st, tail_out, 0) == cudaSuccess) {
    } else if (!rc) {
      rc = SAGE_ERR_CUDA;
    }
    if (tail_in) cudaEventDestroy(tail_in);
    if (tail_out) cudaEventDestroy(tail_out);
  }
  // events may be destroyed while work that records or waits on them is pending
  if (ev_entry) cudaEventDestroy(ev_entry);
  for (int i = 0; i < 2; ++i) {
    if (ev_in[i]) cudaEventDestroy(ev_in[i]);
    if (ev_done[i]) cudaEventDestroy(ev_done[i]);
    if (ev_out[i]) cudaEventDestroy(ev_out[i]);
  }
  if (cudaFreeAsync(ws, st) != cudaSuccess && !rc) rc = SAGE_ERR_CUDA;
  if (rc == SAGE_ERR_CUDA) cudaGetLastError();
  return rc;
}

int sage_attn_fwd_host(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d, int causal,
                       float sm_scale, int granularity, int heads_per_chunk, void* stream) {
  return sage_attn_fwd_host_variant(q, k, v, o, B, H, N, d, causal, sm_scale, granularity, heads_per_chunk,
                                    SAGE_VARIANT_FP16PV, stream);
}

}  // extern "C"
