// prep_kernels.cu -- the two HBM-bound steps in front of the fused attention kernel:
//   smooth_k: per-(b,h) channel mean of K over tokens   (SageAttention summary, first
//             bullet; Interesting idea I1 -- removing a component shared by all tokens of K
//             leaves the softmax unchanged)
//   quant:    symmetric absmax INT8 quantization of Q and of the smoothed K, per token or
//             per block of tokens (Summary, first bullet; Key points: per-token granularity)
//
// Both are bit-exact by construction: the mean comes from an exact fixed-point sum, and
// every floating-point step is a single IEEE-rounded operation written with the _rn
// intrinsics (never contracted into an FMA), in the order the C ABI documents.
#include <cuda_fp16.h>
#include <cstdint>
#include <type_traits>

#include "prep_kernels.cuh"

namespace sage {

// fp16 bits -> the value times 2^24 as an exact integer.  A normal fp16 is
// (1024 + mantissa) * 2^(exponent - 25); a subnormal is mantissa * 2^-24.
// Infinity / NaN (exponent 31) map to a finite value (results are then unspecified).
__device__ __forceinline__ long long half_bits_to_fixed(uint32_t h) {
  const uint32_t e = (h >> 10) & 31u;
  const uint32_t m = h & 1023u;
  const long long mag = e ? (static_cast<long long>(m | 1024u) << (e - 1)) : static_cast<long long>(m);
  return (h & 0x8000u) ? -mag : mag;
}

// One CTA of 1024 threads per (32-channel chunk, head): thread = (token phase 0..255, 16-byte
// piece 0..3 of the 64-byte chunk row).  Each thread keeps four 16-byte loads in flight
// (tokens t, t+256, t+512, t+768) so that the whole GPU has enough bytes in flight to run
// at HBM speed even with few heads.
template <int D>
__global__ void __launch_bounds__(1024) smooth_k_kernel(const __half* __restrict__ k, float* __restrict__ km,
                                                        int N) {
  constexpr int PHASES = 256;
  const int chunk = blockIdx.x;  // 32 channels
  const int bh = blockIdx.y;
  const int piece = threadIdx.x & 3;
  const int tok0 = threadIdx.x >> 2;
  const __half* base = k + (static_cast<size_t>(bh) * N) * D + chunk * 32 + piece * 8;

  long long acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0;

  for (int t = tok0; t < N; t += 4 * PHASES) {
    uint4 w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      w[u] = (t + u * PHASES < N) ? __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(t + u * PHASES) * D))
                                  : make_uint4(0u, 0u, 0u, 0u);  // +0.0 contributes nothing
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t words[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] += half_bits_to_fixed(words[i] & 0xFFFFu);
        acc[2 * i + 1] += half_bits_to_fixed(words[i] >> 16);
      }
    }
  }
  // lanes sharing `piece` differ in lane bits 2..4
#pragma unroll
  for (int i = 0; i < 8; ++i) {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
  }
  __shared__ long long part[32][4][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane < 4) {
#pragma unroll
    for (int i = 0; i < 8; ++i) part[warp][lane][i] = acc[i];
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int p = threadIdx.x >> 3, i = threadIdx.x & 7;  // channel = chunk*32 + p*8 + i
    long long s = 0;
#pragma unroll
    for (int w = 0; w < 32; ++w) s += part[w][p][i];
    const float s32 = __ll2float_rn(s);
    const float mean = __fdiv_rn(s32, static_cast<float>(N));
    km[static_cast<size_t>(bh) * D + chunk * 32 + p * 8 + i] = __fmul_rn(mean, 5.9604644775390625e-08f);
  }
}

__device__ __forceinline__ void unpack8(const uint4& w, float (&x)[8]) {
  const __half2* h = reinterpret_cast<const __half2*>(&w);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ int quant1(float x, float inv) {
  int q = __float2int_rn(__fmul_rn(x, inv));  // round half to even
  return max(-127, min(127, q));
}

__device__ __forceinline__ uint2 pack8(const float (&x)[8], float inv) {
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) lo |= (static_cast<uint32_t>(quant1(x[i], inv)) & 0xFFu) << (8 * i);
#pragma unroll
  for (int i = 0; i < 4; ++i) hi |= (static_cast<uint32_t>(quant1(x[4 + i], inv)) & 0xFFu) << (8 * i);
  return make_uint2(lo, hi);
}

// Quantize groups of G tokens (G = 1: per token).  T = D/8 threads cover one token row with
// one 16-byte vector each; a 256-thread CTA covers P = 256/T tokens per pass.
//   G == 1 : each T-lane team is its own group (team-wide shuffle max); teams past the last
//            row compute on zeros and store nothing;
//   G  > 1 : the CTA is one group of G tokens held in registers (G/P passes), CTA-wide max.
//            Groups tile each head separately: ceil(N/G) groups per head, the last one holding
//            the N mod G remaining tokens when G does not divide N.
template <int D, int G, bool SMOOTH>
__global__ void __launch_bounds__(256) quant_kernel(const __half* __restrict__ x, const float* __restrict__ km,
                                                    int8_t* __restrict__ q, float* __restrict__ scale, int N,
                                                    long long rows) {
  constexpr int T = D / 8;
  constexpr int P = 256 / T;
  const int piece = threadIdx.x % T;
  const int c0 = piece * 8;

  if constexpr (G == 1) {
    const size_t row = static_cast<size_t>(blockIdx.x) * P + threadIdx.x / T;
    const bool live = row < static_cast<size_t>(rows);  // whole T-lane teams; all lanes stay for the shuffles
    // the load always reads an existing row (the last one for teams past the end), then is zeroed
    uint4 w = __ldg(reinterpret_cast<const uint4*>(x + (live ? row : static_cast<size_t>(rows) - 1) * D + c0));
    if (!live) w = make_uint4(0u, 0u, 0u, 0u);
    float v[8];
    unpack8(w, v);
    if constexpr (SMOOTH) {
      const float* mu = km + (live ? row / N : 0) * D + c0;
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __fsub_rn(v[i], __ldg(mu + i));
    }
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
#pragma unroll
    for (int off = T / 2; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    float s = 0.f, inv = 0.f;
    if (a > 0.f) {
      s = __fdiv_rn(a, 127.0f);
      inv = __fdiv_rn(127.0f, a);
    }
    if (live) {
      *reinterpret_cast<uint2*>(q + row * D + c0) = pack8(v, inv);
      if (piece == 0) scale[row] = s;
    }
  } else {
    static_assert(G % P == 0, "group must be a whole number of passes");
    constexpr int PASSES = G / P;
    const int n_groups = (N + G - 1) / G;
    const int bh = static_cast<int>(blockIdx.x) / n_groups;
    const int tok0 = (static_cast<int>(blockIdx.x) % n_groups) * G;  // first token of the group in its head
    const size_t row0 = static_cast<size_t>(bh) * N + tok0;
    const int tok = threadIdx.x / T;
    float mu[8];
    if constexpr (SMOOTH) {
      const float* m = km + static_cast<size_t>(bh) * D + c0;
#pragma unroll
      for (int i = 0; i < 8; ++i) mu[i] = __ldg(m + i);
    }
    float v[PASSES][8];
    float a = 0.f;
    // a whole group (every group but a partial last one of its head) compiles without the
    // per-token guards, so that its PASSES loads are all in flight together
    const bool whole = tok0 + G <= N;
    auto load_pass = [&](auto whole_tag) {
    constexpr bool WHOLE = decltype(whole_tag)::value;
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
      const bool live = WHOLE || tok0 + p * P + tok < N;
      // every pass loads (the group's first token for rows past N, then zeroed): no branch
      // between the loads, so all PASSES of them are in flight together
      uint4 w = __ldg(reinterpret_cast<const uint4*>(x + (row0 + (live ? p * P + tok : 0)) * D + c0));
      if (!live) w = make_uint4(0, 0, 0, 0);
      unpack8(w, v[p]);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if constexpr (SMOOTH) v[p][i] = __fsub_rn(v[p][i], mu[i]);
        if (live) a = fmaxf(a, fabsf(v[p][i]));
      }
    }
    };
    if (whole) load_pass(std::true_type{});
    else load_pass(std::false_type{});
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    __shared__ float wmax[8];
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = a;
    __syncthreads();
    a = wmax[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) a = fmaxf(a, wmax[w]);
    float s = 0.f, inv = 0.f;
    if (a > 0.f) {
      s = __fdiv_rn(a, 127.0f);
      inv = __fdiv_rn(127.0f, a);
    }
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
      const size_t row = row0 + p * P + tok;
      if (whole || tok0 + p * P + tok < N) *reinterpret_cast<uint2*>(q + row * D + c0) = pack8(v[p], inv);
    }
    if (threadIdx.x == 0) scale[blockIdx.x] = s;
  }
}

// ---------------------------------------------------------------- launchers
template <int D>
static cudaError_t launch_smooth_d(const __half* k, float* km, int BH, int N, cudaStream_t st) {
  dim3 grid(D / 32, BH);
  smooth_k_kernel<D><<<grid, 1024, 0, st>>>(k, km, N);
  return cudaGetLastError();
}

cudaError_t launch_smooth_k(const __half* k, float* km, int BH, int N, int D, cudaStream_t st) {
  return D == 128 ? launch_smooth_d<128>(k, km, BH, N, st) : launch_smooth_d<64>(k, km, BH, N, st);
}

template <int D, int G, bool SMOOTH>
static cudaError_t launch_quant_g(const __half* x, const float* km, int8_t* q, float* s, int BH, int N,
                                  cudaStream_t st) {
  constexpr int T = D / 8, P = 256 / T;
  const long long rows = static_cast<long long>(BH) * N;
  const long long blocks = (G == 1) ? (rows + P - 1) / P : static_cast<long long>(BH) * ((N + G - 1) / G);
  quant_kernel<D, G, SMOOTH><<<static_cast<unsigned>(blocks), 256, 0, st>>>(x, km, q, s, N, rows);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_quant_d(const __half* x, const float* km, int8_t* q, float* s, int BH, int N,
                                  int group, cudaStream_t st) {
  const bool sm = km != nullptr;
  switch (group) {
    case 1:
      return sm ? launch_quant_g<D, 1, true>(x, km, q, s, BH, N, st) : launch_quant_g<D, 1, false>(x, km, q, s, BH, N, st);
    case 64:
      return sm ? launch_quant_g<D, 64, true>(x, km, q, s, BH, N, st) : launch_quant_g<D, 64, false>(x, km, q, s, BH, N, st);
    case 128:
      return sm ? launch_quant_g<D, 128, true>(x, km, q, s, BH, N, st) : launch_quant_g<D, 128, false>(x, km, q, s, BH, N, st);
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_quant(const __half* x, const float* km, int8_t* q, float* s, int BH, int N, int D, int group,
                         cudaStream_t st) {
  return D == 128 ? launch_quant_d<128>(x, km, q, s, BH, N, group, st)
                  : launch_quant_d<64>(x, km, q, s, BH, N, group, st);
}

}  // namespace sage
