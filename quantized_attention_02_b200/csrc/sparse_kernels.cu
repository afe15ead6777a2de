// sparse_kernels.cu -- the first stage of the block-sparse variant (SpargeAttn abstract: a
// quick prediction of the attention map decides which block products to skip).
//
//   sparse_pool_kernel    per (head, block): the mean of the block's tokens and its self-
//                         similarity |sum_t x_t / |x_t||^2 / n^2 (the mean cosine over ordered
//                         token pairs), for query blocks of 256 tokens and key blocks of 128;
//   sparse_select_kernel  per (head, query block): the compressed map softmax_j(q_bar . k_bar_j *
//                         sm_scale) over the visible key blocks; keeps the fewest blocks, in
//                         decreasing probability (ties: lower index first), whose probabilities
//                         reach tau; adds every visible block when the query block's similarity
//                         is below theta, each key block whose similarity is below theta, and
//                         (causal) the diagonal blocks; writes the kept blocks' ascending list.
// A query block of 256 tokens is the fused kernel's work unit (two query tiles), a key block of
// 128 tokens its key tile, so the list is what that unit walks.  The arithmetic is fp32 (the
// oracle's is fp64): decisions can differ only where a similarity lies at theta or a cumulative
// probability at tau, to within rounding.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "sparse_kernels.cuh"

namespace sage {

constexpr int kPoolThreads = 256;

template <int D>
__global__ void __launch_bounds__(kPoolThreads) sparse_pool_kernel(const __half* __restrict__ q,
                                                                   const __half* __restrict__ k,
                                                                   float* __restrict__ means, float* __restrict__ sims,
                                                                   int N, int NQB, int NKB) {
  constexpr int T = D / 8;               // threads per token row (8 channels each)
  constexpr int R = kPoolThreads / T;    // rows per pass
  constexpr int WARPS = kPoolThreads / 32;
  const int nb = NQB + NKB;
  const int bh = static_cast<int>(blockIdx.x) / nb, b = static_cast<int>(blockIdx.x) % nb;
  const bool is_q = b < NQB;
  const int size = is_q ? kSparseBQ : kSparseBK;
  const int t0 = (is_q ? b : b - NQB) * size;
  const int n = min(size, N - t0);
  const __half* base = (is_q ? q : k) + (static_cast<size_t>(bh) * N + t0) * D;
  const int piece = threadIdx.x % T, row = threadIdx.x / T;
  float sum[8], usum[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) sum[i] = usum[i] = 0.f;
  // whole passes, so that every lane takes part in the row's shuffles; rows past n read zeros.
  // U passes' loads are issued together (a block is 8 to 32 passes), so the loop is not bound
  // by one load's latency per pass.
  constexpr int U = 4;
  for (int t = row; t < size; t += U * R) {
    uint4 w[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      w[u] = make_uint4(0u, 0u, 0u, 0u);
      if (t + u * R < n) w[u] = __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(t + u * R) * D + piece * 8));
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const __half2* h = reinterpret_cast<const __half2*>(&w[u]);
      float x[8];
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
        ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
      }
#pragma unroll
      for (int off = T / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;  // a zero token adds nothing to either sum
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        sum[i] += x[i];
        usum[i] = fmaf(x[i], inv, usum[i]);
      }
    }
  }
  // lanes of a warp with the same piece differ by multiples of T
#pragma unroll
  for (int i = 0; i < 8; ++i) {
#pragma unroll
    for (int off = T; off < 32; off <<= 1) {
      sum[i] += __shfl_xor_sync(0xffffffffu, sum[i], off);
      usum[i] += __shfl_xor_sync(0xffffffffu, usum[i], off);
    }
  }
  __shared__ float ps[WARPS][T][8], pu[WARPS][T][8];
  __shared__ float sq_part[D / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane < T) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      ps[warp][lane][i] = sum[i];
      pu[warp][lane][i] = usum[i];
    }
  }
  __syncthreads();
  if (threadIdx.x < D) {
    const int p = threadIdx.x >> 3, i = threadIdx.x & 7;  // channel p*8 + i = threadIdx.x
    float s = 0.f, u = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      s += ps[w][p][i];
      u += pu[w][p][i];
    }
    means[(static_cast<size_t>(bh) * nb + b) * D + threadIdx.x] = s / static_cast<float>(n);
    float u2 = u * u;  // sum over the block's channels of (sum of unit vectors)^2
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) u2 += __shfl_xor_sync(0xffffffffu, u2, off);
    if (lane == 0) sq_part[threadIdx.x >> 5] = u2;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float u2 = 0.f;
#pragma unroll
    for (int w = 0; w < D / 32; ++w) u2 += sq_part[w];
    sims[static_cast<size_t>(bh) * nb + b] = u2 / (static_cast<float>(n) * static_cast<float>(n));
  }
}

template <int D>
__global__ void __launch_bounds__(256) sparse_select_kernel(const float* __restrict__ means,
                                                            const float* __restrict__ sims, int N, int NQB, int NKB,
                                                            int causal, float sm_scale, float tau, float theta,
                                                            int* __restrict__ kv_count, int16_t* __restrict__ kv_index) {
  constexpr int WARPS = 8;
  const int nb = NQB + NKB;
  const int bh = static_cast<int>(blockIdx.x) / NQB, i = static_cast<int>(blockIdx.x) % NQB;
  __shared__ float qbar[D];
  __shared__ float p[kSparseMaxKeyBlocks];
  __shared__ int16_t order[kSparseMaxKeyBlocks];
  __shared__ uint8_t keep[kSparseMaxKeyBlocks];
  __shared__ float red[WARPS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* mk = means + (static_cast<size_t>(bh) * nb + NQB) * D;
  const float qs = sims[static_cast<size_t>(bh) * nb + i];
  const float* ks = sims + static_cast<size_t>(bh) * nb + NQB;
  const int last_q = min(N, (i + 1) * kSparseBQ) - 1;
  const int nvis = causal ? last_q / kSparseBK + 1 : NKB;
  for (int c = threadIdx.x; c < D; c += blockDim.x) qbar[c] = means[(static_cast<size_t>(bh) * nb + i) * D + c];
  for (int j = threadIdx.x; j < NKB; j += blockDim.x) keep[j] = 0;
  __syncthreads();
  // compressed scores, one warp per key block
  for (int j = warp; j < nvis; j += WARPS) {
    float s = 0.f;
#pragma unroll
    for (int c = lane; c < D; c += 32) s = fmaf(qbar[c], mk[static_cast<size_t>(j) * D + c], s);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) p[j] = s * sm_scale;
  }
  __syncthreads();
  // softmax over the visible blocks
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < nvis; j += blockDim.x) mx = fmaxf(mx, p[j]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int w = 1; w < WARPS; ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  float z = 0.f;
  for (int j = threadIdx.x; j < nvis; j += blockDim.x) z += (p[j] = __expf(p[j] - mx));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  if (lane == 0) red[warp] = z;
  __syncthreads();
  z = 0.f;
#pragma unroll
  for (int w = 0; w < WARPS; ++w) z += red[w];
  for (int j = threadIdx.x; j < nvis; j += blockDim.x) p[j] /= z;
  __syncthreads();
  // rank of each block in decreasing probability (ties: lower index first)
  for (int j = threadIdx.x; j < nvis; j += blockDim.x) {
    const float pj = p[j];
    int rank = 0;
    for (int m = 0; m < nvis; ++m) rank += (p[m] > pj || (p[m] == pj && m < j)) ? 1 : 0;
    order[rank] = static_cast<int16_t>(j);
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // the fewest most probable blocks whose probabilities reach tau
    float cum = 0.f;
    for (int a = 0; a < nvis && cum < tau; ++a) {
      keep[order[a]] = 1;
      cum += p[order[a]];
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < nvis; j += blockDim.x) {
    if (qs < theta || ks[j] < theta) keep[j] = 1;
    if (causal && (j + 1) * kSparseBK > i * kSparseBQ) keep[j] = 1;  // holds one of the block's queries
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int16_t* out = kv_index + (static_cast<size_t>(bh) * NQB + i) * NKB;
    int cnt = 0;
    for (int j = 0; j < nvis; ++j)
      if (keep[j]) out[cnt++] = static_cast<int16_t>(j);
    kv_count[static_cast<size_t>(bh) * NQB + i] = cnt;
  }
}

template <int D>
static cudaError_t launch_sparse_predict_d(const __half* q, const __half* k, float* means, float* sims, int BH, int N,
                                           int causal, float sm_scale, float tau, float theta, int* kv_count,
                                           int16_t* kv_index, cudaStream_t st) {
  const int NQB = (N + kSparseBQ - 1) / kSparseBQ, NKB = (N + kSparseBK - 1) / kSparseBK;
  sparse_pool_kernel<D><<<static_cast<unsigned>(BH) * (NQB + NKB), kPoolThreads, 0, st>>>(q, k, means, sims, N, NQB,
                                                                                          NKB);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sparse_select_kernel<D><<<static_cast<unsigned>(BH) * NQB, 256, 0, st>>>(means, sims, N, NQB, NKB, causal, sm_scale,
                                                                          tau, theta, kv_count, kv_index);
  return cudaGetLastError();
}

size_t sparse_predict_workspace(int BH, int N, int D) {
  const size_t nb = static_cast<size_t>((N + kSparseBQ - 1) / kSparseBQ + (N + kSparseBK - 1) / kSparseBK);
  return static_cast<size_t>(BH) * nb * (D + 1) * sizeof(float);
}

cudaError_t launch_sparse_predict(const __half* q, const __half* k, void* workspace, int BH, int N, int D, int causal,
                                  float sm_scale, float tau, float theta, int* kv_count, int16_t* kv_index,
                                  cudaStream_t st) {
  const size_t nb = static_cast<size_t>((N + kSparseBQ - 1) / kSparseBQ + (N + kSparseBK - 1) / kSparseBK);
  float* means = static_cast<float*>(workspace);
  float* sims = means + static_cast<size_t>(BH) * nb * D;
  return D == 128 ? launch_sparse_predict_d<128>(q, k, means, sims, BH, N, causal, sm_scale, tau, theta, kv_count,
                                                 kv_index, st)
                  : launch_sparse_predict_d<64>(q, k, means, sims, BH, N, causal, sm_scale, tau, theta, kv_count,
                                                kv_index, st);
}

}  // namespace sage
