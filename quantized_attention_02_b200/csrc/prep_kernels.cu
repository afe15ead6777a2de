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
#include <cooperative_groups.h>
#include <cuda_fp16.h>
#include <algorithm>
#include <cstdint>
#include <type_traits>

#include "fp4_codes.cuh"
#include "prep_kernels.cuh"

namespace sage {

namespace cg = cooperative_groups;

// Exact channel sums without 64-bit integer work per element.  Every finite fp16 value x is
// a multiple of 2^-24 with |x| < 2^16.  One rounding add of C = 1.5 * 2^17 (the sum stays in
// [2^17, 2^18), where the fp32 spacing is 2^-6) gives t = C + h with h = x rounded to a
// multiple of 2^-6; bits(t) - bits(C) = h * 2^6 exactly (an integer, |.| < 2^22); h = t - C and
// lo = x - h are exact in fp32 (lo is a multiple of 2^-24 with |lo| <= 2^-7).  So
//   x * 2^24 = (h * 2^6) * 2^18 + lo * 2^24
// and a thread sums the h * 2^6 in int32 and the lo in fp32 -- both exact for up to 64 tokens
// (|sum h * 2^6| < 2^28, |sum lo| <= 1/2 on the 2^-24 grid) -- then moves them into int64.
// Per element that is fp32 adds (packed two at a time) and one integer add, instead of a
// 64-bit shift-and-add.  Infinity / NaN inputs give unspecified (finite-time) results.
constexpr float kSplitC = 196608.0f;          // 1.5 * 2^17
constexpr int kSplitBits = 0x48400000;        // bits of kSplitC
constexpr int kSplitFlushTokens = 64;         // tokens a thread adds between flushes

__device__ __forceinline__ void split_acc(uint32_t word, int& h0, int& h1, float2& lo) {
  const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&word));
  const float2 t = __fadd2_rn(x, make_float2(kSplitC, kSplitC));
  const float2 h = __fadd2_rn(t, make_float2(-kSplitC, -kSplitC));
  lo = __fadd2_rn(lo, __fadd2_rn(x, make_float2(-h.x, -h.y)));
  h0 += __float_as_int(t.x) - kSplitBits;
  h1 += __float_as_int(t.y) - kSplitBits;
}

// One thread-block cluster of C CTAs per head (C = 1, 2, 4 or 8, chosen from N at launch so
// that every CTA gets at least 2048 tokens), the clusters side by side along grid x.  CTA r of the cluster sums the contiguous
// token slice [r*S, min(N, (r+1)*S)), S = ceil(N / C), reading whole rows: a team of T = D/8
// threads covers one token row with one 16-byte load each (coalesced), a 512-thread CTA covers
// 512/T rows per pass and keeps four passes of loads in flight.  The per-CTA channel sums
// (exact int64) meet in the cluster's rank-0 CTA through distributed shared memory, which
// writes the mean: one read of K, no atomics, no workspace, and the integer total does not
// depend on the order of the additions.
constexpr int kSmoothMaxCtas = 8;
constexpr int kSmoothThreads = 512;
constexpr int kSmoothTokensPerCta = 2048;

// Exact channel sums of the token rows [t0, t1) of one head's K (base points at channel piece*8 of
// token 0), by the whole CTA: every thread accumulates its rows with split_acc, flushing into int64
// every kSplitFlushTokens tokens; the CTA's sums land in csum[D].  Ends with the CTA's threads
// synchronized (csum complete).
template <int D>
__device__ __forceinline__ void cta_k_channel_sums(const __half* __restrict__ base, int t0, int t1,
                                                   long long* __restrict__ csum) {
  constexpr int T = D / 8;                 // threads per token row
  constexpr int R = kSmoothThreads / T;    // rows per pass
  constexpr int U = 4;                     // passes in flight
  constexpr int WARPS = kSmoothThreads / 32;
  const int row = threadIdx.x / T;
  constexpr int ITERS = kSplitFlushTokens / U;  // loop iterations between flushes
  long long acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0;
  for (int t = t0 + row; t < t1;) {
    int hs[8];
    float2 ls[4];
#pragma unroll
    for (int i = 0; i < 8; ++i) hs[i] = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) ls[i] = make_float2(0.f, 0.f);
    for (int it = 0; it < ITERS && t < t1; ++it, t += U * R) {
      uint4 w[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        w[u] = (t + u * R < t1) ? __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(t + u * R) * D))
                                : make_uint4(0u, 0u, 0u, 0u);  // +0.0 contributes nothing
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t words[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) split_acc(words[i], hs[2 * i], hs[2 * i + 1], ls[i]);
      }
    }
    // flush: x * 2^24 summed = (sum h*2^6) * 2^18 + (sum lo) * 2^24, both parts exact integers
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += (static_cast<long long>(hs[2 * i]) << 18) + __float2int_rn(__fmul_rn(ls[i].x, 16777216.0f));
      acc[2 * i + 1] += (static_cast<long long>(hs[2 * i + 1]) << 18) + __float2int_rn(__fmul_rn(ls[i].y, 16777216.0f));
    }
  }
  // lanes of a warp with the same piece differ by multiples of T
#pragma unroll
  for (int i = 0; i < 8; ++i) {
#pragma unroll
    for (int off = T; off < 32; off <<= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
  }
  __shared__ long long part[WARPS][T][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane < T) {
#pragma unroll
    for (int i = 0; i < 8; ++i) part[warp][lane][i] = acc[i];
  }
  __syncthreads();
  if (threadIdx.x < D) {
    const int p = threadIdx.x >> 3, i = threadIdx.x & 7;  // channel = p*8 + i = threadIdx.x
    long long s = 0;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) s += part[w][p][i];
    csum[threadIdx.x] = s;
  }
  __syncthreads();
}

// The K mean of channel c from the cluster's per-CTA sums (distributed shared memory):
// fl32(fl32(S_c) / N) * 2^-24.
__device__ __forceinline__ float cluster_k_mean(cg::cluster_group& cluster, long long* csum, int c, int n_ctas,
                                                int N) {
  long long s = 0;
  for (int r = 0; r < n_ctas; ++r) s += *cluster.map_shared_rank(csum + c, r);
  const float s32 = __ll2float_rn(s);
  const float mean = __fdiv_rn(s32, static_cast<float>(N));
  return __fmul_rn(mean, 5.9604644775390625e-08f);
}

template <int D>
__global__ void __launch_bounds__(kSmoothThreads) smooth_k_kernel(const __half* __restrict__ k,
                                                                  float* __restrict__ km, int N) {
  constexpr int T = D / 8;                 // threads per token row
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int n_ctas = static_cast<int>(cluster.num_blocks());  // consecutive CTAs of grid x
  const int bh = static_cast<int>(blockIdx.x) / n_ctas;      // (grid x holds B*H clusters: no 65535 cap)
  const int piece = threadIdx.x % T;       // channels piece*8 .. piece*8+7
  const int slice = (N + n_ctas - 1) / n_ctas;
  const int t0 = rank * slice;
  const int t1 = min(N, t0 + slice);
  __shared__ long long csum[D];  // this CTA's channel sums, read by rank 0 of the cluster
  cta_k_channel_sums<D>(k + (static_cast<size_t>(bh) * N) * D + piece * 8, t0, t1, csum);
  cluster.sync();
  if (rank == 0 && threadIdx.x < D)
    km[static_cast<size_t>(bh) * D + threadIdx.x] = cluster_k_mean(cluster, csum, threadIdx.x, n_ctas, N);
  cluster.sync();  // every CTA keeps its csum in place until rank 0 has read it
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

// INT8 codes of 8 values: y = fl(x * inv), code = round_half_even(y).  The rounding is one add
// of 1.5 * 2^23: for |y| < 2^22 the sum lies in [2^23, 2^24), where the fp32 spacing is 1, so it
// rounds y to the nearest integer (ties to even) and the low byte of its bits is the code in
// two's complement.  No clamp is needed: |x| <= a and inv = fl(127/a) give
// |y| <= 127 (1 + 2^-24)^2 < 127.5, so |code| <= 127 (a = 0 gives inv = 0 and codes 0).
constexpr float kRoundC = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ uint2 pack8(const float (&x)[8], float inv) {
  // scalar _rn intrinsics: the product must be rounded before the add (a contracted
  // multiply-add would round x * inv + C once and break ties differently)
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) b[i] = __float_as_uint(__fadd_rn(__fmul_rn(x[i], inv), kRoundC));
  const uint32_t lo = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
  return make_uint2(lo, hi);
}

// Quantize groups of G tokens (G = 1: per token).  T = D/8 threads cover one token row with
// one 16-byte vector each; a 256-thread CTA covers P = 256/T tokens per pass.
//   G == 1 : each T-lane team is its own group (team-wide shuffle max); teams past the last
//            row compute on zeros and store nothing;
//   G  > 1 : the CTA is one group of G tokens held in registers (G/P passes), CTA-wide max.
//            Groups tile each head separately: ceil(N/G) groups per head, the last one holding
//            the N mod G remaining tokens when G does not divide N.
// Body of quant_kernel: `blk` is the CTA's group (per-block) or its block of P rows (per-token).
template <int D, int G, bool SMOOTH>
__device__ __forceinline__ void quant_block(const __half* __restrict__ x, const float* __restrict__ km,
                                            int8_t* __restrict__ q, float* __restrict__ scale, int N,
                                            long long rows, unsigned blk) {
  constexpr int T = D / 8;
  constexpr int P = 256 / T;
  const int piece = threadIdx.x % T;
  const int c0 = piece * 8;

  if constexpr (G == 1) {
    const size_t row = static_cast<size_t>(blk) * P + threadIdx.x / T;
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
    const int bh = static_cast<int>(blk) / n_groups;
    const int tok0 = (static_cast<int>(blk) % n_groups) * G;  // first token of the group in its head
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
    if (threadIdx.x == 0) scale[blk] = s;
  }
}

template <int D, int G, bool SMOOTH>
__global__ void __launch_bounds__(256) quant_kernel(const __half* __restrict__ x, const float* __restrict__ km,
                                                    int8_t* __restrict__ q, float* __restrict__ scale, int N,
                                                    long long rows) {
  quant_block<D, G, SMOOTH>(x, km, q, scale, N, rows, blockIdx.x);
}

// ---------------------------------------------------------------- the whole preparation in one launch
// K mean, K codes and Q codes of a head in one launch: one cluster of C CTAs per head (C as for
// smooth_k_kernel) splits the head's tokens into slices of whole 128-token blocks.  Phase 1 sums K
// exactly over the slice (cta_k_channel_sums) and every CTA derives the mean from the cluster's
// sums in distributed shared memory.  Phase 2 quantizes the slice's K groups (K minus the mean)
// and Q groups.  Per-block groups go to teams of G*T/8 threads (eight 16-byte loads each; T = D/8
// threads per token row): a team loads its whole group into registers (fp16, one read), takes the
// absmax with shuffles and one named barrier, and writes the codes from registers.  Per-token groups go to T-lane
// teams within a warp (no barrier).  Same arithmetic as smooth_k_kernel and quant_kernel, so the
// same bits.  Rows past N read as zeros (and are neither smoothed nor stored).
// BAR0: the first named-barrier id of this pass's teams (ids BAR0 .. BAR0 + TEAMS - 1).  Each
// pass needs its own ids: a team that finishes its K groups early enters the Q pass while other
// teams still synchronize on theirs, and one barrier id must never see two thread counts at once.
template <int D, int G, bool SMOOTH, int BAR0>
__device__ __forceinline__ void team_quant_groups(const __half* __restrict__ x, const float (&mu)[8],
                                                  int8_t* __restrict__ out, float* __restrict__ scale, int N,
                                                  int bh, int t0, int t1, float* red) {
  constexpr int T = D / 8;       // threads per token row
  const int piece = threadIdx.x % T;
  const __half* head = x + (static_cast<size_t>(bh) * N) * D + piece * 8;
  int8_t* ohead = out + (static_cast<size_t>(bh) * N) * D + piece * 8;
  auto smooth = [&](float (&v)[8], bool live) {
    if constexpr (SMOOTH) {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = live ? __fsub_rn(v[i], mu[i]) : 0.f;
    }
  };
  if constexpr (G == 1) {
    // one token per T-lane team; all CTA rows, U passes at a time
    constexpr int R = kSmoothThreads / T;
    constexpr int U = 4;
    const int row = threadIdx.x / T;
    for (int t = t0 + row; t - row < t1; t += U * R) {  // t - row is CTA-uniform: whole warps iterate
      uint4 w[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tok = t + u * R;
        w[u] = tok < t1 ? __ldg(reinterpret_cast<const uint4*>(head + static_cast<size_t>(tok) * D))
                        : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tok = t + u * R;
        float v[8];
        unpack8(w[u], v);
        smooth(v, tok < t1);
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
        if (tok < t1) {
          *reinterpret_cast<uint2*>(ohead + static_cast<size_t>(tok) * D) = pack8(v, inv);
          if (piece == 0) scale[static_cast<size_t>(bh) * N + tok] = s;
        }
      }
    }
  } else {
    constexpr int PASSES = 8;               // 16-byte loads per thread, all in flight
    constexpr int TEAM = G * T / PASSES;    // threads per group team (64 .. 256)
    constexpr int TEAMS = kSmoothThreads / TEAM;
    constexpr int P = TEAM / T;             // rows per team pass
    constexpr int TW = TEAM / 32;           // warps per team
    static_assert(TEAM % 32 == 0 && TEAMS <= 8 && P * PASSES == G && BAR0 + TEAMS <= 16, "team shape");
    const int team = threadIdx.x / TEAM, tt = threadIdx.x % TEAM;
    const int row = tt / T;
    const int n_groups = (N + G - 1) / G;
    int parity = 0;
    for (int g = t0 / G + team; g * G < t1; g += TEAMS, parity ^= 1) {
      const int g0 = g * G;
      uint4 w[PASSES];
#pragma unroll
      for (int p = 0; p < PASSES; ++p) {
        const int tok = g0 + p * P + row;
        w[p] = tok < t1 ? __ldg(reinterpret_cast<const uint4*>(head + static_cast<size_t>(tok) * D))
                        : make_uint4(0u, 0u, 0u, 0u);
      }
      float a = 0.f;
#pragma unroll
      for (int p = 0; p < PASSES; ++p) {
        float v[8];
        unpack8(w[p], v);
        smooth(v, g0 + p * P + row < t1);
#pragma unroll
        for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      // the team's warp maxima meet in shared memory (two slots, alternating by group, so a slot
      // is only rewritten after every thread of the team has passed the next barrier)
      float* slot = red + parity * (kSmoothThreads / 32) + team * TW;
      if ((tt & 31) == 0) slot[tt >> 5] = a;
      asm volatile("barrier.sync %0, %1;" ::"r"(BAR0 + team), "r"(TEAM) : "memory");
      a = slot[0];
#pragma unroll
      for (int i = 1; i < TW; ++i) a = fmaxf(a, slot[i]);
      float s = 0.f, inv = 0.f;
      if (a > 0.f) {
        s = __fdiv_rn(a, 127.0f);
        inv = __fdiv_rn(127.0f, a);
      }
      if (tt == 0) scale[static_cast<size_t>(bh) * n_groups + g] = s;
#pragma unroll
      for (int p = 0; p < PASSES; ++p) {
        const int tok = g0 + p * P + row;
        float v[8];
        unpack8(w[p], v);
        smooth(v, tok < t1);
        if (tok < t1) *reinterpret_cast<uint2*>(ohead + static_cast<size_t>(tok) * D) = pack8(v, inv);
      }
    }
  }
}

template <int D, int GQ, int GK>
__global__ void __launch_bounds__(kSmoothThreads) prep_fused_kernel(const __half* __restrict__ q,
                                                                    const __half* __restrict__ k,
                                                                    float* __restrict__ km, int8_t* __restrict__ q8,
                                                                    int8_t* __restrict__ k8, float* __restrict__ sq,
                                                                    float* __restrict__ sk, int N) {
  constexpr int T = D / 8;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int n_ctas = static_cast<int>(cluster.num_blocks());
  const int bh = static_cast<int>(blockIdx.x) / n_ctas;
  const int piece = threadIdx.x % T;
  const int slice = ((N + n_ctas - 1) / n_ctas + 127) / 128 * 128;  // whole 128-token blocks
  const int t0 = min(N, rank * slice);
  const int t1 = min(N, t0 + slice);
  __shared__ long long csum[D];
  __shared__ float s_mu[D];
  cta_k_channel_sums<D>(k + (static_cast<size_t>(bh) * N) * D + piece * 8, t0, t1, csum);
  cluster.sync();
  if (threadIdx.x < D) {
    const float m = cluster_k_mean(cluster, csum, threadIdx.x, n_ctas, N);
    s_mu[threadIdx.x] = m;
    if (rank == 0) km[static_cast<size_t>(bh) * D + threadIdx.x] = m;
  }
  cluster.sync();  // the cluster's sums have been read; s_mu is complete in every CTA
  // group-team warp maxima [parity][warp], one array per pass: a warp moving on to the Q groups
  // must not overwrite a slot another warp of its K team has yet to read
  __shared__ float red_k[2 * (kSmoothThreads / 32)], red_q[2 * (kSmoothThreads / 32)];
  float mu[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mu[i] = s_mu[piece * 8 + i];
  team_quant_groups<D, GK, true, 1>(k, mu, k8, sk, N, bh, t0, t1, red_k);   // barrier ids 1 .. 8
  team_quant_groups<D, GQ, false, 9>(q, mu, q8, sq, N, bh, t0, t1, red_q);  // barrier ids 9 .. 12
}

// ---------------------------------------------------------------- V to FP8 (E4M3)
// The FP8 P.V variant (SageAttention2 abstract: (P~, V) quantized to FP8, V smoothed): per
// (b,h) and channel c,
//   vm = fl32(fl32(S_c) / N) * 2^-24 from the exact sum S_c of V[t][c] * 2^24 (SMOOTH; else 0),
//   a  = max_t |fl32(V[t][c] - vm)|,  sv = fl32(a / 448),  inv = fl32(448 / a)  (a = 0: 0, 0),
//   v8 = e4m3(fl32(fl32(V - vm) * inv)), round to nearest even, saturating at +-448.
// One cluster of C CTAs per head (as smooth_k_kernel) in two passes over the head's tokens:
// pass 1 sums (the exact split of split_acc) and takes the channel maximum and minimum of V; the
// CTAs exchange their partials through distributed shared memory and each derives vm, a, sv and
// inv itself; pass 2 re-reads its token slice (now mostly from L2) and writes the codes.  The
// absmax needs no third pass: fl32(x - vm) is monotonic in x, so
// a = max(fl32(max V - vm), fl32(vm - min V)).
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;  // cvt packs its first source into the upper byte
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// FP4 = true: the statistics of the microscaling FP4 variant's V instead of FP8 codes: the same
// exact channel mean (vm), the channel scale sv = fl32(a / 2688) and its inverse rv =
// fl32(2688 / a) (2688 = 6 * 448: the largest E2M1 code times the largest E4M3 scale); no codes.
template <int D, bool SMOOTH, bool FP4 = false>
__global__ void __launch_bounds__(kSmoothThreads, 2) quant_v_fp8_kernel(const __half* __restrict__ v,
                                                                     uint8_t* __restrict__ v8, float* __restrict__ sv,
                                                                     float* __restrict__ vm, int N,
                                                                     float* __restrict__ rv = nullptr) {
  constexpr int T = D / 8;                 // threads per token row (one 16-byte piece each)
  constexpr int R = kSmoothThreads / T;    // rows per pass
  constexpr int U = 4;                     // passes in flight
  constexpr int WARPS = kSmoothThreads / 32;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int n_ctas = static_cast<int>(cluster.num_blocks());
  const int bh = static_cast<int>(blockIdx.x) / n_ctas;
  const int piece = threadIdx.x % T;
  const int row = threadIdx.x / T;
  const int slice = (N + n_ctas - 1) / n_ctas;
  const int t0 = rank * slice;
  const int t1 = min(N, t0 + slice);
  const __half* base = v + (static_cast<size_t>(bh) * N) * D + piece * 8;

  // ---- pass 1: exact sums, maxima and minima of this thread's 8 channels over its rows (the
  // extrema as fp16 pairs: exact, two channels per instruction)
  long long acc[8];
  __half2 hmx[4], hmn[4];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    hmx[i] = __halves2half2(__ushort_as_half(0xFC00u), __ushort_as_half(0xFC00u));  // -inf
    hmn[i] = __halves2half2(__ushort_as_half(0x7C00u), __ushort_as_half(0x7C00u));  // +inf
  }
  constexpr int ITERS = kSplitFlushTokens / U;
  for (int t = t0 + row; t < t1;) {
    int hs[8];
    float2 ls[4];
#pragma unroll
    for (int i = 0; i < 8; ++i) hs[i] = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) ls[i] = make_float2(0.f, 0.f);
    for (int it = 0; it < ITERS && t < t1; ++it, t += U * R) {
      uint4 w[U];
      bool live[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        live[u] = t + u * R < t1;
        w[u] = live[u] ? __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(t + u * R) * D))
                       : make_uint4(0u, 0u, 0u, 0u);  // +0.0 adds nothing; kept out of max / min below
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t words[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if constexpr (SMOOTH) split_acc(words[i], hs[2 * i], hs[2 * i + 1], ls[i]);
          if (live[u]) {
            const __half2 x = *reinterpret_cast<const __half2*>(&words[i]);
            hmx[i] = __hmax2(hmx[i], x);
            hmn[i] = __hmin2(hmn[i], x);
          }
        }
      }
    }
    if constexpr (SMOOTH) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] += (static_cast<long long>(hs[2 * i]) << 18) + __float2int_rn(__fmul_rn(ls[i].x, 16777216.0f));
        acc[2 * i + 1] += (static_cast<long long>(hs[2 * i + 1]) << 18) + __float2int_rn(__fmul_rn(ls[i].y, 16777216.0f));
      }
    }
  }
  float mx[8], mn[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    mx[2 * i] = __low2float(hmx[i]);
    mx[2 * i + 1] = __high2float(hmx[i]);
    mn[2 * i] = __low2float(hmn[i]);
    mn[2 * i + 1] = __high2float(hmn[i]);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
#pragma unroll
    for (int off = T; off < 32; off <<= 1) {
      acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], off));
      mn[i] = fminf(mn[i], __shfl_xor_sync(0xffffffffu, mn[i], off));
    }
  }
  __shared__ long long part[WARPS][T][8];
  __shared__ float pmax[WARPS][T][8], pmin[WARPS][T][8];
  __shared__ long long csum[D];  // this CTA's channel partials, read by every CTA of the cluster
  __shared__ float cmax[D], cmin[D];
  __shared__ float s_vm[D], s_inv[D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane < T) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      part[warp][lane][i] = acc[i];
      pmax[warp][lane][i] = mx[i];
      pmin[warp][lane][i] = mn[i];
    }
  }
  __syncthreads();
  if (threadIdx.x < D) {
    const int p = threadIdx.x >> 3, i = threadIdx.x & 7;  // channel = p*8 + i = threadIdx.x
    long long s = 0;
    float a = -INFINITY, b = INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      s += part[w][p][i];
      a = fmaxf(a, pmax[w][p][i]);
      b = fminf(b, pmin[w][p][i]);
    }
    csum[threadIdx.x] = s;
    cmax[threadIdx.x] = a;
    cmin[threadIdx.x] = b;
  }
  cluster.sync();
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    long long s = 0;
    float hi = -INFINITY, lo = INFINITY;
    for (int r = 0; r < n_ctas; ++r) {
      s += *cluster.map_shared_rank(csum + c, r);
      hi = fmaxf(hi, *cluster.map_shared_rank(cmax + c, r));
      lo = fminf(lo, *cluster.map_shared_rank(cmin + c, r));
    }
    float mean = 0.f;
    if constexpr (SMOOTH) mean = __fmul_rn(__fdiv_rn(__ll2float_rn(s), static_cast<float>(N)), 5.9604644775390625e-08f);
    const float a = fmaxf(0.f, fmaxf(__fsub_rn(hi, mean), __fsub_rn(mean, lo)));
    constexpr float kRange = FP4 ? 2688.0f : 448.0f;
    float scale = 0.f, inv = 0.f;
    if (a > 0.f) {
      scale = __fdiv_rn(a, kRange);
      inv = __fdiv_rn(kRange, a);
    }
    s_vm[c] = mean;
    s_inv[c] = inv;
    if (rank == 0) {
      sv[static_cast<size_t>(bh) * D + c] = scale;
      if constexpr (SMOOTH) vm[static_cast<size_t>(bh) * D + c] = mean;
      if constexpr (FP4) rv[static_cast<size_t>(bh) * D + c] = inv;
    }
  }
  cluster.sync();  // every CTA keeps its partials in place until all have read them
  if constexpr (!FP4) {

    // ---- pass 2: codes of this CTA's token slice
    float m8[8], i8[8];
  #pragma unroll
    for (int i = 0; i < 8; ++i) {
      m8[i] = s_vm[piece * 8 + i];
      i8[i] = s_inv[piece * 8 + i];
    }
    uint8_t* out = v8 + (static_cast<size_t>(bh) * N) * D + piece * 8;
    for (int t = t0 + row; t < t1; t += U * R) {
      uint4 w[U];
  #pragma unroll
      for (int u = 0; u < U; ++u)
        w[u] = (t + u * R < t1) ? __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(t + u * R) * D))
                                : make_uint4(0u, 0u, 0u, 0u);
  #pragma unroll
      for (int u = 0; u < U; ++u) {
        if (t + u * R >= t1) continue;
        float x[8];
        unpack8(w[u], x);
  #pragma unroll
        for (int i = 0; i < 8; ++i) {
          if constexpr (SMOOTH) x[i] = __fsub_rn(x[i], m8[i]);
          x[i] = __fmul_rn(x[i], i8[i]);
        }
        *reinterpret_cast<uint2*>(out + static_cast<size_t>(t + u * R) * D) =
            make_uint2(e4m3x4(x[0], x[1], x[2], x[3]), e4m3x4(x[4], x[5], x[6], x[7]));
      }
    }
  }
}

// ---------------------------------------------------------------- launchers
template <int D>
static cudaError_t launch_smooth_d(const __half* k, float* km, int BH, int N, cudaStream_t st) {
  int ctas = 1;  // a power of two, at most kSmoothMaxCtas, with >= kSmoothTokensPerCta tokens per CTA
  while (ctas < kSmoothMaxCtas && N / (2 * ctas) >= kSmoothTokensPerCta) ctas *= 2;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas) * static_cast<unsigned>(BH));  // one cluster of `ctas` CTAs per head
  cfg.blockDim = dim3(kSmoothThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(ctas);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, smooth_k_kernel<D>, k, km, N);
}

template <int D, bool FP4 = false>
static cudaError_t launch_quant_v_fp8_d(const __half* v, uint8_t* v8, float* sv, float* vm, int BH, int N,
                                        cudaStream_t st, float* rv = nullptr) {
  int ctas = 1;  // the cluster size of smooth_k: >= kSmoothTokensPerCta tokens per CTA, at most 8
  while (ctas < kSmoothMaxCtas && N / (2 * ctas) >= kSmoothTokensPerCta) ctas *= 2;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas) * static_cast<unsigned>(BH));
  cfg.blockDim = dim3(kSmoothThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(ctas);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (vm) return cudaLaunchKernelEx(&cfg, quant_v_fp8_kernel<D, true, FP4>, v, v8, sv, vm, N, rv);
  return cudaLaunchKernelEx(&cfg, quant_v_fp8_kernel<D, false, FP4>, v, v8, sv, vm, N, rv);
}

cudaError_t launch_quant_v_fp8(const __half* v, uint8_t* v8, float* sv, float* vm, int BH, int N, int D,
                               cudaStream_t st) {
  return D == 128 ? launch_quant_v_fp8_d<128>(v, v8, sv, vm, BH, N, st) : launch_quant_v_fp8_d<64>(v, v8, sv, vm, BH, N, st);
}

template <int D, int GQ, int GK>
static cudaError_t launch_prep_fused_g(const __half* q, const __half* k, float* km, int8_t* q8, int8_t* k8, float* sq,
                                       float* sk, int BH, int N, cudaStream_t st) {
  int ctas = 1;  // the cluster size of smooth_k
  while (ctas < kSmoothMaxCtas && N / (2 * ctas) >= kSmoothTokensPerCta) ctas *= 2;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas) * static_cast<unsigned>(BH));
  cfg.blockDim = dim3(kSmoothThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(ctas);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prep_fused_kernel<D, GQ, GK>, q, k, km, q8, k8, sq, sk, N);
}

template <int D>
static cudaError_t launch_prep_fused_d(const __half* q, const __half* k, float* km, int8_t* q8, int8_t* k8, float* sq,
                                       float* sk, int BH, int N, bool per_token, cudaStream_t st) {
  return per_token ? launch_prep_fused_g<D, 1, 1>(q, k, km, q8, k8, sq, sk, BH, N, st)
                   : launch_prep_fused_g<D, 128, 64>(q, k, km, q8, k8, sq, sk, BH, N, st);
}

cudaError_t launch_prep_fused(const __half* q, const __half* k, float* km, int8_t* q8, int8_t* k8, float* sq,
                              float* sk, int BH, int N, int D, bool per_token, cudaStream_t st) {
  return D == 128 ? launch_prep_fused_d<128>(q, k, km, q8, k8, sq, sk, BH, N, per_token, st)
                  : launch_prep_fused_d<64>(q, k, km, q8, k8, sq, sk, BH, N, per_token, st);
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
static cudaError_t launch_quant_qk_d(const __half* q, const __half* k, const float* km, int8_t* q8, int8_t* k8,
                                     float* sq, float* sk, int BH, int N, bool per_token, cudaStream_t st) {
  // two launches: measured faster than one launch over both tensors (each kernel keeps its own
  // register count, so the K groups run at a higher occupancy)
  cudaError_t e;
  if (per_token) {
    e = launch_quant_g<D, 1, false>(q, nullptr, q8, sq, BH, N, st);
    if (e != cudaSuccess) return e;
    return km ? launch_quant_g<D, 1, true>(k, km, k8, sk, BH, N, st) : launch_quant_g<D, 1, false>(k, km, k8, sk, BH, N, st);
  }
  e = launch_quant_g<D, 128, false>(q, nullptr, q8, sq, BH, N, st);
  if (e != cudaSuccess) return e;
  return km ? launch_quant_g<D, 64, true>(k, km, k8, sk, BH, N, st) : launch_quant_g<D, 64, false>(k, km, k8, sk, BH, N, st);
}

cudaError_t launch_quant_qk(const __half* q, const __half* k, const float* km, int8_t* q8, int8_t* k8, float* sq,
                            float* sk, int BH, int N, int D, bool per_token, cudaStream_t st) {
  return D == 128 ? launch_quant_qk_d<128>(q, k, km, q8, k8, sq, sk, BH, N, per_token, st)
                  : launch_quant_qk_d<64>(q, k, km, q8, k8, sq, sk, BH, N, per_token, st);
}

// ---------------------------------------------------------------- microscaling FP4 variant
// (SageAttention3 entry: microscaling FP4 attention on Blackwell's FP4 tensor cores).  Formats: E2M1
// codes, two per byte (the even element in the low nibble), one UE4M3 scale per 16 elements
// along the contraction dimension, chosen as e4m3(fl32(max|z| / 6)), codes
// e2m1(fl32(z * fl32(1 / scale))).  Scales are stored in the tensor cores' scale atoms: 512 bytes
// per 128 rows x 4 scales (64 elements of the contraction), row r's four scales at byte
// (r % 32) * 16 + (r / 32) * 4.

// Q (SMOOTH = false) or K minus its channel mean km: one CTA per (head, 128-token tile), one
// thread per token.  g[bh, tile] = fl32(a / 2688) with a the tile's largest |x|; z = fl32(x *
// fl32(2688 / a)); codes [BH][N][D/2 bytes].  Scale atoms (D/64 per row group, one per 64
// channels): Q (ROWS64 = false) [BH][tiles][D/64][512], the tile's 128 tokens as rows; K
// (ROWS64 = true) [BH][ceil(N/64)][D/64][512], each 64-token half in the first 64 rows of its own
// atoms (the attention kernel's key tiles are 64 tokens), the other rows zero.
template <int D, bool SMOOTH, bool ROWS64 = false>
__global__ void __launch_bounds__(128) quant_fp4_kernel(const __half* __restrict__ x, const float* __restrict__ km,
                                                        uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                                        float* __restrict__ g, int N) {
  constexpr int NA = D / 64;  // scale atoms per row group
  const int nt = (N + 127) / 128;
  const int bh = static_cast<int>(blockIdx.x) / nt, tile = static_cast<int>(blockIdx.x) % nt;
  const int r = threadIdx.x, row = tile * 128 + r;
  const bool live = row < N;
  __shared__ float s_km[D];
  __shared__ float s_max[4];
  if (r < D) s_km[r] = SMOOTH ? km[static_cast<size_t>(bh) * D + r] : 0.f;
  __syncthreads();
  float v[D];
  const uint4* src = reinterpret_cast<const uint4*>(x + (static_cast<size_t>(bh) * N + (live ? row : 0)) * D);
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    float f[8];
    unpack8(live ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u), f);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      v[8 * i + k] = (SMOOTH && live) ? __fsub_rn(f[k], s_km[8 * i + k]) : f[k];
      a = fmaxf(a, fabsf(v[8 * i + k]));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
  if ((r & 31) == 0) s_max[r >> 5] = a;
  __syncthreads();
  a = fmaxf(fmaxf(s_max[0], s_max[1]), fmaxf(s_max[2], s_max[3]));
  const float rr = a > 0.f ? __fdiv_rn(2688.0f, a) : 0.f;
  if (r == 0) g[static_cast<size_t>(bh) * nt + tile] = __fdiv_rn(a, 2688.0f);
  uint32_t w[D / 8];
  uint32_t sfw[NA];
#pragma unroll
  for (int a2 = 0; a2 < NA; ++a2) sfw[a2] = 0u;
#pragma unroll
  for (int gi = 0; gi < D / 16; ++gi) {
    float z[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) z[k] = __fmul_rn(v[16 * gi + k], rr);
    const uint32_t s8 = microscale16(z, w[2 * gi], w[2 * gi + 1]);
    sfw[gi >> 2] |= (live ? s8 : 0u) << (8 * (gi & 3));
  }
  if (live) {
    uint4* dst = reinterpret_cast<uint4*>(codes + (static_cast<size_t>(bh) * N + row) * (D / 2));
#pragma unroll
    for (int i = 0; i < D / 32; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  }
  if constexpr (ROWS64) {
    const int n64 = (N + 63) / 64, half = tile * 2 + (r >> 6), lr = r & 63;
    if (half < n64) {
      uint8_t* atoms = sf + (static_cast<size_t>(bh) * n64 + half) * (NA * 512) + (lr & 31) * 16 + (lr >> 5) * 4;
#pragma unroll
      for (int a2 = 0; a2 < NA; ++a2) {
        *reinterpret_cast<uint32_t*>(atoms + 512 * a2) = sfw[a2];
        if (lr < 32)  // rows 64..127 of the atom (bytes 8..15 of each 16-byte line): zero
          *reinterpret_cast<uint2*>(atoms + 512 * a2 + 8) = make_uint2(0u, 0u);
      }
    }
  } else {
    uint8_t* atoms = sf + (static_cast<size_t>(bh) * nt + tile) * (NA * 512) + (r & 31) * 16 + (r >> 5) * 4;
#pragma unroll
    for (int a2 = 0; a2 < NA; ++a2) *reinterpret_cast<uint32_t*>(atoms + 512 * a2) = sfw[a2];
  }
}

// V codes along the tokens: one CTA per (head, 128-key tile), one thread per channel.
// z = fl32(fl32(v - vm) * rv), groups of 16 keys; codes transposed [BH][D][n_tiles * 64 bytes]
// (keys past N: zero codes, outside every group's maximum); scale atoms [BH][tiles][2][512] (keys
// 0-63, 64-127 of the tile) with the D channels as rows (D = 64: rows 64..127 zero).
template <int D, bool SMOOTH>
__global__ void __launch_bounds__(D) quant_v_fp4_kernel(const __half* __restrict__ v, const float* __restrict__ vm,
                                                        const float* __restrict__ rv, uint8_t* __restrict__ codes_t,
                                                        uint8_t* __restrict__ sf, int N) {
  const int nt = (N + 127) / 128;
  const int bh = static_cast<int>(blockIdx.x) / nt, tile = static_cast<int>(blockIdx.x) % nt;
  const int c = threadIdx.x;
  const float mean = SMOOTH ? vm[static_cast<size_t>(bh) * D + c] : 0.f;
  const float rr = rv[static_cast<size_t>(bh) * D + c];
  const int n_live = min(128, N - tile * 128);
  // the tile's rows in shared memory (16-byte loads across the CTA), then one channel per thread
  __shared__ uint4 s_tile[128 * D / 8];
  const uint4* gsrc = reinterpret_cast<const uint4*>(v + (static_cast<size_t>(bh) * N + tile * 128) * D);
#pragma unroll 4
  for (int i = c; i < n_live * (D / 8); i += D) s_tile[i] = __ldg(gsrc + i);
  __syncthreads();
  const __half* src = reinterpret_cast<const __half*>(s_tile) + c;
  uint32_t w[16];
  uint32_t sfw[2] = {0u, 0u};
#pragma unroll
  for (int gi = 0; gi < 8; ++gi) {
    float z[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int t = 16 * gi + k;
      const float xv = t < n_live ? __half2float(src[static_cast<size_t>(t) * D]) : 0.f;
      z[k] = t < n_live ? __fmul_rn(SMOOTH ? __fsub_rn(xv, mean) : xv, rr) : 0.f;
    }
    const uint32_t s8 = microscale16(z, w[2 * gi], w[2 * gi + 1]);
    sfw[gi >> 2] |= s8 << (8 * (gi & 3));
  }
  uint4* dst = reinterpret_cast<uint4*>(codes_t + (static_cast<size_t>(bh) * D + c) * (static_cast<size_t>(nt) * 64) +
                                        tile * 64);
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  uint8_t* atoms = sf + (static_cast<size_t>(bh) * nt + tile) * 1024 + (c & 31) * 16 + (c >> 5) * 4;
  *reinterpret_cast<uint32_t*>(atoms) = sfw[0];
  *reinterpret_cast<uint32_t*>(atoms + 512) = sfw[1];
  if (D == 64 && c < 32) {  // rows 64..127 of the atoms: zero
    *reinterpret_cast<uint2*>(atoms + 8) = make_uint2(0u, 0u);
    *reinterpret_cast<uint2*>(atoms + 512 + 8) = make_uint2(0u, 0u);
  }
}

template <int D>
static cudaError_t launch_quant_qk_fp4_d(const __half* q, const __half* k, const float* km, uint8_t* q4, uint8_t* sfq,
                                         float* gq, uint8_t* k4, uint8_t* sfk, float* gk, int BH, int N,
                                         cudaStream_t st) {
  const unsigned blocks = static_cast<unsigned>(BH) * static_cast<unsigned>((N + 127) / 128);
  quant_fp4_kernel<D, false><<<blocks, 128, 0, st>>>(q, nullptr, q4, sfq, gq, N);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (km) quant_fp4_kernel<D, true, true><<<blocks, 128, 0, st>>>(k, km, k4, sfk, gk, N);
  else quant_fp4_kernel<D, false, true><<<blocks, 128, 0, st>>>(k, nullptr, k4, sfk, gk, N);
  return cudaGetLastError();
}

cudaError_t launch_quant_qk_fp4(const __half* q, const __half* k, const float* km, uint8_t* q4, uint8_t* sfq,
                                float* gq, uint8_t* k4, uint8_t* sfk, float* gk, int BH, int N, int D,
                                cudaStream_t st) {
  return D == 128 ? launch_quant_qk_fp4_d<128>(q, k, km, q4, sfq, gq, k4, sfk, gk, BH, N, st)
                  : launch_quant_qk_fp4_d<64>(q, k, km, q4, sfq, gq, k4, sfk, gk, BH, N, st);
}

template <int D>
static cudaError_t launch_quant_v_fp4_d(const __half* v, uint8_t* v4t, uint8_t* sfv, float* gv, float* vm, float* rv,
                                        int BH, int N, cudaStream_t st) {
  cudaError_t e = launch_quant_v_fp8_d<D, true>(v, nullptr, gv, vm, BH, N, st, rv);
  if (e != cudaSuccess) return e;
  const unsigned blocks = static_cast<unsigned>(BH) * static_cast<unsigned>((N + 127) / 128);
  if (vm) quant_v_fp4_kernel<D, true><<<blocks, D, 0, st>>>(v, vm, rv, v4t, sfv, N);
  else quant_v_fp4_kernel<D, false><<<blocks, D, 0, st>>>(v, nullptr, rv, v4t, sfv, N);
  return cudaGetLastError();
}

cudaError_t launch_quant_v_fp4(const __half* v, uint8_t* v4t, uint8_t* sfv, float* gv, float* vm, float* rv, int BH,
                               int N, int D, cudaStream_t st) {
  return D == 128 ? launch_quant_v_fp4_d<128>(v, v4t, sfv, gv, vm, rv, BH, N, st)
                  : launch_quant_v_fp4_d<64>(v, v4t, sfv, gv, vm, rv, BH, N, st);
}

}  // namespace sage
