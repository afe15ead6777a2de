// attn_kernels.cu -- the fused 8-bit attention forward kernel for sm_100a, and the debug
// kernel that exposes its INT32 Q.K^T.
//
// Method (SageAttention summary page, Summary bullets 1-2 and "FlashAttention-style tiling"):
//   S   = q8 . k8^T                       INT8 x INT8 -> INT32 on the tensor cores (tcgen05 kind::i8)
//   s   = S * sq(i) * sk(j) * sm_scale    dequantized in fp32, kept in log2 units (x log2 e)
//   online softmax over key tiles: running row max m, row sum l, exp2
//   P~  = fp16(exp2(s - m))               written back to tensor memory
//   O  += P~ . V                          FP16 x FP16 -> FP32 on the tensor cores (kind::f16,
//                                         A operand read straight from tensor memory)
//   O   = O / l                           stored as fp16
//
// CTA organisation (one CTA per SM: 512 TMEM columns and > 114 KB of shared memory), for head
// dimension 64 (128 has its own kernel, attn_v3.cuh):
//   work unit = (head, pair of 128-row query tiles); 12 warps:
//     warp 0      TMA producer: Q tiles once, then K / V tiles through a STAGES-deep ring
//     warps 1, 2  MMA issuers of query tile 0 / 1 (warp 1 also allocates TMEM)
//     warps 4-7   softmax for query tile 0 (thread = one query row = one TMEM lane)
//     warps 8-11  softmax for query tile 1
//   TMEM columns: S0 [0,128) S1 [128,256) O0 [256,320) O1 [320,384) P~0 [384,448) P~1 [448,512)
//   (P~ fp16, two keys per column).  Per key tile j an MMA warp issues QK_t(j+1) as soon as the
//   softmax has copied S_t(j) into registers (S_t is free), then PV_t(j) as the two halves of
//   P~_t(j) arrive; the softmax waits for PV_t(j-1) before it writes P~_t(j) (one P~ buffer).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <type_traits>

#include "attn_kernels.cuh"
#include "fp4_codes.cuh"
#include "sm100_ptx.cuh"

namespace sage {

template <int D>
struct AttnLayout {
  static constexpr int BM = 128;          // query rows per tile
  static constexpr int BN = 128;          // keys per tile
  static constexpr int NQT = 2;           // query tiles per CTA
  static constexpr int STAGES = D == 128 ? 3 : 4;
  static constexpr int Q_BYTES = BM * D;  // int8 tile
  static constexpr int K_BYTES = BN * D;  // int8 tile
  static constexpr int V_BOX = BN * 128;  // one 64-column fp16 box (128-byte rows)
  static constexpr int V_BYTES = BN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQT * Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * K_BYTES;
  static constexpr int OFF_SK = OFF_V + STAGES * V_BYTES;           // per-token key scales
  static constexpr int OFF_BAR = OFF_SK + STAGES * BN * 4;
  static constexpr int NUM_BARS = 1 + 3 * STAGES + 6 * NQT;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int MAX_LIST = 512;                      // block-sparse variant: key tiles a CTA may visit
  static constexpr int OFF_LIST = OFF_MISC + 16;            // int16 list of the key tiles visited
  static constexpr int OFF_SKIP = OFF_LIST + MAX_LIST * 2;  // [2][3] stage-2 votes, [2][2] P.V keep flags
  static constexpr int USED = OFF_SKIP + 64;
  // at least 116 KB so that two CTAs never share an SM (each holds all 512 TMEM columns)
  static constexpr int SMEM = (USED + 1024 > 116 * 1024 ? USED + 1024 : 116 * 1024);
  __host__ __device__ static constexpr uint32_t s_col(int t) { return 128u * t; }
  __host__ __device__ static constexpr uint32_t o_col(int t) { return 256u + D * t; }
  __host__ __device__ static constexpr uint32_t p_col(int t) { return 256u + 2 * D + 64u * t; }
  static_assert(256 + 2 * D + 128 <= 512, "S, O and P~ of two query tiles fit the 512 TMEM columns");
  static constexpr int THREADS = 384;
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float fast_log2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Magic-number integer -> float: for |S| < 2^22 the bits of S + 0x4B400000 are the float
// 1.5 * 2^23 + S exactly.
constexpr uint32_t kMagicBits = 0x4B400000u;
constexpr float kMagicF = 12582912.0f;

// Scale c with its 3 lowest mantissa bits cleared (21 significant bits): kMagicF * c is then
// exact in fp32 (relative change of c at most 2^-20).
__device__ __forceinline__ float trim_scale(float c) { return __uint_as_float(__float_as_uint(c) & ~7u); }

// 4 ulps of x (a power of two), or the smallest normal for tiny / zero x.
__device__ __forceinline__ float offset_quantum(float x) {
  const int e = static_cast<int>((__float_as_uint(x) >> 23) & 0xFFu);
  return e > 22 ? __uint_as_float(static_cast<uint32_t>(e - 21) << 23) : 0x1p-126f;
}

// Smallest multiple of the power of two q that is >= x (exact).  Floats of magnitude at
// least 2^23 q are multiples of q already (and x / q might overflow).
__device__ __forceinline__ float round_up_to(float x, float q) {
  return fabsf(x) < q * 8388608.0f ? ceilf(x / q) * q : x;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Maximum of 64 signed integers held as bits: four independent chains of one 2-input and
// seven 3-input maxima (4 * (2 + 7 * 2) = 64 elements, x[0..63] exactly).
__device__ __forceinline__ int imax64(const uint32_t* x) {
  int a[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) a[k] = max(static_cast<int>(x[k]), static_cast<int>(x[4 + k]));
#pragma unroll
  for (int i = 8; i < 64; i += 8) {
#pragma unroll
    for (int k = 0; k < 4; ++k) a[k] = __vimax3_s32(a[k], static_cast<int>(x[i + k]), static_cast<int>(x[i + 4 + k]));
  }
  return max(max(a[0], a[1]), max(a[2], a[3]));
}

template <uint32_t N>
__device__ __forceinline__ void reg_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void reg_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Bounded wait used on exit paths: ignores the abort flag, records a timeout.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) {
      atomicExch(&g_device_error, kDevTimeoutBarrier);
      return;
    }
  }
}

__device__ __forceinline__ void group_bar(int id) { asm volatile("barrier.sync %0, 128;" ::"r"(id) : "memory"); }

// TRACE builds record SM clock stamps of the pipeline events of the first trace_ctas CTAs
// (layout documented at sage_debug_attn_trace in include/sage_attn.h).
//
// SPARSE = true is the block-sparse variant of the SpargeAttn abstract, as in the head-dimension
// 128 kernel: kv_count[bh * n_pairs + pair] and the ascending key-tile list
// kv_index[(bh * n_pairs + pair) * ceil(N/128) + i] give the key tiles this CTA visits (stage 1),
// and a softmax group drops key tile j of its query tile when every row below N scores more than
// skip_lambda (log2 units) under its running maximum there (stage 2): no exp2 pass, no P.V.
template <int D, bool CAUSAL, bool PER_TOKEN, bool TRACE, bool RAGGED, bool SPARSE = false>
__global__ void __launch_bounds__(384, 1)
    sage_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const float* __restrict__ sq,
                     const float* __restrict__ sk, __half* __restrict__ o, int BH, int N,
                     float sm_scale_log2, long long* __restrict__ trace, int trace_ctas,
                     const int* __restrict__ kv_count = nullptr, const int16_t* __restrict__ kv_index = nullptr,
                     float skip_lambda = 0.f) {
  using L = AttnLayout<D>;
  constexpr int STAGES = L::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  float* sSK = reinterpret_cast<float*>(smem + L::OFF_SK);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* bar_q = bars;
  uint64_t* bar_k_full = bars + 1;
  uint64_t* bar_v_full = bars + 1 + STAGES;
  uint64_t* bar_kv_empty = bars + 1 + 2 * STAGES;
  uint64_t* bar_s_full = bars + 1 + 3 * STAGES;
  uint64_t* bar_p_full = bar_s_full + 2;  // P~ of keys 64..127 (the whole tile) written
  uint64_t* bar_o_done = bar_s_full + 4;
  uint64_t* bar_drain = bar_s_full + 6;   // one per MMA warp
  uint64_t* bar_p_lo = bar_s_full + 8;    // P~ of keys 0..63 written
  uint64_t* bar_s_free = bar_s_full + 10; // softmax t holds S_t(j) in registers: S_t may be overwritten
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  int* arrived = reinterpret_cast<int*>(smem + L::OFF_MISC + 8);  // trace builds: threads at the final barrier

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: consecutive CTAs share a head (its K/V stay in L2); within a head the
  // query-tile pairs with the most key tiles (causal) come first
  const int n_qtiles = (N + L::BM - 1) / L::BM;  // the last tile may be partial (rows past N: zeros)
  const int n_pairs = (n_qtiles + 1) / 2;
  const int bh = static_cast<int>(blockIdx.x) / n_pairs;
  const int pair = n_pairs - 1 - static_cast<int>(blockIdx.x) % n_pairs;
  const int tile0 = 2 * pair;
  const int n_tiles = min(2, n_qtiles - tile0);
  const int n_kv_total = (N + L::BN - 1) / L::BN;
  int n_iter[2];
  n_iter[0] = CAUSAL ? tile0 + 1 : n_kv_total;
  n_iter[1] = (n_tiles > 1) ? (CAUSAL ? tile0 + 2 : n_kv_total) : 0;
  int16_t* sList = reinterpret_cast<int16_t*>(smem + L::OFF_LIST);
  int* sSkipVote = reinterpret_cast<int*>(smem + L::OFF_SKIP);     // [2 tiles][3]: bit 0 a row keeps the
                                                                   // tile, bit 1 a warp gave up waiting
  int* sPvKeep = reinterpret_cast<int*>(smem + L::OFF_SKIP + 32);  // [2 tiles][2]: P.V of key tile j issued
  if constexpr (SPARSE) {
    // causal lists end with the diagonal tiles: tile 0 stops one step before tile 1 when the
    // list holds tile0 + 1.  Count and entries are clamped into range (a malformed list gives
    // unspecified output, never an access outside the tensors); the cta_sync after the barrier
    // set-up publishes the list.
    const int count = min(max(kv_count[static_cast<size_t>(bh) * n_pairs + pair], 0), min(n_kv_total, L::MAX_LIST));
    const int16_t* lst = kv_index + (static_cast<size_t>(bh) * n_pairs + pair) * n_kv_total;
    for (int i = threadIdx.x; i < count; i += L::THREADS)
      sList[i] = static_cast<int16_t>(min(max(static_cast<int>(lst[i]), 0), n_kv_total - 1));
    const int last = count > 0 ? min(max(static_cast<int>(lst[count - 1]), 0), n_kv_total - 1) : -1;
    n_iter[1] = n_tiles > 1 ? count : 0;
    n_iter[0] = (CAUSAL && n_tiles > 1 && last == tile0 + 1) ? count - 1 : count;
  }
  const int n_kv = max(n_iter[0], n_iter[1]);
  auto key_tile = [&](int j) -> int {  // key tile visited in step j
    if constexpr (SPARSE) return sList[j];
    return j;
  };
  const int row_base = bh * N;  // first row of this head in the [BH*N, D] arrays
  long long* trace_row = nullptr;
  if constexpr (TRACE) {
    if (static_cast<int>(blockIdx.x) < trace_ctas) {
      trace_row = trace + static_cast<size_t>(blockIdx.x) * (2 + 10 * n_kv_total);
      if (threadIdx.x == 0) trace_row[0] = clock_stamp();
    }
  }
  // trace slots: [0] start, [1] end, then per key tile j: softmax group t events e (0 S ready,
  // 1 max done, 2 P~ signalled) at 2 + (3t+e) n_kv_total + j; MMA thread events e (0 P.V issued,
  // 1 next Q.K^T issued) for tile t at 2 + (6 + 2t + e) n_kv_total + j
  auto stamp = [&](int slot) {
    if constexpr (TRACE) {
      if (trace_row) trace_row[2 + slot] = clock_stamp();
    }
  };

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_k_full + s, 1);
      mbar_init(bar_v_full + s, 1);
      mbar_init(bar_kv_empty + s, n_tiles);  // one commit from each MMA warp
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s_full + t, 1);
      mbar_init(bar_p_full + t, 128);
      mbar_init(bar_o_done + t, 1);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_drain + 1, 1);
    mbar_init(bar_p_lo, 128);
    mbar_init(bar_p_lo + 1, 128);
    mbar_init(bar_s_free, 128);
    mbar_init(bar_s_free + 1, 128);
    for (int i = 0; i < 6; ++i) sSkipVote[i] = 0;
    *abort_flag = 0;
    *arrived = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync();  // lane 0 of warp 0 initialised the barriers alone
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Registers: the block is launched with 168 per thread (384 x 168); the control
  // warpgroup hands most of its share to the two softmax warpgroups: 128 x 72 + 256 x 216.
  // Each setmaxnreg is executed by a whole warpgroup and dominates that group's code.
  if (warp < 4) {
    reg_dealloc<72>();
    if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      int issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = 0;
      mbar_arrive_expect_tx(bar_q, n_tiles * L::Q_BYTES);
      for (int t = 0; t < n_tiles; ++t)
        tma_load_3d(sQ + t * L::Q_BYTES, &tm_q, bar_q, 0, (tile0 + t) * L::BM, bh);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % STAGES;
        const int it = j / STAGES;
        if (j >= STAGES && !mbar_wait(bar_kv_empty + s, (it - 1) & 1, abort_flag)) break;
        const int key_row = key_tile(j) * L::BN;  // token row within the head
        // per-token key scales: one bulk copy when the 128 scales exist and start on a 16-byte
        // boundary, else plain loads (zeros past N) stored before the arrival that publishes them
        const bool bulk_sk = PER_TOKEN && (N % 4 == 0) && key_row + L::BN <= N;
        if (PER_TOKEN && !bulk_sk) {
          for (int c = 0; c < L::BN; ++c)
            sSK[s * L::BN + c] = key_row + c < N ? __ldg(sk + row_base + key_row + c) : 0.f;
        }
        mbar_arrive_expect_tx(bar_k_full + s, L::K_BYTES + (bulk_sk ? L::BN * 4 : 0));
        tma_load_3d(sK + s * L::K_BYTES, &tm_k, bar_k_full + s, 0, key_row, bh);
        if (bulk_sk) bulk_load(sSK + s * L::BN, sk + row_base + key_row, L::BN * 4, bar_k_full + s);
        mbar_arrive_expect_tx(bar_v_full + s, L::V_BYTES);
#pragma unroll
        for (int b = 0; b < D / 64; ++b)
          tma_load_3d(sV + s * L::V_BYTES + b * L::V_BOX, &tm_v, bar_v_full + s, 64 * b, key_row, bh);
        issued[s] = it + 1;
      }
      if (*abort_flag) {  // let copies in flight land before the CTA exits
        mbar_drain(bar_q, 0);
        for (int s = 0; s < STAGES; ++s) {
          if (issued[s] > 0) {
            mbar_drain(bar_k_full + s, (issued[s] - 1) & 1);
            mbar_drain(bar_v_full + s, (issued[s] - 1) & 1);
          }
        }
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ================================================================ MMA warps
    // Warp 1 issues the products of query tile 0, warp 2 those of tile 1: one tcgen05.mma stream
    // per warp leaves the tensor core idle between back-to-back instructions (about 110-140
    // cycles each), two independent streams keep it busy.  The whole warp runs the loop
    // (uniform control flow and descriptors); elect.sync lets one lane issue each instruction.
    // Per key tile j: QK(j+1) first (it only needs S_t free and K(j+1)), so that the next scores
    // are ready when the softmax finishes tile j; then PV(j) from the P~ region.
    const int t = warp - 1;
    if (t < n_tiles) {
      constexpr uint32_t IDESC_QK = make_idesc(2 /*s32*/, 1 /*s8*/, 1 /*s8*/, 0, 0, 128, L::BN);
      constexpr uint32_t IDESC_PV = make_idesc(1 /*f32*/, 0 /*f16*/, 0 /*f16*/, 0, 1 /*V is MN-major*/, 128, D);
      constexpr SwizzleMode QK_SWZ = D == 128 ? kSwizzle128B : kSwizzle64B;
      constexpr uint32_t QK_SBO = D == 128 ? 1024 : 512;  // 8 rows of D bytes
      const uint32_t q_base = smem_u32(sQ) + t * L::Q_BYTES, k_base = smem_u32(sK), v_base = smem_u32(sV);
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
      };

      auto issue_qk = [&](int s) {
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
          const uint64_t a = make_smem_desc(q_base + kk * 32, 16, QK_SBO, QK_SWZ);
          const uint64_t b = make_smem_desc(k_base + s * L::K_BYTES + kk * 32, 16, QK_SBO, QK_SWZ);
          mma_i8_ss_warp(tmem + L::s_col(t), a, b, IDESC_QK, kk > 0 ? 1u : 0u);
        }
        mma_commit_warp(bar_s_full + t);
      };
      // P.V for keys [16*k0, 16*k1) of the tile: 16 keys per MMA = 16 rows of 128 B in the V box
      // (LBO jumps to the next 64 columns); P~ columns hold two fp16 keys each
      auto issue_pv = [&](int s, bool first, int k0, int k1) {
#pragma unroll
        for (int kk = k0; kk < k1; ++kk) {
          const uint64_t b = make_smem_desc(v_base + s * L::V_BYTES + kk * 16 * 128, L::V_BOX, 1024, kSwizzle128B);
          mma_f16_ts_warp(tmem + L::o_col(t), tmem + L::p_col(t) + kk * 8, b, IDESC_PV, (first && kk == 0) ? 0u : 1u);
        }
      };

      bool ok = wait(bar_q, 0) && wait(bar_k_full, 0);
      if (ok) {
        tc_fence_after();
        issue_qk(0);
      }
      for (int j = 0; ok && j < n_iter[t]; ++j) {
        const int s = j % STAGES;
        if (j + 1 < n_iter[t]) {
          // S_t(j+1) overwrites S_t(j) once the softmax holds S_t(j) in registers
          const int s1 = (j + 1) % STAGES;
          if (!wait(bar_k_full + s1, ((j + 1) / STAGES) & 1)) break;
          if (!wait(bar_s_free + t, j & 1)) break;
          tc_fence_after();
          issue_qk(s1);
          if (lane == 0) stamp((7 + 2 * t) * n_kv_total + j);
        }
        if (!wait(bar_v_full + s, (j / STAGES) & 1)) break;
        // the first half of P~ is signalled separately, so that its P.V overlaps the exp2
        // work on the second half
        if (!wait(bar_p_lo + t, j & 1)) break;
        tc_fence_after();
        // block-sparse variant: the softmax group may have dropped key tile j (never the first)
        bool issue = true;
        if constexpr (SPARSE) issue = *reinterpret_cast<volatile int*>(sPvKeep + t * 2 + (j & 1)) != 0;
        if (issue) {
          if (j == 0) issue_pv(s, true, 0, L::BN / 32);
          else issue_pv(s, false, 0, L::BN / 32);
        }
        if (!wait(bar_p_full + t, j & 1)) break;
        tc_fence_after();
        if (issue) issue_pv(s, false, L::BN / 32, L::BN / 16);
        mma_commit_warp(bar_o_done + t);
        if (lane == 0) stamp((6 + 2 * t) * n_kv_total + j);
        mma_commit_warp(bar_kv_empty + s);  // this tile's products reading stage s are issued
      }
      // all MMAs issued by this warp must finish before TMEM is released
      mma_commit_warp(bar_drain + t);
      mbar_drain(bar_drain + t, 0);
    }
    }
  } else {
    reg_alloc<216>();
    // ================================================================ softmax warpgroups
    const int t = (warp - 4) >> 2;
    const int quad = warp & 3;  // TMEM lane quadrant this warp may access
    const int r = quad * 32 + lane;
    if (t < n_tiles) {
      const int q_tile = tile0 + t;
      const int q_row = q_tile * L::BM + r;
      const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
      const uint32_t tS = tmem + lane_addr + L::s_col(t);
      const uint32_t tO = tmem + lane_addr + L::o_col(t);
      const uint32_t tP = tmem + lane_addr + L::p_col(t);
      // rows past N (a partial last tile) compute on zeros and are never stored
      const float sq_r = PER_TOKEN ? (q_row < N ? __ldg(sq + row_base + q_row) : 0.f) : __ldg(sq + bh * n_qtiles + q_tile);
      const float a_r = sq_r * sm_scale_log2;  // log2-unit value of one integer step, before sk
      const int n_kgroups = (N + 63) / 64;  // per-block key scales per head
      const float* sk_head = sk + static_cast<size_t>(bh) * (PER_TOKEN ? N : n_kgroups);

      // Offset quantum: the exponent offset m_use is kept a multiple of qm, a power of two at
      // least 4 ulps of kMagic * c for every key scale c of this row.  Then kMagic * c' + m_use
      // is exact in fp32 and fma(f, c', -(kMagic * c' + m_use)) = fl(S * c' - m_use): the
      // integer-to-float conversion by the magic-number add costs no extra rounding.
      float qm = 0x1p-126f;
      if constexpr (!PER_TOKEN) {
        // largest key scale of the head: the warp's lanes split the key scales, then reduce
        float skmax = 0.f;
        for (int i = lane; i < n_kgroups; i += 32) skmax = fmaxf(skmax, __ldg(sk_head + i));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) skmax = fmaxf(skmax, __shfl_xor_sync(0xffffffffu, skmax, off));
        qm = offset_quantum(kMagicF * trim_scale(a_r * skmax));
      }

      float m_use = 0.f;  // exponent offset (log2 units) applied to this row so far
      float m_run = -INFINITY;  // block-sparse variant: the row's largest score so far (log2 units)
      float2 lsum[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
      bool ok = true;
      // Block-sparse variant: the four warps of the group meet at one named barrier per key tile
      // (the stage-2 vote).  A warp whose bounded wait gave up still takes that barrier once for
      // the step it leaves in, with bit 1 in the vote, and the whole group leaves there: no warp
      // is left waiting at a barrier that the others never reach.
      int* vote = sSkipVote + t * 3;
      auto leave_vote = [&](int jj) {
        if constexpr (SPARSE) {
          if (jj < n_iter[t]) {
            if (r == 0) vote[(jj + 1) % 3] = 0;
            if (lane == 0) atomicOr(vote + jj % 3, 2);
            group_bar(1 + t);
          }
        }
      };
      for (int j = 0; j < n_iter[t]; ++j) {
        if (!__all_sync(0xffffffffu, mbar_wait(bar_s_full + t, j & 1, abort_flag))) { leave_vote(j); ok = false; break; }
        tc_fence_after();
        if (r == 0) stamp((3 * t) * n_kv_total + j);
        // masked keys: past the diagonal (causal) and past N (a partial last key tile); keys
        // c > cmax of this tile are left out of the maximum and get P~ = 0.  Such a tile is
        // always the last key tile of its query tile.
        const int kt = key_tile(j);
        const int kvalid = N - kt * L::BN;
        const bool diag = (CAUSAL && kt == q_tile) || (RAGGED && kvalid < L::BN);
        uint32_t x[128];
        tmem_ld64_sync(tS + 0, *reinterpret_cast<uint32_t(*)[64]>(x + 0));
        tmem_ld64_sync(tS + 64, *reinterpret_cast<uint32_t(*)[64]>(x + 64));
        if (!diag) {  // S_t is in registers: the next Q.K^T may overwrite it (masked tiles re-read it)
          tc_fence_before();
          mbar_arrive(bar_s_free + t);
        }
        const int cmax = min((CAUSAL && kt == q_tile) ? r : L::BN - 1, kvalid - 1);
        const int s = j % STAGES;
        float mx;            // row maximum of the dequantized scores (log2 units)
        float cb0 = 0.f, cb1 = 0.f, nb0 = 0.f, nb1 = 0.f;
        const float* skj = sSK + s * L::BN;
        if constexpr (PER_TOKEN) {
          // f = kMagic + S exactly (|S| < 2^22), as float bits; masked keys -inf
          if (diag) {
#pragma unroll
            for (int c = 0; c < 128; ++c) x[c] = c > cmax ? 0xFF800000u : x[c] + kMagicBits;
          } else {
#pragma unroll
            for (int c = 0; c < 128; ++c) x[c] += kMagicBits;
          }
          if (!__all_sync(0xffffffffu, mbar_wait(bar_k_full + s, (j / STAGES) & 1, abort_flag))) { leave_vote(j); ok = false; break; }
          // max of S * sk over the row's keys (masked: -inf), then times a_r >= 0
          float m3 = -INFINITY;
#pragma unroll
          for (int c = 0; c < 128; c += 2) {
            const float2 v = __fmul2_rn(__fadd2_rn(make_float2(__uint_as_float(x[c]), __uint_as_float(x[c + 1])),
                                                   make_float2(-kMagicF, -kMagicF)),
                                        *reinterpret_cast<const float2*>(skj + c));
            m3 = fmaxf(m3, fmaxf(v.x, v.y));
          }
          mx = m3 == -INFINITY ? -INFINITY : a_r * m3;
        } else {
          // integer maxima of the two 64-key halves (one key scale each); masked keys INT_MIN
          cb0 = trim_scale(a_r * __ldg(sk_head + 2 * kt));
          cb1 = 2 * kt + 1 < n_kgroups ? trim_scale(a_r * __ldg(sk_head + 2 * kt + 1)) : 0.f;
          if (diag) {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c > cmax) x[c] = 0x80000000u;
          }
          const int im0 = imax64(x);
          if (diag) {
#pragma unroll
            for (int c = 64; c < 128; ++c)
              if (c > cmax) x[c] = 0x80000000u;
          }
          const int im1 = imax64(x + 64);
          const float m0 = im0 == INT_MIN ? -INFINITY : cb0 * static_cast<float>(im0);
          const float m1 = im1 == INT_MIN ? -INFINITY : cb1 * static_cast<float>(im1);
          mx = fmaxf(m0, m1);
        }

        // ---- stage 2 (block-sparse variant): the group keeps key tile j when one of its rows
        // below N scores within skip_lambda of its running maximum (always the first tile, whose
        // running maximum is -inf).  Vote slots rotate over three steps: slot (j+1) % 3 was last
        // read at step j-2, before every thread reached step j-1's barrier.
        bool keep_tile = true;
        if constexpr (SPARSE) {
          const bool row_keeps = q_row < N && !(mx < m_run - skip_lambda);
          if (r == 0) vote[(j + 1) % 3] = 0;
          if (__any_sync(0xffffffffu, row_keeps) && lane == 0) atomicOr(vote + j % 3, 1);
          group_bar(1 + t);
          const int v = *reinterpret_cast<volatile int*>(vote + j % 3);
          if (v & 2) { ok = false; break; }  // a warp of the group gave up waiting
          keep_tile = (v & 1) != 0;
          if (keep_tile && q_row < N) m_run = fmaxf(m_run, mx);
        }

        // ---- rescale only when the maximum grew by more than 2^8 (bounds P~ by 256)
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m_use = round_up_to(mx, qm);
        } else if (keep_tile && mx > m_use + 8.f) {
          const float m_new = round_up_to(mx, qm);
          alpha = fast_exp2(m_use - m_new);
          m_use = m_new;
          rescale = true;
        }
        // P.V(j-1) must be complete before O is rescaled and before P~(j) overwrites P~(j-1)
        if (j > 0) {
          if (!__all_sync(0xffffffffu, mbar_wait(bar_o_done + t, (j - 1) & 1, abort_flag))) { leave_vote(j + 1); ok = false; break; }
          tc_fence_after();
        }
        // the P.V warp read this slot at step j-2, before P.V(j-1) (complete above) was issued;
        // the flag is published by this thread's arrival on bar_p_lo below
        if (SPARSE && r == 0) sPvKeep[t * 2 + (j & 1)] = keep_tile ? 1 : 0;
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int i = 0; i < 4; ++i) lsum[i] = __fmul2_rn(lsum[i], make_float2(alpha, alpha));
#pragma unroll
          for (int cb = 0; cb < D; cb += 32) {
            uint32_t ov[32];
            tmem_ld32_sync(tO + cb, ov);
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st32(tO + cb, ov);
          }
        }
        if constexpr (!PER_TOKEN) {
          nb0 = -fmaf(kMagicF, cb0, m_use);  // exact: see offset_quantum above
          nb1 = -fmaf(kMagicF, cb1, m_use);
        }
        if (r == 0) stamp((3 * t + 1) * n_kv_total + j);

        // ---- P~ = exp2(s - m_use) in fp16; the row sum takes the unrounded values.  Tiles that
        // mask keys take exp_pass_masked below instead.
        auto exp_pass = [&]() {
#pragma unroll
        for (int cb = 0; cb < 128; cb += 32) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const int c = cb + i;
            float2 tt;
            if constexpr (PER_TOKEN) {
              // fl(fl(S * sk) * a_r - m_use)
              const float2 v = __fmul2_rn(__fadd2_rn(make_float2(__uint_as_float(x[c]), __uint_as_float(x[c + 1])),
                                                     make_float2(-kMagicF, -kMagicF)),
                                          *reinterpret_cast<const float2*>(skj + c));
              tt = __ffma2_rn(v, make_float2(a_r, a_r), make_float2(-m_use, -m_use));
            } else {
              const float cs = c < 64 ? cb0 : cb1;
              const float nb = c < 64 ? nb0 : nb1;
              // kMagic + S as float (exact), then one rounding: fl(S * c' - m_use)
              tt = __ffma2_rn(make_float2(__uint_as_float(x[c] + kMagicBits), __uint_as_float(x[c + 1] + kMagicBits)),
                              make_float2(cs, cs), make_float2(nb, nb));
            }
            const float2 p = make_float2(fast_exp2(tt.x), fast_exp2(tt.y));
            lsum[(i >> 1) & 3] = __fadd2_rn(lsum[(i >> 1) & 3], p);
            pk[i >> 1] = pack_half2(p.x, p.y);
          }
          tmem_st16(tP + (cb >> 1), pk);
          if (cb == 32) {  // keys 0..63 done: let their P.V start
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p_lo + t);
          }
        }
        };
        // ---- the same for a tile with masked keys (c > cmax: the causal diagonal, a partial last
        // tile), at most one per row: a rolled loop over 8-key steps that re-reads S from TMEM
        // 8 columns at a time, so that this rare case adds little code next to the unrolled pass
        auto exp_pass_masked = [&]() {
#pragma unroll 1
          for (int c8 = 0; c8 < 16; ++c8) {
            uint32_t y[8];
            tmem_ld8_sync(tS + 8 * c8, y);
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
              const int c = 8 * c8 + i;
              float2 tt;
              if constexpr (PER_TOKEN) {
                const float2 v = __fmul2_rn(make_float2(static_cast<float>(static_cast<int>(y[i])), static_cast<float>(static_cast<int>(y[i + 1]))),
                                            *reinterpret_cast<const float2*>(skj + c));
                tt = __ffma2_rn(v, make_float2(a_r, a_r), make_float2(-m_use, -m_use));
              } else {
                const float cs = c < 64 ? cb0 : cb1;
                const float nb = c < 64 ? nb0 : nb1;
                tt = __ffma2_rn(make_float2(__uint_as_float(y[i] + kMagicBits), __uint_as_float(y[i + 1] + kMagicBits)),
                                make_float2(cs, cs), make_float2(nb, nb));
              }
              const float2 p = make_float2(c > cmax ? 0.f : fast_exp2(tt.x), c + 1 > cmax ? 0.f : fast_exp2(tt.y));
              lsum[(i >> 1) & 3] = __fadd2_rn(lsum[(i >> 1) & 3], p);
              pk[i >> 1] = pack_half2(p.x, p.y);
            }
            tmem_st4(tP + 4 * c8, pk);
            if (c8 == 7) {  // keys 0..63 done: let their P.V start
              tmem_wait_st();
              tc_fence_before();
              mbar_arrive(bar_p_lo + t);
            }
          }
        };
        if (!keep_tile) {
          // stage 2 dropped the tile: no P~, and the P.V warp issues nothing for it
          if (diag) {
            tc_fence_before();
            mbar_arrive(bar_s_free + t);
          }
          mbar_arrive(bar_p_lo + t);
        } else if (diag) {
          exp_pass_masked();
          tc_fence_before();
          mbar_arrive(bar_s_free + t);  // its re-reads of S_t are done
        } else {
          exp_pass();
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_p_full + t);
        if (r == 0) stamp((3 * t + 2) * n_kv_total + j);
      }

      // ---- epilogue: O / l -> fp16 -> global
      if (ok && __all_sync(0xffffffffu, mbar_wait(bar_o_done + t, (n_iter[t] - 1) & 1, abort_flag))) {
        tc_fence_after();
        const float2 l2 = __fadd2_rn(__fadd2_rn(lsum[0], lsum[1]), __fadd2_rn(lsum[2], lsum[3]));
        const float inv_l = 1.f / (l2.x + l2.y);
        __half* orow = o + (static_cast<size_t>(row_base) + q_row) * D;
#pragma unroll
        for (int cb = 0; cb < D; cb += 32) {
          uint32_t ov[32];
          tmem_ld32_sync(tO + cb, ov);
          uint32_t hv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            hv[i] = pack_half2(__uint_as_float(ov[2 * i]) * inv_l, __uint_as_float(ov[2 * i + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + cb);
          if (q_row < N) {
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
          }
        }
      }
    }
  }

  // roles diverge inside warps (single-lane producers and stores): the thread-counting barrier
  // holds the TMEM release until every thread of the CTA is done
  tc_fence_before();
  if constexpr (TRACE) {  // also checks that the barrier held every thread
    const long long t_end = cta_end_checked(arrived, threadIdx.x == 0);
    if (trace_row && threadIdx.x == 0) trace_row[1] = t_end;
  } else {
    cta_sync();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

#include "attn_v3.cuh"
#include "attn_fp4.cuh"

// ---------------------------------------------------------------- debug: INT32 S = q8 k8^T
// One CTA per (128-row query tile, head), all along grid x.  Thread 0 issues the TMA loads and the same
// kind::i8 MMA as the fused kernel; warps 4-7 copy S from TMEM to global memory.
template <int D>
__global__ void __launch_bounds__(256, 1)
    sage_qk_debug_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         int32_t* __restrict__ s_out, int N) {
  constexpr int BM = 128, BN = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + BM * D;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BM * D + BN * D);
  uint64_t* bar_q = bars;
  uint64_t* bar_k = bars + 1;
  uint64_t* bar_s = bars + 2;
  uint64_t* bar_free = bars + 3;
  uint64_t* bar_drain = bars + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 5) + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = N / BM;  // grid x = B*H heads x n_qt query tiles (no 65535 cap on heads)
  const int q_tile = static_cast<int>(blockIdx.x) % n_qt, bh = static_cast<int>(blockIdx.x) / n_qt;
  const int row_base = bh * N;
  const int n_kv = N / BN;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_k, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_free, 128);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync();  // lane 0 of warp 0 initialised the barriers alone
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      constexpr uint32_t IDESC = make_idesc(2, 1, 1, 0, 0, 128, BN);
      constexpr SwizzleMode SWZ = D == 128 ? kSwizzle128B : kSwizzle64B;
      constexpr uint32_t SBO = D == 128 ? 1024 : 512;
      mbar_arrive_expect_tx(bar_q, BM * D);
      tma_load_2d(sQ, &tm_q, bar_q, 0, row_base + q_tile * BM);
      bool ok = mbar_wait(bar_q, 0, abort_flag);
      int k_loads = 0;
      for (int j = 0; ok && j < n_kv; ++j) {
        if (j > 0 && !mbar_wait(bar_free, (j - 1) & 1, abort_flag)) break;  // S and K buffer free
        mbar_arrive_expect_tx(bar_k, BN * D);
        tma_load_2d(sK, &tm_k, bar_k, 0, row_base + j * BN);
        ++k_loads;
        if (!mbar_wait(bar_k, j & 1, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
          const uint64_t a = make_smem_desc(smem_u32(sQ) + kk * 32, 16, SBO, SWZ);
          const uint64_t b = make_smem_desc(smem_u32(sK) + kk * 32, 16, SBO, SWZ);
          mma_i8_ss(tmem, a, b, IDESC, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_s);
      }
      mma_commit(bar_drain);
      mbar_drain(bar_drain, 0);
      if (k_loads > 0) mbar_drain(bar_k, (k_loads - 1) & 1);
    }
  } else if (warp >= 4) {
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t tS = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    int32_t* srow = s_out + (static_cast<size_t>(row_base) + q_tile * BM + r) * N;
    for (int j = 0; j < n_kv; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar_s, j & 1, abort_flag))) break;
      tc_fence_after();
#pragma unroll
      for (int cb = 0; cb < BN; cb += 32) {
        uint32_t v[32];
        tmem_ld32_sync(tS + cb, v);
        uint4* dst = reinterpret_cast<uint4*>(srow + j * BN + cb);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
      tc_fence_before();
      mbar_arrive(bar_free);
    }
  }
  // roles diverge inside warps (single-lane producers and stores): the thread-counting barrier
  // holds the TMEM release until every thread of the CTA is done
  tc_fence_before();
  cta_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ---------------------------------------------------------------- launchers
template <int D, bool CAUSAL, bool PER_TOKEN, bool TRACE = false, bool RAGGED = false, bool SPARSE = false>
static cudaError_t launch_attn_t(const AttnArgs& a, cudaStream_t st) {
  using L = AttnLayout<D>;
  auto kern = sage_attn_kernel<D, CAUSAL, PER_TOKEN, TRACE, RAGGED, SPARSE>;
  static bool configured = false;  // attribute set once per instantiation (idempotent)
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int n_qtiles = (a.N + L::BM - 1) / L::BM;
  const int n_pairs = (n_qtiles + 1) / 2;
  dim3 grid(static_cast<unsigned>(n_pairs * a.BH));
  kern<<<grid, L::THREADS, L::SMEM, st>>>(*a.tm_q, *a.tm_k, *a.tm_v, a.sq, a.sk, a.o, a.BH, a.N, a.sm_scale_log2,
                                          a.trace, a.trace_ctas, a.kv_count, a.kv_index, a.skip_lambda);
  return cudaGetLastError();
}

template <bool CAUSAL, bool PER_TOKEN, bool TRACE = false, bool RAGGED = false, bool FP8 = false, bool SPARSE = false>
static cudaError_t launch_attn_v3(const AttnArgs& a, cudaStream_t st) {
  using L = V3LayoutT<FP8>;
  auto kern = sage_attn_v3_kernel<CAUSAL, PER_TOKEN, TRACE, RAGGED, FP8, SPARSE>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int n_pairs = ((a.N + L::BM - 1) / L::BM + 1) / 2;
  dim3 grid(static_cast<unsigned>(n_pairs * a.BH));
  kern<<<grid, L::THREADS, L::SMEM, st>>>(*a.tm_q, *a.tm_k, *a.tm_v, *a.tm_o, a.sq, a.sk, a.BH, a.N, a.sm_scale_log2,
                                          a.trace, a.trace_ctas, a.sv, a.vm, a.kv_count, a.kv_index, a.skip_lambda);
  return cudaGetLastError();
}

// RAGGED instantiations carry the key masking of a partial last key tile; whole-tile problems
// (N a multiple of 128) use the others, whose non-causal forms have no masking code at all.
template <int D, bool RAGGED, bool SPARSE = false>
static cudaError_t launch_attn_d(const AttnArgs& a, cudaStream_t st) {
  if (a.causal)
    return a.per_token ? launch_attn_t<D, true, true, false, RAGGED, SPARSE>(a, st)
                       : launch_attn_t<D, true, false, false, RAGGED, SPARSE>(a, st);
  return a.per_token ? launch_attn_t<D, false, true, false, RAGGED, SPARSE>(a, st)
                     : launch_attn_t<D, false, false, false, RAGGED, SPARSE>(a, st);
}

template <bool RAGGED, bool FP8 = false, bool SPARSE = false>
static cudaError_t launch_attn_128(const AttnArgs& a, cudaStream_t st) {
  if (a.causal)
    return a.per_token ? launch_attn_v3<true, true, false, RAGGED, FP8, SPARSE>(a, st)
                       : launch_attn_v3<true, false, false, RAGGED, FP8, SPARSE>(a, st);
  return a.per_token ? launch_attn_v3<false, true, false, RAGGED, FP8, SPARSE>(a, st)
                     : launch_attn_v3<false, false, false, RAGGED, FP8, SPARSE>(a, st);
}

cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st) {
  const bool ragged = a.N % 128 != 0;
  if (a.fp8) {  // the FP8 P.V variant: head dimension 128, untraced
    if (a.D != 128 || a.trace || a.kv_count) return cudaErrorNotSupported;
    return ragged ? launch_attn_128<true, true>(a, st) : launch_attn_128<false, true>(a, st);
  }
  if (a.kv_count) {  // the block-sparse variant: untraced, up to 512 key tiles
    static_assert(AttnLayout<64>::MAX_LIST == V3Layout::MAX_LIST, "one list bound for both head dimensions");
    if (a.trace || (a.N + 127) / 128 > V3Layout::MAX_LIST) return cudaErrorNotSupported;
    if (a.D == 128) return ragged ? launch_attn_128<true, false, true>(a, st) : launch_attn_128<false, false, true>(a, st);
    return ragged ? launch_attn_d<64, true, true>(a, st) : launch_attn_d<64, false, true>(a, st);
  }
  if (a.trace) {  // traced builds exist for per-block granularity and whole tiles only
    if (a.per_token || ragged) return cudaErrorNotSupported;
    if (a.D == 128) return a.causal ? launch_attn_v3<true, false, true>(a, st) : launch_attn_v3<false, false, true>(a, st);
    return a.causal ? launch_attn_t<64, true, false, true>(a, st) : launch_attn_t<64, false, false, true>(a, st);
  }
  if (a.D == 128) return ragged ? launch_attn_128<true>(a, st) : launch_attn_128<false>(a, st);
  return ragged ? launch_attn_d<64, true>(a, st) : launch_attn_d<64, false>(a, st);
}

template <int D, bool CAUSAL, bool RAGGED>
static cudaError_t launch_attn_fp4_t(const Fp4Args& a, cudaStream_t st) {
  using L = Fp4Layout<D>;
  auto kern = sage_attn_fp4_kernel<D, CAUSAL, RAGGED>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const unsigned grid = static_cast<unsigned>((a.N + 127) / 128) * static_cast<unsigned>(a.BH);
  kern<<<grid, L::THREADS, L::SMEM, st>>>(*a.tm_q, *a.tm_k, *a.tm_v, a.sfq, a.sfk, a.sfv, a.gq, a.gk, a.gv, a.vm, a.o,
                                          a.N, a.sm_scale_log2);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_attn_fp4_d(const Fp4Args& a, cudaStream_t st) {
  const bool ragged = a.N % 128 != 0;
  if (a.causal) return ragged ? launch_attn_fp4_t<D, true, true>(a, st) : launch_attn_fp4_t<D, true, false>(a, st);
  return ragged ? launch_attn_fp4_t<D, false, true>(a, st) : launch_attn_fp4_t<D, false, false>(a, st);
}

cudaError_t launch_attn_fp4(const Fp4Args& a, cudaStream_t st) {
  return a.D == 128 ? launch_attn_fp4_d<128>(a, st) : launch_attn_fp4_d<64>(a, st);
}

template <int D>
static cudaError_t launch_qk_debug_d(const CUtensorMap& tq, const CUtensorMap& tk, int32_t* s, int BH, int N,
                                     cudaStream_t st) {
  // 4 CTAs per SM at most (4 x 128 TMEM columns): ask for 56 KB of shared memory each
  constexpr int SMEM = 56 * 1024;
  auto kern = sage_qk_debug_kernel<D>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  dim3 grid(static_cast<unsigned>(N / 128) * static_cast<unsigned>(BH));
  kern<<<grid, 256, SMEM, st>>>(tq, tk, s, N);
  return cudaGetLastError();
}

cudaError_t launch_qk_debug(const CUtensorMap& tq, const CUtensorMap& tk, int32_t* s, int BH, int N, int D,
                            cudaStream_t st) {
  return D == 128 ? launch_qk_debug_d<128>(tq, tk, s, BH, N, st) : launch_qk_debug_d<64>(tq, tk, s, BH, N, st);
}

// Failure detection check: one warp initialises an mbarrier that nothing ever arrives on and
// waits on its first phase with the bounded wait every pipeline role uses.  The wait gives up
// after kWaitLimitCycles, records kDevTimeoutBarrier in the status word and the kernel returns
// normally, so the context stays usable.  out[0] = 1 if the wait completed (it cannot), 0 if
// it gave up.
__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(int* __restrict__ out) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  const bool ok = mbar_wait(&bar, 0, &abort_flag);
  if (threadIdx.x == 0) out[0] = ok ? 1 : 0;
}

cudaError_t launch_wait_timeout(int* out, cudaStream_t st) {
  wait_timeout_kernel<<<1, 32, 0, st>>>(out);
  return cudaGetLastError();
}

int read_and_clear_device_error(cudaStream_t st, cudaError_t* err) {
  *err = cudaStreamSynchronize(st);
  if (*err != cudaSuccess) return -1;
  int h = 0;
  *err = cudaMemcpyFromSymbol(&h, g_device_error, sizeof(int));
  if (*err != cudaSuccess) return -1;
  const int zero = 0;
  *err = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
  if (*err != cudaSuccess) return -1;
  return h;
}

}  // namespace sage
