// attn_v3.cuh -- the fused attention kernel for head dimension 128, with P.V computed
// transposed: O^T[d, q] += V^T[d, keys] . P~^T[keys, q], one product stream per query tile
// (M = 128 = d, N = 128 queries, K = 16 keys), each issued by its own warp.
//
// Why this shape: one warp issuing tcgen05.mma gets about one instruction per 110-140 cycles
// whatever N is (up to 256), so at N = 128 a single issuing warp keeps the tensor core about half
// busy; several issuing warps overlap.  Here three warps issue: Q.K^T for both query tiles, and
// one P.V stream per tile.  Transposed, P~ is the B operand and lives in shared memory in the
// 128-byte-swizzled K-major layout the tensor core reads, and O^T has the head dimension on the
// TMEM lanes, so a separate correction warpgroup (thread = head dimension) rescales the O^T
// columns of the queries whose softmax offset moved, off the softmax warps' path.
//
// Included by attn_kernels.cu inside namespace sage (one translation unit with the PTX helpers).
#pragma once

// FP8: the P.V variant with E4M3 P~ and V (kind::f8f6f4): one 128-byte TMA box per V tile and
// one byte per P~ element; the P~ region keeps its fp16 size because the epilogue stages O there.
template <bool FP8>
struct V3LayoutT {
  static constexpr int D = 128;
  static constexpr int BM = 128, BN = 128;
  static constexpr int SK = 3;                // K stages
  static constexpr int SV = 2;                // V stages
  static constexpr int Q_BYTES = BM * D;      // int8 tile
  static constexpr int K_BYTES = BN * D;      // int8 tile
  static constexpr int V_BOX = BN * 128;      // one 64-column fp16 box (128-byte rows)
  static constexpr int V_BYTES = FP8 ? BN * D : BN * D * 2;  // fp16: two boxes; e4m3: one
  static constexpr int P_ATOM = 256 * 128;    // 64 keys x 256 query rows of fp16 P~
  static constexpr int P_BYTES = 2 * P_ATOM;  // 128 keys
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + SK * K_BYTES;
  static constexpr int OFF_P = OFF_V + SV * V_BYTES;
  static constexpr int OFF_ALPHA = OFF_P + P_BYTES;       // [2][256] fp32 rescale factors
  static constexpr int OFF_L = OFF_ALPHA + 2 * 256 * 4;   // [256] fp32 row sums
  static constexpr int OFF_FLAG = OFF_L + 256 * 4;        // [2][3] int rescale votes
  static constexpr int OFF_SKS = OFF_FLAG + 32;           // [2 tiles][2][128] fp32 per-token key scales
  static constexpr int OFF_BAR = OFF_SKS + 2 * 2 * 128 * 4;
  // q, k_full/empty, v_full/empty, then per tile: s_full, s_free, p_lo, p_hi, o_done, 2 votes,
  // corr_done, drain, key scales staged, plus the Q.K^T warp's drain
  static constexpr int NUM_BARS = 1 + 2 * SK + 2 * SV + 10 * 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  // block-sparse variant: the CTA's key-tile list (int16, up to 512 tiles) and the skip votes
  static constexpr int MAX_LIST = 512;
  static constexpr int OFF_LIST = OFF_MISC + 16;
  static constexpr int OFF_SKIP = OFF_LIST + MAX_LIST * 2;  // [2 tiles][3] group votes, [2 tiles][2] P.V flags
  static constexpr int SMEM = OFF_SKIP + 64 + 1024;
  static constexpr int THREADS = 512;
};
using V3Layout = V3LayoutT<false>;
static_assert(V3LayoutT<false>::SMEM <= 227 * 1024 && V3LayoutT<true>::SMEM <= 227 * 1024, "shared memory budget");

// Exact 2^k for an integer k <= 0 (0 below the normal range): the FP8 variant's offsets are
// integers, so its rescale factors are powers of two and rescaling O and l is exact.
__device__ __forceinline__ float exp2_int(float k) {
  const int e = 127 + static_cast<int>(k);
  return e > 0 ? __int_as_float(e << 23) : 0.f;
}

// Four fp32 values to E4M3 (round to nearest even, saturating), packed little-endian.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;  // cvt packs its first source into the upper byte
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

__device__ __forceinline__ void st_shared_v2(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

// exp2 on the FMA pipe for a pair of arguments (Cody-Waite style range reduction plus a
// polynomial), to take part of the exp2 work off the MUFU unit:
//   t -> max(t, -126); n = round_to_nearest(t) via the 1.5 * 2^23 add; f = t - n in [-1/2, 1/2];
//   2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 with coefficients fitted here to the minimax relative error on
//   [-1/2, 1/2] (max relative error 7.5e-5, below half an fp16 ulp); 2^n by adding n to the
//   exponent field (n << 23, taken from the low bits of the magic sum).
__device__ __forceinline__ float2 exp2_poly2(float2 t) {
  constexpr float c0 = 0.9999281167984009f, c1 = 0.6932609677314758f, c2 = 0.2426108568906784f,
                  c3 = 0.055171459913253784f;
  t.x = fmaxf(t.x, -126.f);
  t.y = fmaxf(t.y, -126.f);
  const float2 y = __fadd2_rn(t, make_float2(kMagicF, kMagicF));
  const float2 n = __fadd2_rn(y, make_float2(-kMagicF, -kMagicF));
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), t);
  float2 p = __ffma2_rn(f, make_float2(c3, c3), make_float2(c2, c2));
  p = __ffma2_rn(p, f, make_float2(c1, c1));
  p = __ffma2_rn(p, f, make_float2(c0, c0));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(y.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(y.y) << 23)));
}

// Barrier of one 128-thread warpgroup: named barrier `id` (1, 2, ...; 0 is the CTA barrier),
// counted per thread, so warps may arrive diverged.
__device__ __forceinline__ void group_sync(int id) { asm volatile("barrier.sync %0, 128;" ::"r"(id) : "memory"); }

// CTA-wide vote helpers -----------------------------------------------------------------
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

__device__ __forceinline__ void bulk_commit_and_wait_read() {
  asm volatile("cp.async.bulk.commit_group;\n\tcp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Warp roles (16 warps):
//   0   TMA producer: Q tiles once, then V tiles through their ring
//   1 / 3  MMA warps: O^T_t += V^T . P~_t^T for query tile 0 / 1 (warp 1 also allocates TMEM)
//   2   MMA warp: S_t = Q_t . K^T for both query tiles; also loads the K ring (TMA)
//   4-7 / 8-11  softmax of query tile 0 / 1 (thread = query row = TMEM lane of S), then that
//               tile's epilogue (thread = head dimension = TMEM lane of O^T): normalizes by 1/l,
//               stages O in shared memory and TMA-stores it, both tiles in parallel
//   12-15       correction (thread = head dimension d = TMEM lane of O^T): rescales the O^T
//               columns of rows whose offset moved, between two P.V products
//
// FP8 = true is the P.V variant of the SageAttention2 abstract ((P~, V) in FP8, P~V accumulated in
// an FP32 buffer -- here the tensor memory accumulator): V arrives as E4M3 codes with per-channel
// scales sv and channel means vm (vm may be null), P~ is rounded to E4M3 and P.V runs as
// tcgen05 kind::f8f6f4 with fp32 accumulation.  The row offsets are integers (quantum >= 1) and
// P~ = 2^(s - m_use + 8), so P~ is rounded on the E4M3 grid of a power-of-two scaling of
// exp(s - max s), as the oracle rounds it, and the offset moves as soon as the row maximum passes
// it by half a unit (P~ <= 2^8.5 < 448); the epilogue applies sv and adds vm.
//
// SPARSE = true is the block-sparse variant of the SpargeAttn abstract (a predicted map skips
// products; a softmax-aware filter skips more).  kv_count[bh * n_pairs + pair] and the ascending
// key-tile list kv_index[(bh * n_pairs + pair) * ceil(N/128) + i] say which key tiles the CTA
// visits (stage 1); every role walks the list instead of 0 .. n_kv-1.  Stage 2: a softmax group
// drops key tile j of its query tile when, for each of its rows below N, the tile's largest score
// lies more than skip_lambda (log2 units) under the row's running maximum; the group agrees
// through a vote and a named barrier, skips its exp2 pass, and its P.V warp issues nothing for
// that tile (the tile adds to neither O nor l).
template <bool CAUSAL, bool PER_TOKEN, bool TRACE, bool RAGGED, bool FP8 = false, bool SPARSE = false>
__global__ void __launch_bounds__(512, 1)
    sage_attn_v3_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                        const float* __restrict__ sq, const float* __restrict__ sk, int BH, int N,
                        float sm_scale_log2, long long* __restrict__ trace, int trace_ctas,
                        const float* __restrict__ sv = nullptr, const float* __restrict__ vm = nullptr,
                        const int* __restrict__ kv_count = nullptr, const int16_t* __restrict__ kv_index = nullptr,
                        float skip_lambda = 0.f) {
  using L = V3LayoutT<FP8>;
  constexpr int D = L::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;
  uint8_t* sP = smem + L::OFF_P;
  float* sAlpha = reinterpret_cast<float*>(smem + L::OFF_ALPHA);  // [2][256] per-query rescale factor
  float* sL = reinterpret_cast<float*>(smem + L::OFF_L);          // [256] 1 / row sum
  int* sFlag = reinterpret_cast<int*>(smem + L::OFF_FLAG);        // [2 tiles][3 slots] rescale votes
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* bar_q = bars;
  uint64_t* bar_k_full = bar_q + 1;
  uint64_t* bar_k_empty = bar_k_full + L::SK;
  uint64_t* bar_v_full = bar_k_empty + L::SK;
  uint64_t* bar_v_empty = bar_v_full + L::SV;
  uint64_t* bar_s_full = bar_v_empty + L::SV;  // [2] Q.K^T of tile t done
  uint64_t* bar_s_free = bar_s_full + 2;       // [2] softmax t has read S_t
  uint64_t* bar_p_lo = bar_s_free + 2;         // [2] P~ keys 0..63 of tile t in shared memory
  uint64_t* bar_p_hi = bar_p_lo + 2;           // [2] P~ keys 64..127 of tile t in shared memory
  uint64_t* bar_o_done = bar_p_hi + 2;         // [2] a whole P.V with tile t's queries done
  uint64_t* bar_vote = bar_o_done + 2;         // [2 tiles][2] softmax t published its rescale factors
                                               // (key tile j uses bar_vote[2t + (j & 1)])
  uint64_t* bar_corr = bar_vote + 4;           // [2] O^T columns of tile t corrected
  uint64_t* bar_drain = bar_corr + 2;          // [3] MMA warps' completion at exit
  uint64_t* bar_sks = bar_drain + 3;           // [2] per-token key scales of softmax t's next key tile staged
  float* sSKs = reinterpret_cast<float*>(smem + L::OFF_SKS);  // [2 tiles][2][128] per-token key scales
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  int* arrived = reinterpret_cast<int*>(smem + L::OFF_MISC + 8);  // trace builds: threads at the final barrier

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: head-major, heavy query-tile pairs first
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
  int* sSkipVote = reinterpret_cast<int*>(smem + L::OFF_SKIP);       // [2 tiles][3]: a row keeps the tile
  int* sPvKeep = reinterpret_cast<int*>(smem + L::OFF_SKIP + 32);    // [2 tiles][2]: P.V of key tile j issued
  if constexpr (SPARSE) {
    // the list is ascending; causal lists end with the diagonal tiles, so tile 0 stops one key
    // tile before tile 1 when the list holds tile0 + 1 (only tile 1 sees it)
    // a malformed list (count or entries out of range) gives unspecified output, never an access
    // outside the tensors: both are clamped into range
    const int count = min(max(kv_count[static_cast<size_t>(bh) * n_pairs + pair], 0), min(n_kv_total, L::MAX_LIST));
    const int16_t* lst = kv_index + (static_cast<size_t>(bh) * n_pairs + pair) * n_kv_total;
    for (int i = threadIdx.x; i < count; i += L::THREADS)
      sList[i] = static_cast<int16_t>(min(max(static_cast<int>(lst[i]), 0), n_kv_total - 1));
    const int last = count > 0 ? min(max(static_cast<int>(lst[count - 1]), 0), n_kv_total - 1) : -1;
    n_iter[1] = n_tiles > 1 ? count : 0;
    n_iter[0] = (CAUSAL && n_tiles > 1 && last == tile0 + 1) ? count - 1 : count;
  }
  const int n_kv = max(n_iter[0], n_iter[1]);
  // key tile visited in step j
  auto key_tile = [&](int j) -> int {
    if constexpr (SPARSE) return sList[j];
    return j;
  };
  const int row_base = bh * N;

  long long* trace_row = nullptr;
  if constexpr (TRACE) {
    if (static_cast<int>(blockIdx.x) < trace_ctas) {
      trace_row = trace + static_cast<size_t>(blockIdx.x) * (2 + 10 * n_kv_total);
      if (threadIdx.x == 0) trace_row[0] = clock_stamp();
    }
  }
  // trace slots as documented at sage_debug_attn_trace; MMA event 0 = the P.V containing
  // tile t's queries issued, event 1 = Q.K^T of tile t issued (for key tile j + 1)
  auto stamp = [&](int slot) {
    if constexpr (TRACE) {
      if (trace_row) trace_row[2 + slot] = clock_stamp();
    }
  };

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < L::SK; ++s) {
      mbar_init(bar_k_full + s, 1);
      mbar_init(bar_k_empty + s, 1);
    }
    for (int s = 0; s < L::SV; ++s) {
      mbar_init(bar_v_full + s, 1);
      mbar_init(bar_v_empty + s, n_tiles);  // one commit from each P.V warp
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s_full + t, 1);
      mbar_init(bar_s_free + t, 128);
      mbar_init(bar_p_lo + t, 128);
      mbar_init(bar_p_hi + t, 128);
      mbar_init(bar_o_done + t, 1);
      mbar_init(bar_vote + 2 * t, 128);
      mbar_init(bar_vote + 2 * t + 1, 128);
      mbar_init(bar_corr + t, 128);
      mbar_init(bar_drain + t, 1);
    }
    mbar_init(bar_drain + 2, 1);
    mbar_init(bar_sks, 128);
    mbar_init(bar_sks + 1, 128);
    for (int i = 0; i < 6; ++i) sFlag[i] = 0;
    for (int i = 0; i < 6; ++i) sSkipVote[i] = 0;
    *abort_flag = 0;
    *arrived = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_o);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync();  // lane 0 of warp 0 initialised the barriers alone
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S_0 [0,128), S_1 [128,256), O^T [256,512) with column 256 + q for the CTA's
  // query q (tile 0: q < 128, tile 1: q >= 128); O^T lane = head dimension d.
  auto wait_warp = [&](uint64_t* bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
  };

  // Registers: launched with 128 per thread (512 x 128); the control and correction groups hand
  // part of theirs to the softmax groups: 128 x 88 + 256 x 168 + 128 x 88.  Each setmaxnreg is
  // executed by a whole warpgroup and dominates that group's code.
  if (warp < 4) {
  reg_dealloc<88>();
  if (warp == 0) {
    // ============================================================ TMA producer: Q once, then V
    // (the Q.K^T warp loads K itself, so that a V stage still in use never holds back a K load)
    if (lane == 0) {
      int v_issued[L::SV];
      for (int s = 0; s < L::SV; ++s) v_issued[s] = 0;
      mbar_arrive_expect_tx(bar_q, n_tiles * L::Q_BYTES);
      for (int t = 0; t < n_tiles; ++t)
        tma_load_3d(sQ + t * L::Q_BYTES, &tm_q, bar_q, 0, (tile0 + t) * L::BM, bh);
      for (int j = 0; j < n_kv; ++j) {
        const int key_row = key_tile(j) * L::BN;  // token row within the head
        const int sv_ = j % L::SV;
        if (j >= L::SV && !mbar_wait(bar_v_empty + sv_, (j / L::SV - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar_v_full + sv_, L::V_BYTES);
        tma_load_3d(sV + sv_ * L::V_BYTES, &tm_v, bar_v_full + sv_, 0, key_row, bh);
        if constexpr (!FP8) tma_load_3d(sV + sv_ * L::V_BYTES + L::V_BOX, &tm_v, bar_v_full + sv_, 64, key_row, bh);
        v_issued[sv_] = j / L::SV + 1;
      }
      if (*abort_flag) {  // let copies in flight land before the CTA exits
        mbar_drain(bar_q, 0);
        for (int s = 0; s < L::SV; ++s)
          if (v_issued[s] > 0) mbar_drain(bar_v_full + s, (v_issued[s] - 1) & 1);
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ============================================================ MMA: O^T_t += V^T . P~_t^T
    // Warp 1 serves query tile 0, warp 3 tile 1: each product has M = 128 (head dims),
    // N = 128 (the tile's queries), K = 16 keys, and the two tiles' streams overlap on the
    // tensor core.  The whole warp runs the loop; elect.sync lets one lane issue.
    const int t = warp == 1 ? 0 : 1;
    if (t < n_tiles) {
      // tile t's P~ rows: fp16, 128 rows of each 64-key atom; e4m3, 128 rows of 128 bytes
      const uint32_t v_base = smem_u32(sV), p_base = smem_u32(sP) + t * 128 * 128;
      constexpr uint32_t IDESC_PV = make_idesc(1 /*f32*/, 0, 0, 1 /*A = V^T MN-major*/, 0, 128, 128);
      // kind::f8f6f4: format 0 = E4M3 for A and B, A = V^T MN-major (allowed for 8-bit E4M3)
      constexpr uint32_t IDESC_PV8 = make_idesc(1 /*f32*/, 0 /*e4m3*/, 0 /*e4m3*/, 1, 0, 128, 128);
      const uint32_t d_tmem = tmem + 256 + 128 * t;
      bool ok = true;
      for (int j = 0; ok && j < n_iter[t]; ++j) {
        const int s = j % L::SV;
        if (!wait_warp(bar_v_full + s, (j / L::SV) & 1)) break;
        // rescaled O^T columns must be in place before this product accumulates into them
        if (j > 0 && !wait_warp(bar_corr + t, (j - 1) & 1)) break;
        for (int half = 0; half < 2; ++half) {
          if (!wait_warp(half == 0 ? bar_p_lo + t : bar_p_hi + t, j & 1)) { ok = false; break; }
          tc_fence_after();
          bool issue = true;  // block-sparse variant: the softmax group may have dropped key tile j
          if constexpr (SPARSE) issue = *reinterpret_cast<volatile int*>(sPvKeep + t * 2 + (j & 1)) != 0;
          if (!issue) {
          } else if constexpr (FP8) {
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
              const int kk = half * 2 + k2;  // 32 keys per MMA
              // A = V^T in E4M3: keys kk*32.. of the V tile (32 rows of 128 B: all 128 head dims)
              const uint64_t a = make_smem_desc(v_base + s * L::V_BYTES + kk * 32 * 128, L::V_BYTES, 1024, kSwizzle128B);
              // B = P~_t^T in E4M3: 32-byte step kk inside the tile's 128-byte swizzled rows
              const uint64_t b = make_smem_desc(p_base + kk * 32, 16, 1024, kSwizzle128B);
              mma_f8_ss_warp(d_tmem, a, b, IDESC_PV8, (j == 0 && kk == 0) ? 0u : 1u);
            }
          } else {
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int kk = half * 4 + k4;  // 16 keys per MMA
            // A = V^T: keys kk*16.. of the V tile (16 rows of 128 B), LBO = next 64 head dims
            const uint64_t a = make_smem_desc(v_base + s * L::V_BYTES + kk * 16 * 128, L::V_BOX, 1024, kSwizzle128B);
            // B = P~_t^T: 64-key atom `half`, 32-byte step k4 inside the 128-byte swizzled rows
            const uint64_t b = make_smem_desc(p_base + half * L::P_ATOM + k4 * 32, 16, 1024, kSwizzle128B);
            mma_f16_ss_warp(d_tmem, a, b, IDESC_PV, (j == 0 && kk == 0) ? 0u : 1u);
          }
          }
          if (half == 1) mma_commit_warp(bar_o_done + t);
        }
        if (!ok) break;
        mma_commit_warp(bar_v_empty + s);  // one of the n_tiles arrivals that free stage s
        if (lane == 0) stamp((6 + 2 * t) * n_kv_total + j);
      }
      mma_commit_warp(bar_drain + t);
      mbar_drain(bar_drain + t, 0);
    }
  } else if (warp == 2) {
    // ============================================================ MMA: S_t = Q_t . K^T, and the
    // K ring's loads: key tile jj goes to stage jj % SK once Q.K^T of the tile before it there
    // (jj - SK) is complete.
    const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK);
    constexpr uint32_t IDESC_QK = make_idesc(2 /*s32*/, 1 /*s8*/, 1 /*s8*/, 0, 0, 128, L::BN);
    int k_loaded = 0;  // key tiles 0 .. k_loaded-1 requested
    auto load_k = [&](int jj) {
      if (lane == 0) {
        mbar_arrive_expect_tx(bar_k_full + jj % L::SK, L::K_BYTES);
        tma_load_3d(sK + (jj % L::SK) * L::K_BYTES, &tm_k, bar_k_full + jj % L::SK, 0, key_tile(jj) * L::BN, bh);
      }
      k_loaded = jj + 1;
    };
    for (int jj = 0; jj < min(L::SK - 1, n_kv); ++jj) load_k(jj);
    bool ok = wait_warp(bar_q, 0);
    for (int j = 0; ok && j < n_kv; ++j) {
      const int s = j % L::SK;
      if (j + L::SK - 1 < n_kv) {  // refill the stage key tile j - 1 used
        if (j > 0 && !wait_warp(bar_k_empty + (j - 1) % L::SK, ((j - 1) / L::SK) & 1)) break;
        load_k(j + L::SK - 1);
      }
      if (!wait_warp(bar_k_full + s, (j / L::SK) & 1)) break;
      for (int t = 0; t < n_tiles; ++t) {
        if (j >= n_iter[t]) continue;
        if (j > 0 && !wait_warp(bar_s_free + t, (j - 1) & 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
          const uint64_t a = make_smem_desc(q_base + t * L::Q_BYTES + kk * 32, 16, 1024, kSwizzle128B);
          const uint64_t b = make_smem_desc(k_base + s * L::K_BYTES + kk * 32, 16, 1024, kSwizzle128B);
          mma_i8_ss_warp(tmem + 128 * t, a, b, IDESC_QK, kk > 0 ? 1u : 0u);
        }
        mma_commit_warp(bar_s_full + t);
        if (lane == 0 && j > 0) stamp((7 + 2 * t) * n_kv_total + j - 1);
      }
      if (!ok) break;
      mma_commit_warp(bar_k_empty + s);
    }
    mma_commit_warp(bar_drain + 2);
    mbar_drain(bar_drain + 2, 0);
    if (*abort_flag && lane == 0) {  // let K copies in flight land before the CTA exits
      for (int jj = max(0, k_loaded - L::SK); jj < k_loaded; ++jj) mbar_drain(bar_k_full + jj % L::SK, (jj / L::SK) & 1);
    }
  }
  } else if (warp < 12) {
    reg_alloc<168>();
    // ============================================================ softmax warpgroups
    const int t = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // query row in the tile = TMEM lane of S
    if (t < n_tiles) {
      const int q_tile = tile0 + t;
      const int q_row = q_tile * L::BM + r;
      const int qi = t * 128 + r;  // the CTA's query index (row of P~, column of O^T)
      const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
      const uint32_t tS = tmem + lane_addr + 128 * t;
      const uint32_t p_row = smem_u32(sP) + qi * 128;   // fp16 P~: this row in each 64-key atom
      const uint32_t p_row8 = smem_u32(sP) + qi * 128;  // e4m3 P~: all 128 keys in one 128-byte row
      // rows past N (a partial last tile) compute on zeros and are never stored
      const float sq_r = PER_TOKEN ? (q_row < N ? __ldg(sq + row_base + q_row) : 0.f) : __ldg(sq + bh * n_qtiles + q_tile);
      const float a_r = sq_r * sm_scale_log2;
      const int n_kgroups = (N + 63) / 64;  // per-block key scales per head
      const float* sk_head = sk + static_cast<size_t>(bh) * (PER_TOKEN ? N : n_kgroups);

      float qm = 0x1p-126f;
      if constexpr (!PER_TOKEN) {
        float skmax = 0.f;
        for (int i = lane; i < n_kgroups; i += 32) skmax = fmaxf(skmax, __ldg(sk_head + i));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) skmax = fmaxf(skmax, __shfl_xor_sync(0xffffffffu, skmax, off));
        qm = offset_quantum(kMagicF * trim_scale(a_r * skmax));
      }
      // FP8: integer offsets (a power-of-two quantum of at least 1), P~ = 2^(s - m_use + p_shift)
      // with the row maximum near 2^8; the offset moves once the maximum passes it by half a unit.
      // (A quantum above 8 -- scores so coarse that one integer step of S moves them by more than
      // 2^21 -- keeps the shift 0.)
      float p_shift = 0.f, lazy = 8.f;
      if constexpr (FP8) {
        qm = fmaxf(qm, 1.f);
        p_shift = qm <= 8.f ? 8.f : 0.f;
        lazy = qm <= 8.f ? 0.5f : 8.f;
      }

      // per-token key scales: thread r fetches scale r of a key tile (zero past N) and the group
      // publishes the 128 of them in shared memory, double-buffered, for all its rows; the fetch
      // for key tile j+1 is issued early in iteration j and stored at its end
      float* sks_t = sSKs + t * 256;
      auto key_scale = [&](int jj) -> float {
        const int key = key_tile(jj) * L::BN + r;
        return key < N ? __ldg(sk_head + key) : 0.f;
      };
      if constexpr (PER_TOKEN) {
        sks_t[r] = key_scale(0);
        mbar_arrive(bar_sks + t);
      }

      float m_use = 0.f;
      float m_run = -INFINITY;  // block-sparse variant: the row's largest score so far (log2 units)
      float2 lsum[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
      bool ok = true;
      // Block-sparse variant: the group's four warps meet at one named barrier per key tile (the
      // stage-2 vote).  A warp whose bounded wait gave up still takes that barrier once for the
      // step it leaves in, with bit 1 in the vote, and the whole group leaves there: no warp is
      // left waiting at a barrier that the others never reach.
      int* vote = sSkipVote + t * 3;
      auto leave_vote = [&](int jj) {
        if constexpr (SPARSE) {
          if (jj < n_iter[t]) {
            if (r == 0) vote[(jj + 1) % 3] = 0;
            if (lane == 0) atomicOr(vote + jj % 3, 2);
            group_sync(3 + t);
          }
        }
      };
      for (int j = 0; j < n_iter[t]; ++j) {
        if (!wait_warp(bar_s_full + t, j & 1)) { leave_vote(j); ok = false; break; }
        tc_fence_after();
        if (r == 0) stamp((3 * t) * n_kv_total + j);
        const float* skj = sks_t + (j & 1) * 128;  // per-token key scales of key tile j (shared memory)
        float sk_next = 0.f;
        if constexpr (PER_TOKEN) {
          if (j + 1 < n_iter[t]) sk_next = key_scale(j + 1);
          if (!wait_warp(bar_sks + t, j & 1)) { leave_vote(j); ok = false; break; }
        }
        // masked keys: past the diagonal (causal) and past N (a partial last key tile); keys
        // c > cmax of this tile are left out of the maximum and get P~ = 0
        const int kt = key_tile(j);
        const int kvalid = N - kt * L::BN;
        const bool diag = (CAUSAL && kt == q_tile) || (RAGGED && kvalid < L::BN);
        const int cmax = min((CAUSAL && kt == q_tile) ? r : L::BN - 1, kvalid - 1);

        // ---- row maximum of the dequantized scores (log2 units), S read in two halves
        float mx = -INFINITY;
        float cb0 = 0.f, cb1 = 0.f;
        if constexpr (!PER_TOKEN) {
          cb0 = trim_scale(a_r * __ldg(sk_head + 2 * kt));
          cb1 = 2 * kt + 1 < n_kgroups ? trim_scale(a_r * __ldg(sk_head + 2 * kt + 1)) : 0.f;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t x[64];
          tmem_ld64_sync(tS + 64 * h, x);
          if constexpr (PER_TOKEN) {
            // max of S * sk over the row's keys (a_r >= 0 multiplies it afterwards)
            float m3 = -INFINITY;
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              const int cc = 64 * h + c;
              float2 v = __fmul2_rn(make_float2(static_cast<float>(static_cast<int>(x[c])), static_cast<float>(static_cast<int>(x[c + 1]))),
                                    *reinterpret_cast<const float2*>(skj + cc));
              if (diag) {
                if (cc > cmax) v.x = -INFINITY;
                if (cc + 1 > cmax) v.y = -INFINITY;
              }
              m3 = fmaxf(m3, fmaxf(v.x, v.y));
            }
            if (m3 != -INFINITY) mx = fmaxf(mx, a_r * m3);
          } else {
            if (diag) {
#pragma unroll
              for (int c = 0; c < 64; ++c)
                if (64 * h + c > cmax) x[c] = 0x80000000u;
            }
            const int im = imax64(x);
            if (im != INT_MIN) mx = fmaxf(mx, (h ? cb1 : cb0) * static_cast<float>(im));
          }
        }

        // ---- stage 2 (block-sparse variant): the group keeps key tile j when one of its rows
        // below N scores within skip_lambda of its running maximum (always the first tile, whose
        // running maximum is -inf).  Vote slots rotate over three steps: slot (j+1) % 3 was last
        // read at step j-2, before every thread arrived at step j-1's barrier.
        bool keep_tile = true;
        if constexpr (SPARSE) {
          const bool row_keeps = q_row < N && !(mx < m_run - skip_lambda);
          if (r == 0) vote[(j + 1) % 3] = 0;
          if (__any_sync(0xffffffffu, row_keeps) && lane == 0) atomicOr(vote + j % 3, 1);
          group_sync(3 + t);
          const int v = *reinterpret_cast<volatile int*>(vote + j % 3);
          if (v & 2) { ok = false; break; }  // a warp of the group gave up waiting
          keep_tile = (v & 1) != 0;
          if (keep_tile && q_row < N) m_run = fmaxf(m_run, mx);
        }

        // ---- offset update; the correction group rescales O^T columns of rows whose offset moved
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m_use = round_up_to(mx, qm);
        } else if (keep_tile && mx > m_use + lazy) {
          const float m_new = round_up_to(mx, qm);
          alpha = FP8 ? exp2_int(m_use - m_new) : fast_exp2(m_use - m_new);
          m_use = m_new;
          rescale = true;
        }
        if (j > 0) {
          // Run-ahead bound, without a wait: this vote's barrier, factor slot and flag slot were
          // last used by key tile j-2, and the correction group has consumed that vote, because
          // the P.V of key tile j-2 (which waits for that correction) completed before this
          // group's exp2 pass of key tile j-1 began.
          sAlpha[(j & 1) * 256 + qi] = alpha;
          int* flag = sFlag + t * 3;
          if (r == 0) flag[(j + 1) % 3] = 0;  // slot of iteration j+1, last read by iteration j-2's correction
          if (__any_sync(0xffffffffu, rescale) && lane == 0) atomicOr(flag + j % 3, 1);
          mbar_arrive(bar_vote + 2 * t + (j & 1));
          if (rescale) {
#pragma unroll
            for (int i = 0; i < 4; ++i) lsum[i] = __fmul2_rn(lsum[i], make_float2(alpha, alpha));
          }
        }
        const float m_exp = m_use - p_shift;  // exponent offset of P~ (= m_use for fp16 P~)
        const float nb0 = -fmaf(kMagicF, cb0, m_exp);  // exact: see offset_quantum
        const float nb1 = -fmaf(kMagicF, cb1, m_exp);
        if (r == 0) stamp((3 * t + 1) * n_kv_total + j);

        // ---- P~ = exp2(s - m_use) in fp16, 32 keys at a time from TMEM (the next chunk's load in
        // flight while this one is computed), into shared memory.  The last chunk is waited for
        // together with the third, so that S_t is released (and the next Q.K^T can start) one
        // chunk before the end.  Tiles that mask keys take exp_pass_masked below instead.
        auto exp_pass = [&]() -> bool {
        // the tile's P~ buffer is reused: the previous P.V must have read it (one wait up front,
        // none inside the unrolled pass; measured 3-4 % faster than a wait per half)
        if (j > 0 && !wait_warp(bar_o_done + t, (j - 1) & 1)) return false;
        uint32_t xs[2][32];
        tmem_ld32_async(tS, xs[0]);
#pragma unroll
        for (int cb = 0; cb < 128; cb += 32) {
          uint32_t (&x)[32] = xs[(cb >> 5) & 1];
          if (cb < 96) tmem_wait_ld_into(x);
          if (cb < 64) {
            tmem_ld32_async(tS + cb + 32, xs[((cb >> 5) + 1) & 1]);
          } else if (cb == 64) {
            tmem_ld32_async(tS + 96, xs[1]);
            tmem_wait_ld_into(xs[1]);
            tc_fence_before();
            mbar_arrive(bar_s_free + t);  // S_t fully read: the next Q.K^T may overwrite it
          }
          uint32_t pk[16];
          float pf[FP8 ? 32 : 1];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const int c = cb + i;
            float2 tt;
            if constexpr (PER_TOKEN) {
              // fl(fl(S * sk) * a_r - m_use)
              const float2 v = __fmul2_rn(make_float2(static_cast<float>(static_cast<int>(x[i])), static_cast<float>(static_cast<int>(x[i + 1]))),
                                          *reinterpret_cast<const float2*>(skj + c));
              tt = __ffma2_rn(v, make_float2(a_r, a_r), make_float2(-m_exp, -m_exp));
            } else {
              const float cs = c < 64 ? cb0 : cb1;
              const float nb = c < 64 ? nb0 : nb1;
              // kMagic + S as float (exact), then one rounding: fl(S * c' - m_use)
              tt = __ffma2_rn(make_float2(__uint_as_float(x[i] + kMagicBits), __uint_as_float(x[i + 1] + kMagicBits)),
                              make_float2(cs, cs), make_float2(nb, nb));
            }
            // one pair in four on the FMA pipe (exp2_poly2), the rest on the MUFU unit
            const float2 p = ((i >> 1) & 3) == 3 ? exp2_poly2(tt) : make_float2(fast_exp2(tt.x), fast_exp2(tt.y));
            lsum[(i >> 1) & 3] = __fadd2_rn(lsum[(i >> 1) & 3], p);
            if constexpr (FP8) {
              pf[i] = p.x;
              pf[i + 1] = p.y;
            } else {
              pk[i >> 1] = pack_half2(p.x, p.y);
            }
          }
          if constexpr (FP8) {
            // keys cb..cb+31 = two 16-byte chunks of 16 keys in the query's 128-byte row
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              const int chunk = (cb >> 4) + g;
              const float* f = pf + 16 * g;
              st_shared_v4(p_row8 + ((chunk ^ (qi & 7)) << 4), pack_e4m3x4(f[0], f[1], f[2], f[3]),
                           pack_e4m3x4(f[4], f[5], f[6], f[7]), pack_e4m3x4(f[8], f[9], f[10], f[11]),
                           pack_e4m3x4(f[12], f[13], f[14], f[15]));
            }
          } else {
          // keys cb..cb+31 = four 16-byte chunks of 8 keys in 64-key atom cb/64
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int chunk = ((cb & 63) >> 3) + g;
            st_shared_v4(p_row + (cb >> 6) * L::P_ATOM + ((chunk ^ (qi & 7)) << 4), pk[4 * g], pk[4 * g + 1],
                         pk[4 * g + 2], pk[4 * g + 3]);
          }
          }
          if (cb == 32 || cb == 96) {
            if constexpr (SPARSE) {
              if (cb == 32 && r == 0) sPvKeep[t * 2 + (j & 1)] = 1;  // read by the P.V warp after bar_p_lo
            }
            fence_proxy_async_shared();
            mbar_arrive(cb == 32 ? bar_p_lo + t : bar_p_hi + t);
          }
        }
        return true;
        };
        // ---- the same for a tile with masked keys (c > cmax: the causal diagonal, a partial last
        // tile), at most one per row: a rolled loop over 8-key steps, S re-read 8 columns at a
        // time, so that this rare case adds little code next to the unrolled pass
        auto exp_pass_masked = [&]() -> bool {
#pragma unroll 1
          for (int c8 = 0; c8 < 16; ++c8) {
            uint32_t x[8];
            tmem_ld8_sync(tS + 8 * c8, x);
            if (c8 == 15) {
              tc_fence_before();
              mbar_arrive(bar_s_free + t);  // S_t fully read
            }
            if (j > 0 && c8 == 0) {  // the previous P.V has read the P~ buffer
              if (!wait_warp(bar_o_done + t, (j - 1) & 1)) return false;
            }
            uint32_t pk[4];
            float pf[FP8 ? 8 : 1];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
              const int c = 8 * c8 + i;
              float2 tt;
              if constexpr (PER_TOKEN) {
                const float2 v = __fmul2_rn(make_float2(static_cast<float>(static_cast<int>(x[i])), static_cast<float>(static_cast<int>(x[i + 1]))),
                                            *reinterpret_cast<const float2*>(skj + c));
                tt = __ffma2_rn(v, make_float2(a_r, a_r), make_float2(-m_exp, -m_exp));
              } else {
                const float cs = c < 64 ? cb0 : cb1;
                const float nb = c < 64 ? nb0 : nb1;
                tt = __ffma2_rn(make_float2(__uint_as_float(x[i] + kMagicBits), __uint_as_float(x[i + 1] + kMagicBits)),
                                make_float2(cs, cs), make_float2(nb, nb));
              }
              const float2 p = make_float2(c > cmax ? 0.f : fast_exp2(tt.x), c + 1 > cmax ? 0.f : fast_exp2(tt.y));
              lsum[(i >> 1) & 3] = __fadd2_rn(lsum[(i >> 1) & 3], p);
              if constexpr (FP8) {
                pf[i] = p.x;
                pf[i + 1] = p.y;
              } else {
                pk[i >> 1] = pack_half2(p.x, p.y);
              }
            }
            if constexpr (FP8) {
              // keys 8*c8 .. 8*c8+7 = half (c8 mod 2) of 16-byte chunk c8/2 of the 128-byte row
              st_shared_v2(p_row8 + (((c8 >> 1) ^ (qi & 7)) << 4) + (c8 & 1) * 8, pack_e4m3x4(pf[0], pf[1], pf[2], pf[3]),
                           pack_e4m3x4(pf[4], pf[5], pf[6], pf[7]));
            } else {
            // keys 8*c8 .. 8*c8+7 = 16-byte chunk (c8 mod 8) of 64-key atom c8/8
            st_shared_v4(p_row + (c8 >> 3) * L::P_ATOM + (((c8 & 7) ^ (qi & 7)) << 4), pk[0], pk[1], pk[2], pk[3]);
            }
            if (c8 == 7 || c8 == 15) {
              if constexpr (SPARSE) {
                if (c8 == 7 && r == 0) sPvKeep[t * 2 + (j & 1)] = 1;
              }
              fence_proxy_async_shared();
              mbar_arrive(c8 == 7 ? bar_p_lo + t : bar_p_hi + t);
            }
          }
          return true;
        };
        if (!keep_tile) {
          // stage 2 dropped the tile: no exp2 pass and no P~.  The wait for the previous P.V keeps
          // this group's bar_o_done waits one phase apart and orders the reuse of the flag slot.
          if (j > 0 && !wait_warp(bar_o_done + t, (j - 1) & 1)) { leave_vote(j + 1); ok = false; break; }
          tc_fence_before();
          mbar_arrive(bar_s_free + t);  // S_t read (for the maximum)
          if (r == 0) sPvKeep[t * 2 + (j & 1)] = 0;
          mbar_arrive(bar_p_lo + t);
          mbar_arrive(bar_p_hi + t);
        } else if (!(diag ? exp_pass_masked() : exp_pass())) { leave_vote(j + 1); ok = false; break; }
        if constexpr (PER_TOKEN) {  // key scales of tile j+1 into the other buffer
          if (j + 1 < n_iter[t]) {
            sks_t[((j + 1) & 1) * 128 + r] = sk_next;
            mbar_arrive(bar_sks + t);
          }
        }
        if (r == 0) stamp((3 * t + 2) * n_kv_total + j);
      }
      // ---- epilogue of this query tile by its own softmax group (both tiles in parallel):
      // O[q][d] = O^T[d][q] / l_q -> fp16, staged in the tile's own P~ rows (two [128 q][64 d]
      // pieces; this thread is TMEM lane d = r of O^T), then TMA-stored by one thread
      // Every thread of the group reaches both group barriers on every path (a warp whose
      // bounded wait gave up skips only the work), so a timeout cannot strand the group.
      const float2 l2 = __fadd2_rn(__fadd2_rn(lsum[0], lsum[1]), __fadd2_rn(lsum[2], lsum[3]));
      sL[qi] = 1.f / (l2.x + l2.y);
      group_sync(1 + t);  // the tile's 1 / l complete
      ok = ok && __all_sync(0xffffffffu, mbar_wait(bar_o_done + t, (n_iter[t] - 1) & 1, abort_flag));
      if (ok) {
        tc_fence_after();
        const uint32_t tOT = tmem + lane_addr + 256 + 128 * t;
        const uint32_t stage = smem_u32(sP) + (r >> 6) * L::P_ATOM + t * 128 * 128 + (r & 63) * 2;
        const float* inv_l = sL + t * 128;
        // FP8: head dimension r's scale and mean (O = O^T acc / l * sv + vm)
        float2 sv2 = make_float2(1.f, 1.f), vm2 = make_float2(0.f, 0.f);
        if constexpr (FP8) {
          const float s_ = __ldg(sv + static_cast<size_t>(bh) * D + r);
          const float m_ = vm ? __ldg(vm + static_cast<size_t>(bh) * D + r) : 0.f;
          sv2 = make_float2(s_, s_);
          vm2 = make_float2(m_, m_);
        }
#pragma unroll
        for (int cb = 0; cb < 128; cb += 64) {
          uint32_t ov[64];
          tmem_ld64_sync(tOT + cb, ov);
          // queries q, q+1 of this head dimension: packed multiply and packed fp16 conversion
          // (each value rounded once, as a scalar multiply and conversion would), then one
          // 16-bit store per query row
#pragma unroll
          for (int i = 0; i < 64; i += 4) {
            const float4 il = *reinterpret_cast<const float4*>(inv_l + cb + i);
            float2 a = __fmul2_rn(make_float2(__uint_as_float(ov[i]), __uint_as_float(ov[i + 1])), make_float2(il.x, il.y));
            float2 b = __fmul2_rn(make_float2(__uint_as_float(ov[i + 2]), __uint_as_float(ov[i + 3])), make_float2(il.z, il.w));
            if constexpr (FP8) {
              a = __ffma2_rn(a, sv2, vm2);
              b = __ffma2_rn(b, sv2, vm2);
            }
            const uint32_t ha = pack_half2(a.x, a.y), hb = pack_half2(b.x, b.y);
            st_shared_u16(stage + (cb + i) * 128, static_cast<uint16_t>(ha));
            st_shared_u16(stage + (cb + i + 1) * 128, static_cast<uint16_t>(ha >> 16));
            st_shared_u16(stage + (cb + i + 2) * 128, static_cast<uint16_t>(hb));
            st_shared_u16(stage + (cb + i + 3) * 128, static_cast<uint16_t>(hb >> 16));
          }
        }
        fence_proxy_async_shared();
      }
      group_sync(1 + t);  // the whole tile staged
      if (r == 0 && !*abort_flag) {
        const int y = q_tile * L::BM;  // rows past N are clipped by the tensor map
        tma_store_3d(&tm_o, sP + t * 128 * 128, 0, y, bh);
        tma_store_3d(&tm_o, sP + L::P_ATOM + t * 128 * 128, 64, y, bh);
        bulk_commit_and_wait_read();
      }
    }
  } else {
    reg_dealloc<88>();
    // ============================================================ correction
    const int quad = warp & 3;  // TMEM lanes (head dimensions) 32 quad .. 32 quad + 31 of O^T
    const uint32_t tOT = tmem + (static_cast<uint32_t>(quad * 32) << 16) + 256;
    bool ok = true;
    for (int j = 1; ok && j < n_kv; ++j) {
      for (int t = 0; t < n_tiles; ++t) {
        if (j >= n_iter[t]) continue;
        if (!wait_warp(bar_vote + 2 * t + (j & 1), ((j - 1) >> 1) & 1)) { ok = false; break; }
        if (sFlag[t * 3 + j % 3]) {
          // O^T holds the products up to key tile j-1: wait for the last of them
          if (!wait_warp(bar_o_done + t, (j - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const float* alpha = sAlpha + (j & 1) * 256 + t * 128;
#pragma unroll
          for (int cb = 0; cb < 128; cb += 32) {
            uint32_t ov[32];
            tmem_ld32_sync(tOT + t * 128 + cb, ov);
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha[cb + i]);
            tmem_st32(tOT + t * 128 + cb, ov);
          }
          tmem_wait_st();
          tc_fence_before();
        }
        mbar_arrive(bar_corr + t);
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
