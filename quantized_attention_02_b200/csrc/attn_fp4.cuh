// attn_fp4.cuh -- the fused attention kernel of the microscaling FP4 variant (included by
// attn_kernels.cu, after the head-dimension-128 kernel whose helpers it uses).
//
// Method (SageAttention3 abstract: attention on Blackwell's FP4 tensor cores with microscaling;
// the readings are the oracle's, oracle/sage_oracle_sa3.c):
//   S   = Q4 . K4^T              E2M1 x E2M1 with one UE4M3 scale per 16 channels
//                                (tcgen05 kind::mxf4nvf4 block16), fp32 in tensor memory
//   u   = S * gq * gk * sm_scale * log2(e)     gq, gk: the fp32 scales of the 128-token tiles
//   online softmax over 128-key tiles with an integer offset m = ceil(max u seen so far); when
//   it grows, O and the row sum are scaled by 2^(m_old - m_new) (exact)
//   p   = 2^(u - m + 10)         the row sum takes p unrounded
//   P~  = microscaled E2M1 of p, one UE4M3 scale per 16 keys
//   O  += P~ . V4                V4: E2M1 codes of (V - vm) / gv along the keys, 16 keys per scale
//   O   = O * gv / l + vm        stored as fp16
//
// CTA: one 128-row query tile of one head; 10 warps: warp 0 TMA producer (Q once, K and V tiles
// and their scale atoms through a 3-stage ring), warp 1 MMA issuer (also allocates tensor
// memory), warps 2-9 softmax (two threads per query row = tensor-memory lane, each with half of
// the row's keys and output columns).  Tensor memory:
// S [0, 128), O [128, 256), then the scale factors copied from shared memory by tcgen05.cp
// (4 columns per 512-byte atom): Q 256, K stage s 264 + 8s, P~ 288, V stage s 296 + 8s.
// Per key tile j the MMA warp issues Q.K^T(j+1) as soon as the softmax holds S(j) in registers,
// then P~.V(j) once P~(j) and its scales are in shared memory.

struct Fp4Layout {
  static constexpr int BM = 128, BN = 128, D = 128, STAGES = 3;
  static constexpr int TILE = 128 * 64;  // 128 rows of 128 E2M1 codes (64 bytes)
  static constexpr int SF = 1024;        // two 512-byte scale atoms (64 elements of K each)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE;
  static constexpr int OFF_V = OFF_K + STAGES * TILE;
  static constexpr int OFF_P = OFF_V + STAGES * TILE;
  static constexpr int OFF_SFQ = OFF_P + TILE;
  static constexpr int OFF_SFK = OFF_SFQ + SF;
  static constexpr int OFF_SFV = OFF_SFK + STAGES * SF;
  static constexpr int OFF_SFP = OFF_SFV + STAGES * SF;
  static constexpr int OFF_GV = OFF_SFP + SF;  // [128] channel scales
  static constexpr int OFF_VM = OFF_GV + 512;  // [128] channel means
  static constexpr int OFF_XCH = OFF_VM + 512;  // row-maximum exchange [3][2][128], fail flags, row sums [2][128]
  static constexpr int OFF_BAR = OFF_XCH + 3 * 1024 + 16 + 1024;
  static constexpr int NUM_BARS = 1 + 3 * STAGES + 5;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr int THREADS = 320;
  static constexpr uint32_t COL_S = 0, COL_O = 128, COL_SFQ = 256, COL_SFK = 264, COL_SFP = 288, COL_SFV = 296;
  static_assert(COL_SFK + 8 * STAGES <= COL_SFP && COL_SFV + 8 * STAGES <= 512, "tensor-memory columns");
};

template <bool CAUSAL, bool RAGGED>
__global__ void __launch_bounds__(320, 1)
    sage_attn_fp4_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const uint8_t* __restrict__ sfq,
                         const uint8_t* __restrict__ sfk, const uint8_t* __restrict__ sfv,
                         const float* __restrict__ gq, const float* __restrict__ gk, const float* __restrict__ gv,
                         const float* __restrict__ vm, __half* __restrict__ o, int N, float sm_scale_log2) {
  using L = Fp4Layout;
  constexpr int S = L::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* sGV = reinterpret_cast<float*>(smem + L::OFF_GV);
  float* sVM = reinterpret_cast<float*>(smem + L::OFF_VM);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* bar_q = bars;
  uint64_t* bar_k_full = bars + 1;
  uint64_t* bar_v_full = bar_k_full + S;
  uint64_t* bar_kv_empty = bar_v_full + S;
  uint64_t* bar_s_full = bar_kv_empty + S;  // Q.K^T(j) complete
  uint64_t* bar_s_free = bar_s_full + 1;    // the softmax holds S(j) in registers (256 arrivals)
  uint64_t* bar_p_full = bar_s_free + 1;    // P~(j) and its scales in shared memory (256 arrivals)
  uint64_t* bar_o_done = bar_p_full + 1;    // P~.V(j) complete
  uint64_t* bar_drain = bar_o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = (N + L::BM - 1) / L::BM;
  const int bh = static_cast<int>(blockIdx.x) / n_qt;
  const int q_tile = n_qt - 1 - static_cast<int>(blockIdx.x) % n_qt;  // causal: the longest rows first
  const int n_kt = n_qt;
  const int n_kv = CAUSAL ? q_tile + 1 : n_kt;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(bar_k_full + s, 1);
      mbar_init(bar_v_full + s, 1);
      mbar_init(bar_kv_empty + s, 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_s_free, 256);
    mbar_init(bar_p_full, 256);
    mbar_init(bar_o_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp >= 2 && warp < 6) {  // the channel scales and means of this head for the epilogue
    const int c = threadIdx.x - 64;
    sGV[c] = __ldg(gv + static_cast<size_t>(bh) * L::D + c);
    sVM[c] = vm ? __ldg(vm + static_cast<size_t>(bh) * L::D + c) : 0.f;
  }
  if (threadIdx.x < 3) reinterpret_cast<int*>(smem + L::OFF_XCH + 3 * 1024)[threadIdx.x] = 0;  // exchange fail flags
  tc_fence_before();
  cta_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ============================================================ TMA producer
    if (lane == 0) {
      int issued[S];
      for (int s = 0; s < S; ++s) issued[s] = 0;
      mbar_arrive_expect_tx(bar_q, L::TILE + L::SF);
      tma_load_3d(smem + L::OFF_Q, &tm_q, bar_q, 0, q_tile * L::BM, bh);
      bulk_load(smem + L::OFF_SFQ, sfq + (static_cast<size_t>(bh) * n_qt + q_tile) * L::SF, L::SF, bar_q);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % S, it = j / S;
        if (j >= S && !mbar_wait(bar_kv_empty + s, (it - 1) & 1, abort_flag)) break;
        const size_t sf_off = (static_cast<size_t>(bh) * n_kt + j) * L::SF;
        mbar_arrive_expect_tx(bar_k_full + s, L::TILE + L::SF);
        tma_load_3d(smem + L::OFF_K + s * L::TILE, &tm_k, bar_k_full + s, 0, j * L::BN, bh);
        bulk_load(smem + L::OFF_SFK + s * L::SF, sfk + sf_off, L::SF, bar_k_full + s);
        mbar_arrive_expect_tx(bar_v_full + s, L::TILE + L::SF);
        tma_load_3d(smem + L::OFF_V + s * L::TILE, &tm_v, bar_v_full + s, j * 64, 0, bh);  // keys j*128.. (bytes)
        bulk_load(smem + L::OFF_SFV + s * L::SF, sfv + sf_off, L::SF, bar_v_full + s);
        issued[s] = it + 1;
      }
      if (*abort_flag) {  // let copies in flight land before the CTA exits
        mbar_drain(bar_q, 0);
        for (int s = 0; s < S; ++s) {
          if (issued[s] > 0) {
            mbar_drain(bar_k_full + s, (issued[s] - 1) & 1);
            mbar_drain(bar_v_full + s, (issued[s] - 1) & 1);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer (whole warp; elect.sync)
    constexpr uint32_t IDESC = make_idesc_fp4(128, 128);
    const uint32_t sbase = smem_u32(smem);
    auto wait = [&](uint64_t* bar, uint32_t parity) { return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag)); };
    // two 512-byte scale atoms at saddr -> columns col .. col + 7
    auto copy_scales = [&](uint32_t col, uint32_t saddr) {
#pragma unroll
      for (int a = 0; a < 2; ++a)
        tmem_cp_32x128b_warp(tmem + col + 4 * a, make_smem_desc(saddr + 512 * a, 16, 128, kSwizzleNone));
    };
    // 128 x 128 x 128 block-scaled product, two K steps of 64 elements (32 bytes of each 64-byte row)
    auto product = [&](uint32_t d_col, uint32_t a_addr, uint32_t b_addr, uint32_t sfa_col, uint32_t sfb_col, bool first) {
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const uint64_t a = make_smem_desc(a_addr + kk * 32, 16, 512, kSwizzle64B);
        const uint64_t b = make_smem_desc(b_addr + kk * 32, 16, 512, kSwizzle64B);
        mma_fp4_ss_warp(tmem + d_col, a, b, IDESC, tmem + sfa_col + 4 * kk, tmem + sfb_col + 4 * kk,
                        (first && kk == 0) ? 0u : 1u);
      }
    };
    auto qk = [&](int s) {
      copy_scales(L::COL_SFK + 8 * s, sbase + L::OFF_SFK + s * L::SF);
      product(L::COL_S, sbase + L::OFF_Q, sbase + L::OFF_K + s * L::TILE, L::COL_SFQ, L::COL_SFK + 8 * s, true);
      mma_commit_warp(bar_s_full);
    };
    bool ok = wait(bar_q, 0) && wait(bar_k_full, 0);
    if (ok) {
      tc_fence_after();
      copy_scales(L::COL_SFQ, sbase + L::OFF_SFQ);
      qk(0);
    }
    for (int j = 0; ok && j < n_kv; ++j) {
      const int s = j % S;
      if (j + 1 < n_kv) {
        const int s1 = (j + 1) % S;
        if (!wait(bar_k_full + s1, ((j + 1) / S) & 1)) break;
        if (!wait(bar_s_free, j & 1)) break;  // S(j) read: S may be overwritten
        tc_fence_after();
        qk(s1);
      }
      if (!wait(bar_p_full, j & 1)) break;
      if (!wait(bar_v_full + s, (j / S) & 1)) break;
      tc_fence_after();
      copy_scales(L::COL_SFP, sbase + L::OFF_SFP);
      copy_scales(L::COL_SFV + 8 * s, sbase + L::OFF_SFV + s * L::SF);
      product(L::COL_O, sbase + L::OFF_P, sbase + L::OFF_V + s * L::TILE, L::COL_SFP, L::COL_SFV + 8 * s, j == 0);
      mma_commit_warp(bar_o_done);
      mma_commit_warp(bar_kv_empty + s);  // this tile's products (and copies) reading stage s are done
    }
    mma_commit_warp(bar_drain);
    mbar_drain(bar_drain, 0);
  } else {
    // ============================================================ softmax
    // Two threads per query row (tensor-memory lane): half h of the row's 128 keys and of its
    // 128 output columns.  They agree on the row maximum through shared memory and a named
    // barrier of the 256 softmax threads, once per key tile.
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = quad * 32 + lane;
    const int q_row = q_tile * L::BM + r;
    const int c0 = 64 * half;  // this thread's first key of a tile and first output column
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + lane_addr + L::COL_S + c0, tO = tmem + lane_addr + L::COL_O + c0;
    const uint32_t p_row = smem_u32(smem + L::OFF_P) + r * 64;  // 64-byte swizzle: chunk c at c ^ ((r >> 1) & 3)
    // this half's four group scales: atom `half`, row r
    uint32_t* sfp_word = reinterpret_cast<uint32_t*>(smem + L::OFF_SFP + 512 * half + (r & 31) * 16 + (r >> 5) * 4);
    float* sMax = reinterpret_cast<float*>(smem + L::OFF_XCH);        // [3 slots][2 halves][128 rows]
    int* sFail = reinterpret_cast<int*>(smem + L::OFF_XCH + 3 * 1024);  // [3 slots]
    const float c_r = __fmul_rn(__ldg(gq + static_cast<size_t>(bh) * n_qt + q_tile), sm_scale_log2);
    const float* gk_head = gk + static_cast<size_t>(bh) * n_kt;
    float m_use = 0.f;
    float2 lsum[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
    bool ok = true;
    // Exchange of step j: slot j % 3 (last read at step j-3); the flag slot of step j+1 is cleared
    // here, its last reads (step j-2) being done before every thread reached step j-1's barrier.
    // A thread whose bounded wait gave up still takes the barrier of the step it leaves in, with
    // its fail flag set, so that all 256 threads leave at the same barrier.
    auto exchange = [&](int j, float hm, bool failed) -> float {
      const int slot = j % 3;
      if (threadIdx.x == 64) sFail[(j + 1) % 3] = 0;
      sMax[(slot * 2 + half) * 128 + r] = hm;
      if (failed) sFail[slot] = 1;
      asm volatile("barrier.sync 1, 256;" ::: "memory");
      if (*reinterpret_cast<volatile int*>(sFail + slot)) return NAN;
      return fmaxf(hm, sMax[(slot * 2 + (half ^ 1)) * 128 + r]);
    };
    for (int j = 0; j < n_kv; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar_s_full, j & 1, abort_flag))) {
        exchange(j, 0.f, true);
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t x[64];
      tmem_ld64_sync(tS, x);
      tc_fence_before();
      mbar_arrive(bar_s_free);
      // u = S * cb with cb > 0 (a zero factor only comes with all-zero codes, S = 0, and is kept
      // off zero so that masked keys, S = -inf, stay -inf): the maximum of the products is the
      // product of the maximum (rounding is monotonic)
      const float cb = fmaxf(__fmul_rn(c_r, __ldg(gk_head + j)), 1.17549435e-38f);
      // masked keys: past the diagonal (causal) and past N (a partial last key tile)
      const bool diag = (CAUSAL && j == q_tile) || (RAGGED && (j + 1) * L::BN > N);
      const int cmax = min((CAUSAL && j == q_tile) ? r : L::BN - 1, N - j * L::BN - 1) - c0;
      if (diag) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c > cmax) x[c] = 0xFF800000u;
      }
      float sm = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; c += 2) sm = max3f(sm, __uint_as_float(x[c]), __uint_as_float(x[c + 1]));
      const float hm = sm == -INFINITY ? -INFINITY : __fmul_rn(sm, cb);
      const float mx = exchange(j, hm, false);
      if (mx != mx) { ok = false; break; }  // a thread of the softmax gave up waiting
      // integer offset: set by the first tile, moved up when a tile's maximum passes it
      const float m_new = ceilf(mx);
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_use = m_new;
      } else if (m_new > m_use) {
        alpha = exp2_int(m_use - m_new);
        m_use = m_new;
        rescale = true;
      }
      // P~.V(j-1) must be complete before O is rescaled and before P~(j) overwrites P~(j-1)
      if (j > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(bar_o_done, (j - 1) & 1, abort_flag))) {
          if (j + 1 < n_kv) exchange(j + 1, 0.f, true);
          ok = false;
          break;
        }
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int i = 0; i < 4; ++i) lsum[i] = __fmul2_rn(lsum[i], make_float2(alpha, alpha));
#pragma unroll
        for (int cb2 = 0; cb2 < 64; cb2 += 32) {
          uint32_t ov[32];
          tmem_ld32_sync(tO + cb2, ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st32(tO + cb2, ov);
        }
        tmem_wait_st();
      }
      const float m_e = m_use - 10.f;  // p = 2^(S * cb - m + 10); exact: m is an integer
      uint32_t w[8];
      uint32_t sfw = 0u;
#pragma unroll
      for (int gi = 0; gi < 4; ++gi) {
        float2 z[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int c = 16 * gi + 2 * k;
          const float2 tt = __ffma2_rn(make_float2(__uint_as_float(x[c]), __uint_as_float(x[c + 1])),
                                       make_float2(cb, cb), make_float2(-m_e, -m_e));
          z[k] = make_float2(fast_exp2(tt.x), fast_exp2(tt.y));  // masked: exp2(-inf) = 0
          lsum[k & 3] = __fadd2_rn(lsum[k & 3], z[k]);
        }
        sfw |= microscale16_pos(z, w[2 * gi], w[2 * gi + 1]) << (8 * gi);
      }
      // P~ row r: keys 32c .. 32c+31 are the 16-byte chunk c of the row's 64 bytes (c = 2 half, 2 half + 1)
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * half + cc;
        st_shared_v4(p_row + ((c ^ ((r >> 1) & 3)) << 4), w[4 * cc], w[4 * cc + 1], w[4 * cc + 2], w[4 * cc + 3]);
      }
      *sfp_word = sfw;
      fence_proxy_async_shared();
      mbar_arrive(bar_p_full);
    }
    // ---- epilogue: O * gv / l + vm -> fp16 -> global (l: the two halves' sums)
    float* sL = reinterpret_cast<float*>(smem + L::OFF_XCH + 3 * 1024 + 16);  // [2 halves][128 rows]
    const float2 l2 = __fadd2_rn(__fadd2_rn(lsum[0], lsum[1]), __fadd2_rn(lsum[2], lsum[3]));
    sL[half * 128 + r] = l2.x + l2.y;
    asm volatile("barrier.sync 1, 256;" ::: "memory");
    if (ok && __all_sync(0xffffffffu, mbar_wait(bar_o_done, (n_kv - 1) & 1, abort_flag))) {
      tc_fence_after();
      const float inv_l = 1.f / (sL[r] + sL[128 + r]);
      __half* orow = o + (static_cast<size_t>(bh) * N + q_row) * L::D + c0;
#pragma unroll
      for (int cb2 = 0; cb2 < 64; cb2 += 32) {
        uint32_t ov[32];
        tmem_ld32_sync(tO + cb2, ov);
        uint32_t hv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = c0 + cb2 + 2 * i;
          const float a0 = __fadd_rn(__fmul_rn(__fmul_rn(__uint_as_float(ov[2 * i]), inv_l), sGV[c]), sVM[c]);
          const float a1 = __fadd_rn(__fmul_rn(__fmul_rn(__uint_as_float(ov[2 * i + 1]), inv_l), sGV[c + 1]), sVM[c + 1]);
          hv[i] = pack_half2(a0, a1);
        }
        if (q_row < N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cb2);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
        }
      }
    }
  }

  tc_fence_before();
  cta_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}
