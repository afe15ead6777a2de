// mma_rate.cu -- tensor-core issue probe for the MMA shapes the fused attention kernel uses.
//
// What it measures is the rate of this loop: one warp issuing one MMA per iteration with the
// destination column and the accumulate flag computed per instruction.  That loop reaches about
// one instruction per 110-140 SM cycles whatever N is, which is below the tensor core's rate for
// N <= 128 (straight-line issue of the same shapes runs at the datasheet per-SM rate), so its
// results are a lower bound on the tensor rate, not the peak.
//
// One CTA per SM; one thread issues `iters` back-to-back tcgen05 MMAs of one kind, rotating
// over `chains` independent TMEM accumulators (operands in shared memory, zero-filled), then
// waits for them with a commit; the CTA's SM-clock cycle count goes to cycles[blockIdx.x].
//   mode 0: kind::i8,  M=128 K=32, A and B from shared memory (Q.K^T shape)
//   mode 1: kind::f16, M=128 K=16, A from TMEM, B MN-major from shared memory (P.V shape)
//   mode 2: kind::f16, M=128 K=16, A and B from shared memory
// N is 64, 128 or 256; chains * N <= 256.
#include <cuda_runtime.h>

#include <cstdint>

#include "sage_attn.h"

namespace sage {
// sm100_ptx.cuh defines the device status word, so it is included in one translation unit
// only; the probe keeps its own copies of the few wrappers it needs.
namespace probe {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// CTA barrier counting threads one by one (non-.aligned): warps may reach it diverged.
__device__ __forceinline__ void cta_sync() { asm volatile("barrier.sync 0;" ::: "memory"); }

__device__ __forceinline__ uint64_t desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t swz) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (static_cast<uint64_t>(1u) << 46) |
         (static_cast<uint64_t>(swz) << 61);
}

constexpr uint32_t idesc(uint32_t d_fmt, uint32_t a_fmt, uint32_t b_fmt, uint32_t b_mn, uint32_t M, uint32_t N) {
  return (d_fmt << 4) | (a_fmt << 7) | (b_fmt << 10) | (b_mn << 16) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int mode, int n, int chains, int issuers, int iters,
                                                          long long* cycles, int* status) {
  extern __shared__ uint8_t raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;              // 16 KB
  uint8_t* sB = smem + 16384;      // 32 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 49152);  // one per issuing warp
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + 49168);
  for (int i = threadIdx.x; i < 49152 / 16; i += blockDim.x) reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bars)) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bars + 1)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // zero fill visible to the tensor core
  if (threadIdx.x < 32) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(slot)) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  cta_sync();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *slot;

  // Each issuing warp runs the loop with warp-uniform operands (elect.sync picks the lane that
  // issues) into its own accumulator columns; with two issuers each does half of the MMAs.
  const int w = threadIdx.x >> 5;
  if (w < issuers) {
    uint64_t* bar = bars + w;
    const int my_iters = iters / issuers;
    const uint32_t a = smem_u32(sA), b = smem_u32(sB);
    const uint32_t mask = static_cast<uint32_t>(chains - 1);  // chains is 1, 2 or 4
    uint32_t id = 0;
    if (mode == 0) id = idesc(2, 1, 1, 0, 128, n);
    else if (mode == 1) id = idesc(1, 0, 0, 1, 128, n);
    else id = idesc(1, 0, 0, 0, 128, n);
    // descriptors for the four K-steps, computed once; the loop body is unrolled by four
    uint64_t da[4], db[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      da[k] = desc(a + k * 32, 16, 1024, 2);
      db[k] = mode == 1 ? desc(b + k * 2048, 16384, 1024, 2) : desc(b + k * 32, 16, 1024, 2);
    }
    const long long t0 = clock64();
    for (int i = 0; i < my_iters; i += 4) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t c = static_cast<uint32_t>(i + k) & mask;
        const uint32_t acc = static_cast<uint32_t>(i + k) > mask ? 1u : 0u;
        const uint32_t d = tmem + 256 + (c + static_cast<uint32_t>(w * chains)) * static_cast<uint32_t>(n);
        if (mode == 1) {
          asm volatile("{\n\t.reg .pred p, e;\n\t.reg .b32 ln;\n\telect.sync ln|e, 0xffffffff;\n\t"
                       "setp.ne.b32 p, %4, 0;\n\t"
                       "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
                       "r"(tmem + k * 8), "l"(db[k]), "r"(id), "r"(acc) : "memory");
        } else if (mode == 0) {
          asm volatile("{\n\t.reg .pred p, e;\n\t.reg .b32 ln;\n\telect.sync ln|e, 0xffffffff;\n\t"
                       "setp.ne.b32 p, %4, 0;\n\t"
                       "@e tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
                       "l"(da[k]), "l"(db[k]), "r"(id), "r"(acc) : "memory");
        } else {
          asm volatile("{\n\t.reg .pred p, e;\n\t.reg .b32 ln;\n\telect.sync ln|e, 0xffffffff;\n\t"
                       "setp.ne.b32 p, %4, 0;\n\t"
                       "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
                       "l"(da[k]), "l"(db[k]), "r"(id), "r"(acc) : "memory");
        }
      }
    }
    asm volatile("{\n\t.reg .pred e;\n\t.reg .b32 ln;\n\telect.sync ln|e, 0xffffffff;\n\t"
                 "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
                     smem_u32(bar))
                 : "memory");
    uint32_t done = 0;
    const long long tw = clock64();
    while (!done) {
      asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
                   "selp.u32 %0, 1, 0, p;\n\t}" : "=r"(done) : "r"(smem_u32(bar)) : "memory");
      if (!done && clock64() - tw > (1ll << 31)) {  // bounded: ~1 s, then report and leave
        atomicExch(status, 1);
        break;
      }
    }
    if (threadIdx.x == 0) cycles[blockIdx.x] = clock64() - t0;  // issuer 0 (both run concurrently)
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  cta_sync();
  if (threadIdx.x < 32) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

}  // namespace probe
}  // namespace sage

extern "C" int sage_debug_mma_rate(int mode, int n, int chains, int issuers, int iters, int ctas, long long* cycles,
                                   int* status, void* stream) {
  if (mode < 0 || mode > 2 || iters <= 0 || iters > (1 << 24) || iters % 4 != 0 || ctas <= 0 || !cycles || !status)
    return SAGE_ERR_INVALID;
  if ((n != 64 && n != 128 && n != 256) || (chains != 1 && chains != 2 && chains != 4) || (issuers != 1 && issuers != 2) ||
      issuers * chains * n > 256 || iters % (4 * issuers) != 0)
    return SAGE_ERR_INVALID;
  if (mode == 1 && n > 128) return SAGE_ERR_INVALID;  // B box of the P.V shape holds 128 columns
  constexpr int SMEM = 49152 + 64 + 1024;
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(sage::probe::mma_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 120 * 1024) !=
        cudaSuccess)
      return SAGE_ERR_CUDA;
    configured = true;
  }
  // 120 KB of shared memory per CTA keeps one CTA (and one 512-column TMEM allocation) per SM
  (void)SMEM;
  sage::probe::mma_rate_kernel<<<ctas, 128, 120 * 1024, static_cast<cudaStream_t>(stream)>>>(mode, n, chains, issuers,
                                                                                              iters, cycles, status);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}
