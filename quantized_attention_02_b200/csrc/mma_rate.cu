// mma_rate.cu -- tensor-core peak probe: the dense MMA rate of one SM per kind, measured on
// straight-line issue, so that the roofline's INT8 : FP16 (and FP8) ratio is a measurement of
// this GPU rather than a datasheet assumption.
//
// One CTA per SM (120 KB of shared memory keeps a second one off), 512 TMEM columns.  Two warps
// each own a 256-column fp32/s32 accumulator and issue `iters` tcgen05 MMAs of shape
// M = 128, N = 256 (the largest single-CTA shape) back to back: the loop body is eight
// instructions with loop-invariant descriptors and the accumulate flag set, so nothing is
// computed between them.  Operands are zero-filled shared memory (128-byte swizzled, K-major).
//   kind 0: kind::i8      (s8 x s8 -> s32),      K = 32 per instruction
//   kind 1: kind::f16     (f16 x f16 -> f32),    K = 16
//   kind 2: kind::f8f6f4  (e4m3 x e4m3 -> f32),  K = 32
// Each instruction is 128 * 256 * K multiply-accumulates.  Warp 0's lane 0 writes the CTA's SM
// cycles from its first issue until both warps' MMAs have completed (a commit per warp) to
// cycles[blockIdx.x]; the host divides 2 * iters * 128 * 256 * K by that.  Every wait is bounded:
// one that gives up sets *status = 1 and the CTA still frees its tensor memory and exits.
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

// instruction descriptor: D format bits 4-5, A / B formats bits 7-9 / 10-12, both K-major,
// N >> 3 in bits 17-22, M >> 4 in bits 24-28
constexpr uint32_t idesc(uint32_t d_fmt, uint32_t ab_fmt, uint32_t M, uint32_t N) {
  return (d_fmt << 4) | (ab_fmt << 7) | (ab_fmt << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

template <int KIND>
__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
  if constexpr (KIND == 0) {
    asm volatile("{\n\t.reg .pred p, e;\n\t.reg .b32 ln;\n\telect.sync ln|e, 0xffffffff;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
                 "l"(a), "l"(b), "r"(id), "r"(acc) : "memory");
  } else if constexpr (KIND == 1) {
    asm volatile("{\n\t.reg .pred p, e;\n\t.reg .b32 ln;\n\telect.sync ln|e, 0xffffffff;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
                 "l"(a), "l"(b), "r"(id), "r"(acc) : "memory");
  } else {
    asm volatile("{\n\t.reg .pred p, e;\n\t.reg .b32 ln;\n\telect.sync ln|e, 0xffffffff;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
                 "l"(a), "l"(b), "r"(id), "r"(acc) : "memory");
  }
}

template <int KIND>
__global__ void __launch_bounds__(128, 1) mma_peak_kernel(int iters, long long* cycles, int* status) {
  extern __shared__ uint8_t raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;          // 128 rows x 128 B
  uint8_t* sB = smem + 16384;  // 256 rows x 128 B
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 49152);  // one per issuing warp
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + 49168);
  volatile long long* t_start = reinterpret_cast<volatile long long*>(smem + 49176);
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

  constexpr uint32_t K_BYTES = 32;  // every kind reads 32 bytes of K per row per instruction
  constexpr uint32_t ID = KIND == 0 ? idesc(2 /*s32*/, 1 /*s8*/, 128, 256)
                        : KIND == 1 ? idesc(1 /*f32*/, 0 /*f16*/, 128, 256)
                                    : idesc(1 /*f32*/, 0 /*e4m3*/, 128, 256);
  const int w = threadIdx.x >> 5;
  if (w < 2) {
    const uint32_t d = tmem + 256u * static_cast<uint32_t>(w);  // this warp's accumulator columns
    const uint32_t a = smem_u32(sA), b = smem_u32(sB);
    const uint64_t da0 = desc(a, 16, 1024, 2), da1 = desc(a + K_BYTES, 16, 1024, 2);
    const uint64_t da2 = desc(a + 2 * K_BYTES, 16, 1024, 2), da3 = desc(a + 3 * K_BYTES, 16, 1024, 2);
    const uint64_t db0 = desc(b, 16, 1024, 2), db1 = desc(b + K_BYTES, 16, 1024, 2);
    const uint64_t db2 = desc(b + 2 * K_BYTES, 16, 1024, 2), db3 = desc(b + 3 * K_BYTES, 16, 1024, 2);
    if (threadIdx.x == 0) *t_start = clock64();
    mma<KIND>(d, da0, db0, ID, 0u);  // first instruction initialises the accumulator
    for (int i = 8; i < iters; i += 8) {
      mma<KIND>(d, da1, db1, ID, 1u);
      mma<KIND>(d, da2, db2, ID, 1u);
      mma<KIND>(d, da3, db3, ID, 1u);
      mma<KIND>(d, da0, db0, ID, 1u);
      mma<KIND>(d, da1, db1, ID, 1u);
      mma<KIND>(d, da2, db2, ID, 1u);
      mma<KIND>(d, da3, db3, ID, 1u);
      mma<KIND>(d, da0, db0, ID, 1u);
    }
    mma<KIND>(d, da1, db1, ID, 1u);  // iters is a multiple of 8: 1 + 8 (iters/8 - 1) + 7 = iters
    mma<KIND>(d, da2, db2, ID, 1u);
    mma<KIND>(d, da3, db3, ID, 1u);
    mma<KIND>(d, da0, db0, ID, 1u);
    mma<KIND>(d, da1, db1, ID, 1u);
    mma<KIND>(d, da2, db2, ID, 1u);
    mma<KIND>(d, da3, db3, ID, 1u);
    asm volatile("{\n\t.reg .pred e;\n\t.reg .b32 ln;\n\telect.sync ln|e, 0xffffffff;\n\t"
                 "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
                     smem_u32(bars + w))
                 : "memory");
  }
  if (threadIdx.x == 0) {  // both warps' products complete (bounded waits, ~1 s each)
    for (int i = 0; i < 2; ++i) {
      uint32_t done = 0;
      const long long tw = clock64();
      while (!done) {
        asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}" : "=r"(done) : "r"(smem_u32(bars + i)) : "memory");
        if (!done && clock64() - tw > (1ll << 31)) {
          atomicExch(status, 1);
          break;
        }
      }
    }
    cycles[blockIdx.x] = clock64() - *t_start;
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  cta_sync();
  if (threadIdx.x < 32) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

template <int KIND>
int launch_peak(int iters, int ctas, long long* cycles, int* status, cudaStream_t st) {
  static bool configured = false;
  constexpr int SMEM = 120 * 1024;  // one CTA (and one 512-column TMEM allocation) per SM
  if (!configured) {
    if (cudaFuncSetAttribute(mma_peak_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess)
      return SAGE_ERR_CUDA;
    configured = true;
  }
  mma_peak_kernel<KIND><<<ctas, 128, SMEM, st>>>(iters, cycles, status);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

}  // namespace probe
}  // namespace sage

extern "C" int sage_debug_mma_peak(int kind, int iters, int ctas, long long* cycles, int* status, void* stream) {
  if (kind < 0 || kind > 2 || iters < 8 || iters > (1 << 24) || iters % 8 != 0 || ctas <= 0 || !cycles || !status)
    return SAGE_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (kind == 0) return sage::probe::launch_peak<0>(iters, ctas, cycles, status, st);
  if (kind == 1) return sage::probe::launch_peak<1>(iters, ctas, cycles, status, st);
  return sage::probe::launch_peak<2>(iters, ctas, cycles, status, st);
}
