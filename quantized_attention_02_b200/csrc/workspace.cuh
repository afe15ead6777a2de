// workspace.cuh -- stream-ordered device workspace for the entry points that need one
// (sage_attn_fwd, sage_attn_fwd_host).
//
// Allocations come from a memory pool owned by the library (one per device, created on first
// use), not from the process's default pool, whose settings belong to the application.  The
// pool's release threshold is unlimited: memory freed by a call stays reserved for the next
// call instead of being handed back to the driver at every synchronization, which would make
// the first call after each synchronize map the workspace again (measured: 2-15 ms of host
// time for that call).  The pool therefore keeps the largest workspace used so far reserved
// until the process exits.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>

namespace sage {

// cudaMallocFromPoolAsync on the library's pool of the current device; returns the CUDA
// error (cudaSuccess on success).  Free with cudaFreeAsync on a stream ordered after the uses.
cudaError_t workspace_alloc(void** p, size_t bytes, cudaStream_t st);

}  // namespace sage
