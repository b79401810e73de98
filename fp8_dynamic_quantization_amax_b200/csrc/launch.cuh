// launch.cuh -- kernel launches with programmatic dependent launch (PDL).
//
// A kernel launched with programmatic stream serialization may start (be
// scheduled, run its set-up) while the previous kernel in the stream is
// still finishing; it must then execute griddepcontrol.wait before its first
// access to global memory, which returns once the previous grid has
// completed and its writes are visible.  Every kernel launched through
// launch_pdl() does that, so back-to-back kernels of a step (and the nodes
// of a captured CUDA graph) lose most of the launch gap between them.  A
// kernel launched without the attribute ignores the wait.
#pragma once

#include <cuda_runtime.h>

namespace hq {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Lets the next kernel in the stream launch now rather than when this grid's
// CTAs exit: its CTAs are dispatched as this grid's leave the SMs (or into
// room they leave free) and run their set-up up to their own pdl_wait(),
// which still returns only once this grid has completed.  Every kernel calls
// it right after its pdl_wait(), so once all of a grid's CTAs have started
// the next launch is already in flight.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              bool cooperative, Args... args) {
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cooperative) {
    attr[n].id = cudaLaunchAttributeCooperative;
    attr[n].val.cooperative = 1;
    ++n;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  if (e == cudaErrorNotSupported || e == cudaErrorInvalidValue) {
    // this launch form refused the attribute: launch serialised instead
    cudaGetLastError();
    cfg.attrs = attr + 1;
    cfg.numAttrs = n - 1;
    e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  }
  return e;
}

}  // namespace hq
