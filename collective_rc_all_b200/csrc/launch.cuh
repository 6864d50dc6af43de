// launch.cuh -- how every kernel of this library is launched.
//
// Kernels can go out with programmatic dependent launch: the launch carries the
// programmatic stream-serialization attribute, so the GPU may schedule the
// kernel's thread blocks while the previous kernel in the stream is still
// draining, and each kernel triggers its own dependents as soon as all of its
// blocks are running.  The contract that keeps this exact: every kernel runs
// pdl_wait() (griddepcontrol.wait) before its first global-memory access.
// That instruction returns once the kernels it depends on have completed and
// their memory operations are visible, so a kernel reads and writes global
// memory only after everything earlier in the stream is finished, exactly as
// with an ordinary launch; only the launch latency and the kernel's prologue
// (shared-memory tables, mbarrier set-up) overlap the previous kernel's tail.
// Stream capture turns the attribute into programmatic graph edges.
//
// Off by default: RC_PDL=1 in the environment (read once per process) turns
// it on.  Measured on a sequence of seven different collectives captured in
// one graph, it changed nothing with the bulk-copy fan-out (133.8 vs 133.5 us)
// and cost 5% with the register fan-out (138.8 vs 131.1 us), presumably
// because the dependents' blocks, resident early and waiting at
// griddepcontrol.wait, take issue slots from the running kernel.  Without
// the attribute griddepcontrol.wait returns at once.
#pragma once

#include <cuda_runtime.h>

#include <utility>

#include "internal.h"

namespace rc {

bool pdl_enabled();

template <class... KArgs, class... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          Args &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (pdl_enabled()) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  cudaError_t err = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (err != cudaSuccess) {
    (void)cudaGetLastError();  // clear the launch error; it is returned here
    return err;
  }
  note_launches(1);
  return cudaSuccess;
}

}  // namespace rc
