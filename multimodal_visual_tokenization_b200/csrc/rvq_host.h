// rvq_host.h -- host-side helpers shared by the translation units of librvq.so:
// argument checks, CUDA error mapping, the kernel launch counter and the GEMM
// profiling events.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "rvq.h"

namespace rvq {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Every kernel launch of the library goes through note_launch() so that
// rvq_launch_count() reports how many kernels ran.
void note_launch(int n = 1);

// Profiling of the distance-GEMM launches (see rvq_profile_enable in rvq.h).
bool profiling_enabled();
void profile_begin(cudaStream_t s);
void profile_end(cudaStream_t s, int levels = 1);  // levels: RVQ levels the launch covers

inline int check_launch() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? RVQ_OK : RVQ_ERR_CUDA;
}

int device_sm_count(int *sms);

// Launch with programmatic stream serialization (see griddep_* in rvq_device.cuh).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace rvq
