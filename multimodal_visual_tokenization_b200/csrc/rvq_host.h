// rvq_host.h -- host-side helpers shared by the translation units of librvq.so:
// argument checks, CUDA error mapping, the kernel launch counter, the GEMM
// profiling events, NVTX ranges and host-side fault injection.
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
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

// NVTX range over one entry-point call, named after the entry point (shown by nsys / ncu
// timelines; a push and a pop that do nothing while no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

// Host-side fault injection, for testing how callers handle errors without making a GPU fault:
// RVQ_FAULT="<entry point>:<status>[,<entry point>:<status>...]" (read once, at the first call)
// makes each named entry point return that negative rvq_status before it checks its arguments or
// touches the device.  0 when the entry point is not named (the normal case).
int injected_fault(const char *entry);

#define RVQ_ENTRY(name)                                        \
  ::rvq::NvtxRange rvq_nvtx_range_(name);                      \
  if (const int rvq_fault_ = ::rvq::injected_fault(name)) return rvq_fault_

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
