// rvq_ipc.cu -- device pointers shared between the processes of one node (one per GPU), so
// that a kernel can read another GPU's buffer directly over NVLink (the codebook-sharded
// encode reads each winning codeword from the rank that holds it).  Host code only.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "rvq_host.h"

namespace rvq {
namespace {

typedef CUresult (*AddressRangeFn)(CUdeviceptr *, size_t *, CUdeviceptr);

AddressRangeFn address_range_fn() {
  static AddressRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(p);
  });
  return fn;
}

static_assert(sizeof(cudaIpcMemHandle_t) == RVQ_IPC_HANDLE_BYTES, "IPC handle size");

}  // namespace
}  // namespace rvq

extern "C" int rvq_ipc_export(const void *ptr, void *handle, size_t *offset) {
  using namespace rvq;
  if (!ptr || !handle || !offset) return RVQ_ERR_ARG;
  AddressRangeFn range = address_range_fn();
  if (!range) return RVQ_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return RVQ_ERR_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base)) != cudaSuccess) return RVQ_ERR_CUDA;
  std::memcpy(handle, &h, sizeof h);
  *offset = static_cast<size_t>(reinterpret_cast<CUdeviceptr>(ptr) - base);
  return RVQ_OK;
}

extern "C" int rvq_ipc_import(const void *handle, size_t offset, void **ptr) {
  using namespace rvq;
  if (!handle || !ptr) return RVQ_ERR_ARG;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof h);
  void *base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return RVQ_ERR_CUDA;
  *ptr = static_cast<uint8_t *>(base) + offset;
  return RVQ_OK;
}

extern "C" int rvq_ipc_close(void *ptr, size_t offset) {
  using namespace rvq;
  if (!ptr) return RVQ_ERR_ARG;
  return cudaIpcCloseMemHandle(static_cast<uint8_t *>(ptr) - offset) == cudaSuccess ? RVQ_OK : RVQ_ERR_CUDA;
}
