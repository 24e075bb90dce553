// Peer mappings of device buffers between processes (one process per GPU): a cache replica's planes
// are exported by their owner and imported by every other rank, whose compress kernels then store the
// chunk's latents into them directly.  A pointer may lie inside a larger allocation (PyTorch's caching
// allocator sub-allocates), so the handle carries the offset from the allocation's base.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>
#include <unordered_map>

#include "vmla_internal.cuh"

namespace {

using GetRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

GetRangeFn range_fn() {
  static GetRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetRangeFn>(p);
  });
  return fn;
}

std::mutex g_mu;
std::unordered_map<uintptr_t, void*> g_bases;   // imported pointer -> mapped allocation base

}  // namespace

extern "C" {

vmla_status vmla_ipc_export(const void* dev_ptr, vmla_ipc_handle* out) {
  if (!dev_ptr || !out) return vmla::report(VMLA_ERR_INVALID_ARG, "dev_ptr and out must not be NULL");
  GetRangeFn fn = range_fn();
  if (!fn) return vmla::report(VMLA_ERR_CUDA, "cuMemGetAddressRange is not available");
  CUdeviceptr base = 0;
  size_t size = 0;
  if (fn(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
    return vmla::report(VMLA_ERR_INVALID_ARG, "dev_ptr is not device memory of this context");
  cudaIpcMemHandle_t h;
  cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
  if (e != cudaSuccess) return vmla::report(VMLA_ERR_CUDA, cudaGetErrorString(e));
  static_assert(sizeof(h) <= sizeof(out->bytes), "IPC handle size");
  std::memset(out, 0, sizeof(*out));
  std::memcpy(out->bytes, &h, sizeof(h));
  out->offset = (int64_t)(reinterpret_cast<uintptr_t>(dev_ptr) - (uintptr_t)base);
  return VMLA_OK;
}

vmla_status vmla_ipc_import(const vmla_ipc_handle* h, void** dev_ptr) {
  if (!h || !dev_ptr) return vmla::report(VMLA_ERR_INVALID_ARG, "handle and dev_ptr must not be NULL");
  *dev_ptr = nullptr;
  cudaIpcMemHandle_t mh;
  std::memcpy(&mh, h->bytes, sizeof(mh));
  void* base = nullptr;
  cudaError_t e = cudaIpcOpenMemHandle(&base, mh, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return vmla::report(VMLA_ERR_CUDA, cudaGetErrorString(e));
  void* p = static_cast<uint8_t*>(base) + h->offset;
  std::lock_guard<std::mutex> lk(g_mu);
  g_bases[reinterpret_cast<uintptr_t>(p)] = base;
  *dev_ptr = p;
  return VMLA_OK;
}

vmla_status vmla_ipc_release(void* dev_ptr) {
  void* base = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_bases.find(reinterpret_cast<uintptr_t>(dev_ptr));
    if (it == g_bases.end()) return vmla::report(VMLA_ERR_INVALID_ARG, "pointer was not returned by vmla_ipc_import");
    base = it->second;
    g_bases.erase(it);
  }
  cudaError_t e = cudaIpcCloseMemHandle(base);
  if (e != cudaSuccess) return vmla::report(VMLA_ERR_CUDA, cudaGetErrorString(e));
  return VMLA_OK;
}

}  // extern "C"
