// Host helpers shared by the tensor-core kernels: TMA descriptor encoding through the driver entry
// point (no link-time dependency on libcuda) and the bound of device-side waits.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace vmla {

// Tensor maps of one latent attention launch: query boxes (q, and its rope part qr), the cache planes
// (k = c, also read as V; kr = k^R) and, for the fused layer, W^K_up and W^V_up.
struct AttnMaps {
  CUtensorMap q, qr, k, kr;
  CUtensorMap wuk, wuv;
};

// Checked builds (compiled with -DVMLA_CHECKED=1): every computed global store of the tensor-core
// kernels is tested against the extent of the buffer it writes; a store outside it is skipped and its
// site (90 + site) is recorded in the device status word.  Release builds compile the test away.
#ifndef VMLA_CHECKED
#define VMLA_CHECKED 0
#endif
struct Span {
  const void* base;
  int64_t bytes;
};
__host__ __device__ inline Span make_span(const void* base, int64_t bytes) { return Span{base, bytes}; }
#ifdef __CUDACC__
__device__ __forceinline__ bool store_ok(const Span& s, const void* p, int bytes, int* status, int site) {
#if VMLA_CHECKED
  const char* b = static_cast<const char*>(s.base);
  const char* q = static_cast<const char*>(p);
  if (q < b || q + bytes > b + s.bytes) {
    if (status) atomicCAS(status, 0, 90 + site);
    return false;
  }
#else
  (void)s; (void)p; (void)bytes; (void)status; (void)site;
#endif
  return true;
}
#endif
// Extent of a buffer of `bytes` as the checked build records it: less `vmla_debug_shrink_extents`
// bytes when that test hook is set, so that correct stores at the end of the buffer are reported.
int64_t checked_extent(int64_t bytes);

// Encode a 4-D bf16 tensor map {d0 (contiguous), d1, d2, d3} with byte strides s1, s2, s3 of the
// three outer dimensions and box {b0, b1, b2, 1}; swizzle_bytes is 128, 64, 32 or 0.  Out-of-range
// rows read as zeros.
cudaError_t make_map_4d(CUtensorMap* map, const void* base, int64_t d0, int64_t d1, int64_t d2,
                        int64_t d3, int64_t s1, int64_t s2, int64_t s3, int b0, int b1, int b2,
                        int swizzle_bytes);

// Bound of every device-side mbarrier wait, in nanoseconds (vmla_set_wait_timeout_ms).
uint64_t wait_limit_ns();

// Raise a kernel's dynamic shared-memory limit once per device (bit d of `done` marks device d).
cudaError_t ensure_smem_attr(const void* kernel, int bytes, std::atomic<uint64_t>& done);

// Test hook of vmla_debug_drop_kv_tile: returns the pending tile index (or -1) and clears it.
int take_drop_kv_tile();

// Reason of the last refusal by a tc_check_* function (thread-local).
void set_tc_reason(const char* why);

}  // namespace vmla
