// Host helpers shared by the tensor-core kernels: TMA descriptor encoding through the driver entry
// point (no link-time dependency on libcuda) and the bound of device-side waits.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace vmla {

struct TmaMaps5 {
  CUtensorMap q, qr, k, kr, v;
  CUtensorMap wuk, wuv;   // fused latent attention: W^K_up and W^V_up
};

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
