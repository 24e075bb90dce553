// TMA descriptor encoding and the device-wait bound shared by the tensor-core kernels.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "ptx_sm100.cuh"
#include "tc_common.cuh"
#include "vmla_internal.cuh"

namespace vmla {
namespace {

std::atomic<uint64_t> g_wait_limit_ns{1000000000ull};   // 1 s
std::atomic<int> g_drop_kv_tile{-1};

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(); }

int take_drop_kv_tile() { return g_drop_kv_tile.exchange(-1); }

namespace {
std::atomic<int64_t> g_shrink_extents{0};
}

int64_t checked_extent(int64_t bytes) {
  const int64_t s = g_shrink_extents.load();
  return bytes > s ? bytes - s : 0;
}

cudaError_t ensure_smem_attr(const void* kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load() & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit);
  return e;
}

namespace {
thread_local const char* t_reason = "";
}
void set_tc_reason(const char* why) { t_reason = why; }
const char* tc_last_reason() { return t_reason; }

cudaError_t make_map_4d(CUtensorMap* map, const void* base, int64_t d0, int64_t d1, int64_t d2,
                        int64_t d3, int64_t s1, int64_t s2, int64_t s3, int b0, int b1, int b2,
                        int swizzle_bytes) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[4] = {(cuuint64_t)d0, (cuuint64_t)d1, (cuuint64_t)d2, (cuuint64_t)d3};
  cuuint64_t strides[3] = {(cuuint64_t)s1, (cuuint64_t)s2, (cuuint64_t)s3};
  cuuint32_t box[4] = {(cuuint32_t)b0, (cuuint32_t)b1, (cuuint32_t)b2, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                          : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                          : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace vmla

extern "C" VMLA_API int32_t vmla_set_wait_timeout_ms(int32_t ms) {
  const uint64_t old = vmla::g_wait_limit_ns.load() / 1000000ull;
  if (ms > 0) vmla::g_wait_limit_ns.store((uint64_t)ms * 1000000ull);
  return (int32_t)old;
}

extern "C" VMLA_API void vmla_debug_drop_kv_tile(int32_t tile) { vmla::g_drop_kv_tile.store(tile); }

extern "C" VMLA_API int32_t vmla_debug_shrink_extents(int64_t bytes) {
  vmla::g_shrink_extents.store(bytes > 0 ? bytes : 0);
  return VMLA_CHECKED;
}

namespace vmla {
namespace {
// One pair of arguments per thread through exactly the device function the softmax warps call.
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t stride = 2 * (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x); i < n; i += stride) {
    const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.f;
    float y0, y1;
    sm100::exp2_poly2(y0, y1, x0, x1);
    y[i] = y0;
    if (i + 1 < n) y[i + 1] = y1;
  }
}
}  // namespace
}  // namespace vmla

extern "C" VMLA_API vmla_status vmla_debug_exp2_poly(const float* x, float* y, int64_t n, void* stream) {
  if (n < 0) return vmla::report(VMLA_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return VMLA_OK;                       // nothing to do (empty buffers may be NULL)
  if (!x || !y) return vmla::report(VMLA_ERR_INVALID_ARG, "x and y must not be NULL");
  const int64_t pairs = (n + 1) / 2;
  const int threads = 256;
  const int64_t want = (pairs + threads - 1) / threads;
  const int blocks = (int)(want < 148 * 8 ? want : 148 * 8);
  vmla::exp2_poly_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  vmla::count_launches(1);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? VMLA_OK : vmla::report(VMLA_ERR_CUDA, cudaGetErrorString(e));
}
