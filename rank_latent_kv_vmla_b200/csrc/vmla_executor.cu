// Streaming executor: runs layer steps whose inputs and outputs live in host memory, overlapping the
// host -> device copies of the next step and the device -> host copy of the previous step with the
// current step's kernels (two staging slots in a caller-provided device workspace, two copy streams).
//
// Step i uses slot s = i % 2:
//   h2d stream      waits for compute(i-2) (slot s inputs free), copies x, q_nope, q_rope, records h2d[s]
//   compute stream  waits for h2d[s] and d2h(i-2) (slot s output free), runs vmla_compress_append and
//                   vmla_latent_attention_fused on the slot, records compute[s]
//   d2h stream      waits for compute[s], copies the slot's output to the host, records d2h[s]
#include <cuda_runtime.h>

#include <new>

#include "vmla_internal.cuh"

namespace {

constexpr int kSlots = 2;

int64_t round_up(int64_t v) { return (v + 255) / 256 * 256; }

struct Sizes {
  int64_t x, qn, qr, out, slot;
};

Sizes sizes(const vmla_config& c, int batch) {
  const int64_t nq = (int64_t)c.chunk_frames * c.grid_h * c.grid_w;
  const int64_t e = c.dtype == VMLA_BF16 ? 2 : 4;
  Sizes s;
  s.x = batch * nq * c.dim * e;
  s.qn = batch * nq * c.n_heads * c.d_nope * e;
  s.qr = batch * nq * c.n_heads * c.d_rope * e;
  s.out = batch * nq * c.n_heads * c.d_v * e;
  s.slot = round_up(s.x) + round_up(s.qn) + round_up(s.qr) + round_up(s.out);
  return s;
}

}  // namespace

struct vmla_executor {
  vmla_config cfg;
  int batch;
  Sizes sz;
  uint8_t* slot[kSlots];
  cudaStream_t compute, h2d, d2h;
  cudaEvent_t h2d_done[kSlots], compute_done[kSlots], d2h_done[kSlots];
  int64_t submitted;
};

extern "C" {

int64_t vmla_executor_workspace_bytes(const vmla_config* cfg, int32_t batch) {
  if (!cfg || batch <= 0) return -1;
  return kSlots * sizes(*cfg, batch).slot;
}

vmla_status vmla_executor_create(const vmla_config* cfg, int32_t batch, void* workspace,
                                 int64_t workspace_bytes, void* stream, vmla_executor** out) {
  if (!cfg || !out) return vmla::report(VMLA_ERR_INVALID_ARG, "cfg and out must not be NULL");
  *out = nullptr;
  if (batch <= 0) return vmla::report(VMLA_ERR_INVALID_ARG, "batch must be >= 1");
  if (cfg->dtype != VMLA_BF16) return vmla::report(VMLA_ERR_UNSUPPORTED, "the executor runs the bf16 fused path");
  const Sizes sz = sizes(*cfg, batch);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return vmla::report(VMLA_ERR_MISALIGNED, "workspace must be a 256-byte aligned device buffer");
  if (workspace_bytes < kSlots * sz.slot)
    return vmla::report(VMLA_ERR_INVALID_ARG, "workspace smaller than vmla_executor_workspace_bytes()");
  vmla_executor* ex = new (std::nothrow) vmla_executor();
  if (!ex) return vmla::report(VMLA_ERR_CUDA, "out of host memory");
  ex->cfg = *cfg;
  ex->batch = batch;
  ex->sz = sz;
  for (int s = 0; s < kSlots; ++s) ex->slot[s] = static_cast<uint8_t*>(workspace) + s * sz.slot;
  ex->compute = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamCreateWithFlags(&ex->h2d, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&ex->d2h, cudaStreamNonBlocking);
  for (int s = 0; e == cudaSuccess && s < kSlots; ++s) {
    e = cudaEventCreateWithFlags(&ex->h2d_done[s], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ex->compute_done[s], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ex->d2h_done[s], cudaEventDisableTiming);
  }
  if (e != cudaSuccess) {
    vmla_executor_destroy(ex);
    return vmla::report(VMLA_ERR_CUDA, cudaGetErrorString(e));
  }
  *out = ex;
  return VMLA_OK;
}

vmla_status vmla_executor_submit(vmla_executor* ex, vmla_cache* cache, const void* w_dkv_kr, const void* w_uk,
                                 const void* w_uv, const void* x_host, const void* q_nope_host,
                                 const void* q_rope_host, void* out_host) {
  if (!ex || !cache || !x_host || !q_nope_host || !q_rope_host || !out_host)
    return vmla::report(VMLA_ERR_INVALID_ARG, "executor, cache and host buffers must not be NULL");
  if (cache->batch != ex->batch) return vmla::report(VMLA_ERR_INVALID_ARG, "cache batch differs from the executor's");
  // everything the two calls below check on the host is checked here first, so that a refused step
  // enqueues nothing: no copy, no compress (which would advance frames_written and evict a frame)
  for (const void* p : {(const void*)cache->c, (const void*)cache->k_r, w_dkv_kr, w_uk, w_uv}) {
    if (!p) return vmla::report(VMLA_ERR_INVALID_ARG, "cache planes and weights must not be NULL");
    if (reinterpret_cast<uintptr_t>(p) & 15u)
      return vmla::report(VMLA_ERR_MISALIGNED, "cache planes and weights must be 16-byte aligned");
  }
  vmla_status chk = vmla_check_fused(&ex->cfg);
  if (chk != VMLA_OK) return chk;
  chk = vmla_check_attention_window(&ex->cfg, cache->frames_written + ex->cfg.chunk_frames,
                                    cache->frames_written, 1);
  if (chk != VMLA_OK) return chk;
  const int s = (int)(ex->submitted % kSlots);
  uint8_t* x = ex->slot[s];
  uint8_t* qn = x + round_up(ex->sz.x);
  uint8_t* qr = qn + round_up(ex->sz.qn);
  uint8_t* o = qr + round_up(ex->sz.qr);
  const bool reuse = ex->submitted >= kSlots;
  cudaError_t e = cudaSuccess;
  // inputs of this slot: free once the step that last read them has finished
  if (reuse) e = cudaStreamWaitEvent(ex->h2d, ex->compute_done[s], 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(x, x_host, ex->sz.x, cudaMemcpyHostToDevice, ex->h2d);
  if (e == cudaSuccess) e = cudaMemcpyAsync(qn, q_nope_host, ex->sz.qn, cudaMemcpyHostToDevice, ex->h2d);
  if (e == cudaSuccess) e = cudaMemcpyAsync(qr, q_rope_host, ex->sz.qr, cudaMemcpyHostToDevice, ex->h2d);
  if (e == cudaSuccess) e = cudaEventRecord(ex->h2d_done[s], ex->h2d);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ex->compute, ex->h2d_done[s], 0);
  // output of this slot: free once the copy of the step that last wrote it has finished
  if (e == cudaSuccess && reuse) e = cudaStreamWaitEvent(ex->compute, ex->d2h_done[s], 0);
  if (e != cudaSuccess) return vmla::report(VMLA_ERR_CUDA, cudaGetErrorString(e));
  const int64_t f0 = cache->frames_written;
  vmla_status st = vmla_compress_append(&ex->cfg, x, w_dkv_kr, f0, cache, ex->compute);
  if (st != VMLA_OK) return st;
  st = vmla_latent_attention_fused(&ex->cfg, qn, qr, w_uk, w_uv, cache, f0, 1, o, nullptr, ex->compute);
  if (st != VMLA_OK) return st;
  e = cudaEventRecord(ex->compute_done[s], ex->compute);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ex->d2h, ex->compute_done[s], 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(out_host, o, ex->sz.out, cudaMemcpyDeviceToHost, ex->d2h);
  if (e == cudaSuccess) e = cudaEventRecord(ex->d2h_done[s], ex->d2h);
  if (e != cudaSuccess) return vmla::report(VMLA_ERR_CUDA, cudaGetErrorString(e));
  ++ex->submitted;
  return VMLA_OK;
}

vmla_status vmla_executor_wait(vmla_executor* ex) {
  if (!ex) return vmla::report(VMLA_ERR_INVALID_ARG, "executor is NULL");
  cudaError_t e = cudaStreamSynchronize(ex->d2h);
  if (e == cudaSuccess) e = cudaStreamSynchronize(ex->h2d);
  if (e != cudaSuccess) return vmla::report(VMLA_ERR_CUDA, cudaGetErrorString(e));
  int32_t code = 0;
  return vmla_device_status(ex->compute, &code);
}

vmla_status vmla_executor_destroy(vmla_executor* ex) {
  if (!ex) return VMLA_OK;
  if (ex->d2h) cudaStreamSynchronize(ex->d2h);
  if (ex->h2d) cudaStreamSynchronize(ex->h2d);
  for (int s = 0; s < kSlots; ++s) {
    if (ex->h2d_done[s]) cudaEventDestroy(ex->h2d_done[s]);
    if (ex->compute_done[s]) cudaEventDestroy(ex->compute_done[s]);
    if (ex->d2h_done[s]) cudaEventDestroy(ex->d2h_done[s]);
  }
  if (ex->h2d) cudaStreamDestroy(ex->h2d);
  if (ex->d2h) cudaStreamDestroy(ex->d2h);
  delete ex;
  return VMLA_OK;
}

}  // extern "C"
