// mla_noalloc.cu -- sparse MLA decode for callers that cannot allocate device memory.
//
// dsa_sparse_mla_decode splits each query's selected rows across CTAs and needs caller-provided
// workspace for the partial results.  Some callers cannot call cudaMalloc at the point where
// they run the layer: code that runs inside another framework's memory pool with no allocator
// handle, plugins whose host process forbids allocation after start-up, or code paths that must
// not allocate because allocation can synchronise the device.  For them this file provides
// dsa_sparse_mla_decode_noalloc, which takes the same inputs and outputs but keeps the partial
// results in a fixed scratch array that lives in the library itself.
//
// The scratch is a file-scope __device__ array of kScratchBytes (32 MiB).  It exists on a device
// once the library's scratch module is loaded there: under lazy module loading (the CUDA default)
// that happens at the first call of this entry point on the device, whose address lookup loads
// the module, reserves the 32 MiB and may synchronise the device.  Make that first call during
// set-up, before timing-critical work and before any stream capture; later calls do neither.  The
// array then stays reserved until the process exits.  All calls on a device share it, so two calls
// whose kernels overlap on the GPU (different streams, no ordering) race on it; calls on one stream
// are ordered and safe.  Each call overwrites every partial it later reads, so nothing in the array
// has to start at zero and the previous call's contents are harmless.
#include <cuda_runtime.h>
#include <stdio.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

constexpr size_t kScratchBytes = 32ull << 20;

// Device-side scratch for the split-K partial outputs and log-sum-exps.
static __device__ __align__(256) unsigned char g_mla_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
struct ScratchEntry {
  CUcontext ctx;
  void* ptr;
};
ScratchEntry g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  In host code the array's name is
// only a host-side stand-in, so the real address is looked up with cudaGetSymbolAddress: once per
// device (the set-up done by the first call there), and again if the device's context has changed
// since (a device reset releases the old array).
void* scratch_address(int dev) {
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  ScratchEntry& e = g_scratch[dev];
  const CUcontext ctx = current_cuda_context();
  if (!e.ptr || !ctx || ctx != e.ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mla_scratch) != cudaSuccess) return nullptr;
    e.ptr = p;
    e.ctx = current_cuda_context();
  }
  return e.ptr;
}

}  // namespace
}  // namespace dsa

extern "C" dsa_status dsa_sparse_mla_decode_noalloc(const void* q, int32_t q_dtype, int32_t H,
                                                    int32_t d_v, int32_t d_rope,
                                                    const dsa_paged_cache* latent,
                                                    const dsa_batch* batch, const int32_t* idx,
                                                    int32_t k, float softmax_scale, void* out,
                                                    float* lse, dsa_stream stream) {
  int dev = 0;
  int sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= dsa::kMaxDevices ||
      !dsa::current_device_sms(&sms)) {
    dsa::set_last_error_message("dsa_sparse_mla_decode_noalloc: no usable CUDA device");
    return DSA_ERR_CUDA;
  }
  // the scratch this call needs: the split plan of the workspace entry point for the same call
  // (arguments it would reject need none here; it rejects them below)
  size_t need = 0;
  if (batch && latent && batch->num_queries > 0)
    need = dsa::mla_plan(true, q, q_dtype, H, d_v, d_rope, *latent, batch->num_queries, k, out, sms)
               .workspace_bytes;
  if (need > dsa::kScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "dsa_sparse_mla_decode_noalloc: these sizes need %zu bytes of split scratch, more than "
             "the library's fixed %zu bytes; call dsa_sparse_mla_decode with a workspace instead",
             need, dsa::kScratchBytes);
    dsa::set_last_error_message(msg);
    return DSA_ERR_INVALID_ARG;
  }
  void* scratch = dsa::scratch_address(dev);
  if (!scratch) {
    dsa::set_last_error_message("dsa_sparse_mla_decode_noalloc: cannot resolve the scratch address");
    return DSA_ERR_CUDA;
  }
  return dsa_sparse_mla_decode(q, q_dtype, H, d_v, d_rope, latent, batch, idx, k, softmax_scale,
                               out, lse, scratch, dsa::kScratchBytes, stream);
}
