// dsa_api.cu -- the C ABI declared in include/dsa.h: host-side argument checks, the device
// error word, kernel selection and tensor-map encoding.  All compute happens in the kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"

// The library's one piece of device state: a word of DSA_DEVERR_* bits per device.
__device__ int g_dsa_device_error;

namespace dsa {
namespace {

thread_local char g_msg[256];
constexpr int kMaxDevices = 64;

dsa_status fail(dsa_status st, const char* fmt, const char* detail = "") {
  snprintf(g_msg, sizeof g_msg, fmt, detail);
  return st;
}

std::mutex g_mu;
std::atomic<long long> g_launches{0};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The calling thread's current CUDA context (NULL when none is current yet).
CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
  return c;
}

struct DeviceEntry {
  CUcontext ctx;
  int* err;
  int num_sms;
};
DeviceEntry g_dev[kMaxDevices];

// Device address of the error word and the SM count of the current device, looked up once per
// device and looked up again whenever the device's context is not the one they were found in
// (after a device reset the old addresses are gone).
bool device_state(int** err, int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceEntry& d = g_dev[dev];
  CUcontext ctx = current_context();
  if (!d.err || !ctx || ctx != d.ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dsa_device_error) != cudaSuccess) return false;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    d.num_sms = sms;
    d.err = static_cast<int*>(p);
    d.ctx = current_context();
  }
  *err = d.err;
  *num_sms = d.num_sms;
  return true;
}

dsa_status cuda_status(cudaError_t e, const char* where, int kernels = 0) {
  if (e == cudaSuccess) {
    g_launches += kernels;
    return DSA_OK;
  }
  snprintf(g_msg, sizeof g_msg, "%s: %s", where, cudaGetErrorString(e));
  return DSA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dsa_status check_batch(const dsa_batch* b) {
  if (!b) return fail(DSA_ERR_INVALID_ARG, "batch is NULL%s");
  if (b->num_queries < 0 || b->num_reqs < 0) return fail(DSA_ERR_INVALID_ARG, "negative batch size%s");
  if (b->num_queries == 0) return DSA_OK;
  if (!b->q_req || !b->q_pos || !b->block_table)
    return fail(DSA_ERR_INVALID_ARG, "batch has a NULL device array%s");
  if (b->num_reqs < 1 || b->max_blocks < 1 || b->max_context < 1)
    return fail(DSA_ERR_INVALID_ARG, "batch needs num_reqs, max_blocks, max_context >= 1%s");
  if (b->query_group < 1 || b->num_queries % b->query_group != 0)
    return fail(DSA_ERR_INVALID_ARG, "query_group must be >= 1 and divide num_queries%s");
  return DSA_OK;
}

dsa_status check_cache(const dsa_paged_cache* c, const dsa_batch* b, const char* name) {
  if (!c) return fail(DSA_ERR_INVALID_ARG, "%s cache is NULL", name);
  if (!c->data) return fail(DSA_ERR_INVALID_ARG, "%s cache data is NULL", name);
  if (c->num_blocks < 1 || c->block_size < 1 || c->dim < 1)
    return fail(DSA_ERR_INVALID_ARG, "%s cache has an empty shape", name);
  if (c->dtype != DSA_F32 && c->dtype != DSA_BF16 && c->dtype != DSA_E4M3)
    return fail(DSA_ERR_INVALID_ARG, "%s cache dtype is unknown", name);
  if (c->dtype == DSA_E4M3 && !c->scale)
    return fail(DSA_ERR_INVALID_ARG, "%s cache is e4m3 but has no scale", name);
  if (!aligned16(c->data)) return fail(DSA_ERR_INVALID_ARG, "%s cache data is not 16-byte aligned", name);
  if ((int64_t)b->max_blocks * c->block_size < (int64_t)b->max_context)
    return fail(DSA_ERR_INVALID_ARG, "%s: max_blocks * block_size < max_context", name);
  return DSA_OK;
}

// ---------------------------------------------------------------------------------------------
// tensor maps
// ---------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

void set_last_error_message(const char* msg) { snprintf(g_msg, sizeof g_msg, "%s", msg); }

CUcontext current_cuda_context() { return current_context(); }

bool current_device_sms(int* num_sms) {
  int* err;
  return device_state(&err, num_sms);
}

MlaPlan mla_plan(bool decode, const void* q, int32_t q_dtype, int32_t H, int32_t d_v, int32_t d_rope,
                 const dsa_paged_cache& latent, int32_t T, int32_t k, const void* out, int num_sms) {
  MlaPlan pl{false, 1, 0};
  pl.tensor_cores = (H == 128 || H == 64) && d_v == 512 && d_rope == 64 && q_dtype == DSA_BF16 &&
                    latent.block_size == 64 && aligned16(q) && aligned16(out) && aligned16(latent.data);
  if (pl.tensor_cores && T > 0) {
    pl.nsplit = decode ? mla_tc_num_splits(T, k, num_sms) : 1;
    pl.workspace_bytes = mla_tc_workspace_bytes(T, H, d_v, pl.nsplit);
  }
  return pl;
}

bool encode_tmap_2d(void* tmap_out, const void* base, int elem_bytes, uint64_t inner,
                    uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                    uint32_t box_outer, bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  CUtensorMapDataType dt = elem_bytes == 1   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                           : elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                             : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(reinterpret_cast<CUtensorMap*>(tmap_out), dt, 2, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace dsa

using namespace dsa;

extern "C" {

int32_t dsa_abi_version(void) { return DSA_ABI_VERSION; }

int64_t dsa_kernel_launch_count(void) { return g_launches.load(); }

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported combination";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_DEVICE_FAULT: return "device-detected fault";
  }
  return "unknown status";
}

const char* dsa_last_error_message(void) { return g_msg; }

dsa_status dsa_get_device_error(int32_t* code, dsa_stream stream) {
  if (!code) return fail(DSA_ERR_INVALID_ARG, "code is NULL%s");
  int* err;
  int sms;
  if (!device_state(&err, &sms)) return fail(DSA_ERR_CUDA, "no CUDA device%s");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, err, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e, "dsa_get_device_error");
  *code = host;
  return host ? DSA_ERR_DEVICE_FAULT : DSA_OK;
}

dsa_status dsa_clear_device_error(dsa_stream stream) {
  int* err;
  int sms;
  if (!device_state(&err, &sms)) return fail(DSA_ERR_CUDA, "no CUDA device%s");
  return cuda_status(cudaMemsetAsync(err, 0, sizeof(int), static_cast<cudaStream_t>(stream)),
                     "dsa_clear_device_error");
}

// The indexer call behind dsa_indexer_scores; *hist_built tells whether the launched kernel adds
// the scores to key_hist (the generic kernel and the tensor-core kernel for one query per tile
// with bf16 keys do; the others leave it untouched).
static dsa_status indexer_scores_impl(const void* q, int32_t q_dtype, const float* q_scale, int32_t Hi,
                                      int32_t Di, const float* w, const dsa_paged_cache* keys,
                                      const dsa_batch* batch, float* scores, int64_t ld,
                                      uint32_t* key_hist, dsa_stream stream, bool* hist_built) {
  *hist_built = false;
  dsa_status st = check_batch(batch);
  if (st != DSA_OK) return st;
  if (batch->num_queries == 0) return DSA_OK;
  if ((st = check_cache(keys, batch, "indexer key")) != DSA_OK) return st;
  if (!q || !w || !scores) return fail(DSA_ERR_INVALID_ARG, "indexer: NULL q, w or scores%s");
  if (Hi < 1 || Di < 1 || Hi * Di > 16384) return fail(DSA_ERR_INVALID_ARG, "indexer: Hi*Di must be in [1, 16384]%s");
  if (keys->dim != Di) return fail(DSA_ERR_INVALID_ARG, "indexer: key dim != Di%s");
  if (q_dtype != DSA_F32 && q_dtype != DSA_BF16 && q_dtype != DSA_E4M3)
    return fail(DSA_ERR_INVALID_ARG, "indexer: q dtype must be f32, bf16 or e4m3%s");
  if (q_dtype == DSA_E4M3 && !q_scale) return fail(DSA_ERR_INVALID_ARG, "indexer: e4m3 q needs q_scale%s");
  if (ld < batch->max_context) return fail(DSA_ERR_INVALID_ARG, "indexer: ld < max_context%s");
  if (key_hist && !aligned16(key_hist)) return fail(DSA_ERR_INVALID_ARG, "indexer: key_hist not 16-byte aligned%s");
  int* err;
  int sms;
  if (!device_state(&err, &sms)) return fail(DSA_ERR_CUDA, "no CUDA device%s");
  IndexerArgs a{q, q_dtype, q_dtype == DSA_E4M3 ? q_scale : nullptr, Hi, Di, w, *keys, *batch, scores, ld,
                key_hist, err};
  // tensor-core operand pairs: bf16 x bf16, e4m3 keys x bf16 queries, e4m3 x e4m3
  const bool tc_pair = (q_dtype == DSA_BF16 && (keys->dtype == DSA_BF16 || keys->dtype == DSA_E4M3)) ||
                       (q_dtype == DSA_E4M3 && keys->dtype == DSA_E4M3);
  const bool tc_shape = Hi == 64 && Di == 128 && tc_pair && keys->block_size == 64 && aligned16(q) &&
                        (ld % 4) == 0 && aligned16(scores);
  cudaError_t e;
  if (tc_shape && batch->query_group % 4 == 0) {
    e = launch_indexer_tc_prefill(a, sms, static_cast<cudaStream_t>(stream));
  } else if (tc_shape) {
    e = launch_indexer_tc_decode(a, sms, static_cast<cudaStream_t>(stream));
    *hist_built = key_hist && keys->dtype == DSA_BF16;
  } else {
    e = launch_indexer_generic(a, static_cast<cudaStream_t>(stream));
    *hist_built = key_hist != nullptr;
  }
  return cuda_status(e, "dsa_indexer_scores launch", 1);
}

dsa_status dsa_indexer_scores(const void* q, int32_t q_dtype, const float* q_scale, int32_t Hi,
                              int32_t Di, const float* w, const dsa_paged_cache* keys,
                              const dsa_batch* batch, float* scores, int64_t ld,
                              uint32_t* key_hist, dsa_stream stream) {
  bool built;
  return indexer_scores_impl(q, q_dtype, q_scale, Hi, Di, w, keys, batch, scores, ld, key_hist, stream, &built);
}

dsa_status dsa_topk_select(const float* scores, int64_t ld, const int32_t* q_pos, int32_t T,
                           int32_t k, int32_t* idx, uint32_t* key_hist, dsa_stream stream) {
  if (T < 0) return fail(DSA_ERR_INVALID_ARG, "topk: T < 0%s");
  if (T == 0) return DSA_OK;
  if (!scores || !q_pos || !idx) return fail(DSA_ERR_INVALID_ARG, "topk: NULL pointer%s");
  if (k < 1 || k > 4096) return fail(DSA_ERR_INVALID_ARG, "topk: k must be in [1, 4096]%s");
  if (ld < 1) return fail(DSA_ERR_INVALID_ARG, "topk: ld < 1%s");
  if (key_hist && !aligned16(key_hist)) return fail(DSA_ERR_INVALID_ARG, "topk: key_hist not 16-byte aligned%s");
  int* err;
  int sms;
  if (!device_state(&err, &sms)) return fail(DSA_ERR_CUDA, "no CUDA device%s");
  return cuda_status(launch_topk(scores, ld, q_pos, T, k, idx, key_hist, err, static_cast<cudaStream_t>(stream)),
                     "dsa_topk_select launch", 1);
}

dsa_status dsa_indexer_topk(const void* q, int32_t q_dtype, const float* q_scale, int32_t Hi,
                            int32_t Di, const float* w, const dsa_paged_cache* keys,
                            const dsa_batch* batch, int32_t k, float* scores, int64_t ld,
                            int32_t* idx, void* workspace, size_t workspace_bytes,
                            dsa_stream stream) {
  dsa_status st = check_batch(batch);
  if (st != DSA_OK) return st;
  if (batch->num_queries == 0) return DSA_OK;
  if (!idx) return fail(DSA_ERR_INVALID_ARG, "indexer_topk: idx is NULL%s");
  if (k < 1 || k > 4096) return fail(DSA_ERR_INVALID_ARG, "indexer_topk: k must be in [1, 4096]%s");
  uint32_t* key_hist = nullptr;
  if (workspace) {
    if (workspace_bytes < dsa_indexer_topk_workspace_size(batch->num_queries) || !aligned16(workspace))
      return fail(DSA_ERR_INVALID_ARG, "indexer_topk: workspace too small or not 16-byte aligned%s");
    key_hist = static_cast<uint32_t*>(workspace);
  }
  bool built = false;
  if ((st = indexer_scores_impl(q, q_dtype, q_scale, Hi, Di, w, keys, batch, scores, ld, key_hist, stream,
                                &built)) != DSA_OK)
    return st;
  // the selection takes the histogram only when the indexer kernel built it (else it samples)
  return dsa_topk_select(scores, ld, batch->q_pos, batch->num_queries, k, idx, built ? key_hist : nullptr, stream);
}

size_t dsa_indexer_topk_workspace_size(int32_t num_queries) {
  return num_queries > 0 ? (size_t)num_queries * kKeyBins * sizeof(uint32_t) : 0;
}

static dsa_status mla_common(bool decode, const void* q, int32_t q_dtype, int32_t H, int32_t d_v,
                             int32_t d_rope, const dsa_paged_cache* latent, const dsa_batch* batch,
                             const int32_t* idx, int32_t k, float softmax_scale, void* out,
                             float* lse, void* workspace, size_t workspace_bytes,
                             dsa_stream stream) {
  dsa_status st = check_batch(batch);
  if (st != DSA_OK) return st;
  if (batch->num_queries == 0) return DSA_OK;
  if ((st = check_cache(latent, batch, "latent")) != DSA_OK) return st;
  if (!q || !out) return fail(DSA_ERR_INVALID_ARG, "mla: NULL q or out%s");
  if (!idx && k < batch->max_context)
    return fail(DSA_ERR_INVALID_ARG, "mla: without a selection (idx NULL) k must be >= max_context%s");
  if (H < 1 || d_v < 1 || d_rope < 0) return fail(DSA_ERR_INVALID_ARG, "mla: bad H, d_v or d_rope%s");
  if (d_v > 1024 || d_v + d_rope > 4096) return fail(DSA_ERR_INVALID_ARG, "mla: d_v <= 1024 and d_v + d_rope <= 4096 required%s");
  if (latent->dim != d_v + d_rope) return fail(DSA_ERR_INVALID_ARG, "mla: latent dim != d_v + d_rope%s");
  if (q_dtype != DSA_F32 && q_dtype != DSA_BF16) return fail(DSA_ERR_INVALID_ARG, "mla: dtype must be f32 or bf16%s");
  if (latent->dtype != q_dtype) return fail(DSA_ERR_INVALID_ARG, "mla: latent dtype != q dtype%s");
  if (k < 1 || k > 65536) return fail(DSA_ERR_INVALID_ARG, "mla: k must be in [1, 65536]%s");
  if (!(softmax_scale > 0.0f)) return fail(DSA_ERR_INVALID_ARG, "mla: softmax_scale must be > 0%s");
  int* err;
  int sms;
  if (!device_state(&err, &sms)) return fail(DSA_ERR_CUDA, "no CUDA device%s");
  MlaArgs a{q, q_dtype, H, d_v, d_rope, *latent, *batch, idx, k, softmax_scale, out, lse,
            workspace, workspace_bytes, err};
  const int T = batch->num_queries;
  const MlaPlan pl = mla_plan(decode, q, q_dtype, H, d_v, d_rope, *latent, T, k, out, sms);
  cudaError_t e;
  int kernels = 1;
  if (pl.tensor_cores) {
    const size_t need = pl.workspace_bytes;
    if (need > 0 && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)))
      return fail(DSA_ERR_INVALID_ARG, "mla: workspace missing, too small or not 256-byte aligned%s");
    kernels = pl.nsplit > 1 ? 2 : 1;
    e = launch_mla_tc(a, pl.nsplit, sms, static_cast<cudaStream_t>(stream));
  } else {
    e = launch_mla_generic(a, static_cast<cudaStream_t>(stream));
  }
  return cuda_status(e, decode ? "dsa_sparse_mla_decode launch" : "dsa_sparse_mla_prefill launch",
                     kernels);
}

dsa_status dsa_sparse_mla_decode(const void* q, int32_t q_dtype, int32_t H, int32_t d_v,
                                 int32_t d_rope, const dsa_paged_cache* latent,
                                 const dsa_batch* batch, const int32_t* idx, int32_t k,
                                 float softmax_scale, void* out, float* lse, void* workspace,
                                 size_t workspace_bytes, dsa_stream stream) {
  return mla_common(true, q, q_dtype, H, d_v, d_rope, latent, batch, idx, k, softmax_scale, out,
                    lse, workspace, workspace_bytes, stream);
}

dsa_status dsa_sparse_mla_prefill(const void* q, int32_t q_dtype, int32_t H, int32_t d_v,
                                  int32_t d_rope, const dsa_paged_cache* latent,
                                  const dsa_batch* batch, const int32_t* idx, int32_t k,
                                  float softmax_scale, void* out, float* lse, void* workspace,
                                  size_t workspace_bytes, dsa_stream stream) {
  return mla_common(false, q, q_dtype, H, d_v, d_rope, latent, batch, idx, k, softmax_scale, out,
                    lse, workspace, workspace_bytes, stream);
}

dsa_status dsa_selftest_bounded_wait(int64_t limit_cycles, dsa_stream stream) {
  if (limit_cycles < 1 || limit_cycles > kWaitCycles)
    return fail(DSA_ERR_INVALID_ARG, "selftest: limit_cycles must be in [1, 4e9]%s");
  int* err;
  int sms;
  if (!device_state(&err, &sms)) return fail(DSA_ERR_CUDA, "no CUDA device%s");
  return cuda_status(launch_bounded_wait_selftest(limit_cycles, err, static_cast<cudaStream_t>(stream)),
                     "dsa_selftest_bounded_wait launch", 1);
}

dsa_status dsa_selftest_gather_rate(const dsa_paged_cache* latent, const int32_t* rows, int32_t tiles_per_cta,
                                    int32_t num_ctas, int64_t* cycles, dsa_stream stream) {
  if (!latent || !latent->data || !rows || !cycles) return fail(DSA_ERR_INVALID_ARG, "gather rate: NULL argument%s");
  if (latent->dtype != DSA_BF16 || latent->block_size != 64 || latent->dim != 576 || latent->num_blocks < 1 ||
      (reinterpret_cast<uintptr_t>(latent->data) & 15u))
    return fail(DSA_ERR_INVALID_ARG, "gather rate: latent must be bf16, 64-token blocks of 576, 16-byte aligned%s");
  if ((uint64_t)latent->num_blocks * 64u >= 0x7FFFFFFFull)
    return fail(DSA_ERR_INVALID_ARG, "gather rate: pool rows must fit 31 bits%s");
  if (tiles_per_cta < 1 || tiles_per_cta > 65536 || num_ctas < 1 || num_ctas > 1024)
    return fail(DSA_ERR_INVALID_ARG, "gather rate: tiles_per_cta in [1, 65536], num_ctas in [1, 1024]%s");
  int* err;
  int sms;
  if (!device_state(&err, &sms)) return fail(DSA_ERR_CUDA, "no CUDA device%s");
  return cuda_status(launch_gather_rate_selftest(*latent, rows, tiles_per_cta, num_ctas, cycles, err,
                                                 static_cast<cudaStream_t>(stream)),
                     "dsa_selftest_gather_rate launch", 1);
}

size_t dsa_mla_workspace_size(int32_t num_queries, int32_t H, int32_t d_v, int32_t k) {
  if (num_queries <= 0 || (H != 128 && H != 64) || d_v != 512 || k < 1) return 0;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return mla_tc_workspace_bytes(num_queries, H, d_v, mla_tc_num_splits(num_queries, k, sms));
}

}  // extern "C"
