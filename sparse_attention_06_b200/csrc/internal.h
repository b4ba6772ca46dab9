// internal.h -- launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dsa.h"

namespace dsa {

// Arguments of an indexer launch after host validation.
struct IndexerArgs {
  const void* q;
  int q_dtype;
  const float* q_scale;  // [T, Hi] for e4m3 queries, else null
  int Hi, Di;
  const float* w;
  dsa_paged_cache keys;
  dsa_batch batch;
  float* scores;
  int64_t ld;
  uint32_t* key_hist;  // [T, kKeyBins] order-key digit counts to add to, or null
  int* err;
};

struct MlaArgs {
  const void* q;
  int dtype;
  int H, d_v, d_rope;
  dsa_paged_cache latent;
  dsa_batch batch;
  const int32_t* idx;
  int k;
  float scale;
  void* out;
  float* lse;
  void* workspace;
  size_t workspace_bytes;
  int* err;
};

// generic CUDA-core path (any shape)
cudaError_t launch_indexer_generic(const IndexerArgs& a, cudaStream_t s);
cudaError_t launch_mla_generic(const MlaArgs& a, cudaStream_t s);

// radix top-k (any k <= 4096); key_hist (or null): [T, kKeyBins] digit counts of each row's
// scores, read to place the threshold and left zeroed
cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* q_pos, int T, int k,
                        int32_t* idx, uint32_t* key_hist, int* err, cudaStream_t s);

// tcgen05 paths (production shapes)
cudaError_t launch_indexer_tc_decode(const IndexerArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_indexer_tc_prefill(const IndexerArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_mla_tc(const MlaArgs& a, int nsplit, int num_sms, cudaStream_t s);
int mla_tc_num_splits(int T, int k, int num_sms);
size_t mla_tc_workspace_bytes(int T, int H, int d_v, int nsplit);

// Launch configuration with programmatic stream serialization (the kernel may start while the
// previous kernel of the stream finishes; every kernel here waits for it with griddepcontrol.wait
// before its first global-memory access) and, when cluster_x > 0, thread-block clusters of
// cluster_x CTAs.  `attrs` must hold two entries and outlive the launch call.
inline cudaLaunchConfig_t launch_config(dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                        cudaLaunchAttribute* attrs, unsigned cluster_x = 0) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  if (cluster_x > 0) {
    attrs[1].id = cudaLaunchAttributeClusterDimension;
    attrs[1].val.clusterDim.x = cluster_x;
    attrs[1].val.clusterDim.y = 1;
    attrs[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  return cfg;
}

// detail text returned by dsa_last_error_message() on this host thread
void set_last_error_message(const char* msg);

// the calling thread's current CUDA context (NULL when none is current)
CUcontext current_cuda_context();

// SM count of the current device (false when there is no usable device)
bool current_device_sms(int* num_sms);

// How an MLA call runs: on the tensor-core kernels or the generic ones, with how many key splits
// per query, and the workspace bytes of the split partials (0 with one split or the generic path).
struct MlaPlan {
  bool tensor_cores;
  int nsplit;
  size_t workspace_bytes;
};
MlaPlan mla_plan(bool decode, const void* q, int32_t q_dtype, int32_t H, int32_t d_v, int32_t d_rope,
                 const dsa_paged_cache& latent, int32_t T, int32_t k, const void* out, int num_sms);

// diagnostic: one thread waits on an mbarrier that nothing arrives on, bounded by limit_cycles
cudaError_t launch_bounded_wait_selftest(long long limit_cycles, int* err, cudaStream_t s);
cudaError_t launch_gather_rate_selftest(const dsa_paged_cache& latent, const int32_t* rows, int tiles, int ctas,
                                        int64_t* cycles, int* err, cudaStream_t s);

// tensor-map encoding through the driver entry point (no link-time libcuda dependency)
bool encode_tmap_2d(void* tmap_out, const void* base, int elem_bytes, uint64_t inner,
                    uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                    uint32_t box_outer, bool swizzle128);

}  // namespace dsa
