// generic.cu -- CUDA-core kernels for any indexer / MLA shape and dtype.
//
// These run the shapes the tensor-core kernels do not cover (for example the tiny fp32 layer:
// indexer 4 heads x 32, MLA 8 heads over 64 + 16) and serve as the bring-up path.  They follow
// the definitions directly:
//   indexer (page "How GLM5.3 Sparse Attention Affects HBM Memory Usage", section "Lightning
//   Indexer"): score = sum_h w_h * ReLU(q_h . khat), khat = key * per-token scale for e4m3
//   (e4m3 queries likewise: qhat = code * per-(query, head) scale);
//   sparse MLA (same page, "Sparse MLA"): softmax over the selected rows of scale * q . row,
//   output = softmax-weighted sum of the rows' first d_v dims, computed with a running max.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {

namespace {

constexpr int kGenericTile = 128;

__device__ __forceinline__ bool lookup_row(const dsa_batch& b, const dsa_paged_cache& c, int req,
                                           int64_t pos, int64_t* row, int* err) {
  int64_t lblk = pos / c.block_size;
  if (lblk >= b.max_blocks) {
    raise_error(err, DSA_DEVERR_BLOCK_ID);
    return false;
  }
  int32_t blk = b.block_table[(int64_t)req * b.max_blocks + lblk];
  if (blk < 0 || blk >= c.num_blocks) {
    raise_error(err, DSA_DEVERR_BLOCK_ID);
    return false;
  }
  *row = (int64_t)blk * c.block_size + pos % c.block_size;
  return true;
}

// grid (ceil(max_context / 128), T), block 128: one thread per key position.
__global__ void indexer_generic_kernel(IndexerArgs a) {
  extern __shared__ float sm[];
  float* qs = sm;                       // [Hi * Di]
  float* ws = sm + (size_t)a.Hi * a.Di;  // [Hi]
  const int t = blockIdx.y;
  const int req = a.batch.q_req[t];
  const int pos = a.batch.q_pos[t];
  if (req < 0 || req >= a.batch.num_reqs || pos < 0 || pos >= a.batch.max_context) {
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_error(a.err, DSA_DEVERR_REQUEST);
    return;
  }
  const int64_t s0 = (int64_t)blockIdx.x * kGenericTile;
  if (s0 > pos) return;  // uniform over the block
  for (int e = threadIdx.x; e < a.Hi * a.Di; e += blockDim.x) {
    const float qsc = a.q_scale ? a.q_scale[(int64_t)t * a.Hi + e / a.Di] : 1.0f;  // e4m3 queries
    qs[e] = load_elem(a.q, a.q_dtype, (int64_t)t * a.Hi * a.Di + e) * qsc;
  }
  for (int h = threadIdx.x; h < a.Hi; h += blockDim.x) ws[h] = a.w[(int64_t)t * a.Hi + h];
  __syncthreads();
  const int64_t s = s0 + threadIdx.x;
  if (s > pos) return;
  int64_t row;
  if (!lookup_row(a.batch, a.keys, req, s, &row, a.err)) return;
  const float sc = (a.keys.dtype == DSA_E4M3) ? a.keys.scale[row] : 1.0f;
  const int64_t kbase = row * a.Di;
  float score = 0.0f;
  for (int h = 0; h < a.Hi; ++h) {
    float dot = 0.0f;
    const float* qh = qs + (size_t)h * a.Di;
    for (int i = 0; i < a.Di; ++i) dot = fmaf(qh[i], load_elem(a.keys.data, a.keys.dtype, kbase + i), dot);
    dot *= sc;
    score = fmaf(ws[h], fmaxf(dot, 0.0f), score);
  }
  a.scores[(int64_t)t * a.ld + s] = score;
  if (a.key_hist) {  // the selection's threshold histogram
    bool nan = false;
    atomicAdd(&a.key_hist[(int64_t)t * kKeyBins + key_digit(order_key(score, nan))], 1u);
  }
}

constexpr int kMlaThreads = 128;
constexpr int kMaxVPerThread = 8;  // d_v <= 1024

__device__ __forceinline__ float block_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float tot = 0.0f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += red[w];
  return tot;
}

// grid (H, T), block 128: one CTA per (query, head), rows visited in order with a running max.
__global__ void mla_generic_kernel(MlaArgs a) {
  extern __shared__ float sm[];
  const int dqk = a.d_v + a.d_rope;
  float* qs = sm;          // [dqk]
  float* red = sm + dqk;   // [32]
  const int h = blockIdx.x, t = blockIdx.y;
  const int req = a.batch.q_req[t];
  const int pos = a.batch.q_pos[t];
  const int64_t qo = ((int64_t)t * a.H + h);
  if (req < 0 || req >= a.batch.num_reqs || pos < 0 || pos >= a.batch.max_context) {
    if (threadIdx.x == 0 && h == 0) raise_error(a.err, DSA_DEVERR_REQUEST);
    return;
  }
  for (int i = threadIdx.x; i < dqk; i += blockDim.x) qs[i] = load_elem(a.q, a.dtype, qo * dqk + i);
  __syncthreads();
  float m = -INFINITY, l = 0.0f;
  float o[kMaxVPerThread];
#pragma unroll
  for (int c = 0; c < kMaxVPerThread; ++c) o[c] = 0.0f;
  // without a selection (idx null) every visible position is attended: slot j holds position j
  const int nslots = a.idx ? a.k : min(a.k, pos + 1);
  for (int j = 0; j < nslots; ++j) {
    const int p = a.idx ? a.idx[(int64_t)t * a.k + j] : j;
    if (p == -1) continue;
    if (p < -1 || p > pos) {
      if (threadIdx.x == 0 && h == 0) raise_error(a.err, DSA_DEVERR_INDEX);
      continue;
    }
    int64_t row;
    if (!lookup_row(a.batch, a.latent, req, p, &row, threadIdx.x == 0 ? a.err : nullptr)) continue;
    const int64_t rb = row * dqk;
    float part = 0.0f;
    for (int i = threadIdx.x; i < dqk; i += blockDim.x)
      part = fmaf(qs[i], load_elem(a.latent.data, a.latent.dtype, rb + i), part);
    const float logit = block_sum(part, red) * a.scale;
    const float m_new = fmaxf(m, logit);
    const float corr = expf(m - m_new);
    const float pe = expf(logit - m_new);
    l = l * corr + pe;
#pragma unroll
    for (int c = 0; c < kMaxVPerThread; ++c) {
      const int col = threadIdx.x + c * blockDim.x;
      if (col < a.d_v) o[c] = fmaf(pe, load_elem(a.latent.data, a.latent.dtype, rb + col), o[c] * corr);
    }
    m = m_new;
  }
  const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll
  for (int c = 0; c < kMaxVPerThread; ++c) {
    const int col = threadIdx.x + c * blockDim.x;
    if (col >= a.d_v) continue;
    const float v = o[c] * inv;
    if (a.dtype == DSA_F32)
      static_cast<float*>(a.out)[qo * a.d_v + col] = v;
    else
      static_cast<__nv_bfloat16*>(a.out)[qo * a.d_v + col] = __float2bfloat16_rn(v);
  }
  if (a.lse && threadIdx.x == 0) a.lse[qo] = l > 0.0f ? m + logf(l) : -INFINITY;
}

}  // namespace

cudaError_t launch_indexer_generic(const IndexerArgs& a, cudaStream_t s) {
  const int T = a.batch.num_queries;
  if (T == 0) return cudaSuccess;
  dim3 grid((a.batch.max_context + kGenericTile - 1) / kGenericTile, T);
  size_t smem = sizeof(float) * ((size_t)a.Hi * a.Di + a.Hi);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(indexer_generic_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  indexer_generic_kernel<<<grid, kGenericTile, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_mla_generic(const MlaArgs& a, cudaStream_t s) {
  const int T = a.batch.num_queries;
  if (T == 0) return cudaSuccess;
  dim3 grid(a.H, T);
  size_t smem = sizeof(float) * ((size_t)a.d_v + a.d_rope + 32);
  mla_generic_kernel<<<grid, kMlaThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
