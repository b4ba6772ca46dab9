// topk.cu -- per-query top-K selection over indexer scores.
//
// Page "How GLM5.3 Sparse Attention Affects HBM Memory Usage", section "Lightning Indexer": the
// K highest indexer scores are kept per query (one selection shared by all heads); a query that
// sees fewer than K positions keeps all of them.  Ties go to the lower position, and the chosen
// positions are emitted in ascending order, so the result is unique and deterministic.
//
// Method (one CTA of 1024 threads per query row):
//   1. every score is mapped to an order-preserving 32-bit key (larger score -> larger key,
//      -0.0 folded onto +0.0, NaN -> lowest key plus an error bit);
//   2. three radix passes (11 + 11 + 10 bits, shared-memory histograms) find the exact key value
//      Tk of the K-th largest element and how many elements equal to Tk must be taken (need);
//   3. one in-order pass over the row takes every key > Tk and the first `need` keys == Tk,
//      using block-wide prefix counts, and writes their positions in ascending order.
// All counts are order-independent, so the result does not depend on atomic ordering.
#include "common.cuh"
#include "internal.h"

namespace dsa {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;

__device__ __forceinline__ uint32_t order_key(float f, bool& is_nan) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) {
    is_nan = true;
    return 0u;
  }
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum of `v` over the block; returns the prefix, writes the block total.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_tot,
                                                         uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t wv = lane < kWarps ? warp_tot[lane] : 0u;
    uint32_t wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xFFFFFFFFu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < kWarps) warp_tot[lane] = wi - wv;  // exclusive warp offsets
    if (lane == 31) warp_tot[kWarps] = wi;        // block total
  }
  __syncthreads();
  uint32_t res = warp_tot[warp] + incl - v;
  total = warp_tot[kWarps];
  __syncthreads();
  return res;
}

__global__ void __launch_bounds__(kThreads) topk_kernel(const float* __restrict__ scores,
                                                        int64_t ld, const int32_t* __restrict__ q_pos,
                                                        int k, int32_t* __restrict__ idx, int* err) {
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t warp_tot[kWarps + 1];
  __shared__ uint32_t s_digit, s_above;
  __shared__ int s_nan;

  const int t = blockIdx.x;
  int64_t n = (int64_t)q_pos[t] + 1;
  if (n > ld) {  // a row cannot hold more scores than its stride
    if (threadIdx.x == 0) raise_error(err, DSA_DEVERR_REQUEST);
    n = ld;
  }
  int32_t* out = idx + (int64_t)t * k;
  if (n <= k) {
    for (int j = threadIdx.x; j < k; j += kThreads) out[j] = j < n ? j : -1;
    return;
  }
  const float* row = scores + (int64_t)t * ld;
  if (threadIdx.x == 0) s_nan = 0;

  uint32_t prefix = 0u, hmask = 0u, krem = (uint32_t)k;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  bool saw_nan = false;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass];
    const uint32_t dmask = (1u << widths[pass]) - 1u;
    const int nbins = 1 << widths[pass];
    for (int b = threadIdx.x; b < kBins; b += kThreads) hist[b] = 0u;
    __syncthreads();
    for (int64_t i = threadIdx.x; i < n; i += kThreads) {
      uint32_t key = order_key(row[i], saw_nan);
      if ((key & hmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane L owns bins [L*per, (L+1)*per); find the digit holding the krem-th largest key
      const int lane = threadIdx.x;
      const int per = nbins / 32;
      uint32_t mine = 0u;
      for (int b = 0; b < per; ++b) mine += hist[lane * per + b];
      // suffix sums over lanes (bins above and including lane L)
      uint32_t suf = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_down_sync(0xFFFFFFFFu, suf, o);
        if (lane + o < 32) suf += y;
      }
      const uint32_t above_lane = suf - mine;  // bins of higher lanes
      const bool hit = suf >= krem && above_lane < krem;
      const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, hit);
      if (hit && lane == 31 - __clz(ballot)) {
        uint32_t run = above_lane;
        for (int b = per - 1; b >= 0; --b) {
          const uint32_t h = hist[lane * per + b];
          if (run + h >= krem) {
            s_digit = (uint32_t)(lane * per + b);
            s_above = run;
            break;
          }
          run += h;
        }
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    hmask |= dmask << shift;
    krem -= s_above;
    __syncthreads();
  }
  if (saw_nan) s_nan = 1;  // benign race: every writer stores 1
  const uint32_t tk = prefix;
  const uint32_t need = krem;  // number of keys equal to tk to take, lowest positions first

  uint32_t base = 0u, eq_seen = 0u;
  for (int64_t c0 = 0; c0 < n; c0 += kThreads) {
    const int64_t i = c0 + threadIdx.x;
    bool dummy = false;
    const uint32_t key = i < n ? order_key(row[i], dummy) : 0u;
    const bool valid = i < n;
    const uint32_t eq = (valid && key == tk) ? 1u : 0u;
    uint32_t eq_tot;
    const uint32_t eq_rank = block_exclusive_scan(eq, warp_tot, eq_tot);
    const uint32_t take = (valid && (key > tk || (eq && eq_seen + eq_rank < need))) ? 1u : 0u;
    uint32_t take_tot;
    const uint32_t at = block_exclusive_scan(take, warp_tot, take_tot);
    if (take && base + at < (uint32_t)k) out[base + at] = (int32_t)i;
    base += take_tot;
    eq_seen += eq_tot;
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_nan) raise_error(err, DSA_DEVERR_NAN_SCORE);
}

}  // namespace

cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* q_pos, int T, int k,
                        int32_t* idx, int* err, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  topk_kernel<<<T, kThreads, 0, s>>>(scores, ld, q_pos, k, idx, err);
  return cudaGetLastError();
}

}  // namespace dsa
