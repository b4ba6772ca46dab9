// topk.cu -- per-query top-K selection over indexer scores.
//
// Page "How GLM5.3 Sparse Attention Affects HBM Memory Usage", section "Lightning Indexer": the
// K highest indexer scores are kept per query (one selection shared by all heads); a query that
// sees fewer than K positions keeps all of them.  Ties go to the lower position, and the chosen
// positions are emitted in ascending order, so the result is unique and deterministic.
//
// Scores are compared through an order-preserving 32-bit key (larger score -> larger key, -0.0
// folded onto +0.0, NaN -> the lowest key and an error bit).  Each row is handled by a cluster of
// C CTAs (C = 1..8, chosen so that rows x C fills the SMs); CTA r owns a contiguous slice of the
// row's positions.
//
//   1. Threshold.  Every CTA reads the same strided sample of the row (8-score chunks; the loads
//      of its own slice are already in flight) and finds, by radix steps of 12-bit digits, a key
//      tau with at least js sample keys >= tau, where js is the sample rank expected to leave
//      ~1.15 K + 4 sqrt(K) scores of the row at or above tau.  Rows of at most kCap positions take
//      every score (no threshold).
//   2. Filter.  One coalesced pass over the slice appends every (key, position) with
//      score >= tau to shared memory (one shared atomic per warp and 256 scores), and the CTA
//      stores its candidate count into every CTA of the cluster.
//   3. Exact K-th key.  After a cluster barrier every CTA gathers all candidate keys of the row
//      through distributed shared memory and radix-selects the K-th largest key Tk among them.
//      If the row had at least K candidates, every score >= Tk is a candidate, so Tk is the
//      row's K-th key.  (Fewer than K or more than kCap candidates: CTA 0 runs the exact path
//      below over the whole row.)
//   4. Output.  Each CTA marks its candidates with key > Tk in a bitmap of its slice, counts its
//      ties (key == Tk) and stores both counts into every CTA; after a second cluster barrier it
//      knows how many selections and ties the lower slices hold, takes the lowest-position ties
//      up to the row's remaining quota and writes its marked positions, in ascending order, at
//      its offset in the output row.
// Exact path: a radix select over the row finds Tk and the number of ties to take, and an
// in-order pass over 8192-score chunks writes the positions.
// Every count is order-independent, so the result does not depend on the order of atomics.
#include "common.cuh"
#include "internal.h"

namespace dsa {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kDigit = 12;                 // radix digit width of the selections
constexpr int kHBins = 1 << kDigit;
constexpr int kCap = 6144;                 // candidates of one row (all CTAs of its cluster together)
constexpr int kMaxSlice = 1 << 17;         // positions one CTA's bitmap covers
constexpr int kMaxCluster = 8;
constexpr int kSample = 4096;              // sampled keys (512 chunks of 8)
constexpr int kPer = 16;                   // scores per thread per filter step

struct Smem {
  uint32_t bitmap[kMaxSlice / 32];      // selected positions of this CTA's slice
  uint32_t cand_key[kCap];              // this CTA's candidates (read by the whole cluster)
  uint32_t cand_pos[kCap];
  uint32_t pool[kCap];                  // the row's candidate keys, then this CTA's ties
  uint32_t hist[2][kHBins];             // radix histograms, alternating between steps
  uint32_t red[2 * kWarps];
  uint32_t wsum[kWarps];
  uint32_t warp_tot[kWarps + 1];
  uint32_t res[2][4];                   // digit, keys above it, keys in it
  uint32_t scal[12];
  uint32_t cnt_all[kMaxCluster];        // written by every CTA of the cluster: its candidates
  uint32_t above_all[kMaxCluster];      // ... its keys above Tk
  uint32_t ties_all[kMaxCluster];       // ... its keys equal to Tk
};
static_assert(kCap >= kSample, "the sample fits the candidate key buffer");

// ---------------------------------------------------------------------------------------------
// cluster primitives (thread-block clusters, distributed shared memory)
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_nctas() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_index() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

// Every thread of every CTA of the cluster arrives (release) / waits (acquire).
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_sync() {
  cluster_arrive();
  cluster_wait();
}

__device__ __forceinline__ uint32_t cluster_addr(const void* local, uint32_t rank) {
  uint32_t remote;
  asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  return remote;
}

// 32-bit load from the shared memory of CTA `rank` of this cluster, at the offset of `local`.
// Ordered after the last cluster barrier by that barrier's acquire; no compiler barrier here, so
// that several of these loads can be in flight at once.
__device__ __forceinline__ uint32_t ld_cluster_u32(const uint32_t* local, uint32_t rank) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr(local, rank)));
  return v;
}

// 32-bit store into the shared memory of CTA `rank`; made visible by the next cluster barrier.
__device__ __forceinline__ void st_cluster_u32(uint32_t* local, uint32_t rank, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr(local, rank)), "r"(v) : "memory");
}

// ---------------------------------------------------------------------------------------------
// keys, scans, radix selection
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t order_key(float f, bool& is_nan) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) {
    is_nan = true;
    return 0u;
  }
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inverse of order_key on the keys it produces: the float whose key is `key` (keys below the key
// of -inf map to a NaN pattern, which no comparison accepts).
__device__ __forceinline__ float key_to_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

__device__ __forceinline__ uint32_t warp_inclusive_scan(uint32_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// Exclusive prefix sum of `v` over the block; returns the prefix, writes the block total.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_tot, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t incl = warp_inclusive_scan(v);
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  uint32_t before = 0u, all = 0u;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const uint32_t x = warp_tot[w];
    before += w < warp ? x : 0u;
    all += x;
  }
  total = all;
  __syncthreads();  // warp_tot is reused by the next scan
  return before + incl - v;
}

// Clears both radix histograms (each thread its share).  Call before the first kth_key of a CTA;
// kth_key leaves them clear again.
__device__ __forceinline__ void clear_hists(Smem& S) {
  constexpr int kPerT = kHBins / kThreads;
#pragma unroll
  for (int b = 0; b < kPerT; ++b) {
    S.hist[0][threadIdx.x * kPerT + b] = 0u;
    S.hist[1][threadIdx.x * kPerT + b] = 0u;
  }
}

// j-th largest (1-based) of the keys that each(f) hands to f, over the block, by radix steps of
// 12-bit digits taken from the highest bit in which the keys differ (bits every key shares are
// skipped).  After each step only the keys in the chosen digit bin stay in play.
//   exact:  returns that key; *above = the number of keys strictly greater.
//   !exact: stops after the first step whose chosen bin holds at most `limit` keys and returns the
//           bin's lower edge (the undecided low bits zero): at least j keys are >= the result.
// j must not exceed the number of keys.  Three block barriers per step (histogram, warp sums,
// result); the histograms alternate between steps, so clearing one overlaps the other's use.
template <class Each>
__device__ uint32_t kth_key(Smem& S, uint32_t j, Each each, bool exact, uint32_t limit, uint32_t* above) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t a = 0xFFFFFFFFu, o = 0u;
  each([&](uint32_t key) {
    a &= key;
    o |= key;
  });
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    a &= __shfl_xor_sync(0xFFFFFFFFu, a, off);
    o |= __shfl_xor_sync(0xFFFFFFFFu, o, off);
  }
  if (lane == 0) {
    S.red[warp] = a;
    S.red[kWarps + warp] = o;
  }
  __syncthreads();
  a = 0xFFFFFFFFu;
  o = 0u;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    a &= S.red[w];
    o |= S.red[kWarps + w];
  }
  uint32_t fixed = ~(a ^ o);  // decided bits: those every key shares, then each chosen digit
  uint32_t prefix = a & fixed;
  uint32_t krem = j;
  int buf = 0;
  constexpr int kPerLane = kHBins / kThreads;  // bins per thread (8)
  constexpr int kPerWarp = kHBins / kWarps;    // bins per warp (256)
  while (fixed != 0xFFFFFFFFu) {
    const int hb = 31 - __clz(~fixed);
    const int lb = hb >= kDigit - 1 ? hb - (kDigit - 1) : 0;
    const uint32_t dmask = (2u << (hb - lb)) - 1u;
    uint32_t* hist = S.hist[buf];
    each([&](uint32_t key) {
      if ((key & fixed) == prefix) atomicAdd(&hist[(key >> lb) & dmask], 1u);
    });
#pragma unroll
    for (int b = 0; b < kPerLane; ++b) S.hist[buf ^ 1][tid * kPerLane + b] = 0u;
    __syncthreads();
    // warp w owns bins [kHBins - kPerWarp (w + 1), kHBins - kPerWarp w), lane l the kPerLane bins
    // below kHBins - kPerWarp w - kPerLane l: counts run downward from the top bin
    uint32_t h[kPerLane];
    uint32_t lsum = 0u;
    const int top = kHBins - 1 - warp * kPerWarp - lane * kPerLane;
#pragma unroll
    for (int b = 0; b < kPerLane; ++b) {
      h[b] = hist[top - b];
      lsum += h[b];
    }
    const uint32_t lincl = warp_inclusive_scan(lsum);
    if (lane == 31) S.wsum[warp] = lincl;
    __syncthreads();
    uint32_t wabove = 0u;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) wabove += w < warp ? S.wsum[w] : 0u;
    uint32_t abv = wabove + lincl - lsum;
    if (abv < krem && krem <= abv + lsum) {
#pragma unroll
      for (int b = 0; b < kPerLane; ++b) {
        if (abv < krem && krem <= abv + h[b]) {
          S.res[buf][0] = (uint32_t)(top - b);
          S.res[buf][1] = abv;
          S.res[buf][2] = h[b];
        }
        abv += h[b];
      }
    }
    __syncthreads();
    const uint32_t d = S.res[buf][0], d_above = S.res[buf][1], d_count = S.res[buf][2];
    prefix |= d << lb;
    fixed |= dmask << lb;
    krem -= d_above;
    buf ^= 1;
    if (!exact && d_count <= limit) break;
  }
  // the histogram of the last step is the dirty one: clear it for the next call (the next call
  // writes it only after a barrier that follows this)
#pragma unroll
  for (int b = 0; b < kPerLane; ++b) S.hist[buf ^ 1][tid * kPerLane + b] = 0u;
  if (above) *above = j - krem;
  return prefix & fixed;
}

// Keys held in registers: element e of this thread is valid when tid + e * kThreads < m.
template <int N>
struct RegKeys {
  uint32_t v[N];
  int m;
  template <class F>
  __device__ __forceinline__ void operator()(F f) const {
#pragma unroll
    for (int e = 0; e < N; ++e)
      if ((int)threadIdx.x + e * kThreads < m) f(v[e]);
  }
};

template <int N>
__device__ __forceinline__ RegKeys<N> load_keys(const uint32_t* src, int m, bool complement) {
  RegKeys<N> r;
  r.m = m;
#pragma unroll
  for (int e = 0; e < N; ++e) {
    const int i = threadIdx.x + e * kThreads;
    const uint32_t x = i < m ? src[i] : 0u;
    r.v[e] = complement ? ~x : x;
  }
  return r;
}

// Exact path over a whole row in global memory: radix select of Tk, then an in-order pass over
// chunks of kPer * kThreads scores (each thread takes kPer consecutive positions) with two
// block-wide prefix sums per chunk, one over ties and one over the positions taken.
__device__ void topk_exact(Smem& S, const float* row, int64_t n, int k, int32_t* out, bool& saw_nan) {
  clear_hists(S);
  __syncthreads();
  uint32_t above;
  auto each = [&](auto f) {
    for (int64_t i = threadIdx.x; i < n; i += kThreads) f(order_key(row[i], saw_nan));
  };
  const uint32_t tk = kth_key(S, (uint32_t)k, each, true, 0u, &above);
  const uint32_t need = (uint32_t)k - above;  // keys equal to tk to take, lowest positions first
  uint32_t base = 0u, eq_seen = 0u;
  for (int64_t c0 = 0; c0 < n; c0 += (int64_t)kPer * kThreads) {
    const int64_t p0 = c0 + (int64_t)threadIdx.x * kPer;
    uint32_t key[kPer];
    uint32_t eq = 0u;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      bool dummy = false;
      key[e] = p0 + e < n ? order_key(row[p0 + e], dummy) : 0u;
      eq += (p0 + e < n && key[e] == tk) ? 1u : 0u;
    }
    uint32_t eq_tot, take_tot;
    uint32_t eq_rank = eq_seen + block_exclusive_scan(eq, S.warp_tot, eq_tot);
    uint32_t mask = 0u;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      if (p0 + e < n) {
        if (key[e] > tk) {
          mask |= 1u << e;
        } else if (key[e] == tk) {
          if (eq_rank < need) mask |= 1u << e;
          ++eq_rank;
        }
      }
    }
    uint32_t at = base + block_exclusive_scan((uint32_t)__popc(mask), S.warp_tot, take_tot);
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      if (mask & (1u << e)) {
        if (at < (uint32_t)k) out[at] = (int32_t)(p0 + e);
        ++at;
      }
    }
    base += take_tot;
    eq_seen += eq_tot;
  }
}

// kPer scores of a slice for this thread, from 16-byte loads where the slice allows: element
// j sits at base + ((j / 4) * kThreads + tid) * 4 + j % 4.
__device__ __forceinline__ void load_batch(const float* srow, int len, int base, bool vec, float (&v)[kPer]) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int u = 0; u < kPer / 4; ++u) {
    const int i = base + (u * kThreads + tid) * 4;
    if (vec && i + 4 <= len) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(srow + i));
      v[4 * u] = f.x; v[4 * u + 1] = f.y; v[4 * u + 2] = f.z; v[4 * u + 3] = f.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) v[4 * u + e] = i + e < len ? srow[i + e] : 0.f;
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    topk_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ q_pos, int k,
                int32_t* __restrict__ idx, int* err) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31;
  griddep_launch_dependents();
  const uint32_t C = cluster_nctas(), r = cluster_rank();
  const int64_t t = cluster_index();
  griddep_wait();  // the scores come from the previous kernel of the stream
  int64_t n = (int64_t)q_pos[t] + 1;
  if (n > ld) {  // a row cannot hold more scores than its stride
    if (tid == 0 && r == 0) raise_error(err, DSA_DEVERR_REQUEST);
    n = ld;
  }
  int32_t* out = idx + t * k;
  if (n <= k) {  // dense: every visible position, then -1 padding
    for (int64_t j = (int64_t)r * kThreads + tid; j < k; j += (int64_t)C * kThreads) out[j] = j < n ? (int32_t)j : -1;
    return;
  }
  const float* row = scores + t * ld;
  bool saw_nan = false;
  if (tid == 0) S.scal[4] = 0u;  // NaN seen
  const int64_t per = (((n + C - 1) / C) + 31) & ~int64_t(31);
  if (per > kMaxSlice) {  // slices too long for the bitmap: exact path on one CTA
    if (r == 0) {
      topk_exact(S, row, n, k, out, saw_nan);
      if (saw_nan) S.scal[4] = 1u;
      __syncthreads();
      if (tid == 0 && S.scal[4]) raise_error(err, DSA_DEVERR_NAN_SCORE);
    }
    return;
  }
  const int64_t lo = min(n, (int64_t)r * per);
  const int64_t hi = min(n, lo + per);
  const int len = (int)(hi - lo);
  const int words = (len + 31) >> 5;
  const float* srow = row + lo;
  const bool vec = ((reinterpret_cast<uintptr_t>(srow) & 15u) == 0);
  constexpr int kStep = kPer * kThreads;
  float v[kPer];
  load_batch(srow, len, 0, vec, v);  // the first batch of this slice, in flight during step 1
  for (int w = tid; w < words; w += kThreads) S.bitmap[w] = 0u;
  clear_hists(S);
  if (tid == 0) {
    S.scal[5] = 0u;  // candidates of this CTA
    S.scal[6] = 0u;  // ties of this CTA
    S.scal[7] = 0u;  // keys above Tk in this CTA
  }

  // 1. threshold from a strided sample (identical in every CTA of the cluster)
  const bool take_all = n <= kCap;
  float tau_f = -INFINITY;
  if (!take_all) {
    constexpr int kChunks = kSample / 8;
    constexpr int kSPT = kSample / kThreads;
    RegKeys<kSPT> smp;
    smp.m = kSample;
    float sv[kSPT];
#pragma unroll
    for (int e = 0; e < kSPT; ++e) {
      const int s = tid + e * kThreads;
      const int64_t p = (((int64_t)(s >> 3) * n / kChunks) & ~int64_t(7)) + (s & 7);
      sv[e] = row[p];
    }
#pragma unroll
    for (int e = 0; e < kSPT; ++e) smp.v[e] = order_key(sv[e], saw_nan);
    __syncthreads();  // histograms cleared
    const float rk = (float)k * (float)kSample / (float)n;  // sample rank of the row's K-th score
    int js = (int)ceilf(1.15f * rk + 4.f * sqrtf(rk) + 8.f);
    js = min(js, kSample);
    const uint32_t tau = kth_key(S, (uint32_t)js, smp, false, (uint32_t)(js / 8 + 2), nullptr);
    tau_f = key_to_float(tau);
  }
  __syncthreads();

  // 2. filter: append (key, position) of every score >= tau in this slice; the next batch's loads
  //    are issued before the current batch is processed
  for (int base = 0; base < len; base += kStep) {
    float vn[kPer];
    if (base + kStep < len) load_batch(srow, len, base + kStep, vec, vn);
    uint32_t mask = 0u;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = base + ((j >> 2) * kThreads + tid) * 4 + (j & 3);
      const bool valid = i < len;
      saw_nan |= valid && (v[j] != v[j]);
      const bool pass = valid && (take_all || v[j] >= tau_f);
      mask |= (uint32_t)pass << j;
    }
    const uint32_t c = (uint32_t)__popc(mask);
    const uint32_t incl = warp_inclusive_scan(c);
    const uint32_t tot = __shfl_sync(0xFFFFFFFFu, incl, 31);
    if (tot) {
      uint32_t wbase = 0u;
      if (lane == 0) wbase = atomicAdd(&S.scal[5], tot);
      uint32_t at = __shfl_sync(0xFFFFFFFFu, wbase, 0) + incl - c;
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        if (mask & (1u << j)) {
          if (at < (uint32_t)kCap) {
            bool dummy = false;
            S.cand_key[at] = order_key(v[j], dummy);
            S.cand_pos[at] = (uint32_t)(lo + base + ((j >> 2) * kThreads + tid) * 4 + (j & 3));
          }
          ++at;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) v[j] = vn[j];
  }
  __syncthreads();
  if (tid < (int)C) st_cluster_u32(&S.cnt_all[r], (uint32_t)tid, S.scal[5]);
  cluster_sync();  // A: every CTA's candidates and counts are visible to the cluster

  uint32_t m = 0u;  // the row's candidates
#pragma unroll
  for (int q = 0; q < kMaxCluster; ++q) m += q < (int)C ? S.cnt_all[q] : 0u;
  if (m < (uint32_t)k || m > (uint32_t)kCap) {
    // the threshold missed (too high, or too many scores tie at it): exact path on CTA 0
    cluster_sync();  // no CTA reads another's shared memory after this point
    if (r == 0) topk_exact(S, row, n, k, out, saw_nan);
    if (saw_nan) S.scal[4] = 1u;
    __syncthreads();
    if (tid == 0 && S.scal[4]) raise_error(err, DSA_DEVERR_NAN_SCORE);
    return;
  }

  // 3. exact K-th key among the row's candidates (gathered from every CTA of the cluster)
  constexpr int kKPT = kCap / kThreads;
  RegKeys<kKPT> cand;
  cand.m = (int)m;
  if (C > 1) {
    uint32_t pre[kMaxCluster];  // candidate offsets of the cluster's CTAs
    pre[0] = 0u;
#pragma unroll
    for (int q = 1; q < kMaxCluster; ++q) pre[q] = pre[q - 1] + (q - 1 < (int)C ? S.cnt_all[q - 1] : 0u);
#pragma unroll
    for (int e = 0; e < kKPT; ++e) {
      const uint32_t i = (uint32_t)(tid + e * kThreads);
      uint32_t src = 0u, off = 0u;
#pragma unroll
      for (int q = 1; q < kMaxCluster; ++q) {
        if (pre[q] <= i && q < (int)C) {
          src = (uint32_t)q;
          off = pre[q];
        }
      }
      cand.v[e] = i < m ? ld_cluster_u32(&S.cand_key[i - off], src) : 0u;
    }
  } else {
    cand = load_keys<kKPT>(S.cand_key, (int)m, false);
  }
  uint32_t above;
  const uint32_t tk = kth_key(S, (uint32_t)k, cand, true, 0u, &above);
  const uint32_t need = (uint32_t)k - above;  // keys equal to tk to take, lowest positions first

  // 4. this CTA's keys above tk go to the bitmap; its ties are listed
  const uint32_t mine = S.cnt_all[r];
  for (uint32_t c0 = 0; c0 < mine; c0 += kThreads) {
    const uint32_t c = c0 + tid;
    uint32_t key = 0u, pos = 0u;
    if (c < mine) {
      key = S.cand_key[c];
      pos = S.cand_pos[c];
    }
    const bool gt = c < mine && key > tk;
    if (gt) atomicOr(&S.bitmap[(pos - lo) >> 5], 1u << ((pos - lo) & 31));
    if (c < mine && key == tk) {
      const uint32_t e = atomicAdd(&S.scal[6], 1u);
      S.pool[e] = pos;
    }
    const uint32_t b = __ballot_sync(0xFFFFFFFFu, gt);
    if (lane == 0 && b) atomicAdd(&S.scal[7], (uint32_t)__popc(b));
  }
  __syncthreads();
  if (tid < (int)C) {
    st_cluster_u32(&S.above_all[r], (uint32_t)tid, S.scal[7]);
    st_cluster_u32(&S.ties_all[r], (uint32_t)tid, S.scal[6]);
  }
  cluster_sync();  // B: every CTA's counts are visible
  cluster_arrive();  // this CTA reads no other CTA's shared memory from here on

  // output offset of this CTA, and the ties it takes (the lowest positions of the row win)
  uint32_t offset = 0u, ties_before = 0u;
#pragma unroll
  for (int q = 0; q < kMaxCluster; ++q) {
    if (q < (int)r) {
      const uint32_t ti = S.ties_all[q];
      const uint32_t qq = need > ties_before ? min(ti, need - ties_before) : 0u;
      offset += S.above_all[q] + qq;
      ties_before += ti;
    }
  }
  const uint32_t nties = S.ties_all[r];
  const uint32_t quota = need > ties_before ? min(nties, need - ties_before) : 0u;
  if (quota > 0u) {
    uint32_t pos_cut = 0xFFFFFFFFu;  // take tied positions <= pos_cut
    if (quota < nties) {
      // the `quota` lowest positions among the ties: select on the complemented position
      const RegKeys<kKPT> tp = load_keys<kKPT>(S.pool, (int)nties, true);
      pos_cut = ~kth_key(S, quota, tp, true, 0u, nullptr);
    }
    for (uint32_t e = tid; e < nties; e += kThreads) {
      const uint32_t pos = S.pool[e];
      if (pos <= pos_cut) atomicOr(&S.bitmap[(pos - lo) >> 5], 1u << ((pos - lo) & 31));
    }
    __syncthreads();
  }
  // ascending output: prefix sum of per-thread popcounts over contiguous word ranges
  const int wpt = (words + kThreads - 1) / kThreads;
  const int w0 = min(words, tid * wpt);
  const int w1 = min(words, w0 + wpt);
  uint32_t cnt = 0u;
  for (int w = w0; w < w1; ++w) cnt += (uint32_t)__popc(S.bitmap[w]);
  uint32_t total;
  uint32_t at = offset + block_exclusive_scan(cnt, S.warp_tot, total);
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = S.bitmap[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1u;
      if (at < (uint32_t)k) out[at] = (int32_t)(lo + w * 32 + b);
      ++at;
    }
  }
  if (saw_nan) S.scal[4] = 1u;  // benign race: every writer stores 1
  __syncthreads();
  if (tid == 0 && S.scal[4]) raise_error(err, DSA_DEVERR_NAN_SCORE);
  cluster_wait();  // no CTA exits while another may still read its shared memory
}

}  // namespace

cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* q_pos, int T, int k,
                        int32_t* idx, int* err, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // CTAs per row: fill the SMs when there are few rows; keep every slice within the bitmap
  int C = 1;
  while (C < kMaxCluster && (int64_t)T * 2 * C <= sms && ld > (int64_t)C * 4096) C *= 2;
  while (C < kMaxCluster && (ld + C - 1) / C > kMaxSlice) C *= 2;
  const int smem = (int)sizeof(Smem);
  e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attrs[2];
  const cudaLaunchConfig_t cfg = launch_config(dim3((unsigned)((int64_t)T * C)), dim3(kThreads), (size_t)smem, s,
                                               attrs, (unsigned)C);
  return cudaLaunchKernelEx(&cfg, topk_kernel, scores, ld, q_pos, k, idx, err);
}

}  // namespace dsa
