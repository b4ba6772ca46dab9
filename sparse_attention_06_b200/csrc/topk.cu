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
//   1. Threshold.  With the row's order-key digit histogram (12-bit digits: the sign, exponent
//      and three mantissa bits of the score; the indexer builds it as it writes the scores) every
//      CTA finds the digit bin that holds the row's K-th key, and tau is that bin's lower edge: the
//      keys >= tau are exactly the keys of that bin and above, whose number the histogram gives.
//      Without a histogram, or when that number exceeds the candidate capacity, every CTA reads
//      the same strided sample of the row (8-score chunks) and finds, by radix steps of 12-bit
//      digits, a key tau with at least js sample keys >= tau, js = rk + 4 sqrt(rk) + 8 where rk
//      is the sample rank of the row's K-th score: the count of sample keys above that score is
//      about binomial with mean rk, so fewer than K candidates (and the exact path below) needs a
//      deviation of more than four standard deviations (~1e-6 per row).  Rows of at most kCap
//      positions take every score (no threshold).  A histogram that does not describe the row
//      (one left dirty) only leads to a wrong tau, which step 2's count catches (exact path).
//      Each CTA clears its share of the histogram row once every CTA has used it.
//   2. Filter.  One coalesced pass over the slice appends every (key, position) with
//      score >= tau to shared memory (one shared atomic per warp and 512 scores), and the CTA
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
//
// Code size.  With few rows the kernel is one serial chain of short phases, each run once per
// launch, so fetching instructions is a large part of its time.  The radix selection is therefore
// one out-of-line function over keys in shared memory, shared by the sample, the candidates and
// the ties; reductions use redux.sync; the exact fallback path is out of line as well.
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
constexpr int kPer = 16;                   // scores per thread per step of the exact path
constexpr int kFPer = 16;                  // scores per thread per filter batch
static_assert(kHBins == 8 * kThreads, "each thread scans 8 histogram bins");
static_assert(kCap >= kSample, "the sample fits the key pool");
static_assert(kKeyBins == 8 * kThreads, "each thread reads 8 bins of a digit histogram row");
static_assert(kKeyBins % (4 * kMaxCluster) == 0, "every CTA clears whole 16-byte pieces of a histogram row");

struct Smem {
  uint32_t bitmap[kMaxSlice / 32];      // selected positions of this CTA's slice
  uint32_t cand_key[kCap];              // this CTA's candidates (read by the whole cluster)
  uint32_t cand_pos[kCap];
  uint32_t pool[kCap];                  // sample keys, then the row's candidate keys, then this CTA's ties
  alignas(16) uint32_t hist[2][kHBins]; // radix histograms, alternating between steps
  uint32_t red[2 * kWarps];
  uint32_t wsum[kWarps];
  uint32_t warp_tot[kWarps];
  uint32_t res[2][4];                   // digit, keys above it, keys in it
  uint32_t scal[12];
  uint32_t cnt_all[kMaxCluster];        // written by every CTA of the cluster: its candidates
  uint32_t above_all[kMaxCluster];      // ... its keys above Tk
  uint32_t ties_all[kMaxCluster];       // ... its keys equal to Tk
};

extern __shared__ __align__(16) uint8_t topk_smem[];
__device__ __forceinline__ Smem& smem() { return *reinterpret_cast<Smem*>(topk_smem); }

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
// Arrive without release semantics: only for an arrive that publishes no memory operation.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_sync() {
  cluster_arrive();
  cluster_wait();
}

__device__ __forceinline__ uint32_t cluster_addr(const void* local, uint32_t rank) {
  uint32_t remote;
  asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  return remote;
}

// Four consecutive 32-bit words (16-byte aligned) from the shared memory of CTA `rank`.
__device__ __forceinline__ uint4 ld_cluster_u32x4(const uint32_t* local, uint32_t rank) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(cluster_addr(local, rank)));
  return v;
}

// 32-bit store into the shared memory of CTA `rank`; made visible by the next cluster barrier.
__device__ __forceinline__ void st_cluster_u32(uint32_t* local, uint32_t rank, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr(local, rank)), "r"(v) : "memory");
}

// ---------------------------------------------------------------------------------------------
// keys, scans, radix selection
// ---------------------------------------------------------------------------------------------
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
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t& total) {
  Smem& S = smem();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t incl = warp_inclusive_scan(v);
  if (lane == 31) S.warp_tot[warp] = incl;
  __syncthreads();
  const uint32_t x = lane < kWarps ? S.warp_tot[lane] : 0u;
  total = __reduce_add_sync(0xFFFFFFFFu, x);
  const uint32_t before = __reduce_add_sync(0xFFFFFFFFu, lane < warp ? x : 0u);
  __syncthreads();  // warp_tot is reused by the next scan
  return before + incl - v;
}

// Clears both radix histograms (each thread its 8 bins of each).  Call before the first kth_key
// of a CTA; kth_key leaves them clear again.
__device__ __forceinline__ void clear_hist(int which) {
  uint4* h = reinterpret_cast<uint4*>(smem().hist[which]) + 2 * threadIdx.x;
  h[0] = make_uint4(0u, 0u, 0u, 0u);
  h[1] = make_uint4(0u, 0u, 0u, 0u);
}

// Keys held in registers: element e of this thread is key tid + e * kThreads, valid below m.
struct RegKeys {
  static constexpr int N = kCap / kThreads;
  uint32_t v[N];
  int m;
  template <class F>
  __device__ __forceinline__ void operator()(F f) const {
#pragma unroll
    for (int e = 0; e < N; ++e)
      if ((int)threadIdx.x + e * kThreads < m) f(v[e]);
  }
};

// Keys in shared memory: the first m entries of the pool, or of this CTA's candidate keys.  They
// are loaded into registers once per selection (load()), so that the histogram passes issue
// their atomics back to back.
struct SmemKeys {
  int m;
  bool cand;
  __device__ __forceinline__ RegKeys load() const {
    const uint32_t* keys = cand ? smem().cand_key : smem().pool;
    RegKeys r;
    r.m = m;
#pragma unroll
    for (int e = 0; e < RegKeys::N; ++e) {
      const int i = threadIdx.x + e * kThreads;
      r.v[e] = i < m ? keys[i] : 0u;
    }
    return r;
  }
};

// The keys of a whole row in global memory (exact path); a NaN score sets the CTA's NaN flag.
struct RowKeys {
  const float* row;
  int64_t n;
  __device__ __forceinline__ RowKeys load() const { return *this; }
  template <class F>
  __device__ __forceinline__ void operator()(F f) const {
    bool nan = false;
    for (int64_t i = threadIdx.x; i < n; i += kThreads) f(order_key(row[i], nan));
    if (nan) smem().scal[4] = 1u;  // benign race: every writer stores 1
  }
};

struct Kth {
  uint32_t key;    // the selected key (exact) or the threshold (not exact)
  uint32_t above;  // exact: keys strictly greater than `key`
};

// j-th largest (1-based) of the keys that src(f) hands to f, over the block, by radix steps of
// 12-bit digits taken from the highest bit in which the keys differ (bits every key shares are
// skipped).  After each step only the keys in the chosen digit bin stay in play.
//   exact:  returns that key and the number of keys strictly greater.
//   !exact: stops after the first step whose chosen bin holds at most `limit` keys and returns the
//           bin's lower edge (the undecided low bits zero): at least j keys are >= the result.
// j must not exceed the number of keys.  Three block barriers per step (histogram, warp sums,
// result); the histograms alternate between steps, so clearing one overlaps the other's use.
template <class Src>
__device__ __noinline__ Kth kth_key(Src keys, uint32_t j, bool exact, uint32_t limit) {
  Smem& S = smem();
  const auto src = keys.load();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t a = 0xFFFFFFFFu, o = 0u;
  src([&](uint32_t key) {
    a &= key;
    o |= key;
  });
  a = __reduce_and_sync(0xFFFFFFFFu, a);
  o = __reduce_or_sync(0xFFFFFFFFu, o);
  if (lane == 0) {
    S.red[warp] = a;
    S.red[kWarps + warp] = o;
  }
  __syncthreads();
  a = __reduce_and_sync(0xFFFFFFFFu, lane < kWarps ? S.red[lane] : 0xFFFFFFFFu);
  o = __reduce_or_sync(0xFFFFFFFFu, lane < kWarps ? S.red[kWarps + lane] : 0u);
  uint32_t fixed = ~(a ^ o);  // decided bits: those every key shares, then each chosen digit
  uint32_t prefix = a & fixed;
  uint32_t krem = j;
  int buf = 0;
  while (fixed != 0xFFFFFFFFu) {
    const int hb = 31 - __clz(~fixed);
    const int lb = hb >= kDigit - 1 ? hb - (kDigit - 1) : 0;
    const uint32_t dmask = (2u << (hb - lb)) - 1u;
    uint32_t* hist = S.hist[buf];
    src([&](uint32_t key) {
      if ((key & fixed) == prefix) atomicAdd(&hist[(key >> lb) & dmask], 1u);
    });
    clear_hist(buf ^ 1);
    __syncthreads();
    // thread tid owns the 8 bins [8 (kThreads - 1 - tid), 8 (kThreads - tid)); counts run downward
    // from the top bin (thread 0) to bin 0 (the last thread)
    const uint4* mine = reinterpret_cast<const uint4*>(hist) + 2 * (kThreads - 1 - tid);
    const uint4 lo4 = mine[0], hi4 = mine[1];
    const uint32_t h[8] = {hi4.w, hi4.z, hi4.y, hi4.x, lo4.w, lo4.z, lo4.y, lo4.x};
    const uint32_t lsum = (lo4.x + lo4.y) + (lo4.z + lo4.w) + (hi4.x + hi4.y) + (hi4.z + hi4.w);
    const uint32_t lincl = warp_inclusive_scan(lsum);
    if (lane == 31) S.wsum[warp] = lincl;
    __syncthreads();
    uint32_t abv = __reduce_add_sync(0xFFFFFFFFu, lane < warp ? S.wsum[lane] : 0u) + lincl - lsum;
    if (abv < krem && krem <= abv + lsum) {
      const int top = kHBins - 1 - 8 * tid;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
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
  clear_hist(buf ^ 1);
  return Kth{prefix & fixed, j - krem};
}

// Exact path over a whole row in global memory: radix select of Tk, then an in-order pass over
// chunks of kPer * kThreads scores (each thread takes kPer consecutive positions) with two
// block-wide prefix sums per chunk, one over ties and one over the positions taken.
__device__ __noinline__ void topk_exact(const float* row, int64_t n, int k, int32_t* out) {
  clear_hist(0);
  clear_hist(1);
  __syncthreads();
  const Kth tk = kth_key(RowKeys{row, n}, (uint32_t)k, true, 0u);
  const uint32_t need = (uint32_t)k - tk.above;  // keys equal to Tk to take, lowest positions first
  uint32_t base = 0u, eq_seen = 0u;
  for (int64_t c0 = 0; c0 < n; c0 += (int64_t)kPer * kThreads) {
    const int64_t p0 = c0 + (int64_t)threadIdx.x * kPer;
    uint32_t key[kPer];
    uint32_t eq = 0u;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      bool dummy = false;
      key[e] = p0 + e < n ? order_key(row[p0 + e], dummy) : 0u;
      eq += (p0 + e < n && key[e] == tk.key) ? 1u : 0u;
    }
    uint32_t eq_tot, take_tot;
    uint32_t eq_rank = eq_seen + block_exclusive_scan(eq, eq_tot);
    uint32_t mask = 0u;
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      if (p0 + e < n) {
        if (key[e] > tk.key) {
          mask |= 1u << e;
        } else if (key[e] == tk.key) {
          if (eq_rank < need) mask |= 1u << e;
          ++eq_rank;
        }
      }
    }
    uint32_t at = base + block_exclusive_scan((uint32_t)__popc(mask), take_tot);
    while (mask) {
      const int e = __ffs(mask) - 1;
      mask &= mask - 1u;
      if (at < (uint32_t)k) out[at] = (int32_t)(p0 + e);
      ++at;
    }
    base += take_tot;
    eq_seen += eq_tot;
  }
}

// max(a, b), NaN when either is NaN
__device__ __forceinline__ float max_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// v[j] for a j known only at run time, without indexing the register array
__device__ __forceinline__ float pick(const float (&v)[kFPer], int j) {
  float x = v[0];
#pragma unroll
  for (int e = 1; e < kFPer; ++e) x = j == e ? v[e] : x;
  return x;
}

// kFPer scores of a slice for this thread, from 16-byte loads where the slice allows: element
// j sits at base + ((j / 4) * kThreads + tid) * 4 + j % 4.
__device__ __forceinline__ void load_batch(const float* srow, int len, int base, bool vec, float (&v)[kFPer]) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int u = 0; u < kFPer / 4; ++u) {
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

// Place of the k-th largest key of a row in its order-key digit histogram (global memory, one
// row of kKeyBins counters): the bin b holding it, the keys in higher bins and the keys in b.
// Thread tid owns the 8 bins [8 (kThreads - 1 - tid), 8 (kThreads - tid)), so counts run
// downward from the top bin (thread 0) to bin 0 (the last thread).  found = false when the
// histogram holds fewer than k keys.
struct HistPlace {
  uint32_t bin, above, count;
  bool found;
};
__device__ __noinline__ HistPlace place_in_histogram(const uint32_t* __restrict__ hrow, uint32_t k) {
  Smem& S = smem();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint4* mine = reinterpret_cast<const uint4*>(hrow) + 2 * (kThreads - 1 - tid);
  const uint4 lo4 = __ldg(mine), hi4 = __ldg(mine + 1);
  const uint32_t h[8] = {hi4.w, hi4.z, hi4.y, hi4.x, lo4.w, lo4.z, lo4.y, lo4.x};
  const uint32_t lsum = (lo4.x + lo4.y) + (lo4.z + lo4.w) + (hi4.x + hi4.y) + (hi4.z + hi4.w);
  const uint32_t lincl = warp_inclusive_scan(lsum);
  if (lane == 31) S.wsum[warp] = lincl;
  if (tid == 0) S.res[0][3] = 0u;  // found
  __syncthreads();
  uint32_t abv = __reduce_add_sync(0xFFFFFFFFu, lane < warp ? S.wsum[lane] : 0u) + lincl - lsum;
  if (abv < k && k <= abv + lsum) {
    const int top = kKeyBins - 1 - 8 * tid;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      if (abv < k && k <= abv + h[b]) {
        S.res[0][0] = (uint32_t)(top - b);
        S.res[0][1] = abv;
        S.res[0][2] = h[b];
        S.res[0][3] = 1u;
      }
      abv += h[b];
    }
  }
  __syncthreads();
  HistPlace r{S.res[0][0], S.res[0][1], S.res[0][2], S.res[0][3] != 0u};
  __syncthreads();  // res is reused by the radix selections
  return r;
}

__global__ void __launch_bounds__(kThreads, 1)
    topk_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ q_pos, int k,
                int32_t* __restrict__ idx, uint32_t* __restrict__ key_hist, int* err) {
  Smem& S = smem();
  const int tid = threadIdx.x, lane = tid & 31;
  griddep_launch_dependents();
  const uint32_t C = cluster_nctas(), r = cluster_rank();
  const int64_t t = cluster_index();
  // warm the address translation of this row (a prefetch reads nothing that the previous kernel
  // may still write: the loads below come after the wait)
  if (tid == 0) asm volatile("prefetch.global.L2 [%0];" ::"l"(scores + t * ld + min((int64_t)r * 4096, ld - 1)));
  griddep_wait();  // the scores (and their histogram) come from the previous kernel of the stream
  int64_t n = (int64_t)q_pos[t] + 1;
  if (n > ld) {  // a row cannot hold more scores than its stride
    if (tid == 0 && r == 0) raise_error(err, DSA_DEVERR_REQUEST);
    n = ld;
  }
  int32_t* out = idx + t * k;
  // The row's digit histogram (when given): read for the threshold below, then this CTA clears its
  // share of it, once no CTA of the cluster reads it any more, so that it starts at zero next call.
  uint32_t* hrow = key_hist ? key_hist + t * kKeyBins : nullptr;
  auto clear_histogram_share = [&]() {
    if (!hrow) return;
    const int per = kKeyBins / (int)C;
    uint4* h4 = reinterpret_cast<uint4*>(hrow + (int)r * per);
    for (int e = tid; e < per / 4; e += kThreads) h4[e] = make_uint4(0u, 0u, 0u, 0u);
  };
  if (n <= k) {  // dense: every visible position, then -1 padding
    for (int64_t j = (int64_t)r * kThreads + tid; j < k; j += (int64_t)C * kThreads) out[j] = j < n ? (int32_t)j : -1;
    clear_histogram_share();
    return;
  }
  const float* row = scores + t * ld;
  if (tid == 0) S.scal[4] = 0u;  // NaN seen
  if (n > (int64_t)kMaxSlice * C) {  // slices too long for the bitmap: exact path on one CTA
    clear_histogram_share();
    if (r == 0) {
      __syncthreads();  // the NaN flag is clear
      topk_exact(row, n, k, out);
      __syncthreads();
      if (tid == 0 && S.scal[4]) raise_error(err, DSA_DEVERR_NAN_SCORE);
    }
    return;
  }
  // slices of a multiple of 32 positions (whole bitmap words), at most kMaxSlice; n < 2^20 here
  const int nn = (int)n;
  const int per = (int)((((uint32_t)nn + C - 1u) / C + 31u) & ~31u);
  const int lo = min(nn, (int)r * per);
  const int len = min(nn, lo + per) - lo;
  const int words = (len + 31) >> 5;
  const float* srow = row + lo;
  const bool vec = ((reinterpret_cast<uintptr_t>(srow) & 15u) == 0);
  constexpr int kStep = kFPer * kThreads;
  float v[kFPer];
  load_batch(srow, len, 0, vec, v);  // the first batch of this slice, in flight during step 1
  for (int w = tid; w < words; w += kThreads) S.bitmap[w] = 0u;
  clear_hist(0);
  clear_hist(1);
  if (tid == 0) {
    S.scal[5] = 0u;  // candidates of this CTA
    S.scal[6] = 0u;  // ties of this CTA
    S.scal[7] = 0u;  // keys above Tk in this CTA
  }
  bool saw_nan = false;

  // 1. threshold (identical in every CTA of the cluster): the lower edge of the digit bin that holds
  //    the row's K-th key, from the row's histogram when it has one that places at most kCap
  //    candidates; else from a strided sample
  const bool take_all = n <= kCap;
  float tau_f = -INFINITY;
  if (!take_all) {
    bool placed = false;
    if (hrow) {
      const HistPlace hp = place_in_histogram(hrow, (uint32_t)k);
      if (hp.found && hp.above + hp.count <= (uint32_t)kCap) {
        placed = true;
        tau_f = key_to_float(hp.bin << (32 - kKeyDigitBits));
      }
    }
    if (!placed) {
      constexpr int kChunks = kSample / 8;
      constexpr int kSPT = kSample / kThreads;
      float sv[kSPT];
#pragma unroll
      for (int e = 0; e < kSPT; ++e) {
        const int s = tid + e * kThreads;
        const int64_t p = (((int64_t)(s >> 3) * n / kChunks) & ~int64_t(7)) + (s & 7);
        sv[e] = row[p];
      }
      // the first batch is consumed here (NaN check), so that its loads complete with the sample's
      // rather than after step 1
#pragma unroll
      for (int j = 0; j < kFPer; ++j) saw_nan |= v[j] != v[j];
#pragma unroll
      for (int e = 0; e < kSPT; ++e) S.pool[tid + e * kThreads] = order_key(sv[e], saw_nan);
      __syncthreads();  // sample keys and cleared histograms visible
      const float rk = (float)k * (float)kSample / (float)n;  // sample rank of the row's K-th score
      int js = (int)ceilf(rk + 4.f * sqrtf(rk) + 8.f);
      js = min(js, kSample);
      tau_f = key_to_float(kth_key(SmemKeys{kSample, false}, (uint32_t)js, false, (uint32_t)(js / 8 + 2)).key);
    }
  } else {
    __syncthreads();  // the counters are clear
  }

  // 2. filter: append (key, position) of every score >= tau in this slice; the next batch's loads
  //    are issued before the current batch is processed.  Every score takes a comparison and a
  //    NaN-propagating max (NaN in the slice <=> NaN max; load_batch gives 0 past the slice, and
  //    only a last, partial batch tests positions).  With take_all the threshold is -inf: a NaN
  //    score is then no candidate, which changes no result (its key is the lowest: it is selected
  //    only when fewer than K other scores exist, and then the exact path below runs).
  const float tau_eff = take_all ? -INFINITY : tau_f;
  float nan_max = 0.0f;
  for (int base = 0; base < len; base += kStep) {
    float vn[kFPer];
    if (base + kStep < len) load_batch(srow, len, base + kStep, vec, vn);
    uint32_t mask = 0u;
    if (base + kStep <= len) {
#pragma unroll
      for (int j = 0; j < kFPer; ++j) {
        nan_max = max_nan(nan_max, v[j]);
        mask |= (uint32_t)(v[j] >= tau_eff) << j;
      }
    } else {
#pragma unroll
      for (int j = 0; j < kFPer; ++j) {
        const int i = base + ((j >> 2) * kThreads + tid) * 4 + (j & 3);
        nan_max = max_nan(nan_max, v[j]);
        mask |= (uint32_t)(i < len && v[j] >= tau_eff) << j;
      }
    }
    const uint32_t c = (uint32_t)__popc(mask);
    const uint32_t incl = warp_inclusive_scan(c);
    const uint32_t tot = __shfl_sync(0xFFFFFFFFu, incl, 31);
    if (tot) {
      uint32_t wbase = 0u;
      if (lane == 0) wbase = atomicAdd(&S.scal[5], tot);
      uint32_t at = __shfl_sync(0xFFFFFFFFu, wbase, 0) + incl - c;
      for (uint32_t mm = mask; mm != 0u && at < (uint32_t)kCap; mm &= mm - 1u, ++at) {
        const int j = __ffs(mm) - 1;
        bool dummy = false;
        S.cand_key[at] = order_key(pick(v, j), dummy);
        S.cand_pos[at] = (uint32_t)(lo + base + ((j >> 2) * kThreads + tid) * 4 + (j & 3));
      }
    }
#pragma unroll
    for (int j = 0; j < kFPer; ++j) v[j] = vn[j];
  }
  saw_nan |= nan_max != nan_max;
  if (saw_nan) S.scal[4] = 1u;  // benign race: every writer stores 1
  __syncthreads();
  if (tid < (int)C) st_cluster_u32(&S.cnt_all[r], (uint32_t)tid, S.scal[5]);
  cluster_sync();  // A: every CTA's candidates and counts are visible to the cluster
  clear_histogram_share();  // every CTA of the cluster has placed its threshold

  uint32_t m = 0u;  // the row's candidates
  for (int q = 0; q < (int)C; ++q) m += S.cnt_all[q];
  if (m < (uint32_t)k || m > (uint32_t)kCap) {
    // the threshold missed (too high, or too many scores tie at it): exact path on CTA 0
    cluster_sync();  // no CTA reads another's shared memory after this point
    if (r == 0) {
      topk_exact(row, n, k, out);
      __syncthreads();
      if (tid == 0 && S.scal[4]) raise_error(err, DSA_DEVERR_NAN_SCORE);
    }
    return;
  }

  // 3. exact K-th key among the row's candidates (gathered from every CTA of the cluster into the
  //    pool, CTA by CTA, four keys per remote load; the first 2048 of each CTA's keys at once)
  if (C > 1) {
    constexpr uint32_t kSpan = 4 * kThreads;
    const uint32_t i0 = 4u * (uint32_t)tid;
    uint4 val[kMaxCluster];
#pragma unroll
    for (int q = 0; q < kMaxCluster; ++q) {
      const uint32_t cq = q < (int)C ? S.cnt_all[q] : 0u;
      val[q] = i0 < cq ? ld_cluster_u32x4(&S.cand_key[i0], (uint32_t)q) : make_uint4(0u, 0u, 0u, 0u);
    }
    uint32_t pre = 0u;
#pragma unroll
    for (int q = 0; q < kMaxCluster; ++q) {
      const uint32_t cq = q < (int)C ? S.cnt_all[q] : 0u;
      for (uint32_t i = i0; i < cq; i += kSpan) {
        const uint4 x = i == i0 ? val[q] : ld_cluster_u32x4(&S.cand_key[i], (uint32_t)q);
        S.pool[pre + i] = x.x;  // entries at or past cq are stale: not copied
        if (i + 1 < cq) S.pool[pre + i + 1] = x.y;
        if (i + 2 < cq) S.pool[pre + i + 2] = x.z;
        if (i + 3 < cq) S.pool[pre + i + 3] = x.w;
      }
      pre += cq;
    }
    __syncthreads();
  }
  const Kth tk = kth_key(SmemKeys{(int)m, C == 1}, (uint32_t)k, true, 0u);
  const uint32_t need = (uint32_t)k - tk.above;  // keys equal to Tk to take, lowest positions first

  // 4. this CTA's keys above Tk go to the bitmap; its ties are listed
  const uint32_t mine = S.cnt_all[r];
  for (uint32_t c0 = 0; c0 < mine; c0 += kThreads) {
    const uint32_t c = c0 + tid;
    uint32_t key = 0u, pos = 0u;
    if (c < mine) {
      key = S.cand_key[c];
      pos = S.cand_pos[c];
    }
    const bool gt = c < mine && key > tk.key;
    if (gt) atomicOr(&S.bitmap[(pos - lo) >> 5], 1u << ((pos - lo) & 31));
    if (c < mine && key == tk.key) {
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
  cluster_arrive_relaxed();  // this CTA reads no other CTA's shared memory from here on

  // output offset of this CTA, and the ties it takes (the lowest positions of the row win)
  uint32_t offset = 0u, ties_before = 0u;
  for (int q = 0; q < (int)r; ++q) {
    const uint32_t ti = S.ties_all[q];
    const uint32_t qq = need > ties_before ? min(ti, need - ties_before) : 0u;
    offset += S.above_all[q] + qq;
    ties_before += ti;
  }
  const uint32_t nties = S.ties_all[r];
  const uint32_t quota = need > ties_before ? min(nties, need - ties_before) : 0u;
  if (quota > 0u) {
    // take the `quota` lowest tied positions: when not all, select on the complemented position
    const bool some = quota < nties;
    uint32_t pos_cut = 0xFFFFFFFFu;  // take tied positions <= pos_cut
    if (some) {
      for (uint32_t e = tid; e < nties; e += kThreads) S.pool[e] = ~S.pool[e];
      __syncthreads();
      pos_cut = ~kth_key(SmemKeys{(int)nties, false}, quota, true, 0u).key;
    }
    for (uint32_t e = tid; e < nties; e += kThreads) {
      const uint32_t pos = some ? ~S.pool[e] : S.pool[e];
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
  uint32_t at = offset + block_exclusive_scan(cnt, total);
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = S.bitmap[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1u;
      if (at < (uint32_t)k) out[at] = (int32_t)(lo + w * 32 + b);
      ++at;
    }
  }
  if (tid == 0 && S.scal[4]) raise_error(err, DSA_DEVERR_NAN_SCORE);  // set before the filter's barrier
  cluster_wait();  // no CTA exits while another may still read its shared memory
}

}  // namespace

cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* q_pos, int T, int k,
                        int32_t* idx, uint32_t* key_hist, int* err, cudaStream_t s) {
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
  return cudaLaunchKernelEx(&cfg, topk_kernel, scores, ld, q_pos, k, idx, key_hist, err);
}

}  // namespace dsa
