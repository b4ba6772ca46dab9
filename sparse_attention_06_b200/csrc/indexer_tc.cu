// indexer_tc.cu -- lightning-indexer scores on the 5th-generation tensor cores (sm_100a).
//
// Computes, for every query t and visible key position s (page "How GLM5.3 Sparse Attention
// Affects HBM Memory Usage", section "Lightning Indexer"):
//     score[t, s] = sum_h w[t,h] * ReLU(q[t,h,:] . khat[s,:])
// with 64 indexer heads of 128 dims and three operand modes:
//   bf16 keys, bf16 queries  -- kind::f16 products of the operands exactly as stored;
//   e4m3 keys, bf16 queries  -- kind::f8f6f4 products that read the e4m3 key pages as stored (no
//       conversion of the keys at all).  Each bf16 query head row q_h is written as two e4m3
//       terms at a power-of-two scale: x = q_h * 2^s_h with s_h chosen so that max|x| lies in
//       [128, 256), a = e4m3(x) and b = e4m3(x - a).  A bf16 value has 8 significant bits and an
//       e4m3 value 4, so a + b = x exactly for every element down to 2^-10 of the head's largest
//       (smaller ones keep an absolute error below 2^-18 of it).  The product runs as
//       k . a + k . b, accumulated in f32, and the epilogue weights head h by w_h * 2^-s_h: ReLU
//       is positively homogeneous, so ReLU(q_h . k) = 2^-s_h ReLU(x . k).  Any bf16 range works;
//   e4m3 keys, e4m3 queries with a per-(query, head) f32 scale -- one kind::f8f6f4 product, the
//       epilogue weights head h by w_h * q_scale[t,h].
// For e4m3 keys the per-token scale is applied after the head sum (equal for scale > 0).
//
// Shape of the computation: per tile of 128 consecutive key positions (two 64-token pages of the
// paged key cache) one tensor-core product D[128 keys, 64*NQ] = K[128 keys, 128] . Q[64*NQ, 128]^T
// with f32 accumulation in tensor memory (TMEM), where the N side holds the 64 heads of NQ
// queries (NQ = 1 for decode, NQ = 4 for prefill chunks whose queries share one request; with
// one query the two terms of split bf16 queries are 128 rows of N, summed by the epilogue).  Each
// TMEM lane then holds one key's head logits, so the ReLU and the w-weighted head sum are
// in-thread work of the epilogue.
//
// One persistent CTA per SM walks a contiguous range of the (query group, key tile) list.  Roles:
//   warp 0      producer: looks up the block ids of the next 32 tiles at once (one lane per tile,
//               the following batch already in flight), checks them and publishes 8-32 tiles'
//               block ids in a tile-info ring in one lane-parallel pass, then (lane 0) issues the
//               TMA copies of key pages (and, for bf16 keys, of query tiles) into 128B-swizzled
//               shared memory; key pages that only one tile reads (one query per request) are
//               copied with an L2 evict-first policy
//   warp 1      TMEM allocation and the thread that issues tcgen05.mma / tcgen05.commit (with one
//               query per tile, of the even tiles; the last warp issues the odd ones)
//   epilogue    sets of 4 warps: with one query per tile three sets (e4m3 keys) or two (bf16)
//               take tiles in turn, over six or four accumulator buffers; with four queries two
//               sets score half of the queries each, over two buffers.  Each reads the tile info
//               LOOK tiles ahead (and, for e4m3, starts a
//               4-byte cp.async of its key's scale then), then per tile: tcgen05.ld of the
//               accumulator, ReLU, head sum, scale, score stores (and, when the selection is
//               fused and one query is scored per tile against bf16 keys, a count per score in a
//               shared order-key digit histogram, added to the query's global row at the query's
//               end)
//   query prep  (e4m3 keys only) 1 or 4 warps write each query group's operand: the two e4m3 terms of
//               the bf16 queries, or the e4m3 query codes, into a 128B-swizzled slot
// Every wait is bounded (DSA_DEVERR_TIMEOUT); bad block ids and bad query metadata are flagged in
// the device error word and skipped, never trapped.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {

namespace {

constexpr int kTileKeys = 128;
constexpr int kPage = 64;
constexpr int kHeads = 64;
constexpr int kDim = 128;

// Operand modes.
enum KeyMode {
  kBf16 = 0,     // bf16 keys x bf16 queries (kind::f16)
  kE4m3 = 1,     // e4m3 keys x bf16 queries as two e4m3 terms (kind::f8f6f4)
  kE4m3Q8 = 2,   // e4m3 keys x e4m3 queries with a per-head scale (kind::f8f6f4)
};

template <int NQ, int KM>
struct Cfg {
  static constexpr bool FP8 = KM != kBf16;
  static constexpr int TERMS = KM == kE4m3 ? 2 : 1;            // e4m3 terms of each query row
  static constexpr int N = kHeads * NQ;                        // query rows of a tile
  // Accumulator buffers in tensor memory: the MMA of a tile waits until the epilogue has released
  // the buffer NACC tiles back, so more buffers let the products run further ahead of the
  // epilogue; with alternating epilogue sets and issuers every buffer belongs to one set and one
  // issuer.  One query per tile: e4m3 queries (four N = 64 products per tile) over six buffers
  // and three epilogue sets; split bf16 queries with e4m3 keys over four buffers of 128 columns
  // and two sets, which is what tensor memory holds; bf16 keys over four buffers and two sets.
  // Four queries per tile: two buffers of N = 256.
  static constexpr bool SPLIT1 = FP8 && TERMS == 2 && NQ == 1;
  static constexpr int NACC = NQ == 1 ? (FP8 && !SPLIT1 ? 6 : 4) : 2;
  // With one query per tile the two e4m3 terms of the split bf16 queries sit side by side in the
  // MMA's N (rows 0..63 the first term, 64..127 the second): one N = 128 product per K step and
  // the epilogue adds the halves.  With four queries they take two passes into one N = 256 sum.
  static constexpr bool SPLIT_N = TERMS == 2 && NQ == 1 && NACC * 2 * N <= 512;
  static constexpr int NMMA = SPLIT_N ? 2 * N : N;            // MMA N = accumulator columns
  // Epilogue sets of four warps (each set covers the 128 TMEM lanes).  With one query per tile
  // the sets take tiles in turn (three for e4m3 keys and queries, whose 16 KB tiles come twice as
  // fast as bf16 ones); with four queries two sets take every tile, each scoring two queries.
  static constexpr int EPI_SETS = NQ == 1 ? (FP8 && !SPLIT1 ? 3 : 2) : 2;
  static constexpr int EPI_WARPS = 4 * EPI_SETS;
  static constexpr bool EPI_ALT = NQ == 1;
  static constexpr int TSTEP = EPI_ALT ? EPI_SETS : 1;        // tiles between one set's tiles
  static constexpr int OPS = FP8 ? (NQ == 1 ? 8 : 4) : 4;      // key-tile stages
  static constexpr int QS = FP8 ? 2 : (NQ == 1 ? 2 : 1);       // query operand slots
  static constexpr int TIS = NQ == 1 ? (FP8 ? 64 : 32) : 16;  // tile-info ring entries (a power of two)
  // Tiles whose info the producer publishes in one lane-parallel pass.  A ring entry is free again
  // once the epilogue has looked at its previous tile, which it does after finishing the tile LOOK
  // of its own tiles earlier; so a pass never waits on the epilogue while TIS - PUB - LOOK * TSTEP
  // covers the tiles in flight (at most OPS + 2), and it can never wait on tiles of its own.
  static constexpr int PUB = NQ == 1 && FP8 ? 32 : 8;
  // Tiles (of its own) an epilogue warp reads ahead in the tile-info ring.  The producer runs at
  // most OPS + 2 tiles ahead of the epilogue's last finished tile, so the distance stays below
  // that; only e4m3 needs it (its scale copies).
  static constexpr int LOOK = FP8 ? 4 : 1;
  static constexpr int OP_BYTES = kTileKeys * kDim * (FP8 ? 1 : 2);  // 16 KB e4m3 / 32 KB bf16 key tile
  static constexpr int CHUNK_BYTES = kTileKeys * 128;         // one 128-byte-row block of a key tile
  static constexpr int Q_CHUNK = N * 128;                     // one 128-byte-row block of a query tile
  static constexpr int Q_BYTES = FP8 ? TERMS * Q_CHUNK : 2 * Q_CHUNK;
  static constexpr int TMEM_COLS = NACC * NMMA <= 256 ? (NACC * NMMA <= 128 ? 128 : 256) : 512;
  static constexpr int EPI_NQ = EPI_ALT ? NQ : NQ / EPI_SETS;  // queries per epilogue warp
  static_assert(EPI_ALT || EPI_NQ * EPI_SETS == NQ, "the epilogue sets score every query of a group once");
  static constexpr int EPI_ARRIVE = EPI_ALT ? 4 : EPI_WARPS;  // epilogue arrivals per tile
  // (one prep warp with one query per tile keeps the CTA at 16 warps, four per SM sub-partition,
  // which leaves every thread 128 registers)
  static constexpr int PREP_WARPS = FP8 ? (NQ == 1 ? 1 : 4) : 0;
  static constexpr int PREP0 = 2 + EPI_WARPS;                 // first query-prep warp
  // One thread issues a tcgen05 instruction about every 60-75 cycles, which with one query per
  // tile (N = 64) is slower than the rest of the pipeline: a second warp issues the odd tiles.
  static constexpr int MMA_WARPS = NQ == 1 ? 2 : 1;
  static constexpr int MMA2 = PREP0 + PREP_WARPS;             // the second issuing warp
  static constexpr int THREADS = 32 * (PREP0 + PREP_WARPS + MMA_WARPS - 1);
  // Each issuer waits on a key stage's and an accumulator's mbarriers by phase parity, which is
  // only sound when it has seen every phase of them: with two issuers alternating tiles, every
  // stage and buffer must belong to one of them (even counts).
  static_assert(MMA_WARPS == 1 || (OPS % 2 == 0 && NACC % 2 == 0), "stages and buffers must not alternate between issuers");
  // a publication pass waits only on tiles issued before it, and not while the pipeline is full
  static_assert(TIS + LOOK * TSTEP >= PUB, "tile-info ring too small for a publication pass");
  static_assert(TIS + LOOK * TSTEP - PUB >= OPS + 2, "a publication pass would wait on the pipeline");
  static_assert((TIS & (TIS - 1)) == 0, "ring index by mask");
  static_assert(PUB <= 32, "one lane per tile");
  // One query per tile with bf16 keys: the epilogue counts its scores' order-key digits in a
  // shared histogram (when the selection's histogram is wanted) and adds it to the query's global
  // row at each query boundary of the CTA's range.  (With e4m3 keys the epilogue is the kernel's
  // bottleneck, and the counting cost the kernel more than the histogram saves the selection.)
  static constexpr bool HIST = NQ == 1 && !FP8;
  static_assert(NACC * NMMA <= 512, "accumulators fit tensor memory");
  static_assert(!EPI_ALT || NACC % EPI_SETS == 0, "each epilogue set owns whole accumulator buffers");
  // shared-memory carve-up (offsets from a 1024-aligned base)
  static constexpr int OFF_OP = 0;
  static constexpr int OFF_Q = OFF_OP + OPS * OP_BYTES;
  static constexpr int OFF_W = OFF_Q + QS * Q_BYTES;
  static constexpr int OFF_SC = OFF_W + EPI_WARPS * EPI_NQ * kHeads * 4;  // w, one copy per epilogue warp
  static constexpr int OFF_PR = OFF_SC + (FP8 ? TIS * kTileKeys * 4 : 0);  // key scales of ring tiles
  static constexpr int OFF_TI = OFF_PR + TIS * kTileKeys;                  // row present, per ring tile
  static constexpr int OFF_BT = OFF_TI + TIS * 8;                          // block ids of ring tiles
  static constexpr int OFF_HIST = OFF_BT + 32 * 16;                        // the producer's batch table
  static constexpr int OFF_BAR = OFF_HIST + (HIST ? kKeyBins * 4 : 0);     // the digit histogram
  static constexpr int NBAR = 2 * OPS + 2 * QS + 2 * NACC + 1 + 2 * TIS + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 64;
  static constexpr int SMEM = BYTES + 1024;  // slack for aligning the base
};

struct Params {
  const int32_t* q_req;
  const int32_t* q_pos;
  const int32_t* block_table;
  const void* q;                 // [T, 64, 128] bf16 or e4m3 codes
  const float* q_scale;          // [T, 64] (e4m3 queries)
  const float* w;
  const float* key_scale;
  float* scores;
  int64_t ld;
  uint32_t* key_hist;            // [T, kKeyBins] order-key digit counts to add to, or null
  int64_t num_blocks;
  int num_queries, num_reqs, max_blocks, max_context;
  int* err;
  int stream_keys;               // each key page is read by one query tile: load keys evict-first
};

// One query group (NQ consecutive queries of one request) and its tile count.
struct Group {
  int req;
  int nmax;   // keys visible to the group (max over its queries)
  int tiles;  // 128-key tiles to score (0 = group skipped)
};

template <int NQ>
__device__ __forceinline__ Group group_info(const Params& p, int g, bool report) {
  Group G{0, 0, 0};
  const int t0 = g * NQ;
  const int req = p.q_req[t0];
  bool ok = req >= 0 && req < p.num_reqs;
  int nmax = 0;
#pragma unroll
  for (int i = 0; i < NQ; ++i) {
    const int pos = p.q_pos[t0 + i];
    if (pos < 0 || pos >= p.max_context) ok = false;
    if (NQ > 1 && p.q_req[t0 + i] != req) {
      ok = false;
      if (report) raise_error(p.err, DSA_DEVERR_QUERY_GROUP);
    }
    nmax = max(nmax, pos + 1);
  }
  if (!ok) {
    if (report) raise_error(p.err, DSA_DEVERR_REQUEST);
    return G;
  }
  G.req = req;
  G.nmax = nmax;
  G.tiles = (nmax + kTileKeys - 1) / kTileKeys;
  return G;
}

// Walk over the global (group, tile) list, restricted to [lo, hi).
template <int NQ>
struct Walk {
  int64_t g, hi, grp_start;
  int grp, ngroups;
  Group G;

  __device__ void init(const Params& p, int64_t lo, int64_t hi_) {
    g = lo;
    hi = hi_;
    ngroups = p.num_queries / NQ;
    grp = 0;
    grp_start = 0;
    G = Group{0, 0, 0};
    if (lo >= hi) return;
    while (grp < ngroups) {
      G = group_info<NQ>(p, grp, false);
      if (grp_start + G.tiles > lo) break;
      grp_start += G.tiles;
      ++grp;
    }
  }

  // Next tile of the range: sets group index and tile-in-group; false at the end.
  __device__ bool next(const Params& p, int& group, int& tile) {
    if (g >= hi) return false;
    while (g >= grp_start + G.tiles) {
      grp_start += G.tiles;
      ++grp;
      G = group_info<NQ>(p, grp, false);
    }
    group = grp;
    tile = (int)(g - grp_start);
    ++g;
    return true;
  }
};

// Raw block-table entry of page `pg` (0/1) of tile `j` of a group: -1 when the page holds no
// visible key, -2 when its logical block is past the table.  Only the load; check_block() judges
// the value when it is used, so that the load stays in flight until then.  A negative table entry
// for a page with visible keys is an error like any other id outside the pool (it reads as -3).
__device__ __forceinline__ int lookup_block(const Params& p, const Group& G, int j, int pg) {
  const int first = j * kTileKeys + pg * kPage;
  if (G.tiles == 0 || first >= G.nmax) return -1;
  const int lblk = first / kPage;
  if (lblk >= p.max_blocks) return -2;
  const int b = p.block_table[(int64_t)G.req * p.max_blocks + lblk];
  return b < 0 ? -3 : b;
}

// The physical block of a looked-up entry, or -1 (flagging entries outside the pool).
__device__ __forceinline__ int check_block(const Params& p, int raw) {
  if (raw == -1) return -1;
  if (raw < 0 || raw >= p.num_blocks) {
    raise_error(p.err, DSA_DEVERR_BLOCK_ID);
    return -1;
  }
  return raw;
}

// Bounded wait that ignores the abort flag (used to drain in-flight copies when giving up).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int* err) {
  mbar_wait(bar, parity, err, nullptr);
}

// D[tmem] (+)= A * B^T, kind::f8f6f4 with e4m3 A and B from shared-memory descriptors, f32
// accumulate.  Same issue-lean form as umma_ss.
template <int ACC>
__device__ __forceinline__ void umma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "n"(ACC));
}

// Power-of-two exponent s with which a bf16 query head row whose largest magnitude is `amax` is
// scaled before it is split into e4m3 terms: amax * 2^s lies in [128, 256).  Rows of zeros (and
// rows holding an infinity or NaN, whose products are not finite anyway) keep s = 0; s is at most
// 126, so that 2^-s stays a normal f32.  The query-prep warps and the epilogue both call this on
// the same values, so they agree on s.
__device__ __forceinline__ int q_head_shift(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const int ex = (int)((bits >> 23) & 0xFFu);
  if (!(amax > 0.0f) || ex == 0xFF) return 0;
  const int e = ex == 0 ? -127 : ex - 127;  // floor(log2(amax)); subnormals count as 2^-127
  return min(7 - e, 126);
}

// 2^s for |s| <= 126 (an exact power of two)
__device__ __forceinline__ float exp2i(int s) { return __uint_as_float((uint32_t)(s + 127) << 23); }

// Largest magnitude of 8 bf16 values (one 16-byte piece)
__device__ __forceinline__ float amax_bf16x8(const uint4& v) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&v);
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = fmaxf(m, fabsf(__uint_as_float(w[i] << 16)));
    m = fmaxf(m, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
  }
  return m;
}

// The two e4m3 terms of 8 bf16 values scaled by 2^s: a = e4m3(x), b = e4m3(x - a); 8 bytes each.
__device__ __forceinline__ void split_bf16x8(const uint4& v, float scale, uint2& a, uint2& b) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&v);
  uint32_t pa[2] = {0u, 0u}, pb[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float x0 = __uint_as_float(w[i] << 16) * scale;
    const float x1 = __uint_as_float(w[i] & 0xFFFF0000u) * scale;
    const __nv_fp8x2_storage_t ca = __nv_cvt_float2_to_fp8x2(make_float2(x0, x1), __NV_SATFINITE, __NV_E4M3);
    const __half2_raw ha = __nv_cvt_fp8x2_to_halfraw2(ca, __NV_E4M3);
    const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&ha));
    const __nv_fp8x2_storage_t cb =
        __nv_cvt_float2_to_fp8x2(make_float2(x0 - fa.x, x1 - fa.y), __NV_SATFINITE, __NV_E4M3);
    pa[i >> 1] |= (uint32_t)ca << (16 * (i & 1));
    pb[i >> 1] |= (uint32_t)cb << (16 * (i & 1));
  }
  a = make_uint2(pa[0], pa[1]);
  b = make_uint2(pb[0], pb[1]);
}

// (a0, a1) * (b0, b1) + c as one packed f32x2 FMA (round to nearest, per lane).
__device__ __forceinline__ uint64_t ffma2(float a0, float a1, float b0, float b1, uint64_t c) {
  uint64_t d;
  asm("{\n\t.reg .b64 a, b;\n\t"
      "mov.b64 a, {%1, %2};\n\t"
      "mov.b64 b, {%3, %4};\n\t"
      "fma.rn.f32x2 %0, a, b, %5;\n\t}"
      : "=l"(d)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "l"(c));
  return d;
}

__device__ __forceinline__ void unpack2(uint64_t x, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(x));
}

template <int NQ, int KM>
__global__ void __launch_bounds__(Cfg<NQ, KM>::THREADS, 1)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                      const Params p) {
  using C = Cfg<NQ, KM>;
  constexpr bool FP8 = C::FP8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* op_ring = smem + C::OFF_OP;
  uint8_t* q_slots = smem + C::OFF_Q;
  float* w_s = reinterpret_cast<float*>(smem + C::OFF_W);
  float* sc_ring = reinterpret_cast<float*>(smem + C::OFF_SC);  // [TIS][128] (e4m3) key scales
  uint8_t* pr_ring = smem + C::OFF_PR;                           // [TIS][128] row's page present
  int2* ti_ring = reinterpret_cast<int2*>(smem + C::OFF_TI);     // [TIS] block ids of the pages
  int4* batch_tab = reinterpret_cast<int4*>(smem + C::OFF_BT);   // [32] producer: (block ids, group) per tile
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* op_full = bars;
  uint64_t* op_empty = op_full + C::OPS;
  uint64_t* q_full = op_empty + C::OPS;  // query operand in place (TMA bytes, or the prep warps)
  uint64_t* q_empty = q_full + C::QS;
  uint64_t* acc_full = q_empty + C::QS;
  uint64_t* acc_empty = acc_full + C::NACC;
  uint64_t* mma_done = acc_empty + C::NACC;
  uint64_t* ti_full = mma_done + 1;       // [TIS] tile info (and scales) in place
  uint64_t* ti_empty = ti_full + C::TIS;  // [TIS] tile info read by every epilogue warp
  uint64_t* hb_ready = ti_empty + C::TIS;  // every epilogue warp done with the histogram's query
  uint64_t* hb_done = hb_ready + 1;        // the histogram added to its query's row and cleared
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + C::OFF_HIST);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  unsigned long long* total_tiles = reinterpret_cast<unsigned long long*>(smem + C::OFF_MISC + 16);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  griddep_launch_dependents();

  if (tid == 0) {
    for (int i = 0; i < C::OPS; ++i) {
      mbar_init(&op_full[i], 1);
      mbar_init(&op_empty[i], 1);
    }
    for (int i = 0; i < C::QS; ++i) {
      mbar_init(&q_full[i], FP8 ? C::PREP_WARPS : 1);
      mbar_init(&q_empty[i], C::MMA_WARPS);
    }
    for (int i = 0; i < C::NACC; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::EPI_ARRIVE);
    }
    mbar_init(mma_done, C::MMA_WARPS);
    for (int i = 0; i < C::TIS; ++i) {
      mbar_init(&ti_full[i], 1);
      mbar_init(&ti_empty[i], C::EPI_ARRIVE);
    }
    mbar_init(hb_ready, C::EPI_WARPS);
    mbar_init(hb_done, C::EPI_WARPS);
    *abort_flag = 0;
    *total_tiles = 0ull;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if constexpr (C::HIST)
    for (int b = tid; b < kKeyBins; b += blockDim.x) hist_s[b] = 0u;
  __syncthreads();
  griddep_wait();  // inputs may come from the previous kernel of the stream
  // total tile count of the whole call (every CTA computes the same value)
  {
    unsigned long long part = 0;
    for (int g = tid; g < p.num_queries / NQ; g += blockDim.x) part += (unsigned long long)group_info<NQ>(p, g, false).tiles;
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xFFFFFFFFu, part, o);
    if (lane == 0 && part) atomicAdd(total_tiles, part);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int64_t N = (int64_t)*total_tiles;
  const int64_t lo = N * blockIdx.x / gridDim.x;
  const int64_t hi = N * (blockIdx.x + 1) / gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lo < hi) {
      if (lane == 0) {
        prefetch_tmap(&kmap);
        if (!FP8) prefetch_tmap(&qmap);
      }
      // Every lane runs the same walk; lane l keeps tile l of each batch of 32 and loads its two
      // block ids.  The next batch is looked up before the current one is issued.
      Walk<NQ> W;
      W.init(p, lo, hi);
      int n_cnt = 0, n_grp = -1, n_r0 = -1, n_r1 = -1;
      auto fetch = [&]() {
        n_cnt = 0;
        n_grp = -1;
        int mj = 0;
        Group mG{0, 0, 0};
        for (int l = 0; l < 32; ++l) {
          int g, j;
          if (!W.next(p, g, j)) break;
          if (lane == l) {
            n_grp = g;
            mj = j;
            mG = W.G;
          }
          ++n_cnt;
        }
        n_r0 = n_grp >= 0 ? lookup_block(p, mG, mj, 0) : -1;
        n_r1 = n_grp >= 0 ? lookup_block(p, mG, mj, 1) : -1;
      };
      fetch();
      int last = -1, m = -1;  // (lane 0) group of the last query tile issued, query tiles issued
      int64_t i = 0;          // tiles whose copies were issued (the first tile of the batch below)
      // keys read once (decode) are loaded evict-first, so that they do not push the scores this
      // kernel writes out of L2 before the selection reads them
      const bool hint = p.stream_keys != 0;
      const uint64_t key_policy = hint ? l2_policy_evict_first() : 0ull;
      auto load_key = [&](uint8_t* dst, int32_t c0, int32_t row, uint64_t* bar) {
        if (hint) tma_load_2d_hint(dst, &kmap, bar, c0, row, key_policy);
        else tma_load_2d(dst, &kmap, bar, c0, row);
      };
      bool ok = true;
      while (ok && n_cnt > 0) {
        const int cnt = n_cnt;
        // this lane's tile of the batch (tile i + lane): block ids checked, into the batch table
        const int b0 = lane < cnt ? check_block(p, n_r0) : -1;
        const int b1 = lane < cnt ? check_block(p, n_r1) : -1;
        batch_tab[lane] = make_int4(b0, b1, n_grp, 0);
        fetch();  // the next batch's lookups, in flight while this one is issued
        __syncwarp();
        for (int l0 = 0; l0 < cnt && ok; l0 += C::PUB) {
          const int n = min(C::PUB, cnt - l0);
          // tile info of tiles l0 .. l0 + n - 1 of the batch, one lane each: published before any
          // wait of these tiles below, which depend on the epilogue
          bool lok = true;
          if (lane < n) {
            const int4 e = batch_tab[l0 + lane];
            const int64_t x = i + l0 + lane;
            const int c = (int)(x & (C::TIS - 1)), cu = (int)(x / C::TIS);
            if (cu >= 1 && !mbar_wait(&ti_empty[c], (cu - 1) & 1, p.err, abort_flag)) {
              lok = false;
            } else {
              ti_ring[c] = make_int2(e.x, e.y);
              mbar_arrive(&ti_full[c]);
            }
          }
          ok = __all_sync(0xFFFFFFFFu, lok);
          if (!ok) break;
          // the query tiles (bf16 keys) and key copies of these tiles, in order, from lane 0
          int64_t issued = i + l0;
          if (lane == 0) {
            for (int l = l0; l < l0 + n; ++l) {
              const int4 e = batch_tab[l];
              const int grp = e.z, t0 = e.x, t1 = e.y;
              if (!FP8 && grp != last) {
                const int mm = m + 1;  // m counts the query tiles issued so far
                const int slot = mm % C::QS, use = mm / C::QS;
                if (use >= 1 && !(ok = mbar_wait(&q_empty[slot], (use - 1) & 1, p.err, abort_flag))) break;
                mbar_arrive_expect_tx(&q_full[slot], C::Q_BYTES);
                uint8_t* qd = q_slots + slot * C::Q_BYTES;
                tma_load_2d(qd, &qmap, &q_full[slot], 0, grp * NQ * kHeads);
                tma_load_2d(qd + C::Q_CHUNK, &qmap, &q_full[slot], 64, grp * NQ * kHeads);
                m = mm;
                last = grp;
              }
              const int st = (int)(issued % C::OPS), use = (int)(issued / C::OPS);
              if (use >= 1 && !(ok = mbar_wait(&op_empty[st], (use - 1) & 1, p.err, abort_flag))) break;
              constexpr uint32_t kPageBytes = C::OP_BYTES / 2;
              mbar_arrive_expect_tx(&op_full[st], (t0 >= 0 ? kPageBytes : 0u) + (t1 >= 0 ? kPageBytes : 0u));
              uint8_t* dst = op_ring + st * C::OP_BYTES;
              if constexpr (FP8) {
                // a 64-token e4m3 page is one 8 KB box of 128-byte rows
                if (t0 >= 0) load_key(dst, 0, t0 * kPage, &op_full[st]);
                if (t1 >= 0) load_key(dst + 8192, 0, t1 * kPage, &op_full[st]);
              } else {
                // a bf16 page is two 8 KB boxes (dims 0..63 and 64..127), one per column block
                if (t0 >= 0) {
                  load_key(dst, 0, t0 * kPage, &op_full[st]);
                  load_key(dst + C::CHUNK_BYTES, 64, t0 * kPage, &op_full[st]);
                }
                if (t1 >= 0) {
                  load_key(dst + 8192, 0, t1 * kPage, &op_full[st]);
                  load_key(dst + C::CHUNK_BYTES + 8192, 64, t1 * kPage, &op_full[st]);
                }
              }
              ++issued;
            }
          }
          ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
          if (!ok) i = __shfl_sync(0xFFFFFFFFu, issued, 0);
        }
        if (ok) i += cnt;
        __syncwarp();  // the batch table is rewritten by the next batch
      }
      if (!ok && lane == 0) {
        // give up: let the copies already issued land before the CTA's memory goes away
        for (int s = 0; s < C::OPS; ++s)
          if (i > s) drain_wait(&op_full[s], (uint32_t)(((i - 1 - s) / C::OPS) & 1), p.err);
        if constexpr (!FP8) {
          for (int q = 0; q < C::QS; ++q)
            if (m >= q) drain_wait(&q_full[q], (uint32_t)(((m - q) / C::QS) & 1), p.err);
        }
      }
    }
  } else if (warp == 1 || (C::MMA_WARPS == 2 && warp == C::MMA2)) {
    // ------------------------------------------------------------------ MMA issuer(s)
    const int par = warp == 1 ? 0 : 1;  // with two issuers: the parity of the tiles this one issues
    if (lane == 0 && lo < hi) {
      // f16 kind: bf16 operands; f8f6f4 kind: e4m3 operands (format code 0 in both fields)
      const uint32_t idesc = idesc_f16(FP8 ? 0u : 1u, 0u, 128u, (uint32_t)C::NMMA);
      Walk<NQ> W;
      W.init(p, lo, hi);
      int grp, j, last = -1, m = -1, slot = -1;
      int64_t i = 0;
      bool ok = true;
      while (W.next(p, grp, j)) {
        if (grp != last) {
          if (slot >= 0) mma_commit(&q_empty[slot]);
          last = grp;
          ++m;
          slot = m % C::QS;
          if (!(ok = mbar_wait(&q_full[slot], (m / C::QS) & 1, p.err, abort_flag))) break;
        }
        // both issuers take every query-slot hand-off above (each commits q_empty once per group)
        if (C::MMA_WARPS == 2 && (int)(i & 1) != par) {  // the other issuer's tile
          ++i;
          continue;
        }
        const int s = (int)(i % C::OPS), use = (int)(i / C::OPS);
        if (!(ok = mbar_wait(&op_full[s], use & 1, p.err, abort_flag))) break;
        const int a = (int)(i % C::NACC), ause = (int)(i / C::NACC);
        if (ause >= 1 && !(ok = mbar_wait(&acc_empty[a], (ause - 1) & 1, p.err, abort_flag))) break;
        tc_fence_after();
        // K steps of 32 bytes each (16 bf16 or 32 e4m3 dims); the descriptor's start-address
        // field counts 16-byte units
        const uint64_t ad = sw128_desc(smem_u32(op_ring + s * C::OP_BYTES), 16, 1024);
        const uint64_t bd = sw128_desc(smem_u32(q_slots + slot * C::Q_BYTES), 16, 1024);
        const uint32_t d = tmem_base + (uint32_t)(a * C::NMMA);
        constexpr uint64_t ac = C::CHUNK_BYTES >> 4, bc = C::Q_CHUNK >> 4;
        if constexpr (FP8) {
          // one 128-byte row holds all 128 dims: four K steps (with SPLIT_N over both terms at
          // once); with four queries the second term (the residual of the bf16 queries)
          // accumulates into the same D with the same key operand in a second pass
          umma_ss_f8<0>(d, ad, bd, idesc);
          umma_ss_f8<1>(d, ad + 2, bd + 2, idesc);
          umma_ss_f8<1>(d, ad + 4, bd + 4, idesc);
          umma_ss_f8<1>(d, ad + 6, bd + 6, idesc);
          if constexpr (C::TERMS == 2 && !C::SPLIT_N) {
            umma_ss_f8<1>(d, ad, bd + bc, idesc);
            umma_ss_f8<1>(d, ad + 2, bd + bc + 2, idesc);
            umma_ss_f8<1>(d, ad + 4, bd + bc + 4, idesc);
            umma_ss_f8<1>(d, ad + 6, bd + bc + 6, idesc);
          }
        } else {
          // two 64-dim column blocks of four K steps each
          umma_ss<0>(d, ad, bd, idesc);
          umma_ss<1>(d, ad + 2, bd + 2, idesc);
          umma_ss<1>(d, ad + 4, bd + 4, idesc);
          umma_ss<1>(d, ad + 6, bd + 6, idesc);
          umma_ss<1>(d, ad + ac, bd + bc, idesc);
          umma_ss<1>(d, ad + ac + 2, bd + bc + 2, idesc);
          umma_ss<1>(d, ad + ac + 4, bd + bc + 4, idesc);
          umma_ss<1>(d, ad + ac + 6, bd + bc + 6, idesc);
        }
        mma_commit(&op_empty[s]);
        mma_commit(&acc_full[a]);
        ++i;
      }
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(mma_done);
      drain_wait(mma_done, 0, p.err);
    }
  } else if (warp < C::PREP0) {
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - 2;                   // epilogue warp
    const int eset = ew >> 2;                  // its set
    const int quarter = warp & 3;              // TMEM lanes this warp may access
    const int q0 = C::EPI_ALT ? 0 : eset * C::EPI_NQ;  // first query of the group this warp scores
    const int t0 = C::EPI_ALT ? eset : 0;      // first tile of this warp, then every tstep-th
    constexpr int tstep = C::TSTEP;
    const int r = quarter * 32 + lane;         // key row of the tile
    float* w_mine = w_s + ew * C::EPI_NQ * kHeads;  // this warp's copy of its queries' head weights
    const int64_t ntl = hi - lo;               // tiles of this CTA
    bool ok = true;
    // Tile `it` seen C::LOOK of this warp's tiles ahead: note whether this row's page exists and
    // (e4m3) start the copy of the row's key scale; each thread reads back only what it wrote
    // itself, after its own cp.async group of that tile has completed.  One group is committed per
    // tile of this warp (empty past the end) so that the group count stays in step.
    auto look = [&](int64_t it) {
      if (it < ntl && ok) {
        const int c = (int)(it & (C::TIS - 1));
        ok = warp_wait(&ti_full[c], (uint32_t)((it / C::TIS) & 1), p.err, abort_flag);
        if (ok) {
          const int2 blk = ti_ring[c];
          const int b = r < kPage ? blk.x : blk.y;
          pr_ring[c * kTileKeys + r] = b >= 0 ? 1 : 0;
          if (FP8 && b >= 0)
            cp_async_4(smem_u32(sc_ring + c * kTileKeys + r), p.key_scale + (int64_t)b * kPage + (r & (kPage - 1)));
          __syncwarp();
          if (lane == 0) mbar_arrive(&ti_empty[c]);
        }
      }
      cp_async_commit();
    };
#pragma unroll 1
    for (int d = 0; d < C::LOOK; ++d) look(t0 + (int64_t)d * tstep);
    // The shared digit histogram holds the counts of query hgrp.  Every epilogue warp walks every
    // tile, so all of them see each query boundary: there each one signals that its tiles of the
    // query are done, waits for the others, adds its share of the bins to the query's global row
    // (one reduction per nonzero bin), clears them, and waits until every share is cleared.
    // Each warp notes the range of digits its lanes counted ([hlo, hhi]), and at a boundary
    // sweeps only its range (the scores of a query span a few binades: tens of bins of 4096).
    const bool use_hist = C::HIST && p.key_hist != nullptr;
    int hgrp = -1;
    uint32_t hphase = 0, hlo = 0xFFFFFFFFu, hhi = 0u;
    auto flush_hist = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(hb_ready);
      if (!warp_wait(hb_ready, hphase, p.err, abort_flag)) return false;
      uint32_t* grow = p.key_hist + (int64_t)hgrp * kKeyBins;
      const uint32_t wlo = __reduce_min_sync(0xFFFFFFFFu, hlo), whi = __reduce_max_sync(0xFFFFFFFFu, hhi);
      for (uint32_t b = wlo + lane; b <= whi; b += 32) {
        const uint32_t c = atomicExch(&hist_s[b], 0u);  // ranges of warps overlap: take each count once
        if (c) atomicAdd(&grow[b], c);
      }
      hlo = 0xFFFFFFFFu;
      hhi = 0u;
      __syncwarp();
      if (lane == 0) mbar_arrive(hb_done);
      if (!warp_wait(hb_done, hphase, p.err, abort_flag)) return false;
      hphase ^= 1u;
      return true;
    };
    Walk<NQ> W;
    W.init(p, lo, hi);
    int grp, j, last = -1;
    int npos[C::EPI_NQ];
    int64_t i = 0;
    int turn = 0;  // i % tstep
    while (ok && W.next(p, grp, j)) {
      if (use_hist && grp != hgrp) {
        if (hgrp >= 0 && !(ok = flush_hist())) break;
        hgrp = grp;
      }
      const bool mine = turn == t0;
      turn = turn + 1 == tstep ? 0 : turn + 1;
      if (!mine) {  // another set's tile
        ++i;
        continue;
      }
      if (grp != last) {
        // this warp's head weights for the group, with the query operand's per-head factor folded
        // in: 2^-s_h for split bf16 queries, the per-head scale for e4m3 queries
        __syncwarp();
        for (int e = lane; e < C::EPI_NQ * kHeads; e += 32) {
          const int64_t th = (int64_t)(grp * NQ + q0) * kHeads + e;  // (query, head) row
          float f = 1.0f;
          if constexpr (KM == kE4m3) {
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q) + th * kDim);
            float amax = 0.0f;
#pragma unroll
            for (int c = 0; c < kDim / 8; ++c) amax = fmaxf(amax, amax_bf16x8(__ldg(src + c)));
            f = exp2i(-q_head_shift(amax));
          } else if constexpr (KM == kE4m3Q8) {
            f = p.q_scale[th];
          }
          w_mine[e] = p.w[th] * f;
        }
        __syncwarp();
#pragma unroll
        for (int qi = 0; qi < C::EPI_NQ; ++qi) npos[qi] = p.q_pos[grp * NQ + q0 + qi] + 1;
        last = grp;
      }
      cp_async_wait<C::LOOK - 1>();  // this tile's group (committed LOOK tiles ago) has landed
      const int c = (int)(i & (C::TIS - 1));
      const bool present = pr_ring[c * kTileKeys + r] != 0;
      const float scale = FP8 ? sc_ring[c * kTileKeys + r] : 1.0f;
      const int a = (int)(i % C::NACC), use = (int)(i / C::NACC);
      if (!warp_wait(&acc_full[a], use & 1, p.err, abort_flag)) break;
      tc_fence_after();
      const int s = j * kTileKeys + r;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * C::NMMA + q0 * kHeads);
#pragma unroll
      for (int qi = 0; qi < C::EPI_NQ; ++qi) {
        const float4* w4 = reinterpret_cast<const float4*>(w_mine + qi * kHeads);
        // head pairs in packed f32x2 FMAs, four independent pair accumulators; the heads in two
        // halves of 32 columns (with SPLIT_N, each the sum of its two term columns)
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        if constexpr (!C::SPLIT_N && NQ > 1) {
          // (four queries per tile: all 64 head columns in flight before one wait)
          uint32_t v[64];
#pragma unroll
          for (int c16 = 0; c16 < 4; ++c16)
            tmem_ld16(tbase + qi * 64 + c16 * 16, *reinterpret_cast<uint32_t(*)[16]>(&v[c16 * 16]));
          tmem_wait_ld();
#pragma unroll
          for (int h4 = 0; h4 < 16; ++h4) {
            const float4 wv = w4[h4];
            uint64_t* ac = acc + (h4 & 1) * 2;
            ac[0] = ffma2(wv.x, wv.y, fmaxf(__uint_as_float(v[4 * h4 + 0]), 0.0f), fmaxf(__uint_as_float(v[4 * h4 + 1]), 0.0f), ac[0]);
            ac[1] = ffma2(wv.z, wv.w, fmaxf(__uint_as_float(v[4 * h4 + 2]), 0.0f), fmaxf(__uint_as_float(v[4 * h4 + 3]), 0.0f), ac[1]);
          }
        } else
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t v[32];
          tmem_ld16(tbase + qi * 64 + hh * 32, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
          tmem_ld16(tbase + qi * 64 + hh * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
          if constexpr (C::SPLIT_N) {
            uint32_t u[32];
            tmem_ld16(tbase + kHeads + hh * 32, *reinterpret_cast<uint32_t(*)[16]>(&u[0]));
            tmem_ld16(tbase + kHeads + hh * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&u[16]));
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) v[c] = __float_as_uint(__uint_as_float(v[c]) + __uint_as_float(u[c]));
          } else {
            tmem_wait_ld();
          }
#pragma unroll
          for (int h4 = 0; h4 < 8; ++h4) {
            const float4 wv = w4[hh * 8 + h4];
            uint64_t* ac = acc + (h4 & 1) * 2;
            ac[0] = ffma2(wv.x, wv.y, fmaxf(__uint_as_float(v[4 * h4 + 0]), 0.0f), fmaxf(__uint_as_float(v[4 * h4 + 1]), 0.0f), ac[0]);
            ac[1] = ffma2(wv.z, wv.w, fmaxf(__uint_as_float(v[4 * h4 + 2]), 0.0f), fmaxf(__uint_as_float(v[4 * h4 + 3]), 0.0f), ac[1]);
          }
        }
        float sum = 0.0f;
        {
          float lo[4], hi[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) unpack2(acc[e], lo[e], hi[e]);
          sum = ((lo[0] + hi[0]) + (lo[1] + hi[1])) + ((lo[2] + hi[2]) + (lo[3] + hi[3]));
        }
        const bool written = present && s < npos[qi];
        const float score = sum * scale;
        if (written) p.scores[(int64_t)(grp * NQ + q0 + qi) * p.ld + s] = score;
        if (use_hist && written) {  // the selection's threshold histogram (the query is hgrp)
          bool nan = false;
          const uint32_t dg = key_digit(order_key(score, nan));
          atomicAdd(&hist_s[dg], 1u);
          hlo = min(hlo, dg);
          hhi = max(hhi, dg);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[a]);
      look(i + (int64_t)C::LOOK * tstep);  // after this tile is released, so that the producer can get there
      ++i;
    }
    if (ok && use_hist && hgrp >= 0) ok = flush_hist();  // the range's last query
    cp_async_wait_all();  // no copy may land after the CTA's shared memory is released
  } else if constexpr (FP8) {
    // ------------------------------------------------------------------ query prep (e4m3 keys)
    // Each query group's operand slot: rows n = (query n / 64, head n % 64) of N 128-byte rows in
    // the 128B-swizzled K-major layout (16-byte piece c of row n at n * 128 + ((c ^ (n % 8)) * 16)),
    // one block per term.  A thread handles half a row (64 dims); the two halves of a row sit in
    // adjacent lanes, which share the row's largest magnitude.
    const int pt = tid - 32 * C::PREP0;  // 0 .. 32 * PREP_WARPS - 1
    Walk<NQ> W;
    W.init(p, lo, hi);
    int grp, j, last = -1, m = -1;
    while (W.next(p, grp, j)) {
      if (grp == last) continue;
      last = grp;
      ++m;
      const int slot = m % C::QS, use = m / C::QS;
      if (use >= 1 && !warp_wait(&q_empty[slot], (use - 1) & 1, p.err, abort_flag)) break;
      uint8_t* dst = q_slots + slot * C::Q_BYTES;
#pragma unroll 1
      for (int task = pt; task < 2 * C::N; task += 32 * C::PREP_WARPS) {
        const int n = task >> 1, half = task & 1;
        const int64_t th = (int64_t)grp * NQ * kHeads + n;  // (query, head) row of q
        if constexpr (KM == kE4m3) {
          const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q) + th * kDim) + 8 * half;
          uint4 v[8];
          float amax = 0.0f;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            v[c] = __ldg(src + c);
            amax = fmaxf(amax, amax_bf16x8(v[c]));
          }
          amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
          const float sc = exp2i(q_head_shift(amax));
#pragma unroll
          for (int c = 0; c < 4; ++c) {  // 16-byte pieces 4 half + c of both terms
            uint2 a0, b0, a1, b1;
            split_bf16x8(v[2 * c], sc, a0, b0);
            split_bf16x8(v[2 * c + 1], sc, a1, b1);
            const uint32_t off = sw128_offset((uint32_t)n, (uint32_t)(4 * half + c));
            *reinterpret_cast<uint4*>(dst + off) = make_uint4(a0.x, a0.y, a1.x, a1.y);
            *reinterpret_cast<uint4*>(dst + C::Q_CHUNK + off) = make_uint4(b0.x, b0.y, b1.x, b1.y);
          }
        } else {
          const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.q) + th * kDim) + 4 * half;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(dst + sw128_offset((uint32_t)n, (uint32_t)(4 * half + c))) = __ldg(src + c);
        }
      }
      fence_proxy_async_smem();  // the generic-proxy stores above are read by the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_full[slot]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int NQ, int KM>
cudaError_t launch_impl(const IndexerArgs& a, int num_sms, cudaStream_t s) {
  using C = Cfg<NQ, KM>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  alignas(64) CUtensorMap kmap, qmap;
  const uint64_t rows = (uint64_t)a.keys.num_blocks * kPage;
  bool ok;
  if (C::FP8) {
    ok = encode_tmap_2d(&kmap, a.keys.data, 1, kDim, rows, kDim, 128, kPage, true);
    qmap = kmap;  // unused: the query operand is written by the prep warps
  } else {
    ok = encode_tmap_2d(&kmap, a.keys.data, 2, kDim, rows, kDim * 2, 64, kPage, true) &&
         encode_tmap_2d(&qmap, a.q, 2, kDim, (uint64_t)a.batch.num_queries * kHeads, kDim * 2, 64,
                        (uint32_t)(kHeads * NQ), true);
  }
  if (!ok) return cudaErrorInvalidValue;
  Params p{a.batch.q_req, a.batch.q_pos, a.batch.block_table, a.q, a.q_scale, a.w, a.keys.scale, a.scores, a.ld,
           a.key_hist, a.keys.num_blocks, a.batch.num_queries, a.batch.num_reqs, a.batch.max_blocks,
           a.batch.max_context, a.err,
           // one query per request (decode): every key page is read by one query tile only
           (NQ == 1 && a.batch.num_queries <= a.batch.num_reqs) ? 1 : 0};
  auto kern = indexer_tc_kernel<NQ, KM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attrs[2];
  const cudaLaunchConfig_t cfg = launch_config(dim3(num_sms), dim3(C::THREADS), C::SMEM, s, attrs);
  return cudaLaunchKernelEx(&cfg, kern, kmap, qmap, p);
}

template <int NQ>
cudaError_t launch_mode(const IndexerArgs& a, int num_sms, cudaStream_t s) {
  if (a.keys.dtype != DSA_E4M3) return launch_impl<NQ, kBf16>(a, num_sms, s);
  if (a.q_dtype == DSA_E4M3) return launch_impl<NQ, kE4m3Q8>(a, num_sms, s);
  return launch_impl<NQ, kE4m3>(a, num_sms, s);
}

}  // namespace

cudaError_t launch_indexer_tc_decode(const IndexerArgs& a, int num_sms, cudaStream_t s) {
  return launch_mode<1>(a, num_sms, s);
}

cudaError_t launch_indexer_tc_prefill(const IndexerArgs& a, int num_sms, cudaStream_t s) {
  return launch_mode<4>(a, num_sms, s);
}

}  // namespace dsa
