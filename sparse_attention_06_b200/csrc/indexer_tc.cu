// indexer_tc.cu -- lightning-indexer scores on the 5th-generation tensor cores (sm_100a).
//
// Computes, for every query t and visible key position s (page "How GLM5.3 Sparse Attention
// Affects HBM Memory Usage", section "Lightning Indexer"):
//     score[t, s] = sum_h w[t,h] * ReLU(q[t,h,:] . khat[s,:])
// with 64 indexer heads of 128 dims, bf16 queries, and bf16 keys or e4m3 keys with a per-token
// scale (khat = code * scale; for scale > 0 the scale is applied after the head sum, which is the
// same value).  bf16 keys multiply bf16 queries exactly as stored.  For e4m3 keys the product runs
// in f16: each code is re-encoded by integer bit operations as the f16 holding code * 2^-8 (exact
// for every finite code, subnormals included), the epilogue multiplies the per-token scale by 2^8,
// and each query tile is converted bf16 -> f16 once, which is exact for |q| in [2^-14, 65504]
// (smaller values keep an absolute error below 2^-25).
//
// Shape of the computation: per tile of 128 consecutive key positions (two 64-token pages of the
// paged key cache) one tensor-core product D[128 keys, 64*NQ] = K[128 keys, 128] . Q[64*NQ, 128]^T
// with f32 accumulation in tensor memory (TMEM), where the N side holds the 64 heads of NQ
// queries (NQ = 1 for decode, NQ = 4 for prefill chunks whose queries share one request).  Each
// TMEM lane then holds one key's head logits, so the ReLU and the w-weighted head sum are
// in-thread work of the epilogue.
//
// One persistent CTA per SM walks a contiguous range of the (query group, key tile) list.  Roles:
//   warp 0      TMA producer: key pages and query tiles into 128B-swizzled shared memory
//   warp 1      TMEM allocation and the single thread that issues tcgen05.mma / tcgen05.commit
//   warps 2-5   epilogue: tcgen05.ld of the accumulator, ReLU, head sum, scale, score stores
//   warps 6-9   (e4m3 keys only) convert the fp8 staging tile into the f16 operand ring and each
//               query tile to f16 in place
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

template <int NQ, bool FP8>
struct Cfg {
  static constexpr int N = kHeads * NQ;                       // MMA N
  static constexpr int OPS = FP8 ? (NQ == 1 ? 3 : 2) : (NQ == 1 ? 5 : 4);  // operand stages
  static constexpr int STS = FP8 ? (NQ == 1 ? 6 : 4) : 0;     // fp8 staging stages
  static constexpr int QS = NQ == 1 ? 2 : 1;                  // query slots
  static constexpr int OP_BYTES = kTileKeys * kDim * 2;       // 32 KB bf16 key tile
  static constexpr int CHUNK_BYTES = kTileKeys * 128;         // one 64-dim column block
  static constexpr int ST_BYTES = kTileKeys * kDim;           // 16 KB fp8 key tile
  static constexpr int Q_BYTES = N * kDim * 2;
  static constexpr int Q_CHUNK = N * 128;
  static constexpr int TMEM_COLS = 2 * N;
  static constexpr int THREADS = FP8 ? 320 : 192;
  // shared-memory carve-up (offsets from a 1024-aligned base)
  static constexpr int OFF_OP = 0;
  static constexpr int OFF_ST = OFF_OP + OPS * OP_BYTES;
  static constexpr int OFF_Q = OFF_ST + STS * ST_BYTES;
  static constexpr int OFF_W = OFF_Q + QS * Q_BYTES;
  static constexpr int OFF_BAR = OFF_W + 4 * NQ * kHeads * 4;  // one copy of w per epilogue warp
  static constexpr int NBAR = 2 * OPS + 2 * STS + 3 * QS + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 64;
  static constexpr int SMEM = BYTES + 1024;  // slack for aligning the base
};

struct Params {
  const int32_t* q_req;
  const int32_t* q_pos;
  const int32_t* block_table;
  const float* w;
  const float* key_scale;
  float* scores;
  int64_t ld;
  int64_t num_blocks;
  int num_queries, num_reqs, max_blocks, max_context;
  int* err;
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

// Physical block of page `pg` (0/1) of tile `j` of a group, or -1 when the page holds no
// visible key or its block id is outside the pool.
__device__ __forceinline__ int page_block(const Params& p, const Group& G, int j, int pg, bool report) {
  const int first = j * kTileKeys + pg * kPage;
  if (first >= G.nmax) return -1;
  const int lblk = first / kPage;
  if (lblk >= p.max_blocks) {
    if (report) raise_error(p.err, DSA_DEVERR_BLOCK_ID);
    return -1;
  }
  const int blk = p.block_table[(int64_t)G.req * p.max_blocks + lblk];
  if (blk < 0 || blk >= p.num_blocks) {
    if (report) raise_error(p.err, DSA_DEVERR_BLOCK_ID);
    return -1;
  }
  return blk;
}

// Bounded wait that ignores the abort flag (used to drain in-flight copies when giving up).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int* err) {
  mbar_wait(bar, parity, err, nullptr);
}

// Two e4m3 codes -> two f16 holding code * 2^-8, exactly.  An e4m3 code s.eeee.mmm has value
// (1 + m/8) 2^(e-7) (or (m/8) 2^-6 when e = 0); its 7 magnitude bits placed at f16 bits 7..13 read
// as (1 + m/8) 2^(e-15) (or, as an f16 subnormal, (m/8) 2^-14): the same value times 2^-8 in both
// cases.  The sign moves from bit 7 to bit 15.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2_times_2m8(uint32_t w, uint32_t byte_sel) {
  const uint32_t x = __byte_perm(w, 0u, byte_sel);  // code a in bits 0..7, code b in bits 16..23
  return ((x << 7) & 0x3F803F80u) | ((x << 8) & 0x80008000u);
}

// fp8 e4m3 x16 -> f16 x16, each value scaled by 2^-8 (exact)
__device__ __forceinline__ void e4m3x16_to_f16(const uint4& in, uint4& lo, uint4& hi) {
  lo.x = e4m3x2_to_f16x2_times_2m8(in.x, 0x4140u);
  lo.y = e4m3x2_to_f16x2_times_2m8(in.x, 0x4342u);
  lo.z = e4m3x2_to_f16x2_times_2m8(in.y, 0x4140u);
  lo.w = e4m3x2_to_f16x2_times_2m8(in.y, 0x4342u);
  hi.x = e4m3x2_to_f16x2_times_2m8(in.z, 0x4140u);
  hi.y = e4m3x2_to_f16x2_times_2m8(in.z, 0x4342u);
  hi.z = e4m3x2_to_f16x2_times_2m8(in.w, 0x4140u);
  hi.w = e4m3x2_to_f16x2_times_2m8(in.w, 0x4342u);
}

// bf16 x8 -> f16 x8 in place (16 bytes)
__device__ __forceinline__ uint4 bf16x8_to_f16(const uint4& in) {
  uint4 out;
  const uint32_t* a = reinterpret_cast<const uint32_t*>(&in);
  uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a[i]));
    const __half2 h = __float22half2_rn(f);
    o[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return out;
}

template <int NQ, bool FP8>
__global__ void __launch_bounds__(Cfg<NQ, FP8>::THREADS, 1)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                      const Params p) {
  using C = Cfg<NQ, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* op_ring = smem + C::OFF_OP;
  uint8_t* st_ring = smem + C::OFF_ST;
  uint8_t* q_slots = smem + C::OFF_Q;
  float* w_s = reinterpret_cast<float*>(smem + C::OFF_W);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* op_full = bars;
  uint64_t* op_empty = op_full + C::OPS;
  uint64_t* st_full = op_empty + C::OPS;
  uint64_t* st_empty = st_full + C::STS;
  uint64_t* q_full = st_empty + C::STS;
  uint64_t* q_empty = q_full + C::QS;
  uint64_t* q_ready = q_empty + C::QS;  // (e4m3) query tile converted to f16
  uint64_t* acc_full = q_ready + C::QS;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  unsigned long long* total_tiles = reinterpret_cast<unsigned long long*>(smem + C::OFF_MISC + 16);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < C::OPS; ++i) {
      mbar_init(&op_full[i], FP8 ? 128 : 1);
      mbar_init(&op_empty[i], 1);
    }
    for (int i = 0; i < C::STS; ++i) {
      mbar_init(&st_full[i], 1);
      mbar_init(&st_empty[i], 128);
    }
    for (int i = 0; i < C::QS; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&q_ready[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    *total_tiles = 0ull;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
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
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && lo < hi) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&qmap);
      Walk<NQ> W;
      W.init(p, lo, hi);
      int grp, j, last = -1, m = -1;
      int64_t i = 0;
      bool ok = true;
      while (ok && W.next(p, grp, j)) {
        if (grp != last) {
          last = grp;
          ++m;
          const int slot = m % C::QS, use = m / C::QS;
          if (use >= 1 && !(ok = mbar_wait(&q_empty[slot], (use - 1) & 1, p.err, abort_flag))) break;
          mbar_arrive_expect_tx(&q_full[slot], C::Q_BYTES);
          uint8_t* qd = q_slots + slot * C::Q_BYTES;
          tma_load_2d(qd, &qmap, &q_full[slot], 0, grp * NQ * kHeads);
          tma_load_2d(qd + C::Q_CHUNK, &qmap, &q_full[slot], 64, grp * NQ * kHeads);
        }
        const int b0 = page_block(p, W.G, j, 0, true);
        const int b1 = page_block(p, W.G, j, 1, true);
        if (FP8) {
          const int s = (int)(i % C::STS), use = (int)(i / C::STS);
          if (use >= 1 && !(ok = mbar_wait(&st_empty[s], (use - 1) & 1, p.err, abort_flag))) break;
          const uint32_t bytes = (b0 >= 0 ? 8192u : 0u) + (b1 >= 0 ? 8192u : 0u);
          mbar_arrive_expect_tx(&st_full[s], bytes);
          uint8_t* dst = st_ring + s * C::ST_BYTES;
          if (b0 >= 0) tma_load_2d(dst, &kmap, &st_full[s], 0, b0 * kPage);
          if (b1 >= 0) tma_load_2d(dst + 8192, &kmap, &st_full[s], 0, b1 * kPage);
        } else {
          const int s = (int)(i % C::OPS), use = (int)(i / C::OPS);
          if (use >= 1 && !(ok = mbar_wait(&op_empty[s], (use - 1) & 1, p.err, abort_flag))) break;
          const uint32_t bytes = (b0 >= 0 ? 16384u : 0u) + (b1 >= 0 ? 16384u : 0u);
          mbar_arrive_expect_tx(&op_full[s], bytes);
          uint8_t* dst = op_ring + s * C::OP_BYTES;
          if (b0 >= 0) {
            tma_load_2d(dst, &kmap, &op_full[s], 0, b0 * kPage);
            tma_load_2d(dst + C::CHUNK_BYTES, &kmap, &op_full[s], 64, b0 * kPage);
          }
          if (b1 >= 0) {
            tma_load_2d(dst + 8192, &kmap, &op_full[s], 0, b1 * kPage);
            tma_load_2d(dst + C::CHUNK_BYTES + 8192, &kmap, &op_full[s], 64, b1 * kPage);
          }
        }
        ++i;
      }
      if (!ok) {
        // give up: let the copies already issued land before the CTA's memory goes away
        for (int s = 0; s < C::OPS && !FP8; ++s)
          if (i > s) drain_wait(&op_full[s], (uint32_t)(((i - 1 - s) / C::OPS) & 1), p.err);
        for (int s = 0; s < C::STS; ++s)
          if (i > s) drain_wait(&st_full[s], (uint32_t)(((i - 1 - s) / C::STS) & 1), p.err);
        for (int q = 0; q < C::QS; ++q)
          if (m >= q) drain_wait(&q_full[q], (uint32_t)(((m - q) / C::QS) & 1), p.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && lo < hi) {
      const uint32_t idesc = idesc_f16(FP8 ? 0u : 1u, 0u, 128u, (uint32_t)C::N);  // f16 or bf16
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
          if (!(ok = mbar_wait(FP8 ? &q_ready[slot] : &q_full[slot], (m / C::QS) & 1, p.err, abort_flag))) break;
        }
        const int s = (int)(i % C::OPS), use = (int)(i / C::OPS);
        if (!(ok = mbar_wait(&op_full[s], use & 1, p.err, abort_flag))) break;
        const int a = (int)(i & 1), ause = (int)(i >> 1);
        if (ause >= 1 && !(ok = mbar_wait(&acc_empty[a], (ause - 1) & 1, p.err, abort_flag))) break;
        tc_fence_after();
        // 8 MMAs of K = 16: two 64-dim column blocks, four K steps of 32 bytes each (the
        // descriptor's start-address field counts 16-byte units)
        const uint64_t ad = sw128_desc(smem_u32(op_ring + s * C::OP_BYTES), 16, 1024);
        const uint64_t bd = sw128_desc(smem_u32(q_slots + slot * C::Q_BYTES), 16, 1024);
        const uint32_t d = tmem_base + (uint32_t)(a * C::N);
        constexpr uint64_t ac = C::CHUNK_BYTES >> 4, bc = C::Q_CHUNK >> 4;
        umma_ss<0>(d, ad, bd, idesc);
        umma_ss<1>(d, ad + 2, bd + 2, idesc);
        umma_ss<1>(d, ad + 4, bd + 4, idesc);
        umma_ss<1>(d, ad + 6, bd + 6, idesc);
        umma_ss<1>(d, ad + ac, bd + bc, idesc);
        umma_ss<1>(d, ad + ac + 2, bd + bc + 2, idesc);
        umma_ss<1>(d, ad + ac + 4, bd + bc + 4, idesc);
        umma_ss<1>(d, ad + ac + 6, bd + bc + 6, idesc);
        mma_commit(&op_empty[s]);
        mma_commit(&acc_full[a]);
        ++i;
      }
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(mma_done);
      drain_wait(mma_done, 0, p.err);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;              // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;         // key row of the tile
    float* w_mine = w_s + (warp - 2) * NQ * kHeads;  // this warp's copy of the group's w
    const int pg = r >> 6;                           // page of the tile holding this row
    // Tiles are looked up ahead of their accumulator: the block id two tiles ahead and the e4m3
    // scale one tile ahead, so that neither global load is waited on in the tile that issued it.
    Walk<NQ> W;
    W.init(p, lo, hi);
    int g0 = -1, j0 = 0, g1 = -1, j1 = 0, g2 = -1, j2 = 0;
    Group G0{0, 0, 0}, G1{0, 0, 0}, G2{0, 0, 0};
    int b0 = -1, b1 = -1, b2 = -1;
    float sc0 = 1.0f, sc1 = 1.0f;
    if (W.next(p, g1, j1)) {
      G1 = W.G;
      b1 = page_block(p, G1, j1, pg, false);
      if (W.next(p, g2, j2)) {
        G2 = W.G;
        b2 = page_block(p, G2, j2, pg, false);
      } else {
        g2 = -1;
      }
      if (FP8 && b1 >= 0) sc1 = 256.0f * p.key_scale[(int64_t)b1 * kPage + (r & 63)];
    } else {
      g1 = -1;
    }
    int last = -1;
    int npos[NQ];
    int64_t i = 0;
    while (g1 >= 0) {
      // rotate: the tile to finish now is the one looked up last iteration
      g0 = g1; j0 = j1; G0 = G1; b0 = b1; sc0 = sc1;
      g1 = g2; j1 = j2; G1 = G2; b1 = b2;
      sc1 = 1.0f;
      if (g1 >= 0 && FP8 && b1 >= 0) sc1 = 256.0f * p.key_scale[(int64_t)b1 * kPage + (r & 63)];  // undo 2^-8
      if (g1 >= 0 && W.next(p, g2, j2)) {
        G2 = W.G;
        b2 = page_block(p, G2, j2, pg, false);
      } else {
        g2 = -1;
      }
      if (g0 != last) {
        __syncwarp();
        for (int e = lane; e < NQ * kHeads; e += 32) w_mine[e] = p.w[(int64_t)g0 * NQ * kHeads + e];
        __syncwarp();
#pragma unroll
        for (int qi = 0; qi < NQ; ++qi) npos[qi] = p.q_pos[g0 * NQ + qi] + 1;
        last = g0;
      }
      const int a = (int)(i & 1), use = (int)(i >> 1);
      if (!warp_wait(&acc_full[a], use & 1, p.err, abort_flag)) break;
      tc_fence_after();
      const int s = j0 * kTileKeys + r;
      const float scale = FP8 ? sc0 : 1.0f;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * C::N);
#pragma unroll
      for (int qi = 0; qi < NQ; ++qi) {
        uint32_t v[64];
        tmem_ld16(tbase + qi * 64 + 0, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
        tmem_ld16(tbase + qi * 64 + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
        tmem_ld16(tbase + qi * 64 + 32, *reinterpret_cast<uint32_t(*)[16]>(&v[32]));
        tmem_ld16(tbase + qi * 64 + 48, *reinterpret_cast<uint32_t(*)[16]>(&v[48]));
        tmem_wait_ld();
        const float4* w4 = reinterpret_cast<const float4*>(w_mine + qi * kHeads);
        float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
        for (int h4 = 0; h4 < 16; ++h4) {
          const float4 wv = w4[h4];
          acc0 = fmaf(wv.x, fmaxf(__uint_as_float(v[4 * h4 + 0]), 0.0f), acc0);
          acc1 = fmaf(wv.y, fmaxf(__uint_as_float(v[4 * h4 + 1]), 0.0f), acc1);
          acc0 = fmaf(wv.z, fmaxf(__uint_as_float(v[4 * h4 + 2]), 0.0f), acc0);
          acc1 = fmaf(wv.w, fmaxf(__uint_as_float(v[4 * h4 + 3]), 0.0f), acc1);
        }
        if (b0 >= 0 && s < npos[qi]) p.scores[(int64_t)(g0 * NQ + qi) * p.ld + s] = (acc0 + acc1) * scale;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[a]);
      ++i;
    }
  } else if (FP8) {
    // ------------------------------------------------------------------ fp8 -> bf16 converter
    const int ct = tid - 192;  // 0..127
    Walk<NQ> W;
    W.init(p, lo, hi);
    int grp, j, last = -1, m = -1;
    int64_t i = 0;
    while (W.next(p, grp, j)) {
      if (grp != last) {
        // a new query tile: convert it to f16 in place once it has landed
        last = grp;
        ++m;
        const int slot = m % C::QS;
        if (!warp_wait(&q_full[slot], (m / C::QS) & 1, p.err, abort_flag)) break;
        uint8_t* q = q_slots + slot * C::Q_BYTES;
        for (int off = ct * 16; off < C::Q_BYTES; off += 128 * 16)
          *reinterpret_cast<uint4*>(q + off) = bf16x8_to_f16(*reinterpret_cast<const uint4*>(q + off));
        fence_proxy_async_smem();
        mbar_arrive(&q_ready[slot]);
      }
      const int s8 = (int)(i % C::STS), u8 = (int)(i / C::STS);
      if (!warp_wait(&st_full[s8], u8 & 1, p.err, abort_flag)) break;
      const int so = (int)(i % C::OPS), uo = (int)(i / C::OPS);
      if (uo >= 1 && !warp_wait(&op_empty[so], (uo - 1) & 1, p.err, abort_flag)) break;
      const uint8_t* src = st_ring + s8 * C::ST_BYTES;
      uint8_t* dst = op_ring + so * C::OP_BYTES;
#pragma unroll 2
      for (int k = 0; k < 8; ++k) {
        const int piece = ct + 128 * k;  // 16-byte piece of the fp8 tile: row piece/8, column piece%8
        const int row = piece >> 3, c = piece & 7;
        const uint4 in = *reinterpret_cast<const uint4*>(src + row * 128 + c * 16);
        uint4 lo4, hi4;
        e4m3x16_to_f16(in, lo4, hi4);
        uint8_t* chunk = dst + (c >> 2) * C::CHUNK_BYTES;
        const uint32_t p0 = (uint32_t)((c & 3) * 2);
        *reinterpret_cast<uint4*>(chunk + sw128_offset(row, p0)) = lo4;
        *reinterpret_cast<uint4*>(chunk + sw128_offset(row, p0 + 1)) = hi4;
      }
      fence_proxy_async_smem();
      mbar_arrive(&op_full[so]);
      mbar_arrive(&st_empty[s8]);
      ++i;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int NQ, bool FP8>
cudaError_t launch_impl(const IndexerArgs& a, int num_sms, cudaStream_t s) {
  using C = Cfg<NQ, FP8>;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  alignas(64) CUtensorMap kmap, qmap;
  const uint64_t rows = (uint64_t)a.keys.num_blocks * kPage;
  bool ok;
  if (FP8)
    ok = encode_tmap_2d(&kmap, a.keys.data, 1, kDim, rows, kDim, 128, kPage, false);
  else
    ok = encode_tmap_2d(&kmap, a.keys.data, 2, kDim, rows, kDim * 2, 64, kPage, true);
  ok = ok && encode_tmap_2d(&qmap, a.q, 2, kDim, (uint64_t)a.batch.num_queries * kHeads, kDim * 2, 64,
                            (uint32_t)(kHeads * NQ), true);
  if (!ok) return cudaErrorInvalidValue;
  Params p{a.batch.q_req, a.batch.q_pos, a.batch.block_table, a.w, a.keys.scale, a.scores, a.ld,
           a.keys.num_blocks, a.batch.num_queries, a.batch.num_reqs, a.batch.max_blocks,
           a.batch.max_context, a.err};
  auto kern = indexer_tc_kernel<NQ, FP8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<num_sms, C::THREADS, C::SMEM, s>>>(kmap, qmap, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_indexer_tc_decode(const IndexerArgs& a, int num_sms, cudaStream_t s) {
  return a.keys.dtype == DSA_E4M3 ? launch_impl<1, true>(a, num_sms, s) : launch_impl<1, false>(a, num_sms, s);
}

cudaError_t launch_indexer_tc_prefill(const IndexerArgs& a, int num_sms, cudaStream_t s) {
  return a.keys.dtype == DSA_E4M3 ? launch_impl<4, true>(a, num_sms, s) : launch_impl<4, false>(a, num_sms, s);
}

}  // namespace dsa
