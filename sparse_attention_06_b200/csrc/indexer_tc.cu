// indexer_tc.cu -- lightning-indexer scores on the 5th-generation tensor cores (sm_100a).
//
// Computes, for every query t and visible key position s (page "How GLM5.3 Sparse Attention
// Affects HBM Memory Usage", section "Lightning Indexer"):
//     score[t, s] = sum_h w[t,h] * ReLU(q[t,h,:] . khat[s,:])
// with 64 indexer heads of 128 dims, bf16 queries, and bf16 keys or e4m3 keys with a per-token
// scale (khat = code * scale; for scale > 0 the scale is applied after the head sum, which is the
// same value).  bf16 keys multiply bf16 queries exactly as stored.  For e4m3 keys the product runs
// in f16: each pair of codes becomes two f16 by the hardware conversion (cvt.rn.f16x2.e4m3x2, exact:
// every e4m3 value, subnormals included, is an f16), and each query tile is converted bf16 -> f16
// once, which is exact for |q| in [2^-14, 65504] (smaller values keep an absolute error below 2^-25).
//
// Shape of the computation: per tile of 128 consecutive key positions (two 64-token pages of the
// paged key cache) one tensor-core product D[128 keys, 64*NQ] = K[128 keys, 128] . Q[64*NQ, 128]^T
// with f32 accumulation in tensor memory (TMEM), where the N side holds the 64 heads of NQ
// queries (NQ = 1 for decode, NQ = 4 for prefill chunks whose queries share one request).  Each
// TMEM lane then holds one key's head logits, so the ReLU and the w-weighted head sum are
// in-thread work of the epilogue.
//
// One persistent CTA per SM walks a contiguous range of the (query group, key tile) list.  Roles:
//   warp 0      producer: looks up the block ids of the next 32 tiles at once (one lane per tile,
//               the following batch already in flight), checks them and publishes 8-32 tiles'
//               block ids in a tile-info ring in one lane-parallel pass, then (lane 0) issues the
//               TMA copies of key pages and query tiles into 128B-swizzled shared memory
//   warp 1      TMEM allocation and the thread that issues tcgen05.mma / tcgen05.commit (for e4m3
//               keys with one query per tile, of the even tiles; the last warp issues the odd ones)
//   epilogue    8 warps in two sets (alternate tiles with one query per tile, else half of the
//               queries each): reads the tile
//               info LOOK tiles ahead (and, for e4m3, starts a 4-byte cp.async of its key's scale
//               then), then per tile: tcgen05.ld of the accumulator, ReLU, head sum, scale, score
//               stores
//   converter   (e4m3 keys only) converts the fp8 staging tile to f16 -- into tensor memory, where
//               the MMA reads it as the A operand, when one query uses the tile (8 warps), else
//               into the shared-memory operand ring (4 warps) -- and each query tile to f16 in place
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
  // e4m3 keys with one query per tile: the converted key tile goes to tensor memory and the MMA
  // reads its A operand from there (the accumulators of N = 64 leave room for four A stages)
  static constexpr bool TMEM_A = FP8 && NQ == 1;
  static constexpr int OPS = TMEM_A ? 4 : FP8 ? 2 : (NQ == 1 ? 5 : 4);  // operand stages
  static constexpr int STS = FP8 ? (NQ == 1 ? 8 : 4) : 0;     // fp8 staging stages
  static constexpr int QS = NQ == 1 ? 2 : 1;                  // query slots
  static constexpr int TIS = NQ == 1 ? (FP8 ? 48 : 24) : 16;  // tile-info ring entries
  // Tiles whose info the producer publishes in one lane-parallel pass.  A ring entry is free again
  // once the epilogue has looked at its previous tile, which it does after finishing the tile LOOK
  // of its own tiles earlier; so a pass never waits on the epilogue while TIS - PUB - LOOK * tstep
  // covers the tiles in flight (at most STS + OPS + 2), and it can never wait on tiles of its own.
  static constexpr int PUB = NQ == 1 && FP8 ? 32 : 8;
  // Tiles (of its own) an epilogue warp reads ahead in the tile-info ring.  The producer runs at
  // most STS + OPS + 2 tiles (e4m3) or OPS + 2 tiles (bf16) ahead of the epilogue's last finished
  // tile, so the distance stays below that; only e4m3 needs it (its scale copies).
  static constexpr int LOOK = FP8 ? (NQ == 1 ? 4 : 4) : 1;
  static constexpr int OP_BYTES = kTileKeys * kDim * 2;       // 32 KB bf16 key tile
  static constexpr int CHUNK_BYTES = kTileKeys * 128;         // one 64-dim column block
  static constexpr int ST_BYTES = kTileKeys * kDim;           // 16 KB fp8 key tile
  static constexpr int Q_BYTES = N * kDim * 2;
  static constexpr int Q_CHUNK = N * 128;
  static constexpr int TMEM_COLS = TMEM_A ? 512 : 2 * N;
  // Epilogue: two sets of four warps (each set covers the 128 TMEM lanes).  With one query per
  // tile the sets take alternate tiles (set s owns accumulator s); with four queries both sets
  // take every tile, each scoring two of the queries.
  static constexpr int EPI_WARPS = 8;
  static constexpr bool EPI_ALT = NQ == 1;
  static constexpr int EPI_NQ = EPI_ALT ? NQ : NQ / 2;       // queries per epilogue warp
  static constexpr int EPI_ARRIVE = EPI_ALT ? 4 : 8;          // epilogue arrivals per tile
  static constexpr int CONV_WARPS = FP8 ? 4 : 0;
  static constexpr int CONV0 = 2 + EPI_WARPS;                 // first converter warp
  // One thread issues a tcgen05.mma about every 60 cycles, which at N = 64 is half the tensor
  // pipe's rate: for e4m3 keys with one query per tile (A in tensor memory) a second warp issues
  // the odd tiles (accumulator 1).
  static constexpr int MMA_WARPS = TMEM_A ? 2 : 1;
  static constexpr int MMA2 = CONV0 + CONV_WARPS;             // the second issuing warp
  static constexpr int THREADS = 32 * (CONV0 + CONV_WARPS + MMA_WARPS - 1);
  // Each issuer waits on an operand stage's mbarrier by phase parity, which is only sound when it
  // has seen the stage's previous phase: with two issuers alternating tiles, every stage must
  // belong to one of them (an even number of stages).
  static_assert(MMA_WARPS == 1 || OPS % 2 == 0, "operand stages must not alternate between issuers");
  // a publication pass waits only on tiles issued before it, and not while the pipeline is full
  static_assert(TIS + LOOK * (EPI_ALT ? 2 : 1) >= PUB, "tile-info ring too small for a publication pass");
  static_assert(TIS + LOOK * (EPI_ALT ? 2 : 1) - PUB >= STS + OPS + 2, "a publication pass would wait on the pipeline");
  static_assert(PUB <= 32, "one lane per tile");
  // shared-memory carve-up (offsets from a 1024-aligned base)
  static constexpr int OFF_OP = 0;
  static constexpr int OFF_ST = OFF_OP + (TMEM_A ? 0 : OPS * OP_BYTES);
  static constexpr int OFF_Q = OFF_ST + STS * ST_BYTES;
  static constexpr int OFF_W = OFF_Q + QS * Q_BYTES;
  static constexpr int OFF_SC = OFF_W + EPI_WARPS * EPI_NQ * kHeads * 4;  // w, one copy per epilogue warp
  static constexpr int OFF_PR = OFF_SC + (FP8 ? TIS * kTileKeys * 4 : 0);  // key scales of ring tiles
  static constexpr int OFF_TI = OFF_PR + TIS * kTileKeys;                  // row present, per ring tile
  static constexpr int OFF_BT = OFF_TI + TIS * 8;                          // block ids of ring tiles
  static constexpr int OFF_BAR = OFF_BT + 32 * 16;                         // the producer's batch table
  static constexpr int NBAR = 2 * OPS + 2 * STS + 3 * QS + 4 + 1 + 2 * TIS;
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

// Raw block-table entry of page `pg` (0/1) of tile `j` of a group: -1 when the page holds no
// visible key, -2 when its logical block is past the table.  Only the load; check_block() judges
// the value when it is used, so that the load stays in flight until then.  A negative table entry
// for a page with visible keys is an error like any other id outside the pool (it reads as -3).
// TMEM_A: tensor-memory column of converted key-tile stage s (after the two accumulators of N
// columns; one f16 key tile = 128 dims = 64 columns)
template <int N>
__device__ __forceinline__ uint32_t a_stage_col(int s) { return (uint32_t)(2 * N + s * (kDim / 2)); }

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

// Four e4m3 codes (one 32-bit word, lowest byte first) -> four f16 in two words, exactly, by the
// hardware conversion.
__device__ __forceinline__ void e4m3x4_to_f16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 a, b;\n\t"
      "mov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// fp8 e4m3 x16 -> f16 x16 (exact)
__device__ __forceinline__ void e4m3x16_to_f16(const uint4& in, uint4& lo, uint4& hi) {
  e4m3x4_to_f16x4(in.x, lo.x, lo.y);
  e4m3x4_to_f16x4(in.y, lo.z, lo.w);
  e4m3x4_to_f16x4(in.z, hi.x, hi.y);
  e4m3x4_to_f16x4(in.w, hi.z, hi.w);
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
  float* sc_ring = reinterpret_cast<float*>(smem + C::OFF_SC);  // [TIS][128] (e4m3) key scales
  uint8_t* pr_ring = smem + C::OFF_PR;                           // [TIS][128] row's page present
  int2* ti_ring = reinterpret_cast<int2*>(smem + C::OFF_TI);     // [TIS] block ids of the pages
  int4* batch_tab = reinterpret_cast<int4*>(smem + C::OFF_BT);   // [32] producer: (block ids, group) per tile
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
  uint64_t* ti_full = mma_done + 1;     // [TIS] tile info (and scales) in place
  uint64_t* ti_empty = ti_full + C::TIS;  // [TIS] tile info read by every epilogue warp
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  unsigned long long* total_tiles = reinterpret_cast<unsigned long long*>(smem + C::OFF_MISC + 16);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  griddep_launch_dependents();

  if (tid == 0) {
    for (int i = 0; i < C::OPS; ++i) {
      mbar_init(&op_full[i], FP8 ? C::CONV_WARPS : 1);
      mbar_init(&op_empty[i], 1);
    }
    for (int i = 0; i < C::STS; ++i) {
      mbar_init(&st_full[i], 1);
      mbar_init(&st_empty[i], C::CONV_WARPS);
    }
    for (int i = 0; i < C::QS; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], C::MMA_WARPS);
      mbar_init(&q_ready[i], C::CONV_WARPS);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::EPI_ARRIVE);
    }
    mbar_init(mma_done, C::MMA_WARPS);
    for (int i = 0; i < C::TIS; ++i) {
      mbar_init(&ti_full[i], 1);
      mbar_init(&ti_empty[i], C::EPI_ARRIVE);
    }
    *abort_flag = 0;
    *total_tiles = 0ull;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
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
        prefetch_tmap(&qmap);
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
            const int c = (int)(x % C::TIS), cu = (int)(x / C::TIS);
            if (cu >= 1 && !mbar_wait(&ti_empty[c], (cu - 1) & 1, p.err, abort_flag)) {
              lok = false;
            } else {
              ti_ring[c] = make_int2(e.x, e.y);
              mbar_arrive(&ti_full[c]);
            }
          }
          ok = __all_sync(0xFFFFFFFFu, lok);
          if (!ok) break;
          // the query tiles and key copies of these tiles, in order, from lane 0
          int64_t issued = i + l0;
          if (lane == 0) {
            for (int l = l0; l < l0 + n; ++l) {
              const int4 e = batch_tab[l];
              const int grp = e.z, t0 = e.x, t1 = e.y;
              if (grp != last) {
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
              if constexpr (FP8) {
                const int st = (int)(issued % C::STS), use = (int)(issued / C::STS);
                if (use >= 1 && !(ok = mbar_wait(&st_empty[st], (use - 1) & 1, p.err, abort_flag))) break;
                mbar_arrive_expect_tx(&st_full[st], (t0 >= 0 ? 8192u : 0u) + (t1 >= 0 ? 8192u : 0u));
                uint8_t* dst = st_ring + st * C::ST_BYTES;
                if (t0 >= 0) tma_load_2d(dst, &kmap, &st_full[st], 0, t0 * kPage);
                if (t1 >= 0) tma_load_2d(dst + 8192, &kmap, &st_full[st], 0, t1 * kPage);
              } else {
                const int st = (int)(issued % C::OPS), use = (int)(issued / C::OPS);
                if (use >= 1 && !(ok = mbar_wait(&op_empty[st], (use - 1) & 1, p.err, abort_flag))) break;
                mbar_arrive_expect_tx(&op_full[st], (t0 >= 0 ? 16384u : 0u) + (t1 >= 0 ? 16384u : 0u));
                uint8_t* dst = op_ring + st * C::OP_BYTES;
                if (t0 >= 0) {
                  tma_load_2d(dst, &kmap, &op_full[st], 0, t0 * kPage);
                  tma_load_2d(dst + C::CHUNK_BYTES, &kmap, &op_full[st], 64, t0 * kPage);
                }
                if (t1 >= 0) {
                  tma_load_2d(dst + 8192, &kmap, &op_full[st], 0, t1 * kPage);
                  tma_load_2d(dst + C::CHUNK_BYTES + 8192, &kmap, &op_full[st], 64, t1 * kPage);
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
        for (int s = 0; s < C::OPS && !FP8; ++s)
          if (i > s) drain_wait(&op_full[s], (uint32_t)(((i - 1 - s) / C::OPS) & 1), p.err);
        if constexpr (FP8) {
          for (int s = 0; s < C::STS; ++s)
            if (i > s) drain_wait(&st_full[s], (uint32_t)(((i - 1 - s) / C::STS) & 1), p.err);
        }
        for (int q = 0; q < C::QS; ++q)
          if (m >= q) drain_wait(&q_full[q], (uint32_t)(((m - q) / C::QS) & 1), p.err);
      }
    }
  } else if (warp == 1 || (C::MMA_WARPS == 2 && warp == C::MMA2)) {
    // ------------------------------------------------------------------ MMA issuer(s)
    const int par = warp == 1 ? 0 : 1;  // with two issuers: the parity of the tiles this one issues
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
        if (C::MMA_WARPS == 2 && (int)(i & 1) != par) {  // the other issuer's tile
          ++i;
          continue;
        }
        const int s = (int)(i % C::OPS), use = (int)(i / C::OPS);
        if (!(ok = mbar_wait(&op_full[s], use & 1, p.err, abort_flag))) break;
        const int a = (int)(i & 1), ause = (int)(i >> 1);
        if (ause >= 1 && !(ok = mbar_wait(&acc_empty[a], (ause - 1) & 1, p.err, abort_flag))) break;
        tc_fence_after();
        // 8 MMAs of K = 16: two 64-dim column blocks, four K steps of 32 bytes each (the
        // descriptor's start-address field counts 16-byte units)
        const uint64_t bd = sw128_desc(smem_u32(q_slots + slot * C::Q_BYTES), 16, 1024);
        const uint32_t d = tmem_base + (uint32_t)(a * C::N);
        constexpr uint64_t ac = C::CHUNK_BYTES >> 4, bc = C::Q_CHUNK >> 4;
        if constexpr (C::TMEM_A) {
          // A = the f16 key tile in tensor memory: one K step of 16 dims = 8 columns
          const uint32_t at = tmem_base + a_stage_col<C::N>(s);
          umma_ts<0>(d, at, bd, idesc);
          umma_ts<1>(d, at + 8, bd + 2, idesc);
          umma_ts<1>(d, at + 16, bd + 4, idesc);
          umma_ts<1>(d, at + 24, bd + 6, idesc);
          umma_ts<1>(d, at + 32, bd + bc, idesc);
          umma_ts<1>(d, at + 40, bd + bc + 2, idesc);
          umma_ts<1>(d, at + 48, bd + bc + 4, idesc);
          umma_ts<1>(d, at + 56, bd + bc + 6, idesc);
        } else {
          const uint64_t ad = sw128_desc(smem_u32(op_ring + s * C::OP_BYTES), 16, 1024);
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
  } else if (warp < C::CONV0) {
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - 2;                   // epilogue warp
    const int eset = ew >> 2;                  // its set
    const int quarter = warp & 3;              // TMEM lanes this warp may access
    const int q0 = C::EPI_ALT ? 0 : eset * C::EPI_NQ;  // first query of the group this warp scores
    const int t0 = C::EPI_ALT ? eset : 0;      // first tile of this warp, then every tstep-th
    constexpr int tstep = C::EPI_ALT ? 2 : 1;
    const int r = quarter * 32 + lane;         // key row of the tile
    float* w_mine = w_s + ew * C::EPI_NQ * kHeads;  // this warp's copy of its queries' w
    const int64_t ntl = hi - lo;               // tiles of this CTA
    bool ok = true;
    // Tile `it` seen C::LOOK of this warp's tiles ahead: note whether this row's page exists and
    // (e4m3) start the copy of the row's key scale; each thread reads back only what it wrote
    // itself, after its own cp.async group of that tile has completed.  One group is committed per
    // tile of this warp (empty past the end) so that the group count stays in step.
    auto look = [&](int64_t it) {
      if (it < ntl && ok) {
        const int c = (int)(it % C::TIS);
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
    Walk<NQ> W;
    W.init(p, lo, hi);
    int grp, j, last = -1;
    int npos[C::EPI_NQ];
    int64_t i = 0;
    while (ok && W.next(p, grp, j)) {
      if ((i & (tstep - 1)) != t0) {  // the other set's tile
        ++i;
        continue;
      }
      if (grp != last) {
        __syncwarp();
        for (int e = lane; e < C::EPI_NQ * kHeads; e += 32) w_mine[e] = p.w[(int64_t)(grp * NQ + q0) * kHeads + e];
        __syncwarp();
#pragma unroll
        for (int qi = 0; qi < C::EPI_NQ; ++qi) npos[qi] = p.q_pos[grp * NQ + q0 + qi] + 1;
        last = grp;
      }
      cp_async_wait<C::LOOK - 1>();  // this tile's group (committed LOOK tiles ago) has landed
      const int c = (int)(i % C::TIS);
      const bool present = pr_ring[c * kTileKeys + r] != 0;
      const float scale = FP8 ? sc_ring[c * kTileKeys + r] : 1.0f;
      const int a = (int)(i & 1), use = (int)(i >> 1);
      if (!warp_wait(&acc_full[a], use & 1, p.err, abort_flag)) break;
      tc_fence_after();
      const int s = j * kTileKeys + r;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * C::N + q0 * kHeads);
#pragma unroll
      for (int qi = 0; qi < C::EPI_NQ; ++qi) {
        uint32_t v[64];
        tmem_ld16(tbase + qi * 64 + 0, *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
        tmem_ld16(tbase + qi * 64 + 16, *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
        tmem_ld16(tbase + qi * 64 + 32, *reinterpret_cast<uint32_t(*)[16]>(&v[32]));
        tmem_ld16(tbase + qi * 64 + 48, *reinterpret_cast<uint32_t(*)[16]>(&v[48]));
        tmem_wait_ld();
        const float4* w4 = reinterpret_cast<const float4*>(w_mine + qi * kHeads);
        // head pairs in packed f32x2 FMAs, four independent pair accumulators
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int h4 = 0; h4 < 16; ++h4) {
          const float4 wv = w4[h4];
          uint64_t* ac = acc + (h4 & 1) * 2;
          ac[0] = ffma2(wv.x, wv.y, fmaxf(__uint_as_float(v[4 * h4 + 0]), 0.0f), fmaxf(__uint_as_float(v[4 * h4 + 1]), 0.0f), ac[0]);
          ac[1] = ffma2(wv.z, wv.w, fmaxf(__uint_as_float(v[4 * h4 + 2]), 0.0f), fmaxf(__uint_as_float(v[4 * h4 + 3]), 0.0f), ac[1]);
        }
        float sum = 0.0f;
        {
          float lo[4], hi[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) unpack2(acc[e], lo[e], hi[e]);
          sum = ((lo[0] + hi[0]) + (lo[1] + hi[1])) + ((lo[2] + hi[2]) + (lo[3] + hi[3]));
        }
        if (present && s < npos[qi]) p.scores[(int64_t)(grp * NQ + q0 + qi) * p.ld + s] = sum * scale;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[a]);
      look(i + (int64_t)C::LOOK * tstep);  // after this tile is released, so that the producer can get there
      ++i;
    }
    cp_async_wait_all();  // no copy may land after the CTA's shared memory is released
  } else if constexpr (FP8) {
    // ------------------------------------------------------------------ fp8 -> f16 converter
    const int cw = warp - C::CONV0;  // 0 .. CONV_WARPS-1
    const int ct = tid - 32 * C::CONV0;
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
        for (int off = ct * 16; off < C::Q_BYTES; off += 32 * C::CONV_WARPS * 16)
          *reinterpret_cast<uint4*>(q + off) = bf16x8_to_f16(*reinterpret_cast<const uint4*>(q + off));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_ready[slot]);
      }
      const int s8 = (int)(i % C::STS), u8 = (int)(i / C::STS);
      if (!warp_wait(&st_full[s8], u8 & 1, p.err, abort_flag)) break;
      const int so = (int)(i % C::OPS), uo = (int)(i / C::OPS);
      if (uo >= 1 && !warp_wait(&op_empty[so], (uo - 1) & 1, p.err, abort_flag)) break;
      const uint8_t* src = st_ring + s8 * C::ST_BYTES;
      if constexpr (C::TMEM_A) {
        // this thread: key row `row` (its TMEM lane); the staging tile is 128B-swizzled, so the
        // lanes of a warp read distinct banks
        tc_fence_after();
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const uint32_t ta = tmem_base + ((uint32_t)(quarter * 32) << 16) + a_stage_col<C::N>(so);
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // dims [64 h, 64 h + 64) -> 32 columns
          uint32_t f[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 in = *reinterpret_cast<const uint4*>(src + sw128_offset(row, h * 4 + c));
            uint4 lo4, hi4;
            e4m3x16_to_f16(in, lo4, hi4);
            f[8 * c + 0] = lo4.x; f[8 * c + 1] = lo4.y; f[8 * c + 2] = lo4.z; f[8 * c + 3] = lo4.w;
            f[8 * c + 4] = hi4.x; f[8 * c + 5] = hi4.y; f[8 * c + 6] = hi4.z; f[8 * c + 7] = hi4.w;
          }
          tmem_st16(ta + h * 32, *reinterpret_cast<uint32_t(*)[16]>(&f[0]));
          tmem_st16(ta + h * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&f[16]));
        }
        tmem_wait_st();
        tc_fence_before();
      } else {
        // 16 codes -> two 16-byte chunks (2 c16, 2 c16 + 1) of the swizzled operand; the 8 threads of a
        // quarter-warp cover one 128-byte row of codes, so the loads are contiguous, and the threads
        // of the second 64-dim block store their odd chunk first, so that each store instruction
        // hits eight distinct 16-byte bank groups
        uint8_t* dst = op_ring + so * C::OP_BYTES;
        constexpr int kSteps = (kTileKeys * kDim / 16) / (32 * (C::CONV_WARPS > 0 ? C::CONV_WARPS : 1));
#pragma unroll
        for (int k = 0; k < kSteps; ++k) {
          const int piece = ct + 32 * C::CONV_WARPS * k;  // 16-byte piece: row piece/8, codes 16 (piece%8) ..
          const int row = piece >> 3, c16 = piece & 7;
          const uint4 in = *reinterpret_cast<const uint4*>(src + row * 128 + c16 * 16);
          uint4 o0, o1;
          e4m3x16_to_f16(in, o0, o1);
          uint8_t* blk = dst + (c16 >> 2) * C::CHUNK_BYTES;
          const uint32_t ch = (uint32_t)(2 * c16) & 7u;
          const bool odd_first = c16 >= 4;
          *reinterpret_cast<uint4*>(blk + sw128_offset(row, ch + (odd_first ? 1u : 0u))) = odd_first ? o1 : o0;
          *reinterpret_cast<uint4*>(blk + sw128_offset(row, ch + (odd_first ? 0u : 1u))) = odd_first ? o0 : o1;
        }
        fence_proxy_async_smem();
      }
      (void)cw;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&op_full[so]);
        mbar_arrive(&st_empty[s8]);
      }
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
    ok = encode_tmap_2d(&kmap, a.keys.data, 1, kDim, rows, kDim, 128, kPage, C::TMEM_A);
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
  cudaLaunchAttribute attrs[2];
  const cudaLaunchConfig_t cfg = launch_config(dim3(num_sms), dim3(C::THREADS), C::SMEM, s, attrs);
  return cudaLaunchKernelEx(&cfg, kern, kmap, qmap, p);
}

}  // namespace

cudaError_t launch_indexer_tc_decode(const IndexerArgs& a, int num_sms, cudaStream_t s) {
  return a.keys.dtype == DSA_E4M3 ? launch_impl<1, true>(a, num_sms, s) : launch_impl<1, false>(a, num_sms, s);
}

cudaError_t launch_indexer_tc_prefill(const IndexerArgs& a, int num_sms, cudaStream_t s) {
  return a.keys.dtype == DSA_E4M3 ? launch_impl<4, true>(a, num_sms, s) : launch_impl<4, false>(a, num_sms, s);
}

}  // namespace dsa
