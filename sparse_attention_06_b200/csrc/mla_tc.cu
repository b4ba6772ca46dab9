// mla_tc.cu -- sparse MLA (MQA mode) over the selected latent rows on tcgen05 tensor cores.
//
// Page "How GLM5.3 Sparse Attention Affects HBM Memory Usage", sections "Sparse MLA" and "MLA
// Modifications": all H heads (128, or GLM-5's 64) share each selected 576-wide latent row (512
// latent + 64 RoPE); the logits are P = Q[H, 576] K^T over the selected rows and the output is
// O = softmax(P) V, where V is the first 512 dims of the same rows.  The softmax is the usual
// scaled one.
//
// Work unit = (query t, key split sp, value half v).  A unit computes, for its slice of the
// query's selected rows (64-row tiles), S = Q K^T on the tensor cores (M = H heads, N = 64 rows,
// K = 576), an online softmax per head row, and O_v += P V_v (M = H heads, N = 256 value dims,
// K = 64 rows) into tensor memory.  With M = 64 the products use lanes 0..15 of each 32-lane
// tensor-memory quarter (GLM-5 shape; every other place is the same).  The full O (512 f32 columns) would fill tensor memory, so the
// two value halves run on two CTAs, each recomputing S.
// Tensor memory (512 columns): O_v [0, 256), S [256, 320), and the first 384 dims of Q
// [320, 512) -- the S products read those as the A operand straight from tensor memory, so only
// Q's last 192 dims (48 KB) are read from shared memory.  Shared memory holds a two-stage ring of
// gathered rows (72 KB per 64-row tile, 128B-swizzled: the same bytes serve as the K-major B of
// Q K^T and the MN-major B of P V) and P (16 KB).  A tensor-core instruction costs a roughly fixed
// issue time of ~40-50 cycles below N = 128, so 64-row tiles halve the issue cost per row
// against 32-row tiles.
// With several key splits per query each unit writes (O / l, LSE) partials that a small combine
// kernel merges: O = sum_sp exp(LSE_sp - LSE) O_sp, LSE = log sum_sp exp(LSE_sp).
//
// Roles (320 threads): warps 0-3 look up the rows of their 16 keys per tile and gather them with
// TMA (tile::gather4: four rows x 128 bytes per instruction, 128B-swizzled by the copy itself;
// unused slots point past the pool and read as zeros), and write Q into tensor memory (warp 0
// lane 0 also loads Q's shared-memory part by TMA) after issuing the unit's first gathers, so
// that both loads are in flight together; warp 4 owns tensor memory and issues the Q K^T
// products; warps 5-8 run the softmax and the epilogue (one head row per thread); warp 9 issues
// the P V products.  One thread issues a tensor-core instruction about every 60 cycles, so the two
// product chains get separate issuing threads: the Q K^T chain of the next tile does not hold
// back P V, which frees the row-ring stage for the next gather.
// When every CTA runs a single unit (few queries, latency-bound), Q instead arrives by TMA: the
// P V thread loads it at the start, dims [0, 320) into the then idle ring stage 1 and P buffer,
// and the softmax warps, idle until the first S, move each head row from there to tensor memory
// (per-lane loads of 16-byte pieces of 128 rows would keep L1 busy for microseconds); and the
// gather warps, idle by the epilogue, store half of O.
// All waits are bounded; bad indices / block ids set the device error word and are skipped.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {


constexpr int kDqk = 576;       // latent + rope
constexpr int kDv = 512;        // value dims
constexpr int kHalf = 256;      // value dims per CTA
constexpr int kTile = 64;       // rows per tile (MMA N of Q K^T, MMA K of P V)
constexpr int kChunks = 9;      // 64-dim column blocks of a row
constexpr int kTmemQChunks = 6; // Q column blocks held in tensor memory
constexpr int kPage = 64;
constexpr int kStages = 2;      // gathered-row ring
constexpr int kGatherWarps = 4;
constexpr int kKeysPerWarp = kTile / kGatherWarps;  // 16
constexpr int kPvWarp = kGatherWarps + 5;                 // issues the P V products
constexpr int kThreads = 32 * (kGatherWarps + 1 + 4 + 1);

constexpr int K_CHUNK = kTile * 128;                         // 8 KB: 64 rows x 64 dims
constexpr int K_BYTES = kChunks * K_CHUNK;                   // 72 KB
constexpr int NBAR = 2 + 3 * kStages + 8;
constexpr int kQStaged = 5;                                  // staged Q: 64-dim boxes through shared memory
static_assert(kQStaged + 1 == kTmemQChunks, "the last tensor-memory Q box is loaded directly");

// Shapes that depend on the head count H (the MMA M: 128, or 64 for the GLM-5 shape).  With
// M = 64 a product's rows sit in lanes 0..15 of each 32-lane tensor-memory quarter (row m in lane
// 32 (m / 16) + m % 16), so a warp owns RQ = H / 4 head rows of its quarter: lanes 0..RQ-1.
template <int H>
struct HCfg {
  static_assert(H == 64 || H == 128, "tensor-core MLA heads");
  static constexpr int RQ = H / 4;                              // head rows per lane quarter
  static constexpr int Q_CHUNK = H * 128;                       // H head rows x 64 dims
  static constexpr int QS_BYTES = (kChunks - kTmemQChunks) * Q_CHUNK;  // Q in shared memory
  static constexpr int P_BYTES = H * kTile * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QS_BYTES;
  static constexpr int OFF_P = OFF_K + kStages * K_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int OFF_MASK = OFF_BAR + NBAR * 8;         // valid-row masks [stage][gather warp]
  static constexpr int OFF_MISC = OFF_MASK + kStages * kGatherWarps * 4;
  static constexpr int OFF_STATS = OFF_MISC + 32;             // 1 / l of each head row (last unit)
  static constexpr int BYTES = OFF_STATS + H * 4;
  static constexpr int SMEM = BYTES + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(4 * Q_CHUNK <= K_BYTES && Q_CHUNK == P_BYTES, "staging: 4 boxes in ring stage 1, 1 in P");
};

constexpr uint32_t TM_O = 0;       // O half: columns [0, 256)
constexpr uint32_t TM_S = 256;     // S: [256, 320)
constexpr uint32_t TM_Q = 320;     // Q dims [0, 384) as bf16 pairs: [320, 512)
constexpr uint32_t TM_COLS = 512;

struct Params {
  const __nv_bfloat16* latent;   // pool rows of 576
  const __nv_bfloat16* q;        // [T, H, 576]
  const int32_t* idx;
  const int32_t* q_req;
  const int32_t* q_pos;
  const int32_t* block_table;
  __nv_bfloat16* out;            // [T, H, 512] (single split)
  float* lse;                    // [T, H] or null (single split)
  float* part_o;                 // [T, nsplit, H, 512] (several splits)
  float* part_lse;               // [T, nsplit, H]
  int64_t num_blocks;
  int32_t oob_row;               // first row past the pool (gathered as zeros)
  int T, k, ks, nsplit, num_reqs, max_blocks, max_context;
  bool dense;                    // no selection (idx null): every visible position, slot j = position j
  float scale_log2;              // softmax scale * log2(e)
  int* err;
};

// 2^x by the hardware approximation (relative error ~2^-22, far below the bf16 rounding of P);
// 2^-inf = 0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Unit u -> (t, split, half): the two halves of one (t, split) are adjacent so that they run
// concurrently and the second gather of each row hits L2.
__device__ __forceinline__ void unit_coords(const Params& p, int u, int& t, int& sp, int& v) {
  v = u & 1;
  const int ts = u >> 1;
  t = ts / p.nsplit;
  sp = ts % p.nsplit;
}

// Row lookup of selection slot `slot` of query t in two halves, so that the dependent loads
// can be issued a tile apart: the selected position of a slot (kNoSlot when the slot is outside
// the split or the selection) ...
constexpr int kNoSlot = -2;
// (Not gated by the query's validity, so that the load does not wait for the loads behind it:
// pos_block applies that gate where the position is used, a tile later.)
__device__ __forceinline__ int slot_pos(const Params& p, int t, int sp, int slot) {
  if (slot >= min(p.k, (sp + 1) * p.ks)) return kNoSlot;
  if (p.dense) return slot;
  return p.idx[(int64_t)t * p.k + slot];
}
// ... and the physical block holding it (-1 when unused or out of range; flagged when `report`).
__device__ __forceinline__ int pos_block(const Params& p, bool qok, int req, int pos, int ps, bool report) {
  if (!qok || ps == kNoSlot || ps == -1) return -1;
  if (ps < 0 || ps > pos) {
    if (report && !p.dense) raise_error(p.err, DSA_DEVERR_INDEX);  // dense: slots past the query are unused
    return -1;
  }
  const int lblk = ps / kPage;
  const int blk = lblk < p.max_blocks ? p.block_table[(int64_t)req * p.max_blocks + lblk] : -1;
  if (blk < 0 || blk >= p.num_blocks) {
    if (report) raise_error(p.err, DSA_DEVERR_BLOCK_ID);
    return -1;
  }
  return blk;
}

// Pull the H x 576 query block of query t into L2 ahead of its use (16 KB pieces).
template <int H>
__device__ __forceinline__ void prefetch_q(const Params& p, int t) {
  const uint8_t* src = reinterpret_cast<const uint8_t*>(p.q + (int64_t)t * H * kDqk);
#pragma unroll 1
  for (int off = 0; off < H * kDqk * 2; off += 16384) prefetch_l2_bulk(src + off, 16384u);
}

// Staging place of the staged Q's box c (dims [64 c, 64 c + 64), H rows, 128B-swizzled,
// 1024-byte aligned): boxes 0..3 in ring stage 1, box 4 in the P buffer.
template <int H>
__device__ __forceinline__ uint8_t* q_stage_box(uint8_t* smem, int c) {
  using HC = HCfg<H>;
  return c < 4 ? smem + HC::OFF_K + K_BYTES + c * HC::Q_CHUNK : smem + HC::OFF_P;
}

// 64-row tiles of unit (t, sp): its split's share of the k selection slots, or, without a
// selection, of the query's visible positions.
__device__ __forceinline__ int unit_tiles(const Params& p, int t, int sp) {
  const int first = sp * p.ks;
  const int slots = p.dense ? min(p.k, max(0, p.q_pos[t] + 1)) : p.k;
  const int n = min(p.ks, slots - first);
  return n > 0 ? (n + kTile - 1) / kTile : 0;
}

// The RQ head rows of this warp's tensor-memory lane quarter (lanes 0..RQ-1), columns [c_lo,
// c_hi) of O_v / l (multiples of 64), from tensor memory to the partials (f32, with key splits) or
// the output (bf16), through a 4 KB staging area: lane i stages its row (128 bytes per block,
// 16-byte pieces XOR-permuted by i mod 8), then the warp writes rows 4k + lane/8, piece lane mod
// 8, so that each global store instruction writes four whole 128-byte row pieces (lanes past RQ
// stage nothing that is written).  prow / orow: this lane's partial / output row (rows of a
// quarter are consecutive).  have_o false (a unit without rows) stores zeros.
template <int H>
__device__ __forceinline__ void store_o(const Params& p, uint32_t lane_base, int c_lo, int c_hi, uint8_t* stage,
                                        float inv, bool have_o, int64_t prow, int64_t orow, int v) {
  constexpr int RQ = HCfg<H>::RQ;
  const int lane = threadIdx.x & 31;
  const int srow = lane >> 3, spiece = lane & 7;
  const bool f32out = p.nsplit > 1;
  // partial / output row of the quarter's first head row (every lane's r is that plus lane % RQ)
  const int64_t prow0 = prow - lane % RQ, orow0 = orow - lane % RQ;
  // write the staged 128-byte block of each of this warp's rows to columns [col, col + 128 B)
  auto flush = [&](int col) {
    __syncwarp();
#pragma unroll
    for (int k4 = 0; k4 < HCfg<H>::RQ / 4; ++k4) {
      const int rr = k4 * 4 + srow;  // row within this warp's RQ
      const uint4 x = *reinterpret_cast<const uint4*>(stage + rr * 128 + ((spiece ^ (rr & 7)) << 4));
      if (f32out)
        *reinterpret_cast<uint4*>(p.part_o + (prow0 + rr) * kDv + v * kHalf + col + spiece * 4) = x;
      else
        *reinterpret_cast<uint4*>(p.out + (orow0 + rr) * kDv + v * kHalf + col + spiece * 8) = x;
    }
    __syncwarp();
  };
#pragma unroll 1
  for (int c0 = c_lo; c0 < c_hi; c0 += 64) {
    uint32_t o[64];
    if (have_o) {
      tmem_ld16(lane_base + TM_O + c0, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
      tmem_ld16(lane_base + TM_O + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&o[16]));
      tmem_ld16(lane_base + TM_O + c0 + 32, *reinterpret_cast<uint32_t(*)[16]>(&o[32]));
      tmem_ld16(lane_base + TM_O + c0 + 48, *reinterpret_cast<uint32_t(*)[16]>(&o[48]));
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int c = 0; c < 64; ++c) o[c] = 0u;
    }
    uint8_t* srow_ptr = stage + lane * 128;  // (staged only by lanes 0..RQ-1: RQ * 128 bytes)
    if (f32out) {
      // two blocks of 32 f32 columns
#pragma unroll
      for (int b = 0; b < 2; ++b) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int c = 32 * b + 4 * j;
          if (lane < RQ)
            *reinterpret_cast<float4*>(srow_ptr + ((j ^ (lane & 7)) << 4)) =
                make_float4(__uint_as_float(o[c]) * inv, __uint_as_float(o[c + 1]) * inv,
                            __uint_as_float(o[c + 2]) * inv, __uint_as_float(o[c + 3]) * inv);
        }
        flush(c0 + 32 * b);
      }
    } else {
      // one block of 64 bf16 columns
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 hv = __floats2bfloat162_rn(__uint_as_float(o[8 * j + 2 * e]) * inv,
                                                          __uint_as_float(o[8 * j + 2 * e + 1]) * inv);
          pk[e] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        if (lane < RQ) *reinterpret_cast<uint4*>(srow_ptr + ((j ^ (lane & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      flush(c0);
    }
  }
}

template <int H, bool kStagedQ, bool kDense>
__global__ void __launch_bounds__(kThreads, 1)
    mla_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap lmap,
                  const __grid_constant__ CUtensorMap pmap, const Params p) {
  using HC = HCfg<H>;
  constexpr int RQ = HC::RQ;
  constexpr int Q_CHUNK = HC::Q_CHUNK;
  constexpr int QS_BYTES = HC::QS_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem + HC::OFF_Q;
  uint8_t* k_ring = smem + HC::OFF_K;
  uint8_t* p_s = smem + HC::OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + HC::OFF_BAR);
  uint64_t* q_full = bars + 0;                 // Q of the unit in place (TMEM part + smem part)
  uint64_t* q_empty = bars + 1;                // the unit's last Q K^T has completed
  uint64_t* k_full = bars + 2;                 // [kStages] rows landed
  uint64_t* k_empty = k_full + kStages;        // [kStages] P V of the stage done
  uint64_t* m_full = k_empty + kStages;        // [kStages] valid-row masks published
  uint64_t* s_full = m_full + kStages;         // S computed
  uint64_t* s_empty = s_full + 1;              // S read by the softmax
  uint64_t* p_full = s_empty + 1;              // P written
  uint64_t* pv_done = p_full + 1;              // P V completed
  uint64_t* mma_fin = pv_done + 1;
  uint64_t* q_first = mma_fin + 1;             // staged Q: all of it in place
  uint64_t* q_stage = q_first + 1;             // staged Q: dims [0, 320) in shared memory
  uint64_t* ep_half = q_stage + 1;             // last unit: row statistics published after its last P V
  float* stats = reinterpret_cast<float*>(smem + HC::OFF_STATS);
  uint32_t* masks = reinterpret_cast<uint32_t*>(smem + HC::OFF_MASK);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + HC::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + HC::OFF_MISC + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int units = p.T * p.nsplit * 2;
  // kStagedQ (every CTA runs one unit: few queries): Q is staged by TMA in the then idle ring
  // stage 1 and P buffer and moved to tensor memory by the softmax warps; otherwise the gather
  // warps copy each unit's Q.  Two instantiations, so that neither carries the other's code.
  constexpr bool staged_q = kStagedQ;
  griddep_launch_dependents();

  if (tid == 0) {
    if (blockIdx.x < units) {
      int t0, sp0, v0;
      unit_coords(p, blockIdx.x, t0, sp0, v0);
      prefetch_q<H>(p, t0);
    }
    mbar_init(q_full, 32 * kGatherWarps + 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&k_full[i], kGatherWarps);
      mbar_init(&k_empty[i], 1);
      mbar_init(&m_full[i], kGatherWarps);
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, 4);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(mma_fin, 2);  // both issuing threads
    mbar_init(q_first, 128 + 1);  // softmax threads + the TMA issue
    mbar_init(q_stage, 1);
    mbar_init(ep_half, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kGatherWarps) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // the selection comes from the previous kernel of the stream

  if (warp < kGatherWarps) {
    // ------------------------------------------------------------------ Q and row gather
    const int gw = warp;                  // keys gw*16 .. gw*16+15 of each tile; head rows gw*RQ..
    // this lane's head row (lanes past RQ, which hold no row with H = 64, repeat one: they fill
    // tensor-memory lanes no product reads)
    const int h = gw * RQ + (lane % RQ);
    const uint32_t my_lanes = tmem + ((uint32_t)(gw * 32) << 16);
    int gi = 0;  // CTA-wide tile counter
    int ui = 0;  // CTA-wide unit counter
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++ui) {
      int t, sp, v;
      unit_coords(p, u, t, sp, v);
      if (gw == 0 && lane == 0 && u + (int)gridDim.x < units) {
        int tn, spn, vn;
        unit_coords(p, u + gridDim.x, tn, spn, vn);
        if (tn != t) prefetch_q<H>(p, tn);  // the next unit's queries, while this one runs
      }
      // Row lookups of this warp's 16 keys per tile (lanes 0..15), software-pipelined so that no
      // load is waited on in the tile it is issued: the selected position two tiles ahead and the
      // block id one tile ahead.  The first ones are issued before the Q copy below.
      const int req = p.q_req[t];
      const int pos = p.q_pos[t];
      const bool qok = req >= 0 && req < p.num_reqs && pos >= 0 && pos < p.max_context;
      const int ntiles = unit_tiles(p, t, sp);
      const bool mine = lane < kKeysPerWarp;
      const int kslot = sp * p.ks + gw * kKeysPerWarp + lane;
      int ps_j = mine && ntiles > 0 ? slot_pos(p, t, sp, kslot) : kNoSlot;
      int ps_j1 = mine && ntiles > 1 ? slot_pos(p, t, sp, kslot + kTile) : kNoSlot;
      // Q of the unit (unless staged), once the previous unit's Q K^T products are done with it,
      // after the unit's first row gathers are issued: the shared-memory part by TMA, and this
      // thread's head row, dims [0, 384), into tensor-memory columns [320, 512)
      auto copy_q = [&]() -> bool {
        if (ui >= 1 && !warp_wait(q_empty, (ui - 1) & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        if (gw == 0 && lane == 0) {
          mbar_arrive_expect_tx(q_full, QS_BYTES);
          for (int c = kTmemQChunks; c < kChunks; ++c)
            tma_load_2d(q_s + (c - kTmemQChunks) * Q_CHUNK, &qmap, q_full, c * 64, t * H);
        }
        const uint4* src = reinterpret_cast<const uint4*>(p.q + ((int64_t)t * H + h) * kDqk);
#pragma unroll 1
        for (int b = 0; b < 2; ++b) {  // 192 dims = 96 columns per batch, all loads in flight
          uint32_t w[96];
#pragma unroll
          for (int e = 0; e < 24; ++e) {
            const uint4 x = __ldg(src + b * 24 + e);
            w[4 * e] = x.x; w[4 * e + 1] = x.y; w[4 * e + 2] = x.z; w[4 * e + 3] = x.w;
          }
#pragma unroll
          for (int c = 0; c < 6; ++c)
            tmem_st16(my_lanes + TM_Q + b * 96 + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&w[c * 16]));
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(q_full);
        return true;
      };
      if (!qok && tid == 0 && v == 0 && sp == 0) raise_error(p.err, DSA_DEVERR_REQUEST);
      int blk_j = mine ? pos_block(p, qok, req, pos, ps_j, v == 0) : -1;
      for (int j = 0; j < ntiles; ++j, ++gi) {
        const int s = gi % kStages;
        const int64_t row = blk_j >= 0 ? (int64_t)blk_j * kPage + (ps_j % kPage) : -1;
        const int blk_j1 = mine && j + 1 < ntiles ? pos_block(p, qok, req, pos, ps_j1, v == 0) : -1;
        const int ps_j2 = mine && j + 2 < ntiles ? slot_pos(p, t, sp, kslot + (j + 2) * kTile) : kNoSlot;
        if (gi >= kStages && !(ok = warp_wait(&k_empty[s], ((gi / kStages) - 1) & 1, p.err, abort_flag))) break;
        // a staged Q sits in ring stage 1 until the softmax warps have moved it
        if constexpr (staged_q)
          if (gi == 1 && !(ok = warp_wait(q_first, 0, p.err, abort_flag))) break;
        // publish which of this warp's rows are real to the softmax warps
        const uint32_t vmask = __ballot_sync(0xFFFFFFFFu, row >= 0) & ((1u << kKeysPerWarp) - 1u);
        if (lane == 0) {
          masks[s * kGatherWarps + gw] = vmask;
          mbar_arrive(&m_full[s]);
        }
        ps_j = ps_j1;
        ps_j1 = ps_j2;
        blk_j = blk_j1;
        // Without a selection a tile is 64 consecutive positions starting at a multiple of 64:
        // one whole page when every position is visible and the page exists.  Such a tile comes
        // in as nine 64-row boxes (warp 0), every other tile as gathered rows, this warp's 16 as
        // four gather4 groups of four rows x nine 64-dim column blocks (rows past the pool,
        // never read, for the unused slots).  The byte count is the same either way.
        const int32_t rc = row >= 0 ? (int32_t)row : p.oob_row;
        uint8_t* stage = k_ring + s * K_BYTES + gw * kKeysPerWarp * 128;
        bool whole_page = false;
        if constexpr (kDense)
          whole_page = sp * p.ks + j * kTile + kTile - 1 <= pos && __all_sync(0xFFFFFFFFu, !mine || row >= 0);
        if (lane == 0) mbar_arrive_expect_tx(&k_full[s], kKeysPerWarp * kDqk * 2);
        if (whole_page) {
          const int32_t prow = __shfl_sync(0xFFFFFFFFu, rc, 0) & ~(kPage - 1);  // the page's first row
          if (gw == 0 && lane == 0) {
#pragma unroll
            for (int c = 0; c < kChunks; ++c) tma_load_2d(k_ring + s * K_BYTES + c * K_CHUNK, &pmap, &k_full[s], c * 64, prow);
          }
        } else
#pragma unroll
        for (int g4 = 0; g4 < kKeysPerWarp / 4; ++g4) {
          const int32_t r0 = __shfl_sync(0xFFFFFFFFu, rc, 4 * g4 + 0);
          const int32_t r1 = __shfl_sync(0xFFFFFFFFu, rc, 4 * g4 + 1);
          const int32_t r2 = __shfl_sync(0xFFFFFFFFu, rc, 4 * g4 + 2);
          const int32_t r3 = __shfl_sync(0xFFFFFFFFu, rc, 4 * g4 + 3);
          if (lane == 0) {
#pragma unroll
            for (int c = 0; c < kChunks; ++c)
              tma_gather4(stage + c * K_CHUNK + g4 * 512, &lmap, &k_full[s], c * 64, r0, r1, r2, r3);
          }
        }
        if constexpr (!staged_q)
          if (j == 0 && !(ok = copy_q())) break;
      }
      if constexpr (!staged_q)
        if (ok && ntiles == 0) ok = copy_q();
      if (ok && u + (int)gridDim.x >= units) {
        // the CTA's last unit: columns [128, 256) of O_v / l, once the softmax warps have published
        // 1 / l (after the unit's last P V, which also frees the row ring for the staging)
        if (!(ok = warp_wait(ep_half, 0, p.err, abort_flag))) break;
        tc_fence_after();
        const int64_t orow = (int64_t)t * H + h;
        const int64_t prow = ((int64_t)t * p.nsplit + sp) * H + h;
        store_o<H>(p, my_lanes, kHalf / 2, kHalf, k_ring + gw * RQ * 128, stats[h], ntiles > 0, prow, orow, v);
        tc_fence_before();
      }
    }
    if (!ok && lane == 0) {
      // gave up: the row copies of the last use of each stage must land before the CTA exits
      for (int t = gi - 1; t >= 0 && t >= gi - kStages; --t)
        mbar_wait(&k_full[t % kStages], (uint32_t)((t / kStages) & 1), p.err, nullptr);
    }
  } else if (warp == kGatherWarps) {
    // ------------------------------------------------------------------ Q K^T issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_f16(1u, 0u, (uint32_t)H, (uint32_t)kTile);  // S: B K-major
      int gi = 0, ui = 0;
      bool ok = true;
      const uint64_t qd = sw128_desc(smem_u32(q_s), 16, 1024);
      const uint32_t d_s = tmem + TM_S, a_q = tmem + TM_Q;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++ui) {
        int t, sp, v;
        unit_coords(p, u, t, sp, v);
        const int ntiles = unit_tiles(p, t, sp);
        if constexpr (staged_q) {
          if (!(ok = mbar_wait(q_first, 0, p.err, abort_flag))) break;
        } else {
          if (!(ok = mbar_wait(q_full, ui & 1, p.err, abort_flag))) break;
        }
        if (ntiles == 0) mma_commit(q_empty);
        for (int j = 0; j < ntiles; ++j) {
          const int g = gi + j, s = g % kStages;
          if (!(ok = mbar_wait(&k_full[s], (g / kStages) & 1, p.err, abort_flag))) break;
          if (g >= 1 && !(ok = mbar_wait(s_empty, (g - 1) & 1, p.err, abort_flag))) break;
          // S[g] = Q K^T: Q dims 0..383 from tensor memory, 384..575 from shared memory
          fence_proxy_async_smem();
          tc_fence_after();
          const uint64_t kd = sw128_desc(smem_u32(k_ring + s * K_BYTES), 16, 1024);
          constexpr uint64_t kc = K_CHUNK >> 4, qc = Q_CHUNK >> 4;
          umma_ts<0>(d_s, a_q + 0, kd + 0, idesc_s);
#pragma unroll
          for (int i = 1; i < 4 * kTmemQChunks; ++i)  // chunk i/4, K step i%4: 8 TMEM columns, 32 B
            umma_ts<1>(d_s, a_q + (uint32_t)(i * 8), kd + (uint64_t)(i >> 2) * kc + (uint64_t)(i & 3) * 2, idesc_s);
#pragma unroll
          for (int i = 0; i < 4 * (kChunks - kTmemQChunks); ++i)
            umma_ss<1>(d_s, qd + (uint64_t)(i >> 2) * qc + (uint64_t)(i & 3) * 2,
                       kd + (uint64_t)(kTmemQChunks + (i >> 2)) * kc + (uint64_t)(i & 3) * 2, idesc_s);
          mma_commit(s_full);
          if (j == ntiles - 1) mma_commit(q_empty);  // last use of Q by this unit
        }
        gi += ntiles;
      }
      // every MMA issued by this thread has completed before TMEM is released
      mma_commit(mma_fin);
      mbar_wait(mma_fin, 0, p.err, nullptr);
    }
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------------ P V issuer
    if (lane == 0) {
      if constexpr (staged_q) {
        // the unit's Q by TMA: dims [384, 576) to their place, dims [0, 320) staged in ring stage 1
        // (64-dim boxes 0..3) and the P buffer (box 4) for the softmax warps
        int t0, sp0, v0;
        unit_coords(p, blockIdx.x, t0, sp0, v0);
        mbar_arrive_expect_tx(q_first, QS_BYTES);
        for (int c = kTmemQChunks; c < kChunks; ++c)
          tma_load_2d(q_s + (c - kTmemQChunks) * Q_CHUNK, &qmap, q_first, c * 64, t0 * H);
        mbar_arrive_expect_tx(q_stage, kQStaged * Q_CHUNK);
        for (int c = 0; c < kQStaged; ++c)
          tma_load_2d(q_stage_box<H>(smem, c), &qmap, q_stage, c * 64, t0 * H);
      }
      const uint32_t idesc_o = idesc_f16(1u, 1u, (uint32_t)H, (uint32_t)kHalf);  // O: B (V) MN-major
      // P [128 x 64] K-major, no swizzle: 8x16-byte core matrices 128 B apart along K and 1024 B
      // apart along M; one K step (16 keys) is two core matrices = 256 bytes
      const uint64_t pd = noswz_desc(smem_u32(p_s), 128, 1024);
      const uint32_t d_o = tmem + TM_O;
      int gi = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int t, sp, v;
        unit_coords(p, u, t, sp, v);
        const int ntiles = unit_tiles(p, t, sp);
        for (int j = 0; j < ntiles; ++j) {
          const int g = gi + j, s = g % kStages;
          if (!(ok = mbar_wait(p_full, g & 1, p.err, abort_flag))) break;
          // O_v += P V_v; V is MN-major 128B-swizzled: 64-dim blocks K_CHUNK apart, 8-row groups
          // 1024 B apart, one K step (16 rows) = 2048 bytes
          tc_fence_after();
          const uint64_t vd = sw128_desc(smem_u32(k_ring + s * K_BYTES) + (uint32_t)(v * 4 * K_CHUNK), K_CHUNK, 1024);
          if (j > 0)
            umma_ss<1>(d_o, pd, vd, idesc_o);
          else
            umma_ss<0>(d_o, pd, vd, idesc_o);
          umma_ss<1>(d_o, pd + 16, vd + 128, idesc_o);
          umma_ss<1>(d_o, pd + 32, vd + 256, idesc_o);
          umma_ss<1>(d_o, pd + 48, vd + 384, idesc_o);
          mma_commit(pv_done);
          mma_commit(&k_empty[s]);
        }
        gi += ntiles;
      }
      mma_commit(mma_fin);
      mbar_wait(mma_fin, 0, p.err, nullptr);
    }
  } else if (warp < kPvWarp) {
    // ------------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    // this lane's head row; with H = 64 lanes RQ..31 of the quarter hold no row: they see every
    // key as masked and write nothing (their r repeats a row only to keep addresses in range)
    const bool row_lane = lane < RQ;
    const int r = quarter * RQ + (lane % RQ);
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    if constexpr (staged_q) {
      // the staged Q, head row r, dims [0, 384) into tensor-memory columns [320, 512): dims
      // [0, 320) from the staged 128B-swizzled boxes (16-byte piece j of row r sits at piece
      // j ^ (r mod 8)), dims [320, 384) straight from global memory
      int t0, sp0, v0;
      unit_coords(p, blockIdx.x, t0, sp0, v0);
      const uint4* src = reinterpret_cast<const uint4*>(p.q + ((int64_t)t0 * H + r) * kDqk) + 5 * 8;
      uint32_t w[32];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint4 x = __ldg(src + e);
        w[4 * e] = x.x; w[4 * e + 1] = x.y; w[4 * e + 2] = x.z; w[4 * e + 3] = x.w;
      }
      const bool qs_ok = mbar_wait(q_stage, 0, p.err, abort_flag);
#pragma unroll 1
      for (int c = 0; c < kQStaged && qs_ok; ++c) {
        const uint8_t* row = q_stage_box<H>(smem, c) + r * 128;
        uint32_t x[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 y = *reinterpret_cast<const uint4*>(row + ((j ^ (r & 7)) << 4));
          x[4 * j] = y.x; x[4 * j + 1] = y.y; x[4 * j + 2] = y.z; x[4 * j + 3] = y.w;
        }
        tmem_st16(lane_base + TM_Q + c * 32, *reinterpret_cast<uint32_t(*)[16]>(&x[0]));
        tmem_st16(lane_base + TM_Q + c * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&x[16]));
      }
      tmem_st16(lane_base + TM_Q + kQStaged * 32, *reinterpret_cast<uint32_t(*)[16]>(&w[0]));
      tmem_st16(lane_base + TM_Q + kQStaged * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&w[16]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(q_first);
    }
    int gi = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      int t, sp, v;
      unit_coords(p, u, t, sp, v);
      const int ntiles = unit_tiles(p, t, sp);
      float m_used = -INFINITY, l = 0.0f;
      for (int j = 0; j < ntiles; ++j) {
        const int g = gi + j, s = g % kStages;
        if (!(ok = warp_wait(s_full, g & 1, p.err, abort_flag))) break;
        if (!(ok = warp_wait(&m_full[s], (g / kStages) & 1, p.err, abort_flag))) break;
        tc_fence_after();
        uint32_t sv[64];
        tmem_ld16(lane_base + TM_S, *reinterpret_cast<uint32_t(*)[16]>(&sv[0]));
        tmem_ld16(lane_base + TM_S + 16, *reinterpret_cast<uint32_t(*)[16]>(&sv[16]));
        tmem_ld16(lane_base + TM_S + 32, *reinterpret_cast<uint32_t(*)[16]>(&sv[32]));
        tmem_ld16(lane_base + TM_S + 48, *reinterpret_cast<uint32_t(*)[16]>(&sv[48]));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_empty);
        uint64_t valid = 0u;
#pragma unroll
        for (int w = 0; w < kGatherWarps; ++w) valid |= (uint64_t)masks[s * kGatherWarps + w] << (w * kKeysPerWarp);
        if (!row_lane) valid = 0u;
        float mt = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float xv = ((valid >> c) & 1u) ? __uint_as_float(sv[c]) * p.scale_log2 : -INFINITY;
          sv[c] = __float_as_uint(xv);
          mt = fmaxf(mt, xv);
        }
        // the P buffer and O are free once the previous tile's P V has completed
        if (g >= 1 && !(ok = warp_wait(pv_done, (g - 1) & 1, p.err, abort_flag))) break;
        // Lazy rescale: the exponent base m_used only moves when some row's tile maximum exceeds
        // it by more than 2^8 (so P stays <= 256).  The decision is taken for the whole warp,
        // because the tensor-memory loads and stores below are warp-collective; rows whose
        // maximum did not grow get the factor 1.
        if (__any_sync(0xFFFFFFFFu, mt > m_used + 8.0f)) {
          const float m_new = fmaxf(m_used, mt);
          const float f = m_new == -INFINITY ? 1.0f : exp2f(m_used - m_new);  // 0 when m_used = -inf
          if (j > 0) {
            // rescale this row of O before the next P V accumulates into it
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < kHalf; c0 += 32) {
              uint32_t o[32];
              tmem_ld16(lane_base + TM_O + c0, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
              tmem_ld16(lane_base + TM_O + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&o[16]));
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
              tmem_st16(lane_base + TM_O + c0, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
              tmem_st16(lane_base + TM_O + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&o[16]));
            }
            tmem_wait_st();
          }
          l *= f;
          m_used = m_new;
        }
        float psum = 0.0f;
        uint32_t pk[32];
        // 2^(x - m): x = -inf gives 0; while no real row has been seen m_used is -inf and every x is
        // -inf, so the base 0 is used instead
        const float msub = m_used == -INFINITY ? 0.0f : m_used;
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const float p0 = fast_exp2(__uint_as_float(sv[c]) - msub);
          const float p1 = fast_exp2(__uint_as_float(sv[c + 1]) - msub);
          const __nv_bfloat162 b = __floats2bfloat162_rn(p0, p1);
          // the normaliser sums the rounded weights that P V actually uses
          const float2 bf = __bfloat1622float2(b);
          psum += bf.x + bf.y;
          pk[c >> 1] = *reinterpret_cast<const uint32_t*>(&b);
        }
        l += psum;
        // P row r: 8 core-matrix rows of 16 B (8 keys each), no swizzle
        if (row_lane) {
          uint8_t* prow = p_s + (r >> 3) * 1024 + (r & 7) * 16;
#pragma unroll
          for (int kc = 0; kc < 8; ++kc)
            *reinterpret_cast<uint4*>(prow + kc * 128) = make_uint4(pk[4 * kc], pk[4 * kc + 1], pk[4 * kc + 2], pk[4 * kc + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full);
      }
      if (!ok) break;
      gi += ntiles;
      // epilogue: wait for the unit's last P V, then O / l and the LSE
      if (ntiles > 0 && !(ok = warp_wait(pv_done, (gi - 1) & 1, p.err, abort_flag))) break;
      tc_fence_after();
      const float inv = l > 0.0f ? 1.0f / l : 0.0f;
      const float lse = l > 0.0f ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
      const int64_t orow = (int64_t)t * H + r;
      const int64_t prow = ((int64_t)t * p.nsplit + sp) * H + r;
      // O / l leaves through this warp's quarter of the P buffer (RQ * 128 bytes; free: the last
      // P V has completed).  In the CTA's last unit the gather warps, idle by then, store the columns
      // [128, 256) of the half: they get 1 / l through shared memory once the last P V is done.
      const bool last = u + (int)gridDim.x >= units;
      if (last) {
        if (row_lane) stats[r] = inv;
        mbar_arrive(ep_half);
      }
      store_o<H>(p, lane_base, 0, last ? kHalf / 2 : kHalf, p_s + quarter * RQ * 128, inv, ntiles > 0, prow, orow, v);
      if (v == 0 && row_lane) {
        if (p.nsplit == 1) {
          if (p.lse) p.lse[orow] = lse;
        } else {
          p.part_lse[prow] = lse;
        }
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kGatherWarps) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

// grid (T, H heads), block 256: merge the split partials of one (query, head) row.  The split
// weights exp(LSE_sp - max) go to shared memory first; then thread i sums column group i % 128
// (4 of the 512 value columns) over the splits i / 128, i / 128 + 2, ... with up to 16 loads in
// flight, and the two halves are added through shared memory.
constexpr int kMaxSplits = 64;
constexpr int kCombThreads = 256;
template <int H>
__global__ void __launch_bounds__(kCombThreads) mla_combine_kernel(const float* __restrict__ part_o,
                                                                   const float* __restrict__ part_lse, int nsplit,
                                                                   __nv_bfloat16* __restrict__ out,
                                                                   float* __restrict__ lse_out) {
  __shared__ float wts[kMaxSplits];
  __shared__ float4 red[kCombThreads / 2];
  __shared__ float s_inv, s_lse;
  const int t = blockIdx.x, h = blockIdx.y;
  const int c4 = threadIdx.x & 127, half = threadIdx.x >> 7;
  griddep_launch_dependents();
  griddep_wait();  // the partials come from the kernel before
  const int64_t row0 = (int64_t)t * nsplit * H + h;  // partial row of split 0; split sp adds sp*H
  if (threadIdx.x < 32) {
    float mx = -INFINITY;
    for (int sp = threadIdx.x; sp < nsplit; sp += 32) mx = fmaxf(mx, part_lse[row0 + (int64_t)sp * H]);
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    float sum = 0.0f;
    for (int sp = threadIdx.x; sp < nsplit; sp += 32) {
      const float ls = part_lse[row0 + (int64_t)sp * H];
      const float wgt = ls == -INFINITY ? 0.0f : expf(ls - mx);
      wts[sp] = wgt;
      sum += wgt;
    }
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    if (threadIdx.x == 0) {
      s_inv = sum > 0.0f ? 1.0f / sum : 0.0f;
      s_lse = sum > 0.0f ? mx + logf(sum) : -INFINITY;
    }
  }
  __syncthreads();
  float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  const float4* src = reinterpret_cast<const float4*>(part_o + row0 * kDv) + c4;
  const int64_t step = (int64_t)H * kDv / 4;  // float4s from one split's row to the next
  for (int sp0 = half; sp0 < nsplit; sp0 += 32) {
    float4 a[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {  // every load of the batch in flight before the first use
      const int sp = sp0 + 2 * e;
      a[e] = sp < nsplit ? __ldg(src + sp * step) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int sp = sp0 + 2 * e;
      const float wgt = sp < nsplit ? wts[sp] : 0.0f;
      acc.x = fmaf(wgt, a[e].x, acc.x);
      acc.y = fmaf(wgt, a[e].y, acc.y);
      acc.z = fmaf(wgt, a[e].z, acc.z);
      acc.w = fmaf(wgt, a[e].w, acc.w);
    }
  }
  if (half) red[c4] = acc;
  __syncthreads();
  if (!half) {
    const float4 o = red[c4];
    const float inv = s_inv;
    const __nv_bfloat162 lo = __floats2bfloat162_rn((acc.x + o.x) * inv, (acc.y + o.y) * inv);
    const __nv_bfloat162 hi = __floats2bfloat162_rn((acc.z + o.z) * inv, (acc.w + o.w) * inv);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&lo);
    pk.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(out + ((int64_t)t * H + h) * kDv + 4 * c4) = pk;
    if (lse_out && threadIdx.x == 0) lse_out[(int64_t)t * H + h] = s_lse;
  }
}

int split_size(int k, int nsplit) { return ((k + nsplit - 1) / nsplit + kTile - 1) / kTile * kTile; }

// Key splits per query.  Cost model in 64-row tile times: a unit costs its tiles plus a fixed
// ~2.5 (query load, pipeline fill, epilogue), units run in waves of one per SM, and more than one
// split adds the combine pass (a launch, ~2 tiles, plus reading the partials, ~0.02 tile per
// query and split).
int splits_for(int T, int k, int num_sms) {
  double best_cost = 1e300;
  int best = 1;
  for (int n = 1; n <= kMaxSplits; n *= 2) {
    const int ks = split_size(k, n);
    const int ns = (k + ks - 1) / ks;
    const long long units = 2LL * T * ns;
    const double waves = (double)((units + num_sms - 1) / num_sms);
    double cost = waves * ((double)(ks / kTile) + 2.5);
    if (ns > 1) cost += 2.0 + 0.02 * T * ns;
    if (cost < best_cost) {
      best_cost = cost;
      best = ns;
    }
    if (ks == kTile) break;
  }
  return best;
}

}  // namespace

int mla_tc_num_splits(int T, int k, int num_sms) { return splits_for(T, k, num_sms); }

size_t mla_tc_workspace_bytes(int T, int H, int d_v, int nsplit) {
  if (nsplit <= 1) return 0;
  const size_t o = (size_t)T * nsplit * H * d_v * sizeof(float);
  const size_t l = (size_t)T * nsplit * H * sizeof(float);
  return ((o + 255) / 256) * 256 + ((l + 255) / 256) * 256;
}

namespace {

template <int H>
cudaError_t launch_mla_tc_h(const MlaArgs& a, int nsplit, int num_sms, cudaStream_t s) {
  using HC = HCfg<H>;
  const int T = a.batch.num_queries;
  alignas(64) CUtensorMap qmap, lmap, pmap;
  if (!encode_tmap_2d(&qmap, a.q, 2, kDqk, (uint64_t)T * H, kDqk * 2, 64, H, true)) return cudaErrorInvalidValue;
  const uint64_t pool_rows = (uint64_t)a.latent.num_blocks * kPage;
  if (pool_rows >= 0x7FFFFFFFull) return cudaErrorInvalidValue;  // row coordinates are 32-bit
  if (!encode_tmap_2d(&lmap, a.latent.data, 2, kDqk, pool_rows, (uint64_t)kDqk * 2, 64, 1, true))
    return cudaErrorInvalidValue;
  // whole 64-token pages (the dense case): 64-row boxes of one 64-dim column block
  if (!encode_tmap_2d(&pmap, a.latent.data, 2, kDqk, pool_rows, (uint64_t)kDqk * 2, 64, kPage, true))
    return cudaErrorInvalidValue;
  Params p;
  p.latent = static_cast<const __nv_bfloat16*>(a.latent.data);
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.idx = a.idx;
  p.dense = a.idx == nullptr;
  p.q_req = a.batch.q_req;
  p.q_pos = a.batch.q_pos;
  p.block_table = a.batch.block_table;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.num_blocks = a.latent.num_blocks;
  p.oob_row = (int32_t)pool_rows;
  p.T = T;
  p.k = a.k;
  p.nsplit = nsplit;
  p.ks = split_size(a.k, nsplit);
  p.num_reqs = a.batch.num_reqs;
  p.max_blocks = a.batch.max_blocks;
  p.max_context = a.batch.max_context;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.err = a.err;
  p.part_o = nullptr;
  p.part_lse = nullptr;
  if (nsplit > 1) {
    const size_t o = (size_t)T * nsplit * H * kDv * sizeof(float);
    p.part_o = static_cast<float*>(a.workspace);
    p.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(a.workspace) + ((o + 255) / 256) * 256);
  }
  const int units = T * nsplit * 2;
  const int grid = units < num_sms ? units : num_sms;
  // one unit per CTA: staged Q; without a selection: whole pages by 64-row boxes
  auto kernel = units <= grid ? (p.dense ? mla_tc_kernel<H, true, true> : mla_tc_kernel<H, true, false>)
                              : (p.dense ? mla_tc_kernel<H, false, true> : mla_tc_kernel<H, false, false>);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, HC::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attrs[2];
  const cudaLaunchConfig_t cfg = launch_config(dim3(grid), dim3(kThreads), HC::SMEM, s, attrs);
  e = cudaLaunchKernelEx(&cfg, kernel, qmap, lmap, pmap, p);
  if (e != cudaSuccess || nsplit == 1) return e;
  cudaLaunchAttribute cattrs[2];
  const cudaLaunchConfig_t ccfg = launch_config(dim3(T, H), dim3(kCombThreads), 0, s, cattrs);
  return cudaLaunchKernelEx(&ccfg, mla_combine_kernel<H>, (const float*)p.part_o, (const float*)p.part_lse, nsplit,
                            p.out, a.lse);
}

}  // namespace

cudaError_t launch_mla_tc(const MlaArgs& a, int nsplit, int num_sms, cudaStream_t s) {
  return a.H == 64 ? launch_mla_tc_h<64>(a, nsplit, num_sms, s) : launch_mla_tc_h<128>(a, nsplit, num_sms, s);
}

}  // namespace dsa
