// mla_tc.cu -- sparse MLA (MQA mode) over the selected latent rows on tcgen05 tensor cores.
//
// Page "How GLM5.3 Sparse Attention Affects HBM Memory Usage", sections "Sparse MLA" and "MLA
// Modifications": all 128 heads share each selected 576-wide latent row (512 latent + 64 RoPE);
// the logits are P = Q[H, 576] K^T over the selected rows and the output is O = softmax(P) V,
// where V is the first 512 dims of the same rows.  The softmax is the usual scaled one.
//
// Work unit = (query t, key split sp, value half v).  A unit computes, for its slice of the
// query's selected rows (32-row tiles), S = Q K^T on the tensor cores (M = 128 heads, N = 32 rows,
// K = 576), an online softmax per head row, and O_v += P V_v (M = 128 heads, N = 256 value dims,
// K = 32 rows) into tensor memory.  Tensor memory holds O_v (256 columns) and two S buffers
// (32 columns each): the full O (512 columns) would leave no room for S, so the two value halves
// run on two CTAs, each recomputing S.  Q (128 x 576 bf16, 144 KB) stays in shared memory for the
// whole unit; rows are gathered from the paged pool with cp.async into a two-stage ring.
// With several key splits per query each unit writes (O / l, LSE) partials that a small combine
// kernel merges: O = sum_sp exp(LSE_sp - LSE) O_sp, LSE = log sum_sp exp(LSE_sp).
//
// Roles (224 threads): warps 0-1 gather rows (warp 0 lane 0 also loads Q by TMA), warp 2 owns
// TMEM and issues the MMAs, warps 3-6 run the softmax and the epilogue (one head row per thread).
// All waits are bounded; bad indices / block ids set the device error word and are skipped.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {

namespace {

constexpr int kH = 128;         // heads (MMA M)
constexpr int kDqk = 576;       // latent + rope
constexpr int kDv = 512;        // value dims
constexpr int kHalf = 256;      // value dims per CTA
constexpr int kTile = 32;       // rows per tile (MMA N of Q K^T, MMA K of P V)
constexpr int kChunks = 9;      // 64-dim column blocks of a row
constexpr int kPage = 64;
constexpr int kThreads = 224;

constexpr int Q_CHUNK = kH * 128;            // 16 KB: 128 head rows x 64 dims
constexpr int Q_BYTES = kChunks * Q_CHUNK;   // 144 KB
constexpr int K_CHUNK = kTile * 128;         // 4 KB: 32 rows x 64 dims
constexpr int K_BYTES = kChunks * K_CHUNK;   // 36 KB
constexpr int P_BYTES = kH * kTile * 2;      // 8 KB
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + Q_BYTES;
constexpr int OFF_P = OFF_K + 2 * K_BYTES;
constexpr int OFF_BAR = OFF_P + P_BYTES;
constexpr int NBAR = 15;
constexpr int OFF_MASK = OFF_BAR + NBAR * 8;   // valid-row masks: 2 stages x 2 gather warps
constexpr int OFF_MISC = OFF_MASK + 16;
constexpr int BYTES = OFF_MISC + 32;
constexpr int SMEM = BYTES + 1024;
static_assert(SMEM <= 232448, "shared memory budget");

constexpr uint32_t TM_O = 0;       // O half: columns [0, 256)
constexpr uint32_t TM_S = 256;     // S buffers: [256, 288), [288, 320)
constexpr uint32_t TM_COLS = 512;

struct Params {
  const __nv_bfloat16* latent;   // pool rows of 576
  const int32_t* idx;
  const int32_t* q_req;
  const int32_t* q_pos;
  const int32_t* block_table;
  __nv_bfloat16* out;            // [T, 128, 512] (single split)
  float* lse;                    // [T, 128] or null (single split)
  float* part_o;                 // [T, nsplit, 128, 512] (several splits)
  float* part_lse;               // [T, nsplit, 128]
  int64_t num_blocks;
  int T, k, ks, nsplit, num_reqs, max_blocks, max_context;
  float scale_log2;              // softmax scale * log2(e)
  int* err;
};

__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
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
// can be issued a tile apart: the selected position of a slot (kNoSlot when the slot is outside the split or the selection) ...
constexpr int kNoSlot = -2;
__device__ __forceinline__ int slot_pos(const Params& p, int t, bool qok, int sp, int slot) {
  if (!qok || slot >= min(p.k, (sp + 1) * p.ks)) return kNoSlot;
  return p.idx[(int64_t)t * p.k + slot];
}
// ... and the physical block holding it (-1 when unused or out of range; flagged when `report`).
__device__ __forceinline__ int pos_block(const Params& p, int req, int pos, int ps, bool report) {
  if (ps == kNoSlot || ps == -1) return -1;
  if (ps < 0 || ps > pos) {
    if (report) raise_error(p.err, DSA_DEVERR_INDEX);
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

__device__ __forceinline__ int unit_tiles(const Params& p, int sp) {
  const int first = sp * p.ks;
  const int n = min(p.ks, p.k - first);
  return n > 0 ? (n + kTile - 1) / kTile : 0;
}

__global__ void __launch_bounds__(kThreads, 1)
    mla_tc_kernel(const __grid_constant__ CUtensorMap qmap, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_s = smem + OFF_Q;
  uint8_t* k_ring = smem + OFF_K;
  uint8_t* p_s = smem + OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;   // [2]
  uint64_t* k_empty = bars + 4;  // [2]
  uint64_t* s_full = bars + 6;   // [2]
  uint64_t* s_empty = bars + 8;  // [2]
  uint64_t* p_full = bars + 10;
  uint64_t* pv_done = bars + 11;
  uint64_t* mma_fin = bars + 12;
  uint64_t* m_full = bars + 13;  // [2] valid-row mask of a stage published
  uint32_t* masks = reinterpret_cast<uint32_t*>(smem + OFF_MASK);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int units = p.T * p.nsplit * 2;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 64);
      mbar_init(&k_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(mma_fin, 1);
    mbar_init(&m_full[0], 2);
    mbar_init(&m_full[1], 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 2) {
    // ------------------------------------------------------------------ Q TMA + row gather
    const int gw = warp;  // rows 16*gw .. 16*gw+15 of each tile
    int gi = 0;           // CTA-wide tile counter
    int ui = 0;           // CTA-wide unit counter
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++ui) {
      int t, sp, v;
      unit_coords(p, u, t, sp, v);
      const int req = p.q_req[t];
      const int pos = p.q_pos[t];
      const bool qok = req >= 0 && req < p.num_reqs && pos >= 0 && pos < p.max_context;
      if (!qok && tid == 0 && v == 0 && sp == 0) raise_error(p.err, DSA_DEVERR_REQUEST);
      if (warp == 0) {
        if (ui >= 1 && !(ok = warp_wait(q_empty, (ui - 1) & 1, p.err, abort_flag))) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(q_full, Q_BYTES);
          for (int c = 0; c < kChunks; ++c) tma_load_2d(q_s + c * Q_CHUNK, &qmap, q_full, c * 64, t * kH);
        }
      }
      const int ntiles = unit_tiles(p, sp);
      // Row lookups of this warp's 16 keys per tile (lanes 0..15), software-pipelined so that no
      // load is waited on in the tile it is issued: the selected position two tiles ahead and the
      // block id one tile ahead.
      const bool mine = lane < 16;
      const int kslot = sp * p.ks + gw * 16 + lane;
      int ps_j = mine && ntiles > 0 ? slot_pos(p, t, qok, sp, kslot) : kNoSlot;
      int ps_j1 = mine && ntiles > 1 ? slot_pos(p, t, qok, sp, kslot + kTile) : kNoSlot;
      int blk_j = mine ? pos_block(p, req, pos, ps_j, v == 0) : -1;
      for (int j = 0; j < ntiles; ++j, ++gi) {
        const int s = gi & 1;
        const int64_t row = blk_j >= 0 ? (int64_t)blk_j * kPage + (ps_j % kPage) : -1;
        const int blk_j1 = mine && j + 1 < ntiles ? pos_block(p, req, pos, ps_j1, v == 0) : -1;
        const int ps_j2 = mine && j + 2 < ntiles ? slot_pos(p, t, qok, sp, kslot + (j + 2) * kTile) : kNoSlot;
        if (gi >= 2 && !(ok = warp_wait(&k_empty[s], ((gi >> 1) - 1) & 1, p.err, abort_flag))) break;
        // publish which rows of the tile are real to the softmax warps
        const uint32_t vmask = __ballot_sync(0xFFFFFFFFu, row >= 0) & 0xFFFFu;
        if (lane == 0) {
          masks[s * 2 + gw] = vmask;
          mbar_arrive(&m_full[s]);
        }
        ps_j = ps_j1;
        ps_j1 = ps_j2;
        blk_j = blk_j1;
        uint8_t* stage = k_ring + s * K_BYTES;
        const uint32_t stage_u32 = smem_u32(stage);
#pragma unroll 1
        for (int kk = 0; kk < 16; ++kk) {
          const int64_t r = __shfl_sync(0xFFFFFFFFu, row, kk);
          const int key = gw * 16 + kk;
          const char* src = reinterpret_cast<const char*>(p.latent) + (r >= 0 ? r : 0) * (kDqk * 2);
          const uint32_t nbytes = r >= 0 ? 16u : 0u;
#pragma unroll
          for (int rep = 0; rep < 3; ++rep) {
            const int piece = lane + 32 * rep;  // 72 pieces of 16 bytes per row
            if (piece < 72) {
              const int c = piece >> 3, sub = piece & 7;
              cp_async_16(stage_u32 + c * K_CHUNK + sw128_offset(key, sub), src + piece * 16, nbytes);
            }
          }
        }
        cp_async_mbar_arrive_noinc(&k_full[s]);
      }
    }
    // let every copy this thread issued land before the CTA may exit
    cp_async_wait<0>();
  } else if (warp == 2) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_f16(1u, 0u, 128u, (uint32_t)kTile);  // S: B K-major
      const uint32_t idesc_o = idesc_f16(1u, 1u, 128u, (uint32_t)kHalf);  // O: B (V) MN-major
      int gi = 0, ui = 0;
      bool ok = true;
      const uint32_t q_base = smem_u32(q_s);
      const uint32_t p_base = smem_u32(p_s);
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++ui) {
        int t, sp, v;
        unit_coords(p, u, t, sp, v);
        const int ntiles = unit_tiles(p, sp);
        if (!(ok = mbar_wait(q_full, ui & 1, p.err, abort_flag))) break;
        if (ntiles == 0) mma_commit(q_empty);
        for (int j = 0; j <= ntiles && ok; ++j) {
          if (j < ntiles) {
            // S[gi] = Q K^T
            const int g = gi + j, s = g & 1;
            if (!(ok = mbar_wait(&k_full[s], (g >> 1) & 1, p.err, abort_flag))) break;
            if (g >= 2 && !(ok = mbar_wait(&s_empty[s], ((g >> 1) - 1) & 1, p.err, abort_flag))) break;
            fence_proxy_async_smem();
            tc_fence_after();
            const uint32_t k_base = smem_u32(k_ring + s * K_BYTES);
            const uint32_t d = tmem + TM_S + (uint32_t)(s * kTile);
#pragma unroll 1
            for (int c = 0; c < kChunks; ++c) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = sw128_desc(q_base + c * Q_CHUNK + kk * 32, 16, 1024);
                const uint64_t bd = sw128_desc(k_base + c * K_CHUNK + kk * 32, 16, 1024);
                mma_f16_ss(d, ad, bd, idesc_s, (c | kk) ? 1u : 0u);
              }
            }
            mma_commit(&s_full[s]);
            if (j == ntiles - 1) mma_commit(q_empty);  // last use of Q by this unit
          }
          if (j >= 1) {
            // O_v += P[gi + j - 1] V_v
            const int g = gi + j - 1, s = g & 1;
            if (!(ok = mbar_wait(p_full, g & 1, p.err, abort_flag))) break;
            tc_fence_after();
            const uint32_t v_base = smem_u32(k_ring + s * K_BYTES) + (uint32_t)(v * 4 * K_CHUNK);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              // A = P [128 x 32] K-major, no swizzle: 8x16B core matrices, 128 B apart along K,
              // 512 B apart along M.  B = V [256 x 32] MN-major 128B-swizzled: 64-dim blocks
              // K_CHUNK apart, 8-row groups 1024 B apart.
              const uint64_t ad = noswz_desc(p_base + kk * 256, 128, 512);
              const uint64_t bd = sw128_desc(v_base + kk * 2048, K_CHUNK, 1024);
              mma_f16_ss(tmem + TM_O, ad, bd, idesc_o, (j > 1 || kk) ? 1u : 0u);
            }
            mma_commit(pv_done);
            mma_commit(&k_empty[s]);
          }
        }
        gi += ntiles;
      }
      // every MMA issued by this thread has completed before TMEM is released
      mma_commit(mma_fin);
      mbar_wait(mma_fin, 0, p.err, nullptr);
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // head row
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    int gi = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      int t, sp, v;
      unit_coords(p, u, t, sp, v);
      const int ntiles = unit_tiles(p, sp);
      float m_used = -INFINITY, l = 0.0f;
      for (int j = 0; j < ntiles; ++j) {
        const int g = gi + j, s = g & 1;
        if (!(ok = warp_wait(&s_full[s], (g >> 1) & 1, p.err, abort_flag))) break;
        if (!(ok = warp_wait(&m_full[s], (g >> 1) & 1, p.err, abort_flag))) break;
        tc_fence_after();
        uint32_t sv[32];
        tmem_ld16(lane_base + TM_S + s * kTile, *reinterpret_cast<uint32_t(*)[16]>(&sv[0]));
        tmem_ld16(lane_base + TM_S + s * kTile + 16, *reinterpret_cast<uint32_t(*)[16]>(&sv[16]));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[s]);
        const uint32_t valid = masks[s * 2 + 0] | (masks[s * 2 + 1] << 16);
        float x[32];
        float mt = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = ((valid >> c) & 1u) ? __uint_as_float(sv[c]) * p.scale_log2 : -INFINITY;
          mt = fmaxf(mt, x[c]);
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
            for (int c0 = 0; c0 < kHalf; c0 += 16) {
              uint32_t o[16];
              tmem_ld16(lane_base + TM_O + c0, o);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * f);
              tmem_st16(lane_base + TM_O + c0, o);
            }
            tmem_wait_st();
          }
          l *= f;
          m_used = m_new;
        }
        float psum = 0.0f;
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float p0 = x[c] == -INFINITY ? 0.0f : exp2f(x[c] - m_used);
          const float p1 = x[c + 1] == -INFINITY ? 0.0f : exp2f(x[c + 1] - m_used);
          const __nv_bfloat162 b = __floats2bfloat162_rn(p0, p1);
          // the normaliser sums the rounded weights that P V actually uses
          const float2 bf = __bfloat1622float2(b);
          psum += bf.x + bf.y;
          pk[c >> 1] = *reinterpret_cast<const uint32_t*>(&b);
        }
        l += psum;
        // P row r: 4 core-matrix rows of 16 B (8 keys each), no swizzle
        uint8_t* prow = p_s + (r >> 3) * 512 + (r & 7) * 16;
#pragma unroll
        for (int kc = 0; kc < 4; ++kc)
          *reinterpret_cast<uint4*>(prow + kc * 128) = make_uint4(pk[4 * kc], pk[4 * kc + 1], pk[4 * kc + 2], pk[4 * kc + 3]);
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
      const int64_t orow = (int64_t)t * kH + r;
      // O / l in 64-column pieces: four TMEM loads in flight per wait, then the stores
      const int64_t prow = ((int64_t)t * p.nsplit + sp) * kH + r;
#pragma unroll 1
      for (int c0 = 0; c0 < kHalf; c0 += 64) {
        uint32_t o[64];
        if (ntiles > 0) {
          tmem_ld16(lane_base + TM_O + c0, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
          tmem_ld16(lane_base + TM_O + c0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&o[16]));
          tmem_ld16(lane_base + TM_O + c0 + 32, *reinterpret_cast<uint32_t(*)[16]>(&o[32]));
          tmem_ld16(lane_base + TM_O + c0 + 48, *reinterpret_cast<uint32_t(*)[16]>(&o[48]));
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) o[c] = 0u;
        }
        if (p.nsplit == 1) {
          __nv_bfloat16* dst = p.out + orow * kDv + v * kHalf + c0;
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(o[c + e]) * inv, __uint_as_float(o[c + e + 1]) * inv);
              pk[e >> 1] = *reinterpret_cast<const uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(dst + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        } else {
          float* dst = p.part_o + prow * kDv + v * kHalf + c0;
#pragma unroll
          for (int c = 0; c < 64; c += 4)
            *reinterpret_cast<float4*>(dst + c) = make_float4(__uint_as_float(o[c]) * inv, __uint_as_float(o[c + 1]) * inv,
                                                              __uint_as_float(o[c + 2]) * inv, __uint_as_float(o[c + 3]) * inv);
        }
      }
      if (v == 0) {
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
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

// grid (T, 128 heads), block 128: merge the split partials of one (query, head) row; each thread
// owns 4 of the 512 value columns.  The split weights exp(LSE_sp - max) are computed once into
// shared memory, so the per-split loads of the accumulation loop are independent.
constexpr int kMaxSplits = 64;
__global__ void __launch_bounds__(128) mla_combine_kernel(const float* __restrict__ part_o,
                                                          const float* __restrict__ part_lse, int nsplit,
                                                          __nv_bfloat16* __restrict__ out,
                                                          float* __restrict__ lse_out) {
  __shared__ float wts[kMaxSplits];
  __shared__ float s_mx, s_inv, s_lse;
  const int t = blockIdx.x, h = blockIdx.y, c = threadIdx.x * 4;
  const int64_t row0 = (int64_t)t * nsplit * kH + h;  // partial row of split 0; split sp adds sp*kH
  if (threadIdx.x < 32) {
    float mx = -INFINITY;
    for (int sp = threadIdx.x; sp < nsplit; sp += 32) mx = fmaxf(mx, part_lse[row0 + (int64_t)sp * kH]);
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    float sum = 0.0f;
    for (int sp = threadIdx.x; sp < nsplit; sp += 32) {
      const float ls = part_lse[row0 + (int64_t)sp * kH];
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
#pragma unroll 8
  for (int sp = 0; sp < nsplit; ++sp) {
    const float wgt = wts[sp];
    const float4 a = __ldg(reinterpret_cast<const float4*>(part_o + (row0 + (int64_t)sp * kH) * kDv + c));
    acc.x = fmaf(wgt, a.x, acc.x);
    acc.y = fmaf(wgt, a.y, acc.y);
    acc.z = fmaf(wgt, a.z, acc.z);
    acc.w = fmaf(wgt, a.w, acc.w);
  }
  const float inv = s_inv;
  const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  uint2 pk;
  pk.x = *reinterpret_cast<const uint32_t*>(&lo);
  pk.y = *reinterpret_cast<const uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out + ((int64_t)t * kH + h) * kDv + c) = pk;
  if (lse_out && threadIdx.x == 0) lse_out[(int64_t)t * kH + h] = s_lse;
}

int splits_for(int T, int k, int num_sms) {
  const int tiles_q = (k + kTile - 1) / kTile;  // tiles per (query, half)
  const double ideal = 2.0 * T * tiles_q / num_sms;
  int best = 1;
  for (int n = 1; n <= kMaxSplits; n *= 2) {
    int ks = ((k + n - 1) / n + kTile - 1) / kTile * kTile;
    if (ks < 2 * kTile && n > 1) break;
    const int ns = (k + ks - 1) / ks;
    const long long units = 2LL * T * ns;
    const double per_cta = (double)((units + num_sms - 1) / num_sms) * (ks / kTile);
    best = ns;
    if (per_cta <= 1.1 * ideal + 1) break;
  }
  return best;
}

int split_size(int k, int nsplit) { return ((k + nsplit - 1) / nsplit + kTile - 1) / kTile * kTile; }

}  // namespace

int mla_tc_num_splits(int T, int k, int num_sms) { return splits_for(T, k, num_sms); }

size_t mla_tc_workspace_bytes(int T, int H, int d_v, int nsplit) {
  if (nsplit <= 1) return 0;
  const size_t o = (size_t)T * nsplit * H * d_v * sizeof(float);
  const size_t l = (size_t)T * nsplit * H * sizeof(float);
  return ((o + 255) / 256) * 256 + ((l + 255) / 256) * 256;
}

cudaError_t launch_mla_tc(const MlaArgs& a, int nsplit, int num_sms, cudaStream_t s) {
  const int T = a.batch.num_queries;
  alignas(64) CUtensorMap qmap;
  if (!encode_tmap_2d(&qmap, a.q, 2, kDqk, (uint64_t)T * kH, kDqk * 2, 64, kH, true)) return cudaErrorInvalidValue;
  Params p;
  p.latent = static_cast<const __nv_bfloat16*>(a.latent.data);
  p.idx = a.idx;
  p.q_req = a.batch.q_req;
  p.q_pos = a.batch.q_pos;
  p.block_table = a.batch.block_table;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.num_blocks = a.latent.num_blocks;
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
    const size_t o = (size_t)T * nsplit * kH * kDv * sizeof(float);
    p.part_o = static_cast<float*>(a.workspace);
    p.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(a.workspace) + ((o + 255) / 256) * 256);
  }
  cudaError_t e = cudaFuncSetAttribute(mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  const int units = T * nsplit * 2;
  const int grid = units < num_sms ? units : num_sms;
  mla_tc_kernel<<<grid, kThreads, SMEM, s>>>(qmap, p);
  e = cudaGetLastError();
  if (e != cudaSuccess || nsplit == 1) return e;
  mla_combine_kernel<<<dim3(T, kH), 128, 0, s>>>(p.part_o, p.part_lse, nsplit, p.out, a.lse);
  return cudaGetLastError();
}

}  // namespace dsa
