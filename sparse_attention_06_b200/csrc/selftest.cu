// selftest.cu -- diagnostic kernels: the library's bounded waits, and the row-gather rate of the
// sparse MLA's TMA pattern.
//
// Every wait of the tensor-core kernels on an mbarrier phase is bounded: after a limit it sets
// DSA_DEVERR_TIMEOUT in the device error word and the kernel returns instead of hanging.  This
// kernel exercises that path on purpose, with a short limit: one thread initialises an mbarrier
// that nothing ever arrives on and waits for its first phase through the same bounded wait the
// kernels use.  The wait runs out after `limit_cycles` SM cycles, the error bit is set, and the
// kernel exits normally, leaving the context usable.
//
// The tensor-core sparse MLA brings each 64-row tile of selected latent rows (576 bf16 = 1152
// bytes per row) into shared memory by TMA tile::gather4 (four rows x 128 bytes per instruction,
// nine 64-dim column blocks per row, 128B-swizzled), in a two-stage ring, and that gather rate is
// what bounds it.  gather_rate_kernel runs the same gathers with nothing else: four warps issue
// each tile's gathers (16 rows each) once the stage is free, one thread waits for the tile to land
// and frees the stage, and the CTA's SM cycles over all its tiles are written out.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {
namespace {

__global__ void bounded_wait_kernel(long long limit_cycles, int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait(&bar, 0, err, nullptr, limit_cycles);  // no thread arrives: this wait gives up
}

constexpr int kGTile = 64;                  // rows per tile
constexpr int kGBlocks = 9;                 // 64-dim column blocks of a 576-dim row
constexpr int kGBlock = kGTile * 128;       // 8 KB
constexpr int kGStageBytes = kGBlocks * kGBlock;
constexpr int kGStages = 2;
constexpr int kGThreads = 160;              // four gathering warps + the waiting one
constexpr int kGSmem = kGStages * kGStageBytes + 4 * 8 + 1024;

__global__ void __launch_bounds__(kGThreads, 1)
    gather_rate_kernel(const __grid_constant__ CUtensorMap lmap, const int32_t* __restrict__ rows, int tiles,
                       int32_t pool_rows, long long* __restrict__ cycles, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGStages * kGStageBytes);
  uint64_t* empty = full + kGStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGStages; ++i) {
      mbar_init(&full[i], 4);
      mbar_init(&empty[i], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();
  bool ok = true;
  if (warp < 4) {
    int j = 0;
    for (; j < tiles; ++j) {
      const int s = j % kGStages;
      if (j >= kGStages && !(ok = warp_wait(&empty[s], ((j / kGStages) - 1) & 1, err, nullptr))) break;
      int32_t r = pool_rows;  // rows past the pool read as zeros
      if (lane < 16) {
        r = rows[((int64_t)blockIdx.x * tiles + j) * kGTile + warp * 16 + lane];
        if (r < 0 || r >= pool_rows) {
          raise_error(err, DSA_DEVERR_INDEX);
          r = pool_rows;
        }
      }
      uint8_t* stage = smem + s * kGStageBytes + warp * 16 * 128;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], 16 * kGBlocks * 128);
#pragma unroll
      for (int g4 = 0; g4 < 4; ++g4) {
        const int32_t r0 = __shfl_sync(0xFFFFFFFFu, r, 4 * g4), r1 = __shfl_sync(0xFFFFFFFFu, r, 4 * g4 + 1);
        const int32_t r2 = __shfl_sync(0xFFFFFFFFu, r, 4 * g4 + 2), r3 = __shfl_sync(0xFFFFFFFFu, r, 4 * g4 + 3);
        if (lane == 0)
#pragma unroll
          for (int c = 0; c < kGBlocks; ++c)
            tma_gather4(stage + c * kGBlock + g4 * 512, &lmap, &full[s], c * 64, r0, r1, r2, r3);
      }
    }
    if (!ok && lane == 0)  // gave up: the copies of the last use of each stage land before exit
      for (int t = j - 1; t >= 0 && t >= j - kGStages; --t)
        mbar_wait(&full[t % kGStages], (uint32_t)((t / kGStages) & 1), err, nullptr);
  } else if (lane == 0) {
    const long long t0 = clock64();
    for (int j = 0; j < tiles && ok; ++j) {
      const int s = j % kGStages;
      if (!(ok = mbar_wait(&full[s], (uint32_t)((j / kGStages) & 1), err, nullptr))) break;
      mbar_arrive(&empty[s]);
    }
    cycles[blockIdx.x] = ok ? clock64() - t0 : -1;
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_gather_rate_selftest(const dsa_paged_cache& latent, const int32_t* rows, int tiles, int ctas,
                                        int64_t* cycles, int* err, cudaStream_t s) {
  const uint64_t pool_rows = (uint64_t)latent.num_blocks * (uint64_t)latent.block_size;
  alignas(64) CUtensorMap lmap;
  if (!encode_tmap_2d(&lmap, latent.data, 2, (uint64_t)latent.dim, pool_rows, (uint64_t)latent.dim * 2, 64, 1,
                      true))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gather_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmem);
  if (e != cudaSuccess) return e;
  gather_rate_kernel<<<ctas, kGThreads, kGSmem, s>>>(lmap, rows, tiles, (int32_t)pool_rows,
                                                     reinterpret_cast<long long*>(cycles), err);
  return cudaGetLastError();
}

cudaError_t launch_bounded_wait_selftest(long long limit_cycles, int* err, cudaStream_t s) {
  bounded_wait_kernel<<<1, 32, 0, s>>>(limit_cycles, err);
  return cudaGetLastError();
}

}  // namespace dsa
