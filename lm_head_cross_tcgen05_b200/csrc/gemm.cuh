// gemm.cuh — persistent, warp-specialised bf16 GEMM on the sm_100a tensor cores.
//
// One CTA per SM (grid = min(tiles, SMs)); each CTA walks the output tiles
// t = blockIdx.x, blockIdx.x + gridDim.x, ... in a fixed order. Every output tile is owned
// by exactly one CTA and its K loop runs in ascending order, so the fp32 result of a tile
// does not depend on which CTA ran it or on the SM count: the GEMM is deterministic with no
// cross-CTA reduction.
//
// Roles (192 threads):
//   warp 0, lane 0  TMA producer: 128-byte-swizzled operand tiles into a STAGES-deep ring.
//   warp 1, lane 0  MMA issuer: tcgen05.mma (M=128, N=256, K=16 per instruction) into one of
//                   two TMEM accumulators (2 x 256 fp32 columns = all 512 TMEM columns), so
//                   the epilogue of tile i overlaps the main loop of tile i+1.
//   warps 2..5      epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//                   32*(w%4) .. +31, i.e. tile rows), then the fused math of `Epi`.
//
// Operand layouts: A is [M, K] and B is [N, K] in the tensor core's view. Each may sit in
// global memory K-major (K contiguous: box 64 x rows) or MN-major (M or N contiguous: boxes
// of 64 MN x 64 K); the MMA reads MN-major operands through the descriptor's transpose bit,
// so no operand is ever transposed in memory.
#pragma once

#include "sm100.cuh"

namespace lmh {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_STAGE_BYTES = BM * BK * 2;  // 16 KiB
constexpr int B_STAGE_BYTES = BN * BK * 2;  // 32 KiB
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int MN_BLOCK_BYTES = 64 * BK * 2;  // one 64 (MN) x 64 (K) box: 8 KiB
constexpr int GEMM_THREADS = 192;
constexpr int GEMM_SMEM_BYTES = STAGES * STAGE_BYTES + 1024;  // + slack to 1 KiB-align
constexpr uint32_t TMEM_COLS = 512;

struct GemmGrid {
  int m_tiles;
  int n_tiles;
  int k_blocks;     // ceil(K / 64)
  int n_fastest;    // tile order: 0 -> consecutive tiles walk M, 1 -> walk N
  uint32_t* err;    // device error word
};

__device__ __forceinline__ void tile_coords(const GemmGrid& g, int t, int& mb, int& nb) {
  if (g.n_fastest) {
    nb = t % g.n_tiles;
    mb = t / g.n_tiles;
  } else {
    mb = t % g.m_tiles;
    nb = t / g.m_tiles;
  }
}

template <class Epi>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                   const __grid_constant__ CUtensorMap tmB, const GemmGrid g,
                   const typename Epi::Params ep) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  const uint32_t smem_base = (smem_u32(dsmem) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = g.m_tiles * g.n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull_bar[b]), 1);
      mbar_init(smem_u32(&tempty_bar[b]), 4);
    }
    mbar_init(smem_u32(&drain_bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(&tmem_slot), TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      uint32_t kbg = 0;
      for (int t = blockIdx.x; t < num_tiles && !abort_flag; t += gridDim.x) {
        int mb, nb;
        tile_coords(g, t, mb, nb);
        for (int kb = 0; kb < g.k_blocks; ++kb, ++kbg) {
          const uint32_t s = kbg % STAGES;
          const uint32_t ph = (kbg / STAGES) & 1u;
          if (!mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, g.err)) {
            abort_flag = 1;
            break;
          }
          const uint32_t fb = smem_u32(&full_bar[s]);
          const uint32_t a_dst = smem_base + s * STAGE_BYTES;
          const uint32_t b_dst = a_dst + A_STAGE_BYTES;
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          if (!Epi::kAMajorMN) {
            tma_load_2d(a_dst, &tmA, fb, kb * BK, mb * BM);
          } else {
#pragma unroll
            for (int j = 0; j < BM / 64; ++j)
              tma_load_2d(a_dst + j * MN_BLOCK_BYTES, &tmA, fb, mb * BM + 64 * j, kb * BK);
          }
          if (!Epi::kBMajorMN) {
            tma_load_2d(b_dst, &tmB, fb, kb * BK, nb * BN);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_2d(b_dst + j * MN_BLOCK_BYTES, &tmB, fb, nb * BN + 64 * j, kb * BK);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc_bf16(BM, BN, Epi::kAMajorMN, Epi::kBMajorMN);
      uint32_t kbg = 0;
      int it = 0;
      for (int t = blockIdx.x; t < num_tiles && !abort_flag; t += gridDim.x, ++it) {
        const int b = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (!mbar_wait(smem_u32(&tempty_bar[b]), (use & 1u) ^ 1u, g.err)) {
          abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * BN);
        bool ok = true;
        for (int kb = 0; kb < g.k_blocks; ++kb, ++kbg) {
          const uint32_t s = kbg % STAGES;
          const uint32_t ph = (kbg / STAGES) & 1u;
          if (!mbar_wait(smem_u32(&full_bar[s]), ph, g.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_base + s * STAGE_BYTES;
          const uint32_t b_base = a_base + A_STAGE_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t adesc = Epi::kAMajorMN
                                       ? make_sw128_desc(a_base + k * 2048, MN_BLOCK_BYTES, 1024)
                                       : make_sw128_desc(a_base + k * 32, 16, 1024);
            const uint64_t bdesc = Epi::kBMajorMN
                                       ? make_sw128_desc(b_base + k * 2048, MN_BLOCK_BYTES, 1024)
                                       : make_sw128_desc(b_base + k * 32, 16, 1024);
            mma_bf16(d_tmem, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&empty_bar[s]));  // frees the smem stage once read
        }
        if (!ok) {
          abort_flag = 1;
          break;
        }
        mma_commit(smem_u32(&tfull_bar[b]));  // accumulator b is complete
      }
      // No MMA may still be writing TMEM when the columns are released.
      mma_commit(smem_u32(&drain_bar));
      mbar_wait(smem_u32(&drain_bar), 0, g.err);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;  // the TMEM lane quarter this warp may access
    const int row_in_tile = q * 32 + lane;
    int it = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      const int b = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      bool ok = !abort_flag && mbar_wait(smem_u32(&tfull_bar[b]), use & 1u, g.err);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        abort_flag = 1;
        break;
      }
      tc_fence_after();
      int mb, nb;
      tile_coords(g, t, mb, nb);
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * BN);
      Epi::tile(ep, mb, nb, taddr, row_in_tile);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty_bar[b]));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace lmh
