// gemm.cuh — persistent, warp-specialised bf16 GEMM on the sm_100a tensor cores, run by CTA
// pairs (clusters of 2) that share one 256 x 256 output tile per MMA (tcgen05 cta_group::2).
//
// Each CTA of a pair owns 128 of the tile's 256 rows: it stages its 128 rows of A and its 128
// rows (of 256) of B in its own shared memory, and its half of the fp32 accumulator lives in
// its own TMEM. The pair's rank-0 CTA issues the MMAs, which read the operand halves of both
// CTAs. Per SM this halves the B operand traffic of a 128 x 256 single-CTA tile.
//
// Persistent schedule: grid = 2 x (number of co-resident pairs); pair p walks the work units
// p, p + pairs, ... of a fixed, grouped order (group_m row tiles at a time, rows fastest). A
// work unit is an output tile, or a tile and one of k_splits consecutive K ranges when a
// launch has too few tiles to fill the GPU (its epilogue then writes an fp32 partial).
// Every output tile is owned by one pair and its K loop runs in ascending order, so the fp32
// result of a tile does not depend on which SMs ran it or how many there are: the GEMM is
// deterministic without any cross-CTA reduction.
//
// Roles (192 threads per CTA):
//   warp 0, lane 0  TMA producer (both CTAs): its own operand halves into a STAGES-deep ring;
//                   every load completes its bytes on the rank-0 CTA's `full` barrier.
//   warp 1, lane 0  MMA issuer (rank 0 only): tcgen05.mma 256x256x16 into one of two TMEM
//                   accumulators (2 x 256 fp32 columns = all 512), so the epilogue of tile i
//                   overlaps the main loop of tile i+1; commits free the smem stage and signal
//                   the accumulator in both CTAs (multicast commit, no multicast loads). A wide
//                   instantiation (Pipe::WIDE = 2) has 256 x 512 pair tiles instead: two MMAs
//                   per K step, one per 256-column half, share the staged A, and the single
//                   accumulator fills all 512 columns (no overlap with the next tile).
//   warps 2..5      epilogue (both CTAs): tcgen05.ld of the CTA's accumulator half (warp w
//                   reads TMEM lanes 32*(w%4) .. +31), then the fused math of `Epi`; releases
//                   the accumulator with an arrival on the rank-0 CTA's `tmem_empty` barrier.
//
// Operand layouts: A is [M, K] and B is [N, K] in the tensor core's view. Each may be K-major
// in global memory (K contiguous: boxes of 64 K x 128 rows, two per stage) or MN-major (M or N
// contiguous: boxes of 64 MN x 128 K); MN-major operands are read through the descriptor's
// transpose bit, so no operand is ever transposed in memory.
#pragma once

#include "sm100.cuh"

namespace lmh {

constexpr int BM = 128;   // accumulator rows per CTA (half of a pair tile)
constexpr int PM = 256;   // rows per pair tile
constexpr int BN = 256;   // columns per tile
constexpr int BNH = 128;  // B rows staged per CTA
constexpr int A_SUB_BYTES = BM * 128;        // one K-major sub-tile of A (rows x 64 K)
constexpr int B_SUB_BYTES = BNH * 128;
constexpr int GEMM_THREADS = 192;
constexpr int EPI_BUF_BYTES = 32 * 128;      // 32 rows x 64 bf16 (or 32 fp32), 128B-swizzled
constexpr int kMaxDynSmem = 232448;          // 227 KiB per CTA on sm_100

// Pipeline shape of a GEMM instantiation, taken from its epilogue: K per stage (kBK), ring
// depth (kStages) and staging buffers per epilogue warp (kEpiBufs). The default is K = 128 per
// stage, i.e. 8 MMAs per barrier round trip: each round trip (wait for the stage, commit its
// release) costs the tensor pipe a roughly fixed bubble, so the deeper stage runs about 18 %
// more MMAs per clock than a 64-deep one; 3 stages of 64 KiB per CTA, two 4 KiB staging buffers
// per epilogue warp. Every 256 x 256 epilogue uses this shape: the alternatives measured
// (64-deep stages, 2 stages of 192, ring depth traded for staging in the dW accumulation) were
// slower. kWide = 2 makes the pair tile 256 x 512: two MMAs per K step share the A stage, the one
// accumulator takes all 512 TMEM columns, so the epilogue no longer overlaps the next tile's
// main loop; the wide dH and dW epilogues run 2 stages of 96 KiB (16 MMAs per round trip).
struct PipeDefault {
  static constexpr int kBK = 128, kStages = 3, kEpiBufs = 2, kWide = 1;
};

template <class Epi>
struct Pipe {
  static constexpr int BK = Epi::kBK;
  static constexpr int STAGES = Epi::kStages;
  static constexpr int EPI_BUFS = Epi::kEpiBufs;
  static constexpr int WIDE = Epi::kWide;             // 256-column halves of a pair tile
  static constexpr int NACC = 2 / WIDE;               // accumulators in the 512 TMEM columns
  static constexpr int KSUB = BK / 64;                // 128-byte-wide K sub-tiles (K-major)
  static constexpr int A_STAGE_BYTES = BM * BK * 2;
  static constexpr int B_HALF_BYTES = BNH * BK * 2;   // this CTA's B rows of one half
  static constexpr int B_STAGE_BYTES = WIDE * B_HALF_BYTES;
  static constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
  static constexpr int MN_BLOCK_BYTES = 64 * BK * 2;  // one 64 (MN) x BK (K) box
  static constexpr int EPI_STAGE_BYTES = 4 * EPI_BUFS * EPI_BUF_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_STAGE_BYTES + 1024;  // + align
  static_assert(BK % 16 == 0 && STAGES >= 2 && EPI_BUFS >= 2 && EPI_BUFS <= 8, "pipeline shape");
  static_assert(WIDE == 1 || WIDE == 2, "a pair tile is 256 or 512 columns wide");
  static_assert(NACC * BN * WIDE == 512, "the accumulators fill the 512 TMEM columns");
  static_assert((Epi::kAMajorMN && Epi::kBMajorMN) || BK % 64 == 0,
                "a K-major operand is staged in 64-wide K boxes");
  static_assert(SMEM_BYTES + 256 <= kMaxDynSmem, "shared memory per CTA");
};

// What an epilogue warp needs to stage bf16 output through shared memory and store it with
// TMA: the output tensor map (bf16, box 64 columns x 32 rows, 128-byte swizzle), its two
// staging buffers, and a running count of its stores (which selects the buffer).
struct EpiCtx {
  const CUtensorMap* tmC;
  const CUtensorMap* tmD;  // a second map some epilogues read through (else tmC again)
  uint32_t stage;
  int lane;
  int row_w;         // first accumulator row of this warp within the CTA's 128
  uint32_t nstore;
  int split;         // K range of the current work unit (0 unless K is split)
  uint32_t bar;      // this warp's mbarrier for TMA loads into its staging buffers
  uint32_t bar_phase;
  uint32_t* err;
};
constexpr uint32_t TMEM_COLS = 512;

struct GemmGrid {
  int m_tiles;   // pair tiles along M (256 rows each)
  int n_tiles;   // tiles along N (256 x Pipe<Epi>::WIDE columns each)
  int k_blocks;  // ceil(K / Pipe<Epi>::BK)
  int k_splits;  // K split into this many consecutive ranges (work units = tiles x splits)
  int group_m;   // tile order: group_m row tiles at a time, rows fastest within a group
  int hint_a;    // L2 eviction priority of A's loads (L2Hint)
  int hint_b;    // L2 eviction priority of B's loads
  uint32_t* err; // device error word
};

// Work unit u = split * tiles + tile: the split's K blocks are [kb0, kb1).
__device__ __forceinline__ void unit_coords(const GemmGrid& g, int u, int& mb, int& nb, int& split,
                                            int& kb0, int& kb1) {
  const int tiles = g.m_tiles * g.n_tiles;
  split = u / tiles;
  int t = u - split * tiles;
  const int per_group = g.group_m * g.n_tiles;
  const int grp = t / per_group;
  const int rem = t - grp * per_group;
  const int m0 = grp * g.group_m;
  const int gm = min(g.group_m, g.m_tiles - m0);
  mb = m0 + rem % gm;
  nb = rem / gm;
  kb0 = static_cast<int>(static_cast<long long>(g.k_blocks) * split / g.k_splits);
  kb1 = static_cast<int>(static_cast<long long>(g.k_blocks) * (split + 1) / g.k_splits);
}

template <class Epi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                   const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC,
                   const __grid_constant__ CUtensorMap tmD, const GemmGrid g,
                   const typename Epi::Params ep) {
  using P = Pipe<Epi>;
  constexpr int BK = P::BK, STAGES = P::STAGES, STAGE_BYTES = P::STAGE_BYTES;
  constexpr int A_STAGE_BYTES = P::A_STAGE_BYTES, MN_BLOCK_BYTES = P::MN_BLOCK_BYTES;
  constexpr int KSUB = P::KSUB;
  constexpr int WIDE = P::WIDE, NACC = P::NACC, B_HALF_BYTES = P::B_HALF_BYTES;
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];   // rank 0: operands of a stage landed
  __shared__ __align__(8) uint64_t empty_bar[STAGES];  // both: the stage was read by the MMAs
  __shared__ __align__(8) uint64_t tfull_bar[2];       // both: accumulator b is complete
  __shared__ __align__(8) uint64_t tempty_bar[2];      // rank 0: both CTAs drained accumulator b
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ __align__(8) uint64_t epi_bar[4];         // epilogue warp w-2: its staged loads
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  const uint32_t smem_base = (smem_u32(dsmem) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int num_tiles = g.m_tiles * g.n_tiles * g.k_splits;  // work units

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull_bar[b]), 1);
      mbar_init(smem_u32(&tempty_bar[b]), 8);  // 4 epilogue warps x 2 CTAs
    }
    mbar_init(smem_u32(&drain_bar), 1);
    for (int w = 0; w < 4; ++w) mbar_init(smem_u32(&epi_bar[w]), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc_pair(smem_u32(&tmem_slot), TMEM_COLS);
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      const uint64_t pol_a = l2_policy(g.hint_a);
      const uint64_t pol_b = l2_policy(g.hint_b);
      uint32_t kbg = 0;
      for (int t = pair; t < num_tiles && !abort_flag; t += npairs) {
        int mb, nb, sp, kb0, kb1;
        unit_coords(g, t, mb, nb, sp, kb0, kb1);
        const int arow = mb * PM + static_cast<int>(rank) * BM;    // this CTA's A rows
        const int brow = nb * BN * WIDE + static_cast<int>(rank) * BNH;  // its B rows, half 0
        for (int kb = kb0; kb < kb1; ++kb, ++kbg) {
          const uint32_t s = kbg % STAGES;
          const uint32_t ph = (kbg / STAGES) & 1u;
          if (!mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, g.err)) {
            abort_flag = 1;
            break;
          }
          const uint32_t lfull = map_to_rank(smem_u32(&full_bar[s]), 0);
          if (rank == 0) mbar_arrive_expect_tx(smem_u32(&full_bar[s]), 2 * STAGE_BYTES);
          const uint32_t a_dst = smem_base + s * STAGE_BYTES;
          const uint32_t b_dst = a_dst + A_STAGE_BYTES;
          if (!Epi::kAMajorMN) {
#pragma unroll
            for (int j = 0; j < KSUB; ++j)
              tma_load_2d_pair(a_dst + j * A_SUB_BYTES, &tmA, lfull, kb * BK + 64 * j, arow, pol_a);
          } else {
#pragma unroll
            for (int j = 0; j < BM / 64; ++j)
              tma_load_2d_pair(a_dst + j * MN_BLOCK_BYTES, &tmA, lfull, arow + 64 * j, kb * BK,
                               pol_a);
          }
#pragma unroll
          for (int h = 0; h < WIDE; ++h) {  // half h: the pair tile's columns h*256 .. +255
            const uint32_t bh = b_dst + h * B_HALF_BYTES;
            if (!Epi::kBMajorMN) {
#pragma unroll
              for (int j = 0; j < KSUB; ++j)
                tma_load_2d_pair(bh + j * B_SUB_BYTES, &tmB, lfull, kb * BK + 64 * j,
                                 brow + h * BN, pol_b);
            } else {
#pragma unroll
              for (int j = 0; j < BNH / 64; ++j)
                tma_load_2d_pair(bh + j * MN_BLOCK_BYTES, &tmB, lfull, brow + h * BN + 64 * j,
                                 kb * BK, pol_b);
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (rank 0)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = make_idesc_bf16(PM, BN, Epi::kAMajorMN, Epi::kBMajorMN);
      uint32_t kbg = 0;
      int it = 0;
      for (int t = pair; t < num_tiles && !abort_flag; t += npairs, ++it) {
        const int b = it % NACC;
        const uint32_t use = static_cast<uint32_t>(it / NACC);
        if (!mbar_wait(smem_u32(&tempty_bar[b]), (use & 1u) ^ 1u, g.err)) {
          abort_flag = 1;
          break;
        }
        tc_fence_after();
        int mb, nb, sp, kb0, kb1;
        unit_coords(g, t, mb, nb, sp, kb0, kb1);
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * BN * WIDE);
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb, ++kbg) {
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
            // K-major: sub-tile k/4, 32-byte step inside its 128-byte rows; MN-major: 16 rows
            const uint64_t adesc =
                Epi::kAMajorMN
                    ? make_sw128_desc(a_base + k * 2048, MN_BLOCK_BYTES, 1024)
                    : make_sw128_desc(a_base + (k >> 2) * A_SUB_BYTES + (k & 3) * 32, 16, 1024);
#pragma unroll
            for (int h = 0; h < WIDE; ++h) {  // both halves reuse this A step
              const uint32_t bh = b_base + h * B_HALF_BYTES;
              const uint64_t bdesc =
                  Epi::kBMajorMN
                      ? make_sw128_desc(bh + k * 2048, MN_BLOCK_BYTES, 1024)
                      : make_sw128_desc(bh + (k >> 2) * B_SUB_BYTES + (k & 3) * 32, 16, 1024);
              mma_bf16_pair(d_tmem + h * BN, adesc, bdesc, idesc,
                            (kb != kb0 || k != 0) ? 1u : 0u);
            }
          }
          mma_commit_pair(smem_u32(&empty_bar[s]), 0x3);  // both CTAs may refill stage s
        }
        if (!ok) {
          abort_flag = 1;
          break;
        }
        mma_commit_pair(smem_u32(&tfull_bar[b]), 0x3);  // accumulator b done in both CTAs
      }
      // No MMA may still be writing TMEM when the columns are released.
      mma_commit_pair_local(smem_u32(&drain_bar));
      mbar_wait(smem_u32(&drain_bar), 0, g.err);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;  // the TMEM lane quarter this warp may access
    const int row_in_tile = q * 32 + lane;
    const uint32_t stage_w =
        smem_base + STAGES * STAGE_BYTES + (warp - 2) * P::EPI_BUFS * EPI_BUF_BYTES;
    EpiCtx ctx{&tmC, &tmD, stage_w, lane, q * 32, 0u, 0, smem_u32(&epi_bar[warp - 2]), 0u, g.err};
    if (lane == 0) tma_prefetch_desc(&tmC);
    int it = 0;
    for (int t = pair; t < num_tiles; t += npairs, ++it) {
      const int b = it % NACC;
      const uint32_t use = static_cast<uint32_t>(it / NACC);
      bool ok = !abort_flag && mbar_wait(smem_u32(&tfull_bar[b]), use & 1u, g.err);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        abort_flag = 1;
        break;
      }
      tc_fence_after();
      int mb, nb, sp, kb0, kb1;
      unit_coords(g, t, mb, nb, sp, kb0, kb1);
      ctx.split = sp;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(b * BN * WIDE);
#pragma unroll 1
      for (int h = 0; h < WIDE; ++h)  // each 256-column half as a tile of its own
        Epi::tile(ep, mb * 2 + static_cast<int>(rank), nb * WIDE + h, taddr + h * BN,
                  row_in_tile, ctx);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(smem_u32(&tempty_bar[b]), 0));
    }
    if (lane == 0) bulk_wait_all();  // every staged output has reached global memory
  }

  tc_fence_before();
  cluster_sync();  // MMAs drained in rank 0, accumulator reads done in both CTAs
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

}  // namespace lmh
