// epilogues.cuh — what each GEMM does with its fp32 accumulator tile (128 rows x 256
// columns of TMEM per CTA). Each epilogue thread owns one tile row and reads it as four
// 64-column slabs (two tcgen05.ld of 32 columns each). bf16 outputs are staged per warp in
// shared memory (32 rows x 64 columns, 128-byte swizzled) and written with one TMA store, so
// global writes are full 128-byte lines instead of 32 scattered 16-byte pieces.
#pragma once

#include <cuda_bf16.h>
#include <limits.h>

#include "gemm.cuh"

namespace lmh {

constexpr int kSlabs = BN / 64;
constexpr float kNegInf = -__builtin_huge_valf();

// ---------------------------------------------------------------------------- targets
// The ids whose logits a row needs individually: its label (TK = kLabel), or the sorted,
// de-duplicated valid candidate ids of the support entries (TK = kCands).
enum TargetKind { kLabel = 0, kCands = 1 };

struct Targets {
  const int32_t* labels;  // [N]        (kLabel)
  const int32_t* sorted;  // [N, K]     ascending distinct valid ids of each row (kCands)
  const int32_t* nuniq;   // [N]        number of sorted ids of each row
  int K;
};

template <int TK>
struct TargetCursor;

template <>
struct TargetCursor<kLabel> {
  int lab;  // -1: no target in this row
  __device__ __forceinline__ void init(const Targets& tg, long long grow, int n0, int V) {
    const int y = tg.labels[grow];
    lab = (y >= 0 && y < V) ? y : -1;
  }
  __device__ __forceinline__ void none() { lab = -1; }
  // Calls hit(j, 0) for the target column col0 + j of this 32-column slice, if any.
  template <class F>
  __device__ __forceinline__ void slice(int col0, F&& hit) {
    if (static_cast<unsigned>(lab - col0) < 32u) {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j == lab) hit(j, 0);
    }
  }
};

template <>
struct TargetCursor<kCands> {
  const int32_t* srow;
  int ptr, nu, next;
  __device__ __forceinline__ void init(const Targets& tg, long long grow, int n0, int V) {
    srow = tg.sorted + grow * tg.K;
    nu = tg.nuniq[grow];
    int lo = 0, hi = nu;  // first sorted id >= n0
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (srow[mid] < n0) lo = mid + 1; else hi = mid;
    }
    ptr = lo;
    next = ptr < nu ? srow[ptr] : INT_MAX;
  }
  __device__ __forceinline__ void none() { nu = 0; ptr = 0; next = INT_MAX; }
  // Calls hit(j, p) for every target column col0 + j of this slice, p = its sorted index.
  template <class F>
  __device__ __forceinline__ void slice(int col0, F&& hit) {
    if (next < col0 + 32) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (col0 + j == next) {
          hit(j, ptr);
          ++ptr;
          next = ptr < nu ? srow[ptr] : INT_MAX;
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------- staged store
// The warp writes its 32 rows x 64 columns (a: columns 0..31, b: 32..63 of each thread's
// row) into one of its two staging buffers and lane 0 stores the block at (x, y) of ctx.tmC.
// A buffer is reused only after the store issued from it two calls earlier has finished
// reading it. All lanes of the warp must call this together.
__device__ __forceinline__ void stage_store_64(EpiCtx& c, const float (&a)[32],
                                               const float (&b)[32], int x, int y,
                                               bool do_store) {
  const uint32_t buf = c.stage + (c.nstore & 1u) * EPI_BUF_BYTES;
  if (c.lane == 0) bulk_wait_read_le1();
  __syncwarp();
  const uint32_t row = buf + static_cast<uint32_t>(c.lane) * 128u;
  const uint32_t sw = static_cast<uint32_t>(c.lane & 7);
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const float* v = u < 4 ? a : b;
    const int o = (u & 3) * 8;
    uint4 w;
    w.x = pack_bf16x2(v[o + 0], v[o + 1]);
    w.y = pack_bf16x2(v[o + 2], v[o + 3]);
    w.z = pack_bf16x2(v[o + 4], v[o + 5]);
    w.w = pack_bf16x2(v[o + 6], v[o + 7]);
    st_shared_v4(row + ((static_cast<uint32_t>(u) ^ sw) << 4), w);  // 16-byte chunk swizzle
  }
  fence_async_smem();
  __syncwarp();
  if (c.lane == 0 && do_store) {
    tma_store_2d(c.tmC, buf, x, y);
    bulk_commit();
  }
  ++c.nstore;
}

// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read_le() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// The fp32 counterpart: the warp's 32 rows x 64 columns of fp32 (a: columns x .. x+31, b:
// x+32 .. x+63 of each thread's row) go through both of its staging buffers with one proxy
// fence, then to two TMA stores, or with `reduce` two TMA adds into the destination, at (x, y)
// and (x + 32, y) of ctx.tmC (fp32, box 32 columns x 32 rows, 128-byte swizzle), committed as
// one group. The buffers are reused once the previous group has read them. (One fence per
// 64 columns instead of per 32: 3 % off the accumulating dW GEMM.)
__device__ __forceinline__ uint4 f32x4_bits(const float (&v)[32], int u) {
  return make_uint4(__float_as_uint(v[u * 4 + 0]), __float_as_uint(v[u * 4 + 1]),
                    __float_as_uint(v[u * 4 + 2]), __float_as_uint(v[u * 4 + 3]));
}

// Each thread's 64 fp32 (a: columns 0..31, b: 32..63 of its row) into the warp's two staging
// buffers, each the 128-byte-swizzled layout of a 32 x 32 fp32 TMA box. The buffers must be
// free; the caller fences before a TMA operation reads them.
__device__ __forceinline__ void write_f32_pair(const EpiCtx& c, const float (&a)[32],
                                               const float (&b)[32]) {
  const uint32_t b0 = c.stage, b1 = c.stage + EPI_BUF_BYTES;
  const uint32_t row = static_cast<uint32_t>(c.lane) * 128u;
  const uint32_t sw = static_cast<uint32_t>(c.lane & 7);
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const uint32_t ch = row + ((static_cast<uint32_t>(u) ^ sw) << 4);
    st_shared_v4(b0 + ch, f32x4_bits(a, u));
    st_shared_v4(b1 + ch, f32x4_bits(b, u));
  }
}

__device__ __forceinline__ void stage_f32_64(EpiCtx& c, const float (&a)[32], const float (&b)[32],
                                             int x, int y, bool do_op, bool reduce) {
  const uint32_t b0 = c.stage, b1 = c.stage + EPI_BUF_BYTES;
  if (c.lane == 0) bulk_wait_read_le<0>();
  __syncwarp();
  write_f32_pair(c, a, b);
  fence_async_smem();
  __syncwarp();
  if (c.lane == 0 && do_op) {
    if (reduce) {
      tma_reduce_add_2d(c.tmC, b0, x, y);
      tma_reduce_add_2d(c.tmC, b1, x + 32, y);
    } else {
      tma_store_2d(c.tmC, b0, x, y);
      tma_store_2d(c.tmC, b1, x + 32, y);
    }
    bulk_commit();
  }
  c.nstore += 2;
}

// ------------------------------------------------------------------ logits statistics
// Forward epilogue of z = H_c W^T. Per (row, 256-wide vocabulary tile t) it writes the tile
// maximum m_t, s_t = sum_v exp(z_v - m_t), the first column attaining m_t, and the logits at
// the row's targets; with kStoreP it also stores p~ = exp(z - m_t) in bf16 (zero past V),
// which the fused backward rescales into the softmax gradient. Columns >= V are masked.
// ctx.tmC (kStoreP): the chunk's [rows, ldp] bf16 buffer.
template <int TK, bool kStoreP>
struct EpiStats : PipeDefault {
  static constexpr int kId = kStoreP ? 3 : 2;  // gemm_logits_stats(_store)
  static constexpr int kAMajorMN = 0;          // H chunk [rows, d], K-major
  static constexpr int kBMajorMN = 0;          // W [V, d], K-major
  struct Params {
    int rows;           // rows of this chunk
    long long row0;     // global index of the chunk's first row
    int V;
    int T;              // vocabulary tiles, ceil(V / 256)
    long long ldp;      // row stride of the chunk buffer (elements), round_up(V, 8)
    Targets tg;
    float* zt;          // target logits: [N] (kLabel) or [N, K] by sorted index (kCands)
    float* part_m;      // [rows, T]
    float* part_s;      // [rows, T]
    int32_t* part_i;    // [rows, T]
    Temperature temp;   // logits are z / tau_i
  };

  static __device__ __forceinline__ void tile(const Params& p, int mb, int nb, uint32_t taddr,
                                              int rit, EpiCtx& ctx) {
    const int row = mb * BM + rit;
    const bool rv = row < p.rows;
    const long long grow = p.row0 + row;
    const int n0 = nb * BN;
    const bool full = n0 + BN <= p.V;
    const float it = rv ? inv_temperature(p.temp, grow) : 1.f;
    TargetCursor<TK> cur;
    if (rv) cur.init(p.tg, grow, n0, p.V); else cur.none();

    // pass 1: maximum, its first column, target logits (of the tempered logits)
    float m = kNegInf;
    int am = n0;
#pragma unroll 1
    for (int sl = 0; sl < 2 * kSlabs; ++sl) {
      float v[32];
      tmem_ld32(taddr + sl * 32, v);
      const int col0 = n0 + sl * 32;
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= it;
      if (!full) {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j >= p.V) v[j] = kNegInf;
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (v[j] > m) {
          m = v[j];
          am = col0 + j;
        }
      }
      cur.slice(col0, [&](int j, int idx) {
        if (TK == kLabel) p.zt[grow] = v[j];
        else p.zt[grow * p.tg.K + idx] = v[j];
      });
    }

    // pass 2: sum of exp(z - m); optionally p~ = exp(z - m) to the chunk buffer
    const float moff = -m * kLog2e;
    const float sc = it * kLog2e;
    float s0 = 0.f, s1 = 0.f;
    const int wrow = mb * BM + ctx.row_w;  // first chunk row of this warp
#pragma unroll 1
    for (int sb = 0; sb < kSlabs; ++sb) {
      float a[32], b[32];
      const int col0 = n0 + sb * 64;
      tmem_ld32(taddr + sb * 64, a);
      tmem_ld32(taddr + sb * 64 + 32, b);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float ea = fast_exp2(fmaf(a[j], sc, moff));
        const float eb = fast_exp2(fmaf(b[j], sc, moff));
        a[j] = (full || col0 + j < p.V) ? ea : 0.f;
        b[j] = (full || col0 + 32 + j < p.V) ? eb : 0.f;
        s0 += a[j];
        s1 += b[j];
      }
      if (kStoreP) stage_store_64(ctx, a, b, col0, wrow, wrow < p.rows && col0 < p.ldp);
    }
    if (rv) {
      const long long o = static_cast<long long>(row) * p.T + nb;
      p.part_m[o] = m;
      p.part_s[o] = s0 + s1;
      p.part_i[o] = am;
    }
  }
};

// ------------------------------------------------------------------ softmax gradient
// Backward epilogue with recomputed logits: G = alpha_i exp(z - lse_i) - beta at the row's
// targets, written in bf16 to the chunk's G buffer (zero past column V; ctx.tmC maps it).
template <int TK>
struct EpiGrad : PipeDefault {
  static constexpr int kId = 4;  // gemm_logits_grad
  static constexpr int kAMajorMN = 0;
  static constexpr int kBMajorMN = 0;
  struct Params {
    int rows;
    long long row0;
    int V;
    long long ldp;
    Targets tg;
    const float* lse;    // [N]
    const float* alpha;  // [N]
    const float* beta;   // [N] (kLabel) or [N, K] in sorted order (kCands)
    Temperature temp;    // logits are z / tau_i (alpha and beta carry the 1 / tau_i factor)
  };

  static __device__ __forceinline__ void tile(const Params& p, int mb, int nb, uint32_t taddr,
                                              int rit, EpiCtx& ctx) {
    const int row = mb * BM + rit;
    const bool rv = row < p.rows;
    const long long grow = p.row0 + row;
    const int n0 = nb * BN;
    const bool full = n0 + BN <= p.V;
    const float al = rv ? p.alpha[grow] : 0.f;
    const float loff = rv ? -p.lse[grow] * kLog2e : 0.f;
    const float sc = (rv ? inv_temperature(p.temp, grow) : 1.f) * kLog2e;
    TargetCursor<TK> cur;
    if (rv) cur.init(p.tg, grow, n0, p.V); else cur.none();
    const int wrow = mb * BM + ctx.row_w;
#pragma unroll 1
    for (int sb = 0; sb < kSlabs; ++sb) {
      float a[32], b[32];
      const int col0 = n0 + sb * 64;
      tmem_ld32(taddr + sb * 64, a);
      tmem_ld32(taddr + sb * 64 + 32, b);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float ea = al * fast_exp2(fmaf(a[j], sc, loff));
        const float eb = al * fast_exp2(fmaf(b[j], sc, loff));
        a[j] = (full || col0 + j < p.V) ? ea : 0.f;
        b[j] = (full || col0 + 32 + j < p.V) ? eb : 0.f;
      }
      cur.slice(col0, [&](int j, int idx) {
        a[j] -= (TK == kLabel) ? p.beta[grow] : p.beta[grow * p.tg.K + idx];
      });
      cur.slice(col0 + 32, [&](int j, int idx) {
        b[j] -= (TK == kLabel) ? p.beta[grow] : p.beta[grow * p.tg.K + idx];
      });
      stage_store_64(ctx, a, b, col0, wrow, wrow < p.rows && col0 < p.ldp);
    }
  }
};

// ------------------------------------------------------------------ row scatter
// Where the fp32 rows of a vocabulary shard's dH contribution go when each is written straight
// to the rank that reduces it: the N rows form R consecutive slices (the first N % R hold one
// row more), slice j belongs to rank j, and rank j's receive buffer dest[j] is [R][rows_j][d]
// fp32 with this rank's rows at slot `rank`. dest[j] may be another GPU's memory (a peer
// pointer): the epilogue reaches it with ordinary stores, tile by tile, while the GEMM runs.
struct RowScatter {
  float* const* dest = nullptr;  // [R] receive buffers (a device array), or null: no scatter
  long long N = 0;
  long long row0 = 0;            // global index of the chunk's first row
  int R = 1;
  int rank = 0;
  __device__ __forceinline__ float* row(long long g, int d) const {
    const long long base = N / R, extra = N % R, big = extra * (base + 1);
    long long j, start, rows;
    if (g < big) {
      j = g / (base + 1);
      start = j * (base + 1);
      rows = base + 1;
    } else {  // base >= 1 here: g >= big only when some slice holds base rows
      j = extra + (g - big) / base;
      start = big + (j - extra) * base;
      rows = base;
    }
    return dest[j] + (static_cast<long long>(rank) * rows + (g - start)) * d;
  }
};

// ------------------------------------------------------------------ dH = G W
// ctx.tmC maps this chunk's rows of dH ([rows, d] at row r0). With K (= V) split, each unit
// writes its fp32 partial to part[split][row][col] instead; a fixed-order reduction over the
// splits then produces dH. With a row scatter each fp32 row goes to its reducing rank.
// kWide_ = 2: 256 x 512 pair tiles. dH's K loop runs over the whole vocabulary (about 1000
// K blocks per tile at V = 128256), so an epilogue that no longer overlaps the next tile costs
// under 1 %, while reading each staged block of G for two MMAs cuts a quarter of the operand
// bytes moved from L2 into shared memory (at 8192 x 128256 x 4096 the step ran 3-7 % faster
// on two boxes: less power, higher clock). K per stage is 128 in 2 stages of 96 KiB: 16 MMAs per barrier
// round trip (4 stages of 64 measured 3 % slower). The tensor core adds the same K steps in
// the same order either way, so an unsplit wide tile gives the narrow tile's bits.
struct DhParams {
  int rows;
  int d;
  float* part;    // [splits, rows, d] fp32, or null when K is not split
  RowScatter sc;  // with sc.dest: fp32 rows to their reducing ranks instead (one split)
};
template <int kWide_, int kBK_, int kStages_>
struct EpiDHT {
  static constexpr int kBK = kBK_, kStages = kStages_, kEpiBufs = 2, kWide = kWide_;
  static constexpr int kId = 5;        // gemm_dH
  static constexpr int kAMajorMN = 0;  // G chunk [rows, V], K-major
  static constexpr int kBMajorMN = 1;  // W [V, d] read as [K = V, N = d], N contiguous
  using Params = DhParams;
  static __device__ __forceinline__ void tile(const Params& p, int mb, int nb, uint32_t taddr,
                                              int rit, EpiCtx& ctx) {
    const int n0 = nb * BN;
    const int wrow = mb * BM + ctx.row_w;
    const int row = mb * BM + rit;
#pragma unroll 1
    for (int sb = 0; sb < kSlabs; ++sb) {
      const int col0 = n0 + sb * 64;
      if (col0 >= p.d) break;  // uniform across the warp (d is a multiple of 64)
      float a[32], b[32];
      tmem_ld32(taddr + sb * 64, a);
      tmem_ld32(taddr + sb * 64 + 32, b);
      if (p.sc.dest || p.part) {
        if (row < p.rows) {
          float4* o = reinterpret_cast<float4*>(
              (p.sc.dest ? p.sc.row(p.sc.row0 + row, p.d)
                         : p.part + (static_cast<long long>(ctx.split) * p.rows + row) * p.d) +
              col0);
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float* v = u < 8 ? a : b;
            const int q = (u & 7) * 4;
            __stcs(o + u, make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]));
          }
        }
      } else {
        stage_store_64(ctx, a, b, col0, wrow, wrow < p.rows);
      }
    }
  }
};

using EpiDH = EpiDHT<1, PipeDefault::kBK, PipeDefault::kStages>;
using EpiDHWide = EpiDHT<2, 128, 2>;

// ------------------------------------------------------------------ dW = G^T H_c
// acc_mode 0: the tile sum is the whole dW, stored in bf16 (ctx.tmC: bf16 dW [V, d]).
// acc_mode 1: acc = 0 + sum (first chunk), stored in fp32.
// acc_mode 2: acc += sum, one fp32 add per element done by the TMA unit at L2.
// acc_mode 3: dW = bf16(acc + sum) (last chunk of an internal accumulator, which is not
//             written back): the accumulator block is loaded by TMA into the warp's staging
//             buffers, added in registers, and the bf16 result stored through ctx.tmC.
// acc_mode 4: 0 + sum in fp32, each row stored straight into the receive buffer of the rank
//             that reduces it (p.sc: row data-parallel dW over peer memory; one chunk).
// acc_mode 5: as mode 3, and the fp32 sum is also stored back into the accumulator (last
//             chunk of a caller-owned accumulator that must end up holding the sum): the
//             bf16 cast of the final accumulator needs no separate pass.
// In modes 1 and 2 ctx.tmC maps the fp32 accumulator [V, d]; in modes 3 and 5 ctx.tmD does
// (fp32, box 32 x 32 rows, 128-byte swizzle) and ctx.tmC maps bf16 dW. Every
// element has one owner tile per launch and the launches of a call run in chunk order, so the
// accumulation order is fixed. Every add (modes 1 and 3 in registers, mode 2 in the TMA unit)
// is an IEEE fp32 add rounded to nearest even, so an internal accumulator gives the same bits
// as a zeroed caller-owned one. The accumulator is never read by 16-byte register loads that
// wait on DRAM one row at a time: writes are staged stores and L2 reduce-adds, and the one
// read (mode 3) is a TMA block load.
// kBK_, kStages_, kEpiBufs_: the pipeline shape (Pipe). Trading ring depth for more staging
// buffers (more reduce-adds in flight per warp) made the accumulate modes slower, not faster
// (96 x 3 stages with 5 buffers, 64 x 5 with 4, 64 x 4 with 6: 2.94 -> 3.27 ms per 2048-row
// chunk at 16384 x 5120 x 151936), so every mode runs the default shape. kWide_ = 2: 256 x 512
// pair tiles (2 stages of 128-deep K), used for the bf16 output of a single chunk of at least
// 8192 rows (64 K blocks): a quarter less operand traffic outweighs the exposed epilogue there
// (8192 x 128256 x 4096: the step 2 % faster), while the fp32 accumulate modes, whose epilogue
// is several times heavier, keep 256 x 256. No tile width changes dW's bits.
template <int kBK_, int kStages_, int kEpiBufs_, int kWide_ = 1>
struct EpiDWT {
  static constexpr int kBK = kBK_, kStages = kStages_, kEpiBufs = kEpiBufs_, kWide = kWide_;
  static constexpr int kId = 6;        // gemm_dW
  static constexpr int kAMajorMN = 1;  // G^T: G chunk [rows, V] read as [K = rows, M = V]
  static constexpr int kBMajorMN = 1;  // H chunk [rows, d] read as [K = rows, N = d]
  struct Params {
    int V;
    int d;
    int acc_mode;
    RowScatter sc;  // acc_mode 4: the receive buffers of the R ranks, N = V
  };
  static __device__ __forceinline__ void tile(const Params& p, int mb, int nb, uint32_t taddr,
                                              int rit, EpiCtx& ctx) {
    const int n0 = nb * BN;
    const int wrow = mb * BM + ctx.row_w;
    const bool wv = wrow < p.V;  // rows past V are clipped by the tensor maps
#pragma unroll 1
    for (int sb = 0; sb < kSlabs; ++sb) {
      const int col0 = n0 + sb * 64;
      if (col0 >= p.d) break;  // uniform across the warp (d is a multiple of 64)
      float a[32], b[32];
      tmem_ld32(taddr + sb * 64, a);
      tmem_ld32(taddr + sb * 64 + 32, b);
      if (p.acc_mode == 0) {
        stage_store_64(ctx, a, b, col0, wrow, wv);
      } else if (p.acc_mode == 4) {
        const int row = mb * BM + rit;
        if (row < p.V) {
          float4* o = reinterpret_cast<float4*>(p.sc.row(row, p.d) + col0);
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float* v = u < 8 ? a : b;
            const int q = (u & 7) * 4;
            __stcs(o + u, make_float4(__fadd_rn(0.f, v[q]), __fadd_rn(0.f, v[q + 1]),
                                      __fadd_rn(0.f, v[q + 2]), __fadd_rn(0.f, v[q + 3])));
          }
        }
      } else if (p.acc_mode == 3 || p.acc_mode == 5) {
        if (!wv) continue;  // warp-uniform: nothing of this block exists
        add_loaded_64(ctx, col0, wrow, a, b);
        if (p.acc_mode == 5) store_sum_64(ctx, col0, wrow, a, b);
        stage_store_64(ctx, a, b, col0, wrow, true);
      } else {
        if (p.acc_mode == 1) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            a[j] = __fadd_rn(0.f, a[j]);
            b[j] = __fadd_rn(0.f, b[j]);
          }
        }
        stage_f32_64(ctx, a, b, col0, wrow, wv, p.acc_mode == 2);
      }
    }
  }
  // The warp's 32 x 64 fp32 sums back into the accumulator at (col0, wrow) through both
  // staging buffers (free after add_loaded_64); returns once the TMA has read them, so the
  // bf16 store that follows may reuse either buffer. Rows past V are clipped by the map.
  static __device__ __forceinline__ void store_sum_64(EpiCtx& c, int col0, int wrow,
                                                      const float (&a)[32], const float (&b)[32]) {
    const uint32_t b0 = c.stage, b1 = c.stage + EPI_BUF_BYTES;
    write_f32_pair(c, a, b);
    fence_async_smem();
    __syncwarp();
    if (c.lane == 0) {
      tma_store_2d(c.tmD, b0, col0, wrow);
      tma_store_2d(c.tmD, b1, col0 + 32, wrow);
      bulk_commit();
      bulk_wait_read_all();
    }
    __syncwarp();
  }
  // a (+)= acc[wrow + lane, col0 .. col0+31], b (+)= acc[.., col0+32 .. col0+63], the 32 x 64
  // fp32 block loaded by TMA into the warp's two staging buffers (zero past V).
  static __device__ __forceinline__ void add_loaded_64(EpiCtx& c, int col0, int wrow,
                                                       float (&a)[32], float (&b)[32]) {
    const uint32_t b0 = c.stage, b1 = c.stage + EPI_BUF_BYTES;
    if (c.lane == 0) {
      bulk_wait_read_all();  // earlier staged stores have finished reading both buffers
      mbar_arrive_expect_tx(c.bar, 2 * EPI_BUF_BYTES);
      tma_load_2d(b0, c.tmD, c.bar, col0, wrow);
      tma_load_2d(b1, c.tmD, c.bar, col0 + 32, wrow);
    }
    __syncwarp();
    // bounded: on expiry the error word is set; wait once more for the copies in flight
    if (!mbar_wait(c.bar, c.bar_phase, c.err)) mbar_wait(c.bar, c.bar_phase, c.err);
    c.bar_phase ^= 1u;
    const uint32_t sw = static_cast<uint32_t>(c.lane & 7);
    const uint32_t off = static_cast<uint32_t>(c.lane) * 128u;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t ch = ((static_cast<uint32_t>(u) ^ sw) << 4) + off;
      const uint4 x = ld_shared_v4(b0 + ch);
      const uint4 y = ld_shared_v4(b1 + ch);
      a[u * 4 + 0] = __fadd_rn(__uint_as_float(x.x), a[u * 4 + 0]);
      a[u * 4 + 1] = __fadd_rn(__uint_as_float(x.y), a[u * 4 + 1]);
      a[u * 4 + 2] = __fadd_rn(__uint_as_float(x.z), a[u * 4 + 2]);
      a[u * 4 + 3] = __fadd_rn(__uint_as_float(x.w), a[u * 4 + 3]);
      b[u * 4 + 0] = __fadd_rn(__uint_as_float(y.x), b[u * 4 + 0]);
      b[u * 4 + 1] = __fadd_rn(__uint_as_float(y.y), b[u * 4 + 1]);
      b[u * 4 + 2] = __fadd_rn(__uint_as_float(y.z), b[u * 4 + 2]);
      b[u * 4 + 3] = __fadd_rn(__uint_as_float(y.w), b[u * 4 + 3]);
    }
    __syncwarp();  // every lane has read both buffers before the bf16 staging reuses one
  }
};
using EpiDW = EpiDWT<PipeDefault::kBK, PipeDefault::kStages, PipeDefault::kEpiBufs>;
using EpiDWWide = EpiDWT<128, 2, 2, 2>;

}  // namespace lmh
