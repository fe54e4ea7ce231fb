// epilogues.cuh — what each GEMM does with its fp32 accumulator tile (128 rows x 256
// columns in TMEM). Each epilogue thread owns one tile row and reads it as eight 32-column
// slices with tcgen05.ld; nothing here synchronises across threads.
#pragma once

#include <cuda_bf16.h>
#include <limits.h>

#include "gemm.cuh"

namespace lmh {

constexpr int kSlices = BN / 32;
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

// kStream: the data is read once, much later (the chunk's softmax / gradient buffer): store
// with the streaming hint so it does not push reused operands out of L2.
template <bool kStream = false>
__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float (&v)[32],
                                              int nvec) {
  // nvec: how many of the four 8-column vectors to write (the rest lie past the row end)
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    if (u < nvec) {
      uint4 w;
      w.x = pack_bf16x2(v[8 * u + 0], v[8 * u + 1]);
      w.y = pack_bf16x2(v[8 * u + 2], v[8 * u + 3]);
      w.z = pack_bf16x2(v[8 * u + 4], v[8 * u + 5]);
      w.w = pack_bf16x2(v[8 * u + 6], v[8 * u + 7]);
      if (kStream) __stcs(d4 + u, w); else d4[u] = w;
    }
  }
}

// ------------------------------------------------------------------ logits statistics
// Forward epilogue of z = H_c W^T. Per (row, 256-wide vocabulary tile t) it writes the tile
// maximum m_t, s_t = sum_v exp(z_v - m_t), the first column attaining m_t, and the logits at
// the row's targets; with kStoreP it also stores p~ = exp(z - m_t) in bf16, which the fused
// backward rescales into the softmax gradient. Columns >= V are masked to -inf.
template <int TK, bool kStoreP>
struct EpiStats {
  static constexpr int kId = kStoreP ? 3 : 2;  // gemm_logits_stats(_store)
  static constexpr int kAMajorMN = 0;  // H chunk [rows, d], K-major
  static constexpr int kBMajorMN = 0;  // W [V, d], K-major
  struct Params {
    int rows;           // rows of this chunk
    long long row0;     // global index of the chunk's first row
    int V;
    int T;              // vocabulary tiles, ceil(V / 256)
    long long ldp;      // row stride of P (elements), round_up(V, 8)
    Targets tg;
    float* zt;          // target logits: [N] (kLabel) or [N, K] by sorted index (kCands)
    float* part_m;      // [rows, T]
    float* part_s;      // [rows, T]
    int32_t* part_i;    // [rows, T]
    __nv_bfloat16* P;   // [rows, ldp] (kStoreP)
  };

  static __device__ __forceinline__ void tile(const Params& p, int mb, int nb, uint32_t taddr,
                                              int rit) {
    const int row = mb * BM + rit;
    const bool rv = row < p.rows;
    const long long grow = p.row0 + row;
    const int n0 = nb * BN;
    const bool full = n0 + BN <= p.V;
    TargetCursor<TK> cur;
    if (rv) cur.init(p.tg, grow, n0, p.V); else cur.none();

    // pass 1: maximum, its first column, target logits
    float m = kNegInf;
    int am = n0;
#pragma unroll 1
    for (int sl = 0; sl < kSlices; ++sl) {
      float v[32];
      tmem_ld32(taddr + sl * 32, v);
      const int col0 = n0 + sl * 32;
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

    // pass 2: sum of exp(z - m), optionally p~ = exp(z - m) to P
    const float moff = -m * kLog2e;
    float s0 = 0.f, s1 = 0.f;
    __nv_bfloat16* prow = kStoreP ? p.P + static_cast<long long>(row) * p.ldp : nullptr;
#pragma unroll 1
    for (int sl = 0; sl < kSlices; ++sl) {
      float v[32];
      tmem_ld32(taddr + sl * 32, v);
      const int col0 = n0 + sl * 32;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float e = fast_exp2(fmaf(v[j], kLog2e, moff));
        v[j] = (full || col0 + j < p.V) ? e : 0.f;
      }
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        s0 += v[j];
        s1 += v[j + 1];
      }
      if (kStoreP && rv) {
        const long long rem = p.ldp - col0;
        const int nvec = rem >= 32 ? 4 : (rem > 0 ? static_cast<int>(rem >> 3) : 0);
        store_bf16x32<true>(prow + col0, v, nvec);
      }
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
// targets, written in bf16 to the chunk's G buffer (zero past column V).
template <int TK>
struct EpiGrad {
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
    __nv_bfloat16* P;    // [rows, ldp]
  };

  static __device__ __forceinline__ void tile(const Params& p, int mb, int nb, uint32_t taddr,
                                              int rit) {
    const int row = mb * BM + rit;
    const bool rv = row < p.rows;
    const long long grow = p.row0 + row;
    const int n0 = nb * BN;
    const bool full = n0 + BN <= p.V;
    const float a = rv ? p.alpha[grow] : 0.f;
    const float loff = rv ? -p.lse[grow] * kLog2e : 0.f;
    TargetCursor<TK> cur;
    if (rv) cur.init(p.tg, grow, n0, p.V); else cur.none();
    __nv_bfloat16* prow = p.P + static_cast<long long>(row) * p.ldp;
#pragma unroll 1
    for (int sl = 0; sl < kSlices; ++sl) {
      float v[32];
      tmem_ld32(taddr + sl * 32, v);
      const int col0 = n0 + sl * 32;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float e = a * fast_exp2(fmaf(v[j], kLog2e, loff));
        v[j] = (full || col0 + j < p.V) ? e : 0.f;
      }
      cur.slice(col0, [&](int j, int idx) {
        v[j] -= (TK == kLabel) ? p.beta[grow] : p.beta[grow * p.tg.K + idx];
      });
      if (rv) {
        const long long rem = p.ldp - col0;
        const int nvec = rem >= 32 ? 4 : (rem > 0 ? static_cast<int>(rem >> 3) : 0);
        store_bf16x32<true>(prow + col0, v, nvec);
      }
    }
  }
};

// ------------------------------------------------------------------ dH = G W
struct EpiDH {
  static constexpr int kId = 5;  // gemm_dH
  static constexpr int kAMajorMN = 0;  // G chunk [rows, V], K-major
  static constexpr int kBMajorMN = 1;  // W [V, d] read as [K = V, N = d], N contiguous
  struct Params {
    int rows;
    long long row0;
    int d;
    __nv_bfloat16* dH;  // [N, d]
  };
  static __device__ __forceinline__ void tile(const Params& p, int mb, int nb, uint32_t taddr,
                                              int rit) {
    const int row = mb * BM + rit;
    const bool rv = row < p.rows;
    const int n0 = nb * BN;
    __nv_bfloat16* out = p.dH + (p.row0 + row) * static_cast<long long>(p.d);
#pragma unroll 1
    for (int sl = 0; sl < kSlices; ++sl) {
      const int col0 = n0 + sl * 32;
      if (col0 >= p.d) break;  // uniform across the warp
      float v[32];
      tmem_ld32(taddr + sl * 32, v);
      if (rv) store_bf16x32(out + col0, v, 4);
    }
  }
};

// ------------------------------------------------------------------ dW = G^T H_c
// acc_mode 0: the tile sum is the whole dW; 1: acc = 0 + sum (first chunk into a fresh
// internal accumulator); 2: acc += sum (the caller's or a later chunk). With `out` set the
// bf16 cast of the resulting value is written as well (last chunk).
struct EpiDW {
  static constexpr int kId = 6;  // gemm_dW
  static constexpr int kAMajorMN = 1;  // G^T: G chunk [rows, V] read as [K = rows, M = V]
  static constexpr int kBMajorMN = 1;  // H chunk [rows, d] read as [K = rows, N = d]
  struct Params {
    int V;
    int d;
    float* acc;           // [V, d] or null
    int acc_mode;
    __nv_bfloat16* out;   // [V, d] or null
  };
  static __device__ __forceinline__ void tile(const Params& p, int mb, int nb, uint32_t taddr,
                                              int rit) {
    const int vrow = mb * BM + rit;
    const bool vv = vrow < p.V;
    const int n0 = nb * BN;
    const long long base = static_cast<long long>(vrow) * p.d;
#pragma unroll 1
    for (int sl = 0; sl < kSlices; ++sl) {
      const int col0 = n0 + sl * 32;
      if (col0 >= p.d) break;
      float v[32];
      tmem_ld32(taddr + sl * 32, v);
      if (!vv) continue;
      if (p.acc_mode != 0) {
        float4* a4 = reinterpret_cast<float4*>(p.acc + base + col0);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float4 a;
          if (p.acc_mode == 2) {
            a = a4[u];
            a.x += v[4 * u + 0];
            a.y += v[4 * u + 1];
            a.z += v[4 * u + 2];
            a.w += v[4 * u + 3];
          } else {
            a.x = v[4 * u + 0] + 0.f;
            a.y = v[4 * u + 1] + 0.f;
            a.z = v[4 * u + 2] + 0.f;
            a.w = v[4 * u + 3] + 0.f;
          }
          a4[u] = a;
          v[4 * u + 0] = a.x;
          v[4 * u + 1] = a.y;
          v[4 * u + 2] = a.z;
          v[4 * u + 3] = a.w;
        }
      }
      if (p.out) store_bf16x32(p.out + base + col0, v, 4);
    }
  }
};

}  // namespace lmh
