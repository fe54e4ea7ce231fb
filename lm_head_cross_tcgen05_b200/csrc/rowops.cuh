// rowops.cuh — the row-wise (HBM- or latency-bound) kernels around the GEMMs: label
// counting, candidate preparation, the row finalize that combines vocabulary-tile partials
// into lse / loss / log-prob / argmax, the in-place rescale of p~ into the softmax gradient,
// the target fix-up, fixed-order means, the support outputs and the backward coefficients.
// Every reduction runs in a fixed order (lane-strided partial sums in ascending index order,
// then a fixed butterfly), and no kernel uses floating-point atomics.
#pragma once

#include <cuda_bf16.h>
#include <math.h>

#include "sm100.cuh"

namespace lmh {

struct WsHeader {
  uint32_t err;     // device error bits
  int32_t n_valid;  // rows with 0 <= label < V
  uint32_t pad[62];
};
static_assert(sizeof(WsHeader) == 256, "header is one 256-byte block");

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
// Butterfly sum: every lane ends with the same bits (each level adds a commuted pair).
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ int warp_min_int(int x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = min(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// mean-reduction weight of a valid row: 1 / count (0 if count == 0), or 1 for a sum
__device__ __forceinline__ float row_weight(bool valid, int mean, const int32_t* n_given,
                                            const WsHeader* h) {
  if (!valid) return 0.f;
  if (!mean) return 1.f;
  const int n = n_given ? *n_given : h->n_valid;
  return n > 0 ? 1.f / static_cast<float>(n) : 0.f;
}

// ---------------------------------------------------------------------------- labels

__global__ void count_labels_kernel(const int32_t* __restrict__ labels, long long N, int V,
                                    WsHeader* h) {
  int cnt = 0;
  bool bad = false;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < N;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int y = labels[i];
    cnt += (y >= 0 && y < V) ? 1 : 0;
    bad |= (y >= V);
  }
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  const bool any_bad = __any_sync(0xffffffffu, bad);
  if ((threadIdx.x & 31) == 0) {
    if (cnt) atomicAdd(&h->n_valid, cnt);  // integer: exact in any order
    if (any_bad) atomicOr(&h->err, kErrLabelRange);
  }
}

// Rows with 0 <= label < V, added into *out (zeroed before the launch).
__global__ void count_valid_kernel(const int32_t* __restrict__ labels, long long N, int V,
                                   int32_t* out) {
  int cnt = 0;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < N;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int y = labels[i];
    cnt += (y >= 0 && y < V) ? 1 : 0;
  }
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  if ((threadIdx.x & 31) == 0 && cnt) atomicAdd(out, cnt);  // integer: exact in any order
}

// out[i] = sum over r = 0..R-1 of parts[r * n + i], added in ascending r.
__global__ void reduce_ranks_kernel(int R, long long n, const float* __restrict__ parts,
                                    float* __restrict__ out) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float a = parts[i];
    for (int r = 1; r < R; ++r) a += parts[static_cast<long long>(r) * n + i];
    out[i] = a;
  }
}

// ---------------------------------------------------------------------------- candidates
// One block per row (grid-stride), blockDim >= K. For row i: the distinct valid ids in
// ascending order (sorted[i, 0..nuniq)), and for every slot k the sorted index of its id
// (rank[i, k], -1 for padding or out-of-range ids).
__global__ void prep_cands_kernel(const int32_t* __restrict__ ids, long long N, int K, int V,
                                  int32_t* __restrict__ sorted, int32_t* __restrict__ nuniq,
                                  int32_t* __restrict__ rank, WsHeader* h) {
  extern __shared__ int32_t sh[];
  int32_t* s_id = sh;         // [K] valid id or -1
  int32_t* s_first = sh + K;  // [K] 1 if the first slot holding a valid id
  int32_t* s_rank = sh + 2 * K;
  const int k = threadIdx.x;
  for (long long i = blockIdx.x; i < N; i += gridDim.x) {
    int id = -1;
    if (k < K) {
      id = ids[i * K + k];
      if (id >= V) atomicOr(&h->err, kErrLabelRange);
      if (id < 0 || id >= V) id = -1;
      s_id[k] = id;
    }
    __syncthreads();
    int canon = -1;
    if (k < K && id >= 0) {
      canon = k;
      for (int j = 0; j < k; ++j)
        if (s_id[j] == id) { canon = j; break; }
      s_first[k] = canon == k;
    } else if (k < K) {
      s_first[k] = 0;
    }
    __syncthreads();
    if (k < K && id >= 0 && canon == k) {
      int r = 0;
      for (int j = 0; j < K; ++j) r += (s_first[j] && s_id[j] < id) ? 1 : 0;
      s_rank[k] = r;
      sorted[i * K + r] = id;
    }
    if (k == 0) {
      int u = 0;
      for (int j = 0; j < K; ++j) u += s_first[j];
      nuniq[i] = u;
    }
    __syncthreads();
    if (k < K) rank[i * K + k] = (id >= 0) ? s_rank[canon] : -1;
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------- finalize
// One warp per row of the chunk. Combines the row's T tile partials (m_t, s_t, first
// argmax) into lse = M + log sum_t s_t exp(m_t - M), M = max_t m_t; the argmax is that of the
// first tile attaining M. kind 0: CE (loss, logprob, argmax); 1: logprob only; 2: lse only.
// With write_scale (fused CE) s_t is overwritten by alpha_i exp(m_t - lse_i), the factor
// that turns the stored p~ of tile t into the softmax gradient.
struct FinParams {
  int rows;
  long long row0;
  int T;
  int V;
  int kind;
  const float* part_m;
  float* part_s;
  const int32_t* part_i;
  const int32_t* labels;
  const float* zt;
  float* lse;
  float* loss;
  float* logprob;
  int32_t* argmax;
  int write_scale;
  int mean;
  const int32_t* n_given;
  WsHeader* h;
  Temperature temp;
  const float* alpha;  // write_scale: alpha_i given per row (it includes 1 / tau_i), or null
};

__global__ void finalize_rows_kernel(const FinParams p) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= p.rows) return;
  const long long grow = p.row0 + row;
  const float* pm = p.part_m + static_cast<long long>(row) * p.T;
  float* ps = p.part_s + static_cast<long long>(row) * p.T;
  float M = -__int_as_float(0x7f800000);
  for (int t = lane; t < p.T; t += 32) M = fmaxf(M, pm[t]);
  M = warp_max(M);
  const float moff = -M * kLog2e;
  float S = 0.f;
  int tfirst = 0x7fffffff;
  for (int t = lane; t < p.T; t += 32) {
    const float mt = pm[t];
    S += ps[t] * fast_exp2(fmaf(mt, kLog2e, moff));
    if (mt == M && t < tfirst) tfirst = t;
  }
  S = warp_sum(S);
  const float lse = M + logf(S);
  if (lane == 0) {
    p.lse[grow] = lse;
    if (!isfinite(lse)) atomicOr(&p.h->err, kErrNonFinite);
    if (p.temp.rows && !temperature_ok(p.temp.rows[grow])) atomicOr(&p.h->err, kErrTemperature);
  }
  bool valid = false;
  if (p.kind <= 1) {
    const int y = p.labels[grow];
    valid = (y >= 0 && y < p.V);
    if (lane == 0) {
      const float zl = valid ? p.zt[grow] : 0.f;
      const float lossv = valid ? lse - zl : 0.f;
      if (p.kind == 0) p.loss[grow] = lossv;
      if (p.logprob) p.logprob[grow] = valid ? zl - lse : 0.f;
    }
  }
  if (p.argmax) {
    tfirst = warp_min_int(tfirst);
    if (lane == 0) p.argmax[grow] = (tfirst < p.T) ? p.part_i[static_cast<long long>(row) * p.T + tfirst] : 0;
  }
  if (p.write_scale) {
    const float a = p.alpha ? p.alpha[grow]
                            : row_weight(valid, p.mean, p.n_given, p.h) * inv_temperature(p.temp, grow);
    const float loff = -lse * kLog2e;
    for (int t = lane; t < p.T; t += 32) ps[t] = a * fast_exp2(fmaf(pm[t], kLog2e, loff));
  }
}

// ---------------------------------------------------------------------------- G rescale
// In place over the chunk's [rows, ldp] bf16 buffer: G = scale[row, t] * p~ (t = col / 256).
// Grid (x: spans of a row, y: rows). Each thread moves four 16-byte vectors a blockDim apart
// (coalesced), issuing all four loads before any store.
constexpr int kGbuildThreads = 256;
constexpr int kGbuildVec = 4;

__device__ __forceinline__ uint4 scale_bf16x8(uint4 w, float f) {
  float2 a = unpack_bf16x2(w.x), b = unpack_bf16x2(w.y), e = unpack_bf16x2(w.z),
         g = unpack_bf16x2(w.w);
  w.x = pack_bf16x2(a.x * f, a.y * f);
  w.y = pack_bf16x2(b.x * f, b.y * f);
  w.z = pack_bf16x2(e.x * f, e.y * f);
  w.w = pack_bf16x2(g.x * f, g.y * f);
  return w;
}

__global__ void __launch_bounds__(kGbuildThreads)
    gbuild_kernel(int rows, long long ldp, int T, const float* __restrict__ scale,
                  __nv_bfloat16* __restrict__ P) {
  const long long nv = ldp >> 3;  // 16-byte vectors per row
  const long long span = static_cast<long long>(kGbuildThreads) * kGbuildVec;
  for (long long r = blockIdx.y; r < rows; r += gridDim.y) {
    uint4* row4 = reinterpret_cast<uint4*>(P + r * ldp);
    const float* sc = scale + r * T;
    for (long long c0 = blockIdx.x * span + threadIdx.x; c0 < nv; c0 += gridDim.x * span) {
      uint4 w[kGbuildVec];
#pragma unroll
      for (int u = 0; u < kGbuildVec; ++u) {
        const long long c = c0 + u * kGbuildThreads;
        if (c < nv) w[u] = __ldcs(row4 + c);
      }
#pragma unroll
      for (int u = 0; u < kGbuildVec; ++u) {
        const long long c = c0 + u * kGbuildThreads;
        if (c < nv) row4[c] = scale_bf16x8(w[u], sc[c >> 5]);  // 32 vectors per 256-wide tile
      }
    }
  }
}

// Label column of each valid row: G = alpha exp(z_y - lse) - beta, from the fp32 logit, with
// alpha = beta = the mean / sum weight of the row over tau_i, or alpha_i, beta_i given.
__global__ void fix_labels_kernel(int rows, long long row0, int V, long long ldp,
                                  const int32_t* __restrict__ labels,
                                  const float* __restrict__ zt, const float* __restrict__ lse,
                                  int mean, const int32_t* n_given, const WsHeader* h,
                                  Temperature temp, __nv_bfloat16* __restrict__ P,
                                  const float* __restrict__ alpha = nullptr,
                                  const float* __restrict__ beta = nullptr) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  const long long g = row0 + r;
  const int y = labels[g];
  if (y < 0 || y >= V) return;
  const float a = alpha ? alpha[g] : row_weight(true, mean, n_given, h) * inv_temperature(temp, g);
  const float b = beta ? beta[g] : a;
  const float v = a * fast_exp2(fmaf(zt[g], kLog2e, -lse[g] * kLog2e)) - b;
  P[r * ldp + y] = __float2bfloat16_rn(v);
}

// Candidate columns of each row (fused support backward), one warp per row:
// G = alpha_i exp(z_ic - lse_i) - beta_ic at every distinct valid candidate c, from the fp32
// logit (zt and beta are indexed by the sorted candidate position).
__global__ void fix_cands_kernel(int rows, long long row0, int K, long long ldp,
                                 const int32_t* __restrict__ sorted,
                                 const int32_t* __restrict__ nuniq,
                                 const float* __restrict__ zt, const float* __restrict__ lse,
                                 const float* __restrict__ alpha,
                                 const float* __restrict__ beta,
                                 __nv_bfloat16* __restrict__ P) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const long long g = row0 + r;
  const int nu = nuniq[g];
  const float a = alpha[g], loff = -lse[g] * kLog2e;
  for (int u = lane; u < nu; u += 32) {
    const long long o = g * K + u;
    const float v = a * fast_exp2(fmaf(zt[o], kLog2e, loff)) - beta[o];
    P[r * ldp + sorted[o]] = __float2bfloat16_rn(v);
  }
}

// ---------------------------------------------------------------------------- means
// Single block, fixed order: thread t sums elements t, t + blockDim, ... in fp64, then a
// fixed tree over threads. divisor: count from the header / given count (by_count) or n.
__global__ void mean_kernel(const float* __restrict__ vals, long long n, int by_count,
                            const int32_t* n_given, const WsHeader* h, float* out) {
  __shared__ double sh[1024];
  double acc = 0.0;
  for (long long i = threadIdx.x; i < n; i += blockDim.x) acc += static_cast<double>(vals[i]);
  sh[threadIdx.x] = acc;
  __syncthreads();
  for (int s = blockDim.x >> 1; s > 0; s >>= 1) {
    if (threadIdx.x < s) sh[threadIdx.x] += sh[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const long long den = by_count ? (n_given ? *n_given : h->n_valid) : n;
    *out = den > 0 ? static_cast<float>(sh[0] / static_cast<double>(den)) : 0.f;
  }
}

// ---------------------------------------------------------------------------- support
// One warp per row: lp_ik = z_i,c_ik - lse_i (0 for padding), KL_i = sum_k e^r (r - lp).
__global__ void support_out_kernel(long long N, int K, const int32_t* __restrict__ rank,
                                   const float* __restrict__ zt, const float* __restrict__ lse,
                                   const float* __restrict__ ref, float* lp, float* kl) {
  const int lane = threadIdx.x & 31;
  const long long i = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (i >= N) return;
  const float l = lse[i];
  float acc = 0.f;
  for (int k = lane; k < K; k += 32) {
    const int r = rank[i * K + k];
    float v = 0.f;
    if (r >= 0) {
      v = zt[i * K + r] - l;
      if (ref) {
        const float rr = ref[i * K + k];
        acc += expf(rr) * (rr - v);
      }
    }
    if (lp) lp[i * K + k] = v;
  }
  acc = warp_sum(acc);
  if (kl && lane == 0) kl[i] = acc;
}

// ---------------------------------------------------------------------------- backward
// alpha_i and beta (per label, or per sorted candidate id summed over repeated slots) of
// G = alpha P - sum beta e_t for the four objectives; one warp per row.
// Without `grad` every row term has the weight 1, or 1 / count with `mean` (count: the valid
// rows of the labels for CE / LOGPROB, N for the support objectives); with `scalar` grad[0]
// multiplies that weight instead of grad holding one weight per term. beta covers the
// candidates of `rank` (this vocabulary or shard); alpha all valid ones (see alpha_ids).
__global__ void bwd_coef_kernel(int mode, long long N, int K, int V,
                                const int32_t* __restrict__ targets,
                                const float* __restrict__ grad, const float* __restrict__ ref,
                                const int32_t* __restrict__ rank,
                                const int32_t* __restrict__ nuniq, Temperature temp, int mean,
                                int scalar, WsHeader* h, float* __restrict__ alpha,
                                float* __restrict__ beta, const int32_t* n_given = nullptr,
                                const int32_t* __restrict__ alpha_ids = nullptr,
                                int alpha_V = 0) {
  const int lane = threadIdx.x & 31;
  const long long i = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (i >= N) return;
  const float it = inv_temperature(temp, i);  // chain-rule factor of the tempered logits
  if (lane == 0 && temp.rows && !temperature_ok(temp.rows[i])) atomicOr(&h->err, kErrTemperature);
  float unit = 1.f;  // weight of a row term when no per-term grad is given
  if (mean) {
    const long long cnt = n_given ? *n_given : (mode <= 1) ? h->n_valid : N;
    unit = cnt > 0 ? 1.f / static_cast<float>(cnt) : 0.f;
  }
  if (scalar) {
    unit *= grad[0];
    grad = nullptr;
  }
  if (mode <= 1) {  // CE / LOGPROB over labels
    if (lane == 0) {
      const int y = targets[i];
      const bool ok = (y >= 0 && y < V);
      const float g = ok ? (grad ? grad[i] : unit) * it : 0.f;
      const float a = (mode == 0) ? g : -g;
      alpha[i] = a;
      beta[i] = a;
    }
    return;
  }
  // support: weight w_k = gamma_ik (SUPPORT_LOGPROB, alpha = -sum, beta = -w) or
  // g_i exp(r_ik) (SUPPORT_KL, alpha = sum, beta = w)
  const float gi = (mode == 3) ? (grad ? grad[i] : unit) * it : 0.f;
  float sum = 0.f;
  for (int k = lane; k < K; k += 32) {
    // alpha sums every valid candidate: of this vocabulary (rank >= 0), or, for one shard of a
    // split vocabulary, of the whole one (alpha_ids: the global ids, valid below alpha_V)
    const bool counted = alpha_ids ? (alpha_ids[i * K + k] >= 0 && alpha_ids[i * K + k] < alpha_V)
                                   : rank[i * K + k] >= 0;
    if (!counted) continue;
    sum += (mode == 2) ? (grad ? grad[i * K + k] : unit) * it : gi * expf(ref[i * K + k]);
  }
  sum = warp_sum(sum);
  if (lane == 0) alpha[i] = (mode == 2) ? -sum : sum;
  const int nu = nuniq[i];
  for (int r = lane; r < nu; r += 32) {
    float b = 0.f;
    for (int k = 0; k < K; ++k) {
      if (rank[i * K + k] != r) continue;
      b += (mode == 2) ? (grad ? grad[i * K + k] : unit) * it : gi * expf(ref[i * K + k]);
    }
    beta[i * K + r] = (mode == 2) ? -b : b;
  }
}

// ---------------------------------------------------------------------------- split-K sum
// dH[r, j] = bf16(sum over s = 0, 1, ... of part[s, r, j]): the fixed-order reduction of the
// split dH GEMM's fp32 partials. Pairs of columns per thread, grid-stride.
__global__ void split_sum_kernel(int splits, long long rows, int d, const float* __restrict__ part,
                                 __nv_bfloat16* __restrict__ out) {
  const long long n2 = rows * d / 2;
  const long long plane = rows * d;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < n2;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    float2 acc = __ldcs(reinterpret_cast<const float2*>(part) + e);
    for (int sp = 1; sp < splits; ++sp) {
      const float2 v = __ldcs(reinterpret_cast<const float2*>(part + sp * plane) + e);
      acc.x += v.x;
      acc.y += v.y;
    }
    reinterpret_cast<uint32_t*>(out)[e] = pack_bf16x2(acc.x, acc.y);
  }
}

// ---------------------------------------------------------------------------- self-test
// One thread waits on an mbarrier that nothing ever arrives on, with the same bounded wait
// the GEMMs use: the wait gives up after timeout_ns and records kErrTimeout.
__global__ void wait_selftest_kernel(uint32_t* err, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, err, timeout_ns);
}

// ---------------------------------------------------------------------------- dW cast
// dst = bf16(src) over n4 groups of 4 elements (round to nearest even).
__global__ void cast_bf16_kernel(const float* __restrict__ src, long long n4,
                                 __nv_bfloat16* __restrict__ dst) {
  const float4* s4 = reinterpret_cast<const float4*>(src);
  uint2* d4 = reinterpret_cast<uint2*>(dst);
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 v = __ldcs(s4 + i);
    __stcs(d4 + i, make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w)));
  }
}

// ---------------------------------------------------------------------------- gradient scale
// x = bf16(x * g[0]) in place over n4 groups of 4 elements (round to nearest even; g = 1
// leaves every bit unchanged).
__global__ void scale_bf16_kernel(long long n4, const float* __restrict__ g,
                                  __nv_bfloat16* __restrict__ x) {
  const float s = *g;
  uint2* x4 = reinterpret_cast<uint2*>(x);
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint2 w = x4[i];
    const float2 a = unpack_bf16x2(w.x), b = unpack_bf16x2(w.y);
    x4[i] = make_uint2(pack_bf16x2(a.x * s, a.y * s), pack_bf16x2(b.x * s, b.y * s));
  }
}

}  // namespace lmh
