// sparse.cuh — the support-set entries renormalised over each row's candidate set: only the
// K candidate logits of a row take part, so the work is K dot products per row forward and a
// gather (dH) plus a scatter (dW) backward, with no vocabulary-wide contraction.
//
// Definitions (row i, distinct valid candidate ids s_iu, u < nuniq_i; tau_i the temperature):
//   z_iu   = <H_i, W_{s_iu}> / tau_i
//   lse_i  = log sum_u exp(z_iu)              (the log-normaliser over the support)
//   lp_ik  = z_i,u(k) - lse_i                 (u(k): the distinct id of slot k)
//   q_iu   = exp(z_iu - lse_i)
//   G_iu   = alpha_i q_iu - beta_iu           (alpha, beta: the same coefficients as the
//                                               full-vocabulary objectives, 1/tau_i included)
//   dH_i   = sum_u G_iu W_{s_iu},   dW_v = sum_{(i,u): s_iu = v} G_iu H_i
// Every sum runs in a fixed order: dot products lane-strided then a butterfly; dH over u
// ascending; dW over the rows i of each vocabulary id in ascending order (the pairs of an id
// are sorted by row before they are summed), so results are bitwise reproducible.
#pragma once

#include <cuda_bf16.h>

#include "rowops.cuh"

namespace lmh {

__device__ __forceinline__ float dot_bf16_row(const __nv_bfloat16* a, const __nv_bfloat16* b,
                                              int d, int lane) {
  // d is a multiple of 64: each lane takes 8-element vectors lane, lane + 32, ...
  const uint4* a4 = reinterpret_cast<const uint4*>(a);
  const uint4* b4 = reinterpret_cast<const uint4*>(b);
  float acc = 0.f;
  for (int v = lane; v < d / 8; v += 32) {
    const uint4 x = a4[v], y = b4[v];
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 p = unpack_bf16x2(xs[u]), q = unpack_bf16x2(ys[u]);
      acc = fmaf(p.x, q.x, acc);
      acc = fmaf(p.y, q.y, acc);
    }
  }
  return warp_sum(acc);
}

// One block per row (grid-stride), one warp per distinct candidate: zt[i, u] = z_iu.
__global__ void support_dots_kernel(long long N, int K, int d, const __nv_bfloat16* __restrict__ H,
                                    const __nv_bfloat16* __restrict__ W,
                                    const int32_t* __restrict__ sorted,
                                    const int32_t* __restrict__ nuniq, Temperature temp,
                                    float* __restrict__ zt) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (long long i = blockIdx.x; i < N; i += gridDim.x) {
    const int nu = nuniq[i];
    const float it = inv_temperature(temp, i);
    const __nv_bfloat16* h = H + i * d;
    for (int u = warp; u < nu; u += nw) {
      const float z = dot_bf16_row(h, W + static_cast<long long>(sorted[i * K + u]) * d, d, lane);
      if (lane == 0) zt[i * K + u] = z * it;
    }
  }
}

// One warp per row: lse over the row's distinct candidates (0 for a row without any).
__global__ void support_lse_kernel(long long N, int K, const int32_t* __restrict__ nuniq,
                                   const float* __restrict__ zt, float* __restrict__ lse,
                                   WsHeader* h) {
  const int lane = threadIdx.x & 31;
  const long long i = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (i >= N) return;
  const int nu = nuniq[i];
  float m = -__int_as_float(0x7f800000);
  for (int u = lane; u < nu; u += 32) m = fmaxf(m, zt[i * K + u]);
  m = warp_max(m);
  float s = 0.f;
  for (int u = lane; u < nu; u += 32) s += fast_exp2((zt[i * K + u] - m) * kLog2e);
  s = warp_sum(s);
  if (lane == 0) {
    const float l = nu > 0 ? m + logf(s) : 0.f;
    lse[i] = l;
    if (!isfinite(l)) atomicOr(&h->err, kErrNonFinite);
  }
}

// Backward, per row: gu[i, u] = alpha_i exp(z_iu - lse_i) - beta_iu, then
// dH_i = sum_u gu[i, u] W_{s_iu} (u ascending). One block per row; threads over d.
__global__ void support_grad_dh_kernel(long long N, int K, int d,
                                       const __nv_bfloat16* __restrict__ W,
                                       const int32_t* __restrict__ sorted,
                                       const int32_t* __restrict__ nuniq,
                                       const float* __restrict__ zt,
                                       const float* __restrict__ lse,
                                       const float* __restrict__ alpha,
                                       const float* __restrict__ beta, float* __restrict__ gu,
                                       __nv_bfloat16* __restrict__ dH) {
  extern __shared__ float sg[];  // [K] this row's gu
  for (long long i = blockIdx.x; i < N; i += gridDim.x) {
    const int nu = nuniq[i];
    const float a = alpha[i], l = lse[i];
    for (int u = threadIdx.x; u < nu; u += blockDim.x) {
      const float g = a * fast_exp2((zt[i * K + u] - l) * kLog2e) - beta[i * K + u];
      sg[u] = g;
      gu[i * K + u] = g;
    }
    __syncthreads();
    if (dH) {
      for (int j = threadIdx.x * 2; j < d; j += blockDim.x * 2) {
        float acc0 = 0.f, acc1 = 0.f;
        for (int u = 0; u < nu; ++u) {
          const float2 w = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(
              W + static_cast<long long>(sorted[i * K + u]) * d + j));
          acc0 = fmaf(sg[u], w.x, acc0);
          acc1 = fmaf(sg[u], w.y, acc1);
        }
        *reinterpret_cast<uint32_t*>(dH + i * d + j) = pack_bf16x2(acc0, acc1);
      }
    }
    __syncthreads();
  }
}

// Scatter support: count the (row, distinct id) pairs of every vocabulary id.
__global__ void support_count_kernel(long long N, int K, const int32_t* __restrict__ sorted,
                                     const int32_t* __restrict__ nuniq, int32_t* __restrict__ cnt) {
  for (long long p = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; p < N * K;
       p += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long i = p / K;
    const int u = static_cast<int>(p - i * K);
    if (u < nuniq[i]) atomicAdd(&cnt[sorted[p]], 1);  // integer counts: exact in any order
  }
}

// Exclusive scan of cnt[0..V) into off[0..V] with one block (fixed order, V up to 2^31).
__global__ void scan_kernel(int V, const int32_t* __restrict__ cnt, int32_t* __restrict__ off) {
  __shared__ int32_t part[1024];
  const int t = threadIdx.x, T = blockDim.x;
  const long long per = (static_cast<long long>(V) + T - 1) / T;
  const long long b = t * per, e = b + per < V ? b + per : V;
  int32_t s = 0;
  for (long long v = b; v < e; ++v) s += cnt[v];
  part[t] = s;
  __syncthreads();
  if (t == 0) {
    int32_t run = 0;
    for (int k = 0; k < T; ++k) {
      const int32_t x = part[k];
      part[k] = run;
      run += x;
    }
  }
  __syncthreads();
  int32_t run = part[t];
  for (long long v = b; v < e; ++v) {
    off[v] = run;
    run += cnt[v];
  }
  if (t == T - 1) off[V] = run;
}

// Place every pair's row index into its id's bucket (order inside a bucket is not yet fixed).
__global__ void support_place_kernel(long long N, int K, const int32_t* __restrict__ sorted,
                                     const int32_t* __restrict__ nuniq,
                                     const int32_t* __restrict__ off, int32_t* __restrict__ fill,
                                     int32_t* __restrict__ pair_row,
                                     int32_t* __restrict__ pair_slot) {
  for (long long p = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; p < N * K;
       p += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long i = p / K;
    const int u = static_cast<int>(p - i * K);
    if (u >= nuniq[i]) continue;
    const int v = sorted[p];
    const int at = off[v] + atomicAdd(&fill[v], 1);
    pair_row[at] = static_cast<int32_t>(i);
    pair_slot[at] = u;
  }
}

// One warp per vocabulary id: sort its bucket by row (insertion sort; buckets are short),
// which fixes the summation order of dW whatever order the pairs were placed in.
__global__ void support_sort_buckets_kernel(int V, const int32_t* __restrict__ off,
                                            int32_t* __restrict__ pair_row,
                                            int32_t* __restrict__ pair_slot) {
  const long long v = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (v >= V) return;
  const int b = off[v], e = off[v + 1];
  for (int x = b + 1; x < e; ++x) {
    const int r = pair_row[x], s = pair_slot[x];
    int y = x - 1;
    while (y >= b && pair_row[y] > r) {
      pair_row[y + 1] = pair_row[y];
      pair_slot[y + 1] = pair_slot[y];
      --y;
    }
    pair_row[y + 1] = r;
    pair_slot[y + 1] = s;
  }
}

// dW_v = sum over the bucket of v (rows ascending) of gu[i, u] H_i; one block per id,
// threads over d. acc_mode as for the dense dW: 0 the sum is dW, 1 acc = sum, 2 acc += sum.
__global__ void support_dw_kernel(int V, int K, int d, const __nv_bfloat16* __restrict__ H,
                                  const int32_t* __restrict__ off,
                                  const int32_t* __restrict__ pair_row,
                                  const int32_t* __restrict__ pair_slot,
                                  const float* __restrict__ gu, float* __restrict__ acc,
                                  int acc_mode, __nv_bfloat16* __restrict__ dW) {
  for (long long v = blockIdx.x; v < V; v += gridDim.x) {
    const int b = off[v], e = off[v + 1];
    for (int j = threadIdx.x * 2; j < d; j += blockDim.x * 2) {
      float s0 = 0.f, s1 = 0.f;
      for (int x = b; x < e; ++x) {
        const long long i = pair_row[x];
        const float g = gu[i * K + pair_slot[x]];
        const float2 hv = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(H + i * d + j));
        s0 = fmaf(g, hv.x, s0);
        s1 = fmaf(g, hv.y, s1);
      }
      if (acc_mode == 1) {
        *reinterpret_cast<float2*>(acc + v * d + j) = make_float2(s0, s1);
      } else if (acc_mode == 2) {
        float2* a2 = reinterpret_cast<float2*>(acc + v * d + j);
        float2 a = *a2;
        a.x += s0;
        a.y += s1;
        *a2 = a;
        s0 = a.x;
        s1 = a.y;
      }
      if (dW) *reinterpret_cast<uint32_t*>(dW + v * d + j) = pack_bf16x2(s0, s1);
    }
  }
}

}  // namespace lmh
