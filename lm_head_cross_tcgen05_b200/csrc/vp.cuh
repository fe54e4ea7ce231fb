// vp.cuh — the row kernels of the vocabulary-parallel cross entropy. W is split by rows into R
// contiguous shards [v0_r, v0_r + V_r), one per rank. Each rank runs the logits GEMM over its
// shard and reduces every row to a 4-word record; the records of all ranks, gathered in rank
// order, combine into the row's lse, loss, log-prob and argmax. The backward recomputes G on
// each shard with the global lse; the shards' fp32 dH contributions are summed in rank order.
//
// Record of row i on rank r (4 x 32 bits, the layout every rank and the combine share):
//   [0] lse_r  = log sum_{v in shard} exp(z_iv)        (fp32)
//   [1] max_r  = max_{v in shard} z_iv                  (fp32)
//   [2] arg_r  = the smallest global id attaining max_r (int32 bits)
//   [3] zy_r   = z_i,y_i if the label lies in the shard, else -inf (fp32)
// z is the tempered logit (z / tau_i) when a temperature is given.
#pragma once

#include "epilogues.cuh"
#include "rowops.cuh"

namespace lmh {

// labels_local[i] = y_i - v0 when v0 <= y_i < v0 + Vr, else -1 (no target column here).
__global__ void vp_local_labels_kernel(long long N, const int32_t* __restrict__ labels,
                                       long long v0, long long Vr,
                                       int32_t* __restrict__ local) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < N;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long y = labels[i];
    local[i] = (y >= v0 && y < v0 + Vr) ? static_cast<int32_t>(y - v0) : -1;
  }
}

// One warp per row of a chunk: the row's T tile partials of this shard (ascending t) into its
// record. Same arithmetic as the single-device row finalize.
__global__ void vp_finalize_kernel(int rows, long long row0, int T, long long v0,
                                   const float* __restrict__ part_m,
                                   const float* __restrict__ part_s,
                                   const int32_t* __restrict__ part_i,
                                   const int32_t* __restrict__ local,
                                   const float* __restrict__ zt, Temperature temp, WsHeader* h,
                                   float4* __restrict__ rec) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const long long grow = row0 + row;
  const float* pm = part_m + static_cast<long long>(row) * T;
  const float* ps = part_s + static_cast<long long>(row) * T;
  float M = -__int_as_float(0x7f800000);
  for (int t = lane; t < T; t += 32) M = fmaxf(M, pm[t]);
  M = warp_max(M);
  const float moff = -M * kLog2e;
  float S = 0.f;
  int tfirst = 0x7fffffff;
  for (int t = lane; t < T; t += 32) {
    const float mt = pm[t];
    S += ps[t] * fast_exp2(fmaf(mt, kLog2e, moff));
    if (mt == M && t < tfirst) tfirst = t;
  }
  S = warp_sum(S);
  tfirst = warp_min_int(tfirst);
  if (lane == 0) {
    const float l = M + logf(S);
    if (!isfinite(l)) atomicOr(&h->err, kErrNonFinite);
    if (temp.rows && !temperature_ok(temp.rows[grow])) atomicOr(&h->err, kErrTemperature);
    const int arg = (tfirst < T) ? part_i[static_cast<long long>(row) * T + tfirst] : 0;
    const float zy = local[grow] >= 0 ? zt[grow] : -__int_as_float(0x7f800000);
    rec[grow] = make_float4(l, M, __int_as_float(static_cast<int32_t>(v0 + arg)), zy);
  }
}

// One thread per row: combine the R records (rank order) of the row.
//   lse  = m + log sum_r exp(lse_r - m), m = max_r lse_r, summed in ascending r
//   argmax: the record with the largest max_r, the first rank on ties (shards ascend, so the
//           smallest global id wins, as on one device)
//   loss = lse - zy and logprob = zy - lse for rows with 0 <= y < V, else 0; zy is the one
//          finite zy_r (a valid row whose label no shard holds is flagged non-finite)
__global__ void vp_combine_kernel(long long N, int R, int V, const float4* __restrict__ rec,
                                  const int32_t* __restrict__ labels, float* __restrict__ lse,
                                  float* __restrict__ loss, float* __restrict__ logprob,
                                  int32_t* __restrict__ argmax, WsHeader* h) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < N;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float m = -__int_as_float(0x7f800000);
    for (int r = 0; r < R; ++r) m = fmaxf(m, rec[static_cast<long long>(r) * N + i].x);
    const float moff = -m * kLog2e;
    float s = 0.f, best = -__int_as_float(0x7f800000), zy = -__int_as_float(0x7f800000);
    int arg = 0;
    bool first = true;
    for (int r = 0; r < R; ++r) {
      const float4 q = rec[static_cast<long long>(r) * N + i];
      s += fast_exp2(fmaf(q.x, kLog2e, moff));
      if (first || q.y > best) {
        best = q.y;
        arg = __float_as_int(q.z);
        first = false;
      }
      if (q.w > zy) zy = q.w;
    }
    const float l = m + logf(s);
    lse[i] = l;
    const int y = labels[i];
    const bool valid = (y >= 0 && y < V);
    if (!isfinite(l) || (valid && !isfinite(zy))) atomicOr(&h->err, kErrNonFinite);
    if (loss) loss[i] = valid ? l - zy : 0.f;
    if (logprob) logprob[i] = valid ? zy - l : 0.f;
    if (argmax) argmax[i] = arg;
  }
}

// ---------------------------------------------------------------------------- support entries
// Record of row i on rank r for the support entries (K + 1 floats): [0] lse_r as above, then
// for every slot k the logit of candidate c_ik if it lies in the shard, else -inf.
// One warp per row of a chunk; sorted / rank describe the shard-local candidates.
__global__ void vp_support_finalize_kernel(int rows, long long row0, int T, int K,
                                           const float* __restrict__ part_m,
                                           const float* __restrict__ part_s,
                                           const int32_t* __restrict__ rank,
                                           const float* __restrict__ zt, Temperature temp,
                                           WsHeader* h, float* __restrict__ rec) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const long long grow = row0 + row;
  const float* pm = part_m + static_cast<long long>(row) * T;
  const float* ps = part_s + static_cast<long long>(row) * T;
  float M = -__int_as_float(0x7f800000);
  for (int t = lane; t < T; t += 32) M = fmaxf(M, pm[t]);
  M = warp_max(M);
  const float moff = -M * kLog2e;
  float S = 0.f;
  for (int t = lane; t < T; t += 32) S += ps[t] * fast_exp2(fmaf(pm[t], kLog2e, moff));
  S = warp_sum(S);
  float* out = rec + grow * (K + 1);
  if (lane == 0) {
    const float l = M + logf(S);
    if (!isfinite(l)) atomicOr(&h->err, kErrNonFinite);
    if (temp.rows && !temperature_ok(temp.rows[grow])) atomicOr(&h->err, kErrTemperature);
    out[0] = l;
  }
  for (int k = lane; k < K; k += 32) {
    const int r = rank[grow * K + k];
    out[1 + k] = r >= 0 ? zt[grow * K + r] : -__int_as_float(0x7f800000);
  }
}

// One warp per row: the R support records (rank order) of the row into lse (as for the CE
// records), lp_ik = z_ik - lse_i with z_ik the one finite candidate logit over the ranks (0 for
// padding ids < 0; ids >= V flagged and treated as padding), and with ref the KL term
// sum_k exp(r_ik) (r_ik - lp_ik) over the valid slots.
__global__ void vp_support_combine_kernel(long long N, int R, int K, int V,
                                          const float* __restrict__ rec,
                                          const int32_t* __restrict__ ids,
                                          const float* __restrict__ ref, float* __restrict__ lp,
                                          float* __restrict__ lse, float* __restrict__ kl,
                                          WsHeader* h) {
  const int lane = threadIdx.x & 31;
  const long long i = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (i >= N) return;
  const long long rs = N * (K + 1);  // one rank's records
  float l = 0.f;
  if (lane == 0) {
    float m = -__int_as_float(0x7f800000);
    for (int r = 0; r < R; ++r) m = fmaxf(m, rec[r * rs + i * (K + 1)]);
    const float moff = -m * kLog2e;
    float s = 0.f;
    for (int r = 0; r < R; ++r) s += fast_exp2(fmaf(rec[r * rs + i * (K + 1)], kLog2e, moff));
    l = m + logf(s);
    lse[i] = l;
    if (!isfinite(l)) atomicOr(&h->err, kErrNonFinite);
  }
  l = __shfl_sync(0xffffffffu, l, 0);
  float acc = 0.f;
  for (int k = lane; k < K; k += 32) {
    const int id = ids[i * K + k];
    if (id >= V) atomicOr(&h->err, kErrLabelRange);
    const bool valid = id >= 0 && id < V;
    float z = -__int_as_float(0x7f800000);
    for (int r = 0; r < R; ++r) z = fmaxf(z, rec[r * rs + i * (K + 1) + 1 + k]);
    if (valid && !isfinite(z)) atomicOr(&h->err, kErrNonFinite);
    const float v = valid ? z - l : 0.f;
    if (lp) lp[i * K + k] = v;
    if (ref && valid) {
      const float rr = ref[i * K + k];
      acc += expf(rr) * (rr - v);
    }
  }
  acc = warp_sum(acc);
  if (kl && lane == 0) kl[i] = acc;
}

// Fused backward of a shard, one warp per row: the tile factors that turn the stored
// p~ = exp(z - m_t) into the softmax gradient with the combined lse,
//   s_t = alpha_i exp(m_t - lse_i),  alpha_i = weight of row i / tau_i,
// the weight being 1 (sum) or 1 / count (mean) for rows with 0 <= y_i < V (all ranks' count).
__global__ void vp_scale_kernel(int rows, int T, int V, const int32_t* __restrict__ labels,
                                const float* __restrict__ lse, const float* __restrict__ part_m,
                                int mean, const int32_t* n_given, const WsHeader* h,
                                Temperature temp, float* __restrict__ part_s) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int y = labels[row];
  const float a = row_weight(y >= 0 && y < V, mean, n_given, h) * inv_temperature(temp, row);
  const float loff = -lse[row] * kLog2e;
  const float* pm = part_m + static_cast<long long>(row) * T;
  float* ps = part_s + static_cast<long long>(row) * T;
  for (int t = lane; t < T; t += 32) ps[t] = a * fast_exp2(fmaf(pm[t], kLog2e, loff));
}

// out[j] = bf16(sum_{r = 0..R-1} parts[r][j]) over n elements (a multiple of 4), the ranks'
// fp32 contributions added in ascending rank order.
__global__ void vp_reduce_rows_kernel(int R, long long n4, const float4* __restrict__ parts,
                                      __nv_bfloat16* __restrict__ out) {
  uint2* o = reinterpret_cast<uint2*>(out);
  for (long long j = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; j < n4;
       j += static_cast<long long>(gridDim.x) * blockDim.x) {
    float4 a = __ldcs(parts + j);
    for (int r = 1; r < R; ++r) {
      const float4 b = __ldcs(parts + static_cast<long long>(r) * n4 + j);
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    __stcs(o + j, make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w)));
  }
}

// A rank without rows still owns one slot of rows in every receive buffer of a row scatter
// (its fp32 contribution to each slice): zero them, V x d elements in float4 groups.
__global__ void zero_slots_kernel(RowScatter sc, long long V, int d) {
  const long long q = d / 4;  // float4 groups per row
  for (long long j = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; j < V * q;
       j += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long v = j / q;
    reinterpret_cast<float4*>(sc.row(v, d))[j - v * q] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// The same sum, stored to n_out copies of the output (the full dH of every rank, other GPUs'
// memory through peer pointers), at an offset of off4 groups of 4 elements.
__global__ void vp_reduce_rows_to_kernel(int R, long long n4, const float4* __restrict__ parts,
                                         __nv_bfloat16* const* __restrict__ outs, int n_out,
                                         long long off4) {
  for (long long j = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; j < n4;
       j += static_cast<long long>(gridDim.x) * blockDim.x) {
    float4 a = __ldcs(parts + j);
    for (int r = 1; r < R; ++r) {
      const float4 b = __ldcs(parts + static_cast<long long>(r) * n4 + j);
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    const uint2 v = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
    for (int k = 0; k < n_out; ++k) reinterpret_cast<uint2*>(outs[k])[off4 + j] = v;
  }
}

}  // namespace lmh
