// lmh_api.cu — the C ABI of include/lmh.h, one translation unit: the shared host code
// (api_common.cuh: checks, plan, launches), the single-device entries below, the
// vocabulary-parallel entries (api_vp.cuh) and the allocation-free entry (api_noalloc.cuh).
// Nothing here allocates device memory or waits for the device (except lmh_read_errors,
// whose job is to).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/lmh.h"
#include "epilogues.cuh"
#include "gemm.cuh"
#include "rowops.cuh"
#include "sparse.cuh"
#include "vp.cuh"
#include "peer.cuh"

using namespace lmh;

#include "api_common.cuh"

// ============================================================================ C ABI

extern "C" size_t lmh_workspace_size(const lmh_shape* shape, int entry) {
  if (!shape_ok(shape) || entry < LMH_ENTRY_LOSS_FWD || entry > LMH_ENTRY_VP_SUPPORT_BWD) return 0;
  if ((entry == LMH_ENTRY_SUPPORT_LOGPROB || entry == LMH_ENTRY_SUPPORT_KL ||
       entry == LMH_ENTRY_VP_SUPPORT_PARTIALS || entry == LMH_ENTRY_VP_SUPPORT_COMBINE ||
       entry == LMH_ENTRY_VP_SUPPORT_BWD) &&
      (shape->K < 1 || shape->K > LMH_MAX_K))
    return 0;
  const bool fused = (entry == LMH_ENTRY_LOSS_FWD || entry == LMH_ENTRY_VP_PARTIALS ||
                      entry == LMH_ENTRY_SUPPORT_KL || entry == LMH_ENTRY_LOSS_FWD_BWD) &&
                     (shape->flags & LMH_F_FUSED_BWD);
  const bool want_acc = !(shape->flags & LMH_F_DW_ACC_GIVEN);
  return make_plan(shape, entry, fused, want_acc).total;
}

extern "C" lmh_status lmh_dh_plan(int64_t rows, int64_t d, int64_t V, int32_t* wide,
                                  int32_t* splits) {
  if (rows < 1 || d <= 0 || (d % 64) != 0 || V < 1 || V > 0x7fffffffLL || !wide || !splits)
    return LMH_ERR_INVALID_ARG;
  const DhPlan p = dh_plan(rows, d, V);
  *wide = p.wide ? 1 : 0;
  *splits = p.splits;
  return LMH_OK;
}

// The CE forward, and with dH / dW its fused backward. weighted: the backward is that of
// L = sum_i w_i l_i for the objective `mode` (loss or log-prob rows), with the row weights and
// target coefficients from bwd_coef_kernel; otherwise of the mean (or summed) loss.
static lmh_status loss_fwd_impl(const lmh_shape* shape, bool weighted, int mode,
                                const float* grad, const lmh_bf16* H, const lmh_bf16* W,
                                const int32_t* labels, float* loss_rows, float* lse,
                                float* logprob, int32_t* argmax, float* loss_mean,
                                int32_t* n_valid, const int32_t* n_valid_given, lmh_bf16* dH,
                                lmh_bf16* dW, float* dW_acc, void* workspace,
                                size_t workspace_bytes, void* stream,
                                const RowScatter* dw_scatter = nullptr) {
  if (!shape_ok(shape)) return LMH_ERR_INVALID_ARG;
  const bool fused = dH || dW || dW_acc || dw_scatter;
  const Plan P = make_plan(shape, weighted ? LMH_ENTRY_LOSS_FWD_BWD : LMH_ENTRY_LOSS_FWD, fused,
                           dW && !dW_acc);
  int dev, sms;
  LMH_TRY(common_checks(shape, H, W, workspace, workspace_bytes, P.total, &dev, &sms));
  if (P.N > 0 && (!labels || !loss_rows || !lse)) return LMH_ERR_INVALID_ARG;
  if (!aligned16(dH) || !aligned16(dW) || !aligned16(dW_acc)) return LMH_ERR_ALIGNMENT;
  if (weighted && (shape->flags & LMH_F_GRAD_SCALAR) && !grad) return LMH_ERR_INVALID_ARG;
  if (dw_scatter && (dW || dW_acc || P.nchunks > 1)) return LMH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{static_cast<uint8_t*>(workspace), static_cast<WsHeader*>(workspace)};
  LMH_TRY(clear_header(ws, st));
  if (P.N == 0 && dw_scatter) {  // this rank's slots of every receive buffer are zero
    const int64_t n4 = P.V * P.d / 4;
    const int64_t blocks = cdiv(n4, 256);
    ProfScope ps(KID_ZERO_SLOTS, st);
    zero_slots_kernel<<<static_cast<unsigned>(blocks < 8192 ? blocks : 8192), 256, 0, st>>>(
        *dw_scatter, P.V, static_cast<int>(P.d));
    LMH_TRY(last_launch());
  }
  if (P.N == 0) return empty_call(P, loss_mean, n_valid, dW, dW_acc, st);
  LMH_TRY(count_labels(P, labels, ws, st));
  const int mean = (shape->flags & LMH_F_MEAN) ? 1 : 0;
  float* alpha = nullptr;
  float* beta = nullptr;
  if (fused && weighted) {
    alpha = ws.at<float>(P.o_alpha);
    beta = ws.at<float>(P.o_beta);
    ProfScope ps(KID_BWD_COEF, st);
    bwd_coef_kernel<<<static_cast<unsigned>(cdiv(P.N, 8)), 256, 0, st>>>(
        mode, P.N, 1, static_cast<int>(P.V), labels, grad, nullptr, nullptr, nullptr, P.temp,
        mean, (shape->flags & LMH_F_GRAD_SCALAR) ? 1 : 0, ws.h, alpha, beta, n_valid_given);
  }
  LMH_TRY(last_launch());
  Targets tg{};
  tg.labels = labels;
  tg.K = 1;
  for (int64_t ci = 0; ci < P.nchunks; ++ci) {
    const int64_t r0 = ci * P.c;
    const int rows = static_cast<int>(P.N - r0 < P.c ? P.N - r0 : P.c);
    if (fused) {
      LMH_TRY((run_stats<kLabel, true>(P, dev, sms, H, W, tg, r0, rows, ws, st)));
    } else {
      LMH_TRY((run_stats<kLabel, false>(P, dev, sms, H, W, tg, r0, rows, ws, st)));
    }
    LMH_TRY(run_finalize(P, 0, r0, rows, labels, lse, loss_rows, logprob, argmax, fused ? 1 : 0,
                         mean, n_valid_given, ws, st, alpha));
    if (fused) {
      __nv_bfloat16* G = ws.at<__nv_bfloat16>(P.o_gbuf);
      const int64_t nv = P.Vp / 8;
      const int64_t bx = cdiv(nv, kGbuildThreads * kGbuildVec);
      dim3 grid(static_cast<unsigned>(bx < 64 ? bx : 64),
                static_cast<unsigned>(rows < 65535 ? rows : 65535));
      {
        ProfScope ps(KID_GBUILD, st);
        gbuild_kernel<<<grid, kGbuildThreads, 0, st>>>(rows, P.Vp, static_cast<int>(P.T),
                                                       ws.at<float>(P.o_ps), G);
      }
      LMH_TRY(last_launch());
      {
        ProfScope ps(KID_FIX_LABELS, st);
        fix_labels_kernel<<<static_cast<unsigned>(cdiv(rows, 256)), 256, 0, st>>>(
            rows, r0, static_cast<int>(P.V), P.Vp, labels, ws.at<float>(P.o_zt), lse, mean,
            n_valid_given, ws.h, P.temp, G, alpha, beta);
      }
      LMH_TRY(last_launch());
      LMH_TRY(run_backward_gemms(P, dev, sms, H, W, r0, rows, static_cast<int>(ci), dH, dW,
                                 dW_acc, ws, st, nullptr, nullptr, dw_scatter));
    }
  }
  if (loss_mean) {
    ProfScope ps(KID_MEAN, st);
    mean_kernel<<<1, 1024, 0, st>>>(loss_rows, P.N, 1, n_valid_given, ws.h, loss_mean);
    LMH_TRY(last_launch());
  }
  if (n_valid &&
      cudaMemcpyAsync(n_valid, &ws.h->n_valid, 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return LMH_ERR_CUDA;
  return LMH_OK;
}

extern "C" lmh_status lmh_loss_fwd(const lmh_shape* shape, const lmh_bf16* H, const lmh_bf16* W,
                                   const int32_t* labels, float* loss_rows, float* lse,
                                   float* logprob, int32_t* argmax, float* loss_mean,
                                   int32_t* n_valid, const int32_t* n_valid_given, lmh_bf16* dH,
                                   lmh_bf16* dW, float* dW_acc, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  return loss_fwd_impl(shape, false, LMH_BWD_CE, nullptr, H, W, labels, loss_rows, lse, logprob,
                       argmax, loss_mean, n_valid, n_valid_given, dH, dW, dW_acc, workspace,
                       workspace_bytes, stream);
}

extern "C" lmh_status lmh_loss_fwd_bwd(const lmh_shape* shape, int mode, const lmh_bf16* H,
                                       const lmh_bf16* W, const int32_t* labels,
                                       const float* grad, float* loss_rows, float* lse,
                                       float* logprob, int32_t* argmax, float* loss_mean,
                                       int32_t* n_valid, const int32_t* n_valid_given,
                                       lmh_bf16* dH, lmh_bf16* dW, float* dW_acc,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  if (mode != LMH_BWD_CE && mode != LMH_BWD_LOGPROB) return LMH_ERR_INVALID_ARG;
  return loss_fwd_impl(shape, true, mode, grad, H, W, labels, loss_rows, lse, logprob, argmax,
                       loss_mean, n_valid, n_valid_given, dH, dW, dW_acc, workspace,
                       workspace_bytes, stream);
}

extern "C" lmh_status lmh_logprob(const lmh_shape* shape, const lmh_bf16* H, const lmh_bf16* W,
                                  const int32_t* labels, float* logprob, float* lse,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (!shape_ok(shape)) return LMH_ERR_INVALID_ARG;
  const Plan P = make_plan(shape, LMH_ENTRY_LOGPROB, false, false);
  int dev, sms;
  LMH_TRY(common_checks(shape, H, W, workspace, workspace_bytes, P.total, &dev, &sms));
  if (P.N > 0 && (!labels || !logprob || !lse)) return LMH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{static_cast<uint8_t*>(workspace), static_cast<WsHeader*>(workspace)};
  LMH_TRY(clear_header(ws, st));
  if (P.N == 0) return LMH_OK;
  LMH_TRY(count_labels(P, labels, ws, st));
  Targets tg{};
  tg.labels = labels;
  tg.K = 1;
  for (int64_t ci = 0; ci < P.nchunks; ++ci) {
    const int64_t r0 = ci * P.c;
    const int rows = static_cast<int>(P.N - r0 < P.c ? P.N - r0 : P.c);
    LMH_TRY((run_stats<kLabel, false>(P, dev, sms, H, W, tg, r0, rows, ws, st)));
    LMH_TRY(run_finalize(P, 1, r0, rows, labels, lse, nullptr, logprob, nullptr, 0, 0, nullptr,
                         ws, st));
  }
  return LMH_OK;
}

static lmh_status support_fwd(const lmh_shape* shape, int entry, const lmh_bf16* H,
                              const lmh_bf16* W, const int32_t* ids, const float* ref,
                              float* lp, float* kl_rows, float* kl_mean, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream) {
  if (!shape_ok(shape) || shape->K < 1 || shape->K > LMH_MAX_K) return LMH_ERR_INVALID_ARG;
  const Plan P = make_plan(shape, entry, false, false);
  int dev, sms;
  LMH_TRY(common_checks(shape, H, W, workspace, workspace_bytes, P.total, &dev, &sms));
  if (P.N > 0 && (!ids || !lse)) return LMH_ERR_INVALID_ARG;
  if (entry == LMH_ENTRY_SUPPORT_LOGPROB && P.N > 0 && !lp) return LMH_ERR_INVALID_ARG;
  if (entry == LMH_ENTRY_SUPPORT_KL && P.N > 0 && (!ref || !kl_rows)) return LMH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{static_cast<uint8_t*>(workspace), static_cast<WsHeader*>(workspace)};
  LMH_TRY(clear_header(ws, st));
  if (P.N == 0) {
    if (kl_mean && cudaMemsetAsync(kl_mean, 0, 4, st) != cudaSuccess) return LMH_ERR_CUDA;
    return LMH_OK;
  }
  LMH_TRY(prep_cands(P, ids, ws, st));
  if (P.renorm) {
    LMH_TRY(support_logits(P, H, W, ws, st));
    ProfScope ps(KID_SUPPORT_LSE, st);
    support_lse_kernel<<<static_cast<unsigned>(cdiv(P.N, 8)), 256, 0, st>>>(
        P.N, static_cast<int>(P.K), ws.at<int32_t>(P.o_nuniq), ws.at<float>(P.o_zt), lse, ws.h);
    LMH_TRY(last_launch());
  } else {
    Targets tg{};
    tg.sorted = ws.at<int32_t>(P.o_sorted);
    tg.nuniq = ws.at<int32_t>(P.o_nuniq);
    tg.K = static_cast<int>(P.K);
    for (int64_t ci = 0; ci < P.nchunks; ++ci) {
      const int64_t r0 = ci * P.c;
      const int rows = static_cast<int>(P.N - r0 < P.c ? P.N - r0 : P.c);
      LMH_TRY((run_stats<kCands, false>(P, dev, sms, H, W, tg, r0, rows, ws, st)));
      LMH_TRY(run_finalize(P, 2, r0, rows, nullptr, lse, nullptr, nullptr, nullptr, 0, 0,
                           nullptr, ws, st));
    }
  }
  {
    ProfScope ps(KID_SUPPORT_OUT, st);
    support_out_kernel<<<static_cast<unsigned>(cdiv(P.N, 8)), 256, 0, st>>>(
      P.N, static_cast<int>(P.K), ws.at<int32_t>(P.o_rank), ws.at<float>(P.o_zt), lse,
      entry == LMH_ENTRY_SUPPORT_KL ? ref : nullptr, lp,
      entry == LMH_ENTRY_SUPPORT_KL ? kl_rows : nullptr);
  }
  LMH_TRY(last_launch());
  if (entry == LMH_ENTRY_SUPPORT_KL && kl_mean) {
    ProfScope ps(KID_MEAN, st);
    mean_kernel<<<1, 1024, 0, st>>>(kl_rows, P.N, 0, nullptr, ws.h, kl_mean);
    LMH_TRY(last_launch());
  }
  return LMH_OK;
}

extern "C" lmh_status lmh_support_logprob(const lmh_shape* shape, const lmh_bf16* H,
                                          const lmh_bf16* W, const int32_t* ids, float* lp,
                                          float* lse, void* workspace, size_t workspace_bytes,
                                          void* stream) {
  return support_fwd(shape, LMH_ENTRY_SUPPORT_LOGPROB, H, W, ids, nullptr, lp, nullptr, nullptr,
                     lse, workspace, workspace_bytes, stream);
}

extern "C" lmh_status lmh_support_kl(const lmh_shape* shape, const lmh_bf16* H,
                                     const lmh_bf16* W, const int32_t* ids,
                                     const float* ref_logp, float* kl_rows, float* kl_mean,
                                     float* lp, float* lse, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  return support_fwd(shape, LMH_ENTRY_SUPPORT_KL, H, W, ids, ref_logp, lp, kl_rows, kl_mean, lse,
                     workspace, workspace_bytes, stream);
}

extern "C" lmh_status lmh_support_fwd_bwd(const lmh_shape* shape, int mode, const lmh_bf16* H,
                                          const lmh_bf16* W, const int32_t* ids,
                                          const float* ref_logp, const float* grad,
                                          float* kl_rows, float* kl_mean, float* lp, float* lse,
                                          lmh_bf16* dH, lmh_bf16* dW, float* dW_acc,
                                          void* workspace, size_t workspace_bytes,
                                          void* stream) {
  if (!shape_ok(shape) || shape->K < 1 || shape->K > LMH_MAX_K) return LMH_ERR_INVALID_ARG;
  if (shape->flags & LMH_F_SUPPORT_RENORM) return LMH_ERR_INVALID_ARG;  // sparse path: two calls
  if (mode != LMH_BWD_SUPPORT_LOGPROB && mode != LMH_BWD_SUPPORT_KL) return LMH_ERR_INVALID_ARG;
  const bool kl = mode == LMH_BWD_SUPPORT_KL;
  const bool grads = dH || dW || dW_acc;
  const Plan P = make_plan(shape, LMH_ENTRY_SUPPORT_KL, grads, dW && !dW_acc);
  int dev, sms;
  LMH_TRY(common_checks(shape, H, W, workspace, workspace_bytes, P.total, &dev, &sms));
  if (P.N > 0 && (!ids || !lse)) return LMH_ERR_INVALID_ARG;
  if (kl && P.N > 0 && (!ref_logp || !kl_rows)) return LMH_ERR_INVALID_ARG;
  if ((shape->flags & LMH_F_GRAD_SCALAR) && !grad) return LMH_ERR_INVALID_ARG;
  if (!aligned16(dH) || !aligned16(dW) || !aligned16(dW_acc)) return LMH_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{static_cast<uint8_t*>(workspace), static_cast<WsHeader*>(workspace)};
  LMH_TRY(clear_header(ws, st));
  if (P.N == 0) return empty_call(P, kl_mean, nullptr, dW, dW_acc, st);
  LMH_TRY(prep_cands(P, ids, ws, st));
  const int K = static_cast<int>(P.K);
  float* alpha = grads ? ws.at<float>(P.o_alpha) : nullptr;
  float* beta = grads ? ws.at<float>(P.o_beta) : nullptr;
  if (grads) {
    // the coefficients depend on the weights (and the reference log-probs) only, not on lse:
    // KL: alpha_i = g_i sum_k exp(r_ik), beta_ic = g_i sum_{k: c_ik = c} exp(r_ik);
    // log-probs: alpha_i = -sum_k g_ik, beta_ic = -sum_{k: c_ik = c} g_ik
    ProfScope ps(KID_BWD_COEF, st);
    bwd_coef_kernel<<<static_cast<unsigned>(cdiv(P.N, 8)), 256, 0, st>>>(
        mode, P.N, K, static_cast<int>(P.V), ids, grad, ref_logp, ws.at<int32_t>(P.o_rank),
        ws.at<int32_t>(P.o_nuniq), P.temp, (shape->flags & LMH_F_MEAN) ? 1 : 0,
        (shape->flags & LMH_F_GRAD_SCALAR) ? 1 : 0, ws.h, alpha, beta);
  }
  LMH_TRY(last_launch());
  Targets tg{};
  tg.sorted = ws.at<int32_t>(P.o_sorted);
  tg.nuniq = ws.at<int32_t>(P.o_nuniq);
  tg.K = K;
  for (int64_t ci = 0; ci < P.nchunks; ++ci) {
    const int64_t r0 = ci * P.c;
    const int rows = static_cast<int>(P.N - r0 < P.c ? P.N - r0 : P.c);
    if (!grads) {
      LMH_TRY((run_stats<kCands, false>(P, dev, sms, H, W, tg, r0, rows, ws, st)));
      LMH_TRY(run_finalize(P, 2, r0, rows, nullptr, lse, nullptr, nullptr, nullptr, 0, 0,
                           nullptr, ws, st));
      continue;
    }
    LMH_TRY((run_stats<kCands, true>(P, dev, sms, H, W, tg, r0, rows, ws, st)));
    LMH_TRY(run_finalize(P, 2, r0, rows, nullptr, lse, nullptr, nullptr, nullptr, 1, 0, nullptr,
                         ws, st, alpha));
    __nv_bfloat16* G = ws.at<__nv_bfloat16>(P.o_gbuf);
    {
      const int64_t nv = P.Vp / 8;
      const int64_t bx = cdiv(nv, kGbuildThreads * kGbuildVec);
      dim3 grid(static_cast<unsigned>(bx < 64 ? bx : 64),
                static_cast<unsigned>(rows < 65535 ? rows : 65535));
      ProfScope ps(KID_GBUILD, st);
      gbuild_kernel<<<grid, kGbuildThreads, 0, st>>>(rows, P.Vp, static_cast<int>(P.T),
                                                     ws.at<float>(P.o_ps), G);
    }
    LMH_TRY(last_launch());
    {
      ProfScope ps(KID_FIX_CANDS, st);
      fix_cands_kernel<<<static_cast<unsigned>(cdiv(rows, 8)), 256, 0, st>>>(
          rows, r0, K, P.Vp, ws.at<int32_t>(P.o_sorted), ws.at<int32_t>(P.o_nuniq),
          ws.at<float>(P.o_zt), lse, alpha, beta, G);
    }
    LMH_TRY(last_launch());
    LMH_TRY(run_backward_gemms(P, dev, sms, H, W, r0, rows, static_cast<int>(ci), dH, dW, dW_acc,
                               ws, st));
  }
  {
    ProfScope ps(KID_SUPPORT_OUT, st);
    support_out_kernel<<<static_cast<unsigned>(cdiv(P.N, 8)), 256, 0, st>>>(
        P.N, K, ws.at<int32_t>(P.o_rank), ws.at<float>(P.o_zt), lse, kl ? ref_logp : nullptr,
        lp, kl ? kl_rows : nullptr);
  }
  LMH_TRY(last_launch());
  if (kl && kl_mean) {
    ProfScope ps(KID_MEAN, st);
    mean_kernel<<<1, 1024, 0, st>>>(kl_rows, P.N, 0, nullptr, ws.h, kl_mean);
    LMH_TRY(last_launch());
  }
  return LMH_OK;
}

extern "C" lmh_status lmh_support_kl_fwd_bwd(const lmh_shape* shape, const lmh_bf16* H,
                                             const lmh_bf16* W, const int32_t* ids,
                                             const float* ref_logp, float* kl_rows,
                                             float* kl_mean, float* lp, float* lse,
                                             lmh_bf16* dH, lmh_bf16* dW, float* dW_acc,
                                             void* workspace, size_t workspace_bytes,
                                             void* stream) {
  if (shape && (shape->flags & LMH_F_GRAD_SCALAR)) return LMH_ERR_INVALID_ARG;  // no grad here
  return lmh_support_fwd_bwd(shape, LMH_BWD_SUPPORT_KL, H, W, ids, ref_logp, nullptr, kl_rows,
                             kl_mean, lp, lse, dH, dW, dW_acc, workspace, workspace_bytes,
                             stream);
}

extern "C" lmh_status lmh_loss_bwd(const lmh_shape* shape, int mode, const lmh_bf16* H,
                                   const lmh_bf16* W, const int32_t* targets, const float* lse,
                                   const float* grad, const float* ref_logp, lmh_bf16* dH,
                                   lmh_bf16* dW, float* dW_acc, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  if (!shape_ok(shape) || mode < LMH_BWD_CE || mode > LMH_BWD_SUPPORT_KL)
    return LMH_ERR_INVALID_ARG;
  const bool cands = mode >= LMH_BWD_SUPPORT_LOGPROB;
  if (cands && (shape->K < 1 || shape->K > LMH_MAX_K)) return LMH_ERR_INVALID_ARG;
  lmh_shape sh = *shape;  // the renormalised path exists for the support objectives only
  if (!cands) sh.flags &= ~LMH_F_SUPPORT_RENORM;
  const Plan P = make_plan(&sh, LMH_ENTRY_LOSS_BWD, true, dW && !dW_acc);
  int dev, sms;
  LMH_TRY(common_checks(shape, H, W, workspace, workspace_bytes, P.total, &dev, &sms));
  if (P.N > 0 && (!targets || !lse)) return LMH_ERR_INVALID_ARG;
  if (mode == LMH_BWD_SUPPORT_KL && P.N > 0 && !ref_logp) return LMH_ERR_INVALID_ARG;
  if ((shape->flags & LMH_F_GRAD_SCALAR) && !grad) return LMH_ERR_INVALID_ARG;
  if (!aligned16(dH) || !aligned16(dW) || !aligned16(dW_acc)) return LMH_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{static_cast<uint8_t*>(workspace), static_cast<WsHeader*>(workspace)};
  LMH_TRY(clear_header(ws, st));
  if (P.N == 0) return empty_call(P, nullptr, nullptr, dW, dW_acc, st);
  if (!dH && !dW && !dW_acc) return LMH_OK;
  Targets tg{};
  if (cands) {
    LMH_TRY(prep_cands(P, targets, ws, st));
    tg.sorted = ws.at<int32_t>(P.o_sorted);
    tg.nuniq = ws.at<int32_t>(P.o_nuniq);
    tg.K = static_cast<int>(P.K);
  } else {
    LMH_TRY(count_labels(P, targets, ws, st));
    tg.labels = targets;
    tg.K = 1;
  }
  float* alpha = ws.at<float>(P.o_alpha);
  float* beta = ws.at<float>(P.o_beta);
  {
    ProfScope ps(KID_BWD_COEF, st);
    bwd_coef_kernel<<<static_cast<unsigned>(cdiv(P.N, 8)), 256, 0, st>>>(
      mode, P.N, cands ? static_cast<int>(P.K) : 1, static_cast<int>(P.V), targets, grad,
      ref_logp, cands ? ws.at<int32_t>(P.o_rank) : nullptr,
      cands ? ws.at<int32_t>(P.o_nuniq) : nullptr, P.temp,
      (shape->flags & LMH_F_MEAN) ? 1 : 0, (shape->flags & LMH_F_GRAD_SCALAR) ? 1 : 0, ws.h,
      alpha, beta);
  }
  LMH_TRY(last_launch());
  if (P.renorm) return sparse_backward(P, H, W, lse, dH, dW, dW_acc, ws, st);
  for (int64_t ci = 0; ci < P.nchunks; ++ci) {
    const int64_t r0 = ci * P.c;
    const int rows = static_cast<int>(P.N - r0 < P.c ? P.N - r0 : P.c);
    CUtensorMap ta, tb, tc;
    if (!tmap_2d(&ta, H + r0 * P.d, P.d, rows, P.d, BM) || !tmap_2d(&tb, W, P.d, P.V, P.d, BNH) ||
        !tmap_out(&tc, ws.at<__nv_bfloat16>(P.o_gbuf), P.Vp, rows, P.Vp))
      return LMH_ERR_CUDA;
    if (cands) {
      EpiGrad<kCands>::Params ep{rows, r0, static_cast<int>(P.V), P.Vp, tg, lse, alpha, beta,
                                 P.temp};
      LMH_TRY(launch_gemm<EpiGrad<kCands>>(dev, sms, ta, tb, tc, rows, P.V, P.d, kOrderLogits,
                                           &ws.h->err, ep, st));
    } else {
      EpiGrad<kLabel>::Params ep{rows, r0, static_cast<int>(P.V), P.Vp, tg, lse, alpha, beta,
                                 P.temp};
      LMH_TRY(launch_gemm<EpiGrad<kLabel>>(dev, sms, ta, tb, tc, rows, P.V, P.d, kOrderLogits,
                                           &ws.h->err, ep, st));
    }
    LMH_TRY(run_backward_gemms(P, dev, sms, H, W, r0, rows, static_cast<int>(ci), dH, dW, dW_acc,
                               ws, st));
  }
  return LMH_OK;
}

#include "api_vp.cuh"

extern "C" lmh_status lmh_count_valid(int64_t N, int64_t V, const int32_t* labels,
                                      int32_t* n_valid, void* stream) {
  if (N < 0 || V <= 0 || V > 0x7fffffffLL || !n_valid) return LMH_ERR_INVALID_ARG;
  if (N > 0 && !labels) return LMH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(labels) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(n_valid) & 3u) != 0)
    return LMH_ERR_ALIGNMENT;
  int dev, sms;
  LMH_TRY(current_device(&dev, &sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(n_valid, 0, 4, st) != cudaSuccess) return LMH_ERR_CUDA;
  if (N == 0) return LMH_OK;
  const int64_t blocks = cdiv(N, 256);
  ProfScope ps(KID_COUNT_VALID, st);
  count_valid_kernel<<<static_cast<unsigned>(blocks < 1024 ? blocks : 1024), 256, 0, st>>>(
      labels, N, static_cast<int>(V), n_valid);
  return last_launch();
}

extern "C" lmh_status lmh_reduce_ranks_f32(int R, int64_t n, const float* parts, float* out,
                                           void* stream) {
  if (R < 1 || n < 0) return LMH_ERR_INVALID_ARG;
  if (n == 0) return LMH_OK;
  if (!parts || !out) return LMH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(parts) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(out) & 3u) != 0)
    return LMH_ERR_ALIGNMENT;
  int dev, sms;
  LMH_TRY(current_device(&dev, &sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t blocks = cdiv(n, 256);
  ProfScope ps(KID_REDUCE_RANKS, st);
  reduce_ranks_kernel<<<static_cast<unsigned>(blocks < 8192 ? blocks : 8192), 256, 0, st>>>(
      R, n, parts, out);
  return last_launch();
}

extern "C" lmh_status lmh_scale_bf16(lmh_bf16* x, int64_t n, const float* g, void* stream) {
  if (n < 0 || (n % 4) != 0) return LMH_ERR_INVALID_ARG;
  if (n == 0) return LMH_OK;
  if (!x || !g) return LMH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 7u) != 0 || (reinterpret_cast<uintptr_t>(g) & 3u) != 0)
    return LMH_ERR_ALIGNMENT;
  int dev, sms;
  LMH_TRY(current_device(&dev, &sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t blocks = cdiv(n / 4, 256);
  ProfScope ps(KID_SCALE, st);
  scale_bf16_kernel<<<static_cast<unsigned>(blocks < 8192 ? blocks : 8192), 256, 0, st>>>(
      n / 4, g, reinterpret_cast<__nv_bfloat16*>(x));
  return last_launch();
}

extern "C" lmh_status lmh_read_errors(const void* workspace, uint32_t* errors, void* stream) {
  if (!workspace || !errors) return LMH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return LMH_ERR_CUDA;
  if (cudaMemcpy(errors, workspace, 4, cudaMemcpyDeviceToHost) != cudaSuccess)
    return LMH_ERR_CUDA;
  return LMH_OK;
}

extern "C" lmh_status lmh_selftest_wait_timeout(void* workspace, uint32_t timeout_ms,
                                                void* stream) {
  if (!workspace || timeout_ms < 1 || timeout_ms > 5000) return LMH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return LMH_ERR_ALIGNMENT;
  int dev, sms;
  LMH_TRY(current_device(&dev, &sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{static_cast<uint8_t*>(workspace), static_cast<WsHeader*>(workspace)};
  LMH_TRY(clear_header(ws, st));
  wait_selftest_kernel<<<1, 32, 0, st>>>(&ws.h->err, uint64_t(timeout_ms) * 1000000ull);
  return last_launch();
}

extern "C" lmh_status lmh_profile_enable(int on) {
  g_prof_on.store(on != 0);
  return LMH_OK;
}

extern "C" int lmh_profile_read(int max_records, int32_t* kernel_ids, float* ms) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  int n = 0;
  for (const ProfRec& r : g_prof_recs) {
    if (n < max_records && kernel_ids && ms) {
      float t = -1.f;
      if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
        t = -1.f;
      kernel_ids[n] = r.id;
      ms[n] = t;
      ++n;
    }
    g_prof_pool.push_back(r.a);
    g_prof_pool.push_back(r.b);
  }
  g_prof_recs.clear();
  return n;
}

extern "C" const char* lmh_kernel_name(int kernel_id) {
  return (kernel_id >= 0 && kernel_id < KID_COUNT) ? kKernelNames[kernel_id] : "";
}

#include "api_noalloc.cuh"
