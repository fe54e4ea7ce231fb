// api_vp.cuh — the C ABI's vocabulary-parallel entries (lmh_vp_*). Part of the one
// translation unit lmh_api.cu (included there once, after the shared host code).
#pragma once

// ============================================================================ vocab-parallel
namespace {

// The receive buffers of a row scatter: R ranks, this one among them, N rows split over R.
lmh_status vp_dest_ok(const lmh_vp_dest* dest, const float* dH_part, int64_t N,
                      RowScatter* sc) {
  if (!dest) return LMH_OK;
  if (dH_part || !dest->recv || dest->R < 1 || dest->rank < 0 || dest->rank >= dest->R)
    return LMH_ERR_INVALID_ARG;
  sc->dest = dest->recv;
  sc->R = dest->R;
  sc->rank = dest->rank;
  sc->N = N;
  return LMH_OK;
}

lmh_status vp_args_ok(const lmh_shape* shard, int64_t v0, int64_t V_total) {
  if (!shape_ok(shard) || v0 < 0 || V_total <= 0 || V_total > 0x7fffffffLL ||
      v0 + shard->V > V_total)
    return LMH_ERR_INVALID_ARG;
  return LMH_OK;
}

lmh_status vp_local_labels(const Plan& P, const int32_t* labels, int64_t v0, const Ws& ws,
                           cudaStream_t st) {
  const int64_t blocks = cdiv(P.N, 256);
  ProfScope ps(KID_VP_LABELS, st);
  vp_local_labels_kernel<<<static_cast<unsigned>(blocks < 1024 ? blocks : 1024), 256, 0, st>>>(
      P.N, labels, v0, P.V, ws.at<int32_t>(P.o_lloc));
  return last_launch();
}

// Valid rows of the full vocabulary (0 <= y < V_total) into the header; flags y >= V_total.
lmh_status count_labels_total(const Plan& P, const int32_t* labels, int64_t V_total,
                              const Ws& ws, cudaStream_t st) {
  const int64_t blocks = cdiv(P.N, 256);
  ProfScope ps(KID_COUNT_LABELS, st);
  count_labels_kernel<<<static_cast<unsigned>(blocks < 1024 ? blocks : 1024), 256, 0, st>>>(
      labels, P.N, static_cast<int>(V_total), ws.h);
  return last_launch();
}

}  // namespace

extern "C" lmh_status lmh_vp_partials(const lmh_shape* shard, int64_t v0, int64_t V_total,
                                      const lmh_bf16* H, const lmh_bf16* W_shard,
                                      const int32_t* labels, float* records, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  LMH_TRY(vp_args_ok(shard, v0, V_total));
  const bool fused = (shard->flags & LMH_F_FUSED_BWD) != 0;
  const Plan P = make_plan(shard, LMH_ENTRY_VP_PARTIALS, fused, false);
  int dev, sms;
  LMH_TRY(common_checks(shard, H, W_shard, workspace, workspace_bytes, P.total, &dev, &sms));
  if (P.N > 0 && (!labels || !records)) return LMH_ERR_INVALID_ARG;
  if (fused && P.nchunks > 1) return LMH_ERR_INVALID_ARG;  // p~ of every row is kept
  if (!aligned16(records)) return LMH_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{static_cast<uint8_t*>(workspace), static_cast<WsHeader*>(workspace)};
  LMH_TRY(clear_header(ws, st));
  if (P.N == 0) return LMH_OK;
  LMH_TRY(vp_local_labels(P, labels, v0, ws, st));
  Targets tg{};
  tg.labels = ws.at<int32_t>(P.o_lloc);
  tg.K = 1;
  for (int64_t ci = 0; ci < P.nchunks; ++ci) {
    const int64_t r0 = ci * P.c;
    const int rows = static_cast<int>(P.N - r0 < P.c ? P.N - r0 : P.c);
    if (fused) {
      LMH_TRY((run_stats<kLabel, true>(P, dev, sms, H, W_shard, tg, r0, rows, ws, st)));
    } else {
      LMH_TRY((run_stats<kLabel, false>(P, dev, sms, H, W_shard, tg, r0, rows, ws, st)));
    }
    ProfScope ps(KID_VP_FINALIZE, st);
    vp_finalize_kernel<<<static_cast<unsigned>(cdiv(rows, 8)), 256, 0, st>>>(
        rows, r0, static_cast<int>(P.T), v0, ws.at<float>(P.o_pm), ws.at<float>(P.o_ps),
        ws.at<int32_t>(P.o_pi), ws.at<int32_t>(P.o_lloc), ws.at<float>(P.o_zt), P.temp, ws.h,
        reinterpret_cast<float4*>(records));
    LMH_TRY(last_launch());
  }
  return LMH_OK;
}

extern "C" lmh_status lmh_vp_combine(const lmh_shape* shape, int R, const float* records,
                                     const int32_t* labels, float* loss_rows, float* lse,
                                     float* logprob, int32_t* argmax, float* loss_mean,
                                     int32_t* n_valid, const int32_t* n_valid_given,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  if (!shape_ok(shape) || R < 1) return LMH_ERR_INVALID_ARG;
  const Plan P = make_plan(shape, LMH_ENTRY_VP_COMBINE, false, false);
  if (!workspace) return LMH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return LMH_ERR_ALIGNMENT;
  if (workspace_bytes < P.total) return LMH_ERR_WORKSPACE_TOO_SMALL;
  if (P.N > 0 && (!records || !labels || !loss_rows || !lse)) return LMH_ERR_INVALID_ARG;
  if (!aligned16(records)) return LMH_ERR_ALIGNMENT;
  int dev, sms;
  LMH_TRY(current_device(&dev, &sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{static_cast<uint8_t*>(workspace), static_cast<WsHeader*>(workspace)};
  LMH_TRY(clear_header(ws, st));
  if (P.N == 0) return empty_call(P, loss_mean, n_valid, nullptr, nullptr, st);
  LMH_TRY(count_labels_total(P, labels, P.V, ws, st));
  {
    const int64_t blocks = cdiv(P.N, 256);
    ProfScope ps(KID_VP_COMBINE, st);
    vp_combine_kernel<<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), 256, 0, st>>>(
        P.N, R, static_cast<int>(P.V), reinterpret_cast<const float4*>(records), labels, lse,
        loss_rows, logprob, argmax, ws.h);
  }
  LMH_TRY(last_launch());
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

extern "C" lmh_status lmh_vp_loss_bwd(const lmh_shape* shard, int mode, int64_t v0,
                                      int64_t V_total, const lmh_bf16* H,
                                      const lmh_bf16* W_shard, const int32_t* labels,
                                      const float* lse, const float* grad, float* dH_part,
                                      lmh_bf16* dW_shard, float* dW_acc_shard,
                                      const lmh_vp_dest* dest, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  LMH_TRY(vp_args_ok(shard, v0, V_total));
  RowScatter sc;
  LMH_TRY(vp_dest_ok(dest, dH_part, shard->N, &sc));
  if (mode != LMH_BWD_CE && mode != LMH_BWD_LOGPROB) return LMH_ERR_INVALID_ARG;
  lmh_shape sh = *shard;
  sh.flags &= ~LMH_F_SUPPORT_RENORM;
  sh.K = 1;
  const Plan P = make_plan(&sh, LMH_ENTRY_VP_BWD, true, dW_shard && !dW_acc_shard);
  int dev, sms;
  LMH_TRY(common_checks(&sh, H, W_shard, workspace, workspace_bytes, P.total, &dev, &sms));
  if (P.N > 0 && (!labels || !lse)) return LMH_ERR_INVALID_ARG;
  if ((sh.flags & LMH_F_GRAD_SCALAR) && !grad) return LMH_ERR_INVALID_ARG;
  if (!aligned16(dH_part) || !aligned16(dW_shard) || !aligned16(dW_acc_shard))
    return LMH_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{static_cast<uint8_t*>(workspace), static_cast<WsHeader*>(workspace)};
  LMH_TRY(clear_header(ws, st));
  if (P.N == 0) return empty_call(P, nullptr, nullptr, dW_shard, dW_acc_shard, st);
  if (!dH_part && !dest && !dW_shard && !dW_acc_shard) return LMH_OK;
  LMH_TRY(count_labels_total(P, labels, V_total, ws, st));
  LMH_TRY(vp_local_labels(P, labels, v0, ws, st));
  float* alpha = ws.at<float>(P.o_alpha);
  float* beta = ws.at<float>(P.o_beta);
  {
    // the row coefficients see the global label (valid rows over the full vocabulary); the
    // one-hot term lands in this shard only if the label is one of its columns
    ProfScope ps(KID_BWD_COEF, st);
    bwd_coef_kernel<<<static_cast<unsigned>(cdiv(P.N, 8)), 256, 0, st>>>(
        mode, P.N, 1, static_cast<int>(V_total), labels, grad, nullptr, nullptr, nullptr, P.temp,
        (sh.flags & LMH_F_MEAN) ? 1 : 0, (sh.flags & LMH_F_GRAD_SCALAR) ? 1 : 0, ws.h, alpha,
        beta);
  }
  LMH_TRY(last_launch());
  Targets tg{};
  tg.labels = ws.at<int32_t>(P.o_lloc);
  tg.K = 1;
  for (int64_t ci = 0; ci < P.nchunks; ++ci) {
    const int64_t r0 = ci * P.c;
    const int rows = static_cast<int>(P.N - r0 < P.c ? P.N - r0 : P.c);
    CUtensorMap ta, tb, tc;
    if (!tmap_2d(&ta, H + r0 * P.d, P.d, rows, P.d, BM) ||
        !tmap_2d(&tb, W_shard, P.d, P.V, P.d, BNH) ||
        !tmap_out(&tc, ws.at<__nv_bfloat16>(P.o_gbuf), P.Vp, rows, P.Vp))
      return LMH_ERR_CUDA;
    EpiGrad<kLabel>::Params ep{rows, r0, static_cast<int>(P.V), P.Vp, tg, lse, alpha, beta,
                               P.temp};
    LMH_TRY(launch_gemm<EpiGrad<kLabel>>(dev, sms, ta, tb, tc, rows, P.V, P.d, kOrderLogits,
                                         &ws.h->err, ep, st));
    LMH_TRY(run_backward_gemms(P, dev, sms, H, W_shard, r0, rows, static_cast<int>(ci), nullptr,
                               dW_shard, dW_acc_shard, ws, st, dH_part,
                               dest ? &sc : nullptr));
  }
  return LMH_OK;
}

extern "C" lmh_status lmh_vp_fused_bwd(const lmh_shape* shard, int64_t v0, int64_t V_total,
                                       const lmh_bf16* H, const lmh_bf16* W_shard,
                                       const int32_t* labels, const float* lse,
                                       const int32_t* n_valid_given, float* dH_part,
                                       lmh_bf16* dW_shard, float* dW_acc_shard,
                                       const lmh_vp_dest* dest, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  LMH_TRY(vp_args_ok(shard, v0, V_total));
  if (!(shard->flags & LMH_F_FUSED_BWD)) return LMH_ERR_INVALID_ARG;
  RowScatter sc;
  LMH_TRY(vp_dest_ok(dest, dH_part, shard->N, &sc));
  const Plan P = make_plan(shard, LMH_ENTRY_VP_PARTIALS, true, false);
  int dev, sms;
  LMH_TRY(common_checks(shard, H, W_shard, workspace, workspace_bytes, P.total, &dev, &sms));
  if (P.nchunks > 1) return LMH_ERR_INVALID_ARG;
  if (P.N > 0 && (!labels || !lse)) return LMH_ERR_INVALID_ARG;
  if (!aligned16(dH_part) || !aligned16(dW_shard) || !aligned16(dW_acc_shard))
    return LMH_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{static_cast<uint8_t*>(workspace), static_cast<WsHeader*>(workspace)};
  LMH_TRY(clear_header(ws, st));
  if (P.N == 0) return empty_call(P, nullptr, nullptr, dW_shard, dW_acc_shard, st);
  if (!dH_part && !dest && !dW_shard && !dW_acc_shard) return LMH_OK;
  const int mean = (shard->flags & LMH_F_MEAN) ? 1 : 0;
  const int rows = static_cast<int>(P.N);
  LMH_TRY(count_labels_total(P, labels, V_total, ws, st));
  LMH_TRY(vp_local_labels(P, labels, v0, ws, st));
  {
    // s_t of each (row, tile) becomes alpha_i exp(m_t - lse_i) with the combined lse
    ProfScope ps(KID_VP_SCALE, st);
    vp_scale_kernel<<<static_cast<unsigned>(cdiv(rows, 8)), 256, 0, st>>>(
        rows, static_cast<int>(P.T), static_cast<int>(V_total), labels, lse,
        ws.at<float>(P.o_pm), mean, n_valid_given, ws.h, P.temp, ws.at<float>(P.o_ps));
  }
  LMH_TRY(last_launch());
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
    // the one-hot term, in the shard that holds the label's column
    ProfScope ps(KID_FIX_LABELS, st);
    fix_labels_kernel<<<static_cast<unsigned>(cdiv(rows, 256)), 256, 0, st>>>(
        rows, 0, static_cast<int>(P.V), P.Vp, ws.at<int32_t>(P.o_lloc), ws.at<float>(P.o_zt),
        lse, mean, n_valid_given, ws.h, P.temp, G);
  }
  LMH_TRY(last_launch());
  return run_backward_gemms(P, dev, sms, H, W_shard, 0, rows, 0, nullptr, dW_shard,
                            dW_acc_shard, ws, st, dH_part, dest ? &sc : nullptr);
}

// ---------------------------------------------------------------- support entries
namespace {

// Shard-local candidate ids: c - v0 inside [v0, v0 + Vr), else -1 (padding here).
lmh_status vp_local_ids(const Plan& P, const int32_t* ids, int64_t v0, const Ws& ws,
                        cudaStream_t st) {
  const int64_t n = P.N * P.K;
  const int64_t blocks = cdiv(n, 256);
  ProfScope ps(KID_VP_LABELS, st);
  vp_local_labels_kernel<<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), 256, 0, st>>>(
      n, ids, v0, P.V, ws.at<int32_t>(P.o_lloc));
  return last_launch();
}

bool vp_support_shape_ok(const lmh_shape* s) {
  return s->K >= 1 && s->K <= LMH_MAX_K && !(s->flags & LMH_F_SUPPORT_RENORM);
}

}  // namespace

extern "C" lmh_status lmh_vp_support_partials(const lmh_shape* shard, int64_t v0,
                                              int64_t V_total, const lmh_bf16* H,
                                              const lmh_bf16* W_shard, const int32_t* ids,
                                              float* records, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  LMH_TRY(vp_args_ok(shard, v0, V_total));
  if (!vp_support_shape_ok(shard)) return LMH_ERR_INVALID_ARG;
  const Plan P = make_plan(shard, LMH_ENTRY_VP_SUPPORT_PARTIALS, false, false);
  int dev, sms;
  LMH_TRY(common_checks(shard, H, W_shard, workspace, workspace_bytes, P.total, &dev, &sms));
  if (P.N > 0 && (!ids || !records)) return LMH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{static_cast<uint8_t*>(workspace), static_cast<WsHeader*>(workspace)};
  LMH_TRY(clear_header(ws, st));
  if (P.N == 0) return LMH_OK;
  LMH_TRY(vp_local_ids(P, ids, v0, ws, st));
  LMH_TRY(prep_cands(P, ws.at<int32_t>(P.o_lloc), ws, st));
  Targets tg{};
  tg.sorted = ws.at<int32_t>(P.o_sorted);
  tg.nuniq = ws.at<int32_t>(P.o_nuniq);
  tg.K = static_cast<int>(P.K);
  for (int64_t ci = 0; ci < P.nchunks; ++ci) {
    const int64_t r0 = ci * P.c;
    const int rows = static_cast<int>(P.N - r0 < P.c ? P.N - r0 : P.c);
    LMH_TRY((run_stats<kCands, false>(P, dev, sms, H, W_shard, tg, r0, rows, ws, st)));
    ProfScope ps(KID_VP_FINALIZE, st);
    vp_support_finalize_kernel<<<static_cast<unsigned>(cdiv(rows, 8)), 256, 0, st>>>(
        rows, r0, static_cast<int>(P.T), static_cast<int>(P.K), ws.at<float>(P.o_pm),
        ws.at<float>(P.o_ps), ws.at<int32_t>(P.o_rank), ws.at<float>(P.o_zt), P.temp, ws.h,
        records);
    LMH_TRY(last_launch());
  }
  return LMH_OK;
}

extern "C" lmh_status lmh_vp_support_combine(const lmh_shape* shape, int R,
                                             const float* records, const int32_t* ids,
                                             const float* ref_logp, float* lp, float* lse,
                                             float* kl_rows, float* kl_mean, void* workspace,
                                             size_t workspace_bytes, void* stream) {
  if (!shape_ok(shape) || R < 1 || shape->K < 1 || shape->K > LMH_MAX_K)
    return LMH_ERR_INVALID_ARG;
  const Plan P = make_plan(shape, LMH_ENTRY_VP_SUPPORT_COMBINE, false, false);
  if (!workspace) return LMH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return LMH_ERR_ALIGNMENT;
  if (workspace_bytes < P.total) return LMH_ERR_WORKSPACE_TOO_SMALL;
  if (P.N > 0 && (!records || !ids || !lse)) return LMH_ERR_INVALID_ARG;
  if ((kl_rows || kl_mean) && !ref_logp) return LMH_ERR_INVALID_ARG;
  if (kl_mean && !kl_rows) return LMH_ERR_INVALID_ARG;
  int dev, sms;
  LMH_TRY(current_device(&dev, &sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{static_cast<uint8_t*>(workspace), static_cast<WsHeader*>(workspace)};
  LMH_TRY(clear_header(ws, st));
  if (P.N == 0) return empty_call(P, kl_mean, nullptr, nullptr, nullptr, st);
  {
    ProfScope ps(KID_VP_COMBINE, st);
    vp_support_combine_kernel<<<static_cast<unsigned>(cdiv(P.N, 8)), 256, 0, st>>>(
        P.N, R, static_cast<int>(shape->K), static_cast<int>(P.V), records, ids,
        kl_rows ? ref_logp : nullptr, lp, lse, kl_rows, ws.h);
  }
  LMH_TRY(last_launch());
  if (kl_mean) {
    ProfScope ps(KID_MEAN, st);
    mean_kernel<<<1, 1024, 0, st>>>(kl_rows, P.N, 0, nullptr, ws.h, kl_mean);
    LMH_TRY(last_launch());
  }
  return LMH_OK;
}

extern "C" lmh_status lmh_vp_support_bwd(const lmh_shape* shard, int mode, int64_t v0,
                                         int64_t V_total, const lmh_bf16* H,
                                         const lmh_bf16* W_shard, const int32_t* ids,
                                         const float* lse, const float* grad,
                                         const float* ref_logp, float* dH_part,
                                         lmh_bf16* dW_shard, float* dW_acc_shard,
                                         const lmh_vp_dest* dest, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  LMH_TRY(vp_args_ok(shard, v0, V_total));
  if (!vp_support_shape_ok(shard)) return LMH_ERR_INVALID_ARG;
  if (mode != LMH_BWD_SUPPORT_LOGPROB && mode != LMH_BWD_SUPPORT_KL) return LMH_ERR_INVALID_ARG;
  RowScatter sc;
  LMH_TRY(vp_dest_ok(dest, dH_part, shard->N, &sc));
  const Plan P = make_plan(shard, LMH_ENTRY_VP_SUPPORT_BWD, true, dW_shard && !dW_acc_shard);
  int dev, sms;
  LMH_TRY(common_checks(shard, H, W_shard, workspace, workspace_bytes, P.total, &dev, &sms));
  if (P.N > 0 && (!ids || !lse)) return LMH_ERR_INVALID_ARG;
  if (mode == LMH_BWD_SUPPORT_KL && P.N > 0 && !ref_logp) return LMH_ERR_INVALID_ARG;
  if ((shard->flags & LMH_F_GRAD_SCALAR) && !grad) return LMH_ERR_INVALID_ARG;
  if (!aligned16(dH_part) || !aligned16(dW_shard) || !aligned16(dW_acc_shard))
    return LMH_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{static_cast<uint8_t*>(workspace), static_cast<WsHeader*>(workspace)};
  LMH_TRY(clear_header(ws, st));
  if (P.N == 0) return empty_call(P, nullptr, nullptr, dW_shard, dW_acc_shard, st);
  if (!dH_part && !dest && !dW_shard && !dW_acc_shard) return LMH_OK;
  LMH_TRY(vp_local_ids(P, ids, v0, ws, st));
  LMH_TRY(prep_cands(P, ws.at<int32_t>(P.o_lloc), ws, st));
  const int K = static_cast<int>(P.K);
  float* alpha = ws.at<float>(P.o_alpha);
  float* beta = ws.at<float>(P.o_beta);
  {
    // beta over this shard's candidates; alpha over every valid candidate of the vocabulary
    ProfScope ps(KID_BWD_COEF, st);
    bwd_coef_kernel<<<static_cast<unsigned>(cdiv(P.N, 8)), 256, 0, st>>>(
        mode, P.N, K, static_cast<int>(P.V), ws.at<int32_t>(P.o_lloc), grad, ref_logp,
        ws.at<int32_t>(P.o_rank), ws.at<int32_t>(P.o_nuniq), P.temp,
        (shard->flags & LMH_F_MEAN) ? 1 : 0, (shard->flags & LMH_F_GRAD_SCALAR) ? 1 : 0, ws.h,
        alpha, beta, nullptr, ids, static_cast<int>(V_total));
  }
  LMH_TRY(last_launch());
  Targets tg{};
  tg.sorted = ws.at<int32_t>(P.o_sorted);
  tg.nuniq = ws.at<int32_t>(P.o_nuniq);
  tg.K = K;
  for (int64_t ci = 0; ci < P.nchunks; ++ci) {
    const int64_t r0 = ci * P.c;
    const int rows = static_cast<int>(P.N - r0 < P.c ? P.N - r0 : P.c);
    CUtensorMap ta, tb, tc;
    if (!tmap_2d(&ta, H + r0 * P.d, P.d, rows, P.d, BM) ||
        !tmap_2d(&tb, W_shard, P.d, P.V, P.d, BNH) ||
        !tmap_out(&tc, ws.at<__nv_bfloat16>(P.o_gbuf), P.Vp, rows, P.Vp))
      return LMH_ERR_CUDA;
    EpiGrad<kCands>::Params ep{rows, r0, static_cast<int>(P.V), P.Vp, tg, lse, alpha, beta,
                               P.temp};
    LMH_TRY(launch_gemm<EpiGrad<kCands>>(dev, sms, ta, tb, tc, rows, P.V, P.d, kOrderLogits,
                                         &ws.h->err, ep, st));
    LMH_TRY(run_backward_gemms(P, dev, sms, H, W_shard, r0, rows, static_cast<int>(ci), nullptr,
                               dW_shard, dW_acc_shard, ws, st, dH_part,
                               dest ? &sc : nullptr));
  }
  return LMH_OK;
}

// Row data-parallel one-pass step whose dW GEMM stores each fp32 row of the rank's dW into the
// receive buffer of the rank that reduces that vocabulary row (the row scatter over V).
extern "C" lmh_status lmh_dp_loss_fwd_bwd(const lmh_shape* shape, int mode, const lmh_bf16* H,
                                          const lmh_bf16* W, const int32_t* labels,
                                          const float* grad, float* loss_rows, float* lse,
                                          float* logprob, int32_t* argmax, float* loss_mean,
                                          const int32_t* n_valid_given, lmh_bf16* dH,
                                          const lmh_vp_dest* dW_dest, void* workspace,
                                          size_t workspace_bytes, void* stream) {
  if (!shape_ok(shape) || !dW_dest) return LMH_ERR_INVALID_ARG;
  if (mode != LMH_BWD_CE && mode != LMH_BWD_LOGPROB) return LMH_ERR_INVALID_ARG;
  RowScatter sc;
  LMH_TRY(vp_dest_ok(dW_dest, nullptr, shape->V, &sc));
  return loss_fwd_impl(shape, true, mode, grad, H, W, labels, loss_rows, lse, logprob, argmax,
                       loss_mean, nullptr, n_valid_given, dH, nullptr, nullptr, workspace,
                       workspace_bytes, stream, &sc);
}

extern "C" lmh_status lmh_vp_reduce_rows(int R, int64_t rows, int64_t d, const float* parts,
                                         lmh_bf16* out, void* stream) {
  if (R < 1 || rows < 0 || d <= 0 || (d % 64) != 0) return LMH_ERR_INVALID_ARG;
  if (rows == 0) return LMH_OK;
  if (!parts || !out) return LMH_ERR_INVALID_ARG;
  if (!aligned16(parts) || !aligned16(out)) return LMH_ERR_ALIGNMENT;
  int dev, sms;
  LMH_TRY(current_device(&dev, &sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t n4 = rows * d / 4;
  const int64_t blocks = cdiv(n4, 256);
  ProfScope ps(KID_VP_REDUCE, st);
  vp_reduce_rows_kernel<<<static_cast<unsigned>(blocks < 8192 ? blocks : 8192), 256, 0, st>>>(
      R, n4, reinterpret_cast<const float4*>(parts), reinterpret_cast<__nv_bfloat16*>(out));
  return last_launch();
}

extern "C" lmh_status lmh_vp_reduce_rows_to(int R, int64_t rows, int64_t d, const float* parts,
                                            lmh_bf16* const* outs, int n_out, int64_t row_offset,
                                            void* stream) {
  if (R < 1 || rows < 0 || d <= 0 || (d % 64) != 0 || n_out < 1 || row_offset < 0)
    return LMH_ERR_INVALID_ARG;
  if (rows == 0) return LMH_OK;
  if (!parts || !outs) return LMH_ERR_INVALID_ARG;
  if (!aligned16(parts)) return LMH_ERR_ALIGNMENT;
  int dev, sms;
  LMH_TRY(current_device(&dev, &sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t n4 = rows * d / 4;
  const int64_t blocks = cdiv(n4, 256);
  ProfScope ps(KID_VP_REDUCE, st);
  vp_reduce_rows_to_kernel<<<static_cast<unsigned>(blocks < 8192 ? blocks : 8192), 256, 0, st>>>(
      R, n4, reinterpret_cast<const float4*>(parts),
      reinterpret_cast<__nv_bfloat16* const*>(outs), n_out, row_offset * d / 4);
  return last_launch();
}

// The barrier that orders the peer-memory exchanges (peer.cuh). The error word is the
// workspace header's; this entry never clears it, so a time-out stays recorded until the
// caller reads and clears it.
extern "C" lmh_status lmh_peer_barrier(void* workspace, uint32_t* const* signals, int32_t R,
                                       int32_t rank, uint32_t epoch, uint32_t timeout_ms,
                                       void* stream) {
  if (!workspace || !signals || R < 1 || R > 1024 || rank < 0 || rank >= R || epoch == 0 ||
      timeout_ms < 1 || timeout_ms > 60000)
    return LMH_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0 ||
      (reinterpret_cast<uintptr_t>(signals) & 7u) != 0)
    return LMH_ERR_ALIGNMENT;
  int dev, sms;
  LMH_TRY(current_device(&dev, &sms));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned threads = static_cast<unsigned>((R + 31) / 32 * 32);
  ProfScope ps(KID_PEER_BARRIER, st);
  peer_barrier_kernel<<<1, threads, 0, st>>>(signals, R, rank, epoch,
                                             uint64_t(timeout_ms) * 1000000ull,
                                             &static_cast<WsHeader*>(workspace)->err);
  return last_launch();
}
