/*
 * lmh.h — C ABI of the deterministic chunked LM-head + loss for NVIDIA B200 (sm_100a).
 *
 * The operation (FlashInfer PR #8059 "feat(cake_lm_head_det_loss): det names for the
 * chunked LM-head + loss backend", description): logits z = H W^T are computed chunk by
 * chunk over rows and vocabulary, never stored as a full N x V matrix in HBM, and reduced
 * to a per-row log-sum-exp, cross-entropy loss and target log-probability; the backward
 * recomputes (or reuses) softmax minus one-hot and contracts it into dH and dW. The same
 * description names the entries chunked_lm_head_det_{loss, logprob, support_logprob,
 * support_kl} and states the determinism contract: for fixed inputs, hardware, chunk plan
 * and initial accumulation buffers, forward and backward give bitwise-identical results run
 * to run. This library keeps that contract: no floating-point atomics, every reduction in a
 * fixed order, and no result depends on how many SMs the GPU has or which SM ran which tile.
 *
 * Conventions shared by every entry
 * ---------------------------------
 * - H [N, d] and W [V, d] are bf16, row-major and contiguous (row stride d elements);
 *   lmh_bf16 is the raw 16-bit pattern. d must be a positive multiple of 64.
 * - Every pointer argument is a DEVICE pointer unless marked "host", 16-byte aligned, and
 *   owned by the caller. The library sees no buffer sizes: each buffer must hold what the
 *   shape declares for it (the sizes given below); a smaller one is read or written past
 *   its end. The Python binding checks every size before the call. The library never allocates device memory, never frees it, and
 *   never synchronises the host: each call only enqueues work on `stream` (a cudaStream_t;
 *   NULL is the legacy default stream) and returns.
 * - The workspace must hold at least lmh_workspace_size(shape, entry) bytes, be 256-byte
 *   aligned, and must not be used by another call in flight at the same time.
 * - Labels (miles-ext-kernels PR #14 "[Cake 13/13]", lm_head op commit, "Review items"):
 *   every negative label marks an ignored row (LMH_IGNORE_INDEX = -100 is the customary
 *   value). A label >= V is out of range: the row is treated as ignored and the device
 *   error word gets LMH_DEVERR_LABEL_RANGE (no trap; read it with lmh_read_errors).
 * - Rows are processed in chunks of shape->chunk_rows rows (0 selects 4096, the default of
 *   the same commit's --cake-lm-head-chunk-size), in ascending order. The chunk plan changes
 *   the summation order of dW across chunks and, where a chunk's dH tiling splits the
 *   vocabulary sum into ranges added in a fixed order (lmh_dh_plan), of dH. The forward
 *   outputs (loss, lse, log-probs, argmax, counts) do not depend on it; no output depends on
 *   the GPU's SM count.
 * - Return value: LMH_OK, or an error found on the host before anything was enqueued
 *   (invalid argument, misalignment, short workspace, unsupported device), or
 *   LMH_ERR_CUDA when a launch failed. Errors found on the device go to the error word.
 */
#ifndef LMH_H_
#define LMH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LMH_API __attribute__((visibility("default")))
#else
#define LMH_API
#endif

typedef uint16_t lmh_bf16;

typedef enum lmh_status {
  LMH_OK = 0,
  LMH_ERR_INVALID_ARG = 1,
  LMH_ERR_UNSUPPORTED_DEVICE = 2,
  LMH_ERR_WORKSPACE_TOO_SMALL = 3,
  LMH_ERR_ALIGNMENT = 4,
  LMH_ERR_CUDA = 5,
  LMH_ERR_SCRATCH_LIMIT = 6
} lmh_status;

#define LMH_IGNORE_INDEX (-100)

/* Bits of the device error word (first 4 bytes of the workspace). */
#define LMH_DEVERR_LABEL_RANGE 0x1u /* a label or candidate id was >= V          */
#define LMH_DEVERR_TIMEOUT 0x2u     /* a bounded wait inside a kernel gave up     */
#define LMH_DEVERR_NONFINITE 0x4u   /* a row's log-sum-exp came out inf or NaN    */
#define LMH_DEVERR_TEMPERATURE 0x8u /* a per-row temperature was not finite and > 0 (used 1) */

/* shape->flags */
#define LMH_F_MEAN 0x1u         /* fused CE gradient is of the mean over valid rows    */
#define LMH_F_FUSED_BWD 0x2u    /* sizing only: lmh_loss_fwd will also produce dH/dW   */
#define LMH_F_DW_ACC_GIVEN 0x4u /* sizing only: the caller passes an fp32 dW_acc       */
#define LMH_F_SUPPORT_RENORM 0x8u /* support entries: renormalise over the candidates   */
#define LMH_F_GRAD_SCALAR 0x10u   /* backward: grad is one float shared by every term    */
#define LMH_F_DW_ACC_STORE 0x20u  /* dW_acc receives this call's dW instead of adding it */

/* entries, for lmh_workspace_size */
#define LMH_ENTRY_LOSS_FWD 0
#define LMH_ENTRY_LOSS_BWD 1
#define LMH_ENTRY_LOGPROB 2
#define LMH_ENTRY_SUPPORT_LOGPROB 3
#define LMH_ENTRY_SUPPORT_KL 4
#define LMH_ENTRY_VP_PARTIALS 5 /* vocabulary-parallel entries, below */
#define LMH_ENTRY_VP_COMBINE 6
#define LMH_ENTRY_VP_BWD 7
#define LMH_ENTRY_LOSS_FWD_BWD 8
#define LMH_ENTRY_VP_SUPPORT_PARTIALS 9
#define LMH_ENTRY_VP_SUPPORT_COMBINE 10
#define LMH_ENTRY_VP_SUPPORT_BWD 11

/* objectives of lmh_loss_bwd */
#define LMH_BWD_CE 0              /* L = sum_i g_i loss_i                                */
#define LMH_BWD_LOGPROB 1         /* L = sum_i g_i logprob_i                             */
#define LMH_BWD_SUPPORT_LOGPROB 2 /* L = sum_ik g_ik lp_ik                               */
#define LMH_BWD_SUPPORT_KL 3      /* L = sum_i g_i KL_i                                  */

#define LMH_MAX_K 1024 /* largest candidate count per row of the support entries */

/*
 * Temperature (miles-ext-kernels PR #14, lm_head op commit: temperature stages, tested off,
 * scalar, per row and 1.0): every entry works on the tempered logits z_iv / tau_i with
 * tau_i = temperature * row_temperature[i] (a factor that is 0 or absent counts as 1), and
 * the gradients carry the chain-rule factor 1 / tau_i. With both off the results are bit for
 * bit those without temperature. A per-row value that is not finite and > 0 is used as 1
 * and flags LMH_DEVERR_TEMPERATURE.
 */
typedef struct lmh_shape {
  int64_t N;                    /* rows (tokens), >= 0                                 */
  int64_t d;                    /* hidden size, multiple of 64                         */
  int64_t V;                    /* vocabulary size, 1 .. 2^31 - 1                      */
  int64_t K;                    /* candidates per row (support entries), 1..LMH_MAX_K  */
  int64_t chunk_rows;           /* rows per chunk; 0 selects 4096                      */
  uint32_t flags;               /* LMH_F_*                                             */
  float temperature;            /* scalar temperature, finite and >= 0; 0 or 1: none   */
  const float* row_temperature; /* device [N] per-row temperatures, or NULL            */
} lmh_shape;

/*
 * lmh_workspace_size — bytes of workspace the entry needs for `shape` (host, pure; no CUDA
 * call). Memory budget (FlashInfer PR #8059, CodeRabbit summary: "memory-budgeted backend
 * options ... workspace reporting"): the largest term is one chunk's bf16 softmax/gradient
 * buffer, chunk_rows x round_up(V, 8) x 2 bytes, present for LMH_ENTRY_LOSS_BWD and for
 * LMH_ENTRY_LOSS_FWD with LMH_F_FUSED_BWD; an fp32 [V, d] dW accumulator is added when the
 * plan has more than one chunk, dW is produced, and LMH_F_DW_ACC_GIVEN is not set.
 * Returns 0 for an invalid shape or entry.
 */
LMH_API size_t lmh_workspace_size(const lmh_shape* shape, int entry);

/*
 * lmh_dh_plan — how the dH = G W contraction of one chunk of `rows` rows is tiled (host,
 * pure; no CUDA call). Not an operation of the method: it makes inspectable a part of what
 * FlashInfer PR #8059's determinism contract (description) calls the chunk plan. *wide (host) receives 1 for 256 x 512 CTA-pair tiles, whose two MMAs
 * per K step share one staged block of G, or 0 for 256 x 256 tiles; *splits (host) the
 * number of vocabulary ranges whose fp32 partial products are summed in ascending order
 * (1: no split). The plan reads (rows, d, V) only, never the device, so dH's bits do not
 * depend on the GPU; a split changes dH's summation order, so two chunk plans whose chunks
 * get different plans round dH differently. The wide tile with one range gives the bits of
 * the 256 x 256 tile. Entries that write dH as fp32 rows (the vocabulary-parallel backward,
 * the row scatters) always use 256 x 256 tiles without a split.
 * Returns LMH_ERR_INVALID_ARG if rows < 1, d is not a positive multiple of 64, V is not in
 * 1 .. 2^31 - 1, or an output pointer is null.
 */
LMH_API lmh_status lmh_dh_plan(int64_t rows, int64_t d, int64_t V, int32_t* wide,
                               int32_t* splits);

/*
 * lmh_loss_fwd — cross-entropy forward, optionally fused with its backward.
 * Passage: FlashInfer PR #8059, description (chunked_lm_head_det_loss; "covers the CE and
 * policy losses"); miles-ext-kernels PR #14, lm_head op commit (labels, FP32 dW accumulator
 * cast to BF16 dW).
 *   labels    [N] int32.
 *   loss_rows [N] fp32 out (required): lse_i - z_i,y_i, 0 for ignored rows.
 *   lse       [N] fp32 out (required): log sum_v exp z_iv, for every row.
 *   logprob   [N] fp32 out, nullable: z_i,y_i - lse_i, 0 for ignored rows.
 *   argmax    [N] int32 out, nullable: smallest v attaining max_v z_iv (fp32 logits).
 *   loss_mean [1] fp32 out, nullable: sum of loss_rows over valid rows / n_valid (0 if none).
 *   n_valid   [1] int32 out, nullable: rows with 0 <= label < V.
 *   n_valid_given [1] int32 in, nullable: if given, the mean divides by this count instead.
 *   dH [N, d] bf16 out, dW [V, d] bf16 out, dW_acc [V, d] fp32 in/out — all nullable. If dH
 *     or dW is given the call also runs the backward of loss_mean (LMH_F_MEAN set) or of
 *     sum_i loss_i (not set), reusing the forward's softmax instead of recomputing logits.
 *     dW_acc, if given, is incremented by this call's dW in chunk order (zero it first for
 *     a fresh gradient) and dW, if given, receives its round-to-nearest-even bf16 cast.
 *     With LMH_F_DW_ACC_STORE in shape->flags the first chunk overwrites dW_acc instead (no
 *     zeroing needed; a call without rows zeroes it), so dW_acc holds exactly this call's
 *     fp32 dW. The flag applies wherever dW_acc is taken.
 *     Each increment is one IEEE fp32 add per element and chunk, rounded to nearest even.
 *     Without dW_acc and with one chunk, dW is the bf16 cast of the fp32 tile sums.
 */
LMH_API lmh_status lmh_loss_fwd(const lmh_shape* shape, const lmh_bf16* H, const lmh_bf16* W,
                        const int32_t* labels, float* loss_rows, float* lse, float* logprob,
                        int32_t* argmax, float* loss_mean, int32_t* n_valid,
                        const int32_t* n_valid_given, lmh_bf16* dH, lmh_bf16* dW,
                        float* dW_acc, void* workspace, size_t workspace_bytes, void* stream);

/*
 * lmh_loss_bwd — backward of any of the four row objectives, recomputing the logits chunk
 * by chunk from H and W (FlashInfer PR #8059, CodeRabbit walkthrough: "memory-budget
 * planning and recomputation"). With P = softmax(z) it forms
 *   G_iv = alpha_i P_iv - sum_k beta_ik [v = t_ik]
 * and returns dH = G W and dW = G^T H, where, by `mode`:
 *   LMH_BWD_CE:              targets = labels [N];  grad [N] = dL/dloss_i;
 *                            alpha_i = beta_i = g_i (valid rows; 0 for ignored rows).
 *   LMH_BWD_LOGPROB:         targets = labels [N];  grad [N] = dL/dlogprob_i;
 *                            alpha_i = beta_i = -g_i.
 *   LMH_BWD_SUPPORT_LOGPROB: targets = ids [N, K]; grad [N, K] = dL/dlp_ik;
 *                            alpha_i = -sum_k g_ik, beta_ik = -g_ik.
 *   LMH_BWD_SUPPORT_KL:      targets = ids [N, K]; grad [N] = dL/dKL_i; ref_logp [N, K];
 *                            alpha_i = g_i sum_k exp(r_ik), beta_ik = g_i exp(r_ik).
 * Candidate ids < 0 are padding and are skipped. lse [N] is the forward's output.
 * A given grad is taken as is (LMH_F_MEAN does not scale it).
 * grad may be NULL: every row term then has the weight 1, or 1 / count with LMH_F_MEAN in
 * shape->flags (count: the valid rows of the labels for CE / LOGPROB, N for the support
 * objectives), taken on the device without a host synchronisation. With LMH_F_GRAD_SCALAR,
 * grad points to one float g (device memory, e.g. the upstream gradient of a summed or
 * averaged loss) and every term has the weight g, or g / count with LMH_F_MEAN.
 * dH, dW, dW_acc: as in lmh_loss_fwd (nullable; dW_acc accumulates in chunk order).
 */
LMH_API lmh_status lmh_loss_bwd(const lmh_shape* shape, int mode, const lmh_bf16* H,
                        const lmh_bf16* W, const int32_t* targets, const float* lse,
                        const float* grad, const float* ref_logp, lmh_bf16* dH, lmh_bf16* dW,
                        float* dW_acc, void* workspace, size_t workspace_bytes, void* stream);

/*
 * lmh_loss_fwd_bwd — lmh_loss_fwd with the fused backward of a weighted row objective known
 * before the call: L = sum_i w_i loss_i (mode LMH_BWD_CE) or L = sum_i w_i logprob_i (mode
 * LMH_BWD_LOGPROB), e.g. a policy-gradient loss whose per-row weights (advantages) are fixed
 * before the forward (FlashInfer PR #8059, description: "the CE and policy losses"). The
 * weights are those of lmh_loss_bwd: w_i = grad[i], taken as given (LMH_F_MEAN does not
 * scale per-row weights); or one shared grad[0] with LMH_F_GRAD_SCALAR, or 1 with grad NULL,
 * these two times 1 / count with LMH_F_MEAN, the count being *n_valid_given if given, else
 * the valid rows. Ignored rows get 0. The forward outputs
 * are those of lmh_loss_fwd (loss_mean is always the mean loss); dH, dW, dW_acc as there.
 * The softmax is reused as in lmh_loss_fwd's fused path: three GEMMs per chunk.
 * Workspace: lmh_workspace_size(shape, LMH_ENTRY_LOSS_FWD_BWD) with LMH_F_FUSED_BWD.
 */
LMH_API lmh_status lmh_loss_fwd_bwd(const lmh_shape* shape, int mode, const lmh_bf16* H,
                                    const lmh_bf16* W, const int32_t* labels, const float* grad,
                                    float* loss_rows, float* lse, float* logprob,
                                    int32_t* argmax, float* loss_mean, int32_t* n_valid,
                                    const int32_t* n_valid_given, lmh_bf16* dH, lmh_bf16* dW,
                                    float* dW_acc, void* workspace, size_t workspace_bytes,
                                    void* stream);

/*
 * lmh_logprob — per-row target log-probability (FlashInfer PR #8059, description:
 * chunked_lm_head_det_logprob; miles-ext-kernels PR #14, lm_head op commit: log_probs).
 *   logprob [N] fp32 out: z_i,y_i - lse_i, 0 for ignored rows.  lse [N] fp32 out (required).
 */
LMH_API lmh_status lmh_logprob(const lmh_shape* shape, const lmh_bf16* H, const lmh_bf16* W,
                       const int32_t* labels, float* logprob, float* lse, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * lmh_support_logprob — "candidate-restricted log-probabilities" (FlashInfer PR #8059,
 * CodeRabbit summary and walkthrough). Reading taken: the full-vocabulary log-probability
 * evaluated at each candidate, lp_ik = z_i,c_ik - lse_i.
 *   ids [N, K] int32 in (K = shape->K; ids < 0 are padding, lp = 0 there; ids >= V flag
 *   LMH_DEVERR_LABEL_RANGE and are treated as padding). lp [N, K] fp32 out. lse [N] out.
 */
LMH_API lmh_status lmh_support_logprob(const lmh_shape* shape, const lmh_bf16* H, const lmh_bf16* W,
                               const int32_t* ids, float* lp, float* lse, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * lmh_support_kl — forward KL over the candidate set (FlashInfer PR #8059, CodeRabbit
 * walkthrough: "candidate-support log-probability and forward-KL APIs"). Reading taken:
 * KL(ref || model) = sum_k exp(r_ik) (r_ik - lp_ik) over the valid candidates of row i,
 * with r = ref_logp the given reference log-probs.
 *   ids [N, K], ref_logp [N, K] fp32 in. kl_rows [N] fp32 out. kl_mean [1] fp32 out,
 *   nullable (mean over all N rows). lp [N, K] fp32 out, nullable. lse [N] out (required).
 */
/*
 * LMH_F_SUPPORT_RENORM (the other reading of "candidate-restricted"): with this flag the
 * support entries normalise over each row's distinct valid candidate ids instead of the whole
 * vocabulary: lp_ik = z_i,c_ik - log sum_{distinct valid c} exp z_ic, and `lse` receives that
 * log-normaliser (0 for a row without candidates). Only the K candidate logits are computed
 * (K dot products per row). lmh_loss_bwd with LMH_BWD_SUPPORT_LOGPROB / LMH_BWD_SUPPORT_KL and
 * the same flag takes that `lse` and forms the gradient on the candidates only: dH by a
 * gather of W rows, dW by a scatter summed per vocabulary row in ascending row order (rows of
 * dW with no candidate get 0, or keep dW_acc). chunk_rows plays no part in this path.
 */
LMH_API lmh_status lmh_support_kl(const lmh_shape* shape, const lmh_bf16* H, const lmh_bf16* W,
                          const int32_t* ids, const float* ref_logp, float* kl_rows,
                          float* kl_mean, float* lp, float* lse, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * Row scatter of the shards' dH contributions (instead of dH_part, see lmh_vp_loss_bwd): the
 * N rows form R consecutive slices (the first N % R hold one row more; slice j: rows
 * [a_j, a_{j+1})), and rank j reduces slice j. recv is a DEVICE array of R pointers; recv[j]
 * is rank j's receive buffer, [R][a_{j+1} - a_j][d] fp32, and this rank's rows land at slot
 * `rank`. recv[j] may point into another GPU's memory (a peer mapping over NVLink, e.g.
 * symmetric memory): the dH GEMM's epilogue writes each fp32 row there with ordinary stores
 * while the GEMM runs, so the exchange needs no separate collective. The caller orders it:
 * every rank's call must finish before rank j reduces its buffer (e.g. a barrier on the
 * stream), and rank j then calls lmh_vp_reduce_rows_to.
 */
typedef struct lmh_vp_dest {
  float* const* recv; /* [R] device array of receive buffers */
  int32_t R;
  int32_t rank;       /* this rank, 0 <= rank < R */
} lmh_vp_dest;

/*
 * Vocabulary-parallel cross entropy. The pages run the head at tensor-parallel size 1 only
 * (miles-ext-kernels PR #14, lm_head op commit: the validate hook's startup checks). These
 * entries split the same definitions over R ranks that each hold a contiguous row range
 * [v0, v0 + V_r) of W (the shard); every rank passes the whole H, the global labels and the
 * same chunk_rows, temperature and flags. Per step:
 *   1. lmh_vp_partials on every rank: a 4-word record per row over the rank's shard.
 *   2. The caller gathers the records of all ranks, in rank order, into [R, N, 4].
 *   3. lmh_vp_combine (any rank, or every rank): lse, loss, log-prob, argmax and the mean, as
 *      lmh_loss_fwd gives them for the whole vocabulary, combined over the ranks in ascending
 *      order.
 *   4. lmh_vp_loss_bwd on every rank with the combined lse: the rank's fp32 contribution to
 *      dH (the sum over its shard) and its shard's dW. dW needs no exchange.
 *   5. The caller sums the dH contributions with lmh_vp_reduce_rows, in rank order (for
 *      example: each rank gathers one row slice from every rank, reduces it, and the bf16
 *      slices are gathered back).
 * With a fixed R and shard plan every output is bitwise reproducible. Against the one-device
 * entries the lse is combined in a different grouping (tiles within a shard, then shards), so
 * the values agree to fp32 rounding, not bit for bit. Label rules as lmh_loss_fwd, against the
 * full vocabulary V_total.
 *
 * lmh_vp_partials: shard->V = V_r (the shard's rows of W), shard->N, d, chunk_rows, flags,
 *   temperature as for lmh_logprob. W_shard [V_r, d] bf16. records [N, 4] out, 16-byte
 *   aligned: { lse_r (fp32) = log sum over the shard of exp z_iv; max_r (fp32) = the shard's
 *   largest logit; arg_r (int32 bits) = the smallest global id attaining it; zy_r (fp32) =
 *   the label's logit if 0 <= y_i - v0 < V_r, else -inf }. Requires 0 <= v0 and
 *   v0 + V_r <= V_total. Workspace: lmh_workspace_size(shard, LMH_ENTRY_VP_PARTIALS).
 *   With LMH_F_FUSED_BWD in shard->flags the call also keeps the shard's softmax numerators
 *   p~ = exp(z - m_t) and tile maxima in the workspace for lmh_vp_fused_bwd (all rows in one
 *   chunk: chunk_rows >= N, else LMH_ERR_INVALID_ARG; size the workspace with the flag).
 */
LMH_API lmh_status lmh_vp_partials(const lmh_shape* shard, int64_t v0, int64_t V_total,
                                   const lmh_bf16* H, const lmh_bf16* W_shard,
                                   const int32_t* labels, float* records, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * lmh_vp_combine: shape->N rows, shape->V = V_total, shape->d as the shards'. records
 * [R, N, 4] in (the ranks' records in rank order, 16-byte aligned). Outputs as lmh_loss_fwd:
 * loss_rows, lse (required), logprob, argmax, loss_mean, n_valid (nullable), n_valid_given
 * (nullable). A valid row whose label logit no record holds sets LMH_DEVERR_NONFINITE.
 * Workspace: lmh_workspace_size(shape, LMH_ENTRY_VP_COMBINE) (256 bytes).
 */
LMH_API lmh_status lmh_vp_combine(const lmh_shape* shape, int R, const float* records,
                                  const int32_t* labels, float* loss_rows, float* lse,
                                  float* logprob, int32_t* argmax, float* loss_mean,
                                  int32_t* n_valid, const int32_t* n_valid_given, void* workspace,
                                  size_t workspace_bytes, void* stream);

/*
 * lmh_vp_loss_bwd: the shard's part of lmh_loss_bwd (mode LMH_BWD_CE or LMH_BWD_LOGPROB; grad
 * nullable as there, with the count over the full vocabulary). lse [N] is the combined one.
 * dH_part [N, d] fp32 out (nullable): sum over the shard's columns of G_iv W_v, to be summed
 * over the ranks; or, with dest (then dH_part must be null), the same rows scattered to the
 * ranks that reduce them. dW_shard [V_r, d] bf16 out and dW_acc_shard [V_r, d] fp32 in/out
 * (nullable, as dW and dW_acc of lmh_loss_bwd). Workspace: lmh_workspace_size(shard, LMH_ENTRY_VP_BWD)
 * (with LMH_F_DW_ACC_GIVEN in shard->flags if dW_acc_shard is passed).
 */
LMH_API lmh_status lmh_vp_loss_bwd(const lmh_shape* shard, int mode, int64_t v0,
                                   int64_t V_total, const lmh_bf16* H, const lmh_bf16* W_shard,
                                   const int32_t* labels, const float* lse, const float* grad,
                                   float* dH_part, lmh_bf16* dW_shard, float* dW_acc_shard,
                                   const lmh_vp_dest* dest, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * lmh_vp_fused_bwd: the shard's backward of the summed loss (or of the mean over the valid
 * rows of all ranks with LMH_F_MEAN) from the p~ that lmh_vp_partials kept, as lmh_loss_fwd's
 * fused path does on one device: G = alpha_i exp(m_t - lse_i) p~ minus alpha_i at the label,
 * with the combined lse. Three GEMMs per step instead of the four of partials + lmh_vp_loss_bwd.
 * Call it with the same shard, flags and workspace as that lmh_vp_partials call, after it and
 * before the workspace is reused. n_valid_given (nullable) as in lmh_loss_fwd. Outputs (and
 * dest) as lmh_vp_loss_bwd.
 */
LMH_API lmh_status lmh_vp_fused_bwd(const lmh_shape* shard, int64_t v0, int64_t V_total,
                                    const lmh_bf16* H, const lmh_bf16* W_shard,
                                    const int32_t* labels, const float* lse,
                                    const int32_t* n_valid_given, float* dH_part,
                                    lmh_bf16* dW_shard, float* dW_acc_shard,
                                    const lmh_vp_dest* dest, void* workspace,
                                    size_t workspace_bytes, void* stream);

/*
 * Vocabulary-parallel support entries (the split of lmh_support_logprob / lmh_support_kl and
 * of lmh_loss_bwd's support objectives; full-vocabulary reading only, LMH_F_SUPPORT_RENORM is
 * refused). shape->K candidates per row; ids [N, K] are the global candidate ids.
 * lmh_vp_support_partials: records [N, K + 1] fp32 out: { lse_r as for lmh_vp_partials; for
 *   each slot k the logit of c_ik if it lies in the shard, else -inf }. Workspace:
 *   lmh_workspace_size(shard, LMH_ENTRY_VP_SUPPORT_PARTIALS).
 * lmh_vp_support_combine: shape->V = V_total; records [R, N, K + 1] in rank order. Outputs as
 *   lmh_support_kl: lp [N, K] (nullable), lse [N], kl_rows [N] and kl_mean [1] (nullable; they
 *   need ref_logp [N, K]). Candidate ids >= V_total set LMH_DEVERR_LABEL_RANGE and count as
 *   padding. Workspace: lmh_workspace_size(shape, LMH_ENTRY_VP_SUPPORT_COMBINE).
 * lmh_vp_support_bwd: mode LMH_BWD_SUPPORT_LOGPROB or LMH_BWD_SUPPORT_KL, grad / ref_logp /
 *   flags as lmh_loss_bwd, lse the combined one; outputs and dest as lmh_vp_loss_bwd. G is
 *   formed on the shard's columns with alpha over all of a row's valid candidates and beta at
 *   the shard's own. Workspace: lmh_workspace_size(shard, LMH_ENTRY_VP_SUPPORT_BWD).
 */
LMH_API lmh_status lmh_vp_support_partials(const lmh_shape* shard, int64_t v0, int64_t V_total,
                                           const lmh_bf16* H, const lmh_bf16* W_shard,
                                           const int32_t* ids, float* records, void* workspace,
                                           size_t workspace_bytes, void* stream);
LMH_API lmh_status lmh_vp_support_combine(const lmh_shape* shape, int R, const float* records,
                                          const int32_t* ids, const float* ref_logp, float* lp,
                                          float* lse, float* kl_rows, float* kl_mean,
                                          void* workspace, size_t workspace_bytes, void* stream);
LMH_API lmh_status lmh_vp_support_bwd(const lmh_shape* shard, int mode, int64_t v0,
                                      int64_t V_total, const lmh_bf16* H,
                                      const lmh_bf16* W_shard, const int32_t* ids,
                                      const float* lse, const float* grad, const float* ref_logp,
                                      float* dH_part, lmh_bf16* dW_shard, float* dW_acc_shard,
                                      const lmh_vp_dest* dest, void* workspace,
                                      size_t workspace_bytes, void* stream);

/*
 * lmh_vp_reduce_rows: out[j] = bf16(sum_{r = 0..R-1} parts[r, j]) over rows x d elements, the
 * R fp32 contributions added in ascending r (round to nearest even). parts [R, rows, d] fp32,
 * out [rows, d] bf16, both 16-byte aligned; d a multiple of 64. No workspace.
 */
LMH_API lmh_status lmh_vp_reduce_rows(int R, int64_t rows, int64_t d, const float* parts,
                                      lmh_bf16* out, void* stream);

/*
 * lmh_vp_reduce_rows_to: the same sum, stored into n_out outputs at row row_offset: outs is a
 * DEVICE array of n_out pointers to [*, d] bf16 buffers, which may be other GPUs' memory (each
 * rank's full dH, so that rank j's reduced slice reaches every rank with ordinary stores).
 * parts 16-byte aligned; every outs[k] + row_offset * d 8-byte aligned.
 */
LMH_API lmh_status lmh_vp_reduce_rows_to(int R, int64_t rows, int64_t d, const float* parts,
                                         lmh_bf16* const* outs, int n_out, int64_t row_offset,
                                         void* stream);

/*
 * lmh_support_kl_fwd_bwd — lmh_support_kl plus the backward of the mean KL (LMH_F_MEAN:
 * weight 1 / N per row) or of the summed KL, in one pass that reuses the forward's softmax as
 * lmh_loss_fwd's fused path does. The KL's coefficients (alpha_i = g_i sum_k exp(r_ik),
 * beta_ic = g_i sum over the slots of c of exp(r_ik)) depend on the reference log-probs only,
 * so the forward's softmax numerators p~ = exp(z - m_t) are kept per chunk, scaled into
 * alpha_i P by the row finalize, and the candidate columns rewritten from their fp32 logits.
 * Three GEMMs per chunk instead of the four of lmh_support_kl followed by lmh_loss_bwd.
 *   Arguments as lmh_support_kl (kl_rows, lse and ref_logp required), plus dH, dW, dW_acc as
 *   in lmh_loss_fwd (all null: the forward alone). Workspace: lmh_workspace_size(shape,
 *   LMH_ENTRY_SUPPORT_KL) with LMH_F_FUSED_BWD (and LMH_F_DW_ACC_GIVEN) in shape->flags.
 *   LMH_F_SUPPORT_RENORM is refused (LMH_ERR_INVALID_ARG): that reading's backward is the
 *   sparse path of lmh_loss_bwd, which has no logits GEMM to save.
 */
/*
 * lmh_support_fwd_bwd — the general one-pass support entry: the forward of lmh_support_kl
 * (mode LMH_BWD_SUPPORT_KL; ref_logp and kl_rows required) or of lmh_support_logprob (mode
 * LMH_BWD_SUPPORT_LOGPROB; kl outputs and ref_logp unused), plus the backward of
 * L = sum_i g_i KL_i or L = sum_ik g_ik lp_ik with weights known before the call: grad [N]
 * (KL) or [N, K] (log-probs), taken as given; or one shared grad[0] with LMH_F_GRAD_SCALAR,
 * or 1 with grad NULL, these two times 1 / N with LMH_F_MEAN. Workspace and outputs as
 * lmh_support_kl_fwd_bwd, which is this entry with mode LMH_BWD_SUPPORT_KL and grad NULL.
 */
LMH_API lmh_status lmh_support_fwd_bwd(const lmh_shape* shape, int mode, const lmh_bf16* H,
                                       const lmh_bf16* W, const int32_t* ids,
                                       const float* ref_logp, const float* grad, float* kl_rows,
                                       float* kl_mean, float* lp, float* lse, lmh_bf16* dH,
                                       lmh_bf16* dW, float* dW_acc, void* workspace,
                                       size_t workspace_bytes, void* stream);

LMH_API lmh_status lmh_support_kl_fwd_bwd(const lmh_shape* shape, const lmh_bf16* H,
                                          const lmh_bf16* W, const int32_t* ids,
                                          const float* ref_logp, float* kl_rows, float* kl_mean,
                                          float* lp, float* lse, lmh_bf16* dH, lmh_bf16* dW,
                                          float* dW_acc, void* workspace,
                                          size_t workspace_bytes, void* stream);

/*
 * Row data-parallel steps. Every rank holds all of W and its own rows of the batch; the mean
 * loss divides by the valid rows of all ranks, and dW is the sum of the ranks' dW. The pages'
 * ops sum a weight gradient over the rows of one call and leave its reduction across ranks
 * to the caller (miles-ext-kernels PR #14, gated RMSNorm commit notes). These two entries
 * let the caller make that reduction reproducible, with the arithmetic in this library:
 *   1. lmh_count_valid on every rank; the caller sums the counts over the ranks (an integer
 *      all-reduce, exact in any order).
 *   2. lmh_loss_fwd or lmh_loss_fwd_bwd on every rank with LMH_F_MEAN, n_valid_given = that
 *      sum, dW = NULL and an fp32 dW_acc with LMH_F_DW_ACC_STORE: loss_mean is then the rank's
 *      share of the global mean, dH its own rows' gradient, dW_acc its fp32 dW.
 *   3. The caller gathers the R shares of the mean and adds them in rank order
 *      (lmh_reduce_ranks_f32), and sums the fp32 dW in rank order by row slices with
 *      lmh_vp_reduce_rows (each rank reduces the rows of its slice from every rank; the bf16
 *      slices are then gathered), as for the vocabulary-parallel dH.
 * With a fixed rank count and batch split every output is bitwise reproducible; against one
 * device on the concatenated batch the values agree to fp32 rounding.
 *
 * lmh_count_valid: *n_valid = the number of rows with 0 <= labels[i] < V (int32 device out).
 *   labels [N] int32 device. No workspace; labels >= V are not flagged here (the loss entries
 *   flag them). N = 0 writes 0.
 * lmh_reduce_ranks_f32: out[i] = sum_{r = 0..R-1} parts[r * n + i] in ascending r, fp32
 *   (round to nearest even). parts [R, n] and out [n] fp32 device, 4-byte aligned; any n.
 */
LMH_API lmh_status lmh_count_valid(int64_t N, int64_t V, const int32_t* labels,
                                   int32_t* n_valid, void* stream);

/*
 * lmh_dp_loss_fwd_bwd — step 2 above with the dW exchange fused into the dW GEMM: instead of
 * writing the rank's fp32 dW locally for a collective to move, the GEMM's epilogue stores
 * each fp32 row (0 + tile sum) straight into the receive buffer of the rank that reduces it,
 * while the GEMM runs (ordinary stores; the buffers may be other GPUs' memory through peer
 * mappings). The vocabulary rows are split as evenly as possible into R slices in order;
 * rank j reduces slice j, and its buffer dW_dest->recv[j] is [R][rows_j][d] fp32 with slot r
 * for rank r (16-byte aligned). A rank without rows zeroes its slots. The caller orders the
 * steps: every rank's call has finished before rank j adds its R slots in rank order with
 * lmh_vp_reduce_rows_to (which can store the bf16 slice into every rank's dW). The additions
 * are those of the collective route, so the bits are the same.
 *   Arguments as lmh_loss_fwd_bwd (mode LMH_BWD_CE or LMH_BWD_LOGPROB; grad NULL for the
 *   plain mean or summed CE), without n_valid, dW and dW_acc. One chunk only:
 *   shape->chunk_rows >= N (LMH_ERR_INVALID_ARG otherwise). Workspace:
 *   lmh_workspace_size(shape, LMH_ENTRY_LOSS_FWD_BWD) with LMH_F_FUSED_BWD.
 */
LMH_API lmh_status lmh_dp_loss_fwd_bwd(const lmh_shape* shape, int mode, const lmh_bf16* H,
                                       const lmh_bf16* W, const int32_t* labels,
                                       const float* grad, float* loss_rows, float* lse,
                                       float* logprob, int32_t* argmax, float* loss_mean,
                                       const int32_t* n_valid_given, lmh_bf16* dH,
                                       const lmh_vp_dest* dW_dest, void* workspace,
                                       size_t workspace_bytes, void* stream);
LMH_API lmh_status lmh_reduce_ranks_f32(int R, int64_t n, const float* parts, float* out,
                                        void* stream);

/*
 * lmh_scale_bf16 — x = bf16(x * g[0]) in place over n elements (n a multiple of 4, x 8-byte
 * aligned; g one float in device memory; rounding to nearest even, so g = 1 changes no bit).
 * Not part of the method: it lets a training framework apply the upstream gradient g of a
 * summed or averaged loss to the dH and dW that a one-pass entry (lmh_loss_fwd with dH/dW,
 * lmh_support_kl_fwd_bwd) computed for g = 1, with no host synchronisation.
 */
LMH_API lmh_status lmh_scale_bf16(lmh_bf16* x, int64_t n, const float* g, void* stream);

/*
 * lmh_read_errors — synchronises `stream`, then copies the device error word of the last
 * call that used `workspace` into *errors (host). Each entry clears the word when it starts.
 */
LMH_API lmh_status lmh_read_errors(const void* workspace, uint32_t* errors, void* stream);

/*
 * lmh_logprob_noalloc — the same per-row target log-probability and log-sum-exp as
 * lmh_logprob, for callers that cannot allocate device memory. The pages have no counterpart
 * of this entry.
 *
 * Who needs it: code that is handed its input and output buffers but may not call
 * cudaMalloc on the call path, so it cannot provide the workspace lmh_logprob needs. Examples
 * are a plugin inside an inference engine that owns and pre-reserves the whole device heap,
 * and a hot loop that must not change a memory pool's accounting.
 *
 * What it does instead: its scratch (error word, label logits, per-tile partials) lives in
 * one fixed 32 MiB array inside this library, which every GPU that loads the library keeps
 * until the process exits. The call allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine. Results are bit-identical to lmh_logprob's. The rows are split
 * into chunks small enough for the array; the chunk plan does not change any log-prob bit.
 *   - The first call on each device looks up the array's device address (with that device
 *     current) and caches it. Make that first call before any stream capture.
 *   - All calls share the one array, and it keeps the last call's contents. Calls whose work
 *     overlaps on the GPU (other streams, other host threads, the same device) race on it and
 *     give wrong results. Order such calls on one stream or synchronise between them.
 *   - A shape whose plan does not fit the array even one row at a time (about 2.6 million
 *     vocabulary entries per row, or fewer with very many rows) returns
 *     LMH_ERR_SCRATCH_LIMIT before anything is enqueued.
 * Arguments as lmh_logprob, without the workspace. The error word cannot be read back; use
 * lmh_logprob where that matters.
 */
LMH_API lmh_status lmh_logprob_noalloc(const lmh_shape* shape, const lmh_bf16* H,
                                       const lmh_bf16* W, const int32_t* labels, float* logprob,
                                       float* lse, void* stream);

/*
 * lmh_peer_barrier — a stream-ordered barrier of R ranks through peer memory, with a bounded
 * wait. Not part of the method: it orders the peer-memory exchanges of the multi-rank steps
 * (the RowScatter of lmh_vp_loss_bwd / lmh_vp_fused_bwd / lmh_dp_loss_fwd_bwd writes into
 * another rank's receive buffer, and that rank may reduce the buffer only after every rank's
 * stores have landed; lmh_vp_reduce_rows_to writes into every rank's output, which the
 * owners may read only after every rank's reduce).
 *   signals: DEVICE array of R pointers, 8-byte aligned. signals[j] is rank j's signal array
 *     of R uint32 words, which may live in another GPU's memory (a peer mapping over NVLink,
 *     e.g. symmetric memory). Zero every rank's array once, and make sure every rank has done
 *     so (e.g. a host-side collective), before the first barrier.
 *   epoch: the barrier's number, 1, 2, 3, ... in the same sequence on every rank (0 is
 *     invalid). Words are compared modulo 2^32.
 *   The kernel makes this rank's earlier writes on `stream` (peer stores included) visible
 *   system-wide, stores `epoch` into word `rank` of every rank's array, then waits until
 *   every word of signals[rank] has reached `epoch`. Later work on `stream` sees what the
 *   other ranks wrote before their signals.
 *   timeout_ms (1..60000): the wait gives up after this long, sets LMH_DEVERR_TIMEOUT in the
 *     workspace's error word and returns; the context stays usable. The word is never cleared
 *     here: read it with lmh_read_errors (which synchronises the stream) before trusting the
 *     exchange that the barrier ordered, and clear it before the next use.
 *   workspace: at least 256 bytes, 256-byte aligned (only its error word is used).
 *   R in 1..1024, 0 <= rank < R. LMH_ERR_INVALID_ARG / LMH_ERR_ALIGNMENT before any launch.
 * Never run two ranks of one barrier as separate launches on the same GPU: nothing makes them
 * run at the same time, so they would wait out the time-out on each other.
 */
LMH_API lmh_status lmh_peer_barrier(void* workspace, uint32_t* const* signals, int32_t R,
                                    int32_t rank, uint32_t epoch, uint32_t timeout_ms,
                                    void* stream);

/*
 * lmh_selftest_wait_timeout — failure-path self-test (not part of the method). Enqueues one
 * thread that waits, with the bounded wait every kernel of this library uses, on an mbarrier
 * that nothing arrives on. The wait gives up after timeout_ms (1..5000) and sets
 * LMH_DEVERR_TIMEOUT in the workspace's error word (read it with lmh_read_errors); the
 * context stays usable. workspace: at least 256 bytes, 256-byte aligned.
 */
LMH_API lmh_status lmh_selftest_wait_timeout(void* workspace, uint32_t timeout_ms, void* stream);

/*
 * Measurement hook (not part of the method). lmh_profile_enable(1) makes every later call
 * bracket each kernel it enqueues with a pair of CUDA events on the call's stream (host-side
 * event objects only; process-wide; lmh_profile_enable(0) stops). lmh_profile_read
 * synchronises the recorded events, writes up to max_records (kernel id, milliseconds)
 * pairs to the host arrays, returns how many it wrote and forgets all records.
 * lmh_kernel_name maps an id to a stable name ("gemm_dW", "row_finalize", ...).
 */
LMH_API lmh_status lmh_profile_enable(int on);
LMH_API int lmh_profile_read(int max_records, int32_t* kernel_ids, float* ms);
LMH_API const char* lmh_kernel_name(int kernel_id);

#ifdef __cplusplus
}
#endif

#endif /* LMH_H_ */
