// lmh_api.cu — the C ABI of include/lmh.h: argument validation, the chunk plan and the
// workspace carve-up, TMA descriptor encoding, and the stream-ordered sequence of kernels of
// each entry. Nothing here allocates device memory or waits for the device (except
// lmh_read_errors, whose job is to).
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

using namespace lmh;

namespace {

constexpr int64_t kDefaultChunk = 4096;
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ------------------------------------------------------------------------ plan
// The row partition and the byte offsets of every workspace region.
struct Plan {
  int64_t N, d, V, K, Vp, T, c, nchunks;
  bool cands;   // per-row candidate lists (support entries, candidate backward)
  bool gbuf;    // chunk softmax / gradient buffer
  bool acc;     // internal fp32 dW accumulator
  bool renorm;  // support entries renormalised over the candidate set (sparse path)
  size_t o_zt, o_sorted, o_nuniq, o_rank, o_pm, o_ps, o_pi, o_alpha, o_beta, o_gbuf, o_acc;
  size_t o_gu, o_cnt, o_off, o_fill, o_prow, o_pslot;  // sparse backward
  size_t o_dhpart;                                     // split-K partials of dH
  size_t o_lloc;                                       // vocab-parallel: shard-local labels
  size_t total;
  Temperature temp;  // logits are z / tau_i
};

bool shape_ok(const lmh_shape* s) {
  if (!s) return false;
  if (s->N < 0 || s->d <= 0 || (s->d % 64) != 0 || s->V <= 0 || s->V > 0x7fffffffLL)
    return false;
  if (s->d > (1LL << 24) || s->chunk_rows < 0) return false;
  if (!(s->temperature >= 0.f && s->temperature < 3.0e38f)) return false;  // NaN fails too
  if ((reinterpret_cast<uintptr_t>(s->row_temperature) & 3u) != 0) return false;
  return true;
}

// K splits of the dH GEMM of a chunk with `rows` rows. Chunks with too few output tiles to keep
// every SM busy (fewer than 384 pair tiles) split the vocabulary into up to 8 ranges, aiming at
// 512 work units. Each split costs a write and a read of an fp32 [rows, d] partial, i.e. 8 / V
// bytes per flop of the GEMM: a range must span at least 32768 vocabulary rows, which keeps
// that traffic near 3 % of the GEMM's time (at V = 32000 no split pays). The rule reads the
// shape only (never the SM count), so the result bits do not depend on the GPU's size.
int dh_splits(int64_t rows, int64_t d, int64_t V) {
  const int64_t tiles = cdiv(rows, PM) * cdiv(d, BN);
  if (tiles >= 384) return 1;
  int64_t sp = cdiv(512, tiles);
  const int64_t by_v = V / 32768;
  if (sp > 8) sp = 8;
  if (sp > by_v) sp = by_v;
  return sp < 1 ? 1 : static_cast<int>(sp);
}

// fused: the entry keeps a [c, Vp] bf16 buffer; need_acc: an fp32 [V, d] accumulator.
Plan make_plan(const lmh_shape* s, int entry, bool fused, bool dw_without_acc) {
  Plan p{};
  const float t = s->temperature;
  p.temp.inv_scalar = (t > 0.f && t != 1.f) ? 1.f / t : 1.f;
  p.temp.rows = s->row_temperature;
  p.N = s->N;
  p.d = s->d;
  p.V = s->V;
  p.Vp = (s->V + 7) / 8 * 8;
  p.T = cdiv(s->V, BN);
  const int64_t c = s->chunk_rows > 0 ? s->chunk_rows : kDefaultChunk;
  p.c = p.N > 0 ? (c < p.N ? c : p.N) : 0;
  p.nchunks = p.N > 0 ? cdiv(p.N, p.c) : 0;
  const bool vp_bwd = entry == LMH_ENTRY_VP_BWD;
  const bool bwd = entry == LMH_ENTRY_LOSS_BWD || vp_bwd;
  p.cands = (entry == LMH_ENTRY_SUPPORT_LOGPROB || entry == LMH_ENTRY_SUPPORT_KL ||
             entry == LMH_ENTRY_LOSS_BWD);
  p.K = p.cands ? (s->K > 0 ? s->K : 1) : 1;
  p.renorm = p.cands && (s->flags & LMH_F_SUPPORT_RENORM);
  const bool fwd_fused = fused && (entry == LMH_ENTRY_LOSS_FWD || entry == LMH_ENTRY_VP_PARTIALS ||
                                   entry == LMH_ENTRY_SUPPORT_KL ||
                                   entry == LMH_ENTRY_LOSS_FWD_BWD);
  p.gbuf = !p.renorm && (bwd || fwd_fused);
  p.acc = p.gbuf && dw_without_acc && p.nchunks > 1;
  const bool stats = !bwd && entry != LMH_ENTRY_VP_COMBINE;
  const bool partials = stats && !p.renorm;
  size_t o = sizeof(WsHeader);
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes);
    return at;
  };
  const size_t N = static_cast<size_t>(p.N);
  p.o_zt = (stats || p.renorm) ? take(N * p.K * 4) : 0;
  p.o_sorted = p.cands ? take(N * p.K * 4) : 0;
  p.o_nuniq = p.cands ? take(N * 4) : 0;
  p.o_rank = p.cands ? take(N * p.K * 4) : 0;
  const size_t cT = static_cast<size_t>(p.c) * p.T;
  p.o_pm = partials ? take(cT * 4) : 0;
  p.o_ps = partials ? take(cT * 4) : 0;
  p.o_pi = partials ? take(cT * 4) : 0;
  const bool coef = bwd || (fwd_fused && (entry == LMH_ENTRY_SUPPORT_KL ||
                                          entry == LMH_ENTRY_LOSS_FWD_BWD));
  p.o_alpha = coef ? take(N * 4) : 0;
  p.o_beta = coef ? take(N * p.K * 4) : 0;
  p.o_lloc = (vp_bwd || entry == LMH_ENTRY_VP_PARTIALS) ? take(N * 4) : 0;
  p.o_gbuf = p.gbuf ? take(static_cast<size_t>(p.c) * p.Vp * 2) : 0;
  p.o_acc = p.acc ? take(static_cast<size_t>(p.V) * p.d * 4) : 0;
  const bool vp = vp_bwd || entry == LMH_ENTRY_VP_PARTIALS;  // dH leaves in fp32, unsplit
  if (p.gbuf && p.nchunks > 0 && !vp) {  // the largest split-K partial of any chunk
    const int64_t last = p.N - (p.nchunks - 1) * p.c;
    const int64_t a = dh_splits(p.c, p.d, p.V) > 1 ? dh_splits(p.c, p.d, p.V) * p.c : 0;
    const int64_t b = dh_splits(last, p.d, p.V) > 1 ? dh_splits(last, p.d, p.V) * last : 0;
    const int64_t r = a > b ? a : b;
    p.o_dhpart = r ? take(static_cast<size_t>(r) * p.d * 4) : 0;
  }
  const bool sparse_bwd = p.renorm && entry == LMH_ENTRY_LOSS_BWD;
  p.o_gu = sparse_bwd ? take(N * p.K * 4) : 0;
  p.o_cnt = sparse_bwd ? take(static_cast<size_t>(p.V) * 4) : 0;
  p.o_off = sparse_bwd ? take((static_cast<size_t>(p.V) + 1) * 4) : 0;
  p.o_fill = sparse_bwd ? take(static_cast<size_t>(p.V) * 4) : 0;
  p.o_prow = sparse_bwd ? take(N * p.K * 4) : 0;
  p.o_pslot = sparse_bwd ? take(N * p.K * 4) : 0;
  p.total = o;
  return p;
}

// ------------------------------------------------------------------------ device state
struct DevState {
  bool init = false;
  bool ok = false;
  int sms = 0;
};
std::mutex g_mu;
DevState g_dev[64];

lmh_status current_device(int* dev_out, int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LMH_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DevState& ds = g_dev[dev];
  if (!ds.init) {
    int major = 0, minor = 0, n = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return LMH_ERR_CUDA;
    ds.ok = (major == 10 && minor == 0);
    ds.sms = n;
    ds.init = true;
  }
  if (!ds.ok) return LMH_ERR_UNSUPPORTED_DEVICE;
  *dev_out = dev;
  *sms = ds.sms;
  return LMH_OK;
}

// ------------------------------------------------------------------------ stage timing
// Measurement hook: while enabled, every kernel the library enqueues is bracketed by a pair
// of CUDA events on its stream (host-side objects; no device memory is allocated).
enum KernelId {
  KID_COUNT_LABELS, KID_PREP_CANDS, KID_GEMM_LOGITS, KID_GEMM_LOGITS_P, KID_GEMM_GRAD,
  KID_GEMM_DH, KID_GEMM_DW, KID_FINALIZE, KID_GBUILD, KID_FIX_LABELS, KID_MEAN,
  KID_SUPPORT_OUT, KID_BWD_COEF, KID_CAST, KID_SUPPORT_DOTS, KID_SUPPORT_LSE,
  KID_SUPPORT_DH, KID_SUPPORT_DW, KID_SPLIT_SUM, KID_VP_LABELS, KID_VP_FINALIZE,
  KID_VP_COMBINE, KID_VP_REDUCE, KID_VP_SCALE, KID_FIX_CANDS, KID_SCALE, KID_COUNT
};
const char* const kKernelNames[KID_COUNT] = {
    "count_labels", "prep_cands", "gemm_logits_stats", "gemm_logits_stats_store",
    "gemm_logits_grad", "gemm_dH", "gemm_dW", "row_finalize", "gbuild", "fix_labels",
    "mean", "support_out", "bwd_coef", "cast_bf16", "support_dots", "support_lse",
    "support_grad_dh", "support_dw", "split_sum", "vp_local_labels", "vp_finalize",
    "vp_combine", "vp_reduce_rows", "vp_scale", "fix_cands", "scale_bf16"};

struct ProfRec {
  int id;
  cudaEvent_t a, b;
};
std::atomic<bool> g_prof_on{false};
std::mutex g_prof_mu;
std::vector<ProfRec> g_prof_recs;
std::vector<cudaEvent_t> g_prof_pool;

cudaEvent_t prof_event() {
  if (!g_prof_pool.empty()) {
    cudaEvent_t e = g_prof_pool.back();
    g_prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

struct ProfScope {
  int id = -1;
  cudaEvent_t a = nullptr;
  cudaStream_t st;
  ProfScope(int kid, cudaStream_t s) : st(s) {
    if (!g_prof_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    a = prof_event();
    if (a && cudaEventRecord(a, st) == cudaSuccess) id = kid;
  }
  ~ProfScope() {
    if (id < 0) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    cudaEvent_t b = prof_event();
    if (b && cudaEventRecord(b, st) == cudaSuccess) g_prof_recs.push_back({id, a, b});
  }
};

// ------------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2-D bf16 tensor [outer, inner] with row stride `ld` elements; box {64, box_outer}, 128-byte
// swizzle, zero fill out of bounds.
bool tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t ld,
             uint32_t box_outer) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {64, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map of an epilogue's staged TMA stores: bf16 [outer, inner], box 64 x 32 rows.
bool tmap_out(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t ld) {
  return tmap_2d(m, base, inner, outer, ld, 32);
}

// Accumulator map of the dW epilogue's staged fp32 stores and adds: fp32 [outer, inner] with
// row stride `ld` elements, box 32 x 32 rows, 128-byte swizzle.
bool tmap_acc(CUtensorMap* m, const float* base, uint64_t inner, uint64_t outer, uint64_t ld) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------------ launches
// Tile orders and L2 priorities of the three contractions.
struct GemmOrder {
  int group_m;  // pair-row tiles per group (rows fastest inside a group)
  int hint_a, hint_b;
};

template <class Epi>
lmh_status launch_gemm(int dev, int sms, const CUtensorMap& a, const CUtensorMap& b,
                       const CUtensorMap& c, int64_t M, int64_t Ncols, int64_t K,
                       GemmOrder order, uint32_t* err, const typename Epi::Params& ep,
                       cudaStream_t st, int k_splits = 1, const CUtensorMap* d = nullptr) {
  static std::atomic<uint64_t> attr_done{0};
  static std::atomic<int> pairs_cache[64];
  const uint64_t bit = 1ull << dev;
  if (!(attr_done.load() & bit)) {
    if (cudaFuncSetAttribute(gemm_tc_kernel<Epi>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GEMM_SMEM_BYTES) != cudaSuccess)
      return LMH_ERR_CUDA;
    // how many CTA pairs can be resident at once (one CTA per SM)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(sms / 2 * 2));
    cfg.blockDim = dim3(GEMM_THREADS);
    cfg.dynamicSmemBytes = GEMM_SMEM_BYTES;
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, gemm_tc_kernel<Epi>, &cfg) != cudaSuccess ||
        nclusters < 1) {
      cudaGetLastError();
      nclusters = sms / 2;
    }
    pairs_cache[dev].store(nclusters);
    attr_done.fetch_or(bit);
  }
  GemmGrid g;
  g.m_tiles = static_cast<int>(cdiv(M, PM));
  g.n_tiles = static_cast<int>(cdiv(Ncols, BN));
  g.k_blocks = static_cast<int>(cdiv(K, BK));
  g.k_splits = k_splits;
  g.group_m = order.group_m < 1 ? g.m_tiles : (order.group_m < g.m_tiles ? order.group_m : g.m_tiles);
  g.hint_a = order.hint_a;
  g.hint_b = order.hint_b;
  g.err = err;
  const int64_t tiles = static_cast<int64_t>(g.m_tiles) * g.n_tiles * k_splits;
  if (tiles <= 0) return LMH_OK;
  const int64_t pairs_max = pairs_cache[dev].load();
  const int pairs = static_cast<int>(tiles < pairs_max ? tiles : pairs_max);
  ProfScope ps(Epi::kId, st);
  gemm_tc_kernel<Epi><<<2 * pairs, GEMM_THREADS, GEMM_SMEM_BYTES, st>>>(a, b, c, d ? *d : c,
                                                                        g, ep);
  return cudaGetLastError() == cudaSuccess ? LMH_OK : LMH_ERR_CUDA;
}

// logits: 16 row tiles (4096 rows of H, 34 MB) across all vocabulary tiles, then the next
// 16: the H slice stays in L2 while W streams (measured 2.5 GB of DRAM reads per launch at
// 8192 x 128256 x 4096 instead of 12 GB when all 32 row tiles share each vocabulary tile)
constexpr GemmOrder kOrderLogits{16, kL2Normal, kL2Normal};
// dH: two 256-row tiles at a time across all hidden tiles (13.8 GB of DRAM reads per launch
// at the headline size, against 19.7 GB for groups of eight and 22.7 GB for rows fastest)
constexpr GemmOrder kOrderDH{2, kL2Normal, kL2Normal};
// dW: one 256-word vocabulary tile across all hidden tiles (each G tile is read once while
// its 16 hidden tiles run side by side; keeping H at evict-last priority measured worse)
constexpr GemmOrder kOrderDW{1, kL2Normal, kL2Normal};

#define LMH_TRY(x)                      \
  do {                                  \
    lmh_status _s = (x);                \
    if (_s != LMH_OK) return _s;        \
  } while (0)

lmh_status last_launch() { return cudaGetLastError() == cudaSuccess ? LMH_OK : LMH_ERR_CUDA; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Ws {
  uint8_t* base;
  WsHeader* h;
  template <class T>
  T* at(size_t off) const { return reinterpret_cast<T*>(base + off); }
};

lmh_status common_checks(const lmh_shape* s, const void* H, const void* W, void* ws,
                         size_t ws_bytes, size_t need, int* dev, int* sms) {
  if (!shape_ok(s)) return LMH_ERR_INVALID_ARG;
  if (s->N > 0 && (!H || !W)) return LMH_ERR_INVALID_ARG;
  if (!ws) return LMH_ERR_INVALID_ARG;
  if (!aligned16(H) || !aligned16(W)) return LMH_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return LMH_ERR_ALIGNMENT;
  if (ws_bytes < need) return LMH_ERR_WORKSPACE_TOO_SMALL;
  return current_device(dev, sms);
}

// Per-chunk logits statistics GEMM + row finalize.
template <int TK, bool kStoreP>
lmh_status run_stats(const Plan& P, int dev, int sms, const lmh_bf16* H, const lmh_bf16* W,
                     const Targets& tg, int64_t r0, int rows, const Ws& ws, cudaStream_t st) {
  CUtensorMap ta, tb, tc;
  if (!tmap_2d(&ta, H + r0 * P.d, P.d, rows, P.d, BM) || !tmap_2d(&tb, W, P.d, P.V, P.d, BNH))
    return LMH_ERR_CUDA;
  if (kStoreP) {
    if (!tmap_out(&tc, ws.at<__nv_bfloat16>(P.o_gbuf), P.Vp, rows, P.Vp)) return LMH_ERR_CUDA;
  } else {
    tc = ta;  // not used without the store
  }
  typename EpiStats<TK, kStoreP>::Params ep;
  ep.rows = rows;
  ep.row0 = r0;
  ep.V = static_cast<int>(P.V);
  ep.T = static_cast<int>(P.T);
  ep.ldp = P.Vp;
  ep.tg = tg;
  ep.zt = ws.at<float>(P.o_zt);
  ep.part_m = ws.at<float>(P.o_pm);
  ep.part_s = ws.at<float>(P.o_ps);
  ep.part_i = ws.at<int32_t>(P.o_pi);
  ep.temp = P.temp;
  return launch_gemm<EpiStats<TK, kStoreP>>(dev, sms, ta, tb, tc, rows, P.V, P.d, kOrderLogits,
                                           &ws.h->err, ep, st);
}

lmh_status run_finalize(const Plan& P, int kind, int64_t r0, int rows, const int32_t* labels,
                        float* lse, float* loss, float* logprob, int32_t* argmax, int write_scale,
                        int mean, const int32_t* n_given, const Ws& ws, cudaStream_t st,
                        const float* alpha = nullptr) {
  FinParams f;
  f.rows = rows;
  f.row0 = r0;
  f.T = static_cast<int>(P.T);
  f.V = static_cast<int>(P.V);
  f.kind = kind;
  f.part_m = ws.at<float>(P.o_pm);
  f.part_s = ws.at<float>(P.o_ps);
  f.part_i = ws.at<int32_t>(P.o_pi);
  f.labels = labels;
  f.zt = ws.at<float>(P.o_zt);
  f.lse = lse;
  f.loss = loss;
  f.logprob = logprob;
  f.argmax = argmax;
  f.write_scale = write_scale;
  f.mean = mean;
  f.n_given = n_given;
  f.h = ws.h;
  f.temp = P.temp;
  f.alpha = alpha;
  const int warps = 8;
  ProfScope ps(KID_FINALIZE, st);
  finalize_rows_kernel<<<static_cast<unsigned>(cdiv(rows, warps)), 32 * warps, 0, st>>>(f);
  return last_launch();
}

// dW = bf16(acc) over [V, d] (V * d is a multiple of 4; both buffers 16-byte aligned).
lmh_status cast_dw(const Plan& P, const float* acc, lmh_bf16* dW, cudaStream_t st) {
  ProfScope ps(KID_CAST, st);
  const int64_t n4 = P.V * P.d / 4;
  const int64_t blocks = cdiv(n4, 256);
  cast_bf16_kernel<<<static_cast<unsigned>(blocks < 8192 ? blocks : 8192), 256, 0, st>>>(
      acc, n4, reinterpret_cast<__nv_bfloat16*>(dW));
  return last_launch();
}

// dH = G W and dW (+)= G^T H_c for one chunk whose G sits in the workspace buffer.
// With dH_f32 (vocabulary-parallel shards) dH's rows go to it in fp32 instead, unsplit.
lmh_status run_backward_gemms(const Plan& P, int dev, int sms, const lmh_bf16* H,
                              const lmh_bf16* W, int64_t r0, int rows, int chunk_idx,
                              lmh_bf16* dH, lmh_bf16* dW, float* dW_acc, const Ws& ws,
                              cudaStream_t st, float* dH_f32 = nullptr,
                              const RowScatter* scatter = nullptr) {
  const __nv_bfloat16* G = ws.at<__nv_bfloat16>(P.o_gbuf);
  if (scatter) {  // each fp32 row straight to the rank that reduces it
    CUtensorMap ta, tb;
    if (!tmap_2d(&ta, G, P.V, rows, P.Vp, BM) || !tmap_2d(&tb, W, P.d, P.V, P.d, BK))
      return LMH_ERR_CUDA;
    EpiDH::Params ep;
    ep.rows = rows;
    ep.d = static_cast<int>(P.d);
    ep.part = nullptr;
    ep.sc = *scatter;
    ep.sc.row0 = r0;
    LMH_TRY(launch_gemm<EpiDH>(dev, sms, ta, tb, ta, rows, P.d, P.V, kOrderDH, &ws.h->err, ep,
                               st, 1));
  } else if (dH_f32) {
    CUtensorMap ta, tb;
    if (!tmap_2d(&ta, G, P.V, rows, P.Vp, BM) || !tmap_2d(&tb, W, P.d, P.V, P.d, BK))
      return LMH_ERR_CUDA;
    EpiDH::Params ep;
    ep.rows = rows;
    ep.d = static_cast<int>(P.d);
    ep.part = dH_f32 + r0 * P.d;  // split 0 of a one-split partial: the rows themselves
    LMH_TRY(launch_gemm<EpiDH>(dev, sms, ta, tb, ta, rows, P.d, P.V, kOrderDH, &ws.h->err, ep,
                               st, 1));
  } else if (dH) {
    CUtensorMap ta, tb, tc;
    if (!tmap_2d(&ta, G, P.V, rows, P.Vp, BM) || !tmap_2d(&tb, W, P.d, P.V, P.d, BK) ||
        !tmap_out(&tc, dH + r0 * P.d, P.d, rows, P.d))
      return LMH_ERR_CUDA;
    EpiDH::Params ep;
    ep.rows = rows;
    ep.d = static_cast<int>(P.d);
    const int sp = dh_splits(rows, P.d, P.V);
    ep.part = sp > 1 ? ws.at<float>(P.o_dhpart) : nullptr;
    LMH_TRY(launch_gemm<EpiDH>(dev, sms, ta, tb, tc, rows, P.d, P.V, kOrderDH, &ws.h->err, ep,
                               st, sp));
    if (sp > 1) {
      ProfScope ps(KID_SPLIT_SUM, st);
      const int64_t blocks = cdiv(static_cast<int64_t>(rows) * P.d / 2, 256);
      split_sum_kernel<<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), 256, 0, st>>>(
          sp, rows, static_cast<int>(P.d), ws.at<float>(P.o_dhpart),
          reinterpret_cast<__nv_bfloat16*>(dH + r0 * P.d));
      LMH_TRY(last_launch());
    }
  }
  if (dW || dW_acc) {
    CUtensorMap ta, tb, tc;
    if (!tmap_2d(&ta, G, P.V, rows, P.Vp, BK) || !tmap_2d(&tb, H + r0 * P.d, P.d, rows, P.d, BK))
      return LMH_ERR_CUDA;
    // Internal accumulator (several chunks, no caller dW_acc): store, add, ..., and the last
    // chunk adds and casts in its epilogue without writing the sum back. Caller's dW_acc:
    // add in every chunk, then cast it. One chunk without dW_acc: bf16 tile sums directly.
    const bool last = chunk_idx == P.nchunks - 1;
    float* acc = dW_acc ? dW_acc : (P.acc ? ws.at<float>(P.o_acc) : nullptr);
    EpiDW::Params ep;
    ep.V = static_cast<int>(P.V);
    ep.d = static_cast<int>(P.d);
    if (!acc) ep.acc_mode = 0;
    else if (dW_acc) ep.acc_mode = 2;
    else ep.acc_mode = chunk_idx == 0 ? 1 : (last ? 3 : 2);
    CUtensorMap td;  // mode 3: the accumulator, read by the epilogue
    bool ok;
    if (ep.acc_mode == 0) {
      ok = tmap_out(&tc, dW, P.d, P.V, P.d);
    } else if (ep.acc_mode == 3) {
      ok = tmap_out(&tc, dW, P.d, P.V, P.d) && tmap_acc(&td, acc, P.d, P.V, P.d);
    } else {
      ok = tmap_acc(&tc, acc, P.d, P.V, P.d);
    }
    if (!ok) return LMH_ERR_CUDA;
    LMH_TRY(launch_gemm<EpiDW>(dev, sms, ta, tb, tc, P.V, P.d, rows, kOrderDW, &ws.h->err, ep,
                               st, 1, ep.acc_mode == 3 ? &td : nullptr));
    if (dW_acc && dW && last) LMH_TRY(cast_dw(P, acc, dW, st));
  }
  return LMH_OK;
}

lmh_status clear_header(const Ws& ws, cudaStream_t st) {
  return cudaMemsetAsync(ws.h, 0, sizeof(WsHeader), st) == cudaSuccess ? LMH_OK : LMH_ERR_CUDA;
}

lmh_status count_labels(const Plan& P, const int32_t* labels, const Ws& ws, cudaStream_t st) {
  if (P.N == 0) return LMH_OK;
  const int64_t blocks = cdiv(P.N, 256);
  ProfScope ps(KID_COUNT_LABELS, st);
  count_labels_kernel<<<static_cast<unsigned>(blocks < 1024 ? blocks : 1024), 256, 0, st>>>(
      labels, P.N, static_cast<int>(P.V), ws.h);
  return last_launch();
}

lmh_status prep_cands(const Plan& P, const int32_t* ids, const Ws& ws, cudaStream_t st) {
  if (P.N == 0) return LMH_OK;
  const int threads = static_cast<int>(cdiv(P.K, 32) * 32);
  const int64_t blocks = P.N < 65535 ? P.N : 65535;
  ProfScope ps(KID_PREP_CANDS, st);
  prep_cands_kernel<<<static_cast<unsigned>(blocks), threads, 3 * P.K * sizeof(int32_t), st>>>(
      ids, P.N, static_cast<int>(P.K), static_cast<int>(P.V), ws.at<int32_t>(P.o_sorted),
      ws.at<int32_t>(P.o_nuniq), ws.at<int32_t>(P.o_rank), ws.h);
  return last_launch();
}

// Logits of each row's distinct candidates (renormalised support entries): zt [N, K].
lmh_status support_logits(const Plan& P, const lmh_bf16* H, const lmh_bf16* W, const Ws& ws,
                          cudaStream_t st) {
  ProfScope ps(KID_SUPPORT_DOTS, st);
  const int64_t blocks = P.N < 65535 ? P.N : 65535;
  support_dots_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      P.N, static_cast<int>(P.K), static_cast<int>(P.d),
      reinterpret_cast<const __nv_bfloat16*>(H), reinterpret_cast<const __nv_bfloat16*>(W),
      ws.at<int32_t>(P.o_sorted), ws.at<int32_t>(P.o_nuniq), P.temp, ws.at<float>(P.o_zt));
  return last_launch();
}

// Backward of the renormalised support objectives: G on the candidates only, dH by a gather
// of W rows, dW by a scatter whose pairs are grouped by id and summed in row order.
lmh_status sparse_backward(const Plan& P, const lmh_bf16* H, const lmh_bf16* W, const float* lse,
                           lmh_bf16* dH, lmh_bf16* dW, float* dW_acc, const Ws& ws,
                           cudaStream_t st) {
  const int K = static_cast<int>(P.K), d = static_cast<int>(P.d), V = static_cast<int>(P.V);
  LMH_TRY(support_logits(P, H, W, ws, st));
  const int64_t rblocks = P.N < 65535 ? P.N : 65535;
  {
    ProfScope ps(KID_SUPPORT_DH, st);
    support_grad_dh_kernel<<<static_cast<unsigned>(rblocks), 256, K * sizeof(float), st>>>(
        P.N, K, d, reinterpret_cast<const __nv_bfloat16*>(W), ws.at<int32_t>(P.o_sorted),
        ws.at<int32_t>(P.o_nuniq), ws.at<float>(P.o_zt), lse, ws.at<float>(P.o_alpha),
        ws.at<float>(P.o_beta), ws.at<float>(P.o_gu), reinterpret_cast<__nv_bfloat16*>(dH));
  }
  LMH_TRY(last_launch());
  if (!dW && !dW_acc) return LMH_OK;
  if (cudaMemsetAsync(ws.at<int32_t>(P.o_cnt), 0, size_t(V) * 4, st) != cudaSuccess ||
      cudaMemsetAsync(ws.at<int32_t>(P.o_fill), 0, size_t(V) * 4, st) != cudaSuccess)
    return LMH_ERR_CUDA;
  ProfScope ps(KID_SUPPORT_DW, st);
  const int64_t pb = cdiv(P.N * K, 256);
  const unsigned pblocks = static_cast<unsigned>(pb < 4096 ? pb : 4096);
  support_count_kernel<<<pblocks, 256, 0, st>>>(P.N, K, ws.at<int32_t>(P.o_sorted),
                                                ws.at<int32_t>(P.o_nuniq), ws.at<int32_t>(P.o_cnt));
  LMH_TRY(last_launch());
  scan_kernel<<<1, 1024, 0, st>>>(V, ws.at<int32_t>(P.o_cnt), ws.at<int32_t>(P.o_off));
  LMH_TRY(last_launch());
  support_place_kernel<<<pblocks, 256, 0, st>>>(
      P.N, K, ws.at<int32_t>(P.o_sorted), ws.at<int32_t>(P.o_nuniq), ws.at<int32_t>(P.o_off),
      ws.at<int32_t>(P.o_fill), ws.at<int32_t>(P.o_prow), ws.at<int32_t>(P.o_pslot));
  LMH_TRY(last_launch());
  support_sort_buckets_kernel<<<static_cast<unsigned>(cdiv(V, 256)), 256, 0, st>>>(
      V, ws.at<int32_t>(P.o_off), ws.at<int32_t>(P.o_prow), ws.at<int32_t>(P.o_pslot));
  LMH_TRY(last_launch());
  const int64_t vblocks = V < 65535 ? V : 65535;
  support_dw_kernel<<<static_cast<unsigned>(vblocks), 256, 0, st>>>(
      V, K, d, reinterpret_cast<const __nv_bfloat16*>(H), ws.at<int32_t>(P.o_off),
      ws.at<int32_t>(P.o_prow), ws.at<int32_t>(P.o_pslot), ws.at<float>(P.o_gu), dW_acc,
      dW_acc ? 2 : 0, reinterpret_cast<__nv_bfloat16*>(dW));
  return last_launch();
}

// Outputs of a call without rows: zero counts / means, dW = cast of the given accumulator.
lmh_status empty_call(const Plan& P, float* mean_out, int32_t* nvalid_out, lmh_bf16* dW,
                      float* dW_acc, cudaStream_t st) {
  if (mean_out && cudaMemsetAsync(mean_out, 0, 4, st) != cudaSuccess) return LMH_ERR_CUDA;
  if (nvalid_out && cudaMemsetAsync(nvalid_out, 0, 4, st) != cudaSuccess) return LMH_ERR_CUDA;
  if (dW) {
    const int64_t n = P.V * P.d;
    if (dW_acc) return cast_dw(P, dW_acc, dW, st);
    if (cudaMemsetAsync(dW, 0, n * 2, st) != cudaSuccess) return LMH_ERR_CUDA;
  }
  return LMH_OK;
}

}  // namespace

// ============================================================================ C ABI

extern "C" size_t lmh_workspace_size(const lmh_shape* shape, int entry) {
  if (!shape_ok(shape) || entry < LMH_ENTRY_LOSS_FWD || entry > LMH_ENTRY_LOSS_FWD_BWD) return 0;
  if ((entry == LMH_ENTRY_SUPPORT_LOGPROB || entry == LMH_ENTRY_SUPPORT_KL) &&
      (shape->K < 1 || shape->K > LMH_MAX_K))
    return 0;
  const bool fused = (entry == LMH_ENTRY_LOSS_FWD || entry == LMH_ENTRY_VP_PARTIALS ||
                      entry == LMH_ENTRY_SUPPORT_KL || entry == LMH_ENTRY_LOSS_FWD_BWD) &&
                     (shape->flags & LMH_F_FUSED_BWD);
  const bool want_acc = !(shape->flags & LMH_F_DW_ACC_GIVEN);
  return make_plan(shape, entry, fused, want_acc).total;
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
                                size_t workspace_bytes, void* stream) {
  if (!shape_ok(shape)) return LMH_ERR_INVALID_ARG;
  const bool fused = dH || dW || dW_acc;
  const Plan P = make_plan(shape, weighted ? LMH_ENTRY_LOSS_FWD_BWD : LMH_ENTRY_LOSS_FWD, fused,
                           dW && !dW_acc);
  int dev, sms;
  LMH_TRY(common_checks(shape, H, W, workspace, workspace_bytes, P.total, &dev, &sms));
  if (P.N > 0 && (!labels || !loss_rows || !lse)) return LMH_ERR_INVALID_ARG;
  if (!aligned16(dH) || !aligned16(dW) || !aligned16(dW_acc)) return LMH_ERR_ALIGNMENT;
  if (weighted && (shape->flags & LMH_F_GRAD_SCALAR) && !grad) return LMH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{static_cast<uint8_t*>(workspace), static_cast<WsHeader*>(workspace)};
  LMH_TRY(clear_header(ws, st));
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
                                 dW_acc, ws, st));
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

extern "C" lmh_status lmh_support_kl_fwd_bwd(const lmh_shape* shape, const lmh_bf16* H,
                                             const lmh_bf16* W, const int32_t* ids,
                                             const float* ref_logp, float* kl_rows,
                                             float* kl_mean, float* lp, float* lse,
                                             lmh_bf16* dH, lmh_bf16* dW, float* dW_acc,
                                             void* workspace, size_t workspace_bytes,
                                             void* stream) {
  if (!shape_ok(shape) || shape->K < 1 || shape->K > LMH_MAX_K) return LMH_ERR_INVALID_ARG;
  if (shape->flags & LMH_F_SUPPORT_RENORM) return LMH_ERR_INVALID_ARG;  // sparse path: two calls
  const bool grads = dH || dW || dW_acc;
  const Plan P = make_plan(shape, LMH_ENTRY_SUPPORT_KL, grads, dW && !dW_acc);
  int dev, sms;
  LMH_TRY(common_checks(shape, H, W, workspace, workspace_bytes, P.total, &dev, &sms));
  if (P.N > 0 && (!ids || !lse || !ref_logp || !kl_rows)) return LMH_ERR_INVALID_ARG;
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
    // the KL's coefficients depend on the reference log-probs only, not on lse: alpha_i =
    // g_i sum_k exp(r_ik), beta_ic = g_i sum_{k: c_ik = c} exp(r_ik), g_i = 1 / N or 1
    ProfScope ps(KID_BWD_COEF, st);
    bwd_coef_kernel<<<static_cast<unsigned>(cdiv(P.N, 8)), 256, 0, st>>>(
        LMH_BWD_SUPPORT_KL, P.N, K, static_cast<int>(P.V), ids, nullptr, ref_logp,
        ws.at<int32_t>(P.o_rank), ws.at<int32_t>(P.o_nuniq), P.temp,
        (shape->flags & LMH_F_MEAN) ? 1 : 0, 0, ws.h, alpha, beta);
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
        P.N, K, ws.at<int32_t>(P.o_rank), ws.at<float>(P.o_zt), lse, ref_logp, lp, kl_rows);
  }
  LMH_TRY(last_launch());
  if (kl_mean) {
    ProfScope ps(KID_MEAN, st);
    mean_kernel<<<1, 1024, 0, st>>>(kl_rows, P.N, 0, nullptr, ws.h, kl_mean);
    LMH_TRY(last_launch());
  }
  return LMH_OK;
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

// ============================================================================ no-allocation
// lmh_logprob_noalloc: the log-prob entry with its scratch in a fixed device array of this
// file instead of a caller workspace, for callers that cannot allocate device memory.
namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB on every device
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

uint8_t* g_static_scratch_addr[64] = {};  // device address per device, guarded by g_mu

// The array's name is only a host-side stand-in; its device address is looked up once per
// device, with that device current, and cached.
lmh_status static_scratch_addr(int dev, uint8_t** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_static_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
      return LMH_ERR_CUDA;
    g_static_scratch_addr[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_static_scratch_addr[dev];
  return LMH_OK;
}

// Largest chunk (at most `want` rows) whose log-prob plan fits the static array, or 0.
int64_t static_chunk_rows(const lmh_shape* s, int64_t want) {
  lmh_shape t = *s;
  t.chunk_rows = want;
  if (make_plan(&t, LMH_ENTRY_LOGPROB, false, false).total <= kStaticScratchBytes) return want;
  int64_t lo = 0, hi = want;  // fits(lo) or lo == 0; !fits(hi)
  while (hi - lo > 1) {
    const int64_t mid = lo + (hi - lo) / 2;
    t.chunk_rows = mid;
    if (make_plan(&t, LMH_ENTRY_LOGPROB, false, false).total <= kStaticScratchBytes) lo = mid;
    else hi = mid;
  }
  return lo;
}

}  // namespace

extern "C" lmh_status lmh_logprob_noalloc(const lmh_shape* shape, const lmh_bf16* H,
                                          const lmh_bf16* W, const int32_t* labels,
                                          float* logprob, float* lse, void* stream) {
  if (!shape_ok(shape)) return LMH_ERR_INVALID_ARG;
  if (shape->N > 0 && (!H || !W || !labels || !logprob || !lse)) return LMH_ERR_INVALID_ARG;
  if (!aligned16(H) || !aligned16(W)) return LMH_ERR_ALIGNMENT;
  lmh_shape s = *shape;
  const int64_t want = s.N > 0 ? (s.chunk_rows > 0 && s.chunk_rows < s.N ? s.chunk_rows : s.N) : 1;
  s.chunk_rows = static_chunk_rows(&s, want);
  if (s.chunk_rows < 1) return LMH_ERR_SCRATCH_LIMIT;
  int dev, sms;
  LMH_TRY(current_device(&dev, &sms));
  uint8_t* scratch = nullptr;
  LMH_TRY(static_scratch_addr(dev, &scratch));
  const Plan P = make_plan(&s, LMH_ENTRY_LOGPROB, false, false);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ws ws{scratch, reinterpret_cast<WsHeader*>(scratch)};
  LMH_TRY(clear_header(ws, st));  // error word and count start at zero on every call
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
