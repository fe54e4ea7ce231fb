// api_common.cuh — the host side shared by every entry of the C ABI: argument checks, the chunk
// plan and the workspace carve-up, device state, the kernel timing hook, TMA descriptor
// encoding, the persistent-GEMM launch, and the stream-ordered steps several entries run.
// Part of the one translation unit lmh_api.cu (included there once, inside no namespace).
#pragma once

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
  bool acc_store;  // the caller's dW_acc is overwritten by the first chunk, not added to
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

// K splits of the narrow (256 x 256) dH GEMM of a chunk with `rows` rows. Chunks with too few
// output tiles to keep every SM busy (fewer than 384 pair tiles) split the vocabulary into up
// to 8 ranges, aiming at 512 work units. Each split costs a write and a read of an fp32
// [rows, d] partial, i.e. 8 / V bytes per flop of the GEMM: a range must span at least 32768
// vocabulary rows, which keeps that traffic near 3 % of the GEMM's time (at V = 32000 no split
// pays).
int dh_splits(int64_t rows, int64_t d, int64_t V) {
  const int64_t tiles = cdiv(rows, PM) * cdiv(d, BN);
  if (tiles >= 384) return 1;
  int64_t sp = cdiv(512, tiles);
  const int64_t by_v = V / 32768;
  if (sp > 8) sp = 8;
  if (sp > by_v) sp = by_v;
  return sp < 1 ? 1 : static_cast<int>(sp);
}

// The dH GEMM of a chunk: narrow (256 x 256) or wide (256 x 512) pair tiles, and its K splits.
// Work is counted in rounds of the 74 CTA pairs of a 148-SM B200 (a wide unit takes two narrow
// units' time); the wide tile, whose operand traffic is a quarter lower, is taken when its
// rounds cost less than 0.95 of the narrow tile's (the 0.95: a step measured 5 % faster with a
// quarter of dH's operand loads left out). Its splits (up to 8, each range at least 32768
// vocabulary rows) minimise its rounds. The rule reads the shape only, never the device, so
// the result bits do not depend on the GPU that runs it.
struct DhPlan {
  bool wide;
  int splits;
};
constexpr int kPlanPairs = 74;
DhPlan dh_plan(int64_t rows, int64_t d, int64_t V) {
  const int sn = dh_splits(rows, d, V);
  const int64_t tn = cdiv(rows, PM) * cdiv(d, BN);
  const double narrow = static_cast<double>(cdiv(tn * sn, kPlanPairs)) / sn;
  const int64_t tw = cdiv(rows, PM) * cdiv(d, 2 * BN);
  int64_t max_sp = V / 32768;
  if (max_sp > 8) max_sp = 8;
  if (max_sp < 1) max_sp = 1;
  int best_sp = 1;
  double best = 2.0 * cdiv(tw, kPlanPairs);
  for (int sp = 2; sp <= max_sp; ++sp) {
    const double t = 2.0 * cdiv(tw * sp, kPlanPairs) / sp;
    if (t < best) {
      best = t;
      best_sp = sp;
    }
  }
  if (best * 0.95 < narrow) return DhPlan{true, best_sp};
  return DhPlan{false, sn};
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
  const bool vp_sup = entry == LMH_ENTRY_VP_SUPPORT_PARTIALS || entry == LMH_ENTRY_VP_SUPPORT_BWD;
  const bool vp_bwd = entry == LMH_ENTRY_VP_BWD || entry == LMH_ENTRY_VP_SUPPORT_BWD;
  const bool bwd = entry == LMH_ENTRY_LOSS_BWD || vp_bwd;
  p.cands = (entry == LMH_ENTRY_SUPPORT_LOGPROB || entry == LMH_ENTRY_SUPPORT_KL ||
             entry == LMH_ENTRY_LOSS_BWD || vp_sup);
  p.K = p.cands ? (s->K > 0 ? s->K : 1) : 1;
  p.renorm = p.cands && (s->flags & LMH_F_SUPPORT_RENORM);
  const bool fwd_fused = fused && (entry == LMH_ENTRY_LOSS_FWD || entry == LMH_ENTRY_VP_PARTIALS ||
                                   entry == LMH_ENTRY_SUPPORT_KL ||
                                   entry == LMH_ENTRY_LOSS_FWD_BWD);
  p.gbuf = !p.renorm && (bwd || fwd_fused);
  p.acc = p.gbuf && dw_without_acc && p.nchunks > 1;
  p.acc_store = (s->flags & LMH_F_DW_ACC_STORE) != 0;
  const bool stats = !bwd && entry != LMH_ENTRY_VP_COMBINE &&
                     entry != LMH_ENTRY_VP_SUPPORT_COMBINE;
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
  // shard-local labels [N], or shard-local candidate ids [N, K]
  p.o_lloc = (vp_bwd || entry == LMH_ENTRY_VP_PARTIALS || vp_sup) ? take(N * p.K * 4) : 0;
  p.o_gbuf = p.gbuf ? take(static_cast<size_t>(p.c) * p.Vp * 2) : 0;
  p.o_acc = p.acc ? take(static_cast<size_t>(p.V) * p.d * 4) : 0;
  const bool vp = vp_bwd || entry == LMH_ENTRY_VP_PARTIALS || vp_sup;  // dH in fp32, unsplit
  if (p.gbuf && p.nchunks > 0 && !vp) {  // the largest split-K partial of any chunk
    const int64_t last = p.N - (p.nchunks - 1) * p.c;
    const int sa = dh_plan(p.c, p.d, p.V).splits, sb = dh_plan(last, p.d, p.V).splits;
    const int64_t a = sa > 1 ? sa * p.c : 0;
    const int64_t b = sb > 1 ? sb * last : 0;
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
  KID_VP_COMBINE, KID_VP_REDUCE, KID_VP_SCALE, KID_FIX_CANDS, KID_SCALE, KID_COUNT_VALID,
  KID_REDUCE_RANKS, KID_ZERO_SLOTS, KID_PEER_BARRIER, KID_COUNT
};
const char* const kKernelNames[KID_COUNT] = {
    "count_labels", "prep_cands", "gemm_logits_stats", "gemm_logits_stats_store",
    "gemm_logits_grad", "gemm_dH", "gemm_dW", "row_finalize", "gbuild", "fix_labels",
    "mean", "support_out", "bwd_coef", "cast_bf16", "support_dots", "support_lse",
    "support_grad_dh", "support_dw", "split_sum", "vp_local_labels", "vp_finalize",
    "vp_combine", "vp_reduce_rows", "vp_scale", "fix_cands", "scale_bf16", "count_valid",
    "reduce_ranks", "zero_slots", "peer_barrier"};

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
                             Pipe<Epi>::SMEM_BYTES) != cudaSuccess)
      return LMH_ERR_CUDA;
    // how many CTA pairs can be resident at once (one CTA per SM)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(sms / 2 * 2));
    cfg.blockDim = dim3(GEMM_THREADS);
    cfg.dynamicSmemBytes = Pipe<Epi>::SMEM_BYTES;
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
  g.n_tiles = static_cast<int>(cdiv(Ncols, BN * Pipe<Epi>::WIDE));
  g.k_blocks = static_cast<int>(cdiv(K, Pipe<Epi>::BK));
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
  gemm_tc_kernel<Epi><<<2 * pairs, GEMM_THREADS, Pipe<Epi>::SMEM_BYTES, st>>>(
      a, b, c, d ? *d : c, g, ep);
  return cudaGetLastError() == cudaSuccess ? LMH_OK : LMH_ERR_CUDA;
}

// logits: 16 row tiles (4096 rows of H, 34 MB) across all vocabulary tiles, then the next
// 16: the H slice stays in L2 while W streams (measured 2.5 GB of DRAM reads per launch at
// 8192 x 128256 x 4096 instead of 12 GB when all 32 row tiles share each vocabulary tile)
constexpr GemmOrder kOrderLogits{16, kL2Normal, kL2Normal};
// dH: two 256-row tiles at a time across all hidden tiles (13.8 GB of DRAM reads per launch
// at the headline size, against 19.7 GB for groups of eight and 22.7 GB for rows fastest)
constexpr GemmOrder kOrderDH{2, kL2Normal, kL2Normal};
// dH split over vocabulary ranges (a chunk with few row tiles): every row tile of the chunk
// in one group, so a wave spans all rows and a few hidden tiles of one range and each slice
// of W is read by one wave (2048 x 5120 x 151936 in 4 ranges: 5.2-5.5 GB of DRAM reads per
// launch instead of 7.2-7.5 GB for groups of two)
constexpr GemmOrder kOrderDHSplit{0, kL2Normal, kL2Normal};
// dH with wide tiles: two 256-row tiles at a time across all 512-column tiles, split-major
constexpr GemmOrder kOrderDHWide{2, kL2Normal, kL2Normal};
// dW: one 256-word vocabulary tile across all hidden tiles (each G tile is read once while
// its 16 hidden tiles run side by side; keeping H at evict-last priority measured worse)
constexpr GemmOrder kOrderDW{1, kL2Normal, kL2Normal};
// dW's bf16 output of one chunk in 256 x 512 tiles from this many rows (64 K blocks) up
constexpr int kDwWideRows = 8192;

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

// One chunk's dW GEMM in accumulate mode acc_mode (EpiDW); its tensor maps use the
// instantiation's K per stage.
template <class Epi>
lmh_status run_dw(const Plan& P, int dev, int sms, const __nv_bfloat16* G, const lmh_bf16* H,
                  int64_t r0, int rows, int acc_mode, float* acc, lmh_bf16* dW,
                  const RowScatter* dw_scatter, const Ws& ws, cudaStream_t st) {
  CUtensorMap ta, tb, tc, td;  // td: mode 3 reads the accumulator through it
  if (!tmap_2d(&ta, G, P.V, rows, P.Vp, Pipe<Epi>::BK) ||
      !tmap_2d(&tb, H + r0 * P.d, P.d, rows, P.d, Pipe<Epi>::BK))
    return LMH_ERR_CUDA;
  typename Epi::Params ep;
  ep.V = static_cast<int>(P.V);
  ep.d = static_cast<int>(P.d);
  ep.acc_mode = acc_mode;
  if (acc_mode == 4) ep.sc = *dw_scatter;
  bool ok;
  if (acc_mode == 4) {
    tc = ta;
    ok = true;
  } else if (acc_mode == 0) {
    ok = tmap_out(&tc, dW, P.d, P.V, P.d);
  } else if (acc_mode == 3 || acc_mode == 5) {
    ok = tmap_out(&tc, dW, P.d, P.V, P.d) && tmap_acc(&td, acc, P.d, P.V, P.d);
  } else {
    ok = tmap_acc(&tc, acc, P.d, P.V, P.d);
  }
  if (!ok) return LMH_ERR_CUDA;
  return launch_gemm<Epi>(dev, sms, ta, tb, tc, P.V, P.d, rows, kOrderDW, &ws.h->err, ep, st, 1,
                          (acc_mode == 3 || acc_mode == 5) ? &td : nullptr);
}

// dH = G W and dW (+)= G^T H_c for one chunk whose G sits in the workspace buffer.
// With dH_f32 (vocabulary-parallel shards) dH's rows go to it in fp32 instead, unsplit.
lmh_status run_backward_gemms(const Plan& P, int dev, int sms, const lmh_bf16* H,
                              const lmh_bf16* W, int64_t r0, int rows, int chunk_idx,
                              lmh_bf16* dH, lmh_bf16* dW, float* dW_acc, const Ws& ws,
                              cudaStream_t st, float* dH_f32 = nullptr,
                              const RowScatter* scatter = nullptr,
                              const RowScatter* dw_scatter = nullptr) {
  const __nv_bfloat16* G = ws.at<__nv_bfloat16>(P.o_gbuf);
  if (scatter) {  // each fp32 row straight to the rank that reduces it
    CUtensorMap ta, tb;
    if (!tmap_2d(&ta, G, P.V, rows, P.Vp, BM) || !tmap_2d(&tb, W, P.d, P.V, P.d, Pipe<EpiDH>::BK))
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
    if (!tmap_2d(&ta, G, P.V, rows, P.Vp, BM) || !tmap_2d(&tb, W, P.d, P.V, P.d, Pipe<EpiDH>::BK))
      return LMH_ERR_CUDA;
    EpiDH::Params ep;
    ep.rows = rows;
    ep.d = static_cast<int>(P.d);
    ep.part = dH_f32 + r0 * P.d;  // split 0 of a one-split partial: the rows themselves
    LMH_TRY(launch_gemm<EpiDH>(dev, sms, ta, tb, ta, rows, P.d, P.V, kOrderDH, &ws.h->err, ep,
                               st, 1));
  } else if (dH) {
    const DhPlan dp = dh_plan(rows, P.d, P.V);
    const int sp = dp.splits;
    CUtensorMap ta, tb, tc;
    if (!tmap_2d(&ta, G, P.V, rows, P.Vp, BM) ||
        !tmap_2d(&tb, W, P.d, P.V, P.d, dp.wide ? Pipe<EpiDHWide>::BK : Pipe<EpiDH>::BK) ||
        !tmap_out(&tc, dH + r0 * P.d, P.d, rows, P.d))
      return LMH_ERR_CUDA;
    EpiDH::Params ep;  // the same parameters for both tile widths
    ep.rows = rows;
    ep.d = static_cast<int>(P.d);
    ep.part = sp > 1 ? ws.at<float>(P.o_dhpart) : nullptr;
    if (dp.wide)
      LMH_TRY(launch_gemm<EpiDHWide>(dev, sms, ta, tb, tc, rows, P.d, P.V, kOrderDHWide,
                                     &ws.h->err, ep, st, sp));
    else
      LMH_TRY(launch_gemm<EpiDH>(dev, sms, ta, tb, tc, rows, P.d, P.V,
                                 sp > 1 ? kOrderDHSplit : kOrderDH, &ws.h->err, ep, st, sp));
    if (sp > 1) {
      ProfScope ps(KID_SPLIT_SUM, st);
      const int64_t blocks = cdiv(static_cast<int64_t>(rows) * P.d / 2, 256);
      split_sum_kernel<<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), 256, 0, st>>>(
          sp, rows, static_cast<int>(P.d), ws.at<float>(P.o_dhpart),
          reinterpret_cast<__nv_bfloat16*>(dH + r0 * P.d));
      LMH_TRY(last_launch());
    }
  }
  if (dW || dW_acc || dw_scatter) {
    // Internal accumulator (several chunks, no caller dW_acc): store, add, ..., and the last
    // chunk adds and casts in its epilogue without writing the sum back. Caller's dW_acc:
    // add in every chunk (the first stores with LMH_F_DW_ACC_STORE), then cast it. One chunk
    // without dW_acc: bf16 tile sums directly.
    const bool last = chunk_idx == P.nchunks - 1;
    float* acc = dW_acc ? dW_acc : (P.acc ? ws.at<float>(P.o_acc) : nullptr);
    int acc_mode;
    if (dw_scatter) {  // one chunk: fp32 rows to the reducing ranks (no output map)
      acc_mode = 4;
    } else if (!acc) {
      acc_mode = 0;
    } else if (dW_acc) {
      const bool first_store = P.acc_store && chunk_idx == 0;
      // the last chunk adds, stores the sum and casts it in one pass, unless it is also the
      // stored first chunk (then: store, and the cast below)
      acc_mode = (dW && last && !first_store) ? 5 : (first_store ? 1 : 2);
    } else {
      acc_mode = chunk_idx == 0 ? 1 : (last ? 3 : 2);
    }
    if (acc_mode == 0 && rows >= kDwWideRows)
      LMH_TRY(run_dw<EpiDWWide>(P, dev, sms, G, H, r0, rows, acc_mode, acc, dW, dw_scatter, ws,
                                st));
    else
      LMH_TRY(run_dw<EpiDW>(P, dev, sms, G, H, r0, rows, acc_mode, acc, dW, dw_scatter, ws, st));
    if (dW_acc && dW && last && acc_mode != 5) LMH_TRY(cast_dw(P, acc, dW, st));
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
      dW_acc ? (P.acc_store ? 1 : 2) : 0, reinterpret_cast<__nv_bfloat16*>(dW));
  return last_launch();
}

// Outputs of a call without rows: zero counts / means, dW = cast of the given accumulator
// (zeroed first with LMH_F_DW_ACC_STORE: the call's dW is zero).
lmh_status empty_call(const Plan& P, float* mean_out, int32_t* nvalid_out, lmh_bf16* dW,
                      float* dW_acc, cudaStream_t st) {
  if (mean_out && cudaMemsetAsync(mean_out, 0, 4, st) != cudaSuccess) return LMH_ERR_CUDA;
  if (nvalid_out && cudaMemsetAsync(nvalid_out, 0, 4, st) != cudaSuccess) return LMH_ERR_CUDA;
  if (dW_acc && P.acc_store &&
      cudaMemsetAsync(dW_acc, 0, static_cast<size_t>(P.V) * P.d * 4, st) != cudaSuccess)
    return LMH_ERR_CUDA;
  if (dW) {
    const int64_t n = P.V * P.d;
    if (dW_acc) return cast_dw(P, dW_acc, dW, st);
    if (cudaMemsetAsync(dW, 0, n * 2, st) != cudaSuccess) return LMH_ERR_CUDA;
  }
  return LMH_OK;
}

}  // namespace
