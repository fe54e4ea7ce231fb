// api_noalloc.cuh — lmh_logprob_noalloc, the log-prob entry whose scratch is a fixed device
// array of this library. Part of the one translation unit lmh_api.cu (included there once).
#pragma once

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
