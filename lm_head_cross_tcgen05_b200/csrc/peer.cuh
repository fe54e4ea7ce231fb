// peer.cuh — the stream-ordered barrier that orders the peer-memory exchanges of the
// multi-rank steps (a rank's GEMM epilogue stores rows into another rank's receive buffer;
// that rank may reduce the buffer only after every rank's stores have landed).
//
// Each rank owns a signal array of R uint32 words, which every rank can write (peer-mapped
// memory over NVLink, zeroed once before the first barrier). Barrier number e (1, 2, 3, ...,
// the same sequence on every rank) stores e into word `rank` of every rank's array, then waits
// until every word of this rank's own array has reached e. The wait is bounded by
// %globaltimer: on expiry it sets kErrTimeout in the error word and the kernel returns, so a
// rank that never arrives costs the others one time-out, never a hung GPU.
#pragma once

#include "sm100.cuh"

namespace lmh {

__device__ __forceinline__ void st_release_sys_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_sys_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// One block of at least R threads. Thread j signals rank j and then waits for rank j's word.
// Epochs are compared wrap-safe (a peer may already be one barrier ahead).
__global__ void peer_barrier_kernel(uint32_t* const* __restrict__ signals, int R, int rank,
                                    uint32_t epoch, uint64_t timeout_ns, uint32_t* err) {
  const int j = threadIdx.x;
  // Everything this rank wrote before the barrier on its stream (peer stores of an epilogue
  // included) is visible system-wide before any rank can observe the signal.
  __threadfence_system();
  __syncthreads();
  if (j < R) st_release_sys_u32(signals[j] + rank, epoch);
  if (j < R) {
    const uint32_t* mine = signals[rank] + j;
    const uint64_t t0 = global_timer_ns();
    while (static_cast<int32_t>(ld_acquire_sys_u32(mine) - epoch) < 0) {
      if (global_timer_ns() - t0 > timeout_ns) {
        atomicOr(err, kErrTimeout);
        break;
      }
      __nanosleep(128);
    }
  }
  __syncthreads();
  // What the peers wrote before their signals is visible to this rank's later kernels.
  __threadfence_system();
}

}  // namespace lmh
