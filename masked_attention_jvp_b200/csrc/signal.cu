// Stream-ordered barrier of the ranks of a context-parallel group over mapped
// signal words (caj_signal_barrier in include/causaljvp.h).
//
// The fused output all-to-all (caj_attn_fwd_jvp_scatter) stores rows straight
// into the other ranks' slice buffers. Each rank must know that no peer still
// reads its slice before the stores start, and that every peer's stores have
// landed before it copies its slice out. This kernel is that fence: rank r
// writes the call's epoch into word r of every rank's pad, then waits until
// every word of its own pad has reached the epoch. Every wait is bounded: on
// expiry the kernel records an error word that caj_last_device_status reports,
// and returns, so a rank that stalls or leaves ends its peers' barriers with
// an error status, never with a trap or a hang.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace caj {
namespace {

__device__ uint32_t g_signal_error = 0;

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void store_release_sys(uint32_t *addr, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t load_acquire_sys(const uint32_t *addr) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(addr) : "memory");
  return v;
}

// One block of kMaxShards threads; thread t < shards signals rank t and waits
// for rank t's signal.
__global__ void signal_barrier_kernel(SignalParams p) {
  const int t = threadIdx.x;
  if (t < p.shards) {
    // this rank's earlier work on the stream (the scattered stores) is ordered
    // before the signal that peers acquire
    __threadfence_system();
    store_release_sys(p.pads[t] + p.rank, p.epoch);
    const uint32_t *mine = p.pads[p.rank] + t;
    const uint64_t start = now_ns();
    // bounded by time and, should the timer misbehave, by a poll count as well
    for (uint32_t it = 0; int32_t(load_acquire_sys(mine) - p.epoch) < 0; ++it) {
      if (now_ns() - start > p.timeout_ns || it >= (1u << 30)) {
        atomicCAS(&g_signal_error, 0u, uint32_t(kErrTimeoutBase | kSiteSignalBarrier));
        break;
      }
      __nanosleep(128);
    }
    __threadfence_system();
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_signal_barrier(const SignalParams &p, cudaStream_t stream) {
  signal_barrier_kernel<<<1, kMaxShards, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t read_and_clear_signal_error(uint32_t *out) {
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_signal_error, sizeof(v));
  if (e == cudaSuccess && v) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_signal_error, &zero, sizeof(zero));
  }
  *out = v;
  return e;
}

}  // namespace caj
