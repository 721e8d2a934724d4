// Host-buffer forward + JVP whose device staging area is a fixed array inside
// the library (caj_attn_fwd_jvp_host_static in include/causaljvp.h).
//
// The ordinary host-buffer call takes its device workspace from the caller.
// Some callers have no way to obtain one: a plain C program or plugin that
// holds its tensors in host memory and links no device allocator, or a host
// runtime whose memory manager owns every device allocation and forbids
// cudaMalloc from its extensions. This file gives them the same call with the
// workspace taken from a file-scope __device__ array of a fixed size. Nothing
// here allocates: no cudaMalloc, no cudaFree, no allocating library routine.
//
// The array lives in every device that loads this module, for the life of the
// process. Its device address is looked up once per device with
// cudaGetSymbolAddress (in host code the symbol's name is only a host-side
// stand-in and must never be handed to a kernel).
#include "causaljvp.h"

#include <cuda_runtime.h>

#include <mutex>
#include <vector>

namespace {

constexpr size_t kScratchBytes = size_t(CAJ_HOST_STATIC_MAX_BYTES);

// The staging area: the six inputs, O, tO, LSE and tLSE of one call, laid out
// exactly as caj_attn_fwd_jvp_host lays out a caller's workspace. Every call
// overwrites what it reads back, so nothing needs to start at zero.
__device__ __align__(256) unsigned char g_host_scratch[kScratchBytes];

std::mutex g_scratch_mu;
std::vector<void *> g_scratch_addr;  // per device ordinal; null until looked up

// Device address of the staging area on the current device (looked up on the
// first call on each device, with that device current).
caj_status scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CAJ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (int(g_scratch_addr.size()) <= dev) g_scratch_addr.resize(dev + 1, nullptr);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_host_scratch) != cudaSuccess || !p) return CAJ_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return CAJ_OK;
}

}  // namespace

extern "C" caj_status caj_attn_fwd_jvp_host_static(const void *q, const void *k, const void *v,
                                                   const void *tq, const void *tk, const void *tv,
                                                   const caj_problem *prob, const caj_mask_desc *mask,
                                                   void *o, void *to, float *lse, float *tlse,
                                                   void *stream) {
  size_t need = 0;
  caj_status st = caj_attn_fwd_jvp_host_workspace(prob, &need);
  if (st != CAJ_OK) return st;
  if (need > kScratchBytes) return CAJ_ERR_UNSUPPORTED;  // problem too large for the fixed area
  void *ws = nullptr;
  st = scratch_address(&ws);
  if (st != CAJ_OK) return st;
  return caj_attn_fwd_jvp_host(q, k, v, tq, tk, tv, prob, mask, o, to, lse, tlse, ws, kScratchBytes,
                               stream);
}
