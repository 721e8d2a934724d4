// Output projection of the attention block in primal-tangent form on B200
// tensor cores (sm_100a):
//   y = x W^T + b,   ty = tx W^T
// Causal-rCM runs the JVP layer by layer, each layer mapping a (primal, tangent)
// pair to a pair (section 3.2.2, "JVP FSDP2"). The projection is linear, so the
// tangent goes through the same weight without the bias.
//
// One persistent kernel does both products. The rows of x and tx form one
// operand of 2M rows, so every weight tile is used by the primal and the
// tangent rows alike while it sits in L2, and one launch covers both.
//
// Design (clusters of two CTAs, one CTA per SM, 6 warps per CTA):
//   Each CTA pair computes 256 x 256 output tiles with tcgen05 cta_group::2:
//   CTA r of the pair loads rows [128 r, +128) of the A tile (x or tx) and rows
//   [128 r, +128) of the B tile (half of the tile's 256 weight rows) into its
//   own shared memory; the pair's leader (r = 0) issues one M = 256, N = 256
//   product per 16-wide K step that reads both CTAs' halves, and each CTA's
//   tensor memory receives its own 128 rows of the result. Per CTA and 64-wide
//   K block that is 32 KiB of copies for 4.2 MFLOP, against 48 KiB for a single
//   CTA's 128 x 256 tile, so L2 -> SM traffic drops by a third and the ring
//   holds 6 stages. No copy is multicast: each CTA loads only its own halves;
//   both CTAs' copies complete on the leader's barrier.
//   warp 0      TMA producer (both CTAs).
//   warp 1      tcgen05 MMA issuer (the leader's elected lane); both CTAs'
//               warp 1 allocate and free the pair's tensor memory. fp32
//               accumulators are double-buffered in TMEM (2 x 256 columns) so
//               the epilogue of one tile overlaps the products of the next.
//   warps 2-5   epilogue (both CTAs): warp w reads TMEM lanes [32 (w%4), +32),
//               i.e. 32 rows of the CTA's half, 64 columns at a time; adds the
//               bias (primal rows only), rounds to bf16, writes a
//               128-byte-swizzled staging tile and stores it with a TMA tile
//               store (two staging buffers per warp).
// Tiles (which of x / tx, 256-row block, 256-column block) are visited with the
// column block fastest, so the column blocks of one row block run at about the
// same time on neighbouring SMs and the row block is read from DRAM once.
// Measured against a single-CTA 128 x 256 version of the same kernel on the
// Wan-1.3B projection (M = 65520 tokens, K = C = 1536, best of rounds): 0.418
// against 0.453 ms; PyTorch's cuBLAS matmuls on the same tensors took 0.432 ms.
//
// Every mbarrier wait is bounded: on expiry the kernel records an error code,
// drains its in-flight copies, products and stores, frees TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "ptx_sm100.cuh"

namespace caj {
namespace {

using namespace ptx;

__device__ uint32_t g_proj_error = 0;

constexpr int PM = 128;          // rows of a CTA's half tile (TMEM lanes)
constexpr int PN = 256;          // columns of a tile (one MMA's N)
constexpr int PK = 64;           // K per stage: one 128-byte swizzle atom of bf16
constexpr int kStages = 6;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr uint32_t A_BYTES = PM * PK * 2;                 // this CTA's 128 A rows, 16 KiB
constexpr uint32_t B_BYTES = (PN / 2) * PK * 2;           // this CTA's 128 B rows, 16 KiB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int OUT_ROWS = 32, OUT_COLS = 64;               // one epilogue warp's store box
constexpr uint32_t OUT_BYTES = OUT_ROWS * OUT_COLS * 2;   // 4 KiB
constexpr int kOutBufs = 2;
constexpr uint32_t OFF_OUT = kStages * STAGE_BYTES;
constexpr uint32_t OFF_BAR = OFF_OUT + kEpiWarps * kOutBufs * OUT_BYTES;
// barriers: full[kStages] (the leader's count both CTAs' copies), empty[kStages],
// acc_full[2], acc_empty[2] (the leader's: both CTAs' epilogue warps arrive),
// drain; then the TMEM base address and the abort flag
constexpr uint32_t BAR_FULL = 0, BAR_EMPTY = 8 * kStages, BAR_ACC_FULL = 16 * kStages,
                   BAR_ACC_EMPTY = BAR_ACC_FULL + 16, BAR_DRAIN = BAR_ACC_EMPTY + 16,
                   OFF_TMEM_SLOT = BAR_DRAIN + 8, OFF_ABORT = OFF_TMEM_SLOT + 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + OFF_ABORT + 4 + 1024;  // + slack for the 1 KiB alignment
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
constexpr uint32_t kTmemCols = 2 * PN;

// wait sites (low byte of the error code)
enum : uint32_t { kSiteEmpty = 1, kSiteFull = 2, kSiteAccEmpty = 3, kSiteAccFull = 4 };

__device__ __noinline__ void raise_proj_error(volatile int *abort_flag, uint32_t code) {
  atomicCAS(&g_proj_error, 0u, code);
  *abort_flag = 1;
}

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                             uint64_t timeout_ns, uint32_t site) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1; it < 0x40000000u; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > timeout_ns) {
        raise_proj_error(abort_flag, kErrTimeoutBase | site);
        return false;
      }
    }
  }
  raise_proj_error(abort_flag, kErrTimeoutBase | site);
  return false;
}

// Ignores the abort flag: only drains this CTA's own copies and products.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1; it < 0x40000000u; ++it) {
    if (mbar_try_wait(bar, parity)) return;
    if ((it & 31u) == 0 && globaltimer_ns() - t0 > timeout_ns) return;
  }
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          uint64_t timeout_ns, uint32_t site) {
  return __all_sync(0xffffffffu, wait_bounded(bar, parity, abort_flag, timeout_ns, site));
}

// 2-D tile store shared -> global (rows and columns past the tensor are not written).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *m, uint32_t src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N committed store groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t n_clusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// The shared::cluster address of this CTA's shared-memory word `saddr` in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 2-D tile load into this CTA's shared memory whose completion is counted on an
// mbarrier of either CTA of the pair (`bar` a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t pred, uint32_t dst, const CUtensorMap *m,
                                                 uint32_t bar, int32_t x, int32_t y) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %0, 0;\n\t"
      "@p cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%1], [%2, {%4, %5}], [%3];\n\t}" ::"r"(pred), "r"(dst), "l"(reinterpret_cast<uint64_t>(m)),
      "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void mma_ss_pair(uint32_t pred, uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "setp.ne.b32 q, %0, 0;\n\t"
      "@q tcgen05.mma.cta_group::2.kind::f16 [%1], %2, %3, %4, p;\n\t}" ::"r"(pred),
      "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the mbarrier at offset `bar` of BOTH CTAs of the pair when the
// pair's products issued so far are done (a commit, not a copy).
__device__ __forceinline__ void tc_commit_pair(uint32_t pred, uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %0, 0;\n\t"
      "@p tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%1], %2;\n\t}" ::"r"(
          pred),
      "r"(bar), "h"(uint16_t(3))
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster_addr) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
    out_proj_sm100_kernel(const __grid_constant__ OutProjParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t *sgen = smem_raw + (sbase - raw);
  const uint32_t bars = sbase + OFF_BAR;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sgen + OFF_BAR + OFF_ABORT);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sgen + OFF_BAR + OFF_TMEM_SLOT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();               // 0: the pair's leader
  const int32_t pair = int32_t(cluster_id_x()), n_pairs = int32_t(n_clusters_x());

  const int32_t m_blocks = (p.M + 2 * PM - 1) / (2 * PM);   // 256-row blocks per operand
  const int32_t n_blocks = (p.C + PN - 1) / PN;
  const int32_t k_blocks = (p.K + PK - 1) / PK;
  const int32_t n_tiles = 2 * m_blocks * n_blocks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars + BAR_FULL + 8 * s, 1);
      mbar_init(bars + BAR_EMPTY + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bars + BAR_ACC_FULL + 8 * b, 1);
      mbar_init(bars + BAR_ACC_EMPTY + 8 * b, 2 * kEpiWarps);  // both CTAs' epilogue warps
    }
    mbar_init(bars + BAR_DRAIN, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.tm_x);
    prefetch_tmap(&p.tm_tx);
    prefetch_tmap(&p.tm_w);
    prefetch_tmap(&p.tm_y);
    prefetch_tmap(&p.tm_ty);
  }
  if (warp == 1) {  // both CTAs, same warp, same slot: one allocation for the pair
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (both CTAs)
    const uint32_t leader = elect_one();
    uint32_t stage = 0, phase = 0, issued = 0;
    bool ok = true;
    for (int32_t t = pair; ok && t < n_tiles; t += n_pairs) {
      const int32_t nb = t % n_blocks, rest = t / n_blocks, which = rest / m_blocks;
      const int32_t a_row = (rest % m_blocks) * 2 * PM + int32_t(rank) * PM;
      const int32_t b_row = nb * PN + int32_t(rank) * (PN / 2);
      const CUtensorMap *am = which ? &p.tm_tx : &p.tm_x;
      for (int32_t kb = 0; kb < k_blocks; ++kb) {
        if (!warp_wait(bars + BAR_EMPTY + 8 * stage, phase ^ 1u, abort_flag, p.timeout_ns, kSiteEmpty)) {
          ok = false;
          break;
        }
        if (p.fault_mode == 0) {
          const uint32_t sa = sbase + stage * STAGE_BYTES, sb = sa + A_BYTES;
          const uint32_t fb = map_to_rank(bars + BAR_FULL + 8 * stage, 0);  // the leader's barrier
          if (rank == 0) mbar_arrive_expect_tx_if(leader, bars + BAR_FULL + 8 * stage, 2 * STAGE_BYTES);
          tma_load_2d_pair(leader, sa, am, fb, kb * PK, a_row);
          tma_load_2d_pair(leader, sb, &p.tm_w, fb, kb * PK, b_row);
          ++issued;
        }
        __syncwarp();
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok && leader && rank == 0) {  // the leader's barriers count both CTAs' copies
      const uint32_t inflight = issued < uint32_t(kStages) ? issued : uint32_t(kStages);
      uint32_t s = stage, ph = phase;
      for (uint32_t i = 0; i < inflight; ++i) {
        if (s == 0) {
          s = kStages;
          ph ^= 1u;
        }
        --s;
        drain_wait(bars + BAR_FULL + 8 * s, ph, p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // ------------------------------------------------ MMA issuer (leader only)
      const uint32_t leader = elect_one();
      constexpr uint32_t IDESC = idesc_bf16_f32(2 * PM, PN, 0);
      uint32_t stage = 0, phase = 0, tcount = 0;
      bool ok = true;
      for (int32_t t = pair; ok && t < n_tiles; t += n_pairs, ++tcount) {
        const uint32_t buf = tcount & 1u, use = tcount >> 1;
        if (!warp_wait(bars + BAR_ACC_EMPTY + 8 * buf, (use & 1u) ^ 1u, abort_flag, p.timeout_ns, kSiteAccEmpty)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + buf * PN;
        for (int32_t kb = 0; kb < k_blocks; ++kb) {
          if (!warp_wait(bars + BAR_FULL + 8 * stage, phase, abort_flag, p.timeout_ns, kSiteFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + stage * STAGE_BYTES, sb = sa + A_BYTES;
          const uint64_t da = sdesc_sw128(sa, 16, 1024), db = sdesc_sw128(sb, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < PK / 16; ++kk)
            mma_ss_pair(leader, d_tmem, da + uint64_t(kk * 2), db + uint64_t(kk * 2), IDESC, (kb | kk) != 0);
          tc_commit_pair(leader, bars + BAR_EMPTY + 8 * stage);  // both CTAs' stage is free
          __syncwarp();
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(leader, bars + BAR_ACC_FULL + 8 * buf);   // both CTAs' accumulator half is complete
        __syncwarp();
      }
      tc_commit_pair(leader, bars + BAR_DRAIN);
      __syncwarp();
      if (leader) drain_wait(bars + BAR_DRAIN, 0, p.timeout_ns);
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int ew = warp - 2;
    const uint32_t lane_taddr = tmem + (uint32_t(32 * q) << 16);
    const uint32_t stage_base = sbase + OFF_OUT + uint32_t(ew) * kOutBufs * OUT_BYTES;
    const uint32_t acc_empty_leader = map_to_rank(bars + BAR_ACC_EMPTY, 0);
    uint32_t tcount = 0, chunk_count = 0;
    for (int32_t t = pair; t < n_tiles; t += n_pairs, ++tcount) {
      const int32_t nb = t % n_blocks, rest = t / n_blocks, which = rest / m_blocks;
      const int32_t m0 = (rest % m_blocks) * 2 * PM + int32_t(rank) * PM, n0 = nb * PN;
      const uint32_t buf = tcount & 1u, use = tcount >> 1;
      if (!warp_wait(bars + BAR_ACC_FULL + 8 * buf, use & 1u, abort_flag, p.timeout_ns, kSiteAccFull)) break;
      tc_fence_after();
      const int32_t row0 = m0 + 32 * q;
      const bool rows_in = row0 < p.M;
      const bool primal = which == 0 && p.bias != nullptr;
      const CUtensorMap *om = which ? &p.tm_ty : &p.tm_y;
#pragma unroll 1
      for (int c = 0; c < PN / OUT_COLS; ++c) {
        uint32_t ra[32], rb[32];
        tmem_ld32x2(lane_taddr + buf * PN + c * OUT_COLS, lane_taddr + buf * PN + c * OUT_COLS + 32, ra, rb);
        if (c == PN / OUT_COLS - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(acc_empty_leader + 8 * buf);
        }
        const int32_t col0 = n0 + c * OUT_COLS;
        if (!rows_in || col0 >= p.C) continue;
        if (primal) {
          const uint4 *bp = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.bias) + col0);
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            if (col0 + 8 * g < p.C) {
              const uint4 bw = __ldg(bp + g);
              uint32_t *acc = g < 4 ? ra + 8 * g : rb + 8 * (g - 4);
              const uint32_t w4[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                acc[2 * e] = __float_as_uint(__uint_as_float(acc[2 * e]) + bf16_lo(w4[e]));
                acc[2 * e + 1] = __float_as_uint(__uint_as_float(acc[2 * e + 1]) + bf16_hi(w4[e]));
              }
            }
          }
        }
        const uint32_t sb_idx = chunk_count & 1u;
        if (lane == 0) bulk_wait_read<kOutBufs - 1>();
        __syncwarp();
        const uint32_t sbuf = stage_base + sb_idx * OUT_BYTES;
        const uint32_t row_addr = sbuf + uint32_t(lane) * 128u;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t *src = u < 4 ? ra + 8 * u : rb + 8 * (u - 4);
          const uint32_t w0 = pack_bf16(__uint_as_float(src[0]), __uint_as_float(src[1]));
          const uint32_t w1 = pack_bf16(__uint_as_float(src[2]), __uint_as_float(src[3]));
          const uint32_t w2 = pack_bf16(__uint_as_float(src[4]), __uint_as_float(src[5]));
          const uint32_t w3 = pack_bf16(__uint_as_float(src[6]), __uint_as_float(src[7]));
          const uint32_t dst = row_addr + ((uint32_t(u) ^ (uint32_t(lane) & 7u)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w0), "r"(w1), "r"(w2),
                       "r"(w3)
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(om, sbuf, col0, row0);
          bulk_commit();
        }
        __syncwarp();
        ++chunk_count;
      }
    }
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }

  // neither CTA leaves while the pair's products may still read its shared
  // memory or the peer may still signal its barriers
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}
}  // namespace

cudaError_t launch_out_proj_sm100(const OutProjParams &p, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(2);
  // Per device, once: the shared-memory limit and how many CTA pairs fit at a
  // time (the persistent grid).
  static std::atomic<uint64_t> set_up{0};
  static std::atomic<int> max_pairs_of[64];
  e = once_per_device(set_up, [&] {
    cudaError_t r = cudaFuncSetAttribute(out_proj_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM_BYTES);
    int sms = 0, pairs = 0;
    if (r == cudaSuccess) r = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (r == cudaSuccess) r = cudaOccupancyMaxActiveClusters(&pairs, out_proj_sm100_kernel, &cfg);
    if (r == cudaSuccess && dev < 64) max_pairs_of[dev].store(pairs >= 1 ? pairs : sms / 2);
    return r;
  });
  if (e != cudaSuccess) return e;
  const int max_pairs = dev < 64 ? max_pairs_of[dev].load() : 74;
  const int64_t m_blocks = (p.M + 2 * PM - 1) / (2 * PM), n_blocks = (p.C + PN - 1) / PN;
  const int64_t tiles = 2 * m_blocks * n_blocks;
  const int64_t pairs = tiles < max_pairs ? tiles : max_pairs;
  cfg.gridDim = dim3(unsigned(2 * pairs));
  e = cudaLaunchKernelEx(&cfg, out_proj_sm100_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t read_and_clear_proj_error(uint32_t *out) {
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_proj_error, sizeof(v));
  if (e == cudaSuccess && v) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_proj_error, &zero, sizeof(zero));
  }
  *out = v;
  return e;
}

}  // namespace caj
