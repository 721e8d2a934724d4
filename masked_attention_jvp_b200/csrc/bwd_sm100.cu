// Backward of the primal block-causal attention on B200 tensor cores (sm_100a).
//
// The student's gradient step in TF-sCM backpropagates through the masked
// attention forward; the JVP branch is stop-gradient (Causal-rCM, appendix A)
// and needs no backward. With P_ij = exp(scale <q_i,k_j> - LSE_i) on visible
// pairs, the gradients are
//   dV_j = sum_i P_ij dO_i,        dP_ij = <dO_i, v_j>,   Delta_i = <dO_i, O_i>
//   dS_ij = P_ij (dP_ij - Delta_i),  dQ_i = scale sum_j dS_ij k_j,
//   dK_j = scale sum_i dS_ij q_i.
// Three kernels, no atomics, deterministic:
//   delta      Delta_i = <dO_i, O_i> (HBM-bound pre-pass, also an output);
//   dq         one CTA per 128-query tile, streams the visible key tiles:
//              S = Q K^T and dP = dO V^T (tcgen05, TMEM), dS in registers,
//              dQ += dS K with dS read back from TMEM;
//   dkdv       one CTA per 128-key tile, streams the query tiles that see it
//              (the transposed block-causal schedule): S^T = K Q^T and
//              dP^T = V dO^T, then dV += P^T dO and dK += dS^T Q.
// Both main kernels reuse the forward kernel's organisation: warp 0 issues TMA
// copies, warp 1 the MMAs (elected lane, warp-uniform loop). Warps 2-9 form two
// warpgroups that each take one 32-column half of every 64-column tile. P and
// dS are written back to TMEM as bf16 over the columns their thread read. (Four
// warpgroups of 16 columns each, 576 threads, measured 8% slower: the softmax
// is bound by the exponential unit and by fixed load/store/barrier latencies,
// which more warps do not shorten, and the extra warps share sub-partitions
// with the copy and MMA warps.)
// The CTA's own 128 rows that serve as the A operand of the score products
// (Q and dO in dq, K in dkdv) are copied once into TMEM by the softmax warps,
// so those N = 64 products read only the streamed 64-row tile from shared
// memory: shared-memory bandwidth, not the tensor core, bounded them when A
// came from shared memory too. (Writing dS to a TMEM area of its own, so the
// next scores need not wait for the dQ product, measured 14% slower: it left no
// TMEM for the operands above, and the products they feed went back to
// reading both operands from shared memory.)
// Every mbarrier wait is bounded; on expiry the kernel records an error code,
// drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "mask_schedule.h"
#include "ptx_sm100.cuh"

namespace caj {

__device__ uint32_t g_bwd_device_error = 0;

namespace {

using namespace ptx;

constexpr int BM = 128;  // rows owned by a CTA (queries for dq, keys for dkdv)
constexpr int BN = 64;   // streamed tile width (keys for dq, queries for dkdv)
constexpr int kGroups = 2;                  // softmax warpgroups
constexpr int kCols = BN / kGroups;         // tile columns per warpgroup
constexpr int kSoftmaxWarps = 4 * kGroups;
constexpr int kThreads = 64 + 32 * kSoftmaxWarps;
constexpr uint32_t kColMask = kCols == 32 ? 0xffffffffu : (1u << kCols) - 1u;

// TMEM column offset of the packed bf16 pairs of tile columns [16 kk, 16 kk + 16)
// inside a buffer, when warpgroup g packs its kCols columns at g * kCols.
__host__ __device__ constexpr uint32_t packed_col(int kk) {
  return uint32_t((16 * kk / kCols) * kCols + (16 * kk % kCols) / 2);
}
constexpr float kLog2e = 1.4426950408889634f;

__device__ __noinline__ void bwd_raise(volatile int *abort_flag, uint32_t code) {
  atomicCAS(&g_bwd_device_error, 0u, code);
  *abort_flag = 1;
}

__device__ __forceinline__ bool bwait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                      uint64_t timeout_ns, uint32_t site) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1; it < 0x40000000u; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > timeout_ns) {
        bwd_raise(abort_flag, kErrTimeoutBase | site);
        return false;
      }
    }
  }
  bwd_raise(abort_flag, kErrTimeoutBase | site);
  return false;
}

__device__ __forceinline__ bool bwarp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                           uint64_t timeout_ns, uint32_t site) {
  return __all_sync(0xffffffffu, bwait(bar, parity, abort_flag, timeout_ns, site));
}

// Bounded wait of the MMA warp, with no warp vote (see the forward kernels: a
// vote after queued tensor-core instructions holds the warp until the queue
// takes them); the warp reconverges after its loop.
__device__ __forceinline__ bool bissuer_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                             uint64_t timeout_ns, uint32_t site) {
  return bwait(bar, parity, abort_flag, timeout_ns, site);
}

__device__ __forceinline__ void bdrain(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1; it < 0x40000000u; ++it) {
    if (mbar_try_wait(bar, parity)) return;
    if ((it & 31u) == 0 && globaltimer_ns() - t0 > timeout_ns) return;
  }
}

__device__ __forceinline__ uint32_t bits_in(int32_t lo, int32_t hi) {
  lo = max(lo, 0);
  hi = min(hi, 32);
  if (hi <= lo) return 0u;
  return uint32_t(((1ull << hi) - 1ull) & ~((1ull << lo) - 1ull));
}

// Up to three ascending tile ranges, held in registers (the schedule functions
// fill an array with computed indices, which would otherwise live in local
// memory and be re-read for every tile).
struct TileRanges {
  int32_t s0, n0, s1, n1, s2;  // starts of the ranges; lengths of the first two
  __device__ __forceinline__ explicit TileRanges(const int32_t (&t)[6])
      : s0(t[0]), n0(t[1] - t[0]), s1(t[2]), n1(t[3] - t[2]), s2(t[4]) {}
};

// Tile index of the j-th visited tile.
__device__ __forceinline__ int32_t nth_tile(int32_t j, const TileRanges &r) {
  if (j < r.n0) return r.s0 + j;
  if (j < r.n0 + r.n1) return r.s1 + (j - r.n0);
  return r.s2 + (j - r.n0 - r.n1);
}

// TMEM accesses of 8, 16 or 32 columns, chosen by the register array's size.
__device__ __forceinline__ void tmem_ld_pair(uint32_t a, uint32_t b, uint32_t (&x)[16], uint32_t (&y)[16]) {
  tmem_ld16x2(a, b, x, y);
}
__device__ __forceinline__ void tmem_ld_pair(uint32_t a, uint32_t b, uint32_t (&x)[32], uint32_t (&y)[32]) {
  tmem_ld32x2(a, b, x, y);
}
__device__ __forceinline__ void tmem_ld_cols(uint32_t a, uint32_t (&x)[16]) { tmem_ld16(a, x); }
__device__ __forceinline__ void tmem_ld_cols(uint32_t a, uint32_t (&x)[32]) { tmem_ld32(a, x); }
__device__ __forceinline__ void tmem_st_cols(uint32_t a, const uint32_t (&x)[8]) { tmem_st8(a, x); }
__device__ __forceinline__ void tmem_st_cols(uint32_t a, const uint32_t (&x)[16]) { tmem_st16(a, x); }
__device__ __forceinline__ void tmem_st_cols(uint32_t a, const uint32_t (&x)[32]) { tmem_st32(a, x); }

// NRES: resident 128-row tiles kept in shared memory (0 in dq, V in dkdv).
template <int D, int NRES>
struct BCfg {
  static constexpr int NB = D / 64;          // 128-byte column blocks per row
  static constexpr int RBLK = BM * 128;      // one column block of a resident 128-row tile
  static constexpr int SBLK = BN * 128;      // one column block of a streamed 64-row tile
  static constexpr int R_BYTES = NB * RBLK;  // a resident 128 x D tile
  static constexpr int S_BYTES = NB * SBLK;  // a streamed 64 x D tile
  static constexpr int STAGES = 4;
  // stage: two streamed tiles + 2 x 64 fp32 row statistics (dkdv), padded so
  // every stage starts on a 1 KiB boundary (128-byte swizzle)
  static constexpr int STAGE = 2 * S_BYTES + 1024;
  static constexpr int OFF_R = 0;
  static constexpr int OFF_ST = NRES * R_BYTES;
  static constexpr int OFF_BAR = OFF_ST + STAGES * STAGE;
  // barriers: a_ready, r_full, st_full[S], st_empty[S], s_full[2], p_full[2],
  // o_done[2], drain, dp_free
  static constexpr int NBAR = 2 + 2 * STAGES + 8;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static_assert(SMEM_BYTES <= 232448, "shared memory overflow");
  static constexpr uint32_t TMEM_COLS = 512;
};

struct BBars {
  uint32_t a_ready, r_full, st_full, st_empty, s_full, p_full, o_done, drain, dp_free;
};

template <int STAGES>
__device__ __forceinline__ BBars bbars(uint32_t base) {
  BBars b;
  b.a_ready = base;
  b.r_full = base + 8;
  b.st_full = base + 16;
  b.st_empty = b.st_full + 8 * STAGES;
  b.s_full = b.st_empty + 8 * STAGES;
  b.p_full = b.s_full + 16;
  b.o_done = b.p_full + 16;
  b.drain = b.o_done + 16;
  b.dp_free = b.drain + 8;
  return b;
}

// Copies part g (of kGroups) of this thread's bf16 row into TMEM as packed
// pairs: column taddr + i holds elements (2i, 2i+1) of the row, the layout in
// which the tensor core reads an A operand from TMEM (one 16-element K step per
// 8 columns). Rows past the sequence are zero, as a TMA copy would fill them.
template <int D>
__device__ __forceinline__ void row_to_tmem(const uint16_t *row, bool live, uint32_t taddr, int g) {
  constexpr int W = D / (2 * kGroups);  // 32-bit words in one part of a row
  static_assert(W % 4 == 0 && W >= 8, "row part must be whole 16-byte loads and >= 8 columns");
  uint32_t w[W];
  const uint4 *s4 = reinterpret_cast<const uint4 *>(row) + g * (W / 4);
#pragma unroll
  for (int v = 0; v < W / 4; ++v) {
    const uint4 x = live ? __ldg(s4 + v) : make_uint4(0u, 0u, 0u, 0u);
    w[4 * v] = x.x;
    w[4 * v + 1] = x.y;
    w[4 * v + 2] = x.z;
    w[4 * v + 3] = x.w;
  }
  tmem_st_cols(taddr + g * W, w);
}

// Shared prologue of both kernels: barriers, TMEM, error checks. Returns false
// when the CTA must return at once.
template <class C>
__device__ __forceinline__ bool bwd_setup(uint32_t sbase, uint8_t *sgen, const BBars &bar,
                                          int warp) {
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sgen + C::OFF_MISC + 4);
  if (threadIdx.x == 0) {
    mbar_init(bar.a_ready, kSoftmaxWarps);
    mbar_init(bar.r_full, 1);
    mbar_init(bar.dp_free, kSoftmaxWarps);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar.st_full + 8 * s, 1);
      mbar_init(bar.st_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar.s_full + 8 * b, 1);
      mbar_init(bar.p_full + 8 * b, kSoftmaxWarps);
      mbar_init(bar.o_done + 8 * b, 1);
    }
    mbar_init(bar.drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sbase + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return true;
}

// ============================================================== dQ kernel
template <int D>
__global__ void __launch_bounds__(kThreads, 1) bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  using C = BCfg<D, 0>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicCAS(&g_bwd_device_error, 0u, uint32_t(kErrSmemMisaligned));
    return;
  }
  uint8_t *sgen = smem_raw;
  const BBars bar = bbars<C::STAGES>(sbase + C::OFF_BAR);
  volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sgen + C::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sgen + C::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int32_t bh = blockIdx.x / p.n_row_tiles;
  const int32_t qt = p.row_order[blockIdx.x % p.n_row_tiles];
  const int32_t q0 = qt * BM, q1 = min(q0 + BM, p.geom.N);
  int32_t tr[6];
  const int32_t ntiles = qtile_key_tiles(p.geom, q0, q1, BN, tr[0], tr[1], tr[2], tr[3]);
  tr[4] = tr[5] = tr[3];
  const TileRanges t(tr);

  bwd_setup<C>(sbase, sgen, bar, warp);
  const uint32_t tmem = *tmem_slot;
  // TMEM: dQ accumulator [0, D) | Q [D, 3D/2) | dO [3D/2, 2D) (packed bf16, the
  // A operands of the score products) | buffer b: S [2D + 128b, +64), dP [+64, +128)
  constexpr uint32_t COL_Q = D, COL_DO = D + D / 2, COL_S0 = 2 * D;
  static_assert(COL_S0 + 256 <= C::TMEM_COLS, "TMEM overflow");

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // (test hook, fault_mode 1: no copies at all, so the MMA warp's first
    // bounded wait runs out with nothing in flight)
    if (p.fault_mode != 1) {
      const uint32_t leader = elect_one();
      int32_t armed = 0;
      for (int32_t j = 0; j < ntiles; ++j) {
        const int s = j % C::STAGES;
        if (j >= C::STAGES && !bwarp_wait(bar.st_empty + 8 * s, ((j / C::STAGES) - 1) & 1, abort_flag,
                                          p.timeout_ns, 21))
          break;
        const int32_t key0 = nth_tile(j, t) * BN;
        const uint32_t dst = sbase + C::OFF_ST + s * C::STAGE, fb = bar.st_full + 8 * s;
        mbar_arrive_expect_tx_if(leader, fb, 2 * C::S_BYTES);
#pragma unroll
        for (int c = 0; c < C::NB; ++c) {
          tma_load_3d(leader, dst + c * C::SBLK, &p.tm_k_s, fb, c * 64, key0, bh);
          tma_load_3d(leader, dst + C::S_BYTES + c * C::SBLK, &p.tm_v_s, fb, c * 64, key0, bh);
        }
        armed = j + 1;
      }
      for (int32_t j = (armed > C::STAGES ? armed - C::STAGES : 0); j < armed; ++j)
        bdrain(bar.st_full + 8 * (j % C::STAGES), (j / C::STAGES) & 1, p.timeout_ns);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    const uint32_t leader = elect_one();
    constexpr uint32_t ID_S = idesc_bf16_f32(BM, BN, 0);  // Q K^T, dO V^T
    constexpr uint32_t ID_Q = idesc_bf16_f32(BM, D, 1);   // dS K, K read MN-major
    const uint64_t dK0 = sdesc_sw128(sbase + C::OFF_ST, 16, 1024);
    const uint64_t dV0 = sdesc_sw128(sbase + C::OFF_ST + C::S_BYTES, 16, 1024);
    const uint64_t dKmn0 = sdesc_sw128(sbase + C::OFF_ST, C::SBLK, 1024);
    bool ok = bissuer_wait(bar.a_ready, 0, abort_flag, p.timeout_ns, 22);
    tc_fence_after();
    for (int32_t j = 0; ok && j <= ntiles; ++j) {
      if (j < ntiles) {
        const int s = j % C::STAGES;
        if (!(ok = bissuer_wait(bar.st_full + 8 * s, (j / C::STAGES) & 1, abort_flag, p.timeout_ns, 23)))
          break;
        const uint64_t so = uint64_t((s * C::STAGE) >> 4);
        const uint32_t cS = tmem + COL_S0 + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t st = uint64_t(((kk >> 2) * C::SBLK + (kk & 3) * 32) >> 4);
          mma_ts(leader, cS, tmem + COL_Q + 8 * kk, dK0 + so + st, ID_S, kk > 0 ? 1u : 0u);
          mma_ts(leader, cS + 64, tmem + COL_DO + 8 * kk, dV0 + so + st, ID_S, kk > 0 ? 1u : 0u);
        }
        tc_commit(leader, bar.s_full + 8 * (j & 1));
      }
      if (j >= 1) {
        const int32_t i = j - 1;
        if (!(ok = bissuer_wait(bar.p_full + 8 * (i & 1), (i >> 1) & 1, abort_flag, p.timeout_ns, 24)))
          break;
        tc_fence_after();
        const int s = i % C::STAGES;
        const uint64_t so = uint64_t((s * C::STAGE) >> 4);
        const uint32_t aS = tmem + COL_S0 + (i & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t pc = packed_col(kk);  // packed dS columns of keys 16kk..
          mma_ts(leader, tmem, aS + pc, dKmn0 + so + uint64_t((kk * 16 * 128) >> 4), ID_Q,
                 (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(leader, bar.o_done + 8 * (i & 1));
        tc_commit(leader, bar.st_empty + 8 * s);
      }
    }
    __syncwarp();  // lanes may leave the loop apart on an abort
    tc_commit(leader, bar.drain);
    bdrain(bar.drain, 0, p.timeout_ns);
  } else {
    // ------------------------------------------------- softmax + epilogue
    const int g = (warp - 2) >> 2, sub = warp & 3, row = sub * 32 + lane;
    const int32_t q = q0 + row;
    const uint32_t lane_addr = tmem + (uint32_t(sub * 32) << 16);
    const bool live = q < p.geom.N;
    const size_t ri = size_t(bh) * p.geom.N + (live ? q : 0);
    const float lse2 = live ? p.lse[ri] * kLog2e : 0.f;
    const float dl = live ? p.delta[ri] : 0.f;
    int32_t a0, b0, a1, b1;
    if (live) {
      row_key_ranges(p.geom, q, a0, b0, a1, b1);
    } else {
      a0 = 0; b0 = p.geom.N; a1 = b1 = 0;
    }
    const float sl2 = p.scale * kLog2e;
    {  // this thread's rows of Q and dO become the A operands in TMEM
      const size_t off = (size_t(bh) * p.geom.N + (live ? q : 0)) * D;
      row_to_tmem<D>(static_cast<const uint16_t *>(p.q) + off, live, lane_addr + COL_Q, g);
      row_to_tmem<D>(static_cast<const uint16_t *>(p.dout) + off, live, lane_addr + COL_DO, g);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.a_ready);
    }
    bool ok = true;
    for (int32_t j = 0; j < ntiles; ++j) {
      const int b = j & 1;
      if (!bwarp_wait(bar.s_full + 8 * b, (j >> 1) & 1, abort_flag, p.timeout_ns, 25)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int32_t kh = nth_tile(j, t) * BN + kCols * g;
      const uint32_t cS = lane_addr + COL_S0 + b * 128 + kCols * g;
      uint32_t rs[kCols], rp[kCols];
      tmem_ld_pair(cS, cS + 64, rs, rp);
      const uint32_t vis = (bits_in(a0 - kh, b0 - kh) | bits_in(a1 - kh, b1 - kh)) & kColMask;
      if (vis != kColMask) {  // hidden keys: p = 0 and no dP (select, NaN-safe)
#pragma unroll
        for (int i = 0; i < kCols; ++i) {
          const bool v = (vis >> i) & 1u;
          rs[i] = v ? rs[i] : __float_as_uint(-INFINITY);
          rp[i] = v ? rp[i] : __float_as_uint(dl);
        }
      }
      // element pairs in packed fp32x2 arithmetic (exponentials scalar)
      const uint64_t sl2x2 = f2(sl2, sl2), nlse2 = f2(-lse2, -lse2), dl2 = f2(dl, dl);
      uint32_t pk[kCols / 2];
#pragma unroll
      for (int i = 0; i < kCols / 2; ++i) {
        float xa, xb, da, db;
        f2_split(fma2(f2(__uint_as_float(rs[2 * i]), __uint_as_float(rs[2 * i + 1])), sl2x2, nlse2), xa, xb);
        const uint64_t p2 = f2(ex2(xa), ex2(xb));
        f2_split(mul2(p2, sub2(f2(__uint_as_float(rp[2 * i]), __uint_as_float(rp[2 * i + 1])), dl2)), da, db);
        pk[i] = pack_bf16(da, db);
      }
      tmem_st_cols(cS, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.p_full + 8 * b);
    }
    if (ok && ntiles > 0) {
      const int32_t last = ntiles - 1;
      if (bwarp_wait(bar.o_done + 8 * (last & 1), (last >> 1) & 1, abort_flag, p.timeout_ns, 26)) {
        tc_fence_after();
        uint4 *out = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.dq) + ri * D);
        constexpr int GC = D / kGroups, EC = GC < 32 ? GC : 32;  // columns per group, per load
#pragma unroll 1
        for (int c = g * GC; c < (g + 1) * GC; c += EC) {
          uint32_t r[EC];
          tmem_ld_cols(lane_addr + c, r);
          uint32_t po[EC / 2];
#pragma unroll
          for (int i = 0; i < EC / 2; ++i)
            po[i] = pack_bf16(__uint_as_float(r[2 * i]) * p.scale, __uint_as_float(r[2 * i + 1]) * p.scale);
          if (live) {
#pragma unroll
            for (int v = 0; v < EC / 8; ++v)
              out[c / 8 + v] = make_uint4(po[4 * v], po[4 * v + 1], po[4 * v + 2], po[4 * v + 3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ============================================================ dK dV kernel
template <int D>
__global__ void __launch_bounds__(kThreads, 1) bwd_dkdv_kernel(const __grid_constant__ BwdParams p) {
  using C = BCfg<D, 1>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicCAS(&g_bwd_device_error, 0u, uint32_t(kErrSmemMisaligned));
    return;
  }
  uint8_t *sgen = smem_raw;
  const BBars bar = bbars<C::STAGES>(sbase + C::OFF_BAR);
  volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sgen + C::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sgen + C::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int32_t bh = blockIdx.x / p.n_row_tiles;
  const int32_t kt = p.row_order[blockIdx.x % p.n_row_tiles];
  const int32_t k0 = kt * BM, k1 = min(k0 + BM, p.geom.N);
  int32_t tr[6];
  const int32_t ntiles = ktile_query_tiles(p.geom, k0, k1, BN, tr);
  const TileRanges t(tr);

  bwd_setup<C>(sbase, sgen, bar, warp);
  const uint32_t tmem = *tmem_slot;
  // TMEM: dV [0, D) | dK [D, 2D) | K [2D, 5D/2) (packed bf16, the A operand of
  // S^T) | buffer b: S^T [COL_S0 + 64b, +64), then P^T and dS^T packed over it
  // | dP^T [COL_S0 + 128, +64), one buffer, free once the softmax has read it
  constexpr uint32_t COL_K = 2 * D, COL_S0 = (5 * D / 2 + 63) / 64 * 64, COL_DP = COL_S0 + 128;
  static_assert(COL_DP + 64 <= C::TMEM_COLS, "TMEM overflow");

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // (test hook, fault_mode 1: no copies at all, so the MMA warp's first
    // bounded wait runs out with nothing in flight)
    if (p.fault_mode != 1) {
      const uint32_t leader = elect_one();
      mbar_arrive_expect_tx_if(leader, bar.r_full, C::R_BYTES);
      for (int c = 0; c < C::NB; ++c)
        tma_load_3d(leader, sbase + C::OFF_R + c * C::RBLK, &p.tm_v_r, bar.r_full, c * 64, k0, bh);
      int32_t armed = 0;
      for (int32_t j = 0; j < ntiles; ++j) {
        const int s = j % C::STAGES;
        if (j >= C::STAGES && !bwarp_wait(bar.st_empty + 8 * s, ((j / C::STAGES) - 1) & 1, abort_flag,
                                          p.timeout_ns, 31))
          break;
        const int32_t qb = nth_tile(j, t) * BN;
        const uint32_t dst = sbase + C::OFF_ST + s * C::STAGE, fb = bar.st_full + 8 * s;
        // row statistics of the 64 queries (LSE in base 2, Delta), +inf / 0 past N
        float *stat = reinterpret_cast<float *>(sgen + C::OFF_ST + s * C::STAGE + 2 * C::S_BYTES);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int32_t qi = qb + 32 * h + lane;
          const bool in = qi < p.geom.N;
          const size_t idx = size_t(bh) * p.geom.N + (in ? qi : 0);
          stat[32 * h + lane] = in ? p.lse[idx] * kLog2e : INFINITY;
          stat[64 + 32 * h + lane] = in ? p.delta[idx] : 0.f;
        }
        __syncwarp();
        mbar_arrive_expect_tx_if(leader, fb, 2 * C::S_BYTES);
#pragma unroll
        for (int c = 0; c < C::NB; ++c) {
          tma_load_3d(leader, dst + c * C::SBLK, &p.tm_q_s, fb, c * 64, qb, bh);
          tma_load_3d(leader, dst + C::S_BYTES + c * C::SBLK, &p.tm_do_s, fb, c * 64, qb, bh);
        }
        armed = j + 1;
      }
      bdrain(bar.r_full, 0, p.timeout_ns);
      for (int32_t j = (armed > C::STAGES ? armed - C::STAGES : 0); j < armed; ++j)
        bdrain(bar.st_full + 8 * (j % C::STAGES), (j / C::STAGES) & 1, p.timeout_ns);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    const uint32_t leader = elect_one();
    constexpr uint32_t ID_S = idesc_bf16_f32(BM, BN, 0);  // K Q^T, V dO^T
    constexpr uint32_t ID_A = idesc_bf16_f32(BM, D, 1);   // P^T dO, dS^T Q (B read MN-major)
    const uint64_t dV = sdesc_sw128(sbase + C::OFF_R, 16, 1024);
    const uint64_t dQ0 = sdesc_sw128(sbase + C::OFF_ST, 16, 1024);
    const uint64_t dO0 = sdesc_sw128(sbase + C::OFF_ST + C::S_BYTES, 16, 1024);
    const uint64_t dQmn0 = sdesc_sw128(sbase + C::OFF_ST, C::SBLK, 1024);
    const uint64_t dOmn0 = sdesc_sw128(sbase + C::OFF_ST + C::S_BYTES, C::SBLK, 1024);
    bool ok = bissuer_wait(bar.a_ready, 0, abort_flag, p.timeout_ns, 38) &&
              bissuer_wait(bar.r_full, 0, abort_flag, p.timeout_ns, 32);
    tc_fence_after();
    for (int32_t j = 0; ok && j <= ntiles; ++j) {
      if (j < ntiles) {
        const int s = j % C::STAGES;
        if (!(ok = bissuer_wait(bar.st_full + 8 * s, (j / C::STAGES) & 1, abort_flag, p.timeout_ns, 33)))
          break;
        const uint64_t so = uint64_t((s * C::STAGE) >> 4);
        const uint32_t cS = tmem + COL_S0 + (j & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t st = uint64_t(((kk >> 2) * C::SBLK + (kk & 3) * 32) >> 4);
          mma_ts(leader, cS, tmem + COL_K + 8 * kk, dQ0 + so + st, ID_S, kk > 0 ? 1u : 0u);
        }
        // dP^T has one buffer: the softmax must have read dP^T(j-1)
        if (j >= 1) {
          if (!(ok = bissuer_wait(bar.dp_free, (j - 1) & 1, abort_flag, p.timeout_ns, 39))) break;
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ro = uint64_t(((kk >> 2) * C::RBLK + (kk & 3) * 32) >> 4);
          const uint64_t st = uint64_t(((kk >> 2) * C::SBLK + (kk & 3) * 32) >> 4);
          mma_ss(leader, tmem + COL_DP, dV + ro, dO0 + so + st, ID_S, kk > 0 ? 1u : 0u);
        }
        tc_commit(leader, bar.s_full + 8 * (j & 1));
      }
      if (j >= 1) {
        const int32_t i = j - 1;
        if (!(ok = bissuer_wait(bar.p_full + 8 * (i & 1), (i >> 1) & 1, abort_flag, p.timeout_ns, 34)))
          break;
        tc_fence_after();
        const int s = i % C::STAGES;
        const uint64_t so = uint64_t((s * C::STAGE) >> 4);
        const uint32_t aP = tmem + COL_S0 + (i & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // queries 16kk..: packed P^T in the first half of its warpgroup's
          // columns, dS^T in the second half
          const uint32_t pc = packed_col(kk);
          const uint64_t ko = uint64_t((kk * 16 * 128) >> 4);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          mma_ts(leader, tmem, aP + pc, dOmn0 + so + ko, ID_A, acc);           // dV += P^T dO
          mma_ts(leader, tmem + D, aP + kCols / 2 + pc, dQmn0 + so + ko, ID_A, acc);  // dK += dS^T Q
        }
        tc_commit(leader, bar.o_done + 8 * (i & 1));
        tc_commit(leader, bar.st_empty + 8 * s);
      }
    }
    __syncwarp();  // lanes may leave the loop apart on an abort
    tc_commit(leader, bar.drain);
    bdrain(bar.drain, 0, p.timeout_ns);
  } else {
    // ------------------------------------------------- softmax + epilogue
    const int g = (warp - 2) >> 2, sub = warp & 3, krow = sub * 32 + lane;
    const int32_t key = k0 + krow;
    const uint32_t lane_addr = tmem + (uint32_t(sub * 32) << 16);
    const bool live = key < p.geom.N;
    int32_t a0 = 0, b0 = 0, a1 = 0, b1 = 0;  // queries that see this key (none past N)
    if (live) key_query_ranges(p.geom, key, a0, b0, a1, b1);
    const float sl2 = p.scale * kLog2e;
    {  // this thread's row of K becomes the A operand of S^T in TMEM
      const size_t off = (size_t(bh) * p.geom.N + (live ? key : 0)) * D;
      row_to_tmem<D>(static_cast<const uint16_t *>(p.k) + off, live, lane_addr + COL_K, g);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.a_ready);
    }
    bool ok = true;
    for (int32_t j = 0; j < ntiles; ++j) {
      const int b = j & 1, s = j % C::STAGES;
      if (!bwarp_wait(bar.s_full + 8 * b, (j >> 1) & 1, abort_flag, p.timeout_ns, 35) ||
          !bwarp_wait(bar.st_full + 8 * s, (j / C::STAGES) & 1, abort_flag, p.timeout_ns, 36)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int32_t qh = nth_tile(j, t) * BN + kCols * g;
      const uint32_t cS = lane_addr + COL_S0 + b * 64 + kCols * g;
      uint32_t rs[kCols], rp[kCols];
      tmem_ld_pair(cS, lane_addr + COL_DP + kCols * g, rs, rp);
      tc_fence_before();  // dP^T is in registers: its buffer may be overwritten
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.dp_free);
      const uint32_t vis = (bits_in(a0 - qh, b0 - qh) | bits_in(a1 - qh, b1 - qh)) & kColMask;
      if (vis != kColMask) {  // queries that do not see this key: p = 0, no dP
#pragma unroll
        for (int i = 0; i < kCols; ++i) {
          const bool v = (vis >> i) & 1u;
          rs[i] = v ? rs[i] : __float_as_uint(-INFINITY);
          rp[i] = v ? rp[i] : 0u;
        }
      }
      const float4 *st4 = reinterpret_cast<const float4 *>(sgen + C::OFF_ST + s * C::STAGE +
                                                           2 * C::S_BYTES) + (kCols / 4) * g;
      uint32_t pk[kCols / 2], dk[kCols / 2];
      // element pairs in packed fp32x2 arithmetic (exponentials scalar)
      const uint64_t sl2x2 = f2(sl2, sl2);
#pragma unroll
      for (int i4 = 0; i4 < kCols / 4; ++i4) {
        const float4 l4 = st4[i4], d4 = st4[16 + i4];
        const uint64_t nl2[2] = {f2(-l4.x, -l4.y), f2(-l4.z, -l4.w)}, dv2[2] = {f2(d4.x, d4.y), f2(d4.z, d4.w)};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int i = 2 * i4 + h, c0 = 2 * i, c1 = 2 * i + 1;
          // hidden pairs: s = -inf gives p = 0, so dS = 0 whatever dP - Delta is
          float xa, xb, qa, qb;
          f2_split(fma2(f2(__uint_as_float(rs[c0]), __uint_as_float(rs[c1])), sl2x2, nl2[h]), xa, xb);
          const float pa = ex2(xa), pb = ex2(xb);
          f2_split(mul2(f2(pa, pb), sub2(f2(__uint_as_float(rp[c0]), __uint_as_float(rp[c1])), dv2[h])), qa, qb);
          pk[i] = pack_bf16(pa, pb);
          dk[i] = pack_bf16(qa, qb);
        }
      }
      tmem_st_cols(cS, pk);
      tmem_st_cols(cS + kCols / 2, dk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.p_full + 8 * b);
    }
    const size_t ri = size_t(bh) * p.geom.N + (live ? key : 0);
    if (ok && ntiles > 0) {
      const int32_t last = ntiles - 1;
      if (bwarp_wait(bar.o_done + 8 * (last & 1), (last >> 1) & 1, abort_flag, p.timeout_ns, 37)) {
        tc_fence_after();
        uint4 *odv = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.dv) + ri * D);
        uint4 *odk = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.dk) + ri * D);
        constexpr int GC = D / kGroups, EC = GC < 32 ? GC : 32;  // columns per group, per load
#pragma unroll 1
        for (int c = g * GC; c < (g + 1) * GC; c += EC) {
          uint32_t rv[EC], rk[EC];
          tmem_ld_pair(lane_addr + c, lane_addr + D + c, rv, rk);
          uint32_t pv[EC / 2], pkk[EC / 2];
#pragma unroll
          for (int i = 0; i < EC / 2; ++i) {
            pv[i] = pack_bf16(__uint_as_float(rv[2 * i]), __uint_as_float(rv[2 * i + 1]));
            pkk[i] = pack_bf16(__uint_as_float(rk[2 * i]) * p.scale, __uint_as_float(rk[2 * i + 1]) * p.scale);
          }
          if (live) {
#pragma unroll
            for (int v = 0; v < EC / 8; ++v) {
              odv[c / 8 + v] = make_uint4(pv[4 * v], pv[4 * v + 1], pv[4 * v + 2], pv[4 * v + 3]);
              odk[c / 8 + v] = make_uint4(pkk[4 * v], pkk[4 * v + 1], pkk[4 * v + 2], pkk[4 * v + 3]);
            }
          }
        }
      }
    } else if (ok && live) {
      // a key no query sees (cannot happen for valid masks): zero gradients
      uint4 *odv = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.dv) + ri * D);
      uint4 *odk = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.dk) + ri * D);
      for (int c = g * (D / kGroups); c < (g + 1) * (D / kGroups); c += 8) {
        odv[c / 8] = make_uint4(0, 0, 0, 0);
        odk[c / 8] = make_uint4(0, 0, 0, 0);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ============================================================ Delta pre-pass
// Delta_i = <dO_i, O_i> in fp32; D/8 lanes per row, 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const void *o, const void *dout, float *delta,
                                                        int64_t rows) {
  constexpr int LPR = D / 8;  // lanes per row
  const int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) / LPR;
  const int part = threadIdx.x % LPR;
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = __ldg(static_cast<const uint4 *>(o) + row * LPR + part);
    const uint4 b = __ldg(static_cast<const uint4 *>(dout) + row * LPR + part);
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(__uint_as_float(wa[i] << 16), __uint_as_float(wb[i] << 16), acc);
      acc = fmaf(__uint_as_float(wa[i] & 0xffff0000u), __uint_as_float(wb[i] & 0xffff0000u), acc);
    }
  }
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off, LPR);
  if (row < rows && part == 0) delta[row] = acc;
}

template <int D>
cudaError_t launch_bwd_impl(const BwdParams &p, cudaStream_t stream) {
  using CQ = BCfg<D, 0>;
  using CK = BCfg<D, 1>;
  static std::atomic<uint64_t> attr_set{0};
  cudaError_t e = once_per_device(attr_set, [] {
    cudaError_t r = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         CQ::SMEM_BYTES);
    if (r == cudaSuccess)
      r = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, CK::SMEM_BYTES);
    return r;
  });
  if (e != cudaSuccess) return e;
  const int64_t rows = int64_t(p.BH) * p.geom.N;
  const int64_t threads = rows * (D / 8);
  bwd_delta_kernel<D><<<unsigned((threads + 255) / 256), 256, 0, stream>>>(p.o, p.dout, p.delta, rows);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const unsigned grid = unsigned(p.n_row_tiles) * unsigned(p.BH);
  bwd_dq_kernel<D><<<grid, kThreads, CQ::SMEM_BYTES, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  BwdParams pk = p;  // the key-major kernel takes the key-tile order
  for (int32_t i = 0; i < p.n_row_tiles; ++i) pk.row_order[i] = p.col_order[i];
  bwd_dkdv_kernel<D><<<grid, kThreads, CK::SMEM_BYTES, stream>>>(pk);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd_sm100(const BwdParams &p, int D, cudaStream_t stream) {
  if (D == 128) return launch_bwd_impl<128>(p, stream);
  if (D == 64) return launch_bwd_impl<64>(p, stream);
  return cudaErrorInvalidValue;
}

cudaError_t read_and_clear_bwd_error(uint32_t *out) {
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_bwd_device_error, sizeof(v));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_bwd_device_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return e;
  }
  *out = v;
  return cudaSuccess;
}

}  // namespace caj
