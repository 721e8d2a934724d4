// Fused forward + JVP of block-causal attention on B200 tensor cores (sm_100a).
//
// Computes, per (batch*head, 128-row query tile), the masked attention output
// and its forward-mode tangent of the Causal-rCM paper, appendix B (eq. 42-45,
// Algorithm 1): the online softmax of FlashAttention carries, next to the usual
// running max m, normaliser l and output accumulator O, the JVP accumulators
//   T = sum_j p~_j (ts_j v_j + tv_j)      (value-tangent + score-tangent terms)
//   r = sum_j p~_j ts_j                    (row scalar)
// all rescaled by the same online factor; after the last key tile
//   O = O / l,  mu = r / l,  tO = T / l - mu O,  LSE = ln l + m,  tLSE = mu.
//
// Design (sm_100a, one CTA per query tile, 10 warps):
//   warp 0      TMA producer: Q, tQ once; then, per step j, the K|tK tile of
//               key tile j and the V|tV tile of key tile j-1, both completing on
//               one barrier, through 2-deep shared-memory rings (128-byte swizzle).
//               K stage j%2 is released by the score-MMA commit of tile j, V stage
//               j%2 by the value-MMA commit of tile j.
//   warp 1      tcgen05 MMA issuer (one thread), also owns the TMEM allocation:
//                 [S | tS_1] = Q [K ; tK]^T        (one N=128 MMA per k-step)
//                 tS += tQ K^T                      (N=64)
//                 [O | T] += P [V | tV]             (A = P from TMEM, N=2D)
//                 T += (P o tS) V                   (A = P o tS from TMEM, N=D)
//               S/tS are double-buffered in TMEM so the scores of tile j+1 are
//               computed while tile j's softmax runs.
//   warps 2-9   softmax / epilogue: two warpgroups, each thread owns one query
//               row and one 32-key half of every key tile (warpgroup g takes
//               keys [32g, 32g+32)). TMEM -> registers, mask (only where the half
//               tile is not entirely visible to the row), exp2-domain online
//               softmax with a lazily updated max shared by the two halves
//               through shared memory, bf16 P and P o tS written back into the
//               score columns in TMEM, and the final normalisation and JVP
//               epilogue (warpgroup g writes output columns [gD/2, (g+1)D/2)).
// TMEM (512 columns x 128 lanes, fp32): O [0,D) | T [D,2D) | S/tS buffer 0 |
// S/tS buffer 1, each buffer S [64 cols] then tS [64 cols]. The bf16 P of keys
// [32g, 32g+32) is packed into S columns [32g, 32g+16) and P o tS into the same
// columns of tS, so each thread only overwrites score columns it has read.
//
// Under clean-tangent-zero teacher forcing, the query tiles of clean rows need
// no tangent at all; they run in a primal-only kernel further down.
//
// Every wait on an mbarrier is bounded by a time limit; on expiry the kernel
// records an error code in a device word, drains its own in-flight copies and
// MMAs, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "mask_schedule.h"
#include "ptx_sm100.cuh"

namespace caj {

__device__ uint32_t g_device_error = 0;

namespace {

using namespace ptx;

constexpr int BM = kBlockM;  // query rows per tile
constexpr int BN = kBlockN;  // keys per tile
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = 64 + 32 * kSoftmaxWarps;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale once the max grew by 2^8
// How many k-steps before the end of the score (S) / value (V) MMA batch the MMA
// warp probes the barrier the next batch needs (0: after the batch).
constexpr int kProbeLeadS = 0;
constexpr int kProbeLeadV = 0;

template <int D>
struct Cfg {
  static constexpr int NB = D / 64;                    // 128-byte column blocks per row
  static constexpr int QBLK = BM * 128;                // one column block of a Q tile
  static constexpr int Q_BYTES = NB * QBLK;
  static constexpr int KBLK = 2 * BN * 128;            // one column block of [K ; tK]
  static constexpr int KT_STAGE = NB * KBLK;
  static constexpr int VBLK = BN * 128;                // one column block of V (or tV)
  static constexpr int V_STAGE = 2 * NB * VBLK;        // V blocks, then tV blocks
  // K stage j%2 is released by s_full[j%2], V stage j%2 by o_done[j%2]
  static constexpr int KS = 2;
  static constexpr int VS = 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_TQ = Q_BYTES;
  static constexpr int OFF_KT = 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_KT + KS * KT_STAGE;
  static constexpr int OFF_BAR = OFF_V + VS * V_STAGE;
  // barriers: q_full, x_full[2], s_full[2], p_full[2], o_done[2], drain,
  //           pair[4 lane quarters][2 slots], pair_end[4 lane quarters]
  static constexpr int NBAR = 1 + 2 + 7 + 12;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag
  // row-max exchange between the two softmax warpgroups: [2 slots][2 halves][BM] fp32
  static constexpr int OFF_XCH = OFF_MISC + 16;
  static constexpr int SMEM_BYTES = OFF_XCH + 2 * 2 * BM * 4;
  // tensor memory columns
  static constexpr uint32_t COL_O = 0;
  static constexpr uint32_t COL_T = D;
  static constexpr uint32_t COL_S0 = 2 * D;
  static constexpr uint32_t BUF_COLS = 2 * BN;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(COL_S0 + 2 * BUF_COLS <= TMEM_COLS, "tensor memory overflow");
  static_assert(SMEM_BYTES <= 232448, "shared memory overflow");
  static constexpr uint32_t Q_TX = 2 * Q_BYTES;
  static constexpr uint32_t KT_TX = KT_STAGE;
  static constexpr uint32_t V_TX = V_STAGE;
  static_assert(KT_TX + V_TX < (1u << 20), "transaction count limit");
};

struct Barriers {
  uint32_t q_full, x_full, s_full, p_full, o_done, drain, pair, pair_end;
};

template <int D>
__device__ __forceinline__ Barriers make_barriers(uint32_t base) {
  using C = Cfg<D>;
  Barriers b;
  b.q_full = base;
  b.x_full = base + 8;
  b.s_full = b.x_full + 16;
  b.p_full = b.s_full + 16;
  b.o_done = b.p_full + 16;
  b.drain = b.o_done + 16;
  b.pair = b.drain + 8;
  b.pair_end = b.pair + 64;
  return b;
}

// Record the first device error and raise the CTA's abort flag.
__device__ __noinline__ void raise_error(volatile int *abort_flag, uint32_t code) {
  atomicCAS(&g_device_error, 0u, code);
  *abort_flag = 1;
}

// Wait for completion of the phase with parity `parity`. Gives up (returns
// false) when the CTA has aborted or after `timeout_ns`, recording `site`.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity,
                                             volatile int *abort_flag, uint64_t timeout_ns,
                                             uint32_t site) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1; it < 0x40000000u; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > timeout_ns) {
        raise_error(abort_flag, kErrTimeoutBase | site);
        return false;
      }
    }
  }
  raise_error(abort_flag, kErrTimeoutBase | site);
  return false;
}

// Same, ignoring the abort flag: used only to drain this CTA's own in-flight
// copies and MMAs before it releases shared and tensor memory.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1; it < 0x40000000u; ++it) {
    if (mbar_try_wait(bar, parity)) return;
    if ((it & 31u) == 0 && globaltimer_ns() - t0 > timeout_ns) return;
  }
}

// Bits [lo, hi) of a 32-bit mask, bounds clamped to [0, 32].
__device__ __forceinline__ uint32_t range_bits(int32_t lo, int32_t hi) {
  lo = max(lo, 0);
  hi = min(hi, 32);
  if (hi <= lo) return 0u;
  return uint32_t(((1ull << hi) - 1ull) & ~((1ull << lo) - 1ull));
}

// Key tile index of the j-th visited tile.
__device__ __forceinline__ int32_t tile_at(int32_t j, int32_t t0, int32_t n0, int32_t t2) {
  return j < n0 ? t0 + j : t2 + (j - n0);
}

// Rendezvous of the two softmax warps that share a lane quarter, through an
// mbarrier with two arrivals (bounded, unlike a named barrier, so an aborting
// CTA cannot strand the partner). Orders each warp's shared-memory writes
// before the partner's subsequent reads (arrive releases, the wait acquires).
__device__ __forceinline__ bool pair_sync(uint32_t mbar, uint32_t parity, int lane,
                                          volatile int *abort_flag, uint64_t timeout_ns,
                                          uint32_t site) {
  __syncwarp();
  if (lane == 0) mbar_arrive(mbar);
  const bool got = wait_bounded(mbar, parity, abort_flag, timeout_ns, site);
  return __all_sync(0xffffffffu, got);
}

// Bounded wait by a whole warp, with a warp-uniform outcome.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          uint64_t timeout_ns, uint32_t site) {
  return __all_sync(0xffffffffu, wait_bounded(bar, parity, abort_flag, timeout_ns, site));
}

// Bounded wait of the MMA warp, with no warp vote: a vote right after the
// elected lane has queued tensor-core instructions holds the whole warp until
// the queue takes them (about 390 cycles with a full queue). Every lane polls
// the same barrier, so the lanes agree but for an abort or a timeout, where a
// lane that gives up raises the CTA's abort flag and the others follow at
// their next wait; the warp reconverges after its loop.
__device__ __forceinline__ bool issuer_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                            uint64_t timeout_ns, uint32_t site) {
  return wait_bounded(bar, parity, abort_flag, timeout_ns, site);
}

// The slice-map arithmetic of the scattering epilogues, kept out of line.
// Inlined, it changed the register allocation of the kernels' main loop:
// the scattering kernel then ran 4.7% slower than the plain one, against
// 2.5-4.2% out of line (3 heads of the TF frame-wise workload, round-robin).
__device__ __noinline__ void scatter_rows(const OutMap &m, int32_t bh, int32_t q, int D, uint4 **o,
                                          uint4 **to) {
  const OutRow dst = slice_row(m, bh, q);
  *o = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(m.o[dst.shard]) + dst.row * D);
  *to = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(m.to[dst.shard]) + dst.row * D);
}

__device__ __noinline__ void scatter_stats(const OutMap &m, int32_t bh, int32_t q, float lse, float tlse) {
  const OutRow dst = slice_row(m, bh, q);
  m.lse[dst.shard][dst.stat] = lse;
  m.tlse[dst.shard][dst.stat] = tlse;
}

// KIND (a TileKind): dense tangents (kTilesAll), or the query tiles with a noisy
// row under clean-tangent-zero teacher forcing (kTilesNoisyCTZ: the caller
// guarantees tq, tk, tv vanish on rows < L). Each is its own instantiation, so
// the dense kernel carries no trace of the specialisation; the clean query
// tiles have a kernel of their own (fwd_primal_sm100_kernel). Measured on the
// TF frame-wise workload: one kernel branching on the kind of each tile took
// 16.0 ms, the two specialised launches 12.0 ms.
// SCATTER: the epilogue stores each row into its sequence slice through the
// slice map (caj_attn_fwd_jvp_scatter, the Ulysses output all-to-all) instead
// of the one-slice output; a separate instantiation, so the one-slice kernel
// keeps its plain addressing.
template <int D, int KIND, bool SCATTER>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_jvp_sm100_kernel(const __grid_constant__ Sm100Params p) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  // 128-byte-swizzled tiles need a 1 KiB aligned base; refuse to run otherwise.
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicCAS(&g_device_error, 0u, uint32_t(kErrSmemMisaligned));
    return;
  }
  uint8_t *sgen = smem_raw;
  const Barriers bar = make_barriers<D>(sbase + C::OFF_BAR);
  volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sgen + C::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sgen + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Work item: head by head (its K/V stay in L2 while its tiles run), and
  // inside a head the heaviest query tiles first.
  const int32_t bh = blockIdx.x / p.n_qtiles;
  const int32_t qt = p.qtile_order[blockIdx.x % p.n_qtiles];
  const int32_t q0 = qt * BM;
  const int32_t q1 = min(q0 + BM, p.geom.N);
  int32_t t0, t1, t2, t3;
  const int32_t ntiles = qtile_key_tiles(p.geom, q0, q1, BN, t0, t1, t2, t3);
  const int32_t n0 = t1 - t0;
  // Clean-tangent-zero teacher forcing: a key tile of clean tokens has
  // tK = tV = 0. (Tiles of clean query rows have no tangent at all and run in
  // fwd_primal_sm100_kernel below.)
  static_assert(KIND == kTilesAll || KIND == kTilesNoisyCTZ, "clean tiles run in the primal kernel");
  constexpr bool CTZ = KIND != kTilesAll;
  auto clean_keys = [&](int32_t key0) { return CTZ && key0 + BN <= p.geom.L; };
  // The host partitions the query tiles by kind; a tile of the other kind is
  // refused before any barrier or TMEM use (the whole CTA leaves together).
  if (CTZ && q1 <= p.geom.L) {
    if (threadIdx.x == 0) atomicCAS(&g_device_error, 0u, uint32_t(kErrTileKind));
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(bar.q_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar.x_full + 8 * b, 1);
      mbar_init(bar.s_full + 8 * b, 1);
      mbar_init(bar.p_full + 8 * b, kSoftmaxWarps);  // one arrival per softmax warp
      mbar_init(bar.o_done + 8 * b, 1);
    }
    mbar_init(bar.drain, 1);
    for (int i = 0; i < 8; ++i) mbar_init(bar.pair + 8 * i, 2);  // the two warps of a lane quarter
    for (int i = 0; i < 4; ++i) mbar_init(bar.pair_end + 8 * i, 2);
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
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop (warp-uniform addresses stay in uniform
    // registers); one elected lane issues the copies.
    const uint32_t leader = elect_one();
    if (leader) {
      prefetch_tmap(&p.tm_q);
      prefetch_tmap(&p.tm_k);
      prefetch_tmap(&p.tm_v);
    }
    const uint32_t sq = sbase + C::OFF_Q, stq = sbase + C::OFF_TQ;
    const bool load_q = p.fault_mode != 1;  // test hook: leave q_full unarmed
    if (load_q) {
      mbar_arrive_expect_tx_if(leader, bar.q_full, C::Q_TX);
      for (int c = 0; c < C::NB; ++c) {
        tma_load_3d(leader, sq + c * C::QBLK, &p.tm_q, bar.q_full, c * 64, q0, bh);
        tma_load_3d(leader, stq + c * C::QBLK, &p.tm_tq, bar.q_full, c * 64, q0, bh);
      }
    }
    // Step j loads K|tK of key tile j (j < ntiles) into K stage j%2 and V|tV
    // of key tile j-1 (j >= 1) into V stage (j-1)%2, completing on x_full[j%2].
    int32_t steps_armed = 0;
    for (int32_t j = 0; j <= ntiles; ++j) {
      const int b = j & 1;
      // S(j-2) done: K stage b and x_full[b]'s previous phase are consumed
      if (j >= 2 && !warp_wait(bar.s_full + 8 * b, ((j >> 1) - 1) & 1, abort_flag, p.timeout_ns, 1))
        break;
      // OT(j-3) done: V stage (j-1)%2 is free
      if (j >= 3 && !warp_wait(bar.o_done + 8 * ((j - 1) & 1), (((j - 1) >> 1) - 1) & 1,
                               abort_flag, p.timeout_ns, 2))
        break;
      const bool has_k = j < ntiles, has_v = j >= 1;
      const int32_t kkey0 = has_k ? tile_at(j, t0, n0, t2) * BN : 0;
      const int32_t vkey0 = has_v ? tile_at(j - 1, t0, n0, t2) * BN : 0;
      const bool k_tan = has_k && !clean_keys(kkey0);  // tK needed
      const bool v_tan = has_v && !clean_keys(vkey0);  // tV needed
      const uint32_t fb = bar.x_full + 8 * b;
      mbar_arrive_expect_tx_if(leader, fb,
                               (has_k ? (k_tan ? C::KT_TX : C::KT_TX / 2) : 0u) +
                                   (has_v ? (v_tan ? C::V_TX : C::V_TX / 2) : 0u));
      if (has_k) {
        const uint32_t dst = sbase + C::OFF_KT + b * C::KT_STAGE;
#pragma unroll
        for (int c = 0; c < C::NB; ++c) {
          tma_load_3d(leader, dst + c * C::KBLK, &p.tm_k, fb, c * 64, kkey0, bh);
          if (k_tan)
            tma_load_3d(leader, dst + c * C::KBLK + BN * 128, &p.tm_tk, fb, c * 64, kkey0, bh);
        }
      }
      if (has_v) {
        const uint32_t dst = sbase + C::OFF_V + ((j - 1) & 1) * C::V_STAGE;
#pragma unroll
        for (int c = 0; c < C::NB; ++c) {
          tma_load_3d(leader, dst + c * C::VBLK, &p.tm_v, fb, c * 64, vkey0, bh);
          if (v_tan)
            tma_load_3d(leader, dst + (C::NB + c) * C::VBLK, &p.tm_tv, fb, c * 64, vkey0, bh);
        }
      }
      steps_armed = j + 1;
    }
    // Drain: every copy this warp issued must land before the CTA exits.
    if (load_q) drain_wait(bar.q_full, 0, p.timeout_ns);
    for (int32_t j = (steps_armed > 2 ? steps_armed - 2 : 0); j < steps_armed; ++j)
      drain_wait(bar.x_full + 8 * (j & 1), (j >> 1) & 1, p.timeout_ns);
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // Warp-uniform loop; the elected lane issues every MMA and commit (so one
    // thread's commits track all of them).
    const uint32_t leader = elect_one();
    constexpr uint32_t ID_S = idesc_bf16_f32(BM, 2 * BN, 0);   // Q [K;tK]^T
    constexpr uint32_t ID_TS = idesc_bf16_f32(BM, BN, 0);      // tQ K^T
    constexpr uint32_t ID_OT = idesc_bf16_f32(BM, 2 * D, 1);   // P [V|tV]
    constexpr uint32_t ID_T = idesc_bf16_f32(BM, D, 1);        // (P o tS) V
    // Operand descriptors: one base per buffer, then compile-time byte offsets
    // (added to the start-address field, which cannot carry out of its 14 bits
    // for shared-memory addresses below 256 KiB).
    const uint64_t dQ = sdesc_sw128(sbase + C::OFF_Q, 16, 1024);
    const uint64_t dTQ = sdesc_sw128(sbase + C::OFF_TQ, 16, 1024);
    const uint64_t dK0 = sdesc_sw128(sbase + C::OFF_KT, 16, 1024);
    // MN-major B: 64-element column blocks C::VBLK apart, 8-key groups 1 KiB apart.
    const uint64_t dV0 = sdesc_sw128(sbase + C::OFF_V, C::VBLK, 1024);
    const uint32_t tS0 = tmem + C::COL_S0;
    bool ok = issuer_wait(bar.q_full, 0, abort_flag, p.timeout_ns, 3);
    // Step j: scores of key tile j, then value products of key tile j-1. One
    // probe covers K(j) and V(j-1), a second one P(j-1). A probe issued while
    // earlier MMAs are still queued overlaps their execution, so each probe is
    // placed kProbeLead k-steps before the end of the batch that precedes its use.
    if (ok) ok = issuer_wait(bar.x_full, 0, abort_flag, p.timeout_ns, 4);
    for (int32_t j = 0; ok && j <= ntiles; ++j) {
      const int32_t i = j - 1;  // key tile whose value products this step issues
      bool have_p = i < 0;
      if (j < ntiles) {
        const bool s_clean = clean_keys(tile_at(j, t0, n0, t2) * BN);
        const uint64_t dK = dK0 + uint64_t(((j & 1) * C::KT_STAGE) >> 4);
        const uint32_t dS = tS0 + (j & 1) * C::BUF_COLS;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          if (kk == D / 16 - kProbeLeadS && !have_p) {
            if (!(ok = issuer_wait(bar.p_full + 8 * (i & 1), (i >> 1) & 1, abort_flag, p.timeout_ns, 5)))
              break;
            have_p = true;
          }
          // 16 bf16 (32 bytes) per k-step inside a 128-byte swizzle atom, 64 per column block
          const uint64_t qo = uint64_t(((kk >> 2) * C::QBLK + (kk & 3) * 32) >> 4);
          const uint64_t ko = uint64_t(((kk >> 2) * C::KBLK + (kk & 3) * 32) >> 4);
          if (!s_clean) {  // [S | Q tK^T] = Q [K;tK]^T, then tS += tQ K^T
            mma_ss(leader, dS, dQ + qo, dK + ko, ID_S, kk > 0 ? 1u : 0u);
            mma_ss(leader, dS + BN, dTQ + qo, dK + ko, ID_TS, 1u);
          } else {         // clean keys (tK = 0): S = Q K^T, tS = tQ K^T
            mma_ss(leader, dS, dQ + qo, dK + ko, ID_TS, kk > 0 ? 1u : 0u);
            mma_ss(leader, dS + BN, dTQ + qo, dK + ko, ID_TS, kk > 0 ? 1u : 0u);
          }
        }
        if (!ok) break;
        tc_commit(leader, bar.s_full + 8 * (j & 1));
      }
      const bool next = j + 1 <= ntiles;  // another step follows
      bool have_x = !next;
      if (i >= 0) {
        if (!have_p &&
            !(ok = issuer_wait(bar.p_full + 8 * (i & 1), (i >> 1) & 1, abort_flag, p.timeout_ns, 5)))
          break;
        tc_fence_after();
        const uint64_t dV = dV0 + uint64_t(((i & 1) * C::V_STAGE) >> 4);
        const uint32_t aP = tS0 + (i & 1) * C::BUF_COLS;
        const uint32_t first = i > 0 ? 1u : 0u;
        const bool v_clean = clean_keys(tile_at(i, t0, n0, t2) * BN);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          if (kk == BN / 16 - kProbeLeadV && !have_x) {
            if (!(ok = issuer_wait(bar.x_full + 8 * ((j + 1) & 1), ((j + 1) >> 1) & 1, abort_flag,
                                 p.timeout_ns, 4)))
              break;
            have_x = true;
          }
          const uint64_t vo = uint64_t((kk * 16 * 128) >> 4);  // 16 keys of 128-byte rows
          const uint32_t pc = (kk >> 1) * 32 + (kk & 1) * 8;   // packed P columns of keys 16kk..
          if (!v_clean) {  // [O | T] += P [V | tV], then T += (P o tS) V
            mma_ts(leader, tmem + C::COL_O, aP + pc, dV + vo, ID_OT, kk > 0 ? 1u : first);
            mma_ts(leader, tmem + C::COL_T, aP + BN + pc, dV + vo, ID_T, 1u);
          } else {         // clean keys (tV = 0): O += P V, T += (P o tS) V
            mma_ts(leader, tmem + C::COL_O, aP + pc, dV + vo, ID_T, kk > 0 ? 1u : first);
            mma_ts(leader, tmem + C::COL_T, aP + BN + pc, dV + vo, ID_T, kk > 0 ? 1u : first);
          }
        }
        if (!ok) break;
        tc_commit(leader, bar.o_done + 8 * (i & 1));
      }
      if (!have_x &&
          !(ok = issuer_wait(bar.x_full + 8 * ((j + 1) & 1), ((j + 1) >> 1) & 1, abort_flag,
                           p.timeout_ns, 4)))
        break;
    }
    // Drain: all MMAs issued by the elected lane complete before TMEM is freed.
    __syncwarp();  // lanes may leave the loop apart on an abort
    tc_commit(leader, bar.drain);
    drain_wait(bar.drain, 0, p.timeout_ns);
  } else {
    // ------------------------------------------------- softmax + epilogue
    const int g = (warp - 2) >> 2;            // key half of each tile owned by this warpgroup
    const int sub = warp & 3;                 // TMEM lane quarter this warp may access
    const int row = sub * 32 + lane;          // query row within the tile
    const int32_t q = q0 + row;
    const uint32_t lane_addr = tmem + (uint32_t(sub * 32) << 16);
    float *xch = reinterpret_cast<float *>(sgen + C::OFF_XCH);  // [slot][half][row]
    int32_t a0, b0, a1, b1;
    if (q < p.geom.N) {
      row_key_ranges(p.geom, q, a0, b0, a1, b1);
    } else {  // padding row past the sequence end: keep it finite, never stored
      a0 = 0;
      b0 = p.geom.N;
      a1 = b1 = 0;
    }
    const float sl2 = p.scale_log2e;
    const float scale = p.scale;
    float m_run = -INFINITY;  // running max of s * scale * log2(e), possibly stale by < 2^8
    float l_run = 0.f, r_run = 0.f;  // partial sums over this thread's key halves
    bool ok = true;

    for (int32_t j = 0; j < ntiles; ++j) {
      const int b = j & 1;
      const bool got = wait_bounded(bar.s_full + 8 * b, (j >> 1) & 1, abort_flag, p.timeout_ns, 7);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int32_t kh = tile_at(j, t0, n0, t2) * BN + 32 * g;  // first key of this half
      const uint32_t cS = lane_addr + C::COL_S0 + b * C::BUF_COLS + 32 * g;
      const uint32_t cT = cS + BN;
      uint32_t rs[32], rt[32];
      tmem_ld32x2(cS, cT, rs, rt);
      float s[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) s[i] = __uint_as_float(rs[i]);
      // Keys of this half tile the row may see; mask only where some are hidden.
      // Hidden keys get s = -inf (so p = 0) and a zero score tangent (select, so
      // a non-finite tangent of a hidden key cannot leak in as 0 * inf).
      const uint32_t vis = range_bits(a0 - kh, b0 - kh) | range_bits(a1 - kh, b1 - kh);
      if (vis != 0xffffffffu) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const bool v = (vis >> i) & 1u;
          s[i] = v ? s[i] : -INFINITY;
          rt[i] = v ? rt[i] : 0u;
        }
      }
      const float hmax = max_of32(s);
      // Exchange the half-row max with the other warpgroup.
      xch[(b * 2 + g) * BM + row] = hmax;
      if (!pair_sync(bar.pair + 8 * (sub * 2 + b), (j >> 1) & 1, lane, abort_flag, p.timeout_ns,
                     10)) {
        ok = false;
        break;
      }
      const float tmax = fmaxf(hmax, xch[(b * 2 + (g ^ 1)) * BM + row]);
      const float m_tile = tmax * sl2;  // -inf if the row sees nothing in this tile
      // Lazy rescale: keep the old max unless the new one exceeds it by 2^8.
      const bool grow = m_tile > m_run + kRescaleThreshold;
      const bool had_acc = m_run != -INFINITY;  // accumulators hold non-zero data
      float alpha = 1.f;
      if (grow) {
        alpha = had_acc ? ex2(m_run - m_tile) : 0.f;
        l_run *= alpha;
        r_run *= alpha;
        m_run = m_tile;
      }
      if (__any_sync(0xffffffffu, grow && had_acc) && j > 0) {
        // This warpgroup's accumulator (O for g=0, T for g=1) must be scaled by
        // alpha once the value MMAs of the previous tile have landed.
        const int pb = (j - 1) & 1;
        const bool g2 =
            wait_bounded(bar.o_done + 8 * pb, ((j - 1) >> 1) & 1, abort_flag, p.timeout_ns, 8);
        if (!__all_sync(0xffffffffu, g2)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = lane_addr + (g ? C::COL_T : C::COL_O);
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t r[32];
          tmem_ld32(acc + c, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(acc + c, r);
        }
      }
      const float ref = (m_run == -INFINITY) ? 0.f : m_run;
      // P = 2^(s*scale*log2e - ref) and P o tS, rounded to bf16 and packed into
      // this half's first 16 score columns.
      // Element pairs go through packed fp32x2 arithmetic (the exponentials
      // stay scalar): the same roundings per element, half the instructions.
      const uint64_t sl2x2 = f2(sl2, sl2), nref2 = f2(-ref, -ref), scale2 = f2(scale, scale);
      uint64_t ls2[2] = {0ull, 0ull}, rs2[2] = {0ull, 0ull};
      uint32_t pk[16], tk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float xa, xb;
        f2_split(fma2(f2(s[2 * i], s[2 * i + 1]), sl2x2, nref2), xa, xb);
        const float pa = ex2(xa), pb = ex2(xb);
        const uint64_t p2 = f2(pa, pb);
        const uint64_t q2 = mul2(p2, mul2(f2(__uint_as_float(rt[2 * i]), __uint_as_float(rt[2 * i + 1])), scale2));
        ls2[i & 1] = add2(ls2[i & 1], p2);
        rs2[i & 1] = add2(rs2[i & 1], q2);
        float qa, qb;
        f2_split(q2, qa, qb);
        pk[i] = pack_bf16(pa, pb);
        tk[i] = pack_bf16(qa, qb);
      }
      tmem_st16(cS, pk);
      tmem_st16(cT, tk);
      float la, lb, lc, ld, ra, rb, rc, rd;
      f2_split(ls2[0], la, lb);
      f2_split(ls2[1], lc, ld);
      f2_split(rs2[0], ra, rb);
      f2_split(rs2[1], rc, rd);
      l_run += (la + lb) + (lc + ld);
      r_run += (ra + rb) + (rc + rd);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.p_full + 8 * b);
    }

    if (ok && ntiles > 0) {
      // Combine the two halves' partial sums (both relative to the same max).
      // Slot ntiles&1 was last read at tile ntiles-2, before the partner's
      // final pair rendezvous; slot (ntiles-1)&1 is free once the first
      // rendezvous below has passed.
      const int s0 = ntiles & 1, s1 = s0 ^ 1;
      xch[(s0 * 2 + g) * BM + row] = l_run;
      bool got = pair_sync(bar.pair_end + 8 * sub, 0, lane, abort_flag, p.timeout_ns, 11);
      const float l_tot = l_run + xch[(s0 * 2 + (g ^ 1)) * BM + row];
      if (got) {
        xch[(s1 * 2 + g) * BM + row] = r_run;
        got = pair_sync(bar.pair_end + 8 * sub, 1, lane, abort_flag, p.timeout_ns, 11);
      }
      const float r_tot = r_run + xch[(s1 * 2 + (g ^ 1)) * BM + row];
      const int32_t last = ntiles - 1;
      if (got)
        got = wait_bounded(bar.o_done + 8 * (last & 1), (last >> 1) & 1, abort_flag, p.timeout_ns, 9);
      if (__all_sync(0xffffffffu, got)) {
        tc_fence_after();
        const float inv_l = 1.f / l_tot;
        const float mu = r_tot * inv_l;
        const bool store = q < p.geom.N;
        uint4 *orow, *torow;
        if constexpr (SCATTER) {
          scatter_rows(p.scatter, bh, store ? q : 0, D, &orow, &torow);
        } else {
          const size_t rowoff = out_row(bh, store ? q : 0, p.geom.N, p.out_heads, D);
          orow = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.o) + rowoff);
          torow = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.to) + rowoff);
        }
#pragma unroll 1
        for (int c = g * (D / 2); c < (g + 1) * (D / 2); c += 32) {
          uint32_t ro[32], rt[32];
          tmem_ld32x2(lane_addr + C::COL_O + c, lane_addr + C::COL_T + c, ro, rt);
          uint32_t po[16], pt[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float oa = __uint_as_float(ro[2 * i]) * inv_l;
            const float ob = __uint_as_float(ro[2 * i + 1]) * inv_l;
            const float ta = fmaf(__uint_as_float(rt[2 * i]), inv_l, -mu * oa);
            const float tb = fmaf(__uint_as_float(rt[2 * i + 1]), inv_l, -mu * ob);
            po[i] = pack_bf16(oa, ob);
            pt[i] = pack_bf16(ta, tb);
          }
          if (store) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              orow[c / 8 + v] = make_uint4(po[4 * v], po[4 * v + 1], po[4 * v + 2], po[4 * v + 3]);
              torow[c / 8 + v] = make_uint4(pt[4 * v], pt[4 * v + 1], pt[4 * v + 2], pt[4 * v + 3]);
            }
          }
        }
        if (store && g == 0) {
          const float lse = (m_run + __log2f(l_tot)) * 0.69314718055994530942f;
          if constexpr (SCATTER) {
            scatter_stats(p.scatter, bh, q, lse, mu);
          } else {
            const size_t ri = size_t(bh) * p.geom.N + q;
            p.lse[ri] = lse;
            p.tlse[ri] = mu;
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

// ================================================================ primal only
// Query tiles of clean rows under clean-tangent-zero teacher forcing: their
// tangents vanish, so tO = 0 and tLSE = 0 exactly, and only O = softmax(S) V
// and LSE are computed.
// The two softmax warpgroups split the key tiles, not the keys of a tile:
// warpgroup g takes tiles j = g (mod 2), each thread a whole 64-key row of
// them, with its own running max m_g, sum l_g and accumulator O_g in TMEM.
// The two online softmaxes run side by side with no rendezvous per tile; the
// epilogue merges them once: with m = max(m_0, m_1) and a_g = 2^(m_g - m),
//   O = (a_0 O_0 + a_1 O_1) / (a_0 l_0 + a_1 l_1),  LSE = ln 2 (m + log2 of that sum).
// (Measured against the JVP kernel's scheme, where the two warpgroups take the
// two 32-key halves of every tile and meet each tile to agree on a row max: the
// per-tile chain of a warp - TMEM load, rendezvous, exponentials, store - was
// the limit, with the tensor pipe 35% busy.)
// TMEM: O_0 [0, D) | O_1 [D, 2D) | four 64-column score buffers. K and V have
// 4-deep rings; the MMA warp issues the scores of tile j, then O_(i%2) += P V
// of tile i = j - 3, so the tensor core runs up to three tiles of scores ahead.
// Roles and masking are those of the JVP kernel above.
constexpr int kPrimalBufs = 4;
constexpr int kPrimalLag = kPrimalBufs - 1;

template <int D>
struct PCfg {
  static constexpr int NS = kPrimalBufs;
  static constexpr int NB = D / 64;
  static constexpr int QBLK = BM * 128;
  static constexpr int Q_BYTES = NB * QBLK;
  static constexpr int KBLK = BN * 128;      // one column block of a K (or V) tile
  static constexpr int K_STAGE = NB * KBLK;
  static constexpr int V_STAGE = NB * KBLK;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * K_STAGE;
  static constexpr int OFF_BAR = OFF_V + NS * V_STAGE;
  // barriers: q_full, k_full[NS], v_full[NS], s_full[NS], p_full[NS], o_done[NS],
  //           drain, pair_end[4 lane quarters]
  static constexpr int NBAR = 1 + 5 * NS + 1 + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_XCH = OFF_MISC + 16;  // [m, l][2 warpgroups][BM] fp32
  static constexpr int SMEM_BYTES = OFF_XCH + 2 * 2 * BM * 4;
  static constexpr uint32_t COL_O = 0;       // O_g at COL_O + g D
  static constexpr uint32_t COL_S0 = 2 * D;  // score buffer b: [COL_S0 + BN b, +BN)
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(COL_S0 + NS * BN <= TMEM_COLS, "tensor memory overflow");
  static_assert(SMEM_BYTES <= 232448, "shared memory overflow");
  static_assert(OFF_K % 1024 == 0 && K_STAGE % 1024 == 0, "128-byte swizzle needs 1 KiB aligned tiles");
  static_assert(NS % 2 == 0, "buffer b serves warpgroup b % 2");
};

struct PBarriers {
  uint32_t q_full, k_full, v_full, s_full, p_full, o_done, drain, pair_end;
};

template <int D>
__device__ __forceinline__ PBarriers make_pbarriers(uint32_t base) {
  constexpr int NS = PCfg<D>::NS;
  PBarriers b;
  b.q_full = base;
  b.k_full = base + 8;
  b.v_full = b.k_full + 8 * NS;
  b.s_full = b.v_full + 8 * NS;
  b.p_full = b.s_full + 8 * NS;
  b.o_done = b.p_full + 8 * NS;
  b.drain = b.o_done + 8 * NS;
  b.pair_end = b.drain + 8;
  return b;
}

template <int D, bool SCATTER>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_primal_sm100_kernel(const __grid_constant__ Sm100Params p) {
  using C = PCfg<D>;
  constexpr int NS = C::NS;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicCAS(&g_device_error, 0u, uint32_t(kErrSmemMisaligned));
    return;
  }
  uint8_t *sgen = smem_raw;
  const PBarriers bar = make_pbarriers<D>(sbase + C::OFF_BAR);
  volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sgen + C::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sgen + C::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int32_t bh = blockIdx.x / p.n_qtiles;
  const int32_t qt = p.qtile_order[blockIdx.x % p.n_qtiles];
  const int32_t q0 = qt * BM;
  const int32_t q1 = min(q0 + BM, p.geom.N);
  int32_t t0, t1, t2, t3;
  const int32_t ntiles = qtile_key_tiles(p.geom, q0, q1, BN, t0, t1, t2, t3);
  const int32_t n0 = t1 - t0;
  // only clean query rows come here; the host partitions the tiles
  if (p.tile_kind != kTilesCleanCTZ || q1 > p.geom.L) {
    if (threadIdx.x == 0) atomicCAS(&g_device_error, 0u, uint32_t(kErrTileKind));
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(bar.q_full, 1);
    for (int b = 0; b < NS; ++b) {
      mbar_init(bar.k_full + 8 * b, 1);
      mbar_init(bar.v_full + 8 * b, 1);
      mbar_init(bar.s_full + 8 * b, 1);
      mbar_init(bar.p_full + 8 * b, kSoftmaxWarps / 2);  // the four warps of one warpgroup
      mbar_init(bar.o_done + 8 * b, 1);
    }
    mbar_init(bar.drain, 1);
    for (int i = 0; i < 4; ++i) mbar_init(bar.pair_end + 8 * i, 2);
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
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint32_t leader = elect_one();
    if (leader) {
      prefetch_tmap(&p.tm_q);
      prefetch_tmap(&p.tm_k);
      prefetch_tmap(&p.tm_v);
    }
    const bool load_q = p.fault_mode != 1;  // test hook: leave q_full unarmed
    if (load_q) {
      mbar_arrive_expect_tx_if(leader, bar.q_full, C::Q_BYTES);
      for (int c = 0; c < C::NB; ++c)
        tma_load_3d(leader, sbase + C::OFF_Q + c * C::QBLK, &p.tm_q, bar.q_full, c * 64, q0, bh);
    }
    int32_t armed = 0;
    for (int32_t j = 0; j < ntiles; ++j) {
      const int b = j % NS;
      const uint32_t ph = ((j / NS) - 1) & 1;  // phase of the previous use of stage b
      const int32_t key0 = tile_at(j, t0, n0, t2) * BN;
      // K stage b held tile j - NS: its scores must have completed
      if (j >= NS && !warp_wait(bar.s_full + 8 * b, ph, abort_flag, p.timeout_ns, 12)) break;
      mbar_arrive_expect_tx_if(leader, bar.k_full + 8 * b, C::K_STAGE);
#pragma unroll
      for (int c = 0; c < C::NB; ++c)
        tma_load_3d(leader, sbase + C::OFF_K + b * C::K_STAGE + c * C::KBLK, &p.tm_k, bar.k_full + 8 * b,
                    c * 64, key0, bh);
      // V stage b held tile j - NS: its value product must have completed
      if (j >= NS && !warp_wait(bar.o_done + 8 * b, ph, abort_flag, p.timeout_ns, 13)) {
        armed = -(j + 1);  // K of tile j is in flight, V is not
        break;
      }
      mbar_arrive_expect_tx_if(leader, bar.v_full + 8 * b, C::V_STAGE);
#pragma unroll
      for (int c = 0; c < C::NB; ++c)
        tma_load_3d(leader, sbase + C::OFF_V + b * C::V_STAGE + c * C::KBLK, &p.tm_v, bar.v_full + 8 * b,
                    c * 64, key0, bh);
      armed = j + 1;
    }
    // Drain every copy this warp issued before the CTA releases its memory.
    if (load_q) drain_wait(bar.q_full, 0, p.timeout_ns);
    const int32_t k_armed = armed < 0 ? -armed : armed, v_armed = armed < 0 ? -armed - 1 : armed;
    for (int32_t j = (k_armed > NS ? k_armed - NS : 0); j < k_armed; ++j)
      drain_wait(bar.k_full + 8 * (j % NS), (j / NS) & 1, p.timeout_ns);
    for (int32_t j = (v_armed > NS ? v_armed - NS : 0); j < v_armed; ++j)
      drain_wait(bar.v_full + 8 * (j % NS), (j / NS) & 1, p.timeout_ns);
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    const uint32_t leader = elect_one();
    constexpr uint32_t ID_S = idesc_bf16_f32(BM, BN, 0);  // Q K^T
    constexpr uint32_t ID_O = idesc_bf16_f32(BM, D, 1);   // P V, V read MN-major
    const uint64_t dQ = sdesc_sw128(sbase + C::OFF_Q, 16, 1024);
    const uint64_t dK0 = sdesc_sw128(sbase + C::OFF_K, 16, 1024);
    const uint64_t dV0 = sdesc_sw128(sbase + C::OFF_V, C::KBLK, 1024);
    bool ok = issuer_wait(bar.q_full, 0, abort_flag, p.timeout_ns, 14);
    for (int32_t j = 0; ok && j < ntiles + kPrimalLag; ++j) {
      if (j < ntiles) {
        // Buffer j%NS last held P of tile j - NS, read by its value product,
        // which was issued earlier (step j - 1): the tensor pipe runs in order.
        const int b = j % NS;
        if (!(ok = issuer_wait(bar.k_full + 8 * b, (j / NS) & 1, abort_flag, p.timeout_ns, 15))) break;
        tc_fence_after();
        const uint64_t dK = dK0 + uint64_t((b * C::K_STAGE) >> 4);
        const uint32_t dS = tmem + C::COL_S0 + b * BN;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t qo = uint64_t(((kk >> 2) * C::QBLK + (kk & 3) * 32) >> 4);
          const uint64_t ko = uint64_t(((kk >> 2) * C::KBLK + (kk & 3) * 32) >> 4);
          mma_ss(leader, dS, dQ + qo, dK + ko, ID_S, kk > 0 ? 1u : 0u);
        }
        tc_commit(leader, bar.s_full + 8 * b);
      }
      const int32_t i = j - kPrimalLag;
      if (i >= 0) {
        const int b = i % NS;
        if (!(ok = issuer_wait(bar.p_full + 8 * b, (i / NS) & 1, abort_flag, p.timeout_ns, 16))) break;
        if (!(ok = issuer_wait(bar.v_full + 8 * b, (i / NS) & 1, abort_flag, p.timeout_ns, 17))) break;
        tc_fence_after();
        const uint64_t dV = dV0 + uint64_t((b * C::V_STAGE) >> 4);
        const uint32_t aP = tmem + C::COL_S0 + b * BN;
        const uint32_t dO = tmem + C::COL_O + (i & 1) * D;  // warpgroup i%2's accumulator
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t vo = uint64_t((kk * 16 * 128) >> 4);  // 16 keys of 128-byte rows
          const uint32_t pc = (kk >> 1) * 32 + (kk & 1) * 8;   // packed P columns of keys 16kk..
          mma_ts(leader, dO, aP + pc, dV + vo, ID_O, (i > 1 || kk > 0) ? 1u : 0u);
        }
        tc_commit(leader, bar.o_done + 8 * b);
      }
    }
    __syncwarp();  // lanes may leave the loop apart on an abort
    tc_commit(leader, bar.drain);
    drain_wait(bar.drain, 0, p.timeout_ns);
  } else {
    // ------------------------------------------------- softmax + epilogue
    const int g = (warp - 2) >> 2;  // this warpgroup takes key tiles j = g (mod 2)
    const int sub = warp & 3;
    const int row = sub * 32 + lane;
    const int32_t q = q0 + row;
    const uint32_t lane_addr = tmem + (uint32_t(sub * 32) << 16);
    const uint32_t cO = lane_addr + C::COL_O + g * D;
    float *xch = reinterpret_cast<float *>(sgen + C::OFF_XCH);  // [m, l][warpgroup][row]
    int32_t a0, b0, a1, b1;
    if (q < p.geom.N) {
      row_key_ranges(p.geom, q, a0, b0, a1, b1);
    } else {
      a0 = 0;
      b0 = p.geom.N;
      a1 = b1 = 0;
    }
    const float sl2 = p.scale_log2e;
    float m_run = -INFINITY;  // of this warpgroup's tiles, possibly stale by < 2^8
    float l_run = 0.f;
    bool ok = true;
    for (int32_t j = g; j < ntiles; j += 2) {
      const int b = j % NS;
      if (!warp_wait(bar.s_full + 8 * b, (j / NS) & 1, abort_flag, p.timeout_ns, 18)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int32_t kh = tile_at(j, t0, n0, t2) * BN;
      const uint32_t cS = lane_addr + C::COL_S0 + b * BN;
      uint32_t ra[32], rb[32];
      tmem_ld32x2(cS, cS + 32, ra, rb);
      float s[64];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        s[i] = __uint_as_float(ra[i]);
        s[32 + i] = __uint_as_float(rb[i]);
      }
      // keys of this tile the row may see; mask only where some are hidden
      const uint32_t v0 = range_bits(a0 - kh, b0 - kh) | range_bits(a1 - kh, b1 - kh);
      const uint32_t v1 = range_bits(a0 - kh - 32, b0 - kh - 32) | range_bits(a1 - kh - 32, b1 - kh - 32);
      if ((v0 & v1) != 0xffffffffu) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = ((v0 >> i) & 1u) ? s[i] : -INFINITY;
          s[32 + i] = ((v1 >> i) & 1u) ? s[32 + i] : -INFINITY;
        }
      }
      const float m_tile = fmaxf(max_of32(s), max_of32(s + 32)) * sl2;
      const bool grow = m_tile > m_run + kRescaleThreshold;
      const bool had_acc = m_run != -INFINITY;
      float alpha = 1.f;
      if (grow) {
        alpha = had_acc ? ex2(m_run - m_tile) : 0.f;
        l_run *= alpha;
        m_run = m_tile;
      }
      if (__any_sync(0xffffffffu, grow && had_acc) && j >= 2) {
        // O_g must be scaled once this warpgroup's previous tile (j - 2) has
        // landed in it (value products complete in order).
        const int pb = (j - 2) % NS;
        if (!warp_wait(bar.o_done + 8 * pb, ((j - 2) / NS) & 1, abort_flag, p.timeout_ns, 20)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t r[32];
          tmem_ld32(cO + c, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(cO + c, r);
        }
      }
      const float ref = (m_run == -INFINITY) ? 0.f : m_run;
      // P = 2^(s*scale*log2e - ref) in bf16: keys 0-31 packed into columns
      // 0-15, keys 32-63 into columns 32-47 (the layout the value MMA reads)
      // element pairs in packed fp32x2 arithmetic (exponentials scalar)
      const uint64_t sl2x2 = f2(sl2, sl2), nref2 = f2(-ref, -ref);
      uint64_t ls2[2] = {0ull, 0ull};
      uint32_t pk0[16], pk1[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float xa, xb, xc, xd;
        f2_split(fma2(f2(s[2 * i], s[2 * i + 1]), sl2x2, nref2), xa, xb);
        f2_split(fma2(f2(s[32 + 2 * i], s[32 + 2 * i + 1]), sl2x2, nref2), xc, xd);
        const float pa = ex2(xa), pb = ex2(xb), pc = ex2(xc), pd = ex2(xd);
        ls2[i & 1] = add2(ls2[i & 1], add2(f2(pa, pb), f2(pc, pd)));
        pk0[i] = pack_bf16(pa, pb);
        pk1[i] = pack_bf16(pc, pd);
      }
      tmem_st16(cS, pk0);
      tmem_st16(cS + 32, pk1);
      float la, lb, lc, ld;
      f2_split(ls2[0], la, lb);
      f2_split(ls2[1], lc, ld);
      l_run += (la + lb) + (lc + ld);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.p_full + 8 * b);
    }

    if (ok && ntiles > 0) {
      // Merge the two warpgroups' partial softmaxes (a warpgroup without tiles,
      // or whose tiles the row cannot see, has m = -inf and contributes 0).
      xch[(0 * 2 + g) * BM + row] = m_run;
      xch[(1 * 2 + g) * BM + row] = l_run;
      bool got = pair_sync(bar.pair_end + 8 * sub, 0, lane, abort_flag, p.timeout_ns, 21);
      const float m_o = xch[(0 * 2 + (g ^ 1)) * BM + row], l_o = xch[(1 * 2 + (g ^ 1)) * BM + row];
      const float m_0 = g ? m_o : m_run, m_1 = g ? m_run : m_o;
      const float l_0 = g ? l_o : l_run, l_1 = g ? l_run : l_o;
      const float m = fmaxf(m_0, m_1);
      const bool has0 = m_0 != -INFINITY, has1 = m_1 != -INFINITY;
      const float f0 = has0 ? ex2(m_0 - m) : 0.f, f1 = has1 ? ex2(m_1 - m) : 0.f;
      const float l_tot = f0 * l_0 + f1 * l_1;
      const int32_t last = ntiles - 1;
      if (got)
        got = wait_bounded(bar.o_done + 8 * (last % NS), (last / NS) & 1, abort_flag, p.timeout_ns, 22);
      if (__all_sync(0xffffffffu, got)) {
        tc_fence_after();
        const float w0 = f0 / l_tot, w1 = f1 / l_tot;
        const bool store = q < p.geom.N;
        uint4 *orow, *torow;
        if constexpr (SCATTER) {
          scatter_rows(p.scatter, bh, store ? q : 0, D, &orow, &torow);
        } else {
          const size_t rowoff = out_row(bh, store ? q : 0, p.geom.N, p.out_heads, D);
          orow = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.o) + rowoff);
          torow = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.to) + rowoff);
        }
        // warpgroup g writes output columns [g D/2, (g+1) D/2)
#pragma unroll 1
        for (int c = g * (D / 2); c < (g + 1) * (D / 2); c += 32) {
          uint32_t r0[32], r1[32];
          tmem_ld32x2(lane_addr + C::COL_O + c, lane_addr + C::COL_O + D + c, r0, r1);
          uint32_t po[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            // select, not multiply: an accumulator never written holds garbage
            const float x0 = has0 ? __uint_as_float(r0[2 * i]) * w0 : 0.f;
            const float y0 = has0 ? __uint_as_float(r0[2 * i + 1]) * w0 : 0.f;
            const float x1 = has1 ? __uint_as_float(r1[2 * i]) * w1 : 0.f;
            const float y1 = has1 ? __uint_as_float(r1[2 * i + 1]) * w1 : 0.f;
            po[i] = pack_bf16(x0 + x1, y0 + y1);
          }
          if (store) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              orow[c / 8 + v] = make_uint4(po[4 * v], po[4 * v + 1], po[4 * v + 2], po[4 * v + 3]);
              torow[c / 8 + v] = make_uint4(0u, 0u, 0u, 0u);  // clean rows: the tangent vanishes
            }
          }
        }
        if (store && g == 0) {
          const float lse = (m + __log2f(l_tot)) * 0.69314718055994530942f;
          if constexpr (SCATTER) {
            scatter_stats(p.scatter, bh, q, lse, 0.f);
          } else {
            const size_t ri = size_t(bh) * p.geom.N + q;
            p.lse[ri] = lse;
            p.tlse[ri] = 0.f;
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

template <int D, bool SCATTER>
cudaError_t launch_primal_impl(const Sm100Params &p, cudaStream_t stream) {
  using C = PCfg<D>;
  static std::atomic<uint64_t> attr_set{0};
  cudaError_t e = once_per_device(attr_set, [] {
    return cudaFuncSetAttribute(fwd_primal_sm100_kernel<D, SCATTER>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::SMEM_BYTES);
  });
  if (e != cudaSuccess) return e;
  const unsigned grid = unsigned(p.n_qtiles) * unsigned(p.BH);
  fwd_primal_sm100_kernel<D, SCATTER><<<grid, kThreads, C::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError();
}

template <int D, int KIND, bool SCATTER>
cudaError_t launch_impl(const Sm100Params &p, cudaStream_t stream) {
  using C = Cfg<D>;
  static std::atomic<uint64_t> attr_set{0};
  cudaError_t e = once_per_device(attr_set, [] {
    return cudaFuncSetAttribute(fwd_jvp_sm100_kernel<D, KIND, SCATTER>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::SMEM_BYTES);
  });
  if (e != cudaSuccess) return e;
  const unsigned grid = unsigned(p.n_qtiles) * unsigned(p.BH);
  fwd_jvp_sm100_kernel<D, KIND, SCATTER><<<grid, kThreads, C::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError();
}

// The scattering epilogue is an instantiation of its own: the one-slice
// kernels keep their plain addressing. (One kernel for both, through the
// slice map, measured 3-5% slower on the dense path under the power cap.)
template <bool SCATTER>
cudaError_t dispatch(const Sm100Params &p, int D, cudaStream_t stream) {
  switch (p.tile_kind * 256 + D) {
    case kTilesAll * 256 + 128: return launch_impl<128, kTilesAll, SCATTER>(p, stream);
    case kTilesNoisyCTZ * 256 + 128: return launch_impl<128, kTilesNoisyCTZ, SCATTER>(p, stream);
    case kTilesCleanCTZ * 256 + 128: return launch_primal_impl<128, SCATTER>(p, stream);
    case kTilesAll * 256 + 64: return launch_impl<64, kTilesAll, SCATTER>(p, stream);
    case kTilesNoisyCTZ * 256 + 64: return launch_impl<64, kTilesNoisyCTZ, SCATTER>(p, stream);
    case kTilesCleanCTZ * 256 + 64: return launch_primal_impl<64, SCATTER>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_fwd_jvp_sm100(const Sm100Params &p, int D, cudaStream_t stream) {
  return p.scatter.shards > 0 ? dispatch<true>(p, D, stream) : dispatch<false>(p, D, stream);
}

cudaError_t read_and_clear_device_error(cudaStream_t stream, uint32_t *out) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  uint32_t v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return e;
  }
  *out = v;
  return cudaSuccess;
}

}  // namespace caj
