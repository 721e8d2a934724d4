// Internal launch interface between the C-ABI front end (api.cpp) and the CUDA
// translation units. Not part of the public header.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "mask_schedule.h"

namespace caj {

// Query-tile height of both kernels' work decomposition (rows per tile).
constexpr int kBlockM = 128;
// Key-tile width of the tensor-core kernel.
constexpr int kBlockN = 64;
// Largest number of query tiles per head the launch order table can hold.
constexpr int kMaxQTiles = 4096;

// Device error word values (first error wins). Low byte: where a wait gave up.
enum DeviceError : uint32_t {
  kErrNone = 0,
  kErrTimeoutBase = 0x100,     // | wait site
  kErrSmemMisaligned = 0x200,  // dynamic shared memory not 1 KiB aligned
  kErrTileKind = 0x300,        // a query tile outside the kind its launch covers
};

// Wait site of the signal barrier (kErrTimeoutBase | site when it gives up).
constexpr uint32_t kSiteSignalBarrier = 0xF0;

// Query tiles of one launch of the tensor-core forward. With clean-tangent-zero
// teacher forcing (tq, tk, tv vanish on rows < L) a call runs as two launches,
// one per kind of query tile: each kernel instantiation carries only its own
// kind's code, with no runtime branch on the kind.
enum TileKind : int32_t {
  kTilesAll = 0,       // dense tangents, every query tile
  kTilesNoisyCTZ = 1,  // clean-tangent-zero: tiles with a noisy row (q1 > L)
  kTilesCleanCTZ = 2,  // clean-tangent-zero: tiles of clean rows only (primal only)
};

// Largest number of sequence slices one output map scatters to: the GPUs of
// one NVSwitch domain.
constexpr int kMaxShards = 8;

// Where the output rows of a launch go. The packed sequence of N rows is cut
// into `shards` equal slices of `shard_len` rows; slice r lives in buffers
// o[r], to[r], lse[r], tlse[r]. In context-parallel (Ulysses) attention slice r
// belongs to rank r and those buffers are its memory, reached over NVLink, so
// the epilogue itself performs the output all-to-all. Head h of the launch
// (bh = b * heads + h) is head head_base + h of the heads_total heads each slice
// holds. O, tO: [B, heads_total, shard_len, D], or [B, shard_len, heads_total, D]
// when token_major (the input layout of the output projection). LSE, tLSE:
// [B, heads_total, shard_len]. One slice with head_base = 0 and
// heads_total = heads is the plain [B, H, N, D] output.
struct OutMap {
  void *o[kMaxShards], *to[kMaxShards];
  float *lse[kMaxShards], *tlse[kMaxShards];
  int32_t shards, shard_len;
  int32_t heads, head_base, heads_total;
  int32_t token_major;
};

// Output row q of head bh: its slice, its O/tO row (in units of D elements)
// and its LSE/tLSE element.
struct OutRow {
  int32_t shard;
  size_t row, stat;
};

__host__ __device__ inline OutRow slice_row(const OutMap &m, int32_t bh, int32_t q) {
  const int32_t b = bh / m.heads, h = m.head_base + bh % m.heads;
  const int32_t r = q / m.shard_len, ql = q - r * m.shard_len;
  OutRow o;
  o.shard = r;
  o.stat = (size_t(b) * m.heads_total + h) * m.shard_len + ql;
  o.row = m.token_major ? (size_t(b) * m.shard_len + ql) * m.heads_total + h : o.stat;
  return o;
}

// Element offset of output row q of head bh (= b H + h) in a one-slice output:
// [B, H, N, D] when out_heads == 0, else token-major [B, N, H, D] with
// H = out_heads. Equal to slice_row of the one-slice map, times D.
__host__ __device__ inline size_t out_row(int32_t bh, int32_t q, int32_t N, int32_t out_heads, int D) {
  if (out_heads == 0) return (size_t(bh) * N + q) * D;
  const int32_t b = bh / out_heads, h = bh % out_heads;
  return ((size_t(b) * N + q) * out_heads + h) * D;
}

struct Sm100Params {
  CUtensorMap tm_q, tm_tq, tm_k, tm_tk, tm_v, tm_tv;  // 3-D maps over [B*H, N, D]
  void *o, *to;          // one-slice output: [B*H, N, D] bf16
  float *lse, *tlse;     // [B*H, N]
  MaskGeom geom;
  int32_t BH;
  int32_t n_qtiles;
  float scale;           // softmax scale
  float scale_log2e;     // scale * log2(e)
  uint64_t timeout_ns;   // bounded-wait limit
  int32_t fault_mode;    // test hook: 1 = skip the query-tile copies
  int32_t tile_kind;     // TileKind: the query tiles this launch covers
  int32_t out_heads;     // H when O, tO are token-major [B, N, H, D]; 0: [B, H, N, D]
  uint16_t qtile_order[kMaxQTiles];  // heaviest query tiles first
  // Sequence slices of a context-parallel output. shards == 0: the launch
  // writes the one-slice output above; otherwise the scattering
  // instantiations write through this map and o, to, lse, tlse are unused.
  OutMap scatter;
};

struct SimtParams {
  const void *q, *k, *v, *tq, *tk, *tv;
  OutMap out;  // where O, tO (fp32) and LSE, tLSE rows go
  MaskGeom geom;
  int32_t BH;
  float scale;
};

struct PrologueParams {
  const void *xq, *xk, *xv, *txq, *txk, *txv;  // [B, N, H*D] bf16
  const float *gq, *gk;                        // [H*D]
  const float *rope_cos, *rope_sin;            // [N, D/2]
  void *q, *k, *v, *tq, *tk, *tv;              // [B, H, N, D] bf16
  int32_t B, N, H, D;
  float eps;
  int32_t per_head;
};

struct BwdParams {
  // dq kernel: streamed K, V (64-row boxes); Q and dO rows are read into TMEM;
  // dkdv kernel: resident V (128-row box), streamed Q, dO (64-row boxes); K
  // rows are read into TMEM
  CUtensorMap tm_k_s, tm_v_s, tm_v_r, tm_q_s, tm_do_s;
  const void *q, *k;      // [B*H, N, D] bf16
  const void *o, *dout;   // [B*H, N, D] bf16 (o for Delta only)
  const float *lse;       // [B*H, N] natural log, from the forward
  float *delta;           // [B*H, N] Delta = <dO, O> (written by the pre-pass)
  void *dq, *dk, *dv;     // [B*H, N, D] bf16
  MaskGeom geom;
  int32_t BH;
  int32_t n_row_tiles;    // ceil(N / 128), for both query and key tiles
  float scale;
  uint64_t timeout_ns;
  uint16_t row_order[kMaxQTiles];  // query tiles, heaviest first (dq kernel)
  uint16_t col_order[kMaxQTiles];  // key tiles, heaviest first (dkdv kernel)
  int32_t fault_mode;     // test hook: 1 = the producers issue no copies
};

// Output projection in primal-tangent form: y = x W^T + b, ty = tx W^T.
// 2-D bf16 maps, innermost dimension first, 128-byte swizzle:
//   tm_x, tm_tx over [M, K], box 64 x 128 (a CTA's half of a 256-row tile);
//   tm_w over [C, K], box 64 x 128 (a CTA's half of a 256-row weight tile);
//   tm_y, tm_ty over [M, C], box 64 x 32 (the epilogue's store box).
struct OutProjParams {
  CUtensorMap tm_x, tm_tx, tm_w, tm_y, tm_ty;
  const void *bias;      // [C] bf16 or null
  int32_t M, K, C;
  uint64_t timeout_ns;
  int32_t fault_mode;    // test hook: 1 = the producer issues no copies
};

// Signal barrier of a context-parallel group: pads[r] is rank r's pad of
// kMaxShards words as mapped in this process.
struct SignalParams {
  uint32_t *pads[kMaxShards];
  int32_t shards, rank;
  uint32_t epoch;
  uint64_t timeout_ns;
};

// Runs `set` (a per-device kernel attribute setting, e.g. its shared-memory
// limit) the first time a call site launches on the current device: function
// attributes hold per device, so a process that drives several GPUs sets them
// on each. `done` is the call site's bit set of devices (ordinals below 64).
template <class F>
inline cudaError_t once_per_device(std::atomic<uint64_t> &done, F set) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load() & bit)) return cudaSuccess;
  e = set();
  if (e == cudaSuccess && bit) done.fetch_or(bit);
  return e;
}

// Each returns the launch's cudaError_t (cudaSuccess when enqueued).
cudaError_t launch_fwd_jvp_sm100(const Sm100Params &p, int D, cudaStream_t stream);
cudaError_t launch_fwd_jvp_simt_f32(const SimtParams &p, int D, cudaStream_t stream);
cudaError_t launch_qk_norm_rope_jvp(const PrologueParams &p, cudaStream_t stream);
cudaError_t launch_attn_bwd_sm100(const BwdParams &p, int D, cudaStream_t stream);
cudaError_t read_and_clear_bwd_error(uint32_t *out);
cudaError_t launch_signal_barrier(const SignalParams &p, cudaStream_t stream);
cudaError_t launch_out_proj_sm100(const OutProjParams &p, cudaStream_t stream);
cudaError_t read_and_clear_proj_error(uint32_t *out);
cudaError_t read_and_clear_signal_error(uint32_t *out);

// Device error word access (defined next to the kernels that write it).
cudaError_t read_and_clear_device_error(cudaStream_t stream, uint32_t *out);

}  // namespace caj
