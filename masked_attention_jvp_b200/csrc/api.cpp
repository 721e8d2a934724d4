// C-ABI front end of libcausaljvp: argument validation, the query-tile launch
// order, TMA descriptor construction and kernel dispatch. See
// include/causaljvp.h for the contract of every entry point.
#include "causaljvp.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <limits>
#include <map>
#include <memory>
#include <utility>
#include <mutex>
#include <vector>

#include "kernels.h"
#include "mask_schedule.h"

namespace {

thread_local char g_cuda_msg[256] = "";
uint32_t g_last_device_code = 0;

caj_status cuda_fail(cudaError_t e) {
  std::snprintf(g_cuda_msg, sizeof g_cuda_msg, "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return CAJ_ERR_CUDA;
}

bool geom_from_desc(const caj_mask_desc *m, caj::MaskGeom *g) {
  if (!m) return false;
  const int64_t T = m->tokens_per_frame, c = m->frames_per_chunk, F = m->n_frames;
  if (T <= 0 || c <= 0 || F <= 0) return false;
  if (m->tf_layout != 0 && m->tf_layout != 1) return false;
  if (F % c != 0) return false;
  const int64_t L = F * T, N = L * (m->tf_layout ? 2 : 1);
  if (N > (int64_t(1) << 30)) return false;
  g->G = int32_t(c * T);
  g->L = int32_t(L);
  g->N = int32_t(N);
  g->tf = m->tf_layout;
  return true;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// cuTensorMapEncodeTiled, fetched from the driver through the runtime so the
// library needs no link-time dependency on libcuda.
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_tiled() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 3-D bf16 map over [BH, N, D] (innermost first), box = 64 columns x rows x 1,
// 128-byte swizzle, zero fill outside the tensor.
bool encode_map(EncodeTiledFn enc, CUtensorMap *map, const void *base, int BH, int N, int D,
                int box_rows) {
  cuuint64_t dims[3] = {cuuint64_t(D), cuuint64_t(N), cuuint64_t(BH)};
  cuuint64_t strides[2] = {cuuint64_t(D) * 2, cuuint64_t(N) * D * 2};
  cuuint32_t box[3] = {64, cuuint32_t(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Per-device check that this is an sm_100 part (cached).
caj_status check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  static std::mutex mu;
  static std::vector<int> state;  // 0 unknown, 1 ok, 2 unsupported
  std::lock_guard<std::mutex> lock(mu);
  if (int(state.size()) <= dev) state.resize(dev + 1, 0);
  if (state[dev] == 0) {
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return cuda_fail(e);
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_fail(e);
    state[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return state[dev] == 1 ? CAJ_OK : CAJ_ERR_UNSUPPORTED;
}

std::atomic<uint64_t> g_timeout_override_ns{0};
std::atomic<int32_t> g_fault_mode{0};

uint64_t wait_timeout_ns() {
  const uint64_t o = g_timeout_override_ns.load();
  if (o) return o;
  static uint64_t ns = [] {
    const char *s = std::getenv("CAJ_WAIT_TIMEOUT_MS");
    double ms = s ? std::atof(s) : 0.0;
    if (!(ms > 0.0)) ms = 2000.0;
    return uint64_t(ms * 1e6);
  }();
  return ns;
}

}  // namespace

namespace {

// ------------------------------------------------ output projection
// 2-D bf16 map over a row-major [rows, cols] matrix, box = 64 columns x box_rows,
// 128-byte swizzle, zero fill outside the matrix.
bool encode_map_2d(EncodeTiledFn enc, CUtensorMap *map, const void *base, int64_t rows, int64_t cols,
                   int box_rows) {
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(cols) * 2};
  cuuint32_t box[2] = {64, cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Shape, dtype, flag and mask checks shared by the device and host forms of
// the forward.
caj_status validate_fwd(const caj_problem *prob, const caj_mask_desc *mask, caj::MaskGeom *g) {
  if (!prob || !mask) return CAJ_ERR_INVALID_ARG;
  if (prob->B <= 0 || prob->H <= 0 || prob->N <= 0 || prob->D <= 0) return CAJ_ERR_INVALID_ARG;
  if (!geom_from_desc(mask, g) || g->N != prob->N) return CAJ_ERR_INVALID_ARG;
  if (prob->dtype != CAJ_DTYPE_F32 && prob->dtype != CAJ_DTYPE_BF16) return CAJ_ERR_INVALID_ARG;
  if (!(prob->scale >= 0.f) || std::isinf(prob->scale)) return CAJ_ERR_INVALID_ARG;
  if (prob->flags & ~int32_t(CAJ_FLAG_CLEAN_TANGENT_ZERO | CAJ_FLAG_TOKEN_MAJOR_OUT))
    return CAJ_ERR_INVALID_ARG;
  if ((prob->flags & CAJ_FLAG_CLEAN_TANGENT_ZERO) && !mask->tf_layout) return CAJ_ERR_INVALID_ARG;
  if (prob->D != 64 && prob->D != 128) return CAJ_ERR_UNSUPPORTED;
  const int64_t BH = int64_t(prob->B) * prob->H;
  if (BH > 65535 || prob->N > (1 << 20)) return CAJ_ERR_UNSUPPORTED;
  return CAJ_OK;
}

// Device workspace of the host-buffer forward: the six inputs, O, tO, LSE and
// tLSE, each region 256-byte aligned.
struct HostWorkspace {
  size_t in[6], o, to, lse, tlse, total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool host_workspace(const caj_problem *prob, HostWorkspace *w) {
  if (!prob || prob->B <= 0 || prob->H <= 0 || prob->N <= 0 || prob->D <= 0) return false;
  const size_t es = prob->dtype == CAJ_DTYPE_BF16 ? 2 : prob->dtype == CAJ_DTYPE_F32 ? 4 : 0;
  if (!es) return false;
  const size_t rows = size_t(prob->B) * size_t(prob->H) * size_t(prob->N);
  const size_t tensor = align256(rows * size_t(prob->D) * es), stats = align256(rows * 4);
  size_t off = 0;
  for (int i = 0; i < 6; ++i, off += tensor) w->in[i] = off;
  w->o = off;
  off += tensor;
  w->to = off;
  off += tensor;
  w->lse = off;
  off += stats;
  w->tlse = off;
  off += stats;
  w->total = off;
  return true;
}

// Copy streams and events of the host-buffer forward, one set per device,
// created on first use and kept for the life of the process.
constexpr int kHostChunks = 16;  // at most this many head chunks per call
constexpr int kEndPieces = 2;  // the first and the last chunk go in this many pieces
constexpr int kHostPieces = kHostChunks + 2 * (kEndPieces - 1);
struct HostPipe {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t in_ready[kHostPieces] = {}, out_ready[kHostPieces] = {};
};
std::mutex g_pipe_mu;
std::vector<std::unique_ptr<HostPipe>> g_pipes;

cudaError_t host_pipe(int dev, HostPipe **out) {
  if (int(g_pipes.size()) <= dev) g_pipes.resize(dev + 1);
  if (!g_pipes[dev]) {
    std::unique_ptr<HostPipe> p(new HostPipe());
    cudaError_t e = cudaStreamCreateWithFlags(&p->in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->out, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->start, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->done, cudaEventDisableTiming);
    for (int c = 0; c < kHostPieces && e == cudaSuccess; ++c) {
      e = cudaEventCreateWithFlags(&p->in_ready[c], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->out_ready[c], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) return e;  // the partial set is not kept; nothing was enqueued
    g_pipes[dev] = std::move(p);
  }
  *out = g_pipes[dev].get();
  return cudaSuccess;
}

}  // namespace

extern "C" {

const char *caj_status_string(caj_status s) {
  switch (s) {
    case CAJ_OK: return "CAJ_OK";
    case CAJ_ERR_INVALID_ARG: return "CAJ_ERR_INVALID_ARG";
    case CAJ_ERR_UNSUPPORTED: return "CAJ_ERR_UNSUPPORTED";
    case CAJ_ERR_CUDA: return "CAJ_ERR_CUDA";
    case CAJ_ERR_DEVICE_TIMEOUT: return "CAJ_ERR_DEVICE_TIMEOUT";
  }
  return "CAJ_ERR_UNKNOWN";
}

const char *caj_last_cuda_error(void) { return g_cuda_msg; }

caj_status caj_set_wait_timeout_ms(double ms) {
  g_timeout_override_ns.store(ms > 0.0 ? uint64_t(ms * 1e6) : 0);
  return CAJ_OK;
}

caj_status caj_debug_set_fault(int32_t mode) {
  if (mode != 0 && mode != 1) return CAJ_ERR_INVALID_ARG;
  g_fault_mode.store(mode);
  return CAJ_OK;
}

int32_t caj_version(void) { return 100; }

caj_status caj_validate_mask(const caj_mask_desc *mask, int32_t N) {
  caj::MaskGeom g;
  if (!geom_from_desc(mask, &g)) return CAJ_ERR_INVALID_ARG;
  return g.N == N ? CAJ_OK : CAJ_ERR_INVALID_ARG;
}

int64_t caj_visible_pairs(const caj_mask_desc *mask) {
  caj::MaskGeom g;
  if (!geom_from_desc(mask, &g)) return -1;
  return caj::visible_pairs(g);
}

caj_status caj_row_key_ranges(const caj_mask_desc *mask, int32_t row, int32_t r[4]) {
  caj::MaskGeom g;
  if (!geom_from_desc(mask, &g) || !r || row < 0 || row >= g.N) return CAJ_ERR_INVALID_ARG;
  caj::row_key_ranges(g, row, r[0], r[1], r[2], r[3]);
  return CAJ_OK;
}

int32_t caj_qtile_key_tiles(const caj_mask_desc *mask, int32_t q0, int32_t q1, int32_t block_n,
                            int32_t t[4]) {
  caj::MaskGeom g;
  if (!geom_from_desc(mask, &g) || !t || block_n <= 0 || q0 < 0 || q1 <= q0 || q1 > g.N)
    return -1;
  return caj::qtile_key_tiles(g, q0, q1, block_n, t[0], t[1], t[2], t[3]);
}

caj_status caj_key_query_ranges(const caj_mask_desc *mask, int32_t key, int32_t r[4]) {
  caj::MaskGeom g;
  if (!geom_from_desc(mask, &g) || !r || key < 0 || key >= g.N) return CAJ_ERR_INVALID_ARG;
  caj::key_query_ranges(g, key, r[0], r[1], r[2], r[3]);
  return CAJ_OK;
}

int32_t caj_ktile_query_tiles(const caj_mask_desc *mask, int32_t k0, int32_t k1, int32_t block_q,
                              int32_t t[6]) {
  caj::MaskGeom g;
  if (!geom_from_desc(mask, &g) || !t || block_q <= 0 || k0 < 0 || k1 <= k0 || k1 > g.N) return -1;
  int32_t tt[6];
  const int32_t n = caj::ktile_query_tiles(g, k0, k1, block_q, tt);
  for (int i = 0; i < 6; ++i) t[i] = tt[i];
  return n;
}

namespace {

// The query tiles (of kBlockM rows) in heaviest-first order: by decreasing
// number of visited key tiles, ties later tile first.
std::vector<std::pair<int32_t, int32_t>> qtile_costs(const caj::MaskGeom &g) {
  const int32_t n_qtiles = (g.N + caj::kBlockM - 1) / caj::kBlockM;
  std::vector<std::pair<int32_t, int32_t>> cost(n_qtiles);
  for (int32_t t = 0; t < n_qtiles; ++t) {
    int32_t r[4];
    const int32_t q0 = t * caj::kBlockM, q1 = std::min(q0 + caj::kBlockM, g.N);
    cost[t] = {caj::qtile_key_tiles(g, q0, q1, caj::kBlockN, r[0], r[1], r[2], r[3]), t};
  }
  std::sort(cost.begin(), cost.end(), [](const auto &a, const auto &b) {
    return a.first != b.first ? a.first > b.first : a.second > b.second;
  });
  return cost;
}

// Part `part` of `nparts` of the query tiles, balanced by cost: the tiles go
// heaviest first, each to the part with the least work so far (lowest index on
// ties), so parts differ by at most one tile's work. Every head has the same
// mask, so a part runs its tiles for all heads. Heaviest-first order is kept.
std::vector<std::pair<int32_t, int32_t>> part_of(const std::vector<std::pair<int32_t, int32_t>> &cost,
                                                 int32_t part, int32_t nparts) {
  if (nparts <= 1) return cost;
  std::vector<int64_t> load(nparts, 0);
  std::vector<std::pair<int32_t, int32_t>> mine;
  for (const auto &c : cost) {
    int32_t best = 0;
    for (int32_t r = 1; r < nparts; ++r)
      if (load[r] < load[best]) best = r;
    load[best] += c.first;
    if (best == part) mine.push_back(c);
  }
  return mine;
}

// Launches the forward + JVP of a validated problem on `s`, the output rows
// placed by `out`: a one-slice output, or (scatter) the slices of a
// context-parallel output. With nparts > 1 only the query tiles of part
// `part` run, and only those in [tile_lo, tile_hi) (tensor-core path).
caj_status fwd_launch(const void *const in[6], const caj_problem *prob, const caj::MaskGeom &g,
                      const caj::OutMap &out, bool scatter, cudaStream_t s, int32_t part = 0,
                      int32_t nparts = 1, int32_t tile_lo = 0,
                      int32_t tile_hi = std::numeric_limits<int32_t>::max()) {
  const void *q = in[0], *k = in[1], *v = in[2], *tq = in[3], *tk = in[4], *tv = in[5];
  const int64_t BH = int64_t(prob->B) * prob->H;
  const float scale = prob->scale > 0.f ? prob->scale : 1.0f / std::sqrt(float(prob->D));

  if (prob->dtype == CAJ_DTYPE_F32) {
    caj::SimtParams p{};
    p.q = q; p.k = k; p.v = v; p.tq = tq; p.tk = tk; p.tv = tv;
    p.out = out;
    p.geom = g;
    p.BH = int32_t(BH);
    p.scale = scale;
    cudaError_t e = caj::launch_fwd_jvp_simt_f32(p, prob->D, s);
    return e == cudaSuccess ? CAJ_OK : cuda_fail(e);
  }
  const int32_t n_qtiles = (prob->N + caj::kBlockM - 1) / caj::kBlockM;
  if (n_qtiles > caj::kMaxQTiles) return CAJ_ERR_UNSUPPORTED;
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return cuda_fail(cudaErrorNotSupported);

  // Parameters live in a heap block: the struct carries the launch order table.
  std::unique_ptr<caj::Sm100Params> hp(new caj::Sm100Params());
  caj::Sm100Params &p = *hp;
  const int N = prob->N, D = prob->D;
  bool okm = encode_map(enc, &p.tm_q, q, int(BH), N, D, caj::kBlockM) &&
             encode_map(enc, &p.tm_tq, tq, int(BH), N, D, caj::kBlockM) &&
             encode_map(enc, &p.tm_k, k, int(BH), N, D, caj::kBlockN) &&
             encode_map(enc, &p.tm_tk, tk, int(BH), N, D, caj::kBlockN) &&
             encode_map(enc, &p.tm_v, v, int(BH), N, D, caj::kBlockN) &&
             encode_map(enc, &p.tm_tv, tv, int(BH), N, D, caj::kBlockN);
  if (!okm) return cuda_fail(cudaErrorInvalidValue);
  if (scatter) {
    p.scatter = out;
  } else {
    p.o = out.o[0]; p.to = out.to[0]; p.lse = out.lse[0]; p.tlse = out.tlse[0];
    p.out_heads = out.token_major ? prob->H : 0;
  }
  p.geom = g;
  p.BH = int32_t(BH);
  p.n_qtiles = n_qtiles;
  p.scale = scale;
  p.scale_log2e = scale * 1.4426950408889634f;
  p.timeout_ns = wait_timeout_ns();
  p.fault_mode = g_fault_mode.load();
  p.tile_kind = caj::kTilesAll;
  // Launch order: query tiles by decreasing number of key tiles (ties: later
  // first); with parts, this part's tiles only.
  std::vector<std::pair<int32_t, int32_t>> cost = part_of(qtile_costs(g), part, nparts);
  if (tile_lo > 0 || tile_hi < n_qtiles)
    cost.erase(std::remove_if(cost.begin(), cost.end(),
                              [&](const std::pair<int32_t, int32_t> &c) {
                                return c.second < tile_lo || c.second >= tile_hi;
                              }),
               cost.end());
  if (cost.empty()) return CAJ_OK;  // a part with no tile: nothing to launch
  p.n_qtiles = int32_t(cost.size());
  if (prob->flags & CAJ_FLAG_CLEAN_TANGENT_ZERO) {
    // Two launches, each over one kind of query tile in the same heaviest-first
    // order: tiles with a noisy row (the dearer ones) first, then the clean ones.
    std::unique_ptr<caj::Sm100Params> hc(new caj::Sm100Params(p));
    int32_t nn = 0, nc = 0;
    for (const auto &c : cost) {
      const int32_t t = c.second;
      if (std::min((t + 1) * caj::kBlockM, N) <= g.L)
        hc->qtile_order[nc++] = uint16_t(t);
      else
        p.qtile_order[nn++] = uint16_t(t);
    }
    p.tile_kind = caj::kTilesNoisyCTZ;
    p.n_qtiles = nn;
    hc->tile_kind = caj::kTilesCleanCTZ;
    hc->n_qtiles = nc;
    cudaError_t e = nn ? caj::launch_fwd_jvp_sm100(p, D, s) : cudaSuccess;
    if (e == cudaSuccess && nc) e = caj::launch_fwd_jvp_sm100(*hc, D, s);
    return e == cudaSuccess ? CAJ_OK : cuda_fail(e);
  }
  for (size_t i = 0; i < cost.size(); ++i) p.qtile_order[i] = uint16_t(cost[i].second);

  cudaError_t e = caj::launch_fwd_jvp_sm100(p, D, s);
  return e == cudaSuccess ? CAJ_OK : cuda_fail(e);
}

}  // namespace

caj_status caj_attn_fwd_jvp(const void *q, const void *k, const void *v, const void *tq,
                            const void *tk, const void *tv, const caj_problem *prob,
                            const caj_mask_desc *mask, void *o, void *to, float *lse, float *tlse,
                            void *stream) {
  const void *ins[6] = {q, k, v, tq, tk, tv};
  for (const void *p : ins)
    if (!p || !aligned16(p)) return CAJ_ERR_INVALID_ARG;
  if (!o || !to || !aligned16(o) || !aligned16(to)) return CAJ_ERR_INVALID_ARG;
  if (!lse || !tlse || !aligned4(lse) || !aligned4(tlse)) return CAJ_ERR_INVALID_ARG;
  caj::MaskGeom g;
  caj_status st = validate_fwd(prob, mask, &g);
  if (st != CAJ_OK) return st;
  st = check_device();
  if (st != CAJ_OK) return st;

  caj::OutMap out{};
  out.o[0] = o; out.to[0] = to; out.lse[0] = lse; out.tlse[0] = tlse;
  out.shards = 1;
  out.shard_len = prob->N;
  out.heads = out.heads_total = prob->H;
  out.head_base = 0;
  out.token_major = (prob->flags & CAJ_FLAG_TOKEN_MAJOR_OUT) ? 1 : 0;
  return fwd_launch(ins, prob, g, out, false, static_cast<cudaStream_t>(stream));
}

caj_status caj_attn_fwd_jvp_part(const void *q, const void *k, const void *v, const void *tq,
                                 const void *tk, const void *tv, const caj_problem *prob,
                                 const caj_mask_desc *mask, int32_t part, int32_t nparts, void *o,
                                 void *to, float *lse, float *tlse, void *stream) {
  const void *ins[6] = {q, k, v, tq, tk, tv};
  for (const void *p : ins)
    if (!p || !aligned16(p)) return CAJ_ERR_INVALID_ARG;
  if (!o || !to || !aligned16(o) || !aligned16(to)) return CAJ_ERR_INVALID_ARG;
  if (!lse || !tlse || !aligned4(lse) || !aligned4(tlse)) return CAJ_ERR_INVALID_ARG;
  if (nparts < 1 || part < 0 || part >= nparts) return CAJ_ERR_INVALID_ARG;
  caj::MaskGeom g;
  caj_status st = validate_fwd(prob, mask, &g);
  if (st != CAJ_OK) return st;
  if (prob->dtype != CAJ_DTYPE_BF16 && nparts > 1) return CAJ_ERR_UNSUPPORTED;  // tensor-core path only
  st = check_device();
  if (st != CAJ_OK) return st;
  caj::OutMap out{};
  out.o[0] = o; out.to[0] = to; out.lse[0] = lse; out.tlse[0] = tlse;
  out.shards = 1;
  out.shard_len = prob->N;
  out.heads = out.heads_total = prob->H;
  out.head_base = 0;
  out.token_major = (prob->flags & CAJ_FLAG_TOKEN_MAJOR_OUT) ? 1 : 0;
  return fwd_launch(ins, prob, g, out, false, static_cast<cudaStream_t>(stream), part, nparts);
}

int32_t caj_part_query_tiles(const caj_mask_desc *mask, int32_t part, int32_t nparts, int32_t *tiles,
                             int32_t capacity) {
  caj::MaskGeom g;
  if (!geom_from_desc(mask, &g) || nparts < 1 || part < 0 || part >= nparts || capacity < 0) return -1;
  const auto mine = part_of(qtile_costs(g), part, nparts);
  if (tiles)
    for (size_t i = 0; i < mine.size() && int32_t(i) < capacity; ++i) tiles[i] = mine[i].second;
  return int32_t(mine.size());
}

static_assert(CAJ_MAX_SHARDS == caj::kMaxShards, "slice count of the public and kernel output maps");

caj_status caj_attn_fwd_jvp_scatter(const void *q, const void *k, const void *v, const void *tq,
                                    const void *tk, const void *tv, const caj_problem *prob,
                                    const caj_mask_desc *mask, const caj_seq_scatter *dst,
                                    void *stream) {
  const void *ins[6] = {q, k, v, tq, tk, tv};
  for (const void *p : ins)
    if (!p || !aligned16(p)) return CAJ_ERR_INVALID_ARG;
  caj::MaskGeom g;
  caj_status st = validate_fwd(prob, mask, &g);
  if (st != CAJ_OK) return st;
  if (!dst || dst->shards < 1 || dst->shards > CAJ_MAX_SHARDS || prob->N % dst->shards)
    return CAJ_ERR_INVALID_ARG;
  if (dst->head_base < 0 || dst->heads_total < prob->H || dst->head_base > dst->heads_total - prob->H)
    return CAJ_ERR_INVALID_ARG;
  for (int32_t r = 0; r < dst->shards; ++r) {
    if (!dst->o[r] || !dst->to[r] || !aligned16(dst->o[r]) || !aligned16(dst->to[r]))
      return CAJ_ERR_INVALID_ARG;
    if (!dst->lse[r] || !dst->tlse[r] || !aligned4(dst->lse[r]) || !aligned4(dst->tlse[r]))
      return CAJ_ERR_INVALID_ARG;
  }
  st = check_device();
  if (st != CAJ_OK) return st;
  // the epilogue writes the slices with device stores: host memory (pinned or
  // not) is refused here rather than met by the kernel
  for (int32_t r = 0; r < dst->shards; ++r) {
    const void *slice[4] = {dst->o[r], dst->to[r], dst->lse[r], dst->tlse[r]};
    for (const void *ptr : slice) {
      cudaPointerAttributes a{};
      cudaError_t e = cudaPointerGetAttributes(&a, ptr);
      if (e != cudaSuccess) {
        (void)cudaGetLastError();  // the failed query leaves its error behind: clear it
        return CAJ_ERR_INVALID_ARG;
      }
      if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return CAJ_ERR_INVALID_ARG;
    }
  }

  caj::OutMap out{};
  for (int32_t r = 0; r < dst->shards; ++r) {
    out.o[r] = dst->o[r]; out.to[r] = dst->to[r];
    out.lse[r] = dst->lse[r]; out.tlse[r] = dst->tlse[r];
  }
  out.shards = dst->shards;
  out.shard_len = prob->N / dst->shards;
  out.heads = prob->H;
  out.head_base = dst->head_base;
  out.heads_total = dst->heads_total;
  out.token_major = (prob->flags & CAJ_FLAG_TOKEN_MAJOR_OUT) ? 1 : 0;
  return fwd_launch(ins, prob, g, out, true, static_cast<cudaStream_t>(stream));
}

caj_status caj_attn_fwd_jvp_host_workspace(const caj_problem *prob, size_t *bytes) {
  HostWorkspace w;
  if (!bytes || !host_workspace(prob, &w)) return CAJ_ERR_INVALID_ARG;
  *bytes = w.total;
  return CAJ_OK;
}

caj_status caj_attn_fwd_jvp_host(const void *q, const void *k, const void *v, const void *tq,
                                 const void *tk, const void *tv, const caj_problem *prob,
                                 const caj_mask_desc *mask, void *o, void *to, float *lse,
                                 float *tlse, void *workspace, size_t workspace_bytes,
                                 void *stream) {
  const void *hin[6] = {q, k, v, tq, tk, tv};
  for (const void *p : hin)
    if (!p) return CAJ_ERR_INVALID_ARG;
  if (!o || !to || !lse || !tlse) return CAJ_ERR_INVALID_ARG;
  caj::MaskGeom g;
  caj_status st = validate_fwd(prob, mask, &g);
  if (st != CAJ_OK) return st;
  // head chunks are copied as contiguous blocks: head-major outputs only
  if (prob->flags & CAJ_FLAG_TOKEN_MAJOR_OUT) return CAJ_ERR_INVALID_ARG;
  HostWorkspace w;
  if (!host_workspace(prob, &w) || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < w.total)
    return CAJ_ERR_INVALID_ARG;
  st = check_device();
  if (st != CAJ_OK) return st;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);

  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe *pp = nullptr;
  if ((e = host_pipe(dev, &pp)) != cudaSuccess) return cuda_fail(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  const size_t es = prob->dtype == CAJ_DTYPE_BF16 ? 2 : 4;
  const int64_t BH = int64_t(prob->B) * prob->H;
  const int64_t hpc = (BH + kHostChunks - 1) / kHostChunks;  // heads per chunk
  const int64_t nchunks = (BH + hpc - 1) / hpc;
  const int32_t N = prob->N;
  const size_t row_bytes = size_t(prob->D) * es, head_bytes = size_t(N) * row_bytes;

  // Pieces: a chunk of heads, the query tiles [t_lo, t_hi) that run on it, its
  // query rows [r0, r1) and the key rows [k0, k1) first copied for it (earlier
  // pieces of the chunk copied the rest of what its tiles read). The first and
  // the last chunk go in kEndPieces pieces of consecutive query tiles; piece p
  // copies the keys its tiles read beyond those of the pieces before it. The
  // kernels then start after a fraction of a chunk's copy, and after the last
  // copy only that fraction is left to run and copy back. (tensor-core path;
  // the fp32 path runs whole heads.) Measured on the TF frame-wise workload:
  // two pieces are 3% faster end to end than whole chunks, four pieces 2%; the
  // extra launches and strided copies of more pieces cost more than they save.
  struct Piece {
    int64_t h0, nh;
    int32_t t_lo, t_hi, r0, r1, k0, k1;
  };
  const int32_t n_qt = (N + caj::kBlockM - 1) / caj::kBlockM;
  const int32_t P = prob->dtype == CAJ_DTYPE_BF16 ? std::min<int32_t>(kEndPieces, n_qt) : 1;
  int32_t tb[kEndPieces + 1], rb[kEndPieces + 1], kb[kEndPieces + 1];
  for (int32_t i = 0; i <= P; ++i) tb[i] = int32_t(int64_t(i) * n_qt / P);
  // teacher forcing: the first piece ends with the clean rows where it can, so
  // that it reads no noisy keys
  if (P == 2 && g.tf && g.L / caj::kBlockM >= 1) tb[1] = std::min(tb[1], g.L / caj::kBlockM);
  for (int32_t i = 0; i <= P; ++i) rb[i] = std::min(tb[i] * caj::kBlockM, N);
  kb[0] = 0;
  for (int32_t i = 1, t = 0, kmax = 0; i <= P; ++i) {  // running maximum of the key rows read
    for (; t < tb[i]; ++t) {
      int32_t r[4];
      caj::qtile_key_tiles(g, t * caj::kBlockM, std::min((t + 1) * caj::kBlockM, N), caj::kBlockN, r[0], r[1],
                           r[2], r[3]);
      kmax = std::max(kmax, std::max(r[1], r[3]) * caj::kBlockN);
    }
    kb[i] = i == P ? N : std::min(kmax, N);
  }
  Piece pieces[kHostPieces];
  int np = 0;
  for (int64_t c = 0; c < nchunks; ++c) {
    const int64_t h0 = c * hpc, nh = std::min(hpc, BH - h0);
    if (P > 1 && (c == 0 || c == nchunks - 1)) {
      for (int32_t i = 0; i < P; ++i) pieces[np++] = Piece{h0, nh, tb[i], tb[i + 1], rb[i], rb[i + 1], kb[i], kb[i + 1]};
    } else {
      pieces[np++] = Piece{h0, nh, 0, n_qt, 0, N, 0, N};
    }
  }

  // Both copy streams start after the work already on `stream` (an earlier
  // call may still read this workspace), and `stream` ends after both.
  auto ok = [&](cudaError_t r) { return r == cudaSuccess || (e = r, false); };
  // rows [a, b) of every head of a piece, between the caller's tensor and the
  // workspace (one strided copy: the heads are `head_bytes` apart on both sides)
  auto copy_rows = [&](uint8_t *dst, const uint8_t *src, size_t rbytes, size_t pitch, const Piece &pc,
                       int32_t a, int32_t b, cudaMemcpyKind kind, cudaStream_t st) {
    if (b <= a) return true;
    const size_t off = size_t(pc.h0) * pitch + size_t(a) * rbytes;
    return ok(cudaMemcpy2DAsync(dst + off, pitch, src + off, pitch, size_t(b - a) * rbytes, size_t(pc.nh),
                                kind, st));
  };
  bool good = ok(cudaEventRecord(pp->start, s)) && ok(cudaStreamWaitEvent(pp->in, pp->start, 0)) &&
              ok(cudaStreamWaitEvent(pp->out, pp->start, 0));
  caj_status kst = CAJ_OK;
  const size_t stat_pitch = size_t(N) * 4;
  for (int i = 0; good && i < np; ++i) {
    const Piece &pc = pieces[i];
    for (int t = 0; good && t < 6; ++t) {
      const bool query = t == 0 || t == 3;  // q, tq: the piece's own rows; k, v, tk, tv: its key rows
      good = copy_rows(ws + w.in[t], static_cast<const uint8_t *>(hin[t]), row_bytes, head_bytes, pc,
                       query ? pc.r0 : pc.k0, query ? pc.r1 : pc.k1, cudaMemcpyHostToDevice, pp->in);
    }
    good = good && ok(cudaEventRecord(pp->in_ready[i], pp->in)) &&
           ok(cudaStreamWaitEvent(s, pp->in_ready[i], 0));
    if (!good) break;
    // the chunk's heads form a problem of their own: [1, nh, N, D] at head h0
    caj_problem sub = *prob;
    sub.B = 1;
    sub.H = int32_t(pc.nh);
    const size_t off = size_t(pc.h0) * head_bytes, soff = size_t(pc.h0) * stat_pitch;
    const void *ins[6];
    for (int t = 0; t < 6; ++t) ins[t] = ws + w.in[t] + off;
    caj::OutMap out{};
    out.o[0] = ws + w.o + off;
    out.to[0] = ws + w.to + off;
    out.lse[0] = reinterpret_cast<float *>(ws + w.lse + soff);
    out.tlse[0] = reinterpret_cast<float *>(ws + w.tlse + soff);
    out.shards = 1;
    out.shard_len = N;
    out.heads = out.heads_total = sub.H;
    kst = fwd_launch(ins, &sub, g, out, false, s, 0, 1, pc.t_lo, pc.t_hi);
    if (kst != CAJ_OK) break;
    good = ok(cudaEventRecord(pp->out_ready[i], s)) && ok(cudaStreamWaitEvent(pp->out, pp->out_ready[i], 0)) &&
           copy_rows(static_cast<uint8_t *>(o), ws + w.o, row_bytes, head_bytes, pc, pc.r0, pc.r1,
                     cudaMemcpyDeviceToHost, pp->out) &&
           copy_rows(static_cast<uint8_t *>(to), ws + w.to, row_bytes, head_bytes, pc, pc.r0, pc.r1,
                     cudaMemcpyDeviceToHost, pp->out) &&
           copy_rows(reinterpret_cast<uint8_t *>(lse), ws + w.lse, 4, stat_pitch, pc, pc.r0, pc.r1,
                     cudaMemcpyDeviceToHost, pp->out) &&
           copy_rows(reinterpret_cast<uint8_t *>(tlse), ws + w.tlse, 4, stat_pitch, pc, pc.r0, pc.r1,
                     cudaMemcpyDeviceToHost, pp->out);
  }
  // Join both copy streams back into `stream`, also after a failure, so that no
  // copy touches the caller's buffers once `stream` has passed this call.
  cudaError_t je = cudaEventRecord(pp->done, pp->in);
  if (je == cudaSuccess) je = cudaStreamWaitEvent(s, pp->done, 0);
  if (je == cudaSuccess) je = cudaEventRecord(pp->done, pp->out);
  if (je == cudaSuccess) je = cudaStreamWaitEvent(s, pp->done, 0);
  if (kst != CAJ_OK) return kst;
  if (!good) return cuda_fail(e);
  return je == cudaSuccess ? CAJ_OK : cuda_fail(je);
}

caj_status caj_out_proj_jvp(const void *x, const void *tx, const void *w, const void *bias,
                            const caj_linear_shape *shape, void *y, void *ty, void *stream) {
  if (!shape || shape->M <= 0 || shape->K <= 0 || shape->C <= 0) return CAJ_ERR_INVALID_ARG;
  if (shape->K % 8 || shape->C % 8) return CAJ_ERR_UNSUPPORTED;  // 16-byte rows
  const void *ptrs[5] = {x, tx, w, y, ty};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return CAJ_ERR_INVALID_ARG;
  if (bias && !aligned16(bias)) return CAJ_ERR_INVALID_ARG;
  if (shape->M > (int64_t(1) << 31) - 1) return CAJ_ERR_UNSUPPORTED;  // TMA row coordinates are 32-bit
  caj_status st = check_device();
  if (st != CAJ_OK) return st;
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return cuda_fail(cudaErrorNotSupported);
  caj::OutProjParams p{};
  const int64_t M = shape->M, K = shape->K, C = shape->C;
  const bool okm = encode_map_2d(enc, &p.tm_x, x, M, K, 128) && encode_map_2d(enc, &p.tm_tx, tx, M, K, 128) &&
                   encode_map_2d(enc, &p.tm_w, w, C, K, 128) && encode_map_2d(enc, &p.tm_y, y, M, C, 32) &&
                   encode_map_2d(enc, &p.tm_ty, ty, M, C, 32);
  if (!okm) return cuda_fail(cudaErrorInvalidValue);
  p.bias = bias;
  p.M = int32_t(M);
  p.K = K;
  p.C = C;
  p.timeout_ns = wait_timeout_ns();
  p.fault_mode = g_fault_mode.load();
  cudaError_t e = caj::launch_out_proj_sm100(p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CAJ_OK : cuda_fail(e);
}

caj_status caj_qk_norm_rope_jvp(const void *xq, const void *xk, const void *xv, const void *txq,
                                const void *txk, const void *txv, const float *gq, const float *gk,
                                const float *rope_cos, const float *rope_sin,
                                const caj_prologue_shape *shape, void *q, void *k, void *v, void *tq,
                                void *tk, void *tv, void *stream) {
  if (!shape) return CAJ_ERR_INVALID_ARG;
  const void *ptrs16[] = {xq, xk, xv, txq, txk, txv, gq, gk, rope_cos, rope_sin, q, k, v, tq, tk, tv};
  for (const void *p : ptrs16)
    if (!p || !aligned16(p)) return CAJ_ERR_INVALID_ARG;
  if (shape->B <= 0 || shape->N <= 0 || shape->H <= 0 || shape->D <= 0) return CAJ_ERR_INVALID_ARG;
  if (!(shape->eps >= 0.f) || std::isinf(shape->eps)) return CAJ_ERR_INVALID_ARG;
  if (shape->norm_per_head != 0 && shape->norm_per_head != 1) return CAJ_ERR_INVALID_ARG;
  if (shape->D != 64 && shape->D != 128) return CAJ_ERR_UNSUPPORTED;
  const int64_t C = int64_t(shape->H) * shape->D;
  if (C % 256 != 0 || C > 8192) return CAJ_ERR_UNSUPPORTED;
  if (int64_t(shape->B) * shape->N > (int64_t(1) << 31) - 1) return CAJ_ERR_UNSUPPORTED;
  caj_status st = check_device();
  if (st != CAJ_OK) return st;
  caj::PrologueParams p{};
  p.xq = xq; p.xk = xk; p.xv = xv; p.txq = txq; p.txk = txk; p.txv = txv;
  p.gq = gq; p.gk = gk; p.rope_cos = rope_cos; p.rope_sin = rope_sin;
  p.q = q; p.k = k; p.v = v; p.tq = tq; p.tk = tk; p.tv = tv;
  p.B = shape->B; p.N = shape->N; p.H = shape->H; p.D = shape->D;
  p.eps = shape->eps;
  p.per_head = shape->norm_per_head;
  cudaError_t e = caj::launch_qk_norm_rope_jvp(p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CAJ_OK : cuda_fail(e);
}

caj_status caj_attn_bwd(const void *q, const void *k, const void *v, const void *o,
                        const void *dout, const float *lse, const caj_problem *prob,
                        const caj_mask_desc *mask, void *dq, void *dk, void *dv, float *delta,
                        void *stream) {
  if (!prob || !mask) return CAJ_ERR_INVALID_ARG;
  const void *ins[] = {q, k, v, o, dout, dq, dk, dv};
  for (const void *p : ins)
    if (!p || !aligned16(p)) return CAJ_ERR_INVALID_ARG;
  if (!lse || !delta || !aligned4(lse) || !aligned4(delta)) return CAJ_ERR_INVALID_ARG;
  if (prob->B <= 0 || prob->H <= 0 || prob->N <= 0 || prob->D <= 0) return CAJ_ERR_INVALID_ARG;
  caj::MaskGeom g;
  if (!geom_from_desc(mask, &g) || g.N != prob->N) return CAJ_ERR_INVALID_ARG;
  if (prob->dtype != CAJ_DTYPE_F32 && prob->dtype != CAJ_DTYPE_BF16) return CAJ_ERR_INVALID_ARG;
  if (!(prob->scale >= 0.f) || std::isinf(prob->scale)) return CAJ_ERR_INVALID_ARG;
  if (prob->flags != 0) return CAJ_ERR_INVALID_ARG;
  if (prob->dtype != CAJ_DTYPE_BF16) return CAJ_ERR_UNSUPPORTED;
  if (prob->D != 64 && prob->D != 128) return CAJ_ERR_UNSUPPORTED;
  const int64_t BH = int64_t(prob->B) * prob->H;
  if (BH > 65535 || prob->N > (1 << 20)) return CAJ_ERR_UNSUPPORTED;
  const int32_t ntile = (prob->N + caj::kBlockM - 1) / caj::kBlockM;
  if (ntile > caj::kMaxQTiles) return CAJ_ERR_UNSUPPORTED;
  caj_status st = check_device();
  if (st != CAJ_OK) return st;
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return cuda_fail(cudaErrorNotSupported);
  std::unique_ptr<caj::BwdParams> hp(new caj::BwdParams());
  caj::BwdParams &p = *hp;
  const int N = prob->N, D = prob->D;
  // q, k and dout are also read row by row with 16-byte loads (checked above)
  const bool okm = encode_map(enc, &p.tm_k_s, k, int(BH), N, D, 64) &&
                   encode_map(enc, &p.tm_v_s, v, int(BH), N, D, 64) &&
                   encode_map(enc, &p.tm_v_r, v, int(BH), N, D, 128) &&
                   encode_map(enc, &p.tm_q_s, q, int(BH), N, D, 64) &&
                   encode_map(enc, &p.tm_do_s, dout, int(BH), N, D, 64);
  if (!okm) return cuda_fail(cudaErrorInvalidValue);
  p.q = q; p.k = k; p.o = o; p.dout = dout; p.lse = lse; p.delta = delta; p.dq = dq; p.dk = dk; p.dv = dv;
  p.geom = g;
  p.BH = int32_t(BH);
  p.n_row_tiles = ntile;
  p.scale = prob->scale > 0.f ? prob->scale : 1.0f / std::sqrt(float(D));
  p.timeout_ns = wait_timeout_ns();
  p.fault_mode = g_fault_mode.load();
  // Launch orders: query tiles by decreasing key-tile count, key tiles by
  // decreasing query-tile count (ties: later first).
  std::vector<std::pair<int32_t, int32_t>> cq(ntile), ck(ntile);
  for (int32_t t = 0; t < ntile; ++t) {
    int32_t r[6];
    const int32_t a = t * caj::kBlockM, b = std::min(a + caj::kBlockM, N);
    cq[t] = {caj::qtile_key_tiles(g, a, b, caj::kBlockN, r[0], r[1], r[2], r[3]), t};
    ck[t] = {caj::ktile_query_tiles(g, a, b, caj::kBlockN, r), t};
  }
  auto heavier = [](const auto &x, const auto &y) {
    return x.first != y.first ? x.first > y.first : x.second > y.second;
  };
  std::sort(cq.begin(), cq.end(), heavier);
  std::sort(ck.begin(), ck.end(), heavier);
  for (int32_t i = 0; i < ntile; ++i) {
    p.row_order[i] = uint16_t(cq[i].second);
    p.col_order[i] = uint16_t(ck[i].second);
  }
  cudaError_t e = caj::launch_attn_bwd_sm100(p, D, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CAJ_OK : cuda_fail(e);
}

caj_status caj_signal_barrier(uint32_t *const *pads, int32_t shards, int32_t rank, uint32_t epoch,
                              double timeout_ms, void *stream) {
  if (!pads || shards < 1 || shards > CAJ_MAX_SHARDS || rank < 0 || rank >= shards || epoch == 0)
    return CAJ_ERR_INVALID_ARG;
  caj::SignalParams p{};
  for (int32_t r = 0; r < shards; ++r) {
    if (!pads[r] || !aligned4(pads[r])) return CAJ_ERR_INVALID_ARG;
    p.pads[r] = pads[r];
  }
  caj_status st = check_device();
  if (st != CAJ_OK) return st;
  p.shards = shards;
  p.rank = rank;
  p.epoch = epoch;
  p.timeout_ns = timeout_ms > 0.0 ? uint64_t(timeout_ms * 1e6) : wait_timeout_ns();
  cudaError_t e = caj::launch_signal_barrier(p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CAJ_OK : cuda_fail(e);
}

namespace {
using AddressRangeFn = CUresult (*)(CUdeviceptr *, size_t *, CUdeviceptr);

AddressRangeFn get_address_range() {
  static std::once_flag once;
  static AddressRangeFn fn = nullptr;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(ptr);
  });
  return fn;
}

// Addresses handed out by caj_ipc_open, with the mapped allocation's base and
// how many opens are outstanding (opening a handle that is already mapped in
// this context returns the same mapping, reference-counted by the runtime).
std::mutex g_ipc_mu;
std::map<uintptr_t, std::pair<void *, int>> g_ipc_open;
}  // namespace

caj_status caj_ipc_export(const void *ptr, caj_ipc_handle *out) {
  if (!ptr || !out) return CAJ_ERR_INVALID_ARG;
  AddressRangeFn range = get_address_range();
  if (!range) return cuda_fail(cudaErrorNotSupported);
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return CAJ_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base));
  if (e != cudaSuccess) return cuda_fail(e);
  static_assert(sizeof(h) == sizeof(out->handle), "IPC handle size");
  std::memcpy(out->handle, &h, sizeof(h));
  out->offset = uint64_t(reinterpret_cast<uintptr_t>(ptr) - uintptr_t(base));
  return CAJ_OK;
}

caj_status caj_ipc_open(const caj_ipc_handle *h, void **ptr) {
  if (!h || !ptr) return CAJ_ERR_INVALID_ARG;
  cudaIpcMemHandle_t ch;
  std::memcpy(&ch, h->handle, sizeof(ch));
  void *base = nullptr;
  cudaError_t e = cudaIpcOpenMemHandle(&base, ch, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return cuda_fail(e);
  void *p = static_cast<uint8_t *>(base) + h->offset;
  std::lock_guard<std::mutex> lock(g_ipc_mu);
  auto &entry = g_ipc_open[reinterpret_cast<uintptr_t>(p)];
  entry.first = base;
  entry.second += 1;
  *ptr = p;
  return CAJ_OK;
}

caj_status caj_ipc_close(void *ptr) {
  void *base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_ipc_mu);
    auto it = g_ipc_open.find(reinterpret_cast<uintptr_t>(ptr));
    if (!ptr || it == g_ipc_open.end()) return CAJ_ERR_INVALID_ARG;
    base = it->second.first;
    if (--it->second.second == 0) g_ipc_open.erase(it);
  }
  cudaError_t e = cudaIpcCloseMemHandle(base);
  return e == cudaSuccess ? CAJ_OK : cuda_fail(e);
}

caj_status caj_last_device_status(void *stream) {
  uint32_t code = 0, bcode = 0, scode = 0;
  cudaError_t e = caj::read_and_clear_device_error(static_cast<cudaStream_t>(stream), &code);
  if (e != cudaSuccess) return cuda_fail(e);
  e = caj::read_and_clear_bwd_error(&bcode);
  if (e != cudaSuccess) return cuda_fail(e);
  e = caj::read_and_clear_signal_error(&scode);
  if (e != cudaSuccess) return cuda_fail(e);
  uint32_t pcode = 0;
  e = caj::read_and_clear_proj_error(&pcode);
  if (e != cudaSuccess) return cuda_fail(e);
  if (!code) code = bcode;
  if (!code) code = scode;
  if (!code) code = pcode;
  if (code != 0) {
    g_last_device_code = code;
    return CAJ_ERR_DEVICE_TIMEOUT;
  }
  return CAJ_OK;
}

uint32_t caj_last_device_error_code(void) { return g_last_device_code; }

}  // extern "C"
