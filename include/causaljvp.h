/*
 * libcausaljvp -- fused forward + forward-mode JVP of block-causal softmax
 * attention on NVIDIA B200 (sm_100a).
 *
 * The operation is the masked FlashAttention JVP of the Causal-rCM paper
 * (arXiv 2606.25473), appendix B "FlashAttention-2 JVP kernel with custom
 * mask", eq. 42-45 and Algorithm 1. Per (batch, head), with S = scale*Q K^T + M,
 * P = softmax(S), O = P V:
 *   tS   = scale * (tQ K^T + Q tK^T)                          (eq. 43)
 *   tO   = (P o (tS - rowsum(P o tS))) V + P tV               (eq. 44)
 *   LSE  = log sum_j exp(S_ij)         (natural log)
 *   tLSE = rowsum(P o tS)
 * M is 0 where a query may attend to a key and -inf elsewhere; it carries no
 * tangent (appendix B, text after eq. 43). The mask family is the block-causal
 * one of section 3.1.1 (teacher forcing, eq. 8) and section 4 (frame-wise c1-1
 * and chunk-wise c3-3 chunking), described by caj_mask_desc below.
 *
 * Conventions for every entry point:
 *  - Pointers named q, k, v, tq, tk, tv, o, to, lse, tlse are DEVICE pointers on
 *    the current CUDA device. The caller owns and allocates every buffer; the
 *    library allocates no device memory per call.
 *  - Tensors q..tv, o, to are [B, H, N, D] contiguous (D fastest), 16-byte
 *    aligned. lse and tlse are [B, H, N] fp32, 4-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls are asynchronous on that stream; nothing synchronises implicitly.
 *  - Argument errors are detected on the host, before anything is launched, and
 *    leave the outputs untouched.
 */
#ifndef CAUSALJVP_H
#define CAUSALJVP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CAJ_OK = 0,
  CAJ_ERR_INVALID_ARG = 1,    /* null/misaligned pointer, bad shape or mask descriptor */
  CAJ_ERR_UNSUPPORTED = 2,    /* valid request this build does not implement (e.g. D=96) */
  CAJ_ERR_CUDA = 3,           /* a CUDA runtime/driver call failed; see caj_last_cuda_error */
  CAJ_ERR_DEVICE_TIMEOUT = 4  /* a kernel gave up on a bounded wait (reported asynchronously) */
} caj_status;

typedef enum { CAJ_DTYPE_F32 = 0, CAJ_DTYPE_BF16 = 1 } caj_dtype;

/*
 * Block-causal mask (Causal-rCM section 3.1.1 and section 4). Tokens come in
 * frames of `tokens_per_frame` (T) tokens and frames in chunks of
 * `frames_per_chunk` (c) frames; G = c*T tokens per chunk, L = n_frames*T.
 *   tf_layout = 0: N = L. Query i sees every key of its own chunk and of all
 *                  earlier chunks (diffusion-forcing / inference layout).
 *   tf_layout = 1: N = 2L, packed [clean | noisy] (teacher forcing, eq. 8).
 *                  A clean query of chunk j sees clean chunks <= j. A noisy
 *                  query of chunk j sees clean chunks < j and its own noisy
 *                  chunk j. Clean queries see no noisy key.
 * Requirements: all fields > 0 (tf_layout in {0,1}), n_frames % frames_per_chunk == 0.
 */
typedef struct {
  int32_t tokens_per_frame;
  int32_t frames_per_chunk;
  int32_t n_frames;
  int32_t tf_layout;
} caj_mask_desc;

/* Problem shape. dtype is a caj_dtype and applies to q..tv, o and to.
 * scale <= 0 selects 1/sqrt(D). flags is a bitwise OR of caj_flags. */
typedef struct {
  int32_t B, H, N, D;
  int32_t dtype;
  float scale;
  int32_t flags;
} caj_problem;

/*
 * CAJ_FLAG_CLEAN_TANGENT_ZERO (teacher-forcing layout only): the caller
 * guarantees that tq, tk and tv are exactly zero on the clean half (token
 * rows < L). In TF-sCM the clean context has zero tangent and only the noisy
 * branch follows the teacher velocity (Causal-rCM section 3.1.2, the paragraph
 * after eq. 17). The call then skips every product that vanishes: query tiles
 * of clean rows compute only the primal (tO = 0, tLSE = 0), and key tiles of
 * clean tokens skip Q tK^T and P tV. It runs as two kernel launches on
 * `stream`, one per kind of query tile (tiles with a noisy row, then tiles of
 * clean rows). With the guarantee the results equal the dense definition;
 * without it they do not.
 */
/*
 * CAJ_FLAG_TOKEN_MAJOR_OUT: o and to are written token-major, [B, N, H, D]
 * (= [B, N, H*D], the input layout of the output projection,
 * caj_out_proj_jvp) instead of [B, H, N, D]. lse and tlse keep [B, H, N].
 * Not accepted by caj_attn_fwd_jvp_host.
 */
typedef enum { CAJ_FLAG_CLEAN_TANGENT_ZERO = 1, CAJ_FLAG_TOKEN_MAJOR_OUT = 2 } caj_flags;

/*
 * Forward + JVP of block-causal attention (appendix B eq. 42-45, Algorithm 1).
 *   in : q, k, v, tq, tk, tv   [B,H,N,D] of prob->dtype, read only
 *   out: o, to                 [B,H,N,D] of prob->dtype, fully overwritten
 *                              ([B,N,H,D] with CAJ_FLAG_TOKEN_MAJOR_OUT)
 *        lse, tlse             [B,H,N] fp32, fully overwritten
 * Supported: D in {64, 128}; dtype BF16 (tensor-core path, fp32 accumulation)
 * or F32 (CUDA-core fp32 path); N == n_frames*tokens_per_frame*(tf_layout?2:1);
 * B*H <= 65535; N <= 1048576.
 * Returns CAJ_OK once the kernel(s) are enqueued on `stream` (asynchronous),
 * CAJ_ERR_INVALID_ARG / CAJ_ERR_UNSUPPORTED without launching, or
 * CAJ_ERR_CUDA if a launch failed. Device-side bounded-wait failures are
 * reported by caj_last_device_status.
 */
caj_status caj_attn_fwd_jvp(const void *q, const void *k, const void *v,
                            const void *tq, const void *tk, const void *tv,
                            const caj_problem *prob, const caj_mask_desc *mask,
                            void *o, void *to, float *lse, float *tlse,
                            void *stream);

/*
 * One part of caj_attn_fwd_jvp, for splitting one call over `nparts` GPUs with
 * no collective: every (batch, head) and every query row is an independent
 * problem (appendix B: each query block runs on its own over the key ranges its
 * mask allows), so rank r may compute any subset of the query tiles (128 rows)
 * while holding all of q..tv. The tiles are dealt out by cost, heaviest first,
 * each to the part with the least work so far, so parts differ by at most one
 * tile's work; a part runs its tiles for every head.
 *   in / out     as caj_attn_fwd_jvp (full-size buffers); only the rows of this
 *                part's query tiles are written, the others are left as they are
 *   part, nparts 0 <= part < nparts; nparts = 1 is caj_attn_fwd_jvp
 * The union over parts 0..nparts-1 equals caj_attn_fwd_jvp bit for bit.
 * bf16 only when nparts > 1 (CAJ_ERR_UNSUPPORTED for fp32). Returns as
 * caj_attn_fwd_jvp; a part without tiles launches nothing and returns CAJ_OK.
 */
caj_status caj_attn_fwd_jvp_part(const void *q, const void *k, const void *v,
                                 const void *tq, const void *tk, const void *tv,
                                 const caj_problem *prob, const caj_mask_desc *mask,
                                 int32_t part, int32_t nparts, void *o, void *to, float *lse,
                                 float *tlse, void *stream);

/*
 * Context-parallel form of caj_attn_fwd_jvp, with the output all-to-all done by
 * the kernel's epilogue. Causal-rCM trains with flattened Ulysses context
 * parallelism (section 3.2.1, "Parallelism"; section 3.2.2, "JVP Ulysses CP").
 * Each of P ranks holds N/P tokens of every head. An all-to-all gives each rank
 * H/P heads over the whole sequence. Local attention runs, and the outputs and
 * their tangents return through a second all-to-all. The tangents follow the
 * same route as their primals.
 * Here the second all-to-all is not a separate collective: each output row is
 * written directly into the buffers of the rank that owns its sequence slice.
 *   in : q, k, v, tq, tk, tv   this rank's heads over the whole sequence,
 *                              [B,H,N,D] of prob->dtype (H = heads of this rank)
 *   dst->shards                P, 1..CAJ_MAX_SHARDS; N must be a multiple of P
 *   dst->head_base             global index of this call's head 0
 *   dst->heads_total           heads of each slice buffer, at least
 *                              head_base + H
 *   dst->o[r], dst->to[r]      slice r (token rows [r N/P, (r+1) N/P)):
 *                              [B, heads_total, N/P, D] of prob->dtype, or
 *                              [B, N/P, heads_total, D] with
 *                              CAJ_FLAG_TOKEN_MAJOR_OUT; 16-byte aligned
 *   dst->lse[r], dst->tlse[r]  slice r: [B, heads_total, N/P] fp32
 * Only the rows of this call's heads are written. The other heads' rows in
 * the slice buffers are left as they are. Values and rounding equal those of
 * caj_attn_fwd_jvp on the same inputs.
 * On a multi-GPU run the slice buffers of the other ranks are their device
 * memory mapped into this process: CUDA IPC or symmetric memory, with peer
 * access enabled. The kernel writes them with plain stores over NVLink.
 * The library does not synchronise with the peers. Before the call the caller
 * makes sure that no rank still reads the slice buffers. After it, the caller
 * orders every rank's reads after all P calls, e.g. with a barrier on the
 * stream. The buffers are owned by the caller.
 * Returns as caj_attn_fwd_jvp. CAJ_ERR_INVALID_ARG is also returned for a null
 * dst, a shard count or head range out of bounds, a null or misaligned slice
 * pointer, or a slice pointer that is not device memory (host memory, pinned
 * or not, by cudaPointerGetAttributes): the kernel writes the slices with
 * device stores.
 */
#define CAJ_MAX_SHARDS 8
typedef struct {
  int32_t shards;
  int32_t head_base;
  int32_t heads_total;
  void *o[CAJ_MAX_SHARDS];
  void *to[CAJ_MAX_SHARDS];
  float *lse[CAJ_MAX_SHARDS];
  float *tlse[CAJ_MAX_SHARDS];
} caj_seq_scatter;
caj_status caj_attn_fwd_jvp_scatter(const void *q, const void *k, const void *v,
                                    const void *tq, const void *tk, const void *tv,
                                    const caj_problem *prob, const caj_mask_desc *mask,
                                    const caj_seq_scatter *dst, void *stream);

/*
 * Stream-ordered barrier of the P ranks of a context-parallel group, the fence
 * around caj_attn_fwd_jvp_scatter (section 3.2.2, "JVP Ulysses CP": the output
 * all-to-all; here every rank writes rows into its peers' memory, so each rank
 * must know when its peers have finished reading, and later writing, its slice).
 *   pads[r]     device pointer, as mapped in this process, to rank r's pad of
 *               CAJ_MAX_SHARDS uint32 words (symmetric memory or CUDA IPC with
 *               peer access; pads[rank] is this rank's own). Every pad starts
 *               zeroed before any rank's first call.
 *   shards      P, 1..CAJ_MAX_SHARDS;  rank: this rank, 0..P-1
 *   epoch       nonzero, larger than on any earlier call over these pads
 *               (wrapping compare: a counter from 1 serves for 2^31 calls);
 *               every rank passes the same value to the same barrier
 *   timeout_ms  limit on the wait; <= 0 takes the library's wait limit
 *               (caj_set_wait_timeout_ms)
 * One small kernel on `stream`: rank r stores `epoch` into word r of every
 * rank's pad (system-scope release, after a system fence that orders this
 * rank's earlier work on the stream before it), then waits until every word of
 * its own pad has reached `epoch` (system-scope acquire). Work enqueued on
 * `stream` after the call starts once every rank has arrived. The wait is
 * bounded: if a peer does not arrive in time the kernel records
 * CAJ_ERR_DEVICE_TIMEOUT (caj_last_device_error_code 0x1F0), read by
 * caj_last_device_status, and returns; it never traps.
 * Returns CAJ_OK once enqueued, CAJ_ERR_INVALID_ARG (null or misaligned pad,
 * rank or shard count out of range, epoch 0) without launching, or CAJ_ERR_CUDA.
 */
caj_status caj_signal_barrier(uint32_t *const *pads, int32_t shards, int32_t rank, uint32_t epoch,
                              double timeout_ms, void *stream);

/*
 * Peer mappings for the slice buffers of caj_attn_fwd_jvp_scatter (section
 * 3.2.1 "Parallelism": each rank's output slice must be writable by every
 * rank). Plain CUDA IPC: a rank exports a handle for device memory it owns,
 * the other ranks open it as a peer mapping over NVLink. No multicast object
 * is created or bound.
 *   caj_ipc_export  ptr: device memory from cudaMalloc on the current device
 *                   (e.g. PyTorch's default allocator; not memory from
 *                   cudaMallocAsync or cuMemCreate). Writes an opaque handle
 *                   (the allocation's IPC handle and ptr's offset inside it).
 *   caj_ipc_open    maps a handle exported by ANOTHER process (same node) and
 *                   returns the address of the exported ptr in this process;
 *                   peer access is enabled on first touch.
 *   caj_ipc_close   unmaps an address returned by caj_ipc_open. An address
 *                   opened n times needs n closes. The exporter keeps its
 *                   memory until every opener has closed it.
 * Return CAJ_OK, CAJ_ERR_INVALID_ARG (null argument; an address not opened
 * here) or CAJ_ERR_CUDA (caj_last_cuda_error names the CUDA error).
 */
typedef struct {
  unsigned char handle[64];
  uint64_t offset;
} caj_ipc_handle;
caj_status caj_ipc_export(const void *ptr, caj_ipc_handle *out);
caj_status caj_ipc_open(const caj_ipc_handle *h, void **ptr);
caj_status caj_ipc_close(void *ptr);

/*
 * Host-buffer form of caj_attn_fwd_jvp: the same operation, with the inputs
 * and outputs in host memory. The heads are split into at most 16 chunks.
 * Three things run at once on three streams: the copy of chunk c's six inputs
 * to the device, the kernel on chunk c-1, and the copy of an earlier chunk's
 * outputs back to the host. (bf16: the first and the last chunk go in two
 * pieces by query rows, the first piece copying only the key rows its query
 * tiles read, so the pipeline fills and drains in half the time.) Pinned host memory lets the copies overlap;
 * pageable memory gives the same results, but its copies do not overlap.
 *   in : q, k, v, tq, tk, tv   host, [B,H,N,D] of prob->dtype, read only
 *   out: o, to                 host, [B,H,N,D] of prob->dtype
 *        lse, tlse             host, [B,H,N] fp32
 *   workspace                  device memory, 256-byte aligned, of at least
 *                              caj_attn_fwd_jvp_host_workspace() bytes. It is
 *                              owned by the caller and not freed here. No other
 *                              work may use it until the call has completed.
 *   stream                     the call runs after the work already on
 *                              `stream`. The outputs are complete in host
 *                              memory once `stream` has passed the call, e.g.
 *                              after cudaStreamSynchronize(stream).
 * The library keeps two copy streams and a set of events per device, created
 * on first use. Returns as caj_attn_fwd_jvp, and CAJ_ERR_INVALID_ARG also
 * for a null, misaligned or too small workspace. After a failure, `stream`
 * still waits for every copy the call enqueued.
 */
caj_status caj_attn_fwd_jvp_host_workspace(const caj_problem *prob, size_t *bytes);
caj_status caj_attn_fwd_jvp_host(const void *q, const void *k, const void *v,
                                 const void *tq, const void *tk, const void *tv,
                                 const caj_problem *prob, const caj_mask_desc *mask,
                                 void *o, void *to, float *lse, float *tlse,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * caj_attn_fwd_jvp_host with no device memory from the caller. The paper has
 * no counterpart to this call; it exists for callers that cannot allocate
 * device memory: a plain C program or plugin that keeps its tensors in host
 * memory and links no device allocator, or a host runtime whose memory manager
 * owns every device allocation and forbids cudaMalloc from its extensions.
 * The device staging area is a fixed array of CAJ_HOST_STATIC_MAX_BYTES inside
 * the library (a file-scope __device__ array). Every device that loads the
 * library holds it until the process exits. Nothing is allocated or freed by
 * the call: no cudaMalloc, no cudaFree, no allocating library routine.
 *   in / out       as caj_attn_fwd_jvp_host (host buffers; pinned memory lets
 *                  the copies overlap the kernels)
 *   size limit     the problem's caj_attn_fwd_jvp_host_workspace() size must
 *                  not exceed CAJ_HOST_STATIC_MAX_BYTES (for bf16, D = 128:
 *                  B*H*N up to about 32 000 rows). A larger problem returns
 *                  CAJ_ERR_UNSUPPORTED and touches nothing.
 *   first call     the first call on each device looks up the array's device
 *                  address (cudaGetSymbolAddress, with that device current).
 *                  Make that first call before any stream capture.
 *   sharing        every call on a device uses the same array, which keeps the
 *                  last call's contents. Each call overwrites every byte it
 *                  reads back, so nothing needs clearing. Calls whose work
 *                  overlaps on the GPU (other streams, other host threads)
 *                  race on the array: order them, e.g. on one stream.
 * Returns as caj_attn_fwd_jvp_host, CAJ_ERR_UNSUPPORTED for a problem beyond
 * the limit, or CAJ_ERR_CUDA if the array's address cannot be looked up.
 */
#define CAJ_HOST_STATIC_MAX_BYTES (64u << 20)
caj_status caj_attn_fwd_jvp_host_static(const void *q, const void *k, const void *v,
                                        const void *tq, const void *tk, const void *tv,
                                        const caj_problem *prob, const caj_mask_desc *mask,
                                        void *o, void *to, float *lse, float *tlse, void *stream);

/*
 * Output projection of the attention block in primal-tangent form. Causal-rCM
 * runs the JVP layer by layer, each layer mapping a (primal, tangent) pair to a
 * pair (section 3.2.2, "JVP FSDP2"); the projection after attention is
 * linear, so its tangent is the same map without the bias:
 *   y = x W^T + b,   ty = tx W^T
 *   in : x, tx   [M, K] bf16 row-major: M = B*N tokens, K = H*D (the attention
 *                output written with CAJ_FLAG_TOKEN_MAJOR_OUT)
 *        w       [C, K] bf16 row-major (the layer's weight)
 *        bias    [C] bf16, or null for none
 *   out: y, ty   [M, C] bf16, fully overwritten
 * One launch of a tcgen05 kernel computes both products (the rows of x and tx
 * form one operand, so each weight tile serves both), bf16 in, fp32
 * accumulation, the bias added in fp32 to primal rows before the rounding to
 * bf16. Nothing is allocated per call. Pointers 16-byte aligned; K and C
 * multiples of 8 and M < 2^31 (CAJ_ERR_UNSUPPORTED otherwise). Returns CAJ_OK
 * once enqueued on `stream`, CAJ_ERR_INVALID_ARG without launching, or
 * CAJ_ERR_CUDA. Bounded-wait failures are reported by caj_last_device_status.
 */
typedef struct {
  int64_t M;
  int32_t K, C;
} caj_linear_shape;

caj_status caj_out_proj_jvp(const void *x, const void *tx, const void *w, const void *bias,
                            const caj_linear_shape *shape, void *y, void *ty, void *stream);

/*
 * Attention-block prologue in primal-tangent form. Causal-rCM implements the
 * JVP layer by layer, each layer taking and returning a (primal, tangent) pair
 * (section 3.2.2, "JVP FSDP2"). For q and k:
 *   y  = g * x / r, r = sqrt(mean(x^2) + eps)                    (RMSNorm)
 *   ty = g * (tx / r - x * mean(x * tx) / r^3)                    (its JVP)
 * then the rotary embedding of interleaved pairs (2i, 2i+1) of each head by the
 * angle whose cosine/sine are rope_cos/rope_sin[n][i] (linear: the tangent is
 * rotated the same way). v and tv are copied. The mean runs over the whole
 * token (norm_per_head = 0, width H*D) or over each head (1, width D).
 *   in : xq, xk, xv, txq, txk, txv   [B, N, H*D] bf16 (the projections' layout)
 *        gq, gk                      [H*D] fp32 RMSNorm gains, 16-byte aligned
 *        rope_cos, rope_sin          [N, D/2] fp32, 16-byte aligned
 *   out: q, k, v, tq, tk, tv         [B, H, N, D] bf16 (caj_attn_fwd_jvp's layout)
 * Supported: D in {64, 128}; H*D a multiple of 256 and at most 8192; eps >= 0.
 * Returns CAJ_OK once enqueued, CAJ_ERR_INVALID_ARG / CAJ_ERR_UNSUPPORTED
 * without launching, or CAJ_ERR_CUDA.
 */
typedef struct {
  int32_t B, N, H, D;
  float eps;
  int32_t norm_per_head;
} caj_prologue_shape;

caj_status caj_qk_norm_rope_jvp(const void *xq, const void *xk, const void *xv,
                                const void *txq, const void *txk, const void *txv,
                                const float *gq, const float *gk,
                                const float *rope_cos, const float *rope_sin,
                                const caj_prologue_shape *shape,
                                void *q, void *k, void *v, void *tq, void *tk, void *tv,
                                void *stream);

/*
 * Backward of the primal block-causal attention: the student's gradient step in
 * TF-sCM (the JVP branch is stop-gradient and needs none). With
 * P_ij = exp(scale <q_i, k_j> - LSE_i) on visible pairs and dO the gradient of O:
 *   dV = P^T dO,  dP = dO V^T,  Delta_i = <dO_i, O_i>,  dS = P o (dP - Delta),
 *   dQ = scale dS K,  dK = scale dS^T Q.
 *   in : q, k, v, o, dout      [B,H,N,D] bf16 (o from caj_attn_fwd_jvp)
 *        lse                   [B,H,N] fp32, natural log (from caj_attn_fwd_jvp)
 *   out: dq, dk, dv            [B,H,N,D] bf16, fully overwritten
 *        delta                 [B,H,N] fp32, Delta_i = <dO_i, O_i>
 * prob->dtype must be CAJ_DTYPE_BF16 and D in {64, 128}; prob->flags must be 0.
 * Deterministic (no atomics). Returns like caj_attn_fwd_jvp.
 */
caj_status caj_attn_bwd(const void *q, const void *k, const void *v, const void *o,
                        const void *dout, const float *lse, const caj_problem *prob,
                        const caj_mask_desc *mask, void *dq, void *dk, void *dv, float *delta,
                        void *stream);

/* Synchronises `stream`, then reads and clears the library's device error word.
 * Returns CAJ_OK, CAJ_ERR_DEVICE_TIMEOUT (a kernel gave up: it abandoned a wait
 * or refused to run; its outputs are undefined) or CAJ_ERR_CUDA. */
caj_status caj_last_device_status(void *stream);

/* Detail of the last device error (0 if none). Valid after
 * caj_last_device_status returned CAJ_ERR_DEVICE_TIMEOUT:
 *   0x100 | site   a bounded wait expired at the numbered wait site (site 0xF0:
 *                  the signal barrier, caj_signal_barrier);
 *   0x200          the dynamic shared memory was not 1 KiB aligned;
 *   0x300          a forward launch met a query tile of the other kind than it
 *                  was built for (an internal partitioning error). */
uint32_t caj_last_device_error_code(void);

/* Sets the limit, in milliseconds, on every bounded wait inside the kernels of
 * later calls on this process (default 2000, or the CAJ_WAIT_TIMEOUT_MS
 * environment variable). ms <= 0 restores the default. Returns CAJ_OK. */
caj_status caj_set_wait_timeout_ms(double ms);

/* Test hook for the bounded-wait path: mode 1 makes later tensor-core launches
 * skip their copies (the forward kernels: the query-tile copies; the backward's
 * dQ and dK/dV kernels: every copy), so the MMA warp's first wait runs out, the
 * kernel records CAJ_ERR_DEVICE_TIMEOUT with the site of that wait and every
 * role exits cleanly. Nothing is in flight when the roles exit, and nothing
 * faults or hangs; outputs of such a call are undefined. mode 0 (default)
 * restores normal operation. Returns CAJ_OK, or CAJ_ERR_INVALID_ARG. */
caj_status caj_debug_set_fault(int32_t mode);

/* Human-readable name of a status. Never NULL. */
const char *caj_status_string(caj_status s);

/* Text of the last CUDA error seen by this library on this thread ("" if none). */
const char *caj_last_cuda_error(void);

/* ---- host-side mask and schedule queries (no GPU needed) ---- */

/* Checks a mask descriptor against N. Returns CAJ_OK or CAJ_ERR_INVALID_ARG. */
caj_status caj_validate_mask(const caj_mask_desc *mask, int32_t N);

/* Visible (query, key) pairs of one head, in closed form; -1 on a bad mask.
 * Work of one call is 12 * D * visible_pairs * B * H floating-point operations. */
int64_t caj_visible_pairs(const caj_mask_desc *mask);

/* Keys that query row `row` may attend to, as up to two half-open intervals
 * [r[0], r[1]) and [r[2], r[3]) (an empty interval has r[2] == r[3]).
 * Returns CAJ_OK or CAJ_ERR_INVALID_ARG. */
caj_status caj_row_key_ranges(const caj_mask_desc *mask, int32_t row, int32_t r[4]);

/* The key tiles of width `block_n` the kernel visits for the query tile
 * [q0, q1): up to two half-open tile-index ranges [t[0], t[1]) and [t[2], t[3]),
 * ascending and disjoint. Returns the number of tiles, or -1 on a bad argument. */
int32_t caj_qtile_key_tiles(const caj_mask_desc *mask, int32_t q0, int32_t q1,
                            int32_t block_n, int32_t t[4]);

/* Queries that may attend to key `key` (the transposed mask), as up to two
 * half-open intervals [r[0], r[1]) and [r[2], r[3]). CAJ_OK or CAJ_ERR_INVALID_ARG. */
caj_status caj_key_query_ranges(const caj_mask_desc *mask, int32_t key, int32_t r[4]);

/* The query tiles of height `block_q` the backward's key-major kernel visits for
 * the key tile [k0, k1): up to three ascending disjoint half-open tile ranges
 * t[0..5]. Returns the number of tiles, or -1 on a bad argument. */
int32_t caj_ktile_query_tiles(const caj_mask_desc *mask, int32_t k0, int32_t k1,
                              int32_t block_q, int32_t t[6]);

/* The query tiles (of 128 rows) that part `part` of `nparts` runs in
 * caj_attn_fwd_jvp_part, in launch order (heaviest first): writes up to
 * `capacity` tile indices to `tiles` (may be NULL) and returns how many the
 * part has, or -1 on a bad argument. */
int32_t caj_part_query_tiles(const caj_mask_desc *mask, int32_t part, int32_t nparts, int32_t *tiles,
                             int32_t capacity);

/* Library version, major*10000 + minor*100 + patch. */
int32_t caj_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CAUSALJVP_H */
