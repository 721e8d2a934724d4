// Layer prologue of the attention block in primal-tangent form.
//
// Causal-rCM implements the JVP layer by layer: every layer takes and returns a
// (primal, tangent) pair (section 3.2.2, "JVP FSDP2"). Before attention, q and k
// are RMS-normalised and rotated by the rotary embedding; v passes through.
// RMSNorm is nonlinear, so its tangent needs the primal:
//   y  = g * x / r,                r = sqrt(mean(x^2) + eps)
//   ty = g * (tx / r - x * mean(x * tx) / r^3)
// and the rotary embedding of interleaved pairs (2i, 2i+1) is linear, so it
// rotates the tangent by the same angle:
//   (a, b) -> (a cos t - b sin t, a sin t + b cos t).
// This kernel reads the six projections in the linear layer's layout
// [B, N, H*D], applies the above to q and k, and writes all six tensors in the
// attention kernel's layout [B, H, N, D] (bf16 in, fp32 arithmetic, bf16 out).
//
// It moves data and does little arithmetic: HBM-bound. One CTA per token, one
// thread per 8 channels (16-byte loads and stores); the mean over the token is
// a block reduction, the mean over a head a shuffle reduction.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace caj {
namespace {

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
}

// Sums of 4 values over `width` consecutive lanes (a power of two <= 32).
__device__ __forceinline__ void lane_group_sum4(float (&v)[4], int width) {
  for (int o = width / 2; o > 0; o >>= 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o, width);
  }
}

// RMSNorm + JVP of 8 channels, then rotation of their 4 pairs.
__device__ __forceinline__ void norm_rope8(float (&x)[8], float (&tx)[8], const float (&g)[8],
                                           float rinv, float mean_xtx, const float (&cs)[4],
                                           const float (&sn)[4]) {
  const float r3 = rinv * rinv * rinv * mean_xtx;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = g[2 * i] * x[2 * i] * rinv, b = g[2 * i + 1] * x[2 * i + 1] * rinv;
    const float ta = g[2 * i] * fmaf(tx[2 * i], rinv, -x[2 * i] * r3);
    const float tb = g[2 * i + 1] * fmaf(tx[2 * i + 1], rinv, -x[2 * i + 1] * r3);
    x[2 * i] = a * cs[i] - b * sn[i];
    x[2 * i + 1] = a * sn[i] + b * cs[i];
    tx[2 * i] = ta * cs[i] - tb * sn[i];
    tx[2 * i + 1] = ta * sn[i] + tb * cs[i];
  }
}

template <int D>
__global__ void __launch_bounds__(1024) qk_norm_rope_jvp_kernel(const PrologueParams p) {
  extern __shared__ float red[];  // [warps][4] partial sums for the whole-token mean
  const int C = p.H * D;
  const int tid = threadIdx.x;          // channels [8 tid, 8 tid + 8)
  const int64_t tok = blockIdx.x;       // b * N + n
  const int n = int(tok % p.N);
  const int64_t b = tok / p.N;
  const int c0 = 8 * tid;
  const int h = c0 / D, d0 = c0 % D;

  const size_t in_off = size_t(tok) * C + c0;
  const uint4 *in[6] = {static_cast<const uint4 *>(p.xq), static_cast<const uint4 *>(p.xk),
                        static_cast<const uint4 *>(p.xv), static_cast<const uint4 *>(p.txq),
                        static_cast<const uint4 *>(p.txk), static_cast<const uint4 *>(p.txv)};
  uint4 raw[6];
#pragma unroll
  for (int i = 0; i < 6; ++i) raw[i] = __ldcs(in[i] + in_off / 8);

  float xq[8], xk[8], txq[8], txk[8];
  unpack8(raw[0], xq);
  unpack8(raw[1], xk);
  unpack8(raw[3], txq);
  unpack8(raw[4], txk);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};  // sum xq^2, sum xq*txq, sum xk^2, sum xk*txk
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    acc[0] = fmaf(xq[i], xq[i], acc[0]);
    acc[1] = fmaf(xq[i], txq[i], acc[1]);
    acc[2] = fmaf(xk[i], xk[i], acc[2]);
    acc[3] = fmaf(xk[i], txk[i], acc[3]);
  }
  float len;
  if (p.per_head) {
    lane_group_sum4(acc, D / 8);
    len = float(D);
  } else {
    lane_group_sum4(acc, 32);
    const int warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
    if (lane == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) red[warp * 4 + i] = acc[i];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float s = 0.f;
      for (int w = 0; w < nw; ++w) s += red[w * 4 + i];
      acc[i] = s;
    }
    len = float(C);
  }
  const float inv_len = 1.f / len;
  const float rq = rsqrtf(fmaf(acc[0], inv_len, p.eps));
  const float rk = rsqrtf(fmaf(acc[2], inv_len, p.eps));

  float gq[8], gk[8], cs[4], sn[4];
  {
    const float4 *g4q = reinterpret_cast<const float4 *>(p.gq + c0);
    const float4 *g4k = reinterpret_cast<const float4 *>(p.gk + c0);
    const float4 a = __ldg(g4q), bq = __ldg(g4q + 1), c = __ldg(g4k), dk = __ldg(g4k + 1);
    gq[0] = a.x; gq[1] = a.y; gq[2] = a.z; gq[3] = a.w;
    gq[4] = bq.x; gq[5] = bq.y; gq[6] = bq.z; gq[7] = bq.w;
    gk[0] = c.x; gk[1] = c.y; gk[2] = c.z; gk[3] = c.w;
    gk[4] = dk.x; gk[5] = dk.y; gk[6] = dk.z; gk[7] = dk.w;
    const float4 cc = __ldg(reinterpret_cast<const float4 *>(p.rope_cos + size_t(n) * (D / 2) + d0 / 2));
    const float4 ss = __ldg(reinterpret_cast<const float4 *>(p.rope_sin + size_t(n) * (D / 2) + d0 / 2));
    cs[0] = cc.x; cs[1] = cc.y; cs[2] = cc.z; cs[3] = cc.w;
    sn[0] = ss.x; sn[1] = ss.y; sn[2] = ss.z; sn[3] = ss.w;
  }
  norm_rope8(xq, txq, gq, rq, acc[1] * inv_len, cs, sn);
  norm_rope8(xk, txk, gk, rk, acc[3] * inv_len, cs, sn);

  const size_t out_off = ((size_t(b) * p.H + h) * p.N + n) * D + d0;
  uint4 *out[6] = {static_cast<uint4 *>(p.q), static_cast<uint4 *>(p.k), static_cast<uint4 *>(p.v),
                   static_cast<uint4 *>(p.tq), static_cast<uint4 *>(p.tk), static_cast<uint4 *>(p.tv)};
  __stcs(out[0] + out_off / 8, pack8(xq));
  __stcs(out[1] + out_off / 8, pack8(xk));
  __stcs(out[2] + out_off / 8, raw[2]);
  __stcs(out[3] + out_off / 8, pack8(txq));
  __stcs(out[4] + out_off / 8, pack8(txk));
  __stcs(out[5] + out_off / 8, raw[5]);
}

}  // namespace

cudaError_t launch_qk_norm_rope_jvp(const PrologueParams &p, cudaStream_t stream) {
  const int threads = p.H * p.D / 8;
  const unsigned grid = unsigned(int64_t(p.B) * p.N);
  const size_t smem = size_t((threads + 31) / 32) * 4 * sizeof(float);
  if (p.D == 128) {
    qk_norm_rope_jvp_kernel<128><<<grid, threads, smem, stream>>>(p);
  } else if (p.D == 64) {
    qk_norm_rope_jvp_kernel<64><<<grid, threads, smem, stream>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace caj
