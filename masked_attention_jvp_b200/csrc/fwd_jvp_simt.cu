// fp32 forward + JVP of block-causal attention on CUDA cores.
//
// The fp32 path exists for fp32 inputs, where the tensor cores' bf16/tf32
// rounding would exceed a 1e-5 relative error. Same mathematics as the
// tensor-core kernel (Causal-rCM appendix B, eq. 42-45): an online softmax in
// fp32 that carries, besides m, l and O, the JVP accumulators
// T = sum_j p~_j (ts_j v_j + tv_j) and r = sum_j p~_j ts_j, rescaled by the same
// factor, then tO = T/l - (r/l) O.
//
// One warp per query row. Keys are visited 32 at a time, one per lane (each lane
// forms its key's score and score tangent as full dot products), then the warp
// applies the chunk to O and T with lane-owned slices of D.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kernels.h"
#include "mask_schedule.h"

namespace caj {
namespace {

constexpr int kWarps = 4;

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32) fwd_jvp_simt_f32_kernel(const __grid_constant__ SimtParams p) {
  constexpr int PER = D / 32;  // elements of D owned by each lane
  __shared__ float4 sq[kWarps][D / 4], stq[kWarps][D / 4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gid = int64_t(blockIdx.x) * kWarps + warp;
  const int32_t N = p.geom.N;
  if (gid >= int64_t(p.BH) * N) return;
  const int32_t bh = int32_t(gid / N), qi = int32_t(gid % N);
  const size_t head = size_t(bh) * N * D;
  const float *Q = static_cast<const float *>(p.q) + head;
  const float *TQ = static_cast<const float *>(p.tq) + head;
  const float *K = static_cast<const float *>(p.k) + head;
  const float *TK = static_cast<const float *>(p.tk) + head;
  const float *V = static_cast<const float *>(p.v) + head;
  const float *TV = static_cast<const float *>(p.tv) + head;

  for (int i = lane; i < D / 4; i += 32) {
    sq[warp][i] = reinterpret_cast<const float4 *>(Q + size_t(qi) * D)[i];
    stq[warp][i] = reinterpret_cast<const float4 *>(TQ + size_t(qi) * D)[i];
  }
  __syncwarp();

  int32_t r[4];
  row_key_ranges(p.geom, qi, r[0], r[1], r[2], r[3]);
  float m_run = -INFINITY, l_run = 0.f, r_run = 0.f;
  float oacc[PER], tacc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) oacc[e] = tacc[e] = 0.f;

  for (int rg = 0; rg < 2; ++rg) {
    const int32_t a = r[2 * rg], b = r[2 * rg + 1];
    for (int32_t base = a; base < b; base += 32) {
      const int32_t j = base + lane;
      const bool valid = j < b;
      float s = -INFINITY, ts = 0.f;
      if (valid) {
        const float4 *kr = reinterpret_cast<const float4 *>(K + size_t(j) * D);
        const float4 *tkr = reinterpret_cast<const float4 *>(TK + size_t(j) * D);
        float d0 = 0.f, d1 = 0.f, d2 = 0.f;
#pragma unroll 4
        for (int i = 0; i < D / 4; ++i) {
          const float4 kv = kr[i], tkv = tkr[i], qv = sq[warp][i], tqv = stq[warp][i];
          d0 = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, d0))));
          d1 = fmaf(tqv.x, kv.x, fmaf(tqv.y, kv.y, fmaf(tqv.z, kv.z, fmaf(tqv.w, kv.w, d1))));
          d2 = fmaf(qv.x, tkv.x, fmaf(qv.y, tkv.y, fmaf(qv.z, tkv.z, fmaf(qv.w, tkv.w, d2))));
        }
        s = d0 * p.scale;
        ts = (d1 + d2) * p.scale;
      }
      const float m_new = fmaxf(m_run, warp_max(s));
      const float alpha = (m_run == -INFINITY) ? 0.f : expf(m_run - m_new);
      const float pj = valid ? expf(s - m_new) : 0.f;
      const float ptj = pj * ts;
      l_run = l_run * alpha + warp_sum(pj);
      r_run = r_run * alpha + warp_sum(ptj);
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        oacc[e] *= alpha;
        tacc[e] *= alpha;
      }
      const int cnt = min(32, b - base);
      for (int kk = 0; kk < cnt; ++kk) {
        const float pk = __shfl_sync(0xffffffffu, pj, kk);
        const float ptk = __shfl_sync(0xffffffffu, ptj, kk);
        const float *vr = V + size_t(base + kk) * D;
        const float *tvr = TV + size_t(base + kk) * D;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
          const float vv = vr[lane + 32 * e];
          oacc[e] = fmaf(pk, vv, oacc[e]);
          tacc[e] = fmaf(ptk, vv, fmaf(pk, tvr[lane + 32 * e], tacc[e]));
        }
      }
      m_run = m_new;
    }
  }

  const float inv_l = 1.f / l_run;
  const float mu = r_run * inv_l;
  const OutRow dst = slice_row(p.out, bh, qi);
  float *O = static_cast<float *>(p.out.o[dst.shard]) + dst.row * D;
  float *TO = static_cast<float *>(p.out.to[dst.shard]) + dst.row * D;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const float ov = oacc[e] * inv_l;
    O[lane + 32 * e] = ov;
    TO[lane + 32 * e] = fmaf(tacc[e], inv_l, -mu * ov);
  }
  if (lane == 0) {
    p.out.lse[dst.shard][dst.stat] = m_run + logf(l_run);
    p.out.tlse[dst.shard][dst.stat] = mu;
  }
}

}  // namespace

cudaError_t launch_fwd_jvp_simt_f32(const SimtParams &p, int D, cudaStream_t stream) {
  const int64_t rows = int64_t(p.BH) * p.geom.N;
  const unsigned grid = unsigned((rows + kWarps - 1) / kWarps);
  if (D == 128) {
    fwd_jvp_simt_f32_kernel<128><<<grid, kWarps * 32, 0, stream>>>(p);
  } else if (D == 64) {
    fwd_jvp_simt_f32_kernel<64><<<grid, kWarps * 32, 0, stream>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace caj
