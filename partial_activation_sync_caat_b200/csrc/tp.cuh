// tp.cuh - the finishing kernel of the layer split over real devices, one tensor-parallel rank
// per GPU ("Tensor-Parallelism with Partially Synchronized Activations", App. A.2 Eq. 22; §3:
// only the first floor(h p) channels are exchanged; §4 Eq. 9: residual add, then the norm).
//
// The local step (the CTA-pair GEMM kernel in its split-output mode, rowpar_common.cuh) leaves
// this rank's fp32 partial of the shared channels in zs [T, n_s] and the finished private
// channels in h [T, H] (c >= n_s: private_scale * partial + residual, bf16).  The caller sums zs
// over the ranks (its collective).  This kernel then, per token row: h[:, c] = bf16(zs_sum[:, c]
// + R[:, c]) for c < n_s (stored, so that h is the complete pre-norm residual stream), the
// fp32 sum of squares of the whole bf16 row, and out = h / sqrt(sum / H + eps) * gamma.  One
// warp per row, the row in registers (H <= 4096); rows in any order; out may alias h.
#pragma once

#include "ptx.cuh"

namespace caat {

constexpr int KT_FIN_THREADS = 256;

template <int VPL>
__global__ void __launch_bounds__(KT_FIN_THREADS, 2)
    tp_finish_kernel(const float* __restrict__ zs, const __nv_bfloat16* __restrict__ R, __nv_bfloat16* h,
                     __nv_bfloat16* out, const __nv_bfloat16* __restrict__ gamma, int64_t T, int H, int n_s,
                     float eps) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * KT_FIN_THREADS + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * KT_FIN_THREADS) >> 5;
  const int nvec = H >> 3;
  const float inv_h = 1.0f / static_cast<float>(H);
  const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
  for (int64_t t = warp_global; t < T; t += nwarps) {
    uint4* hp = reinterpret_cast<uint4*>(h + t * H);
    const uint4* rp = reinterpret_cast<const uint4*>(R + t * H);
    const float4* zp = reinterpret_cast<const float4*>(zs + t * n_s);
    uint4 x[VPL];
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const int idx = 32 * u + lane;  // channels 8 idx .. 8 idx + 7
      x[u] = make_uint4(0, 0, 0, 0);
      if (idx < nvec) {
        if (8 * idx + 8 <= n_s) {
          // shared: the ranks' summed partial plus this rank's residual, rounded once
          const uint4 r = __ldg(rp + idx);
          const float4 z0 = __ldg(zp + 2 * idx), z1 = __ldg(zp + 2 * idx + 1);
          x[u].x = pack_bf16x2(z0.x + bf16lo(r.x), z0.y + bf16hi(r.x));
          x[u].y = pack_bf16x2(z0.z + bf16lo(r.y), z0.w + bf16hi(r.y));
          x[u].z = pack_bf16x2(z1.x + bf16lo(r.z), z1.y + bf16hi(r.z));
          x[u].w = pack_bf16x2(z1.z + bf16lo(r.w), z1.w + bf16hi(r.w));
          hp[idx] = x[u];
        } else {
          x[u] = hp[idx];  // private channels, finished by the local step
        }
      }
    }
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const uint32_t w[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = bf16lo(w[e]), b = bf16hi(w[e]);
        ss = fmaf(a, a, ss);
        ss = fmaf(b, b, ss);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, off);
    const float rstd = rsqrtf(ss * inv_h + eps);
    uint4* op = reinterpret_cast<uint4*>(out + t * H);
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const int idx = 32 * u + lane;
      if (idx < nvec) {
        const uint4 g = __ldg(g4 + idx);
        const uint32_t w[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
        const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          o[e] = pack_bf16x2(bf16lo_p(w[e]) * rstd * bf16lo(gw[e]), bf16hi_p(w[e]) * rstd * bf16hi(gw[e]));
        op[idx] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

}  // namespace caat
