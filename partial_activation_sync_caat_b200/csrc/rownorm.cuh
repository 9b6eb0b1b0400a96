// rownorm.cuh - per-rank, per-token RMSNorm of the pre-norm residual stream h.
//
// out[r, t, :] = h[r, t, :] / sqrt(mean_c h[r, t, c]^2 + eps) * gamma, with gamma shared by
// the ranks ("Tensor-Parallelism with Partially Synchronized Activations", §4 Eq. 9: the
// norm follows the partial channel-reduce and the residual add; §4: norm parameters are
// synchronized across ranks).  fp32 math, bf16 round-to-nearest-even stores.
//
// One warp per row; each lane keeps up to NV 16-byte vectors of its row in registers
// (H <= NV * 256), longer rows are read a second time.  128-bit loads and stores, the
// warp's 32 lanes covering 512 contiguous bytes per instruction.  h and out may alias.
#pragma once

#include "ptx.cuh"

namespace caat {

constexpr int K2_THREADS = 256;

template <int NV>
__global__ void __launch_bounds__(K2_THREADS)
    rownorm_kernel(const __nv_bfloat16* h, __nv_bfloat16* out, const __nv_bfloat16* __restrict__ gamma,
                   int64_t rows, int H, float eps) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * K2_THREADS + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * K2_THREADS) >> 5;
  const int nvec = H >> 3;
  const float inv_h = 1.0f / static_cast<float>(H);
  const uint4* g4 = reinterpret_cast<const uint4*>(gamma);

  for (int64_t row = warp_global; row < rows; row += nwarps) {
    const uint4* hp = reinterpret_cast<const uint4*>(h + row * H);
    uint4* op = reinterpret_cast<uint4*>(out + row * H);
    uint4 v[NV];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int idx = lane + 32 * i;
      v[i] = make_uint4(0, 0, 0, 0);
      if (idx < nvec) v[i] = hp[idx];
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = bf16lo(w[e]), b = bf16hi(w[e]);
        ss = fmaf(a, a, ss);
        ss = fmaf(b, b, ss);
      }
    }
    for (int idx = lane + 32 * NV; idx < nvec; idx += 32) {
      const uint4 t = hp[idx];
      const uint32_t w[4] = {t.x, t.y, t.z, t.w};
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

#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int idx = lane + 32 * i;
      if (idx < nvec) {
        const uint4 g = g4[idx];
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          o[e] = pack_bf16x2(bf16lo(w[e]) * rstd * bf16lo(gw[e]), bf16hi(w[e]) * rstd * bf16hi(gw[e]));
        op[idx] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    for (int idx = lane + 32 * NV; idx < nvec; idx += 32) {
      const uint4 t = hp[idx];
      const uint4 g = g4[idx];
      const uint32_t w[4] = {t.x, t.y, t.z, t.w};
      const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        o[e] = pack_bf16x2(bf16lo(w[e]) * rstd * bf16lo(gw[e]), bf16hi(w[e]) * rstd * bf16hi(gw[e]));
      op[idx] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace caat
