// rownorm.cuh - per-rank, per-token RMSNorm of the pre-norm residual stream h.
//
// out[r, t, :] = h[r, t, :] / sqrt(mean_c h[r, t, c]^2 + eps) * gamma, with gamma shared by
// the ranks ("Tensor-Parallelism with Partially Synchronized Activations", §4 Eq. 9: the
// norm follows the partial channel-reduce and the residual add; §4: norm parameters are
// synchronized across ranks).  fp32 math, bf16 round-to-nearest-even stores.
//
// HBM-bound: one read of h and one write of out per element, the row held in registers between
// the sum of squares and the rescale.  H <= 4096: a warp per row (rownorm_reg_kernel); wider
// rows: a CTA per row (rownorm_block_kernel).  Rows are taken in reverse order (the rows the
// GEMM wrote last may still be in L2).  h and out may alias.
#pragma once

#include "ptx.cuh"

namespace caat {

constexpr int K2_THREADS = 256;

// H <= 256 * VPL: one warp per row, the row kept in registers (VPL 128-bit vectors per lane),
// so h is read exactly once.  All VPL loads of a row are issued before the first use.
template <int VPL>
__global__ void __launch_bounds__(K2_THREADS, 2)
    rownorm_reg_kernel(const __nv_bfloat16* h, __nv_bfloat16* out, const __nv_bfloat16* __restrict__ gamma, int P,
                       int64_t T, int64_t t0, int64_t tc, int H, float eps) {
  const int64_t rows = static_cast<int64_t>(P) * tc;
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * K2_THREADS + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * K2_THREADS) >> 5;
  const int nvec = H >> 3;
  const float inv_h = 1.0f / static_cast<float>(H);
  const uint4* g4 = reinterpret_cast<const uint4*>(gamma);

  // Rows in reverse order: the rows the GEMM wrote last (rank P-1's) may still be in L2.
  for (int64_t i0 = warp_global; i0 < rows; i0 += nwarps) {
    const int64_t i = rows - 1 - i0;
    const int64_t r = i / tc;
    const int64_t row = r * T + t0 + (i - r * tc);
    const uint4* hp = reinterpret_cast<const uint4*>(h + row * H);
    uint4* op = reinterpret_cast<uint4*>(out + row * H);
    uint4 t[VPL];
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const int idx = 32 * u + lane;
      t[u] = idx < nvec ? hp[idx] : make_uint4(0, 0, 0, 0);
    }
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const uint32_t w[4] = {t[u].x, t[u].y, t[u].z, t[u].w};
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
    for (int u = 0; u < VPL; ++u) {
      const int idx = 32 * u + lane;
      if (idx < nvec) {
        const uint4 g = __ldg(g4 + idx);
        const uint32_t w[4] = {t[u].x, t[u].y, t[u].z, t[u].w};
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

// Wide rows (H > 4096): one CTA per (rank, token) row, the row held in registers (VPT 128-bit
// vectors per thread, H <= 8 * THREADS * VPT), sum of squares reduced over the block.  Rows
// are dealt to CTAs in reverse order (as in rownorm_reg_kernel).  h and out may alias.
template <int THREADS, int VPT>
__global__ void __launch_bounds__(THREADS)
    rownorm_block_kernel(const __nv_bfloat16* h, __nv_bfloat16* out, const __nv_bfloat16* __restrict__ gamma, int P,
                         int64_t T, int64_t t0, int64_t tc, int H, float eps) {
  __shared__ float red[THREADS / 32];
  const int64_t rows = static_cast<int64_t>(P) * tc;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nvec = H >> 3;
  const float inv_h = 1.0f / static_cast<float>(H);
  const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
  for (int64_t i0 = blockIdx.x; i0 < rows; i0 += gridDim.x) {
    const int64_t i = rows - 1 - i0;
    const int64_t r = i / tc;
    const int64_t row = r * T + t0 + (i - r * tc);
    const uint4* hp = reinterpret_cast<const uint4*>(h + row * H);
    uint4* op = reinterpret_cast<uint4*>(out + row * H);
    uint4 t[VPT];
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
      const int idx = THREADS * u + threadIdx.x;
      t[u] = idx < nvec ? hp[idx] : make_uint4(0, 0, 0, 0);
    }
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
      const uint32_t w[4] = {t[u].x, t[u].y, t[u].z, t[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = bf16lo(w[e]), b = bf16hi(w[e]);
        ss = fmaf(a, a, ss);
        ss = fmaf(b, b, ss);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, off);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < THREADS / 32; ++w2) tot += red[w2];
    const float rstd = rsqrtf(tot * inv_h + eps);
    __syncthreads();  // red is rewritten for the next row
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
      const int idx = THREADS * u + threadIdx.x;
      if (idx < nvec) {
        const uint4 g = __ldg(g4 + idx);
        const uint32_t w[4] = {t[u].x, t[u].y, t[u].z, t[u].w};
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
