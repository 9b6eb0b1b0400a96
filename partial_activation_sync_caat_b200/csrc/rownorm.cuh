// rownorm.cuh - per-rank, per-token RMSNorm of the pre-norm residual stream h.
//
// out[r, t, :] = h[r, t, :] / sqrt(mean_c h[r, t, c]^2 + eps) * gamma, with gamma shared by
// the ranks ("Tensor-Parallelism with Partially Synchronized Activations", §4 Eq. 9: the
// norm follows the partial channel-reduce and the residual add; §4: norm parameters are
// synchronized across ranks).  fp32 math, bf16 round-to-nearest-even stores.
//
// HBM-bound: one read of h and one write of out per element.  One warp per row, two passes
// over the row: the first pass streams it (8 independent 128-bit loads per lane in flight)
// and accumulates the sum of squares; the second pass reads it again (an L1/L2 hit: the row
// was just brought in) and writes the scaled values.  Few registers, so many warps per SM keep
// enough bytes in flight to cover HBM latency (32 warps per SM at most 64 registers).  h and out may alias.
#pragma once

#include "ptx.cuh"

namespace caat {

constexpr int K2_THREADS = 256;

// Normalizes the rows (r, t) for every rank r and t in [t0, t0 + tc) of [P, T, H] tensors.
__global__ void __launch_bounds__(K2_THREADS, 4)
    rownorm_kernel(const __nv_bfloat16* h, __nv_bfloat16* out, const __nv_bfloat16* __restrict__ gamma, int P,
                   int64_t T, int64_t t0, int64_t tc, int H, float eps) {
  const int64_t rows = static_cast<int64_t>(P) * tc;
  constexpr int U = 8;  // vectors per lane in flight
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * K2_THREADS + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * K2_THREADS) >> 5;
  const int nvec = H >> 3;
  const float inv_h = 1.0f / static_cast<float>(H);
  const uint4* g4 = reinterpret_cast<const uint4*>(gamma);

  for (int64_t i = warp_global; i < rows; i += nwarps) {
    const int64_t r = i / tc;
    const int64_t row = r * T + t0 + (i - r * tc);
    const uint4* hp = reinterpret_cast<const uint4*>(h + row * H);
    uint4* op = reinterpret_cast<uint4*>(out + row * H);
    float ss = 0.f;
    for (int v0 = 0; v0 < nvec; v0 += 32 * U) {
      uint4 t[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int idx = v0 + 32 * u + lane;
        t[u] = idx < nvec ? hp[idx] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t w[4] = {t[u].x, t[u].y, t[u].z, t[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = bf16lo(w[e]), b = bf16hi(w[e]);
          ss = fmaf(a, a, ss);
          ss = fmaf(b, b, ss);
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, off);
    const float rstd = rsqrtf(ss * inv_h + eps);

    for (int v0 = 0; v0 < nvec; v0 += 32 * U) {
      uint4 t[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int idx = v0 + 32 * u + lane;
        t[u] = idx < nvec ? hp[idx] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int idx = v0 + 32 * u + lane;
        if (idx < nvec) {
          const uint4 g = __ldg(g4 + idx);
          const uint32_t w[4] = {t[u].x, t[u].y, t[u].z, t[u].w};
          const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            o[e] = pack_bf16x2(bf16lo(w[e]) * rstd * bf16lo(gw[e]), bf16hi(w[e]) * rstd * bf16hi(gw[e]));
          op[idx] = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }
  }
}

// Single-pass variant for H <= 256 * VPL: the warp keeps its row in registers (VPL 128-bit
// vectors per lane), so h is read exactly once (no second pass through L1/L2).  All VPL loads
// of a row are issued before the first use.
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
          o[e] = pack_bf16x2(bf16lo(w[e]) * rstd * bf16lo(gw[e]), bf16hi(w[e]) * rstd * bf16hi(gw[e]));
        op[idx] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

}  // namespace caat
