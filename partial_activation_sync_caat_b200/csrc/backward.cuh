// backward.cuh - the backward of the partially synchronized row-parallel layer.
//
// "Tensor-Parallelism with Partially Synchronized Activations", §4 Eq. 10-13 and Fig. 2b:
// with partial synchronization the reduction over the ranks in the backward pass must come
// AFTER the derivative of the normalization (the 'h' operation), and the shared norm
// weight's gradient is reduced over the ranks; reduced gradients are accumulated in fp32
// (§4, "Numerical stability via 32 bit gradient accumulation").  Given dout = dL/d(out) and
// the pre-norm stream h saved by the forward:
//
//   r = 1/sqrt(mean_c h^2 + eps), g = dout * gamma
//   dh = r g - h r^3 (sum_c g h) / H              (RMSNorm backward, per rank and token)
//   dR = dh                                        (residual add)
//   dZt_m[:, c] = sum_q dh_q[:, c]  for c in S     (reduction over ranks, fp32)
//              = s * dh_m[:, c]    otherwise      (private scale s)
//   dgamma = sum over ranks and tokens of dout * h * r
//   dX_m = dZt_m W_m,  dW_m = dZt_m^T X_m          (two batched tcgen05 GEMMs on the CTA-pair
//                                                   kernel reading W, dZt and X MN-major; the
//                                                   transposes below serve calls of <= 128
//                                                   tokens or channels)
#pragma once

#include "ptx.cuh"
#include "rowpar_common.cuh"

namespace caat {

constexpr int KB_THREADS = 512;
constexpr int KB_VEC = 2;      // 8-channel vectors per thread: H <= 8 * 512 * 2 = 8192
constexpr int KB_MAXP = 16;
constexpr size_t KB_SMEM_MAX = 200 * 1024;  // staging of the shared-memory norm backward

struct BwdParams {
  const __nv_bfloat16* h;      // [P, T, H]
  const __nv_bfloat16* dout;   // [P, T, H]
  const __nv_bfloat16* gamma;  // [H]
  __nv_bfloat16* dR;           // [P, T, H] or null
  __nv_bfloat16* dZt;          // [P, T, H]
  float* dg_part;              // [gridDim.x][H] per-CTA partial dgamma
  int P, H;
  int64_t T;
  float eps, private_scale;
  int zk_regs;                 // 1 (P <= 8): bf16(s dh) kept in registers between passes 2 and 3
  uint32_t mask_bits[K1_MASK_WORDS];
};

__device__ __forceinline__ void unpack8(uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = bf16lo(w[e]);
    f[2 * e + 1] = bf16hi(w[e]);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

// KB1: RMSNorm backward + the reduction over ranks.  Persistent CTAs walk the tokens; a CTA
// handles every rank of its token so that the shared channels' sum over ranks stays on chip.
// Pass 1 reduces sum h^2 and sum g h per rank over the block; pass 2 forms dh, stores dR,
// accumulates the shared sum (ranks in order 0..P-1) and this CTA's dgamma; pass 3 stores dZt.
// The token's h and dout are re-read in passes 2 and 3 (L1/L2 hits).
__global__ void __launch_bounds__(KB_THREADS, 1) rownorm_bwd_kernel(const __grid_constant__ BwdParams prm) {
  __shared__ float red[2 * KB_MAXP][KB_THREADS / 32];
  __shared__ float s_r[KB_MAXP], s_k[KB_MAXP];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int H = prm.H, P = prm.P;
  const int nvec = H >> 3;
  const float inv_h = 1.0f / static_cast<float>(H);
  const size_t rstride = static_cast<size_t>(prm.T) * H;
  float gam[KB_VEC][8];
  float dg[KB_VEC][8];
#pragma unroll
  for (int k = 0; k < KB_VEC; ++k) {
    const int v = threadIdx.x + k * KB_THREADS;
    const uint4 g = v < nvec ? *reinterpret_cast<const uint4*>(prm.gamma + 8 * v) : make_uint4(0, 0, 0, 0);
    unpack8(g, gam[k]);
#pragma unroll
    for (int e = 0; e < 8; ++e) dg[k][e] = 0.f;
  }

  for (int64_t t = blockIdx.x; t < prm.T; t += gridDim.x) {
    const size_t toff = static_cast<size_t>(t) * H;
    // pass 1: per-rank sums of h^2 and g h
    float ss[KB_MAXP], gd[KB_MAXP];
#pragma unroll
    for (int m = 0; m < KB_MAXP; ++m) {
      ss[m] = 0.f;
      gd[m] = 0.f;
      if (m < P) {
#pragma unroll
        for (int k = 0; k < KB_VEC; ++k) {
          const int v = threadIdx.x + k * KB_THREADS;
          if (v < nvec) {
            float hf[8], df[8];
            unpack8(*reinterpret_cast<const uint4*>(prm.h + m * rstride + toff + 8 * v), hf);
            unpack8(*reinterpret_cast<const uint4*>(prm.dout + m * rstride + toff + 8 * v), df);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              ss[m] = fmaf(hf[e], hf[e], ss[m]);
              gd[m] = fmaf(df[e] * gam[k][e], hf[e], gd[m]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < KB_MAXP; ++m) {
      if (m < P) {
        float a = ss[m], b = gd[m];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          a += __shfl_xor_sync(0xFFFFFFFFu, a, off);
          b += __shfl_xor_sync(0xFFFFFFFFu, b, off);
        }
        if (lane == 0) {
          red[2 * m][warp] = a;
          red[2 * m + 1][warp] = b;
        }
      }
    }
    __syncthreads();
    if (threadIdx.x < P) {
      float a = 0.f, b = 0.f;
      for (int w = 0; w < KB_THREADS / 32; ++w) {
        a += red[2 * threadIdx.x][w];
        b += red[2 * threadIdx.x + 1][w];
      }
      const float r = rsqrtf(a * inv_h + prm.eps);
      s_r[threadIdx.x] = r;
      s_k[threadIdx.x] = r * r * r * b * inv_h;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < KB_VEC; ++k) {
      const int v = threadIdx.x + k * KB_THREADS;
      if (v >= nvec) continue;
      const int c = 8 * v;
      const uint32_t bits = (prm.mask_bits[c >> 5] >> (c & 31)) & 0xFFu;
      // pass 2: dh per rank -> dR, the shared sum S, dgamma
      float S[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) S[e] = 0.f;
      for (int m = 0; m < P; ++m) {
        const size_t off = m * rstride + toff + c;
        float hf[8], df[8], dh[8];
        unpack8(*reinterpret_cast<const uint4*>(prm.h + off), hf);
        unpack8(*reinterpret_cast<const uint4*>(prm.dout + off), df);
        const float r = s_r[m], kk = s_k[m];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          dh[e] = r * df[e] * gam[k][e] - hf[e] * kk;
          S[e] += dh[e];
          dg[k][e] = fmaf(df[e], hf[e] * r, dg[k][e]);
        }
        if (prm.dR != nullptr) *reinterpret_cast<uint4*>(prm.dR + off) = pack8(dh);
      }
      // pass 3: dZt per rank (shared channels: S, private: s dh)
      for (int m = 0; m < P; ++m) {
        const size_t off = m * rstride + toff + c;
        float z[8];
        if (bits != 0xFFu) {
          float hf[8], df[8];
          unpack8(*reinterpret_cast<const uint4*>(prm.h + off), hf);
          unpack8(*reinterpret_cast<const uint4*>(prm.dout + off), df);
          const float r = s_r[m], kk = s_k[m];
#pragma unroll
          for (int e = 0; e < 8; ++e) z[e] = prm.private_scale * (r * df[e] * gam[k][e] - hf[e] * kk);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if ((bits >> e) & 1u) z[e] = S[e];
        *reinterpret_cast<uint4*>(prm.dZt + off) = pack8(z);
      }
    }
    __syncthreads();  // red / s_r / s_k are rewritten for the next token
  }
#pragma unroll
  for (int k = 0; k < KB_VEC; ++k) {
    const int v = threadIdx.x + k * KB_THREADS;
    if (v >= nvec) continue;
    float4* dst = reinterpret_cast<float4*>(prm.dg_part + static_cast<size_t>(blockIdx.x) * H + 8 * v);
    dst[0] = make_float4(dg[k][0], dg[k][1], dg[k][2], dg[k][3]);
    dst[1] = make_float4(dg[k][4], dg[k][5], dg[k][6], dg[k][7]);
  }
}

// KB1s: the same as KB1 with the token's h and dout staged in shared memory (cp.async, P H 4
// bytes), so that each is read from memory once.  One 8-channel vector of every rank per thread
// (H <= 8 * KB_THREADS); each thread stages and reads back only its own vectors, so the staging
// needs no block barrier.  Pass 2 leaves in the h slot the private channels' bf16 result
// s * dh, so pass 3 only selects; as soon as pass 2 is done with a token's dout, the next
// token's dout is requested into its slot (and its h after pass 3), so those loads overlap the
// stores of dZt.
template <int MAXP>  // P <= MAXP (8 or 16)
__global__ void __launch_bounds__(KB_THREADS, 1) rownorm_bwd_smem_kernel(const __grid_constant__ BwdParams prm) {
  extern __shared__ __align__(16) uint8_t kb_smem[];
  __shared__ float red[2 * KB_MAXP][KB_THREADS / 32];
  __shared__ float s_r[KB_MAXP], s_k[KB_MAXP];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int H = prm.H, P = prm.P;
  const int nvec = H >> 3;
  const float inv_h = 1.0f / static_cast<float>(H);
  const size_t rstride = static_cast<size_t>(prm.T) * H;
  uint4* sh = reinterpret_cast<uint4*>(kb_smem);                    // [P][nvec] h, then s dh
  uint4* sd = sh + static_cast<size_t>(P) * nvec;                  // [P][nvec] dout
  const int v = threadIdx.x;
  const bool active = v < nvec;
  const int c = 8 * v;
  float gam[8], dg[8];
  unpack8(active ? *reinterpret_cast<const uint4*>(prm.gamma + c) : make_uint4(0, 0, 0, 0), gam);
#pragma unroll
  for (int e = 0; e < 8; ++e) dg[e] = 0.f;
  const uint32_t bits = active ? (prm.mask_bits[c >> 5] >> (c & 31)) & 0xFFu : 0u;

  auto stage = [&](uint4* dst, const __nv_bfloat16* src, int64_t t) {
    if (!active) return;
    const size_t toff = static_cast<size_t>(t) * H + c;
    for (int m = 0; m < P; ++m)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst + m * nvec + v)),
                   "l"(src + m * rstride + toff) : "memory");
  };
  if (blockIdx.x < prm.T) {
    stage(sh, prm.h, blockIdx.x);
    stage(sd, prm.dout, blockIdx.x);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");

  for (int64_t t = blockIdx.x; t < prm.T; t += gridDim.x) {
    const size_t toff = static_cast<size_t>(t) * H + c;
    const int64_t tn = t + gridDim.x;  // this CTA's next token
    asm volatile("cp.async.wait_group 0;" ::: "memory");  // this token's h and dout (own vectors)
    // per rank m: value m = sum of h^2, value MAXP + m = sum of g h over this thread's channels
    float sums[2 * MAXP];
#pragma unroll
    for (int m = 0; m < MAXP; ++m) {
      float a = 0.f, b = 0.f;
      if (active && m < P) {
        float hf[8], df[8];
        unpack8(sh[m * nvec + v], hf);
        unpack8(sd[m * nvec + v], df);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          a = fmaf(hf[e], hf[e], a);
          b = fmaf(df[e] * gam[e], hf[e], b);
        }
      }
      sums[m] = a;
      sums[MAXP + m] = b;
    }
    warp_sum_many<2 * MAXP>(sums, lane);
    {
      constexpr int kShift = (2 * MAXP == 32) ? 0 : (2 * MAXP == 16 ? 1 : 2);
      const int idx = lane >> kShift;  // the value this lane holds the warp total of
      if ((lane & ((1 << kShift) - 1)) == 0) {
        const int m = idx % MAXP;
        if (m < P) red[2 * m + (idx >= MAXP ? 1 : 0)][warp] = sums[0];
      }
    }
    __syncthreads();
    if (threadIdx.x < P) {
      float a = 0.f, b = 0.f;
      for (int w = 0; w < KB_THREADS / 32; ++w) {
        a += red[2 * threadIdx.x][w];
        b += red[2 * threadIdx.x + 1][w];
      }
      const float r = rsqrtf(a * inv_h + prm.eps);
      s_r[threadIdx.x] = r;
      s_k[threadIdx.x] = r * r * r * b * inv_h;
    }
    __syncthreads();
    float S[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) S[e] = 0.f;
    if (MAXP <= 8 && prm.zk_regs) {
      // pass 2: dh per rank -> dR, the shared sum S, dgamma; bf16(s dh) kept in registers, so
      // both of this token's slots are free before pass 3 and the next token's loads start now
      uint4 zk[MAXP];
#pragma unroll
      for (int m = 0; m < MAXP; ++m) {
        zk[m] = make_uint4(0u, 0u, 0u, 0u);
        if (active && m < P) {
          float hf[8], df[8], dh[8], zp[8];
          unpack8(sh[m * nvec + v], hf);
          unpack8(sd[m * nvec + v], df);
          const float r = s_r[m], kk = s_k[m];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            dh[e] = r * df[e] * gam[e] - hf[e] * kk;
            S[e] += dh[e];
            dg[e] = fmaf(df[e], hf[e] * r, dg[e]);
            zp[e] = prm.private_scale * dh[e];
          }
          if (prm.dR != nullptr) *reinterpret_cast<uint4*>(prm.dR + m * rstride + toff) = pack8(dh);
          zk[m] = pack8(zp);
        }
      }
      if (tn < prm.T) {  // this thread's slots of this token are no longer read
        stage(sd, prm.dout, tn);
        stage(sh, prm.h, tn);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      // pass 3: dZt per rank (shared channels: S, private: s dh)
#pragma unroll
      for (int m = 0; m < MAXP; ++m) {
        if (active && m < P) {
          float z[8];
          unpack8(zk[m], z);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if ((bits >> e) & 1u) z[e] = S[e];
          *reinterpret_cast<uint4*>(prm.dZt + m * rstride + toff) = pack8(z);
        }
      }
    } else {
      if (active) {
        // pass 2: dh per rank -> dR, the shared sum S, dgamma; the h slot gets bf16(s dh)
        for (int m = 0; m < P; ++m) {
          float hf[8], df[8], dh[8], zp[8];
          unpack8(sh[m * nvec + v], hf);
          unpack8(sd[m * nvec + v], df);
          const float r = s_r[m], kk = s_k[m];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            dh[e] = r * df[e] * gam[e] - hf[e] * kk;
            S[e] += dh[e];
            dg[e] = fmaf(df[e], hf[e] * r, dg[e]);
            zp[e] = prm.private_scale * dh[e];
          }
          if (prm.dR != nullptr) *reinterpret_cast<uint4*>(prm.dR + m * rstride + toff) = pack8(dh);
          sh[m * nvec + v] = pack8(zp);
        }
      }
      if (tn < prm.T) stage(sd, prm.dout, tn);  // dout of this token is no longer needed
      asm volatile("cp.async.commit_group;" ::: "memory");
      if (active) {
        // pass 3: dZt per rank (shared channels: S, private: s dh)
        for (int m = 0; m < P; ++m) {
          float z[8];
          unpack8(sh[m * nvec + v], z);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if ((bits >> e) & 1u) z[e] = S[e];
          *reinterpret_cast<uint4*>(prm.dZt + m * rstride + toff) = pack8(z);
        }
      }
      if (tn < prm.T) stage(sh, prm.h, tn);  // the h slots were read back by this thread only
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    __syncthreads();  // red / s_r / s_k are reused next token
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  if (active) {
    float4* dst = reinterpret_cast<float4*>(prm.dg_part + static_cast<size_t>(blockIdx.x) * H + c);
    dst[0] = make_float4(dg[0], dg[1], dg[2], dg[3]);
    dst[1] = make_float4(dg[4], dg[5], dg[6], dg[7]);
  }
}

// Dynamic shared memory of rownorm_bwd_smem_kernel.
inline size_t bwd_smem_bytes(int P, int H) { return static_cast<size_t>(P) * H * 2 * 2; }

// KB2: dgamma[c] = sum over the CTAs of KB1 (in CTA order) of their partials.
__global__ void dgamma_reduce_kernel(const float* __restrict__ part, float* __restrict__ dgamma, int nparts, int H) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= H) return;
  float a = 0.f;
  for (int b = 0; b < nparts; ++b) a += part[static_cast<size_t>(b) * H + c];
  dgamma[c] = a;
}

// KB3: batched transpose of bf16 matrices, in [B][R][C] -> out [B][C][Rp], out[b][c][r] =
// in[b][r][c] for r < R and 0 for R <= r < Rp (the zero tail makes the reduction length of the
// GEMM that reads it a multiple of 8).  KT_ROWS x KT_COLS tiles through shared memory; 16-byte
// loads (a warp reads 4 rows x 128 bytes) and 16-byte stores (a warp reads one shared row
// segment of 32 consecutive columns: no bank conflicts).  C % 8 == 0 and Rp % 8 == 0.
constexpr int KT_ROWS = 128;
constexpr int KT_COLS = 64;
constexpr int KT_PITCH = KT_COLS + 8;  // u16 per shared row (16-byte aligned rows)
constexpr int KT_THREADS = 256;
__global__ void __launch_bounds__(KT_THREADS) transpose_pad_kernel(const __nv_bfloat16* __restrict__ in,
                                                                   __nv_bfloat16* __restrict__ out, int64_t R,
                                                                   int64_t C, int64_t Rp) {
  __shared__ __align__(16) uint16_t tile[KT_ROWS][KT_PITCH];
  const int64_t b = blockIdx.z;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * KT_COLS;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * KT_ROWS;
  const __nv_bfloat16* src = in + b * R * C;
  __nv_bfloat16* dst = out + b * C * Rp;
  constexpr int VPR = KT_COLS / 8;  // 16-byte vectors per tile row
#pragma unroll
  for (int i = 0; i < KT_ROWS * VPR / KT_THREADS; ++i) {
    const int idx = threadIdx.x + i * KT_THREADS;
    const int rr = idx / VPR, vv = idx % VPR;
    const int64_t r = r0 + rr, c = c0 + 8 * vv;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < R && c < C) v = *reinterpret_cast<const uint4*>(src + r * C + c);
    *reinterpret_cast<uint4*>(&tile[rr][8 * vv]) = v;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < KT_COLS * (KT_ROWS / 8) / KT_THREADS; ++i) {
    const int idx = threadIdx.x + i * KT_THREADS;
    const int cc = idx % KT_COLS, vv = idx / KT_COLS;
    const int64_t c = c0 + cc, r = r0 + 8 * vv;
    if (c < C && r < Rp) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        w[e] = static_cast<uint32_t>(tile[8 * vv + 2 * e][cc]) | (static_cast<uint32_t>(tile[8 * vv + 2 * e + 1][cc]) << 16);
      *reinterpret_cast<uint4*>(dst + c * Rp + r) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

}  // namespace caat
