// permuted.cuh - the channel-permuted path for a sync set given as a sorted channel list.
//
// "Tensor-Parallelism with Partially Synchronized Activations" (§3, App. A.2 Eq. 22) shares
// the first floor(h p) channels; with a sync set S given as an arbitrary sorted list, nearly
// every 256-channel block of the output holds both shared and private channels, and such a
// block costs the row-parallel GEMM two accumulations (all ranks' K for its shared channels,
// each rank's K/P for its private ones).  Permuting the output channels so that S comes
// first makes the set contiguous again (pure blocks, one accumulation each):
//
//   perm(i) = the i-th channel of S for i < n_s, the (i - n_s)-th channel outside S otherwise
//   W'_m[i, :] = W_m[perm(i), :]          (K5 permute_rows_kernel, once per weight)
//   Z'_m = GEMM + partial channel-reduce of X_m W'_m^T with S' = {0 .. n_s - 1}
//   h_m[:, c] = Z'_m[:, pos(c)] + R_m[:, c],  pos = perm^{-1}    (K2p rownorm_gather_kernel)
//   out_m = RMSNorm(h_m) * gamma
//
// Everything is a pure relabelling of channels: Eq. 22's sums and the residual add and norm
// of Eq. 9 are unchanged.  Z' is rounded to bf16 once before the residual add (the GEMM's
// epilogue writes it; the norm kernel adds R), where the unpermuted path rounds h once.
#pragma once

#include "ptx.cuh"
#include "rowpar_common.cuh"

namespace caat {

constexpr int K5_THREADS = 256;
constexpr int K2P_THREADS = 256;

struct PermParams {
  int P, H, Kp, n_s;
  int64_t T;
  float eps;
  uint32_t mask_bits[K1_MASK_WORDS];  // bit c = original channel c is shared
};

// s_pre[w] = number of shared channels in mask words [0, w), w = 0..nw; s_mask = the words.
// Whole block; nw <= K1_MASK_WORDS.
__device__ __forceinline__ void mask_prefix(const uint32_t* mask, int nw, uint32_t* s_mask, int* s_pre) {
  __shared__ int warp_tot[32];
  const int nthr = blockDim.x;
  const int per = (nw + nthr - 1) / nthr;
  const int w0 = min(nw, threadIdx.x * per), w1 = min(nw, w0 + per);
  int local = 0;
  for (int w = w0; w < w1; ++w) {
    const uint32_t m = mask[w];
    s_mask[w] = m;
    local += __popc(m);
  }
  // block exclusive scan of `local`
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nwarps = nthr >> 5;
    int t = lane < nwarps ? warp_tot[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, t, off);
      if (lane >= off) t += y;
    }
    if (lane < nwarps) warp_tot[lane] = t;  // inclusive over warps
  }
  __syncthreads();
  int run = incl - local + (warp > 0 ? warp_tot[warp - 1] : 0);
  for (int w = w0; w < w1; ++w) {
    s_pre[w] = run;
    run += __popc(mask[w]);
  }
  if (w1 == nw && w0 < w1) s_pre[nw] = run;
  if (nw == 0 && threadIdx.x == 0) s_pre[0] = 0;
  __syncthreads();
}

// Position of the k-th (0-based) set bit of m (k < popc(m)).
__device__ __forceinline__ int select_bit(uint32_t m, int k) {
  for (int j = 0; j < k; ++j) m &= m - 1u;
  return __ffs(static_cast<int>(m)) - 1;
}

// perm(i): the original channel at permuted position i.
__device__ __forceinline__ int perm_src(int i, int n_s, int H, int nw, const uint32_t* s_mask, const int* s_pre) {
  if (i < n_s) {
    int lo = 0, hi = nw - 1;  // last word w with s_pre[w] <= i
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= i) lo = mid; else hi = mid - 1;
    }
    return 32 * lo + select_bit(s_mask[lo], i - s_pre[lo]);
  }
  const int k = i - n_s;
  int lo = 0, hi = nw - 1;  // last word w with (clear bits before w) <= k
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (32 * mid - s_pre[mid] <= k) lo = mid; else hi = mid - 1;
  }
  const int valid = min(32, H - 32 * lo);
  const uint32_t clear = ~s_mask[lo] & (valid == 32 ? 0xFFFFFFFFu : ((1u << valid) - 1u));
  return 32 * lo + select_bit(clear, k - (32 * lo - s_pre[lo]));
}

// pos(c) = perm^{-1}(c): the permuted position of original channel c.
__device__ __forceinline__ int perm_pos(int c, int n_s, const uint32_t* s_mask, const int* s_pre) {
  const int w = c >> 5, b = c & 31;
  const uint32_t m = s_mask[w];
  const int before = s_pre[w] + __popc(m & ((1u << b) - 1u));
  return ((m >> b) & 1u) ? before : n_s + c - before;
}

// K5: W'[m][i, :] = W[m][perm(i), :] for every rank m; one warp per row, 16-byte copies.
__global__ void __launch_bounds__(K5_THREADS)
    permute_rows_kernel(const __nv_bfloat16* __restrict__ W, __nv_bfloat16* __restrict__ Wp,
                        const __grid_constant__ PermParams prm) {
  __shared__ uint32_t s_mask[K1_MASK_WORDS];
  __shared__ int s_pre[K1_MASK_WORDS + 1];
  const int nw = (prm.H + 31) >> 5;
  mask_prefix(prm.mask_bits, nw, s_mask, s_pre);
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(prm.P) * prm.H;
  const int nvec = prm.Kp >> 3;
  for (int64_t i = (static_cast<int64_t>(blockIdx.x) * K5_THREADS + threadIdx.x) >> 5; i < rows;
       i += (static_cast<int64_t>(gridDim.x) * K5_THREADS) >> 5) {
    const int64_t m = i / prm.H;
    const int c = static_cast<int>(i - m * prm.H);
    const int src = perm_src(c, prm.n_s, prm.H, nw, s_mask, s_pre);
    const uint4* s4 = reinterpret_cast<const uint4*>(W + (m * prm.H + src) * prm.Kp);
    uint4* d4 = reinterpret_cast<uint4*>(Wp + (m * prm.H + c) * prm.Kp);
    for (int v = lane; v < nvec; v += 32) d4[v] = s4[v];
  }
}

// K2p: per (rank, token) row, one warp: Z' row (permuted channels) into shared memory, then
// for each original channel c: h = bf16(Z'[pos(c)] + R[c]); sum of squares of the stored h;
// out = h / sqrt(mean + eps) * gamma.  pos is a per-block table (the same for every row);
// h stays in registers (VPL 128-bit vectors per lane, H <= 256 * VPL).  Z' may be the h or
// out buffer itself: a row is read completely before the warp writes it.  Dynamic shared
// memory (gather_smem_bytes): mask words, prefix counts, pos table, one H-wide row per warp.
template <int VPL>
__global__ void __launch_bounds__(K2P_THREADS, VPL >= 16 ? 1 : 2)
    rownorm_gather_kernel(const __nv_bfloat16* Zp, const __nv_bfloat16* R, __nv_bfloat16* Hout,
                          __nv_bfloat16* Out, const __nv_bfloat16* __restrict__ gamma,
                          const __grid_constant__ PermParams prm) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int H = prm.H;
  const int nw = (H + 31) >> 5;
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(smem_raw);
  int* s_pre = reinterpret_cast<int*>(smem_raw + 4 * nw);
  uint16_t* s_pos = reinterpret_cast<uint16_t*>(smem_raw + ((8 * nw + 4 + 15) & ~15));
  uint8_t* rows_base = reinterpret_cast<uint8_t*>(s_pos) + ((2 * H + 15) & ~15);
  mask_prefix(prm.mask_bits, nw, s_mask, s_pre);
  for (int c = threadIdx.x; c < H; c += blockDim.x) s_pos[c] = static_cast<uint16_t>(perm_pos(c, prm.n_s, s_mask, s_pre));
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nvec = H >> 3;
  const float inv_h = 1.0f / static_cast<float>(H);
  uint4* srow4 = reinterpret_cast<uint4*>(rows_base + static_cast<size_t>(warp) * H * 2);
  const unsigned short* s16 = reinterpret_cast<const unsigned short*>(srow4);
  const uint4* pos4 = reinterpret_cast<const uint4*>(s_pos);
  const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
  const int64_t rows = static_cast<int64_t>(prm.P) * prm.T;

  for (int64_t i = (static_cast<int64_t>(blockIdx.x) * K2P_THREADS + threadIdx.x) >> 5; i < rows;
       i += (static_cast<int64_t>(gridDim.x) * K2P_THREADS) >> 5) {
    const size_t off = static_cast<size_t>(i) * H;
    const uint4* zp4 = reinterpret_cast<const uint4*>(Zp + off);
    const uint4* r4 = reinterpret_cast<const uint4*>(R + off);
    __syncwarp();  // the previous row's gathers are done with the row buffer
    // Z' row straight into shared memory (cp.async, no registers) while R comes into registers
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const int idx = 32 * u + lane;
      if (idx < nvec)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(srow4 + idx)), "l"(zp4 + idx)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    uint4 t[VPL];
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const int idx = 32 * u + lane;
      t[u] = idx < nvec ? r4[idx] : make_uint4(0, 0, 0, 0);
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncwarp();  // every lane's part of the row has landed
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const int idx = 32 * u + lane;
      if (idx < nvec) {
        const uint4 pv = pos4[idx];  // pos of channels 8 idx .. 8 idx + 7 (u16 each)
        const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
        const uint32_t rw[4] = {t[u].x, t[u].y, t[u].z, t[u].w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float z0 = __uint_as_float(static_cast<uint32_t>(s16[pw[e] & 0xFFFFu]) << 16);
          const float z1 = __uint_as_float(static_cast<uint32_t>(s16[pw[e] >> 16]) << 16);
          o[e] = pack_bf16x2(z0 + bf16lo(rw[e]), z1 + bf16hi(rw[e]));
          const float lo = bf16lo(o[e]), hi = bf16hi(o[e]);
          ss = fmaf(lo, lo, ss);
          ss = fmaf(hi, hi, ss);
        }
        t[u] = make_uint4(o[0], o[1], o[2], o[3]);  // h
      }
    }
#pragma unroll
    for (int sh = 16; sh > 0; sh >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, sh);
    const float rstd = rsqrtf(ss * inv_h + prm.eps);
    __syncwarp();  // every lane's reads of this row (Z' may be Hout or Out) are done
    uint4* h4 = reinterpret_cast<uint4*>(Hout + off);
    uint4* o4 = reinterpret_cast<uint4*>(Out + off);
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const int idx = 32 * u + lane;
      if (idx < nvec) {
        if (Hout != nullptr) h4[idx] = t[u];
        const uint4 g = __ldg(g4 + idx);
        const uint32_t w[4] = {t[u].x, t[u].y, t[u].z, t[u].w};
        const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          o[e] = pack_bf16x2(bf16lo(w[e]) * rstd * bf16lo(gw[e]), bf16hi(w[e]) * rstd * bf16hi(gw[e]));
        o4[idx] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

// Dynamic shared memory of rownorm_gather_kernel for hidden size H (<= 4096).
inline size_t gather_smem_bytes(int H) {
  const size_t nw = static_cast<size_t>(H + 31) / 32;
  return ((8 * nw + 4 + 15) & ~size_t(15)) + ((2 * static_cast<size_t>(H) + 15) & ~size_t(15)) +
         static_cast<size_t>(K2P_THREADS / 32) * H * 2;
}

}  // namespace caat
