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

// The same row norm as rownorm_reg_kernel, fed by the GEMM kernel's row-block counters instead
// of a fixed row range, so that it runs while the GEMM is still computing.  The GEMM kernel
// (launched just before, with a grid that leaves some SMs free) adds 1 to the counter of a
// (128-row block, rank) for every epilogue warp's finished tile of it; the block is complete
// when its counter reaches `target` (tiles per row x 4 warps).  This kernel is launched as a
// programmatic dependent of the GEMM, so its blocks (one per SM: the row ring below fills the
// SM's shared memory, which also keeps them off the SMs that hold a GEMM CTA) start on the
// free SMs as soon as every GEMM CTA has started, and spread to the other SMs as GEMM CTAs exit.
//   * Jobs (128-row blocks of one rank) are taken in the order the GEMM's tile order completes
//     them (`order`: 0 = rank by rank, else row block by row block, ranks in order), as 8-row
//     pieces claimed from a counter.  Each warp keeps a ring of up to 8 rows in flight: every row
//     is one bulk copy (cp.async.bulk, H*2 bytes) into the warp's slot, so a few SMs pull h at a
//     high rate.  The row is then normalized from shared memory (fp32 sum of squares, warp
//     reduction, rsqrt, gamma) and stored with 16-byte stores.  The arithmetic, and so every
//     bit of out, is that of rownorm_reg_kernel.
//   * A warp only blocks on a piece whose row block is not complete when it has no row in
//     flight; that wait gives up after `timeout_ns` without progress of the GEMM (its unit
//     counter, `progress`; the GEMM as a whole may run longer than the timeout), or when another
//     wait set the status word.
//   * h and out may alias.
//   * With target 0 it is the plain bulk-copy row norm of every row (launched after the GEMM).
constexpr int K2C_THREADS = 256;
constexpr int K2C_ROWS_PER_JOB = 128;
constexpr int K2C_ROWS_PER_PIECE = 8;
constexpr int K2C_WARP_BYTES = 24576;   // ring of row slots per warp
constexpr int K2C_MAX_SLOTS = 8;
constexpr int K2C_SMEM_BYTES = 128 + (K2C_THREADS / 32) * (K2C_WARP_BYTES + K2C_MAX_SLOTS * 16);

__device__ __forceinline__ uint32_t ld_acquire_u32(const unsigned int* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_relaxed_u32(const unsigned int* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) global -> this CTA's
// shared memory, completing on `bar` (complete_tx).
__device__ __forceinline__ void bulk_load_g2s(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// The j-th row-block job in completion order: its 128-row block and rank.
__device__ __forceinline__ void k2c_job(int j, int order, int P, int n_m128, int& m128, int& rank) {
  if (order == 0) {  // private tiles rank by rank, row blocks in order within a rank
    rank = j / n_m128;
    m128 = j - rank * n_m128;
  } else {           // row block (pair of 128-row blocks) by row block, ranks in order
    const int m = j / (2 * P);
    const int rem = j - m * 2 * P;
    rank = rem >> 1;
    m128 = 2 * m + (rem & 1);
  }
}

template <int VPL>
__global__ void __launch_bounds__(K2C_THREADS, 1)
    rownorm_consumer_kernel(const __nv_bfloat16* h, __nv_bfloat16* out, const __nv_bfloat16* __restrict__ gamma,
                            int P, int64_t T, int H, float eps, const unsigned int* rb_count, unsigned int target,
                            int n_m128, int order, const unsigned int* progress, unsigned int* piece_claim,
                            uint64_t timeout_ns) {
  extern __shared__ uint8_t k2c_raw[];
  uint8_t* smem = k2c_raw + ((128u - (smem_u32(k2c_raw) & 127u)) & 127u);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t stride = (static_cast<uint32_t>(H) * 2u + 127u) & ~127u;  // slot size
  const int nslot = min(K2C_MAX_SLOTS, static_cast<int>(K2C_WARP_BYTES / stride));
  uint8_t* ring = smem + warp * K2C_WARP_BYTES;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + (K2C_THREADS / 32) * K2C_WARP_BYTES) + warp * K2C_MAX_SLOTS;
  int64_t* rowid = reinterpret_cast<int64_t*>(smem + (K2C_THREADS / 32) * K2C_WARP_BYTES +
                                              (K2C_THREADS / 32) * K2C_MAX_SLOTS * 8) + warp * K2C_MAX_SLOTS;
  if (lane == 0) {
    for (int i = 0; i < nslot; ++i) mbar_init(&bar[i], 1);
    fence_mbar_init();  // the initialized barriers are visible to the bulk copies' complete_tx
  }
  __syncwarp();

  const int nvec = H >> 3;
  const float inv_h = 1.0f / static_cast<float>(H);
  const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
  const uint32_t row_bytes = static_cast<uint32_t>(H) * 2u;
  constexpr int kPieces = K2C_ROWS_PER_JOB / K2C_ROWS_PER_PIECE;
  const int total = n_m128 * P * kPieces;

  int m128 = 0, rk = 0, part = 0, next_i = K2C_ROWS_PER_PIECE;  // current piece (exhausted)
  int pend = -1;                                                // claimed piece, job not yet read
  bool no_more = false, failed = false;
  int issued = 0, consumed = 0;
  uint32_t phases = 0;
  for (;;) {
    // ------------------------------------------------ fill the ring
    while (!no_more && issued - consumed < nslot) {
      if (next_i >= K2C_ROWS_PER_PIECE) {
        if (pend < 0) {
          int c = 0;
          if (lane == 0) c = static_cast<int>(atomicAdd(piece_claim, 1u));
          c = __shfl_sync(0xFFFFFFFFu, c, 0);
          if (c >= total) {
            no_more = true;
            break;
          }
          pend = c;
        }
        const int j = pend / kPieces;
        int jm = 0, jr = 0;
        k2c_job(j, order, P, n_m128, jm, jr);
        if (static_cast<int64_t>(jm) * K2C_ROWS_PER_JOB >= T) {  // a block past the last token
          pend = -1;
          continue;
        }
        const unsigned int* cnt = rb_count + static_cast<size_t>(jm) * P + jr;
        uint32_t v = 0;
        // target 0: launched after the GEMM has finished (stream order), nothing to wait for
        if (lane == 0) v = (target == 0u || ld_acquire_u32(cnt) >= target) ? 1u : 0u;
        v = __shfl_sync(0xFFFFFFFFu, v, 0);
        if (v == 0u && issued > consumed) break;  // not complete yet: work on the rows in flight
        if (v == 0u) {
          if (lane == 0) {
            uint64_t t0 = globaltimer_ns();
            uint32_t seen = ld_relaxed_u32(progress);
            for (uint32_t n = 1;; ++n) {
              if (ld_acquire_u32(cnt) >= target) {
                v = 1u;
                break;
              }
              __nanosleep(512);
              if ((n & 15u) == 0u) {
                if (status_poll() != 0) break;
                const uint32_t now = ld_relaxed_u32(progress);
                if (now != seen) {  // the GEMM is making progress: restart the clock
                  seen = now;
                  t0 = globaltimer_ns();
                } else if (globaltimer_ns() - t0 > timeout_ns) {
                  status_raise(4, 40);
                  break;
                }
              }
            }
          }
          v = __shfl_sync(0xFFFFFFFFu, v, 0);
          if (v == 0u) {
            no_more = true;
            failed = true;
            break;
          }
        }
        m128 = jm;
        rk = jr;
        part = pend - j * kPieces;
        next_i = 0;
        pend = -1;
        // h of this row block was stored by the GEMM (async proxy, other SMs) and published
        // (release / acquire above); the bulk copies that read it are async-proxy reads.
        if (lane == 0) asm volatile("fence.proxy.async.global;" ::: "memory");
      }
      const int64_t t = static_cast<int64_t>(m128) * K2C_ROWS_PER_JOB + part * K2C_ROWS_PER_PIECE + next_i;
      ++next_i;
      if (t >= T) {  // rows beyond T end the piece
        next_i = K2C_ROWS_PER_PIECE;
        continue;
      }
      const int slot = issued % nslot;
      if (lane == 0) {
        const int64_t row = static_cast<int64_t>(rk) * T + t;
        rowid[slot] = row;
        mbar_arrive_expect_tx(&bar[slot], row_bytes);
        bulk_load_g2s(ring + slot * stride, h + row * H, row_bytes, &bar[slot]);
      }
      ++issued;
    }
    if (issued == consumed) break;  // nothing in flight and nothing more to claim
    // ------------------------------------------------ normalize the oldest row in flight
    const int slot = consumed % nslot;
    // every lane waits: the phase completion is what makes the copied bytes visible to it
    const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&bar[slot], (phases >> slot) & 1u, timeout_ns, 41));
    phases ^= 1u << slot;
    ++consumed;
    if (!ok) {
      failed = true;
      break;
    }
    const int64_t row = rowid[slot];
    const uint4* sp = reinterpret_cast<const uint4*>(ring + slot * stride);
    uint4 x[VPL];
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const int idx = 32 * u + lane;
      x[u] = idx < nvec ? sp[idx] : make_uint4(0, 0, 0, 0);
    }
    __syncwarp();
    if (lane == 0) fence_proxy_async_smem();  // the slot's next bulk copy follows these reads
    {
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
      uint4* op = reinterpret_cast<uint4*>(out + row * H);
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
  if (failed) {
    // Error path: give every copy still in flight into this warp's ring time to land (bounded,
    // whatever the status word says) before the block can leave.
    for (; consumed < issued; ++consumed) {
      const int slot = consumed % nslot;
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&bar[slot], (phases >> slot) & 1u) && globaltimer_ns() - t0 < 1000000ull) {
      }
      phases ^= 1u << slot;
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
