// tp.cuh - the layer split over real devices, one tensor-parallel rank per GPU ("Tensor-
// Parallelism with Partially Synchronized Activations", App. A.2 Eq. 22; §3: only the first
// floor(h p) channels are exchanged; §4: their sum accumulated in fp32; §4 Eq. 9: residual add,
// then the norm).
//
// Two ways to exchange the shared channels' partials:
//   * through the caller's collective (an all-reduce of zs [T, n_s]), then tp_finish_kernel;
//   * over peer memory, with no library collective: the local GEMM's epilogue pushes each
//     rank's fp32 partial of the shared channels straight into the receive buffer of the rank
//     that owns those columns (owner q owns columns [q w, (q + 1) w), w = n_s / world), the
//     owner sums the world partials of its slice in rank order and writes the sum into every
//     rank's gather buffer (tp_reduce_kernel), and each rank finishes from its gather buffer
//     (tp_finish_kernel after a wait).  The exchange is a reduce-scatter fused into the GEMM
//     epilogue plus an all-gather: (world - 1) / world of T n_s fp32 values sent per rank in
//     each half, as a ring all-reduce of the same buffer.  Completion is signalled with
//     per-call epochs in each rank's flag array [2][world] (phase 0: partials pushed by rank
//     r; phase 1: slice reduced by owner q): the last CTA of a launch to finish raises them
//     (release, system scope) after every CTA's stores are fenced at system scope; waiters
//     poll them (acquire, system scope) with a bounded wait.
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
constexpr int TP_MAX_WORLD = 8;
constexpr int KT_RED_THREADS = 256;

// Bounded wait until flags[0..n) all reach `epoch`.  Returns false (and raises the device status
// word as a timeout tagged `site`) if they do not within timeout_ns, or if another waiter
// already raised it.
__device__ __forceinline__ bool tp_wait_flags(const unsigned int* flags, int n, uint32_t epoch, uint64_t timeout_ns,
                                              int site) {
  const uint64_t t0 = globaltimer_ns();
  for (int i = 0; i < n; ++i) {
    for (uint32_t k = 1;; ++k) {
      if (static_cast<int32_t>(ld_acquire_sys_u32(flags + i) - epoch) >= 0) break;
      if ((k & 63u) == 0u) {
        if (status_poll() != 0) return false;
        if (globaltimer_ns() - t0 > timeout_ns) {
          status_raise(4, site);
          return false;
        }
      }
    }
  }
  return true;
}

// One thread per CTA, after a CTA barrier that orders the CTA's stores (to this and other GPUs)
// before it: fence at system scope and count the CTA as done; the last of `total` raises flags[q][phase * world + rank] = epoch on
// every rank q.  Nothing is raised once the device status word is set (an error: the waiters
// time out instead of reading incomplete data).
__device__ __forceinline__ void tp_signal_done(unsigned int* done, uint32_t total, unsigned int* const* flags,
                                               int world, int phase, int rank, uint32_t epoch) {
  fence_sc_sys();
  const uint32_t old = atom_add_acq_rel_gpu_u32(done, 1u);
  if (old != total - 1u || status_poll() != 0) return;
  fence_sc_sys();
  for (int q = 0; q < world; ++q) st_release_sys_u32(flags[q] + phase * world + rank, epoch);
}

// The owner's step of the peer-memory exchange.
struct TpReduceParams {
  const float* recv;                   // this rank's receive buffer [world][T][w]
  float* gather[TP_MAX_WORLD];         // every rank's gather buffer [T][n_s]
  unsigned int* flags[TP_MAX_WORLD];   // every rank's flag array [2][world]
  unsigned int* done;                  // CTAs of this launch done, zero at launch
  int64_t T;
  int w, n_s, world, rank;
  uint32_t epoch;
  uint64_t timeout_ns;
};

// Waits until every rank has pushed its partials of this rank's slice, sums the world partials
// per element in rank order (fp32), and stores the sum into columns [rank w, (rank + 1) w) of
// every rank's gather buffer; then signals phase 1.  16-byte accesses (w % 4 == 0).
__global__ void __launch_bounds__(KT_RED_THREADS)
    tp_reduce_kernel(const __grid_constant__ TpReduceParams prm) {
  __shared__ int s_ok;
  if (threadIdx.x == 0)
    s_ok = tp_wait_flags(prm.flags[prm.rank], prm.world, prm.epoch, prm.timeout_ns, 81) ? 1 : 0;
  __syncthreads();
  if (!s_ok) return;
  const int w4 = prm.w >> 2;
  const int64_t n4 = prm.T * w4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * KT_RED_THREADS;
  const int64_t slab = prm.T * prm.w;  // between the partials of two ranks
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * KT_RED_THREADS + threadIdx.x; i < n4; i += stride) {
    const int64_t t = i / w4;
    const int j = static_cast<int>(i - t * w4) * 4;
    const float* src = prm.recv + t * prm.w + j;
    float4 s = __ldcg(reinterpret_cast<const float4*>(src));
    for (int r = 1; r < prm.world; ++r) {
      const float4 z = __ldcg(reinterpret_cast<const float4*>(src + r * slab));
      s.x += z.x;
      s.y += z.y;
      s.z += z.z;
      s.w += z.w;
    }
    const int64_t off = t * prm.n_s + static_cast<int64_t>(prm.rank) * prm.w + j;
    for (int g = 0; g < prm.world; ++g) *reinterpret_cast<float4*>(prm.gather[g] + off) = s;
  }
  __syncthreads();  // the CTA's stores precede thread 0's system-scope fence in tp_signal_done
  if (threadIdx.x == 0) tp_signal_done(prm.done, gridDim.x, prm.flags, prm.world, 1, prm.rank, prm.epoch);
}

// wait_flags (optional): the peer-memory exchange's phase-1 flags of this rank [world]; the
// kernel first waits (bounded) until they all reach `epoch`.  The T rows are `ranks` x `tokens`
// ([ranks, tokens, H]; ranks = 1 for one device's rank), and the row of token tk of any rank takes
// its shared sums from zs row tk: the single-device layer's P ranks add their own residual to the
// same cross-rank sum.
template <int VPL>
__global__ void __launch_bounds__(KT_FIN_THREADS, 2)
    tp_finish_kernel(const float* __restrict__ zs, const __nv_bfloat16* __restrict__ R, __nv_bfloat16* h, __nv_bfloat16* out,
                     const __nv_bfloat16* __restrict__ gamma, int64_t T, int H, int n_s, float eps,
                     const unsigned int* wait_flags, int wait_n, uint32_t epoch, uint64_t timeout_ns,
                     int64_t tokens, int ranks) {
  if (wait_flags != nullptr) {
    __shared__ int s_ok;
    if (threadIdx.x == 0) s_ok = tp_wait_flags(wait_flags, wait_n, epoch, timeout_ns, 82) ? 1 : 0;
    __syncthreads();
    if (!s_ok) return;
  }
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * KT_FIN_THREADS + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * KT_FIN_THREADS) >> 5;
  const int nvec = H >> 3;
  const float inv_h = 1.0f / static_cast<float>(H);
  const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
  for (int64_t i = warp_global; i < T; i += nwarps) {
    // row i: token tk = i / ranks of rank m = i % ranks, so the ranks of a token are neighbouring
    // warps and read its shared sums (zs row tk) while they are in cache
    const int64_t tk = i / ranks;
    const int64_t t = (i - tk * ranks) * tokens + tk;  // the row in [ranks, tokens, H]
    uint4* hp = reinterpret_cast<uint4*>(h + t * H);
    const uint4* rp = reinterpret_cast<const uint4*>(R + t * H);
    const float4* zp = reinterpret_cast<const float4*>(zs + tk * n_s);
    uint4 x[VPL];
#pragma unroll
    for (int u = 0; u < VPL; ++u) {
      const int idx = 32 * u + lane;  // channels 8 idx .. 8 idx + 7
      x[u] = make_uint4(0, 0, 0, 0);
      if (idx < nvec) {
        if (8 * idx + 8 <= n_s) {
          // shared: the ranks' summed partial plus this rank's residual, rounded once
          const uint4 r = __ldg(rp + idx);
          const float4 z0 = __ldcg(zp + 2 * idx), z1 = __ldcg(zp + 2 * idx + 1);
          x[u].x = pack_bf16x2(z0.x + bf16lo(r.x), z0.y + bf16hi(r.x));
          x[u].y = pack_bf16x2(z0.z + bf16lo(r.y), z0.w + bf16hi(r.y));
          x[u].z = pack_bf16x2(z1.x + bf16lo(r.z), z1.y + bf16hi(r.z));
          x[u].w = pack_bf16x2(z1.z + bf16lo(r.w), z1.w + bf16hi(r.w));
        } else {
          x[u] = hp[idx];  // private channels, finished by the local step
        }
      }
    }
    // (no store in the loop above, so that its loads can all be in flight together)
    if (h != out) {  // h and out the same buffer: out below overwrites it
#pragma unroll
      for (int u = 0; u < VPL; ++u) {
        const int idx = 32 * u + lane;
        if (idx < nvec && 8 * idx + 8 <= n_s) hp[idx] = x[u];
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

// The norm of the single-device layer's shared-sum mode: one CTA (8 warps) per token, the ranks
// of that token on its warps.  The token's shared sums (zs row, n_s fp32) are copied once into
// shared memory (cp.async, a ring of three rows across the CTA's tokens, so that one barrier per
// token both publishes a row and frees the one refilled next) and read from there by every
// rank's warp: rank m's row gets h[c] = bf16(zs[c] + R_m[c]) for c < n_s and its private h[c]
// (stored by the GEMM) otherwise, then the RMSNorm (fp32 sum of squares of the bf16 row, one
// warp, the row in registers) and out = h / sqrt(sum / H + eps) * gamma.  h is stored for the
// shared channels only when it is not the out buffer.  Same arithmetic as tp_finish_kernel.
//   * Tokens are taken from the last one down: the GEMM stores its last rank's private tiles
//     last, so some of those rows may still be in L2.
constexpr int KZ_THREADS = 256;
constexpr int KZ_MAX_NS = 4096;

template <int VPL>
__global__ void __launch_bounds__(KZ_THREADS, 2)
    rownorm_zs_kernel(const float* __restrict__ zs, const __nv_bfloat16* __restrict__ R, __nv_bfloat16* h,
                      __nv_bfloat16* out, const __nv_bfloat16* __restrict__ gamma, int64_t tokens, int P, int H,
                      int n_s, float eps) {
  __shared__ __align__(16) float s_z[3][KZ_MAX_NS];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nvec = H >> 3;
  const int nz4 = n_s >> 2;  // float4 of a zs row
  const float inv_h = 1.0f / static_cast<float>(H);
  const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
  auto fetch = [&](int64_t tk, int b) {
    const float4* src = reinterpret_cast<const float4*>(zs + tk * n_s);
    float4* dst = reinterpret_cast<float4*>(s_z[b]);
    for (int q = threadIdx.x; q < nz4; q += KZ_THREADS)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst + q)), "l"(src + q) : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  int64_t j = blockIdx.x;  // the CTA's k-th token is tokens - 1 - (blockIdx.x + k gridDim.x)
  if (j < tokens) fetch(tokens - 1 - j, 0);
  for (int k = 0; j < tokens; j += gridDim.x, ++k) {
    const int64_t tk = tokens - 1 - j;
    const int b = k % 3;
    const bool more = j + gridDim.x < tokens;
    // the row refilled here held token k - 2, which every warp finished before the last barrier
    if (more) fetch(tk - gridDim.x, b == 2 ? 0 : b + 1);
    if (more) asm volatile("cp.async.wait_group 1;" ::: "memory");
    else asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();  // every thread's part of this token's zs row has landed
    const float4* z4 = reinterpret_cast<const float4*>(s_z[b]);
    for (int m = warp; m < P; m += KZ_THREADS / 32) {
      const int64_t row = static_cast<int64_t>(m) * tokens + tk;
      uint4* hp = reinterpret_cast<uint4*>(h + row * H);
      const uint4* rp = reinterpret_cast<const uint4*>(R + row * H);
      uint4 x[VPL];
#pragma unroll
      for (int u = 0; u < VPL; ++u) {
        const int idx = 32 * u + lane;
        x[u] = make_uint4(0, 0, 0, 0);
        if (idx < nvec) x[u] = (8 * idx + 8 <= n_s) ? __ldg(rp + idx) : hp[idx];  // residual / private h
      }
#pragma unroll
      for (int u = 0; u < VPL; ++u) {
        const int idx = 32 * u + lane;
        if (idx < nvec && 8 * idx + 8 <= n_s) {
          const uint4 r = x[u];
          const float4 z0 = z4[2 * idx], z1 = z4[2 * idx + 1];
          x[u].x = pack_bf16x2(z0.x + bf16lo(r.x), z0.y + bf16hi(r.x));
          x[u].y = pack_bf16x2(z0.z + bf16lo(r.y), z0.w + bf16hi(r.y));
          x[u].z = pack_bf16x2(z1.x + bf16lo(r.z), z1.y + bf16hi(r.z));
          x[u].w = pack_bf16x2(z1.z + bf16lo(r.w), z1.w + bf16hi(r.w));
        }
      }
      if (h != out) {
#pragma unroll
        for (int u = 0; u < VPL; ++u) {
          const int idx = 32 * u + lane;
          if (idx < nvec && 8 * idx + 8 <= n_s) hp[idx] = x[u];
        }
      }
      float ss = 0.f;
#pragma unroll
      for (int u = 0; u < VPL; ++u) {
        const uint32_t w[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = bf16lo(w[e]), c = bf16hi(w[e]);
          ss = fmaf(a, a, ss);
          ss = fmaf(c, c, ss);
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
}

}  // namespace caat
