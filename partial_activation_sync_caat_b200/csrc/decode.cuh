// decode.cuh - the partially synchronized row-parallel layer for decode-sized token counts
// (T <= 64): the same result as rowpar_gemm*.cuh + rownorm.cuh, reorganized for a call
// whose cost is streaming W once from HBM.
//
// "Tensor-Parallelism with Partially Synchronized Activations": partial products Zt_m =
// X_m W_m^T (App. A.2 Eq. 22, first line), partial channel-reduce (Eq. 22, second line),
// private scale (§4 Eq. 14-15), residual add and RMSNorm (§4 Eq. 9); §3.2 describes running
// all tensor-parallel ranks on one device ("logical devices").
//
// K4a decode_partials_kernel: the work is the sequence of items (unit, k-block), a unit being
//     (rank m, 128-channel block), k-blocks fastest.  Persistent CTA i takes the contiguous items
//     [floor(i N / G), floor((i + 1) N / G)) (stream-K: every CTA streams the same number of W
//     bytes, within one k-block).  It streams its W slices with TMA through a ring whose depth
//     follows the token count (the X tile of a stage is T padded to 16 rows), and computes the
//     swapped product D[c, t] = W_m[c,:] . X_m[t,:] with tcgen05.mma (M = 128 channels, N = T
//     padded, fp32 in TMEM).  Each run of a CTA's items inside one unit (a segment) is one
//     accumulation, written as an fp32 partial to Zp[slot][m][t][c]: slot 0 for the segment
//     that starts the unit, slot 1 for the one that ends a unit split between two CTAs (the
//     grid never exceeds the unit count, so a unit has at most two segments).  The tokens are
//     the N side, so W (the only large operand) is read exactly once.
// K4b decode_reduce_norm_kernel: one CTA per (rank m, token t) row.  It adds the two slots of
//     a split unit, forms the shared channels' cross-rank sum (ranks in order, fp32), applies
//     the private scale, adds the residual, stores h (bf16), reduces the sum of squares of the
//     stored h over the CTA and rescales the row held in registers:
//     out = h / sqrt(sum/H + eps) * gamma.
#pragma once

#include "permuted.cuh"
#include "ptx.cuh"
#include "rowpar_common.cuh"

namespace caat {

constexpr int K4_BM = 128;                 // channels per unit
constexpr int K4_BK = 64;
constexpr int K4_MAXN = 64;                // max padded token count
constexpr int K4_A_BYTES = K4_BM * K4_BK * 2;       // 16 KiB of W per stage
constexpr int K4_RING_BYTES = 229376;      // stages of (W tile + X tile)
constexpr int K4_MAX_STAGES = 12;
constexpr int K4_THREADS = 192;
constexpr int K4_SMEM_BYTES = 1024 + K4_RING_BYTES + 512;
constexpr int K4_TMEM_COLS = 128;          // two accumulators of up to 64 columns
constexpr int K4_MAXP = 16;                // ranks supported by the reduce kernel
// The reduce kernels: 1024 threads, VEC 4-channel groups per thread, H <= 4 * 1024 * VEC = 8192.
// Few tokens (T <= 8): one CTA per (rank, token) row; more tokens: one CTA per token, all ranks.
constexpr int K4B_THREADS = 1024;
constexpr int K4B_VEC = 2;
constexpr int K4B_MAX_H = 4 * K4B_THREADS * K4B_VEC;
constexpr int K4T_THREADS = 512;            // the per-token kernel (registers for every rank's sums)
constexpr int K4T_VEC = K4B_MAX_H / (4 * K4T_THREADS);
// The reduce kernels' channel mask covers only the decode path's rows (a small parameter block).
constexpr int K4_MASK_WORDS = K4B_MAX_H / 32;

// A ring for two streaming CTAs per SM (shared memory of both, with their reservations, fits).
constexpr int K4_RING_BYTES_HALF = 112640;

// Ring depth for a padded token count: stages of 16 KiB of W + Tpad x 128 B of X.
__host__ __device__ constexpr int k4_stages(int Tpad, int ring_bytes = K4_RING_BYTES) {
  return (ring_bytes / (K4_A_BYTES + Tpad * 128)) < K4_MAX_STAGES ? (ring_bytes / (K4_A_BYTES + Tpad * 128))
                                                                    : K4_MAX_STAGES;
}

// The streaming kernel's parameters (no channel mask: a small parameter block).
struct DecodeGemmParams {
  float* Zp;                  // [2][P][T][H] fp32 partials (slot 1: second segments of split units)
  int T, Tpad, H, P;
  int n_cb;                   // ceil(H / 128)
  int kblk;                   // ceil(Kp / 64)
  int last_k16;               // 16-wide steps in the last k-block of a rank
  int n_items;                // P * n_cb * kblk
  int stages;                 // ring depth
  int stream_k;               // 1: split the items evenly (units may be cut); 0: whole units
  int ring_bytes;             // shared memory of the ring (the barriers follow it)
  uint64_t timeout_ns;
};

// The reduce kernel's parameters.
struct DecodeParams {
  const float* Zp;            // [2][P][T][H]
  const __nv_bfloat16* R;     // residual [P, T, H]
  __nv_bfloat16* Hout;        // h [P, T, H]
  __nv_bfloat16* Out;         // out [P, T, H]
  const __nv_bfloat16* gamma;
  int T, H, P;
  int n_cb, kblk;
  float private_scale, eps;
  int permuted;               // 1: W's rows are channel-permuted (permuted.cuh): Zp columns are permuted
  int n_s;                    // shared channels (the permuted path's prefix length)
  uint32_t mask_bits[K4_MASK_WORDS];         // bit c = channel c is shared (H <= K4B_MAX_H)
  uint32_t split_bits[K4_MAXP * 64 / 32];  // bit u: unit u = m * n_cb + cb has a second partial
};

// CTA of the streaming kernel that owns item x: the largest i with floor(i N / G) <= x.
__host__ __device__ __forceinline__ int64_t k4_cta_of(int64_t x, int64_t N, int64_t G) {
  return ((x + 1) * G + N - 1) / N - 1;
}

__global__ void __launch_bounds__(K4_THREADS, 1)
    decode_partials_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                           const __grid_constant__ DecodeGemmParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int S = prm.stages;
  const uint32_t b_bytes = static_cast<uint32_t>(prm.Tpad) * K4_BK * 2;
  uint8_t* sA = smem;                               // [S] W tiles (16 KiB, 1024-aligned)
  uint8_t* sB = smem + S * K4_A_BYTES;              // [S] X tiles (Tpad x 128 B, 1024-aligned)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + prm.ring_bytes);
  uint64_t* full = bars;                            // [K4_MAX_STAGES]
  uint64_t* empty = full + K4_MAX_STAGES;           // [K4_MAX_STAGES]
  uint64_t* tfull = empty + K4_MAX_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, K4_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // K4b may be scheduled now: it waits (griddepcontrol.wait) for this grid to complete.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint32_t tmem_base = *tmem_holder;
  const uint64_t tmo = prm.timeout_ns;
  const int64_t N = prm.n_items, G = gridDim.x;
  // stream-K: an even share of the items; otherwise an even share of whole units
  const int64_t U = N / prm.kblk;
  const int item0 = prm.stream_k ? static_cast<int>(static_cast<int64_t>(blockIdx.x) * N / G)
                                 : static_cast<int>(static_cast<int64_t>(blockIdx.x) * U / G) * prm.kblk;
  const int item1 = prm.stream_k ? static_cast<int>((static_cast<int64_t>(blockIdx.x) + 1) * N / G)
                                 : static_cast<int>((static_cast<int64_t>(blockIdx.x) + 1) * U / G) * prm.kblk;
  const int kblk = prm.kblk;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();  // W is streamed once
      const uint64_t pol_x = policy_evict_last();   // X is reused by every unit of its rank
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      for (int it = item0; it < item1; ++it) {
        const int u = it / kblk;
        const int kb = it - u * kblk;
        const int r = u / prm.n_cb;
        const int cb = u - r * prm.n_cb;
        if (!mbar_wait(&empty[stage], phase ^ 1, tmo, 61)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[stage], K4_A_BYTES + b_bytes);
        tma_load_3d(sA + stage * K4_A_BYTES, &tmW, &full[stage], kb * K4_BK, cb * K4_BM, r, pol_w);
        tma_load_3d(sB + stage * b_bytes, &tmX, &full[stage], kb * K4_BK, 0, r, pol_x);
        issued = true;
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
      if (!ok && issued) spin_ns(1000000);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(K4_BM, prm.Tpad);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int seg = item0; seg < item1 && ok;) {
        const int u = seg / kblk;
        const int seg_end = min(item1, (u + 1) * kblk);
        const int buf = local & 1;
        const uint32_t bph = (local >> 1) & 1;
        if (!mbar_wait(&tempty[buf], bph ^ 1, tmo, 62)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dt = tmem_base + static_cast<uint32_t>(buf * K4_MAXN);
        for (int it = seg; it < seg_end; ++it) {
          if (!mbar_wait(&full[stage], phase, tmo, 63)) { ok = false; break; }
          const int kb = it - u * kblk;
          const int nk16 = (kb == kblk - 1) ? prm.last_k16 : (K4_BK / 16);
          const uint32_t a_addr = smem_u32(sA + stage * K4_A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * b_bytes);
          for (int kk = 0; kk < nk16; ++kk)
            umma_bf16(dt, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32), idesc,
                      (it > seg || kk > 0) ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&tfull[buf]);
        ++local;
        seg = seg_end;
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, tmo, 64);
    }
  } else {
    const int q = warp & 3;
    int local = 0;
    for (int seg = item0; seg < item1;) {
      const int u = seg / kblk;
      const int seg_end = min(item1, (u + 1) * kblk);
      const int r = u / prm.n_cb;
      const int cb = u - r * prm.n_cb;
      const int slot = (seg == u * kblk) ? 0 : 1;  // the unit's first or second segment
      const int buf = local & 1;
      const uint32_t bph = (local >> 1) & 1;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&tfull[buf], bph, tmo, 65) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * K4_MAXN);
      uint32_t v[64];
      __syncwarp();
      tmem_ld_32x32b_x32(trow, *reinterpret_cast<uint32_t(*)[32]>(v));
      if (prm.Tpad > 32) tmem_ld_32x32b_x32(trow + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      const int c = cb * K4_BM + q * 32 + lane;
      if (c < prm.H) {
        float* zp = prm.Zp + ((static_cast<size_t>(slot) * prm.P + r) * prm.T) * prm.H + c;
#pragma unroll
        for (int t = 0; t < K4_MAXN; ++t)
          if (t < prm.T) zp[static_cast<size_t>(t) * prm.H] = __uint_as_float(v[t]);
      }
      ++local;
      seg = seg_end;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, K4_TMEM_COLS);
}

// K4b: one CTA per (rank m, token t) row, 4 channels per thread and pass.  All loads a thread
// needs for its 4 channels go out before any is used: the residual, and the fp32 partials of
// every rank (the shared channels' cross-rank sum, in rank order 0..P-1; rank m's own partial
// for the private ones), in batches of 8 ranks; a unit split between two streaming CTAs adds
// its second slot.  The stored h stays in registers for the rescale after the block's
// sum-of-squares reduction.  Launched as a programmatic dependent of K4a: the launch overlaps
// K4a's tail and griddepcontrol.wait orders the reads.
__device__ __forceinline__ bool k4_split(const DecodeParams& prm, int m, int cb) {
  const int u = m * prm.n_cb + cb;
  return (prm.split_bits[u >> 5] >> (u & 31)) & 1u;
}

template <int THREADS, int VEC>
__global__ void __launch_bounds__(THREADS, THREADS >= 1024 ? 1 : 2)
    decode_reduce_norm_kernel(const __grid_constant__ DecodeParams prm) {
  __shared__ float red[THREADS / 32];
  __shared__ float s_rstd;
  const int r = blockIdx.x % prm.P;
  const int t = blockIdx.x / prm.P;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nq = prm.H >> 2;  // 4-channel groups
  const size_t rowoff = (static_cast<size_t>(r) * prm.T + t) * prm.H;
  const size_t zstride = static_cast<size_t>(prm.T) * prm.H;   // between ranks
  const size_t slot1 = static_cast<size_t>(prm.P) * zstride;    // between the two slots
  const float* zrow = prm.Zp + static_cast<size_t>(t) * prm.H;
  __shared__ uint32_t s_mask[K4_MASK_WORDS];
  __shared__ int s_pre[K4_MASK_WORDS + 1];
  if (prm.permuted) mask_prefix(prm.mask_bits, (prm.H + 31) >> 5, s_mask, s_pre);
  asm volatile("griddepcontrol.wait;" ::: "memory");  // K4a's partials are complete and visible

  // the stored h of the thread's groups, in registers (selected by constant indices: the loop
  // over groups itself is not unrolled, which keeps the 1024-thread shape within its registers)
  uint2 hv[VEC];
#pragma unroll
  for (int j = 0; j < VEC; ++j) hv[j] = make_uint2(0u, 0u);
  float ss = 0.f;
#pragma unroll 1
  for (int k = 0; k < VEC; ++k) {
    const int g = threadIdx.x + k * THREADS;
    if (g >= nq) continue;
    const int c = 4 * g;
    const uint32_t bits = (prm.mask_bits[c >> 5] >> (c & 31)) & 0xFu;  // 4 channels, 4-aligned
    const uint2 rv = *reinterpret_cast<const uint2*>(prm.R + rowoff + c);
    float S[4] = {0.f, 0.f, 0.f, 0.f};
    float own[4] = {0.f, 0.f, 0.f, 0.f};
    if (prm.permuted) {
      // channel c + e's partials sit at column pos(c + e) of Zp; one channel at a time
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int pe = perm_pos(c + e, prm.n_s, s_mask, s_pre);
        const bool shared_e = (bits >> e) & 1u;
        const int cbe = pe / K4_BM;
        for (int m0 = 0; m0 < prm.P; m0 += 8) {
          float z[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int m = m0 + j;
            z[j] = 0.f;
            if (m < prm.P && (shared_e || m == r)) {
              z[j] = __ldcg(zrow + m * zstride + pe);
              if (k4_split(prm, m, cbe)) z[j] += __ldcg(zrow + slot1 + m * zstride + pe);
            }
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            S[e] += z[j];
            if (m0 + j == r) own[e] += z[j];
          }
        }
      }
    } else if (bits != 0u) {
      const int cb = c / K4_BM;
      for (int m0 = 0; m0 < prm.P; m0 += 4) {
        const float* zb = zrow + static_cast<size_t>(m0) * zstride + c;
        float4 z[4], w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const bool in = m0 + j < prm.P;
          z[j] = in ? __ldcg(reinterpret_cast<const float4*>(zb + j * zstride)) : make_float4(0.f, 0.f, 0.f, 0.f);
          w[j] = (in && k4_split(prm, m0 + j, cb)) ? __ldcg(reinterpret_cast<const float4*>(zb + slot1 + j * zstride))
                                                   : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          z[j].x += w[j].x; z[j].y += w[j].y; z[j].z += w[j].z; z[j].w += w[j].w;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          S[0] += z[j].x; S[1] += z[j].y; S[2] += z[j].z; S[3] += z[j].w;
          if (m0 + j == r) { own[0] += z[j].x; own[1] += z[j].y; own[2] += z[j].z; own[3] += z[j].w; }
        }
      }
    } else {
      const float* zb = zrow + static_cast<size_t>(r) * zstride + c;
      float4 w = __ldcg(reinterpret_cast<const float4*>(zb));
      if (k4_split(prm, r, c / K4_BM)) {
        const float4 w2 = __ldcg(reinterpret_cast<const float4*>(zb + slot1));
        w.x += w2.x; w.y += w2.y; w.z += w2.z; w.w += w2.w;
      }
      own[0] = w.x; own[1] = w.y; own[2] = w.z; own[3] = w.w;
    }
    const uint32_t rw[2] = {rv.x, rv.y};
    uint32_t o[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float z0 = ((bits >> (2 * e)) & 1u) ? S[2 * e] : prm.private_scale * own[2 * e];
      const float z1 = ((bits >> (2 * e + 1)) & 1u) ? S[2 * e + 1] : prm.private_scale * own[2 * e + 1];
      o[e] = pack_bf16x2(z0 + bf16lo(rw[e]), z1 + bf16hi(rw[e]));
      const float lo = bf16lo(o[e]), hi = bf16hi(o[e]);
      ss = fmaf(lo, lo, ss);
      ss = fmaf(hi, hi, ss);
    }
    const uint2 hk = make_uint2(o[0], o[1]);
#pragma unroll
    for (int j = 0; j < VEC; ++j)
      if (j == k) hv[j] = hk;
    *reinterpret_cast<uint2*>(prm.Hout + rowoff + c) = hk;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, off);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = 0.f;
    for (int w = 0; w < THREADS / 32; ++w) v += red[w];
    s_rstd = rsqrtf(v / static_cast<float>(prm.H) + prm.eps);
  }
  __syncthreads();
  const float rs = s_rstd;
#pragma unroll
  for (int k = 0; k < VEC; ++k) {
    const int g = threadIdx.x + k * THREADS;
    if (g >= nq) continue;
    const uint2 gv = *reinterpret_cast<const uint2*>(prm.gamma + 4 * g);
    uint2 hk = hv[0];
#pragma unroll
    for (int j = 1; j < VEC; ++j)
      if (j == k) hk = hv[j];
    const uint32_t w[2] = {hk.x, hk.y};
    const uint32_t gw[2] = {gv.x, gv.y};
    uint32_t o[2];
#pragma unroll
    for (int e = 0; e < 2; ++e)
      o[e] = pack_bf16x2(bf16lo(w[e]) * rs * bf16lo(gw[e]), bf16hi(w[e]) * rs * bf16hi(gw[e]));
    *reinterpret_cast<uint2*>(prm.Out + rowoff + 4 * g) = make_uint2(o[0], o[1]);
  }
}

// K4b' (T > 8): one CTA per token (512 threads), all ranks, 4 channels per thread and group.  For a
// group, every rank's fp32 partial (a split unit's two slots added) and residual are loaded in one
// round before anything is stored (the loads of later ranks cannot wait behind earlier ranks'
// stores); the shared channels' cross-rank sum is formed once (ranks in order), each rank's h is
// stored (shared: the sum; private: scale x the rank's own partial; plus the residual) and its sum
// of squares accumulated.  The per-rank sums are reduced over the block (warp_sum_many), then
// every rank's h of the group is read back in one round and out written.  The same arithmetic per
// element as K4b.
template <int MAXP>  // P <= MAXP
__global__ void __launch_bounds__(K4T_THREADS, 1)
    decode_reduce_token_kernel(const __grid_constant__ DecodeParams prm) {
  __shared__ float red[MAXP][K4T_THREADS / 32];
  __shared__ float s_rstd[MAXP];
  __shared__ uint32_t s_mask[K4_MASK_WORDS];
  __shared__ int s_pre[K4_MASK_WORDS + 1];
  const int t = blockIdx.x;
  const int P = prm.P;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nq = prm.H >> 2;
  const size_t zstride = static_cast<size_t>(prm.T) * prm.H;    // between ranks
  const size_t slot1 = static_cast<size_t>(P) * zstride;         // between the two slots
  const size_t rstride = static_cast<size_t>(prm.T) * prm.H;     // between ranks of R, h, out
  const float* zrow = prm.Zp + static_cast<size_t>(t) * prm.H;
  const size_t trow = static_cast<size_t>(t) * prm.H;
  if (prm.permuted) mask_prefix(prm.mask_bits, (prm.H + 31) >> 5, s_mask, s_pre);
  asm volatile("griddepcontrol.wait;" ::: "memory");  // K4a's partials are complete and visible

  float ss[MAXP];
#pragma unroll
  for (int m = 0; m < MAXP; ++m) ss[m] = 0.f;
#pragma unroll 1
  for (int k = 0; k < K4T_VEC; ++k) {
    const int g = threadIdx.x + k * K4T_THREADS;
    if (g >= nq) continue;
    const int c = 4 * g;
    const uint32_t bits = (prm.mask_bits[c >> 5] >> (c & 31)) & 0xFu;
    // every rank's partial and residual for these 4 channels, in one round of loads
    float4 z[MAXP];
    uint2 rv[MAXP];
    if (!prm.permuted) {
#pragma unroll
      for (int m = 0; m < MAXP; ++m) {
        z[m] = make_float4(0.f, 0.f, 0.f, 0.f);
        rv[m] = make_uint2(0u, 0u);
        if (m < P) {
          z[m] = __ldcg(reinterpret_cast<const float4*>(zrow + m * zstride + c));
          rv[m] = *reinterpret_cast<const uint2*>(prm.R + m * rstride + trow + c);
        }
      }
#pragma unroll
      for (int m = 0; m < MAXP; ++m) {
        if (m < P && k4_split(prm, m, c / K4_BM)) {
          const float4 w = __ldcg(reinterpret_cast<const float4*>(zrow + slot1 + m * zstride + c));
          z[m].x += w.x; z[m].y += w.y; z[m].z += w.z; z[m].w += w.w;
        }
      }
    } else {
      int col[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) col[e] = perm_pos(c + e, prm.n_s, s_mask, s_pre);
#pragma unroll
      for (int m = 0; m < MAXP; ++m) {
        float zz[4] = {0.f, 0.f, 0.f, 0.f};
        rv[m] = make_uint2(0u, 0u);
        if (m < P) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            zz[e] = __ldcg(zrow + m * zstride + col[e]);
            if (k4_split(prm, m, col[e] / K4_BM)) zz[e] += __ldcg(zrow + slot1 + m * zstride + col[e]);
          }
          rv[m] = *reinterpret_cast<const uint2*>(prm.R + m * rstride + trow + c);
        }
        z[m] = make_float4(zz[0], zz[1], zz[2], zz[3]);
      }
    }
    // the shared sum, once for every rank (ranks in order)
    float S[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < MAXP; ++m) {
      if (m < P) {
        S[0] += z[m].x; S[1] += z[m].y; S[2] += z[m].z; S[3] += z[m].w;
      }
    }
    // every rank's h for these channels
#pragma unroll
    for (int m = 0; m < MAXP; ++m) {
      if (m >= P) break;
      const float own[4] = {z[m].x, z[m].y, z[m].z, z[m].w};
      const uint32_t rw[2] = {rv[m].x, rv[m].y};
      uint32_t o[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float z0 = ((bits >> (2 * e)) & 1u) ? S[2 * e] : prm.private_scale * own[2 * e];
        const float z1 = ((bits >> (2 * e + 1)) & 1u) ? S[2 * e + 1] : prm.private_scale * own[2 * e + 1];
        o[e] = pack_bf16x2(z0 + bf16lo(rw[e]), z1 + bf16hi(rw[e]));
        const float lo = bf16lo(o[e]), hi = bf16hi(o[e]);
        ss[m] = fmaf(lo, lo, ss[m]);
        ss[m] = fmaf(hi, hi, ss[m]);
      }
      *reinterpret_cast<uint2*>(prm.Hout + m * rstride + trow + c) = make_uint2(o[0], o[1]);
    }
  }
  warp_sum_many<MAXP>(ss, lane);
  {
    constexpr int kShift = (MAXP == 32) ? 0 : (MAXP == 16 ? 1 : 2);
    const int idx = lane >> kShift;  // the rank whose warp total this lane holds
    if ((lane & ((1 << kShift) - 1)) == 0 && idx < P) red[idx][warp] = ss[0];
  }
  __syncthreads();
  if (threadIdx.x < P) {
    float v = 0.f;
    for (int w = 0; w < K4T_THREADS / 32; ++w) v += red[threadIdx.x][w];
    s_rstd[threadIdx.x] = rsqrtf(v / static_cast<float>(prm.H) + prm.eps);
  }
  __syncthreads();
  // out = h / rms * gamma: every rank's stored h of a group read back in one round
#pragma unroll 1
  for (int k = 0; k < K4T_VEC; ++k) {
    const int g = threadIdx.x + k * K4T_THREADS;
    if (g >= nq) continue;
    const uint2 gv = *reinterpret_cast<const uint2*>(prm.gamma + 4 * g);
    const uint32_t gw[2] = {gv.x, gv.y};
    uint2 hv[MAXP];
#pragma unroll
    for (int m = 0; m < MAXP; ++m)
      hv[m] = (m < P) ? *reinterpret_cast<const uint2*>(prm.Hout + m * rstride + trow + 4 * g) : make_uint2(0u, 0u);
#pragma unroll
    for (int m = 0; m < MAXP; ++m) {
      if (m >= P) break;
      const float rs = s_rstd[m];
      const uint32_t w[2] = {hv[m].x, hv[m].y};
      uint32_t o[2];
#pragma unroll
      for (int e = 0; e < 2; ++e)
        o[e] = pack_bf16x2(bf16lo(w[e]) * rs * bf16lo(gw[e]), bf16hi(w[e]) * rs * bf16hi(gw[e]));
      *reinterpret_cast<uint2*>(prm.Out + m * rstride + trow + 4 * g) = make_uint2(o[0], o[1]);
    }
  }
}

}  // namespace caat
