// rowpar_gemm.cuh - the partially synchronized row-parallel GEMM with its fused epilogue.
//
// Computes, for P ranks emulated in one GPU ("logical devices", "Tensor-Parallelism with
// Partially Synchronized Activations" §3.2), the partial products Zt_m = X_m W_m^T
// (App. A.2 Eq. 22, first line), the partial channel-reduce (Eq. 22, second line: shared
// channels get sum_m Zt_m, private ones keep Zt_m times the §4 private scale) and the
// residual add h_m = Z_m + R_m (§4 Eq. 9), writing h in bf16, and the RMSNorm that follows
// (fused; see rowpar_common.cuh).  This is the single-CTA variant (128-token tiles) used for
// small token counts; rowpar_gemm2.cuh has the CTA-pair variant.
//
// Work decomposition.  Output tiles are 128 tokens x 256 channels.  Each n-block (256
// channels) is classified on the host as all-shared, all-private or mixed:
//   * shared unit (m, n): one accumulation over the concatenated K of all P ranks, so the
//     cross-rank sum of Eq. 22 rides on the tensor-core accumulation in fp32; the epilogue
//     then makes P passes over the same TMEM accumulator, one per rank's residual.
//   * private unit (m, n, r): one accumulation over rank r's K/P slice, one epilogue pass.
//   * a mixed n-block gets both: the shared unit writes only its shared channels, the
//     private units only their private channels (element-masked stores).
//
// Kernel structure (one persistent CTA per SM, 320 threads):
//   warp 0      TMA producer: fetches units from a global atomic counter (dynamic
//               scheduling), streams X and W k-blocks (64 wide, 128-byte swizzle) into a
//               4-stage shared-memory ring.
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer (M=128, N=256, K=16),
//               accumulating into one of two 256-column TMEM buffers (double-buffered so
//               the epilogue of one unit overlaps the mainloop of the next).
//   warps 2-5   epilogue: residual loads issued ahead, tcgen05.ld 32 lanes x 32 columns,
//               residual add, bf16 stores, per-row sum-of-squares partials, row-block counts.
//   warps 6-9   normalizers (fused RMSNorm of completed row blocks).
// Every wait is bounded (about 1 s): on expiry the device status word is set and all
// roles leave their loops; in-flight TMA loads and MMAs are waited for before exit.
#pragma once

#include "rowpar_common.cuh"

namespace caat {

constexpr int K1_BM = 128;
constexpr int K1_BN = 256;
constexpr int K1_BK = 64;
constexpr int K1_STAGES = 4;
constexpr int K1_A_BYTES = K1_BM * K1_BK * 2;   // 16 KiB
constexpr int K1_B_BYTES = K1_BN * K1_BK * 2;   // 32 KiB
constexpr int K1_SMEM_BYTES = 1024 /*alignment slack*/ + K1_STAGES * (K1_A_BYTES + K1_B_BYTES) + K1_EPI_BYTES + 512;

template <bool kFused>
__global__ void __launch_bounds__(K1Threads<kFused>::value, 1)
    rowpar_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                            const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmH,
                       const __grid_constant__ RowparParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + K1_STAGES * K1_A_BYTES;
  uint8_t* sEpi = smem + K1_STAGES * (K1_A_BYTES + K1_B_BYTES);  // [4 warps][K1_EPI_NBUF] boxes
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + K1_EPI_BYTES);
  uint64_t* full = bars;                         // [K1_STAGES]
  uint64_t* empty = full + K1_STAGES;            // [K1_STAGES]
  uint64_t* tfull = empty + K1_STAGES;           // [2]
  uint64_t* tempty = tfull + 2;                  // [2]
  uint64_t* sfull = tempty + 2;                  // [K1_SCHED]
  uint64_t* sempty = sfull + K1_SCHED;           // [K1_SCHED]
  uint64_t* mma_done = sempty + K1_SCHED;        // [1]
  uint64_t* sig = mma_done + 1;                   // [4] epilogue warps meet per tile
  uint64_t* rbar = sig + 4;                        // [4 warps][K1_EPI_NBUF]
  int* sched_unit = reinterpret_cast<int*>(rbar + 4 * K1_EPI_NBUF);   // [K1_SCHED]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sched_unit + K1_SCHED);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < K1_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 1 * K1Threads<kFused>::epi_warps);
    }
    for (int s = 0; s < K1_SCHED; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 1 + K1Threads<kFused>::epi_warps);
    }
    mbar_init(mma_done, 1);
    for (int b = 0; b < 4; ++b) mbar_init(&sig[b], K1Threads<kFused>::epi_warps);
    for (int b = 0; b < 4 * K1_EPI_NBUF; ++b) mbar_init(&rbar[b], 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmR);
    tma_prefetch_desc(&tmH);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, K1_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint64_t tmo = prm.timeout_ns;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const uint64_t pol_x = policy_evict_normal();
      const uint64_t pol_w = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, last_parity = 0;  // for the drain on abort
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int slot = i % K1_SCHED;
        const uint32_t sph = (i / K1_SCHED) & 1;
        if (!mbar_wait(&sempty[slot], sph ^ 1, tmo, 1)) { ok = false; break; }
        const int u = static_cast<int>(atomicAdd(prm.counter, 1u));
        sched_unit[slot] = u;
        mbar_arrive(&sfull[slot]);
        if (u >= prm.n_units) break;
        const K1Unit un = k1_decode(u, prm);
        const int r0 = un.rank < 0 ? 0 : un.rank;
        const int r1 = un.rank < 0 ? prm.P : un.rank + 1;
        for (int r = r0; r < r1 && ok; ++r) {
          for (int kb = 0; kb < prm.kblk_per_rank; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1, tmo, 2)) { ok = false; break; }
            mbar_arrive_expect_tx(&full[stage], K1_A_BYTES + K1_B_BYTES);
            tma_load_3d(sA + stage * K1_A_BYTES, &tmX, &full[stage], kb * K1_BK, prm.t_begin + un.m * K1_BM, r, pol_x);
            tma_load_3d(sB + stage * K1_B_BYTES, &tmW, &full[stage], kb * K1_BK, un.n * K1_BN, r, pol_w);
            issued_mask |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == K1_STAGES) { stage = 0; phase ^= 1; }
          }
        }
      }
      if (!ok) {
        // Drain: every TMA load issued must land before the CTA may exit.
        for (int s = 0; s < K1_STAGES; ++s)
          if (issued_mask & (1u << s)) mbar_wait(&full[s], (last_parity >> s) & 1u, tmo, 3);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(K1_BM, K1_BN);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int slot = i % K1_SCHED;
        const uint32_t sph = (i / K1_SCHED) & 1;
        if (!mbar_wait(&sfull[slot], sph, tmo, 4)) { ok = false; break; }
        const int u = sched_unit[slot];
        mbar_arrive(&sempty[slot]);
        if (u >= prm.n_units) break;
        const K1Unit un = k1_decode(u, prm);
        const int buf = local & 1;
        const uint32_t bph = (local >> 1) & 1;
        if (!mbar_wait(&tempty[buf], bph ^ 1, tmo, 5)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dt = tmem_base + static_cast<uint32_t>(buf * K1_BN);
        const int nkb = (un.rank < 0 ? prm.P : 1) * prm.kblk_per_rank;
        int kb_in_rank = 0;
        for (int j = 0; j < nkb; ++j) {
          if (!mbar_wait(&full[stage], phase, tmo, 6)) { ok = false; break; }
          const int nk16 = (kb_in_rank == prm.kblk_per_rank - 1) ? prm.last_k16 : (K1_BK / 16);
          const uint32_t a_addr = smem_u32(sA + stage * K1_A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * K1_B_BYTES);
          for (int kk = 0; kk < nk16; ++kk) {
            umma_bf16(dt, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32), idesc,
                      (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == K1_STAGES) { stage = 0; phase ^= 1; }
          if (++kb_in_rank == prm.kblk_per_rank) kb_in_rank = 0;
        }
        if (!ok) break;
        if (!(prm.flags & K1_FLAG_TEST_STALL)) umma_commit(&tfull[buf]);
        ++local;
      }
      // All issued MMAs must complete before TMEM is released.
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, tmo, 7);
    }
  } else if (kFused && warp >= K1_NORM_WARP0) {
    // ---------------------------------------------------------------- normalizer warps
    if constexpr (kFused) k1_normalizer(prm, lane);
  } else {
    // ---------------------------------------------------------------- epilogue warps
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint8_t* my_bufs = sEpi + (warp - 2) * K1_EPI_NBUF * K1_EPI_BOX_BYTES;
    uint64_t* my_rbar = rbar + (warp - 2) * K1_EPI_NBUF;
    uint32_t rphase = 0;
    const uint64_t pol_r = policy_evict_first();
    const uint64_t pol_h = kFused ? policy_evict_normal() : policy_evict_first();
    int local = 0;
    for (int i = 0;; ++i) {
      const int slot = i % K1_SCHED;
      const uint32_t sph = (i / K1_SCHED) & 1;
      int u = 0;
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait(&sfull[slot], sph, tmo, 8) ? 1 : 0;
        if (ok) {
          u = sched_unit[slot];
          mbar_arrive(&sempty[slot]);
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      u = __shfl_sync(0xFFFFFFFFu, u, 0);
      if (!ok || u >= prm.n_units) break;
      const K1Unit un = k1_decode(u, prm);
      const int buf = local & 1;
      const uint32_t bph = (local >> 1) & 1;
      if (lane == 0) ok = mbar_wait(&tfull[buf], bph, tmo, 9) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * K1_BN);
      const int row = prm.t_begin + un.m * K1_BM + q * 32 + lane;
      const int n0 = un.n * K1_BN;
      const bool mixed = prm.ncls[un.n] == 2;
      if (!mixed) {
        const int row0 = prm.t_begin + un.m * K1_BM + q * 32;
        if (!k1_epilogue_tma(trow, prm, &tmR, &tmH, row0, n0, un.rank, un.slot, my_bufs, my_rbar, rphase, lane,
                             pol_r, pol_h))
          break;
      } else if (un.rank < 0) {
        k1_epilogue_shared(trow, prm, row, n0, un.slot, mixed, 0, 8);
      } else {
        k1_epilogue_private(trow, prm, row, un.rank, n0, un.slot, mixed, 0, 2);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      k1_signal_tile(prm, sig, local, un.m, un.rank);
      ++local;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, K1_TMEM_COLS);
}

}  // namespace caat
