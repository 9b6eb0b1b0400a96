// rowpar_gemm2.cuh - the partially synchronized row-parallel GEMM on CTA pairs.
//
// Same computation and work decomposition as rowpar_gemm.cuh ("Tensor-Parallelism with
// Partially Synchronized Activations", App. A.2 Eq. 22 with the §4 residual add), but each
// tile is 256 tokens x 256 channels computed by a pair of CTAs (a 2-CTA cluster on one TPC)
// with tcgen05.mma.cta_group::2:
//   * CTA c of the pair loads X rows [256 m + 128 c, +128) and W rows [256 n + 128 c, +128)
//     (half of A and half of B) into its own shared memory; the leader CTA (c = 0) issues
//     one M=256, N=256, K=16 MMA that reads both halves and leaves in each CTA's TMEM the
//     128 x 256 accumulator of that CTA's tokens.  Per SM this halves the W bytes each k
//     block costs, so a 32 KiB stage holds the same MMA work a 48 KiB stage did, and 6
//     stages fit in shared memory.
//   * Both CTAs' TMA loads signal the leader's full barrier (cta_group::2 form, no
//     multicast); the leader's MMA commits arrive on both CTAs' empty / TMEM-full barriers
//     (multicast commit); both CTAs' epilogues release the accumulator on the leader's
//     TMEM-empty barrier.
//   * Dynamic scheduling: the leader's producer draws a unit from the global counter and
//     writes it into both CTAs' broadcast ring.
//   * Wide shared units (zs_mode 3, forward only): two adjacent whole shared column blocks as one
//     256 x 512 unit.  Per k-block one ring stage holds X and the first block's W half, the
//     next only the second block's W half; the MMA issuer runs both N = 256 halves on the same
//     X stage, into the two TMEM buffers, so the unit counts as two tiles for the buffers'
//     phases.  The epilogue stores each half's fp32 sums and releases its buffer in turn.
// The RMSNorm is fused (rowpar_common.cuh): warps 6-9 of each CTA normalize completed row
// blocks.
// kMajor (GEMM-only use by the backward): bit 0 = A stored MN-major ([K][M], M contiguous),
// bit 1 = B stored MN-major ([K][N]).  Such an operand half is loaded as two 64-wide boxes of
// 64 K rows and read through MN-major descriptors, so the gradient GEMMs need no transposes.
// kMajor = 0 is the forward kernel.  Every wait is bounded; on expiry the device status word is set, all roles leave their
// loops, copies in flight are given time to land, and both CTAs meet at a final cluster
// barrier before TMEM is freed.
#pragma once

#include "ptx.cuh"
#include "rowpar_common.cuh"

namespace caat {

constexpr int K2P_BM = 128;                     // rows per CTA (pair tile: 256)
constexpr int K2P_BN = 256;                     // channels per pair tile (per CTA B half: 128)
constexpr int K2P_BK = 64;
constexpr int K2P_A_BYTES = K2P_BM * K2P_BK * 2;        // 16 KiB
constexpr int K2P_B_BYTES = (K2P_BN / 2) * K2P_BK * 2;  // 16 KiB
constexpr int K2P_STAGE_BYTES = K2P_A_BYTES + K2P_B_BYTES;
// Two shared-memory splits of the same size: 6 operand stages + 2 epilogue boxes per epilogue
// warp (the default), or 5 stages + 4 boxes for workloads whose units are short in K (few k-blocks
// per tile), where the epilogue's residual loads and h stores, not the operands, set the pace.
constexpr int K2P_STAGES = 6;
constexpr int K2P_STAGES_EPI = 5;
constexpr int K2P_EPI_NBUF_EPI = 4;
__host__ __device__ constexpr int k2p_smem_bytes(int stages, int nbuf) {
  return 1024 + stages * K2P_STAGE_BYTES + 4 * nbuf * K1_EPI_BOX_BYTES + 512;
}
constexpr int K2P_SMEM_BYTES = k2p_smem_bytes(K2P_STAGES, K1_EPI_NBUF);
static_assert(k2p_smem_bytes(K2P_STAGES_EPI, K2P_EPI_NBUF_EPI) <= K2P_SMEM_BYTES, "both splits fit the same size");
constexpr uint64_t K2P_DRAIN_NS = 1000000;      // error path only: let copies in flight land

template <bool kFused, int kMajor = 0, int kStages = K2P_STAGES, int kEpiBuf = K1_EPI_NBUF>
__global__ void __launch_bounds__(K1Threads<kFused>::value, 1)
    rowpar_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                            const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmH,
                            const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ RowparParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * K2P_A_BYTES;
  uint8_t* sEpi = smem + kStages * K2P_STAGE_BYTES;  // [4 warps][kEpiBuf] boxes
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + (4 * kEpiBuf * K1_EPI_BOX_BYTES));
  uint64_t* full = bars;                    // [STAGES]  used in the leader
  uint64_t* empty = full + kStages;      // [STAGES]  both CTAs (multicast commit)
  uint64_t* tfull = empty + kStages;     // [2]       both CTAs (multicast commit)
  uint64_t* tempty = tfull + 2;             // [2]       leader: 4 local + 4 peer warps
  uint64_t* sfull = tempty + 2;             // [SCHED]   both CTAs (leader producer arrives)
  uint64_t* sempty = sfull + K1_SCHED;      // [SCHED]   leader: 5 local + 5 peer arrivals
  uint64_t* mma_done = sempty + K1_SCHED;   // [1]       leader
  uint64_t* sig = mma_done + 1;                   // [4] epilogue warps meet per tile
  uint64_t* rbar = sig + 4;                        // [4 warps][kEpiBuf]
  int* sched_unit = reinterpret_cast<int*>(rbar + 4 * kEpiBuf);  // [SCHED] both CTAs
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sched_unit + K1_SCHED);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t cta = cluster_ctarank();   // 0 = leader, 1 = peer
  const bool leader = cta == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * K1Threads<kFused>::epi_warps);
    }
    for (int s = 0; s < K1_SCHED; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 2 * (1 + K1Threads<kFused>::epi_warps));
    }
    mbar_init(mma_done, 1);
    for (int b = 0; b < 4; ++b) mbar_init(&sig[b], K1Threads<kFused>::epi_warps);
    for (int b = 0; b < 4 * kEpiBuf; ++b) mbar_init(&rbar[b], 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmR);
    tma_prefetch_desc(&tmH);
    if (prm.zs_mode == 1 || prm.zs_mode == 3) tma_prefetch_desc(&tmZ);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, K1_TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialized, TMEM allocated, before any remote access
  tc_fence_after();
  // A row-norm kernel launched as a programmatic dependent may start now, on the SMs this
  // grid leaves free: it waits on the row-block job list, never on this grid's completion.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint32_t tmem_base = *tmem_holder;
  const uint64_t tmo = prm.timeout_ns;
  const uint32_t peer = cta ^ 1u;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producers
    if (lane == 0) {
      const uint64_t pol_x = policy_evict_last();
      const uint64_t pol_w = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      for (int i = 0; ok; ++i) {
        const int slot = i % K1_SCHED;
        const uint32_t sph = (i / K1_SCHED) & 1;
        int u;
        if (leader) {
          if (!mbar_wait_cluster(&sempty[slot], sph ^ 1, tmo, 21)) { ok = false; break; }
          u = static_cast<int>(atomicAdd(prm.counter, 1u));
          sched_unit[slot] = u;
          st_shared_cluster_u32(mapa_shared(smem_u32(&sched_unit[slot]), peer), static_cast<uint32_t>(u));
          mbar_arrive(&sfull[slot]);
          mbar_arrive_cluster(mapa_shared(smem_u32(&sfull[slot]), peer));
        } else {
          if (!mbar_wait_cluster(&sfull[slot], sph, tmo, 22)) { ok = false; break; }
          u = sched_unit[slot];
          mbar_arrive_cluster(mapa_shared(smem_u32(&sempty[slot]), 0));
        }
        if (u >= prm.n_units) break;
        const K1Unit un = k1_decode(u, prm);
        const int r0 = un.rank < 0 ? 0 : un.rank;
        const int r1 = un.rank < 0 ? prm.P : un.rank + 1;
        const int xrow = prm.t_begin + un.m * (2 * K2P_BM) + static_cast<int>(cta) * K2P_BM;
        const int wrow = un.n * K2P_BN + static_cast<int>(cta) * (K2P_BN / 2);
        if constexpr (kMajor == 0) {
          if (un.wide) {
            // 256 x 512: per k-block one stage with X and the first block's W half, one with
            // the second block's W half only
            for (int r = r0; r < r1 && ok; ++r) {
              for (int kb = 0; kb < prm.kblk_per_rank; ++kb) {
                if (!mbar_wait(&empty[stage], phase ^ 1, tmo, 23)) { ok = false; break; }
                uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
                if (leader) mbar_arrive_expect_tx(&full[stage], 2 * K2P_STAGE_BYTES);
                tma_load_3d_pair(sA + stage * K2P_A_BYTES, &tmX, fbar, kb * K2P_BK, xrow, r, pol_x);
                tma_load_3d_pair(sB + stage * K2P_B_BYTES, &tmW, fbar, kb * K2P_BK, wrow, r, pol_w);
                issued = true;
                if (++stage == kStages) { stage = 0; phase ^= 1; }
                if (!mbar_wait(&empty[stage], phase ^ 1, tmo, 23)) { ok = false; break; }
                fbar = mapa_shared(smem_u32(&full[stage]), 0);
                if (leader) mbar_arrive_expect_tx(&full[stage], 2 * K2P_B_BYTES);
                tma_load_3d_pair(sB + stage * K2P_B_BYTES, &tmW, fbar, kb * K2P_BK, wrow + K2P_BN, r, pol_w);
                if (++stage == kStages) { stage = 0; phase ^= 1; }
              }
            }
            continue;
          }
        }
        for (int r = r0; r < r1 && ok; ++r) {
          for (int kb = 0; kb < prm.kblk_per_rank; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1, tmo, 23)) { ok = false; break; }
            const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * K2P_STAGE_BYTES);
            if constexpr ((kMajor & 1) != 0) {
              tma_load_3d_pair(sA + stage * K2P_A_BYTES, &tmX, fbar, xrow, kb * K2P_BK, r, pol_x);
              tma_load_3d_pair(sA + stage * K2P_A_BYTES + K2P_A_BYTES / 2, &tmX, fbar, xrow + 64, kb * K2P_BK, r,
                               pol_x);
            } else {
              tma_load_3d_pair(sA + stage * K2P_A_BYTES, &tmX, fbar, kb * K2P_BK, xrow, r, pol_x);
            }
            if constexpr ((kMajor & 2) != 0) {
              tma_load_3d_pair(sB + stage * K2P_B_BYTES, &tmW, fbar, wrow, kb * K2P_BK, r, pol_w);
              tma_load_3d_pair(sB + stage * K2P_B_BYTES + K2P_B_BYTES / 2, &tmW, fbar, wrow + 64, kb * K2P_BK, r,
                               pol_w);
            } else {
              tma_load_3d_pair(sB + stage * K2P_B_BYTES, &tmW, fbar, kb * K2P_BK, wrow, r, pol_w);
            }
            issued = true;
            if (++stage == kStages) { stage = 0; phase ^= 1; }
          }
        }
      }
      if (!ok && issued) spin_ns(K2P_DRAIN_NS);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader)
    if (leader && lane == 0) {
      const uint32_t idesc = idesc_bf16_f32_major(2 * K2P_BM, K2P_BN, (kMajor & 1) != 0, (kMajor & 2) != 0);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int slot = i % K1_SCHED;
        const uint32_t sph = (i / K1_SCHED) & 1;
        if (!mbar_wait(&sfull[slot], sph, tmo, 24)) { ok = false; break; }
        const int u = sched_unit[slot];
        mbar_arrive(&sempty[slot]);
        if (u >= prm.n_units) break;
        const K1Unit un = k1_decode(u, prm);
        if constexpr (kMajor == 0) {
          if (un.wide) {
            // both accumulators: the first block's columns in buffer local & 1, the second's in
            // the other (the buffers of tiles local and local + 1)
            const int b0 = local & 1;
            const uint32_t ph0 = (local >> 1) & 1, ph1 = ((local + 1) >> 1) & 1;
            if (!mbar_wait_cluster(&tempty[b0], ph0 ^ 1, tmo, 25)) { ok = false; break; }
            if (!mbar_wait_cluster(&tempty[b0 ^ 1], ph1 ^ 1, tmo, 25)) { ok = false; break; }
            tc_fence_after();
            const uint32_t dt0 = tmem_base + static_cast<uint32_t>(b0 * K2P_BN);
            const uint32_t dt1 = tmem_base + static_cast<uint32_t>((b0 ^ 1) * K2P_BN);
            const int nkb = prm.P * prm.kblk_per_rank;
            int kb_in_rank = 0;
            for (int j = 0; j < nkb; ++j) {
              const int sa = stage;  // X and the first block's W half
              if (!mbar_wait(&full[stage], phase, tmo, 26)) { ok = false; break; }
              if (++stage == kStages) { stage = 0; phase ^= 1; }
              const int sb = stage;  // the second block's W half
              if (!mbar_wait(&full[stage], phase, tmo, 26)) { ok = false; break; }
              if (++stage == kStages) { stage = 0; phase ^= 1; }
              const int nk16 = (kb_in_rank == prm.kblk_per_rank - 1) ? prm.last_k16 : (K2P_BK / 16);
              const uint32_t a_addr = smem_u32(sA + sa * K2P_A_BYTES);
              const uint32_t b0_addr = smem_u32(sB + sa * K2P_B_BYTES);
              const uint32_t b1_addr = smem_u32(sB + sb * K2P_B_BYTES);
              for (int kk = 0; kk < nk16; ++kk)
                umma_bf16_pair(dt0, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b0_addr + kk * 32), idesc,
                               (j > 0 || kk > 0) ? 1u : 0u);
              for (int kk = 0; kk < nk16; ++kk)
                umma_bf16_pair(dt1, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b1_addr + kk * 32), idesc,
                               (j > 0 || kk > 0) ? 1u : 0u);
              umma_commit_pair_mc(&empty[sa], 0x3);
              umma_commit_pair_mc(&empty[sb], 0x3);
              if (++kb_in_rank == prm.kblk_per_rank) kb_in_rank = 0;
            }
            if (!ok) break;
            if (!(prm.flags & K1_FLAG_TEST_STALL)) {
              umma_commit_pair_mc(&tfull[b0], 0x3);
              umma_commit_pair_mc(&tfull[b0 ^ 1], 0x3);
            }
            local += 2;
            continue;
          }
        }
        const int buf = local & 1;
        const uint32_t bph = (local >> 1) & 1;
        if (!mbar_wait_cluster(&tempty[buf], bph ^ 1, tmo, 25)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dt = tmem_base + static_cast<uint32_t>(buf * K2P_BN);
        const int nkb = (un.rank < 0 ? prm.P : 1) * prm.kblk_per_rank;
        int kb_in_rank = 0;
        for (int j = 0; j < nkb; ++j) {
          if (!mbar_wait(&full[stage], phase, tmo, 26)) { ok = false; break; }
          const int nk16 = (kb_in_rank == prm.kblk_per_rank - 1) ? prm.last_k16 : (K2P_BK / 16);
          const uint32_t a_addr = smem_u32(sA + stage * K2P_A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * K2P_B_BYTES);
          for (int kk = 0; kk < nk16; ++kk) {
            const uint64_t ad = (kMajor & 1) ? sw128_mnmajor_desc(a_addr + kk * 2048) : sw128_kmajor_desc(a_addr + kk * 32);
            const uint64_t bd = (kMajor & 2) ? sw128_mnmajor_desc(b_addr + kk * 2048) : sw128_kmajor_desc(b_addr + kk * 32);
            umma_bf16_pair(dt, ad, bd, idesc, (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
          if (++kb_in_rank == prm.kblk_per_rank) kb_in_rank = 0;
        }
        if (!ok) break;
        if (!(prm.flags & K1_FLAG_TEST_STALL)) umma_commit_pair_mc(&tfull[buf], 0x3);
        ++local;
      }
      umma_commit_pair(mma_done);
      mbar_wait(mma_done, 0, tmo, 27);
    }
  } else if (kFused && warp >= K1_NORM_WARP0) {
    // ---------------------------------------------------------------- normalizer warps
    if constexpr (kFused) k1_normalizer(prm, lane);
  } else {
    // ---------------------------------------------------------------- epilogue warps
    const int q = warp & 3;
    uint8_t* my_bufs = sEpi + (warp - 2) * kEpiBuf * K1_EPI_BOX_BYTES;
    uint64_t* my_rbar = rbar + (warp - 2) * kEpiBuf;
    uint32_t rphase = 0;
    const uint64_t pol_r = policy_evict_first();
    // h is read back soon by the norm (fused, or the row-norm kernel beside this one), maybe
    // still from L2; otherwise streamed out, behind X and W
    const uint64_t pol_h = prm.publish ? policy_evict_normal() : policy_evict_first();
    const uint32_t tempty_leader[2] = {mapa_shared(smem_u32(&tempty[0]), 0), mapa_shared(smem_u32(&tempty[1]), 0)};
    int local = 0;
    int pend_m128 = -1, pend_rank = 0;  // publish mode 2: the tile still to be counted
    for (int i = 0;; ++i) {
      const int slot = i % K1_SCHED;
      const uint32_t sph = (i / K1_SCHED) & 1;
      int u = 0;
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait_cluster(&sfull[slot], sph, tmo, 28) ? 1 : 0;
        if (ok) {
          u = sched_unit[slot];
          if (leader) mbar_arrive(&sempty[slot]);
          else mbar_arrive_cluster(mapa_shared(smem_u32(&sempty[slot]), 0));
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      u = __shfl_sync(0xFFFFFFFFu, u, 0);
      if (!ok || u >= prm.n_units) break;
      const K1Unit un = k1_decode(u, prm);
      if (un.wide) {
        // shared-sum mode, 256 x 512: the two column blocks' accumulators in turn, each released
        // as soon as it is stored (the next unit's first block may start in it)
        const int row0 = prm.t_begin + un.m * (2 * K2P_BM) + static_cast<int>(cta) * K2P_BM + q * 32;
        for (int hh = 0; hh < 2 && ok; ++hh) {
          const int bh = (local + hh) & 1;
          if (lane == 0) ok = mbar_wait(&tfull[bh], ((local + hh) >> 1) & 1, tmo, 29) ? 1 : 0;
          ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
          if (!ok) break;
          tc_fence_after();
          const uint32_t trow = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(bh * K2P_BN);
          k1_epilogue_zs(trow, prm, &tmZ, row0, (un.n + hh) * K2P_BN, my_bufs, lane, pol_h);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(tempty_leader[bh]);
        }
        if (!ok) break;
        local += 2;
        continue;
      }
      const int buf = local & 1;
      const uint32_t bph = (local >> 1) & 1;
      if (lane == 0) ok = mbar_wait(&tfull[buf], bph, tmo, 29) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      if (pend_m128 >= 0) {  // the previous tile's stores have had this tile's mainloop to land
        k1_publish_counts(prm, pend_m128, pend_rank);
        pend_m128 = -1;
      }
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * K2P_BN);
      const int row = prm.t_begin + un.m * (2 * K2P_BM) + static_cast<int>(cta) * K2P_BM + q * 32 + lane;
      const int n0 = un.n * K2P_BN;
      const bool mixed = prm.ncls[un.n] == 2;
      const bool merge = mixed && !kFused && prm.merge_mixed;
      if (prm.zs_mode == 3) {
        const int row0 = prm.t_begin + un.m * (2 * K2P_BM) + static_cast<int>(cta) * K2P_BM + q * 32;
        if (un.rank < 0) {
          k1_epilogue_zs(trow, prm, &tmZ, row0, n0, my_bufs, lane, pol_h);
        } else if (!k1_epilogue_tma<kEpiBuf>(trow, prm, &tmR, &tmH, row0, n0, un.rank, un.slot, my_bufs, my_rbar,
                                             rphase, lane, pol_r, pol_h, false)) {
          break;  // private: full h boxes (a mixed block's shared columns are rewritten from Zs)
        }
      } else if (prm.zs_mode) {
        const int row0 = prm.t_begin + un.m * (2 * K2P_BM) + static_cast<int>(cta) * K2P_BM + q * 32;
        if (!k1_epilogue_split(trow, prm, &tmR, &tmH, &tmZ, row0, n0, un.rank, my_bufs, my_rbar, rphase, lane,
                               pol_r, pol_h))
          break;
      } else if (!mixed || merge) {
        const int row0 = prm.t_begin + un.m * (2 * K2P_BM) + static_cast<int>(cta) * K2P_BM + q * 32;
        // flag of this warp's 32 rows in column block n: [row group][n-block]
        unsigned int* flag =
            merge ? prm.sdone + (static_cast<size_t>((row0 - prm.t_begin) >> 5) * ((prm.H + K2P_BN - 1) / K2P_BN) +
                                 un.n)
                  : nullptr;
        if (merge && un.rank >= 0 && !k1_wait_sdone(prm, flag)) break;
        if (!k1_epilogue_tma<kEpiBuf>(trow, prm, &tmR, &tmH, row0, n0, un.rank, un.slot, my_bufs, my_rbar, rphase, lane,
                             pol_r, pol_h, merge && un.rank >= 0))
          break;
        if (merge && un.rank < 0) k1_signal_sdone(flag);
      } else if (un.rank < 0) {
        k1_epilogue_shared(trow, prm, row, n0, un.slot, mixed, 0, 8);
      } else {
        k1_epilogue_private(trow, prm, row, un.rank, n0, un.slot, mixed, 0, 2);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader[buf]);
      if (prm.publish == 2) {
        pend_m128 = 2 * un.m + static_cast<int>(cta);
        pend_rank = un.rank;
      } else {
        k1_signal_tile(prm, sig, local, 2 * un.m + static_cast<int>(cta), un.rank);
      }
      ++local;
    }
    if (pend_m128 >= 0) k1_publish_counts(prm, pend_m128, pend_rank);
    if (prm.zs_mode == 2) fence_sc_sys();  // this warp's pushes to other GPUs, before the signal
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the other may still touch its shared memory
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, K1_TMEM_COLS);
  // peer-memory exchange: the launch's last CTA tells every owner that this rank's partials are in
  if (prm.zs_mode == 2 && threadIdx.x == 0)
    tp_signal_done(prm.tp_done, gridDim.x, prm.tp_flags, prm.tp_world, 0, prm.tp_rank, prm.tp_epoch);
}

}  // namespace caat
