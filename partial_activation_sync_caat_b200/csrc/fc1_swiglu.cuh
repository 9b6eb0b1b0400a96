// fc1_swiglu.cuh - column-parallel FC1 with SwiGLU of the CAAT-Net MLP block, per rank.
//
// "Tensor-Parallelism with Partially Synchronized Activations" §3.1 Eq. 6: with partial
// channel-reduce every rank m has its own input X_m, and Y_m = sigma(X_m A_m) with A split
// by columns (Eq. 2).  sigma is SwiGLU here: rank m's A_m holds F/P gate rows followed by
// F/P up rows (nn.Linear orientation, H contiguous), and
//     Y_m[t, j] = silu(X_m[t,:] . A_m[j,:]) * (X_m[t,:] . A_m[F/P + j,:]),
// silu(x) = x / (1 + exp(-x)), fp32 accumulation, Y rounded to bf16 (it feeds the
// partially synchronized FC2 of rowpar_gemm*.cuh).
//
// CTA-pair tcgen05 kernel (same pipeline as rowpar_gemm2.cuh): a tile is 256 tokens x 128
// output features of one rank.  The leader CTA loads the 128 gate rows and the peer CTA the
// 128 matching up rows as the two halves of the MMA's B operand, so one M=256, N=256 MMA
// leaves in each CTA's TMEM its 128 tokens x [gate | up] (256 columns).  The epilogue
// computes silu(gate) * up for 128 columns and stores bf16 Y boxes with TMA.  A is viewed
// by TMA as a 4-D tensor (H, F/P, {gate, up}, P) so the last, partial feature block never
// reads the other half's rows (out-of-range rows are zero-filled, stores are clipped).
#pragma once

#include "ptx.cuh"
#include "rowpar_common.cuh"

namespace caat {

constexpr int K3_BM = 128;                      // tokens per CTA (pair tile: 256)
constexpr int K3_BN = 128;                      // output features per tile
constexpr int K3_BK = 64;
constexpr int K3_STAGES = 6;
constexpr int K3_A_BYTES = K3_BM * K3_BK * 2;   // 16 KiB of X
constexpr int K3_B_BYTES = K3_BN * K3_BK * 2;   // 16 KiB: gate rows (leader) or up rows (peer)
constexpr int K3_STAGE_BYTES = K3_A_BYTES + K3_B_BYTES;
constexpr int K3_THREADS = 192;                 // producer, MMA, 4 epilogue warps
constexpr int K3_SMEM_BYTES = 1024 + K3_STAGES * K3_STAGE_BYTES + K1_EPI_BYTES + 512;
constexpr uint64_t K3_DRAIN_NS = 1000000;       // error path only: let copies in flight land

struct Fc1Params {
  unsigned int* counter;   // dynamic unit counter, zero at launch
  int T, H, Fp, P;
  int n_mblk;              // ceil(T / 256)
  int n_nblk;              // ceil(Fp / 128)
  int kblk;                // ceil(H / 64)
  int last_k16;            // 16-wide K steps in the last k-block (1..4)
  int n_units;             // P * n_mblk * n_nblk, rank-major
  uint64_t timeout_ns;
  uint32_t flags;
};

__device__ __forceinline__ void tma_load_4d_pair(void* smem_dst, const void* map, uint32_t mbar_cluster_addr, int c0,
                                                 int c1, int c2, int c3, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar_cluster_addr), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(policy)
      : "memory");
}

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + __expf(-x)); }

__global__ void __launch_bounds__(K3_THREADS, 1)
    fc1_swiglu_pair_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmY, const __grid_constant__ Fc1Params prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + K3_STAGES * K3_A_BYTES;
  uint8_t* sEpi = smem + K3_STAGES * K3_STAGE_BYTES;  // [4 warps][K1_EPI_NBUF] boxes
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + K1_EPI_BYTES);
  uint64_t* full = bars;                   // [STAGES] leader
  uint64_t* empty = full + K3_STAGES;      // [STAGES] both CTAs (multicast commit)
  uint64_t* tfull = empty + K3_STAGES;     // [2] both CTAs (multicast commit)
  uint64_t* tempty = tfull + 2;            // [2] leader: 4 local + 4 peer epilogue warps
  uint64_t* sfull = tempty + 2;            // [SCHED] both CTAs
  uint64_t* sempty = sfull + K1_SCHED;     // [SCHED] leader: 5 local + 5 peer arrivals
  uint64_t* mma_done = sempty + K1_SCHED;  // [1] leader
  int* sched_unit = reinterpret_cast<int*>(mma_done + 1);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sched_unit + K1_SCHED);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t cta = cluster_ctarank();
  const bool leader = cta == 0;
  const uint32_t peer = cta ^ 1u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < K3_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);
    }
    for (int s = 0; s < K1_SCHED; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 10);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, K1_TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint64_t tmo = prm.timeout_ns;
  const int per_rank = prm.n_mblk * prm.n_nblk;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producers
    if (lane == 0) {
      const uint64_t pol_x = policy_evict_normal();
      const uint64_t pol_a = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      for (int i = 0; ok; ++i) {
        const int slot = i % K1_SCHED;
        const uint32_t sph = (i / K1_SCHED) & 1;
        int u;
        if (leader) {
          if (!mbar_wait_cluster(&sempty[slot], sph ^ 1, tmo, 41)) { ok = false; break; }
          u = static_cast<int>(atomicAdd(prm.counter, 1u));
          sched_unit[slot] = u;
          st_shared_cluster_u32(mapa_shared(smem_u32(&sched_unit[slot]), peer), static_cast<uint32_t>(u));
          mbar_arrive(&sfull[slot]);
          mbar_arrive_cluster(mapa_shared(smem_u32(&sfull[slot]), peer));
        } else {
          if (!mbar_wait_cluster(&sfull[slot], sph, tmo, 42)) { ok = false; break; }
          u = sched_unit[slot];
          mbar_arrive_cluster(mapa_shared(smem_u32(&sempty[slot]), 0));
        }
        if (u >= prm.n_units) break;
        const int r = u / per_rank;
        const int rem = u - r * per_rank;
        const int m = rem / prm.n_nblk;
        const int n = rem - m * prm.n_nblk;
        const int xrow = m * (2 * K3_BM) + static_cast<int>(cta) * K3_BM;
        for (int kb = 0; kb < prm.kblk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, tmo, 43)) { ok = false; break; }
          const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * K3_STAGE_BYTES);
          tma_load_3d_pair(sA + stage * K3_A_BYTES, &tmX, fbar, kb * K3_BK, xrow, r, pol_x);
          // leader: gate rows, peer: up rows of features [128 n, 128 n + 128)
          tma_load_4d_pair(sB + stage * K3_B_BYTES, &tmA, fbar, kb * K3_BK, n * K3_BN, static_cast<int>(cta), r,
                           pol_a);
          issued = true;
          if (++stage == K3_STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok && issued) spin_ns(K3_DRAIN_NS);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader)
    if (leader && lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(2 * K3_BM, 2 * K3_BN);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int slot = i % K1_SCHED;
        const uint32_t sph = (i / K1_SCHED) & 1;
        if (!mbar_wait(&sfull[slot], sph, tmo, 44)) { ok = false; break; }
        const int u = sched_unit[slot];
        mbar_arrive(&sempty[slot]);
        if (u >= prm.n_units) break;
        const int buf = local & 1;
        const uint32_t bph = (local >> 1) & 1;
        if (!mbar_wait_cluster(&tempty[buf], bph ^ 1, tmo, 45)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dt = tmem_base + static_cast<uint32_t>(buf * 2 * K3_BN);
        for (int j = 0; j < prm.kblk; ++j) {
          if (!mbar_wait(&full[stage], phase, tmo, 46)) { ok = false; break; }
          const int nk16 = (j == prm.kblk - 1) ? prm.last_k16 : (K3_BK / 16);
          const uint32_t a_addr = smem_u32(sA + stage * K3_A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * K3_B_BYTES);
          for (int kk = 0; kk < nk16; ++kk)
            umma_bf16_pair(dt, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32), idesc,
                           (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == K3_STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (!(prm.flags & K1_FLAG_TEST_STALL)) umma_commit_pair_mc(&tfull[buf], 0x3);
        ++local;
      }
      umma_commit_pair(mma_done);
      mbar_wait(mma_done, 0, tmo, 47);
    }
  } else {
    // ---------------------------------------------------------------- epilogue warps
    const int q = warp & 3;
    uint8_t* my_bufs = sEpi + (warp - 2) * K1_EPI_NBUF * K1_EPI_BOX_BYTES;
    const uint32_t tempty_leader[2] = {mapa_shared(smem_u32(&tempty[0]), 0), mapa_shared(smem_u32(&tempty[1]), 0)};
    int local = 0;
    for (int i = 0;; ++i) {
      const int slot = i % K1_SCHED;
      const uint32_t sph = (i / K1_SCHED) & 1;
      int u = 0;
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait_cluster(&sfull[slot], sph, tmo, 48) ? 1 : 0;
        if (ok) {
          u = sched_unit[slot];
          if (leader) mbar_arrive(&sempty[slot]);
          else mbar_arrive_cluster(mapa_shared(smem_u32(&sempty[slot]), 0));
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      u = __shfl_sync(0xFFFFFFFFu, u, 0);
      if (!ok || u >= prm.n_units) break;
      const int r = u / per_rank;
      const int rem = u - r * per_rank;
      const int m = rem / prm.n_nblk;
      const int n = rem - m * prm.n_nblk;
      const int buf = local & 1;
      const uint32_t bph = (local >> 1) & 1;
      if (lane == 0) ok = mbar_wait(&tfull[buf], bph, tmo, 49) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t trow =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * 2 * K3_BN);
      const int row0 = m * (2 * K3_BM) + static_cast<int>(cta) * K3_BM + q * 32;
      for (int c = 0; c < 2; ++c) {
        const int f0 = n * K3_BN + 64 * c;
        if (f0 >= prm.Fp) break;  // warp-uniform
        uint32_t g[64], v[64];
        __syncwarp();
        tmem_ld_32x32b_x32(trow + 64 * c, *reinterpret_cast<uint32_t(*)[32]>(g));
        tmem_ld_32x32b_x32(trow + 64 * c + 32, *reinterpret_cast<uint32_t(*)[32]>(g + 32));
        tmem_ld_32x32b_x32(trow + K3_BN + 64 * c, *reinterpret_cast<uint32_t(*)[32]>(v));
        tmem_ld_32x32b_x32(trow + K3_BN + 64 * c + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
        tmem_wait_ld();
        uint8_t* rowp = my_bufs + c * K1_EPI_BOX_BYTES + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float y0 = silu_f(__uint_as_float(g[8 * j + 2 * e])) * __uint_as_float(v[8 * j + 2 * e]);
            const float y1 = silu_f(__uint_as_float(g[8 * j + 2 * e + 1])) * __uint_as_float(v[8 * j + 2 * e + 1]);
            o[e] = pack_bf16x2(y0, y1);
          }
          *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tmY, my_bufs + c * K1_EPI_BOX_BYTES, f0, row0, r);
          bulk_commit_group();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_cluster(tempty_leader[buf]);
        bulk_wait_group_read0();  // the boxes are reused by the next tile
      }
      __syncwarp();
      ++local;
    }
    if (lane == 0) bulk_wait_group0();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, K1_TMEM_COLS);
}

}  // namespace caat
