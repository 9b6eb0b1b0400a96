// rowpar_gemm.cuh - the partially synchronized row-parallel GEMM with its fused epilogue.
//
// Computes, for P ranks emulated in one GPU ("logical devices", "Tensor-Parallelism with
// Partially Synchronized Activations" §3.2), the partial products Zt_m = X_m W_m^T
// (App. A.2 Eq. 22, first line), the partial channel-reduce (Eq. 22, second line: shared
// channels get sum_m Zt_m, private ones keep Zt_m times the §4 private scale) and the
// residual add h_m = Z_m + R_m (§4 Eq. 9), writing h in bf16.  The RMSNorm that follows
// is a separate row kernel (rownorm.cuh).
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
// Kernel structure (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: fetches units from a global atomic counter (dynamic
//               scheduling), streams X and W k-blocks (64 wide, 128-byte swizzle) into a
//               4-stage shared-memory ring.
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer (M=128, N=256, K=16),
//               accumulating into one of two 256-column TMEM buffers (double-buffered so
//               the epilogue of one unit overlaps the mainloop of the next).
//   warps 2-5   epilogue: residual loads issued ahead (a whole row segment, or one chunk for
//               up to 8 ranks), tcgen05.ld 32 lanes x 32 columns, residual add, bf16 stores.
// Every wait is bounded (about 1 s): on expiry the device status word is set and all
// roles leave their loops; in-flight TMA loads and MMAs are waited for before exit.
#pragma once

#include "ptx.cuh"

namespace caat {

constexpr int K1_BM = 128;
constexpr int K1_BN = 256;
constexpr int K1_BK = 64;
constexpr int K1_STAGES = 4;
constexpr int K1_THREADS = 192;
constexpr int K1_A_BYTES = K1_BM * K1_BK * 2;   // 16 KiB
constexpr int K1_B_BYTES = K1_BN * K1_BK * 2;   // 32 KiB
constexpr int K1_SCHED = 4;                      // depth of the unit broadcast ring
constexpr int K1_MAX_NBLK = 65536 / K1_BN;       // n-blocks at the largest supported H
constexpr int K1_MASK_WORDS = 65536 / 32;
constexpr int K1_TMEM_COLS = 512;                // two 256-column fp32 accumulators
constexpr int K1_SMEM_BYTES = 1024 /*alignment slack*/ + K1_STAGES * (K1_A_BYTES + K1_B_BYTES) + 512;

enum : uint32_t { K1_FLAG_TEST_STALL = 0x100u };

struct RowparParams {
  const __nv_bfloat16* R;      // residual [P, T, H]
  __nv_bfloat16* Hout;         // pre-norm h [P, T, H]
  unsigned int* counter;       // dynamic unit counter, zero at launch
  int T, H, Kp, P;
  int n_mblk;                  // ceil(T / 128)
  int kblk_per_rank;           // ceil(Kp / 64)
  int last_k16;                // 16-wide K steps in the last k-block of a rank (1..4)
  int nS, nPriv;               // n-blocks that have a shared unit / private units
  int n_units;
  float private_scale;
  uint64_t timeout_ns;
  uint32_t flags;
  uint16_t slist[K1_MAX_NBLK];
  uint16_t plist[K1_MAX_NBLK];
  uint8_t ncls[K1_MAX_NBLK];   // 0 all-private, 1 all-shared, 2 mixed
  uint32_t mask_bits[K1_MASK_WORDS];  // bit c = channel c is shared
};

struct K1Unit {
  int m, n, rank;   // rank < 0: shared unit
};

__device__ __forceinline__ K1Unit k1_decode(int u, const RowparParams& prm) {
  K1Unit un;
  const int n_shared_units = prm.n_mblk * prm.nS;
  if (u < n_shared_units) {
    un.m = u / prm.nS;
    un.n = prm.slist[u % prm.nS];
    un.rank = -1;
  } else {
    // private units: rank-major, then m-block, then n-block (n fastest), so that units
    // running concurrently share rank r's W slice and X m-blocks in L2.
    const int w = u - n_shared_units;
    const int per_rank = prm.n_mblk * prm.nPriv;
    un.rank = w / per_rank;
    const int rem = w - un.rank * per_rank;
    un.m = rem / prm.nPriv;
    un.n = prm.plist[rem - un.m * prm.nPriv];
  }
  return un;
}

// Converts 8 accumulator values (+ residual) to bf16 and stores them for one 16-byte piece.
// want: bit e set = column e of the piece is written (mixed column blocks), 0xFF = all.
__device__ __forceinline__ void k1_store_piece(__nv_bfloat16* dst, const uint32_t* v8, uint4 r, float scale,
                                               uint32_t want) {
  const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
  uint32_t o[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float a0 = __uint_as_float(v8[2 * e]) * scale + bf16lo(rw[e]);
    const float a1 = __uint_as_float(v8[2 * e + 1]) * scale + bf16hi(rw[e]);
    o[e] = pack_bf16x2(a0, a1);
  }
  if (want == 0xFFu) {
    st_v4(dst, make_uint4(o[0], o[1], o[2], o[3]));
  } else if (want != 0u) {
    unsigned short* d16 = reinterpret_cast<unsigned short*>(dst);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (want & (1u << e)) d16[e] = static_cast<unsigned short>((o[e >> 1] >> (16 * (e & 1))) & 0xFFFFu);
  }
}

// Epilogue of a private unit (one rank): 32 rows (one per lane) x up to 256 columns.  All 32
// residual pieces of the row segment are loaded up front (memory-level parallelism), then
// the accumulator is read from TMEM 32 columns at a time.
__device__ __forceinline__ void k1_epilogue_private(uint32_t trow, const RowparParams& prm, int row, int rank,
                                                    int n0, bool mixed) {
  const bool row_ok = row < prm.T;
  const size_t rowoff = (static_cast<size_t>(rank) * prm.T + (row_ok ? row : 0)) * prm.H;
  const __nv_bfloat16* Rp = prm.R + rowoff + n0;
  __nv_bfloat16* Op = prm.Hout + rowoff + n0;
  const int ncols = min(K1_BN, prm.H - n0);
  uint4 rv[K1_BN / 8];
#pragma unroll
  for (int j = 0; j < K1_BN / 8; ++j) {
    rv[j] = make_uint4(0, 0, 0, 0);
    if (row_ok && 8 * j < ncols) rv[j] = ld_nc_v4(Rp + 8 * j);
  }
  const float scale = prm.private_scale;
#pragma unroll
  for (int c = 0; c < K1_BN / 32; ++c) {
    if (32 * c >= ncols) break;  // warp-uniform
    uint32_t v[32];
    __syncwarp();
    tmem_ld_32x32b_x32(trow + 32 * c, v);
    tmem_wait_ld();
    const uint32_t want = mixed ? ~prm.mask_bits[(n0 + 32 * c) >> 5] : 0xFFFFFFFFu;
    if (row_ok) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (32 * c + 8 * k < ncols)
          k1_store_piece(Op + 32 * c + 8 * k, v + 8 * k, rv[4 * c + k], scale, (want >> (8 * k)) & 0xFFu);
    }
  }
}

// Epilogue of a shared unit: the one accumulator (the cross-rank sum) serves every rank.  Per
// 32-column chunk: one TMEM read, then the residual pieces of up to 8 ranks loaded together,
// then one store per rank.
__device__ __forceinline__ void k1_epilogue_shared(uint32_t trow, const RowparParams& prm, int row, int n0,
                                                   bool mixed) {
  constexpr int RG = 8;  // ranks per residual group
  const bool row_ok = row < prm.T;
  const size_t rstride = static_cast<size_t>(prm.T) * prm.H;
  const size_t base = static_cast<size_t>(row_ok ? row : 0) * prm.H + n0;
  const int ncols = min(K1_BN, prm.H - n0);
#pragma unroll 1
  for (int c = 0; c < K1_BN / 32; ++c) {
    if (32 * c >= ncols) break;  // warp-uniform
    uint32_t v[32];
    __syncwarp();
    tmem_ld_32x32b_x32(trow + 32 * c, v);
    const uint32_t want = mixed ? prm.mask_bits[(n0 + 32 * c) >> 5] : 0xFFFFFFFFu;
#pragma unroll 1
    for (int r0 = 0; r0 < prm.P; r0 += RG) {
      uint4 rv[RG][4];
#pragma unroll
      for (int rr = 0; rr < RG; ++rr)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          rv[rr][k] = make_uint4(0, 0, 0, 0);
          if (row_ok && r0 + rr < prm.P && 32 * c + 8 * k < ncols)
            rv[rr][k] = ld_nc_v4(prm.R + (r0 + rr) * rstride + base + 32 * c + 8 * k);
        }
      if (r0 == 0) tmem_wait_ld();
      if (row_ok) {
#pragma unroll
        for (int rr = 0; rr < RG; ++rr) {
          if (r0 + rr >= prm.P) break;
          __nv_bfloat16* Op = prm.Hout + (r0 + rr) * rstride + base + 32 * c;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (32 * c + 8 * k < ncols) k1_store_piece(Op + 8 * k, v + 8 * k, rv[rr][k], 1.0f, (want >> (8 * k)) & 0xFFu);
        }
      }
    }
  }
}

__global__ void __launch_bounds__(K1_THREADS, 1)
    rowpar_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ RowparParams prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = smem + K1_STAGES * K1_A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K1_STAGES * (K1_A_BYTES + K1_B_BYTES));
  uint64_t* full = bars;                         // [K1_STAGES]
  uint64_t* empty = full + K1_STAGES;            // [K1_STAGES]
  uint64_t* tfull = empty + K1_STAGES;           // [2]
  uint64_t* tempty = tfull + 2;                  // [2]
  uint64_t* sfull = tempty + 2;                  // [K1_SCHED]
  uint64_t* sempty = sfull + K1_SCHED;           // [K1_SCHED]
  uint64_t* mma_done = sempty + K1_SCHED;        // [1]
  int* sched_unit = reinterpret_cast<int*>(mma_done + 1);   // [K1_SCHED]
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
      mbar_init(&tempty[b], 4);
    }
    for (int s = 0; s < K1_SCHED; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 5);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
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
            tma_load_3d(sA + stage * K1_A_BYTES, &tmX, &full[stage], kb * K1_BK, un.m * K1_BM, r, pol_x);
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
          tc_fence_after();
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
  } else {
    // ---------------------------------------------------------------- epilogue warps
    const int q = warp & 3;  // TMEM lane quarter this warp may access
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
      const int row = un.m * K1_BM + q * 32 + lane;
      const int n0 = un.n * K1_BN;
      const bool mixed = prm.ncls[un.n] == 2;
      if (un.rank < 0) {
        k1_epilogue_shared(trow, prm, row, n0, mixed);
      } else {
        k1_epilogue_private(trow, prm, row, un.rank, n0, mixed);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      ++local;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, K1_TMEM_COLS);
}

}  // namespace caat
