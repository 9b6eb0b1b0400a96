// rowpar_common.cuh - pieces shared by the two GEMM kernels of the partially synchronized
// row-parallel layer (rowpar_gemm.cuh: one CTA per tile; rowpar_gemm2.cuh: CTA pairs):
// parameters, work-unit decoding, the fused epilogue (partial channel-reduce, private scale,
// residual add, bf16 stores, per-row sum-of-squares partials) and the fused RMSNorm.
//
// "Tensor-Parallelism with Partially Synchronized Activations": App. A.2 Eq. 22 (partial
// channel-reduce), §4 Eq. 14-15 (private-channel scale), §4 Eq. 9 (residual add, then Norm;
// RMSNorm here, gamma shared by the ranks).
//
// Fused RMSNorm.  RMSNorm needs a complete row (all H channels) of one rank, which spans
// ceil(H/256) tiles computed by different CTAs.  Each tile epilogue therefore also writes
// the sum of squares of its (bf16) h values per row into a partial slot, and counts the
// tile into its (128-token row block, rank) counter.  The CTA that completes a row block
// publishes it to a global job list (in completion order).  Dedicated normalizer warps in
// every CTA claim 8-row pieces of published row blocks in order, sum the partial slots of
// each row, and rescale the row: out = h / sqrt(sum/H + eps) * gamma.  Row blocks are
// normalized while their h is still in L2, and the last blocks are spread over all SMs.
#pragma once

#include "ptx.cuh"
#include "tp.cuh"

namespace caat {

constexpr int K1_SCHED = 4;                      // depth of the unit broadcast ring
constexpr int K1_MAX_NBLK = 65536 / 256;         // 256-channel blocks at the largest H
constexpr int K1_MASK_WORDS = 65536 / 32;
constexpr int K1_TMEM_COLS = 512;                // two 256-column fp32 accumulators
// Warps per CTA: producer, MMA, 4 epilogue warps (one per TMEM lane quarter), then (fused
// RMSNorm only) 4 normalizer warps.
template <bool kFused>
struct K1Threads {
  static constexpr int epi_warps = 4;
  static constexpr int value = 32 * (2 + epi_warps + (kFused ? 4 : 0));
};

// TMA epilogue of pure column blocks: per epilogue warp, K1_EPI_NBUF shared-memory buffers of
// one 32-row x 64-column bf16 box (128-byte rows, 128-byte swizzle).
constexpr int K1_EPI_NBUF = 2;
constexpr int K1_EPI_BOX_BYTES = 32 * 64 * 2;
constexpr int K1_EPI_BYTES = 4 * K1_EPI_NBUF * K1_EPI_BOX_BYTES;  // per CTA
constexpr int K1_NORM_WARP0 = 6;                 // first normalizer warp (fused RMSNorm)
constexpr int K1_ROWS_PER_JOB = 128;             // rows of a row block
constexpr int K1_ROWS_PER_PIECE = 8;             // rows a normalizer warp claims at a time
constexpr int K1_PIECES_PER_JOB = K1_ROWS_PER_JOB / K1_ROWS_PER_PIECE;

enum : uint32_t { K1_FLAG_TEST_STALL = 0x100u };

struct RowparParams {
  const __nv_bfloat16* R;      // residual [P, T, H]
  __nv_bfloat16* Hout;         // pre-norm h [P, T, H] (== Out when no h_out is requested)
  __nv_bfloat16* Out;          // normalized output [P, T, H]
  const __nv_bfloat16* gamma;  // [H]
  unsigned int* counter;       // dynamic unit counter, zero at launch
  unsigned int* piece_claim;   // normalizer piece counter, zero at launch
  unsigned int* job_pub;       // published row blocks, zero at launch
  unsigned int* rb_count;      // [n_rb] tiles done per (row block, rank), zero at launch
  unsigned int* job_slots;     // [n_rb] published row-block ids + 1, zero at launch
  float* ss_part;              // [P][T_pad][nslots] per-row sum-of-squares partials
  unsigned int* sdone;         // [T_pad/32][n-blocks] shared unit of a mixed block stored, zero at launch
  int merge_mixed;             // 1: mixed blocks use the TMA epilogue (see k1_epilogue_tma)
  int no_residual;             // 1: store Z (no residual add) -- channel-permuted path, see rownorm.cuh
  int zs_mode;                 // 1: split output of one rank of a multi-device layer (tp.cuh):
                               // channels c < zs_ns go to Zs as the fp32 partial, the others to h;
                               // 2: the same, the partials pushed to their owners' receive buffers;
                               // 3: one device, P ranks: a shared unit stores its accumulator (the
                               // cross-rank sum) as fp32 to Zs [T, zs_ns] once, the norm kernel
                               // adds the residual; private units store h as usual
  int zs_ns;                   // shared channels (zs_mode)
  // zs_mode 2 (peer-memory exchange, tp.cuh): owner q's receive buffer [world][T][tp_w] as this
  // process maps it, every rank's flag array [2][world], the launch's done-CTA counter (zero at
  // launch), and this call's epoch
  float* tp_recv[TP_MAX_WORLD];
  unsigned int* tp_flags[TP_MAX_WORLD];
  unsigned int* tp_done;
  int tp_world, tp_rank, tp_w;
  uint32_t tp_epoch;
  int T, H, Kp, P;             // T: token rows of the tensors (the row stride of rank blocks)
  int t_begin, t_end;          // token rows this launch processes: [t_begin, t_end)
  int n_mblk;                  // row blocks of the kernel's tile height over [t_begin, t_end)
  int kblk_per_rank;           // ceil(Kp / 64)
  int last_k16;                // 16-wide K steps in the last k-block of a rank (1..4)
  int nS, nPriv;               // n-blocks that have a shared unit / private units
  int wide;                    // unit order 0, shared-sum mode: the first 2 * wide shared blocks
                               // (pure, adjacent) run as `wide` 256 x 512 units per row block
  int n_units;
  int fuse_norm;               // 1: normalizer warps produce `Out`; 0: h only
  int publish;                 // 1 (fused norm): count each tile into its (128-row block, rank)
                               // counter and publish completed row blocks to the job list;
                               // 2 (row-norm kernel beside this one): each epilogue warp adds 1 to
                               // the counters of its tile's (128-row block, rank)s once the tile's
                               // stores are complete (checked when the warp's next tile starts)
  int order;                   // unit order: 0 shared units first, then private rank-major;
                               // 1 row-block-major (each row block's units together);
                               // 2 grouped: order 0 within groups of group_m row blocks;
                               // 3 staggered: row block s's shared units, then row block
                               //   (s - group_m)'s private units, for s = 0, 1, ...
  int group_m;                 // row blocks per group (order 2) / stagger distance (order 3)
  int n_rb;                    // (128-row block, rank) pairs = n_m128 * P
  int T_pad;                   // n_m128 * 128
  int nslots;                  // nS + nPriv partial slots per row
  float private_scale;
  float eps;
  uint64_t timeout_ns;
  uint32_t flags;
  uint16_t slist[K1_MAX_NBLK];
  uint16_t plist[K1_MAX_NBLK];
  uint8_t ncls[K1_MAX_NBLK];   // 0 all-private, 1 all-shared, 2 mixed
  uint32_t mask_bits[K1_MASK_WORDS];  // bit c = channel c is shared
};

struct K1Unit {
  int m, n, rank;   // rank < 0: shared unit
  int slot;         // partial slot of this unit's contribution to each row
  int wide;         // 1: shared unit of the column blocks n and n + 1 (a 256 x 512 tile)
};

__device__ __forceinline__ K1Unit k1_decode(int u, const RowparParams& prm) {
  K1Unit un;
  un.wide = 0;
  if (prm.order == 3) {
    // Staggered: step s holds the shared units of row block s (if s < n_mblk), then the
    // private units of row block s - D (rank-major, n fastest).  Row blocks complete at an even
    // rate over the whole kernel (a row block is complete with its private units), and every
    // step mixes long shared and short private units.  D >= 0 keeps each mixed block's shared
    // unit ahead of its private units.
    const int D = min(prm.group_m, prm.n_mblk);
    const int np = prm.P * prm.nPriv;
    const int per = prm.nS + np;
    const int head = D * prm.nS;
    const int n_mid = prm.n_mblk - D;
    int m, v;  // v < 0: shared unit -v - 1; v >= 0: private unit v
    if (u < head) {
      m = u / prm.nS;
      v = -(u - m * prm.nS) - 1;
    } else if (u - head < n_mid * per) {
      const int s = (u - head) / per;
      const int w = (u - head) - s * per;
      if (w < prm.nS) {
        m = D + s;
        v = -w - 1;
      } else {
        m = s;
        v = w - prm.nS;
      }
    } else {
      const int w = u - head - n_mid * per;
      m = n_mid + w / np;
      v = w - (m - n_mid) * np;
    }
    un.m = m;
    if (v < 0) {
      un.slot = -v - 1;
      un.n = prm.slist[un.slot];
      un.rank = -1;
    } else {
      un.rank = v / prm.nPriv;
      const int pi = v - un.rank * prm.nPriv;
      un.n = prm.plist[pi];
      un.slot = prm.nS + pi;
    }
    return un;
  }
  if (prm.order == 2) {
    // Grouped: for each group of group_m row blocks, its shared units (row block major),
    // then its private units rank by rank.  Row blocks of a group complete together, while
    // the next group's tiles are being computed.
    const int G = prm.group_m;
    const int per_m = prm.nS + prm.P * prm.nPriv;
    const int full_groups = prm.n_mblk / G;
    int g = u / (G * per_m);
    if (g > full_groups) g = full_groups;
    const int gm = g < full_groups ? G : prm.n_mblk - full_groups * G;
    const int v = u - g * G * per_m;
    if (v < prm.nS * gm) {
      const int mi = v / prm.nS;
      un.m = g * G + mi;
      un.slot = v - mi * prm.nS;
      un.n = prm.slist[un.slot];
      un.rank = -1;
    } else {
      const int w = v - prm.nS * gm;
      un.rank = w / (gm * prm.nPriv);
      const int rem = w - un.rank * gm * prm.nPriv;
      const int mi = rem / prm.nPriv;
      un.m = g * G + mi;
      const int pi = rem - mi * prm.nPriv;
      un.n = prm.plist[pi];
      un.slot = prm.nS + pi;
    }
    return un;
  }
  if (prm.order == 1) {
    // Row-block-major: the nS shared units of row block m, then its private units rank by
    // rank, then row block m + 1.  A row block's h is complete soon after it is written, so
    // the fused norm finds it in L2.
    const int per_m = prm.nS + prm.P * prm.nPriv;
    un.m = u / per_m;
    const int v = u - un.m * per_m;
    if (v < prm.nS) {
      un.slot = v;
      un.n = prm.slist[v];
      un.rank = -1;
    } else {
      const int w = v - prm.nS;
      un.rank = w / prm.nPriv;
      const int pi = w - un.rank * prm.nPriv;
      un.n = prm.plist[pi];
      un.slot = prm.nS + pi;
    }
    return un;
  }
  // shared units: every row block's wide units first (two blocks each), then the remaining
  // ordinary shared units of every row block (short ones last), then the private units
  const int nSu = prm.nS - prm.wide;   // shared units per row block
  const int nSo = nSu - prm.wide;      // ordinary ones among them
  const int n_wide_units = prm.n_mblk * prm.wide;
  const int n_shared_units = prm.n_mblk * nSu;
  if (u < n_wide_units) {
    un.m = u / prm.wide;
    un.slot = 2 * (u - un.m * prm.wide);
    un.wide = 1;
    un.n = prm.slist[un.slot];
    un.rank = -1;
  } else if (u < n_shared_units) {
    const int v = u - n_wide_units;
    un.m = v / nSo;
    un.slot = 2 * prm.wide + (v - un.m * nSo);
    un.n = prm.slist[un.slot];
    un.rank = -1;
  } else {
    // private units: rank-major, then m-block, then n-block (n fastest), so that units
    // running concurrently share rank r's W slice and X m-blocks in L2.
    const int w = u - n_shared_units;
    const int per_rank = prm.n_mblk * prm.nPriv;
    un.rank = w / per_rank;
    const int rem = w - un.rank * per_rank;
    un.m = rem / prm.nPriv;
    const int pi = rem - un.m * prm.nPriv;
    un.n = prm.plist[pi];
    un.slot = prm.nS + pi;
  }
  return un;
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const unsigned int* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu(unsigned int* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint4 ld_cg_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float ld_cg_f32(const float* p) {
  float v;
  asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

// Converts 8 accumulator values (+ residual) to bf16 and stores them as one 16-byte piece.
// want: bit e set = column e of the piece is written (mixed column blocks), 0xFF = all.
// Returns the sum of squares of the bf16 values written.
__device__ __forceinline__ float k1_store_piece(__nv_bfloat16* dst, const uint32_t* v8, uint4 r, float scale,
                                                uint32_t want) {
  const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
  uint32_t o[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float a0 = __uint_as_float(v8[2 * e]) * scale + bf16lo(rw[e]);
    const float a1 = __uint_as_float(v8[2 * e + 1]) * scale + bf16hi(rw[e]);
    o[e] = pack_bf16x2(a0, a1);
  }
  float ss = 0.f;
  if (want == 0xFFu) {
    st_v4(dst, make_uint4(o[0], o[1], o[2], o[3]));
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = bf16lo(o[e]), hi = bf16hi(o[e]);
      ss = fmaf(lo, lo, ss);
      ss = fmaf(hi, hi, ss);
    }
  } else if (want != 0u) {
    unsigned short* d16 = reinterpret_cast<unsigned short*>(dst);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if (want & (1u << e)) {
        const uint32_t bits = (o[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
        d16[e] = static_cast<unsigned short>(bits);
        const float x = __uint_as_float(bits << 16);
        ss = fmaf(x, x, ss);
      }
    }
  }
  return ss;
}

__device__ __forceinline__ void k1_put_partial(const RowparParams& prm, int rank, int row, int slot, float ss) {
  if (prm.fuse_norm) prm.ss_part[(static_cast<size_t>(rank) * prm.T_pad + row) * prm.nslots + slot] = ss;
}

// Epilogue of a private unit (one rank): 32 rows (one per lane) x the 128-column halves
// [h0, h1) of the tile, each half's 16 residual pieces loaded up front.
__device__ __forceinline__ void k1_epilogue_private(uint32_t trow, const RowparParams& prm, int row, int rank,
                                                    int n0, int slot, bool mixed, int h0, int h1) {
  const bool row_ok = row < prm.t_end;
  const size_t rowoff = (static_cast<size_t>(rank) * prm.T + (row_ok ? row : 0)) * prm.H;
  const __nv_bfloat16* Rp = prm.R + rowoff + n0;
  __nv_bfloat16* Op = prm.Hout + rowoff + n0;
  const int ncols = min(256, prm.H - n0);
  const float scale = prm.private_scale;
  float ss = 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    if (half < h0 || half >= h1) continue;
    const int cb = 128 * half;
    if (cb >= ncols) break;  // warp-uniform
    uint4 rv[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      rv[j] = make_uint4(0, 0, 0, 0);
      if (row_ok && !prm.no_residual && cb + 8 * j < ncols) rv[j] = ld_nc_v4(Rp + cb + 8 * j);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int cc = cb + 32 * c;
      if (cc >= ncols) break;  // warp-uniform
      uint32_t v[32];
      __syncwarp();
      tmem_ld_32x32b_x32(trow + cc, v);
      tmem_wait_ld();
      const uint32_t want = mixed ? ~prm.mask_bits[(n0 + cc) >> 5] : 0xFFFFFFFFu;
      if (row_ok) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (cc + 8 * k < ncols)
            ss += k1_store_piece(Op + cc + 8 * k, v + 8 * k, rv[4 * c + k], scale, (want >> (8 * k)) & 0xFFu);
      }
    }
  }
  if (row_ok) k1_put_partial(prm, rank, row, slot, ss);
}

// Epilogue of a shared unit: the one accumulator (the cross-rank sum) serves every rank.
// Ranks are taken 4 at a time; per 32-column chunk (chunks [c0, c1) of the tile) one TMEM
// read, the residual pieces of the 4 ranks loaded together, then one store per rank.
__device__ __forceinline__ void k1_epilogue_shared(uint32_t trow, const RowparParams& prm, int row, int n0,
                                                   int slot, bool mixed, int c0, int c1) {
  constexpr int RG = 4;
  const bool row_ok = row < prm.t_end;
  const size_t rstride = static_cast<size_t>(prm.T) * prm.H;
  const size_t base = static_cast<size_t>(row_ok ? row : 0) * prm.H + n0;
  const int ncols = min(256, prm.H - n0);
#pragma unroll 1
  for (int r0 = 0; r0 < prm.P; r0 += RG) {
    float ss[RG];
#pragma unroll
    for (int rr = 0; rr < RG; ++rr) ss[rr] = 0.f;
#pragma unroll 1
    for (int c = c0; c < c1; ++c) {
      const int cc = 32 * c;
      if (cc >= ncols) break;  // warp-uniform
      uint32_t v[32];
      __syncwarp();
      tmem_ld_32x32b_x32(trow + cc, v);
      const uint32_t want = mixed ? prm.mask_bits[(n0 + cc) >> 5] : 0xFFFFFFFFu;
      uint4 rv[RG][4];
#pragma unroll
      for (int rr = 0; rr < RG; ++rr)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          rv[rr][k] = make_uint4(0, 0, 0, 0);
          if (row_ok && !prm.no_residual && r0 + rr < prm.P && cc + 8 * k < ncols)
            rv[rr][k] = ld_nc_v4(prm.R + (r0 + rr) * rstride + base + cc + 8 * k);
        }
      tmem_wait_ld();
      if (row_ok) {
#pragma unroll
        for (int rr = 0; rr < RG; ++rr) {
          if (r0 + rr >= prm.P) break;
          __nv_bfloat16* Op = prm.Hout + (r0 + rr) * rstride + base + cc;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (cc + 8 * k < ncols)
              ss[rr] += k1_store_piece(Op + 8 * k, v + 8 * k, rv[rr][k], 1.0f, (want >> (8 * k)) & 0xFFu);
        }
      }
    }
    if (row_ok) {
#pragma unroll
      for (int rr = 0; rr < RG; ++rr)
        if (r0 + rr < prm.P) k1_put_partial(prm, r0 + rr, row, slot, ss[rr]);
    }
  }
}

// Epilogue of a pure column block (all-shared or all-private) through TMA: for each 64-column
// chunk of the warp's 32 rows and each rank (all P ranks for a shared unit, whose one
// accumulator is their common cross-rank sum), the residual box is loaded by TMA into a
// swizzled shared buffer, every lane (one row) adds its accumulator row chunk (fp32, times
// the private scale for private units), rounds to bf16 in place, and the box is stored to h
// by TMA.  Full 128-byte lines move in bulk; rows beyond T and columns beyond H are
// zero-filled on load and clipped on store by the tensor maps.  Items are pipelined over
// NBUF buffers (K1_EPI_NBUF by default).  Returns false if a wait ran out.
// Mixed column blocks (merge = true, private units only): the shared unit of the block has
// already stored full boxes of h whose shared columns are final; the private unit loads that
// h box together with the residual box, keeps the shared columns, writes its private columns
// and stores the full box again (single-buffered).
template <int NBUF = K1_EPI_NBUF>
__device__ __forceinline__ bool k1_epilogue_tma(uint32_t trow, const RowparParams& prm, const void* tmR,
                                                const void* tmH, int row0, int n0, int rank, int slot, uint8_t* bufs,
                                                uint64_t* rbar, uint32_t& phase, int lane, uint64_t pol_r,
                                                uint64_t pol_h, bool merge = false) {
  if (merge) {
    const int nch = min(4, (prm.H - n0 + 63) / 64);
    const float scale = prm.private_scale;
    for (int c = 0; c < nch; ++c) {
      if (lane == 0) {
        mbar_arrive_expect_tx(&rbar[0], (prm.no_residual ? 1 : 2) * K1_EPI_BOX_BYTES);
        if (!prm.no_residual) tma_load_3d(bufs, tmR, &rbar[0], n0 + 64 * c, row0, rank, pol_r);
        tma_load_3d(bufs + K1_EPI_BOX_BYTES, tmH, &rbar[0], n0 + 64 * c, row0, rank, pol_r);
      }
      uint32_t v[64];
      __syncwarp();
      tmem_ld_32x32b_x32(trow + 64 * c, *reinterpret_cast<uint32_t(*)[32]>(v));
      tmem_ld_32x32b_x32(trow + 64 * c + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tmem_wait_ld();
      const bool ok = mbar_wait(&rbar[0], phase & 1u, prm.timeout_ns, 33);
      phase ^= 1u;
      if (!__all_sync(0xFFFFFFFFu, ok)) return false;
      uint8_t* rrow = bufs + lane * 128;
      uint8_t* hrow = bufs + K1_EPI_BOX_BYTES + lane * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int col = n0 + 64 * c + 8 * j;
        const uint32_t bits = (prm.mask_bits[col >> 5] >> (col & 31)) & 0xFFu;
        const int g = (j ^ (lane & 7)) << 4;
        const uint4 rr = prm.no_residual ? make_uint4(0u, 0u, 0u, 0u) : *reinterpret_cast<const uint4*>(rrow + g);
        const uint4 hh = *reinterpret_cast<const uint4*>(hrow + g);
        const uint32_t rw[4] = {rr.x, rr.y, rr.z, rr.w};
        const uint32_t hw[4] = {hh.x, hh.y, hh.z, hh.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t priv = pack_bf16x2(__uint_as_float(v[8 * j + 2 * e]) * scale + bf16lo(rw[e]),
                                            __uint_as_float(v[8 * j + 2 * e + 1]) * scale + bf16hi(rw[e]));
          const uint32_t keep = (((bits >> (2 * e)) & 1u) ? 0x0000FFFFu : 0u) |
                                (((bits >> (2 * e + 1)) & 1u) ? 0xFFFF0000u : 0u);
          o[e] = (hw[e] & keep) | (priv & ~keep);
        }
        *reinterpret_cast<uint4*>(hrow + g) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(tmH, bufs + K1_EPI_BOX_BYTES, n0 + 64 * c, row0, rank, pol_h);
        bulk_commit_group();
        bulk_wait_group_read0();  // both boxes are reused by the next chunk
      }
      __syncwarp();
    }
    if (prm.publish == 1) {  // the row blocks are published after this tile: complete its stores
      if (lane == 0) {
        bulk_wait_group0();
        asm volatile("fence.proxy.async.global;" ::: "memory");
      }
      __syncwarp();
    }
    return true;
  }
  const int nch = min(4, (prm.H - n0 + 63) / 64);
  const int nr = rank < 0 ? prm.P : 1;
  const int n_items = nch * nr;  // rank-major: item i = (rank i / nch, chunk i % nch)
  const float scale = rank < 0 ? 1.0f : prm.private_scale;
  const int row = row0 + lane;
  if (prm.no_residual) {
    // Z only: no residual boxes to load; each item is composed straight into a free buffer.
    for (int i = 0; i < n_items; ++i) {
      const int ri = i / nch, c = i - ri * nch;
      const int r = rank < 0 ? ri : rank;
      const int b = i % NBUF;
      uint32_t v[64];
      __syncwarp();
      tmem_ld_32x32b_x32(trow + 64 * c, *reinterpret_cast<uint32_t(*)[32]>(v));
      tmem_ld_32x32b_x32(trow + 64 * c + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tmem_wait_ld();
      if (lane == 0 && i >= NBUF) bulk_wait_group_read<NBUF - 1>();  // the store from buffer b has read it
      __syncwarp();
      uint8_t* rowp = bufs + b * K1_EPI_BOX_BYTES + lane * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          o[e] = pack_bf16x2(__uint_as_float(v[8 * j + 2 * e]) * scale, __uint_as_float(v[8 * j + 2 * e + 1]) * scale);
        *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(tmH, bufs + b * K1_EPI_BOX_BYTES, n0 + 64 * c, row0, r, pol_h);
        bulk_commit_group();
      }
    }
    if (lane == 0) {
      if (prm.publish == 1) {
        bulk_wait_group0();
        asm volatile("fence.proxy.async.global;" ::: "memory");
      } else {
        bulk_wait_group_read0();
      }
    }
    __syncwarp();
    return true;
  }
  const int npre = min(NBUF, n_items);
  for (int i = 0; i < npre; ++i) {
    const int ri = i / nch, c = i - ri * nch;
    const int r = rank < 0 ? ri : rank;
    if (lane == 0) {
      mbar_arrive_expect_tx(&rbar[i], K1_EPI_BOX_BYTES);
      tma_load_3d(bufs + i * K1_EPI_BOX_BYTES, tmR, &rbar[i], n0 + 64 * c, row0, r, pol_r);
    }
  }
  float ss = 0.f;
  for (int i = 0; i < n_items; ++i) {
    const int ri = i / nch, c = i - ri * nch;
    const int r = rank < 0 ? ri : rank;
    const int b = i % NBUF;
    uint32_t v[64];
    __syncwarp();
    tmem_ld_32x32b_x32(trow + 64 * c, *reinterpret_cast<uint32_t(*)[32]>(v));
    tmem_ld_32x32b_x32(trow + 64 * c + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
    tmem_wait_ld();
    const bool ok = mbar_wait(&rbar[b], (phase >> b) & 1u, prm.timeout_ns, 32);
    phase ^= 1u << b;
    if (!__all_sync(0xFFFFFFFFu, ok)) return false;
    uint8_t* rowp = bufs + b * K1_EPI_BOX_BYTES + lane * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint4* ptr = reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4));
      const uint4 rr = *ptr;
      const uint32_t rw[4] = {rr.x, rr.y, rr.z, rr.w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        o[e] = pack_bf16x2(__uint_as_float(v[8 * j + 2 * e]) * scale + bf16lo(rw[e]),
                           __uint_as_float(v[8 * j + 2 * e + 1]) * scale + bf16hi(rw[e]));
        if (prm.fuse_norm && n0 + 64 * c + 8 * j < prm.H) {
          const float lo = bf16lo(o[e]), hi = bf16hi(o[e]);
          ss = fmaf(lo, lo, ss);
          ss = fmaf(hi, hi, ss);
        }
      }
      *ptr = make_uint4(o[0], o[1], o[2], o[3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(tmH, bufs + b * K1_EPI_BOX_BYTES, n0 + 64 * c, row0, r, pol_h);
      bulk_commit_group();
    }
    if (prm.fuse_norm && c == nch - 1) {  // this rank's row segment is complete
      if (row < prm.t_end) k1_put_partial(prm, r, row, slot, ss);
      ss = 0.f;
    }
    const int nx = i + NBUF;
    if (nx < n_items) {
      if (lane == 0) {
        bulk_wait_group_read0();  // the store that read buffer b is done with it
        const int r2i = nx / nch, c2 = nx - r2i * nch;
        const int r2 = rank < 0 ? r2i : rank;
        mbar_arrive_expect_tx(&rbar[b], K1_EPI_BOX_BYTES);
        tma_load_3d(bufs + b * K1_EPI_BOX_BYTES, tmR, &rbar[b], n0 + 64 * c2, row0, r2, pol_r);
      }
      __syncwarp();
    }
  }
  if (lane == 0) {
    if (prm.publish == 1) {
      // The normalizers of other CTAs read this tile's h: complete the stores and order
      // them (async proxy) before the generic-proxy signal that follows.
      bulk_wait_group0();
      asm volatile("fence.proxy.async.global;" ::: "memory");
    } else {
      bulk_wait_group_read0();
    }
  }
  __syncwarp();
  return true;
}

// Shared unit in zs_mode 3: the accumulator of the columns below zs_ns (the cross-rank sum of
// Eq. 22, exact fp32) is stored to Zs [T, zs_ns] by 32 x 32 fp32 boxes (128-byte rows,
// 128-byte swizzle, clipped at zs_ns and T by the tensor map) through the warp's first two
// boxes in turn.  Nothing else: the residual add and the store of h for every rank move to the
// norm kernel, which reads Zs once per token.
__device__ __forceinline__ void k1_epilogue_zs(uint32_t trow, const RowparParams& prm, const void* tmZ, int row0,
                                               int n0, uint8_t* bufs, int lane, uint64_t pol) {
  const int nch = min(4, (prm.H - n0 + 63) / 64);
  int nb = 0;  // boxes stored so far; box nb goes through buffer nb % 2
  for (int c = 0; c < nch; ++c) {
    const int col = n0 + 64 * c;
    if (col >= prm.zs_ns) break;  // warp-uniform
    uint32_t v[64];
    __syncwarp();
    tmem_ld_32x32b_x32(trow + 64 * c, *reinterpret_cast<uint32_t(*)[32]>(v));
    tmem_ld_32x32b_x32(trow + 64 * c + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
    tmem_wait_ld();
    for (int hf = 0; hf < 2; ++hf) {
      if (col + 32 * hf >= prm.zs_ns) break;  // warp-uniform
      uint8_t* box = bufs + (nb & 1) * K1_EPI_BOX_BYTES;
      if (lane == 0 && nb >= 2) bulk_wait_group_read1();  // the store two boxes back has read this buffer
      __syncwarp();
      uint8_t* rowp = box + lane * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) =
            make_uint4(v[32 * hf + 4 * j], v[32 * hf + 4 * j + 1], v[32 * hf + 4 * j + 2], v[32 * hf + 4 * j + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(tmZ, box, col + 32 * hf, row0, 0, pol);
        bulk_commit_group();
      }
      ++nb;
    }
  }
  if (lane == 0) bulk_wait_group_read0();
  __syncwarp();
}

// Epilogue of one tile of the split-output mode (one tensor-parallel rank per device, every
// unit private): for each 64-column chunk of the warp's 32 rows, the columns below zs_ns (the
// shared channels, exchanged between devices) are stored as the fp32 partial to Zs [T, zs_ns]
// (two 32-column boxes, clipped at zs_ns by the tensor map), and a chunk reaching beyond zs_ns
// gets its private columns finished as in the plain epilogue (private scale, residual, bf16)
// and stored to h.  A chunk straddling zs_ns also stores its first columns to h with private
// arithmetic; the finishing kernel overwrites them with the exchanged values.  Returns false
// if a wait ran out.
__device__ __forceinline__ bool k1_epilogue_split(uint32_t trow, const RowparParams& prm, const void* tmR,
                                                  const void* tmH, const void* tmZ, int row0, int n0, int rank,
                                                  uint8_t* bufs, uint64_t* rbar, uint32_t& phase, int lane,
                                                  uint64_t pol_r, uint64_t pol_h) {
  const int nch = min(4, (prm.H - n0 + 63) / 64);
  const float scale = prm.private_scale;
  for (int c = 0; c < nch; ++c) {
    const int col = n0 + 64 * c;
    const bool has_shared = col < prm.zs_ns;
    const bool has_private = col + 64 > prm.zs_ns;
    if (has_private && lane == 0) {  // the residual box, while the accumulator is read
      bulk_wait_group_read0();       // earlier stores from the buffers are done reading them
      mbar_arrive_expect_tx(&rbar[0], K1_EPI_BOX_BYTES);
      tma_load_3d(bufs, tmR, &rbar[0], col, row0, rank, pol_r);
    }
    uint32_t v[64];
    __syncwarp();
    tmem_ld_32x32b_x32(trow + 64 * c, *reinterpret_cast<uint32_t(*)[32]>(v));
    tmem_ld_32x32b_x32(trow + 64 * c + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
    tmem_wait_ld();
    if (has_shared && prm.zs_mode == 2) {
      // each 32-column half goes to the owner of its columns: 8 16-byte stores per row
      const int row = row0 + lane;
      for (int hf = 0; hf < 2; ++hf) {
        const int cc = col + 32 * hf;
        if (cc >= prm.zs_ns) break;  // warp-uniform
        const int q = cc / prm.tp_w;
        const int j = cc - q * prm.tp_w;
        if (row < prm.t_end) {
          float4* dst = reinterpret_cast<float4*>(
              prm.tp_recv[q] + (static_cast<size_t>(prm.tp_rank) * prm.T + row) * prm.tp_w + j);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dst[k] = make_float4(__uint_as_float(v[32 * hf + 4 * k]), __uint_as_float(v[32 * hf + 4 * k + 1]),
                                 __uint_as_float(v[32 * hf + 4 * k + 2]), __uint_as_float(v[32 * hf + 4 * k + 3]));
        }
      }
    } else if (has_shared) {
      // fp32 boxes of 32 rows x 32 columns (128-byte rows, 128-byte swizzle) in buffer 1
      for (int hf = 0; hf < 2; ++hf) {
        if (col + 32 * hf >= prm.zs_ns) break;  // warp-uniform
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
        uint8_t* rowp = bufs + K1_EPI_BOX_BYTES + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) =
              make_uint4(v[32 * hf + 4 * j], v[32 * hf + 4 * j + 1], v[32 * hf + 4 * j + 2], v[32 * hf + 4 * j + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(tmZ, bufs + K1_EPI_BOX_BYTES, col + 32 * hf, row0, 0, pol_h);
          bulk_commit_group();
        }
      }
    }
    if (has_private) {
      const bool ok = mbar_wait(&rbar[0], phase & 1u, prm.timeout_ns, 34);
      phase ^= 1u;
      if (!__all_sync(0xFFFFFFFFu, ok)) return false;
      uint8_t* rowp = bufs + lane * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint4* ptr = reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4));
        const uint4 rr = *ptr;
        const uint32_t rw[4] = {rr.x, rr.y, rr.z, rr.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          o[e] = pack_bf16x2(__uint_as_float(v[8 * j + 2 * e]) * scale + bf16lo(rw[e]),
                             __uint_as_float(v[8 * j + 2 * e + 1]) * scale + bf16hi(rw[e]));
        *ptr = make_uint4(o[0], o[1], o[2], o[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(tmH, bufs, col, row0, rank, pol_h);
        bulk_commit_group();
      }
    }
  }
  if (lane == 0) bulk_wait_group_read0();
  __syncwarp();
  return true;
}

// Shared unit of a mixed block, after its TMA epilogue (one epilogue warp, 32 rows): complete
// the warp's box stores, make them visible to the async proxy of other CTAs, and mark the
// 32-row group's column block as stored.
__device__ __forceinline__ void k1_signal_sdone(unsigned int* flag) {
  if ((threadIdx.x & 31) == 0) {
    bulk_wait_group0();
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __threadfence();
    st_release_gpu(flag, 1u);
  }
  __syncwarp();
}

// Private unit of a mixed block: wait (bounded) until the block's shared unit has stored its
// boxes; returns false if the wait ran out.  Lane 0 polls, the warp follows.
__device__ __forceinline__ bool k1_wait_sdone(const RowparParams& prm, const unsigned int* flag) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) {
    if (ld_acquire_gpu(flag) == 0u) {
      const uint64_t t0 = globaltimer_ns();
      while (ld_acquire_gpu(flag) == 0u) {
        __nanosleep(500);
        if (status_poll() != 0 || globaltimer_ns() - t0 > prm.timeout_ns) {
          if (status_poll() == 0) status_raise(4, 35);
          ok = 0;
          break;
        }
      }
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");  // the TMA loads that follow see the boxes
  }
  return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

// After a tile's epilogue (all 128 epilogue threads): make its h and partials visible, count
// it into the row-block counters of its rank(s), and publish every row block it completes.
// The four epilogue warps meet on one of four mbarriers `sig[tile_idx % 4]` (count 4): every
// warp arrives after its stores and a gpu-scope fence, and warp 2's lane 0 waits (bounded)
// and then does the counting, so a warp that has left its loop on an error cannot block
// the others.  Four barriers: a warp can be at most two tiles ahead of another (the TMEM
// double buffer), so no warp arrives twice on a barrier before its phase completes.
// Publication of one finished tile for the row-norm kernel running beside the GEMM (publish
// mode 2), by one epilogue warp: complete the warp's box stores of the tile, order them (async
// proxy, then a gpu-scope fence) before the counter updates, and add 1 to the counter of each
// (128-row block, rank) the tile belongs to (every rank for a shared tile).  Called one tile
// late, when the warp starts its next tile (or leaves), so the stores have had a mainloop's
// time to complete and the wait rarely stalls.  Fire-and-forget reductions: no round trip.
__device__ __forceinline__ void k1_publish_counts(const RowparParams& prm, int m128, int rank) {
  if ((threadIdx.x & 31) == 0) {
    bulk_wait_group0();
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __threadfence();
    const int r0 = rank < 0 ? 0 : rank;
    const int r1 = rank < 0 ? prm.P : rank + 1;
    unsigned int* c = prm.rb_count + static_cast<size_t>(m128) * prm.P;
    for (int r = r0; r < r1; ++r) asm volatile("red.relaxed.gpu.global.add.u32 [%0], 1;" ::"l"(c + r) : "memory");
  }
  __syncwarp();
}

__device__ __forceinline__ void k1_signal_tile(const RowparParams& prm, uint64_t* sig, int tile_idx, int m128,
                                               int rank) {
  if (prm.publish != 1) return;
  __threadfence();
  __syncwarp();
  const int lane = threadIdx.x & 31;
  uint64_t* bar = &sig[tile_idx & 3];
  if (lane == 0) mbar_arrive(bar);
  if ((threadIdx.x & 127) == 64) {  // warp 2, lane 0
    if (!mbar_wait(bar, static_cast<uint32_t>(tile_idx >> 2) & 1u, prm.timeout_ns, 31)) return;
    const unsigned int target = static_cast<unsigned int>(prm.nS + prm.nPriv);
    const int r0 = rank < 0 ? 0 : rank;
    const int r1 = rank < 0 ? prm.P : rank + 1;
    for (int r = r0; r < r1; ++r) {
      const unsigned int rb = static_cast<unsigned int>(m128 * prm.P + r);
      const unsigned int old = atomicAdd(&prm.rb_count[rb], 1u);
      if (old + 1u == target) {
        __threadfence();
        const unsigned int pos = atomicAdd(prm.job_pub, 1u);
        st_release_gpu(&prm.job_slots[pos], rb + 1u);
      }
    }
  }
}

// Normalizer warp: claims 8-row pieces of published row blocks in publication order and
// rescales them.  Leaves when every piece of every row block is claimed (or on abort).
__device__ __forceinline__ void k1_normalizer(const RowparParams& prm, int lane) {
  const int total = prm.n_rb * K1_PIECES_PER_JOB;
  const int H = prm.H;
  const int nvec = H >> 3;
  const float inv_h = 1.0f / static_cast<float>(H);
  const uint4* g4 = reinterpret_cast<const uint4*>(prm.gamma);
  for (;;) {
    int c = 0;
    if (lane == 0) c = static_cast<int>(atomicAdd(prm.piece_claim, 1u));
    c = __shfl_sync(0xFFFFFFFFu, c, 0);
    if (c >= total) break;
    const int j = c / K1_PIECES_PER_JOB;
    const int part = c - j * K1_PIECES_PER_JOB;
    uint32_t v = 0;
    if (lane == 0) {
      v = ld_acquire_gpu(&prm.job_slots[j]);
      if (v == 0u) {
        const uint64_t t0 = globaltimer_ns();
        while ((v = ld_acquire_gpu(&prm.job_slots[j])) == 0u) {
          __nanosleep(1000);
          if (status_poll() != 0) break;
          if (globaltimer_ns() - t0 > prm.timeout_ns) {
            status_raise(4, 30);
            break;
          }
        }
      }
    }
    v = __shfl_sync(0xFFFFFFFFu, v, 0);
    if (v == 0u) break;
    const int rb = static_cast<int>(v) - 1;
    const int m128 = rb / prm.P;
    const int r = rb - m128 * prm.P;
#pragma unroll 1
    for (int i = 0; i < K1_ROWS_PER_PIECE; ++i) {
      const int row = m128 * K1_ROWS_PER_JOB + part * K1_ROWS_PER_PIECE + i;
      if (row >= prm.T) break;
      const float* sp = prm.ss_part + (static_cast<size_t>(r) * prm.T_pad + row) * prm.nslots;
      float s = 0.f;
      for (int k = lane; k < prm.nslots; k += 32) s += ld_cg_f32(sp + k);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, off);
      const float rstd = rsqrtf(s * inv_h + prm.eps);
      const size_t rowoff = (static_cast<size_t>(r) * prm.T + row) * H;
      const uint4* hp = reinterpret_cast<const uint4*>(prm.Hout + rowoff);
      uint4* op = reinterpret_cast<uint4*>(prm.Out + rowoff);
#pragma unroll 1
      for (int idx0 = 0; idx0 < nvec; idx0 += 32 * 8) {
        uint4 t[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int idx = idx0 + 32 * q + lane;
          t[q] = make_uint4(0, 0, 0, 0);
          if (idx < nvec) t[q] = ld_cg_v4(hp + idx);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int idx = idx0 + 32 * q + lane;
          if (idx < nvec) {
            const uint4 g = __ldg(g4 + idx);
            const uint32_t w[4] = {t[q].x, t[q].y, t[q].z, t[q].w};
            const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              o[e] = pack_bf16x2(bf16lo(w[e]) * rstd * bf16lo(gw[e]), bf16hi(w[e]) * rstd * bf16hi(gw[e]));
            st_v4(op + idx, make_uint4(o[0], o[1], o[2], o[3]));
          }
        }
      }
    }
  }
}

}  // namespace caat
