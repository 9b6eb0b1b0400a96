// caat_api.cu - host side of the C ABI declared in include/caat.h: argument validation,
// sync-set bookkeeping, tensor-map construction, kernel launches, timing and status.
//
// Source of the operations: "Tensor-Parallelism with Partially Synchronized Activations"
// (App. A.2 Eq. 22; §3 shared channels = first floor(h p); §3.1 Eq. 6 and 8; §4 Eq. 9 and
// 14-15).  The device code lives in the *.cuh files included below.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <mutex>
#include <queue>
#include <unordered_map>
#include <new>
#include <vector>

#include "caat.h"
#include "ptx.cuh"
#include "rowpar_gemm.cuh"
#include "rowpar_gemm2.cuh"
#include "fc1_swiglu.cuh"
#include "backward.cuh"
#include "decode.cuh"
#include "permuted.cuh"
#include "rownorm.cuh"
#include "tp.cuh"

namespace {

using caat::RowparParams;

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // bounded device waits: 2 s

// ---------------------------------------------------------------------------------------
// The current CUDA context (driver entry point fetched through the runtime).  Per-device state
// below (kernel attributes, streams, the no-alloc scratch address) is tied to the context it
// was made in: after a device reset the next call finds a new context and sets it up again.
// ---------------------------------------------------------------------------------------
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CUcontext current_context() {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<CtxGetCurrentFn>(nullptr);
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  CUcontext c = nullptr;
  if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
  return c;
}

// ---------------------------------------------------------------------------------------
// Device info and one-time kernel attributes (per device and context)
// ---------------------------------------------------------------------------------------
struct DeviceInfo {
  bool init = false;
  CUcontext ctx = nullptr;
  bool supported = false;
  int sm_count = 0;
  int max_pairs = 0;  // co-resident 2-CTA clusters of the pair GEMM kernel
};

std::mutex g_mu;
DeviceInfo g_dev[64];

caat_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CAAT_ERR_CUDA;
  if (dev < 0 || dev >= 64) return CAAT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  const CUcontext ctx = current_context();
  if (d.init && d.ctx != ctx) d = DeviceInfo();  // a new context (device reset): set up again
  if (!d.init) {
    d.ctx = ctx;
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return CAAT_ERR_CUDA;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return CAAT_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return CAAT_ERR_CUDA;
    d.sm_count = sms;
    d.supported = (major == 10 && minor == 0);
    if (d.supported) {
      if (cudaFuncSetAttribute(caat::rowpar_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               caat::K1_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(caat::rowpar_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               caat::K1_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(caat::rowpar_gemm_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               caat::K2P_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(caat::rowpar_gemm_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               caat::K2P_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(caat::rowpar_gemm_pair_kernel<false, 0, caat::K2P_STAGES_EPI, caat::K2P_EPI_NBUF_EPI>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, caat::K2P_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(caat::rowpar_gemm_pair_kernel<false, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               caat::K2P_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(caat::rowpar_gemm_pair_kernel<false, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               caat::K2P_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(caat::fc1_swiglu_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               caat::K3_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(caat::decode_partials_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               caat::K4_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(caat::rownorm_bwd_smem_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(caat::KB_SMEM_MAX)) != cudaSuccess ||
          cudaFuncSetAttribute(caat::rownorm_bwd_smem_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(caat::KB_SMEM_MAX)) != cudaSuccess ||
          cudaFuncSetAttribute(caat::rownorm_gather_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(caat::gather_smem_bytes(1024))) != cudaSuccess ||
          cudaFuncSetAttribute(caat::rownorm_gather_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(caat::gather_smem_bytes(2048))) != cudaSuccess ||
          cudaFuncSetAttribute(caat::rownorm_gather_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(caat::gather_smem_bytes(4096))) != cudaSuccess ||
          cudaFuncSetAttribute(caat::rownorm_consumer_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               caat::K2C_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(caat::rownorm_consumer_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               caat::K2C_SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(caat::rownorm_consumer_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               caat::K2C_SMEM_BYTES) != cudaSuccess)
        return CAAT_ERR_CUDA;
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
      cfg.blockDim = dim3(caat::K1Threads<true>::value, 1, 1);
      cfg.dynamicSmemBytes = caat::K2P_SMEM_BYTES;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, caat::rowpar_gemm_pair_kernel<true>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        clusters = 0;
      }
      d.max_pairs = clusters;
    }
    d.init = true;
  }
  if (!d.supported) return CAAT_ERR_UNSUPPORTED;
  *out = &d;
  return CAAT_OK;
}

// Row blocks per group of the grouped tile order (tuning; CAAT_GROUP_M overrides).
int group_m_setting() {
  static int v = [] {
    const char* e = std::getenv("CAAT_GROUP_M");
    const int g = (e && *e) ? std::atoi(e) : 0;
    return g > 0 ? g : 8;
  }();
  return v;
}

// Upper bounds on the GEMM kernel's CTA pairs and the row norm's blocks (tuning; 0 = none).
int env_cap(const char* name) {
  const char* e = std::getenv(name);
  const int v = (e && *e) ? std::atoi(e) : 0;
  return v > 0 ? v : 0;
}
int gemm_pairs_cap() {
  static int v = env_cap("CAAT_GEMM_PAIRS");
  return v;
}
int norm_blocks_cap() {
  static int v = env_cap("CAAT_NORM_BLOCKS");
  return v;
}
// SMs the GEMM kernel leaves to the row norm running beside it (tuning; CAAT_NORM_SMS).
int norm_sms_setting() {
  static int v = [] {
    const char* e = std::getenv("CAAT_NORM_SMS");
    return (e && *e) ? std::max(0, std::atoi(e)) : 16;
  }();
  return v;
}
// Unit order and stagger distance of the GEMM when the row norm runs beside it (tuning;
// CAAT_ORDER, CAAT_STAGGER).
int consumer_order_setting() {
  static int v = [] {
    const char* e = std::getenv("CAAT_ORDER");
    const int o = (e && *e) ? std::atoi(e) : 0;
    return (o >= 0 && o <= 3) ? o : 0;
  }();
  return v;
}
// Largest k-blocks per rank for which the GEMM takes the epilogue-heavy shared-memory split
// (tuning; CAAT_EPI_HEAVY_KBLK).
int epi_heavy_kblk_setting() {
  static int v = [] {
    const char* e = std::getenv("CAAT_EPI_HEAVY_KBLK");
    return (e && *e) ? std::atoi(e) : 12;
  }();
  return v;
}
// Smallest token count whose decode reduce runs one CTA per token (tuning; CAAT_DECODE_TOKEN_T).
int decode_token_min_t() {
  static int v = [] {
    const char* e = std::getenv("CAAT_DECODE_TOKEN_T");
    return (e && *e) ? std::max(1, std::atoi(e)) : 9;
  }();
  return v;
}
// Whether the decode streaming kernel splits its items evenly, cutting units (tuning;
// CAAT_DECODE_STREAMK: 1 always, 0 never; unset: with the per-row reduce (few tokens) only.
// Measured on one box: T = 8 30.8 us with the split against 32.1 us with whole units; T = 64
// 38.6 us against 37.1 us, the per-token reduce then paying for the split units' second slots).
int decode_stream_k_setting() {
  static int v = [] {
    const char* e = std::getenv("CAAT_DECODE_STREAMK");
    return (e && *e) ? (*e == '1' ? 1 : 0) : -1;
  }();
  return v;
}
// Streaming CTAs per SM on the decode path, each with half the ring (tuning; CAAT_DECODE_CTAS:
// 1 or 2).  Two measured faster at T = 1 / 8 / 64 on one box: 30.9 / 30.8 / 37.0 us with one,
// 28.8 / 28.9 / 34.7 us with two (more copies in flight against DRAM at once).
int decode_ctas_per_sm_setting() {
  static int v = [] {
    const char* e = std::getenv("CAAT_DECODE_CTAS");
    return (e && *e == '1') ? 1 : 2;
  }();
  return v;
}
// Norm backward: bf16(s dh) kept in registers between its passes 2 and 3, so that the next
// token's loads start a pass earlier (tuning; CAAT_BWD_ZK: 1 on, 0 off).
bool bwd_zk_regs_setting() {
  static bool v = [] {
    const char* e = std::getenv("CAAT_BWD_ZK");
    return (e && *e) ? (*e == '1') : true;
  }();
  return v;
}
// The shared units store their cross-rank sums once (fp32) and the norm kernel adds each rank's
// residual, instead of every shared tile storing h for all P ranks (tuning; CAAT_ZS_SUM: 1 on,
// 0 off).
bool zs_sum_setting() {
  static bool v = [] {
    const char* e = std::getenv("CAAT_ZS_SUM");
    return (e && *e) ? (*e == '1') : true;
  }();
  return v;
}
// Shared-sum mode: pairs of pure shared column blocks run as one 256 x 512 unit (tuning;
// CAAT_WIDE: 1 every pair, 0 never; unset: for K >= 8192, every pair when there are private
// units, else the count a simulated schedule favours).
int wide_setting() {
  static int v = [] {
    const char* e = std::getenv("CAAT_WIDE");
    return (e && *e) ? (*e == '1' ? 1 : 0) : -1;
  }();
  return v;
}
// How many pairs of whole shared column blocks per row block to run as 256 x 512 units when
// there are no private units (every shared block pure): the dynamic scheduler's makespan,
// simulated on `pairs` CTA pairs for wide units first (each worth 1.84 ordinary units, as
// measured at fc2-7b p = 1), then the ordinary shared units; the count with the shortest
// makespan (the fewer wide units on a tie).  Cached per shape.
int wide_count_by_schedule(int n_mblk, int nS, int pure_pairs, int pairs) {
  static std::mutex mu;
  static std::unordered_map<uint64_t, int> memo;
  const uint64_t key = (uint64_t(n_mblk) << 40) ^ (uint64_t(nS) << 24) ^ (uint64_t(pure_pairs) << 12) ^ uint64_t(pairs);
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = memo.find(key);
    if (it != memo.end()) return it->second;
  }
  constexpr double kWideCost = 1.84;
  double best = 0.0;
  int best_w = 0;
  for (int w = 0; w <= pure_pairs; ++w) {
    std::priority_queue<double, std::vector<double>, std::greater<double>> free_at;
    for (int q = 0; q < std::max(pairs, 1); ++q) free_at.push(0.0);
    double end = 0.0;
    auto run = [&](int count, double cost) {
      for (int i = 0; i < count; ++i) {
        const double t = free_at.top() + cost;
        free_at.pop();
        free_at.push(t);
        end = std::max(end, t);
      }
    };
    run(n_mblk * w, kWideCost);
    run(n_mblk * (nS - 2 * w), 1.0);
    if (w == 0 || end < best - 1e-9) {
      best = end;
      best_w = w;
    }
  }
  std::lock_guard<std::mutex> lk(mu);
  memo[key] = best_w;
  return best_w;
}
bool order_env_set() {
  static bool v = [] {
    const char* e = std::getenv("CAAT_ORDER");
    return e && *e;
  }();
  return v;
}
int stagger_setting() {
  static int v = [] {
    const char* e = std::getenv("CAAT_STAGGER");
    const int d = (e && *e) ? std::atoi(e) : 6;
    return d >= 0 ? d : 6;
  }();
  return v;
}

uint64_t timeout_ns() {
  static uint64_t v = [] {
    const char* e = std::getenv("CAAT_TIMEOUT_MS");
    if (e && *e) {
      const double ms = std::atof(e);
      if (ms > 0) return static_cast<uint64_t>(ms * 1e6);
    }
    return kDefaultTimeoutNs;
  }();
  return v;
}

// ---------------------------------------------------------------------------------------
// Tensor maps (driver entry point fetched through the runtime; no link to libcuda)
// ---------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 3-D bf16 tensor [d2][d1][d0] (d0 contiguous), box {b0, b1, 1}, 128-byte swizzle.
caat_status make_map_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                        uint32_t b1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return CAAT_ERR_CUDA;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  const cuuint32_t box[3] = {b0, b1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CAAT_OK : CAAT_ERR_CUDA;
}

// 3-D fp32 tensor [d2][d1][d0] (d0 contiguous), box {b0, b1, 1}, 128-byte swizzle.
caat_status make_map_3d_f32(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                            uint32_t b1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return CAAT_ERR_CUDA;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * 4, d0 * d1 * 4};
  const cuuint32_t box[3] = {b0, b1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CAAT_OK : CAAT_ERR_CUDA;
}

// 4-D bf16 tensor [d3][d2][d1][d0] (d0 contiguous), box {b0, b1, 1, 1}, 128-byte swizzle.
caat_status make_map_4d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
                        uint32_t b0, uint32_t b1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return CAAT_ERR_CUDA;
  const cuuint64_t dims[4] = {d0, d1, d2, d3};
  const cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
  const cuuint32_t box[4] = {b0, b1, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CAAT_OK : CAAT_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------
// Validation and sync-set bookkeeping
// ---------------------------------------------------------------------------------------
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

caat_status check_shapes(int64_t T, int64_t K, int64_t H, int P, double p) {
  if (P < 1 || P > CAAT_MAX_P) return CAAT_ERR_INVALID_ARG;
  if (T < 0 || K <= 0 || H <= 0) return CAAT_ERR_INVALID_ARG;
  if (!(p >= 0.0 && p <= 1.0)) return CAAT_ERR_INVALID_ARG;
  if (K % P != 0) return CAAT_ERR_UNSUPPORTED;
  const int64_t Kp = K / P;
  if (Kp % 8 != 0 || Kp > (int64_t(1) << 30)) return CAAT_ERR_UNSUPPORTED;
  if (H % 8 != 0 || H > CAAT_MAX_H) return CAAT_ERR_UNSUPPORTED;
  if (T > (int64_t(1) << 30)) return CAAT_ERR_UNSUPPORTED;
  return CAAT_OK;
}

int64_t n_sync_of(int64_t H, double p) {
  return static_cast<int64_t>(std::floor(static_cast<double>(H) * p));
}

// Fills mask (H entries, 1 = shared) from (H, p, sync_idx); validates sync_idx.
caat_status build_mask(int64_t H, double p, const int32_t* sync_idx, std::vector<uint8_t>& mask, int64_t* ns_out) {
  if (H <= 0 || !(p >= 0.0 && p <= 1.0)) return CAAT_ERR_INVALID_ARG;
  const int64_t ns = n_sync_of(H, p);
  mask.assign(static_cast<size_t>(H), 0);
  if (sync_idx == nullptr) {
    for (int64_t c = 0; c < ns; ++c) mask[c] = 1;
  } else {
    int64_t prev = -1;
    for (int64_t i = 0; i < ns; ++i) {
      const int64_t c = sync_idx[i];
      if (c < 0 || c >= H || c <= prev) return CAAT_ERR_INVALID_ARG;
      mask[c] = 1;
      prev = c;
    }
  }
  if (ns_out) *ns_out = ns;
  return CAAT_OK;
}

constexpr size_t kCounterBytes = 256;

// Internal (not in caat.h): run only the GEMM kernel of the row-parallel path, storing the
// per-rank products without residual or norm -- a batched GEMM C_b = A_b B_b^T (p = 0, P = b).
constexpr uint32_t kFlagGemmOnly = 0x40000000u;
// Internal, with kFlagGemmOnly on the CTA-pair kernel: A is stored [b][Kr][M] (M contiguous) /
// B is stored [b][Kr][N], read MN-major by the tensor cores (no transposed copies).
constexpr uint32_t kFlagAMn = 0x20000000u;
constexpr uint32_t kFlagBMn = 0x10000000u;

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

// Workspace of the row-parallel layer.  Fused norm: [counters (256 B) | rb_count[n_rb] |
// job_slots[n_rb] | ss_part[P][T_pad][nslots_max] floats]; the counter region (first `zeroed`
// bytes) is cleared on the stream before every launch; ss_part needs no clearing (every slot
// of every valid row is written once).  Separate norm: [counters (256 B) | rb_count[n_rb] |
// sdone]: the tile counters (cleared before the launch when used) let the row norm run beside
// the GEMM; the optional sdone flags ([T_pad/32][n-blocks] u32, cleared before the launch when
// used) let the CTA-pair kernel give mixed column blocks the TMA epilogue.  With a workspace of
// only the 256 B (`min_total`) the norm runs after the GEMM and mixed blocks take the register
// epilogue.  Sized for the larger of the two GEMM kernels' row blocking.
struct RowparWs {
  size_t rb_count, job_slots, ss_part, zeroed, total, min_total, sdone, sdone_bytes, consumer_total;
  int64_t T_pad, n_rb, nslots_max;
};

RowparWs rowpar_ws_layout(int64_t T, int64_t H, int P, bool fused) {
  RowparWs L{};
  L.T_pad = (T + 255) / 256 * 256;
  L.n_rb = (L.T_pad / 128) * P;
  L.nslots_max = 2 * ((H + 255) / 256);
  if (fused) {
    L.rb_count = kCounterBytes;
    L.job_slots = L.rb_count + size_t(L.n_rb) * 4;
    L.zeroed = L.job_slots + size_t(L.n_rb) * 4;
    L.ss_part = align256(L.zeroed);
    L.total = L.ss_part + align256(size_t(P) * L.T_pad * L.nslots_max * 4);
    L.min_total = L.total;
  } else {
    // [counters | rb_count | sdone]: the per-(128-row block, rank) tile counters let the row
    // norm run beside the GEMM (a workspace that ends before sdone still allows it).
    L.rb_count = kCounterBytes;
    L.zeroed = kCounterBytes;
    L.consumer_total = L.rb_count + size_t(L.n_rb) * 4;
    L.sdone = align256(L.consumer_total);
    L.sdone_bytes = size_t(L.T_pad / 32) * size_t((H + 255) / 256) * 4;
    L.total = L.sdone + align256(L.sdone_bytes);
    L.min_total = kCounterBytes;
  }
  return L;
}

// The GEMM path's shared-sum mode: after the counters, Zs [T, n_s] fp32 (the cross-rank sums of
// the shared channels, stored once by the shared units, read by the norm kernel for every rank).
constexpr size_t kZsOffset = kCounterBytes;
size_t zs_workspace(int64_t T, int64_t n_s) { return kZsOffset + align256(size_t(T) * size_t(n_s) * 4); }

// Decode path (T <= CAAT_DECODE_MAX_T, P <= 16): the weight-streaming kernel splits the stream
// of (unit, k-block) items evenly over its CTAs; a unit cut in two leaves two fp32 partials.
bool decode_eligible(int64_t T, int P, int64_t H) {
  return T >= 1 && T <= CAAT_DECODE_MAX_T && P <= caat::K4_MAXP && H <= caat::K4B_MAX_H;
}

// Decode workspace: [256 B | Zp fp32 [2 slots][P][T][H]].
size_t decode_workspace(int64_t T, int64_t H, int P) {
  return kCounterBytes + align256(size_t(2) * P * T * H * 4);
}

// Whether a call with these shapes and flags runs the decode (weight-streaming) kernels.
bool takes_decode_path(int64_t T, int P, int64_t H, uint32_t flags) {
  if (!decode_eligible(T, P, H)) return false;
  if (flags & CAAT_FLAG_FORCE_DECODE_PATH) return true;
  return !(flags & (CAAT_FLAG_FORCE_GEMM_PATH | CAAT_FLAG_FUSED_NORM | CAAT_FLAG_TEST_STALL));
}

// The size that enables every path and fast path of a call of this shape (the value
// caat_workspace_size reports).
size_t rowpar_workspace(int64_t T, int64_t K, int64_t H, int P) {
  (void)K;
  size_t n = std::max(rowpar_ws_layout(T, H, P, true).total, rowpar_ws_layout(T, H, P, false).total);
  if (decode_eligible(T, P, H)) n = std::max(n, decode_workspace(T, H, P));
  if (H <= 4096) n = std::max(n, zs_workspace(T, H));  // the shared sums, up to every channel
  return n;
}

// The workspace a call with these flags needs at least: the decode path's partials if it takes
// that path, else the GEMM path's minimum (the fused norm's partials, or the 256-byte counters).
size_t rowpar_workspace_min(int64_t T, int64_t H, int P, uint32_t flags) {
  if (takes_decode_path(T, P, H, flags)) return decode_workspace(T, H, P);
  return rowpar_ws_layout(T, H, P, (flags & CAAT_FLAG_FUSED_NORM) != 0).min_total;
}

// Device staging of caat_rowpar_forward_host.  Token rows are independent through the whole
// path, so the call is pipelined over chunks of kHostChunk tokens: W and gamma are copied once,
// then per chunk X and R are copied in, the kernels run and out (and h) are copied back, with
// two chunk buffers so that copies in both directions overlap the kernels of other chunks.
// Layout: [row-parallel workspace for one chunk | W | gamma | 2 x (X_c | R_c | O_c | H_c)].
constexpr int64_t kHostChunk = 1024;

struct HostLayout {
  int64_t Tc;
  size_t ws, w, g, buf0, x, r, o, h, buf_bytes, total;
};

HostLayout host_layout(int64_t T, int64_t K, int64_t H, int P) {
  HostLayout L{};
  const size_t Kp = static_cast<size_t>(K / P);
  L.Tc = std::min<int64_t>(T, kHostChunk);
  L.ws = 0;
  L.w = align256(rowpar_workspace(L.Tc, K, H, P));
  L.g = L.w + align256(size_t(P) * H * Kp * 2);
  L.buf0 = L.g + align256(size_t(H) * 2);
  L.x = 0;
  L.r = align256(size_t(P) * L.Tc * Kp * 2);
  L.o = L.r + align256(size_t(P) * L.Tc * H * 2);
  L.h = L.o + align256(size_t(P) * L.Tc * H * 2);
  L.buf_bytes = L.h + align256(size_t(P) * L.Tc * H * 2);
  L.total = L.buf0 + 2 * L.buf_bytes;
  return L;
}

constexpr int64_t kNormChunk = 2048;  // tokens per GEMM launch when the norm is overlapped

// Side stream and events that let the row norm of one chunk of tokens run while the GEMM
// kernel computes the next chunk (created once per device).
struct NormSide {
  bool init = false;
  CUcontext ctx = nullptr;
  cudaStream_t s = nullptr;
  cudaEvent_t ev_gemm = nullptr, ev_done = nullptr;
};
NormSide g_side[64];

caat_status norm_side(NormSide** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CAAT_ERR_CUDA;
  if (dev < 0 || dev >= 64) return CAAT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  NormSide& ns = g_side[dev];
  const CUcontext ctx = current_context();
  if (ns.init && ns.ctx != ctx) ns = NormSide();  // handles of a context that no longer exists
  if (!ns.init) {
    ns.ctx = ctx;
    if (cudaStreamCreateWithFlags(&ns.s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ns.ev_gemm, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ns.ev_done, cudaEventDisableTiming) != cudaSuccess)
      return CAAT_ERR_CUDA;
    ns.init = true;
  }
  *out = &ns;
  return CAAT_OK;
}

// Copy streams and events of the host-buffer pipeline (created once per device).
struct HostPipe {
  bool init = false;
  CUcontext ctx = nullptr;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev_start = nullptr, ev_w = nullptr, ev_in[2] = {}, ev_comp[2] = {}, ev_out[2] = {};
};
HostPipe g_pipe[64];

caat_status host_pipe(HostPipe** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CAAT_ERR_CUDA;
  if (dev < 0 || dev >= 64) return CAAT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  HostPipe& hp = g_pipe[dev];
  const CUcontext ctx = current_context();
  if (hp.init && hp.ctx != ctx) hp = HostPipe();  // handles of a context that no longer exists
  if (!hp.init) {
    hp.ctx = ctx;
    if (cudaStreamCreateWithFlags(&hp.s_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&hp.s_out, cudaStreamNonBlocking) != cudaSuccess)
      return CAAT_ERR_CUDA;
    cudaEvent_t* evs[] = {&hp.ev_start, &hp.ev_w, &hp.ev_in[0], &hp.ev_in[1], &hp.ev_comp[0],
                          &hp.ev_comp[1], &hp.ev_out[0], &hp.ev_out[1]};
    for (cudaEvent_t* e : evs)
      if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return CAAT_ERR_CUDA;
    hp.init = true;
  }
  *out = &hp;
  return CAAT_OK;
}

// Workspace of the MLP block: [FC1 unit counter (256 B) | row-parallel workspace | Y [P,T,F/P]].
struct MlpWs {
  size_t rowpar, y, total;
};

MlpWs mlp_ws_layout(int64_t T, int64_t H, int64_t F, int P, bool fused) {
  MlpWs L{};
  L.rowpar = kCounterBytes;
  (void)fused;
  L.y = L.rowpar + align256(rowpar_workspace(T, F, H, P));
  L.total = L.y + align256(size_t(P) * T * (F / P) * 2);
  return L;
}

}  // namespace

// ---------------------------------------------------------------------------------------
// Timing recorder
// ---------------------------------------------------------------------------------------
struct caat_timing {
  int capacity = 0;
  int max_kernels = 8;
  int n = 0;
  std::vector<cudaEvent_t> ev;
  std::vector<int> nk;
};

namespace {

struct Recorder {
  caat_timing* t = nullptr;
  int rec = -1;
  int k = 0;
  void begin(caat_timing* tm, cudaStream_t s) {
    t = tm;
    if (!t || t->n >= t->capacity) {
      t = nullptr;
      return;
    }
    rec = t->n++;
    k = 0;
    cudaEventRecord(t->ev[rec * (t->max_kernels + 1)], s);
  }
  void after_kernel(cudaStream_t s) {
    if (!t || k >= t->max_kernels) return;
    ++k;
    cudaEventRecord(t->ev[rec * (t->max_kernels + 1) + k], s);
    t->nk[rec] = k;
  }
};

// ---------------------------------------------------------------------------------------
// The row-parallel layer: GEMM + partial channel-reduce + residual (K1), RMSNorm (K2)
// ---------------------------------------------------------------------------------------
// The decode path: weight-streaming partial products (K4a), then reduce + residual + norm (K4b).
caat_status launch_decode(const caat_rowpar_args* a, const std::vector<uint8_t>& mask, const DeviceInfo* dev,
                          uint8_t* ws, Recorder* outer) {
  const int P = a->P;
  const int64_t T = a->T, H = a->H, Kp = a->K / P;
  cudaStream_t st = a->stream;
  caat::DecodeGemmParams gp{};
  gp.Zp = reinterpret_cast<float*>(ws + kCounterBytes);
  gp.T = static_cast<int>(T);
  gp.Tpad = static_cast<int>((T + 15) / 16 * 16);
  gp.H = static_cast<int>(H);
  gp.P = P;
  gp.n_cb = static_cast<int>((H + caat::K4_BM - 1) / caat::K4_BM);
  gp.kblk = static_cast<int>((Kp + caat::K4_BK - 1) / caat::K4_BK);
  const int64_t tail = Kp - int64_t(gp.kblk - 1) * caat::K4_BK;
  gp.last_k16 = static_cast<int>((tail + 15) / 16);
  const int64_t units = int64_t(P) * gp.n_cb;
  const int64_t items = units * gp.kblk;
  if (items > INT32_MAX / 2) return CAAT_ERR_UNSUPPORTED;
  gp.n_items = static_cast<int>(items);
  const int per_sm = decode_ctas_per_sm_setting();
  gp.ring_bytes = per_sm == 2 ? caat::K4_RING_BYTES_HALF : caat::K4_RING_BYTES;
  gp.stages = caat::k4_stages(gp.Tpad, gp.ring_bytes);
  gp.timeout_ns = timeout_ns();
  // No more CTAs than units: every CTA then streams at least one unit's worth of items, so a
  // unit is cut at most once (two partials).
  const int grid = static_cast<int>(std::min<int64_t>(int64_t(per_sm) * dev->sm_count, units));
  const int k4_smem = 1024 + gp.ring_bytes + 512;

  static thread_local caat::DecodeParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.Zp = gp.Zp;
  prm.R = reinterpret_cast<const __nv_bfloat16*>(a->residual);
  prm.Hout = reinterpret_cast<__nv_bfloat16*>(a->h_out ? a->h_out : a->out);
  prm.Out = reinterpret_cast<__nv_bfloat16*>(a->out);
  prm.gamma = reinterpret_cast<const __nv_bfloat16*>(a->gamma);
  prm.T = static_cast<int>(T);
  prm.H = static_cast<int>(H);
  prm.P = P;
  prm.n_cb = gp.n_cb;
  prm.kblk = gp.kblk;
  // units cut between two streaming CTAs (their first and last k-block have different owners)
  if (units > int64_t(caat::K4_MAXP) * 64) return CAAT_ERR_UNSUPPORTED;
  gp.stream_k = decode_stream_k_setting() >= 0 ? decode_stream_k_setting() : (T < decode_token_min_t() ? 1 : 0);
  for (int64_t u = 0; gp.stream_k && u < units; ++u) {
    const int64_t first = u * gp.kblk;
    if (caat::k4_cta_of(first, items, grid) != caat::k4_cta_of(first + gp.kblk - 1, items, grid))
      prm.split_bits[u >> 5] |= 1u << (u & 31);
  }
  prm.private_scale = a->private_scale;
  prm.eps = a->eps;
  prm.permuted = (a->flags & CAAT_FLAG_W_PERMUTED) ? 1 : 0;
  for (int64_t c = 0; c < H; ++c)
    if (mask[c]) {
      prm.mask_bits[c >> 5] |= 1u << (c & 31);
      ++prm.n_s;
    }

  CUtensorMap tmW, tmX;
  caat_status s = make_map_3d(&tmW, a->W, Kp, H, P, caat::K4_BK, caat::K4_BM);
  if (s != CAAT_OK) return s;
  s = make_map_3d(&tmX, a->X, Kp, T, P, caat::K4_BK, static_cast<uint32_t>(gp.Tpad));
  if (s != CAAT_OK) return s;
  Recorder own;
  Recorder& rec = outer ? *outer : own;
  if (!outer) rec.begin(a->timing, st);
  caat::decode_partials_kernel<<<grid, caat::K4_THREADS, k4_smem, st>>>(tmW, tmX, gp);
  if (cudaGetLastError() != cudaSuccess) return CAAT_ERR_CUDA;
  rec.after_kernel(st);
  // The reduce kernel is a programmatic dependent of the partials kernel: its launch overlaps
  // the partials kernel's tail, and it waits in-kernel for that grid's completion.
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  // few tokens: one CTA per (rank, token) row; more: one CTA per token (shared sum formed once)
  const bool per_row = T < decode_token_min_t();
  cfg.gridDim = dim3(static_cast<unsigned>(per_row ? P * T : T), 1, 1);
  cfg.blockDim = dim3(per_row ? caat::K4B_THREADS : caat::K4T_THREADS, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e =
      per_row  ? cudaLaunchKernelEx(&cfg, caat::decode_reduce_norm_kernel<caat::K4B_THREADS, caat::K4B_VEC>, prm)
      : P <= 8 ? cudaLaunchKernelEx(&cfg, caat::decode_reduce_token_kernel<8>, prm)
               : cudaLaunchKernelEx(&cfg, caat::decode_reduce_token_kernel<16>, prm);
  if (e != cudaSuccess) return CAAT_ERR_CUDA;
  rec.after_kernel(st);
  return CAAT_OK;
}

// The split-output local step of one rank of a multi-device layer (caat_rowpar_tp_local):
// the fp32 partial of the first n_s channels goes to zs [T, n_s], the other channels are
// finished into h.
struct TpSplit {
  float* zs;
  int64_t n_s;
  const caat_tp_peers* peers;  // non-null: push the partials to their owners (peer memory)
};

caat_status launch_rowpar(const caat_rowpar_args* a, const std::vector<uint8_t>& mask, const DeviceInfo* dev,
                          unsigned int* counter, Recorder* outer = nullptr, const TpSplit* split = nullptr) {
  // Decode-sized calls stream W once through the dedicated path.
  if (!split && takes_decode_path(a->T, a->P, a->H, a->flags))
    return launch_decode(a, mask, dev, reinterpret_cast<uint8_t*>(counter), outer);
  const int P = a->P;
  const int64_t T = a->T, H = a->H, Kp = a->K / P;
  cudaStream_t st = a->stream;
  __nv_bfloat16* hdst = reinterpret_cast<__nv_bfloat16*>(a->h_out ? a->h_out : a->out);

  // Channel-permuted W (caat_permute_weights): the GEMM runs on a contiguous sync set and
  // writes Z' (no residual) into zdst; the gather norm restores the channel order.
  const bool permuted = (a->flags & CAAT_FLAG_W_PERMUTED) != 0;
  std::vector<uint8_t> pmask;
  const std::vector<uint8_t>* tmask = &mask;  // the mask the GEMM's tiles see
  int n_s = 0;
  for (int64_t c = 0; c < H; ++c) n_s += mask[c];
  if (permuted) {
    if (a->flags & CAAT_FLAG_FUSED_NORM) return CAAT_ERR_UNSUPPORTED;
    if (H > 4096) return CAAT_ERR_UNSUPPORTED;
    void* zd = (a->h_out && a->h_out != a->residual) ? a->h_out : a->out;
    if (zd == a->residual) return CAAT_ERR_UNSUPPORTED;
    hdst = reinterpret_cast<__nv_bfloat16*>(zd);
    pmask.assign(static_cast<size_t>(H), 0);
    for (int c = 0; c < n_s; ++c) pmask[c] = 1;
    tmask = &pmask;
  }

  static thread_local RowparParams prm;  // ~10 KiB: keep it off the stack
  std::memset(&prm, 0, sizeof(prm));
  const bool fused = (a->flags & CAAT_FLAG_FUSED_NORM) != 0;
  const bool gemm_only = (a->flags & kFlagGemmOnly) != 0;
  prm.no_residual = (permuted || gemm_only) ? 1 : 0;
  const RowparWs wl = rowpar_ws_layout(T, H, P, fused);
  uint8_t* wsb = reinterpret_cast<uint8_t*>(counter);
  prm.R = reinterpret_cast<const __nv_bfloat16*>(a->residual);
  prm.Hout = hdst;
  prm.Out = reinterpret_cast<__nv_bfloat16*>(a->out);
  prm.gamma = reinterpret_cast<const __nv_bfloat16*>(a->gamma);
  prm.counter = counter;
  prm.piece_claim = counter + 1;
  prm.job_pub = counter + 2;
  prm.rb_count = fused ? reinterpret_cast<unsigned int*>(wsb + wl.rb_count) : nullptr;
  prm.job_slots = fused ? reinterpret_cast<unsigned int*>(wsb + wl.job_slots) : nullptr;
  prm.ss_part = fused ? reinterpret_cast<float*>(wsb + wl.ss_part) : nullptr;
  prm.fuse_norm = fused ? 1 : 0;
  // Tile order: the fused norm wants row blocks to complete throughout the kernel (grouped
  // order); otherwise shared tiles first, then private tiles rank by rank.
  prm.order = (a->flags & CAAT_FLAG_ORDER_ROWBLOCK) ? 1 : ((fused || (a->flags & CAAT_FLAG_ORDER_GROUPED)) ? 2 : 0);
  prm.group_m = group_m_setting();
  // The row norm beside the GEMM (CTA-pair kernel, separate norm, rows of at most 4096
  // channels): the GEMM publishes each completed (128-row block, rank), and the norm kernel,
  // launched as its programmatic dependent, normalizes published rows on the SMs the GEMM
  // leaves free, while the GEMM computes the others.
  const bool pair_possible =
      dev->max_pairs > 0 && (split != nullptr || (!(a->flags & CAAT_FLAG_SINGLE_CTA) && T > caat::K1_BM));
  const bool consumer = pair_possible && !split && !fused && !permuted && !gemm_only && H <= 4096 &&
                        (a->flags & CAAT_FLAG_NORM_BESIDE_GEMM) && !(a->flags & CAAT_FLAG_OVERLAP_NORM) &&
                        a->ws_bytes >= wl.consumer_total;
  prm.publish = fused ? 1 : (consumer ? 2 : 0);
  // Shared-sum mode: S the first n_s channels, rows of at most 4096 channels, room for Zs, h
  // not stored over the residual (a mixed block's private tiles write whole h boxes, whose
  // shared columns the norm kernel rewrites from Zs and the residual).
  bool contiguous = true;
  for (int64_t c = 0; c < H && contiguous; ++c) contiguous = (mask[c] != 0) == (c < n_s);
  const bool zs3 = zs_sum_setting() && pair_possible && !split && !fused && !permuted && !gemm_only && !consumer &&
                   !(a->flags & CAAT_FLAG_OVERLAP_NORM) && contiguous && n_s > 0 && n_s % 8 == 0 && H <= 4096 &&
                   a->ws_bytes >= zs_workspace(T, n_s) && static_cast<const void*>(hdst) != a->residual;
  if (consumer) {
    prm.rb_count = reinterpret_cast<unsigned int*>(wsb + wl.rb_count);
    if (!(a->flags & (CAAT_FLAG_ORDER_ROWBLOCK | CAAT_FLAG_ORDER_GROUPED))) {
      prm.order = consumer_order_setting();
      if (prm.order == 3) prm.group_m = stagger_setting();
    }
  } else if (!fused && !(a->flags & (CAAT_FLAG_ORDER_ROWBLOCK | CAAT_FLAG_ORDER_GROUPED)) && order_env_set()) {
    prm.order = consumer_order_setting();  // tuning: the same tile orders with the norm after the GEMM
    if (prm.order == 3) prm.group_m = stagger_setting();
  }
  prm.eps = a->eps;
  prm.T = static_cast<int>(T);
  prm.H = static_cast<int>(H);
  prm.Kp = static_cast<int>(Kp);
  prm.P = P;
  prm.kblk_per_rank = static_cast<int>((Kp + caat::K1_BK - 1) / caat::K1_BK);
  const int64_t tail = Kp - int64_t(prm.kblk_per_rank - 1) * caat::K1_BK;
  prm.last_k16 = static_cast<int>((tail + 15) / 16);
  prm.private_scale = a->private_scale;
  prm.timeout_ns = timeout_ns();
  prm.flags = a->flags;
  const int nblk = static_cast<int>((H + caat::K1_BN - 1) / caat::K1_BN);
  for (int nb = 0; nb < nblk; ++nb) {
    const int64_t c0 = int64_t(nb) * caat::K1_BN;
    const int64_t c1 = std::min<int64_t>(H, c0 + caat::K1_BN);
    int64_t cnt = 0;
    for (int64_t c = c0; c < c1; ++c) cnt += (*tmask)[c];
    const uint8_t cls = cnt == 0 ? 0 : (cnt == c1 - c0 ? 1 : 2);
    prm.ncls[nb] = cls;
    if (cls != 0) prm.slist[prm.nS++] = static_cast<uint16_t>(nb);
    if (cls != 1) prm.plist[prm.nPriv++] = static_cast<uint16_t>(nb);
  }
  for (int64_t c = 0; c < H; ++c)
    if ((*tmask)[c]) prm.mask_bits[c >> 5] |= 1u << (c & 31);
  prm.nslots = prm.nS + prm.nPriv;
  // Shared-sum mode in unit order 0: adjacent pure shared blocks two by two as 256 x 512 units
  // (the MMA of both halves reads one X stage: a quarter fewer operand bytes per FLOP).  The
  // first blocks of a contiguous S are pure except perhaps the last.  Only for K >= 8192 (a
  // wide unit's epilogue no longer overlaps the next wide unit's mainloop, so the mainloop must
  // be long): measured on one box, fc2-7b 0.766 -> 0.748 ms, K = 4096 0.501 -> 0.507 ms.  The
  // wide units run first and the short units after them fill the last round: the private
  // units, or without any (p = 1) the ordinary shared units, with the wide count taken from a
  // simulated schedule (fc2-7b p = 1: 0.736 -> 0.710 ms; all pairs wide: 0.751 ms).
  prm.wide = 0;
  if (zs3 && prm.order == 0 && wide_setting() != 0 && (wide_setting() == 1 || a->K >= 8192)) {
    int pure = 0;
    while (pure < prm.nS && prm.slist[pure] == pure && prm.ncls[pure] == 1) ++pure;
    prm.wide = pure / 2;
    // without private units the short ordinary shared units fill the last round: take the
    // number of wide units with the shortest simulated schedule
    if (wide_setting() < 0 && prm.nPriv == 0)
      prm.wide = wide_count_by_schedule(static_cast<int>((T + 2 * caat::K2P_BM - 1) / (2 * caat::K2P_BM)), prm.nS,
                                        pure / 2, dev->max_pairs);
  }
  // The CTA-pair kernel (256-token tiles) for all but the smallest token counts.
  const bool pair = pair_possible;
  const int major = ((a->flags & kFlagAMn) ? 1 : 0) | ((a->flags & kFlagBMn) ? 2 : 0);
  if (major != 0 && (!pair || !gemm_only || fused || major == 1)) return CAAT_ERR_UNSUPPORTED;
  const int64_t bm = pair ? 2 * caat::K2P_BM : caat::K1_BM;
  if ((T + bm - 1) / bm * (prm.nS + int64_t(P) * prm.nPriv) > INT32_MAX / 2) return CAAT_ERR_UNSUPPORTED;
  prm.T_pad = static_cast<int>((T + bm - 1) / bm * bm);
  prm.n_rb = static_cast<int>(prm.T_pad / 128 * P);
  // Mixed column blocks on the pair kernel: TMA epilogue behind per-32-row completion flags of
  // their shared tiles, when the workspace holds the flags.
  bool any_mixed = false;
  for (int nb = 0; nb < nblk; ++nb) any_mixed |= prm.ncls[nb] == 2;
  const bool merge = pair && !fused && any_mixed && a->ws_bytes >= wl.total && !zs3;
  prm.merge_mixed = merge ? 1 : 0;
  prm.sdone = merge ? reinterpret_cast<unsigned int*>(wsb + wl.sdone) : nullptr;
  const size_t zero_bytes = merge ? wl.sdone + wl.sdone_bytes : (consumer ? wl.consumer_total : wl.zeroed);

  prm.zs_mode = split ? (split->peers ? 2 : 1) : (zs3 ? 3 : 0);
  prm.zs_ns = split ? static_cast<int>(split->n_s) : (zs3 ? n_s : 0);
  if (split && split->peers) {
    const caat_tp_peers* pe = split->peers;
    for (int q = 0; q < pe->world; ++q) {
      prm.tp_recv[q] = pe->recv[q];
      prm.tp_flags[q] = pe->flags[q];
    }
    prm.tp_done = counter + 8;  // zeroed with the counters at launch
    prm.tp_world = pe->world;
    prm.tp_rank = pe->rank;
    prm.tp_w = static_cast<int>(split->n_s / pe->world);
    prm.tp_epoch = pe->epoch;
  }
  if (split && (!pair || fused || permuted || gemm_only)) return CAAT_ERR_UNSUPPORTED;
  CUtensorMap tmX, tmW, tmR, tmH, tmZ;
  // K-major operands: boxes of 64 K x (128 rows); MN-major ones: 64 MN x 64 K rows, two per half
  caat_status s = (major & 1) ? make_map_3d(&tmX, a->X, T, Kp, P, 64, caat::K2P_BK)
                              : make_map_3d(&tmX, a->X, Kp, T, P, caat::K1_BK, caat::K1_BM);
  if (s != CAAT_OK) return s;
  s = (major & 2) ? make_map_3d(&tmW, a->W, H, Kp, P, 64, caat::K2P_BK)
                  : make_map_3d(&tmW, a->W, Kp, H, P, caat::K1_BK, pair ? caat::K2P_BN / 2 : caat::K1_BN);
  if (s != CAAT_OK) return s;
  // residual in / pre-norm h out of the TMA epilogue: 32-row x 64-column boxes
  s = make_map_3d(&tmR, a->residual, H, T, P, 64, 32);
  if (s != CAAT_OK) return s;
  s = make_map_3d(&tmH, hdst, H, T, P, 64, 32);
  if (s != CAAT_OK) return s;
  // the split output's fp32 shared-channel partials: 32-row x 32-column boxes
  tmZ = tmH;
  float* zs_buf = zs3 ? reinterpret_cast<float*>(wsb + kZsOffset) : nullptr;
  if (zs3) {
    s = make_map_3d_f32(&tmZ, zs_buf, static_cast<uint64_t>(n_s), T, 1, 32, 32);
    if (s != CAAT_OK) return s;
  }
  if (split && split->n_s > 0 && !split->peers) {
    s = make_map_3d_f32(&tmZ, split->zs, static_cast<uint64_t>(split->n_s), T, 1, 32, 32);
    if (s != CAAT_OK) return s;
  }

  // One GEMM launch over the token rows [t0, t0 + tc) (t0 a multiple of the tile height).
  auto gemm = [&](int64_t t0, int64_t tc) -> caat_status {
    prm.t_begin = static_cast<int>(t0);
    prm.t_end = static_cast<int>(t0 + tc);
    prm.n_mblk = static_cast<int>((tc + bm - 1) / bm);
    const int64_t units = int64_t(prm.n_mblk) * (prm.nS - prm.wide + int64_t(P) * prm.nPriv);
    prm.n_units = static_cast<int>(units);
    if (cudaMemsetAsync(counter, 0, zero_bytes, st) != cudaSuccess) return CAAT_ERR_CUDA;
    if (pair) {
      int pairs = static_cast<int>(std::min<int64_t>(dev->max_pairs, units));
      if (consumer) pairs = std::max(1, std::min(pairs, dev->max_pairs - (norm_sms_setting() + 1) / 2));
      if (gemm_pairs_cap() > 0) pairs = std::min(pairs, gemm_pairs_cap());
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * pairs, 1, 1);
      cfg.blockDim = dim3(fused ? caat::K1Threads<true>::value : caat::K1Threads<false>::value, 1, 1);
      cfg.dynamicSmemBytes = caat::K2P_SMEM_BYTES;
      cfg.stream = st;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      // units short in K (few k-blocks per rank): the split with more epilogue buffers
      const bool epi_heavy = !fused && major == 0 && prm.kblk_per_rank <= epi_heavy_kblk_setting();
      const cudaError_t e =
          fused ? cudaLaunchKernelEx(&cfg, caat::rowpar_gemm_pair_kernel<true>, tmX, tmW, tmR, tmH, tmZ, prm)
          : epi_heavy
              ? cudaLaunchKernelEx(
                    &cfg, caat::rowpar_gemm_pair_kernel<false, 0, caat::K2P_STAGES_EPI, caat::K2P_EPI_NBUF_EPI>, tmX,
                    tmW, tmR, tmH, tmZ, prm)
          : major == 2
              ? cudaLaunchKernelEx(&cfg, caat::rowpar_gemm_pair_kernel<false, 2>, tmX, tmW, tmR, tmH, tmZ, prm)
          : major == 3
              ? cudaLaunchKernelEx(&cfg, caat::rowpar_gemm_pair_kernel<false, 3>, tmX, tmW, tmR, tmH, tmZ, prm)
              : cudaLaunchKernelEx(&cfg, caat::rowpar_gemm_pair_kernel<false>, tmX, tmW, tmR, tmH, tmZ, prm);
      if (e != cudaSuccess) return CAAT_ERR_CUDA;
    } else {
      const int grid = static_cast<int>(std::min<int64_t>(dev->sm_count, units));
      if (fused)
        caat::rowpar_gemm_kernel<true><<<grid, caat::K1Threads<true>::value, caat::K1_SMEM_BYTES, st>>>(
            tmX, tmW, tmR, tmH, prm);
      else
        caat::rowpar_gemm_kernel<false><<<grid, caat::K1Threads<false>::value, caat::K1_SMEM_BYTES, st>>>(
            tmX, tmW, tmR, tmH, prm);
    }
    return cudaGetLastError() == cudaSuccess ? CAAT_OK : CAAT_ERR_CUDA;
  };
  // The row norm of the token rows [t0, t0 + tc) of every rank, on stream `ns`.
  const __nv_bfloat16* g = reinterpret_cast<const __nv_bfloat16*>(a->gamma);
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a->out);
  auto norm = [&](int64_t t0, int64_t tc, cudaStream_t ns, int64_t max_blocks) -> caat_status {
    const int64_t rows = int64_t(P) * tc;
    if (permuted) {
      static thread_local caat::PermParams pp;
      std::memset(&pp, 0, sizeof(pp));
      pp.P = P;
      pp.H = static_cast<int>(H);
      pp.Kp = static_cast<int>(Kp);
      pp.n_s = n_s;
      pp.T = T;
      pp.eps = a->eps;
      for (int64_t c = 0; c < H; ++c)
        if (mask[c]) pp.mask_bits[c >> 5] |= 1u << (c & 31);
      const size_t smem = caat::gather_smem_bytes(static_cast<int>(H));
      const int64_t wpb = caat::K2P_THREADS / 32;
      const int64_t per_sm = H <= 2048 ? 2 : 1;  // blocks resident per SM (registers, shared memory)
      const int64_t gb = std::min<int64_t>((int64_t(P) * T + wpb - 1) / wpb, int64_t(dev->sm_count) * per_sm);
      __nv_bfloat16* hk = reinterpret_cast<__nv_bfloat16*>(a->h_out);  // may equal hdst (in place)
      const __nv_bfloat16* rr = reinterpret_cast<const __nv_bfloat16*>(a->residual);
      if (H <= 1024)
        caat::rownorm_gather_kernel<4><<<gb, caat::K2P_THREADS, smem, ns>>>(hdst, rr, hk, o, g, pp);
      else if (H <= 2048)
        caat::rownorm_gather_kernel<8><<<gb, caat::K2P_THREADS, smem, ns>>>(hdst, rr, hk, o, g, pp);
      else
        caat::rownorm_gather_kernel<16><<<gb, caat::K2P_THREADS, smem, ns>>>(hdst, rr, hk, o, g, pp);
      return cudaGetLastError() == cudaSuccess ? CAAT_OK : CAAT_ERR_CUDA;
    }
    const int64_t warps_per_block = caat::K2_THREADS / 32;
    const int64_t blocks = std::min<int64_t>((rows + warps_per_block - 1) / warps_per_block, max_blocks);
    if (zs3) {
      // one CTA per token (its ranks on the CTA's warps), the token's sums staged once.  A
      // plain launch: as a programmatic dependent of the GEMM the step took 62 us longer.
      const __nv_bfloat16* rr = reinterpret_cast<const __nv_bfloat16*>(a->residual);
      const int Hi = static_cast<int>(H);
      const int64_t fb = std::min<int64_t>(T, int64_t(dev->sm_count) * 2);
      if (H <= 1024)
        caat::rownorm_zs_kernel<4><<<fb, caat::KZ_THREADS, 0, ns>>>(zs_buf, rr, hdst, o, g, T, P, Hi, n_s, a->eps);
      else if (H <= 2048)
        caat::rownorm_zs_kernel<8><<<fb, caat::KZ_THREADS, 0, ns>>>(zs_buf, rr, hdst, o, g, T, P, Hi, n_s, a->eps);
      else
        caat::rownorm_zs_kernel<16><<<fb, caat::KZ_THREADS, 0, ns>>>(zs_buf, rr, hdst, o, g, T, P, Hi, n_s, a->eps);
      return cudaGetLastError() == cudaSuccess ? CAAT_OK : CAAT_ERR_CUDA;
    }
    if (H <= 4096) {
      // row held in registers: VPL 128-bit vectors per lane
      int64_t rb = std::min<int64_t>((rows + warps_per_block - 1) / warps_per_block, int64_t(dev->sm_count) * 2);
      if (norm_blocks_cap() > 0) rb = std::min<int64_t>(rb, norm_blocks_cap());
      if (H <= 1024)
        caat::rownorm_reg_kernel<4><<<rb, caat::K2_THREADS, 0, ns>>>(hdst, o, g, P, T, t0, tc, static_cast<int>(H), a->eps);
      else if (H <= 2048)
        caat::rownorm_reg_kernel<8><<<rb, caat::K2_THREADS, 0, ns>>>(hdst, o, g, P, T, t0, tc, static_cast<int>(H), a->eps);
      else
        caat::rownorm_reg_kernel<16><<<rb, caat::K2_THREADS, 0, ns>>>(hdst, o, g, P, T, t0, tc, static_cast<int>(H), a->eps);
    } else {
      // wide rows: one CTA per row (H <= 65536 = 8 x 1024 x 8)
      const int64_t nb = std::min<int64_t>(rows, int64_t(dev->sm_count) * 8);
      const int Hi = static_cast<int>(H);
      if (H <= 8 * 256 * 4)
        caat::rownorm_block_kernel<256, 4><<<nb, 256, 0, ns>>>(hdst, o, g, P, T, t0, tc, Hi, a->eps);
      else if (H <= 8 * 512 * 4)
        caat::rownorm_block_kernel<512, 4><<<nb, 512, 0, ns>>>(hdst, o, g, P, T, t0, tc, Hi, a->eps);
      else if (H <= 8 * 1024 * 4)
        caat::rownorm_block_kernel<1024, 4><<<nb, 1024, 0, ns>>>(hdst, o, g, P, T, t0, tc, Hi, a->eps);
      else
        caat::rownorm_block_kernel<1024, 8><<<nb, 1024, 0, ns>>>(hdst, o, g, P, T, t0, tc, Hi, a->eps);
    }
    return cudaGetLastError() == cudaSuccess ? CAAT_OK : CAAT_ERR_CUDA;
  };

  Recorder own;
  Recorder& rec = outer ? *outer : own;
  if (!outer) rec.begin(a->timing, st);
  if (consumer) {
    // GEMM, then the row norm as its programmatic dependent (no event between the two: the
    // recorder's one interval covers both kernels).
    s = gemm(0, T);
    if (s != CAAT_OK) return s;
    const int64_t pieces = int64_t(prm.n_rb) * (caat::K2C_ROWS_PER_JOB / caat::K2C_ROWS_PER_PIECE);
    const int64_t warps_per_block = caat::K2C_THREADS / 32;
    const int64_t nb = std::max<int64_t>(
        1, std::min<int64_t>((pieces + warps_per_block - 1) / warps_per_block, int64_t(dev->sm_count)));
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(nb), 1, 1);
    cfg.blockDim = dim3(caat::K2C_THREADS, 1, 1);
    cfg.dynamicSmemBytes = caat::K2C_SMEM_BYTES;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const __nv_bfloat16* hc = hdst;
    const unsigned int* rbc = prm.rb_count;
    // a (128-row block, rank) is complete after every tile of its row, from each epilogue warp
    const unsigned int target = static_cast<unsigned int>((prm.nS + prm.nPriv) * 4);
    const int n_m128 = prm.T_pad / 128;
    const int order = prm.order == 0 ? 0 : 1;
    const unsigned int* prog = counter;     // the GEMM's unit counter: its progress
    unsigned int* pc = counter + 32;        // piece counter, on its own 128-byte line
    const uint64_t tmo = prm.timeout_ns;
    const int64_t Tl = T;
    const int Hi = static_cast<int>(H);
    const float ep = a->eps;
    cudaError_t e;
    if (H <= 1024)
      e = cudaLaunchKernelEx(&cfg, caat::rownorm_consumer_kernel<4>, hc, o, g, P, Tl, Hi, ep, rbc, target, n_m128,
                             order, prog, pc, tmo);
    else if (H <= 2048)
      e = cudaLaunchKernelEx(&cfg, caat::rownorm_consumer_kernel<8>, hc, o, g, P, Tl, Hi, ep, rbc, target, n_m128,
                             order, prog, pc, tmo);
    else
      e = cudaLaunchKernelEx(&cfg, caat::rownorm_consumer_kernel<16>, hc, o, g, P, Tl, Hi, ep, rbc, target, n_m128,
                             order, prog, pc, tmo);
    if (e != cudaSuccess) return CAAT_ERR_CUDA;
    rec.after_kernel(st);
    return CAAT_OK;
  }
  const bool overlap = !fused && !permuted && !gemm_only && !split && (a->flags & CAAT_FLAG_OVERLAP_NORM) &&
                       T >= 2 * kNormChunk;
  if (!overlap) {
    s = gemm(0, T);
    if (s != CAAT_OK) return s;
    rec.after_kernel(st);
    if (fused || gemm_only || split) return CAAT_OK;
    s = norm(0, T, st, int64_t(dev->sm_count) * 4);
    if (s != CAAT_OK) return s;
    rec.after_kernel(st);
    return CAAT_OK;
  }
  // Chunked: the GEMM of chunk i + 1 runs on the caller's stream while the row norm of chunk i
  // runs on the side stream (a norm block fits on an SM beside a GEMM CTA).  Recorded
  // intervals: [start, last GEMM done], [last GEMM done, all norms done].
  NormSide* side = nullptr;
  s = norm_side(&side);
  if (s != CAAT_OK) return s;
  for (int64_t t0 = 0; t0 < T; t0 += kNormChunk) {
    const int64_t tc = std::min<int64_t>(kNormChunk, T - t0);
    s = gemm(t0, tc);
    if (s != CAAT_OK) return s;
    if (cudaEventRecord(side->ev_gemm, st) || cudaStreamWaitEvent(side->s, side->ev_gemm, 0)) return CAAT_ERR_CUDA;
    s = norm(t0, tc, side->s, dev->sm_count);
    if (s != CAAT_OK) return s;
  }
  rec.after_kernel(st);
  if (cudaEventRecord(side->ev_done, side->s) || cudaStreamWaitEvent(st, side->ev_done, 0)) return CAAT_ERR_CUDA;
  rec.after_kernel(st);
  return CAAT_OK;
}

caat_status validate_rowpar(const caat_rowpar_args* a, std::vector<uint8_t>& mask) {
  if (!a) return CAAT_ERR_INVALID_ARG;
  caat_status s = check_shapes(a->T, a->K, a->H, a->P, a->p);
  if (s != CAAT_OK) return s;
  if (!(a->eps >= 0.f) || !std::isfinite(a->eps) || !std::isfinite(a->private_scale)) return CAAT_ERR_INVALID_ARG;
  s = build_mask(a->H, a->p, a->sync_idx, mask, nullptr);
  if (s != CAAT_OK) return s;
  if (a->T == 0) return CAAT_OK;
  if (!a->X || !a->W || !a->residual || !a->gamma || !a->out) return CAAT_ERR_INVALID_ARG;
  if (!aligned16(a->X) || !aligned16(a->W) || !aligned16(a->residual) || !aligned16(a->gamma) ||
      !aligned16(a->out) || (a->h_out && !aligned16(a->h_out)))
    return CAAT_ERR_UNSUPPORTED;
  const size_t need = rowpar_workspace_min(a->T, a->H, a->P, a->flags);
  if (need > 0) {
    if (!a->workspace || a->ws_bytes < need || (reinterpret_cast<uintptr_t>(a->workspace) & 255u))
      return CAAT_ERR_WORKSPACE;
  }
  return CAAT_OK;
}


// ---------------------------------------------------------------------------------------
// Backward
// ---------------------------------------------------------------------------------------
// Workspace of caat_rowpar_backward: [GEMM counters (256 B) | dZt [P,T,H] | dZt^T [P,H,Tp] |
// X^T [P,K/P,Tp] | W^T [P,K/P,H] | dgamma partials [nb, H] fp32], Tp = T rounded up to 8.
struct BwdLayout {
  size_t dzt, dztT, xT, wT, dg, total;
  int64_t Tp;
  int nb;
};

BwdLayout bwd_layout(int64_t T, int64_t K, int64_t H, int P, int sm_count) {
  BwdLayout L{};
  const int64_t Kp = K / P;
  L.Tp = (T + 7) / 8 * 8;
  L.nb = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(T, sm_count)));
  L.dzt = kCounterBytes;
  L.dztT = L.dzt + align256(size_t(P) * T * H * 2);
  L.xT = L.dztT + align256(size_t(P) * H * L.Tp * 2);
  L.wT = L.xT + align256(size_t(P) * Kp * L.Tp * 2);
  L.dg = L.wT + align256(size_t(P) * Kp * H * 2);
  L.total = L.dg + align256(size_t(L.nb) * H * 4);
  return L;
}

// Largest SM count the backward workspace is sized for (the dgamma partials: one row per CTA).
constexpr int kBwdMaxCtas = 1024;

caat_status launch_transpose(const void* in, void* out, int64_t nbatch, int64_t R, int64_t C, int64_t Rp,
                             cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>((C + caat::KT_COLS - 1) / caat::KT_COLS),
                  static_cast<unsigned>((Rp + caat::KT_ROWS - 1) / caat::KT_ROWS), static_cast<unsigned>(nbatch));
  caat::transpose_pad_kernel<<<grid, caat::KT_THREADS, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(in),
                                                   reinterpret_cast<__nv_bfloat16*>(out), R, C, Rp);
  return cudaGetLastError() == cudaSuccess ? CAAT_OK : CAAT_ERR_CUDA;
}

// C_b = A_b B_b^T for b < nb: A [nb, M, Kr], B [nb, N, Kr] (K-major; with kFlagAMn / kFlagBMn in
// `major_flags`: A [nb, Kr, M] / B [nb, Kr, N]), C [nb, M, N] bf16, through the row-parallel GEMM
// kernel with every channel private (p = 0) and no residual.
caat_status launch_batched_gemm(const void* A, const void* B, void* Cm, int nb, int64_t M, int64_t N, int64_t Kr,
                                unsigned int* counter, cudaStream_t st, const DeviceInfo* dev, Recorder* rec,
                                uint32_t major_flags = 0) {
  caat_rowpar_args g;
  std::memset(&g, 0, sizeof(g));
  g.X = reinterpret_cast<const caat_bf16*>(A);
  g.W = reinterpret_cast<const caat_bf16*>(B);
  g.residual = reinterpret_cast<const caat_bf16*>(Cm);
  g.gamma = reinterpret_cast<const caat_bf16*>(Cm);
  g.out = reinterpret_cast<caat_bf16*>(Cm);
  g.h_out = reinterpret_cast<caat_bf16*>(Cm);
  g.workspace = counter;
  g.ws_bytes = kCounterBytes;
  g.stream = st;
  g.T = M;
  g.K = Kr * nb;
  g.H = N;
  g.p = 0.0;
  g.eps = 1e-5f;
  g.private_scale = 1.0f;
  g.P = nb;
  g.flags = CAAT_FLAG_FORCE_GEMM_PATH | kFlagGemmOnly | major_flags;
  static thread_local std::vector<uint8_t> zero_mask;
  zero_mask.assign(static_cast<size_t>(N), 0);
  return launch_rowpar(&g, zero_mask, dev, counter, rec);
}

}  // namespace

// =======================================================================================
// C ABI
// =======================================================================================
extern "C" {

const char* caat_status_string(caat_status s) {
  switch (s) {
    case CAAT_OK: return "CAAT_OK";
    case CAAT_ERR_INVALID_ARG: return "CAAT_ERR_INVALID_ARG";
    case CAAT_ERR_UNSUPPORTED: return "CAAT_ERR_UNSUPPORTED";
    case CAAT_ERR_CUDA: return "CAAT_ERR_CUDA";
    case CAAT_ERR_TIMEOUT: return "CAAT_ERR_TIMEOUT";
    case CAAT_ERR_WORKSPACE: return "CAAT_ERR_WORKSPACE";
  }
  return "CAAT_ERR_UNKNOWN";
}

const char* caat_version(void) { return "caat-b200 0.1.0 (sm_100a)"; }

caat_status caat_sync_mask(int64_t H, double p, const int32_t* sync_idx, uint8_t* mask_out, int64_t* n_sync_out) {
  if (H <= 0 || H > CAAT_MAX_H) return CAAT_ERR_INVALID_ARG;
  std::vector<uint8_t> mask;
  int64_t ns = 0;
  const caat_status s = build_mask(H, p, sync_idx, mask, &ns);
  if (s != CAAT_OK) return s;
  if (mask_out) std::memcpy(mask_out, mask.data(), static_cast<size_t>(H));
  if (n_sync_out) *n_sync_out = ns;
  return CAAT_OK;
}

caat_status caat_rowpar_backward(const caat_rowpar_bwd_args* a) {
  if (!a) return CAAT_ERR_INVALID_ARG;
  caat_status s = check_shapes(a->T, a->K, a->H, a->P, a->p);
  if (s != CAAT_OK) return s;
  if (!(a->eps >= 0.f) || !std::isfinite(a->eps) || !std::isfinite(a->private_scale)) return CAAT_ERR_INVALID_ARG;
  if (a->P > caat::KB_MAXP || a->H > int64_t(8) * caat::KB_THREADS * caat::KB_VEC) return CAAT_ERR_UNSUPPORTED;
  std::vector<uint8_t> mask;
  s = build_mask(a->H, a->p, a->sync_idx, mask, nullptr);
  if (s != CAAT_OK) return s;
  if (a->T == 0) return CAAT_OK;
  if (!a->X || !a->W || !a->h || !a->gamma || !a->dout || !a->dX || !a->dW || !a->dgamma)
    return CAAT_ERR_INVALID_ARG;
  if (!aligned16(a->X) || !aligned16(a->W) || !aligned16(a->h) || !aligned16(a->gamma) || !aligned16(a->dout) ||
      !aligned16(a->dX) || !aligned16(a->dW) || !aligned16(a->dgamma) || (a->dR && !aligned16(a->dR)))
    return CAAT_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CAAT_OK) return s;
  if (dev->sm_count > kBwdMaxCtas) return CAAT_ERR_UNSUPPORTED;
  const int P = a->P;
  const int64_t T = a->T, H = a->H, Kp = a->K / P;
  const BwdLayout L = bwd_layout(T, a->K, H, P, dev->sm_count);
  if (!a->workspace || a->ws_bytes < L.total || (reinterpret_cast<uintptr_t>(a->workspace) & 255u))
    return CAAT_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(a->workspace);
  unsigned int* counter = reinterpret_cast<unsigned int*>(ws);
  cudaStream_t st = a->stream;
  Recorder rec;
  rec.begin(a->timing, st);

  static thread_local caat::BwdParams bp;
  std::memset(&bp, 0, sizeof(bp));
  bp.h = reinterpret_cast<const __nv_bfloat16*>(a->h);
  bp.dout = reinterpret_cast<const __nv_bfloat16*>(a->dout);
  bp.gamma = reinterpret_cast<const __nv_bfloat16*>(a->gamma);
  bp.dR = reinterpret_cast<__nv_bfloat16*>(a->dR);
  bp.dZt = reinterpret_cast<__nv_bfloat16*>(ws + L.dzt);
  bp.dg_part = reinterpret_cast<float*>(ws + L.dg);
  bp.P = P;
  bp.H = static_cast<int>(H);
  bp.T = T;
  bp.eps = a->eps;
  bp.private_scale = a->private_scale;
  bp.zk_regs = bwd_zk_regs_setting() ? 1 : 0;
  for (int64_t c = 0; c < H; ++c)
    if (mask[c]) bp.mask_bits[c >> 5] |= 1u << (c & 31);
  const size_t kb_smem = caat::bwd_smem_bytes(P, static_cast<int>(H));
  if (H <= 8 * caat::KB_THREADS && kb_smem <= caat::KB_SMEM_MAX)
  {
    if (P <= 8)
      caat::rownorm_bwd_smem_kernel<8><<<L.nb, caat::KB_THREADS, kb_smem, st>>>(bp);
    else
      caat::rownorm_bwd_smem_kernel<16><<<L.nb, caat::KB_THREADS, kb_smem, st>>>(bp);
  }
  else
    caat::rownorm_bwd_kernel<<<L.nb, caat::KB_THREADS, 0, st>>>(bp);
  if (cudaGetLastError() != cudaSuccess) return CAAT_ERR_CUDA;
  rec.after_kernel(st);
  caat::dgamma_reduce_kernel<<<static_cast<unsigned>((H + 255) / 256), 256, 0, st>>>(bp.dg_part, a->dgamma, L.nb,
                                                                                     static_cast<int>(H));
  if (cudaGetLastError() != cudaSuccess) return CAAT_ERR_CUDA;
  rec.after_kernel(st);
  if (!(a->flags & CAAT_BWD_FLAG_TRANSPOSED_OPERANDS) && dev->max_pairs > 0 && T > caat::K1_BM && H > caat::K1_BM) {
    // Both gradient GEMMs on the CTA-pair kernel with MN-major operands, straight from the
    // row-major tensors: dX_m = dZt_m W_m (W_m [H][Kp] is B = [Kr=H][N=Kp]); dW_m = dZt_m^T X_m
    // (dZt_m [T][H] is A = [Kr=T][M=H], X_m [T][Kp] is B = [Kr=T][N=Kp]); the token tail of the
    // reduction is zero-filled by the tensor maps.
    s = launch_batched_gemm(ws + L.dzt, a->W, a->dX, P, T, Kp, H, counter, st, dev, &rec, kFlagBMn);
    if (s != CAAT_OK) return s;
    return launch_batched_gemm(ws + L.dzt, a->X, a->dW, P, H, Kp, T, counter, st, dev, &rec, kFlagAMn | kFlagBMn);
  }
  // Fewer than 129 tokens or channels (the one-CTA kernel, K-major operands only): transposes.
  // dX_m = dZt_m W_m = dZt_m (W_m^T)^T
  s = launch_transpose(a->W, ws + L.wT, P, H, Kp, H, st);
  if (s != CAAT_OK) return s;
  rec.after_kernel(st);
  s = launch_batched_gemm(ws + L.dzt, ws + L.wT, a->dX, P, T, Kp, H, counter, st, dev, &rec);
  if (s != CAAT_OK) return s;
  // dW_m = dZt_m^T X_m = (dZt^T)_m ((X^T)_m)^T, reduction over the (zero-padded) tokens
  s = launch_transpose(ws + L.dzt, ws + L.dztT, P, T, H, L.Tp, st);
  if (s != CAAT_OK) return s;
  rec.after_kernel(st);
  s = launch_transpose(a->X, ws + L.xT, P, T, Kp, L.Tp, st);
  if (s != CAAT_OK) return s;
  rec.after_kernel(st);
  return launch_batched_gemm(ws + L.dztT, ws + L.xT, a->dW, P, H, Kp, L.Tp, counter, st, dev, &rec);
}

caat_status caat_speedup_model(double h, double s, double r, double p, double C, double* speedup_out,
                               double* p_star_out) {
  if (!(h > 0.0) || !(s > 0.0) || !(r > 0.0) || !(C > 0.0) || !(p >= 0.0 && p <= 1.0) || !std::isfinite(h) ||
      !std::isfinite(s) || !std::isfinite(r) || !std::isfinite(C))
    return CAAT_ERR_INVALID_ARG;
  const double x = (12.0 * h + 2.0 * s) / (C * r);
  if (speedup_out) *speedup_out = (1.0 - p) / (1.0 + x);
  if (p_star_out) *p_star_out = std::min(x, 1.0);
  return CAAT_OK;
}

caat_status caat_permute_weights(const caat_bf16* W, caat_bf16* W_out, const int32_t* sync_idx, double p, int P,
                                 int64_t H, int64_t K, caat_stream_t stream) {
  caat_status s = check_shapes(0, K, H, P, p);
  if (s != CAAT_OK) return s;
  std::vector<uint8_t> mask;
  int64_t ns = 0;
  s = build_mask(H, p, sync_idx, mask, &ns);
  if (s != CAAT_OK) return s;
  if (!W || !W_out) return CAAT_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(W_out)) return CAAT_ERR_UNSUPPORTED;
  const size_t bytes = static_cast<size_t>(K) * static_cast<size_t>(H) * 2;  // P * H * (K/P) bf16
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(W), b0 = reinterpret_cast<uintptr_t>(W_out);
  if (a0 < b0 + bytes && b0 < a0 + bytes) return CAAT_ERR_INVALID_ARG;  // overlap
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CAAT_OK) return s;
  static thread_local caat::PermParams pp;
  std::memset(&pp, 0, sizeof(pp));
  pp.P = P;
  pp.H = static_cast<int>(H);
  pp.Kp = static_cast<int>(K / P);
  pp.n_s = static_cast<int>(ns);
  for (int64_t c = 0; c < H; ++c)
    if (mask[c]) pp.mask_bits[c >> 5] |= 1u << (c & 31);
  const int64_t rows = int64_t(P) * H;
  const int64_t wpb = caat::K5_THREADS / 32;
  const int64_t blocks = std::min<int64_t>((rows + wpb - 1) / wpb, int64_t(dev->sm_count) * 8);
  caat::permute_rows_kernel<<<static_cast<unsigned>(blocks), caat::K5_THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(W), reinterpret_cast<__nv_bfloat16*>(W_out), pp);
  return cudaGetLastError() == cudaSuccess ? CAAT_OK : CAAT_ERR_CUDA;
}

size_t caat_workspace_size(int64_t T, int64_t K, int64_t H, int P, int variant) {
  if (check_shapes(T, K, H, P, 0.0) != CAAT_OK) return SIZE_MAX;
  if (variant == CAAT_VARIANT_ROWPAR) return rowpar_workspace(T, K, H, P);
  if (variant == CAAT_VARIANT_ROWPAR_HOST) return host_layout(T, K, H, P).total;
  if (variant == CAAT_VARIANT_MLP) return mlp_ws_layout(T, H, K, P, true).total;
  if (variant == CAAT_VARIANT_ROWPAR_BWD) return bwd_layout(T, K, H, P, kBwdMaxCtas).total;
  return SIZE_MAX;
}

caat_status caat_rowpar_forward_ex(const caat_rowpar_args* a) {
  std::vector<uint8_t> mask;
  caat_status s = validate_rowpar(a, mask);
  if (s != CAAT_OK) return s;
  if (a->T == 0) return CAAT_OK;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CAAT_OK) return s;
  return launch_rowpar(a, mask, dev, static_cast<unsigned int*>(a->workspace));
}

}  // extern "C"

struct caat_plan {
  caat_rowpar_args args;
  std::vector<uint8_t> mask;
  DeviceInfo* dev = nullptr;
  int device = 0;
};

extern "C" {

caat_status caat_plan_create(const caat_rowpar_args* a, caat_plan** plan_out) {
  if (!plan_out) return CAAT_ERR_INVALID_ARG;
  *plan_out = nullptr;
  std::vector<uint8_t> mask;
  caat_status s = validate_rowpar(a, mask);
  if (s != CAAT_OK) return s;
  caat_plan* pl = new (std::nothrow) caat_plan();
  if (!pl) return CAAT_ERR_INVALID_ARG;
  pl->args = *a;
  pl->args.sync_idx = nullptr;  // the mask below replaces it
  pl->args.timing = nullptr;
  pl->mask = std::move(mask);
  if (a->T > 0) {
    s = device_info(&pl->dev);
    if (s != CAAT_OK || cudaGetDevice(&pl->device) != cudaSuccess) {
      delete pl;
      return s != CAAT_OK ? s : CAAT_ERR_CUDA;
    }
  }
  *plan_out = pl;
  return CAAT_OK;
}

caat_status caat_plan_execute(const caat_plan* pl, caat_stream_t stream) {
  if (!pl) return CAAT_ERR_INVALID_ARG;
  if (pl->args.T == 0) return CAAT_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CAAT_ERR_CUDA;
  if (dev != pl->device) return CAAT_ERR_INVALID_ARG;  // created for another device
  caat_rowpar_args a = pl->args;
  a.stream = stream;
  return launch_rowpar(&a, pl->mask, pl->dev, static_cast<unsigned int*>(a.workspace));
}

caat_status caat_plan_destroy(caat_plan* pl) {
  delete pl;
  return CAAT_OK;
}

caat_status caat_rowpar_forward_host(const caat_rowpar_args* a) {
  if (!a) return CAAT_ERR_INVALID_ARG;
  caat_status s = check_shapes(a->T, a->K, a->H, a->P, a->p);
  if (s != CAAT_OK) return s;
  if (!(a->eps >= 0.f) || !std::isfinite(a->eps) || !std::isfinite(a->private_scale)) return CAAT_ERR_INVALID_ARG;
  std::vector<uint8_t> mask;
  s = build_mask(a->H, a->p, a->sync_idx, mask, nullptr);
  if (s != CAAT_OK) return s;
  if (a->T == 0) return CAAT_OK;
  if (!a->X || !a->W || !a->residual || !a->gamma || !a->out) return CAAT_ERR_INVALID_ARG;
  const int P = a->P;
  const int64_t T = a->T, H = a->H, Kp = a->K / P;
  const HostLayout L = host_layout(T, a->K, H, P);
  if (!a->workspace || a->ws_bytes < L.total || (reinterpret_cast<uintptr_t>(a->workspace) & 255u))
    return CAAT_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CAAT_OK) return s;
  HostPipe* hp = nullptr;
  s = host_pipe(&hp);
  if (s != CAAT_OK) return s;
  uint8_t* base = static_cast<uint8_t*>(a->workspace);
  cudaStream_t st = a->stream;
  const uint8_t* hX = reinterpret_cast<const uint8_t*>(a->X);
  const uint8_t* hR = reinterpret_cast<const uint8_t*>(a->residual);
  uint8_t* hO = reinterpret_cast<uint8_t*>(a->out);
  uint8_t* hH = reinterpret_cast<uint8_t*>(a->h_out);

  // Copies start after the work already queued on the caller's stream (which may still use
  // this workspace).
  if (cudaEventRecord(hp->ev_start, st) != cudaSuccess || cudaStreamWaitEvent(hp->s_in, hp->ev_start, 0) ||
      cudaStreamWaitEvent(hp->s_out, hp->ev_start, 0))
    return CAAT_ERR_CUDA;
  if (cudaMemcpyAsync(base + L.w, a->W, size_t(P) * H * Kp * 2, cudaMemcpyHostToDevice, hp->s_in) ||
      cudaMemcpyAsync(base + L.g, a->gamma, size_t(H) * 2, cudaMemcpyHostToDevice, hp->s_in) ||
      cudaEventRecord(hp->ev_w, hp->s_in) || cudaStreamWaitEvent(st, hp->ev_w, 0))
    return CAAT_ERR_CUDA;

  // Chunks of L.Tc tokens, the last ones halving (to 256): the copy back of the final chunk
  // is the pipeline's tail, after every upload and kernel.  No chunk is left below 256 tokens
  // (a remainder that small joins the chunk before it), so every chunk of a multi-chunk call
  // takes the GEMM path, whose workspace the per-chunk region is sized for.
  std::vector<int64_t> starts;
  for (int64_t t0 = 0; t0 < T;) {
    const int64_t rem = T - t0;
    int64_t tc = rem >= 2 * L.Tc ? L.Tc : std::max<int64_t>(256, (rem / 2 + 255) / 256 * 256);
    if (rem - tc < 256) tc = rem;
    starts.push_back(t0);
    t0 += tc;
  }
  starts.push_back(T);
  const int64_t nch = static_cast<int64_t>(starts.size()) - 1;
  for (int64_t i = 0; i < nch; ++i) {
    const int b = static_cast<int>(i & 1);
    const int64_t t0 = starts[i];
    const int64_t tc = starts[i + 1] - t0;
    uint8_t* buf = base + L.buf0 + size_t(b) * L.buf_bytes;
    // H2D of the chunk's X and R rows (P strided blocks each)
    if (i >= 2 && cudaStreamWaitEvent(hp->s_in, hp->ev_comp[b], 0)) return CAAT_ERR_CUDA;
    if (cudaMemcpy2DAsync(buf + L.x, size_t(tc) * Kp * 2, hX + size_t(t0) * Kp * 2, size_t(T) * Kp * 2,
                          size_t(tc) * Kp * 2, P, cudaMemcpyHostToDevice, hp->s_in) ||
        cudaMemcpy2DAsync(buf + L.r, size_t(tc) * H * 2, hR + size_t(t0) * H * 2, size_t(T) * H * 2,
                          size_t(tc) * H * 2, P, cudaMemcpyHostToDevice, hp->s_in) ||
        cudaEventRecord(hp->ev_in[b], hp->s_in))
      return CAAT_ERR_CUDA;
    // kernels of the chunk on the caller's stream
    if (cudaStreamWaitEvent(st, hp->ev_in[b], 0)) return CAAT_ERR_CUDA;
    if (i >= 2 && cudaStreamWaitEvent(st, hp->ev_out[b], 0)) return CAAT_ERR_CUDA;
    caat_rowpar_args d = *a;
    d.X = reinterpret_cast<const caat_bf16*>(buf + L.x);
    d.W = reinterpret_cast<const caat_bf16*>(base + L.w);
    d.residual = reinterpret_cast<const caat_bf16*>(buf + L.r);
    d.gamma = reinterpret_cast<const caat_bf16*>(base + L.g);
    d.out = reinterpret_cast<caat_bf16*>(buf + L.o);
    d.h_out = a->h_out ? reinterpret_cast<caat_bf16*>(buf + L.h) : nullptr;
    d.workspace = base;
    d.ws_bytes = L.w;
    d.T = tc;
    std::vector<uint8_t> m2;
    s = validate_rowpar(&d, m2);
    if (s != CAAT_OK) return s;
    s = launch_rowpar(&d, mask, dev, reinterpret_cast<unsigned int*>(base));
    if (s != CAAT_OK) return s;
    if (cudaEventRecord(hp->ev_comp[b], st)) return CAAT_ERR_CUDA;
    // D2H of the chunk's out (and h) rows
    if (cudaStreamWaitEvent(hp->s_out, hp->ev_comp[b], 0) ||
        cudaMemcpy2DAsync(hO + size_t(t0) * H * 2, size_t(T) * H * 2, buf + L.o, size_t(tc) * H * 2,
                          size_t(tc) * H * 2, P, cudaMemcpyDeviceToHost, hp->s_out))
      return CAAT_ERR_CUDA;
    if (hH && cudaMemcpy2DAsync(hH + size_t(t0) * H * 2, size_t(T) * H * 2, buf + L.h, size_t(tc) * H * 2,
                                size_t(tc) * H * 2, P, cudaMemcpyDeviceToHost, hp->s_out))
      return CAAT_ERR_CUDA;
    if (cudaEventRecord(hp->ev_out[b], hp->s_out)) return CAAT_ERR_CUDA;
  }
  // The call is complete on the caller's stream once the last copies back are done.
  if (cudaStreamWaitEvent(st, hp->ev_out[(nch - 1) & 1], 0)) return CAAT_ERR_CUDA;
  if (nch > 1 && cudaStreamWaitEvent(st, hp->ev_out[nch & 1], 0)) return CAAT_ERR_CUDA;
  return CAAT_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// The layer over real devices, one tensor-parallel rank per GPU
// ---------------------------------------------------------------------------------------
namespace {

// `local`: the local step's arguments (K_r is checked only there).
caat_status validate_tp(const caat_tp_args* a, int64_t* n_s_out, bool local) {
  if (!a) return CAAT_ERR_INVALID_ARG;
  if (a->T < 0 || (local && a->K_r <= 0) || a->H <= 0 || !(a->p >= 0.0 && a->p <= 1.0)) return CAAT_ERR_INVALID_ARG;
  if (!(a->eps >= 0.f) || !std::isfinite(a->eps) || !std::isfinite(a->private_scale)) return CAAT_ERR_INVALID_ARG;
  if ((local && (a->K_r % 8 != 0 || a->K_r > (int64_t(1) << 30))) || a->H % 8 != 0 || a->H > 4096 ||
      a->T > (int64_t(1) << 30))
    return CAAT_ERR_UNSUPPORTED;
  const int64_t ns = n_sync_of(a->H, a->p);
  if (ns % 8 != 0) return CAAT_ERR_UNSUPPORTED;
  *n_s_out = ns;
  return CAAT_OK;
}

}  // namespace

extern "C" {

caat_status caat_rowpar_tp_local(const caat_tp_args* a) {
  int64_t ns = 0;
  caat_status s = validate_tp(a, &ns, true);
  if (s != CAAT_OK) return s;
  if (a->T == 0) return CAAT_OK;
  if (!a->X || !a->W || !a->residual || !a->h || (ns > 0 && !a->zs)) return CAAT_ERR_INVALID_ARG;
  if (!aligned16(a->X) || !aligned16(a->W) || !aligned16(a->residual) || !aligned16(a->h) ||
      (ns > 0 && !aligned16(a->zs)))
    return CAAT_ERR_UNSUPPORTED;
  if (!a->workspace || a->ws_bytes < kCounterBytes || (reinterpret_cast<uintptr_t>(a->workspace) & 255u))
    return CAAT_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CAAT_OK) return s;
  if (dev->max_pairs <= 0) return CAAT_ERR_UNSUPPORTED;
  // One rank, every channel a private tile; the split epilogue decides per 64-channel chunk.
  caat_rowpar_args r;
  std::memset(&r, 0, sizeof(r));
  r.X = a->X;
  r.W = a->W;
  r.residual = a->residual;
  r.gamma = a->residual;  // unused by the split mode
  r.out = a->h;
  r.h_out = a->h;
  r.workspace = a->workspace;
  r.ws_bytes = kCounterBytes;
  r.stream = a->stream;
  r.timing = a->timing;
  r.T = a->T;
  r.K = a->K_r;
  r.H = a->H;
  r.p = 0.0;
  r.eps = a->eps;
  r.private_scale = a->private_scale;
  r.P = 1;
  r.flags = CAAT_FLAG_FORCE_GEMM_PATH;
  static thread_local std::vector<uint8_t> zero_mask;
  zero_mask.assign(static_cast<size_t>(a->H), 0);
  const TpSplit split{a->zs, ns, nullptr};
  return launch_rowpar(&r, zero_mask, dev, static_cast<unsigned int*>(a->workspace), nullptr, &split);
}

}  // extern "C"

namespace {

// The peer-memory exchange's descriptor: world, rank, epoch and the per-rank buffers.
caat_status validate_peers(const caat_tp_peers* pe, int64_t ns) {
  if (!pe) return CAAT_ERR_INVALID_ARG;
  if (pe->world < 1 || pe->world > CAAT_TP_MAX_WORLD || pe->rank < 0 || pe->rank >= pe->world || pe->epoch == 0)
    return CAAT_ERR_INVALID_ARG;
  if (ns % (32 * int64_t(pe->world)) != 0) return CAAT_ERR_UNSUPPORTED;
  for (int q = 0; q < pe->world; ++q) {
    if (!pe->recv[q] || !pe->gather[q] || !pe->flags[q]) return CAAT_ERR_INVALID_ARG;
    if (!aligned16(pe->recv[q]) || !aligned16(pe->gather[q]) || (reinterpret_cast<uintptr_t>(pe->flags[q]) & 3u))
      return CAAT_ERR_UNSUPPORTED;
  }
  return CAAT_OK;
}

// The finishing kernel over zs, optionally after waiting for `wait_n` flags to reach `epoch`.
caat_status tp_finish_launch(const caat_tp_args* a, int64_t ns, const float* z, const unsigned int* wait_flags,
                             int wait_n, uint32_t epoch) {
  if (!a->residual || !a->gamma || !a->h || !a->out || (ns > 0 && !z)) return CAAT_ERR_INVALID_ARG;
  if (!aligned16(a->residual) || !aligned16(a->gamma) || !aligned16(a->h) || !aligned16(a->out) ||
      (ns > 0 && !aligned16(z)))
    return CAAT_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  caat_status s = device_info(&dev);
  if (s != CAAT_OK) return s;
  Recorder rec;
  rec.begin(a->timing, a->stream);
  const int64_t warps = caat::KT_FIN_THREADS / 32;
  const int64_t nb = std::max<int64_t>(1, std::min<int64_t>((a->T + warps - 1) / warps, int64_t(dev->sm_count) * 4));
  const __nv_bfloat16* R = reinterpret_cast<const __nv_bfloat16*>(a->residual);
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(a->h);
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a->out);
  const __nv_bfloat16* g = reinterpret_cast<const __nv_bfloat16*>(a->gamma);
  const int Hi = static_cast<int>(a->H), nsi = static_cast<int>(ns);
  cudaStream_t st = a->stream;
  const uint64_t tmo = timeout_ns();
  if (a->H <= 1024)
    caat::tp_finish_kernel<4><<<nb, caat::KT_FIN_THREADS, 0, st>>>(z, R, h, o, g, a->T, Hi, nsi, a->eps, wait_flags,
                                                                   wait_n, epoch, tmo, a->T, 1);
  else if (a->H <= 2048)
    caat::tp_finish_kernel<8><<<nb, caat::KT_FIN_THREADS, 0, st>>>(z, R, h, o, g, a->T, Hi, nsi, a->eps, wait_flags,
                                                                   wait_n, epoch, tmo, a->T, 1);
  else
    caat::tp_finish_kernel<16><<<nb, caat::KT_FIN_THREADS, 0, st>>>(z, R, h, o, g, a->T, Hi, nsi, a->eps,
                                                                    wait_flags, wait_n, epoch, tmo, a->T, 1);
  if (cudaGetLastError() != cudaSuccess) return CAAT_ERR_CUDA;
  rec.after_kernel(st);
  return CAAT_OK;
}

}  // namespace

extern "C" {

caat_status caat_rowpar_tp_finish(const caat_tp_args* a) {
  int64_t ns = 0;
  caat_status s = validate_tp(a, &ns, false);
  if (s != CAAT_OK) return s;
  if (a->T == 0) return CAAT_OK;
  return tp_finish_launch(a, ns, a->zs, nullptr, 0, 0);
}

caat_status caat_rowpar_tp_local_push(const caat_tp_args* a, const caat_tp_peers* pe) {
  int64_t ns = 0;
  caat_status s = validate_tp(a, &ns, true);
  if (s != CAAT_OK) return s;
  s = validate_peers(pe, ns);
  if (s != CAAT_OK) return s;
  if (a->T == 0) return CAAT_OK;
  if (!a->X || !a->W || !a->residual || !a->h) return CAAT_ERR_INVALID_ARG;
  if (!aligned16(a->X) || !aligned16(a->W) || !aligned16(a->residual) || !aligned16(a->h))
    return CAAT_ERR_UNSUPPORTED;
  if (!a->workspace || a->ws_bytes < kCounterBytes || (reinterpret_cast<uintptr_t>(a->workspace) & 255u))
    return CAAT_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CAAT_OK) return s;
  if (dev->max_pairs <= 0) return CAAT_ERR_UNSUPPORTED;
  caat_rowpar_args r;
  std::memset(&r, 0, sizeof(r));
  r.X = a->X;
  r.W = a->W;
  r.residual = a->residual;
  r.gamma = a->residual;  // unused by the split mode
  r.out = a->h;
  r.h_out = a->h;
  r.workspace = a->workspace;
  r.ws_bytes = kCounterBytes;
  r.stream = a->stream;
  r.timing = a->timing;
  r.T = a->T;
  r.K = a->K_r;
  r.H = a->H;
  r.p = 0.0;
  r.eps = a->eps;
  r.private_scale = a->private_scale;
  r.P = 1;
  r.flags = CAAT_FLAG_FORCE_GEMM_PATH;
  static thread_local std::vector<uint8_t> zero_mask;
  zero_mask.assign(static_cast<size_t>(a->H), 0);
  // no shared channels: nothing crosses devices, and the other two steps do not wait
  const TpSplit split{nullptr, ns, ns > 0 ? pe : nullptr};
  return launch_rowpar(&r, zero_mask, dev, static_cast<unsigned int*>(a->workspace), nullptr, &split);
}

caat_status caat_rowpar_tp_reduce(const caat_tp_args* a, const caat_tp_peers* pe) {
  int64_t ns = 0;
  caat_status s = validate_tp(a, &ns, false);
  if (s != CAAT_OK) return s;
  s = validate_peers(pe, ns);
  if (s != CAAT_OK) return s;
  if (a->T == 0 || ns == 0) return CAAT_OK;
  if (!a->workspace || a->ws_bytes < kCounterBytes || (reinterpret_cast<uintptr_t>(a->workspace) & 255u))
    return CAAT_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CAAT_OK) return s;
  caat::TpReduceParams rp{};
  rp.recv = pe->recv[pe->rank];
  for (int q = 0; q < pe->world; ++q) {
    rp.gather[q] = pe->gather[q];
    rp.flags[q] = pe->flags[q];
  }
  rp.done = static_cast<unsigned int*>(a->workspace);
  rp.T = a->T;
  rp.w = static_cast<int>(ns / pe->world);
  rp.n_s = static_cast<int>(ns);
  rp.world = pe->world;
  rp.rank = pe->rank;
  rp.epoch = pe->epoch;
  rp.timeout_ns = timeout_ns();
  const int64_t n4 = a->T * (rp.w / 4);
  const int64_t nb =
      std::max<int64_t>(1, std::min<int64_t>((n4 + caat::KT_RED_THREADS - 1) / caat::KT_RED_THREADS,
                                             int64_t(dev->sm_count) * 4));
  Recorder rec;
  rec.begin(a->timing, a->stream);
  if (cudaMemsetAsync(a->workspace, 0, 4, a->stream) != cudaSuccess) return CAAT_ERR_CUDA;
  caat::tp_reduce_kernel<<<static_cast<unsigned>(nb), caat::KT_RED_THREADS, 0, a->stream>>>(rp);
  if (cudaGetLastError() != cudaSuccess) return CAAT_ERR_CUDA;
  rec.after_kernel(a->stream);
  return CAAT_OK;
}

caat_status caat_rowpar_tp_finish_wait(const caat_tp_args* a, const caat_tp_peers* pe) {
  int64_t ns = 0;
  caat_status s = validate_tp(a, &ns, false);
  if (s != CAAT_OK) return s;
  s = validate_peers(pe, ns);
  if (s != CAAT_OK) return s;
  if (a->T == 0) return CAAT_OK;
  if (ns == 0) return tp_finish_launch(a, 0, nullptr, nullptr, 0, 0);
  return tp_finish_launch(a, ns, pe->gather[pe->rank], pe->flags[pe->rank] + pe->world, pe->world, pe->epoch);
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Entry point without any device allocation: the scratch is a fixed device array.
// ---------------------------------------------------------------------------------------
namespace {

// Scratch of caat_rowpar_forward_noalloc, shared by every call of that entry point on a
// device: whatever workspace the path a call takes needs (the GEMM's unit counter, the
// row-block counters and job list of the norm running beside the GEMM, the mixed-block flags,
// the fused norm's counters and partials, the decode path's fp32 partials), when it fits.  In
// host code `g_noalloc_scratch` is only a host-side stand-in for the symbol: the kernels get its
// device address, looked up with cudaGetSymbolAddress once per device (and again if the
// device's context was replaced, e.g. after a device reset).
static __device__ __align__(256) unsigned char g_noalloc_scratch[CAAT_NOALLOC_SCRATCH_BYTES];

void* g_noalloc_ptr[64];
CUcontext g_noalloc_ctx[64];
bool g_noalloc_ready[64];

caat_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CAAT_ERR_CUDA;
  if (dev < 0 || dev >= 64) return CAAT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  const CUcontext ctx = current_context();
  if (!g_noalloc_ready[dev] || g_noalloc_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return CAAT_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = ctx;
    g_noalloc_ready[dev] = true;
  }
  *out = g_noalloc_ptr[dev];
  return CAAT_OK;
}

}  // namespace

extern "C" {

caat_status caat_rowpar_forward_noalloc(const caat_rowpar_args* a) {
  if (!a) return CAAT_ERR_INVALID_ARG;
  // Per-thread host buffer for the sync mask: after the first call of a thread it is reused
  // without growing (its capacity only increases for a larger H).
  static thread_local std::vector<uint8_t> mask;
  caat_rowpar_args d = *a;
  d.workspace = nullptr;
  d.ws_bytes = 0;
  caat_status s = check_shapes(d.T, d.K, d.H, d.P, d.p);
  if (s != CAAT_OK) return s;
  if (d.T == 0) return validate_rowpar(&d, mask);
  // The fused RMSNorm needs scratch that grows with T; when it does not fit the built-in
  // array, the norm runs as the separate row kernel, which needs only the unit counter.
  if ((d.flags & CAAT_FLAG_FUSED_NORM) &&
      rowpar_workspace_min(d.T, d.H, d.P, d.flags) > CAAT_NOALLOC_SCRATCH_BYTES)
    d.flags &= ~CAAT_FLAG_FUSED_NORM;
  // Likewise the decode path's fp32 partials (4 P T H bytes): a decode-sized call whose partials
  // do not fit takes the GEMM path (unless the caller forces the decode path).
  if (takes_decode_path(d.T, d.P, d.H, d.flags) && !(d.flags & CAAT_FLAG_FORCE_DECODE_PATH) &&
      decode_workspace(d.T, d.H, d.P) > CAAT_NOALLOC_SCRATCH_BYTES)
    d.flags |= CAAT_FLAG_FORCE_GEMM_PATH;
  if (rowpar_workspace_min(d.T, d.H, d.P, d.flags) > CAAT_NOALLOC_SCRATCH_BYTES) return CAAT_ERR_WORKSPACE;
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != CAAT_OK) return s;
  d.workspace = scratch;
  d.ws_bytes = CAAT_NOALLOC_SCRATCH_BYTES;
  s = validate_rowpar(&d, mask);
  if (s != CAAT_OK) return s;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CAAT_OK) return s;
  // launch_rowpar zeroes the counter (cudaMemsetAsync on the stream) before the GEMM kernel.
  return launch_rowpar(&d, mask, dev, static_cast<unsigned int*>(scratch));
}

caat_status caat_rowpar_forward(const caat_bf16* X, const caat_bf16* W, const caat_bf16* residual,
                                const caat_bf16* gamma, const int32_t* sync_idx, int P, double p, caat_bf16* out,
                                int64_t T, int64_t K, int64_t H, void* workspace, size_t ws_bytes,
                                caat_stream_t stream) {
  caat_rowpar_args a;
  std::memset(&a, 0, sizeof(a));
  a.X = X;
  a.W = W;
  a.residual = residual;
  a.gamma = gamma;
  a.sync_idx = sync_idx;
  a.out = out;
  a.workspace = workspace;
  a.ws_bytes = ws_bytes;
  a.stream = stream;
  a.T = T;
  a.K = K;
  a.H = H;
  a.p = p;
  a.eps = 1e-5f;
  a.private_scale = 1.0f;
  a.P = P;
  return caat_rowpar_forward_ex(&a);
}

caat_status caat_mlp_forward_ex(const caat_mlp_args* a) {
  if (!a) return CAAT_ERR_INVALID_ARG;
  caat_status s = check_shapes(a->T, a->F, a->H, a->P, a->p);
  if (s != CAAT_OK) return s;
  if (!(a->eps >= 0.f) || !std::isfinite(a->eps) || !std::isfinite(a->private_scale)) return CAAT_ERR_INVALID_ARG;
  std::vector<uint8_t> mask;
  s = build_mask(a->H, a->p, a->sync_idx, mask, nullptr);
  if (s != CAAT_OK) return s;
  if (a->T == 0) return CAAT_OK;
  if (!a->X || !a->A || !a->W2 || !a->residual || !a->gamma || !a->out) return CAAT_ERR_INVALID_ARG;
  if (!aligned16(a->X) || !aligned16(a->A) || !aligned16(a->W2) || !aligned16(a->residual) || !aligned16(a->gamma) ||
      !aligned16(a->out) || (a->h_out && !aligned16(a->h_out)))
    return CAAT_ERR_UNSUPPORTED;
  const bool fused = (a->flags & CAAT_FLAG_FUSED_NORM) != 0;
  const MlpWs L = mlp_ws_layout(a->T, a->H, a->F, a->P, fused);
  if (!a->workspace || a->ws_bytes < L.total || (reinterpret_cast<uintptr_t>(a->workspace) & 255u))
    return CAAT_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  s = device_info(&dev);
  if (s != CAAT_OK) return s;
  if (dev->max_pairs <= 0) return CAAT_ERR_UNSUPPORTED;

  const int P = a->P;
  const int64_t T = a->T, H = a->H, Fp = a->F / P;
  uint8_t* ws = static_cast<uint8_t*>(a->workspace);
  caat_bf16* Y = reinterpret_cast<caat_bf16*>(ws + L.y);
  cudaStream_t st = a->stream;

  // FC1 + SwiGLU: Y_m = silu(X_m A_gate,m^T) * (X_m A_up,m^T)
  caat::Fc1Params fp{};
  fp.counter = reinterpret_cast<unsigned int*>(ws);
  fp.T = static_cast<int>(T);
  fp.H = static_cast<int>(H);
  fp.Fp = static_cast<int>(Fp);
  fp.P = P;
  fp.n_mblk = static_cast<int>((T + 2 * caat::K3_BM - 1) / (2 * caat::K3_BM));
  fp.n_nblk = static_cast<int>((Fp + caat::K3_BN - 1) / caat::K3_BN);
  fp.kblk = static_cast<int>((H + caat::K3_BK - 1) / caat::K3_BK);
  const int64_t tail = H - int64_t(fp.kblk - 1) * caat::K3_BK;
  fp.last_k16 = static_cast<int>((tail + 15) / 16);
  const int64_t units = int64_t(P) * fp.n_mblk * fp.n_nblk;
  if (units > INT32_MAX / 2) return CAAT_ERR_UNSUPPORTED;
  fp.n_units = static_cast<int>(units);
  fp.timeout_ns = timeout_ns();
  fp.flags = a->flags;
  CUtensorMap tmX, tmA, tmY;
  s = make_map_3d(&tmX, a->X, H, T, P, caat::K3_BK, caat::K3_BM);
  if (s != CAAT_OK) return s;
  s = make_map_4d(&tmA, a->A, H, Fp, 2, P, caat::K3_BK, caat::K3_BN);
  if (s != CAAT_OK) return s;
  s = make_map_3d(&tmY, Y, Fp, T, P, 64, 32);
  if (s != CAAT_OK) return s;

  Recorder rec;
  rec.begin(a->timing, st);
  if (cudaMemsetAsync(ws, 0, kCounterBytes, st) != cudaSuccess) return CAAT_ERR_CUDA;
  {
    const int pairs = static_cast<int>(std::min<int64_t>(dev->max_pairs, units));
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(caat::K3_THREADS, 1, 1);
    cfg.dynamicSmemBytes = caat::K3_SMEM_BYTES;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, caat::fc1_swiglu_pair_kernel, tmX, tmA, tmY, fp) != cudaSuccess) return CAAT_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return CAAT_ERR_CUDA;
  }
  rec.after_kernel(st);

  // FC2: the partially synchronized row-parallel layer on Y
  caat_rowpar_args r;
  std::memset(&r, 0, sizeof(r));
  r.X = Y;
  r.W = a->W2;
  r.residual = a->residual;
  r.gamma = a->gamma;
  r.out = a->out;
  r.h_out = a->h_out;
  r.workspace = ws + L.rowpar;
  r.ws_bytes = L.y - L.rowpar;
  r.stream = st;
  r.T = T;
  r.K = a->F;
  r.H = H;
  r.p = a->p;
  r.eps = a->eps;
  r.private_scale = a->private_scale;
  r.P = P;
  r.flags = a->flags;
  return launch_rowpar(&r, mask, dev, reinterpret_cast<unsigned int*>(ws + L.rowpar), &rec);
}

caat_status caat_mlp_forward(const caat_bf16* X, const caat_bf16* A, const caat_bf16* W2, const caat_bf16* residual,
                             const caat_bf16* gamma, const int32_t* sync_idx, int P, double p, caat_bf16* out,
                             int64_t T, int64_t H, int64_t F, void* workspace, size_t ws_bytes,
                             caat_stream_t stream) {
  caat_mlp_args a;
  std::memset(&a, 0, sizeof(a));
  a.X = X;
  a.A = A;
  a.W2 = W2;
  a.residual = residual;
  a.gamma = gamma;
  a.sync_idx = sync_idx;
  a.out = out;
  a.workspace = workspace;
  a.ws_bytes = ws_bytes;
  a.stream = stream;
  a.T = T;
  a.H = H;
  a.F = F;
  a.p = p;
  a.eps = 1e-5f;
  a.private_scale = 1.0f;
  a.P = P;
  return caat_mlp_forward_ex(&a);
}

caat_status caat_get_device_status(caat_stream_t stream, int32_t* status_out) {
  if (!status_out) return CAAT_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return CAAT_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, caat::g_status_word, sizeof(int)) != cudaSuccess) return CAAT_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(caat::g_status_word, &zero, sizeof(int)) != cudaSuccess) return CAAT_ERR_CUDA;
  *status_out = v;
  return (v & 0xFF) == 0 ? CAAT_OK : static_cast<caat_status>(v & 0xFF);
}

caat_status caat_timing_create(int capacity, caat_timing** out) {
  if (capacity <= 0 || capacity > (1 << 20) || !out) return CAAT_ERR_INVALID_ARG;
  caat_timing* t = new caat_timing();
  t->capacity = capacity;
  t->ev.resize(static_cast<size_t>(capacity) * (t->max_kernels + 1), nullptr);
  t->nk.assign(static_cast<size_t>(capacity), 0);
  for (auto& e : t->ev) {
    if (cudaEventCreate(&e) != cudaSuccess) {
      caat_timing_destroy(t);
      return CAAT_ERR_CUDA;
    }
  }
  *out = t;
  return CAAT_OK;
}

caat_status caat_timing_destroy(caat_timing* t) {
  if (!t) return CAAT_ERR_INVALID_ARG;
  for (auto& e : t->ev)
    if (e) cudaEventDestroy(e);
  delete t;
  return CAAT_OK;
}

caat_status caat_timing_reset(caat_timing* t) {
  if (!t) return CAAT_ERR_INVALID_ARG;
  t->n = 0;
  std::fill(t->nk.begin(), t->nk.end(), 0);
  return CAAT_OK;
}

caat_status caat_timing_read(caat_timing* t, float* ms, int max_records, int max_kernels, int* n_records,
                             int* n_kernels) {
  if (!t || !ms || max_records <= 0 || max_kernels <= 0) return CAAT_ERR_INVALID_ARG;
  const int nr = std::min(t->n, max_records);
  int nk_max = 0;
  for (int r = 0; r < nr; ++r) {
    const int nk = t->nk[r];
    nk_max = std::max(nk_max, nk);
    if (nk == 0) continue;
    cudaEvent_t* e = &t->ev[static_cast<size_t>(r) * (t->max_kernels + 1)];
    if (cudaEventSynchronize(e[nk]) != cudaSuccess) return CAAT_ERR_CUDA;
    for (int k = 0; k < std::min(nk, max_kernels); ++k) {
      float v = 0.f;
      if (cudaEventElapsedTime(&v, e[k], e[k + 1]) != cudaSuccess) return CAAT_ERR_CUDA;
      ms[r * max_kernels + k] = v;
    }
  }
  if (n_records) *n_records = nr;
  if (n_kernels) *n_kernels = nk_max;
  return CAAT_OK;
}

}  // extern "C"
