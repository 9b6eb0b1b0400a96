/*
 * caat.h - C ABI of the B200 (sm_100a) library for the partially synchronized
 * row-parallel linear layer of CAAT-Net.
 *
 * Source of every operation: "Tensor-Parallelism with Partially Synchronized Activations"
 * (Lamprecht, Karnieli, Hanani, Giladi, Soudry; arXiv 2506.19645).
 *
 *   - P tensor-parallel ranks are emulated side by side in one GPU's memory, as the paper's
 *     "logical devices" (§3.2): the partial channel-reduce becomes an on-chip sum.
 *   - Partial products: Zt_m = X_m W_m^T over rank m's K/P slice (§3.1 Eq. 4-5, App. A.2
 *     Eq. 21-22; W_m is the row-parallel block B~_m, stored transposed).
 *   - Partial channel-reduce (App. A.2 Eq. 22; §3.1 Eq. 8): for the shared channels
 *     c in S, |S| = floor(H p), every rank gets sum_m Zt_m[:, c]; the private channels keep
 *     the rank's own Zt_m[:, c], optionally times private_scale (§4 Eq. 14-15: sqrt(P)).
 *   - Residual add and norm (§4 Eq. 9, App. B Eq. 25): h_m = Z_m + R_m, then RMSNorm per
 *     rank and token, out_m = h_m / sqrt(mean_c h_m^2 + eps) * gamma (gamma shared by the
 *     ranks, since norm parameters are synchronized, §4).
 *   - MLP block (§3.1 Eq. 6 with sigma = SwiGLU): Y_m = silu(X_m A_gate,m^T) * (X_m A_up,m^T),
 *     then the layer above with X := Y.
 *   - Backward of the layer (§4 Eq. 10-13): the norm derivative per rank, then the reduction
 *     over ranks of the shared channels' gradients, then the gradients of the partial products.
 *   - Speed-up model of partial synchronization (App. C Eq. 31-35), host only.
 *
 * Conventions for every call below
 *   - bf16 tensors are raw bfloat16 bit patterns (caat_bf16), row-major, last dim contiguous.
 *   - Device pointers are owned by the caller, must be 16-byte aligned and stay valid until
 *     the work queued on `stream` has finished.  The library never allocates device memory
 *     and never synchronizes the stream in a forward call.
 *   - Every forward call validates all arguments on the host first; an invalid call queues
 *     no work and returns an error code.  No call throws across the ABI.
 *   - Work is queued asynchronously on `stream` (a cudaStream_t; NULL = legacy default).
 *   - Device-side waits are bounded: a wait that runs out (2 s; the environment variable
 *     CAAT_TIMEOUT_MS overrides) records CAAT_ERR_TIMEOUT in a device status word, which
 *     caat_get_device_status() reads.
 */
#ifndef CAAT_H_
#define CAAT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(CAAT_BUILD) && defined(__GNUC__)
#define CAAT_API __attribute__((visibility("default")))
#else
#define CAAT_API
#endif

typedef uint16_t caat_bf16;                   /* bfloat16 bit pattern */
typedef struct CUstream_st* caat_stream_t;    /* identical to cudaStream_t */
typedef struct caat_timing caat_timing;       /* opaque per-kernel event recorder */

typedef enum caat_status {
  CAAT_OK = 0,
  CAAT_ERR_INVALID_ARG = 1,   /* a pointer, size or value is invalid (nothing queued) */
  CAAT_ERR_UNSUPPORTED = 2,   /* valid, but outside what the kernels handle (alignment,
                                 divisibility, limits) or no sm_100 device */
  CAAT_ERR_CUDA = 3,          /* a CUDA runtime call failed */
  CAAT_ERR_TIMEOUT = 4,       /* a bounded device-side wait ran out (read from the device) */
  CAAT_ERR_WORKSPACE = 5      /* workspace NULL, misaligned or smaller than required */
} caat_status;

/* Limits of this build. */
#define CAAT_MAX_H 65536      /* hidden size H */
#define CAAT_MAX_P 64         /* emulated tensor-parallel ranks */
#define CAAT_DECODE_MAX_T 64  /* 1 <= T <= this (with P <= 16, H <= 8192) uses the decode
                                 (weight-streaming) path */

/* Workspace variants for caat_workspace_size(). */
#define CAAT_VARIANT_ROWPAR 0 /* caat_rowpar_forward[_ex]; K = FFN dim */
#define CAAT_VARIANT_MLP 1    /* caat_mlp_forward[_ex]; K = F */
#define CAAT_VARIANT_ROWPAR_HOST 2 /* caat_rowpar_forward_host; K = FFN dim */
#define CAAT_VARIANT_ROWPAR_BWD 4  /* caat_rowpar_backward; K = FFN dim */

/* Flags of caat_rowpar_args.flags / caat_mlp_args.flags. */
#define CAAT_FLAG_FORCE_GEMM_PATH 0x1u   /* use the tensor-core GEMM path even for small T */
#define CAAT_FLAG_FORCE_DECODE_PATH 0x2u /* use the weight-streaming path even for large T */
#define CAAT_FLAG_FUSED_NORM 0x8u        /* run the RMSNorm inside the GEMM kernel (normalizer
                                            warps fed by row-block completion counters) instead
                                            of as a separate row kernel after it */
#define CAAT_FLAG_ORDER_ROWBLOCK 0x10u   /* schedule the GEMM tiles row block by row block
                                            (default: shared-channel tiles first, then the
                                            private tiles rank by rank) */
#define CAAT_FLAG_OVERLAP_NORM 0x20u     /* T >= 4096: run the GEMM in 2048-token launches and the
                                            row norm of each launch's tokens on a library-owned
                                            side stream, overlapping the next launch */
#define CAAT_FLAG_ORDER_GROUPED 0x40u    /* schedule the GEMM tiles in groups of row blocks
                                            (shared tiles of the group, then its private tiles
                                            rank by rank); the fused norm always does */
#define CAAT_FLAG_SINGLE_CTA 0x4u        /* use the single-CTA GEMM kernel (128-token tiles)
                                            instead of the CTA-pair kernel (256-token tiles) */
#define CAAT_FLAG_W_PERMUTED 0x80u       /* W is the channel-permuted weight written by
                                            caat_permute_weights for this (sync_idx, p):
                                            the GEMM sees a contiguous sync set (no column
                                            block mixes shared and private channels) and the
                                            norm kernel restores the original channel order.
                                            Outputs stay in the original order.  Needs a
                                            buffer for Z' (h_out if given and distinct from
                                            residual, else out, which must then not alias
                                            residual); not with CAAT_FLAG_FUSED_NORM; the
                                            GEMM path needs H <= 4096. */
#define CAAT_FLAG_NORM_BESIDE_GEMM 0x200u /* CTA-pair GEMM path, H <= 4096, separate norm: start the
                                            row norm while the GEMM runs, on SMs the GEMM leaves
                                            free; it normalizes each 128-token block of a rank as
                                            soon as the GEMM has stored all of it (the GEMM counts
                                            its finished tiles per block in the workspace).  Needs
                                            the workspace caat_workspace_size reports; same bits
                                            as the default (norm after the GEMM) */
#define CAAT_FLAG_TEST_STALL 0x100u      /* test hook: the GEMM kernel's MMA warp never signals
                                            its accumulator, so every consumer wait runs out
                                            and the call reports CAAT_ERR_TIMEOUT through
                                            caat_get_device_status().  Nothing faults. */

/*
 * caat_rowpar_forward - the partially synchronized row-parallel layer, residual add and
 * per-rank RMSNorm (App. A.2 Eq. 22, §4 Eq. 9).
 *
 *   X         device, bf16 [P, T, K/P]   rank m's input slice X_m
 *   W         device, bf16 [P, H, K/P]   rank m's weight block (B~_m transposed, K contiguous)
 *   residual  device, bf16 [P, T, H]     per-rank residual R_m (App. B)
 *   gamma     device, bf16 [H]           RMSNorm weight, shared by the ranks
 *   sync_idx  HOST, int32, NULL or floor(H p) strictly increasing channels in [0, H).
 *             NULL selects the first floor(H p) channels (§3).  Read before return.
 *   P, p      ranks (1..CAAT_MAX_P) and sync factor p in [0, 1]; n_s = floor(H p) in double.
 *   out       device, bf16 [P, T, H]     normalized output; may alias `residual`.
 *   T, K, H   tokens (>= 0), FFN dim (K % P == 0, (K/P) % 8 == 0), hidden (H % 8 == 0).
 *   workspace device scratch, 256-byte aligned; contents need not be initialized and are
 *             clobbered.  caat_workspace_size(T, K, H, P, CAAT_VARIANT_ROWPAR) bytes enable
 *             every path: the fused norm's row-block counters and per-row partial sums of
 *             squares (about 64 ceil(H/256) P T bytes), the completion flags that give
 *             column blocks mixing shared and private channels the TMA epilogue (T/8
 *             ceil(H/256) bytes), the decode path's fp32 partials (4 P T H bytes, T <= 64),
 *             and the cross-rank sums of the shared channels stored once for all ranks
 *             (4 T n_s bytes; H <= 4096, S the first n_s channels, n_s % 8 == 0; each rank's
 *             residual is then added by the norm kernel).  The separate-norm GEMM path runs
 *             with 256 bytes (mixed column blocks then take the register epilogue and every
 *             shared tile stores h for all P ranks); a smaller workspace than a call needs
 *             gives CAAT_ERR_WORKSPACE.
 * eps = 1e-5 and private_scale = 1 (use caat_rowpar_forward_ex for other values).
 * Returns CAAT_OK once the work is queued.
 */
CAAT_API caat_status caat_rowpar_forward(const caat_bf16* X, const caat_bf16* W, const caat_bf16* residual,
                                const caat_bf16* gamma, const int32_t* sync_idx, int P, double p,
                                caat_bf16* out, int64_t T, int64_t K, int64_t H,
                                void* workspace, size_t ws_bytes, caat_stream_t stream);

/* Extended arguments of the row-parallel layer (same meaning as above, plus): */
typedef struct caat_rowpar_args {
  const caat_bf16* X;
  const caat_bf16* W;
  const caat_bf16* residual;
  const caat_bf16* gamma;
  const int32_t* sync_idx;     /* host */
  caat_bf16* out;
  caat_bf16* h_out;            /* optional (NULL): device bf16 [P, T, H] receives the pre-norm
                                  residual stream h = Z + R; may alias `residual` */
  void* workspace;
  size_t ws_bytes;
  caat_stream_t stream;
  caat_timing* timing;         /* optional (NULL): records CUDA events around each kernel */
  int64_t T, K, H;
  double p;
  float eps;                   /* RMSNorm epsilon, >= 0, inside the square root */
  float private_scale;         /* multiplies private channels before the residual add */
  int32_t P;
  uint32_t flags;              /* CAAT_FLAG_* */
} caat_rowpar_args;

CAAT_API caat_status caat_rowpar_forward_ex(const caat_rowpar_args* args);

/*
 * caat_rowpar_forward_host - the same layer for callers whose tensors live in HOST memory.
 * args->X, W, residual, gamma, out (and h_out if not NULL) are host pointers (pinned memory
 * for asynchronous copies; pageable memory also works, with synchronous staging).
 * args->workspace is a device buffer of caat_workspace_size(T, K, H, P,
 * CAAT_VARIANT_ROWPAR_HOST) bytes that receives device copies of the inputs and outputs.
 * The call is pipelined over chunks of 1024 tokens, the last ones halving down to 256 (token
 * rows are independent; a small last chunk keeps the final copy back short): W and gamma
 * are copied once, then each chunk's X and residual rows are copied in, its kernels run on
 * args->stream and its out (and h_out) rows are copied back, on two library-owned copy
 * streams (created on the first call on a device) so that both copy directions overlap the
 * kernels.  All of it is ordered after the work already queued on args->stream, and
 * args->stream waits for the last copy back: the call is complete when args->stream reaches
 * that point, and the host buffers must stay valid until then.
 */
CAAT_API caat_status caat_rowpar_forward_host(const caat_rowpar_args* args);

/*
 * caat_rowpar_forward_noalloc - the same layer for callers that cannot allocate device memory
 * at all: code running where cudaMalloc is unavailable or forbidden (a host process whose
 * allocator is owned by someone else, an embedding that may not grow its memory footprint,
 * a hot loop that must never enter the allocator).  No counterpart in the paper: it is a
 * deployment convenience of this library.
 *
 * Arguments as caat_rowpar_forward_ex, except that args->workspace and args->ws_bytes are
 * ignored.  The scratch the kernels need lives in a fixed device array inside the library,
 * CAAT_NOALLOC_SCRATCH_BYTES bytes per GPU, held by every GPU that loads the library until the
 * process exits.  It holds whatever workspace the path the call takes uses, when that fits:
 * the GEMM kernel's work-unit counter (always), the row-block counters and job list of the
 * norm that runs beside the GEMM (8 bytes per 128 tokens per rank), the completion flags of
 * column blocks that mix shared and private channels (T/8 ceil(H/256) bytes), the shared
 * channels' cross-rank sums (4 T n_s bytes), the fused norm's counters and partials, and the
 * decode path's fp32 partials (4 P T H bytes).
 *   - A fused norm (CAAT_FLAG_FUSED_NORM) whose partials do not fit runs as the separate norm;
 *     a decode-sized call whose partials do not fit takes the GEMM path; the optional parts
 *     (job list, flags, shared sums) are simply not used when they do not fit.  A call that still needs
 *     more than the array (a forced decode path that does not fit) returns
 *     CAAT_ERR_WORKSPACE and queues nothing.
 *   - Calls no cudaMalloc, cudaFree or other allocating routine.
 *   - The first call on a device looks up the array's device address (once per device and
 *     context, with that device current); make that first call before any stream capture.
 *   - Every call shares the one array and clears the part that must start at zero; calls
 *     whose work overlaps on the GPU (other streams, other host threads) race on it and must
 *     be serialized by the caller.
 */
#define CAAT_NOALLOC_SCRATCH_BYTES 1048576
CAAT_API caat_status caat_rowpar_forward_noalloc(const caat_rowpar_args* args);

/*
 * Plans: the graph-capture-friendly form of caat_rowpar_forward_ex for calls repeated on the
 * same buffers (a decode loop, a layer in a captured step).  caat_plan_create validates the
 * arguments and builds the sync mask once, binding every pointer, size and option of `args`
 * (which is copied; sync_idx is read before return); caat_plan_execute then only queues the
 * kernels on `stream` (it allocates nothing and never synchronizes, so it can be captured in
 * a CUDA graph once the device's first call has been made outside capture).  The buffers
 * must stay valid for the plan's lifetime.  A plan is host memory owned by the caller
 * through the handle; executing one plan on two streams at once races on its workspace.
 * No counterpart in the paper.
 */
typedef struct caat_plan caat_plan;
CAAT_API caat_status caat_plan_create(const caat_rowpar_args* args, caat_plan** plan_out);
CAAT_API caat_status caat_plan_execute(const caat_plan* plan, caat_stream_t stream);
CAAT_API caat_status caat_plan_destroy(caat_plan* plan);

/*
 * caat_mlp_forward - the MLP block per rank: column-parallel FC1 with SwiGLU (§3.1 Eq. 6),
 * then the partially synchronized FC2 (App. A.2 Eq. 22), residual add and RMSNorm (Eq. 9).
 *
 *   X         device, bf16 [P, T, H]        per-rank block input X_m
 *   A         device, bf16 [P, 2F/P, H]     rank m's FC1 rows: F/P gate rows, then F/P up rows
 *   W2        device, bf16 [P, H, F/P]      rank m's FC2 block
 *   residual, gamma, sync_idx, P, p, out    as for caat_rowpar_forward
 *   T, H, F   F % P == 0, (F/P) % 8 == 0, H % 8 == 0
 *   workspace caat_workspace_size(T, F, H, P, CAAT_VARIANT_MLP) bytes (holds Y [P,T,F/P]).
 */
CAAT_API caat_status caat_mlp_forward(const caat_bf16* X, const caat_bf16* A, const caat_bf16* W2,
                             const caat_bf16* residual, const caat_bf16* gamma,
                             const int32_t* sync_idx, int P, double p, caat_bf16* out,
                             int64_t T, int64_t H, int64_t F,
                             void* workspace, size_t ws_bytes, caat_stream_t stream);

typedef struct caat_mlp_args {
  const caat_bf16* X;
  const caat_bf16* A;
  const caat_bf16* W2;
  const caat_bf16* residual;
  const caat_bf16* gamma;
  const int32_t* sync_idx;     /* host */
  caat_bf16* out;
  caat_bf16* h_out;            /* optional pre-norm residual stream, as in caat_rowpar_args */
  void* workspace;
  size_t ws_bytes;
  caat_stream_t stream;
  caat_timing* timing;
  int64_t T, H, F;
  double p;
  float eps;
  float private_scale;
  int32_t P;
  uint32_t flags;
} caat_mlp_args;

CAAT_API caat_status caat_mlp_forward_ex(const caat_mlp_args* args);

/*
 * caat_rowpar_backward - gradients of the row-parallel layer (forward: caat_rowpar_forward)
 * for training, §4 Eq. 10-13 and Fig. 2b: the RMSNorm derivative per rank first, THEN the
 * reduction over ranks of the shared channels' gradients (fp32 accumulation, §4 "32 bit
 * gradient accumulation"), the private scale on the private channels, then the partial
 * products' gradients dX_m = dZt_m W_m and dW_m = dZt_m^T X_m (tcgen05 GEMMs); the shared
 * RMSNorm weight's gradient is summed over ranks and tokens (§4 Eq. 12-13).
 *
 *   X, W, gamma, sync_idx, p, P, T, K, H, eps, private_scale  as in the forward call
 *   h        device bf16 [P, T, H]: the pre-norm stream of the forward (its h_out)
 *   dout     device bf16 [P, T, H]: dL/d(out)
 *   dX       device bf16 [P, T, K/P]   (out)
 *   dW       device bf16 [P, H, K/P]   (out)
 *   dR       device bf16 [P, T, H] or NULL: dL/d(residual) = dL/dh  (out)
 *   dgamma   device fp32 [H]            (out)
 *   workspace caat_workspace_size(T, K, H, P, CAAT_VARIANT_ROWPAR_BWD) bytes, 256-byte aligned:
 *            dZt, per-CTA dgamma partials, and room for transposed copies of W, dZt and X,
 *            which only calls with T <= 128 or H <= 128 use (larger calls read the three
 *            tensors in place, MN-major).
 * Requires P <= 16 and H <= 8192.  Outputs must not overlap the inputs.  Asynchronous.
 */
typedef struct caat_rowpar_bwd_args {
  const caat_bf16* X;
  const caat_bf16* W;
  const caat_bf16* h;
  const caat_bf16* gamma;
  const caat_bf16* dout;
  const int32_t* sync_idx;     /* host */
  caat_bf16* dX;
  caat_bf16* dW;
  caat_bf16* dR;
  float* dgamma;
  void* workspace;
  size_t ws_bytes;
  caat_stream_t stream;
  caat_timing* timing;         /* optional: events around each of the backward's kernels */
  int64_t T, K, H;
  double p;
  float eps;
  float private_scale;
  int32_t P;
  uint32_t flags;              /* 0, or CAAT_BWD_FLAG_TRANSPOSED_OPERANDS */
} caat_rowpar_bwd_args;

/* Test hook: run the gradient GEMMs on transposed K-major copies of W, dZt and X (the path of
 * calls with T <= 128 or H <= 128) at any size.  The results equal the default path's bit for
 * bit: same MMA steps on the same values, only the operands' layout in memory differs. */
#define CAAT_BWD_FLAG_TRANSPOSED_OPERANDS 0x1u

CAAT_API caat_status caat_rowpar_backward(const caat_rowpar_bwd_args* args);

/*
 * The layer over real devices, one tensor-parallel rank per GPU (App. A.2 Eq. 22; §3: only the
 * first floor(h p) channels are synchronized; App. D: the exchange moves p times the bytes of
 * a full all-reduce).  Each rank r runs, on its own GPU:
 *   1. caat_rowpar_tp_local: its partial product X_r W_r^T (tcgen05 GEMM); the shared channels
 *      c < n_s = floor(H p) are written to zs as fp32 partials, the private channels are
 *      finished into h (private_scale * partial + residual, bf16);
 *   2. the caller's collective: zs summed over the ranks in place (e.g. an NCCL all-reduce,
 *      sum, fp32, of T * n_s elements); every rank then holds the same sums (Eq. 22);
 *   3. caat_rowpar_tp_finish: h[:, c] = bf16(zs[:, c] + residual[:, c]) for c < n_s (so h is the
 *      complete pre-norm residual stream), then out = RMSNorm(h) * gamma (§4 Eq. 9).
 * S is the first n_s channels (the paper's definition); n_s % 8 == 0 and H <= 4096 are
 * required (CAAT_ERR_UNSUPPORTED otherwise).  The single-device entry points above emulate the
 * same layer with the exchange folded into the tensor-core accumulation.
 *
 *   X         device bf16 [T, K_r]   this rank's input slice (local)
 *   W         device bf16 [H, K_r]   this rank's weight block (local)
 *   residual  device bf16 [T, H]     this rank's residual (local, finish)
 *   gamma     device bf16 [H]        RMSNorm weight (finish)
 *   zs        device fp32 [T, n_s]   local: out (this rank's partial); finish: in (the sum over
 *                                    ranks); NULL allowed when n_s == 0
 *   h         device bf16 [T, H]     local: out (private channels); finish: in/out (complete h)
 *   out       device bf16 [T, H]     finish: out; may alias h
 *   workspace local: 256 device bytes, 256-byte aligned (finish: unused)
 * Both calls are asynchronous on `stream`.  Outputs must not overlap other inputs.
 */
typedef struct caat_tp_args {
  const caat_bf16* X;
  const caat_bf16* W;
  const caat_bf16* residual;
  const caat_bf16* gamma;
  float* zs;
  caat_bf16* h;
  caat_bf16* out;
  void* workspace;
  size_t ws_bytes;
  caat_stream_t stream;
  caat_timing* timing;
  int64_t T, K_r, H;
  double p;
  float eps;
  float private_scale;
  uint32_t flags;              /* 0 */
} caat_tp_args;

CAAT_API caat_status caat_rowpar_tp_local(const caat_tp_args* args);
CAAT_API caat_status caat_rowpar_tp_finish(const caat_tp_args* args);

/*
 * The same layer with the exchange done by the library over peer memory (NVLink), no
 * collective library involved (App. A.2 Eq. 22; §3; §4: fp32 sum of the shared channels; App. D:
 * only the n_s shared channels cross devices).  Owner q of the world ranks owns the shared
 * columns [q w, (q + 1) w), w = n_s / world.  Per call, in this order on every rank:
 *   1. caat_rowpar_tp_local_push: the local GEMM (as caat_rowpar_tp_local) whose epilogue
 *      stores this rank's fp32 partial of every shared column straight into its owner's receive
 *      buffer (recv[q][rank][t][c - q w]); the launch's last CTA then raises
 *      flags[q][0 * world + rank] = epoch on every rank q.  args->zs is not used.
 *   2. caat_rowpar_tp_reduce: waits (bounded) until flags[rank][0 * world + r] = epoch for every
 *      r, sums the world partials of its columns in rank order (fp32), writes the sum into
 *      gather[g][t][rank w + j] of every rank g, and raises flags[g][1 * world + rank] = epoch.
 *   3. caat_rowpar_tp_finish_wait: waits until flags[rank][1 * world + q] = epoch for every q,
 *      then finishes as caat_rowpar_tp_finish with zs = gather[rank].
 * A rank's own entries are its local buffers; the others are the peers' buffers mapped into
 * this process (CUDA IPC), all on GPUs with peer access.  The caller allocates, per rank:
 * recv [world][T][w] fp32, gather [T][n_s] fp32, flags [2][world] uint32 zeroed once, and
 * reuses them across calls with an epoch that grows by one per call (0 is never used).  The
 * three calls of one rank go on one stream in order; then no buffer is overwritten while it is
 * still read: a rank's next push follows its finish, which waited for every owner's reduce, and
 * an owner's next reduce waits for every rank's next push.  A wait that runs out (a rank that
 * never arrives) sets
 * the device status word (caat_get_device_status: CAAT_ERR_TIMEOUT) and the kernel returns;
 * after an error nothing is signalled, so the other ranks' waits run out too.
 * Requirements: world = 1..8, rank < world, n_s = floor(H p) a multiple of 32 world, the
 * caat_rowpar_tp_local requirements, all pointers 16-byte aligned.
 */
#define CAAT_TP_MAX_WORLD 8
typedef struct caat_tp_peers {
  int32_t world;
  int32_t rank;
  uint32_t epoch;
  float* recv[CAAT_TP_MAX_WORLD];
  float* gather[CAAT_TP_MAX_WORLD];
  uint32_t* flags[CAAT_TP_MAX_WORLD];
} caat_tp_peers;

CAAT_API caat_status caat_rowpar_tp_local_push(const caat_tp_args* args, const caat_tp_peers* peers);
CAAT_API caat_status caat_rowpar_tp_reduce(const caat_tp_args* args, const caat_tp_peers* peers);
CAAT_API caat_status caat_rowpar_tp_finish_wait(const caat_tp_args* args, const caat_tp_peers* peers);

/*
 * caat_permute_weights - reorders the output channels (rows) of W for a sync set: with
 * perm(i) = the i-th shared channel for i < n_s and the (i - n_s)-th private channel
 * otherwise (both ascending), W_out[m, i, :] = W[m, perm(i), :] for every rank m.  The
 * layer's result does not depend on the order of the output channels (Eq. 22 sums each
 * shared channel over the ranks, whatever its index), so a forward call given W_out and
 * CAAT_FLAG_W_PERMUTED computes the same layer with the shared channels contiguous, which
 * keeps every 256-channel tile of the GEMM pure when S is an arbitrary list.  Done once per
 * weight (static weights: at load time).  No counterpart in the paper.
 *
 *   W, W_out  device, bf16 [P, H, K/P], 16-byte aligned, must not overlap.
 *   sync_idx, p, P, H, K  as for caat_rowpar_forward (same validation).
 * Asynchronous on `stream`; returns CAAT_OK once the copy kernel is queued.
 */
CAAT_API caat_status caat_permute_weights(const caat_bf16* W, caat_bf16* W_out, const int32_t* sync_idx, double p,
                                          int P, int64_t H, int64_t K, caat_stream_t stream);

/*
 * caat_speedup_model - the paper's speed-up model of partial synchronization (App. C,
 * Eq. 31-35), host only.  Per device and transformer layer (forward): G = (24 s h^2 +
 * 4 s^2 h) / r GEMM operations and P(p) = 2 s h p exchanged activations; with C the ratio of
 * compute to communication capacity in operations per exchanged activation, T(p) = G + C P(p),
 *   speedup = (T(1) - T(p)) / T(1) = (1 - p) / (1 + (12 h + 2 s) / (C r)),
 *   p*      = min((12 h + 2 s) / (C r), 1)   (C P(p*) = G: the exchange just fits under the compute).
 * h hidden size, s tokens, r tensor-parallel ranks, p in [0, 1], C > 0; outputs may be NULL.
 */
CAAT_API caat_status caat_speedup_model(double h, double s, double r, double p, double C, double* speedup_out,
                                        double* p_star_out);

/* Bytes of device workspace a forward call of this shape needs (0 for invalid shapes is
 * never returned: invalid shapes give SIZE_MAX).  variant: CAAT_VARIANT_*; for the MLP
 * variant K is F. */
CAAT_API size_t caat_workspace_size(int64_t T, int64_t K, int64_t H, int P, int variant);

/*
 * caat_sync_mask - host-only sync-set bookkeeping (App. A.2 Eq. 22; §3): n_s = floor(H p)
 * in double, S = first n_s channels (sync_idx NULL) or the given list, validated exactly as
 * the forward calls validate it.  mask_out (host, H bytes, may be NULL) receives 1 for
 * shared and 0 for private channels; n_sync_out (may be NULL) receives n_s.  No GPU needed.
 */
CAAT_API caat_status caat_sync_mask(int64_t H, double p, const int32_t* sync_idx, uint8_t* mask_out,
                           int64_t* n_sync_out);

/* Synchronizes `stream`, returns the device status word recorded by bounded waits since the
 * last call (0 = none; low byte = caat_status, upper bits = where) and clears it. */
CAAT_API caat_status caat_get_device_status(caat_stream_t stream, int32_t* status_out);

/* Event recorder for per-kernel device timing (outside the hot path: create once).
 * Each forward call given a recorder appends one record: events before the first kernel and
 * after each kernel it launches.  caat_timing_read synchronizes on the last event and
 * returns, for record i and kernel j, ms[i * max_kernels + j]. */
CAAT_API caat_status caat_timing_create(int capacity, caat_timing** out);
CAAT_API caat_status caat_timing_destroy(caat_timing* t);
CAAT_API caat_status caat_timing_reset(caat_timing* t);
CAAT_API caat_status caat_timing_read(caat_timing* t, float* ms, int max_records, int max_kernels,
                             int* n_records, int* n_kernels);

CAAT_API const char* caat_status_string(caat_status s);
CAAT_API const char* caat_version(void);

#ifdef __cplusplus
}
#endif
#endif /* CAAT_H_ */
