/*
 * twell.h — C ABI of libtwell: the activation-sparse gated FFN hot path with
 * TwELL (tile-wise ELLPACK) packing, for NVIDIA B200 (sm_100a).
 *
 * Sources of the method (news pages; they print no code and no kernel detail):
 *   [aivizor]      "Sakana AI и NVIDIA представили TwELL — формат и CUDA-ядра,
 *                  превращающие активную разреженность в реальные ускорения LLM"
 *                  (edge.aivizor.me), paragraphs 1-4
 *   [aimodelsnavi] "How TwELL by Sakana AI and NVIDIA Accelerates LLMs by 20%
 *                  Using Unstructured Sparsity" (aimodelsnavi.com), sections
 *                  "Technical Explanation" and "Core of TwELL"
 *
 * The block computed (gate / up / down projections, ReLU gate, gate bias):
 *     z = X W_g^T + b_g      g = ReLU(z)      u = X W_u^T      h = g * u
 *     Y = h W_d^T
 * with an optional L1 term lambda * sum(g) on the gate activations in training
 * ([aivizor] ¶1).
 *
 * Conventions shared by every entry point
 *   - Tensors are row-major device arrays. bf16 tensors are passed as uint16_t
 *     bit patterns. Weights follow the nn.Linear layout: W_g, W_u are
 *     [d_ff][d_model], W_d is [d_model][d_ff], b_g is [d_ff].
 *   - Ownership: the caller allocates every buffer, including the workspace;
 *     the library never allocates or frees device memory.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream).
 *     Argument and shape errors are reported synchronously and nothing is
 *     enqueued. Device-side conditions (overflow capacity exceeded, a bounded
 *     wait giving up) set bits in the caller's device status word, read with
 *     twell_status_read.
 *   - Base pointers must be 16-byte aligned; the workspace 256-byte aligned.
 *   - Supported shapes: T_n == 128; K in {8, 16, 32, 64}; d_model a multiple
 *     of 64 in [64, 16384]; d_ff a multiple of 128 in [128, 16384];
 *     0 <= M <= 2^24; 0 <= ovf_cap <= M. Anything else returns
 *     TWELL_EUNSUPPORTED. M == 0 is a valid no-op.
 *   - No entry point keeps state between calls or falls back to another
 *     implementation: every step runs in this library's sm_100a kernels.
 */
#ifndef TWELL_H
#define TWELL_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TWELL_API __attribute__((visibility("default")))
#else
#define TWELL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st* twell_stream_t;

typedef enum twell_status {
  TWELL_OK = 0,
  TWELL_EINVAL = 1,         /* null or misaligned pointer, negative size, inconsistent descriptor */
  TWELL_EUNSUPPORTED = 2,   /* shape outside the supported set above */
  TWELL_EOVERFLOW_CAP = 3,  /* (device bit) more overflow rows than ovf_cap */
  TWELL_ECUDA = 4,          /* a CUDA runtime or driver call failed */
  TWELL_ETIMEOUT = 5,       /* (device bit) a bounded device-side wait gave up */
  TWELL_EWORKSPACE = 6,     /* workspace too small or misaligned */
  TWELL_EBOUNDS = 7         /* (device bit, bounds-checked build only) an index read from a buffer was out of range */
} twell_status;

/* Device status word bits, set by kernels and read by twell_status_read. */
#define TWELL_STATUS_OVERFLOW_CAP (1u << TWELL_EOVERFLOW_CAP)
#define TWELL_STATUS_TIMEOUT (1u << TWELL_ETIMEOUT)
/* The state given to a call cannot serve it (a tile-routed inference state
 * passed to twell_ffn_bwd); the call wrote no result. */
#define TWELL_STATUS_BAD_STATE (1u << TWELL_EINVAL)
/* Set only by the bounds-checked build of the library (libtwell_bounds.so,
 * compiled with -DTWELL_BOUNDS): its kernels check every index they read from
 * a buffer (a slot's in-tile column, a piece's row, an overflow row, a dense
 * slot, a pair-list row or position) against the extent it addresses before the
 * access it steers; an index out of range sets this bit and the access is
 * skipped. The regular build never sets it and does not check. */
#define TWELL_STATUS_BOUNDS (1u << TWELL_EBOUNDS)

/*
 * The hybrid TwELL representation of g = ReLU(z) ([aivizor] ¶2: horizontal
 * tiles of width T_n aligned with the matmul tile, nonzeros packed locally in
 * each tile; the training format routes a row either to the compact ELL matrix
 * or, if it overflows, to a dense backup; [aimodelsnavi] "Core of TwELL":
 * ELLPACK applied per tile). All arrays are caller-owned device memory.
 *
 * Per (row i, tile t), T = d_ff / T_n:
 *   count[i][t]   true number of units c in the tile with z > 0 (0..T_n), also when > K
 *   val[i][t][s]  bf16 RNE of z for the s-th active unit in ascending column order,
 *                 s < min(count, K); 0 in the unused slots
 *   col[i][t][s]  in-tile column of that unit (0..T_n-1); 0 in the unused slots
 * Row routing: row i is an overflow row (row_ovf[i] = 1) when some tile has
 * count > K, or, when dense_min > 0, when its active units (sum over its tiles
 * of count) number at least dense_min. The second rule is this library's
 * addition to the pages' overflow routing: it sends rows whose gathers would
 * cost more than a dense row to the dense backup (results are the same either
 * way; kchoice.py derives the threshold from measured costs). Overflow rows are listed in ascending order in ovf_rows; the first
 * ovf_cap of them get a dense row g_ovf[s][:] = bf16(ReLU(z[i][:])).
 * n_ovf[0] = rows stored (min(flagged, ovf_cap)), n_ovf[1] = rows flagged.
 * The ELL slots of an overflow row still hold its first K actives per tile.
 *
 * u_ell / u_ovf are written by twell_ffn_fwd when non-NULL and read by
 * twell_ffn_bwd (which requires both): the up projection u at the kept ELL
 * slots of non-overflow rows, and the dense u rows of stored overflow rows.
 *
 * row_plan ([twell_plan_ints(M, d_ff, T_n, K)] int32, zero-filled by the
 * caller when allocated) is the schedule of the sparse kernels, written by the
 * routing step of twell_pack / twell_ffn_fwd and read by twell_ffn_fwd and
 * twell_ffn_bwd: the kept entries of every non-overflow row split into pieces
 * of at most S entries, S sized from the batch's total so that heavy rows are
 * spread over the whole GPU. Its contents are internal; the library leaves its
 * per-row turnstile words at zero between calls. The same d_model must be used
 * for the pack and the passes that read the plan.
 */
typedef struct twell_hybrid {
  int32_t M;         /* tokens (rows) */
  int32_t d_ff;      /* hidden width */
  int32_t T_n;       /* tile width (must be 128) */
  int32_t K;         /* ELL slots per (row, tile) */
  int32_t ovf_cap;   /* capacity of the dense backup block, in rows */
  int32_t dense_min; /* 0, or route rows with at least this many active units dense */
  uint16_t* count;   /* [M][T] */
  uint16_t* val;     /* [M][T][K] bf16 bits */
  uint8_t* col;      /* [M][T][K] */
  uint8_t* row_ovf;  /* [M] */
  int32_t* ovf_rows; /* [max(ovf_cap,1)] */
  int32_t* n_ovf;    /* [2] */
  uint16_t* g_ovf;   /* [max(ovf_cap,1)][d_ff] bf16 bits */
  float* u_ell;      /* [M][T][K], nullable */
  float* u_ovf;      /* [max(ovf_cap,1)][d_ff], nullable */
  uint32_t* status;  /* [1] device status word (TWELL_STATUS_* bits), never cleared by kernels */
  int32_t* row_plan; /* [twell_plan_ints(M, d_ff, T_n, K)], zero-filled at allocation */
} twell_hybrid;

/* Which call a workspace is sized for. */
typedef enum twell_op { TWELL_OP_PACK = 0, TWELL_OP_FWD = 1, TWELL_OP_BWD = 2 } twell_op;

/* Short English text for a status code (static storage). */
TWELL_API const char* twell_status_string(twell_status s);

/* Host-only check of a shape against the supported set; enqueues nothing. */
TWELL_API twell_status twell_query_support(int64_t M, int64_t d_model, int64_t d_ff, int64_t T_n, int64_t K,
                                 int64_t ovf_cap);

/* Elements (int32) of twell_hybrid::row_plan for this shape (0 for an invalid
 * one): 4 + 2 * M + 2 * (M + max(65536, ceil(M * (d_ff / T_n) * K / 256))). */
TWELL_API size_t twell_plan_ints(int64_t M, int64_t d_ff, int64_t T_n, int64_t K);

/* Workspace bytes that `op` needs for this shape (0 for an unsupported shape).
 * For TWELL_OP_FWD and TWELL_OP_BWD this includes room for a transposed W_d,
 * used only when the caller passes W_dt == NULL. */
TWELL_API size_t twell_workspace_bytes(twell_op op, int64_t M, int64_t d_model, int64_t d_ff, int64_t T_n,
                             int64_t K, int64_t ovf_cap);

/* W_dt[j][c] = W_d[c][j]: the down-projection weight stored unit-major
 * ([d_ff][d_model]), so that the weights of one hidden unit are contiguous.
 * Inference callers with fixed weights transpose once and pass W_dt to every
 * call; training callers may pass W_dt == NULL and let each call transpose. */
TWELL_API twell_status twell_transpose_wd(const uint16_t* W_d, int64_t d_model, int64_t d_ff, uint16_t* W_dt,
                                twell_stream_t stream);

/*
 * Gate projection with the TwELL pack in its epilogue, then row routing
 * ([aivizor] ¶2 places the packing inside the gate kernel's epilogue, so no
 * separate conversion pass over a dense z exists).
 *   X [M][d_model], W_g [d_ff][d_model], b_g [d_ff]  (bf16 bits)
 *   h        descriptor (M, d_ff, T_n, K, ovf_cap, arrays) filled on the device;
 *            u_ell / u_ovf are not touched
 *   z_debug  nullable [M][d_ff] fp32: z = X W_g^T + b_g as the kernel computed it
 *            (fp32 accumulation, then + b_g), for bit-exact checks of the pack
 *   ws       workspace of twell_workspace_bytes(TWELL_OP_PACK, ...) bytes
 */
TWELL_API twell_status twell_pack(const uint16_t* X, const uint16_t* W_g, const uint16_t* b_g, int64_t d_model,
                        twell_hybrid* h, float* z_debug, void* ws, size_t ws_bytes,
                        twell_stream_t stream);

/*
 * twell_pack without a workspace argument (the pages have no counterpart; this
 * is an integration aid). It is meant for callers that may not allocate device
 * memory: code embedded in a host application whose allocator owns all of the
 * device memory (a plug-in handed only its inputs and outputs), or a latency-
 * critical loop where a cudaMalloc, which can synchronise the device, is not
 * acceptable. It computes exactly what twell_pack computes.
 *   Scratch: the only scratch twell_pack needs, the dense slices spilled for
 *   tiles with more than K actives, lives in a file-scope device array of
 *   TWELL_NOALLOC_SCRATCH_BYTES that the library owns; every device that loads
 *   the library keeps it until the process exits. The call itself never calls
 *   cudaMalloc, cudaFree or an allocating library routine.
 *   Limit: M * d_ff * 2 <= TWELL_NOALLOC_SCRATCH_BYTES (M * d_ff <= 8,388,608);
 *   larger shapes return TWELL_EWORKSPACE and enqueue nothing.
 *   Set-up: the first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with the caller's current device, which must be the
 *   device of `stream`). Under CUDA's lazy module loading (the default since
 *   CUDA 12.2) that lookup is also when the driver loads this code onto the
 *   device and reserves the array's 16 MiB there, so the first call on each
 *   device does take device memory: make it at set-up time, before a host
 *   allocator claims the device's memory (else it can fail with TWELL_ECUDA)
 *   and before any stream capture. Later calls on that device reserve nothing.
 *   Sharing: all calls share the one array and the array keeps whatever the
 *   last call left in it. A call writes every scratch slice before it reads it,
 *   so nothing has to start at zero; but calls whose execution overlaps on the
 *   GPU (for example on two streams) race on the array and must be serialised.
 */
#define TWELL_NOALLOC_SCRATCH_BYTES (16u << 20)

TWELL_API twell_status twell_pack_noalloc(const uint16_t* X, const uint16_t* W_g, const uint16_t* b_g,
                                          int64_t d_model, twell_hybrid* h, float* z_debug,
                                          twell_stream_t stream);

/*
 * Forward pass of the sparse gated FFN ([aivizor] ¶2: a fused kernel reads the
 * TwELL activations and performs the up and down projections without writing
 * the hidden state to global memory; overflow rows take the dense backup path).
 *   W_u [d_ff][d_model], W_d [d_model][d_ff], W_dt nullable [d_ff][d_model]
 *   Y   [M][d_model] bf16 bits, fp32 accumulation. Rows routed to the dense
 *       block beyond ovf_cap are not written (status bit OVERFLOW_CAP is set).
 *   h   as in twell_pack; also writes u_ell / u_ovf when they are non-NULL
 *   ws  workspace of twell_workspace_bytes(TWELL_OP_FWD, ...) bytes
 */
TWELL_API twell_status twell_ffn_fwd(const uint16_t* X, const uint16_t* W_g, const uint16_t* b_g,
                           const uint16_t* W_u, const uint16_t* W_d, const uint16_t* W_dt,
                           int64_t d_model, uint16_t* Y, twell_hybrid* h, float* z_debug, void* ws,
                           size_t ws_bytes, twell_stream_t stream);

/*
 * Inference forward with per-(row, tile) overflow routing, the alternative to
 * the row-level hybrid of twell_ffn_fwd ([aivizor] ¶2 routes overflowing rows
 * to a dense backup; ¶4 notes that rows can hold far more nonzeros than the
 * mean): no row goes dense; a tile with more than K actives keeps its count
 * and its first K slots and is otherwise read whole from the dense slice the
 * gate epilogue spilled for it, so the sparse kernel runs every active unit
 * (an adaptive number of entries per tile). Same arguments and workspace as
 * twell_ffn_fwd; Y is the same function of the inputs.
 *   h   filled as by twell_pack except: row_ovf = 0 for every row, n_ovf = {0, 0},
 *       g_ovf, u_ell and u_ovf untouched (h->dense_min plays no part: no row
 *       goes dense under tile routing). The state serves inference only:
 *       twell_ffn_bwd given it sets TWELL_STATUS_BAD_STATE and writes nothing.
 */
TWELL_API twell_status twell_ffn_fwd_tiles(const uint16_t* X, const uint16_t* W_g, const uint16_t* b_g,
                                 const uint16_t* W_u, const uint16_t* W_d, const uint16_t* W_dt,
                                 int64_t d_model, uint16_t* Y, twell_hybrid* h, float* z_debug, void* ws,
                                 size_t ws_bytes, twell_stream_t stream);

/*
 * 8-bit weights for the gathers ([aimodelsnavi] "Industry Impact" names the
 * combination of the method with 8-bit quantisation as its long-term outlook).
 * twell_quantize_e4m3_rows stores each row r of a bf16 matrix W [rows][len] as
 * FP8 E4M3 codes (the OCP 8-bit format with a 4-bit exponent, bias 7, 3-bit
 * mantissa, largest finite value 448) with one power-of-two scale per row:
 *   scale[r] = 2^e_r, e_r the smallest integer with max_k |W[r][k]| <= 448 * 2^e_r
 *              (2^0 for an all-zero row)
 *   q[r][k]  = W[r][k] / 2^e_r rounded to the nearest E4M3 value, ties to even
 *   deq[r][k] (nullable) = bf16 bits of q[r][k] * 2^e_r, which is exact (the
 *              dequantised value has at most 4 significant bits)
 * len must be a multiple of 16 in [16, 16384], rows in [0, 2^24]; W, q and deq
 * 16-byte aligned, scale 4-byte aligned; all caller-owned device memory,
 * asynchronous on `stream`. For the forward below: quantise W_u (rows = d_ff,
 * len = d_model) and W_d^T (from twell_transpose_wd; rows = d_ff).
 */
TWELL_API twell_status twell_quantize_e4m3_rows(const uint16_t* W, int64_t rows, int64_t len, uint8_t* q,
                                                float* scale, uint16_t* deq, twell_stream_t stream);

/*
 * twell_ffn_fwd with the fused sparse up+down kernel reading 8-bit weights: per
 * active unit j it gathers row j of W_u8 (d_model codes, scale s_u[j]) and row j
 * of W_dt8 (the codes of column j of W_d, scale s_d[j]) instead of 2 * d_model
 * bf16 values, half the bytes. W_u and W_d are the dequantised bf16 weights
 * (deq of the quantisation above, W_d in its [d_model][d_ff] layout): the gate
 * GEMM takes W_g as it is and the dense backup GEMMs take W_u and W_d. Y is the
 * FFN of X with weights (W_g, W_u, W_d), the function twell_ffn_fwd computes on
 * the same arguments, up to fp32 rounding order. Inside the kernel the token
 * row enters the dot products as f16 (exact for magnitudes in [2^-14, 65504];
 * smaller values are rounded to f16's subnormal grid, larger ones saturate).
 * Row-level routing only; arguments, descriptor, workspace (TWELL_OP_FWD) and
 * errors as twell_ffn_fwd; u_ell / u_ovf are written when non-NULL.
 */
TWELL_API twell_status twell_ffn_fwd_e4m3(const uint16_t* X, const uint16_t* W_g, const uint16_t* b_g,
                                          const uint16_t* W_u, const uint16_t* W_d, const uint8_t* W_u8,
                                          const float* s_u, const uint8_t* W_dt8, const float* s_d, int64_t d_model,
                                          uint16_t* Y, twell_hybrid* h, float* z_debug, void* ws, size_t ws_bytes,
                                          twell_stream_t stream);

/*
 * Backward pass over the hybrid format of a previous twell_ffn_fwd (which must
 * have been given non-NULL u_ell and u_ovf), for L = sum(Y * dY) + lambda * sum(g):
 *   dH_ij = dY_i . W_d[:, j] at active units;  dU = dH g;  dZ = (dH u + lambda) [z > 0]
 *   dX = dU W_u + dZ W_g;  dW_d = dY^T H;  dW_u = dU^T X;  dW_g = dZ^T X;  db_g = sum_i dZ
 *   dY [M][d_model] bf16 bits; dX [M][d_model], dW_g / dW_u [d_ff][d_model],
 *   dW_d [d_model][d_ff], db_g [d_ff] (nullable): fp32, overwritten (not accumulated).
 *   ws  workspace of twell_workspace_bytes(TWELL_OP_BWD, ...) bytes
 * Overflow rows that the forward flagged but could not store (more than
 * ovf_cap of them; the forward set TWELL_STATUS_OVERFLOW_CAP) have no stored g
 * or u: their dX rows are not written (they keep whatever the buffer held),
 * their pairs are left out of dW_g, dW_u, dW_d and db_g, and the backward sets
 * TWELL_STATUS_OVERFLOW_CAP again. Every other row is computed as usual.
 * TWELL_EUNSUPPORTED (and a zero TWELL_OP_BWD workspace size) when the weight
 * gradients' pair list could exceed 2^31 - 1 entries, i.e. when
 * (M - ovf_cap) * (d_ff / T_n) * K + ovf_cap * d_ff > 2^31 - 1 (its positions
 * are 32-bit); a smaller ovf_cap or a split batch fits.
 */
TWELL_API twell_status twell_ffn_bwd(const uint16_t* X, const uint16_t* W_g, const uint16_t* W_u,
                           const uint16_t* W_d, const uint16_t* W_dt, int64_t d_model,
                           const twell_hybrid* h, const uint16_t* dY, float lambda, float* dX,
                           float* dW_g, float* dW_u, float* dW_d, float* db_g, void* ws,
                           size_t ws_bytes, twell_stream_t stream);

/*
 * Count statistics of a packed batch, for choosing the ELL width K of later
 * batches ([aivizor] ¶4: in training the largest number of nonzeros per row
 * can exceed the mean by a large factor). Read from h->count, which keeps the
 * true per-tile counts 0..T_n. With bins c = 0..T_n + 1:
 *   rows_by_max[c]     rows whose largest tile count is c, except that a row
 *                      with at least h->dense_min active units (when
 *                      dense_min > 0) is counted in bin T_n + 1
 *   act_by_max[c]      active units of the rows of bin c (summed over tiles)
 *   tiles_by_count[c]  (row, tile) pairs holding c active units (bin T_n + 1
 *                      stays 0)
 * Under row routing with width K the rows of bins c > K are the dense backup
 * rows and the rest keep all their units in ELL slots; under tile routing the
 * tiles of bins c > K are read from their spilled slices.
 * The three outputs are caller-owned device int64 arrays of T_n + 2 entries
 * (8-byte aligned), overwritten; asynchronous on `stream`. Integer sums: the
 * same result on every run. Errors: TWELL_EINVAL (null or misaligned pointer,
 * negative dense_min), TWELL_EUNSUPPORTED (descriptor shape), TWELL_ECUDA
 * (launch failure).
 */
TWELL_API twell_status twell_count_stats(const twell_hybrid* h, int64_t* rows_by_max, int64_t* act_by_max,
                                         int64_t* tiles_by_count, twell_stream_t stream);

/*
 * Schedule of the sparse kernels of twell_ffn_fwd (row routing) and
 * twell_ffn_bwd: a performance setting with no counterpart on the pages. The
 * results are the same under every schedule, bit for bit.
 *   TWELL_SCHED_FUSED   one kernel per direction: each token piece computes
 *                       its dot products and its axpy in turn (x . W_u[j],
 *                       then Y += h W_d[:, j]; dY . W_d[:, j], then
 *                       dX += dU W_u[j] + dZ W_g[j]).
 *   TWELL_SCHED_PASSES  one pass per gathered weight matrix (u per slot, then
 *                       Y; dH, dU, dZ per slot, then dX), each pass walking
 *                       the row plan's pieces once per chunk of its matrix of
 *                       at most l2_budget_bytes (the up and dH passes by
 *                       ranges of hidden tiles, the down and dX passes by
 *                       ranges of d_model columns), so that the weight rows
 *                       gathered at a time stay in L2 when the matrices do
 *                       not; the token rows are re-read once per chunk.
 *   TWELL_SCHED_AUTO    the default: TWELL_SCHED_PASSES when W_g, W_u and W_d
 *                       together (3 d_model d_ff bf16) are larger than the
 *                       device's L2 and M >= 4096, else TWELL_SCHED_FUSED.
 * l2_budget_bytes: the chunk bound, 0 for the default (64 MiB).
 * Process-wide; applies to the calls made after it returns. Tile routing
 * (twell_ffn_fwd_tiles) and the 8-bit forward always run fused. Errors:
 * TWELL_EINVAL for an unknown mode or a negative budget.
 */
typedef enum twell_sched { TWELL_SCHED_AUTO = 0, TWELL_SCHED_FUSED = 1, TWELL_SCHED_PASSES = 2 } twell_sched;

TWELL_API twell_status twell_set_sparse_schedule(int mode, int64_t l2_budget_bytes);

/*
 * Overlap of the dense backup with the sparse kernels (a performance setting
 * with no counterpart on the pages; results do not change). When on,
 * twell_ffn_fwd, twell_ffn_fwd_e4m3 and twell_ffn_bwd run the
 * dense-backup chain (the overflow rows' GEMMs and their gathers) on a second
 * stream owned by the library, created per device at first use at the
 * highest stream priority, forked from the caller's stream after the routing
 * and joined back into it before the call's remaining kernels; the sparse
 * kernels stay on the caller's stream and use what the GEMM leaves of each
 * SM. The call stays asynchronous and stream-ordered for the caller, and is
 * capturable into a CUDA graph. OFF runs every kernel on the caller's stream;
 * AUTO (the default) overlaps calls of fewer than 4096 rows, where the sparse
 * kernels alone leave most of each SM idle. Process-wide; applies to the calls
 * made after it returns. Returns TWELL_EINVAL for any other mode (the setting
 * is then unchanged).
 */
typedef enum twell_overlap { TWELL_OVERLAP_OFF = 0, TWELL_OVERLAP_ON = 1, TWELL_OVERLAP_AUTO = 2 } twell_overlap;

TWELL_API twell_status twell_set_overlap(int mode);

/* Copies the device status word to *out after synchronizing `stream`; clears
 * it when `clear` is non-zero. Returns TWELL_ECUDA if the copy fails. */
TWELL_API twell_status twell_status_read(const twell_hybrid* h, uint32_t* out, int clear, twell_stream_t stream);

/*
 * Test of failure detection (no counterpart on the pages; a test aid). The
 * dense-backup GEMMs of twell_ffn_fwd and twell_ffn_bwd may split their K
 * range when few rows overflow; the four epilogue warps of such a GEMM meet at
 * a bounded barrier before the tile's partial sums are counted and reduced.
 * After this call, the next `launches` of those GEMMs (each launch that can
 * split counts, whether or not it splits on the device) run with one epilogue
 * warp that never arrives at that barrier, as if it had stalled: the wait runs
 * out after its limit (2 s), the kernel sets TWELL_STATUS_TIMEOUT, counts no
 * arrival for the tile (so no CTA reduces partial sums that may be missing),
 * and unwinds; the rows that GEMM should have written are left unwritten.
 * launches <= 0 cancels what is left. Nothing else changes; the context stays
 * usable.
 */
TWELL_API void twell_test_withhold_epilogue_arrival(int launches);

/*
 * Launch accounting and per-kernel timing (no counterpart on the pages; a
 * runtime aid for measuring where a call spends its time without a profiler).
 *   twell_launch_count   number of kernels this library has launched in the
 *                        process so far (monotonic; thread-safe)
 *   twell_trace_enable   while on, every kernel launch is bracketed by two CUDA
 *                        events recorded on its stream (adds two event records
 *                        per kernel; off by default)
 *   twell_trace_collect  waits for the recorded events, writes up to max_recs
 *                        records (kernel name, duration in ms) to out (nullable),
 *                        forgets them and returns how many there were
 */
typedef struct twell_trace_rec {
  char name[32];
  float ms;
} twell_trace_rec;

TWELL_API uint64_t twell_launch_count(void);
TWELL_API void twell_trace_enable(int on);
TWELL_API int twell_trace_collect(twell_trace_rec* out, int max_recs);

#ifdef __cplusplus
}
#endif

#endif /* TWELL_H */
