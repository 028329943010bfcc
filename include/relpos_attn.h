/*
 * relpos_attn.h -- C ABI of the B200 (sm_100a) exact relative-position
 * attention library.
 *
 * The operation is the unified additive score of "Fast and Exact
 * Relative-Position Attention via Structure-Aware Kernels" (digest page,
 * Eq. (1)):
 *
 *   S_ij = tau * ( q_i.k_j + q_i.aQ_phi(i,j) + k_j.aK_phi(i,j) + b_phi(i,j) ) + M_ij
 *   O    = softmax_j(S) V,   LSE_i = log sum_j exp(S_ij)
 *
 * computed without any N x N tensor in device memory: the relation terms
 * are projected to scalars Z^Q = Q aQ^T, Z^K = K aK^T over each 128-row
 * group's reachable offsets (Eq. (2)-(3), "grouped reachable range"), added
 * to the score tiles on chip, and differentiated per offset with a single
 * writer per gradient entry (Eq. (4), "backward ... without atomics").
 * Bucketed maps are expanded to an equivalent truncated map whose copy
 * columns are summed back into their bucket ("constant tiles and the
 * saturated region").
 *
 * Conventions shared by every entry point
 *  - Offsets are delta = j - i (key position minus query position).
 *  - Every pointer named "device" must point to CUDA device memory owned
 *    by the caller; the library never allocates or frees device memory.
 *    Pointers named "host" point to host memory owned by the caller.
 *  - Tensors are dense row-major; [B,H,N,d] means the last index is
 *    contiguous.  Device pointers to 16-bit tensors must be 16-byte aligned.
 *  - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default)
 *    and runs asynchronously; nothing synchronises the host except the
 *    calls marked "synchronous".
 *  - Return value: RELPOS_OK (0) or a negative relpos_status.  On an error
 *    that is detected before any launch nothing is enqueued.  No C++
 *    exception crosses this interface.
 *  - Identical inputs give bit-identical outputs (no atomics anywhere).
 */
#ifndef RELPOS_ATTN_H_
#define RELPOS_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* relpos_stream_t; /* a cudaStream_t */

typedef enum {
  RELPOS_OK = 0,
  RELPOS_ERR_INVALID_ARG = -1,    /* null required pointer, bad size, misaligned pointer */
  RELPOS_ERR_UNSUPPORTED = -2,    /* head dim other than 64, unknown dtype/map/mask */
  RELPOS_ERR_WORKSPACE = -3,      /* workspace null or smaller than relpos_workspace_size */
  RELPOS_ERR_CUDA = -4,           /* a CUDA call failed; see relpos_last_cuda_error() */
  RELPOS_ERR_TIMEOUT = -5         /* a kernel's bounded wait expired (device status word) */
} relpos_status;

/* Offset maps (digest, experimental setup: Shaw truncated, Transformer-XL
 * identity, T5 buckets, DeBERTa log buckets). */
typedef enum {
  RELPOS_MAP_TRUNCATED = 0,   /* phi = clamp(delta, -clip, clip) + clip; R = 2 clip + 1 */
  RELPOS_MAP_IDENTITY = 1,    /* phi = delta + N - 1; R = 2N - 1 */
  RELPOS_MAP_BUCKET_T5 = 2,   /* T5 buckets (num_buckets, max_distance, bidirectional); R = num_buckets */
  RELPOS_MAP_BUCKET_LOG = 3,  /* DeBERTa log buckets (num_buckets = span k, max_distance = max
                                 position); R = 2 num_buckets */
  RELPOS_MAP_BUCKET_LOG_REVERSED = 4
                              /* the LOG row of the reversed offset -delta = i - j: the
                                 query-minus-key position by which DeBERTa's c2p and p2c terms
                                 both index their relation rows; R = 2 num_buckets */
} relpos_map_kind;

typedef struct {
  int32_t kind;           /* relpos_map_kind */
  int32_t clip;           /* TRUNCATED: clip distance c >= 0 */
  int32_t num_buckets;    /* BUCKET_T5 / BUCKET_LOG */
  int32_t max_distance;   /* BUCKET_T5 / BUCKET_LOG */
  int32_t bidirectional;  /* BUCKET_T5: 1 = bidirectional, 0 = causal-style one-sided */
} relpos_map_desc;

/* Additive mask M (bit flags; M = -inf where masked, 0 elsewhere). */
typedef enum {
  RELPOS_MASK_NONE = 0,
  RELPOS_MASK_CAUSAL = 1,       /* masks j > i */
  RELPOS_MASK_KEY_PADDING = 2   /* masks j >= key_len[b] */
} relpos_mask_flags;

typedef enum { RELPOS_F16 = 0, RELPOS_BF16 = 1, RELPOS_F32 = 2 } relpos_dtype;

/* Tile classes of the tile plan (digest, "constant tiles and the saturated region"). */
typedef enum {
  RELPOS_TILE_MASKED = 0,    /* no kept cell: skipped */
  RELPOS_TILE_CONST_LO = 1,  /* every cell has delta <= E_lo: one shared low-saturated row */
  RELPOS_TILE_BAND = 2,      /* intersects the band: per-score gather */
  RELPOS_TILE_CONST_HI = 3   /* every cell has delta >= E_hi: one shared high-saturated row */
} relpos_tile_class;

/* Tile edge of the tile plan and group size of the projections. */
#define RELPOS_TILE 128

typedef struct {
  int32_t B, H, N, d;        /* d must be 64 */
  int32_t dtype;             /* RELPOS_F16 or RELPOS_BF16: q, k, v, aq, ak (and dout, dq, dk, dv) */
  int32_t out_dtype;         /* O: same as dtype, or RELPOS_F32 */
  float tau;                 /* score scale, finite and > 0 (else INVALID_ARG) */
  relpos_map_desc map;
  int32_t mask;              /* relpos_mask_flags */
  int32_t table_per_head;    /* 0: aq/ak are [R,d] shared by all heads; 1: [H,R,d] */
  const int32_t* key_len;    /* device [B]; required iff mask has KEY_PADDING.  Keys j >= key_len[b]
                                are masked; a value below 0 counts as 0 and one above N as N
                                (the kernels clamp it, so no length can make them read past N) */
  const void* q;             /* device [B,H,N,d] dtype */
  const void* k;             /* device [B,H,N,d] dtype */
  const void* v;             /* device [B,H,N,d] dtype */
  const void* aq;            /* device [R,d] / [H,R,d] dtype, or NULL (term absent) */
  const void* ak;            /* device [R,d] / [H,R,d] dtype, or NULL (term absent) */
  const float* b;            /* device [H,R] float32, or NULL (term absent) */
  void* o;                   /* device [B,H,N,d] out_dtype: output (forward) / input (backward) */
  float* lse;                /* device [B,H,N] float32, natural log: output (fwd) / input (bwd);
                                -inf for a row whose keys are all masked (its O row is 0) */
  /* Attention dropout (no counterpart on the paper's pages: the standard form).
   * O = (P o M / (1 - p')) V with P = softmax(S) (LSE is that of S), M_ij in
   * {0, 1} drawn by Philox4x32-10 (Salmon et al., SC 2011), and p' = ceil(256 p)
   * / 256 the rate the mask realises.  One generator call per block of 4 query
   * rows x 4 keys: cell (b*H + h, i, j) uses counter (j >> 2, i >> 2, b*H + h,
   * dropout_offset) and key (low, high 32 bits of dropout_seed); u = byte j & 3
   * (least significant first) of output word i & 3, and M_ij = 1 when
   * u >= ceil(256 p).  The backward regenerates the same mask, so pass the same
   * three values to both calls.  dropout_p in [0, 1); 0 = no dropout. */
  float dropout_p;
  uint32_t dropout_offset;
  uint64_t dropout_seed;
  /* Where the forward takes the query-side projection Z^Q from (digest,
   * ablation "projection precompute" and limitations section):
   * RELPOS_PROJECTION_RETAINED computes Z^Q over each group's reachable
   * columns once and keeps it in the workspace (quadratic for the identity
   * map); RELPOS_PROJECTION_RECOMPUTE recomputes it inside every tile on the
   * tensor cores, so the forward workspace holds no projection at all (linear
   * memory) at the price of more tensor work per tile.  RECOMPUTE supports
   * the aq and b terms; with ak != NULL it returns UNSUPPORTED.  The backward
   * of a RECOMPUTE forward rebuilds Z^Q in its own part of the workspace. */
  int32_t projection;
  /* Packed variable-length batch (the pages benchmark padded batches; this is
   * the layout of FlashAttention's variable-length interface).  NULL: the
   * dense [B, H, N, d] layout above.  Otherwise cu_seqlens is device int32
   * [B + 1], non-decreasing from 0: sequence b owns tokens cu_seqlens[b] ..
   * cu_seqlens[b + 1] - 1, at most N of them (N is the longest sequence and
   * also sets the identity map's 2N - 1 table rows); q, k, v, o (and dout,
   * dq, dk, dv) are token-major [total_tokens, H, d] and lse is
   * [H, total_tokens]; each sequence attends only to its own keys, and no
   * work is spent on the rows a padded batch would add.  KEY_PADDING must not
   * be set (INVALID_ARG), total_tokens >= 1.  The kernels clamp offsets into
   * [0, total_tokens] and lengths into [0, N], so no store leaves the
   * tensors whatever cu_seqlens holds (inconsistent offsets give meaningless
   * outputs).  The workspace keeps a dense [B, H, N] layout. */
  const int32_t* cu_seqlens;
  int32_t total_tokens;
} relpos_fwd_args;

typedef enum { RELPOS_PROJECTION_RETAINED = 0, RELPOS_PROJECTION_RECOMPUTE = 1 } relpos_projection_mode;

typedef struct {
  relpos_fwd_args fwd;       /* the forward's inputs, plus its O and LSE (read) */
  const void* dout;          /* device [B,H,N,d] dtype: upstream gradient dO */
  void* dq;                  /* device [B,H,N,d] dtype, overwritten */
  void* dk;                  /* device [B,H,N,d] dtype, overwritten */
  void* dv;                  /* device [B,H,N,d] dtype, overwritten */
  float* daq;                /* device float32, shape of aq; required iff aq != NULL; overwritten */
  float* dak;                /* device float32, shape of ak; required iff ak != NULL; overwritten */
  float* db;                 /* device [H,R] float32; required iff b != NULL; overwritten */
  int32_t reuse_forward_workspace;
                             /* 1: `workspace` still holds what relpos_attn_fwd left in it
                                for these same forward arguments (expanded tables, group
                                records, projections Z^Q / Z^K and their saturated columns);
                                the backward then reads them instead of rebuilding them (the
                                digest's retained projection; with projection = RECOMPUTE
                                only the tables are reused and Z^Q is rebuilt).  0: rebuild
                                them.  With 1 and a workspace that does not hold that state
                                the gradients are garbage: the library cannot tell. */
} relpos_bwd_args;

/* Number of rows R of a relation table for `map` at sequence length N (host only):
 * the table sizes of the four mechanisms of the digest's experimental setup
 * (truncated 2 clip + 1, identity 2N - 1, T5 num_buckets, DeBERTa 2 num_buckets).
 * Errors: INVALID_ARG for null pointers or N < 1, UNSUPPORTED for an unknown kind. */
int relpos_table_rows(const relpos_map_desc* map, int32_t N, int32_t* R_out);

/* Saturation bounds of the expanded truncated map (host only; digest, "constant
 * tiles and the saturated region": bucketed maps are expanded by copying each
 * bucket row once per offset it covers): every reachable offset <= *e_lo maps
 * to one row, every offset >= *e_hi to one row; the expanded table has one row
 * per offset in [*e_lo, *e_hi].  Errors: INVALID_ARG, UNSUPPORTED as above. */
int relpos_expanded_bounds(const relpos_map_desc* map, int32_t N, int32_t* e_lo, int32_t* e_hi);

/* Workspace bytes needed by relpos_attn_fwd / relpos_attn_bwd for these
 * arguments (pointers are not read; only sizes, map, mask and which of
 * aq/ak/b are non-NULL).  The workspace holds the projections Z^Q/Z^K over
 * each 128-row group's reachable columns (digest, "grouped reachable range":
 * about N + G - 1 columns per group for the identity map, all R_exp columns
 * when one group covers the table; never N x N for the other maps), the
 * expanded tables, and in backward the offset-sharded gradients of Eq. (4).
 * Errors: INVALID_ARG, UNSUPPORTED. */
int relpos_workspace_size(const relpos_fwd_args* a, size_t* fwd_bytes, size_t* bwd_bytes);

/* Forward (digest, pipeline section: grouped projections, then the
 * FlashAttention-style query-tile / key-tile loop with the relation terms
 * added on chip and an online softmax): writes a->o and a->lse.
 * workspace: device, >= fwd_bytes, 256-byte aligned, contents on entry
 * ignored.  Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
int relpos_attn_fwd(const relpos_fwd_args* a, void* workspace, size_t ws_bytes, relpos_stream_t stream);

/* Backward (digest: two-pass backward, Eq. (4)): from dO and the forward's O
 * and LSE, writes dq, dk, dv and the table gradients daq/dak/db.  Shared
 * tables receive the sum over batch and heads, per-head tables the sum over
 * batch, both in a fixed order.  workspace: device, >= bwd_bytes. */
int relpos_attn_bwd(const relpos_bwd_args* a, void* workspace, size_t ws_bytes, relpos_stream_t stream);

/* Device-side status of the last call that used `workspace` (synchronous:
 * waits for `stream`).  No counterpart on the pages: the library's own
 * failure report.  The fused kernels bound every wait on an mbarrier;
 * when one expires the kernel stops its pipeline, frees its tensor memory,
 * returns, and leaves a non-zero status word at the start of the workspace
 * (its outputs are then invalid).  Returns RELPOS_OK, RELPOS_ERR_TIMEOUT
 * (*device_status = 1), or RELPOS_ERR_CUDA.  device_status: host, may be NULL. */
int relpos_check_workspace(const void* workspace, relpos_stream_t stream, int32_t* device_status);

/* Human-readable text of a relpos_status (static storage).  No counterpart on
 * the pages (error reporting of this interface). */
const char* relpos_status_string(int status);

/* The last cudaError_t seen by this thread inside the library (0 = none).  No
 * counterpart on the pages (error reporting of this interface). */
int relpos_last_cuda_error(void);

/* Forward without a caller workspace (no counterpart in the paper; an
 * addition for callers that cannot allocate device memory, e.g. code running
 * while a memory pool or another runtime owns the whole device and forbids
 * outside allocations, or an enqueue step that must not allocate).
 *
 * Same arguments and outputs as relpos_attn_fwd, but the workspace is a fixed
 * 32 MiB array inside the library's device image.  Every GPU on which the
 * library has made its first such call holds that array until the process
 * exits.  Apart from that first call (below), a call calls no cudaMalloc /
 * cudaFree or any allocating routine.
 *  - Shapes whose forward workspace (relpos_workspace_size's fwd_bytes)
 *    exceeds 32 MiB are rejected with RELPOS_ERR_WORKSPACE before any launch.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    outside any stream capture.  CUDA loads modules lazily by default, so
 *    that first call also loads the array's module (committing the 32 MiB)
 *    and each kernel's first launch loads its module: make one small call on
 *    every device before a pool claims the device's memory, or run with
 *    CUDA_MODULE_LOADING=EAGER.
 *  - All calls share the one array and it keeps the previous call's contents;
 *    the forward reads nothing from it that the same call has not written.
 *    Calls whose work overlaps on the GPU (different streams, or several
 *    host threads) race on the array: serialise them.
 *  - A kernel whose bounded wait expired is reported by relpos_check_noalloc
 *    (the status word lives in the array), until the next call clears it. */
int relpos_attn_fwd_noalloc(const relpos_fwd_args* a, relpos_stream_t stream);

/* Device status of the last relpos_attn_fwd_noalloc on the current device
 * (synchronous: waits for `stream`); results as relpos_check_workspace.  No
 * counterpart in the paper (failure report of the no-allocation forward). */
int relpos_check_noalloc(relpos_stream_t stream, int32_t* device_status);

/* --- measurement ---------------------------------------------------------- */

/* Per-phase device time collected between relpos_profile_start and
 * relpos_profile_stop.  Phases: "tables", "projection", "fwd_attention",
 * "bwd_prep", "bwd_dq", "bwd_dkdv", "fold_ranges", "relation_grads",
 * "bwd_attention".  The backward runs its Q-parallel pass (then the query-side
 * relation gradients) on the caller's stream and its K-parallel pass (then the
 * key side) concurrently on a second stream, so "bwd_dkdv" and the key-side
 * "relation_grads" are measured on that stream and overlap other phases.
 * Each side's dQ / dK row update runs on a further stream of its own, joined
 * back inside its "relation_grads" phase;
 * "bwd_attention" spans both passes, from the start of the first to the end
 * of the later one. */
typedef struct {
  char name[32];
  int32_t calls;       /* times the phase ran */
  int32_t kernels;     /* kernels it launched in total */
  float total_ms;      /* summed device time (CUDA events on the stream(s) the phase ran on) */
} relpos_phase_stat;

/* Starts bracketing every phase the library enqueues with CUDA events
 * (host-side bookkeeping only; the events add a few microseconds per phase).
 * Clears earlier statistics. */
int relpos_profile_start(void);

/* Stops collecting, waits for the recorded events (synchronous) and copies up
 * to max_stats phase statistics into stats (host array).  *n_stats receives
 * the number of phases seen. */
int relpos_profile_stop(relpos_phase_stat* stats, int32_t max_stats, int32_t* n_stats);

/* Number of kernels this library has launched in this process so far. */
int64_t relpos_kernel_launches(void);

/* --- data-parallel exchange -------------------------------------------- */

/* Ascending-rank sum of per-rank partial table gradients.
 * The gradient of a table shared across the batch is a sum over every cell
 * that reads it (digest: Eq. (4)), so when the batch is split over ranks each
 * rank's relpos_attn_bwd leaves the partial sum of its own batch elements in
 * daq / dak / db.  After an all-gather puts the partials in rank order, this
 * call adds them in that order, out[i] = ((p[0][i] + p[1][i]) + p[2][i]) + ...,
 * in fp32 with round-to-nearest adds, so every rank obtains the same bits.
 *  partials: device fp32 [world][n] (row r = rank r's partial, rows contiguous),
 *            4-byte aligned.  Not written unless out is its row 0.
 *  out:      device fp32 [n]; either partials itself (row 0) or a range that
 *            overlaps none of the rows.
 *  world >= 1; n >= 0 (n = 0: returns RELPOS_OK without a launch).
 *  Asynchronous on stream.  Errors: INVALID_ARG (world < 1, n < 0, null or
 *  misaligned pointer, overlapping out), CUDA. */
int relpos_sum_partials(const float* partials, int32_t world, int64_t n, float* out, relpos_stream_t stream);

/* --- parity exports (used by the tests) --------------------------------- */

/* Storage of one 128-row projection group (digest, "grouped reachable range",
 * Eq. (3)): its rows hold the expanded columns [e0, e0 + W) (expanded column
 * e is offset E_lo + e) with a row stride of S floats, starting `base` floats
 * into a (batch, head) slice.  Columns [W, S) of a row are padding. */
typedef struct {
  int32_t e0, W, S, pad;
  int64_t base;
} relpos_group_info;

/* Where relpos_debug_projection left the projections in the workspace. */
typedef struct {
  int32_t E_lo, E_hi, R_exp;   /* expanded offset range [E_lo, E_hi], R_exp = E_hi - E_lo + 1 */
  int32_t nT;                  /* groups (= 128-row tiles) per (batch, head) */
  int32_t grouped;             /* 1: per-group reachable columns; 0: every group stores all R_exp */
  int32_t pad;
  int64_t zq_offset, zk_offset;   /* byte offsets of Z^Q / Z^K (float32) in the workspace; -1 if absent */
  int64_t zq_head, zk_head;       /* floats per (batch, head) slice of Z^Q / Z^K */
  int64_t gq_offset, gk_offset;   /* byte offsets of the query / key groups' relpos_group_info [nT] */
} relpos_projection_layout;

/* Runs the forward's table expansion and projections only (digest, Eq. (2)/(3)
 * over each group's reachable range) and leaves Z^Q = Q aQ_exp^T and
 * Z^K = K aK_exp^T in `workspace`: for row i of (b, h), g = i / 128, group
 * record gi, and expanded column e in [gi.e0, gi.e0 + gi.W), Z^Q[b, h, i, e]
 * is the float at byte zq_offset + 4 (((b H + h) zq_head) + gi.base +
 * (i % 128) gi.S + e - gi.e0); Z^K likewise with the key groups.  Arguments
 * as relpos_attn_fwd (o, lse, v are not read).  Synchronous.  Errors:
 * INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
int relpos_debug_projection(const relpos_fwd_args* a, void* workspace, size_t ws_bytes, relpos_stream_t stream,
                            relpos_projection_layout* layout);

/* Limit, in nanoseconds, of every bounded wait in the fused kernels launched
 * after this call (process-wide; 0 restores the default of 2 s).  Exists so
 * that tests can make a wait run out on purpose and check that the kernels
 * stop cleanly and report RELPOS_ERR_TIMEOUT.  No counterpart on the pages
 * (failure detection of this library). */
int relpos_set_wait_limit_ns(uint64_t ns);

/* phi(i, j) for all N x N cells computed on the host. phi_host: host [N*N] int32. */
int relpos_debug_phi(const relpos_map_desc* map, int32_t N, int32_t* phi_host);

/* phi(j - i) for the 2N-1 offsets delta = 1-N .. N-1, computed by the same
 * device code the expansion kernel uses. phi_dev: device [2N-1] int32.
 * Synchronous. */
int relpos_debug_phi_device(const relpos_map_desc* map, int32_t N, int32_t* phi_dev, relpos_stream_t stream);

/* Tile plan on the host: classes host int32 [B][nT][nT] and segments host
 * int32 [B][nT][4] = (end of CONST_LO run, end of BAND run, end of live
 * tiles, nT) with nT = ceil(N / RELPOS_TILE).  key_len_host: host [B] or NULL. */
int relpos_debug_tile_plan(const relpos_map_desc* map, int32_t B, int32_t N, int32_t mask,
                           const int32_t* key_len_host, int32_t* classes_host, int32_t* segs_host);

/* The same tile plan computed by the device code the kernels use; arguments
 * as above but key_len, classes and segs are device pointers.  Synchronous. */
int relpos_debug_tile_plan_device(const relpos_map_desc* map, int32_t B, int32_t N, int32_t mask,
                                  const int32_t* key_len_dev, int32_t* classes_dev, int32_t* segs_dev,
                                  relpos_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* RELPOS_ATTN_H_ */
