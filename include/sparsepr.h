/*
 * sparsepr.h -- C ABI of the SparsePR sparse attention call on NVIDIA B200
 * (sm_100a).
 *
 * The method: "Partition the Support, Reconstruct the Residual: Training-Free
 * Sparse Attention for Video Generation and World Models" (arXiv 2608.18484),
 * as summarised by paperlayer.ai (cited below as [paperlayer §X]) and the
 * gist.science technical summaries ([gist-nl §X]).
 *
 * One call maps Q, K, V of shape [B, H, N, d] (bf16) to O of the same shape
 * (bf16): full-sequence attention approximated by
 *   1. Response-Coupled Partitioning           [paperlayer §4, App. B-B.2]
 *   2. routed variable-block sparse attention under renormalized hard drop,
 *      plus exact dense rows for M probe queries   [paperlayer §4, App. A.2]
 *   3. Probe-Fitted Residual Reconstruction     [paperlayer §4, App. A-A.3]
 * and the output restored to the original query order [paperlayer §4].
 *
 * Conventions for every entry point:
 *  - Every pointer argument named Q, K, V, O or ws is a DEVICE pointer; the
 *    caller owns it.  The library allocates no memory and never synchronises
 *    the stream, except sparsepr_get_stats, which copies to host and waits.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*, 0 = the
 *    legacy default stream) in stream order; a call returns as soon as the
 *    kernels are enqueued.
 *  - Argument errors are reported synchronously by the return value and
 *    nothing is enqueued.  Device-side faults that the kernels detect (an
 *    index out of range, a bounded wait that ran out) set an error word in the
 *    workspace instead of trapping; sparsepr_get_stats returns SPR_EDEVICE
 *    when it is set.
 *  - The workspace (`ws`, `ws_bytes` >= sparsepr_workspace_size) carries all
 *    intermediate state between the stage entry points; it must be 256-byte
 *    aligned and must not be shared by calls that may overlap on the GPU.
 *  - Not thread-safe per workspace; distinct workspaces may be used from
 *    distinct host threads and streams concurrently.
 */
#ifndef SPARSEPR_H
#define SPARSEPR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPR_OK = 0,
  SPR_EINVAL = 1,        /* an argument is out of range or inconsistent */
  SPR_EUNSUPPORTED = 2,  /* valid but not supported by these kernels (d, layout) */
  SPR_EWORKSPACE = 3,    /* workspace too small or misaligned */
  SPR_ECUDA = 4,         /* a CUDA runtime call failed (launch, copy) */
  SPR_EDEVICE = 5,       /* a kernel set the device error word */
  SPR_ESCRATCH = 6       /* too large for the fixed scratch area of
                            sparsepr_attend_routed_noalloc */
} spr_status;

enum { SPR_ROUTE_TAU = 0, SPR_ROUTE_BUDGET = 1 };

/*
 * Partition construction.  SPR_PARTITION_RESPONSE is the method's
 * Response-Coupled Partitioning.  SPR_PARTITION_SEMANTIC is the comparator the
 * pages measure it against [paperlayer §2 "Token Partitioning"; §3.1 O3, a
 * matched comparison]: the same fixed-iteration k-means run on the raw key
 * rows and, independently, on the raw query rows (Euclidean, same initial
 * rows, iterations and tie rule), with routing, renormalized hard drop, probes
 * and reconstruction unchanged.
 */
enum { SPR_PARTITION_RESPONSE = 0, SPR_PARTITION_SEMANTIC = 1 };

/*
 * k-means start [paperlayer App. C.1 names a warm-started GPU k-means].
 * SPR_INIT_SEEDED: G distinct rows from the splitmix64 partial shuffle of
 * `seed`.  SPR_INIT_WARM: the centroids the previous call left in the same
 * workspace: its raw-key group means (zero for an empty group) mapped into
 * this call's key-response coordinates by W (z = W^T k is linear), and its
 * query centroids kept in head-dimension form a_g = mean of (s / rms) q
 * (semantic mode: the raw-row centroids of both sides).  A warm call needs a
 * workspace whose last completed call had the same B, H, N, d, Gk, Gq, p and
 * partition; otherwise its starting centroids are whatever the workspace
 * holds (the call still completes; only the clustering is affected).
 */
enum { SPR_INIT_SEEDED = 0, SPR_INIT_WARM = 1 };

/*
 * Probe weights of the residual fit.  SPR_WEIGHTS_COVERAGE is the method's
 * coverage weighting [paperlayer §4 "Probe-Fitted Residual Reconstruction"]:
 * a probe of query group g weighs |Q_g| / m_g, normalised to sum 1.
 * SPR_WEIGHTS_UNIFORM weighs every probe 1 / M: the unweighted estimator of
 * the probe-selection / estimator ablation [paperlayer §5 "Ablations",
 * Table 4].  (The same ablation's estimator without the subspace restriction
 * is r = d: the basis then spans the whole output space.)
 */
enum { SPR_WEIGHTS_COVERAGE = 0, SPR_WEIGHTS_UNIFORM = 1 };

/*
 * Which rows of a query group become its probes.  The per-group counts m_g
 * (stratified apportionment) and the weights are the same for both.
 * SPR_PROBES_STRATIFIED takes m_g rows evenly spaced through the group in the
 * permuted order (the method's stratified selection [paperlayer App. A.2]).
 * SPR_PROBES_RANKED takes the group's m_g rows nearest its centroid in
 * query-response coordinates (squared distance ||u_n - c_g||^2, ties to the
 * lower original query index): the distance-ranked selection of the
 * probe-selection ablation [paperlayer §4 "Probe-Fitted Residual
 * Reconstruction" (probes drawn from query partitions and query-response
 * coordinates); §5 "Ablations", Table 4].  The distance is evaluated in fp32
 * as ||u_n||^2 - 2 (u_n . c_g - ||c_g||^2 / 2) from the final query
 * centroids; SPR_PARTITION_SEMANTIC has no query-response coordinates and
 * returns SPR_EUNSUPPORTED with it.
 */
enum { SPR_PROBES_STRATIFIED = 0, SPR_PROBES_RANKED = 1 };

/*
 * Parameters of one call.  Shapes: B batches, H heads, N tokens (N_q = N_k =
 * N, full-sequence attention [paperlayer §2]), head dim d in {64, 128}.
 *
 * Strides are in ELEMENTS for the batch, head and token dimensions of each
 * tensor; the head dimension is contiguous.  Every row start must be 16-byte
 * aligned (token stride a multiple of 8 elements, base pointer 16-byte
 * aligned).  A contiguous [B, H, N, d] tensor has strides {H*N*d, N*d, d}.
 */
typedef struct {
  int32_t B, H, N, d;
  int64_t q_strides[3], k_strides[3], v_strides[3], o_strides[3];
  float scale;        /* softmax scale; <= 0 selects 1/sqrt(d) */
  /* Response-Coupled Partitioning [paperlayer App. B.1, B.2] */
  int32_t Ms;         /* sampled queries, 1..N (rows floor(i*N/Ms)) */
  int32_t p;          /* key-response eigen-coordinates, 1..min(d, 32)
                         (SPR_EUNSUPPORTED above 32) */
  int32_t Gk, Gq;     /* K/V groups and query groups, 1..min(N, 256) */
  int32_t iters;      /* Lloyd iterations of both k-means, 1..100 */
  uint64_t seed;      /* k-means initial rows (splitmix64 partial shuffle) */
  /* routing [paperlayer §4 "Sparse Execution"] */
  int32_t route_mode; /* SPR_ROUTE_TAU or SPR_ROUTE_BUDGET */
  double tau;         /* tau mode: keep cells whose entry mass < tau (> 0) */
  double rho_target;  /* budget mode: executed-pair density target, (0, 1e6] */
  /* Probe-Fitted Residual Reconstruction [paperlayer App. A.2, A.3] */
  int32_t M;          /* probe rows per head, 0..min(N, 4096); 0 = hard drop only */
  int32_t r;          /* residual subspace rank, 0..d */
  double lambda;      /* ridge strength (>= 0), weights normalised to sum 1 */
  int32_t partition;  /* SPR_PARTITION_RESPONSE (0, default) or _SEMANTIC;
                         semantic mode ignores Ms and p */
  int32_t init;       /* SPR_INIT_SEEDED (0, default) or SPR_INIT_WARM */
  int32_t weights;    /* SPR_WEIGHTS_COVERAGE (0, default) or SPR_WEIGHTS_UNIFORM */
  int32_t probes;     /* SPR_PROBES_STRATIFIED (0, default) or SPR_PROBES_RANKED */
  int32_t head0;      /* global index of this call's first (batch, head), 0..2^30: the
                         k-means initial rows of flattened head bh come from the stream
                         of head head0 + bh, so a call split over head ranges (each
                         with its own head0) draws exactly what one call would */
} spr_params;

/* Per-(batch, head) results, copied out by sparsepr_get_stats. */
typedef struct {
  int64_t routed_pairs;   /* sum over routed cells of |Q_i| |K_j| */
  int64_t probe_pairs;    /* M * N_k: exact probe rows against all keys */
  int64_t nnz_cells;      /* routed (query-group, K/V-group) cells */
  int64_t tile_pairs;     /* query x key pairs the attention tiles executed */
  double rho_exec;        /* (routed_pairs + probe_pairs) / (N_q N_k) */
  double obj_k;           /* key k-means objective, final labels/centroids */
  double obj_q;           /* query k-means objective, final labels/centroids */
  double route_threshold; /* smallest kept tail mass (budget mode) */
  int32_t gk_nonempty;    /* nonempty K/V groups */
  int32_t gq_nonempty;    /* nonempty query groups */
  int32_t r_eff;          /* residual directions kept by the fit */
  int32_t flags;          /* bit 0: budget mode kept only the top cells */
} spr_head_stats;

/* Bytes of workspace a call with these parameters needs (0 on bad params). */
size_t sparsepr_workspace_size(const spr_params* prm);

/* Validate parameters; returns the status any entry point would return. */
spr_status sparsepr_check_params(const spr_params* prm);

/*
 * Stage 1: Response-Coupled Partitioning [paperlayer §4, App. B.1, B.2;
 * gist-nl §2A].  Per head: sampled queries Q_s give M_K = Q_s^T Q_s / M_s;
 * keys are k-means-clustered on the top-p eigen-coordinates of M_K (each
 * eigenvector weighted by sqrt(lambda_i / sum lambda)) into paired K/V
 * groups (values follow their keys); queries are k-means-clustered on their
 * RMS-normalised logits against the centred nonempty K/V-group centroids;
 * Q, K, V are then permuted into group-major layouts inside the workspace.
 * prm->partition = SPR_PARTITION_SEMANTIC clusters the raw key rows and the
 * raw query rows instead (the comparator); prm->init = SPR_INIT_WARM starts
 * both k-means from the centroids the previous call left in `ws`.
 * Reads Q, K, V (device, bf16, strides from prm); writes only `ws`.
 */
spr_status sparsepr_partition(const spr_params* prm, const void* Q, const void* K,
                              const void* V, void* ws, size_t ws_bytes, void* stream);

/*
 * Stage 2: routing and probe selection [paperlayer §4, App. A.2].  Per query
 * group, the K/V groups are ranked by softmax mass of the centroid logit
 * s*qbar_i.c_j + ln|K_j|; tau mode keeps cells whose cumulative mass before
 * them is below tau, budget mode keeps the largest such prefix set whose
 * true pair cost plus the M*N probe pairs fits rho_target*N^2 (each group's
 * top cell always kept).  Group means, logits, masses and tails are fp64.
 * Emits the routed-cell CSR, merged key ranges, M
 * probe rows stratified over query groups with coverage weights (1 / M each
 * with prm->weights = SPR_WEIGHTS_UNIFORM), and the attention work list.
 * Reads and writes only `ws`.
 */
spr_status sparsepr_route(const spr_params* prm, void* ws, size_t ws_bytes, void* stream);

/*
 * Stage 3: routed attention under renormalized hard drop fused with the
 * exact dense probe rows [paperlayer §1, §4].  Every query row attends, with
 * its softmax renormalised over the retained keys, to the union of the K/V
 * groups routed to its query group; probe rows attend to all keys.  fp32
 * accumulation; results stay in `ws`.
 */
spr_status sparsepr_attend(const spr_params* prm, void* ws, size_t ws_bytes, void* stream);

/*
 * Stage 4: Probe-Fitted Residual Reconstruction and output restoration
 * [paperlayer App. A.3; gist-nl §2B].  R = O_dense - O_sparse on the probes;
 * U_r = leading right singular vectors of the weighted centred R; a weighted
 * ridge fit of (R - Rbar) U_r on the centred sparse output gives the map
 * x -> Rbar + (x - xbar) B U_r^T, added to every unprobed row; probe rows take
 * their exact dense value.  Writes O (device, bf16, o_strides) in the
 * original query order.  With M = 0 O is the hard-drop output.
 */
spr_status sparsepr_reconstruct(const spr_params* prm, void* ws, size_t ws_bytes, void* O,
                                void* stream);

/* The whole call: the four stages above in order, on one stream. */
spr_status sparsepr_call(const spr_params* prm, const void* Q, const void* K, const void* V,
                         void* O, void* ws, size_t ws_bytes, void* stream);

/*
 * Copy the per-head statistics (B*H entries) to `host_out` and the device
 * error word to `*device_error` (either may be NULL).  Synchronises `stream`.
 * Returns SPR_EDEVICE if the error word is non-zero.
 */
spr_status sparsepr_get_stats(const spr_params* prm, const void* ws, size_t ws_bytes,
                              spr_head_stats* host_out, int32_t* device_error, void* stream);

/*
 * Named intermediate buffers inside the workspace, for tests and diagnostics.
 * sparsepr_workspace_view returns the byte offset and size of one of them
 * (layouts are per head, row-major, head-major; int32 unless noted).
 */
typedef enum {
  SPR_VIEW_LAB_K = 0,    /* [BH, N] K/V group of each key */
  SPR_VIEW_LAB_Q = 1,    /* [BH, N] query group of each query */
  SPR_VIEW_PERM_K = 2,   /* [BH, N] original key index at each permuted slot */
  SPR_VIEW_PERM_Q = 3,   /* [BH, N] original query index at each permuted slot */
  SPR_VIEW_KV_OFF = 4,   /* [BH, Gk+1] group offsets in the permuted keys */
  SPR_VIEW_Q_OFF = 5,    /* [BH, Gq+1] group offsets in the permuted queries */
  SPR_VIEW_ROW_PTR = 6,  /* [BH, Gq+1] CSR row pointers of routed cells */
  SPR_VIEW_COL_IDX = 7,  /* [BH, Gq*Gk] CSR K/V-group indices (ascending) */
  SPR_VIEW_PROBE_POS = 8,/* [BH, M] probe slots in the permuted query order */
  SPR_VIEW_PROBE_IDX = 9,/* [BH, M] probe original query indices */
  SPR_VIEW_PROBE_W = 10, /* [BH, M] fp32 coverage weights (sum 1) */
  SPR_VIEW_O_SPARSE = 11,/* [BH, N, d] fp32 hard-drop output, permuted order */
  SPR_VIEW_O_PROBE = 12, /* [BH, M, d] fp32 exact dense probe rows */
  SPR_VIEW_W_KEY = 13,   /* [BH, d, 32] fp32 key-response projection; columns
                            p .. 31 are zero */
  SPR_VIEW_CENT_K = 14,  /* [BH, Gk, 32] fp32 key centroids (eigen-coordinates) */
  SPR_VIEW_CENT_Q = 15,  /* [BH, Gq, d] fp32 query centroids a_g: the u-space
                            centroid is Ctilde a_g */
  SPR_VIEW_CTILDE = 16,  /* [BH, Gk, d] fp32 centred nonempty K/V centroids,
                            compacted (first gk_nonempty rows) */
  SPR_VIEW_RMS = 17,     /* [BH, N] fp32 query RMS (original order) */
  SPR_VIEW_TAIL = 18,    /* [BH, Gq, Gk] fp64 tail mass of each cell: softmax mass of
                            the cells ranked at or after it (-1: empty group) */
  SPR_VIEW_FIT_U = 19,   /* [BH, d, d] fp32 residual basis (first r_eff cols) */
  SPR_VIEW_FIT_B = 20,   /* [BH, d, d] fp32 ridge coefficients B (first r_eff
                            columns); the correction of a row x is b + (x B) U_r^T */
  SPR_VIEW_FIT_BVEC = 21,/* [BH, d] fp32 intercept b = Rbar - (xbar B) U_r^T */
  SPR_VIEW_PROBE_DIST = 22,/* [BH, N] fp32 squared distance of each permuted query
                            to its group's centroid in query-response
                            coordinates (written with SPR_PROBES_RANKED only) */
  SPR_VIEW_COUNT = 23
} spr_view;

spr_status sparsepr_workspace_view(const spr_params* prm, int32_t which, size_t* offset,
                                   size_t* bytes);

/*
 * Routed attention with no device memory allocation.  The paper has no
 * counterpart to this entry point: it runs the computation of
 * sparsepr_attend's routed cells, declared above (every row of query group i
 * attends, softmax renormalised over the kept keys, to the key ranges routed
 * to i), on group-major inputs the caller supplies, for callers that cannot
 * allocate device memory where they run it (a launch sequence replayed
 * with fixed addresses, a memory pool partitioned ahead of time, a thread
 * that must not enter the allocator).  It enqueues kernels only: no
 * cudaMalloc, cudaFree or allocating library call, ever.  Its own state (error
 * word, work cursor, per-head counters, per-group tile counts, work list)
 * lives in a fixed 4 MiB
 * area of device memory inside the library image; nothing has to start at
 * zero, since each call re-initialises that state before using it.
 *
 * Device pointers, caller-owned (bf16 = 16-bit bfloat, row-major):
 *   Qp, Kp, Vp  [BH, N, d] bf16, contiguous, 16-byte aligned: queries, keys
 *               and values of each head in group-major order (the rows of a
 *               group adjacent; V rows follow their keys).
 *   q_off       [BH, Gq + 1] int32: rows q_off[h][i] .. q_off[h][i+1] - 1 of
 *               head h form query group i; 0 <= q_off[h][i] <= q_off[h][i+1]
 *               <= N.  Rows outside every group are not written.
 *   run_ptr     [BH, Gq + 1] int32: the key ranges of group i of head h are
 *               entries run_ptr[h][i] .. run_ptr[h][i+1] - 1 of that head's
 *               slice of `runs`, with 0 <= run_ptr[h][i] <= run_ptr[h][i+1]
 *               <= Gq * Gk.
 *   runs        [BH, Gq * Gk, 2] int32 (8-byte aligned): key range {x, y}
 *               covers keys x .. y - 1, 0 <= x < y <= N.  Ranges of a group
 *               should not overlap (an overlapping key counts twice).
 *   O           [BH, N, d] fp32 (16-byte aligned): row r of group i receives
 *               softmax(scale * q_r K_S^T) V_S over the union S of its ranges.
 *               Rows of groups with no ranges are not written.
 *   status      int32[4] or NULL: after the call's kernels, the device error
 *               word and three info words (0 = no error; 1 = an index out of
 *               range, info = {head, group, 0 q_off | 1 run_ptr | 2 a range};
 *               2 = work list overflow; 4 = a bounded wait in the attention
 *               kernel gave up).  On an index error nothing is computed.
 * Sizes: BH heads (batch x heads) >= 1, N >= 1 with BH * N < 2^31, d in
 * {64, 128}, 1 <= Gq, Gk <= 256.  scale <= 0 selects 1/sqrt(d).
 *
 * Limit: 256 + 80 * BH (rounded up to 256) + 4 * BH * Gq (rounded up to 256)
 * + 16 * (BH * (ceil(N / 128) + Gq) + 1) bytes must fit in 4 MiB (e.g. 40
 * heads of 75,600 tokens with Gq = 256 need 0.56 MiB); larger problems
 * return SPR_ESCRATCH and enqueue nothing.
 *
 * The first call on each device does a one-time set-up: it looks up the
 * scratch area's address, loads every kernel this entry point can launch
 * (both head dimensions, both attention kernels) and resolves the driver's
 * tensor-map encoder.  Loading device code may take device memory, so make
 * that first call before capturing a stream and before any point where
 * allocation is not allowed; later calls on that device take none.
 * All calls on one device share the one scratch area: two calls that may
 * overlap on the GPU (different streams without ordering between them, or
 * different host threads) race on it and both results are undefined.  Calls
 * in one stream order are safe.  Argument errors return synchronously with
 * nothing enqueued.
 */
spr_status sparsepr_attend_routed_noalloc(const void* Qp, const void* Kp, const void* Vp,
                                          const int32_t* q_off, const int32_t* run_ptr,
                                          const int32_t* runs, int32_t BH, int32_t N, int32_t d,
                                          int32_t Gq, int32_t Gk, float scale, float* O,
                                          int32_t* status, void* stream);

/* Library version string (static storage). */
const char* sparsepr_version(void);

/*
 * Kernel launches this library has enqueued since it was loaded, over all
 * threads and devices (diagnostics; the difference around a call is the
 * number of kernels that call launched).
 */
int64_t sparsepr_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* SPARSEPR_H */
