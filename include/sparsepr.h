/*
 * sparsepr.h -- C ABI of the B200 (sm_100a) SparsePR attention library.
 *
 * One SparsePR call, as described on the summary page of "Partition the
 * Support, Reconstruct the Residual: Training-Free Sparse Attention for Video
 * Generation and World Models" (Taghavi, Langari, Pandey, 2026), runs seven
 * steps on bf16 Q/K/V:
 *   (1) sampled queries' pre-softmax responses to all keys        [partition paragraph]
 *   (2) response-coupled key groups and query groups              [partition paragraph]
 *   (3) routing of (query group, key group) cells to rho_exec     [execution paragraph]
 *   (4) group-major permutation of Q/K/V                          [execution paragraph]
 *   (5) exact attention on the selected cells, renormalised       [execution, residual paragraphs]
 *   (6) probe rows, residual R = O_dense - O_sparse, weighted
 *       ridge fit and projection onto the residual subspace       [probe paragraph]
 *   (7) correction and write-back in the original token order     [probe, execution paragraphs]
 *
 * Conventions for every entry point:
 *   - Q is bf16 [B][Hq][N][d]; K and V are bf16 [B][Hkv][N][d]; all tensors
 *     are contiguous with d innermost and 16-byte aligned base pointers.
 *     Query head hq uses KV head hq / (Hq / Hkv) (grouped-query attention).
 *   - Every tensor pointer is DEVICE memory owned by the caller, unless a
 *     struct field says "handle-owned". Handle-owned buffers are allocated by
 *     sparsepr_create, stay valid until sparsepr_destroy, and are overwritten
 *     by the next call on the handle that produces them.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Every call only enqueues work on it and never waits for the
 *     device; argument errors are returned synchronously and leave the
 *     stream untouched. Device-side failures (a bounded wait that ran out, a
 *     failed bounds check) are recorded in a device status word read with
 *     sparsepr_device_status after the caller synchronises.
 *   - A handle is not thread-safe: calls on one handle must be serialised by
 *     the caller, and work from two calls must not overlap on the device
 *     unless the second call's stream waits for the first.
 *   - Integer index arrays are int32 (N < 2^31); pair counts are int64.
 */
#ifndef SPARSEPR_H
#define SPARSEPR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
typedef enum sparsepr_status {
    SPARSEPR_OK = 0,
    SPARSEPR_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad shape or config value */
    SPARSEPR_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. head dim not 64/128) */
    SPARSEPR_ERR_WORKSPACE = 3,     /* workspace allocation failed in sparsepr_create */
    SPARSEPR_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
    SPARSEPR_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up (device status word) */
    SPARSEPR_ERR_DEVICE = 6         /* a device-side bounds/consistency check failed */
} sparsepr_status;

/* Ablation switches (sparsepr_config.flags); the page's ablations compare them. */
#define SPARSEPR_FLAG_HARD_DROP_ONLY    (1u << 0)  /* no probes, no correction; whole budget to the route */
#define SPARSEPR_FLAG_RIDGE_ONLY        (1u << 1)  /* ablation: ridge correction Rbar + A(o - obar), no projection */
#define SPARSEPR_FLAG_RBAR_UNPROJECTED  (1u << 2)  /* ablation: project only A(o - obar), add Rbar unprojected */
#define SPARSEPR_FLAG_UNIFORM_WEIGHTS   (1u << 3)  /* probe weights 1 instead of group coverage */
#define SPARSEPR_FLAG_TOPMASS           (1u << 4)  /* sparsepr_partition also writes the support diagnostic */
#define SPARSEPR_FLAG_PROBES_UNIFORM    (1u << 5)  /* ablation: probes at rows floor((m+1/2)N/M) of the original order */
#define SPARSEPR_FLAG_PROBES_RANDOM     (1u << 6)  /* ablation: M distinct rows from the SplitMix64 stream of state
                                                      seed ^ 0x70726F6265, each output mod N (repeats skipped);
                                                      at most one of the two probe flags */
#define SPARSEPR_FLAG_SEMANTIC_PARTITION (1u << 7) /* ablation: key groups by k-means on the raw keys, query
                                                      groups on the raw mean query of the KV group (fp32 rows
                                                      of width d; `features` then holds the keys); not with
                                                      SPARSEPR_FLAG_TOPMASS */
#define SPARSEPR_FLAG_STAGE_TIMING      (1u << 8)  /* record per-stage CUDA events (sparsepr_get_stats) */
#define SPARSEPR_FLAG_TEST_STALL        (1u << 9)  /* TEST ONLY: the kernel of sparsepr_dense_attn issues
                                                      no loads, so its first bounded wait runs out (about 2 s of SM
                                                      clock), every CTA returns with its TMEM freed and nothing in
                                                      flight, the output rows are written as zeros and the device
                                                      status word reads SPARSEPR_ERR_TIMEOUT; it exercises the
                                                      bounded waits without a fault or a hang */

/*
 * Shape and hyper-parameters of one call. Defaults used by the page: rK=48,
 * rQ=64, M=64, lambda=0.1, r=16, rho_exec=0.22 (0.26 for the world model).
 *   B, Hq, Hkv, N, d  batch, query heads, KV heads (Hq % Hkv == 0), tokens, head dim (64 or 128)
 *   block             attention tile rows, 64 or 128 (performance only; no effect on results)
 *   Gk, Gq            key / query group counts (1..1024, <= N; Gq*Gk <= 2^20)
 *   rK                number of sampled queries = key feature rank (1..64)
 *   rQ                query coordinate rank (1..64): Gk <= rQ uses all Gk centred logits,
 *                     Gk > rQ projects them with a fixed +-1/sqrt(rQ) SplitMix64 matrix
 *   M                 probe rows per query head (1..min(N, 64); ignored under HARD_DROP_ONLY)
 *   r                 residual subspace rank (1..M, <= 32)
 *   kmeans_iters      Lloyd rounds after the first assignment (0..64)
 *   lambda            ridge strength (> 0)
 *   rho_exec          target execution density = route density + M/N (0 < rho_exec; >= 1 keeps all cells)
 *   flags             SPARSEPR_FLAG_* bits
 *   seed              seed of the query-coordinate projection matrix
 */
typedef struct sparsepr_config {
    int B, Hq, Hkv, N, d;
    int block;
    int Gk, Gq;
    int rK, rQ, M, r;
    int kmeans_iters;
    float lambda;
    float rho_exec;
    unsigned int flags;
    unsigned long long seed;
} sparsepr_config;

typedef struct sparsepr_handle_s* sparsepr_handle;

/*
 * Response-coupled partition of every (batch, KV head) pair, P = B*Hkv pairs
 * in (b, kv head) order [partition paragraph]. Group-major order: inside a
 * group, ascending original index.
 *   kgroup [P][N]        key group of each original key
 *   qgroup [P][N]        query group of each original query (shared by the KV head's query heads)
 *   kperm  [P][N]        group-major position -> original key index
 *   koff   [P][Gk+1]     key group g occupies positions koff[g] .. koff[g+1]-1
 *   qperm  [P][N]        group-major position -> original query index
 *   qoff   [P][Gq+1]
 *   kcent  [P][Gk][d]    fp32 mean of the raw keys of each group (0 for an empty group)
 *   radial [P][N]        fp32 squared distance of each query to its group centroid (coordinates)
 *   probe  [P][M]        original index of each probe row
 *   probe_pos [P][M]     position of each probe row in qperm
 *   weights [P][M]       fp32 group-coverage weight of each probe (mean 1)
 *   features [P][N][rK]  fp32 key response features (written by sparsepr_partition; unused as input)
 *   topmass [P][rK]      fp32 support diagnostic [support paragraph]: for sampled query row s, the
 *                        fraction of keys whose largest softmax weights first reach 90% of the row's
 *                        mass (written by sparsepr_partition with SPARSEPR_FLAG_TOPMASS, else NULL;
 *                        unused as input)
 * When the struct is handed IN, only kgroup/qgroup are ignored; every other
 * field except `features` and `topmass` must be set.
 */
typedef struct sparsepr_partition_t {
    int32_t* kgroup;
    int32_t* qgroup;
    int32_t* kperm;
    int32_t* koff;
    int32_t* qperm;
    int32_t* qoff;
    float* kcent;
    float* radial;
    int32_t* probe;
    int32_t* probe_pos;
    float* weights;
    float* features;
    float* topmass;
} sparsepr_partition_t;

/*
 * Selected cells of every (batch, KV head) pair as CSR [execution paragraph].
 *   rowptr [P][Gq+1]     kept key groups of query group a: kg[p*Gq*Gk + rowptr[a] .. rowptr[a+1]-1]
 *   kg     [P][Gq*Gk]    kept key group ids, ascending inside each row
 *   scores [P][Gq][Gk]   fp32 cell scores (written by sparsepr_route; unused as input)
 *   pairs  [P]           int64 routed (query, key) pairs
 */
typedef struct sparsepr_route_t {
    int32_t* rowptr;
    int32_t* kg;
    float* scores;
    int64_t* pairs;
} sparsepr_route_t;

/*
 * Probe fit of every (batch, query head), Hp = B*Hq [probe paragraph].
 * The correction of a sparse output row o is delta(o) = U (c0 + Bm o), i.e.
 * U U^T (Rbar + A (o - obar)) with Bm = U^T A and c0 = U^T Rbar - Bm obar.
 *   obar, Rbar [Hp][d]   weighted means of the probes' sparse outputs and residuals
 *   A      [Hp][d][d]    ridge map (row-major, y = A x)
 *   U      [Hp][d][r]    residual subspace basis (columns beyond rank are 0)
 *   Bm     [Hp][r][d]
 *   c0     [Hp][r]
 *   rank   [Hp]          int32 rank of the subspace actually used (<= r)
 *   R      [Hp][M][d]    fp32 probe residuals O_dense - O_sparse
 *   Odense [Hp][M][d]    fp32 dense attention output of the probe rows
 *   Osp    [Hp][M][d]    fp32 sparse output of the probe rows (bf16 values widened)
 */
typedef struct sparsepr_fit_t {
    float* obar;
    float* Rbar;
    float* A;
    float* U;
    float* Bm;
    float* c0;
    int32_t* rank;
    float* R;
    float* Odense;
    float* Osp;
} sparsepr_fit_t;

/* Per-call statistics, valid after sparsepr_get_stats. */
typedef struct sparsepr_stats {
    double route_density;   /* mean over (b, KV head) of routed pairs / N^2 */
    double rho_exec;        /* route_density + M / N (the page's realised execution density) */
    double useful_pairs;    /* sum over query heads of routed pairs + M*N (executed exact pairs) */
    float stage_ms[8];      /* partition, route, permute, attention, probe+fit, write-back, -, total
                               (only with SPARSEPR_FLAG_STAGE_TIMING; else 0) */
    int device_status;      /* 0 = OK, else a sparsepr_status code recorded on the device */
} sparsepr_stats;

/* Human-readable name of a status code (static string, never NULL). */
const char* sparsepr_status_string(sparsepr_status s);

/* Library version as major*10000 + minor*100 + patch. */
int sparsepr_version(void);

/*
 * Validate `cfg`, allocate the handle and all workspace on the current CUDA
 * device (cudaMalloc; a few GB at N=118800, 24 heads). On error *out is NULL
 * and nothing is allocated.
 */
sparsepr_status sparsepr_create(const sparsepr_config* cfg, sparsepr_handle* out);

/* Free the workspace and the handle (synchronises the device first). NULL is a no-op. */
sparsepr_status sparsepr_destroy(sparsepr_handle h);

/* Bytes of device workspace the handle holds. */
sparsepr_status sparsepr_workspace_bytes(sparsepr_handle h, size_t* out);

/*
 * Steps (1)-(2) [partition paragraph; probe paragraph for the probe rows]:
 * responses of rK evenly strided sampled queries (sample s: row
 * floor((s+1/2)N/rK) of query head s mod (Hq/Hkv)), Lloyd k-means of the key
 * features into Gk groups, key-group means over the raw keys, query
 * coordinates against them (mean query of the KV group, centred, projected to
 * rQ when Gk > rQ, L2-normalised), Lloyd k-means into Gq query groups,
 * group-major orders, stratified radial probe rows and coverage weights.
 * *out receives pointers to handle-owned buffers.
 */
sparsepr_status sparsepr_partition(sparsepr_handle h, const void* Q, const void* K,
                                   sparsepr_partition_t* out, void* stream);

/*
 * Step (3) [execution paragraph]: cell scores from every query head's logits
 * against the key-group means, then whole cells selected to the budget
 * floor(rho_exec*N^2) - M*N: each query group's top cell first, then cells in
 * descending score (ties: lower query group, then lower key group) while the
 * total stays within budget, the crossing cell kept iff its overshoot is
 * smaller than the undershoot without it. A budget below the top cells' cost
 * (negative when rho_exec < M/N) keeps the top cells only; rho_exec >= 1 keeps
 * every cell whose query and key groups are both non-empty. `part` may be
 * handle-owned or handed in. *out receives pointers to handle-owned buffers.
 */
sparsepr_status sparsepr_route(sparsepr_handle h, const void* Q, const sparsepr_partition_t* part,
                               sparsepr_route_t* out, void* stream);

/*
 * Step (4) [execution paragraph]: gather Q (every query head by its KV
 * head's qperm), K and V (by kperm) into group-major order. Qp/Kp/Vp are
 * caller-owned, same shapes as Q/K/V; any of them may be NULL to skip it.
 */
sparsepr_status sparsepr_permute(sparsepr_handle h, const void* Q, const void* K, const void* V,
                                 const sparsepr_partition_t* part, void* Qp, void* Kp, void* Vp,
                                 void* stream);

/*
 * Step (5) [execution and residual paragraphs]: for every group-major query
 * row of group a, exact softmax attention (scale 1/sqrt(d)) over the union
 * of the key groups that route row a keeps, renormalised over those keys.
 * Qp/Kp/Vp are group-major (sparsepr_permute). Osp: bf16 [B][Hq][N][d] in
 * group-major query order (caller-owned). lse: fp32 [B][Hq][N] natural-log
 * softmax denominators of the scaled logits, or NULL.
 */
sparsepr_status sparsepr_blocksparse_attn(sparsepr_handle h, const void* Qp, const void* Kp,
                                          const void* Vp, const sparsepr_partition_t* part,
                                          const sparsepr_route_t* route, void* Osp, float* lse,
                                          void* stream);

/*
 * Step (6) [probe paragraph]: dense attention of the M probe rows of every
 * query head over all N keys, residuals R = O_dense - O_sparse (O_sparse read
 * from Osp at probe_pos), coverage-weighted centred ridge fit of R on
 * O_sparse (lambda), and the top-r left singular subspace of the weighted
 * residuals. Q/K/V in original order; Osp as written by
 * sparsepr_blocksparse_attn. *out receives pointers to handle-owned buffers.
 */
sparsepr_status sparsepr_probe_fit(sparsepr_handle h, const void* Q, const void* K, const void* V,
                                   const sparsepr_partition_t* part, const void* Osp,
                                   sparsepr_fit_t* out, void* stream);

/*
 * Step (7) [probe and execution paragraphs]: O[qperm[p]] = Osp[p] + delta(Osp[p])
 * for every group-major row p, then the probe rows are overwritten with
 * their dense outputs. O: bf16 [B][Hq][N][d], original order, caller-owned.
 * fit = NULL: the rows only return to the original order (no correction, no
 * probe override), e.g. for sparsepr_affine_diagnostics.
 */
sparsepr_status sparsepr_writeback(sparsepr_handle h, const sparsepr_partition_t* part,
                                   const void* Osp, const sparsepr_fit_t* fit, void* O, void* stream);

/*
 * The whole call, steps (1)-(7), with handle-owned intermediates: Q/K/V in,
 * O (bf16 [B][Hq][N][d], original order, caller-owned) out. Enqueues all
 * kernels on `stream` with no host synchronisation.
 */
sparsepr_status sparsepr_attention(sparsepr_handle h, const void* Q, const void* K, const void* V,
                                   void* O, void* stream);

/*
 * Same as sparsepr_attention but Q/K/V/O are HOST buffers (pinned or
 * pageable): copies them to and from the handle's device staging buffers and
 * synchronises before returning. The KV heads are processed in up to nine
 * chunks, each by an internal sub-handle, on up to eight internal streams, so
 * the copies of some chunks overlap the compute of others; the output equals that of
 * sparsepr_attention bit for bit. The first call allocates the staging
 * buffers (4 tensors of the call's size) and the sub-handles.
 */
sparsepr_status sparsepr_attention_host(sparsepr_handle h, const void* Q, const void* K,
                                        const void* V, void* O, void* stream);

/*
 * Shared-route support diagnostic [support paragraph: a route shared by the
 * queries of a group must cover the union of their supports]. For every query
 * group a of every KV head z, up to SPARSEPR_SHARED_ROWS rows stand for the
 * group: its group-major positions lo + floor((m + 1/2) size / R'),
 * R' = min(SPARSEPR_SHARED_ROWS, size), row m taken in query head m mod (Hq/Hkv).
 * Each row's logits against all N keys (q.k/sqrt(d), fp32) give its 90%-mass
 * set (keys in descending logit until 90% of the softmax mass is reached; every
 * key tied with the last one counts) and its count.
 *   row_frac   [B*Hkv][Gq][SPARSEPR_SHARED_ROWS] fp32, device: each row's count / N
 *              (0 past R')
 *   union_frac [B*Hkv][Gq] fp32, device: |union of the R' sets| / N (0 for an
 *              empty group)
 *   workspace  caller-owned device memory of at least the `min_bytes` that
 *              sparsepr_shared_support_workspace reports (16-byte aligned); more
 *              (up to `all_bytes`) lets more KV heads run per pass.
 * `part` may be handle-owned or handed in (only qperm and qoff are read).
 * Not part of the attention call; it writes no handle state. Returns
 * SPARSEPR_ERR_WORKSPACE when the workspace is too small.
 */
#define SPARSEPR_SHARED_ROWS 8
sparsepr_status sparsepr_shared_support_workspace(sparsepr_handle h, size_t* min_bytes, size_t* all_bytes);
sparsepr_status sparsepr_shared_support(sparsepr_handle h, const void* Q, const void* K,
                                        const sparsepr_partition_t* part, float* row_frac, float* union_frac,
                                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * Affine diagnostics of the hard-drop residual [partition paragraph: the residual of a
 * response-coupled partition is closer to an affine function of the sparse output]. For every
 * query head x, R = Od - Os over all N rows and the least-squares affine fit R ~ A Os + b
 * (fp64 throughout). out[2x] = 1 - SSE / sum_i ||R_i - mean R||^2 (affine-explainable
 * fraction), out[2x+1] = SSE / sum_i ||R_i||^2 (affine-orthogonal energy); NaN (and
 * SPARSEPR_DEV_BOUNDS in the device status) if [Os, 1] is rank deficient.
 *   Os, Od     bf16 [B][Hq][N][d], device, original row order: the uncorrected sparse output
 *              (e.g. sparsepr_blocksparse_attn followed by sparsepr_writeback with fit = NULL)
 *              and the dense output (sparsepr_dense_attn)
 *   out        double [B*Hq][2], device
 *   workspace  caller-owned device memory of sparsepr_affine_diagnostics_workspace bytes
 *              (8-byte aligned)
 */
sparsepr_status sparsepr_affine_diagnostics_workspace(sparsepr_handle h, size_t* bytes);
sparsepr_status sparsepr_affine_diagnostics(sparsepr_handle h, const void* Os, const void* Od, double* out,
                                            void* workspace, size_t workspace_bytes, void* stream);

/* Dense softmax attention (scale 1/sqrt(d)) of every query over all keys: the baseline. */
sparsepr_status sparsepr_dense_attn(sparsepr_handle h, const void* Q, const void* K, const void* V,
                                    void* O, void* stream);

/*
 * Statistics of the last sparsepr_attention / sparsepr_route call on the
 * handle. Waits for that call's work to finish (event synchronisation).
 */
sparsepr_status sparsepr_get_stats(sparsepr_handle h, sparsepr_stats* out);

/* Device status word (0 = OK) after the caller has synchronised; clears it. */
sparsepr_status sparsepr_device_status(sparsepr_handle h, int* out);

/*
 * Record the stage boundaries of the following sparsepr_attention calls into
 * the caller's 7 cudaEvent_t handles (passed as void*): events[i] before
 * stage i for i = 0..5 (partition, route, permute, attention, probe + fit,
 * write-back) and events[6] after the write-back. The events are recorded on
 * the call's stream; the caller owns them and reads them after synchronising.
 * NULL stops recording into caller events. No device memory is allocated.
 */
sparsepr_status sparsepr_set_stage_events(sparsepr_handle h, void* const* events);

/*
 * Allocation-free dense attention of given query rows (the probe-row pass of
 * sparsepr_probe_fit without a handle). The paper has no counterpart: this
 * entry point exists for callers that cannot call cudaMalloc -- code inside a
 * framework whose memory manager owns every device allocation, code that runs
 * while an allocator lock is held, or a process that reserves its device
 * memory up front. It allocates nothing: the caller passes inputs and outputs,
 * and the split-key partial results go to a fixed 8 MiB array compiled into the
 * library (every GPU that loads the library holds it until the process exits).
 *   Q        bf16 [B][Hq][N][d], K and V bf16 [B][Hkv][N][d] (device, 16-byte aligned)
 *   rows     int32 [B*Hkv][M] (device, 4-byte aligned): original query rows, shared by the KV
 *            head's query heads; each must satisfy 0 <= row < N. A row outside that range reads
 *            no memory: its query is taken as zero, so its output row is the mean of V.
 *   O        fp32 [B*Hq][M][d] (device, caller-owned): softmax(q K^T / sqrt(d)) V per row
 *   d in {64, 128}, 1 <= M <= min(N, 64)
 * Limit: B*Hq*M*(d+2)*4 bytes must fit in the 8 MiB array (e.g. 24 heads x 64
 * rows x d=128 uses 0.8 MB per key split, so 10 splits); larger requests return
 * SPARSEPR_ERR_UNSUPPORTED without touching the device. Every call looks up the
 * array's device address in the current context (cudaGetSymbolAddress, with the
 * caller's device current), so the address stays right after cudaDeviceReset or a
 * context switch; the first call on a device may load the library's device code, so
 * make that first call before any stream capture.
 * Every call uses the same array: calls whose work overlaps on a GPU (two streams,
 * two threads) race on it and must be serialised by the caller. No part of the
 * array needs to start at zero: each call writes every slot it later reads.
 */
sparsepr_status sparsepr_probe_attention_noalloc(const void* Q, const void* K, const void* V,
                                                 const int32_t* rows, float* O, int B, int Hq, int Hkv,
                                                 int N, int d, int M, void* stream);

/* Number of kernel launches the last sparsepr_attention call enqueued. */
sparsepr_status sparsepr_last_launch_count(sparsepr_handle h, int* out);

#ifdef __cplusplus
}
#endif

#endif /* SPARSEPR_H */
