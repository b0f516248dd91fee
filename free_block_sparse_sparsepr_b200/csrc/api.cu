// C ABI of the SparsePR library: argument validation, workspace, and the
// orchestration of the seven steps on one CUDA stream (no host synchronisation
// inside the call).
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <new>
#include <vector>

#include "sparsepr.h"
#include "common.cuh"
#include "kernels.h"

using spr::bf16;

namespace {

constexpr int kMaxGroups = 1024;
constexpr int kProbeSplits = 32;
constexpr int kSortChunk = 2048;   // rows per counting-sort chunk (matches the sort kernels)
constexpr unsigned kSupportedFlags =
    SPARSEPR_FLAG_HARD_DROP_ONLY | SPARSEPR_FLAG_RIDGE_ONLY | SPARSEPR_FLAG_RBAR_UNPROJECTED |
    SPARSEPR_FLAG_UNIFORM_WEIGHTS | SPARSEPR_FLAG_TOPMASS | SPARSEPR_FLAG_STAGE_TIMING |
    SPARSEPR_FLAG_PROBES_UNIFORM | SPARSEPR_FLAG_PROBES_RANDOM | SPARSEPR_FLAG_SEMANTIC_PARTITION |
    SPARSEPR_FLAG_TEST_STALL;

inline int pad16(int v) { return (v + 15) / 16 * 16; }
inline int pad64(int v) { return (v + 63) / 64 * 64; }

enum Stage { kStPartition = 0, kStRoute, kStPermute, kStAttn, kStProbeFit, kStWriteback, kStUnused, kStTotal, kNumStages };

constexpr int kHostChunks = 9;     // KV-head chunks of the host-buffer pipeline
// Compute streams of the pipeline, taken by the chunks in turn: the latency-bound steps of a
// chunk (the route selection, the fit, the small k-means kernels of a few heads) then overlap
// other chunks' throughput-bound kernels instead of running alone.
constexpr int kHostStreams = 8;
// Relative chunk sizes: small at both ends, so that the first chunk's inputs land and the last
// chunk's output leaves quickly (a head's copy in is shorter than its call, so after the first
// chunks the copies stay ahead of the compute).
constexpr int kChunkWeight[kHostChunks] = {1, 2, 3, 4, 4, 4, 3, 2, 1};

// Chunk boundaries z0[0..nc] of P KV heads: one head per chunk up to kHostChunks heads, else the
// weights scaled to P (largest remainders, at least one head each).
int host_chunks(int P, int* z0) {
    if (P <= kHostChunks) {
        for (int i = 0; i <= P; ++i) z0[i] = i;
        return P;
    }
    int wsum = 0;
    for (int i = 0; i < kHostChunks; ++i) wsum += kChunkWeight[i];
    int size[kHostChunks], left = P;
    long long rem[kHostChunks];
    for (int i = 0; i < kHostChunks; ++i) {
        const long long num = (long long)kChunkWeight[i] * P;
        size[i] = (int)(num / wsum);
        if (size[i] < 1) size[i] = 1;
        rem[i] = num % wsum;
        left -= size[i];
    }
    while (left > 0) {   // the largest remainders (earliest on ties) take the heads still unassigned
        int b = 0;
        for (int i = 1; i < kHostChunks; ++i)
            if (rem[i] > rem[b]) b = i;
        ++size[b];
        rem[b] = -1;
        --left;
    }
    while (left < 0) {   // the clamp to one head overshot: the largest chunks give heads back
        int b = 0;
        for (int i = 1; i < kHostChunks; ++i)
            if (size[i] > size[b]) b = i;
        --size[b];
        ++left;
    }
    z0[0] = 0;
    for (int i = 0; i < kHostChunks; ++i) z0[i + 1] = z0[i] + size[i];
    return kHostChunks;
}

}  // namespace

// Host-buffer pipeline: one sub-handle per contiguous chunk of flattened KV heads (every step is
// per KV head, so the chunks reproduce the whole call), with the copies in, the chunk calls and
// the copies out on three streams so that transfers overlap the compute of other chunks.
struct HostPipe {
    int nc = 0;
    int z0[kHostChunks + 1] = {};
    sparsepr_handle_s* sub[kHostChunks] = {};
    cudaStream_t in = nullptr, comp[kHostStreams] = {}, out = nullptr;   // chunk i on compute stream i % kHostStreams
    cudaEvent_t start = nullptr, end_comp[kHostStreams] = {}, end_out = nullptr;
    cudaEvent_t ev_in[kHostChunks] = {}, ev_done[kHostChunks] = {};
};

struct sparsepr_handle_s {
    sparsepr_config cfg;
    int P = 0, Hp = 0, g = 0, M = 0;     // M = probes actually used (0 under hard drop)
    int DPk = 0, Dy = 0, DPy = 0, Gkp = 0, nch = 0, Gmax = 0;
    bool proj = false;
    size_t bytes = 0;
    std::vector<void*> allocs;
    // partition
    int32_t *kgroup = nullptr, *qgroup = nullptr, *kperm = nullptr, *koff = nullptr, *qperm = nullptr,
            *qoff = nullptr, *probe = nullptr, *probe_pos = nullptr, *probe_seq = nullptr;
    float* topmass = nullptr;
    unsigned* colmax = nullptr;          // column maxima of the responses (support diagnostic)
    float *kcent = nullptr, *radial = nullptr, *weights = nullptr, *features = nullptr, *ycoord = nullptr,
          *kdist = nullptr, *kmC = nullptr;
    int *counts = nullptr, *bases = nullptr, *km_changed = nullptr, *km_done = nullptr;
    bf16 *Qs = nullptr, *chi = nullptr, *clo = nullptr, *uhi = nullptr, *ulo = nullptr, *projT = nullptr;
    float *u = nullptr, *ulse = nullptr;
    // route
    float* scores = nullptr;
    int32_t *rowptr = nullptr, *kg = nullptr, *tile_off = nullptr, *ktile_cnt = nullptr, *ktile_off = nullptr;
    int2* ktile_list = nullptr;
    int64_t* pairs = nullptr;
    // permuted tensors and sparse output
    bf16 *Qp = nullptr, *Kp = nullptr, *Vp = nullptr, *Osp = nullptr;
    bf16* Qpr = nullptr;                 // gathered probe rows [Hp][128][d] (tensor-core probe pass)
    bf16* wbparts = nullptr;             // bf16 parts of Bm and U^T (tensor-core write-back)
    float* lse = nullptr;
    // probes and fit
    float *Opart = nullptr, *mpart = nullptr, *lpart = nullptr, *Odense = nullptr, *R = nullptr,
          *Xprobe = nullptr, *obar = nullptr, *Rbar = nullptr, *A = nullptr, *U = nullptr, *Bm = nullptr,
          *c0 = nullptr;
    int32_t* rank = nullptr;
    int* dev_status = nullptr;
    // host-buffer variant staging (allocated on first use)
    bf16 *sQ = nullptr, *sK = nullptr, *sV = nullptr, *sO = nullptr;
    struct HostPipe* pipe = nullptr;   // host-buffer pipeline over KV-head chunks (first use)
    // timing
    cudaEvent_t ev[kNumStages + 1] = {};
    cudaEvent_t done_ev = nullptr;
    cudaEvent_t user_ev[7] = {};
    bool user_events = false;
    bool timing = false, timed_call = false;
    // tensor-core k-means operands
    bf16 *kmX2 = nullptr, *kmC2 = nullptr;
    float *kmxx = nullptr, *kmcc = nullptr;
    int4* kmfix = nullptr;
    bool semantic = false;   // ablation: k-means on the raw activations
    int launches = 0;
    int device = 0;
    int num_sms = 148;
};

namespace {

#define SPR_TRY(expr)                                   \
    do {                                                \
        cudaError_t e_ = (expr);                        \
        if (e_ != cudaSuccess) return SPARSEPR_ERR_CUDA; \
        ++h->launches;                                  \
    } while (0)

template <typename T>
sparsepr_status alloc(sparsepr_handle h, T** p, size_t count) {
    if (count == 0) count = 1;
    void* q = nullptr;
    if (cudaMalloc(&q, count * sizeof(T)) != cudaSuccess) return SPARSEPR_ERR_WORKSPACE;
    h->allocs.push_back(q);
    h->bytes += count * sizeof(T);
    *p = static_cast<T*>(q);
    return SPARSEPR_OK;
}

void free_all(sparsepr_handle h) {
    for (void* p : h->allocs) cudaFree(p);
    h->allocs.clear();
    for (auto& e : h->ev)
        if (e) cudaEventDestroy(e);
    if (h->done_ev) cudaEventDestroy(h->done_ev);
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sparsepr_status validate(const sparsepr_config* c) {
    if (!c) return SPARSEPR_ERR_INVALID_ARG;
    if (c->B < 1 || c->Hq < 1 || c->Hkv < 1 || c->Hq % c->Hkv != 0 || c->N < 1) return SPARSEPR_ERR_INVALID_ARG;
    if (c->d != 64 && c->d != 128) return SPARSEPR_ERR_UNSUPPORTED;
    if (c->block != 64 && c->block != 128) return SPARSEPR_ERR_INVALID_ARG;
    if (c->Gk < 1 || c->Gq < 1 || c->Gk > c->N || c->Gq > c->N) return SPARSEPR_ERR_INVALID_ARG;
    if (c->Gk > kMaxGroups || c->Gq > kMaxGroups) return SPARSEPR_ERR_UNSUPPORTED;
    if ((long long)c->Gq * c->Gk > (1ll << 20)) return SPARSEPR_ERR_UNSUPPORTED;
    if (c->rK < 1 || c->rK > 64 || c->rQ < 1 || c->rQ > 64) return SPARSEPR_ERR_INVALID_ARG;
    if (c->kmeans_iters < 0 || c->kmeans_iters > 64) return SPARSEPR_ERR_INVALID_ARG;
    if (!(c->lambda > 0.f) || !isfinite(c->lambda)) return SPARSEPR_ERR_INVALID_ARG;
    if (!(c->rho_exec > 0.f) || !isfinite(c->rho_exec)) return SPARSEPR_ERR_INVALID_ARG;
    if (c->flags & ~kSupportedFlags)
        return SPARSEPR_ERR_INVALID_ARG;
    if ((c->flags & SPARSEPR_FLAG_PROBES_UNIFORM) && (c->flags & SPARSEPR_FLAG_PROBES_RANDOM))
        return SPARSEPR_ERR_INVALID_ARG;
    if ((c->flags & SPARSEPR_FLAG_SEMANTIC_PARTITION) && (c->flags & SPARSEPR_FLAG_TOPMASS))
        return SPARSEPR_ERR_INVALID_ARG;
    if ((c->flags & SPARSEPR_FLAG_TEST_STALL) && !spr::attn_tc_supported(c->d)) return SPARSEPR_ERR_UNSUPPORTED;
    if (!(c->flags & SPARSEPR_FLAG_HARD_DROP_ONLY)) {
        if (c->M < 1 || c->M > c->N) return SPARSEPR_ERR_INVALID_ARG;
        if (c->M > 64) return SPARSEPR_ERR_UNSUPPORTED;
        if (c->r < 1 || c->r > c->M || c->r > 32) return SPARSEPR_ERR_INVALID_ARG;
    }
    if ((long long)c->N * c->Gk > (1ll << 31) || (long long)c->N * 128 > (1ll << 31))
        return SPARSEPR_ERR_UNSUPPORTED;
    return SPARSEPR_OK;
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

void mark(sparsepr_handle h, int stage, cudaStream_t s) {
    if (h->user_events) cudaEventRecord(h->user_ev[stage], s);
    else if (h->timing) cudaEventRecord(h->ev[stage], s);
}

long long budget_pairs(const sparsepr_config& c, int M) {
    const double nn = (double)((long long)c.N * c.N);
    return (long long)floor((double)c.rho_exec * nn) - (long long)M * c.N;
}

// Lloyd k-means on X [P][n][DP] into G groups, then the stable group-major order. With
// G <= 256 the assignment runs on tensor cores (bf16 split operands, near ties settled in fp64)
// and the radial distances come from one exact pass after the last assignment.
// rows_split: the caller already wrote the rows' bf16 parts and squared norms (kmX2, kmxx).
// need_dist: the rows' distances to their centroids are used (the query partition's radial
// key); the key partition's are not, so its exact distance pass is skipped.
sparsepr_status kmeans(sparsepr_handle h, const float* X, int DP, int G, int32_t* labels, float* dist,
                       int32_t* perm, int32_t* off, cudaStream_t s, bool rows_split = false,
                       bool need_dist = true) {
    const int P = h->P, n = h->cfg.N;
    const bool tc = spr::km_tc_supported(G) && DP <= 64;
    auto assign = [&](bool first, const int* done) -> cudaError_t {
        if (!tc) return spr::launch_km_assign(X, h->kmC, labels, dist, h->km_changed, done, P, n, G, DP, first, s);
        cudaError_t e = spr::launch_km_split_cent(h->kmC, h->kmC2, h->kmcc, P, G, DP, s);
        if (e != cudaSuccess) return e;
        ++h->launches;
        return spr::launch_km_assign_tc(X, h->kmX2, h->kmxx, h->kmC, h->kmC2, h->kmcc, labels, h->km_changed, done,
                                        h->kmfix, h->dev_status, P, n, G, DP, first, h->num_sms, s);
    };
    SPR_TRY(spr::launch_km_reset(h->km_changed, h->km_done, P, s));
    if (tc && !rows_split) SPR_TRY(spr::launch_km_split_rows(X, h->kmX2, h->kmxx, P, n, DP, s));
    SPR_TRY(spr::launch_km_seed(X, h->kmC, P, n, G, DP, s));
    SPR_TRY(assign(true, nullptr));
    for (int it = 0; it < h->cfg.kmeans_iters; ++it) {
        SPR_TRY(spr::launch_group_sort(labels, perm, off, h->counts, h->bases, h->km_done, P, n, G, s));
        h->launches += 2;  // histogram, scan and scatter kernels
        SPR_TRY(spr::launch_km_update(X, perm, off, h->kmC, h->km_done, P, n, G, DP, s));
        SPR_TRY(assign(false, h->km_done));
        SPR_TRY(spr::launch_km_check(h->km_changed, h->km_done, P, s));
    }
    if (tc && need_dist) SPR_TRY(spr::launch_km_dist(X, h->kmC, labels, dist, P, n, G, DP, s));
    SPR_TRY(spr::launch_group_sort(labels, perm, off, h->counts, h->bases, nullptr, P, n, G, s));
    h->launches += 2;
    return SPARSEPR_OK;
}

// u[x] = Q[x] . kcent[z]^T / sqrt(d) with kcent split into bf16 hi + lo, and the routing normaliser
// ulse[x][i] = log sum_g |K_g| exp(u[x][i][g]) (fused into the tensor-core kernel's epilogue).
sparsepr_status query_logits(sparsepr_handle h, const bf16* Q, const bf16* chi, const bf16* clo,
                             const int32_t* koff, cudaStream_t s) {
    const sparsepr_config& c = h->cfg;
    if (spr::logits_tc_supported(c.d, c.Gk)) {
        SPR_TRY(spr::launch_logits_tc(Q, chi, clo, koff, h->u, h->ulse, h->dev_status, c.B, c.Hq, c.Hkv, c.N, c.Gk,
                                      h->num_sms, s));
        return SPARSEPR_OK;
    }
    spr::GemmArgs a;
    memset(&a, 0, sizeof(a));
    a.A1 = Q; a.A2 = nullptr; a.sA = (long long)c.N * c.d; a.lda = c.d;
    a.B1 = chi; a.B2 = clo; a.sB = (long long)c.Gk * c.d; a.ldb = c.d; a.bdiv = h->g;
    a.C = h->u; a.sC = (long long)c.N * c.Gk; a.ldc = c.Gk;
    a.M = c.N; a.N = c.Gk; a.K = c.d; a.batch = h->Hp;
    a.alpha = (float)(1.0 / sqrt((double)c.d));
    SPR_TRY(spr::launch_gemm_bf16(a, s));
    SPR_TRY(spr::launch_row_lse(h->u, koff, h->ulse, h->Hp, h->g, c.N, c.Gk, s));
    return SPARSEPR_OK;
}

sparsepr_status probes_impl(sparsepr_handle h, cudaStream_t s);

// Semantic-partition ablation ([partition]): key groups from the raw keys and query groups from
// the raw mean query of each KV group (fp32 rows of width d), everything after as in the
// response-coupled partition; the query logits are still formed for the routing.
sparsepr_status partition_semantic(sparsepr_handle h, const bf16* Q, const bf16* K, cudaStream_t s) {
    const sparsepr_config& c = h->cfg;
    const int P = h->P, N = c.N, d = c.d;
    SPR_TRY(spr::launch_mean_heads_f32(K, h->features, P, 1, N, d, s));
    sparsepr_status st = kmeans(h, h->features, d, c.Gk, h->kgroup, h->kdist, h->kperm, h->koff, s, false, false);
    if (st) return st;
    SPR_TRY(spr::launch_group_mean_bf16(K, h->kperm, h->koff, h->kcent, h->chi, h->clo, P, N, c.Gk, d, s));
    st = query_logits(h, Q, h->chi, h->clo, h->koff, s);
    if (st) return st;
    SPR_TRY(spr::launch_mean_heads_f32(Q, h->ycoord, P, h->g, N, d, s));
    st = kmeans(h, h->ycoord, d, c.Gq, h->qgroup, h->radial, h->qperm, h->qoff, s);
    if (st) return st;
    return probes_impl(h, s);
}

sparsepr_status partition_impl(sparsepr_handle h, const bf16* Q, const bf16* K, cudaStream_t s) {
    const sparsepr_config& c = h->cfg;
    const int P = h->P, N = c.N, d = c.d;
    if (h->semantic) return partition_semantic(h, Q, K, s);
    // (1) sampled responses: F[z] = K[z] . Qs[z]^T / sqrt(d); on the tensor cores the same pass
    // writes the key k-means operands and (support diagnostic) the column maxima
    const bool topmass = (c.flags & SPARSEPR_FLAG_TOPMASS) != 0;
    SPR_TRY(spr::launch_gather_samples(Q, h->Qs, c.B, c.Hq, c.Hkv, N, d, c.rK, h->DPk, s));
    const bool resp_tc = spr::resp_tc_supported(d, h->DPk);
    if (resp_tc) {
        SPR_TRY(spr::launch_resp_tc(K, h->Qs, h->features, h->kmX2, h->kmxx, topmass ? h->colmax : nullptr, P, N, d,
                                    h->DPk, c.rK, h->num_sms, h->dev_status, s));
        if (topmass) ++h->launches;   // the memset of the maxima
    } else {
        spr::GemmArgs a;
        memset(&a, 0, sizeof(a));
        a.A1 = K; a.sA = (long long)N * d; a.lda = d;
        a.B1 = h->Qs; a.sB = (long long)h->DPk * d; a.ldb = d; a.bdiv = 1;
        a.C = h->features; a.sC = (long long)N * h->DPk; a.ldc = h->DPk;
        a.M = N; a.N = h->DPk; a.K = d; a.batch = P;
        a.alpha = (float)(1.0 / sqrt((double)d));
        SPR_TRY(spr::launch_gemm_bf16(a, s));
    }
    if (topmass)
        SPR_TRY(spr::launch_topmass(h->features, h->topmass, resp_tc ? h->colmax : nullptr, P, N, h->DPk, c.rK, s));
    // (2a) key groups and their means in the original key space
    const bool key_rows_split = resp_tc && spr::km_tc_supported(c.Gk);
    sparsepr_status st = kmeans(h, h->features, h->DPk, c.Gk, h->kgroup, h->kdist, h->kperm, h->koff, s,
                                key_rows_split, false);
    if (st) return st;
    SPR_TRY(spr::launch_group_mean_bf16(K, h->kperm, h->koff, h->kcent, h->chi, h->clo, P, N, c.Gk, d, s));
    // (2b) query coordinates and query groups
    st = query_logits(h, Q, h->chi, h->clo, h->koff, s);
    if (st) return st;
    if (h->proj && spr::coords_proj_supported(h->DPy, c.Gk, h->Gkp)) {
        // centring, projection and normalisation in one pass over the logits
        SPR_TRY(spr::launch_coords_proj(h->u, h->projT, h->ycoord, P, h->g, N, c.Gk, h->Gkp, h->num_sms, s));
    } else {
        SPR_TRY(spr::launch_coords_center(h->u, h->uhi, h->ulo, h->ycoord, P, h->g, N, c.Gk, h->Gkp, h->DPy, h->proj,
                                          s));
    }
    if (h->proj && !spr::coords_proj_supported(h->DPy, c.Gk, h->Gkp)) {
        spr::GemmArgs b;
        memset(&b, 0, sizeof(b));
        b.A1 = h->uhi; b.A2 = h->ulo; b.sA = (long long)N * h->Gkp; b.lda = h->Gkp;
        b.B1 = h->projT; b.B2 = nullptr; b.sB = 0; b.ldb = h->Gkp; b.bdiv = 1;
        b.C = h->ycoord; b.sC = (long long)N * h->DPy; b.ldc = h->DPy;
        b.M = N; b.N = h->DPy; b.K = h->Gkp; b.batch = P; b.alpha = 1.f;
        SPR_TRY(spr::launch_gemm_bf16(b, s));
        SPR_TRY(spr::launch_rows_normalize(h->ycoord, P * N, h->DPy, s));
    }
    st = kmeans(h, h->ycoord, h->DPy, c.Gq, h->qgroup, h->radial, h->qperm, h->qoff, s);
    if (st) return st;
    return probes_impl(h, s);
}

// Probe rows (stratified, radial order; or an ablation's grid / random draws) and their weights.
sparsepr_status probes_impl(sparsepr_handle h, cudaStream_t s) {
    const sparsepr_config& c = h->cfg;
    const int P = h->P, N = c.N;
    if (h->M) {
        if (c.flags & (SPARSEPR_FLAG_PROBES_UNIFORM | SPARSEPR_FLAG_PROBES_RANDOM))
            SPR_TRY(spr::launch_probe_alt(h->qperm, h->qoff, h->qgroup, h->probe, h->probe_pos, h->probe_seq, P, N,
                                          c.Gq, h->M, (c.flags & SPARSEPR_FLAG_PROBES_RANDOM) != 0, c.seed,
                                          h->dev_status, s));
        else
            SPR_TRY(spr::launch_probe_select(h->qperm, h->qoff, h->radial, h->probe, h->probe_pos, h->probe_seq,
                                         P, N, c.Gq, h->M, s));
        SPR_TRY(spr::launch_probe_weights(h->qoff, h->probe_seq, h->weights, P, N, c.Gq, h->M,
                                          (c.flags & SPARSEPR_FLAG_UNIFORM_WEIGHTS) != 0, s));
    }
    return SPARSEPR_OK;
}

void fill_partition(sparsepr_handle h, sparsepr_partition_t* p) {
    p->kgroup = h->kgroup; p->qgroup = h->qgroup; p->kperm = h->kperm; p->koff = h->koff;
    p->qperm = h->qperm; p->qoff = h->qoff; p->kcent = h->kcent; p->radial = h->radial;
    p->probe = h->probe; p->probe_pos = h->probe_pos; p->weights = h->weights; p->features = h->features;
    p->topmass = (h->cfg.flags & SPARSEPR_FLAG_TOPMASS) ? h->topmass : nullptr;
}

void fill_route(sparsepr_handle h, sparsepr_route_t* r) {
    r->rowptr = h->rowptr; r->kg = h->kg; r->scores = h->scores; r->pairs = h->pairs;
}

void fill_fit(sparsepr_handle h, sparsepr_fit_t* f) {
    f->obar = h->obar; f->Rbar = h->Rbar; f->A = h->A; f->U = h->U; f->Bm = h->Bm; f->c0 = h->c0;
    f->rank = h->rank; f->R = h->R; f->Odense = h->Odense; f->Osp = h->Xprobe;
}

sparsepr_status check_partition(const sparsepr_partition_t* p, bool need_probe) {
    if (!p || !p->kperm || !p->koff || !p->qperm || !p->qoff || !p->kcent) return SPARSEPR_ERR_INVALID_ARG;
    if (need_probe && (!p->probe || !p->probe_pos || !p->weights)) return SPARSEPR_ERR_INVALID_ARG;
    return SPARSEPR_OK;
}

sparsepr_status route_impl(sparsepr_handle h, const bf16* Q, const sparsepr_partition_t* p, bool logits_ready,
                           cudaStream_t s) {
    const sparsepr_config& c = h->cfg;
    if (!logits_ready) {
        SPR_TRY(spr::launch_split_bf16(p->kcent, h->chi, h->clo, (long long)h->P * c.Gk * c.d, s));
        sparsepr_status st = query_logits(h, Q, h->chi, h->clo, p->koff, s);
        if (st) return st;
    }
    SPR_TRY(spr::launch_cell_scores(h->u, h->ulse, p->qperm, p->qoff, p->koff, h->scores, h->P, h->g, c.N,
                                    c.Gq, c.Gk, s));
    SPR_TRY(spr::launch_route_select(h->scores, p->qoff, p->koff, h->rowptr, h->kg, h->pairs, h->P, c.Gq, c.Gk,
                                     budget_pairs(c, h->M), c.rho_exec >= 1.0f, s));
    return SPARSEPR_OK;
}

sparsepr_status permute_impl(sparsepr_handle h, const bf16* Q, const bf16* K, const bf16* V,
                             const sparsepr_partition_t* p, bf16* Qp, bf16* Kp, bf16* Vp, cudaStream_t s) {
    const sparsepr_config& c = h->cfg;
    if (Qp) SPR_TRY(spr::launch_permute_rows(Q, Qp, p->qperm, h->Hp, h->g, c.N, c.d, s));
    if (Kp) SPR_TRY(spr::launch_permute_rows(K, Kp, p->kperm, h->P, 1, c.N, c.d, s));
    if (Vp) SPR_TRY(spr::launch_permute_rows(V, Vp, p->kperm, h->P, 1, c.N, c.d, s));
    return SPARSEPR_OK;
}

sparsepr_status attn_impl(sparsepr_handle h, const bf16* Qp, const bf16* Kp, const bf16* Vp,
                          const sparsepr_partition_t* p, const sparsepr_route_t* r, bf16* Osp, float* lse,
                          cudaStream_t s) {
    const sparsepr_config& c = h->cfg;
    if (spr::attn_tc_supported(c.d)) {
        SPR_TRY(spr::launch_tile_offsets(p->qoff, h->tile_off, h->P, c.Gq, spr::attn_tc_rows_per_cta(h->g), s));
        SPR_TRY(spr::launch_key_tiles(r->rowptr, r->kg, p->koff, h->ktile_cnt, h->ktile_off, h->ktile_list, h->P, c.N,
                                      c.Gq, c.Gk, s));
        h->launches += 2;  // count, scan and write kernels
        SPR_TRY(spr::launch_attn_sparse_tc(Qp, Kp, Vp, p->qoff, h->tile_off, h->ktile_list, h->ktile_off, Osp, lse,
                                           c.B, c.Hq, c.Hkv, c.N, c.d, c.Gq, h->dev_status, s));
        return SPARSEPR_OK;
    }
    SPR_TRY(spr::launch_tile_offsets(p->qoff, h->tile_off, h->P, c.Gq, 64, s));
    SPR_TRY(spr::launch_attn_sparse(Qp, Kp, Vp, p->qoff, p->koff, h->tile_off, r->rowptr, r->kg, Osp, lse,
                                    c.B, c.Hq, c.Hkv, c.N, c.d, c.Gq, c.Gk, s));
    return SPARSEPR_OK;
}

sparsepr_status probe_fit_impl(sparsepr_handle h, const bf16* Q, const bf16* K, const bf16* V,
                               const sparsepr_partition_t* p, const bf16* Osp, cudaStream_t s) {
    const sparsepr_config& c = h->cfg;
    if (!h->M) return SPARSEPR_OK;
    if (spr::attn_tc_supported(c.d)) {
        // dense attention of the probe rows on the tensor cores, split over the keys
        SPR_TRY(spr::launch_gather_probe_rows(Q, p->probe, h->Qpr, c.B, c.Hq, c.Hkv, c.N, h->M, c.d, 128, s));
        SPR_TRY(spr::launch_attn_probe_tc(h->Qpr, K, V, h->Opart, h->mpart, h->lpart, c.B, c.Hq, c.Hkv, c.N, c.d,
                                          h->M, kProbeSplits, h->dev_status, s));
        SPR_TRY(spr::launch_probe_combine(h->Opart, h->mpart, h->lpart, h->Odense, h->Hp, h->M,
                                          spr::probe_tc_splits(c.N, kProbeSplits), c.d, s));
    } else {
        SPR_TRY(spr::launch_attn_probe(Q, K, V, p->probe, h->Opart, h->mpart, h->lpart, h->Odense, c.B, c.Hq, c.Hkv,
                                       c.N, c.d, h->M, kProbeSplits, s));
        ++h->launches;  // combine kernel
    }
    SPR_TRY(spr::launch_probe_residual(h->Odense, Osp, p->probe_pos, h->R, h->Xprobe, h->Hp, h->g, c.N, c.d,
                                       h->M, s));
    SPR_TRY(spr::launch_fit(h->R, h->Xprobe, p->weights, c.lambda, h->obar, h->Rbar, h->A, h->U, h->Bm, h->c0,
                            h->rank, h->Hp, h->g, c.d, h->M, c.r, (c.flags & SPARSEPR_FLAG_RBAR_UNPROJECTED) != 0,
                            h->dev_status, s));
    return SPARSEPR_OK;
}

sparsepr_status writeback_impl(sparsepr_handle h, const sparsepr_partition_t* p, const bf16* Osp,
                               const sparsepr_fit_t* f, bf16* O, cudaStream_t s) {
    const sparsepr_config& c = h->cfg;
    const bool correct = h->M > 0 && f != nullptr;
    if (correct && (c.flags & SPARSEPR_FLAG_RIDGE_ONLY)) {
        SPR_TRY(spr::launch_writeback_ridge(Osp, p->qperm, f->A, f->obar, f->Rbar, O, h->Hp, h->g, c.N, c.d,
                                            h->num_sms, s));
    } else if (correct && h->wbparts && spr::wb_tc_supported(c.d, c.r)) {
        const float* radd = (c.flags & SPARSEPR_FLAG_RBAR_UNPROJECTED) ? f->Rbar : nullptr;
        SPR_TRY(spr::launch_writeback_tc(Osp, p->qperm, f->U, f->Bm, f->c0, radd, h->wbparts, O, h->Hp, h->g, c.N, c.r,
                                         h->dev_status, h->num_sms, s));
        ++h->launches;   // the split of Bm and U^T into bf16 parts
    } else {
        const float* radd = (correct && (c.flags & SPARSEPR_FLAG_RBAR_UNPROJECTED)) ? f->Rbar : nullptr;
        SPR_TRY(spr::launch_writeback(Osp, p->qperm, correct ? f->U : nullptr, correct ? f->Bm : nullptr,
                                      correct ? f->c0 : nullptr, radd, O, h->Hp, h->g, c.N, c.d, correct ? c.r : 1,
                                      correct, h->num_sms, s));
    }
    if (correct) SPR_TRY(spr::launch_probe_override(f->Odense, p->probe, O, h->Hp, h->g, c.N, c.d, h->M, s));
    return SPARSEPR_OK;
}

}  // namespace

extern "C" {

const char* sparsepr_status_string(sparsepr_status s) {
    switch (s) {
        case SPARSEPR_OK: return "ok";
        case SPARSEPR_ERR_INVALID_ARG: return "invalid argument";
        case SPARSEPR_ERR_UNSUPPORTED: return "unsupported configuration";
        case SPARSEPR_ERR_WORKSPACE: return "workspace allocation failed";
        case SPARSEPR_ERR_CUDA: return "CUDA error";
        case SPARSEPR_ERR_TIMEOUT: return "device wait timed out";
        case SPARSEPR_ERR_DEVICE: return "device-side check failed";
    }
    return "unknown status";
}

int sparsepr_version(void) { return 100; }

sparsepr_status sparsepr_create(const sparsepr_config* cfg, sparsepr_handle* out) {
    if (!out) return SPARSEPR_ERR_INVALID_ARG;
    *out = nullptr;
    sparsepr_status st = validate(cfg);
    if (st) return st;
    sparsepr_handle h = new (std::nothrow) sparsepr_handle_s();
    if (!h) return SPARSEPR_ERR_WORKSPACE;
    h->cfg = *cfg;
    const sparsepr_config& c = h->cfg;
    cudaGetDevice(&h->device);
    if (cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess || h->num_sms < 1)
        h->num_sms = 148;
    h->P = c.B * c.Hkv;
    h->Hp = c.B * c.Hq;
    h->g = c.Hq / c.Hkv;
    h->M = (c.flags & SPARSEPR_FLAG_HARD_DROP_ONLY) ? 0 : c.M;
    h->semantic = (c.flags & SPARSEPR_FLAG_SEMANTIC_PARTITION) != 0;
    h->DPk = h->semantic ? c.d : pad16(c.rK);
    h->proj = c.Gk > c.rQ;
    h->Dy = h->proj ? c.rQ : c.Gk;
    h->DPy = h->semantic ? c.d : pad16(h->Dy);
    h->Gkp = pad64(c.Gk);
    h->nch = (c.N + kSortChunk - 1) / kSortChunk;
    h->Gmax = c.Gk > c.Gq ? c.Gk : c.Gq;
    h->timing = (c.flags & SPARSEPR_FLAG_STAGE_TIMING) != 0;
    const size_t P = h->P, Hp = h->Hp, N = c.N, d = c.d, M = h->M > 0 ? h->M : 1, r = c.r > 0 ? c.r : 1;
    const size_t Gk = c.Gk, Gq = c.Gq;
#define A_(ptr, n)                                 \
    do {                                           \
        if ((st = alloc(h, &h->ptr, (n)))) {       \
            free_all(h);                           \
            delete h;                              \
            return st;                             \
        }                                          \
    } while (0)
    A_(kgroup, P * N); A_(qgroup, P * N); A_(kperm, P * N); A_(koff, P * (Gk + 1));
    A_(qperm, P * N); A_(qoff, P * (Gq + 1)); A_(probe, P * M); A_(probe_pos, P * M); A_(probe_seq, P * M);
    A_(kcent, P * Gk * d); A_(radial, P * N); A_(weights, P * M); A_(features, P * N * h->DPk); A_(topmass, P * c.rK);
    A_(colmax, P * h->DPk);
    A_(ycoord, P * N * h->DPy); A_(kdist, P * N); A_(kmC, P * h->Gmax * (size_t)(h->DPk > 64 || h->DPy > 64 ? (h->DPk > h->DPy ? h->DPk : h->DPy) : 64));
    A_(counts, P * h->nch * h->Gmax); A_(bases, P * h->nch * h->Gmax); A_(km_changed, P); A_(km_done, P);
    A_(Qs, P * h->DPk * d); A_(chi, P * Gk * d); A_(clo, P * Gk * d);
    A_(u, Hp * N * Gk); A_(ulse, Hp * N);
    if (h->proj) {
        A_(uhi, P * N * h->Gkp); A_(ulo, P * N * h->Gkp); A_(projT, (size_t)h->DPy * h->Gkp);
    }
    A_(scores, P * Gq * Gk); A_(rowptr, P * (Gq + 1)); A_(kg, P * Gq * Gk); A_(tile_off, P * (Gq + 1));
    A_(pairs, P);
    A_(ktile_cnt, P * Gq); A_(ktile_off, P * (Gq + 1));
    A_(ktile_list, P * (size_t)spr::key_tiles_capacity(c.N, c.Gq, c.Gk));
    A_(Qp, Hp * N * d); A_(Kp, P * N * d); A_(Vp, P * N * d); A_(Osp, Hp * N * d); A_(lse, Hp * N);
    A_(Opart, Hp * kProbeSplits * M * d); A_(mpart, Hp * kProbeSplits * M); A_(lpart, Hp * kProbeSplits * M);
    A_(Odense, Hp * M * d); A_(R, Hp * M * d); A_(Xprobe, Hp * M * d);
    if (spr::attn_tc_supported(c.d)) A_(Qpr, Hp * 128 * d);
    if (spr::wb_tc_supported(c.d, (int)r)) A_(wbparts, spr::wb_tc_parts_elems((int)Hp));
    A_(obar, Hp * d); A_(Rbar, Hp * d); A_(A, Hp * d * d); A_(U, Hp * d * r); A_(Bm, Hp * r * d); A_(c0, Hp * r);
    A_(rank, Hp); A_(dev_status, 1);
    {
        const size_t G16 = (size_t)((h->Gmax + 15) / 16 * 16), G32 = (size_t)((h->Gmax + 31) / 32 * 32);
        A_(kmX2, 2 * P * N * 64); A_(kmxx, P * N);
        A_(kmC2, 2 * P * G16 * 64); A_(kmcc, P * G32);
        A_(kmfix, spr::km_fix_slots(P, N, h->num_sms));

    }
#undef A_
    bool ok = cudaMemset(h->dev_status, 0, sizeof(int)) == cudaSuccess;
    if (h->proj) {
        ok = ok && cudaMemset(h->uhi, 0, P * N * h->Gkp * sizeof(bf16)) == cudaSuccess;
        ok = ok && cudaMemset(h->ulo, 0, P * N * h->Gkp * sizeof(bf16)) == cudaSuccess;
        ok = ok && spr::launch_make_projection(h->projT, c.Gk, h->Gkp, c.rQ, h->DPy, c.seed, 0) == cudaSuccess;
    }
    ok = ok && cudaMemset(h->ycoord, 0, P * N * h->DPy * sizeof(float)) == cudaSuccess;
    for (auto& e : h->ev) ok = ok && cudaEventCreate(&e) == cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&h->done_ev, cudaEventDisableTiming) == cudaSuccess;
    ok = ok && cudaDeviceSynchronize() == cudaSuccess;
    if (!ok) {
        free_all(h);
        delete h;
        return SPARSEPR_ERR_CUDA;
    }
    *out = h;
    return SPARSEPR_OK;
}

static void destroy_pipe(HostPipe* pp) {
    if (!pp) return;
    for (int i = 0; i < pp->nc; ++i)
        if (pp->sub[i]) sparsepr_destroy(pp->sub[i]);
    for (cudaStream_t st : {pp->in, pp->out})
        if (st) cudaStreamDestroy(st);
    for (int k = 0; k < kHostStreams; ++k) {
        if (pp->comp[k]) cudaStreamDestroy(pp->comp[k]);
        if (pp->end_comp[k]) cudaEventDestroy(pp->end_comp[k]);
    }
    for (cudaEvent_t e : {pp->start, pp->end_out})
        if (e) cudaEventDestroy(e);
    for (int i = 0; i < kHostChunks; ++i) {
        if (pp->ev_in[i]) cudaEventDestroy(pp->ev_in[i]);
        if (pp->ev_done[i]) cudaEventDestroy(pp->ev_done[i]);
    }
    delete pp;
}

sparsepr_status sparsepr_destroy(sparsepr_handle h) {
    if (!h) return SPARSEPR_OK;
    cudaDeviceSynchronize();
    destroy_pipe(h->pipe);
    if (h->sQ) { cudaFree(h->sQ); cudaFree(h->sK); cudaFree(h->sV); cudaFree(h->sO); }
    free_all(h);
    delete h;
    return SPARSEPR_OK;
}

sparsepr_status sparsepr_workspace_bytes(sparsepr_handle h, size_t* out) {
    if (!h || !out) return SPARSEPR_ERR_INVALID_ARG;
    *out = h->bytes;
    return SPARSEPR_OK;
}

sparsepr_status sparsepr_partition(sparsepr_handle h, const void* Q, const void* K, sparsepr_partition_t* out,
                                   void* stream) {
    if (!h || !aligned16(Q) || !aligned16(K) || !out) return SPARSEPR_ERR_INVALID_ARG;
    h->launches = 0;
    cudaStream_t s = as_stream(stream);
    sparsepr_status st = partition_impl(h, static_cast<const bf16*>(Q), static_cast<const bf16*>(K), s);
    if (st) return st;
    fill_partition(h, out);
    return SPARSEPR_OK;
}

namespace {
constexpr int kShared = SPARSEPR_SHARED_ROWS;
size_t align256(size_t b) { return (b + 255) / 256 * 256; }
size_t shared_rows_bytes(sparsepr_handle h) {
    return align256((size_t)h->P * h->cfg.Gq * kShared * h->cfg.d * sizeof(bf16));
}
size_t shared_head_bytes(sparsepr_handle h) {
    return align256((size_t)h->cfg.Gq * kShared * h->cfg.N * sizeof(float));
}
}  // namespace

sparsepr_status sparsepr_affine_diagnostics_workspace(sparsepr_handle h, size_t* bytes) {
    if (!h || !bytes) return SPARSEPR_ERR_INVALID_ARG;
    *bytes = spr::affine_diag_workspace(h->Hp, h->cfg.d);
    return SPARSEPR_OK;
}

sparsepr_status sparsepr_affine_diagnostics(sparsepr_handle h, const void* Os, const void* Od, double* out,
                                            void* workspace, size_t workspace_bytes, void* stream) {
    if (!h || !aligned16(Os) || !aligned16(Od) || !out || !workspace) return SPARSEPR_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 7u) != 0) return SPARSEPR_ERR_INVALID_ARG;
    if (workspace_bytes < spr::affine_diag_workspace(h->Hp, h->cfg.d)) return SPARSEPR_ERR_WORKSPACE;
    h->launches = 0;
    SPR_TRY(spr::launch_affine_diag(static_cast<const bf16*>(Os), static_cast<const bf16*>(Od), out, workspace,
                                    h->Hp, h->cfg.N, h->cfg.d, h->dev_status, as_stream(stream)));
    ++h->launches;   // the Gram and the solve kernels
    return SPARSEPR_OK;
}

sparsepr_status sparsepr_shared_support_workspace(sparsepr_handle h, size_t* min_bytes, size_t* all_bytes) {
    if (!h || (!min_bytes && !all_bytes)) return SPARSEPR_ERR_INVALID_ARG;
    if (min_bytes) *min_bytes = shared_rows_bytes(h) + shared_head_bytes(h);
    if (all_bytes) *all_bytes = shared_rows_bytes(h) + (size_t)h->P * shared_head_bytes(h);
    return SPARSEPR_OK;
}

sparsepr_status sparsepr_shared_support(sparsepr_handle h, const void* Q, const void* K,
                                        const sparsepr_partition_t* part, float* row_frac, float* union_frac,
                                        void* workspace, size_t workspace_bytes, void* stream) {
    if (!h || !aligned16(Q) || !aligned16(K) || !row_frac || !union_frac || !aligned16(workspace))
        return SPARSEPR_ERR_INVALID_ARG;
    if (!part || !part->qperm || !part->qoff) return SPARSEPR_ERR_INVALID_ARG;
    const sparsepr_config& c = h->cfg;
    const size_t rows_b = shared_rows_bytes(h), head_b = shared_head_bytes(h);
    if (workspace_bytes < rows_b + head_b) return SPARSEPR_ERR_WORKSPACE;
    int hc = (int)((workspace_bytes - rows_b) / head_b);
    if (hc > h->P) hc = h->P;
    h->launches = 0;
    cudaStream_t s = as_stream(stream);
    bf16* Qsh = static_cast<bf16*>(workspace);
    float* Z = reinterpret_cast<float*>(static_cast<char*>(workspace) + rows_b);
    const long long ldz = (long long)(head_b / sizeof(float)) / ((long long)c.Gq * kShared);
    SPR_TRY(spr::launch_shared_rows(static_cast<const bf16*>(Q), part->qperm, part->qoff, Qsh, h->P, h->g, c.N, c.d,
                                    c.Gq, s));
    for (int z0 = 0; z0 < h->P; z0 += hc) {
        const int nz = h->P - z0 < hc ? h->P - z0 : hc;
        spr::GemmArgs a;
        memset(&a, 0, sizeof(a));
        a.A1 = Qsh + (size_t)z0 * c.Gq * kShared * c.d; a.sA = (long long)c.Gq * kShared * c.d; a.lda = c.d;
        a.B1 = static_cast<const bf16*>(K) + (size_t)z0 * c.N * c.d; a.sB = (long long)c.N * c.d; a.ldb = c.d;
        a.bdiv = 1;
        a.C = Z; a.sC = (long long)c.Gq * kShared * ldz; a.ldc = (int)ldz;
        a.M = c.Gq * kShared; a.N = c.N; a.K = c.d; a.batch = nz;
        a.alpha = (float)(1.0 / sqrt((double)c.d));
        SPR_TRY(spr::launch_gemm_bf16(a, s));
        SPR_TRY(spr::launch_shared_support(Z, ldz, part->qoff, row_frac, union_frac, z0, nz, c.N, c.Gq, s));
    }
    return SPARSEPR_OK;
}

sparsepr_status sparsepr_route(sparsepr_handle h, const void* Q, const sparsepr_partition_t* part,
                               sparsepr_route_t* out, void* stream) {
    if (!h || !aligned16(Q) || !out) return SPARSEPR_ERR_INVALID_ARG;
    sparsepr_status st = check_partition(part, false);
    if (st) return st;
    h->launches = 0;
    cudaStream_t s = as_stream(stream);
    st = route_impl(h, static_cast<const bf16*>(Q), part, false, s);
    if (st) return st;
    cudaEventRecord(h->done_ev, s);
    h->timed_call = false;
    fill_route(h, out);
    return SPARSEPR_OK;
}

sparsepr_status sparsepr_permute(sparsepr_handle h, const void* Q, const void* K, const void* V,
                                 const sparsepr_partition_t* part, void* Qp, void* Kp, void* Vp, void* stream) {
    if (!h) return SPARSEPR_ERR_INVALID_ARG;
    sparsepr_status st = check_partition(part, false);
    if (st) return st;
    if ((Qp && (!aligned16(Q) || !aligned16(Qp))) || (Kp && (!aligned16(K) || !aligned16(Kp))) ||
        (Vp && (!aligned16(V) || !aligned16(Vp))))
        return SPARSEPR_ERR_INVALID_ARG;
    h->launches = 0;
    return permute_impl(h, static_cast<const bf16*>(Q), static_cast<const bf16*>(K), static_cast<const bf16*>(V),
                        part, static_cast<bf16*>(Qp), static_cast<bf16*>(Kp), static_cast<bf16*>(Vp),
                        as_stream(stream));
}

sparsepr_status sparsepr_blocksparse_attn(sparsepr_handle h, const void* Qp, const void* Kp, const void* Vp,
                                          const sparsepr_partition_t* part, const sparsepr_route_t* route, void* Osp,
                                          float* lse, void* stream) {
    if (!h || !aligned16(Qp) || !aligned16(Kp) || !aligned16(Vp) || !aligned16(Osp)) return SPARSEPR_ERR_INVALID_ARG;
    sparsepr_status st = check_partition(part, false);
    if (st) return st;
    if (!route || !route->rowptr || !route->kg) return SPARSEPR_ERR_INVALID_ARG;
    h->launches = 0;
    return attn_impl(h, static_cast<const bf16*>(Qp), static_cast<const bf16*>(Kp), static_cast<const bf16*>(Vp),
                     part, route, static_cast<bf16*>(Osp), lse, as_stream(stream));
}

sparsepr_status sparsepr_probe_fit(sparsepr_handle h, const void* Q, const void* K, const void* V,
                                   const sparsepr_partition_t* part, const void* Osp, sparsepr_fit_t* out,
                                   void* stream) {
    if (!h || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(Osp) || !out)
        return SPARSEPR_ERR_INVALID_ARG;
    sparsepr_status st = check_partition(part, true);
    if (st) return st;
    if (!h->M) return SPARSEPR_ERR_INVALID_ARG;
    h->launches = 0;
    st = probe_fit_impl(h, static_cast<const bf16*>(Q), static_cast<const bf16*>(K), static_cast<const bf16*>(V),
                        part, static_cast<const bf16*>(Osp), as_stream(stream));
    if (st) return st;
    fill_fit(h, out);
    return SPARSEPR_OK;
}

sparsepr_status sparsepr_writeback(sparsepr_handle h, const sparsepr_partition_t* part, const void* Osp,
                                   const sparsepr_fit_t* fit, void* O, void* stream) {
    if (!h || !aligned16(Osp) || !aligned16(O)) return SPARSEPR_ERR_INVALID_ARG;
    sparsepr_status st = check_partition(part, h->M > 0);
    if (st) return st;
    if (h->M && fit && (!fit->U || !fit->Bm || !fit->c0 || !fit->Odense)) return SPARSEPR_ERR_INVALID_ARG;
    if (h->M && fit && (h->cfg.flags & (SPARSEPR_FLAG_RIDGE_ONLY | SPARSEPR_FLAG_RBAR_UNPROJECTED)) &&
        (!fit->A || !fit->obar || !fit->Rbar))
        return SPARSEPR_ERR_INVALID_ARG;
    h->launches = 0;
    return writeback_impl(h, part, static_cast<const bf16*>(Osp), fit, static_cast<bf16*>(O), as_stream(stream));
}

sparsepr_status sparsepr_attention(sparsepr_handle h, const void* Q, const void* K, const void* V, void* O,
                                   void* stream) {
    if (!h || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SPARSEPR_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    const bf16* q = static_cast<const bf16*>(Q);
    const bf16* k = static_cast<const bf16*>(K);
    const bf16* v = static_cast<const bf16*>(V);
    h->launches = 0;
    sparsepr_partition_t part;
    sparsepr_route_t route;
    fill_partition(h, &part);
    fill_route(h, &route);
    mark(h, 0, s);
    sparsepr_status st = partition_impl(h, q, k, s);
    if (st) return st;
    mark(h, 1, s);
    if ((st = route_impl(h, q, &part, true, s))) return st;
    mark(h, 2, s);
    if ((st = permute_impl(h, q, k, v, &part, h->Qp, h->Kp, h->Vp, s))) return st;
    mark(h, 3, s);
    if ((st = attn_impl(h, h->Qp, h->Kp, h->Vp, &part, &route, h->Osp, h->lse, s))) return st;
    mark(h, 4, s);
    if ((st = probe_fit_impl(h, q, k, v, &part, h->Osp, s))) return st;
    mark(h, 5, s);
    sparsepr_fit_t fit;
    fill_fit(h, &fit);
    if ((st = writeback_impl(h, &part, h->Osp, &fit, static_cast<bf16*>(O), s)))
        return st;
    mark(h, 6, s);
    cudaEventRecord(h->done_ev, s);
    h->timed_call = h->timing && !h->user_events;
    return SPARSEPR_OK;
}

sparsepr_status sparsepr_attention_host(sparsepr_handle h, const void* Q, const void* K, const void* V, void* O,
                                        void* stream) {
    if (!h || !Q || !K || !V || !O) return SPARSEPR_ERR_INVALID_ARG;
    const sparsepr_config& c = h->cfg;
    const size_t qb = (size_t)c.B * c.Hq * c.N * c.d * sizeof(bf16);
    const size_t kb = (size_t)c.B * c.Hkv * c.N * c.d * sizeof(bf16);
    if (!h->sQ) {
        void *a = nullptr, *b = nullptr, *cc = nullptr, *dd = nullptr;
        if (cudaMalloc(&a, qb) || cudaMalloc(&b, kb) || cudaMalloc(&cc, kb) || cudaMalloc(&dd, qb)) {
            if (a) cudaFree(a);
            if (b) cudaFree(b);
            if (cc) cudaFree(cc);
            if (dd) cudaFree(dd);
            return SPARSEPR_ERR_WORKSPACE;
        }
        h->sQ = static_cast<bf16*>(a); h->sK = static_cast<bf16*>(b);
        h->sV = static_cast<bf16*>(cc); h->sO = static_cast<bf16*>(dd);
    }
    if (!h->pipe) {
        HostPipe* pp = new (std::nothrow) HostPipe();
        if (!pp) return SPARSEPR_ERR_WORKSPACE;
        pp->nc = host_chunks(h->P, pp->z0);
        bool ok = true;
        for (int i = 0; i < pp->nc && ok; ++i) {
            sparsepr_config sc = c;
            sc.B = 1;
            sc.Hkv = pp->z0[i + 1] - pp->z0[i];
            sc.Hq = sc.Hkv * h->g;
            sc.flags &= ~SPARSEPR_FLAG_STAGE_TIMING;
            ok = sparsepr_create(&sc, &pp->sub[i]) == SPARSEPR_OK;
        }
        ok = ok && cudaStreamCreateWithFlags(&pp->in, cudaStreamNonBlocking) == cudaSuccess &&
             cudaStreamCreateWithFlags(&pp->out, cudaStreamNonBlocking) == cudaSuccess;
        for (int k = 0; k < kHostStreams && ok; ++k)
            ok = cudaStreamCreateWithFlags(&pp->comp[k], cudaStreamNonBlocking) == cudaSuccess &&
                 cudaEventCreateWithFlags(&pp->end_comp[k], cudaEventDisableTiming) == cudaSuccess;
        for (cudaEvent_t* e : {&pp->start, &pp->end_out})
            ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
        for (int i = 0; i < pp->nc && ok; ++i)
            ok = cudaEventCreateWithFlags(&pp->ev_in[i], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&pp->ev_done[i], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) {
            destroy_pipe(pp);
            return SPARSEPR_ERR_WORKSPACE;
        }
        h->pipe = pp;
    }
    HostPipe* pp = h->pipe;
    cudaStream_t s = as_stream(stream);
    const size_t qh = (size_t)h->g * c.N * c.d, kh = (size_t)c.N * c.d;   // elements per KV head
    const bf16* hQ = static_cast<const bf16*>(Q);
    const bf16* hK = static_cast<const bf16*>(K);
    const bf16* hV = static_cast<const bf16*>(V);
    bf16* hO = static_cast<bf16*>(O);
    bool ok = cudaEventRecord(pp->start, s) == cudaSuccess;
    for (cudaStream_t st : {pp->in, pp->out})
        ok = ok && cudaStreamWaitEvent(st, pp->start, 0) == cudaSuccess;
    for (int k = 0; k < kHostStreams; ++k) ok = ok && cudaStreamWaitEvent(pp->comp[k], pp->start, 0) == cudaSuccess;
    // every chunk's inputs in order on the copy-in stream
    for (int i = 0; i < pp->nc && ok; ++i) {
        const size_t z = pp->z0[i], n = pp->z0[i + 1] - pp->z0[i];
        ok = cudaMemcpyAsync(h->sQ + z * qh, hQ + z * qh, n * qh * sizeof(bf16), cudaMemcpyHostToDevice, pp->in) ==
                 cudaSuccess &&
             cudaMemcpyAsync(h->sK + z * kh, hK + z * kh, n * kh * sizeof(bf16), cudaMemcpyHostToDevice, pp->in) ==
                 cudaSuccess &&
             cudaMemcpyAsync(h->sV + z * kh, hV + z * kh, n * kh * sizeof(bf16), cudaMemcpyHostToDevice, pp->in) ==
                 cudaSuccess &&
             cudaEventRecord(pp->ev_in[i], pp->in) == cudaSuccess;
    }
    // each chunk's call once its inputs have landed (chunk i on compute stream i % kHostStreams,
    // so one chunk's latency-bound kernels overlap the others'), its output copied back
    int launches = 0;
    for (int i = 0; i < pp->nc && ok; ++i) {
        const size_t z = pp->z0[i], n = pp->z0[i + 1] - pp->z0[i];
        cudaStream_t cs = pp->comp[i % kHostStreams];
        ok = cudaStreamWaitEvent(cs, pp->ev_in[i], 0) == cudaSuccess;
        if (ok && sparsepr_attention(pp->sub[i], h->sQ + z * qh, h->sK + z * kh, h->sV + z * kh, h->sO + z * qh,
                                     cs) != SPARSEPR_OK)
            ok = false;
        launches += pp->sub[i]->launches;
        ok = ok && cudaMemcpyAsync(h->pairs + z, pp->sub[i]->pairs, n * sizeof(int64_t), cudaMemcpyDeviceToDevice,
                                   cs) == cudaSuccess;
        ok = ok && cudaEventRecord(pp->ev_done[i], cs) == cudaSuccess &&
             cudaStreamWaitEvent(pp->out, pp->ev_done[i], 0) == cudaSuccess &&
             cudaMemcpyAsync(hO + z * qh, h->sO + z * qh, n * qh * sizeof(bf16), cudaMemcpyDeviceToHost, pp->out) ==
                 cudaSuccess;
    }
    for (int k = 0; k < kHostStreams; ++k)
        ok = ok && cudaEventRecord(pp->end_comp[k], pp->comp[k]) == cudaSuccess &&
             cudaStreamWaitEvent(s, pp->end_comp[k], 0) == cudaSuccess;
    ok = ok && cudaEventRecord(pp->end_out, pp->out) == cudaSuccess &&
         cudaStreamWaitEvent(s, pp->end_out, 0) == cudaSuccess;
    // every internal stream drains before returning, even after an error, so no work outlives the call
    bool drained = cudaStreamSynchronize(s) == cudaSuccess;
    for (cudaStream_t st : {pp->in, pp->out}) drained = cudaStreamSynchronize(st) == cudaSuccess && drained;
    for (int k = 0; k < kHostStreams; ++k) drained = cudaStreamSynchronize(pp->comp[k]) == cudaSuccess && drained;
    if (!drained || !ok) return SPARSEPR_ERR_CUDA;
    // statistics and the device status of the chunk calls on the handle
    int worst = 0;
    for (int i = 0; i < pp->nc; ++i) {
        int ds = 0;
        if (cudaMemcpy(&ds, pp->sub[i]->dev_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
            return SPARSEPR_ERR_CUDA;
        if (ds && !worst) worst = ds;
    }
    if (worst && cudaMemcpy(h->dev_status, &worst, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
        return SPARSEPR_ERR_CUDA;
    cudaEventRecord(h->done_ev, s);
    h->timed_call = false;
    h->launches = launches;
    return SPARSEPR_OK;
}

sparsepr_status sparsepr_dense_attn(sparsepr_handle h, const void* Q, const void* K, const void* V, void* O,
                                    void* stream) {
    if (!h || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SPARSEPR_ERR_INVALID_ARG;
    const sparsepr_config& c = h->cfg;
    h->launches = 0;
    if (spr::attn_tc_supported(c.d)) {
        SPR_TRY(spr::launch_attn_dense_tc(static_cast<const bf16*>(Q), static_cast<const bf16*>(K),
                                          static_cast<const bf16*>(V), static_cast<bf16*>(O), nullptr, c.B, c.Hq,
                                          c.Hkv, c.N, c.d, h->dev_status, (c.flags & SPARSEPR_FLAG_TEST_STALL) != 0,
                                          as_stream(stream)));
        return SPARSEPR_OK;
    }
    SPR_TRY(spr::launch_attn_dense(static_cast<const bf16*>(Q), static_cast<const bf16*>(K),
                                   static_cast<const bf16*>(V), static_cast<bf16*>(O), nullptr, c.B, c.Hq, c.Hkv,
                                   c.N, c.d, as_stream(stream)));
    return SPARSEPR_OK;
}

sparsepr_status sparsepr_get_stats(sparsepr_handle h, sparsepr_stats* out) {
    if (!h || !out) return SPARSEPR_ERR_INVALID_ARG;
    memset(out, 0, sizeof(*out));
    if (cudaEventSynchronize(h->done_ev) != cudaSuccess) return SPARSEPR_ERR_CUDA;
    const sparsepr_config& c = h->cfg;
    std::vector<int64_t> pairs(h->P);
    if (cudaMemcpy(pairs.data(), h->pairs, h->P * sizeof(int64_t), cudaMemcpyDeviceToHost) != cudaSuccess)
        return SPARSEPR_ERR_CUDA;
    const double nn = (double)c.N * (double)c.N;
    double dens = 0.0, useful = 0.0;
    for (int z = 0; z < h->P; ++z) {
        dens += (double)pairs[z] / nn;
        useful += (double)h->g * ((double)pairs[z] + (double)h->M * c.N);
    }
    out->route_density = dens / h->P;
    out->rho_exec = out->route_density + (double)h->M / c.N;
    out->useful_pairs = useful;
    if (h->timed_call) {
        for (int i = 0; i < 6; ++i) cudaEventElapsedTime(&out->stage_ms[i], h->ev[i], h->ev[i + 1]);
        cudaEventElapsedTime(&out->stage_ms[kStTotal], h->ev[0], h->ev[6]);
    }
    int ds = 0;
    if (cudaMemcpy(&ds, h->dev_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SPARSEPR_ERR_CUDA;
    out->device_status = ds;
    return SPARSEPR_OK;
}

sparsepr_status sparsepr_device_status(sparsepr_handle h, int* out) {
    if (!h || !out) return SPARSEPR_ERR_INVALID_ARG;
    if (cudaMemcpy(out, h->dev_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SPARSEPR_ERR_CUDA;
    if (cudaMemset(h->dev_status, 0, sizeof(int)) != cudaSuccess) return SPARSEPR_ERR_CUDA;
    return SPARSEPR_OK;
}

sparsepr_status sparsepr_set_stage_events(sparsepr_handle h, void* const* events) {
    if (!h) return SPARSEPR_ERR_INVALID_ARG;
    if (!events) {
        h->user_events = false;
        return SPARSEPR_OK;
    }
    for (int i = 0; i < 7; ++i)
        if (!events[i]) return SPARSEPR_ERR_INVALID_ARG;
    for (int i = 0; i < 7; ++i) h->user_ev[i] = static_cast<cudaEvent_t>(events[i]);
    h->user_events = true;
    return SPARSEPR_OK;
}

sparsepr_status sparsepr_last_launch_count(sparsepr_handle h, int* out) {
    if (!h || !out) return SPARSEPR_ERR_INVALID_ARG;
    *out = h->launches;
    return SPARSEPR_OK;
}

}  // extern "C"
