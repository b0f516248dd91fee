// Internal host-side launchers of the SparsePR kernels. Every launcher only
// enqueues work on `s` and returns the launch error (cudaSuccess on success).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace spr {

typedef __nv_bfloat16 bf16;

// ---------------------------------------------------------------- dense bf16 GEMM
// C[z][m][n] = alpha * sum_k (A1[z][m][k] B1[zb][n][k] + A2[z][m][k] B2[zb][n][k]),
// zb = z / bdiv. A2/B2 may be null (single term). K % 8 == 0, lda/ldb % 8 == 0.
struct GemmArgs {
    const bf16* A1; const bf16* A2; long long sA; int lda;
    const bf16* B1; const bf16* B2; long long sB; int ldb; int bdiv;
    float* C; long long sC; int ldc;
    int M, N, K, batch;
    float alpha;
};
cudaError_t launch_gemm_bf16(const GemmArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- k-means + group-major order
// X: [P][n][DP] fp32 rows (DP in {16,32,48,64,128}); C: [P][G][DP]; labels/dist: [P][n].
// dst [P][N][d] fp32 = mean over the g query heads of src [P*g][N][d] bf16 (g = 1: widening copy).
cudaError_t launch_mean_heads_f32(const bf16* src, float* dst, int P, int g, int N, int d, cudaStream_t s);
cudaError_t launch_km_seed(const float* X, float* C, int P, int n, int G, int DP, cudaStream_t s);
cudaError_t launch_km_assign(const float* X, const float* C, int32_t* labels, float* dist,
                             int* changed, const int* done, int P, int n, int G, int DP, bool first,
                             cudaStream_t s);
cudaError_t launch_km_update(const float* X, const int32_t* perm, const int32_t* off, float* C,
                             const int* done, int P, int n, int G, int DP, cudaStream_t s);
cudaError_t launch_km_check(int* changed, int* done, int P, cudaStream_t s);
cudaError_t launch_km_reset(int* changed, int* done, int P, cudaStream_t s);
// Stable counting sort of labels [P][n] into perm [P][n] and off [P][G+1].
// counts/bases: [P][ceil(n/256)][G] scratch. done may be null (always run).
cudaError_t launch_group_sort(const int32_t* labels, int32_t* perm, int32_t* off, int* counts,
                              int* bases, const int* done, int P, int n, int G, cudaStream_t s);
// Mean of the bf16 rows Y [P][n][d] per group (perm/off order); empty -> 0. Also writes a
// bf16 hi/lo split of the means (hi = bf16(c), lo = bf16(c - hi)) when chi/clo are non-null.
cudaError_t launch_group_mean_bf16(const bf16* Y, const int32_t* perm, const int32_t* off,
                                   float* cent, bf16* chi, bf16* clo, int P, int n, int G, int d,
                                   cudaStream_t s);
// Tensor-core assignment (G <= 256): rows and centroids split into two bf16 parts
// (X2: [2][P][n][DP] compact, C2: [2][P][G16][64]); near ties are settled exactly in fp64 from
// the fp32 rows X and centroids C, so labels are the argmin of the fp32 distances.
bool km_tc_supported(int G);
cudaError_t launch_km_split_rows(const float* X, bf16* X2, float* xx, int P, int n, int DP, cudaStream_t s);
cudaError_t launch_km_split_cent(const float* C, bf16* C2, float* cc, int P, int G, int DP, cudaStream_t s);
// fix: km_fix_slots(P, n, num_sms) int4 slots (each CTA owns a region for the rows it flags and
// settles exactly in fp64 at its end, correcting labels and moved counts).
size_t km_fix_slots(int P, int n, int num_sms);
cudaError_t launch_km_assign_tc(const float* X, const bf16* X2, const float* xx, const float* C, const bf16* C2,
                                const float* cc, int32_t* labels, int* changed, const int* done, int4* fix,
                                int* status, int P, int n, int G, int DP, bool first, int num_sms, cudaStream_t s);
// dist[z][i] = fp32 of the fp64 squared distance of row i to its own centroid.
cudaError_t launch_km_dist(const float* X, const float* C, const int32_t* labels, float* dist, int P, int n, int G,
                           int DP, cudaStream_t s);
bool logits_tc_supported(int d, int Gk);
cudaError_t launch_logits_tc(const bf16* Q, const bf16* chi, const bf16* clo, const int32_t* koff, float* u,
                             float* lse, int* status, int B, int Hq, int Hkv, int N, int Gk, int num_sms,
                             cudaStream_t s);
// Split fp32 group means into bf16 hi/lo (used when the partition is handed in).
cudaError_t launch_split_bf16(const float* x, bf16* hi, bf16* lo, long long count, cudaStream_t s);

// Support diagnostic: out[z][s] = (smallest k whose k largest exp(F[.][s] - max) hold 90% of the
// row's softmax mass) / N, for s < S; F [P][N][DP] fp32 (DP a multiple of 8, S <= DP). colmax
// (optional, [P][DP]): the column maxima as written by launch_resp_tc, which saves one pass.
cudaError_t launch_topmass(const float* F, float* out, const unsigned* colmax, int P, int N, int DP, int S,
                           cudaStream_t s);
// Sampled responses on the tensor cores (d in {64, 128}, DP a multiple of 16 up to 64):
// F[z][j][s] = K[z][j] . Qs[z][s] / sqrt(d) for every key j, with the two bf16 parts of F in X2
// ([2][P*N][DP]) and ||F[z][j]||^2 in xx; colmax (optional, [P][DP]) receives order-preserving
// keys of the maxima of the first S columns over all keys. Qs [P][DP][d], rows >= S zero.
bool resp_tc_supported(int d, int DP);
cudaError_t launch_resp_tc(const bf16* K, const bf16* Qs, float* F, bf16* X2, float* xx, unsigned* colmax, int P,
                           int N, int d, int DP, int S, int num_sms, int* status, cudaStream_t s);
// Affine diagnostics: per query head, [explained fraction, orthogonal energy] of R = Od - Os.
size_t affine_diag_workspace(int Hp, int d);
cudaError_t launch_affine_diag(const bf16* Os, const bf16* Od, double* out, void* ws, int Hp, int N, int d,
                               int* status, cudaStream_t s);
// Shared-route support: Qsh [P][Gq][8][d] bf16 gathered rows (zero past R' of each group), then
// for KV heads z0..z0+nz-1 the row-major logits Z [nz][Gq*8][ldz] give row_frac [P][Gq][8] and
// union_frac [P][Gq].
cudaError_t launch_shared_rows(const bf16* Q, const int32_t* qperm, const int32_t* qoff, bf16* Qsh, int P, int g,
                               int N, int d, int Gq, cudaStream_t s);
cudaError_t launch_shared_support(const float* Z, long long ldz, const int32_t* qoff, float* row_frac,
                                  float* union_frac, int z0, int nz, int N, int Gq, cudaStream_t s);

// ---------------------------------------------------------------- responses and coordinates
// Qs[z][s][:] = Q[b][h*g + s%g][floor((s+1/2)N/S)][:] for s < S, zero rows up to DP.
cudaError_t launch_gather_samples(const bf16* Q, bf16* Qs, int B, int Hq, int Hkv, int N, int d,
                                  int S, int DP, cudaStream_t s);
// Mean over the g query heads of u, centred over the Gk groups. If proj: write bf16 hi/lo
// [P][N][Gkp]; else write the L2-normalised rows into y [P][N][DPy].
cudaError_t launch_coords_center(const float* u, bf16* uhi, bf16* ulo, float* y, int P, int g,
                                 int N, int Gk, int Gkp, int DPy, bool proj, cudaStream_t s);
cudaError_t launch_rows_normalize(float* y, int rows, int DP, cudaStream_t s);
// Gk > rQ in one pass: y [P][N][DPy] = normalise((mean_h u - row mean) . projT^T) (DPy = 64).
bool coords_proj_supported(int DPy, int Gk, int Gkp);
cudaError_t launch_coords_proj(const float* u, const bf16* projT, float* y, int P, int g, int N, int Gk, int Gkp,
                               int num_sms, cudaStream_t s);
// projT [DPy][Gkp] bf16 = +-1 with the sign of bit 0 of splitmix64(seed ^ (g*rQ + t)).
cudaError_t launch_make_projection(bf16* projT, int Gk, int Gkp, int rQ, int DPy,
                                   unsigned long long seed, cudaStream_t s);

// ---------------------------------------------------------------- probes
// Probe rows: systematic positions of the radial-ordered group-major sequence.
cudaError_t launch_probe_select(const int32_t* qperm, const int32_t* qoff, const float* radial,
                                int32_t* probe, int32_t* probe_pos, int32_t* probe_seq, int P,
                                int N, int Gq, int M, cudaStream_t s);
// Probe-sampling ablations: uniform grid of the original order, or seeded SplitMix64 draws.
cudaError_t launch_probe_alt(const int32_t* qperm, const int32_t* qoff, const int32_t* qgroup, int32_t* probe,
                             int32_t* probe_pos, int32_t* probe_seq, int P, int N, int Gq, int M, bool random,
                             unsigned long long seed, int* status, cudaStream_t s);
cudaError_t launch_probe_weights(const int32_t* qoff, const int32_t* probe_seq, float* w, int P,
                                 int N, int Gq, int M, bool uniform, cudaStream_t s);

// ---------------------------------------------------------------- routing
cudaError_t launch_row_lse(const float* u, const int32_t* koff, float* lse, int Hp, int g, int N,
                           int Gk, cudaStream_t s);
cudaError_t launch_cell_scores(const float* u, const float* lse, const int32_t* qperm,
                               const int32_t* qoff, const int32_t* koff, float* scores, int P,
                               int g, int N, int Gq, int Gk, cudaStream_t s);
cudaError_t launch_route_select(const float* scores, const int32_t* qoff, const int32_t* koff,
                                int32_t* rowptr, int32_t* kg, int64_t* pairs, int P, int Gq,
                                int Gk, long long budget, bool keep_all, cudaStream_t s);

// ---------------------------------------------------------------- permutation
// dst[z][p][:] = src[z][perm[z / div][p]][:] for rows of d bf16 (d % 8 == 0).
cudaError_t launch_permute_rows(const bf16* src, bf16* dst, const int32_t* perm, int Z, int div,
                                int N, int d, cudaStream_t s);

// ---------------------------------------------------------------- attention
// Per-pair tile offsets of the query groups: tile_off[z][a] = sum_{a'<a} ceil(|Q_a'| / bm).
cudaError_t launch_tile_offsets(const int32_t* qoff, int32_t* tile_off, int P, int Gq, int bm, cudaStream_t s);
// Block-sparse attention over group-major Qp/Kp/Vp with the route CSR.
cudaError_t launch_attn_sparse(const bf16* Qp, const bf16* Kp, const bf16* Vp,
                               const int32_t* qoff, const int32_t* koff, const int32_t* tile_off,
                               const int32_t* rowptr, const int32_t* kg, bf16* O, float* lse,
                               int B, int Hq, int Hkv, int N, int d, int Gq, int Gk,
                               cudaStream_t s);
// Dense attention of every query over all keys.
cudaError_t launch_attn_dense(const bf16* Q, const bf16* K, const bf16* V, bf16* O, float* lse,
                              int B, int Hq, int Hkv, int N, int d, cudaStream_t s);
// tcgen05/TMEM versions (head dimension 128): two 128-row query tiles per CTA, 128-key tiles.
bool attn_tc_supported(int d);
// Query rows one CTA covers: two 128-row tiles of one head, or (g even) one tile of two heads.
bool attn_tc_head_pairs(int g);
// A lone last query tile of at most 64 rows (or, with head pairs, such a tile of two heads) runs
// as an M = 64 tile: half the softmax work per key tile, the same K/V reads.
bool attn_tc_half_tails(int g);
int attn_tc_rows_per_cta(int g);
// Key tiles (start row, valid keys) of every query group's merged kept runs: cnt [P][Gq]
// scratch, off [P][Gq+1] absolute offsets, list of key_tiles_capacity(N, Gq, Gk) * P entries.
long long key_tiles_capacity(int N, int Gq, int Gk);
cudaError_t launch_key_tiles(const int32_t* rowptr, const int32_t* kg, const int32_t* koff, int32_t* cnt,
                             int32_t* off, int2* list, int P, int N, int Gq, int Gk, cudaStream_t s);
cudaError_t launch_attn_sparse_tc(const bf16* Qp, const bf16* Kp, const bf16* Vp, const int32_t* qoff,
                                  const int32_t* tile_off, const int2* klist, const int32_t* klist_off, bf16* O,
                                  float* lse, int B, int Hq, int Hkv, int N, int d, int Gq, int* status,
                                  cudaStream_t s);
// stall: test only -- the producer issues no loads, so the first bounded wait runs out.
cudaError_t launch_attn_dense_tc(const bf16* Q, const bf16* K, const bf16* V, bf16* O, float* lse, int B, int Hq,
                                 int Hkv, int N, int d, int* status, bool stall, cudaStream_t s);
// Probe rows on the tensor cores (d = 128): the M (<= 128) probe rows of every query head
// gathered into Qpr [B*Hq][128][d] (rows >= M zero), attended against all keys in
// probe_tc_splits(N, ns) splits of probe_tc_chunk(N, ns) keys; partial outputs, maxima and
// sums in the layout of launch_attn_probe, merged by launch_probe_combine.
cudaError_t launch_gather_probe_rows(const bf16* Q, const int32_t* probe, bf16* Qpr, int B, int Hq, int Hkv, int N,
                                    int M, int d, int rows, cudaStream_t s);
int probe_tc_chunk(int N, int ns);
int probe_tc_splits(int N, int ns);
cudaError_t launch_attn_probe_tc(const bf16* Qpr, const bf16* K, const bf16* V, float* Opart, float* mpart,
                                 float* lpart, int B, int Hq, int Hkv, int N, int d, int M, int ns, int* status,
                                 cudaStream_t s);
cudaError_t launch_probe_combine(const float* Opart, const float* mpart, const float* lpart, float* Odense, int Hp,
                                 int M, int ns, int d, cudaStream_t s);
// Dense attention of gathered probe rows, split over ns key chunks, then combined.
cudaError_t launch_attn_probe(const bf16* Q, const bf16* K, const bf16* V, const int32_t* probe,
                              float* Opart, float* mpart, float* lpart, float* Odense, int B,
                              int Hq, int Hkv, int N, int d, int M, int ns, cudaStream_t s);

// ---------------------------------------------------------------- probe fit + write-back
cudaError_t launch_probe_residual(const float* Odense, const bf16* Osp, const int32_t* probe_pos,
                                  float* R, float* Osp_probe, int Hp, int g, int N, int d, int M,
                                  cudaStream_t s);
cudaError_t launch_fit(const float* R, const float* Xp, const float* w, float lambda, float* obar,
                       float* Rbar, float* A, float* U, float* Bm, float* c0, int32_t* rank,
                       int Hp, int g, int d, int M, int r, bool rbar_unprojected, int* status, cudaStream_t s);
// O = Osp + U (c0 + Bm Osp) (+ Radd [Hp][d] when non-null), scattered to the original order.
cudaError_t launch_writeback(const bf16* Osp, const int32_t* qperm, const float* U,
                             const float* Bm, const float* c0, const float* Radd, bf16* O, int Hp, int g, int N,
                             int d, int r, bool correct, int num_sms, cudaStream_t s);
// O = Osp + Rbar + A (Osp - obar) (ridge correction without the projection).
cudaError_t launch_writeback_ridge(const bf16* Osp, const int32_t* qperm, const float* A, const float* obar,
                                   const float* Rbar, bf16* O, int Hp, int g, int N, int d, int num_sms,
                                   cudaStream_t s);
// Correction and write-back on the tensor cores (d = 128, r <= 32): O[qperm[p]] = o + U (c0 + Bm o)
// (+ Radd) for every group-major row o of Osp; parts: wb_tc_parts_elems(Hp) bf16 of scratch for the
// bf16 parts of Bm and U^T.
bool wb_tc_supported(int d, int r);
size_t wb_tc_parts_elems(int Hp);
cudaError_t launch_writeback_tc(const bf16* Osp, const int32_t* qperm, const float* U, const float* Bm,
                                const float* c0, const float* Radd, bf16* parts, bf16* O, int Hp, int g, int N, int r,
                                int* status, int num_sms, cudaStream_t s);
cudaError_t launch_probe_override(const float* Odense, const int32_t* probe, bf16* O, int Hp,
                                  int g, int N, int d, int M, cudaStream_t s);

}  // namespace spr
