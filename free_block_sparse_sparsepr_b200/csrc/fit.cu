// Probe residuals, the group-coverage-weighted ridge fit with its residual
// subspace (one CTA per query head), the correction + un-permute write-back,
// and the exact dense rows written over the probe rows.
#include <float.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace spr {
namespace {

// R = O_dense - O_sparse at each probe row; the bf16 sparse output is widened to fp32.
__global__ void probe_residual_kernel(const float* __restrict__ Od, const bf16* __restrict__ Osp,
                                      const int32_t* __restrict__ probe_pos, float* R, float* Xp,
                                      int g, int N, int d, int M) {
    const int x = blockIdx.y, m = blockIdx.x, c = threadIdx.x, z = x / g;
    const int pos = probe_pos[(long long)z * M + m];
    const float os = __bfloat162float(Osp[((long long)x * N + pos) * d + c]);
    const long long o = ((long long)x * M + m) * d + c;
    Xp[o] = os;
    R[o] = Od[o] - os;
}

// Per query head x (one CTA of 512 threads):
//   xbar, Rbar   w-weighted means of the probes' sparse outputs X and residuals R
//   A            argmin sum_m w_m ||(R_m - Rbar) - A (X_m - xbar)||^2 + lambda ||A||_F^2, via the
//                M x M system: A = Ys^T (Xs Xs^T + lambda I)^-1 Xs, Xs/Ys rows scaled by sqrt(w_m)
//                (Cholesky of the M x M matrix)
//   U            top-r left singular vectors of the d x M matrix W = [sqrt(w_m) R_m]: one-sided
//                (Hestenes) Jacobi rotates column pairs of W until they are mutually orthogonal;
//                the columns are then sigma_m u_m, sorted by norm (ties -> lower index)
//   Bm = U^T A, c0 = U^T Rbar - Bm xbar  so that the correction is U (c0 + Bm o).
constexpr int kFitThreads = 512;
constexpr int kFitWarps = kFitThreads / 32;
template <int D>
__global__ void __launch_bounds__(kFitThreads) fit_kernel(
    const float* __restrict__ Rg, const float* __restrict__ Xg, const float* __restrict__ wts,
    float lambda, float* obar, float* Rbar, float* A, float* U, float* Bm, float* c0,
    int32_t* rank_out, int g, int M, int r, int rbar_unprojected, int* status) {
    constexpr int d = D;
    constexpr int nt = kFitThreads;
    const int x = blockIdx.x, z = x / g, tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int Mp = (M + 1) & ~1;
    const int ld = d + 1;            // padded row stride: column-wise walks hit distinct banks
    extern __shared__ float sm[];
    float* X = sm;                   // [M][ld]   probes' sparse outputs, then Xs, then Z
    float* Y = X + M * ld;           // [M][ld]   residuals, then Ys
    float* Wc = Y + M * ld;          // [M][ld]   sqrt(w_m) R_m (rows = columns of W)
    float* Km = Wc + M * ld;         // [M][M]
    float* Us = Km + M * M;          // [d][r]
    float* w = Us + d * r;           // [M]
    float* sw = w + M;               // [M]
    float* xb = sw + M;              // [d]
    float* yb = xb + d;              // [d]
    float* nrm = yb + d;             // [M]
    int* sel = reinterpret_cast<int*>(nrm + M);   // [r]
    float* inv_diag = nrm;           // [M] 1 / L[j][j] during the solves (nrm is written after them)
    __shared__ float sW;
    __shared__ int s_rank, s_rot;

    const float* Rx = Rg + (long long)x * M * d;
    const float* Xx = Xg + (long long)x * M * d;
    for (int t = tid; t < M; t += nt) { w[t] = wts[(long long)z * M + t]; sw[t] = sqrtf(wts[(long long)z * M + t]); }
    __syncthreads();
    for (int t = tid; t < M * d; t += nt) {
        const int m = t / d, c = t % d;
        X[m * ld + c] = Xx[t];
        Y[m * ld + c] = Rx[t];
        Wc[m * ld + c] = sw[m] * Rx[t];
    }
    if (tid == 0) {
        float W = 0.f;
        for (int m = 0; m < M; ++m) W += w[m];
        sW = W;
    }
    __syncthreads();
    const float W = sW;
    for (int c = tid; c < d; c += nt) {
        float sx = 0.f, sy = 0.f;
        for (int m = 0; m < M; ++m) { sx = fmaf(w[m], X[m * ld + c], sx); sy = fmaf(w[m], Y[m * ld + c], sy); }
        xb[c] = sx / W;
        yb[c] = sy / W;
    }
    __syncthreads();
    for (int t = tid; t < M * d; t += nt) {
        const int m = t / d, c = t % d;
        X[m * ld + c] = sw[m] * (X[m * ld + c] - xb[c]);
        Y[m * ld + c] = sw[m] * (Y[m * ld + c] - yb[c]);
    }
    __syncthreads();
    // Km = Xs Xs^T + lambda I, lower triangle, in 2 x 2 register blocks (rows past M read as 0)
    {
        const int Mb = (M + 1) / 2, nb = Mb * (Mb + 1) / 2;
        for (int e = tid; e < nb; e += nt) {
            int ib = (int)((sqrtf(8.f * (float)e + 1.f) - 1.f) * 0.5f);
            while (ib * (ib + 1) / 2 > e) --ib;
            while ((ib + 1) * (ib + 2) / 2 <= e) ++ib;
            const int jb = e - ib * (ib + 1) / 2;
            const int i0 = 2 * ib, j0 = 2 * jb;
            const bool i1ok = i0 + 1 < M, j1ok = j0 + 1 < M;
            float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
            for (int c = 0; c < d; ++c) {
                const float xi0 = X[i0 * ld + c], xj0 = X[j0 * ld + c];
                const float xi1 = i1ok ? X[(i0 + 1) * ld + c] : 0.f, xj1 = j1ok ? X[(j0 + 1) * ld + c] : 0.f;
                a00 = fmaf(xi0, xj0, a00);
                a01 = fmaf(xi0, xj1, a01);
                a10 = fmaf(xi1, xj0, a10);
                a11 = fmaf(xi1, xj1, a11);
            }
            Km[i0 * M + j0] = a00 + (i0 == j0 ? lambda : 0.f);
            if (j1ok && j0 + 1 <= i0) Km[i0 * M + j0 + 1] = a01;
            if (i1ok) Km[(i0 + 1) * M + j0] = a10;
            if (i1ok && j1ok) Km[(i0 + 1) * M + j0 + 1] = a11 + (i0 == j0 ? lambda : 0.f);
        }
    }
    __syncthreads();
    // Cholesky Km = L L^T (lower triangle, in place), right-looking: scale column j, then
    // update the trailing triangle
    for (int j = 0; j < M; ++j) {
        float djj = Km[j * M + j];
        if (!(djj > 0.f)) {
            if (tid == 0) set_status(status, kDevBounds);
            djj = 1e-30f;
        }
        const float dj = sqrtf(djj);
        for (int i = j + 1 + tid; i < M; i += nt) Km[i * M + j] = Km[i * M + j] / dj;
        __syncthreads();
        if (tid == 0) Km[j * M + j] = dj;
        {
            const int k = j + 1 + (tid & 63);
            if (k < M) {
                const float lk = Km[k * M + j];
#pragma unroll 4
                for (int i = j + 1 + (tid >> 6); i < M; i += nt / 64)
                    if (k <= i) Km[i * M + k] = fmaf(-Km[i * M + j], lk, Km[i * M + k]);
            }
        }
        __syncthreads();
    }
    for (int t = tid; t < M; t += nt) inv_diag[t] = 1.f / Km[t * M + t];
    __syncthreads();
    // Z = Km^-1 Xs, in place in X: L y = Xs then L^T z = y. Each column is owned by kLpc lanes
    // of one warp (rows interleaved among them), so the substitutions need only warp barriers.
    {
        constexpr int lpc = nt / d;                  // lanes per column (4 at d = 128, 8 at d = 64)
        const int col = tid / lpc, rs = tid % lpc;
        for (int jj = 0; jj < M; ++jj) {
            __syncwarp();
            const float yj = X[jj * ld + col] * inv_diag[jj];
            __syncwarp();
            if ((jj & (lpc - 1)) == rs) X[jj * ld + col] = yj;
            const int i0 = jj + 1 + ((rs - jj - 1) & (lpc - 1));
#pragma unroll 4
            for (int i = i0; i < M; i += lpc) X[i * ld + col] = fmaf(-Km[i * M + jj], yj, X[i * ld + col]);
        }
        for (int m = M - 1; m >= 0; --m) {
            __syncwarp();
            const float zm = X[m * ld + col] * inv_diag[m];
            __syncwarp();
            if ((m & (lpc - 1)) == rs) X[m * ld + col] = zm;
#pragma unroll 4
            for (int k = rs; k < m; k += lpc) X[k * ld + col] = fmaf(-Km[m * M + k], zm, X[k * ld + col]);
        }
    }
    __syncthreads();
    // A = Ys^T Z (d x d): each thread a 4 x (d/16) register tile, columns c2 interleaved by 16
    float* Ax = A + (long long)x * d * d;
    {
        const int ne = d / 16;
        for (int t = tid; t < (d / 4) * 16; t += nt) {
            const int cb = t / 16, c2b = t % 16;
            float acc[4][8];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[q][e] = 0.f;
            for (int m = 0; m < M; ++m) {
                float yv[4], zv[8];
#pragma unroll
                for (int q = 0; q < 4; ++q) yv[q] = Y[m * ld + 4 * cb + q];
#pragma unroll
                for (int e = 0; e < 8; ++e) zv[e] = e < ne ? X[m * ld + c2b + 16 * e] : 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[q][e] = fmaf(yv[q], zv[e], acc[q][e]);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (e < ne) Ax[(long long)(4 * cb + q) * d + c2b + 16 * e] = acc[q][e];
        }
    }
    // One-sided Jacobi on the columns of W (round-robin disjoint pairs, one half-warp per pair:
    // every pair of a round at once). Round k pairs column a(i, k) with b(i, k); both indices
    // advance by one (mod Mp - 1) from round to round.
    {
        const int hw = tid >> 4, hl = tid & 15;
        constexpr int kE = D / 16;                   // elements of a column per lane
        // a pair counts as orthogonal once |u1.u2| <= sqrt(d) eps |u1||u2|, the rounding level of
        // an fp32 dot product of length d
        const float jtol = sqrtf((float)d) * FLT_EPSILON, jtol2 = jtol * jtol;
        const int np = Mp / 2, nm = Mp - 1;
        for (int sweep = 0; sweep < 16; ++sweep) {
            if (tid == 0) s_rot = 0;
            __syncthreads();
            int ia = hw == 0 ? 0 : hw - 1, ib = (Mp - 2 - hw) % nm;   // (i - 1 + k), (Mp - 2 - i + k) mod nm at k = 0
            if (ib < 0) ib += nm;
            for (int k = 0; k < nm; ++k) {
                const int a1 = hw == 0 ? 0 : ia + 1, b1 = ib + 1;
                const int pc = min(a1, b1), qc = max(a1, b1);
                const bool valid = hw < np && qc < M;
                float u1[kE], u2[kE];
                float al = 0.f, be = 0.f, ga = 0.f;
#pragma unroll
                for (int e = 0; e < kE; ++e) {
                    u1[e] = valid ? Wc[pc * ld + hl + 16 * e] : 0.f;
                    u2[e] = valid ? Wc[qc * ld + hl + 16 * e] : 0.f;
                }
#pragma unroll
                for (int e = 0; e < kE; ++e) {
                    al = fmaf(u1[e], u1[e], al);
                    be = fmaf(u2[e], u2[e], be);
                    ga = fmaf(u1[e], u2[e], ga);
                }
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) {
                    al += __shfl_xor_sync(kFull, al, o);
                    be += __shfl_xor_sync(kFull, be, o);
                    ga += __shfl_xor_sync(kFull, ga, o);
                }
                if (valid && ga != 0.f && ga * ga > jtol2 * (al * be)) {
                    // tan of the rotation angle: the smaller root of t^2 + 2 zeta t - 1 = 0
                    const float zeta = __fdividef(be - al, 2.f * ga);
                    const float tt = (zeta >= 0.f ? 1.f : -1.f) / (fabsf(zeta) + sqrtf(fmaf(zeta, zeta, 1.f)));
                    const float cs = rsqrtf(fmaf(tt, tt, 1.f)), sn = tt * cs;
#pragma unroll
                    for (int e = 0; e < kE; ++e) {
                        Wc[pc * ld + hl + 16 * e] = cs * u1[e] - sn * u2[e];
                        Wc[qc * ld + hl + 16 * e] = sn * u1[e] + cs * u2[e];
                    }
                    if (hl == 0) s_rot = 1;
                }
                ia = ia + 1 == nm ? 0 : ia + 1;
                ib = ib + 1 == nm ? 0 : ib + 1;
                __syncthreads();
            }
            const int rotated = s_rot;   // read by every thread before thread 0 resets it
            __syncthreads();
            if (!rotated) break;
        }
    }
    // column norms = singular values; top r (descending, ties -> lower index) and the rank
    for (int m = warp; m < M; m += kFitWarps) {
        float s = 0.f;
        for (int c = lane; c < d; c += 32) s = fmaf(Wc[m * ld + c], Wc[m * ld + c], s);
        s = warp_sum(s);
        if (lane == 0) nrm[m] = sqrtf(s);
    }
    __syncthreads();
    if (warp == 0) {
        for (int k = 0; k < r; ++k) {
            float best = -1.f;
            int bi = M;
            for (int m = lane; m < M; m += 32) {
                bool used = false;
                for (int j = 0; j < k; ++j) used |= (sel[j] == m);
                if (!used && (nrm[m] > best || (nrm[m] == best && m < bi))) { best = nrm[m]; bi = m; }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ob = __shfl_xor_sync(kFull, best, o);
                const int oi = __shfl_xor_sync(kFull, bi, o);
                if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
            }
            if (lane == 0) sel[k] = bi;
            __syncwarp();
        }
        if (lane == 0) {
            const float tol = (float)(M > d ? M : d) * FLT_EPSILON;
            const float s0 = nrm[sel[0]];
            int rk = 0;
            for (int k = 0; k < r && k < M; ++k)
                if (nrm[sel[k]] > 0.f && nrm[sel[k]] > s0 * tol) ++rk;
            s_rank = rk;
        }
    }
    __syncthreads();
    const int rank = s_rank;
    for (int t = tid; t < d * r; t += nt) {
        const int c = t / r, k = t % r;
        const float val = k < rank ? Wc[sel[k] * ld + c] / nrm[sel[k]] : 0.f;
        Us[t] = val;
        U[(long long)x * d * r + t] = val;
    }
    __syncthreads();
    // Bm = U^T A = (Ys U)^T Z: T = Ys U (M x r, in Km's space, free since the solves), then T^T Z
    float* T = Km;
    for (int t = tid; t < M * r; t += nt) {
        const int m = t / r, k = t % r;
        float acc = 0.f;
        for (int c = 0; c < d; ++c) acc = fmaf(Y[m * ld + c], Us[c * r + k], acc);
        T[t] = acc;
    }
    __syncthreads();
    float* Bx = Bm + (long long)x * r * d;
    for (int t = tid; t < r * d; t += nt) {
        const int k = t / d, c2 = t % d;
        float acc = 0.f;
        for (int m = 0; m < M; ++m) acc = fmaf(T[m * r + k], X[m * ld + c2], acc);
        Bx[t] = acc;
    }
    __syncthreads();
    for (int k = warp; k < r; k += kFitWarps) {
        float a1 = 0.f, a2 = 0.f;
        for (int c = lane; c < d; c += 32) {
            a1 = fmaf(Us[c * r + k], yb[c], a1);
            a2 = fmaf(Bx[(long long)k * d + c], xb[c], a2);
        }
        a1 = warp_sum(a1);
        a2 = warp_sum(a2);
        // c0 = U^T Rbar - Bm obar; with Rbar added unprojected only the -Bm obar part
        if (lane == 0) c0[(long long)x * r + k] = (rbar_unprojected ? 0.f : a1) - a2;
    }
    for (int c = tid; c < d; c += nt) {
        obar[(long long)x * d + c] = xb[c];
        Rbar[(long long)x * d + c] = yb[c];
    }
    if (tid == 0) rank_out[x] = rank;
}

// O[qperm[p]] = Osp[p] + U (c0 + Bm Osp[p]) (+ Radd, when given: the residual mean added
// unprojected); one warp per group-major row. Each lane holds
// EPL consecutive elements; Bm and U^T are staged row-major in shared memory so every
// vector load is conflict-free. The RP partial dot products are reduced by recursive
// halving (RP/2 + ... + 1 + 1 shuffles); afterwards lane 2k holds t_k.
template <int D, int RP>
__global__ void __launch_bounds__(256) writeback_kernel(const bf16* __restrict__ Osp,
                                                        const int32_t* __restrict__ qperm,
                                                        const float* __restrict__ U,
                                                        const float* __restrict__ Bm,
                                                        const float* __restrict__ c0,
                                                        const float* __restrict__ Radd, bf16* O,
                                                        int g, int N, int r, int correct) {
    constexpr int EPL = D / 32;
    static_assert(RP == 16 || RP == 32, "RP");
    const int x = blockIdx.y, z = x / g;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __shared__ __align__(16) float sB[RP * D];    // Bm[k][c]
    __shared__ __align__(16) float sUt[RP * D];   // U[c][k] transposed to [k][c]
    __shared__ float sc[RP];
    if (correct) {
        for (int t = threadIdx.x; t < RP * D; t += blockDim.x) {
            const int k = t / D, c = t % D;
            sB[t] = k < r ? Bm[((long long)x * r + k) * D + c] : 0.f;
            sUt[t] = k < r ? U[((long long)x * D + c) * r + k] : 0.f;
        }
        for (int t = threadIdx.x; t < RP; t += blockDim.x) sc[t] = t < r ? c0[(long long)x * r + t] : 0.f;
    }
    __syncthreads();
    float radd[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) radd[e] = (correct && Radd) ? Radd[(long long)x * D + lane * EPL + e] : 0.f;
    // kRW rows per warp and iteration: every Bm / U^T value read from shared memory serves kRW rows
    constexpr int kRW = 4;
    const int32_t* perm = qperm + (long long)z * N;
    for (int p0 = (blockIdx.x * 8 + warp) * kRW; p0 < N; p0 += gridDim.x * 8 * kRW) {
        float o[kRW][EPL];
#pragma unroll
        for (int q = 0; q < kRW; ++q) {
            const bf16* src = Osp + ((long long)x * N + p0 + q) * D + lane * EPL;
#pragma unroll
            for (int e = 0; e < EPL; e += 2) {
                float2 f = make_float2(0.f, 0.f);
                if (p0 + q < N) f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(src + e));
                o[q][e] = f.x;
                o[q][e + 1] = f.y;
            }
        }
        if (correct) {
            float a[kRW][RP];
#pragma unroll
            for (int k = 0; k < RP; ++k) {
                float bk[EPL];
#pragma unroll
                for (int e = 0; e < EPL; ++e) bk[e] = sB[k * D + lane * EPL + e];
#pragma unroll
                for (int q = 0; q < kRW; ++q) {
                    float acc = 0.f;
#pragma unroll
                    for (int e = 0; e < EPL; ++e) acc = fmaf(bk[e], o[q][e], acc);
                    a[q][k] = acc;
                }
            }
            // Step with lane bit b: lanes with b set keep the upper half of the remaining
            // partials (adding the partner's upper half), the others the lower half.
            float tk[kRW];
#pragma unroll
            for (int q = 0; q < kRW; ++q) {
#pragma unroll
                for (int n = RP, bit = 16; n > 1; n >>= 1, bit >>= 1) {
                    const bool up = (lane & bit) != 0;
#pragma unroll
                    for (int i = 0; i < n / 2; ++i) {
                        const float send = up ? a[q][i] : a[q][i + n / 2];
                        const float keep = up ? a[q][i + n / 2] : a[q][i];
                        a[q][i] = keep + __shfl_xor_sync(kFull, send, bit);
                    }
                }
                if (RP == 16) a[q][0] += __shfl_xor_sync(kFull, a[q][0], 1);   // lanes 2k, 2k+1 held halves
                tk[q] = a[q][0];
            }
            float delta[kRW][EPL];
#pragma unroll
            for (int q = 0; q < kRW; ++q)
#pragma unroll
                for (int e = 0; e < EPL; ++e) delta[q][e] = 0.f;
#pragma unroll
            for (int k = 0; k < RP; ++k) {
                float uk[EPL];
#pragma unroll
                for (int e = 0; e < EPL; ++e) uk[e] = sUt[k * D + lane * EPL + e];
                const float ck = sc[k];
#pragma unroll
                for (int q = 0; q < kRW; ++q) {
                    const float t = __shfl_sync(kFull, tk[q], (RP == 16) ? 2 * k : k) + ck;
#pragma unroll
                    for (int e = 0; e < EPL; ++e) delta[q][e] = fmaf(uk[e], t, delta[q][e]);
                }
            }
#pragma unroll
            for (int q = 0; q < kRW; ++q)
#pragma unroll
                for (int e = 0; e < EPL; ++e) o[q][e] += delta[q][e] + radd[e];
        }
#pragma unroll
        for (int q = 0; q < kRW; ++q) {
            if (p0 + q >= N) break;
            bf16* dst = O + ((long long)x * N + perm[p0 + q]) * D + lane * EPL;
#pragma unroll
            for (int e = 0; e < EPL; e += 2)
                *reinterpret_cast<__nv_bfloat162*>(dst + e) = __floats2bfloat162_rn(o[q][e], o[q][e + 1]);
        }
    }
}

__global__ void probe_override_kernel(const float* __restrict__ Od, const int32_t* __restrict__ probe,
                                      bf16* O, int g, int N, int d, int M) {
    const int x = blockIdx.y, m = blockIdx.x, c = threadIdx.x, z = x / g;
    const int row = probe[(long long)z * M + m];
    O[((long long)x * N + row) * d + c] = __float2bfloat16_rn(Od[((long long)x * M + m) * d + c]);
}

// Ridge correction without the subspace projection: O[qperm[p]] = o + Rbar + A (o - obar),
// o = Osp[p]. A (d x d, row stride d + 1) and c = Rbar - A obar in shared memory; one warp per
// group-major row, lane l computing outputs l, l + 32, ... (conflict-free A reads), the row
// itself broadcast from a per-warp buffer.
template <int D>
__global__ void __launch_bounds__(256) writeback_ridge_kernel(const bf16* __restrict__ Osp,
                                                              const int32_t* __restrict__ qperm,
                                                              const float* __restrict__ A,
                                                              const float* __restrict__ obar,
                                                              const float* __restrict__ Rbar, bf16* O, int g,
                                                              int N) {
    constexpr int EPL = D / 32;
    extern __shared__ float rsm[];
    float* sA = rsm;                     // [D][D + 1]
    float* sc = sA + D * (D + 1);        // [D]
    float* so = sc + D;                  // [8 warps][D]
    const int x = blockIdx.y, z = x / g;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float* Ax = A + (long long)x * D * D;
    for (int t = threadIdx.x; t < D * D; t += blockDim.x) sA[(t / D) * (D + 1) + t % D] = Ax[t];
    __syncthreads();
    for (int j = threadIdx.x; j < D; j += blockDim.x) {
        float acc = Rbar[(long long)x * D + j];
        for (int c = 0; c < D; ++c) acc = fmaf(-sA[j * (D + 1) + c], obar[(long long)x * D + c], acc);
        sc[j] = acc;
    }
    __syncthreads();
    const int32_t* perm = qperm + (long long)z * N;
    float* row = so + warp * D;
    for (int p = blockIdx.x * 8 + warp; p < N; p += gridDim.x * 8) {
        const bf16* src = Osp + ((long long)x * N + p) * D;
        float o[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            o[e] = __bfloat162float(src[lane + 32 * e]);
            row[lane + 32 * e] = o[e];
        }
        __syncwarp();
        float acc[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = o[e] + sc[lane + 32 * e];
        for (int c = 0; c < D; ++c) {
            const float oc = row[c];
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] = fmaf(sA[(lane + 32 * e) * (D + 1) + c], oc, acc[e]);
        }
        __syncwarp();
        bf16* dst = O + ((long long)x * N + perm[p]) * D;
#pragma unroll
        for (int e = 0; e < EPL; ++e) dst[lane + 32 * e] = __float2bfloat16_rn(acc[e]);
    }
}

}  // namespace

size_t fit_smem_bytes(int d, int M, int r) {
    const size_t ld = (size_t)d + 1;
    size_t floats = 3 * (size_t)M * ld + (size_t)M * M + (size_t)d * r + 2 * (size_t)M + 2 * (size_t)d + (size_t)M;
    return floats * 4 + (size_t)r * 4;
}

cudaError_t launch_probe_residual(const float* Odense, const bf16* Osp, const int32_t* probe_pos,
                                  float* R, float* Osp_probe, int Hp, int g, int N, int d, int M,
                                  cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    probe_residual_kernel<<<dim3(M, Hp), d, 0, s>>>(Odense, Osp, probe_pos, R, Osp_probe, g, N, d, M);
    return cudaGetLastError();
}

cudaError_t launch_fit(const float* R, const float* Xp, const float* w, float lambda, float* obar,
                       float* Rbar, float* A, float* U, float* Bm, float* c0, int32_t* rank,
                       int Hp, int g, int d, int M, int r, bool rbar_unprojected, int* status, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    if (M > 64) return cudaErrorInvalidValue;
    const size_t smem = fit_smem_bytes(d, M, r);
    auto run = [&](auto kern) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<Hp, kFitThreads, smem, s>>>(R, Xp, w, lambda, obar, Rbar, A, U, Bm, c0, rank, g, M, r,
                                           rbar_unprojected ? 1 : 0, status);
        return cudaGetLastError();
    };
    if (d == 64) return run(fit_kernel<64>);
    if (d == 128) return run(fit_kernel<128>);
    return cudaErrorInvalidValue;
}

cudaError_t launch_writeback(const bf16* Osp, const int32_t* qperm, const float* U,
                             const float* Bm, const float* c0, const float* Radd, bf16* O, int Hp, int g, int N,
                             int d, int r, bool correct, int num_sms, cudaStream_t s) {
    const int cf = correct ? 1 : 0;
    // persistent CTAs (one full wave): each stages Bm and U^T once for thousands of rows
    auto run = [&](auto kern) -> cudaError_t {
        int occ = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 256, 0);
        if (e != cudaSuccess) return e;
        if (occ < 1) occ = 1;
        int per = occ * num_sms / Hp;
        const int maxb = (N + 8 * 4 - 1) / (8 * 4);    // 8 warps x 4 rows per iteration
        if (per > maxb) per = maxb;
        if (per < 1) per = 1;
        kern<<<dim3(per, Hp), 256, 0, s>>>(Osp, qperm, U, Bm, c0, Radd, O, g, N, r, cf);
        return cudaGetLastError();
    };
    if (r <= 16) {
        if (d == 64) return run(writeback_kernel<64, 16>);
        if (d == 128) return run(writeback_kernel<128, 16>);
    } else {
        if (d == 64) return run(writeback_kernel<64, 32>);
        if (d == 128) return run(writeback_kernel<128, 32>);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_writeback_ridge(const bf16* Osp, const int32_t* qperm, const float* A, const float* obar,
                                   const float* Rbar, bf16* O, int Hp, int g, int N, int d, int num_sms,
                                   cudaStream_t s) {
    int per = (4 * num_sms + Hp - 1) / Hp;
    const int maxb = (N + 8 * 16 - 1) / (8 * 16);
    if (per > maxb) per = maxb;
    const dim3 grid(per, Hp);
    const size_t smem = ((size_t)d * (d + 1) + d + 8 * d) * sizeof(float);
    cudaError_t e;
    if (d == 64) {
        e = cudaFuncSetAttribute(writeback_ridge_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        writeback_ridge_kernel<64><<<grid, 256, smem, s>>>(Osp, qperm, A, obar, Rbar, O, g, N);
    } else if (d == 128) {
        e = cudaFuncSetAttribute(writeback_ridge_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        writeback_ridge_kernel<128><<<grid, 256, smem, s>>>(Osp, qperm, A, obar, Rbar, O, g, N);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_probe_override(const float* Odense, const int32_t* probe, bf16* O, int Hp,
                                  int g, int N, int d, int M, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    probe_override_kernel<<<dim3(M, Hp), d, 0, s>>>(Odense, probe, O, g, N, d, M);
    return cudaGetLastError();
}

}  // namespace spr
