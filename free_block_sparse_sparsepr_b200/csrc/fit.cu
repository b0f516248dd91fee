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

__device__ __forceinline__ float block_sum(float v, float* red) {
    v = warp_sum(v);
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[w] = v;
    __syncthreads();
    float t = 0.f;
    if (threadIdx.x == 0) {
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
        red[32] = t;
    }
    __syncthreads();
    return red[32];
}

// Per query head x:
//   xbar, Rbar   w-weighted means of the probes' sparse outputs X and residuals R
//   A            argmin sum_m w_m ||(R_m - Rbar) - A (X_m - xbar)||^2 + lambda ||A||_F^2, via the
//                M x M system: A = Ys^T (Xs Xs^T + lambda I)^-1 Xs, Xs/Ys rows scaled by sqrt(w_m)
//   U            top-r eigenvectors of the Gram matrix of [sqrt(w_m) R_m] mapped to output
//                space (= top-r left singular vectors), cyclic Jacobi in fp32
//   Bm = U^T A, c0 = U^T Rbar - Bm xbar  so that the correction is U (c0 + Bm o).
constexpr int kFitThreads = 256;
__global__ void __launch_bounds__(kFitThreads) fit_kernel(
    const float* __restrict__ Rg, const float* __restrict__ Xg, const float* __restrict__ wts,
    float lambda, float* obar, float* Rbar, float* A, float* U, float* Bm, float* c0,
    int32_t* rank_out, int g, int d, int M, int r, int* status) {
    const int x = blockIdx.x, z = x / g, tid = threadIdx.x, nt = blockDim.x;
    const int Mp = (M + 1) & ~1;
    extern __shared__ float sm[];
    float* X = sm;                 // [M][d]
    float* Y = X + M * d;          // [M][d]
    float* Km = Y + M * d;         // [M][M]
    float* Gr = Km + M * M;        // [M][M]
    float* Vv = Gr + M * M;        // [M][M]
    float* Us = Vv + M * M;        // [d][r]
    float* w = Us + d * r;         // [M]
    float* sw = w + M;             // [M]
    float* xb = sw + M;            // [d]
    float* yb = xb + d;            // [d]
    float* rc = yb + d;            // [Mp/2]
    float* rs = rc + Mp / 2;       // [Mp/2]
    float* eig = rs + Mp / 2;      // [M]
    float* red = eig + M;          // [33]
    int* pp = reinterpret_cast<int*>(red + 33);   // [Mp/2]
    int* pq = pp + Mp / 2;                        // [Mp/2]
    int* sel = pq + Mp / 2;                       // [r]
    __shared__ float sW;
    __shared__ int s_rank, s_stop;

    const float* Rx = Rg + (long long)x * M * d;
    const float* Xx = Xg + (long long)x * M * d;
    for (int t = tid; t < M * d; t += nt) { X[t] = Xx[t]; Y[t] = Rx[t]; }
    for (int t = tid; t < M; t += nt) { w[t] = wts[(long long)z * M + t]; sw[t] = sqrtf(wts[(long long)z * M + t]); }
    __syncthreads();
    if (tid == 0) {
        float W = 0.f;
        for (int m = 0; m < M; ++m) W += w[m];
        sW = W;
    }
    __syncthreads();
    const float W = sW;
    for (int c = tid; c < d; c += nt) {
        float sx = 0.f, sy = 0.f;
        for (int m = 0; m < M; ++m) { sx = fmaf(w[m], X[m * d + c], sx); sy = fmaf(w[m], Y[m * d + c], sy); }
        xb[c] = sx / W;
        yb[c] = sy / W;
    }
    // Gram matrix of the weighted, uncentred residuals.
    for (int t = tid; t < M * M; t += nt) {
        const int i = t / M, j = t % M;
        float acc = 0.f;
        for (int c = 0; c < d; ++c) acc = fmaf(Y[i * d + c], Y[j * d + c], acc);
        Gr[t] = sw[i] * sw[j] * acc;
    }
    __syncthreads();
    for (int t = tid; t < M * d; t += nt) {
        const int m = t / d, c = t % d;
        X[t] = sw[m] * (X[t] - xb[c]);
        Y[t] = sw[m] * (Y[t] - yb[c]);
    }
    __syncthreads();
    for (int t = tid; t < M * M; t += nt) {
        const int i = t / M, j = t % M;
        float acc = 0.f;
        for (int c = 0; c < d; ++c) acc = fmaf(X[i * d + c], X[j * d + c], acc);
        Km[t] = acc + (i == j ? lambda : 0.f);
    }
    __syncthreads();
    // Cholesky Km = L L^T (lower triangle, in place).
    for (int j = 0; j < M; ++j) {
        if (tid == 0) {
            float s = Km[j * M + j];
            for (int k = 0; k < j; ++k) s -= Km[j * M + k] * Km[j * M + k];
            if (!(s > 0.f)) { set_status(status, kDevBounds); s = 1e-30f; }
            Km[j * M + j] = sqrtf(s);
        }
        __syncthreads();
        for (int i = j + 1 + tid; i < M; i += nt) {
            float s = Km[i * M + j];
            for (int k = 0; k < j; ++k) s -= Km[i * M + k] * Km[j * M + k];
            Km[i * M + j] = s / Km[j * M + j];
        }
        __syncthreads();
    }
    // Z = Km^-1 Xs, column by column, in place in X.
    for (int c = tid; c < d; c += nt) {
        for (int m = 0; m < M; ++m) {
            float s = X[m * d + c];
            for (int k = 0; k < m; ++k) s -= Km[m * M + k] * X[k * d + c];
            X[m * d + c] = s / Km[m * M + m];
        }
        for (int m = M - 1; m >= 0; --m) {
            float s = X[m * d + c];
            for (int k = m + 1; k < M; ++k) s -= Km[k * M + m] * X[k * d + c];
            X[m * d + c] = s / Km[m * M + m];
        }
    }
    __syncthreads();
    float* Ax = A + (long long)x * d * d;
    for (int t = tid; t < d * d; t += nt) {
        const int c = t / d, c2 = t % d;
        float acc = 0.f;
        for (int m = 0; m < M; ++m) acc = fmaf(Y[m * d + c], X[m * d + c2], acc);
        Ax[t] = acc;
    }
    // Cyclic Jacobi on Gr with round-robin disjoint pairs; V accumulates the rotations.
    for (int t = tid; t < M * M; t += nt) Vv[t] = (t / M == t % M) ? 1.f : 0.f;
    __syncthreads();
    for (int sweep = 0; sweep < 15; ++sweep) {
        float off = 0.f, tot = 0.f;
        for (int t = tid; t < M * M; t += nt) {
            const float v = Gr[t] * Gr[t];
            tot += v;
            if (t / M != t % M) off += v;
        }
        off = block_sum(off, red);
        tot = block_sum(tot, red);
        if (tid == 0) s_stop = (off <= 1e-12f * tot) ? 1 : 0;
        __syncthreads();
        if (s_stop) break;
        for (int k = 0; k < Mp - 1; ++k) {
            for (int i = tid; i < Mp / 2; i += nt) {
                const int a1 = (i == 0) ? 0 : ((i - 1 + k) % (Mp - 1)) + 1;
                const int b1 = ((Mp - 2 - i + k) % (Mp - 1)) + 1;
                const int p = min(a1, b1), q = max(a1, b1);
                float c = 1.f, s = 0.f;
                if (q < M) {
                    const float apq = Gr[p * M + q];
                    if (apq != 0.f) {
                        const float theta = (Gr[q * M + q] - Gr[p * M + p]) / (2.f * apq);
                        const float tt = (theta >= 0.f ? 1.f : -1.f) / (fabsf(theta) + sqrtf(theta * theta + 1.f));
                        c = 1.f / sqrtf(tt * tt + 1.f);
                        s = tt * c;
                    }
                }
                pp[i] = p; pq[i] = q; rc[i] = c; rs[i] = s;
            }
            __syncthreads();
            for (int t = tid; t < (Mp / 2) * M; t += nt) {
                const int i = t / M, col = t % M, p = pp[i], q = pq[i];
                if (q >= M) continue;
                const float c = rc[i], s = rs[i];
                const float gp = Gr[p * M + col], gq = Gr[q * M + col];
                Gr[p * M + col] = c * gp - s * gq;
                Gr[q * M + col] = s * gp + c * gq;
            }
            __syncthreads();
            for (int t = tid; t < (Mp / 2) * M; t += nt) {
                const int i = t / M, row = t % M, p = pp[i], q = pq[i];
                if (q >= M) continue;
                const float c = rc[i], s = rs[i];
                const float gp = Gr[row * M + p], gq = Gr[row * M + q];
                Gr[row * M + p] = c * gp - s * gq;
                Gr[row * M + q] = s * gp + c * gq;
                const float vp = Vv[row * M + p], vq = Vv[row * M + q];
                Vv[row * M + p] = c * vp - s * vq;
                Vv[row * M + q] = s * vp + c * vq;
            }
            __syncthreads();
        }
    }
    // Top-r eigenpairs (descending; ties -> lower index) and the numerical rank.
    for (int t = tid; t < M; t += nt) eig[t] = fmaxf(Gr[t * M + t], 0.f);
    __syncthreads();
    if (tid < 32) {
        const int lane = tid;
        for (int k = 0; k < r; ++k) {
            float best = -1.f;
            int bi = M;
            for (int m = lane; m < M; m += 32) {
                bool used = false;
                for (int j = 0; j < k; ++j) used |= (sel[j] == m);
                if (!used && (eig[m] > best || (eig[m] == best && m < bi))) { best = eig[m]; bi = m; }
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
            const float e0 = eig[sel[0]];
            int rk = 0;
            for (int k = 0; k < r && k < M; ++k) {
                const float e = eig[sel[k]];
                if (e > 0.f && e > e0 * tol * tol) ++rk;
            }
            s_rank = rk;
        }
    }
    __syncthreads();
    const int rank = s_rank;
    for (int t = tid; t < d * r; t += nt) {
        const int c = t / r, k = t % r;
        float val = 0.f;
        if (k < rank) {
            const int e = sel[k];
            float acc = 0.f;
            for (int m = 0; m < M; ++m) acc = fmaf(sw[m] * Rx[m * d + c], Vv[m * M + e], acc);
            val = acc / sqrtf(eig[e]);
        }
        Us[t] = val;
        U[(long long)x * d * r + t] = val;
    }
    __syncthreads();
    float* Bx = Bm + (long long)x * r * d;
    for (int t = tid; t < r * d; t += nt) {
        const int k = t / d, c2 = t % d;
        float acc = 0.f;
        for (int c = 0; c < d; ++c) acc = fmaf(Us[c * r + k], Ax[(long long)c * d + c2], acc);
        Bx[t] = acc;
    }
    __syncthreads();
    for (int k = tid; k < r; k += nt) {
        float a1 = 0.f, a2 = 0.f;
        for (int c = 0; c < d; ++c) {
            a1 = fmaf(Us[c * r + k], yb[c], a1);
            a2 = fmaf(Bx[(long long)k * d + c], xb[c], a2);
        }
        c0[(long long)x * r + k] = a1 - a2;
    }
    for (int c = tid; c < d; c += nt) {
        obar[(long long)x * d + c] = xb[c];
        Rbar[(long long)x * d + c] = yb[c];
    }
    if (tid == 0) rank_out[x] = rank;
}

// O[qperm[p]] = Osp[p] + U (c0 + Bm Osp[p]); one warp per group-major row. Each lane holds
// EPL consecutive elements; Bm and U^T are staged row-major in shared memory so every
// vector load is conflict-free. The RP partial dot products are reduced by recursive
// halving (RP/2 + ... + 1 + 1 shuffles); afterwards lane 2k holds t_k.
template <int D, int RP>
__global__ void __launch_bounds__(256) writeback_kernel(const bf16* __restrict__ Osp,
                                                        const int32_t* __restrict__ qperm,
                                                        const float* __restrict__ U,
                                                        const float* __restrict__ Bm,
                                                        const float* __restrict__ c0, bf16* O,
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
    const int32_t* perm = qperm + (long long)z * N;
    for (int p = blockIdx.x * 8 + warp; p < N; p += gridDim.x * 8) {
        const bf16* src = Osp + ((long long)x * N + p) * D + lane * EPL;
        float o[EPL];
#pragma unroll
        for (int e = 0; e < EPL; e += 2) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(src + e));
            o[e] = f.x;
            o[e + 1] = f.y;
        }
        if (correct) {
            float a[RP];
#pragma unroll
            for (int k = 0; k < RP; ++k) {
                float acc = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; ++e) acc = fmaf(sB[k * D + lane * EPL + e], o[e], acc);
                a[k] = acc;
            }
            // Step with lane bit b: lanes with b set keep the upper half of the remaining
            // partials (adding the partner's upper half), the others the lower half.
#pragma unroll
            for (int n = RP, bit = 16; n > 1; n >>= 1, bit >>= 1) {
                const bool up = (lane & bit) != 0;
#pragma unroll
                for (int i = 0; i < n / 2; ++i) {
                    const float send = up ? a[i] : a[i + n / 2];
                    const float keep = up ? a[i + n / 2] : a[i];
                    a[i] = keep + __shfl_xor_sync(kFull, send, bit);
                }
            }
            if (RP == 16) a[0] += __shfl_xor_sync(kFull, a[0], 1);   // lanes 2k, 2k+1 held halves of t_k
            const float tk = a[0];
            float delta[EPL];
#pragma unroll
            for (int e = 0; e < EPL; ++e) delta[e] = 0.f;
#pragma unroll
            for (int k = 0; k < RP; ++k) {
                const float t = __shfl_sync(kFull, tk, (RP == 16) ? 2 * k : k) + sc[k];
#pragma unroll
                for (int e = 0; e < EPL; ++e) delta[e] = fmaf(sUt[k * D + lane * EPL + e], t, delta[e]);
            }
#pragma unroll
            for (int e = 0; e < EPL; ++e) o[e] += delta[e];
        }
        bf16* dst = O + ((long long)x * N + perm[p]) * D + lane * EPL;
#pragma unroll
        for (int e = 0; e < EPL; e += 2)
            *reinterpret_cast<__nv_bfloat162*>(dst + e) = __floats2bfloat162_rn(o[e], o[e + 1]);
    }
}

__global__ void probe_override_kernel(const float* __restrict__ Od, const int32_t* __restrict__ probe,
                                      bf16* O, int g, int N, int d, int M) {
    const int x = blockIdx.y, m = blockIdx.x, c = threadIdx.x, z = x / g;
    const int row = probe[(long long)z * M + m];
    O[((long long)x * N + row) * d + c] = __float2bfloat16_rn(Od[((long long)x * M + m) * d + c]);
}

}  // namespace

size_t fit_smem_bytes(int d, int M, int r) {
    const int Mp = (M + 1) & ~1;
    size_t floats = (size_t)2 * M * d + 3 * (size_t)M * M + (size_t)d * r + 2 * M + 2 * d + Mp + M + 33;
    size_t ints = (size_t)Mp + r;
    return floats * 4 + ints * 4;
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
                       int Hp, int g, int d, int M, int r, int* status, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    const size_t smem = fit_smem_bytes(d, M, r);
    cudaError_t e = cudaFuncSetAttribute(fit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    fit_kernel<<<Hp, kFitThreads, smem, s>>>(R, Xp, w, lambda, obar, Rbar, A, U, Bm, c0, rank, g, d, M, r, status);
    return cudaGetLastError();
}

cudaError_t launch_writeback(const bf16* Osp, const int32_t* qperm, const float* U,
                             const float* Bm, const float* c0, bf16* O, int Hp, int g, int N,
                             int d, int r, bool correct, cudaStream_t s) {
    const int blocks = (N + 8 * 16 - 1) / (8 * 16);   // 16 rows per warp
    dim3 grid(blocks, Hp);
    const int cf = correct ? 1 : 0;
    if (r <= 16) {
        if (d == 64) writeback_kernel<64, 16><<<grid, 256, 0, s>>>(Osp, qperm, U, Bm, c0, O, g, N, r, cf);
        else if (d == 128) writeback_kernel<128, 16><<<grid, 256, 0, s>>>(Osp, qperm, U, Bm, c0, O, g, N, r, cf);
        else return cudaErrorInvalidValue;
    } else {
        if (d == 64) writeback_kernel<64, 32><<<grid, 256, 0, s>>>(Osp, qperm, U, Bm, c0, O, g, N, r, cf);
        else if (d == 128) writeback_kernel<128, 32><<<grid, 256, 0, s>>>(Osp, qperm, U, Bm, c0, O, g, N, r, cf);
        else return cudaErrorInvalidValue;
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
