// Affine diagnostics of the hard-drop residual of each query head ([partition] diagnostics,
// judged against dense outputs): R = Od - Os over all N rows, and the least-squares affine map
// R ~ A Os + b. With X = [Os, 1] (N x (d+1)), G = X^T X and C = X^T R, the fit leaves
// SSE = sum ||R||^2 - tr(C^T G^-1 C); reported are
//   explained  = 1 - SSE / sum ||R_i - mean R||^2   (mean R = row d of C over N)
//   orthogonal = SSE / sum ||R||^2.
// Everything is accumulated in fp64: a tiled Gram kernel writes per-chunk partials of
// [G | C] ((d+1) x (2d+1)) and of sum ||R||^2, and one CTA per head sums the chunks in a fixed
// order, factors G (Cholesky, shared memory) and forms ||L^-1 c_q||^2 column by column.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace spr {
namespace {

constexpr int kT = 32;            // Gram tile (rows p of X, columns q of [X | R]) and row step
constexpr int kChunks = 8;        // row chunks per head (partials summed in this order)

// Y[i][c]: c < d -> Os[i][c]; c == d -> 1; c > d -> Od[i][c-d-1] - Os[i][c-d-1] (exact in fp64)
__device__ __forceinline__ double yval(const bf16* os, const bf16* od, int d, int c) {
    if (c < d) return (double)__bfloat162float(os[c]);
    if (c == d) return 1.0;
    const int k = c - d - 1;
    return (double)__bfloat162float(od[k]) - (double)__bfloat162float(os[k]);
}

__global__ void __launch_bounds__(256) affine_gram_kernel(const bf16* __restrict__ Os, const bf16* __restrict__ Od,
                                                          double* part, double* rr, int N, int d) {
    const int x = blockIdx.z, chunk = blockIdx.y;
    const int D1 = d + 1, DY = 2 * d + 1;
    const int qtiles = (DY + kT - 1) / kT;
    const int p0 = (blockIdx.x / qtiles) * kT, q0 = (blockIdx.x % qtiles) * kT;
    const int rows = (N + kChunks - 1) / kChunks, lo = chunk * rows, hi = min(N, lo + rows);
    __shared__ double sA[kT][kT + 1], sB[kT][kT + 1];
    const int ty = threadIdx.x / 8, tx = threadIdx.x % 8;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    double r2 = 0.0;
    const bool diag_r = p0 == 0 && q0 == 0;   // one tile per (head, chunk) also sums ||R||^2
    for (int i0 = lo; i0 < hi; i0 += kT) {
        __syncthreads();
        for (int t = threadIdx.x; t < kT * kT; t += blockDim.x) {
            const int r = t / kT, c = t % kT, i = i0 + r;
            const bool ok = i < hi;
            const bf16* os = Os + ((long long)x * N + i) * d;
            const bf16* od = Od + ((long long)x * N + i) * d;
            sA[r][c] = (ok && p0 + c < D1) ? yval(os, od, d, p0 + c) : 0.0;
            sB[r][c] = (ok && q0 + c < DY) ? yval(os, od, d, q0 + c) : 0.0;
        }
        __syncthreads();
#pragma unroll 8
        for (int r = 0; r < kT; ++r) {
            const double a = sA[r][ty];
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[k] = fma(a, sB[r][tx + 8 * k], acc[k]);
        }
        if (diag_r) {
            for (int t = threadIdx.x; t < kT * d; t += blockDim.x) {
                const int i = i0 + t / d, c = t % d;
                if (i < hi) {
                    const long long o = ((long long)x * N + i) * d + c;
                    const double v = (double)__bfloat162float(Od[o]) - (double)__bfloat162float(Os[o]);
                    r2 = fma(v, v, r2);
                }
            }
        }
    }
    double* P = part + ((long long)x * kChunks + chunk) * D1 * DY;
    const int p = p0 + ty;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int q = q0 + tx + 8 * k;
        if (p < D1 && q < DY) P[(long long)p * DY + q] = acc[k];
    }
    if (diag_r) {
        // fixed-order block sum of ||R||^2
        __shared__ double red[256];
        red[threadIdx.x] = r2;
        __syncthreads();
        if (threadIdx.x == 0) {
            double s = 0.0;
            for (int t = 0; t < 256; ++t) s += red[t];
            rr[(long long)x * kChunks + chunk] = s;
        }
    }
}

__global__ void __launch_bounds__(512) affine_solve_kernel(double* part, const double* __restrict__ rr, double* out,
                                                           int N, int d, int* status) {
    const int x = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
    const int D1 = d + 1, DY = 2 * d + 1;
    extern __shared__ double Lsm[];           // [D1][D1], then sum_i R_i [d]
    double* sRsum = Lsm + D1 * D1;
    __shared__ double red[512];
    __shared__ int bad;
    double* P0 = part + (long long)x * kChunks * D1 * DY;
    // sum the chunks into chunk 0 in a fixed order; G to shared memory, the intercept row of C
    // (row d of X^T R = sum_i R_i) aside before the solves overwrite it
    for (int t = tid; t < D1 * DY; t += nt) {
        double s = P0[t];
        for (int ch = 1; ch < kChunks; ++ch) s += P0[(long long)ch * D1 * DY + t];
        P0[t] = s;
        const int p = t / DY, q = t % DY;
        if (q < D1) Lsm[p * D1 + q] = s;
        if (p == d && q >= D1) sRsum[q - D1] = s;
    }
    if (tid == 0) bad = 0;
    __syncthreads();
    // Cholesky G = L L^T, right-looking, lower triangle in place
    for (int j = 0; j < D1; ++j) {
        double djj = Lsm[j * D1 + j];
        if (!(djj > 0.0)) {
            if (tid == 0) bad = 1;
            djj = 1e-300;
        }
        const double dj = sqrt(djj);
        for (int i = j + 1 + tid; i < D1; i += nt) Lsm[i * D1 + j] /= dj;
        __syncthreads();
        if (tid == 0) Lsm[j * D1 + j] = dj;
        const int n1 = D1 - j - 1;
        for (int t = tid; t < n1 * n1; t += nt) {
            const int i = j + 1 + t / n1, k = j + 1 + t % n1;
            if (k <= i) Lsm[i * D1 + k] -= Lsm[i * D1 + j] * Lsm[k * D1 + j];
        }
        __syncthreads();
    }
    // tr(C^T G^-1 C) = sum_q ||L^-1 c_q||^2; column q of C sits in column D1 + q (stride DY)
    double tr = 0.0;
    for (int q = tid; q < d; q += nt) {
        double* c = P0 + D1 + q;
        for (int p = 0; p < D1; ++p) {
            double v = c[(long long)p * DY];
            for (int k = 0; k < p; ++k) v -= Lsm[p * D1 + k] * c[(long long)k * DY];
            v /= Lsm[p * D1 + p];
            c[(long long)p * DY] = v;
            tr += v * v;
        }
    }
    red[tid] = tr;
    __syncthreads();
    if (tid == 0) {
        double t = 0.0;
        for (int k = 0; k < nt; ++k) t += red[k];
        double rsum = 0.0;
        for (int ch = 0; ch < kChunks; ++ch) rsum += rr[(long long)x * kChunks + ch];
        double m2 = 0.0;
        for (int q = 0; q < d; ++q) m2 += sRsum[q] * sRsum[q];
        const double sse = rsum - t;
        const double centred = rsum - m2 / (double)N;
        out[2 * x] = bad ? NAN : 1.0 - sse / centred;
        out[2 * x + 1] = bad ? NAN : sse / rsum;
        if (bad) set_status(status, kDevBounds);
    }
}

}  // namespace

size_t affine_diag_workspace(int Hp, int d) {
    const size_t D1 = d + 1, DY = 2 * (size_t)d + 1;
    return ((size_t)Hp * kChunks * D1 * DY + (size_t)Hp * kChunks) * sizeof(double);
}

cudaError_t launch_affine_diag(const bf16* Os, const bf16* Od, double* out, void* ws, int Hp, int N, int d,
                               int* status, cudaStream_t s) {
    const int D1 = d + 1, DY = 2 * d + 1;
    double* part = static_cast<double*>(ws);
    double* rr = part + (size_t)Hp * kChunks * D1 * DY;
    const int tiles = ((D1 + kT - 1) / kT) * ((DY + kT - 1) / kT);
    affine_gram_kernel<<<dim3(tiles, kChunks, Hp), 256, 0, s>>>(Os, Od, part, rr, N, d);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = ((size_t)D1 * D1 + d) * sizeof(double);
    e = cudaFuncSetAttribute(affine_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    affine_solve_kernel<<<Hp, 512, smem, s>>>(part, rr, out, N, d, status);
    return cudaGetLastError();
}

}  // namespace spr
