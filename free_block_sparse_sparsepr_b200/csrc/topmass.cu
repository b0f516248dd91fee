// Support diagnostics ([support]). For each row of responses z_j (j < N), the fraction of keys
// that carries 90% of its softmax mass: the smallest k such that the k largest
// p_j = exp(z_j - max z) sum to at least 0.9 sum_j p_j, divided by N.
//   - sampled rows: the responses are the key features F[j][s] written by the response GEMM
//     (8 contiguous floats per key row per CTA);
//   - shared rows: up to eight rows of each query group ([support]: the queries of a group share
//     one route), their logits against every key written row-major by a GEMM; the CTA then also
//     counts the union of the eight 90%-mass sets, each taken as the keys whose logit is at least
//     the k-th largest.
//
// One CTA per 8 rows; every pass streams the rows once. Pass 1: per-row maximum. Pass 2: total
// mass, and mass and count per bin of delta = max - z (256 bins of 1/8 nat; the last one
// open-ended). The bin where the cumulative mass from the top crosses 90% is then narrowed (256
// sub-bins per level) until it holds at most kCap keys; those are sorted exactly (bitonic, in
// shared memory, descending logit) and walked in order to the crossing.
#include <limits.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace spr {
namespace {

constexpr int kCols = 8;
constexpr int kThreads = 512;
constexpr int kBins = 256;
constexpr int kCap = 4096;
constexpr int kMaxLevels = 4;
constexpr float kMass = 0.9f;

struct Smem {
    float hmass[kCols][kBins];
    int hcnt[kCols][kBins];
    float red[kThreads / 32][kCols];
    float mx[kCols], total[kCols], lo[kCols], width[kCols], mass0[kCols];
    int count0[kCols], settled[kCols], nval[kCols], result[kCols];
    float tau[kCols];                    // logit of the k-th largest key (-inf: every key)
    int red_i[kThreads / 32];
    unsigned open[kCols];                // 1 if the current range has no upper end (level 0's last bin)
    float vals[kCols][kCap];
};

enum { kLayoutFeatures = 0, kLayoutRows = 1 };

// Inverse of the order-preserving key the response GEMM's epilogue stores for each column maximum.
__device__ __forceinline__ float from_max_key(unsigned k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <int LAYOUT>
__global__ void __launch_bounds__(kThreads) support_kernel(const float* __restrict__ src, float* out,
                                                           float* out_union, const int32_t* __restrict__ qoff,
                                                           const unsigned* __restrict__ colmax, int N, int ld,
                                                           int S, int Gq, int z0) {
    extern __shared__ unsigned char sm_raw[];
    Smem& sm = *reinterpret_cast<Smem*>(sm_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // features: F[z][j][c0 + c] (ld = DP); rows: Z[zl][a * kCols + c][j] (ld = row stride)
    const float* base;
    int ncol;
    long long oidx;
    int z;
    if (LAYOUT == kLayoutFeatures) {
        z = blockIdx.y;
        const int c0 = blockIdx.x * kCols;
        ncol = min(kCols, S - c0);
        base = src + (long long)z * N * ld + c0;
        oidx = (long long)z * S + c0;
    } else {
        const int zl = blockIdx.y, a = blockIdx.x;
        z = z0 + zl;
        const int size = qoff[(long long)z * (Gq + 1) + a + 1] - qoff[(long long)z * (Gq + 1) + a];
        ncol = min(kCols, size);
        base = src + ((long long)zl * Gq + a) * kCols * ld;
        oidx = ((long long)z * Gq + a) * kCols;
        if (ncol <= 0) {
            if (tid < kCols) out[oidx + tid] = 0.f;
            if (tid == 0) out_union[(long long)z * Gq + a] = 0.f;
            return;
        }
    }
    auto load_row = [&](long long j, float (&v)[kCols]) {
        if (LAYOUT == kLayoutFeatures) {
            const float4* p = reinterpret_cast<const float4*>(base + j * ld);
            const float4 a = __ldg(p), b = __ldg(p + 1);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        } else {
#pragma unroll
            for (int c = 0; c < kCols; ++c) v[c] = c < ncol ? __ldg(base + (long long)c * ld + j) : 0.f;
        }
    };

    // ---- pass 1: maxima (taken from the response GEMM's epilogue when it formed them)
    float v[kCols], acc[kCols];
    if (LAYOUT == kLayoutFeatures && colmax) {
        if (tid < kCols)
            sm.red[0][tid] = tid < ncol ? from_max_key(colmax[(long long)z * ld + blockIdx.x * kCols + tid]) : -INFINITY;
    } else {
#pragma unroll
        for (int c = 0; c < kCols; ++c) acc[c] = -INFINITY;
        for (long long j = tid; j < N; j += kThreads) {
            load_row(j, v);
#pragma unroll
            for (int c = 0; c < kCols; ++c) acc[c] = fmaxf(acc[c], v[c]);
        }
#pragma unroll
        for (int c = 0; c < kCols; ++c) {
            const float r = warp_max(acc[c]);
            if (lane == 0) sm.red[warp][c] = r;
        }
    }
    __syncthreads();
    if (tid < kCols) {
        float r = -INFINITY;
        const int nw = (LAYOUT == kLayoutFeatures && colmax) ? 1 : kThreads / 32;
        for (int w = 0; w < nw; ++w) r = fmaxf(r, sm.red[w][tid]);
        sm.mx[tid] = r;
        sm.lo[tid] = 0.f;
        sm.width[tid] = 0.125f;
        sm.open[tid] = 1u;
        sm.mass0[tid] = 0.f;
        sm.count0[tid] = 0;
        sm.settled[tid] = tid < ncol ? 0 : 1;
        sm.tau[tid] = -INFINITY;
    }
    __syncthreads();
    float m[kCols];
#pragma unroll
    for (int c = 0; c < kCols; ++c) m[c] = sm.mx[c];

    // ---- histogram levels: level 0 also yields the total mass
    for (int level = 0; level < kMaxLevels; ++level) {
        for (int t = tid; t < kCols * kBins; t += kThreads) {
            (&sm.hmass[0][0])[t] = 0.f;
            (&sm.hcnt[0][0])[t] = 0;
        }
        __syncthreads();
        float lo[kCols], inv_w[kCols];
        bool act[kCols], open[kCols];
#pragma unroll
        for (int c = 0; c < kCols; ++c) {
            lo[c] = sm.lo[c];
            inv_w[c] = 1.f / sm.width[c];
            act[c] = !sm.settled[c];
            open[c] = sm.open[c] != 0u;
            acc[c] = 0.f;
        }
        for (long long j = tid; j < N; j += kThreads) {
            load_row(j, v);
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
                if (!act[c]) continue;
                const float d = m[c] - v[c];
                const float p = expf(v[c] - m[c]);
                if (level == 0) acc[c] += p;
                const float b = (d - lo[c]) * inv_w[c];
                if (b >= 0.f && (b < (float)kBins || open[c])) {
                    const int bi = min(kBins - 1, (int)b);
                    atomicAdd(&sm.hmass[c][bi], p);
                    atomicAdd(&sm.hcnt[c][bi], 1);
                }
            }
        }
        if (level == 0) {
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
                const float r = warp_sum(acc[c]);
                if (lane == 0) sm.red[warp][c] = r;
            }
        }
        __syncthreads();
        // one warp per column: find the bin where the cumulative mass crosses the target
        if (warp < kCols && !sm.settled[warp]) {
            const int c = warp;
            if (level == 0 && lane == 0) {
                float r = 0.f;
                for (int w = 0; w < kThreads / 32; ++w) r += sm.red[w][c];
                sm.total[c] = r;
            }
            __syncwarp();
            const float target = kMass * sm.total[c];
            float base = sm.mass0[c];
            int cbase = sm.count0[c];
            int hit = -1;
            for (int b0 = 0; b0 < kBins && hit < 0; b0 += 32) {
                const float bm = sm.hmass[c][b0 + lane];
                const int bc = sm.hcnt[c][b0 + lane];
                float inc = bm;
                int cinc = bc;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float tv = __shfl_up_sync(kFull, inc, o);
                    const int tc = __shfl_up_sync(kFull, cinc, o);
                    if (lane >= o) { inc += tv; cinc += tc; }
                }
                const unsigned crossed = __ballot_sync(kFull, base + inc >= target);
                if (crossed) {
                    const int l = __ffs(crossed) - 1;
                    hit = b0 + l;
                    const float before = __shfl_sync(kFull, inc - bm, l);
                    const int cbefore = __shfl_sync(kFull, cinc - bc, l);
                    base += before;
                    cbase += cbefore;
                } else {
                    base += __shfl_sync(kFull, inc, 31);
                    cbase += __shfl_sync(kFull, cinc, 31);
                }
            }
            if (lane == 0) {
                if (hit < 0) {
                    // rounding left the target unreached: every key counts
                    sm.result[c] = N;
                    sm.settled[c] = 2;
                } else {
                    sm.mass0[c] = base;
                    sm.count0[c] = cbase;
                    const bool last_open = sm.open[c] && hit == kBins - 1;
                    sm.lo[c] = sm.lo[c] + (float)hit * sm.width[c];
                    sm.open[c] = last_open ? 1u : 0u;
                    if (!last_open) sm.width[c] = sm.width[c] / (float)kBins;
                    sm.nval[c] = sm.hcnt[c][hit];
                    if (sm.hcnt[c][hit] <= kCap || level + 1 == kMaxLevels) sm.settled[c] = 3;  // gather next
                }
            }
        }
        __syncthreads();
        bool more = false;
        for (int c = 0; c < kCols; ++c) more |= sm.settled[c] == 0;
        if (!more) break;
    }

    // ---- gather the crossing bin's keys and settle each column exactly
    if (tid < kCols) sm.nval[tid] = 0;
    __syncthreads();
    {
        float lo[kCols], hi[kCols];
        bool act[kCols];
#pragma unroll
        for (int c = 0; c < kCols; ++c) {
            act[c] = sm.settled[c] == 3;
            lo[c] = sm.lo[c];
            // the open range of level 0's last bin has no upper end; a narrowed bin is
            // [lo, lo + width * kBins) in the units it was found with
            hi[c] = sm.open[c] ? INFINITY : sm.lo[c] + sm.width[c] * (float)kBins;
        }
        for (long long j = tid; j < N; j += kThreads) {
            load_row(j, v);
#pragma unroll
            for (int c = 0; c < kCols; ++c) {
                if (!act[c]) continue;
                const float d = m[c] - v[c];
                if (d >= lo[c] && d < hi[c]) {
                    const int at = atomicAdd(&sm.nval[c], 1);
                    if (at < kCap) sm.vals[c][at] = v[c];
                }
            }
        }
    }
    __syncthreads();
    for (int c = 0; c < kCols; ++c) {
        if (sm.settled[c] != 3) continue;
        const int n = min(sm.nval[c], kCap);
        int len = 1;
        while (len < n) len <<= 1;
        for (int t = n + tid; t < len; t += kThreads) sm.vals[c][t] = -INFINITY;
        __syncthreads();
        // bitonic sort, descending logit (descending p)
        for (int k = 2; k <= len; k <<= 1)
            for (int jj = k >> 1; jj > 0; jj >>= 1) {
                for (int t = tid; t < len; t += kThreads) {
                    const int u = t ^ jj;
                    if (u > t) {
                        const float a = sm.vals[c][t], b = sm.vals[c][u];
                        const bool up = (t & k) == 0;
                        if ((a < b) == up) { sm.vals[c][t] = b; sm.vals[c][u] = a; }
                    }
                }
                __syncthreads();
            }
        if (warp == 0) {
            const float target = kMass * sm.total[c];
            float base = sm.mass0[c];
            int idx = -1;
            for (int b0 = 0; b0 < n && idx < 0; b0 += 32) {
                const int t = b0 + lane;
                float inc = t < n ? expf(sm.vals[c][t] - m[c]) : 0.f;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float tv = __shfl_up_sync(kFull, inc, o);
                    if (lane >= o) inc += tv;
                }
                const unsigned crossed = __ballot_sync(kFull, t < n && base + inc >= target);
                if (crossed) idx = b0 + __ffs(crossed) - 1;
                else base += __shfl_sync(kFull, inc, 31);
            }
            if (lane == 0) {
                sm.result[c] = sm.count0[c] + (idx >= 0 ? idx + 1 : n);
                sm.tau[c] = n > 0 ? sm.vals[c][idx >= 0 ? idx : n - 1] : -INFINITY;
            }
        }
        __syncthreads();
    }
    if (LAYOUT == kLayoutFeatures) {
        if (tid < ncol) out[oidx + tid] = (float)min(sm.result[tid], N) / (float)N;
        return;
    }
    if (tid < kCols) out[oidx + tid] = tid < ncol ? (float)min(sm.result[tid], N) / (float)N : 0.f;
    // union of the rows' sets: keys whose logit reaches some row's threshold
    float tau[kCols];
#pragma unroll
    for (int c = 0; c < kCols; ++c) tau[c] = c < ncol ? sm.tau[c] : INFINITY;
    int cnt = 0;
    for (long long j = tid; j < N; j += kThreads) {
        load_row(j, v);
        bool in = false;
#pragma unroll
        for (int c = 0; c < kCols; ++c) in |= c < ncol && v[c] >= tau[c];
        cnt += in ? 1 : 0;
    }
    cnt = warp_sum_int(cnt);
    if (lane == 0) sm.red_i[warp] = cnt;
    __syncthreads();
    if (tid == 0) {
        int t = 0;
        for (int w = 0; w < kThreads / 32; ++w) t += sm.red_i[w];
        out_union[(long long)z * Gq + blockIdx.x] = (float)t / (float)N;
    }
}

}  // namespace

cudaError_t launch_topmass(const float* F, float* out, const unsigned* colmax, int P, int N, int DP, int S,
                           cudaStream_t s) {
    if (DP % kCols != 0 || S > DP) return cudaErrorInvalidValue;
    const size_t smem = sizeof(Smem);
    cudaError_t e = cudaFuncSetAttribute(support_kernel<kLayoutFeatures>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    support_kernel<kLayoutFeatures><<<dim3((S + kCols - 1) / kCols, P), kThreads, smem, s>>>(F, out, nullptr, nullptr,
                                                                                            colmax, N, DP, S, 0, 0);
    return cudaGetLastError();
}

cudaError_t launch_shared_support(const float* Z, long long ldz, const int32_t* qoff, float* row_frac,
                                  float* union_frac, int z0, int nz, int N, int Gq, cudaStream_t s) {
    const size_t smem = sizeof(Smem);
    cudaError_t e = cudaFuncSetAttribute(support_kernel<kLayoutRows>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    if (ldz > INT_MAX) return cudaErrorInvalidValue;
    support_kernel<kLayoutRows><<<dim3(Gq, nz), kThreads, smem, s>>>(Z, row_frac, union_frac, qoff, nullptr, N, (int)ldz,
                                                                     kCols, Gq, z0);
    return cudaGetLastError();
}

// Row m of query group a of head z: the group's group-major position
// lo + floor((m + 1/2) size / R'), R' = min(8, size), in query head z * g + (m mod g); rows past
// R' are zero. Qsh[z][a * 8 + m][:] for d-wide bf16 rows.
static __global__ void shared_rows_kernel(const bf16* __restrict__ Q, const int32_t* __restrict__ qperm,
                                   const int32_t* __restrict__ qoff, bf16* Qsh, int g, int N, int d, int Gq) {
    const int z = blockIdx.y, a = blockIdx.x;
    const int lo = qoff[(long long)z * (Gq + 1) + a], size = qoff[(long long)z * (Gq + 1) + a + 1] - lo;
    const int Rp = min(kCols, size);
    for (int t = threadIdx.x; t < kCols * (d / 8); t += blockDim.x) {
        const int m = t / (d / 8), c = (t % (d / 8)) * 8;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (m < Rp) {
            const int pos = lo + (int)(((2ll * m + 1) * size) / (2ll * Rp));
            const int row = qperm[(long long)z * N + pos];
            val = *reinterpret_cast<const uint4*>(Q + (((long long)z * g + m % g) * N + row) * d + c);
        }
        *reinterpret_cast<uint4*>(Qsh + (((long long)z * Gq + a) * kCols + m) * d + c) = val;
    }
}

cudaError_t launch_shared_rows(const bf16* Q, const int32_t* qperm, const int32_t* qoff, bf16* Qsh, int P, int g,
                               int N, int d, int Gq, cudaStream_t s) {
    if (d % 8 != 0) return cudaErrorInvalidValue;
    shared_rows_kernel<<<dim3(Gq, P), 128, 0, s>>>(Q, qperm, qoff, Qsh, g, N, d, Gq);
    return cudaGetLastError();
}

}  // namespace spr
