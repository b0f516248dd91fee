// Lloyd k-means of the response-coupled partition (key features, query
// coordinates), the stable counting sort that gives the group-major order, and
// the per-group means. Everything is deterministic: integer counts, fixed
// summation orders, no floating-point atomics.
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace spr {
namespace {

constexpr int kSortSub = 256;       // rows per sub-chunk (one row per thread)
constexpr int kSortChunk = 2048;    // rows per counting-sort chunk (one CTA, 8 sub-chunks in order)
constexpr int kAssignRows = 128;    // rows per assignment CTA (one row per thread)
constexpr int kAssignCentMax = 128; // centroids staged in shared memory per pass (64 at D = 128)

__global__ void km_seed_kernel(const float* X, float* C, int n, int G, int DP) {
    const int z = blockIdx.x;
    for (int t = threadIdx.x; t < G * DP; t += blockDim.x) {
        int g = t / DP, k = t % DP;
        long long row = sample_pos(g, n, G);
        C[((long long)z * G + g) * DP + k] = X[((long long)z * n + row) * DP + k];
    }
}

// Nearest centroid per row: argmin_g ||c_g||^2 - 2 x.c_g (ties -> lowest g), fp32.
template <int DP>
__global__ void __launch_bounds__(kAssignRows) km_assign_kernel(const float* __restrict__ X,
                                                                const float* __restrict__ C,
                                                                int32_t* labels, float* dist,
                                                                int* changed, const int* done,
                                                                int n, int G, int first) {
    constexpr int kAssignCent = DP > 64 ? 64 : kAssignCentMax;
    const int z = blockIdx.y;
    if (done && done[z]) return;
    __shared__ __align__(16) float sC[kAssignCent * DP];
    __shared__ float sN[kAssignCent];
    const int i = blockIdx.x * kAssignRows + threadIdx.x;
    const bool valid = i < n;
    float x[DP];
    const float4* xr = reinterpret_cast<const float4*>(X + ((long long)z * n + (valid ? i : 0)) * DP);
#pragma unroll
    for (int k4 = 0; k4 < DP / 4; ++k4) {
        float4 v = valid ? xr[k4] : make_float4(0.f, 0.f, 0.f, 0.f);
        x[4 * k4] = v.x; x[4 * k4 + 1] = v.y; x[4 * k4 + 2] = v.z; x[4 * k4 + 3] = v.w;
    }
    float xx = 0.f;
#pragma unroll
    for (int k = 0; k < DP; ++k) xx = fmaf(x[k], x[k], xx);

    float best = FLT_MAX;
    int bi = 0;
    const float* Cz = C + (long long)z * G * DP;
    for (int c0 = 0; c0 < G; c0 += kAssignCent) {
        const int cnt = min(kAssignCent, G - c0);
        __syncthreads();
        for (int t = threadIdx.x; t < cnt * DP; t += kAssignRows) sC[t] = Cz[(long long)c0 * DP + t];
        __syncthreads();
        for (int t = threadIdx.x; t < cnt; t += kAssignRows) {
            float s = 0.f;
            for (int k = 0; k < DP; ++k) s = fmaf(sC[t * DP + k], sC[t * DP + k], s);
            sN[t] = s;
        }
        __syncthreads();
        for (int j = 0; j < cnt; ++j) {
            const float4* cj = reinterpret_cast<const float4*>(sC + j * DP);
            float d0 = 0.f, d1 = 0.f;
#pragma unroll
            for (int k4 = 0; k4 < DP / 4; k4 += 2) {
                float4 c = cj[k4];
                d0 = fmaf(x[4 * k4], c.x, d0); d0 = fmaf(x[4 * k4 + 1], c.y, d0);
                d0 = fmaf(x[4 * k4 + 2], c.z, d0); d0 = fmaf(x[4 * k4 + 3], c.w, d0);
                if (k4 + 1 < DP / 4) {
                    float4 e = cj[k4 + 1];
                    d1 = fmaf(x[4 * k4 + 4], e.x, d1); d1 = fmaf(x[4 * k4 + 5], e.y, d1);
                    d1 = fmaf(x[4 * k4 + 6], e.z, d1); d1 = fmaf(x[4 * k4 + 7], e.w, d1);
                }
            }
            float dd = sN[j] - 2.f * (d0 + d1);
            if (dd < best) { best = dd; bi = c0 + j; }
        }
    }
    int moved = 0;
    if (valid) {
        long long o = (long long)z * n + i;
        if (!first && labels[o] != bi) moved = 1;
        labels[o] = bi;
        dist[o] = fmaxf(xx + best, 0.f);
    }
    unsigned b = __ballot_sync(kFull, moved);
    if ((threadIdx.x & 31) == 0 && b) atomicAdd(&changed[z], __popc(b));
}

// New centroid = mean of its members in fp64, stored fp32; an empty group keeps its centroid.
// One block per group: the group's row indices (perm order) are staged in shared memory, then
// thread t reads feature quad t % (DP/4) (a float4) of the rows at positions slice,
// slice + nslices, ... of the group, eight rows in flight (no index load in the dependence
// chain); the slices are summed in a fixed order, so the result does not depend on scheduling.
constexpr int kUpdThreads = 256;
constexpr int kUpdIdx = 2048;       // row indices staged per round
template <int DP>
__global__ void __launch_bounds__(kUpdThreads) km_update_kernel(const float* __restrict__ X,
                                                                const int32_t* __restrict__ perm,
                                                                const int32_t* __restrict__ off, float* C,
                                                                const int* done, int n, int G) {
    constexpr int kQ = DP / 4;                       // float4 quads per row
    constexpr int kSl = kUpdThreads / kQ;            // row slices
    constexpr int kU = 8;                            // rows in flight per slice
    const int z = blockIdx.y, g = blockIdx.x;
    if (done && done[z]) return;
    const int lo = off[(long long)z * (G + 1) + g], hi = off[(long long)z * (G + 1) + g + 1];
    if (hi <= lo) return;
    const int q = threadIdx.x % kQ, rs = threadIdx.x / kQ;
    __shared__ double red[kSl][DP];
    __shared__ int sIdx[kUpdIdx];
    const int32_t* pz = perm + (long long)z * n;
    const float4* xz = reinterpret_cast<const float4*>(X + (long long)z * n * DP) + q;
    double a[4][4] = {};
    for (int base = lo; base < hi; base += kUpdIdx) {
        const int cnt = min(kUpdIdx, hi - base);
        __syncthreads();
        for (int t = threadIdx.x; t < cnt; t += kUpdThreads) sIdx[t] = __ldg(pz + base + t);
        __syncthreads();
        if (rs < kSl) {
            int j = rs;
            for (; j + (kU - 1) * kSl < cnt; j += kU * kSl) {
                float4 v[kU];
#pragma unroll
                for (int u = 0; u < kU; ++u) v[u] = __ldg(xz + (long long)sIdx[j + u * kSl] * kQ);
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    a[u & 3][0] += (double)v[u].x; a[u & 3][1] += (double)v[u].y;
                    a[u & 3][2] += (double)v[u].z; a[u & 3][3] += (double)v[u].w;
                }
            }
            for (; j < cnt; j += kSl) {
                const float4 v = __ldg(xz + (long long)sIdx[j] * kQ);
                a[0][0] += (double)v.x; a[0][1] += (double)v.y; a[0][2] += (double)v.z; a[0][3] += (double)v.w;
            }
        }
    }
    if (rs < kSl) {
#pragma unroll
        for (int e = 0; e < 4; ++e) red[rs][4 * q + e] = (a[0][e] + a[1][e]) + (a[2][e] + a[3][e]);
    }
    __syncthreads();
    if (threadIdx.x < DP) {
        double t = 0.0;
#pragma unroll 4
        for (int k = 0; k < kSl; ++k) t += red[k][threadIdx.x];
        C[((long long)z * G + g) * DP + threadIdx.x] = (float)(t / (double)(hi - lo));
    }
}

__global__ void km_check_kernel(int* changed, int* done, int P) {
    for (int z = threadIdx.x; z < P; z += blockDim.x) {
        if (changed[z] == 0) done[z] = 1;
        changed[z] = 0;
    }
}

__global__ void km_reset_kernel(int* changed, int* done, int P) {
    for (int z = threadIdx.x; z < P; z += blockDim.x) { changed[z] = 0; done[z] = 0; }
}

__global__ void sort_hist_kernel(const int32_t* __restrict__ labels, int* counts, const int* done,
                                 int n, int G, int nch) {
    const int z = blockIdx.y, ch = blockIdx.x;
    if (done && done[z]) return;
    extern __shared__ int sh[];
    for (int t = threadIdx.x; t < G; t += blockDim.x) sh[t] = 0;
    __syncthreads();
    for (int k = 0; k < kSortChunk / kSortSub; ++k) {
        const int i = ch * kSortChunk + k * kSortSub + threadIdx.x;
        if (i < n) atomicAdd(&sh[labels[(long long)z * n + i]], 1);
    }
    __syncthreads();
    for (int t = threadIdx.x; t < G; t += blockDim.x) counts[((long long)z * nch + ch) * G + t] = sh[t];
}

// bases[z][ch][g] = rows of group g in chunks < ch; off[z][g] = exclusive scan of group sizes.
__global__ void __launch_bounds__(1024) sort_scan_kernel(const int* __restrict__ counts, int* bases, int32_t* off,
                                 const int* done, int G, int nch) {
    const int z = blockIdx.x;
    if (done && done[z]) return;
    extern __shared__ int tot[];
    __shared__ int wsum[32];
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        int s = 0;
        const int* cz = counts + (long long)z * nch * G + g;
        int* bz = bases + (long long)z * nch * G + g;
        for (int ch0 = 0; ch0 < nch; ch0 += 8) {
            int v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = ch0 + e < nch ? cz[(long long)(ch0 + e) * G] : 0;   // 8 loads in flight
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (ch0 + e < nch) { bz[(long long)(ch0 + e) * G] = s; s += v[e]; }
        }
        tot[g] = s;
    }
    __syncthreads();
    // exclusive scan of the group totals (G <= blockDim.x): warp scans, then the warp totals
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int v = t < G ? tot[t] : 0;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(kFull, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) wsum[w] = inc;
    __syncthreads();
    if (w == 0) {
        const int nw = (blockDim.x + 31) >> 5;
        int x = lane < nw ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(kFull, x, o);
            if (lane >= o) x += n;
        }
        wsum[lane] = x;   // inclusive scan of warp totals
    }
    __syncthreads();
    const int base = w > 0 ? wsum[w - 1] : 0;
    if (t < G) off[(long long)z * (G + 1) + t] = base + inc - v;
    if (t == G - 1) off[(long long)z * (G + 1) + G] = base + inc;
}

// Stable scatter: position = off[g] + rows of g in earlier chunks + earlier sub-chunks of this
// chunk + earlier warps of this sub-chunk + earlier lanes of this warp.
__global__ void sort_scatter_kernel(const int32_t* __restrict__ labels, const int* __restrict__ bases,
                                    const int32_t* __restrict__ off, int32_t* perm, const int* done,
                                    int n, int G, int nch) {
    const int z = blockIdx.y, ch = blockIdx.x;
    if (done && done[z]) return;
    extern __shared__ int wc[];  // [8][G] per-warp counts, then [G] running counts
    int* run = wc + 8 * G;
    for (int t = threadIdx.x; t < 9 * G; t += blockDim.x) wc[t] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int k = 0; k < kSortChunk / kSortSub; ++k) {
        const int i = ch * kSortChunk + k * kSortSub + threadIdx.x;
        const bool valid = i < n;
        const int lab = valid ? labels[(long long)z * n + i] : -1;
        const unsigned m = __match_any_sync(kFull, lab);
        const int rank = __popc(m & ((1u << lane) - 1u));
        if (valid && rank == 0) wc[w * G + lab] = __popc(m);
        __syncthreads();
        if (valid) {
            int pre = run[lab];
            for (int w2 = 0; w2 < w; ++w2) pre += wc[w2 * G + lab];
            const int pos = off[(long long)z * (G + 1) + lab] + bases[((long long)z * nch + ch) * G + lab] + pre + rank;
            perm[(long long)z * n + pos] = i;
        }
        __syncthreads();
        for (int g = threadIdx.x; g < G; g += blockDim.x) {
            int add = 0;
            for (int w2 = 0; w2 < 8; ++w2) { add += wc[w2 * G + g]; wc[w2 * G + g] = 0; }
            run[g] += add;
        }
        __syncthreads();
    }
}

// Group means of bf16 rows (d columns x 4 fixed row slices); empty group -> 0.
__global__ void group_mean_bf16_kernel(const bf16* __restrict__ Y, const int32_t* __restrict__ perm,
                                       const int32_t* __restrict__ off, float* cent, bf16* chi,
                                       bf16* clo, int n, int G, int d) {
    const int z = blockIdx.y, g = blockIdx.x;
    const int lo = off[(long long)z * (G + 1) + g], hi = off[(long long)z * (G + 1) + g + 1];
    const int c = threadIdx.x % d, rs = threadIdx.x / d;
    float acc = 0.f;
    for (int j = lo + rs; j < hi; j += 4)
        acc += __bfloat162float(Y[((long long)z * n + perm[(long long)z * n + j]) * d + c]);
    __shared__ float red[4][128];
    red[rs][c] = acc;
    __syncthreads();
    if (rs == 0) {
        float mean = hi > lo ? ((red[0][c] + red[1][c]) + (red[2][c] + red[3][c])) / (float)(hi - lo) : 0.f;
        long long o = ((long long)z * G + g) * d + c;
        cent[o] = mean;
        if (chi) {
            bf16 h = __float2bfloat16_rn(mean);
            chi[o] = h;
            clo[o] = __float2bfloat16_rn(mean - __bfloat162float(h));
        }
    }
}

__global__ void split_bf16_kernel(const float* x, bf16* hi, bf16* lo, long long count) {
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= count) return;
    float v = x[i];
    bf16 h = __float2bfloat16_rn(v);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
}

// dst[z][i][c] = (1/g) sum_j src[z * g + j][i][c] in fp32 (g = 1: the rows widened to fp32).
__global__ void mean_heads_f32_kernel(const bf16* __restrict__ src, float* dst, int g, long long per_head) {
    const int z = blockIdx.y;
    const float inv = 1.f / (float)g;
    for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < per_head;
         t += (long long)gridDim.x * blockDim.x) {
        float a = 0.f;
        for (int j = 0; j < g; ++j) a += __bfloat162float(src[((long long)z * g + j) * per_head + t]);
        dst[(long long)z * per_head + t] = g == 1 ? a : a * inv;
    }
}

}  // namespace

cudaError_t launch_mean_heads_f32(const bf16* src, float* dst, int P, int g, int N, int d, cudaStream_t s) {
    const long long per_head = (long long)N * d;
    long long blocks = (per_head + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    mean_heads_f32_kernel<<<dim3((unsigned)blocks, P), 256, 0, s>>>(src, dst, g, per_head);
    return cudaGetLastError();
}

cudaError_t launch_km_seed(const float* X, float* C, int P, int n, int G, int DP, cudaStream_t s) {
    km_seed_kernel<<<P, 256, 0, s>>>(X, C, n, G, DP);
    return cudaGetLastError();
}

cudaError_t launch_km_assign(const float* X, const float* C, int32_t* labels, float* dist,
                             int* changed, const int* done, int P, int n, int G, int DP, bool first,
                             cudaStream_t s) {
    dim3 grid((n + kAssignRows - 1) / kAssignRows, P);
    switch (DP) {
        case 16: km_assign_kernel<16><<<grid, kAssignRows, 0, s>>>(X, C, labels, dist, changed, done, n, G, first); break;
        case 32: km_assign_kernel<32><<<grid, kAssignRows, 0, s>>>(X, C, labels, dist, changed, done, n, G, first); break;
        case 48: km_assign_kernel<48><<<grid, kAssignRows, 0, s>>>(X, C, labels, dist, changed, done, n, G, first); break;
        case 64: km_assign_kernel<64><<<grid, kAssignRows, 0, s>>>(X, C, labels, dist, changed, done, n, G, first); break;
        case 128: km_assign_kernel<128><<<grid, kAssignRows, 0, s>>>(X, C, labels, dist, changed, done, n, G, first); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_km_update(const float* X, const int32_t* perm, const int32_t* off, float* C,
                             const int* done, int P, int n, int G, int DP, cudaStream_t s) {
    const dim3 grid(G, P);
    switch (DP) {
        case 16: km_update_kernel<16><<<grid, kUpdThreads, 0, s>>>(X, perm, off, C, done, n, G); break;
        case 32: km_update_kernel<32><<<grid, kUpdThreads, 0, s>>>(X, perm, off, C, done, n, G); break;
        case 48: km_update_kernel<48><<<grid, kUpdThreads, 0, s>>>(X, perm, off, C, done, n, G); break;
        case 64: km_update_kernel<64><<<grid, kUpdThreads, 0, s>>>(X, perm, off, C, done, n, G); break;
        case 128: km_update_kernel<128><<<grid, kUpdThreads, 0, s>>>(X, perm, off, C, done, n, G); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_km_check(int* changed, int* done, int P, cudaStream_t s) {
    km_check_kernel<<<1, 1024, 0, s>>>(changed, done, P);
    return cudaGetLastError();
}

cudaError_t launch_km_reset(int* changed, int* done, int P, cudaStream_t s) {
    km_reset_kernel<<<1, 1024, 0, s>>>(changed, done, P);
    return cudaGetLastError();
}

cudaError_t launch_group_sort(const int32_t* labels, int32_t* perm, int32_t* off, int* counts,
                              int* bases, const int* done, int P, int n, int G, cudaStream_t s) {
    const int nch = (n + kSortChunk - 1) / kSortChunk;
    dim3 grid(nch, P);
    sort_hist_kernel<<<grid, kSortSub, G * sizeof(int), s>>>(labels, counts, done, n, G, nch);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    sort_scan_kernel<<<P, 1024, G * sizeof(int), s>>>(counts, bases, off, done, G, nch);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    sort_scatter_kernel<<<grid, kSortSub, 9 * G * sizeof(int), s>>>(labels, bases, off, perm, done, n, G, nch);
    return cudaGetLastError();
}

cudaError_t launch_group_mean_bf16(const bf16* Y, const int32_t* perm, const int32_t* off,
                                   float* cent, bf16* chi, bf16* clo, int P, int n, int G, int d,
                                   cudaStream_t s) {
    group_mean_bf16_kernel<<<dim3(G, P), 4 * d, 0, s>>>(Y, perm, off, cent, chi, clo, n, G, d);
    return cudaGetLastError();
}

cudaError_t launch_split_bf16(const float* x, bf16* hi, bf16* lo, long long count, cudaStream_t s) {
    if (count <= 0) return cudaSuccess;
    split_bf16_kernel<<<(unsigned)((count + 255) / 256), 256, 0, s>>>(x, hi, lo, count);
    return cudaGetLastError();
}

}  // namespace spr
