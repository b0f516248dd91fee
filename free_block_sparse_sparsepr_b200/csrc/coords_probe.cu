// Sampled query rows, query coordinates against the key-group centroids, and
// the stratified radial probe rows with their group-coverage weights.
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace spr {
namespace {

// Qs[z][s] = Q[b][h*g + s%g][floor((s+1/2)N/S)] (bf16 rows), zero rows for S <= s < DP.
__global__ void gather_samples_kernel(const bf16* __restrict__ Q, bf16* Qs, int Hq, int Hkv, int N,
                                      int d, int S, int DP) {
    const int z = blockIdx.x, b = z / Hkv, h = z % Hkv, g = Hq / Hkv;
    const int vpr = d / 8;  // 16-byte vectors per row
    for (int t = threadIdx.x; t < DP * vpr; t += blockDim.x) {
        int sidx = t / vpr, c = t % vpr;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (sidx < S) {
            long long row = sample_pos(sidx, N, S);
            int head = h * g + sidx % g;
            v = reinterpret_cast<const uint4*>(Q + (((long long)b * Hq + head) * N + row) * d)[c];
        }
        reinterpret_cast<uint4*>(Qs + ((long long)z * DP + sidx) * d)[c] = v;
    }
}

// One warp per query row of a KV head: mean of the g heads' logits, centred over the groups.
// VEC (Gk % 8 == 0): lane l owns the 8 consecutive columns 256*b + 8*l .. +7 of each block b of
// 256 columns, read as two float4 and written as one 16-byte bf16 vector per part; otherwise
// lane l owns the strided columns l + 32*t.
template <bool VEC>
__global__ void coords_center_kernel(const float* __restrict__ u, bf16* uhi, bf16* ulo, float* y,
                                     int g, int N, int Gk, int Gkp, int DPy, int proj) {
    const int z = blockIdx.y;
    const int lane = threadIdx.x & 31;
    const int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (i >= N) return;
    auto col = [&](int t) { return VEC ? (t >> 3) * 256 + lane * 8 + (t & 7) : lane + 32 * t; };
    const float invg = 1.f / (float)g;
    float v[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) v[t] = 0.f;
    for (int j = 0; j < g; ++j) {
        const float* ur = u + (((long long)z * g + j) * N + i) * Gk;
        if (VEC) {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int c0 = b * 256 + lane * 8;
                if (c0 < Gk) {
                    const float4 a0 = *reinterpret_cast<const float4*>(ur + c0);
                    const float4 a1 = *reinterpret_cast<const float4*>(ur + c0 + 4);
                    v[8 * b + 0] += a0.x; v[8 * b + 1] += a0.y; v[8 * b + 2] += a0.z; v[8 * b + 3] += a0.w;
                    v[8 * b + 4] += a1.x; v[8 * b + 5] += a1.y; v[8 * b + 6] += a1.z; v[8 * b + 7] += a1.w;
                }
            }
        } else {
#pragma unroll
            for (int t = 0; t < 32; ++t) {             // 32 independent loads in flight per head
                const int gk = col(t);
                if (gk < Gk) v[t] += ur[gk];
            }
        }
    }
    float s = 0.f;
#pragma unroll
    for (int t = 0; t < 32; ++t) {
        v[t] *= invg;
        s += v[t];
    }
    const float mean = warp_sum(s) / (float)Gk;
    float ss = 0.f;
#pragma unroll
    for (int t = 0; t < 32; ++t) {
        const int gk = col(t);
        v[t] = gk < Gk ? v[t] - mean : 0.f;
        ss = fmaf(v[t], v[t], ss);
    }
    if (proj) {
        bf16* hr = uhi + ((long long)z * N + i) * Gkp;
        bf16* lr = ulo + ((long long)z * N + i) * Gkp;
        if (VEC) {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int c0 = b * 256 + lane * 8;
                if (c0 < Gkp) {
                    uint32_t wh[4], wl[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float a = v[8 * b + 2 * e], c = v[8 * b + 2 * e + 1];
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(a, c);
                        const float2 hf = __bfloat1622float2(h2);
                        __nv_bfloat162 l2 = __floats2bfloat162_rn(a - hf.x, c - hf.y);
                        wh[e] = *reinterpret_cast<uint32_t*>(&h2);
                        wl[e] = *reinterpret_cast<uint32_t*>(&l2);
                    }
                    *reinterpret_cast<uint4*>(hr + c0) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
                    *reinterpret_cast<uint4*>(lr + c0) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
                }
            }
        } else {
#pragma unroll
            for (int t = 0; t < 32; ++t) {
                const int gk = col(t);
                if (gk < Gkp) {
                    bf16 hh = __float2bfloat16_rn(v[t]);
                    hr[gk] = hh;
                    lr[gk] = __float2bfloat16_rn(v[t] - __bfloat162float(hh));
                }
            }
        }
    } else {
        const float nrm = sqrtf(warp_sum(ss));
        float* yr = y + ((long long)z * N + i) * DPy;
#pragma unroll
        for (int t = 0; t < 32; ++t) {
            const int gk = col(t);
            if (gk < DPy) yr[gk] = (gk < Gk && nrm > 0.f) ? v[t] / nrm : 0.f;
        }
    }
}

// One warp per row: y / ||y|| (zero rows stay zero), DP <= 64.
__global__ void rows_normalize_kernel(float* y, long long rows, int DP) {
    const long long i = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (i >= rows) return;
    float* r = y + i * DP;
    const float a = lane < DP ? r[lane] : 0.f;
    const float b = lane + 32 < DP ? r[lane + 32] : 0.f;
    const float nrm = sqrtf(warp_sum(fmaf(a, a, b * b)));
    if (lane < DP) r[lane] = nrm > 0.f ? a / nrm : 0.f;
    if (lane + 32 < DP) r[lane + 32] = nrm > 0.f ? b / nrm : 0.f;
}

__global__ void make_projection_kernel(bf16* projT, int Gk, int Gkp, int rQ, int DPy,
                                       unsigned long long seed) {
    long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (long long)DPy * Gkp) return;
    int row = (int)(t / Gkp), gk = (int)(t % Gkp);
    float v = 0.f;
    if (row < rQ && gk < Gk) {
        unsigned long long bit = splitmix64(seed ^ (unsigned long long)((long long)gk * rQ + row)) & 1ull;
        v = bit ? -1.f : 1.f;
    }
    projT[t] = __float2bfloat16_rn(v);
}

// Probe m of a KV head: position p = floor((m+1/2)N/M) of the sequence ordered by
// (group, radial distance, original index). Inside the group the keys (radial bits, position)
// are sorted in shared memory (bitonic; radial distances are >= 0, so their bits order
// like the values) when the group fits, else ranked by counting.
constexpr int kProbeSmem = 4096;
__global__ void __launch_bounds__(256) probe_select_kernel(const int32_t* __restrict__ qperm,
                                                           const int32_t* __restrict__ qoff,
                                                           const float* __restrict__ radial,
                                                           int32_t* probe, int32_t* probe_pos,
                                                           int32_t* probe_seq, int N, int Gq, int M) {
    const int z = blockIdx.y, m = blockIdx.x;
    const int32_t* off = qoff + (long long)z * (Gq + 1);
    const long long p = sample_pos(m, N, M);
    const int a = upper_index(off, Gq, p);
    const int lo = off[a], cnt = off[a + 1] - lo;
    const int k = (int)(p - lo);
    __shared__ unsigned long long key[kProbeSmem];
    const int32_t* perm = qperm + (long long)z * N + lo;
    const float* rad = radial + (long long)z * N;
    if (cnt <= kProbeSmem) {
        int len = 1;
        while (len < cnt) len <<= 1;
        for (int j = threadIdx.x; j < len; j += blockDim.x) {
            // the position j breaks ties: inside a group positions follow the original index
            key[j] = j < cnt ? ((unsigned long long)__float_as_uint(rad[perm[j]]) << 32) | (unsigned)j : ~0ull;
        }
        __syncthreads();
        for (int kk = 2; kk <= len; kk <<= 1)
            for (int jj = kk >> 1; jj > 0; jj >>= 1) {
                for (int t = threadIdx.x; t < len; t += blockDim.x) {
                    const int u = t ^ jj;
                    if (u > t) {
                        const unsigned long long x = key[t], y = key[u];
                        if ((x > y) == ((t & kk) == 0)) { key[t] = y; key[u] = x; }
                    }
                }
                __syncthreads();
            }
        if (threadIdx.x == 0) {
            const int j = (int)(key[k] & 0xffffffffull);
            probe[(long long)z * M + m] = perm[j];
            probe_pos[(long long)z * M + m] = lo + j;
            probe_seq[(long long)z * M + m] = (int)p;
        }
        return;
    }
    for (int j = threadIdx.x; j < cnt; j += blockDim.x) {
        const int ij = perm[j];
        const float rj = rad[ij];
        int rank = 0;
        for (int e = 0; e < cnt; ++e) {
            const int ie = perm[e];
            const float re = rad[ie];
            rank += (re < rj || (re == rj && ie < ij)) ? 1 : 0;
        }
        if (rank == k) {
            probe[(long long)z * M + m] = ij;
            probe_pos[(long long)z * M + m] = lo + j;
            probe_seq[(long long)z * M + m] = (int)p;
        }
    }
}

// Probe-sampling ablations of [probe]: the rows of a uniform grid over the original token order
// (floor((m + 1/2) N / M)), or M distinct rows from the SplitMix64 stream of state
// seed ^ 0x70726F6265 (output i = splitmix64(state + i * 0x9E3779B97F4A7C15), taken mod N,
// repeats skipped). Each row's group-major position is found in its group's slice of qperm, and
// the probes are stored in ascending position (that position also drives the coverage weights).
constexpr unsigned long long kProbeSalt = 0x70726F6265ull;
constexpr int kMaxProbeRows = 64;
__global__ void __launch_bounds__(kMaxProbeRows) probe_alt_kernel(const int32_t* __restrict__ qperm,
                                                                  const int32_t* __restrict__ qoff,
                                                                  const int32_t* __restrict__ qgroup,
                                                                  int32_t* probe, int32_t* probe_pos,
                                                                  int32_t* probe_seq, int N, int Gq, int M,
                                                                  int random, unsigned long long seed, int* status) {
    const int z = blockIdx.x, m = threadIdx.x;
    __shared__ int rows[kMaxProbeRows];
    __shared__ int pos[kMaxProbeRows];
    if (random) {
        if (m == 0) {
            const unsigned long long st = seed ^ kProbeSalt;
            int got = 0;
            // the stream repeats a row rarely; the bound only guards against M close to N
            const long long cap = 64ll * N + 4096;
            for (long long i = 0; got < M && i < cap; ++i) {
                const int c = (int)(splitmix64(st + (unsigned long long)i * 0x9E3779B97F4A7C15ull) %
                                    (unsigned long long)N);
                bool dup = false;
                for (int e = 0; e < got; ++e) dup |= rows[e] == c;
                if (!dup) rows[got++] = c;
            }
            for (; got < M; ++got) {            // only past the bound: flag it and fill distinct rows
                set_status(status, kDevBounds);
                rows[got] = got;
            }
        }
    } else if (m < M) {
        rows[m] = (int)sample_pos(m, N, M);
    }
    __syncthreads();
    int r = 0, p = 0;
    if (m < M) {
        r = rows[m];
        const int a = qgroup[(long long)z * N + r];
        const int lo = qoff[(long long)z * (Gq + 1) + a], hi = qoff[(long long)z * (Gq + 1) + a + 1];
        const int32_t* pz = qperm + (long long)z * N;
        p = lo;
        for (int j = lo; j < hi; ++j)
            if (pz[j] == r) { p = j; break; }
        pos[m] = p;
    }
    __syncthreads();
    if (m < M) {
        int rank = 0;
        for (int e = 0; e < M; ++e) rank += pos[e] < p ? 1 : 0;
        probe[(long long)z * M + rank] = r;
        probe_pos[(long long)z * M + rank] = p;
        probe_seq[(long long)z * M + rank] = p;
    }
}

// Coverage weight of probe m: its group's size split over the group's probes, plus the
// sizes of probe-less groups whose nearest probe (sequence distance, ties -> lower m) is m.
__global__ void probe_weights_kernel(const int32_t* __restrict__ qoff,
                                     const int32_t* __restrict__ probe_seq, float* w, int N,
                                     int Gq, int M, int uniform) {
    const int z = blockIdx.x;
    const int32_t* off = qoff + (long long)z * (Gq + 1);
    const int32_t* ps = probe_seq + (long long)z * M;
    for (int m = threadIdx.x; m < M; m += blockDim.x) {
        if (uniform) { w[(long long)z * M + m] = 1.f; continue; }
        const int pm = ps[m];
        const int am = upper_index(off, Gq, pm);
        const int lo = off[am], hi = off[am + 1];
        int count = 0;
        for (int t = 0; t < M; ++t) count += (ps[t] >= lo && ps[t] < hi) ? 1 : 0;
        float raw = (float)(hi - lo) / (float)count;
        // probe-less groups before a_m (after the previous probe's group)
        const int abeg = m > 0 ? upper_index(off, Gq, ps[m - 1]) + 1 : 0;
        for (int a = abeg; a < am; ++a) {
            const int glo = off[a], ghi = off[a + 1];
            if (ghi <= glo) continue;
            const long long dm = (long long)pm - (ghi - 1);
            const long long dprev = m > 0 ? (long long)glo - ps[m - 1] : LLONG_MAX;
            if (dm < dprev) raw += (float)(ghi - glo);
        }
        // probe-less groups after a_m (before the next probe's group)
        const int aend = m + 1 < M ? upper_index(off, Gq, ps[m + 1]) : Gq;
        for (int a = am + 1; a < aend; ++a) {
            const int glo = off[a], ghi = off[a + 1];
            if (ghi <= glo) continue;
            const long long dm = (long long)glo - pm;
            const long long dnext = m + 1 < M ? (long long)ps[m + 1] - (ghi - 1) : LLONG_MAX;
            if (dm <= dnext) raw += (float)(ghi - glo);
        }
        w[(long long)z * M + m] = raw * (float)M / (float)N;
    }
}

}  // namespace

cudaError_t launch_gather_samples(const bf16* Q, bf16* Qs, int B, int Hq, int Hkv, int N, int d,
                                  int S, int DP, cudaStream_t s) {
    gather_samples_kernel<<<B * Hkv, 256, 0, s>>>(Q, Qs, Hq, Hkv, N, d, S, DP);
    return cudaGetLastError();
}

cudaError_t launch_coords_center(const float* u, bf16* uhi, bf16* ulo, float* y, int P, int g,
                                 int N, int Gk, int Gkp, int DPy, bool proj, cudaStream_t s) {
    dim3 grid((N + 7) / 8, P);
    if (Gk % 8 == 0 && Gkp % 8 == 0)
        coords_center_kernel<true><<<grid, 256, 0, s>>>(u, uhi, ulo, y, g, N, Gk, Gkp, DPy, proj ? 1 : 0);
    else
        coords_center_kernel<false><<<grid, 256, 0, s>>>(u, uhi, ulo, y, g, N, Gk, Gkp, DPy, proj ? 1 : 0);
    return cudaGetLastError();
}

cudaError_t launch_rows_normalize(float* y, int rows, int DP, cudaStream_t s) {
    rows_normalize_kernel<<<(unsigned)(((long long)rows + 7) / 8), 256, 0, s>>>(y, rows, DP);
    return cudaGetLastError();
}

cudaError_t launch_make_projection(bf16* projT, int Gk, int Gkp, int rQ, int DPy,
                                   unsigned long long seed, cudaStream_t s) {
    long long tot = (long long)DPy * Gkp;
    make_projection_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, s>>>(projT, Gk, Gkp, rQ, DPy, seed);
    return cudaGetLastError();
}

cudaError_t launch_probe_select(const int32_t* qperm, const int32_t* qoff, const float* radial,
                                int32_t* probe, int32_t* probe_pos, int32_t* probe_seq, int P,
                                int N, int Gq, int M, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    probe_select_kernel<<<dim3(M, P), 256, 0, s>>>(qperm, qoff, radial, probe, probe_pos, probe_seq, N, Gq, M);
    return cudaGetLastError();
}

cudaError_t launch_probe_alt(const int32_t* qperm, const int32_t* qoff, const int32_t* qgroup, int32_t* probe,
                             int32_t* probe_pos, int32_t* probe_seq, int P, int N, int Gq, int M, bool random,
                             unsigned long long seed, int* status, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    if (M > kMaxProbeRows || M > N) return cudaErrorInvalidValue;
    probe_alt_kernel<<<P, kMaxProbeRows, 0, s>>>(qperm, qoff, qgroup, probe, probe_pos, probe_seq, N, Gq, M,
                                                 random ? 1 : 0, seed, status);
    return cudaGetLastError();
}

cudaError_t launch_probe_weights(const int32_t* qoff, const int32_t* probe_seq, float* w, int P,
                                 int N, int Gq, int M, bool uniform, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    probe_weights_kernel<<<P, 128, 0, s>>>(qoff, probe_seq, w, N, Gq, M, uniform ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace spr
