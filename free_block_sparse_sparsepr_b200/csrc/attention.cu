// Exact softmax attention on tensor cores (bf16 mma.sync, fp32 accumulate,
// online softmax): the block-sparse pass over each query group's kept key
// groups (renormalised over those keys only), the dense baseline, and the
// split-key dense pass of the probe rows.
#include <float.h>
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"

namespace spr {
namespace {

constexpr int kBM = 64;   // query rows per CTA (16 per warp)
constexpr int kBN = 64;   // keys per tile
constexpr float kLn2 = 0.6931471805599453f;
enum { kSparse = 0, kDense = 1, kProbe = 2 };

struct AttnParams {
    const bf16* Q; const bf16* K; const bf16* V;
    bf16* O; float* lse;
    float* Opart; float* mpart; float* lpart;
    const int32_t* qoff; const int32_t* koff; const int32_t* tile_off;
    const int32_t* rowptr; const int32_t* kg; const int32_t* qidx;
    int N, g, Gq, Gk, M, ns, chunk, mt;
    float scale_log2;
};

// Merged runs of consecutive kept key groups (adjacent in group-major order).
struct KeyRanges {
    const int32_t* kept;
    const int32_t* ko;
    int ri, r1;
    __device__ __forceinline__ bool next(int& lo, int& hi) {
        while (ri < r1) {
            const int g0 = kept[ri++];
            lo = ko[g0];
            hi = ko[g0 + 1];
            while (ri < r1 && ko[kept[ri]] == hi) { hi = ko[kept[ri] + 1]; ++ri; }
            if (hi > lo) return true;
        }
        return false;
    }
};

template <int D>
constexpr int attn_smem_bytes() { return (kBM + 4 * kBN) * (D + 8) * 2; }

template <int D, int MODE>
__global__ void __launch_bounds__(128) attn_kernel(const AttnParams p) {
    constexpr int LD = D + 8;
    constexpr int VPR = D / 8;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    bf16* sQ = reinterpret_cast<bf16*>(smem_raw);
    bf16* sK = sQ + kBM * LD;
    bf16* sV = sK + 2 * kBN * LD;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int x = blockIdx.y, z = x / p.g;
    const bf16* Qh = p.Q + (long long)x * p.N * D;
    const bf16* Kh = p.K + (long long)z * p.N * D;
    const bf16* Vh = p.V + (long long)z * p.N * D;

    int qlo = 0, qn = 0, chunk_id = 0, m0 = 0;
    int cur_lo = 0, cur_hi = 0;
    bool have = false;
    KeyRanges rg;
    rg.kept = nullptr; rg.ko = nullptr; rg.ri = 0; rg.r1 = 0;
    if (MODE == kSparse) {
        const int32_t* toff = p.tile_off + (long long)z * (p.Gq + 1);
        const int tile = blockIdx.x;
        if (tile >= toff[p.Gq]) return;
        const int a = upper_index(toff, p.Gq, tile);
        const int32_t* qo = p.qoff + (long long)z * (p.Gq + 1);
        qlo = qo[a] + (tile - toff[a]) * kBM;
        qn = min(kBM, qo[a + 1] - qlo);
        rg.kept = p.kg + (long long)z * p.Gq * p.Gk;
        rg.ko = p.koff + (long long)z * (p.Gk + 1);
        rg.ri = p.rowptr[(long long)z * (p.Gq + 1) + a];
        rg.r1 = p.rowptr[(long long)z * (p.Gq + 1) + a + 1];
        have = rg.next(cur_lo, cur_hi);
    } else if (MODE == kDense) {
        qlo = blockIdx.x * kBM;
        if (qlo >= p.N) return;
        qn = min(kBM, p.N - qlo);
        cur_lo = 0;
        cur_hi = p.N;
        have = true;
    } else {
        chunk_id = blockIdx.x / p.mt;
        m0 = (blockIdx.x % p.mt) * kBM;
        qn = min(kBM, p.M - m0);
        cur_lo = chunk_id * p.chunk;
        cur_hi = min(p.N, cur_lo + p.chunk);
        have = cur_lo < cur_hi;
    }

    // Query tile (zero rows past the tile's end).
    for (int c = tid; c < kBM * VPR; c += 128) {
        const int r = c / VPR, v = c % VPR;
        bool valid = r < qn;
        long long row;
        if (MODE == kProbe) {
            // a row index outside [0, N) reads nothing: its query is zero-filled
            const int32_t ri = valid ? p.qidx[(long long)z * p.M + m0 + r] : 0;
            valid = valid && ri >= 0 && ri < p.N;
            row = valid ? ri : 0;
        } else {
            row = valid ? qlo + r : 0;
        }
        cp_async16(sQ + r * LD + v * 8, Qh + row * D + v * 8, valid);
    }
    cp_async_commit();

    auto load_kv = [&](int stage, int t0) {
        bf16* dk = sK + stage * kBN * LD;
        bf16* dv = sV + stage * kBN * LD;
        for (int c = tid; c < kBN * VPR; c += 128) {
            const int r = c / VPR, v = c % VPR;
            const int row = t0 + r;
            const bool valid = row < p.N;
            const long long off = (long long)(valid ? row : 0) * D + v * 8;
            cp_async16(dk + r * LD + v * 8, Kh + off, valid);
            cp_async16(dv + r * LD + v * 8, Vh + off, valid);
        }
    };

    if (have) load_kv(0, cur_lo);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    uint32_t qf[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
        ldsm_x4(qf[kk], sQ + (warp * 16 + (lane & 15)) * LD + kk * 16 + (lane >> 4) * 8);

    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float mr0 = -INFINITY, mr1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    int stage = 0;

    while (have) {
        int n_lo = cur_lo, n_hi = cur_hi;
        bool nhave = false;
        if (cur_lo + kBN < cur_hi) { n_lo = cur_lo + kBN; nhave = true; }
        else if (MODE == kSparse) nhave = rg.next(n_lo, n_hi);
        if (nhave) load_kv(stage ^ 1, n_lo);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();

        const bf16* cK = sK + stage * kBN * LD;
        const bf16* cV = sV + stage * kBN * LD;
        float s[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t b[4];
                ldsm_x4(b, cK + (np * 16 + (lane & 7) + ((lane >> 4) << 3)) * LD + kk * 16 + ((lane >> 3) & 1) * 8);
                mma_bf16_16816(s[2 * np], qf[kk], b);
                mma_bf16_16816(s[2 * np + 1], qf[kk], b + 2);
            }
        }
        const int lim = cur_hi - cur_lo;
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int col = nt * 8 + 2 * (lane & 3) + (e & 1);
                const float v = col < lim ? s[nt][e] * p.scale_log2 : -INFINITY;
                s[nt][e] = v;
                if (e < 2) mx0 = fmaxf(mx0, v); else mx1 = fmaxf(mx1, v);
            }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, 2));
        const float mn0 = fmaxf(mr0, mx0), mn1 = fmaxf(mr1, mx1);
        const float sc0 = mn0 == -INFINITY ? 1.f : exp2f(mr0 - mn0);
        const float sc1 = mn1 == -INFINITY ? 1.f : exp2f(mr1 - mn1);
        const float sub0 = mn0 == -INFINITY ? 0.f : mn0;
        const float sub1 = mn1 == -INFINITY ? 0.f : mn1;
        float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            s[nt][0] = exp2f(s[nt][0] - sub0);
            s[nt][1] = exp2f(s[nt][1] - sub0);
            s[nt][2] = exp2f(s[nt][2] - sub1);
            s[nt][3] = exp2f(s[nt][3] - sub1);
            rs0 += s[nt][0] + s[nt][1];
            rs1 += s[nt][2] + s[nt][3];
        }
        l0 = l0 * sc0 + rs0;
        l1 = l1 * sc1 + rs1;
        mr0 = mn0;
        mr1 = mn1;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            o[i][0] *= sc0; o[i][1] *= sc0; o[i][2] *= sc1; o[i][3] *= sc1;
        }
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
            uint32_t a[4];
            a[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
            a[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
            a[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
            a[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
            for (int np = 0; np < D / 16; ++np) {
                uint32_t b[4];
                ldsm_x4_trans(b, cV + (kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * LD + np * 16 + (lane >> 4) * 8);
                mma_bf16_16816(o[2 * np], a, b);
                mma_bf16_16816(o[2 * np + 1], a, b + 2);
            }
        }
        __syncthreads();
        stage ^= 1;
        cur_lo = n_lo;
        cur_hi = n_hi;
        have = nhave;
    }

    l0 += __shfl_xor_sync(kFull, l0, 1);
    l0 += __shfl_xor_sync(kFull, l0, 2);
    l1 += __shfl_xor_sync(kFull, l1, 1);
    l1 += __shfl_xor_sync(kFull, l1, 2);
    const int rr[2] = {warp * 16 + (lane >> 2), warp * 16 + (lane >> 2) + 8};
    const float ls[2] = {l0, l1};
    const float ms[2] = {mr0, mr1};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int r = rr[h];
        if (r >= qn) continue;
        if (MODE != kProbe) {
            const float inv = ls[h] > 0.f ? 1.f / ls[h] : 0.f;
            bf16* orow = p.O + ((long long)x * p.N + qlo + r) * D;
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt)
                *reinterpret_cast<uint32_t*>(orow + nt * 8 + 2 * (lane & 3)) =
                    pack_bf16x2(o[nt][2 * h] * inv, o[nt][2 * h + 1] * inv);
            if (p.lse && (lane & 3) == 0)
                p.lse[(long long)x * p.N + qlo + r] = ls[h] > 0.f ? (ms[h] + log2f(ls[h])) * kLn2 : -INFINITY;
        } else {
            const long long base = ((long long)x * p.ns + chunk_id) * p.M + m0 + r;
            float* orow = p.Opart + base * D;
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt) {
                orow[nt * 8 + 2 * (lane & 3)] = o[nt][2 * h];
                orow[nt * 8 + 2 * (lane & 3) + 1] = o[nt][2 * h + 1];
            }
            if ((lane & 3) == 0) {
                p.mpart[base] = ms[h];
                p.lpart[base] = ls[h];
            }
        }
    }
}

__global__ void probe_combine_kernel(const float* __restrict__ Opart, const float* __restrict__ mpart,
                                     const float* __restrict__ lpart, float* Od, int M, int ns, int D) {
    const int x = blockIdx.y, m = blockIdx.x, c = threadIdx.x;
    float mx = -INFINITY;
    for (int k = 0; k < ns; ++k) mx = fmaxf(mx, mpart[((long long)x * ns + k) * M + m]);
    float L = 0.f, acc = 0.f;
    for (int k = 0; k < ns; ++k) {
        const long long b = ((long long)x * ns + k) * M + m;
        const float mk = mpart[b];
        const float w = mk == -INFINITY ? 0.f : exp2f(mk - mx);
        L += lpart[b] * w;
        acc += Opart[b * D + c] * w;
    }
    Od[((long long)x * M + m) * D + c] = L > 0.f ? acc / L : 0.f;
}

// Qpr[x][r] = Q[x][probe[z][r]] for r < M, zero for M <= r < rows (one 16-byte vector per thread
// step); a probe index outside [0, N) gives a zero row.
__global__ void gather_probe_rows_kernel(const bf16* __restrict__ Q, const int32_t* __restrict__ probe, bf16* Qpr,
                                         int g, int N, int M, int d, int rows) {
    const int x = blockIdx.x, z = x / g;
    const int vpr = d / 8;
    for (int t = threadIdx.x; t < rows * vpr; t += blockDim.x) {
        const int r = t / vpr, c = t % vpr;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < M) {
            const int row = probe[(long long)z * M + r];
            if (row >= 0 && row < N) v = reinterpret_cast<const uint4*>(Q + ((long long)x * N + row) * d)[c];
        }
        reinterpret_cast<uint4*>(Qpr + ((long long)x * rows + r) * d)[c] = v;
    }
}

__global__ void tile_offsets_kernel(const int32_t* __restrict__ qoff, int32_t* tile_off, int P, int Gq, int bm) {
    const int z = blockIdx.x * blockDim.x + threadIdx.x;
    if (z >= P) return;
    const int32_t* qo = qoff + (long long)z * (Gq + 1);
    int32_t* to = tile_off + (long long)z * (Gq + 1);
    int s = 0;
    for (int a = 0; a < Gq; ++a) {
        to[a] = s;
        s += (qo[a + 1] - qo[a] + bm - 1) / bm;
    }
    to[Gq] = s;
}

template <int D, int MODE>
cudaError_t launch_attn(const AttnParams& p, dim3 grid, cudaStream_t s) {
    constexpr int smem = attn_smem_bytes<D>();
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_kernel<D, MODE><<<grid, 128, smem, s>>>(p);
    return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_attn_d(int d, const AttnParams& p, dim3 grid, cudaStream_t s) {
    if (d == 64) return launch_attn<64, MODE>(p, grid, s);
    if (d == 128) return launch_attn<128, MODE>(p, grid, s);
    return cudaErrorInvalidValue;
}

AttnParams base_params(int N, int d, int g) {
    AttnParams p;
    memset(&p, 0, sizeof(p));
    p.N = N;
    p.g = g;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)d));
    return p;
}

}  // namespace

cudaError_t launch_tile_offsets(const int32_t* qoff, int32_t* tile_off, int P, int Gq, int bm, cudaStream_t s) {
    tile_offsets_kernel<<<(P + 127) / 128, 128, 0, s>>>(qoff, tile_off, P, Gq, bm);
    return cudaGetLastError();
}

cudaError_t launch_attn_sparse(const bf16* Qp, const bf16* Kp, const bf16* Vp,
                               const int32_t* qoff, const int32_t* koff, const int32_t* tile_off,
                               const int32_t* rowptr, const int32_t* kg, bf16* O, float* lse,
                               int B, int Hq, int Hkv, int N, int d, int Gq, int Gk, cudaStream_t s) {
    AttnParams p = base_params(N, d, Hq / Hkv);
    p.Q = Qp; p.K = Kp; p.V = Vp; p.O = O; p.lse = lse;
    p.qoff = qoff; p.koff = koff; p.tile_off = tile_off; p.rowptr = rowptr; p.kg = kg;
    p.Gq = Gq; p.Gk = Gk;
    dim3 grid((N + kBM - 1) / kBM + Gq, B * Hq);
    return launch_attn_d<kSparse>(d, p, grid, s);
}

cudaError_t launch_attn_dense(const bf16* Q, const bf16* K, const bf16* V, bf16* O, float* lse,
                              int B, int Hq, int Hkv, int N, int d, cudaStream_t s) {
    AttnParams p = base_params(N, d, Hq / Hkv);
    p.Q = Q; p.K = K; p.V = V; p.O = O; p.lse = lse;
    dim3 grid((N + kBM - 1) / kBM, B * Hq);
    return launch_attn_d<kDense>(d, p, grid, s);
}

cudaError_t launch_gather_probe_rows(const bf16* Q, const int32_t* probe, bf16* Qpr, int B, int Hq, int Hkv, int N,
                                    int M, int d, int rows, cudaStream_t s) {
    gather_probe_rows_kernel<<<B * Hq, 256, 0, s>>>(Q, probe, Qpr, Hq / Hkv, N, M, d, rows);
    return cudaGetLastError();
}

cudaError_t launch_probe_combine(const float* Opart, const float* mpart, const float* lpart, float* Odense, int Hp,
                                 int M, int ns, int d, cudaStream_t s) {
    probe_combine_kernel<<<dim3(M, Hp), d, 0, s>>>(Opart, mpart, lpart, Odense, M, ns, d);
    return cudaGetLastError();
}

cudaError_t launch_attn_probe(const bf16* Q, const bf16* K, const bf16* V, const int32_t* probe,
                              float* Opart, float* mpart, float* lpart, float* Odense, int B,
                              int Hq, int Hkv, int N, int d, int M, int ns, cudaStream_t s) {
    if (M <= 0) return cudaSuccess;
    AttnParams p = base_params(N, d, Hq / Hkv);
    p.Q = Q; p.K = K; p.V = V; p.qidx = probe;
    p.Opart = Opart; p.mpart = mpart; p.lpart = lpart;
    p.M = M; p.ns = ns;
    p.mt = (M + kBM - 1) / kBM;
    const int per = (N + ns - 1) / ns;
    p.chunk = (per + kBN - 1) / kBN * kBN;
    dim3 grid(ns * p.mt, B * Hq);
    cudaError_t e = launch_attn_d<kProbe>(d, p, grid, s);
    if (e != cudaSuccess) return e;
    probe_combine_kernel<<<dim3(M, B * Hq), d, 0, s>>>(Opart, mpart, lpart, Odense, M, ns, d);
    return cudaGetLastError();
}

}  // namespace spr
