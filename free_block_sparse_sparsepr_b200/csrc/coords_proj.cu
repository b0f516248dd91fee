// Query coordinates when Gk > rQ, in one pass over the logits ([partition]): for each query i
// of KV head z, the logits of its g query heads are averaged, centred over the Gk groups,
// split into bf16 hi + lo, multiplied by the +-1 projection (projT [DPy][Gkp], exact in bf16)
// on the tensor cores (mma.sync, fp32 accumulation), and the DPy-wide result is L2-normalised
// in the epilogue (the 1/sqrt(rQ) scale of the projection cancels there).
//
// One CTA per 64 queries: the projection and the tile's centred logits are staged in shared
// memory ([rows][Gkp + 8] bf16, conflict-free ldmatrix); four warps of 16 rows each.
#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"

namespace spr {
namespace {

constexpr int kRows = 64;
constexpr int kThreads = 128;
constexpr int kOut = 64;   // DPy

__global__ void __launch_bounds__(kThreads) coords_proj_kernel(const float* __restrict__ u,
                                                               const bf16* __restrict__ projT, float* y, int g,
                                                               int N, int Gk, int Gkp) {
    extern __shared__ __align__(16) unsigned char cp_raw[];
    const int ld = Gkp + 8;
    bf16* sP = reinterpret_cast<bf16*>(cp_raw);     // [kOut][ld]
    bf16* sH = sP + kOut * ld;                        // [kRows][ld]
    bf16* sL = sH + kRows * ld;                       // [kRows][ld]
    const int z = blockIdx.y, i0 = blockIdx.x * kRows;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    for (int t = tid; t < kOut * Gkp / 8; t += kThreads) {
        const int row = t / (Gkp / 8), c = (t % (Gkp / 8)) * 8;
        *reinterpret_cast<uint4*>(sP + row * ld + c) = *reinterpret_cast<const uint4*>(projT + (long long)row * Gkp + c);
    }
    // centred mean logits of each row, as bf16 hi + lo (one warp per row)
    const float invg = 1.f / (float)g;
    for (int rr = warp; rr < kRows; rr += kThreads / 32) {
        const int i = i0 + rr;
        float v[8 * 8];          // up to 8 columns per lane per 256-column block, Gkp <= 1024
        float s = 0.f;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int c0 = b * 256 + lane * 8;
#pragma unroll
            for (int e = 0; e < 8; ++e) v[8 * b + e] = 0.f;
            if (i < N && c0 < Gk) {
                for (int j = 0; j < g; ++j) {
                    const float* ur = u + (((long long)z * g + j) * N + i) * Gk + c0;
                    if (c0 + 8 <= Gk && (Gk & 3) == 0) {
                        const float4 a0 = *reinterpret_cast<const float4*>(ur);
                        const float4 a1 = *reinterpret_cast<const float4*>(ur + 4);
                        v[8 * b + 0] += a0.x; v[8 * b + 1] += a0.y; v[8 * b + 2] += a0.z; v[8 * b + 3] += a0.w;
                        v[8 * b + 4] += a1.x; v[8 * b + 5] += a1.y; v[8 * b + 6] += a1.z; v[8 * b + 7] += a1.w;
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            if (c0 + e < Gk) v[8 * b + e] += ur[e];
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                v[8 * b + e] *= invg;
                s += v[8 * b + e];
            }
        }
        const float mean = warp_sum(s) / (float)Gk;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int c0 = b * 256 + lane * 8;
            if (c0 >= Gkp) continue;
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                const float a = (i < N && c0 + e < Gk) ? v[8 * b + e] - mean : 0.f;
                const float c = (i < N && c0 + e + 1 < Gk) ? v[8 * b + e + 1] - mean : 0.f;
                const __nv_bfloat16 ah = __float2bfloat16_rn(a), ch = __float2bfloat16_rn(c);
                hi[e / 2] = pack_bf16x2(__bfloat162float(ah), __bfloat162float(ch));
                lo[e / 2] = pack_bf16x2(a - __bfloat162float(ah), c - __bfloat162float(ch));
            }
            *reinterpret_cast<uint4*>(sH + rr * ld + c0) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(sL + rr * ld + c0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
    }
    __syncthreads();

    float acc[8][4];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
    for (int k0 = 0; k0 < Gkp; k0 += 16) {
        uint32_t ah[4], al[4];
        ldsm_x4(ah, sH + (warp * 16 + (lane & 15)) * ld + k0 + (lane >> 4) * 8);
        ldsm_x4(al, sL + (warp * 16 + (lane & 15)) * ld + k0 + (lane >> 4) * 8);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
            uint32_t bfr[4];
            ldsm_x4(bfr, sP + (np * 16 + (lane & 7) + ((lane >> 4) << 3)) * ld + k0 + ((lane >> 3) & 1) * 8);
            mma_bf16_16816(acc[2 * np], ah, bfr);
            mma_bf16_16816(acc[2 * np + 1], ah, bfr + 2);
            mma_bf16_16816(acc[2 * np], al, bfr);
            mma_bf16_16816(acc[2 * np + 1], al, bfr + 2);
        }
    }
    // rows warp*16 + lane/4 (+8): each row's 64 outputs spread over the 4 lanes of a quad
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float ss = 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) ss = fmaf(acc[nt][2 * h], acc[nt][2 * h], fmaf(acc[nt][2 * h + 1], acc[nt][2 * h + 1], ss));
        ss += __shfl_xor_sync(kFull, ss, 1);
        ss += __shfl_xor_sync(kFull, ss, 2);
        const float nrm = sqrtf(ss);
        const float inv = nrm > 0.f ? 1.f / nrm : 0.f;
        const int i = i0 + warp * 16 + (lane >> 2) + 8 * h;
        if (i < N) {
            float* yr = y + ((long long)z * N + i) * kOut;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
                *reinterpret_cast<float2*>(yr + nt * 8 + 2 * (lane & 3)) =
                    make_float2(acc[nt][2 * h] * inv, acc[nt][2 * h + 1] * inv);
        }
    }
}

}  // namespace

bool coords_proj_supported(int DPy, int Gkp) { return false && DPy == kOut && Gkp % 64 == 0 && Gkp <= 1024; }

cudaError_t launch_coords_proj(const float* u, const bf16* projT, float* y, int P, int g, int N, int Gk, int Gkp,
                               cudaStream_t s) {
    const size_t smem = (size_t)(kOut + 2 * kRows) * (Gkp + 8) * sizeof(bf16);
    cudaError_t e = cudaFuncSetAttribute(coords_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    coords_proj_kernel<<<dim3((N + kRows - 1) / kRows, P), kThreads, smem, s>>>(u, projT, y, g, N, Gk, Gkp);
    return cudaGetLastError();
}

}  // namespace spr
