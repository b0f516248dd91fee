// Query coordinates when Gk > rQ, in one pass over the logits ([partition]): for each query i
// of KV head z, the logits of its g query heads are averaged and multiplied by the +-1
// projection (projT [DPy][Gkp], exact in bf16) on the tensor cores (mma.sync, fp32
// accumulation; the averaged logits split into three bf16 parts, so the products carry fp32
// accuracy). Centring commutes with the projection: (u - mean 1) P^T = u P^T - mean (1 P^T), so
// the row mean, summed along the way, is taken off in the epilogue, which then L2-normalises
// the DPy-wide row (the 1/sqrt(rQ) scale of the projection cancels there).
//
// Each warp takes 16-row tiles of its head and loads the logits straight into the MMA
// fragment layout; the projection is staged once per CTA in shared memory.
#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"

namespace spr {
namespace {

constexpr int kOut = 64;   // DPy
constexpr int kWarps = 4;

__device__ __forceinline__ void split3(float v, float& a, float& b, float& c) {
    a = __bfloat162float(__float2bfloat16_rn(v));
    const float r = v - a;
    b = __bfloat162float(__float2bfloat16_rn(r));
    c = r - b;
}

// kOneHead: g == 1, so the next 16 columns' loads are issued before this step's MMAs (a
// register double buffer); with several heads their sum is formed as the loads arrive.
template <bool kOneHead>
__global__ void __launch_bounds__(kWarps * 32, 5) coords_proj_kernel(const float* __restrict__ u,
                                                                  const bf16* __restrict__ projT, float* y, int g,
                                                                  int N, int Gk, int Gkp) {
    extern __shared__ __align__(16) unsigned char cp_raw[];
    const int ld = Gkp + 8;
    bf16* sP = reinterpret_cast<bf16*>(cp_raw);                        // [kOut][ld]
    float* sCol = reinterpret_cast<float*>(cp_raw + (size_t)kOut * ld * sizeof(bf16));   // [kOut]
    const int z = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int t = tid; t < kOut * Gkp / 8; t += blockDim.x) {
        const int row = t / (Gkp / 8), c = (t % (Gkp / 8)) * 8;
        *reinterpret_cast<uint4*>(sP + row * ld + c) = *reinterpret_cast<const uint4*>(projT + (long long)row * Gkp + c);
    }
    __syncthreads();
    for (int t = tid; t < kOut; t += blockDim.x) {
        float s = 0.f;
        for (int c = 0; c < Gk; ++c) s += __bfloat162float(sP[t * ld + c]);
        sCol[t] = s;
    }
    __syncthreads();

    const float invg = 1.f / (float)g;
    const int tiles = (N + 15) / 16;
    for (int tile = blockIdx.x * kWarps + warp; tile < tiles; tile += gridDim.x * kWarps) {
        const int ra = tile * 16 + (lane >> 2), rb = ra + 8;
        const bool va = ra < N, vb = rb < N;
        float acc[8][4];
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
        float sa = 0.f, sb = 0.f;
        // the four float2 of the lane's A fragment at column step k0 (rows ra / rb, columns c0 / c1)
        auto load_step = [&](int k0, float2 (&x)[4]) {
            const int c0 = k0 + (lane & 3) * 2, c1 = c0 + 8;
#pragma unroll
            for (int q = 0; q < 4; ++q) x[q] = make_float2(0.f, 0.f);
            for (int j = 0; j < (kOneHead ? 1 : g); ++j) {
                const float* ua = u + (((long long)z * g + j) * N + ra) * Gk;
                const float* ub = ua + 8ll * Gk;
                if (va && c0 < Gk) { const float2 t = __ldg(reinterpret_cast<const float2*>(ua + c0)); x[0].x += t.x; x[0].y += t.y; }
                if (vb && c0 < Gk) { const float2 t = __ldg(reinterpret_cast<const float2*>(ub + c0)); x[1].x += t.x; x[1].y += t.y; }
                if (va && c1 < Gk) { const float2 t = __ldg(reinterpret_cast<const float2*>(ua + c1)); x[2].x += t.x; x[2].y += t.y; }
                if (vb && c1 < Gk) { const float2 t = __ldg(reinterpret_cast<const float2*>(ub + c1)); x[3].x += t.x; x[3].y += t.y; }
            }
        };
        float2 xn[4];
        if (kOneHead) load_step(0, xn);
        for (int k0 = 0; k0 < Gkp; k0 += 16) {
            float2 x[4];
            if (kOneHead) {
#pragma unroll
                for (int q = 0; q < 4; ++q) x[q] = xn[q];
                if (k0 + 16 < Gkp) load_step(k0 + 16, xn);
            } else {
                load_step(k0, x);
            }
            uint32_t af[3][4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float e0 = x[q].x * invg, e1 = x[q].y * invg;
                if (q & 1) sb += e0 + e1; else sa += e0 + e1;
                float h0, m0, l0, h1, m1, l1;
                split3(e0, h0, m0, l0);
                split3(e1, h1, m1, l1);
                af[0][q] = pack_bf16x2(h0, h1);
                af[1][q] = pack_bf16x2(m0, m1);
                af[2][q] = pack_bf16x2(l0, l1);
            }
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t bfr[4];
                ldsm_x4(bfr, sP + (np * 16 + (lane & 7) + ((lane >> 4) << 3)) * ld + k0 + ((lane >> 3) & 1) * 8);
#pragma unroll
                for (int part = 0; part < 3; ++part) {
                    mma_bf16_16816(acc[2 * np], af[part], bfr);
                    mma_bf16_16816(acc[2 * np + 1], af[part], bfr + 2);
                }
            }
        }
        // row sums over the quad's lanes, then y = acc - mean * colsum, normalised
        sa += __shfl_xor_sync(kFull, sa, 1);
        sa += __shfl_xor_sync(kFull, sa, 2);
        sb += __shfl_xor_sync(kFull, sb, 1);
        sb += __shfl_xor_sync(kFull, sb, 2);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float mean = (h ? sb : sa) / (float)Gk;
            float ss = 0.f;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                const int t = nt * 8 + 2 * (lane & 3);
                acc[nt][2 * h] = fmaf(-mean, sCol[t], acc[nt][2 * h]);
                acc[nt][2 * h + 1] = fmaf(-mean, sCol[t + 1], acc[nt][2 * h + 1]);
                ss = fmaf(acc[nt][2 * h], acc[nt][2 * h], fmaf(acc[nt][2 * h + 1], acc[nt][2 * h + 1], ss));
            }
            ss += __shfl_xor_sync(kFull, ss, 1);
            ss += __shfl_xor_sync(kFull, ss, 2);
            const float nrm = sqrtf(ss);
            const float inv = nrm > 0.f ? 1.f / nrm : 0.f;
            const int i = h ? rb : ra;
            if (i < N) {
                float* yr = y + ((long long)z * N + i) * kOut;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
                    *reinterpret_cast<float2*>(yr + nt * 8 + 2 * (lane & 3)) =
                        make_float2(acc[nt][2 * h] * inv, acc[nt][2 * h + 1] * inv);
            }
        }
    }
}

}  // namespace

bool coords_proj_supported(int DPy, int Gk, int Gkp) {
    return DPy == kOut && Gk % 2 == 0 && Gkp % 16 == 0 && Gkp <= 1024;
}

cudaError_t launch_coords_proj(const float* u, const bf16* projT, float* y, int P, int g, int N, int Gk, int Gkp,
                               int num_sms, cudaStream_t s) {
    const size_t smem = (size_t)kOut * (Gkp + 8) * sizeof(bf16) + kOut * sizeof(float);
    auto kern = g == 1 ? coords_proj_kernel<true> : coords_proj_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int tiles = (N + 15) / 16;
    // persistent CTAs: as many as fit on the GPU at once (a second, partial wave would double
    // the time of the slowest CTA)
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kWarps * 32, smem);
    if (e != cudaSuccess) return e;
    if (occ < 1) occ = 1;
    int per = occ * num_sms / P;
    if (per < 1) per = 1;
    const int maxper = (tiles + kWarps - 1) / kWarps;
    if (per > maxper) per = maxper;
    kern<<<dim3(per, P), kWarps * 32, smem, s>>>(u, projT, y, g, N, Gk, Gkp);
    return cudaGetLastError();
}

}  // namespace spr
