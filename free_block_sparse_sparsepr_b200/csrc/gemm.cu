// Small bf16 GEMMs of the partition step: sampled responses z = K Qs^T and the
// query logits u = Q c^T (c split into bf16 hi + lo for fp32-level accuracy),
// and the +-1 projection of the centred logits. C = alpha * sum_t A_t B_t^T.
#include "common.cuh"
#include "kernels.h"
#include "mma_sync.cuh"

namespace spr {
namespace {

constexpr int kBM = 64, kBN = 64, kBK = 64, kLD = kBK + 8;  // +8 bf16 pad: conflict-free ldmatrix

__global__ void __launch_bounds__(128) gemm_bf16_kernel(GemmArgs a) {
    __shared__ __align__(16) bf16 sA[2][kBM * kLD];
    __shared__ __align__(16) bf16 sB[2][kBN * kLD];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int z = blockIdx.z, zb = z / a.bdiv;
    const int m0 = blockIdx.x * kBM, n0 = blockIdx.y * kBN;
    const bool two = (a.A2 != nullptr) || (a.B2 != nullptr);
    const bf16* At[2] = {a.A1 + z * a.sA, (a.A2 ? a.A2 : a.A1) + z * a.sA};
    const bf16* Bt[2] = {a.B1 + zb * a.sB, (a.B2 ? a.B2 : a.B1) + zb * a.sB};
    const int nt = two ? 2 : 1;

    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < a.K; k0 += kBK) {
        // 64 rows x 8 chunks of 16 B per tile; 128 threads x 4 chunks.
        for (int t = 0; t < nt; ++t) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                int c = tid + j * 128;
                int row = c >> 3, col = (c & 7) * 8;
                uint4 va = make_uint4(0, 0, 0, 0), vb = make_uint4(0, 0, 0, 0);
                if (m0 + row < a.M && k0 + col < a.K)
                    va = *reinterpret_cast<const uint4*>(At[t] + (long long)(m0 + row) * a.lda + k0 + col);
                if (n0 + row < a.N && k0 + col < a.K)
                    vb = *reinterpret_cast<const uint4*>(Bt[t] + (long long)(n0 + row) * a.ldb + k0 + col);
                *reinterpret_cast<uint4*>(&sA[t][row * kLD + col]) = va;
                *reinterpret_cast<uint4*>(&sB[t][row * kLD + col]) = vb;
            }
        }
        __syncthreads();
        for (int t = 0; t < nt; ++t) {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
                uint32_t af[4];
                ldsm_x4(af, &sA[t][(warp * 16 + (lane & 15)) * kLD + kk * 16 + (lane >> 4) * 8]);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t bfr[4];
                    ldsm_x4(bfr, &sB[t][(np * 16 + (lane & 7) + ((lane >> 4) << 3)) * kLD + kk * 16 +
                                        ((lane >> 3) & 1) * 8]);
                    mma_bf16_16816(acc[2 * np], af, bfr);
                    mma_bf16_16816(acc[2 * np + 1], af, bfr + 2);
                }
            }
        }
        __syncthreads();
    }

    float* C = a.C + z * a.sC;
    const int r0 = m0 + warp * 16 + (lane >> 2);
#pragma unroll
    for (int ntile = 0; ntile < 8; ++ntile) {
        int col = n0 + ntile * 8 + 2 * (lane & 3);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            int row = r0 + h * 8;
            if (row < a.M) {
                if (col < a.N) C[(long long)row * a.ldc + col] = a.alpha * acc[ntile][2 * h];
                if (col + 1 < a.N) C[(long long)row * a.ldc + col + 1] = a.alpha * acc[ntile][2 * h + 1];
            }
        }
    }
}

}  // namespace

cudaError_t launch_gemm_bf16(const GemmArgs& a, cudaStream_t s) {
    if (a.M <= 0 || a.N <= 0 || a.batch <= 0) return cudaSuccess;
    dim3 grid((a.M + kBM - 1) / kBM, (a.N + kBN - 1) / kBN, a.batch);
    gemm_bf16_kernel<<<grid, 128, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace spr
