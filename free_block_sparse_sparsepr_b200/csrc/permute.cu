// Group-major gather of Q/K/V rows: coalesced 16-byte vectors; each thread moves kVec vectors
// (blockDim apart), their index and data loads all issued before the stores.
#include "common.cuh"
#include "kernels.h"

namespace spr {
namespace {

constexpr int kVec = 4;

__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                           const int32_t* __restrict__ perm, int div, int N,
                                                           int vpr) {
    const int z = blockIdx.y;
    const long long tot = (long long)N * vpr;
    const long long base = (long long)blockIdx.x * blockDim.x * kVec + threadIdx.x;
    const int32_t* pz = perm + (long long)(z / div) * N;
    int row[kVec];
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
        const long long t = base + (long long)u * blockDim.x;
        row[u] = t < tot ? __ldg(pz + t / vpr) : 0;
    }
    uint4 v[kVec];
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
        const long long t = base + (long long)u * blockDim.x;
        if (t < tot) v[u] = __ldg(src + ((long long)z * N + row[u]) * vpr + t % vpr);
    }
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
        const long long t = base + (long long)u * blockDim.x;
        if (t < tot) dst[(long long)z * tot + t] = v[u];
    }
}

}  // namespace

cudaError_t launch_permute_rows(const bf16* src, bf16* dst, const int32_t* perm, int Z, int div,
                                int N, int d, cudaStream_t s) {
    const int vpr = d / 8;
    const long long tot = (long long)N * vpr;
    const long long per_block = 256ll * kVec;
    dim3 grid((unsigned)((tot + per_block - 1) / per_block), Z);
    permute_rows_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint4*>(src),
                                             reinterpret_cast<uint4*>(dst), perm, div, N, vpr);
    return cudaGetLastError();
}

}  // namespace spr
