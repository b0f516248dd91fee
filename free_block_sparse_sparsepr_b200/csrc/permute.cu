// Group-major gather of Q/K/V rows: coalesced 16-byte vectors, one vector per thread.
#include "common.cuh"
#include "kernels.h"

namespace spr {
namespace {

__global__ void permute_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                    const int32_t* __restrict__ perm, int div, int N, int vpr) {
    const int z = blockIdx.y;
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (long long)N * vpr) return;
    const int p = (int)(t / vpr), c = (int)(t % vpr);
    const int row = perm[(long long)(z / div) * N + p];
    dst[((long long)z * N + p) * vpr + c] = src[((long long)z * N + row) * vpr + c];
}

}  // namespace

cudaError_t launch_permute_rows(const bf16* src, bf16* dst, const int32_t* perm, int Z, int div,
                                int N, int d, cudaStream_t s) {
    const int vpr = d / 8;
    const long long tot = (long long)N * vpr;
    dim3 grid((unsigned)((tot + 255) / 256), Z);
    permute_rows_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint4*>(src),
                                             reinterpret_cast<uint4*>(dst), perm, div, N, vpr);
    return cudaGetLastError();
}

}  // namespace spr
