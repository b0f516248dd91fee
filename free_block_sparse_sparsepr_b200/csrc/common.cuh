// Shared device helpers for the SparsePR kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace spr {

constexpr unsigned kFull = 0xffffffffu;

// Device status word values (match sparsepr_status codes).
constexpr int kDevOk = 0;
constexpr int kDevTimeout = 5;
constexpr int kDevBounds = 6;

__device__ __forceinline__ float bf16_to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}

__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// Systematic sample position floor((i + 1/2) * n / s) in exact integer form.
__host__ __device__ __forceinline__ long long sample_pos(long long i, long long n, long long s) {
    return ((2 * i + 1) * n) / (2 * s);
}

// SplitMix64 output for state x (Steele, Lea, Flood 2014): increment by the odd
// constant 0x9E3779B97F4A7C15, then two xor-shift-multiply rounds and a final xor-shift.
__host__ __device__ __forceinline__ unsigned long long splitmix64(unsigned long long x) {
    unsigned long long z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// Largest index i in [0, n) with a[i] <= v, for non-decreasing a (a[0] <= v assumed).
__device__ __forceinline__ int upper_index(const int32_t* a, int n, long long v) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((long long)a[mid] <= v) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ void set_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

}  // namespace spr
