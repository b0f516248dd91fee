// Lloyd assignment step on 5th-generation tensor cores (G <= 256 groups).
//
// For a tile of 128 rows the dot products with every centroid form one
// 128 x G x D GEMM. Rows and centroids are split into three bf16 parts
// (x = x0 + x1 + x2, each part the bf16 rounding of what the previous parts leave,
// so |x - x0 - x1 - x2| <= 2^-27 |x|) and the product is accumulated in fp32 TMEM
// from the six terms x_i c_j with i + j <= 2: the dot product to fp32 accuracy
// (a two-part split, about 1e-5 relative, lets near-tie flips cascade through the
// Lloyd rounds). One epilogue thread per row then takes
// argmin_g (||c_g||^2 - 2 x.c_g) (ties -> lowest g) straight from its TMEM lane.
//
// Warps 0-3 epilogue, warp 4 TMA producer (centroids once, row tiles in a 2-stage
// ring), warp 5 MMA issuer; TMEM holds two 256-column accumulators.
#include <float.h>
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_primitives.cuh"
#include "tmap.h"

namespace spr {
namespace {

constexpr int kRows = 128;
constexpr int kCols = 64;                 // padded feature width (one 128-byte swizzle row)
constexpr int kMaxG = 256;
constexpr int kTile = kRows * kCols * 2;  // 16 KB per hi or lo row tile
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;

constexpr int kParts = 3;
constexpr int kOffC = 0;                                     // part q at kOffC + q * kMaxG * 128
constexpr int kOffX = kOffC + kParts * kMaxG * 128;          // stage s, part q at + (s * kParts + q) * kTile
constexpr int kOffCC = kOffX + 2 * kParts * kTile;           // kMaxG floats
constexpr int kOffBar = kOffCC + kMaxG * 4;
constexpr int kBarC = 0, kBarXF = 1, kBarXE = 3, kBarDF = 5, kBarDE = 7, kBarMma = 9, kNumBars = 10;
constexpr int kOffMisc = kOffBar + 8 * kNumBars;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;

struct KmParams {
    const float* xx;       // [P][n]
    const float* cc;       // [P][G32]  ||c||^2, +inf past G
    int32_t* labels;       // [P][n]
    float* dist;           // [P][n]
    int* changed;          // [P]
    const int* done;       // [P] or null
    int* status;
    int n, G16, G32, ksteps, first;
};

struct KmMaps {
    CUtensorMap x[kParts];   // row parts [P*n][64] bf16
    CUtensorMap c[kParts];   // centroid parts [P*G16][64] bf16
};

__global__ void __launch_bounds__(kThreads, 1) km_assign_tc_kernel(const __grid_constant__ KmMaps maps,
                                                                   const KmParams p) {
    const int z = blockIdx.y;
    if (p.done && p.done[z]) return;
    if (p.status && *reinterpret_cast<volatile int*>(p.status) == kDevTimeout) return;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = tc::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* sbase = smem_raw + (base - raw);
    float* sCC = reinterpret_cast<float*>(sbase + kOffCC);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + kOffMisc + 4);
    auto bar = [&](int i) { return base + kOffBar + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles = (p.n + kRows - 1) / kRows;

    for (int t = threadIdx.x; t < p.G32; t += kThreads) sCC[t] = p.cc[(long long)z * p.G32 + t];
    if (threadIdx.x == 0) {
        tc::mbar_init(bar(kBarC), 1);
        for (int s = 0; s < 2; ++s) {
            tc::mbar_init(bar(kBarXF + s), 1);
            tc::mbar_init(bar(kBarXE + s), 1);
            tc::mbar_init(bar(kBarDF + s), 1);
            tc::mbar_init(bar(kBarDE + s), 128);
        }
        tc::mbar_init(bar(kBarMma), 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 5) {
        tc::tmem_alloc(tc::smem_addr(tmem_slot), kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(bar(kBarC), (uint32_t)kParts * (uint32_t)p.G16 * 128u);
            for (int q = 0; q < kParts; ++q)
                tc::tma_load_2d(base + kOffC + q * kMaxG * 128, &maps.c[q], bar(kBarC), 0, z * p.G16);
            int i = 0;
            for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
                const int s = i & 1;
                if (i >= 2 && !tc::mbar_wait(bar(kBarXE + s), ((i >> 1) - 1) & 1, abort_flag)) break;
                const uint32_t dx = base + kOffX + s * kParts * kTile;
                const int row = z * p.n + t * kRows;
                tc::mbar_arrive_expect_tx(bar(kBarXF + s), kParts * kTile);
                for (int q = 0; q < kParts; ++q) tc::tma_load_2d(dx + q * kTile, &maps.x[q], bar(kBarXF + s), 0, row);
            }
            int never = 0;
            for (int k = (i > 2 ? i - 2 : 0); k < i; ++k) tc::mbar_wait(bar(kBarXF + (k & 1)), (k >> 1) & 1, &never);
            tc::mbar_wait(bar(kBarC), 0, &never);
        }
    } else if (warp == 5) {
        const uint32_t idesc = tc::idesc_bf16_f32(kRows, p.G16, 0);
        bool ok = __all_sync(kFull, tc::mbar_wait(bar(kBarC), 0, abort_flag));
        int i = 0;
        for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++i) {
            const int s = i & 1;
            if (!__all_sync(kFull, tc::mbar_wait(bar(kBarXF + s), (i >> 1) & 1, abort_flag))) break;
            if (i >= 2 && !__all_sync(kFull, tc::mbar_wait(bar(kBarDE + s), ((i >> 1) - 1) & 1, abort_flag))) break;
            tc::fence_after_sync();
            if (lane == 0) {
                const uint32_t d = tmem + (uint32_t)(s * 256);
                const uint32_t xb = base + kOffX + s * kParts * kTile;
                for (int k = 0; k < p.ksteps; ++k) {
                    const uint32_t off = (uint32_t)(k * 32);
                    uint64_t dx[kParts], dc[kParts];
#pragma unroll
                    for (int q = 0; q < kParts; ++q) {
                        dx[q] = tc::smem_desc_sw128(xb + q * kTile + off, 16, 1024);
                        dc[q] = tc::smem_desc_sw128(base + kOffC + q * kMaxG * 128 + off, 16, 1024);
                    }
                    // terms x_i c_j with i + j <= 2, largest first
                    tc::mma_f16_ss(d, dx[0], dc[0], idesc, k > 0 ? 1u : 0u);
                    tc::mma_f16_ss(d, dx[0], dc[1], idesc, 1u);
                    tc::mma_f16_ss(d, dx[1], dc[0], idesc, 1u);
                    tc::mma_f16_ss(d, dx[0], dc[2], idesc, 1u);
                    tc::mma_f16_ss(d, dx[2], dc[0], idesc, 1u);
                    tc::mma_f16_ss(d, dx[1], dc[1], idesc, 1u);
                }
                tc::commit(bar(kBarXE + s));
                tc::commit(bar(kBarDF + s));
            }
            __syncwarp();
        }
        if (lane == 0) tc::commit(bar(kBarMma));
        __syncwarp();
        int never = 0;
        tc::mbar_wait(bar(kBarMma), 0, &never);
    } else {
        const int r = threadIdx.x;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        int i = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
            const int s = i & 1;
            if (!__all_sync(kFull, tc::mbar_wait(bar(kBarDF + s), (i >> 1) & 1, abort_flag))) break;
            tc::fence_after_sync();
            const uint32_t d = tmem + (uint32_t)(s * 256) + lane_off;
            float best = FLT_MAX;
            int bi = 0;
            for (int c = 0; c < p.G32; c += 32) {
                uint32_t v[32];
                tc::tmem_ld32(d + c, v);
                tc::tmem_wait_ld();
                tc::regs_after_wait(v);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float dd = fmaf(-2.f, __uint_as_float(v[e]), sCC[c + e]);
                    if (dd < best) { best = dd; bi = c + e; }
                }
            }
            tc::fence_before_sync();
            tc::mbar_arrive(bar(kBarDE + s));
            const int row = t * kRows + r;
            int moved = 0;
            if (row < p.n) {
                const long long o = (long long)z * p.n + row;
                if (!p.first && p.labels[o] != bi) moved = 1;
                p.labels[o] = bi;
                p.dist[o] = fmaxf(p.xx[o] + best, 0.f);
            }
            const unsigned b = __ballot_sync(kFull, moved);
            if (lane == 0 && b) atomicAdd(&p.changed[z], __popc(b));
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) set_status(p.status, kDevTimeout);
    if (warp == 5) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// The three bf16 parts of v: each part is the bf16 rounding of what the previous ones leave.
__device__ __forceinline__ void split3(float v, bf16& a, bf16& b, bf16& c) {
    a = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(a);
    b = __float2bfloat16_rn(r1);
    c = __float2bfloat16_rn(r1 - __bfloat162float(b));
}

// X [P][n][DP] fp32 -> three bf16 parts [P][n][64] (zero padded, part q at X3 + q*stride)
// and ||x||^2; one warp per row.
__global__ void km_split_rows_kernel(const float* __restrict__ X, bf16* X3, long long stride, float* xx,
                                     long long rows, int DP) {
    const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float ss = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int c = lane + 32 * h;
        const float v = c < DP ? X[row * DP + c] : 0.f;
        ss = fmaf(v, v, ss);
        bf16 a, b, e;
        split3(v, a, b, e);
        X3[row * kCols + c] = a;
        X3[stride + row * kCols + c] = b;
        X3[2 * stride + row * kCols + c] = e;
    }
    ss = warp_sum(ss);
    if (lane == 0) xx[row] = ss;
}

// C [P][G][DP] fp32 -> three bf16 parts [P][G16][64] (zero rows past G, part q at C3 + q*stride)
// and ||c||^2 [P][G32] (+inf past G so padded columns never win).
__global__ void km_split_cent_kernel(const float* __restrict__ C, bf16* C3, long long stride, float* cc, int G,
                                     int G16, int G32, int DP) {
    const int z = blockIdx.y;
    const int g = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (g >= G32) return;
    float ss = 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int c = lane + 32 * h;
        const float v = (g < G && c < DP) ? C[((long long)z * G + g) * DP + c] : 0.f;
        ss = fmaf(v, v, ss);
        if (g < G16) {
            bf16 a, b, e;
            split3(v, a, b, e);
            const long long o = ((long long)z * G16 + g) * kCols + c;
            C3[o] = a;
            C3[stride + o] = b;
            C3[2 * stride + o] = e;
        }
    }
    ss = warp_sum(ss);
    if (lane == 0) cc[(long long)z * G32 + g] = g < G ? ss : INFINITY;
}

}  // namespace

bool km_tc_supported(int G) { return G >= 1 && G <= kMaxG; }

cudaError_t launch_km_split_rows(const float* X, bf16* X3, float* xx, int P, int n, int DP, cudaStream_t s) {
    const long long rows = (long long)P * n;
    km_split_rows_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(X, X3, rows * kCols, xx, rows, DP);
    return cudaGetLastError();
}

cudaError_t launch_km_split_cent(const float* C, bf16* C3, float* cc, int P, int G, int DP, cudaStream_t s) {
    const int G16 = (G + 15) / 16 * 16, G32 = (G + 31) / 32 * 32;
    km_split_cent_kernel<<<dim3((G32 + 7) / 8, P), 256, 0, s>>>(C, C3, (long long)P * G16 * kCols, cc, G, G16, G32,
                                                                 DP);
    return cudaGetLastError();
}

cudaError_t launch_km_assign_tc(const bf16* X3, const float* xx, const bf16* C3, const float* cc, int32_t* labels,
                                float* dist, int* changed, const int* done, int* status, int P, int n, int G,
                                int DP, bool first, int num_sms, cudaStream_t s) {
    const int G16 = (G + 15) / 16 * 16, G32 = (G + 31) / 32 * 32;
    KmMaps maps;
    for (int q = 0; q < kParts; ++q) {
        if (!make_tmap_bf16_sw128(&maps.x[q], X3 + (long long)q * P * n * kCols, (long long)P * n, kCols, kRows, 64) ||
            !make_tmap_bf16_sw128(&maps.c[q], C3 + (long long)q * P * G16 * kCols, (long long)P * G16, kCols, G16, 64))
            return cudaErrorInvalidValue;
    }
    KmParams p;
    memset(&p, 0, sizeof(p));
    p.xx = xx; p.cc = cc; p.labels = labels; p.dist = dist; p.changed = changed; p.done = done; p.status = status;
    p.n = n; p.G16 = G16; p.G32 = G32; p.ksteps = (DP + 15) / 16; p.first = first ? 1 : 0;
    const int tiles = (n + kRows - 1) / kRows;
    int per = num_sms / P;
    if (per < 1) per = 1;
    if (per > tiles) per = tiles;
    cudaError_t e = cudaFuncSetAttribute(km_assign_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    km_assign_tc_kernel<<<dim3(per, P), kThreads, kSmemBytes, s>>>(maps, p);
    return cudaGetLastError();
}

}  // namespace spr
