// Sampled pre-softmax responses on 5th-generation tensor cores ([partition]: the sampled queries'
// responses to every key are the keys' features):
//   F[z][j][s] = (k_j . q_s) / sqrt(d),   s < rK (columns rK..DP-1 are zero),
// with everything the key k-means and the support diagnostic need from F written by the same
// epilogue, so F is formed once and never re-read for them:
//   - the two bf16 parts of every feature (x0 = bf16(f), x1 = bf16(f - x0)) and ||f||^2 in fp32,
//     the operands of the tensor-core assignment;
//   - optionally ([support]), the maximum response of every sampled query over all keys, the
//     first statistic of its 90%-mass count (an order-preserving integer max, so the result
//     does not depend on the order of the updates).
// Persistent CTAs walk 128-key tiles of all KV heads in contiguous ranges. A key tile (128 x d
// bf16) and its head's sampled queries (DP x d) arrive together by TMA in a 3-stage ring; one
// thread issues the MMAs (M = 128, N = DP, K = d) into one of two TMEM accumulators; four
// epilogue warps take one key row per thread and stage the tile's rows of F and of its two
// parts in shared memory, from where bulk copies write them out (the tile's rows are
// contiguous in every output, so the copies are whole contiguous blocks).
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_primitives.cuh"
#include "tmap.h"

namespace spr {
namespace {

constexpr int kRows = 128;
constexpr int kMaxDP = 64;
constexpr int kStages = 3;
constexpr int kARegion = kRows * 128;              // [128 rows][64 bf16], 128B swizzle
constexpr int kBRegion = kMaxDP * 128;             // [<= 64 rows][64 bf16]
constexpr int kStageBytes = 2 * kARegion + 2 * kBRegion;
constexpr int kThreads = 192;                      // warps 0-3 epilogue, 4 TMA, 5 MMA
constexpr uint32_t kTmemCols = 128;                // two accumulators of 64 columns

constexpr int kOffStage = 0;
constexpr int kOffStg = kOffStage + kStages * kStageBytes;   // output staging: F, x0, x1 rows of a tile
constexpr int kStgF = kRows * kMaxDP * 4, kStgX = kRows * kMaxDP * 2;
constexpr int kOffBar = kOffStg + kStgF + 2 * kStgX;
constexpr int kBarF = 0, kBarE = kStages, kBarDF = 2 * kStages, kBarDE = kBarDF + 2, kBarMma = kBarDE + 2,
              kNumBars = kBarMma + 1;
constexpr int kOffMisc = kOffBar + 8 * kNumBars;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct RespParams {
    float* F;              // [P][N][DP]
    bf16* X2;              // [2][P*N][DP] (part q at X2 + q * P * N * DP)
    float* xx;             // [P*N]
    unsigned* colmax;      // [P][DP] order-preserving keys of the column maxima, or null
    int* status;
    int P, N, d, DP, S, tiles_per_head;
    float scale;
};

// Order-preserving map of an fp32 value to an unsigned key (larger value, larger key).
__device__ __forceinline__ unsigned max_key(float f) {
    const unsigned u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kThreads, 1) resp_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                                                              const __grid_constant__ CUtensorMap tmQs,
                                                              const RespParams p) {
    if (p.status && *reinterpret_cast<volatile int*>(p.status) == kDevTimeout) return;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = tc::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* sbase = smem_raw + (base - raw);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + kOffMisc + 4);
    auto bar = [&](int i) { return base + kOffBar + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nreg = p.d / 64;
    // this CTA's contiguous range of tiles over all heads
    const long long total = (long long)p.P * p.tiles_per_head;
    const int t0 = (int)(total * blockIdx.x / gridDim.x), t1 = (int)(total * (blockIdx.x + 1) / gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(bar(kBarF + s), 1);
            tc::mbar_init(bar(kBarE + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(bar(kBarDF + b), 1);
            tc::mbar_init(bar(kBarDE + b), 128);
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
        // ================= TMA producer: key tile + the head's sampled queries per stage
        if (lane == 0) {
            const uint32_t bytes = (uint32_t)nreg * (kARegion + (uint32_t)p.DP * 128u);
            int i = 0;
            for (int t = t0; t < t1; ++t, ++i) {
                const int s = i % kStages;
                if (i >= kStages && !tc::mbar_wait(bar(kBarE + s), ((i / kStages) - 1) & 1, abort_flag)) break;
                const int z = t / p.tiles_per_head, rt = t % p.tiles_per_head;
                const uint32_t st = base + kOffStage + s * kStageBytes;
                tc::mbar_arrive_expect_tx(bar(kBarF + s), bytes);
                for (int r = 0; r < nreg; ++r) {
                    tc::tma_load_2d(st + r * kARegion, &tmK, bar(kBarF + s), 64 * r, z * p.N + rt * kRows);
                    tc::tma_load_2d(st + 2 * kARegion + r * kBRegion, &tmQs, bar(kBarF + s), 64 * r, z * p.DP);
                }
            }
            int never = 0;
            for (int k = (i > kStages ? i - kStages : 0); k < i; ++k)
                tc::mbar_wait(bar(kBarF + k % kStages), (k / kStages) & 1, &never);
        }
    } else if (warp == 5) {
        // ================= MMA issuer
        const uint32_t idesc = tc::idesc_bf16_f32(kRows, p.DP, 0);
        int i = 0;
        for (int t = t0; t < t1; ++t, ++i) {
            const int s = i % kStages, b = i & 1;
            if (!__all_sync(kFull, tc::mbar_wait(bar(kBarF + s), (i / kStages) & 1, abort_flag))) break;
            if (i >= 2 && !__all_sync(kFull, tc::mbar_wait(bar(kBarDE + b), ((i >> 1) - 1) & 1, abort_flag))) break;
            tc::fence_after_sync();
            if (lane == 0) {
                const uint32_t st = base + kOffStage + s * kStageBytes;
                const uint32_t d = tmem + (uint32_t)(b * 64);
                for (int k = 0; k < p.d / 16; ++k) {
                    const uint32_t aoff = (uint32_t)((k >> 2) * kARegion + (k & 3) * 32);
                    const uint32_t boff = (uint32_t)(2 * kARegion + (k >> 2) * kBRegion + (k & 3) * 32);
                    tc::mma_f16_ss(d, tc::smem_desc_sw128(st + aoff, 16, 1024), tc::smem_desc_sw128(st + boff, 16, 1024),
                                   idesc, k > 0 ? 1u : 0u);
                }
                tc::commit(bar(kBarE + s));
                tc::commit(bar(kBarDF + b));
            }
            __syncwarp();
        }
        if (lane == 0) tc::commit(bar(kBarMma));
        __syncwarp();
        int never = 0;
        tc::mbar_wait(bar(kBarMma), 0, &never);
    } else {
        // ================= epilogue: thread r <-> key row r of the tile <-> TMEM lane r
        const int r = threadIdx.x;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const long long part = (long long)p.P * p.N * p.DP;
        int i = 0;
        for (int t = t0; t < t1; ++t, ++i) {
            const int b = i & 1;
            const int z = t / p.tiles_per_head, rt = t % p.tiles_per_head;
            const int row = rt * kRows + r;
            if (!__all_sync(kFull, tc::mbar_wait(bar(kBarDF + b), (i >> 1) & 1, abort_flag))) break;
            tc::fence_after_sync();
            uint32_t v[64];
            const uint32_t ta = tmem + (uint32_t)(b * 64) + lane_off;
            tc::tmem_ld32(ta, v);
            if (p.DP > 32) tc::tmem_ld32(ta + 32, v + 32);
            tc::tmem_wait_ld();
            tc::regs_after_wait(v);
            if (p.DP > 32) tc::regs_after_wait(v + 32);
            tc::fence_before_sync();
            tc::mbar_arrive(bar(kBarDE + b));
            const bool valid = row < p.N;
            const long long o = (long long)z * p.N + row;
            const int nvalid = min(kRows, p.N - rt * kRows);
            // the staging buffer is free once the previous tile's bulk copies have read it
            if (r == 0) tc::bulk_wait_group_read<0>();
            tc::named_bar_sync(1, 128);
            float xx = 0.f;
            {
                float* frow = reinterpret_cast<float*>(sbase + kOffStg) + r * p.DP;
                bf16* x0row = reinterpret_cast<bf16*>(sbase + kOffStg + kStgF) + r * p.DP;
                bf16* x1row = reinterpret_cast<bf16*>(sbase + kOffStg + kStgF + kStgX) + r * p.DP;
#pragma unroll
                for (int c8 = 0; c8 < kMaxDP / 8; ++c8) {
                    if (8 * c8 < p.DP) {
                        float f[8];
                        uint32_t w0[4], w1[4];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            f[e] = __uint_as_float(v[8 * c8 + e]) * p.scale;
                            xx = fmaf(f[e], f[e], xx);
                        }
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const bf16 a0 = __float2bfloat16_rn(f[2 * e]), a1 = __float2bfloat16_rn(f[2 * e + 1]);
                            const bf16 b0 = __float2bfloat16_rn(f[2 * e] - __bfloat162float(a0));
                            const bf16 b1 = __float2bfloat16_rn(f[2 * e + 1] - __bfloat162float(a1));
                            w0[e] = (uint32_t)__bfloat16_as_ushort(a0) | ((uint32_t)__bfloat16_as_ushort(a1) << 16);
                            w1[e] = (uint32_t)__bfloat16_as_ushort(b0) | ((uint32_t)__bfloat16_as_ushort(b1) << 16);
                        }
                        reinterpret_cast<float4*>(frow)[2 * c8] = make_float4(f[0], f[1], f[2], f[3]);
                        reinterpret_cast<float4*>(frow)[2 * c8 + 1] = make_float4(f[4], f[5], f[6], f[7]);
                        reinterpret_cast<uint4*>(x0row)[c8] = make_uint4(w0[0], w0[1], w0[2], w0[3]);
                        reinterpret_cast<uint4*>(x1row)[c8] = make_uint4(w1[0], w1[1], w1[2], w1[3]);
                    }
                }
            }
            if (valid) p.xx[o] = xx;
            tc::fence_proxy_async_smem();
            tc::named_bar_sync(1, 128);
            if (r == 0) {
                const long long o0 = (long long)z * p.N + rt * kRows;
                tc::bulk_store(p.F + o0 * p.DP, base + kOffStg, (uint32_t)(nvalid * p.DP * 4));
                tc::bulk_store(p.X2 + o0 * p.DP, base + kOffStg + kStgF, (uint32_t)(nvalid * p.DP * 2));
                tc::bulk_store(p.X2 + part + o0 * p.DP, base + kOffStg + kStgF + kStgX, (uint32_t)(nvalid * p.DP * 2));
                tc::bulk_commit_group();
            }
            if (p.colmax) {
                // column maxima over the warp's valid rows, one atomic per column per warp
                const unsigned vm = __ballot_sync(kFull, valid);
#pragma unroll
                for (int c = 0; c < kMaxDP; ++c) {
                    if (c < p.S) {
                        unsigned key = valid ? max_key(__uint_as_float(v[c]) * p.scale) : 0u;
#pragma unroll
                        for (int off = 16; off > 0; off >>= 1) key = max(key, __shfl_xor_sync(kFull, key, off));
                        if (lane == 0 && vm) atomicMax(p.colmax + (long long)z * p.DP + c, key);
                    }
                }
            }
        }
    }

    if (threadIdx.x == 0) tc::bulk_wait_group<0>();   // the staged outputs are written out
    tc::fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) set_status(p.status, kDevTimeout);
    if (warp == 5) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool resp_tc_supported(int d, int DP) { return (d == 64 || d == 128) && DP % 16 == 0 && DP >= 16 && DP <= kMaxDP; }

cudaError_t launch_resp_tc(const bf16* K, const bf16* Qs, float* F, bf16* X2, float* xx, unsigned* colmax, int P,
                           int N, int d, int DP, int S, int num_sms, int* status, cudaStream_t s) {
    if (!resp_tc_supported(d, DP) || (long long)P * N >= (1ll << 31)) return cudaErrorInvalidValue;
    CUtensorMap mk, mq;
    if (!make_tmap_bf16_sw128(&mk, K, (long long)P * N, d, kRows, 64) ||
        !make_tmap_bf16_sw128(&mq, Qs, (long long)P * DP, d, DP, 64))
        return cudaErrorInvalidValue;
    RespParams p;
    memset(&p, 0, sizeof(p));
    p.F = F; p.X2 = X2; p.xx = xx; p.colmax = colmax; p.status = status;
    p.P = P; p.N = N; p.d = d; p.DP = DP; p.S = S; p.tiles_per_head = (N + kRows - 1) / kRows;
    p.scale = (float)(1.0 / sqrt((double)d));
    if (colmax) {
        cudaError_t e = cudaMemsetAsync(colmax, 0, (size_t)P * DP * sizeof(unsigned), s);
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = cudaFuncSetAttribute(resp_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    const long long total = (long long)P * p.tiles_per_head;
    const int grid = (int)(total < num_sms ? total : num_sms);
    resp_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(mk, mq, p);
    return cudaGetLastError();
}

}  // namespace spr
