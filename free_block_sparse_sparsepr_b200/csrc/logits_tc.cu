// Query logits against the key-group means on 5th-generation tensor cores (d = 128, Gk <= 256):
//   u[x][i][g] = (q_i . c_g) / sqrt(d),   c_g = c_hi + c_lo (bf16 split of the fp32 mean),
// and, fused in the epilogue, the routing normaliser
//   lse[x][i] = log sum_{g: |K_g| > 0} |K_g| exp(u[x][i][g]).
// One CTA per (query head, slice of row tiles). The centroid splits stay in shared memory; each
// 128-row query tile arrives by TMA and its 128 x Gk accumulator goes to one of two 256-column
// TMEM buffers. Two epilogue warpgroups take alternate tiles (one thread per row): they scale
// the accumulator, keep a streaming log-sum-exp in the log2 domain, and write u through
// 128-byte-swizzled staging buffers with TMA tiled stores (rows past N are clipped per head).
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_primitives.cuh"
#include "tmap.h"

namespace spr {
namespace {

constexpr int kRows = 128;
constexpr int kD = 128;
constexpr int kMaxG = 256;
constexpr int kRegion = 16384;            // [128 rows][64 bf16], 128B swizzle
constexpr int kCRegion = kMaxG * 128;     // [256 rows][64 bf16]
constexpr int kStage = 16384;             // [128 rows][32 fp32], 128B swizzle
constexpr int kThreads = 320;             // warps 0-7 epilogue, 8 TMA, 9 MMA
constexpr uint32_t kTmemCols = 512;

constexpr int kOffC = 0;                         // hi: 2 regions, lo: 2 regions
constexpr int kOffA = kOffC + 4 * kCRegion;      // one query tile (2 regions)
constexpr int kOffS = kOffA + 2 * kRegion;       // staging: [warpgroup][2][kStage]
constexpr int kOffLw = kOffS + 4 * kStage;       // log2 |K_g| (or -inf) as float [kMaxG]
constexpr int kOffBar = kOffLw + kMaxG * 4;
constexpr int kBarC = 0, kBarAF = 1, kBarAE = 2, kBarDF = 3, kBarDE = 5, kBarMma = 7, kNumBars = 8;
constexpr int kOffMisc = kOffBar + 8 * kNumBars;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct LgParams {
    float* u;                 // [Hp][N][Gk]
    float* lse;               // [Hp][N]
    const int32_t* koff;      // [P][Gk+1]
    int* status;
    int N, g, Gk, G16, G32;
    float scale;
};

template <bool kTmaStore>
__global__ void __launch_bounds__(kThreads, 1) logits_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                const __grid_constant__ CUtensorMap tmChi,
                                                                const __grid_constant__ CUtensorMap tmClo,
                                                                const __grid_constant__ CUtensorMap tmU,
                                                                const LgParams p) {
    if (p.status && *reinterpret_cast<volatile int*>(p.status) == kDevTimeout) return;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = tc::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* sbase = smem_raw + (base - raw);
    float* sLw = reinterpret_cast<float*>(sbase + kOffLw);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + kOffMisc + 4);
    auto bar = [&](int i) { return base + kOffBar + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int x = blockIdx.y, z = x / p.g;
    const int tiles = (p.N + kRows - 1) / kRows;

    const int32_t* ko = p.koff + (long long)z * (p.Gk + 1);
    for (int t = threadIdx.x; t < kMaxG; t += kThreads) {
        const int cnt = t < p.Gk ? ko[t + 1] - ko[t] : 0;
        sLw[t] = cnt > 0 ? log2f((float)cnt) : -INFINITY;
    }
    if (threadIdx.x == 0) {
        tc::mbar_init(bar(kBarC), 1);
        tc::mbar_init(bar(kBarAF), 1);
        tc::mbar_init(bar(kBarAE), 1);
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(bar(kBarDF + b), 1);
            tc::mbar_init(bar(kBarDE + b), 128);
        }
        tc::mbar_init(bar(kBarMma), 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 9) {
        tc::tmem_alloc(tc::smem_addr(tmem_slot), kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(bar(kBarC), 4u * (uint32_t)p.G16 * 128u);
            tc::tma_load_2d(base + kOffC, &tmChi, bar(kBarC), 0, z * p.Gk);
            tc::tma_load_2d(base + kOffC + kCRegion, &tmChi, bar(kBarC), 64, z * p.Gk);
            tc::tma_load_2d(base + kOffC + 2 * kCRegion, &tmClo, bar(kBarC), 0, z * p.Gk);
            tc::tma_load_2d(base + kOffC + 3 * kCRegion, &tmClo, bar(kBarC), 64, z * p.Gk);
            int i = 0;
            for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
                if (i >= 1 && !tc::mbar_wait(bar(kBarAE), (i - 1) & 1, abort_flag)) break;
                const int row = x * p.N + t * kRows;
                tc::mbar_arrive_expect_tx(bar(kBarAF), 2 * kRegion);
                tc::tma_load_2d(base + kOffA, &tmQ, bar(kBarAF), 0, row);
                tc::tma_load_2d(base + kOffA + kRegion, &tmQ, bar(kBarAF), 64, row);
            }
            int never = 0;
            if (i >= 1) tc::mbar_wait(bar(kBarAF), (i - 1) & 1, &never);
            tc::mbar_wait(bar(kBarC), 0, &never);
        }
    } else if (warp == 9) {
        const uint32_t idesc = tc::idesc_bf16_f32(kRows, p.G16, 0);
        bool ok = __all_sync(kFull, tc::mbar_wait(bar(kBarC), 0, abort_flag));
        int i = 0;
        for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++i) {
            const int b = i & 1;
            if (!__all_sync(kFull, tc::mbar_wait(bar(kBarAF), i & 1, abort_flag))) break;
            if (i >= 2 && !__all_sync(kFull, tc::mbar_wait(bar(kBarDE + b), ((i >> 1) - 1) & 1, abort_flag))) break;
            tc::fence_after_sync();
            if (lane == 0) {
                const uint32_t d = tmem + (uint32_t)(b * 256);
#pragma unroll
                for (int k = 0; k < kD / 16; ++k) {
                    const uint32_t aoff = (uint32_t)((k >> 2) * kRegion + (k & 3) * 32);
                    const uint32_t coff = (uint32_t)((k >> 2) * kCRegion + (k & 3) * 32);
                    const uint64_t da = tc::smem_desc_sw128(base + kOffA + aoff, 16, 1024);
                    tc::mma_f16_ss(d, da, tc::smem_desc_sw128(base + kOffC + coff, 16, 1024), idesc, k > 0 ? 1u : 0u);
                    tc::mma_f16_ss(d, da, tc::smem_desc_sw128(base + kOffC + 2 * kCRegion + coff, 16, 1024), idesc, 1u);
                }
                tc::commit(bar(kBarAE));
                tc::commit(bar(kBarDF + b));
            }
            __syncwarp();
        }
        if (lane == 0) tc::commit(bar(kBarMma));
        __syncwarp();
        int never = 0;
        tc::mbar_wait(bar(kBarMma), 0, &never);
    } else {
        // Warpgroup wg takes the tiles i = wg, wg + 2, ... of this CTA, from TMEM buffer wg.
        const int wg = warp >> 2, r = threadIdx.x & 127;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tbuf = tmem + (uint32_t)(wg * 256);
        int kc = 0;  // staging buffers used so far by this warpgroup
        for (int i = wg, t = blockIdx.x + wg * gridDim.x; t < tiles; i += 2, t += 2 * gridDim.x) {
            const bool ok = __all_sync(kFull, tc::mbar_wait(bar(kBarDF + wg), (i >> 1) & 1, abort_flag));
            if (!tc::named_bar_and(1 + wg, 128, ok)) break;
            tc::fence_after_sync();
            const int row = t * kRows + r;
            const bool valid = row < p.N;
            float m2 = -INFINITY, ssum = 0.f;
            for (int c = 0; c < p.G32; c += 32) {
                uint32_t v[32];
                tc::tmem_ld32(tbuf + lane_off + (uint32_t)c, v);
                tc::tmem_wait_ld();
                tc::regs_after_wait(v);
                const int lim = p.Gk - c;
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float uv = __uint_as_float(v[e]) * p.scale;
                    v[e] = __float_as_uint(uv);
                    const float t2 = e < lim ? fmaf(uv, kLog2e, sLw[c + e]) : -INFINITY;
                    mx[e & 3] = fmaxf(mx[e & 3], t2);
                }
                const float mn = fmaxf(m2, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])));
                if (mn > -INFINITY) {
                    float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float t2 = e < lim ? fmaf(__uint_as_float(v[e]), kLog2e, sLw[c + e]) : -INFINITY;
                        sm[e & 3] += exp2f(t2 - mn);
                    }
                    ssum = ssum * exp2f(m2 - mn) + ((sm[0] + sm[1]) + (sm[2] + sm[3]));
                    m2 = mn;
                }
                if (kTmaStore) {
                    const int sb = kOffS + (wg * 2 + (kc & 1)) * kStage;
                    if (r == 0) tc::bulk_wait_group_read<1>();
                    tc::named_bar_sync(1 + wg, 128);
                    unsigned char* srow = sbase + sb + r * 128;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<uint4*>(srow + ((q ^ (r & 7)) << 4)) =
                            make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    tc::fence_proxy_async_smem();
                    tc::named_bar_sync(1 + wg, 128);
                    if (r == 0) {
                        tc::tma_store_3d(&tmU, base + (uint32_t)sb, c, t * kRows, x);
                        tc::bulk_commit_group();
                    }
                    ++kc;
                } else if (valid) {
                    float* ur = p.u + ((long long)x * p.N + row) * p.Gk + c;
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (e < lim) ur[e] = __uint_as_float(v[e]);
                }
            }
            tc::fence_before_sync();
            tc::mbar_arrive(bar(kBarDE + wg));
            if (valid) p.lse[(long long)x * p.N + row] = (m2 + log2f(ssum)) * kLn2;
        }
        if (kTmaStore && r == 0) tc::bulk_wait_group<0>();
    }

    tc::fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) set_status(p.status, kDevTimeout);
    if (warp == 9) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool logits_tc_supported(int d, int Gk) { return d == kD && Gk >= 1 && Gk <= kMaxG; }

cudaError_t launch_logits_tc(const bf16* Q, const bf16* chi, const bf16* clo, const int32_t* koff, float* u,
                             float* lse, int* status, int B, int Hq, int Hkv, int N, int Gk, int num_sms,
                             cudaStream_t s) {
    const int G16 = (Gk + 15) / 16 * 16, G32 = (Gk + 31) / 32 * 32;
    const int Hp = B * Hq, P = B * Hkv;
    const bool tma_store = (Gk % 4) == 0;
    CUtensorMap mq, mh, ml, mu;
    memset(&mu, 0, sizeof(mu));
    if (!make_tmap_bf16_sw128(&mq, Q, (long long)Hp * N, kD, kRows, 64) ||
        !make_tmap_bf16_sw128(&mh, chi, (long long)P * Gk, kD, G16, 64) ||
        !make_tmap_bf16_sw128(&ml, clo, (long long)P * Gk, kD, G16, 64) ||
        (tma_store && !make_tmap_f32_3d_sw128(&mu, u, Gk, N, Hp, kRows)))
        return cudaErrorInvalidValue;
    LgParams p;
    memset(&p, 0, sizeof(p));
    p.u = u; p.lse = lse; p.koff = koff; p.status = status;
    p.N = N; p.g = Hq / Hkv; p.Gk = Gk; p.G16 = G16; p.G32 = G32;
    p.scale = (float)(1.0 / sqrt((double)kD));
    const int tiles = (N + kRows - 1) / kRows;
    int per = num_sms / Hp;
    if (per < 1) per = 1;
    if (per > tiles) per = tiles;
    const dim3 grid(per, Hp);
    cudaError_t e;
    if (tma_store) {
        e = cudaFuncSetAttribute(logits_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        logits_tc_kernel<true><<<grid, kThreads, kSmemBytes, s>>>(mq, mh, ml, mu, p);
    } else {
        e = cudaFuncSetAttribute(logits_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        logits_tc_kernel<false><<<grid, kThreads, kSmemBytes, s>>>(mq, mh, ml, mu, p);
    }
    return cudaGetLastError();
}

}  // namespace spr
