// Correction and write-back on 5th-generation tensor cores (d = 128): for every row o of the sparse
// output in group-major order ([probe]: the fitted correction projected onto the residual
// subspace, [execution]: results return to the original token order)
//   t = c0 + Bm o   (r values, Bm = U^T A),   O[qperm[p]] = o + U t (+ Rbar, ablation),
// where the two products are dense contractions of rank r (16 or 32) over 128-row tiles:
//   MMA 1: T = O_s Bm^T      (M = 128, N = RP, K = 128; Bm as two bf16 parts, O_s exact in bf16)
//   MMA 2: D = T U^T         (M = 128, N = 128, K = RP; T and U as two bf16 parts each, three
//                             terms, T read from TMEM as bf16 pairs)
// so the per-element error is about 2^-16 of the correction, far below the bf16 output rounding.
// Persistent CTAs walk 128-row tiles of all query heads in contiguous ranges; a row tile of O_s
// and its head's Bm / U^T parts arrive together by TMA; one thread issues the MMAs; two epilogue
// warpgroups take alternate tiles (thread r <-> row r <-> TMEM lane r): they turn T into c0 + T
// split into bf16 parts (written back to TMEM), then add D to the row of O_s (read from the
// staged tile) and stage the bf16 row in shared memory; each warp then writes whole 256-byte
// rows at their original indices (one coalesced row per store instruction).
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
constexpr int kRegion = kRows * 128;       // [128 rows][64 bf16], 128B swizzle
constexpr int kThreads = 320;              // warps 0-7 epilogue, 8 TMA, 9 MMA
constexpr uint32_t kTmemCols = 512;        // per warpgroup b: D [256b, +128), T [+128, +RP), parts [+160, +RP)

template <int RP>
struct WbLayout {
    static constexpr int kBReg = RP * 128;                     // [RP rows][64 bf16]
    static constexpr int kOffO = 0;                            // O_s tile: 2 regions
    static constexpr int kOffBm = 2 * kRegion;                 // Bm hi, lo: 2 regions each
    static constexpr int kOffUt = kOffBm + 4 * kBReg;          // U^T hi, lo: 2 regions each
    static constexpr int kStage = kOffUt + 4 * kBReg;
    static constexpr int kStages = RP == 16 ? 3 : 2;
    static constexpr int kOffStg = kStages * kStage;            // output rows of each warpgroup: [2][128][256 B]
    static constexpr int kOffDst = kOffStg + 2 * kRows * 256;   // their original row indices: [2][128] int
    static constexpr int kOffBar = kOffDst + 2 * kRows * 4;
    // barriers: full[S], empty[S] (128 epilogue arrivals... per warpgroup tile), tfull[2], tready[2],
    // dfull[2], tmem_empty[2], mma
    static constexpr int kBarF = 0, kBarE = kStages, kBarTF = 2 * kStages, kBarTR = kBarTF + 2, kBarDF = kBarTR + 2,
                         kBarTE = kBarDF + 2, kBarMma = kBarTE + 2, kNumBars = kBarMma + 1;
    static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
    static constexpr int kSmem = kOffMisc + 16 + 1024;
};
static_assert(WbLayout<16>::kSmem <= 232448 && WbLayout<32>::kSmem <= 232448, "shared memory budget");

struct WbParams {
    const int32_t* qperm;   // [P][N]
    const float* c0;        // [Hp][r]
    const float* Radd;      // [Hp][d] or null
    bf16* O;                // [Hp][N][d], original order
    int* status;
    int Hp, g, N, r, tiles_per_head;
};

template <int RP>
__global__ void __launch_bounds__(kThreads, 1) wb_tc_kernel(const __grid_constant__ CUtensorMap tmO,
                                                            const __grid_constant__ CUtensorMap tmBh,
                                                            const __grid_constant__ CUtensorMap tmBl,
                                                            const __grid_constant__ CUtensorMap tmUh,
                                                            const __grid_constant__ CUtensorMap tmUl,
                                                            const WbParams p) {
    using L = WbLayout<RP>;
    if (p.status && *reinterpret_cast<volatile int*>(p.status) == kDevTimeout) return;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = tc::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* sbase = smem_raw + (base - raw);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + L::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + L::kOffMisc + 4);
    auto bar = [&](int i) { return base + L::kOffBar + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long total = (long long)p.Hp * p.tiles_per_head;
    const int t0 = (int)(total * blockIdx.x / gridDim.x), t1 = (int)(total * (blockIdx.x + 1) / gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < L::kStages; ++s) {
            tc::mbar_init(bar(L::kBarF + s), 1);
            tc::mbar_init(bar(L::kBarE + s), 128);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(bar(L::kBarTF + b), 1);
            tc::mbar_init(bar(L::kBarTR + b), 128);
            tc::mbar_init(bar(L::kBarDF + b), 1);
            tc::mbar_init(bar(L::kBarTE + b), 128);
        }
        tc::mbar_init(bar(L::kBarMma), 1);
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
        // ================= TMA producer: O_s tile + its head's Bm and U^T parts
        if (lane == 0) {
            const uint32_t bytes = 2u * kRegion + 8u * (uint32_t)L::kBReg;
            int i = 0;
            for (int t = t0; t < t1; ++t, ++i) {
                const int s = i % L::kStages;
                if (i >= L::kStages && !tc::mbar_wait(bar(L::kBarE + s), ((i / L::kStages) - 1) & 1, abort_flag))
                    break;
                const int x = t / p.tiles_per_head, rt = t % p.tiles_per_head;
                const uint32_t st = base + s * L::kStage;
                const uint32_t b = bar(L::kBarF + s);
                tc::mbar_arrive_expect_tx(b, bytes);
                for (int h = 0; h < 2; ++h) {
                    tc::tma_load_2d(st + L::kOffO + h * kRegion, &tmO, b, 64 * h, x * p.N + rt * kRows);
                    tc::tma_load_2d(st + L::kOffBm + h * L::kBReg, &tmBh, b, 64 * h, x * RP);
                    tc::tma_load_2d(st + L::kOffBm + (2 + h) * L::kBReg, &tmBl, b, 64 * h, x * RP);
                    tc::tma_load_2d(st + L::kOffUt + h * L::kBReg, &tmUh, b, 64 * h, x * RP);
                    tc::tma_load_2d(st + L::kOffUt + (2 + h) * L::kBReg, &tmUl, b, 64 * h, x * RP);
                }
            }
            int never = 0;
            for (int k = (i > L::kStages ? i - L::kStages : 0); k < i; ++k)
                tc::mbar_wait(bar(L::kBarF + k % L::kStages), (k / L::kStages) & 1, &never);
        }
    } else if (warp == 9) {
        // ================= MMA issuer: MMA 1 of tile i, then MMA 2 of tile i - 1
        const uint32_t id1 = tc::idesc_bf16_f32(kRows, RP, 0);
        const uint32_t id2 = tc::idesc_bf16_f32(kRows, kD, 1);
        bool ok = true;
        auto mma2 = [&](int i) -> bool {
            const int s = i % L::kStages, b = i & 1;
            if (!__all_sync(kFull, tc::mbar_wait(bar(L::kBarTR + b), (i >> 1) & 1, abort_flag))) return false;
            tc::fence_after_sync();
            if (lane == 0) {
                const uint32_t st = base + s * L::kStage;
                const uint32_t dD = tmem + (uint32_t)(256 * b);
                const uint32_t th = dD + 160, tl = dD + 192;      // T parts as bf16 pairs
#pragma unroll
                for (int k = 0; k < RP / 16; ++k) {
                    const uint64_t uh = tc::smem_desc_sw128(st + L::kOffUt + k * 2048, L::kBReg, 1024);
                    const uint64_t ul = tc::smem_desc_sw128(st + L::kOffUt + 2 * L::kBReg + k * 2048, L::kBReg, 1024);
                    tc::mma_f16_ts(dD, th + 8 * k, uh, id2, k > 0 ? 1u : 0u);
                    tc::mma_f16_ts(dD, th + 8 * k, ul, id2, 1u);
                    tc::mma_f16_ts(dD, tl + 8 * k, uh, id2, 1u);
                }
                tc::commit(bar(L::kBarDF + b));
            }
            __syncwarp();
            return true;
        };
        int i = 0;
        for (int t = t0; ok && t < t1; ++t, ++i) {
            const int s = i % L::kStages, b = i & 1;
            if (!__all_sync(kFull, tc::mbar_wait(bar(L::kBarF + s), (i / L::kStages) & 1, abort_flag))) break;
            if (i >= 2 && !__all_sync(kFull, tc::mbar_wait(bar(L::kBarTE + b), ((i >> 1) - 1) & 1, abort_flag)))
                break;
            tc::fence_after_sync();
            if (lane == 0) {
                const uint32_t st = base + s * L::kStage;
                const uint32_t dT = tmem + (uint32_t)(256 * b + 128);
#pragma unroll
                for (int k = 0; k < kD / 16; ++k) {
                    const uint32_t off = (uint32_t)((k >> 2) * kRegion + (k & 3) * 32);
                    const uint32_t boff = (uint32_t)((k >> 2) * L::kBReg + (k & 3) * 32);
                    const uint64_t a = tc::smem_desc_sw128(st + L::kOffO + off, 16, 1024);
                    tc::mma_f16_ss(dT, a, tc::smem_desc_sw128(st + L::kOffBm + boff, 16, 1024), id1, k > 0 ? 1u : 0u);
                    tc::mma_f16_ss(dT, a, tc::smem_desc_sw128(st + L::kOffBm + 2 * L::kBReg + boff, 16, 1024), id1,
                                   1u);
                }
                tc::commit(bar(L::kBarTF + b));
            }
            __syncwarp();
            if (i >= 1) ok = mma2(i - 1);
        }
        if (ok && i >= 1) mma2(i - 1);
        if (lane == 0) tc::commit(bar(L::kBarMma));
        __syncwarp();
        int never = 0;
        tc::mbar_wait(bar(L::kBarMma), 0, &never);
    } else {
        // ================= epilogue warpgroup wg: tiles i with i % 2 == wg
        const int wg = warp >> 2, r = threadIdx.x & 127;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tD = tmem + (uint32_t)(256 * wg) + lane_off;
        int i = wg;
        for (int t = t0 + wg; t < t1; t += 2, i += 2) {
            const int s = i % L::kStages;
            const int x = t / p.tiles_per_head, rt = t % p.tiles_per_head, z = x / p.g;
            const int row = rt * kRows + r;
            const bool valid = row < p.N;
            // the original index of this row and the head's c0 are fetched before waiting
            const int dst = valid ? __ldg(p.qperm + (long long)z * p.N + row) : 0;
            if (!__all_sync(kFull, tc::mbar_wait(bar(L::kBarTF + wg), (i >> 1) & 1, abort_flag))) break;
            tc::fence_after_sync();
            {
                uint32_t tv[32];
                tc::tmem_ld32(tD + 128, tv);
                tc::tmem_wait_ld();
                tc::regs_after_wait(tv);
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) { hi[k] = 0u; lo[k] = 0u; }
#pragma unroll
                for (int k2 = 0; k2 < RP / 2; ++k2) {
                    float tk[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int k = 2 * k2 + e;
                        tk[e] = k < p.r ? __uint_as_float(tv[k]) + __ldg(p.c0 + (long long)x * p.r + k) : 0.f;
                    }
                    const bf16 h0 = __float2bfloat16_rn(tk[0]), h1 = __float2bfloat16_rn(tk[1]);
                    const bf16 l0 = __float2bfloat16_rn(tk[0] - __bfloat162float(h0));
                    const bf16 l1 = __float2bfloat16_rn(tk[1] - __bfloat162float(h1));
                    hi[k2] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
                    lo[k2] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
                }
                tc::tmem_st16(tD + 160, hi);
                tc::tmem_st16(tD + 192, lo);
                tc::tmem_wait_st();
            }
            tc::fence_before_sync();
            tc::mbar_arrive(bar(L::kBarTR + wg));
            if (!__all_sync(kFull, tc::mbar_wait(bar(L::kBarDF + wg), (i >> 1) & 1, abort_flag))) break;
            tc::fence_after_sync();
            const unsigned char* orow = sbase + s * L::kStage + L::kOffO + r * 128;
            // staging row r of this warpgroup: 16-byte chunk c at (c ^ (r & 15)) (fewer bank conflicts)
            unsigned char* stg = sbase + L::kOffStg + wg * (kRows * 256) + r * 256;
            reinterpret_cast<int*>(sbase + L::kOffDst)[wg * kRows + r] = valid ? dst : -1;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t dv[32];
                tc::tmem_ld32(tD + 32 * c, dv);
                tc::tmem_wait_ld();
                tc::regs_after_wait(dv);
                // columns 32c .. 32c+31: region c / 2, 16-byte chunks (c % 2) * 4 .. + 3 (swizzled)
                const unsigned char* reg = orow + (c >> 1) * kRegion;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int chunk = (c & 1) * 4 + q;
                    const uint4 ov = *reinterpret_cast<const uint4*>(reg + ((chunk ^ (r & 7)) << 4));
                    const uint32_t w[4] = {ov.x, ov.y, ov.z, ov.w};
                    uint32_t res[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int col = 32 * c + 8 * q + 2 * e;
                        const float2 o2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
                        float a0 = o2.x + __uint_as_float(dv[8 * q + 2 * e]);
                        float a1 = o2.y + __uint_as_float(dv[8 * q + 2 * e + 1]);
                        if (p.Radd) {
                            a0 += __ldg(p.Radd + (long long)x * kD + col);
                            a1 += __ldg(p.Radd + (long long)x * kD + col + 1);
                        }
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(a0, a1);
                        res[e] = *reinterpret_cast<uint32_t*>(&b2);
                    }
                    const int oc = 4 * c + q;   // output chunk 0..15
                    *reinterpret_cast<uint4*>(stg + ((oc ^ (r & 15)) << 4)) = make_uint4(res[0], res[1], res[2], res[3]);
                }
            }
            tc::fence_before_sync();
            tc::mbar_arrive(bar(L::kBarTE + wg));
            tc::mbar_arrive(bar(L::kBarE + s));
            tc::named_bar_sync(1 + wg, 128);
            // each warp writes rows wl, wl + 4, ...: lane l the bytes [8l, 8l + 8) of the row
            {
                const int wl = warp & 3;
                const unsigned char* sw = sbase + L::kOffStg + wg * (kRows * 256);
                const int* sd = reinterpret_cast<const int*>(sbase + L::kOffDst) + wg * kRows;
                const int ch = lane >> 1, half = lane & 1;
                for (int rr = wl; rr < kRows; rr += 4) {
                    const int d = sd[rr];
                    if (d < 0) continue;
                    const uint2 v = *reinterpret_cast<const uint2*>(sw + rr * 256 + ((ch ^ (rr & 15)) << 4) + half * 8);
                    *reinterpret_cast<uint2*>(p.O + ((long long)x * p.N + d) * kD + lane * 4) = v;
                }
            }
            tc::named_bar_sync(1 + wg, 128);   // the staging rows are free for this warpgroup's next tile
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) set_status(p.status, kDevTimeout);
    if (warp == 9) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// Bm [Hp][r][d] and U [Hp][d][r] (fp32) -> bf16 parts of Bm and of U^T, [Hp][RP][d] each, rows
// >= r zero.
__global__ void wb_split_kernel(const float* __restrict__ Bm, const float* __restrict__ U, bf16* Bh, bf16* Bl,
                                bf16* Uh, bf16* Ul, int r, int RP) {
    const int x = blockIdx.x;
    for (int t = threadIdx.x; t < RP * kD; t += blockDim.x) {
        const int k = t / kD, c = t % kD;
        const float b = k < r ? Bm[((long long)x * r + k) * kD + c] : 0.f;
        const float u = k < r ? U[((long long)x * kD + c) * r + k] : 0.f;
        const long long o = (long long)x * RP * kD + t;
        const bf16 bh = __float2bfloat16_rn(b), uh = __float2bfloat16_rn(u);
        Bh[o] = bh;
        Bl[o] = __float2bfloat16_rn(b - __bfloat162float(bh));
        Uh[o] = uh;
        Ul[o] = __float2bfloat16_rn(u - __bfloat162float(uh));
    }
}

template <int RP>
cudaError_t launch_wb(const bf16* Osp, const bf16* parts, const WbParams& p, int num_sms, cudaStream_t s) {
    using L = WbLayout<RP>;
    const long long per = (long long)p.Hp * RP * kD;
    CUtensorMap mo, bh, bl, uh, ul;
    if (!make_tmap_bf16_sw128(&mo, Osp, (long long)p.Hp * p.N, kD, kRows, 64) ||
        !make_tmap_bf16_sw128(&bh, parts, (long long)p.Hp * RP, kD, RP, 64) ||
        !make_tmap_bf16_sw128(&bl, parts + per, (long long)p.Hp * RP, kD, RP, 64) ||
        !make_tmap_bf16_sw128(&uh, parts + 2 * per, (long long)p.Hp * RP, kD, RP, 64) ||
        !make_tmap_bf16_sw128(&ul, parts + 3 * per, (long long)p.Hp * RP, kD, RP, 64))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(wb_tc_kernel<RP>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    const long long total = (long long)p.Hp * p.tiles_per_head;
    const int grid = (int)(total < num_sms ? total : num_sms);
    wb_tc_kernel<RP><<<grid, kThreads, L::kSmem, s>>>(mo, bh, bl, uh, ul, p);
    return cudaGetLastError();
}

}  // namespace

bool wb_tc_supported(int d, int r) { return d == kD && r >= 1 && r <= 32; }

size_t wb_tc_parts_elems(int Hp) { return (size_t)4 * Hp * 32 * kD; }

cudaError_t launch_writeback_tc(const bf16* Osp, const int32_t* qperm, const float* U, const float* Bm,
                                const float* c0, const float* Radd, bf16* parts, bf16* O, int Hp, int g, int N, int r,
                                int* status, int num_sms, cudaStream_t s) {
    if (!wb_tc_supported(kD, r)) return cudaErrorInvalidValue;
    const int RP = r <= 16 ? 16 : 32;
    const long long per = (long long)Hp * RP * kD;
    wb_split_kernel<<<Hp, 256, 0, s>>>(Bm, U, parts, parts + per, parts + 2 * per, parts + 3 * per, r, RP);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    WbParams p;
    memset(&p, 0, sizeof(p));
    p.qperm = qperm; p.c0 = c0; p.Radd = Radd; p.O = O; p.status = status;
    p.Hp = Hp; p.g = g; p.N = N; p.r = r; p.tiles_per_head = (N + kRows - 1) / kRows;
    return RP == 16 ? launch_wb<16>(Osp, parts, p, num_sms, s) : launch_wb<32>(Osp, parts, p, num_sms, s);
}

}  // namespace spr
