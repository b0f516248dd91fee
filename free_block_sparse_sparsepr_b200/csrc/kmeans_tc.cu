// Lloyd assignment step on 5th-generation tensor cores (G <= 256 groups), certified against
// the fp32 value of the exact distance.
//
// For a tile of 128 rows the dot products with every centroid form one 128 x G x D GEMM.
// Rows and centroids are split into two bf16 parts (x = x0 + x1 + e, |e| <= 2^-16 |x|
// elementwise) and the three terms x0 c0 + x0 c1 + x1 c0 are accumulated in fp32 TMEM, so
// each dot product is known to within about 2^-14 ||x|| ||c||. One more K = 16 step multiplies
// a constant tile of ones (columns 0-2) by the three bf16 parts of -||c_g||^2 / 2, so the
// accumulator holds v_g = x.c_g - ||c_g||^2 / 2 = (||x||^2 - dd_g) / 2 and the nearest centroid
// is the largest v. One epilogue thread per row reads v straight from its TMEM lane, 32
// columns at a time, keeps the largest v of every chunk (three-input maxima) and a register
// copy of the chunk holding the largest so far, from which come the argmax (lowest column on
// ties) and the count of values within the certificate's gap (half the gap in dd) of it.
// When no other distance (in that chunk, or as another chunk's minimum) lies within a bound on
// the estimate's error, the estimate decides; otherwise (about 1% of rows) the row goes to a
// list that the same CTA settles exactly at its end: an fp32 pass over all centroids keeps
// those within a relative 1e-4 of the nearest, and each of those gets ||x||^2 - 2 x.c + ||c||^2
// in fp64 from the fp32 rows and centroids, rounded to fp32, ties to the lowest group. The
// labels are therefore those of the fp32 distances themselves.
//
// Warps 0-7 epilogue (two warpgroups taking alternate tiles, one TMEM buffer each), warp 8
// TMA producer (centroids once, row tiles in a 3-stage ring), warp 9 MMA issuer; all ten warps
// share the exact settlement of the flagged rows at the end.
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
constexpr int kCols = 64;                 // feature width of one 128-byte swizzle row
constexpr int kMaxG = 256;
constexpr int kMaxDP = 64;
constexpr int kTile = kRows * kCols * 2;  // 16 KB per part per row tile
constexpr int kParts = 2;
constexpr int kStages = 3;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;

constexpr int kOffC = 0;                                     // part q at kOffC + q * kMaxG * 128
constexpr int kOffX = kOffC + kParts * kMaxG * 128;          // stage s, part q at + (s * kParts + q) * kTile
constexpr int kOffOnes = kOffX + kStages * kParts * kTile;   // [128][64] bf16, ones in columns 0-2
constexpr int kOffCCt = kOffOnes + kTile;                     // [kMaxG][64] bf16, -||c||^2/2 in three parts
constexpr int kOffCC = kOffCCt + kMaxG * 128;                 // kMaxG floats
constexpr int kOffBar = kOffCC + kMaxG * 4;
constexpr int kBarC = 0, kBarXF = 1, kBarXE = kBarXF + kStages, kBarDF = kBarXE + kStages, kBarDE = kBarDF + 2,
              kBarMma = kBarDE + 2, kNumBars = kBarMma + 1;
constexpr int kOffMisc = kOffBar + 8 * kNumBars;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Gap in dd below which a row is recomputed exactly: 4 kKappa ||x|| max_g ||c_g|| covers twice
// the error of two dot-product estimates (each at most ~3.1 * 2^-16 ||x|| ||c|| from the
// dropped split terms plus fp32 accumulation); kSlack (||x||^2 + max ||c||^2) covers the fp32
// rounding of ||c||^2, its three-part bf16 split (about 2^-24 ||c||^2) and the fp32
// accumulation of v, with a wide margin.
constexpr float kKappa = 1.0f / 8192.0f;   // 2^-13
constexpr float kSlack = 1.0f / 32768.0f;  // 2^-15
// ||c||^2 of padding columns: finite (so its bf16 parts never form a NaN) and far above any distance.
constexpr float kFar = 1.0e37f;

struct KmParams {
    const float* X;        // [P][n][DP] fp32 rows
    const float* C;        // [P][G][DP] fp32 centroids
    const float* xx;       // [P][n]
    const float* cc;       // [P][G32]  ||c||^2, +inf past G
    int32_t* labels;       // [P][n]
    int* changed;          // [P]
    const int* done;       // [P] or null
    int* status;
    int4* fix;             // flagged rows {row, previous label, estimate, chunk mask}; fix_cap slots per CTA
    int n, G, G16, G32, DP, ksteps, first, fix_cap;
};

struct KmMaps {
    CUtensorMap x[kParts];   // row parts [P*n][DP] bf16 (columns DP..63 of a box read as zero)
    CUtensorMap c[kParts];   // centroid parts [P*G16][64] bf16
};

// Three-input fp32 maximum.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}


template <int DP>
__device__ __forceinline__ void settle_row(const int4 h, const float* __restrict__ X, const float* sCk,
                                           const float* sCC, float cmax2, int G, int32_t* labels, int* changed,
                                           int z, int lane);

template <int DP>
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
    int* sFix = reinterpret_cast<int*>(sbase + kOffMisc + 8);
    // This CTA's region of the flagged-row list: one slot per row it can own.
    const int cta = z * gridDim.x + blockIdx.x;
    int4* fix = p.fix + (long long)cta * p.fix_cap;
    auto bar = [&](int i) { return base + kOffBar + 8u * (uint32_t)i; };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles = (p.n + kRows - 1) / kRows;

    for (int t = threadIdx.x; t < kMaxG; t += kThreads) sCC[t] = t < p.G32 ? p.cc[(long long)z * p.G32 + t] : kFar;
    // The two constant operands of the extra K step, written in the 128-byte swizzled layout
    // (16-byte chunk k of row r at chunk k ^ (r % 8)): row r of the ones tile holds 1, 1, 1 in
    // columns 0-2, row g of the other the bf16 parts of -||c_g||^2 / 2; every other element is 0.
    {
        uint4* ones = reinterpret_cast<uint4*>(sbase + kOffOnes);
        uint4* cct = reinterpret_cast<uint4*>(sbase + kOffCCt);
        const uint32_t one = 0x3F80u;   // bf16 1.0
        for (int q = threadIdx.x; q < kRows * 8 + p.G16 * 8; q += kThreads) {
            const bool isc = q >= kRows * 8;
            const int row = (isc ? q - kRows * 8 : q) >> 3, k = (q & 7) ^ (row & 7);
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (k == 0) {
                if (!isc) {
                    v.x = one | (one << 16);
                    v.y = one;
                } else {
                    const float a = -0.5f * p.cc[(long long)z * p.G32 + row];
                    const bf16 h0 = __float2bfloat16_rn(a);
                    const float r1 = a - __bfloat162float(h0);
                    const bf16 h1 = __float2bfloat16_rn(r1);
                    const bf16 h2 = __float2bfloat16_rn(r1 - __bfloat162float(h1));
                    v.x = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
                    v.y = (uint32_t)__bfloat16_as_ushort(h2);
                }
            }
            (isc ? cct : ones)[isc ? q - kRows * 8 : q] = v;
        }
        tc::fence_proxy_async_smem();
    }
    if (threadIdx.x == 0) {
        *sFix = 0;
        tc::mbar_init(bar(kBarC), 1);
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(bar(kBarXF + s), 1);
            tc::mbar_init(bar(kBarXE + s), 1);
        }
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
            tc::mbar_arrive_expect_tx(bar(kBarC), (uint32_t)kParts * (uint32_t)p.G16 * 128u);
            for (int q = 0; q < kParts; ++q)
                tc::tma_load_2d(base + kOffC + q * kMaxG * 128, &maps.c[q], bar(kBarC), 0, z * p.G16);
            int i = 0;
            for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
                const int s = i % kStages, u = i / kStages;
                if (u >= 1 && !tc::mbar_wait(bar(kBarXE + s), (u - 1) & 1, abort_flag)) break;
                const uint32_t dx = base + kOffX + s * kParts * kTile;
                const int row = z * p.n + t * kRows;
                tc::mbar_arrive_expect_tx(bar(kBarXF + s), kParts * kTile);
                for (int q = 0; q < kParts; ++q) tc::tma_load_2d(dx + q * kTile, &maps.x[q], bar(kBarXF + s), 0, row);
            }
            int never = 0;
            for (int k = (i > kStages ? i - kStages : 0); k < i; ++k)
                tc::mbar_wait(bar(kBarXF + k % kStages), (k / kStages) & 1, &never);
            tc::mbar_wait(bar(kBarC), 0, &never);
        }
    } else if (warp == 9) {
        const uint32_t idesc = tc::idesc_bf16_f32(kRows, p.G16, 0);
        bool ok = __all_sync(kFull, tc::mbar_wait(bar(kBarC), 0, abort_flag));
        int i = 0;
        for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++i) {
            const int s = i % kStages, b = i & 1;
            if (!__all_sync(kFull, tc::mbar_wait(bar(kBarXF + s), (i / kStages) & 1, abort_flag))) break;
            if (i >= 2 && !__all_sync(kFull, tc::mbar_wait(bar(kBarDE + b), ((i >> 1) - 1) & 1, abort_flag))) break;
            tc::fence_after_sync();
            if (lane == 0) {
                const uint32_t d = tmem + (uint32_t)(b * 256);
                const uint32_t xb = base + kOffX + s * kParts * kTile;
                for (int k = 0; k < p.ksteps; ++k) {
                    const uint32_t off = (uint32_t)(k * 32);
                    const uint64_t x0 = tc::smem_desc_sw128(xb + off, 16, 1024);
                    const uint64_t x1 = tc::smem_desc_sw128(xb + kTile + off, 16, 1024);
                    const uint64_t c0 = tc::smem_desc_sw128(base + kOffC + off, 16, 1024);
                    const uint64_t c1 = tc::smem_desc_sw128(base + kOffC + kMaxG * 128 + off, 16, 1024);
                    tc::mma_f16_ss(d, x0, c0, idesc, k > 0 ? 1u : 0u);
                    tc::mma_f16_ss(d, x0, c1, idesc, 1u);
                    tc::mma_f16_ss(d, x1, c0, idesc, 1u);
                }
                tc::mma_f16_ss(d, tc::smem_desc_sw128(base + kOffOnes, 16, 1024),
                               tc::smem_desc_sw128(base + kOffCCt, 16, 1024), idesc, 1u);
                tc::commit(bar(kBarXE + s));
                tc::commit(bar(kBarDF + b));
            }
            __syncwarp();
        }
        if (lane == 0) tc::commit(bar(kBarMma));
        __syncwarp();
        int never = 0;
        tc::mbar_wait(bar(kBarMma), 0, &never);
    } else {
        const int wg = warp >> 2, wr = (warp & 3) * 32;
        const uint32_t tb = tmem + (uint32_t)(wg * 256) + ((uint32_t)wr << 16);
        // Columns [G16, G32) are never written by the MMA: make them read as -kFar (never the largest).
        if (p.G16 < p.G32) {
            uint32_t zr[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) zr[e] = __float_as_uint(-kFar);
            tc::tmem_st16(tb + (uint32_t)p.G16, zr);
            tc::tmem_wait_st();
        }
        float cmax2 = 0.f;
        for (int g = lane; g < p.G; g += 32) cmax2 = fmaxf(cmax2, sCC[g]);
        cmax2 = warp_max(cmax2);   // the same value in every lane
        const float cmax = sqrtf(cmax2);
        for (int i = wg, t = blockIdx.x + wg * gridDim.x; t < tiles; i += 2, t += 2 * gridDim.x) {
            // The row's ||x||^2 and previous label are fetched before waiting for the tile.
            const int row = t * kRows + wr + lane;
            const bool valid = row < p.n;
            const long long o = (long long)z * p.n + row;
            const float xxr = valid ? __ldg(p.xx + o) : 0.f;
            const int prev = (valid && !p.first) ? p.labels[o] : -1;
            if (!__all_sync(kFull, tc::mbar_wait(bar(kBarDF + wg), (i >> 1) & 1, abort_flag))) break;
            tc::fence_after_sync();
            // One pass over the row's values, 32 columns (one TMEM load) at a time: the chunk's
            // largest v by three-input maxima and, when it is a new best (B1), the chunk's 32
            // values copied into `best` by predicated selects; B2c is the largest of the other
            // chunks' maxima. The near-tie count and the argmax (lowest column on ties) then come
            // from `best` in registers, with no second read of TMEM.
            float B1 = -INFINITY, B2c = -INFINITY;
            int cb = 0;
            float best[32], cm[kMaxG / 32];   // cm: every chunk's largest v
#pragma unroll
            for (int e = 0; e < 32; ++e) best[e] = -INFINITY;
#pragma unroll
            for (int e = 0; e < kMaxG / 32; ++e) cm[e] = -INFINITY;
            auto chunk = [&](const uint32_t* v, int c, float& cmax_c) {
                auto vv = [&](int e) { return __uint_as_float(v[e]); };
                float mm[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mm[j] = fmax3(fmax3(vv(j), vv(j + 4), vv(j + 8)), fmax3(vv(j + 12), vv(j + 16), vv(j + 20)),
                                  fmaxf(vv(j + 24), vv(j + 28)));
                const float mc = fmaxf(fmax3(mm[0], mm[1], mm[2]), mm[3]);
                cmax_c = mc;
                const bool nb = mc > B1;
                B2c = nb ? B1 : fmaxf(B2c, mc);
                B1 = nb ? mc : B1;
                cb = nb ? c : cb;
#pragma unroll
                for (int e = 0; e < 32; ++e) best[e] = nb ? vv(e) : best[e];
            };
            {
                uint32_t va[32], vb[32];
                tc::tmem_ld32(tb, va);
                tc::tmem_wait_ld();
                tc::regs_after_wait(va);
#pragma unroll
                for (int q = 0; q < kMaxG / 64; ++q) {
                    const int c = 64 * q;
                    if (c < p.G32) {
                        const bool hb = c + 32 < p.G32, ha = c + 64 < p.G32;
                        if (hb) tc::tmem_ld32(tb + (uint32_t)(c + 32), vb);
                        chunk(va, c, cm[2 * q]);
                        if (hb) {
                            tc::tmem_wait_ld();
                            tc::regs_after_wait(vb);
                            if (ha) tc::tmem_ld32(tb + (uint32_t)(c + 64), va);
                            chunk(vb, c + 32, cm[2 * q + 1]);
                            if (ha) {
                                tc::tmem_wait_ld();
                                tc::regs_after_wait(va);
                            }
                        }
                    }
                }
            }
            // T bounds the error of a difference of two dd estimates; differences of v are half those of dd
            const float Th = 0.5f * (4.f * kKappa * sqrtf(xxr) * cmax + kSlack * (xxr + cmax2));
            const float thr = B1 - Th;
            int idx = 31;
            float near = 0.f;
#pragma unroll
            for (int e = 31; e >= 0; --e) {
                idx = best[e] == B1 ? e : idx;
                near += best[e] >= thr ? 1.f : 0.f;
            }
            const int I1 = min(cb + idx, p.G - 1);
            // Chunks that can hold the nearest centroid: a chunk whose largest v is more than the
            // gap below B1 holds only centroids certified farther than the estimated best.
            unsigned cmask = 0u;
#pragma unroll
            for (int e = 0; e < kMaxG / 32; ++e) cmask |= (cm[e] >= thr ? 1u : 0u) << e;
            tc::fence_before_sync();
            tc::mbar_arrive(bar(kBarDE + wg));

            const bool flag = valid && !(B1 - B2c > Th && near < 1.5f);
            // Hand each flagged row to the exact settlement at the end of the kernel.
            const unsigned fl = __ballot_sync(kFull, flag);
            if (fl) {
                int slot = 0;
                if (lane == 0) slot = atomicAdd(sFix, __popc(fl));
                slot = __shfl_sync(kFull, slot, 0) + __popc(fl & ((1u << lane) - 1u));
                if (flag) fix[slot] = make_int4((int)o, prev, I1, (int)cmask);
            }
            int moved = 0;
            if (valid) {
                if (!p.first && prev != I1) moved = 1;
                p.labels[o] = I1;
            }
            const unsigned bm = __ballot_sync(kFull, moved);
            if (lane == 0 && bm) atomicAdd(&p.changed[z], __popc(bm));
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) set_status(p.status, kDevTimeout);
    if (warp == 9) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
    // Exact settlement of this CTA's flagged rows, one warp per row. Every copy and MMA has
    // completed, so the row stages hold the fp32 centroids k-major ([DP][G]: lane g of a warp
    // reads centroid g's component k without bank conflicts).
    const int nfix = *sFix;
    if (nfix > 0 && !*abort_flag) {
        float* sCk = reinterpret_cast<float*>(sbase + kOffX);
        const float* src = p.C + (long long)z * p.G * DP;
        for (int t = threadIdx.x; t < p.G * DP; t += kThreads) sCk[(t % DP) * (p.G + 1) + t / DP] = __ldg(src + t);
        __syncthreads();
        float cmax2 = 0.f;
        for (int g = lane; g < p.G; g += 32) cmax2 = fmaxf(cmax2, sCC[g]);
        cmax2 = warp_max(cmax2);   // the same value in every lane
        for (int w = warp; w < nfix; w += kThreads / 32)
            settle_row<DP>(fix[w], p.X, sCk, sCC, cmax2, p.G, p.labels, p.changed, z, lane);
    }
}

// Exact label of one flagged row {row, previous label, estimate, chunk mask}, settled by one warp
// (centroids k-major in sCk with row stride G + 1, so staging and lane-parallel reads avoid bank
// conflicts; lane g + 32j takes centroid g + 32j). Only the 32-centroid chunks in the mask are
// screened: every centroid of another chunk is certified farther than the estimated best, so it
// can neither be the nearest nor tie with it. Candidates are the groups whose fp32 ||x||^2 - 2 x.c + ||c||^2
// (error below 2^-19 (||x||^2 + ||c||^2)) is within 1e-4 (|d_min| + ||x||^2 + max ||c||^2) of the
// smallest; each gets the fp32 value of its fp64 distance (butterfly sums, identical in every
// lane), argmin with ties to the lowest group. Corrects the label and the count of rows that
// moved.
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

template <int DP>
__device__ __forceinline__ void settle_row(const int4 h, const float* __restrict__ X, const float* sCk,
                                           const float* sCC, float cmax2, int G, int32_t* labels, int* changed,
                                           int z, int lane) {
    static_assert(DP <= 64, "two row components per lane");
    const long long o = h.x;
    const float* xr = X + o * DP;
    const float xa = lane < DP ? __ldg(xr + lane) : 0.f;
    const float xb = lane + 32 < DP ? __ldg(xr + lane + 32) : 0.f;
    const float xx = warp_sum(fmaf(xa, xa, xb * xb));
    const int nj = (G + 31) / 32;
    float dj[kMaxG / 32];
#pragma unroll
    for (int j = 0; j < kMaxG / 32; ++j) dj[j] = INFINITY;
    float dmin = INFINITY;
    // the row in every lane's registers, broadcast once
    float xv[DP];
#pragma unroll
    for (int k = 0; k < DP; ++k) xv[k] = __shfl_sync(kFull, k < 32 ? xa : xb, k & 31);
#pragma unroll 1
    for (int j = 0; j < kMaxG / 32; ++j) {
        if (j < nj && ((h.w >> j) & 1)) {
            const int g = 32 * j + lane;
            const int gc = g < G ? g : G - 1;
            float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < DP; ++k) a[k & 3] = fmaf(xv[k], sCk[k * (G + 1) + gc], a[k & 3]);
            const float dg = g < G ? fmaf(-2.f, (a[0] + a[1]) + (a[2] + a[3]), xx + sCC[g]) : INFINITY;
#pragma unroll
            for (int jj = 0; jj < kMaxG / 32; ++jj) dj[jj] = jj == j ? dg : dj[jj];
            dmin = fminf(dmin, dg);
        }
    }
    dmin = warp_min(dmin);
    const float thr = dmin + 1e-4f * (fabsf(dmin) + xx + cmax2);
    const double xxd = warp_sum_d(fma((double)xa, (double)xa, (double)xb * (double)xb));
    float best = INFINITY;
    int bg = h.z;
#pragma unroll
    for (int j = 0; j < kMaxG / 32; ++j) {
        if (j >= nj) break;
        unsigned m = __ballot_sync(kFull, dj[j] <= thr);
        while (m) {
            const int g = 32 * j + __ffs(m) - 1;
            m &= m - 1;
            const double ca = lane < DP ? (double)sCk[lane * (G + 1) + g] : 0.0;
            const double cb = lane + 32 < DP ? (double)sCk[(lane + 32) * (G + 1) + g] : 0.0;
            const double xc = warp_sum_d(fma((double)xa, ca, (double)xb * cb));
            const double ccd = warp_sum_d(fma(ca, ca, cb * cb));
            const float d = (float)fmax((xxd - 2.0 * xc) + ccd, 0.0);
            if (d < best || (d == best && g < bg)) { best = d; bg = g; }
        }
    }
    if (lane == 0) {
        labels[o] = bg;
        const int prev = h.y;
        if (prev >= 0) {
            const int dmoved = (prev != bg ? 1 : 0) - (prev != h.z ? 1 : 0);
            if (dmoved) atomicAdd(&changed[z], dmoved);
        }
    }
}

// The two bf16 parts of v: the bf16 rounding of v and of what it leaves.
__device__ __forceinline__ void split2(float v, bf16& a, bf16& b) {
    a = __float2bfloat16_rn(v);
    b = __float2bfloat16_rn(v - __bfloat162float(a));
}

// X [rows][DP] fp32 -> two bf16 parts [rows][DP] (part q at X2 + q*stride) and ||x||^2 in fp32;
// one warp per row.
constexpr int kSplitRowsPerWarp = 4;
__global__ void km_split_rows_kernel(const float* __restrict__ X, bf16* X2, long long stride, float* xx,
                                     long long rows, int DP) {
    const long long row0 = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * kSplitRowsPerWarp;
    const int lane = threadIdx.x & 31;
    if (row0 >= rows) return;
    float v[kSplitRowsPerWarp][2];
#pragma unroll
    for (int q = 0; q < kSplitRowsPerWarp; ++q)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = lane + 32 * h;
            v[q][h] = (row0 + q < rows && c < DP) ? __ldg(X + (row0 + q) * DP + c) : 0.f;
        }
#pragma unroll
    for (int q = 0; q < kSplitRowsPerWarp; ++q) {
        const long long row = row0 + q;
        if (row >= rows) break;
        float ss = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = lane + 32 * h;
            ss = fmaf(v[q][h], v[q][h], ss);
            if (c < DP) {
                bf16 a, b;
                split2(v[q][h], a, b);
                X2[row * DP + c] = a;
                X2[stride + row * DP + c] = b;
            }
        }
        ss = warp_sum(ss);
        if (lane == 0) xx[row] = ss;
    }
}

// C [P][G][DP] fp32 -> two bf16 parts [P][G16][64] (zero past G and DP, part q at C2 + q*stride)
// and ||c||^2 [P][G32] (kFar past G so padded columns never win).
__global__ void km_split_cent_kernel(const float* __restrict__ C, bf16* C2, long long stride, float* cc, int G,
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
            bf16 a, b;
            split2(v, a, b);
            const long long o = ((long long)z * G16 + g) * kCols + c;
            C2[o] = a;
            C2[stride + o] = b;
        }
    }
    ss = warp_sum(ss);
    if (lane == 0) cc[(long long)z * G32 + g] = g < G ? ss : kFar;
}

// dist[z][i] = fp32(max(||x||^2 - 2 x.c + ||c||^2, 0)) in fp64 for the row's own centroid;
// one thread per row.
__global__ void km_dist_kernel(const float* __restrict__ X, const float* __restrict__ C,
                               const int32_t* __restrict__ labels, float* dist, int n, int G, int DP) {
    const int z = blockIdx.y;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const long long o = (long long)z * n + i;
    const float4* xr = reinterpret_cast<const float4*>(X + o * DP);
    const float4* cr = reinterpret_cast<const float4*>(C + ((long long)z * G + labels[o]) * DP);
    double xx = 0.0, xc = 0.0, cc = 0.0;
    for (int k = 0; k < DP / 4; ++k) {
        const float4 a = xr[k], b = __ldg(cr + k);
        xx = fma((double)a.x, (double)a.x, xx); xx = fma((double)a.y, (double)a.y, xx);
        xx = fma((double)a.z, (double)a.z, xx); xx = fma((double)a.w, (double)a.w, xx);
        xc = fma((double)a.x, (double)b.x, xc); xc = fma((double)a.y, (double)b.y, xc);
        xc = fma((double)a.z, (double)b.z, xc); xc = fma((double)a.w, (double)b.w, xc);
        cc = fma((double)b.x, (double)b.x, cc); cc = fma((double)b.y, (double)b.y, cc);
        cc = fma((double)b.z, (double)b.z, cc); cc = fma((double)b.w, (double)b.w, cc);
    }
    dist[o] = (float)fmax((xx - 2.0 * xc) + cc, 0.0);
}

}  // namespace

bool km_tc_supported(int G) { return G >= 1 && G <= kMaxG; }

// Grid of the assignment: per CTAs for each of the P problems, each owning at most cap rows.
void km_grid(int P, int n, int num_sms, int* per, int* cap) {
    const int tiles = (n + kRows - 1) / kRows;
    int q = num_sms / P;
    if (q < 1) q = 1;
    if (q > tiles) q = tiles;
    *per = q;
    *cap = (tiles + q - 1) / q * kRows;
}

cudaError_t launch_km_split_rows(const float* X, bf16* X2, float* xx, int P, int n, int DP, cudaStream_t s) {
    const long long rows = (long long)P * n;
    const long long per_block = 8ll * kSplitRowsPerWarp;
    km_split_rows_kernel<<<(unsigned)((rows + per_block - 1) / per_block), 256, 0, s>>>(X, X2, rows * DP, xx, rows,
                                                                                        DP);
    return cudaGetLastError();
}

cudaError_t launch_km_split_cent(const float* C, bf16* C2, float* cc, int P, int G, int DP, cudaStream_t s) {
    const int G16 = (G + 15) / 16 * 16, G32 = (G + 31) / 32 * 32;
    km_split_cent_kernel<<<dim3((G32 + 7) / 8, P), 256, 0, s>>>(C, C2, (long long)P * G16 * kCols, cc, G, G16, G32,
                                                                 DP);
    return cudaGetLastError();
}

cudaError_t launch_km_assign_tc(const float* X, const bf16* X2, const float* xx, const float* C, const bf16* C2,
                                const float* cc, int32_t* labels, int* changed, const int* done, int4* fix,
                                int* status, int P, int n, int G, int DP, bool first, int num_sms, cudaStream_t s) {
    if (DP < 16 || DP > kMaxDP || DP % 16 != 0 || (long long)P * n >= (1ll << 31)) return cudaErrorInvalidValue;
    const int G16 = (G + 15) / 16 * 16, G32 = (G + 31) / 32 * 32;
    KmMaps maps;
    for (int q = 0; q < kParts; ++q) {
        if (!make_tmap_bf16_sw128(&maps.x[q], X2 + (long long)q * P * n * DP, (long long)P * n, DP, kRows, 64) ||
            !make_tmap_bf16_sw128(&maps.c[q], C2 + (long long)q * P * G16 * kCols, (long long)P * G16, kCols, G16, 64))
            return cudaErrorInvalidValue;
    }
    KmParams p;
    memset(&p, 0, sizeof(p));
    p.X = X; p.C = C; p.xx = xx; p.cc = cc; p.labels = labels; p.changed = changed; p.done = done;
    p.status = status; p.fix = fix;
    p.n = n; p.G = G; p.G16 = G16; p.G32 = G32; p.DP = DP; p.ksteps = DP / 16; p.first = first ? 1 : 0;
    int per, cap;
    km_grid(P, n, num_sms, &per, &cap);
    p.fix_cap = cap;
#define SPR_ASSIGN(DPV)                                                                                              \
    case DPV: {                                                                                                      \
        cudaError_t e = cudaFuncSetAttribute(km_assign_tc_kernel<DPV>, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                                             kSmemBytes);                                                            \
        if (e != cudaSuccess) return e;                                                                              \
        km_assign_tc_kernel<DPV><<<dim3(per, P), kThreads, kSmemBytes, s>>>(maps, p);                                \
        break;                                                                                                       \
    }
    switch (DP) {
        SPR_ASSIGN(16)
        SPR_ASSIGN(32)
        SPR_ASSIGN(48)
        SPR_ASSIGN(64)
        default: return cudaErrorInvalidValue;
    }
#undef SPR_ASSIGN
    return cudaGetLastError();
}

size_t km_fix_slots(int P, int n, int num_sms) {
    int per, cap;
    km_grid(P, n, num_sms, &per, &cap);
    return (size_t)P * per * cap;
}

cudaError_t launch_km_dist(const float* X, const float* C, const int32_t* labels, float* dist, int P, int n, int G,
                           int DP, cudaStream_t s) {
    if (DP % 4 != 0) return cudaErrorInvalidValue;
    km_dist_kernel<<<dim3((n + 255) / 256, P), 256, 0, s>>>(X, C, labels, dist, n, G, DP);
    return cudaGetLastError();
}

}  // namespace spr
