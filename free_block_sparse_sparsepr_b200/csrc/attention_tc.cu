// Exact softmax attention on 5th-generation tensor cores (d = 128): the
// block-sparse pass over each query group's kept key groups, renormalised over
// those keys only, and the dense baseline (one key range [0, N)).
//
// One CTA per pair of 128-row query tiles (t = 0, 1) of the same query group; both tiles
// stream the same 128-key K/V tiles. Ten warps:
//   warps 0-3 / 4-7  softmax + epilogue of tile 0 / tile 1: thread r owns query row r =
//              TMEM lane r. Per key tile it reads its row of S_t from TMEM into registers,
//              forms 2^(s c - m) against the running max, writes P_t as bf16 pairs into the first 64 columns of S_t's
//              own TMEM buffer, rescales its O_t row when the max grows by more than 2^8, and
//              finally normalises and stores O_t;
//   warp 8     TMA producer: both Q tiles once, then K and V tiles into rings of 2 and 3 stages;
//   warp 9     TMEM allocation and the MMA issue (one thread): S_t = Q_t K^T (A and B from
//              shared memory), O_t += P_t V (A from TMEM), completions via tcgen05.commit.
// The tensor core alternates between the tiles (PV_0(j), S_0(j+1), PV_1(j), S_1(j+1)), so one
// softmax warpgroup works while the other's MMAs run. S_t(j+1) overwrites the columns P_t(j)
// occupied only after PV_t(j) in issue order; its completion also tells softmax t that
// PV_t(j) is done, so O_t may be rescaled and P_t(j+1) written.
// Key tiles are cut from merged runs of consecutive kept key groups; keys past a run's end
// (the next group's, or zero fill past the tensor) are masked to -inf. A tile with at most 64
// valid keys is a half tile: its S and PV MMAs run with 64 keys and the softmax neither loads
// nor writes the other half. A query tile of at most 64 rows (a group's last) runs its MMAs
// with M = 64; its warpgroup then reads S and writes P with the 16-lane TMEM shapes, two rows
// per thread.
#include <cuda.h>
#include <float.h>
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_primitives.cuh"
#include "tmap.h"

namespace spr {
namespace {

constexpr int kBM = 128;            // rows per query tile (two tiles per CTA)
constexpr int kBN = 128;            // keys per tile
constexpr int kKStages = 2;         // K ring depth
constexpr int kVStages = 3;         // V ring depth (a V tile is freed a step later than a K tile)
constexpr int kRegion = 16384;      // one [128 rows][64 bf16] 128B-swizzled region
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512; // S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512)
constexpr float kRescaleLog2 = 8.f; // lazy rescale threshold (P <= 2^8)
constexpr float kRescaleMax = 256.f; // 2^kRescaleLog2
constexpr float kLn2 = 0.6931471805599453f;

constexpr int kOffQ = 0;                                   // tile t at + t * 2 * kRegion
constexpr int kOffK = kOffQ + 2 * 2 * kRegion;
constexpr int kOffV = kOffK + kKStages * 2 * kRegion;
constexpr int kOffBar = kOffV + kVStages * 2 * kRegion;
// barriers: q_full, k_full[KS], v_full[VS], k_empty[KS], v_empty[VS], s_full[2], p_full[2],
// o_last[2], mma_done. K and V stages are released separately: a K tile as soon as the last S MMA
// that reads it completes, a V tile after the last PV MMA. V(j) is read a step after K(j), so its
// ring is one stage deeper: the load of V(j + 3) has two steps to land instead of one.
constexpr int kBarQ = 0, kBarK = 1, kBarV = kBarK + kKStages, kBarEK = kBarV + kVStages, kBarEV = kBarEK + kKStages,
              kBarS = kBarEV + kVStages, kBarP = kBarS + 2, kBarO = kBarP + 2, kBarMma = kBarO + 2,
              kNumBars = kBarMma + 1;
constexpr int kOffMisc = kOffBar + 8 * kNumBars;          // tmem base (u32), abort flag (int)
constexpr int kOffML = kOffMisc + 16;                      // split mode: tile 1's running max and sum [2][128]
constexpr int kSmemBytes = kOffML + 2 * kBM * 4 + 1024;   // + slack to align the base to 1024
static_assert(kSmemBytes <= 232448, "shared memory budget");

enum { kModeSparse = 0, kModeDense = 1, kModeProbe = 2 };

struct TcParams {
    bf16* O;
    float* lse;
    const int32_t* qoff;
    const int32_t* tile_off;      // [P][Gq+1] CTA (query-tile pair) offsets per query group
    const int2* klist;            // key tiles (start row, valid keys) of every query group
    const int32_t* klist_off;     // [P][Gq+1] offsets into klist
    int* status;
    int N, g, Gq;
    int head_pairs;               // sparse mode, g even: one CTA = the same query tile of two query heads
    int half_tails;               // sparse mode: a last query tile of <= 64 rows (of one head, or of both in a head pair) is M = 64
    int stall;                    // test only: issue no loads (the first bounded wait runs out)
    // probe mode: M gathered rows per query head against key split blockIdx.x (chunk keys each);
    // unnormalised partial outputs [x][ns][M][d], running maxima (log2 units) and sums [x][ns][M]
    float* Opart;
    float* mpart;
    float* lpart;
    int M, ns, chunk;
    float scale_log2;
};

// Three-input fp32 maximum.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Half h (64 columns) of this thread's row of S from TMEM, keys at or past `lim` set to -inf;
// mx receives the half's raw maximum.
__device__ __forceinline__ void load_half(uint32_t tS, int h, int lim, uint32_t (&sv)[2][32], float& mx) {
#pragma unroll
    for (int c = 0; c < 2; ++c) tc::tmem_ld32(tS + 64 * h + 32 * c, sv[c]);
    tc::tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 2; ++c) tc::regs_after_wait(sv[c]);
    float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const int c0 = 64 * h + 32 * c;
        if (c0 + 32 > lim) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (c0 + i >= lim) sv[c][i] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int i = 0; i < 32; i += 2)
            pm[(i >> 1) & 3] = fmax3(pm[(i >> 1) & 3], __uint_as_float(sv[c][i]), __uint_as_float(sv[c][i + 1]));
    }
    mx = fmax3(fmaxf(pm[0], pm[1]), pm[2], pm[3]);
}

// Half h (64 columns) of this thread's row of S from TMEM, keys at or past `lim` set to -inf.
__device__ __forceinline__ void load_half_nomax(uint32_t tS, int h, int lim, uint32_t (&sv)[2][32]) {
#pragma unroll
    for (int c = 0; c < 2; ++c) tc::tmem_ld32(tS + 64 * h + 32 * c, sv[c]);
    tc::tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 2; ++c) tc::regs_after_wait(sv[c]);
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const int c0 = 64 * h + 32 * c;
        if (c0 + 32 > lim) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (c0 + i >= lim) sv[c][i] = __float_as_uint(-INFINITY);
        }
    }
}

// 2^x on the special-function unit (flushes results below 2^-126 to zero).
__device__ __forceinline__ float ex2_sfu(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Pairs of fp32 in one 64-bit register, for the packed f32x2 arithmetic of sm_100.
__device__ __forceinline__ uint64_t pk2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void up2(uint64_t v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// p = 2^(s c + neg_m) for a half row, packed as bf16 pairs (32 registers); pair sums into ps
// (four packed accumulators).
__device__ __forceinline__ void exp_half(const uint32_t (&sv)[2][32], float c_log2, float neg_m, uint32_t* pk,
                                         uint64_t* ps) {
    const uint64_t cc = pk2(c_log2, c_log2), nm = pk2(neg_m, neg_m);
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            float x0, x1;
            up2(fma2(pk2(__uint_as_float(sv[c][2 * e]), __uint_as_float(sv[c][2 * e + 1])), cc, nm), x0, x1);
            const float p0 = ex2_sfu(x0), p1 = ex2_sfu(x1);
            ps[e & 3] = add2(ps[e & 3], pk2(p0, p1));
            __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
            pk[16 * c + e] = *reinterpret_cast<uint32_t*>(&b2);
        }
}

// Key tile j of the CTA: start row and number of valid keys (<= kBN).
__device__ __forceinline__ int2 key_tile(const TcParams& p, int mode, const int2* list, int j) {
    if (mode == kModeDense) {
        const int st = j * kBN;
        return make_int2(st, min(kBN, p.N - st));
    }
    if (mode == kModeProbe) {
        const int st = blockIdx.x * p.chunk + j * kBN;
        return make_int2(st, min(kBN, min(p.N, (blockIdx.x + 1) * p.chunk) - st));
    }
    return list[j];
}

template <int MODE, int D>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                              const __grid_constant__ CUtensorMap tmK,
                                                              const __grid_constant__ CUtensorMap tmV,
                                                              const TcParams p) {
    static_assert(D == 64 || D == 128, "head dimension");
    constexpr int kNR = D / 64;          // 128-byte swizzle regions per row of a tile
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = tc::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* sbase = smem_raw + (base - raw);
    const uint32_t sQ = base + kOffQ, sK = base + kOffK, sV = base + kOffV;
    const uint32_t bars = base + kOffBar;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + kOffMisc + 4);
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Query tile t covers rows [qrow[t], qrow[t] + qn_t) of the flattened [B*Hq*N] query rows:
    // either two consecutive 128-row tiles of query head x, or (head pairs, grouped-query
    // attention with an even group) the same 128 rows of query heads x and x + 1, which share
    // the KV head, the query group and therefore every key tile.
    const int hp = p.head_pairs ? p.g / 2 : 1;
    const int z = p.head_pairs ? (int)blockIdx.y / hp : (int)blockIdx.y / p.g;
    const int x = p.head_pairs ? z * p.g + 2 * ((int)blockIdx.y % hp) : (int)blockIdx.y;
    // a CTA that timed out earlier in this launch (or call) makes the rest return at once
    if (p.status && *reinterpret_cast<volatile int*>(p.status) == kDevTimeout) return;

    // ---- which query tiles
    int qlo, qn0, qn1, a = 0, ntk = 0;
    // half0 / half1: query tile 0 / 1 is an M = 64 tile (rows in lanes 0-15 of each 32-lane
    // quarter, read and written with the 16-lane TMEM shapes)
    bool half0 = false, half1 = false;
    long long qrow[2];
    const int2* klist = nullptr;
    if (MODE == kModeSparse) {
        const int32_t* toff = p.tile_off + (long long)z * (p.Gq + 1);
        const int pair = blockIdx.x;
        if (pair >= toff[p.Gq]) return;
        a = upper_index(toff, p.Gq, pair);
        const int32_t* lo = p.klist_off + (long long)z * (p.Gq + 1);
        klist = p.klist + lo[a];
        ntk = lo[a + 1] - lo[a];
        const int32_t* qo = p.qoff + (long long)z * (p.Gq + 1);
        if (p.head_pairs) {
            // one 128-row tile of two heads per CTA; with half tails, a last tile of at most 64 rows
            // runs as two M = 64 tiles (one per head)
            const int c = pair - toff[a];
            qlo = qo[a] + c * kBM;
            qn0 = qn1 = min(kBM, qo[a + 1] - qlo);
            half0 = half1 = p.half_tails && qn0 <= kBM / 2;
            qrow[0] = (long long)x * p.N + qlo;
            qrow[1] = (long long)(x + 1) * p.N + qlo;
        } else {
            // the group's rows in pairs of 128-row tiles; with half tails, a last tile of at most
            // 64 rows (lone, or the second of its pair) runs as an M = 64 tile
            qlo = qo[a] + (pair - toff[a]) * 2 * kBM;
            const int rows = qo[a + 1] - qlo;
            qn0 = min(kBM, rows);
            qn1 = min(kBM, rows - kBM);
            half0 = p.half_tails && qn1 <= 0 && qn0 <= kBM / 2;
            half1 = p.half_tails && qn1 > 0 && qn1 <= kBM / 2;
            qrow[0] = (long long)x * p.N + qlo;
            qrow[1] = qrow[0] + kBM;
        }
    } else if (MODE == kModeProbe) {
        // the head's gathered probe rows (one tile, rows >= M zero) against keys of split blockIdx.x
        qlo = 0;
        qn0 = p.M;
        qn1 = 0;
        const int klo = blockIdx.x * p.chunk, khi = min(p.N, klo + p.chunk);
        ntk = khi > klo ? (khi - klo + kBN - 1) / kBN : 0;
        qrow[0] = (long long)x * kBM;
        qrow[1] = qrow[0];
    } else {
        qlo = blockIdx.x * 2 * kBM;
        if (qlo >= p.N) return;
        qn0 = min(kBM, p.N - qlo);
        qn1 = min(kBM, p.N - qlo - kBM);
        ntk = (p.N + kBN - 1) / kBN;
        qrow[0] = (long long)x * p.N + qlo;
        qrow[1] = qrow[0] + kBM;
    }
    const bool two = qn1 > 0;
    // split mode: a lone query tile with two or more key tiles. Both softmax warpgroups take
    // the same rows, warpgroup t the key tiles j with j % 2 == t, and warpgroup 0 merges the two
    // partial softmax states at the end, so the tensor core still alternates between two S tiles.
    const bool split = !two && ntk >= 2;
    // the M of the S and PV MMAs into S_t / O_t, and the softmax path of warpgroup t
    auto half_of = [&](int t) { return split ? half0 : (t ? half1 : half0); };

    // ---- set-up: barriers (thread 0), TMEM (warp 9)
    if (threadIdx.x == 0) {
        tc::mbar_init(bar(kBarQ), 1);
        for (int s = 0; s < kKStages; ++s) {
            tc::mbar_init(bar(kBarK + s), 1);
            tc::mbar_init(bar(kBarEK + s), 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            tc::mbar_init(bar(kBarV + s), 1);
            tc::mbar_init(bar(kBarEV + s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            tc::mbar_init(bar(kBarS + t), 1);
            tc::mbar_init(bar(kBarP + t), 128);
            tc::mbar_init(bar(kBarO + t), 1);
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
        // ================= TMA producer (with p.stall set it issues nothing, so the MMA warp's
        // wait for Q gives up after its bound and raises the abort flag; no copy is in flight)
        if (lane == 0 && !p.stall) {
            tc::mbar_arrive_expect_tx(bar(kBarQ), (two ? 2 : 1) * kNR * kRegion);
            for (int h = 0; h < kNR; ++h) tc::tma_load_2d(sQ + h * kRegion, &tmQ, bar(kBarQ), 64 * h, (int)qrow[0]);
            if (two)
                for (int h = 0; h < kNR; ++h)
                    tc::tma_load_2d(sQ + (2 + h) * kRegion, &tmQ, bar(kBarQ), 64 * h, (int)qrow[1]);
            // K runs one tile ahead of V: K(0), then K(j+1) before V(j).
            auto load = [&](int m, bool isv) -> bool {
                const int ns = isv ? kVStages : kKStages, s = m % ns;
                if (m >= ns && !tc::mbar_wait(bar((isv ? kBarEV : kBarEK) + s), ((m / ns) - 1) & 1, abort_flag))
                    return false;
                const int krow = z * p.N + key_tile(p, MODE, klist, m).x;
                const uint32_t d = (isv ? sV : sK) + s * 2 * kRegion;
                const uint32_t b = bar((isv ? kBarV : kBarK) + s);
                tc::mbar_arrive_expect_tx(b, kNR * kRegion);
                for (int h = 0; h < kNR; ++h) tc::tma_load_2d(d + h * kRegion, isv ? &tmV : &tmK, b, 64 * h, krow);
                return true;
            };
            int nk = 0, nv = 0;   // K and V tiles issued
            if (ntk > 0 && load(0, false)) nk = 1;
            for (int j = 0; nk > j && j < ntk; ++j) {
                if (j + 1 < ntk) {
                    if (!load(j + 1, false)) break;
                    nk = j + 2;
                }
                if (!load(j, true)) break;
                nv = j + 1;
            }
            // every issued load must land before the CTA can exit
            int never = 0;
            for (int m = (nk > kKStages ? nk - kKStages : 0); m < nk; ++m)
                tc::mbar_wait(bar(kBarK + m % kKStages), (m / kKStages) & 1, &never);
            for (int m = (nv > kVStages ? nv - kVStages : 0); m < nv; ++m)
                tc::mbar_wait(bar(kBarV + m % kVStages), (m / kVStages) & 1, &never);
            tc::mbar_wait(bar(kBarQ), 0, &never);
        }
    } else if (warp == 9) {
        // ================= MMA issuer
        // instruction descriptors of S_t (full and half key tile) and O_t by the M of tile t
        auto idS = [&](int t, bool half_keys) {
            return tc::idesc_bf16_f32(half_of(t) ? kBM / 2 : kBM, half_keys ? 64 : kBN, 0);
        };
        auto idO = [&](int t) { return tc::idesc_bf16_f32(half_of(t) ? kBM / 2 : kBM, D, 1); };
        // PV k-steps of key tile j (16 keys each): 4 for a half tile, else 8
        auto pv_steps = [&](int j) { return key_tile(p, MODE, klist, j).y <= 64 ? 4 : kBN / 16; };
        const int ntiles = two ? 2 : 1;
        bool have = ntk > 0;
        bool ok = __all_sync(kFull, tc::mbar_wait(bar(kBarQ), 0, abort_flag));
        auto issue_S = [&](int t, int j) {
            const uint32_t kb = sK + (j % kKStages) * 2 * kRegion;
            const uint32_t qb = sQ + (split ? 0 : t) * 2 * kRegion;
            const uint32_t id = idS(t, key_tile(p, MODE, klist, j).y <= 64);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint32_t off = (uint32_t)((k >> 2) * kRegion + (k & 3) * 32);
                tc::mma_f16_ss(tmem + (uint32_t)(t * 128), tc::smem_desc_sw128(qb + off, 16, 1024),
                               tc::smem_desc_sw128(kb + off, 16, 1024), id, k > 0 ? 1u : 0u);
            }
            tc::commit(bar(kBarS + t));
        };
        int j = 0;
        if (split) {
            // S_0(0) and S_1(1) first; then per key tile j (softmax t = j % 2): PV_t(j) and S_t(j + 2)
            for (int t = 0; t < 2 && ok; ++t) {
                ok = __all_sync(kFull, tc::mbar_wait(bar(kBarK + t), 0, abort_flag));
                if (!ok) break;
                tc::fence_after_sync();
                if (lane == 0) {
                    issue_S(t, t);
                    tc::commit(bar(kBarEK + t));
                }
                __syncwarp();
            }
            for (; ok && j < ntk; ++j) {
                const int t = j & 1, s = j % kVStages;
                const bool nh = j + 2 < ntk;
                if (!__all_sync(kFull, tc::mbar_wait(bar(kBarV + s), (j / kVStages) & 1, abort_flag))) break;
                if (nh && !__all_sync(kFull, tc::mbar_wait(bar(kBarK + ((j + 2) % kKStages)), ((j + 2) / kKStages) & 1,
                                                          abort_flag)))
                    break;
                if (!__all_sync(kFull, tc::mbar_wait(bar(kBarP + t), (j >> 1) & 1, abort_flag))) break;
                tc::fence_after_sync();
                if (lane == 0) {
                    const uint32_t vb = sV + s * 2 * kRegion;
                    const uint32_t pt = tmem + (uint32_t)(t * 128);
                    const int nk = pv_steps(j);
#pragma unroll
                    for (int k = 0; k < kBN / 16; ++k)
                        if (k < nk)
                            tc::mma_f16_ts(tmem + 256 + (uint32_t)(t * 128), pt + (uint32_t)(8 * k),
                                           tc::smem_desc_sw128(vb + (uint32_t)(k * 2048), kRegion, 1024), idO(t),
                                           (j >= 2 || k > 0) ? 1u : 0u);
                    tc::commit(bar(kBarEV + s));
                    if (nh) {
                        issue_S(t, j + 2);
                        tc::commit(bar(kBarEK + (j + 2) % kKStages));
                    } else {
                        tc::commit(bar(kBarO + t));
                    }
                }
                __syncwarp();
            }
            have = false;
        }
        if (ok && have) {
            ok = __all_sync(kFull, tc::mbar_wait(bar(kBarK), 0, abort_flag));
            if (ok) {
                tc::fence_after_sync();
                if (lane == 0) {
                    for (int t = 0; t < ntiles; ++t) issue_S(t, 0);
                    tc::commit(bar(kBarEK));
                }
                __syncwarp();
            }
        }
        while (ok && have) {
            const bool nhave = j + 1 < ntk;
            const int s = j % kVStages;
            if (!__all_sync(kFull, tc::mbar_wait(bar(kBarV + s), (j / kVStages) & 1, abort_flag))) break;
            if (nhave && !__all_sync(kFull, tc::mbar_wait(bar(kBarK + ((j + 1) % kKStages)), ((j + 1) / kKStages) & 1,
                                                         abort_flag)))
                break;
            for (int t = 0; t < ntiles && ok; ++t) {
                if (!__all_sync(kFull, tc::mbar_wait(bar(kBarP + t), j & 1, abort_flag))) { ok = false; break; }
                tc::fence_after_sync();
                if (lane == 0) {
                    const uint32_t vb = sV + s * 2 * kRegion;
                    const uint32_t pt = tmem + (uint32_t)(t * 128);       // P_t packed in S_t's columns
                    const int nk = pv_steps(j);
#pragma unroll
                    for (int k = 0; k < kBN / 16; ++k)
                        if (k < nk)
                            tc::mma_f16_ts(tmem + 256 + (uint32_t)(t * 128), pt + (uint32_t)(8 * k),
                                           tc::smem_desc_sw128(vb + (uint32_t)(k * 2048), kRegion, 1024), idO(t),
                                           (j > 0 || k > 0) ? 1u : 0u);
                    const bool last = t + 1 == ntiles;
                    if (last) tc::commit(bar(kBarEV + s));                  // V(j) read by every PV
                    if (nhave) {
                        issue_S(t, j + 1);
                        if (last) tc::commit(bar(kBarEK + (j + 1) % kKStages));   // K(j+1) read by every S
                    } else {
                        tc::commit(bar(kBarO + t));
                    }
                }
                __syncwarp();
            }
            if (!ok) break;
            have = nhave;
            ++j;
        }
        // all issued MMAs complete before TMEM can be released
        if (lane == 0) tc::commit(bar(kBarMma));
        __syncwarp();
        int never = 0;
        tc::mbar_wait(bar(kBarMma), 0, &never);
    } else if (half_of(warp >> 2)) {
        // ================= softmax of an M = 64 tile: warp q of warpgroup t reads lanes 32q .. 32q + 15
        // with the 16-lane shapes; thread i holds rows 16q + i/4 (A) and 16q + i/4 + 8 (B) and, of
        // every 8 key columns, the two at 2 (i % 4), so each thread forms half the exponentials of
        // a 128-row tile's thread. In split mode warpgroup t takes key tiles j % 2 == t and
        // warpgroup 0 merges; with a single key tile warpgroup 0 alone.
        const int t = warp >> 2, wq = warp & 3, q4 = lane & 3;
        const int rA = 16 * wq + (lane >> 2), rB = rA + 8;
        const int qn = two ? (t == 0 ? qn0 : qn1) : qn0;     // two: head pairs, tile t = head x + t
        const long long qrow_t = t ? qrow[1] : qrow[0];
        float* sML = reinterpret_cast<float*>(sbase + kOffML);   // split mode: [0][row] max, [1][row] sum
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + (uint32_t)(t * 128) + lane_off;
        const uint32_t tO = tmem + 256 + (uint32_t)(t * 128) + lane_off;
        const float c_log2 = p.scale_log2;
        const int kj0 = split ? t : 0, kjs = split ? 2 : 1;
        const int nloc = split ? (ntk - t + 1) / 2 : ((t == 0 || two) ? ntk : 0);
        int j = 0;
        float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;   // l: this thread's partial sums
        bool ok = true;
        int lim_next = nloc > 0 ? key_tile(p, MODE, klist, kj0).y : 0;
        for (; j < nloc; ++j) {
            const int lim = lim_next;
            if (j + 1 < nloc) lim_next = key_tile(p, MODE, klist, kj0 + (j + 1) * kjs).y;
            const bool got_s = tc::mbar_wait(bar(kBarS + t), j & 1, abort_flag);
            if (!__all_sync(kFull, got_s)) { ok = false; break; }
            tc::fence_after_sync();
            uint32_t v[2][32];
            tc::tmem_ld_16x256b_x8(tS, v[0]);
            if (lim > 64) tc::tmem_ld_16x256b_x8(tS + 64, v[1]);
            tc::tmem_wait_ld();
            tc::regs_after_wait(v[0]);
            if (lim > 64) tc::regs_after_wait(v[1]);
            float xA = -INFINITY, xB = -INFINITY;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (h == 1 && lim <= 64) break;
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        if (64 * h + 8 * jj + 2 * q4 + e >= lim) {
                            v[h][4 * jj + e] = __float_as_uint(-INFINITY);
                            v[h][4 * jj + 2 + e] = __float_as_uint(-INFINITY);
                        }
                        xA = fmaxf(xA, __uint_as_float(v[h][4 * jj + e]));
                        xB = fmaxf(xB, __uint_as_float(v[h][4 * jj + 2 + e]));
                    }
            }
            xA = fmaxf(xA, __shfl_xor_sync(kFull, xA, 1));
            xA = fmaxf(xA, __shfl_xor_sync(kFull, xA, 2));
            xB = fmaxf(xB, __shfl_xor_sync(kFull, xB, 1));
            xB = fmaxf(xB, __shfl_xor_sync(kFull, xB, 2));
            // lazy rescale: only when a row's maximum rises by more than 2^8
            const bool grow = xA > (mA + kRescaleLog2) / c_log2 || xB > (mB + kRescaleLog2) / c_log2;
            if (__any_sync(kFull, grow)) {
                const float nA = fmaxf(mA, xA * c_log2), nB = fmaxf(mB, xB * c_log2);
                const bool rsA = nA > mA + kRescaleLog2, rsB = nB > mB + kRescaleLog2;
                if (j > 0 && __any_sync(kFull, rsA || rsB)) {
                    // S_t(j) complete => PV_t(j-1) complete: O_t may be rescaled now
                    const float fA = rsA ? exp2f(mA - nA) : 1.f, fB = rsB ? exp2f(mB - nB) : 1.f;
#pragma unroll
                    for (int h = 0; h < D / 64; ++h) {
                        uint32_t ov[32];
                        tc::tmem_ld_16x256b_x8(tO + 64 * h, ov);
                        tc::tmem_wait_ld();
                        tc::regs_after_wait(ov);
#pragma unroll
                        for (int jj = 0; jj < 8; ++jj) {
                            ov[4 * jj] = __float_as_uint(__uint_as_float(ov[4 * jj]) * fA);
                            ov[4 * jj + 1] = __float_as_uint(__uint_as_float(ov[4 * jj + 1]) * fA);
                            ov[4 * jj + 2] = __float_as_uint(__uint_as_float(ov[4 * jj + 2]) * fB);
                            ov[4 * jj + 3] = __float_as_uint(__uint_as_float(ov[4 * jj + 3]) * fB);
                        }
                        tc::tmem_st_16x256b_x8(tO + 64 * h, ov);
                    }
                    if (rsA) lA *= fA;
                    if (rsB) lB *= fB;
                }
                if (rsA) mA = nA;
                if (rsB) mB = nB;
            }
            // P = 2^(s c - m) as bf16 pairs: the pair of columns 8jj + 2 q4 is packed column 4jj + q4
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (h == 1 && lim <= 64) break;
                uint32_t pk[16];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const float p0 = ex2_sfu(fmaf(__uint_as_float(v[h][4 * jj]), c_log2, -mA));
                    const float p1 = ex2_sfu(fmaf(__uint_as_float(v[h][4 * jj + 1]), c_log2, -mA));
                    const float p2 = ex2_sfu(fmaf(__uint_as_float(v[h][4 * jj + 2]), c_log2, -mB));
                    const float p3 = ex2_sfu(fmaf(__uint_as_float(v[h][4 * jj + 3]), c_log2, -mB));
                    lA += p0 + p1;
                    lB += p2 + p3;
                    __nv_bfloat162 b0 = __floats2bfloat162_rn(p0, p1), b1 = __floats2bfloat162_rn(p2, p3);
                    pk[2 * jj] = *reinterpret_cast<uint32_t*>(&b0);
                    pk[2 * jj + 1] = *reinterpret_cast<uint32_t*>(&b1);
                }
                tc::tmem_st_16x128b_x8(tS + 32 * h, pk);
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            tc::mbar_arrive(bar(kBarP + t));
        }
        lA += __shfl_xor_sync(kFull, lA, 1);
        lA += __shfl_xor_sync(kFull, lA, 2);
        lB += __shfl_xor_sync(kFull, lB, 1);
        lB += __shfl_xor_sync(kFull, lB, 2);
        // epilogue: O / l written as bf16 pairs of the thread's columns, and lse
        auto store_rows = [&](const uint32_t (&o0)[32], const uint32_t* o1, int h, float a0A, float a1A, float a0B,
                              float a1B) {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int col = 64 * h + 8 * jj + 2 * q4;
                float vA0 = __uint_as_float(o0[4 * jj]) * a0A, vA1 = __uint_as_float(o0[4 * jj + 1]) * a0A;
                float vB0 = __uint_as_float(o0[4 * jj + 2]) * a0B, vB1 = __uint_as_float(o0[4 * jj + 3]) * a0B;
                if (o1) {
                    vA0 = fmaf(__uint_as_float(o1[4 * jj]), a1A, vA0);
                    vA1 = fmaf(__uint_as_float(o1[4 * jj + 1]), a1A, vA1);
                    vB0 = fmaf(__uint_as_float(o1[4 * jj + 2]), a1B, vB0);
                    vB1 = fmaf(__uint_as_float(o1[4 * jj + 3]), a1B, vB1);
                }
                if (rA < qn) {
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(vA0, vA1);
                    *reinterpret_cast<__nv_bfloat162*>(p.O + (qrow_t + rA) * D + col) = b2;
                }
                if (rB < qn) {
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(vB0, vB1);
                    *reinterpret_cast<__nv_bfloat162*>(p.O + (qrow_t + rB) * D + col) = b2;
                }
            }
        };
        if (split) {
            if (t == 1 && q4 == 0) {
                sML[rA] = mA; sML[kBM + rA] = lA;
                sML[rB] = mB; sML[kBM + rB] = lB;
            }
            tc::named_bar_sync(1, 2 * kBM);
            if (t == 0) {
                bool got = false;
                if (ok) got = tc::mbar_wait(bar(kBarO), 0, abort_flag) && tc::mbar_wait(bar(kBarO + 1), 0, abort_flag);
                if (__all_sync(kFull, got)) {
                    tc::fence_after_sync();
                    const float m1A = sML[rA], l1A = sML[kBM + rA], m1B = sML[rB], l1B = sML[kBM + rB];
                    const float mmA = fmaxf(mA, m1A), mmB = fmaxf(mB, m1B);
                    const float f0A = mmA == -INFINITY ? 0.f : exp2f(mA - mmA), f1A = mmA == -INFINITY ? 0.f : exp2f(m1A - mmA);
                    const float f0B = mmB == -INFINITY ? 0.f : exp2f(mB - mmB), f1B = mmB == -INFINITY ? 0.f : exp2f(m1B - mmB);
                    const float LA = lA * f0A + l1A * f1A, LB = lB * f0B + l1B * f1B;
                    const float iA = LA > 0.f ? 1.f / LA : 0.f, iB = LB > 0.f ? 1.f / LB : 0.f;
#pragma unroll
                    for (int h = 0; h < D / 64; ++h) {
                        uint32_t o0[32], o1[32];
                        tc::tmem_ld_16x256b_x8(tO + 64 * h, o0);
                        tc::tmem_ld_16x256b_x8(tO + 128 + 64 * h, o1);
                        tc::tmem_wait_ld();
                        tc::regs_after_wait(o0);
                        tc::regs_after_wait(o1);
                        store_rows(o0, o1, h, f0A * iA, f1A * iA, f0B * iB, f1B * iB);
                    }
                    if (q4 == 0 && p.lse) {
                        if (rA < qn) p.lse[qrow_t + rA] = (mmA + log2f(LA)) * kLn2;
                        if (rB < qn) p.lse[qrow_t + rB] = (mmB + log2f(LB)) * kLn2;
                    }
                }
            }
        } else if (t == 0 || two) {
            bool got_last = false;
            if (ok && j > 0) got_last = tc::mbar_wait(bar(kBarO + t), 0, abort_flag);
            if (j > 0 && __all_sync(kFull, got_last)) {
                tc::fence_after_sync();
                const float iA = lA > 0.f ? 1.f / lA : 0.f, iB = lB > 0.f ? 1.f / lB : 0.f;
#pragma unroll
                for (int h = 0; h < D / 64; ++h) {
                    uint32_t o0[32];
                    tc::tmem_ld_16x256b_x8(tO + 64 * h, o0);
                    tc::tmem_wait_ld();
                    tc::regs_after_wait(o0);
                    store_rows(o0, nullptr, h, iA, 0.f, iB, 0.f);
                }
                if (q4 == 0 && p.lse) {
                    if (rA < qn) p.lse[qrow_t + rA] = (mA + log2f(lA)) * kLn2;
                    if (rB < qn) p.lse[qrow_t + rB] = (mB + log2f(lB)) * kLn2;
                }
            } else if (j == 0) {
                uint32_t zr[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) zr[e] = 0u;
                for (int h = 0; h < D / 64; ++h) store_rows(zr, nullptr, h, 0.f, 0.f, 0.f, 0.f);
                if (q4 == 0 && p.lse) {
                    if (rA < qn) p.lse[qrow_t + rA] = -INFINITY;
                    if (rB < qn) p.lse[qrow_t + rB] = -INFINITY;
                }
            }
        }
    } else {
        // ================= softmax warpgroup t: thread r <-> row r of tile t <-> TMEM lane r
        const int t = warp >> 2;
        const int r = threadIdx.x & 127;
        const long long qrow_t = t ? qrow[1] : qrow[0];   // first flattened query row of tile t
        const int qn = (t == 0 || split) ? qn0 : qn1;
        float* sML = reinterpret_cast<float*>(sbase + kOffML);   // split mode: [0][r] max, [1][r] sum of tile 1
        if (qn > 0) {
            const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
            const uint32_t tS = tmem + (uint32_t)(t * 128) + lane_off;
            const uint32_t tO = tmem + 256 + (uint32_t)(t * 128) + lane_off;
            const float c_log2 = p.scale_log2;
            // this warpgroup's key tiles: all of them, or (split mode) every other one from t
            const int kj0 = split ? t : 0, kjs = split ? 2 : 1;
            const int nloc = split ? (ntk - t + 1) / 2 : ntk;
            int j = 0;
            float m_run = -INFINITY, l_run = 0.f;
            bool ok = true;
            int lim_next = nloc > 0 ? key_tile(p, MODE, klist, kj0).y : 0;
            for (; j < nloc; ++j) {
                const int lim = lim_next;
                if (j + 1 < nloc) lim_next = key_tile(p, MODE, klist, kj0 + (j + 1) * kjs).y;   // prefetch
                // every TMEM access below is warp-collective: decisions are made warp-uniform
                const bool got_s = tc::mbar_wait(bar(kBarS + t), j & 1, abort_flag);
                if (!__all_sync(kFull, got_s)) { ok = false; break; }
                tc::fence_after_sync();
                // Half h of the row (64 columns) at a time. P of the first half is formed
                // against the running max before the second half is seen and kept packed in
                // registers; only when some row of the warp has a logit more than 2^8 above its
                // running max (rare after the first tile) is the tile redone from S, which stays
                // in TMEM until P is written.
                // P is formed against the running max m_run without looking at this tile's maxima:
                // every p is at most the row's sum over the tile, so a sum of at most 2^8 proves
                // that no logit rose by more than 2^8 above m_run (inf and NaN fail the test too).
                // Otherwise, and on the warpgroup's first key tile, the tile is redone from S, which
                // stays in TMEM until P is written: the row maxima are taken, m_run moves up to the
                // new maximum (O and l rescaled), and P is formed again.
                uint32_t pk0[32], pk1[32];                              // P of columns 0..63, 64..127
                uint64_t ps[4] = {0ull, 0ull, 0ull, 0ull};              // packed pair sums
                bool slow = j == 0;
                if (!slow) {
                    {
                        uint32_t sv[2][32];
                        load_half_nomax(tS, 0, lim, sv);
                        exp_half(sv, c_log2, -m_run, pk0, ps);
                    }
                    if (lim > 64) {
                        uint32_t sv[2][32];
                        load_half_nomax(tS, 1, lim, sv);
                        exp_half(sv, c_log2, -m_run, pk1, ps);
                    }
                    float a0, a1, b0, b1;
                    up2(add2(ps[0], ps[1]), a0, a1);
                    up2(add2(ps[2], ps[3]), b0, b1);
                    const float tsum = (a0 + a1) + (b0 + b1);
                    slow = __any_sync(kFull, !(tsum <= kRescaleMax));
                    if (!slow) {
                        tc::tmem_st16(tS, pk0);
                        tc::tmem_st16(tS + 16, pk0 + 16);
                        if (lim > 64) {
                            tc::tmem_st16(tS + 32, pk1);
                            tc::tmem_st16(tS + 48, pk1 + 16);
                        }
                        l_run += tsum;
                    }
                }
                if (slow) {
                    float mx0 = -INFINITY, mx1 = -INFINITY;
                    {
                        uint32_t sv[2][32];
                        load_half(tS, 0, lim, sv, mx0);
                    }
                    if (lim > 64) {
                        uint32_t sv[2][32];
                        load_half(tS, 1, lim, sv, mx1);
                    }
                    const float m_new = fmaxf(m_run, fmaxf(mx0, mx1) * c_log2);
                    const bool rescale = m_new > m_run;
                    if (j > 0 && __any_sync(kFull, rescale)) {
                        // S_t(j) complete => PV_t(j-1) complete: O_t may be rescaled now
                        const float f = rescale ? exp2f(m_run - m_new) : 1.f;
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t ov[32];
                            tc::tmem_ld32(tO + 32 * c, ov);
                            tc::tmem_wait_ld();
                            tc::regs_after_wait(ov);
#pragma unroll
                            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * f);
                            tc::tmem_st32(tO + 32 * c, ov);
                        }
                        if (rescale) l_run *= f;
                    }
                    if (rescale) m_run = m_new;
#pragma unroll
                    for (int e = 0; e < 4; ++e) ps[e] = 0ull;
                    {
                        uint32_t sv[2][32];
                        load_half_nomax(tS, 0, lim, sv);
                        exp_half(sv, c_log2, -m_run, pk0, ps);
                    }
                    if (lim > 64) {
                        uint32_t sv[2][32];
                        load_half_nomax(tS, 1, lim, sv);
                        exp_half(sv, c_log2, -m_run, pk1, ps);
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) pk1[e] = 0u;
                    }
                    tc::tmem_st16(tS, pk0);
                    tc::tmem_st16(tS + 16, pk0 + 16);
                    tc::tmem_st16(tS + 32, pk1);
                    tc::tmem_st16(tS + 48, pk1 + 16);
                    float a0, a1, b0, b1;
                    up2(add2(ps[0], ps[1]), a0, a1);
                    up2(add2(ps[2], ps[3]), b0, b1);
                    l_run += (a0 + a1) + (b0 + b1);
                }
                tc::tmem_wait_st();
                tc::fence_before_sync();
                tc::mbar_arrive(bar(kBarP + t));
            }
            // epilogue: O / l, bf16 row store, lse
            if (split) {
                // tile 1 hands its running max and sum to warpgroup 0, which reads both O_0 and O_1
                // from TMEM (the same lanes) and writes the merged rows
                if (t == 1) {
                    sML[r] = m_run;
                    sML[kBM + r] = l_run;
                }
                tc::named_bar_sync(1, 2 * kBM);
                if (t == 0) {
                    bool got = false;
                    if (ok) got = tc::mbar_wait(bar(kBarO), 0, abort_flag) && tc::mbar_wait(bar(kBarO + 1), 0, abort_flag);
                    if (__all_sync(kFull, got)) {
                        tc::fence_after_sync();
                        const float m1 = sML[r], l1 = sML[kBM + r];
                        const float mm = fmaxf(m_run, m1);
                        const float f0 = mm == -INFINITY ? 0.f : exp2f(m_run - mm);
                        const float f1 = mm == -INFINITY ? 0.f : exp2f(m1 - mm);
                        const float l = l_run * f0 + l1 * f1;
                        const float inv = l > 0.f ? 1.f / l : 0.f;
                        // probe mode keeps the merged partial state unnormalised (scaled to mm)
                        const float a0 = MODE == kModeProbe ? f0 : f0 * inv, a1 = MODE == kModeProbe ? f1 : f1 * inv;
                        bf16* orow = p.O + (qrow[0] + r) * D;
                        const long long pb = ((long long)x * p.ns + blockIdx.x) * p.M + r;
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t o0[32], o1[32];
                            tc::tmem_ld32(tO + 32 * c, o0);
                            tc::tmem_ld32(tO + 128 + 32 * c, o1);
                            tc::tmem_wait_ld();
                            tc::regs_after_wait(o0);
                            tc::regs_after_wait(o1);
                            if (MODE == kModeProbe) {
                                if (r < qn) {
                                    float4* prow = reinterpret_cast<float4*>(p.Opart + pb * D + 32 * c);
#pragma unroll
                                    for (int q = 0; q < 8; ++q)
                                        prow[q] = make_float4(
                                            fmaf(__uint_as_float(o0[4 * q]), a0, __uint_as_float(o1[4 * q]) * a1),
                                            fmaf(__uint_as_float(o0[4 * q + 1]), a0, __uint_as_float(o1[4 * q + 1]) * a1),
                                            fmaf(__uint_as_float(o0[4 * q + 2]), a0, __uint_as_float(o1[4 * q + 2]) * a1),
                                            fmaf(__uint_as_float(o0[4 * q + 3]), a0, __uint_as_float(o1[4 * q + 3]) * a1));
                                }
                            } else if (r < qn) {
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    uint32_t w[4];
#pragma unroll
                                    for (int e = 0; e < 4; ++e) {
                                        const int i0 = 8 * q + 2 * e;
                                        __nv_bfloat162 b2 = __floats2bfloat162_rn(
                                            fmaf(__uint_as_float(o0[i0]), a0, __uint_as_float(o1[i0]) * a1),
                                            fmaf(__uint_as_float(o0[i0 + 1]), a0, __uint_as_float(o1[i0 + 1]) * a1));
                                        w[e] = *reinterpret_cast<uint32_t*>(&b2);
                                    }
                                    *reinterpret_cast<uint4*>(orow + 32 * c + 8 * q) = make_uint4(w[0], w[1], w[2], w[3]);
                                }
                            }
                        }
                        if (MODE == kModeProbe) {
                            if (r < qn) {
                                p.mpart[pb] = mm;
                                p.lpart[pb] = l;
                            }
                        } else if (r < qn && p.lse) {
                            p.lse[qrow[0] + r] = (mm + log2f(l)) * kLn2;
                        }
                    }
                }
            } else {
            bool got_last = false;
            if (ok && j > 0) got_last = tc::mbar_wait(bar(kBarO + t), 0, abort_flag);
            const long long pb = ((long long)x * p.ns + blockIdx.x) * p.M + r;   // probe mode
            if (MODE == kModeProbe && j > 0 && __all_sync(kFull, got_last)) {
                // a single key tile: the unnormalised state as it stands
                tc::fence_after_sync();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t ov[32];
                    tc::tmem_ld32(tO + 32 * c, ov);
                    tc::tmem_wait_ld();
                    tc::regs_after_wait(ov);
                    if (r < qn) {
                        float4* prow = reinterpret_cast<float4*>(p.Opart + pb * D + 32 * c);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            prow[q] = make_float4(__uint_as_float(ov[4 * q]), __uint_as_float(ov[4 * q + 1]),
                                                  __uint_as_float(ov[4 * q + 2]), __uint_as_float(ov[4 * q + 3]));
                    }
                }
                if (r < qn) {
                    p.mpart[pb] = m_run;
                    p.lpart[pb] = l_run;
                }
            } else if (MODE == kModeProbe) {
                if (j == 0 && r < qn) {
                    // an empty key split: no mass
                    float4* prow = reinterpret_cast<float4*>(p.Opart + pb * D);
                    for (int c = 0; c < D / 4; ++c) prow[c] = make_float4(0.f, 0.f, 0.f, 0.f);
                    p.mpart[pb] = -INFINITY;
                    p.lpart[pb] = 0.f;
                }
            } else if (j > 0 && __all_sync(kFull, got_last)) {
                tc::fence_after_sync();
                const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
                bf16* orow = p.O + (qrow_t + r) * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t ov[32];
                    tc::tmem_ld32(tO + 32 * c, ov);
                    tc::tmem_wait_ld();
                    tc::regs_after_wait(ov);
                    if (r < qn) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(ov[8 * q + 2 * e]) * inv,
                                                                          __uint_as_float(ov[8 * q + 2 * e + 1]) * inv);
                                w[e] = *reinterpret_cast<uint32_t*>(&b2);
                            }
                            *reinterpret_cast<uint4*>(orow + 32 * c + 8 * q) = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
                if (r < qn && p.lse)
                    p.lse[qrow_t + r] = (m_run + log2f(l_run)) * kLn2;
            } else if (j == 0 && r < qn) {
                bf16* orow = p.O + (qrow_t + r) * D;
                for (int c = 0; c < D; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
                if (p.lse) p.lse[qrow_t + r] = -INFINITY;
            }
            }
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

// ---------------------------------------------------------------- key-tile lists
// One warp per (KV head z, query group a): walk the kept key groups of route row a in
// ascending order, merge groups whose key ranges touch (empty groups pass through), and
// cut every merged run [lo, hi) into 128-key tiles. WRITE == false counts the tiles,
// WRITE == true stores them at list + off[z][a].
template <bool WRITE>
__global__ void key_tiles_kernel(const int32_t* __restrict__ rowptr, const int32_t* __restrict__ kg,
                                 const int32_t* __restrict__ koff, int32_t* cnt, const int32_t* __restrict__ off,
                                 int2* list, int P, int Gq, int Gk) {
    const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (wid >= P * Gq) return;
    const int z = wid / Gq, a = wid % Gq;
    const int32_t* rp = rowptr + (long long)z * (Gq + 1);
    const int32_t* kept = kg + (long long)z * Gq * Gk;
    const int32_t* ko = koff + (long long)z * (Gk + 1);
    const int r0 = rp[a], r1 = rp[a + 1];
    int2* out = WRITE ? list + off[(long long)z * (Gq + 1) + a] : nullptr;
    int ntiles = 0;
    int cur_lo = 0, cur_hi = 0;
    bool in_run = false;
    auto emit = [&](int lo, int hi) {
        if (hi <= lo) return;
        const int nt = (hi - lo + kBN - 1) / kBN;
        if (WRITE)
            for (int t = lane; t < nt; t += 32) out[ntiles + t] = make_int2(lo + t * kBN, min(kBN, hi - lo - t * kBN));
        ntiles += nt;
    };
    for (int c0 = r0; c0 < r1; c0 += 32) {
        const int n = min(32, r1 - c0);
        int glo = 0, ghi = 0;
        if (lane < n) {
            const int g = kept[c0 + lane];
            glo = ko[g];
            ghi = ko[g + 1];
        }
        for (int i = 0; i < n; ++i) {
            const int lo = __shfl_sync(kFull, glo, i), hi = __shfl_sync(kFull, ghi, i);
            if (in_run && lo == cur_hi) {
                cur_hi = hi;
            } else {
                if (in_run) emit(cur_lo, cur_hi);
                cur_lo = lo;
                cur_hi = hi;
                in_run = true;
            }
        }
    }
    if (in_run) emit(cur_lo, cur_hi);
    if (!WRITE && lane == 0) cnt[(long long)z * Gq + a] = ntiles;
}

// off[z][a] = z * cap + sum_{a' < a} cnt[z][a']; one thread per KV head.
__global__ void key_tiles_scan_kernel(const int32_t* __restrict__ cnt, int32_t* off, int P, int Gq, int cap) {
    const int z = blockIdx.x * blockDim.x + threadIdx.x;
    if (z >= P) return;
    int s = z * cap;
    for (int a = 0; a < Gq; ++a) {
        off[(long long)z * (Gq + 1) + a] = s;
        s += cnt[(long long)z * Gq + a];
    }
    off[(long long)z * (Gq + 1) + Gq] = s;
}

// ---------------------------------------------------------------- host side

template <int MODE, int D>
cudaError_t launch_tc(const bf16* Q, const bf16* K, const bf16* V, const TcParams& p, long long qrows, int B, int Hkv,
                      dim3 grid, cudaStream_t s) {
    CUtensorMap mq, mk, mv;
    if (!make_tmap_bf16_sw128(&mq, Q, qrows, D, kBM, 64) ||
        !make_tmap_bf16_sw128(&mk, K, (long long)B * Hkv * p.N, D, kBN, 64) ||
        !make_tmap_bf16_sw128(&mv, V, (long long)B * Hkv * p.N, D, kBN, 64))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<MODE, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    attn_tc_kernel<MODE, D><<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_tc_d(int d, const bf16* Q, const bf16* K, const bf16* V, const TcParams& p, long long qrows, int B,
                        int Hkv, dim3 grid, cudaStream_t s) {
    if (d == 128) return launch_tc<MODE, 128>(Q, K, V, p, qrows, B, Hkv, grid, s);
    if (d == 64) return launch_tc<MODE, 64>(Q, K, V, p, qrows, B, Hkv, grid, s);
    return cudaErrorInvalidValue;
}

TcParams params(bf16* O, float* lse, int N, int g, int d, int* status) {
    TcParams p;
    memset(&p, 0, sizeof(p));
    p.O = O;
    p.lse = lse;
    p.N = N;
    p.g = g;
    p.status = status;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)d));
    return p;
}

}  // namespace

bool attn_tc_supported(int d) { return d == 64 || d == 128; }

// Keys per probe split (whole 128-key tiles) and the number of non-empty splits.
int probe_tc_chunk(int N, int ns) { return ((N + ns - 1) / ns + kBN - 1) / kBN * kBN; }
int probe_tc_splits(int N, int ns) { return (N + probe_tc_chunk(N, ns) - 1) / probe_tc_chunk(N, ns); }

bool attn_tc_head_pairs(int g) { return g % 2 == 0; }

bool attn_tc_half_tails(int g) { return g >= 1; }

int attn_tc_rows_per_cta(int g) { return attn_tc_head_pairs(g) ? kBM : 2 * kBM; }

long long key_tiles_capacity(int N, int Gq, int Gk) { return (long long)Gq * ((N + kBN - 1) / kBN + Gk); }

cudaError_t launch_key_tiles(const int32_t* rowptr, const int32_t* kg, const int32_t* koff, int32_t* cnt,
                             int32_t* off, int2* list, int P, int N, int Gq, int Gk, cudaStream_t s) {
    const long long warps = (long long)P * Gq;
    const unsigned blocks = (unsigned)((warps * 32 + 255) / 256);
    key_tiles_kernel<false><<<blocks, 256, 0, s>>>(rowptr, kg, koff, cnt, nullptr, nullptr, P, Gq, Gk);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    key_tiles_scan_kernel<<<(P + 127) / 128, 128, 0, s>>>(cnt, off, P, Gq, (int)key_tiles_capacity(N, Gq, Gk));
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    key_tiles_kernel<true><<<blocks, 256, 0, s>>>(rowptr, kg, koff, cnt, off, list, P, Gq, Gk);
    return cudaGetLastError();
}

cudaError_t launch_attn_sparse_tc(const bf16* Qp, const bf16* Kp, const bf16* Vp, const int32_t* qoff,
                                  const int32_t* tile_off, const int2* klist, const int32_t* klist_off, bf16* O,
                                  float* lse, int B, int Hq, int Hkv, int N, int d, int Gq, int* status, cudaStream_t s) {
    const int g = Hq / Hkv;
    TcParams p = params(O, lse, N, g, d, status);
    p.qoff = qoff; p.tile_off = tile_off; p.klist = klist; p.klist_off = klist_off;
    p.Gq = Gq;
    p.head_pairs = attn_tc_head_pairs(g) ? 1 : 0;
    p.half_tails = attn_tc_half_tails(g) ? 1 : 0;
    const int rows = attn_tc_rows_per_cta(g);
    dim3 grid((N + rows - 1) / rows + Gq, p.head_pairs ? B * Hq / 2 : B * Hq);
    return launch_tc_d<kModeSparse>(d, Qp, Kp, Vp, p, (long long)B * Hq * N, B, Hkv, grid, s);
}

cudaError_t launch_attn_probe_tc(const bf16* Qpr, const bf16* K, const bf16* V, float* Opart, float* mpart,
                                 float* lpart, int B, int Hq, int Hkv, int N, int d, int M, int ns, int* status,
                                 cudaStream_t s) {
    if (M < 1 || M > kBM || ns < 1) return cudaErrorInvalidValue;
    TcParams p = params(nullptr, nullptr, N, Hq / Hkv, d, status);
    p.Opart = Opart; p.mpart = mpart; p.lpart = lpart;
    p.M = M;
    p.chunk = probe_tc_chunk(N, ns);
    p.ns = probe_tc_splits(N, ns);      // splits launched = the stride of the partial outputs
    return launch_tc_d<kModeProbe>(d, Qpr, K, V, p, (long long)B * Hq * kBM, B, Hkv, dim3(p.ns, B * Hq), s);
}

cudaError_t launch_attn_dense_tc(const bf16* Q, const bf16* K, const bf16* V, bf16* O, float* lse, int B, int Hq,
                                 int Hkv, int N, int d, int* status, bool stall, cudaStream_t s) {
    TcParams p = params(O, lse, N, Hq / Hkv, d, status);
    p.stall = stall ? 1 : 0;
    dim3 grid((N + 2 * kBM - 1) / (2 * kBM), B * Hq);
    return launch_tc_d<kModeDense>(d, Q, K, V, p, (long long)B * Hq * N, B, Hkv, grid, s);
}

}  // namespace spr
