// Exact softmax attention on 5th-generation tensor cores (d = 128): the
// block-sparse pass over each query group's kept key groups, renormalised over
// those keys only, and the dense baseline (one key range [0, N)).
//
// One CTA per 128-row query tile, six warps:
//   warps 0-3  softmax + epilogue: thread r owns query row r = TMEM lane r; it reads its row
//              of S from TMEM, keeps the running max / sum, writes P (bf16) into one of two
//              shared-memory buffers in the 128-byte-swizzled K-major layout, rescales its O
//              row in TMEM when the max grows by more than 2^8, and finally normalises and
//              stores O;
//   warp 4     TMA producer: Q once, then K and V tiles of 128 keys into a 2-stage ring;
//   warp 5     TMEM allocation and the MMA issue (one elected thread): S = Q K^T into one of
//              two TMEM buffers, O += P V into a third, completion signalled by tcgen05.commit.
// With two P buffers the tensor core runs S(j+1) and PV(j) while the softmax warps work on
// tile j+1; they wait for PV(j) only when their O row needs rescaling.
// Key tiles are cut from merged runs of consecutive kept key groups; keys past a run's end
// (the next group's, or zero fill past the tensor) are masked to -inf.
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

constexpr int kBM = 128;            // query rows per CTA
constexpr int kBN = 128;            // keys per tile
constexpr int kD = 128;             // head dimension
constexpr int kStages = 2;          // K/V ring depth
constexpr int kRegion = 16384;      // one [128 rows][64 bf16] 128B-swizzled region
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512; // S0 [0,128), S1 [128,256), O [256,384)
constexpr float kRescaleLog2 = 8.f; // lazy rescale threshold (P <= 2^8)
constexpr float kLn2 = 0.6931471805599453f;

constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + 2 * kRegion;
constexpr int kOffV = kOffK + kStages * 2 * kRegion;
constexpr int kOffP = kOffV + kStages * 2 * kRegion;
constexpr int kOffBar = kOffP + 2 * 2 * kRegion;          // two P buffers
// barriers: q_full, k_full[S], v_full[S], kv_empty[S], s_full[2], p_full[2], o_done[2], mma_done
// (s/p/o barriers indexed by tile parity so no waiter can fall two phases behind)
constexpr int kBarQ = 0, kBarK = 1, kBarV = kBarK + kStages, kBarE = kBarV + kStages, kBarS = kBarE + kStages,
              kBarP = kBarS + 2, kBarO = kBarP + 2, kBarMma = kBarO + 2, kNumBars = kBarMma + 1;
constexpr int kOffMisc = kOffBar + 8 * kNumBars;          // tmem base (u32), abort flag (int)
constexpr int kSmemBytes = kOffMisc + 16 + 1024;          // + slack to align the base to 1024

enum { kModeSparse = 0, kModeDense = 1 };

struct TcParams {
    bf16* O;
    float* lse;
    const int32_t* qoff;
    const int32_t* koff;
    const int32_t* tile_off;
    const int32_t* rowptr;
    const int32_t* kg;
    int* status;
    int N, g, Gq, Gk;
    float scale_log2;
};

// Sequence of key tiles of one query tile (identical in every warp role).
struct TileIter {
    const int32_t* kept;
    const int32_t* ko;
    int ri, r1;
    int lo, hi;     // current merged run
    int t0;         // next tile start
    bool dense;
    __device__ __forceinline__ bool next_run() {
        while (ri < r1) {
            const int g0 = kept[ri++];
            lo = ko[g0];
            hi = ko[g0 + 1];
            while (ri < r1 && ko[kept[ri]] == hi) { hi = ko[kept[ri] + 1]; ++ri; }
            if (hi > lo) { t0 = lo; return true; }
        }
        return false;
    }
    // Next tile: start row and number of valid keys (<= kBN); false when exhausted.
    __device__ __forceinline__ bool next(int& start, int& lim) {
        if (t0 >= hi) {
            if (dense || !next_run()) return false;
        }
        start = t0;
        lim = min(kBN, hi - t0);
        t0 += kBN;
        return true;
    }
};

__device__ __forceinline__ bool make_iter(const TcParams& p, int mode, int z, int a, TileIter& it) {
    it.dense = mode == kModeDense;
    if (it.dense) {
        it.lo = 0; it.hi = p.N; it.t0 = 0; it.ri = it.r1 = 0; it.kept = nullptr; it.ko = nullptr;
        return true;
    }
    it.kept = p.kg + (long long)z * p.Gq * p.Gk;
    it.ko = p.koff + (long long)z * (p.Gk + 1);
    it.ri = p.rowptr[(long long)z * (p.Gq + 1) + a];
    it.r1 = p.rowptr[(long long)z * (p.Gq + 1) + a + 1];
    it.lo = it.hi = it.t0 = 0;
    return true;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                              const __grid_constant__ CUtensorMap tmK,
                                                              const __grid_constant__ CUtensorMap tmV,
                                                              const TcParams p) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = tc::smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* sbase = smem_raw + (base - raw);
    const uint32_t sQ = base + kOffQ, sK = base + kOffK, sV = base + kOffV, sP = base + kOffP;
    const uint32_t bars = base + kOffBar;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + kOffMisc + 4);
    auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int x = blockIdx.y, z = x / p.g;
    // a CTA that timed out earlier in this launch (or call) makes the rest return at once
    if (p.status && *reinterpret_cast<volatile int*>(p.status) == kDevTimeout) return;

    // ---- which query tile
    int qlo, qn, a = 0;
    if (MODE == kModeSparse) {
        const int32_t* toff = p.tile_off + (long long)z * (p.Gq + 1);
        const int tile = blockIdx.x;
        if (tile >= toff[p.Gq]) return;
        a = upper_index(toff, p.Gq, tile);
        const int32_t* qo = p.qoff + (long long)z * (p.Gq + 1);
        qlo = qo[a] + (tile - toff[a]) * kBM;
        qn = min(kBM, qo[a + 1] - qlo);
    } else {
        qlo = blockIdx.x * kBM;
        if (qlo >= p.N) return;
        qn = min(kBM, p.N - qlo);
    }

    // ---- set-up: barriers (thread 0), TMEM (warp 5)
    if (threadIdx.x == 0) {
        tc::mbar_init(bar(kBarQ), 1);
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(bar(kBarK + s), 1);
            tc::mbar_init(bar(kBarV + s), 1);
            tc::mbar_init(bar(kBarE + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(bar(kBarS + b), 1);
            tc::mbar_init(bar(kBarP + b), 128);
            tc::mbar_init(bar(kBarO + b), 1);
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
    const uint32_t tS0 = tmem, tO = tmem + 256;

    if (warp == 4) {
        // ================= TMA producer
        if (lane == 0) {
            const int qrow = x * p.N + qlo;
            tc::mbar_arrive_expect_tx(bar(kBarQ), 2 * kRegion);
            tc::tma_load_2d(sQ, &tmQ, bar(kBarQ), 0, qrow);
            tc::tma_load_2d(sQ + kRegion, &tmQ, bar(kBarQ), 64, qrow);
            TileIter it;
            make_iter(p, MODE, z, a, it);
            int start, lim, j = 0;
            while (it.next(start, lim)) {
                const int s = j % kStages;
                if (j >= kStages && !tc::mbar_wait(bar(kBarE + s), ((j / kStages) - 1) & 1, abort_flag)) break;
                const int krow = z * p.N + start;
                const uint32_t dk = sK + s * 2 * kRegion, dv = sV + s * 2 * kRegion;
                tc::mbar_arrive_expect_tx(bar(kBarK + s), 2 * kRegion);
                tc::tma_load_2d(dk, &tmK, bar(kBarK + s), 0, krow);
                tc::tma_load_2d(dk + kRegion, &tmK, bar(kBarK + s), 64, krow);
                tc::mbar_arrive_expect_tx(bar(kBarV + s), 2 * kRegion);
                tc::tma_load_2d(dv, &tmV, bar(kBarV + s), 0, krow);
                tc::tma_load_2d(dv + kRegion, &tmV, bar(kBarV + s), 64, krow);
                ++j;
            }
            // every issued load must land before the CTA can exit
            for (int t = (j > kStages ? j - kStages : 0); t < j; ++t) {
                const int s = t % kStages;
                const uint32_t par = (t / kStages) & 1;
                int dummy = 0;
                volatile int* never = &dummy;
                tc::mbar_wait(bar(kBarK + s), par, never);
                tc::mbar_wait(bar(kBarV + s), par, never);
            }
            tc::mbar_wait(bar(kBarQ), 0, abort_flag);
        }
    } else if (warp == 5) {
        // ================= MMA issuer
        const uint32_t idS = tc::idesc_bf16_f32(kBM, kBN, 0);
        const uint32_t idO = tc::idesc_bf16_f32(kBM, kD, 1);
        TileIter it;
        make_iter(p, MODE, z, a, it);
        int start, lim;
        bool have = it.next(start, lim);
        bool ok = __all_sync(kFull, tc::mbar_wait(bar(kBarQ), 0, abort_flag));
        auto issue_S = [&](int j) -> bool {
            const int s = j % kStages;
            if (!__all_sync(kFull, tc::mbar_wait(bar(kBarK + s), (j / kStages) & 1, abort_flag))) return false;
            tc::fence_after_sync();
            if (lane == 0) {
                const uint32_t dS = tS0 + (uint32_t)((j & 1) * 128);
                const uint32_t kb = sK + s * 2 * kRegion;
#pragma unroll
                for (int k = 0; k < kD / 16; ++k) {
                    const uint32_t off = (uint32_t)((k >> 2) * kRegion + (k & 3) * 32);
                    tc::mma_f16_ss(dS, tc::smem_desc_sw128(sQ + off, 16, 1024), tc::smem_desc_sw128(kb + off, 16, 1024),
                                   idS, k > 0 ? 1u : 0u);
                }
                tc::commit(bar(kBarS + (j & 1)));
            }
            __syncwarp();
            return true;
        };
        int j = 0;
        if (ok && have) ok = issue_S(0);
        while (ok && have) {
            bool nhave = it.next(start, lim);
            if (nhave && !issue_S(j + 1)) { ok = false; break; }
            const int s = j % kStages;
            if (!__all_sync(kFull, tc::mbar_wait(bar(kBarP + (j & 1)), (j >> 1) & 1, abort_flag))) { ok = false; break; }
            if (!__all_sync(kFull, tc::mbar_wait(bar(kBarV + s), (j / kStages) & 1, abort_flag))) { ok = false; break; }
            tc::fence_after_sync();
            if (lane == 0) {
                const uint32_t vb = sV + s * 2 * kRegion;
#pragma unroll
                for (int k = 0; k < kBN / 16; ++k) {
                    const uint32_t pa = sP + (uint32_t)((j & 1) * 2 * kRegion + (k >> 2) * kRegion + (k & 3) * 32);
                    const uint32_t vbk = vb + (uint32_t)(k * 2048);
                    tc::mma_f16_ss(tO, tc::smem_desc_sw128(pa, 16, 1024), tc::smem_desc_sw128(vbk, kRegion, 1024), idO,
                                   (j > 0 || k > 0) ? 1u : 0u);
                }
                tc::commit(bar(kBarE + s));
                tc::commit(bar(kBarO + (j & 1)));
            }
            __syncwarp();
            have = nhave;
            ++j;
        }
        // all issued MMAs complete before TMEM can be released
        if (lane == 0) tc::commit(bar(kBarMma));
        __syncwarp();
        int dummy = 0;
        tc::mbar_wait(bar(kBarMma), 0, &dummy);
    } else {
        // ================= softmax warps 0-3: thread r <-> query row r <-> TMEM lane r
        const int r = threadIdx.x;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        TileIter it;
        make_iter(p, MODE, z, a, it);
        int start, lim, j = 0;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        const float c_log2 = p.scale_log2;
        while (it.next(start, lim)) {
            // every TMEM access below is warp-collective: decisions are made warp-uniform
            const bool got_s = tc::mbar_wait(bar(kBarS + (j & 1)), (j >> 1) & 1, abort_flag);
            if (!__all_sync(kFull, got_s)) { ok = false; break; }
            tc::fence_after_sync();
            const uint32_t tS = tS0 + (uint32_t)((j & 1) * 128) + lane_off;
            uint32_t sv[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::tmem_ld32(tS + 32 * c, sv[c]);
            tc::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::regs_after_wait(sv[c]);
            // row max of the raw logits; keys past the run's end are set to -inf
            float mx = -INFINITY;
            if (lim == kBN) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int i = 0; i < 32; ++i) mx = fmaxf(mx, __uint_as_float(sv[c][i]));
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        if (32 * c + i >= lim) sv[c][i] = __float_as_uint(-INFINITY);
                        mx = fmaxf(mx, __uint_as_float(sv[c][i]));
                    }
            }
            const float m_new = fmaxf(m_run, mx * c_log2);
            const bool rescale = m_new > m_run + kRescaleLog2;
            if (j > 0 && __any_sync(kFull, rescale)) {
                // O holds PV(0..j-1): wait for PV(j-1), then scale the rows whose max moved
                const bool got_o = tc::mbar_wait(bar(kBarO + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort_flag);
                if (!__all_sync(kFull, got_o)) { ok = false; break; }
                tc::fence_after_sync();
                const float f = rescale ? exp2f(m_run - m_new) : 1.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t ov[32];
                    tc::tmem_ld32(tO + lane_off + 32 * c, ov);
                    tc::tmem_wait_ld();
                    tc::regs_after_wait(ov);
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * f);
                    tc::tmem_st32(tO + lane_off + 32 * c, ov);
                }
                tc::tmem_wait_st();
                if (rescale) l_run *= f;
            }
            if (rescale) m_run = m_new;
            // P buffer j&1 was last read by PV(j-2)
            if (j >= 2) {
                const bool got_b = tc::mbar_wait(bar(kBarO + (j & 1)), ((j - 2) >> 1) & 1, abort_flag);
                if (!__all_sync(kFull, got_b)) { ok = false; break; }
            }
            // P = 2^(s*c - m_run) as bf16, 16-byte chunks into the swizzled K-major P tile
            unsigned char* prow = sbase + kOffP + (j & 1) * 2 * kRegion + r * 128;
            const float neg_m = -m_run;
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const int h = c >> 3, cc = c & 7;
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float p0 = exp2f(fmaf(__uint_as_float(sv[c >> 2][(c & 3) * 8 + 2 * e]), c_log2, neg_m));
                    const float p1 = exp2f(fmaf(__uint_as_float(sv[c >> 2][(c & 3) * 8 + 2 * e + 1]), c_log2, neg_m));
                    sum += p0 + p1;
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                    w[e] = *reinterpret_cast<uint32_t*>(&b2);
                }
                *reinterpret_cast<uint4*>(prow + h * kRegion + ((cc ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            l_run += sum;
            tc::fence_proxy_async_smem();
            tc::fence_before_sync();
            tc::mbar_arrive(bar(kBarP + (j & 1)));
            ++j;
        }
        // epilogue: O / l, bf16 row store, lse
        bool got_last = false;
        if (ok && j > 0) got_last = tc::mbar_wait(bar(kBarO + ((j - 1) & 1)), ((j - 1) >> 1) & 1, abort_flag);
        if (j > 0 && __all_sync(kFull, got_last)) {
            tc::fence_after_sync();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            bf16* orow = p.O + ((long long)x * p.N + qlo + r) * kD;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t ov[32];
                tc::tmem_ld32(tO + lane_off + 32 * c, ov);
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
            if (r < qn && p.lse) p.lse[(long long)x * p.N + qlo + r] = (m_run + log2f(l_run)) * kLn2;
        } else if (j == 0 && r < qn) {
            bf16* orow = p.O + ((long long)x * p.N + qlo + r) * kD;
            for (int c = 0; c < kD; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
            if (p.lse) p.lse[(long long)x * p.N + qlo + r] = -INFINITY;
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

// ---------------------------------------------------------------- host side

template <int MODE>
cudaError_t launch_tc(const bf16* Q, const bf16* K, const bf16* V, const TcParams& p, int B, int Hq, int Hkv,
                      dim3 grid, cudaStream_t s) {
    CUtensorMap mq, mk, mv;
    if (!make_tmap_bf16_sw128(&mq, Q, (long long)B * Hq * p.N, kD, kBM, 64) ||
        !make_tmap_bf16_sw128(&mk, K, (long long)B * Hkv * p.N, kD, kBN, 64) ||
        !make_tmap_bf16_sw128(&mv, V, (long long)B * Hkv * p.N, kD, kBN, 64))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attn_tc_kernel<MODE><<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

TcParams params(bf16* O, float* lse, int N, int g, int* status) {
    TcParams p;
    memset(&p, 0, sizeof(p));
    p.O = O;
    p.lse = lse;
    p.N = N;
    p.g = g;
    p.status = status;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)kD));
    return p;
}

}  // namespace

bool attn_tc_supported(int d) { return d == kD; }

cudaError_t launch_attn_sparse_tc(const bf16* Qp, const bf16* Kp, const bf16* Vp, const int32_t* qoff,
                                  const int32_t* koff, const int32_t* tile_off, const int32_t* rowptr,
                                  const int32_t* kg, bf16* O, float* lse, int B, int Hq, int Hkv, int N, int Gq,
                                  int Gk, int* status, cudaStream_t s) {
    TcParams p = params(O, lse, N, Hq / Hkv, status);
    p.qoff = qoff; p.koff = koff; p.tile_off = tile_off; p.rowptr = rowptr; p.kg = kg;
    p.Gq = Gq; p.Gk = Gk;
    dim3 grid((N + kBM - 1) / kBM + Gq, B * Hq);
    return launch_tc<kModeSparse>(Qp, Kp, Vp, p, B, Hq, Hkv, grid, s);
}

cudaError_t launch_attn_dense_tc(const bf16* Q, const bf16* K, const bf16* V, bf16* O, float* lse, int B, int Hq,
                                 int Hkv, int N, int* status, cudaStream_t s) {
    TcParams p = params(O, lse, N, Hq / Hkv, status);
    dim3 grid((N + kBM - 1) / kBM, B * Hq);
    return launch_tc<kModeDense>(Q, K, V, p, B, Hq, Hkv, grid, s);
}

}  // namespace spr
