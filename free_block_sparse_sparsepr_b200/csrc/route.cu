// Routing of (query group, key group) cells to the execution-density budget:
// per-row log-normaliser over the key groups, cell scores (estimated softmax
// weight of one key of group g for a query of group a, averaged over the
// group's queries and the KV head's query heads), then whole-cell selection.
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace spr {
namespace {

// lse[x][i] = log sum_{g: |K_g| > 0} |K_g| exp(u[x][i][g]); one warp per row.
__global__ void row_lse_kernel(const float* __restrict__ u, const int32_t* __restrict__ koff,
                               float* lse, int g, int N, int Gk) {
    const int x = blockIdx.y, z = x / g;
    const int lane = threadIdx.x & 31;
    const int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (i >= N) return;
    const float* ur = u + ((long long)x * N + i) * Gk;
    const int32_t* ko = koff + (long long)z * (Gk + 1);
    float m = -FLT_MAX;
    for (int gk = lane; gk < Gk; gk += 32)
        if (ko[gk + 1] > ko[gk]) m = fmaxf(m, ur[gk]);
    m = warp_max(m);
    float s = 0.f;
    for (int gk = lane; gk < Gk; gk += 32) {
        int sz = ko[gk + 1] - ko[gk];
        if (sz > 0) s += (float)sz * expf(ur[gk] - m);
    }
    s = warp_sum(s);
    if (lane == 0) lse[(long long)x * N + i] = m + logf(s);
}

// scores[z][a][g] = mean over the g heads and the queries of group a of exp(u - lse).
// One CTA per (group a, KV head z); thread t takes key-group column t of each 256-column chunk.
// The group's row indices and their log2-scaled normalisers are staged in shared memory a round
// of rows at a time (coalesced, out of the loads' dependence chain), and exp(u - lse) is formed as
// 2^(u log2 e - lse log2 e) on the special-function unit (relative error about 1e-6); eight rows'
// logits are in flight per thread and four partial sums are added in a fixed order.
constexpr int kCsThreads = 256;
constexpr int kCsRows = 1024;   // rows staged per round
constexpr float kLog2eF = 1.4426950408889634f;

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__global__ void __launch_bounds__(kCsThreads) cell_scores_kernel(const float* __restrict__ u,
                                                                 const float* __restrict__ lse,
                                                                 const int32_t* __restrict__ qperm,
                                                                 const int32_t* __restrict__ qoff,
                                                                 const int32_t* __restrict__ koff, float* scores,
                                                                 int g, int N, int Gq, int Gk) {
    __shared__ int sIdx[kCsRows];
    __shared__ float sL[kCsRows];
    const int z = blockIdx.y, a = blockIdx.x, tid = threadIdx.x;
    const int lo = qoff[(long long)z * (Gq + 1) + a], hi = qoff[(long long)z * (Gq + 1) + a + 1];
    const int32_t* ko = koff + (long long)z * (Gk + 1);
    const int32_t* perm = qperm + (long long)z * N;
    for (int gk0 = 0; gk0 < Gk; gk0 += kCsThreads) {
        const int gk = gk0 + tid;
        const bool ok = hi > lo && gk < Gk && ko[gk + 1] > ko[gk];
        float acc = 0.f;
        for (int j = 0; j < g; ++j) {
            const long long x = (long long)z * g + j;
            const float* ux = u + x * N * Gk + gk;
            const float* lx = lse + x * N;
            float a4[4] = {0.f, 0.f, 0.f, 0.f};
            for (int base = lo; base < hi; base += kCsRows) {
                const int cnt = min(kCsRows, hi - base);
                __syncthreads();   // the previous round's rows are no longer read
                for (int t = tid; t < cnt; t += kCsThreads) {
                    const int i = __ldg(perm + base + t);
                    sIdx[t] = i;
                    sL[t] = __ldg(lx + i) * kLog2eF;
                }
                __syncthreads();
                if (ok) {
                    int q = 0;
                    for (; q + 8 <= cnt; q += 8) {
                        float v8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) v8[e] = __ldg(ux + (long long)sIdx[q + e] * Gk);
#pragma unroll
                        for (int e = 0; e < 8; ++e) a4[e & 3] += ex2_approx(fmaf(v8[e], kLog2eF, -sL[q + e]));
                    }
                    for (; q < cnt; ++q) a4[0] += ex2_approx(fmaf(__ldg(ux + (long long)sIdx[q] * Gk), kLog2eF, -sL[q]));
                }
            }
            acc += (a4[0] + a4[1]) + (a4[2] + a4[3]);
        }
        if (gk < Gk) scores[((long long)z * Gq + a) * Gk + gk] = ok ? acc / ((float)g * (float)(hi - lo)) : 0.f;
    }
}

// One CTA per (batch, KV head). Each non-empty query group keeps its top cell; the other
// eligible cells are ordered by key = (~score_bits << 32 | a*Gk + g) (descending score, then
// ascending a, g) and a cost-weighted radix select finds the first cell whose inclusion would
// exceed the remaining budget; it is kept iff its overshoot < the remaining undershoot.
constexpr int kSelThreads = 1024;
constexpr int kRadix = 2048;   // 11-bit digits
static_assert(2 * kSelThreads == kRadix, "two digit bins per thread in the scan");
__global__ void __launch_bounds__(kSelThreads, 1) route_select_kernel(
    const float* __restrict__ scores, const int32_t* __restrict__ qoff, const int32_t* __restrict__ koff,
    int32_t* rowptr, int32_t* kg, int64_t* pairs, int Gq, int Gk, long long budget, int keep_all) {
    const int z = blockIdx.x;
    extern __shared__ int sm[];
    int* qs = sm;             // [Gq]
    int* ks = qs + Gq;        // [Gk]
    int* mand = ks + Gk;      // [Gq]
    int* rowcnt = mand + Gq;  // [Gq]
    __shared__ unsigned long long hist[kRadix];
    __shared__ int hcnt[kRadix];
    __shared__ int s_unique;
    __shared__ long long red[32];
    __shared__ long long s_rem;
    __shared__ unsigned long long s_prefix, s_mask;
    __shared__ int s_found;
    __shared__ int s_dsel;
    __shared__ long long s_cum;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const float* S = scores + (long long)z * Gq * Gk;
    for (int a = tid; a < Gq; a += blockDim.x)
        qs[a] = qoff[(long long)z * (Gq + 1) + a + 1] - qoff[(long long)z * (Gq + 1) + a];
    for (int gk = tid; gk < Gk; gk += blockDim.x)
        ks[gk] = koff[(long long)z * (Gk + 1) + gk + 1] - koff[(long long)z * (Gk + 1) + gk];
    __syncthreads();

    // Mandatory cell per query group: argmax score over eligible key groups, ties -> lowest g.
    for (int a = warp; a < Gq; a += nw) {
        float best = -FLT_MAX;
        int bg = -1;
        if (qs[a] > 0) {
            for (int gk = lane; gk < Gk; gk += 32) {
                if (ks[gk] > 0) {
                    float v = S[(long long)a * Gk + gk];
                    if (bg < 0 || v > best) { best = v; bg = gk; }
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float ov = __shfl_xor_sync(kFull, best, o);
            int og = __shfl_xor_sync(kFull, bg, o);
            if (og >= 0 && (bg < 0 || ov > best || (ov == best && og < bg))) { best = ov; bg = og; }
        }
        if (lane == 0) mand[a] = bg;
    }
    __syncthreads();

    // Cost of the mandatory cells.
    long long loc = 0;
    for (int a = tid; a < Gq; a += blockDim.x)
        if (mand[a] >= 0) loc += (long long)qs[a] * ks[mand[a]];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) loc += __shfl_xor_sync(kFull, loc, o);
    if (lane == 0) red[warp] = loc;
    __syncthreads();
    if (tid == 0) {
        long long b = 0;
        for (int w = 0; w < nw; ++w) b += red[w];
        s_rem = budget - b;
        s_prefix = 0ull;
        s_mask = 0ull;
        s_found = keep_all ? 0 : 1;
        s_unique = 0;
    }
    __syncthreads();

    // Radix select over 64-bit keys (~score bits, cell index), 11 bits at a time from the top,
    // weighted by cell cost; thread t visits the cells a * Gk + gk with gk = t % Gk (no division
    // per cell). A digit bin holding a single candidate ends the descent: one more pass reads
    // that candidate's full key.
    const int gk0 = tid % Gk, astep = blockDim.x / Gk;
    const bool lane_ok = tid < astep * Gk;
    const bool gk_ok = ks[gk0] > 0;
    if (!keep_all) {
        bool unique = false;
        for (int shift = 53; shift > -11 && !unique; shift -= 11) {
            const int sh = shift > 0 ? shift : 0, bits = shift > 0 ? 11 : 11 + shift;
            const unsigned long long dmask = (1ull << bits) - 1ull;
            for (int t = tid; t < kRadix; t += blockDim.x) { hist[t] = 0ull; hcnt[t] = 0; }
            __syncthreads();
            const unsigned long long prefix = s_prefix, mask = s_mask;
            if (lane_ok && gk_ok) {
                for (int a = tid / Gk; a < Gq; a += astep) {
                    if (qs[a] == 0 || mand[a] == gk0) continue;
                    const long long c = (long long)a * Gk + gk0;
                    const unsigned long long key =
                        ((unsigned long long)(~__float_as_uint(S[c])) << 32) | (unsigned long long)c;
                    if ((key & mask) != prefix) continue;
                    const int dg = (int)((key >> sh) & dmask);
                    atomicAdd(&hist[dg], (unsigned long long)((long long)qs[a] * ks[gk0]));
                    atomicAdd(&hcnt[dg], 1);
                }
            }
            __syncthreads();
            // The selected digit is the first bin whose cost, added to the cost of all lower bins,
            // exceeds the remaining budget: a block-wide exclusive scan of the bins (two per
            // thread) and the smallest bin that satisfies the test.
            {
                const int b0 = 2 * tid;
                const long long h0 = (long long)hist[b0], h1 = (long long)hist[b0 + 1];
                long long inc = h0 + h1;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const long long n = __shfl_up_sync(kFull, inc, o);
                    if (lane >= o) inc += n;
                }
                if (lane == 31) red[warp] = inc;
                if (tid == 0) s_dsel = kRadix;
                __syncthreads();
                if (warp == 0) {
                    long long w = lane < nw ? red[lane] : 0;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const long long n = __shfl_up_sync(kFull, w, o);
                        if (lane >= o) w += n;
                    }
                    if (lane < nw) red[lane] = w;   // inclusive totals of warps 0..lane
                }
                __syncthreads();
                const long long before = (warp > 0 ? red[warp - 1] : 0) + inc - (h0 + h1);
                const long long rem = s_rem;
                int mine = kRadix;
                if (h1 > 0 && before + h0 + h1 > rem) mine = b0 + 1;
                if (h0 > 0 && before + h0 > rem) mine = b0;
                if (mine < kRadix) atomicMin(&s_dsel, mine);
                __syncthreads();
                const int dsel = s_dsel;
                if (dsel < kRadix && (dsel >> 1) == tid) s_cum = dsel == b0 ? before : before + h0;
                __syncthreads();
                if (tid == 0) {
                    if (dsel == kRadix) {
                        s_found = 0;  // every remaining candidate fits in the budget
                    } else {
                        s_rem -= s_cum;
                        s_prefix |= (unsigned long long)dsel << sh;
                        s_mask |= dmask << sh;
                        s_unique = hcnt[dsel] == 1;
                    }
                }
            }
            __syncthreads();
            if (!s_found) break;
            unique = s_unique;
        }
        if (s_found && unique) {
            // the lone candidate under the prefix: its full key
            const unsigned long long prefix = s_prefix, mask = s_mask;
            if (lane_ok && gk_ok) {
                for (int a = tid / Gk; a < Gq; a += astep) {
                    if (qs[a] == 0 || mand[a] == gk0) continue;
                    const long long c = (long long)a * Gk + gk0;
                    const unsigned long long key =
                        ((unsigned long long)(~__float_as_uint(S[c])) << 32) | (unsigned long long)c;
                    if ((key & mask) == prefix) s_prefix = key;
                }
            }
            __syncthreads();
        }
    }
    const int found = s_found;
    const unsigned long long kstar = s_prefix;
    const long long under = s_rem;
    bool take_star = false;
    if (found) {
        const long long cstar = (long long)(kstar & 0xffffffffull);
        const long long cost = (long long)qs[cstar / Gk] * ks[cstar % Gk];
        take_star = (cost - under) < under;
    }

    // Row counts, then CSR in ascending key-group order.
    long long psum = 0;
    for (int a = warp; a < Gq; a += nw) {
        int cnt = 0;
        for (int g0 = 0; g0 < Gk; g0 += 32) {
            const int gk = g0 + lane;
            bool sel = false;
            if (gk < Gk && qs[a] > 0 && ks[gk] > 0) {
                const long long c = (long long)a * Gk + gk;
                if (keep_all || mand[a] == gk || !found) {
                    sel = true;
                } else {
                    const unsigned long long key =
                        ((unsigned long long)(~__float_as_uint(S[c])) << 32) | (unsigned long long)c;
                    sel = key < kstar || (key == kstar && take_star);
                }
            }
            const unsigned b = __ballot_sync(kFull, sel);
            cnt += __popc(b);
            if (sel) psum += (long long)qs[a] * ks[gk];
        }
        if (lane == 0) rowcnt[a] = cnt;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(kFull, psum, o);
    __syncthreads();
    if (lane == 0) red[warp] = psum;
    __syncthreads();
    if (tid == 0) {
        long long tot = 0;
        for (int w = 0; w < nw; ++w) tot += red[w];
        pairs[z] = tot;
        int s = 0;
        int32_t* rp = rowptr + (long long)z * (Gq + 1);
        for (int a = 0; a < Gq; ++a) { int v = rowcnt[a]; rp[a] = s; rowcnt[a] = s; s += v; }
        rp[Gq] = s;
    }
    __syncthreads();
    int32_t* kz = kg + (long long)z * Gq * Gk;
    for (int a = warp; a < Gq; a += nw) {
        int base = rowcnt[a];
        for (int g0 = 0; g0 < Gk; g0 += 32) {
            const int gk = g0 + lane;
            bool sel = false;
            if (gk < Gk && qs[a] > 0 && ks[gk] > 0) {
                const long long c = (long long)a * Gk + gk;
                if (keep_all || mand[a] == gk || !found) {
                    sel = true;
                } else {
                    const unsigned long long key =
                        ((unsigned long long)(~__float_as_uint(S[c])) << 32) | (unsigned long long)c;
                    sel = key < kstar || (key == kstar && take_star);
                }
            }
            const unsigned b = __ballot_sync(kFull, sel);
            if (sel) kz[base + __popc(b & ((1u << lane) - 1u))] = gk;
            base += __popc(b);
        }
    }
}

}  // namespace

cudaError_t launch_row_lse(const float* u, const int32_t* koff, float* lse, int Hp, int g, int N,
                           int Gk, cudaStream_t s) {
    dim3 grid((N + 7) / 8, Hp);
    row_lse_kernel<<<grid, 256, 0, s>>>(u, koff, lse, g, N, Gk);
    return cudaGetLastError();
}

cudaError_t launch_cell_scores(const float* u, const float* lse, const int32_t* qperm,
                               const int32_t* qoff, const int32_t* koff, float* scores, int P,
                               int g, int N, int Gq, int Gk, cudaStream_t s) {
    cell_scores_kernel<<<dim3(Gq, P), kCsThreads, 0, s>>>(u, lse, qperm, qoff, koff, scores, g, N, Gq, Gk);
    return cudaGetLastError();
}

cudaError_t launch_route_select(const float* scores, const int32_t* qoff, const int32_t* koff,
                                int32_t* rowptr, int32_t* kg, int64_t* pairs, int P, int Gq,
                                int Gk, long long budget, bool keep_all, cudaStream_t s) {
    size_t smem = (size_t)(3 * Gq + Gk) * sizeof(int);
    route_select_kernel<<<P, kSelThreads, smem, s>>>(scores, qoff, koff, rowptr, kg, pairs, Gq, Gk,
                                                     budget, keep_all ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace spr
