// Dense attention of given query rows for callers that cannot allocate device memory.
//
// Some callers must not call cudaMalloc: code that runs inside another
// framework's memory manager (which owns every device allocation and would be
// bypassed or re-entered), code running while an allocator lock is held, or a
// process that reserves all of its device memory up front. For them this file
// offers a handle-free variant of the probe-row dense attention (the probe step
// of sparsepr_probe_fit). Its only scratch -- the per-split partial outputs,
// maxima and sums of the split-key pass -- lives in one fixed-size array that
// is compiled into the library, so the call allocates nothing.
#include "common.cuh"
#include "kernels.h"
#include "sparsepr.h"

namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;               // 8 MiB per GPU
constexpr size_t kScratchFloats = kScratchBytes / sizeof(float);
constexpr int kMaxSplits = 32;
constexpr int kKeyTile = 64;

// Split-key partials: Opart [B*Hq][ns][M][d], then mpart and lpart [B*Hq][ns][M].
// Every GPU that loads the library keeps these 8 MiB until the process exits.
static __device__ __align__(256) float g_probe_scratch[kScratchFloats];

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of the scratch array in the current context. The host-side name of the array
// is only a stand-in, so the address is looked up on every call, with the caller's device and
// context current: a cached address would go stale after cudaDeviceReset or point into another
// context when the caller switches contexts through the driver API.
sparsepr_status scratch_in_current_context(float** out) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_probe_scratch) != cudaSuccess || p == nullptr) return SPARSEPR_ERR_CUDA;
    *out = static_cast<float*>(p);
    return SPARSEPR_OK;
}

}  // namespace

extern "C" sparsepr_status sparsepr_probe_attention_noalloc(const void* Q, const void* K, const void* V,
                                                            const int32_t* rows, float* O, int B, int Hq,
                                                            int Hkv, int N, int d, int M, void* stream) {
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !rows || !aligned16(O)) return SPARSEPR_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(rows) & 3u) != 0) return SPARSEPR_ERR_INVALID_ARG;
    if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || N < 1 || M < 1 || M > N) return SPARSEPR_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SPARSEPR_ERR_UNSUPPORTED;
    if (M > 64) return SPARSEPR_ERR_UNSUPPORTED;
    const size_t per_split = (size_t)B * Hq * M * (size_t)(d + 2);   // floats of one key split
    if (per_split > kScratchFloats) return SPARSEPR_ERR_UNSUPPORTED;
    int ns = (int)(kScratchFloats / per_split);
    if (ns > kMaxSplits) ns = kMaxSplits;
    const int tiles = (N + kKeyTile - 1) / kKeyTile;
    if (ns > tiles) ns = tiles;
    float* scratch = nullptr;
    sparsepr_status st = scratch_in_current_context(&scratch);
    if (st != SPARSEPR_OK) return st;
    const size_t hp = (size_t)B * Hq;
    float* Opart = scratch;
    float* mpart = Opart + hp * ns * M * d;
    float* lpart = mpart + hp * ns * M;
    cudaError_t e = spr::launch_attn_probe(static_cast<const spr::bf16*>(Q), static_cast<const spr::bf16*>(K),
                                           static_cast<const spr::bf16*>(V), rows, Opart, mpart, lpart, O, B, Hq,
                                           Hkv, N, d, M, ns, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SPARSEPR_OK : SPARSEPR_ERR_CUDA;
}
