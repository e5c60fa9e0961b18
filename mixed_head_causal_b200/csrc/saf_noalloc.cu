// Allocation-free variant of the backward pass.
//
// Some callers cannot hand the library a device workspace: code that runs
// where cudaMalloc is off limits (inside a custom allocator's own callbacks,
// under a framework that owns every device byte and forbids side allocations,
// or on a path that must never block on the allocator), and callers that
// simply have no allocator object to give.  For them,
// saf_mixed_attn_bwd_noalloc keeps its scratch (the per-row terms
// D = rowsum(dO o O) and, when the caller passes no logz, the replaced heads'
// log-normalisers) in one file-scope device array instead of a workspace.
//
// That array is kNoAllocScratchBytes per GPU, is created when the library is
// loaded on a device and lives until the process exits.  Every call shares
// it: two calls that overlap on the GPU (different streams, or different
// host threads) race on it and give wrong results.  The array keeps whatever
// the previous call left; nothing in it has to start at zero, because both
// regions are fully written before they are read in each call.
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "saf_common.cuh"

namespace saf {
namespace {

// 8 MiB: room for B*H*T + H*T fp32 values up to 2,097,152 (for example
// B=4, H=32, T=8192 with the log-normalisers computed in the call).
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
constexpr size_t kNoAllocScratchFloats = kNoAllocScratchBytes / sizeof(float);

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  Host code
// cannot use the symbol itself (that is a host-side stand-in), so this asks
// the runtime once per device, with that device current.
saf_status scratch_on_current_device(float** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SAF_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        float* p = nullptr;
        if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_noalloc_scratch) != cudaSuccess || !p)
            return SAF_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return SAF_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace saf

using namespace saf;

extern "C" {

saf_status saf_mixed_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                      const void* dout, const float* lse, const float* a, const float* r,
                                      const float* logz, const uint8_t* replaced_mask, int B, int H, int T,
                                      int d_h, void* dq, void* dk, void* dv, int grad_dtype, void* stream) {
    if (B < 0 || H < 0 || T < 0) return SAF_ERR_INVALID_ARG;
    if (d_h != kHeadDim || H > kMaxHeads) return SAF_ERR_UNSUPPORTED;
    if (grad_dtype != 0 && grad_dtype != 1) return SAF_ERR_UNSUPPORTED;
    if ((int64_t)T * kHeadDim > (int64_t)INT32_MAX) return SAF_ERR_INVALID_ARG;
    const int64_t rows = (int64_t)B * H * T;
    if (rows == 0) return SAF_OK;
    if (H > 0 && replaced_mask == nullptr) return SAF_ERR_INVALID_ARG;
    HeadList hl;
    memset(&hl, 0, sizeof(hl));
    for (int h = 0; h < H; ++h)
        if (replaced_mask[h]) {
            hl.replaced[h] = 1;
            hl.heads[hl.n++] = (int16_t)h;
        }
    // scratch needed: D for every row, plus log Z when the caller has none
    const int64_t rows_padded = (rows + 63) & ~int64_t(63);
    const int64_t need = rows_padded + ((hl.n > 0 && logz == nullptr) ? (int64_t)H * T : 0);
    if (need > (int64_t)kNoAllocScratchFloats) return SAF_ERR_WORKSPACE;
    if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return SAF_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
        !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return SAF_ERR_INVALID_ARG;
    if (hl.n > 0 && (!a || !r || !aligned16(a) || !aligned16(r) || (logz && !aligned16(logz))))
        return SAF_ERR_INVALID_ARG;

    float* scratch = nullptr;
    saf_status st = scratch_on_current_device(&scratch);
    if (st != SAF_OK) return st;
    float* dvec = scratch;                 // [B, H, T]
    float* lzs = scratch + rows_padded;    // [H, T], 256-byte aligned
    cudaStream_t s = (cudaStream_t)stream;
    const float* lz = logz;
    if (hl.n > 0 && lz == nullptr) {
        if (launch_lognorm(a, r, hl, T, lzs, s) != cudaSuccess) return SAF_ERR_CUDA;
        lz = lzs;
    }
    if (launch_bwd_dot(static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), dvec,
                       hl, B, H, T, s) != cudaSuccess)
        return SAF_ERR_CUDA;
    return launch_bwd_mma(static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                          static_cast<const __nv_bfloat16*>(v), static_cast<const __nv_bfloat16*>(dout), lse,
                          dvec, a, r, lz, hl, B, H, T, dq, dk, dv, grad_dtype, s) == cudaSuccess
               ? SAF_OK
               : SAF_ERR_CUDA;
}

}  // extern "C"
