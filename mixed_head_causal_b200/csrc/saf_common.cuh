// Shared definitions of the sm_100a mixed-head attention library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/saf.h"

namespace saf {

constexpr int kHeadDim = 64;
constexpr int kMaxHeads = 256;         // heads per layer accepted by the ABI
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kNegInf = -__builtin_huge_valf();

// Replaced-head list passed by value to kernels (the mask lives on the host).
struct HeadList {
    int n;
    uint8_t replaced[kMaxHeads];  // per head flag
    int16_t heads[kMaxHeads];     // the first n entries: indices of replaced heads
};

// Problem shape shared by the launchers.
struct Shape {
    int B, H, T;
    int64_t row_stride_bh;  // T * d elements between consecutive (b,h) slices
};

// ---------------------------------------------------------------- workspace
// Offsets of the scratch regions inside the caller's workspace.  Every region
// starts on a 256-byte boundary.
struct WsLayout {
    size_t header;   // device error word + counters (256 B)
    size_t logz;     // [H, T] fp32 (used when the caller passes logz = NULL)
    size_t dvec;     // [B, H, T] fp32 row terms rowsum(dO o O) (backward only)
    size_t total;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(int B, int H, int T, int is_bwd) {
    WsLayout L{};
    size_t off = 0;
    L.header = off; off += 256;
    L.logz = off; off = align256(off + sizeof(float) * (size_t)H * T);
    if (is_bwd) { L.dvec = off; off = align256(off + sizeof(float) * (size_t)B * H * T); }
    L.total = off;
    return L;
}

// Device error word layout (first bytes of the workspace header).
struct WsHeader {
    unsigned int error;       // nonzero after a bounded wait gave up
    unsigned int where;       // which wait (kernel-specific code)
    unsigned int counters[62];
};

// ---------------------------------------------------------------- accounting
// Kernel ids of the launch accounting (names in saf_profile.cu).
enum KernelId {
    KID_LOGNORM = 1, KID_FWD_MMA = 2, KID_DOT = 3, KID_DKDV_MMA = 4, KID_DQ_MMA = 5,
    KID_FWD_TC = 6, KID_BWD_TC = 7, KID_PREP_REPLACED = 8, KID_DQ_CONVERT = 9, KID_BWD_PRE = 10
};
// Every kernel launch of the library is bracketed by these two calls.
void launch_begin(int kid, cudaStream_t s);
void launch_end(int kid, cudaStream_t s);

// ---------------------------------------------------------------- launchers
// (defined in the kernel translation units; all enqueue on `stream`)
cudaError_t launch_lognorm(const float* a, const float* r, const HeadList& hl, int T,
                           float* logz, cudaStream_t stream);
cudaError_t launch_fwd_mma(const __nv_bfloat16* q, const __nv_bfloat16* k,
                           const __nv_bfloat16* v, __nv_bfloat16* o, float* lse,
                           const float* a, const float* r, const float* logz,
                           const HeadList& hl, int B, int H, int T, cudaStream_t stream);
cudaError_t launch_bwd_dot(const __nv_bfloat16* o, const __nv_bfloat16* dout, float* dvec,
                           const HeadList& hl, int B, int H, int T, cudaStream_t stream);
cudaError_t launch_bwd_mma(const __nv_bfloat16* q, const __nv_bfloat16* k,
                           const __nv_bfloat16* v, const __nv_bfloat16* dout,
                           const float* lse, const float* dvec,
                           const float* a, const float* r, const float* logz,
                           const HeadList& hl, int B, int H, int T,
                           void* dq, void* dk, void* dv, int grad_fp32, cudaStream_t stream);

}  // namespace saf
