// Shared definitions of the sm_100a mixed-head attention library.
#pragma once

#include <cuda.h>
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

// Device arrays of the factored replaced-head pattern (see prep_replaced in
// saf_prep.cu), one row per replaced-head slot s (slot order = head order).
struct ReplacedWs {
    int Tp, Lp;          // T rounded up to 128; Tp + 256
    int ntiles;          // 32-row tiles of a head: ceil(T / 32)
    uint32_t* epair;     // [slots][Lp]   bf16 pairs {E[x], E[x-1]} at x + 128
    float* ef;           // [slots][Lp]   fp32 E[x] at x + 128
    uint32_t* cpair;     // [slots][Tp/2] bf16 pairs {c[2m], c[2m+1]}
    float* cf;           // [slots][Tp]   fp32 c[j]
    float* rsc;          // [slots][Tp]   fp32 r_i
    int* tflag;          // [slots][ntiles] 1 = a row of the tile needs the per-element
                         // exp path (a head takes it when any of its tiles does)
};

__host__ __device__ inline int round_up128(int x) { return (x + 127) & ~127; }

// Per replaced slot, whether the head takes the per-element path: the OR of
// its tiles' range flags (written by the pattern preparation), into dfl[slot]
// in shared memory.  Called by one warp; a barrier of the block must follow
// before dfl is read.
__device__ __forceinline__ void slot_flags(const ReplacedWs& w, int nslots, uint8_t* dfl) {
    const int lane = threadIdx.x & 31;
    for (int s = 0; s < nslots; ++s) {
        int any = 0;
        for (int t = lane; t < w.ntiles; t += 32) any |= w.tflag[(size_t)s * w.ntiles + t];
        any = __any_sync(0xffffffffu, any != 0);
        if (lane == 0) dfl[s] = (uint8_t)any;
    }
}

// CTA order of the tensor-core kernels.  A CTA does one block-row of one
// (batch, head) slice; its work shrinks with its causal rank (rank 0 = the
// longest).  Slices are taken a group at a time, so the tiles they share stay
// in L2, and inside a group the CTAs run longest first across all its slices,
// so the last CTAs to start are the shortest and the tail is small.  A group
// holds about kGroupItems items: kGroupItems / nblk slices, at least one (32
// slices of 1 MB of K and V at T = 4096, 16 of 2 MB at T = 8192).
constexpr int kGroupItems = 1024;
__host__ __device__ __forceinline__ int head_group(int nblk) { return nblk >= kGroupItems ? 1 : kGroupItems / nblk; }
__host__ __device__ __forceinline__ void grouped_order(unsigned b, int BH, int nblk, int& bh, int& rank) {
    const int group = head_group(nblk);
    const unsigned per_group = (unsigned)group * (unsigned)nblk;
    const int g = (int)(b / per_group);
    const int r = (int)(b - (unsigned)g * per_group);
    const int left = BH - g * group;  // slices in this group (the last one may be partial)
    const int heads = left < group ? left : group;
    rank = r / heads;
    bh = g * group + (r - rank * heads);
}

// ---------------------------------------------------------------- workspace
// Offsets of the scratch regions inside the caller's workspace.  Every region
// starts on a 256-byte boundary.
struct WsLayout {
    size_t header;   // device error word + counters (256 B)
    size_t logz;     // [H, T] fp32 (used when the caller passes logz = NULL)
    size_t dvec;     // [B, H, T] fp32 row terms rowsum(dO o O) (backward only)
    size_t epair, ef, cpair, cf, rsc, tflag;  // factored replaced-head arrays (H slots)
    size_t nlse2p;    // [B*H, Tp] fp32 -lse * log2(e), -inf past T  (backward)
    size_t dvecp;    // [B*H, Tp] fp32 rowsum(dO o O), 0 past T      (backward)
    size_t dqacc;    // [B*H, T, 64] fp32 dQ accumulator              (backward)
    size_t dkh, dvh; // [B*H, T, 64] fp32 per-query-head dK, dV (backward, shared K/V only)
    size_t total;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Hkv < H: K/V shared by groups of H / Hkv query heads.
inline WsLayout ws_layout(int B, int H, int T, int is_bwd, int Hkv = -1) {
    WsLayout L{};
    size_t off = 0;
    L.header = off; off += 256;
    L.logz = off; off = align256(off + sizeof(float) * (size_t)H * T);
    if (is_bwd) { L.dvec = off; off = align256(off + sizeof(float) * (size_t)B * H * T); }
    const size_t Tp = (size_t)round_up128(T), Lp = Tp + 256;
    L.epair = off; off = align256(off + 4 * (size_t)H * Lp);
    L.ef = off; off = align256(off + 4 * (size_t)H * Lp);
    L.cpair = off; off = align256(off + 4 * (size_t)H * (Tp / 2));
    L.cf = off; off = align256(off + 4 * (size_t)H * Tp);
    L.rsc = off; off = align256(off + 4 * (size_t)H * Tp);
    L.tflag = off; off = align256(off + 4 * (size_t)H * (Tp / 32));
    if (is_bwd) {
        const size_t BH = (size_t)B * H;
        L.nlse2p = off; off = align256(off + 4 * BH * Tp);
        L.dvecp = off; off = align256(off + 4 * BH * Tp);
        L.dqacc = off; off = align256(off + 4 * BH * (size_t)T * kHeadDim);
        if (Hkv > 0 && Hkv != H) {
            L.dkh = off; off = align256(off + 4 * BH * (size_t)T * kHeadDim);
            L.dvh = off; off = align256(off + 4 * BH * (size_t)T * kHeadDim);
        }
    }
    L.total = off;
    return L;
}

inline ReplacedWs replaced_ws(char* ws, const WsLayout& L, int T) {
    ReplacedWs w;
    w.Tp = round_up128(T);
    w.Lp = w.Tp + 256;
    w.epair = reinterpret_cast<uint32_t*>(ws + L.epair);
    w.ef = reinterpret_cast<float*>(ws + L.ef);
    w.cpair = reinterpret_cast<uint32_t*>(ws + L.cpair);
    w.cf = reinterpret_cast<float*>(ws + L.cf);
    w.rsc = reinterpret_cast<float*>(ws + L.rsc);
    w.ntiles = (T + 31) / 32;
    w.tflag = reinterpret_cast<int*>(ws + L.tflag);
    return w;
}

// Device error word layout (first bytes of the workspace header).
struct WsHeader {
    unsigned int error;       // nonzero after a bounded wait gave up
    unsigned int where;       // which wait (kernel-specific code)
    unsigned int counters[62];
};
// Work-queue counters of the persistent kernels, as word indices into the
// header: the next unclaimed item and the number of CTAs that have finished
// (the last one resets both to zero for the next launch).
constexpr int kCtrFwdNext = 2, kCtrFwdDone = 3, kCtrBwdNext = 4, kCtrBwdDone = 5;

// Index checks of the checked build (compiled with -DSAF_CHECKED, built as
// libsaf_checked.so for tests): SAF_CHECKED_OK(err, cond, code) is `cond`
// there and records a failed check in the workspace error word (bit 0, and
// `code` in word 1 if none was recorded yet), so that the caller skips the
// access it guards and the host reads SAF_ERR_TIMEOUT-class status from
// saf_device_status; in the regular build it is `true` and compiles away.
#ifdef SAF_CHECKED
__device__ __forceinline__ bool saf_checked_ok(unsigned int* err, bool cond, unsigned int code) {
    if (!cond) {
        atomicOr(err, 1u);
        atomicCAS(err + 1, 0u, code);
    }
    return cond;
}
#define SAF_CHECKED_OK(err, cond, code) saf_checked_ok((err), (cond), (code))
#else
#define SAF_CHECKED_OK(err, cond, code) true
#endif

// Number of SMs of the current device (cached per device).
int sm_count();

// ---------------------------------------------------------------- accounting
// Kernel ids of the launch accounting (names in saf_profile.cu).
enum KernelId {
    KID_PATTERN = 1, KID_FWD_MMA = 2, KID_DOT = 3, KID_DKDV_MMA = 4, KID_DQ_MMA = 5,
    KID_FWD_TC = 6, KID_BWD_TC = 7, /* 8: retired */ KID_DQ_CONVERT = 9, KID_BWD_PRE = 10,
    KID_GROUP_SUM = 11, KID_PATTERN_GRAD = 12, KID_CALIBRATION = 13, KID_FIT = 14
};
// Every kernel launch of the library is bracketed by these two calls.
void launch_begin(int kid, cudaStream_t s);
void launch_end(int kid, cudaStream_t s);

// ---------------------------------------------------------------- launchers
// (defined in the kernel translation units; all enqueue on `stream`)
// log Z of the replaced heads into logz [H, T] (the pattern preparation with
// no factored arrays).
cudaError_t launch_lognorm(const float* a, const float* r, const HeadList& hl, int T,
                           float* logz, cudaStream_t stream);
// Pattern preparation of the replaced heads, one launch: log Z (taken from
// logz_in, or computed and written to logz_out) and, when w is non-null, the
// factored arrays and their range flags.
cudaError_t launch_pattern(const float* a, const float* r, const float* logz_in, float* logz_out, const HeadList& hl,
                           int T, const ReplacedWs* w, cudaStream_t stream);
// Tensor-core forward of every head (replaced heads whose factored form would
// leave fp32 range, flag 1, take per-element exps of a + r - log Z); returns
// cudaErrorNotSupported when the tensor maps cannot be built.
// k, v hold Hkv heads; query head h reads K/V head h / (H / Hkv).
// after_pattern: the launch right before it on the stream is this call's
// pattern preparation, which the kernel then overlaps (programmatic launch).
cudaError_t launch_fwd_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                          __nv_bfloat16* o, float* lse, const float* a, const float* r, const float* logz,
                          const HeadList& hl, const ReplacedWs& w, int B, int H, int Hkv, int T, unsigned int* err,
                          bool after_pattern, cudaStream_t stream);
// Backward preprocessing for the tensor-core backward, one launch: padded
// -lse*log2(e) and rowsum(dO o O), a zeroed dQ accumulator, and (hl.n > 0)
// the replaced heads' pattern preparation (what launch_pattern does: log Z
// from logz_in or into logz_out, and the factored arrays).
cudaError_t launch_bwd_pre(const __nv_bfloat16* o, const __nv_bfloat16* dout, const float* lse, int BH, int T,
                           float* nlse2p, float* dvecp, float* dqacc, const float* a, const float* r,
                           const float* logz_in, float* logz_out, const HeadList& hl, const ReplacedWs& w,
                           cudaStream_t stream);
// Tensor-core backward (dK, dV written; dQ reduced into dqacc); replaced
// heads with the per-element flag take exps of a + r - log Z.
// (dk, dv per query head: [B, H, T, 64]; with shared K/V the caller sums them
// over each group with launch_group_sum)
cudaError_t launch_bwd_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                          const __nv_bfloat16* dout, const float* nlse2p, const float* dvecp, float* dqacc,
                          const float* a, const float* r, const float* logz, const HeadList& hl,
                          const ReplacedWs& w, int B, int H, int Hkv, int T, void* dk, void* dv, int grad_fp32,
                          unsigned int* err, cudaStream_t stream);
// Failure-path self-test: a bounded wait on an mbarrier nobody completes.
cudaError_t launch_selftest_wait(unsigned int* err, long long limit, cudaStream_t stream);
// Pattern fitting of nslots targets [nslots, T, T]: alpha, rho [nslots, T], kl [nslots];
// `ws` holds fit_workspace_bytes(nslots, T) bytes (256-byte aligned).
size_t fit_workspace_bytes(int nslots, int T);
cudaError_t launch_fit(const float* target, int nslots, int T, int steps, float lr, float* alpha, float* rho,
                       float* kl, void* ws, cudaStream_t stream);
// Calibration statistics over N samples (q, k [N, H, T, 64], lse [N, H, T]):
// A_hat [H, T, T] and s_var [H]; `partial` holds calibration_partial_floats(H, T) floats.
size_t calibration_partial_floats(int H, int T);
cudaError_t launch_calibration(const __nv_bfloat16* q, const __nv_bfloat16* k, const float* lse, int N, int H,
                               int T, float* a_hat, float* svar, float* partial, cudaStream_t stream);
// Trainable pattern: adds dalpha, drho [H, T] of the replaced heads (zeroed by the caller).
cudaError_t launch_pattern_grad(const __nv_bfloat16* v, const __nv_bfloat16* dout, const float* a, const float* r,
                                const float* logz, const HeadList& hl, int B, int H, int T, float* da, float* dr,
                                cudaStream_t stream);
// dst[b, g] = sum of the H / Hkv fp32 rows src[b, h] of group g, [B, Hkv, T, 64] in the output dtype.
// dq = dqacc / sqrt(d_h) in the requested dtype.
cudaError_t launch_dq_convert(const float* dqacc, void* dq, int64_t rows, int grad_fp32, cudaStream_t stream);
cudaError_t launch_group_sum(const float* src, void* dst, int B, int H, int Hkv, int T, int grad_fp32,
                             cudaStream_t stream);
// bf16 [BH, T, 64] as a 3-D tensor map (d, t, bh); boxes of box_rows x
// box_cols (128 or 32 columns, with the 128- or 64-byte swizzle).
bool make_tmap_bhtd(const void* base, int BH, int T, CUtensorMap* out, int box_rows = 128, int box_cols = 64);
bool make_tmap_bhtd_f32(const void* base, int BH, int T, CUtensorMap* out);
// Warp-level (mma.sync) forward and backward of every head, the reference
// path selected by SAF_FORCE_MMA.
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
