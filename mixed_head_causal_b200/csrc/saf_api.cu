// C ABI of libsaf.so (declared in include/saf.h): argument validation,
// workspace carving and kernel sequencing.  No device memory is allocated
// here; every buffer belongs to the caller.
#include <limits.h>
#include <stdlib.h>
#include <stdint.h>
#include <string.h>

#include "saf_common.cuh"

using namespace saf;

namespace {

constexpr int kVersion = 100;  // 0.1.0
// the fitting kernels stage a, r and log Z of a head in shared memory (3 T floats)
constexpr int kFitMaxT = 16384;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

// Shape checks shared by every entry point.  Sizes must be non-negative and
// every tensor's element count must fit the kernels' 64-bit indexing with
// the per-slice offsets they compute in 32-bit (T * d_h < 2^31).
saf_status check_shape(int B, int H, int T, int d_h) {
    if (B < 0 || H < 0 || T < 0) return SAF_ERR_INVALID_ARG;
    if (d_h != kHeadDim) return SAF_ERR_UNSUPPORTED;
    if (H > kMaxHeads) return SAF_ERR_UNSUPPORTED;
    if ((int64_t)T * kHeadDim > (int64_t)INT_MAX) return SAF_ERR_INVALID_ARG;
    if ((int64_t)B * H > 65535LL * 1024) return SAF_ERR_INVALID_ARG;
    const int64_t bht = (int64_t)B * H * T;
    if (bht > (INT64_MAX / 4) / kHeadDim) return SAF_ERR_INVALID_ARG;
    return SAF_OK;
}

saf_status build_headlist(const uint8_t* mask, int H, HeadList* hl) {
    if (H > 0 && mask == nullptr) return SAF_ERR_INVALID_ARG;
    memset(hl, 0, sizeof(*hl));
    for (int h = 0; h < H; ++h) {
        if (mask[h]) {
            hl->replaced[h] = 1;
            hl->heads[hl->n++] = (int16_t)h;
        }
    }
    return SAF_OK;
}

inline saf_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SAF_OK : SAF_ERR_CUDA; }

// K/V heads: at least one, dividing H (H == 0 allows any positive count).
saf_status check_groups(int H, int H_kv) {
    if (H_kv <= 0) return SAF_ERR_INVALID_ARG;
    if (H > 0 && (H_kv > H || H % H_kv != 0)) return SAF_ERR_INVALID_ARG;
    return SAF_OK;
}

// SAF_FORCE_MMA=1 in the environment routes every head through the
// warp-level mma.sync kernels (the per-element path), for comparisons.
bool force_mma_path() {
    const char* e = getenv("SAF_FORCE_MMA");
    return e && e[0] == '1';
}

}  // namespace

extern "C" {

const char* saf_status_string(saf_status status) {
    switch ((int)status) {  // any int a C caller passes, known or not
        case SAF_OK: return "SAF_OK";
        case SAF_ERR_INVALID_ARG: return "SAF_ERR_INVALID_ARG";
        case SAF_ERR_UNSUPPORTED: return "SAF_ERR_UNSUPPORTED";
        case SAF_ERR_WORKSPACE: return "SAF_ERR_WORKSPACE";
        case SAF_ERR_CUDA: return "SAF_ERR_CUDA";
        case SAF_ERR_TIMEOUT: return "SAF_ERR_TIMEOUT";
        default: return "SAF_ERR_UNKNOWN";
    }
}

int saf_version(void) { return kVersion; }

size_t saf_workspace_size_gqa(int B, int H, int H_kv, int T, int d_h, int is_bwd) {
    if (check_shape(B, H, T, d_h) != SAF_OK || check_groups(H, H_kv) != SAF_OK) return (size_t)-1;
    if ((int64_t)B * H * T == 0) return 0;
    return ws_layout(B, H, T, is_bwd ? 1 : 0, H_kv).total;
}

size_t saf_workspace_size(int B, int H, int T, int d_h, int is_bwd) {
    return saf_workspace_size_gqa(B, H, H, T, d_h, is_bwd);
}

saf_status saf_replaced_lognorm(const float* a, const float* r, const uint8_t* replaced_mask,
                                int H, int T, float* logz, void* stream) {
    saf_status st = check_shape(1, H, T, kHeadDim);
    if (st != SAF_OK) return st;
    if ((int64_t)H * T == 0) return SAF_OK;
    HeadList hl;
    st = build_headlist(replaced_mask, H, &hl);
    if (st != SAF_OK) return st;
    if (hl.n == 0) return SAF_OK;
    if (!a || !r || !logz) return SAF_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(r) || !aligned16(logz)) return SAF_ERR_INVALID_ARG;
    return cuda_status(launch_lognorm(a, r, hl, T, logz, (cudaStream_t)stream));
}

saf_status saf_mixed_attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                                  const float* a, const float* r, const float* logz,
                                  const uint8_t* replaced_mask, int B, int H, int H_kv, int T, int d_h,
                                  void* workspace, size_t workspace_bytes, void* stream) {
    saf_status st = check_shape(B, H, T, d_h);
    if (st != SAF_OK) return st;
    st = check_groups(H, H_kv);
    if (st != SAF_OK) return st;
    if ((int64_t)B * H * T == 0) return SAF_OK;
    HeadList hl;
    st = build_headlist(replaced_mask, H, &hl);
    if (st != SAF_OK) return st;
    if (!q || !k || !v || !o || !lse) return SAF_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return SAF_ERR_INVALID_ARG;
    if (hl.n > 0) {
        if (!a || !r) return SAF_ERR_INVALID_ARG;
        if (!aligned16(a) || !aligned16(r) || (logz && !aligned16(logz))) return SAF_ERR_INVALID_ARG;
    }
    const WsLayout L = ws_layout(B, H, T, 0, H_kv);
    if (!workspace || workspace_bytes < L.total) return SAF_ERR_WORKSPACE;
    if (!aligned256(workspace)) return SAF_ERR_INVALID_ARG;

    cudaStream_t s = (cudaStream_t)stream;
    char* ws = static_cast<char*>(workspace);
    // log Z: the caller's, or computed into the workspace
    float* lzw = reinterpret_cast<float*>(ws + L.logz);
    const float* lz = logz ? logz : lzw;
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
    const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k);
    const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(v);
    __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(o);
    if (force_mma_path()) {
        if (H_kv != H) return SAF_ERR_UNSUPPORTED;  // the warp-level path has no shared K/V
        if (hl.n > 0 && !logz && launch_lognorm(a, r, hl, T, lzw, s) != cudaSuccess) return SAF_ERR_CUDA;
        return cuda_status(launch_fwd_mma(qb, kb, vb, ob, lse, a, r, lz, hl, B, H, T, s));
    }
    // one launch prepares the replaced heads' patterns (log Z and the factored
    // arrays), one runs the layer
    const ReplacedWs rw = replaced_ws(ws, L, T);
    if (hl.n > 0 && launch_pattern(a, r, logz, logz ? nullptr : lzw, hl, T, &rw, s) != cudaSuccess)
        return SAF_ERR_CUDA;
    cudaError_t e = launch_fwd_tc(qb, kb, vb, ob, lse, a, r, lz, hl, rw, B, H, H_kv, T,
                                  reinterpret_cast<unsigned int*>(ws), hl.n > 0, s);
    if (e == cudaErrorNotSupported) return SAF_ERR_UNSUPPORTED;
    if (e != cudaSuccess) return SAF_ERR_CUDA;
    return SAF_OK;
}

saf_status saf_mixed_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                              const float* a, const float* r, const float* logz,
                              const uint8_t* replaced_mask, int B, int H, int T, int d_h,
                              void* workspace, size_t workspace_bytes, void* stream) {
    return saf_mixed_attn_fwd_gqa(q, k, v, o, lse, a, r, logz, replaced_mask, B, H, H, T, d_h, workspace,
                                  workspace_bytes, stream);
}

saf_status saf_mixed_attn_bwd_gqa(const void* q, const void* k, const void* v, const void* o,
                                  const void* dout, const float* lse, const float* a, const float* r,
                                  const float* logz, const uint8_t* replaced_mask, int B, int H, int H_kv,
                                  int T, int d_h, void* dq, void* dk, void* dv, int grad_dtype,
                                  void* workspace, size_t workspace_bytes, void* stream) {
    saf_status st = check_shape(B, H, T, d_h);
    if (st != SAF_OK) return st;
    st = check_groups(H, H_kv);
    if (st != SAF_OK) return st;
    if (grad_dtype != 0 && grad_dtype != 1) return SAF_ERR_UNSUPPORTED;
    if ((int64_t)B * H * T == 0) return SAF_OK;
    HeadList hl;
    st = build_headlist(replaced_mask, H, &hl);
    if (st != SAF_OK) return st;
    if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return SAF_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
        !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return SAF_ERR_INVALID_ARG;
    if (hl.n > 0) {
        if (!a || !r) return SAF_ERR_INVALID_ARG;
        if (!aligned16(a) || !aligned16(r) || (logz && !aligned16(logz))) return SAF_ERR_INVALID_ARG;
    }
    const WsLayout L = ws_layout(B, H, T, 1, H_kv);
    if (!workspace || workspace_bytes < L.total) return SAF_ERR_WORKSPACE;
    if (!aligned256(workspace)) return SAF_ERR_INVALID_ARG;

    cudaStream_t s = (cudaStream_t)stream;
    char* ws = static_cast<char*>(workspace);
    float* lzw = reinterpret_cast<float*>(ws + L.logz);
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
    const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k);
    const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(v);
    const __nv_bfloat16* ob = static_cast<const __nv_bfloat16*>(o);
    const __nv_bfloat16* dob = static_cast<const __nv_bfloat16*>(dout);
    if (force_mma_path()) {
        if (H_kv != H) return SAF_ERR_UNSUPPORTED;  // the warp-level path has no shared K/V
        const float* lz = logz ? logz : lzw;
        if (hl.n > 0 && !logz && launch_lognorm(a, r, hl, T, lzw, s) != cudaSuccess) return SAF_ERR_CUDA;
        float* dvec = reinterpret_cast<float*>(ws + L.dvec);
        if (launch_bwd_dot(ob, dob, dvec, hl, B, H, T, s) != cudaSuccess) return SAF_ERR_CUDA;
        return cuda_status(launch_bwd_mma(qb, kb, vb, dob, lse, dvec, a, r, lz, hl, B, H, T, dq, dk, dv,
                                          grad_dtype, s));
    }
    const ReplacedWs rw = replaced_ws(ws, L, T);
    float* nlse2p = reinterpret_cast<float*>(ws + L.nlse2p);
    float* dvecp = reinterpret_cast<float*>(ws + L.dvecp);
    float* dqacc = reinterpret_cast<float*>(ws + L.dqacc);
    // log Z: the caller's, or batch 0's lse rows of the replaced heads (the
    // forward wrote log Z there, laid out [H, T] like logz)
    const float* lz = logz ? logz : lse;
    // one launch: the row terms, the zeroed dQ accumulator, and the replaced
    // heads' factored arrays
    if (launch_bwd_pre(ob, dob, lse, B * H, T, nlse2p, dvecp, dqacc, a, r, lz, nullptr, hl, rw, s) != cudaSuccess)
        return SAF_ERR_CUDA;
    // shared K/V: per-query-head fp32 dK, dV into the workspace, then summed per group
    const bool grouped = H_kv != H;
    float* dkh = grouped ? reinterpret_cast<float*>(ws + L.dkh) : nullptr;
    float* dvh = grouped ? reinterpret_cast<float*>(ws + L.dvh) : nullptr;
    cudaError_t e = launch_bwd_tc(qb, kb, vb, dob, nlse2p, dvecp, dqacc, a, r, lz, hl, rw, B, H, H_kv, T,
                                  grouped ? dkh : dk, grouped ? dvh : dv, grouped ? 1 : grad_dtype,
                                  reinterpret_cast<unsigned int*>(ws), s);
    if (e == cudaErrorNotSupported) return SAF_ERR_UNSUPPORTED;
    if (e != cudaSuccess) return SAF_ERR_CUDA;
    if (launch_dq_convert(dqacc, dq, (int64_t)B * H * T, grad_dtype, s) != cudaSuccess) return SAF_ERR_CUDA;
    if (grouped) {
        if (launch_group_sum(dkh, dk, B, H, H_kv, T, grad_dtype, s) != cudaSuccess) return SAF_ERR_CUDA;
        if (launch_group_sum(dvh, dv, B, H, H_kv, T, grad_dtype, s) != cudaSuccess) return SAF_ERR_CUDA;
    }
    return SAF_OK;
}

saf_status saf_mixed_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                              const void* dout, const float* lse, const float* a, const float* r,
                              const float* logz, const uint8_t* replaced_mask, int B, int H, int T,
                              int d_h, void* dq, void* dk, void* dv, int grad_dtype,
                              void* workspace, size_t workspace_bytes, void* stream) {
    return saf_mixed_attn_bwd_gqa(q, k, v, o, dout, lse, a, r, logz, replaced_mask, B, H, H, T, d_h, dq, dk, dv,
                                  grad_dtype, workspace, workspace_bytes, stream);
}

size_t saf_fit_workspace_size(int n_heads, int T) {
    if (n_heads < 0 || n_heads > kMaxHeads || T < 0 || T > kFitMaxT) return (size_t)-1;
    return fit_workspace_bytes(n_heads, T);
}

saf_status saf_fit_pattern(const float* target, int n_heads, int T, int steps, float lr, float* a, float* r,
                           float* kl, void* workspace, size_t workspace_bytes, void* stream) {
    if (n_heads < 0 || T < 0 || steps < 0 || !(lr > 0.f)) return SAF_ERR_INVALID_ARG;
    if (n_heads > kMaxHeads || T > kFitMaxT) return SAF_ERR_UNSUPPORTED;
    if ((int64_t)n_heads * T == 0) return SAF_OK;
    if (!target || !a || !r || !kl) return SAF_ERR_INVALID_ARG;
    if (!aligned16(target) || !aligned16(a) || !aligned16(r) || !aligned16(kl)) return SAF_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < fit_workspace_bytes(n_heads, T)) return SAF_ERR_WORKSPACE;
    if (!aligned256(workspace)) return SAF_ERR_INVALID_ARG;
    return cuda_status(launch_fit(target, n_heads, T, steps, lr, a, r, kl, workspace, (cudaStream_t)stream));
}

size_t saf_calibration_workspace_size(int H, int T, int d_h) {
    if (check_shape(1, H, T, d_h) != SAF_OK) return (size_t)-1;
    return sizeof(float) * calibration_partial_floats(H, T);
}

saf_status saf_attn_calibration(const void* q, const void* k, const float* lse, int N, int H, int T, int d_h,
                                float* a_hat, float* svar, void* workspace, size_t workspace_bytes, void* stream) {
    saf_status st = check_shape(N, H, T, d_h);
    if (st != SAF_OK) return st;
    if (N < 2) return SAF_ERR_INVALID_ARG;  // Eq. (1) divides by N - 1
    if ((int64_t)H * T == 0) return SAF_OK;
    if ((double)H * T * T > 9.0e18 / sizeof(float)) return SAF_ERR_INVALID_ARG;
    if (!q || !k || !lse || !a_hat || !svar) return SAF_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(lse) || !aligned16(a_hat) || !aligned16(svar))
        return SAF_ERR_INVALID_ARG;
    const size_t need = sizeof(float) * calibration_partial_floats(H, T);
    if (!workspace || workspace_bytes < need) return SAF_ERR_WORKSPACE;
    if (!aligned16(workspace)) return SAF_ERR_INVALID_ARG;
    return cuda_status(launch_calibration(static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                                          lse, N, H, T, a_hat, svar, static_cast<float*>(workspace),
                                          (cudaStream_t)stream));
}

saf_status saf_replaced_pattern_grad(const void* v, const void* dout, const float* a, const float* r,
                                     const float* logz, const uint8_t* replaced_mask, int B, int H, int T,
                                     int d_h, float* da, float* dr, void* workspace, size_t workspace_bytes,
                                     void* stream) {
    saf_status st = check_shape(B, H, T, d_h);
    if (st != SAF_OK) return st;
    if ((int64_t)H * T == 0) return SAF_OK;
    HeadList hl;
    st = build_headlist(replaced_mask, H, &hl);
    if (st != SAF_OK) return st;
    if (!da || !dr || !aligned16(da) || !aligned16(dr)) return SAF_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemsetAsync(da, 0, sizeof(float) * (size_t)H * T, s) != cudaSuccess) return SAF_ERR_CUDA;
    if (cudaMemsetAsync(dr, 0, sizeof(float) * (size_t)H * T, s) != cudaSuccess) return SAF_ERR_CUDA;
    if (hl.n == 0 || B == 0) return SAF_OK;
    if (!v || !dout || !a || !r) return SAF_ERR_INVALID_ARG;
    if (!aligned16(v) || !aligned16(dout) || !aligned16(a) || !aligned16(r) || (logz && !aligned16(logz)))
        return SAF_ERR_INVALID_ARG;
    const float* lz = logz;
    if (lz == nullptr) {
        const WsLayout L = ws_layout(B, H, T, 0);
        if (!workspace || workspace_bytes < L.total) return SAF_ERR_WORKSPACE;
        if (!aligned256(workspace)) return SAF_ERR_INVALID_ARG;
        float* lzw = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.logz);
        if (launch_lognorm(a, r, hl, T, lzw, s) != cudaSuccess) return SAF_ERR_CUDA;
        lz = lzw;
    }
    return cuda_status(launch_pattern_grad(static_cast<const __nv_bfloat16*>(v),
                                           static_cast<const __nv_bfloat16*>(dout), a, r, lz, hl, B, H, T, da, dr,
                                           s));
}

saf_status saf_selftest_wait_timeout(void* workspace, size_t workspace_bytes, long long limit_cycles,
                                     void* stream) {
    if (!workspace || workspace_bytes < sizeof(WsHeader)) return SAF_ERR_WORKSPACE;
    if (!aligned256(workspace) || limit_cycles < 1 || limit_cycles > (1ll << 31)) return SAF_ERR_INVALID_ARG;
    return cuda_status(launch_selftest_wait(static_cast<unsigned int*>(workspace), limit_cycles,
                                            (cudaStream_t)stream));
}

saf_status saf_device_status(void* workspace, size_t workspace_bytes, void* stream) {
    if (!workspace || workspace_bytes < sizeof(WsHeader)) return SAF_ERR_WORKSPACE;
    WsHeader hdr;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&hdr, workspace, sizeof(hdr), cudaMemcpyDeviceToHost, s) != cudaSuccess) return SAF_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SAF_ERR_CUDA;
    if (hdr.error != 0) {
        if (cudaMemsetAsync(workspace, 0, 2 * sizeof(unsigned int), s) != cudaSuccess) return SAF_ERR_CUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return SAF_ERR_CUDA;
        return SAF_ERR_TIMEOUT;
    }
    return SAF_OK;
}

}  // extern "C"
