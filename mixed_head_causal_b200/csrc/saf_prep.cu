// Small preparation kernels of the mixed-head layer.
//
//  * lognorm: the per-row log-normaliser of a replaced head's compact
//    pattern, log Z(i) = log sum_{k<=i} exp(a[k] + r[i-k])  (Eq. (3) of
//    "When Can Attention Heads Be Statically Defined?", section 二.3).  It
//    depends on a and r only, so it is computed once per head, not per batch.
//  * dot: the backward row term D[i] = sum_c dO[i,c] O[i,c] of softmax
//    attention (equal to sum_j P[i,j] dP[i,j]), one fp32 value per row.
#include "saf_common.cuh"

namespace saf {
namespace {


// Merge two (max, sum-of-exp2) pairs of a log2-domain log-sum-exp.
__device__ __forceinline__ void lse2_merge(float& m, float& s, float m2, float s2) {
    float M = fmaxf(m, m2);
    if (M == kNegInf) return;  // both empty
    float a = (m == kNegInf) ? 0.f : s * exp2f(m - M);
    float b = (m2 == kNegInf) ? 0.f : s2 * exp2f(m2 - M);
    m = M;
    s = a + b;
}

// One warp per row i of one replaced head; lanes stride over k and keep an
// online (max, sum) pair, merged across the warp at the end.
__global__ void __launch_bounds__(256) lognorm_kernel(const float* __restrict__ a,
                                                      const float* __restrict__ r,
                                                      HeadList hl, int T,
                                                      float* __restrict__ logz) {
    const int h = hl.heads[blockIdx.y];
    const int i = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (i >= T) return;
    const float* ah = a + (size_t)h * T;
    const float* rh = r + (size_t)h * T;
    float m = kNegInf, s = 0.f;
    for (int k = lane; k <= i; k += 32) {
        float x = (ah[k] + rh[i - k]) * kLog2e;
        if (x == kNegInf) continue;
        if (x > m) {
            s = (m == kNegInf ? 0.f : s * exp2f(m - x)) + 1.f;
            m = x;
        } else {
            s += exp2f(x - m);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        float m2 = __shfl_xor_sync(0xffffffffu, m, off);
        float s2 = __shfl_xor_sync(0xffffffffu, s, off);
        lse2_merge(m, s, m2, s2);
    }
    if (lane == 0) logz[(size_t)h * T + i] = (m == kNegInf) ? kNegInf : (m + log2f(s)) * kLn2;
}

// 8 threads per row, 16 bytes (8 bf16) of O and dO each.
__global__ void __launch_bounds__(256) dot_kernel(const __nv_bfloat16* __restrict__ o,
                                                  const __nv_bfloat16* __restrict__ dout,
                                                  float* __restrict__ dvec, int64_t rows) {
    const int64_t row = (int64_t)blockIdx.x * 32 + (threadIdx.x >> 3);
    const int part = threadIdx.x & 7;
    float acc = 0.f;
    if (row < rows) {
        const uint4 ov = *reinterpret_cast<const uint4*>(o + row * kHeadDim + part * 8);
        const uint4 dv = *reinterpret_cast<const uint4*>(dout + row * kHeadDim + part * 8);
        const __nv_bfloat162* op = reinterpret_cast<const __nv_bfloat162*>(&ov);
        const __nv_bfloat162* dp = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 a = __bfloat1622float2(op[e]);
            float2 b = __bfloat1622float2(dp[e]);
            acc = fmaf(a.x, b.x, acc);
            acc = fmaf(a.y, b.y, acc);
        }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    if (row < rows && part == 0) dvec[row] = acc;
}

}  // namespace

cudaError_t launch_lognorm(const float* a, const float* r, const HeadList& hl, int T,
                           float* logz, cudaStream_t stream) {
    if (hl.n == 0 || T == 0) return cudaSuccess;
    dim3 grid((T + 7) / 8, hl.n);
    launch_begin(KID_LOGNORM, stream);
    lognorm_kernel<<<grid, 256, 0, stream>>>(a, r, hl, T, logz);
    launch_end(KID_LOGNORM, stream);
    return cudaGetLastError();
}

cudaError_t launch_bwd_dot(const __nv_bfloat16* o, const __nv_bfloat16* dout, float* dvec,
                           const HeadList& hl, int B, int H, int T, cudaStream_t stream) {
    (void)hl;
    const int64_t rows = (int64_t)B * H * T;
    if (rows == 0) return cudaSuccess;
    launch_begin(KID_DOT, stream);
    dot_kernel<<<(unsigned)((rows + 31) / 32), 256, 0, stream>>>(o, dout, dvec, rows);
    launch_end(KID_DOT, stream);
    return cudaGetLastError();
}

}  // namespace saf
