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

__device__ float block_reduce(float v, bool is_max, float* red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        float o = __shfl_xor_sync(0xffffffffu, v, off);
        v = is_max ? fmaxf(v, o) : fminf(v, o);
    }
    if (lane == 0) red[wid] = v;
    __syncthreads();
    if (wid == 0) {
        v = lane < (int)(blockDim.x >> 5) ? red[lane] : (is_max ? kNegInf : -kNegInf);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            float o = __shfl_xor_sync(0xffffffffu, v, off);
            v = is_max ? fmaxf(v, o) : fminf(v, o);
        }
        if (lane == 0) red[32] = v;
    }
    __syncthreads();
    v = red[32];
    __syncthreads();
    return v;
}

// Factored form of a replaced head's pattern,
//   P(i,j) = r_i * E[i-j] * c_j,  E[d] = exp(r[d] - R),  c_j = exp(a[j] - A),
//   r_i = exp(A + R - log Z(i)),  A = max a, R = max r,
// which is Eq. (3) rearranged (exp of a sum is the product of exps).  One CTA
// per replaced head writes, for the tensor-core kernels:
//   epair[x + 128] = {bf16 E[x], bf16 E[x-1]}  for x in [-128, Tp + 128)
//   ef[x + 128]    = E[x] (fp32), same range;  E outside [0, T) is 0
//   cpair[m]       = {bf16 c[2m], bf16 c[2m+1]}, cf[j] = c[j]; 0 for j >= T
//   rsc[i]         = r_i (fp32; 0 where log Z(i) = -inf)
//   flag[h]        = 1 when the factors leave fp32 range for terms that matter
//                    (then the head runs the per-element exp path instead).
__global__ void __launch_bounds__(1024) prep_replaced_kernel(const float* __restrict__ a,
                                                             const float* __restrict__ r,
                                                             const float* __restrict__ logz, HeadList hl,
                                                             int T, int Tp, int Lp, uint32_t* __restrict__ epair,
                                                             float* __restrict__ ef, uint32_t* __restrict__ cpair,
                                                             float* __restrict__ cf, float* __restrict__ rsc,
                                                             int* __restrict__ flag) {
    __shared__ float red[33];
    const int slot = blockIdx.x;
    const int h = hl.heads[slot];
    const float* ah = a + (size_t)h * T;
    const float* rh = r + (size_t)h * T;
    const float* lz = logz + (size_t)h * T;
    float amax = kNegInf, amin = -kNegInf, rmax = kNegInf, lzmin = -kNegInf;
    for (int k = threadIdx.x; k < T; k += blockDim.x) {
        const float av = ah[k], rv = rh[k], lv = lz[k];
        amax = fmaxf(amax, av);
        if (av != kNegInf) amin = fminf(amin, av);
        rmax = fmaxf(rmax, rv);
        if (lv != kNegInf) lzmin = fminf(lzmin, lv);
    }
    amax = block_reduce(amax, true, red);
    amin = block_reduce(amin, false, red);
    rmax = block_reduce(rmax, true, red);
    lzmin = block_reduce(lzmin, false, red);
    const float A = (amax == kNegInf) ? 0.f : amax;
    const float R = (rmax == kNegInf) ? 0.f : rmax;
    uint32_t* ep = epair + (size_t)slot * Lp;
    float* efs = ef + (size_t)slot * Lp;
    for (int x = (int)threadIdx.x - 128; x < Tp + 128; x += blockDim.x) {
        const float e0 = (x >= 0 && x < T) ? expf(rh[x] - R) : 0.f;
        const float e1 = (x - 1 >= 0 && x - 1 < T) ? expf(rh[x - 1] - R) : 0.f;
        __nv_bfloat162 pr = __floats2bfloat162_rn(e0, e1);
        ep[x + 128] = *reinterpret_cast<uint32_t*>(&pr);
        efs[x + 128] = e0;
    }
    uint32_t* cp = cpair + (size_t)slot * (Tp / 2);
    float* cfs = cf + (size_t)slot * Tp;
    for (int m = threadIdx.x; m < Tp / 2; m += blockDim.x) {
        const int j = 2 * m;
        const float c0 = j < T ? expf(ah[j] - A) : 0.f;
        const float c1 = j + 1 < T ? expf(ah[j + 1] - A) : 0.f;
        __nv_bfloat162 pr = __floats2bfloat162_rn(c0, c1);
        cp[m] = *reinterpret_cast<uint32_t*>(&pr);
        cfs[j] = c0;
        cfs[j + 1] = c1;
    }
    float* rs = rsc + (size_t)slot * Tp;
    for (int i = threadIdx.x; i < Tp; i += blockDim.x) {
        const float lv = i < T ? lz[i] : kNegInf;
        rs[i] = (lv == kNegInf) ? 0.f : expf(A + R - lv);
    }
    if (threadIdx.x == 0) {
        // forward: r_i = exp(A + R - log Z(i)) and backward: 1 / c_j = exp(A - a_j)
        // must stay well inside fp32 for every term of size > ~1e-15
        const bool ok = (lzmin == -kNegInf || A + R - lzmin <= 80.f) && (amin == -kNegInf || A - amin <= 80.f);
        flag[h] = ok ? 0 : 1;
    }
}

}  // namespace

cudaError_t launch_prep_replaced(const float* a, const float* r, const float* logz, const HeadList& hl, int T,
                                 const ReplacedWs& w, cudaStream_t stream) {
    if (hl.n == 0 || T == 0) return cudaSuccess;
    launch_begin(KID_PREP_REPLACED, stream);
    prep_replaced_kernel<<<hl.n, 1024, 0, stream>>>(a, r, logz, hl, T, w.Tp, w.Lp, w.epair, w.ef, w.cpair, w.cf,
                                                    w.rsc, w.flag);
    launch_end(KID_PREP_REPLACED, stream);
    return cudaGetLastError();
}

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
