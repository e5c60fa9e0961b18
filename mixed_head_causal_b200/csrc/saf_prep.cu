// Small preparation kernels of the mixed-head layer.
//
//  * lognorm: the per-row log-normaliser of a replaced head's compact
//    pattern, log Z(i) = log sum_{k<=i} exp(a[k] + r[i-k])  (Eq. (3) of
//    "When Can Attention Heads Be Statically Defined?", section 二.3).  It
//    depends on a and r only, so it is computed once per head, not per batch.
//  * dot: the backward row term D[i] = sum_c dO[i,c] O[i,c] of softmax
//    attention (equal to sum_j P[i,j] dP[i,j]), one fp32 value per row.
#include <algorithm>

#include "saf_common.cuh"
#include "tc_util.cuh"

namespace saf {
namespace {


// Tiling of the log-normaliser: a block owns 32 consecutive rows i (one per
// lane) of one replaced head.  It stages a[0, kend) and r[0, kend) (kend = the
// tile's last row + 1; chunks of kLnChunk for long heads) in shared memory in
// log2 units, all loads in flight at once, and its 8 warps split the k range
// 8 ways.  In a warp every lane reads the same a[k] (a broadcast) and
// consecutive r[i-k] (no bank conflicts).  Each lane keeps a log2-domain
// (max, sum) pair updated once per 8 terms; the 8 per-warp partials of a row
// are merged at the end.  Blocks start with the last rows (the longest sums).
constexpr int kLnRows = 32;
constexpr int kLnWarps = 8;
constexpr int kLnChunk = 4096;
constexpr float kLnFloor = -3.402823466e38f;  // finite "no term yet" maximum

__global__ void __launch_bounds__(kLnWarps * 32) lognorm_kernel(const float* __restrict__ a,
                                                               const float* __restrict__ r,
                                                               HeadList hl, int T, int chunk,
                                                               float* __restrict__ logz) {
    // dynamic shared memory of 2 * chunk + kLnRows floats, chunk = min(T, kLnChunk)
    extern __shared__ float ln_smem[];
    float* sa = ln_smem;          // [chunk]: a[k0 + u]
    float* sr = ln_smem + chunk;  // [chunk + kLnRows]: r[dbase + q]
    __shared__ float pm[kLnWarps][32], ps[kLnWarps][32];
    const int h = hl.heads[blockIdx.y];
    const int i0 = (gridDim.x - 1 - blockIdx.x) * kLnRows;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float* ah = a + (size_t)h * T;
    const float* rh = r + (size_t)h * T;
    const int kend = min(i0 + kLnRows, T);  // every k a row of this tile can reach
    float m = kLnFloor, s = 0.f;
    for (int k0 = 0; k0 < kend; k0 += chunk) {
        const int n = min(chunk, kend - k0);  // k of this chunk: [k0, k0 + n)
        // sa[u] = a[k0 + u] (u < n) and sr[q] = r[d], d = dbase + q, for the
        // d = i - k this chunk can meet; out-of-range entries are -inf (no term)
        const int dbase = i0 - k0 - (n - 1);
        const int span = n + kLnRows - 1;
        // every load of the chunk in flight before the first store (one
        // round trip to L2 instead of one per pass of the loop)
        constexpr int kPer = (kLnChunk + kLnRows) / (kLnWarps * 32) + 1;
        float va[kPer], vr[kPer];
#pragma unroll
        for (int e = 0; e < kPer; ++e) {
            const int u = (int)threadIdx.x + e * kLnWarps * 32;
            const int d = dbase + u;
            va[e] = u < n ? ah[k0 + u] : 0.f;
            vr[e] = (u < span && d >= 0 && d < T) ? rh[d] : kNegInf;
        }
#pragma unroll
        for (int e = 0; e < kPer; ++e) {
            const int u = (int)threadIdx.x + e * kLnWarps * 32;
            if (u < n) sa[u] = va[e] * kLog2e;
            if (u < span) sr[u] = vr[e] * kLog2e;
        }
        __syncthreads();
        // warp w takes k in [w * per, (w + 1) * per) of the chunk, 8 at a time;
        // row i = i0 + lane, k = k0 + u: d - dbase = lane + (n - 1) - u
        const int per = ((n + 8 * kLnWarps - 1) / (8 * kLnWarps)) * 8;
        const int ub = warp * per, ue = min(n, ub + per);
        for (int u0 = ub; u0 < ue; u0 += 8) {
            float x[8];
            float mx = kNegInf;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int u = u0 + e;
                x[e] = u < ue ? sa[u] + sr[lane + (n - 1) - u] : kNegInf;
                mx = fmaxf(mx, x[e]);
            }
            if (mx > m) {
                s *= tc::ex2(m - mx);
                m = mx;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) s += tc::ex2(x[e] - m);
        }
        __syncthreads();
    }
    pm[warp][lane] = m;
    ps[warp][lane] = s;
    __syncthreads();
    if (warp == 0) {
        float M = kLnFloor;
#pragma unroll
        for (int w = 0; w < kLnWarps; ++w) M = fmaxf(M, pm[w][lane]);
        float S = 0.f;
#pragma unroll
        for (int w = 0; w < kLnWarps; ++w) S += ps[w][lane] * exp2f(pm[w][lane] - M);
        const int i = i0 + lane;
        if (i < T) logz[(size_t)h * T + i] = (S > 0.f) ? (M + log2f(S)) * kLn2 : kNegInf;
    }
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

// Block-wide reduction of four values at once: max, min, max, min.
__device__ float4 block_reduce_mmmm(float4 v, float4* red) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        v.x = fmaxf(v.x, __shfl_xor_sync(0xffffffffu, v.x, off));
        v.y = fminf(v.y, __shfl_xor_sync(0xffffffffu, v.y, off));
        v.z = fmaxf(v.z, __shfl_xor_sync(0xffffffffu, v.z, off));
        v.w = fminf(v.w, __shfl_xor_sync(0xffffffffu, v.w, off));
    }
    if (lane == 0) red[wid] = v;
    __syncthreads();
    v = red[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) {
        const float4 o = red[w];
        v.x = fmaxf(v.x, o.x);
        v.y = fminf(v.y, o.y);
        v.z = fmaxf(v.z, o.z);
        v.w = fminf(v.w, o.w);
    }
    return v;
}

// Factored form of a replaced head's pattern,
//   P(i,j) = r_i * E[i-j] * c_j,  E[d] = exp(r[d] - R),  c_j = exp(a[j] - A),
//   r_i = exp(A + R - log Z(i)),  A = max a, R = max r,
// which is Eq. (3) rearranged (exp of a sum is the product of exps).  A row of
// blocks per replaced head (grid.y = head slot) writes, for the tensor-core
// kernels:
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
    __shared__ float4 red[32];
    const int slot = blockIdx.y;
    const int h = hl.heads[slot];
    const float* ah = a + (size_t)h * T;
    const float* rh = r + (size_t)h * T;
    const float* lz = logz + (size_t)h * T;
    // every block of the head reduces the whole head (a few KB from L2), then
    // writes its own share of the outputs
    float4 v = make_float4(kNegInf, -kNegInf, kNegInf, -kNegInf);  // max a, min a, max r, min log Z
    for (int k = threadIdx.x; k < T; k += blockDim.x) {
        const float av = ah[k], rv = rh[k], lv = lz[k];
        v.x = fmaxf(v.x, av);
        if (av != kNegInf) v.y = fminf(v.y, av);
        v.z = fmaxf(v.z, rv);
        if (lv != kNegInf) v.w = fminf(v.w, lv);
    }
    v = block_reduce_mmmm(v, red);
    const float amin = v.y, lzmin = v.w;
    const float A = (v.x == kNegInf) ? 0.f : v.x;
    const float R = (v.z == kNegInf) ? 0.f : v.z;
    const int g0 = blockIdx.x * blockDim.x + threadIdx.x, gs = gridDim.x * blockDim.x;
    uint32_t* ep = epair + (size_t)slot * Lp;
    float* efs = ef + (size_t)slot * Lp;
    for (int x = g0 - 128; x < Tp + 128; x += gs) {
        const float e0 = (x >= 0 && x < T) ? expf(rh[x] - R) : 0.f;
        const float e1 = (x - 1 >= 0 && x - 1 < T) ? expf(rh[x - 1] - R) : 0.f;
        __nv_bfloat162 pr = __floats2bfloat162_rn(e0, e1);
        ep[x + 128] = *reinterpret_cast<uint32_t*>(&pr);
        efs[x + 128] = e0;
    }
    uint32_t* cp = cpair + (size_t)slot * (Tp / 2);
    float* cfs = cf + (size_t)slot * Tp;
    for (int m = g0; m < Tp / 2; m += gs) {
        const int j = 2 * m;
        const float c0 = j < T ? expf(ah[j] - A) : 0.f;
        const float c1 = j + 1 < T ? expf(ah[j + 1] - A) : 0.f;
        __nv_bfloat162 pr = __floats2bfloat162_rn(c0, c1);
        cp[m] = *reinterpret_cast<uint32_t*>(&pr);
        cfs[j] = c0;
        cfs[j + 1] = c1;
    }
    float* rs = rsc + (size_t)slot * Tp;
    for (int i = g0; i < Tp; i += gs) {
        const float lv = i < T ? lz[i] : kNegInf;
        rs[i] = (lv == kNegInf) ? 0.f : expf(A + R - lv);
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
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
    // enough 1024-thread blocks per head for about one output entry per thread
    const int nb = std::max(1, std::min(32, (w.Lp + 1023) / 1024));
    prep_replaced_kernel<<<dim3(nb, hl.n), 1024, 0, stream>>>(a, r, logz, hl, T, w.Tp, w.Lp, w.epair, w.ef, w.cpair, w.cf,
                                                    w.rsc, w.flag);
    launch_end(KID_PREP_REPLACED, stream);
    return cudaGetLastError();
}

cudaError_t launch_lognorm(const float* a, const float* r, const HeadList& hl, int T,
                           float* logz, cudaStream_t stream) {
    if (hl.n == 0 || T == 0) return cudaSuccess;
    dim3 grid((T + kLnRows - 1) / kLnRows, hl.n);
    const int chunk = std::min(T, kLnChunk);
    const int smem = (int)sizeof(float) * (2 * chunk + kLnRows);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(lognorm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
    }
    launch_begin(KID_LOGNORM, stream);
    lognorm_kernel<<<grid, kLnWarps * 32, smem, stream>>>(a, r, hl, T, chunk, logz);
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
