// Small preparation kernels of the mixed-head layer.
//
//  * pattern preparation of the replaced heads: the per-row log-normaliser
//    of the compact pattern, log Z(i) = log sum_{k<=i} exp(a[k] + r[i-k])
//    (Eq. (3) of "When Can Attention Heads Be Statically Defined?", section
//    二.3), and the factored arrays the tensor-core kernels read.  It depends
//    on a and r only, so it is computed once per head, not per batch.
//  * dot: the backward row term D[i] = sum_c dO[i,c] O[i,c] of softmax
//    attention (equal to sum_j P[i,j] dP[i,j]), one fp32 value per row.
#include <string.h>

#include <algorithm>

#include "saf_common.cuh"
#include "tc_util.cuh"

namespace saf {
namespace {

// ---------------------------------------------------------------- pattern
// The factored form of a replaced head's pattern,
//   P(i,j) = r_i * E[i-j] * c_j,  E[d] = exp(r[d] - R),  c_j = exp(a[j] - A),
//   r_i = exp(A + R - log Z(i)),  A = max a, R = max r,
// is Eq. (3) rearranged (the exponential of a sum is the product of the
// exponentials).  With it the normaliser is a causal convolution of two
// vectors of numbers in (0, 1]:
//   Z(i) = exp(A + R) * S(i),  S(i) = sum_{k<=i} c_k E[i-k],
// T^2/2 multiply-adds per head instead of as many exponentials.  S(i) >= e^-50
// keeps every term lost to fp32 underflow (below about e^-87) under e^-37 of
// the row's sum; a 32-row tile with a smaller S(i) takes the plain
// log-sum-exp of Eq. (3) instead, with a running maximum (exact_tile).
//
// A block of 256 threads owns 32 consecutive rows (one per lane) of one head
// and stages the keys and distances those rows reach in shared memory, 4096
// at a time; its 8 warps split the keys.  It also writes its 32 positions of
// the arrays the tensor-core kernels read (the first and last tiles add the
// padding):
//   epair[x + 128] = {bf16 E[x], bf16 E[x-1]}  for x in [-128, Tp + 128)
//   ef[x + 128]    = E[x] (fp32), same range;  E outside [0, T) is 0
//   cpair[m]       = {bf16 c[2m], bf16 c[2m+1]}, cf[j] = c[j]; 0 for j >= T
//   rsc[i]         = r_i (fp32; 0 where log Z(i) = -inf)
//   tflag[tile]    = 1 when a term that matters could be lost in the
//                    factored form (below); the kernels OR a head's tiles.
constexpr int kPpRows = 32;
constexpr int kPpWarps = 8;
constexpr int kPpThreads = kPpRows * kPpWarps;
constexpr int kPpChunk = 4096;
constexpr float kLnFloor = -3.402823466e38f;   // finite "no term yet" maximum
constexpr float kSafeSum = 1.92874985e-22f;    // e^-50

struct PatternJob {
    const float* a;
    const float* r;
    const float* logz_in;  // [H, T] given log Z, or null: computed here
    float* logz_out;       // [H, T] written when non-null
    ReplacedWs w;          // the factored arrays, when w.epair is non-null
    HeadList hl;
    int T, ntiles, chunk;  // ntiles = ceil(T / 32), chunk = min(T, kPpChunk)
};

struct PatternShared {
    float4 red[kPpWarps];
    float pm[kPpWarps][32], ps[kPpWarps][32];
};

inline int pattern_smem_bytes(int chunk) { return (int)sizeof(float) * (2 * chunk + kPpRows); }

// log Z of the tile's rows straight from Eq. (3): log2-domain (max, sum) pairs
// per lane, updated once per 8 terms, merged over the 8 warps; valid in every
// thread for its lane's row on return.
__device__ float exact_tile(const float* __restrict__ ah, const float* __restrict__ rh, int T, int i0, int chunk,
                            float* dyn, PatternShared& sh) {
    float* sa = dyn;          // [chunk]: a[k0 + u] log2 e
    float* sr = dyn + chunk;  // [chunk + 32]: r[dbase + q] log2 e
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int kend = min(i0 + kPpRows, T);
    float m = kLnFloor, s = 0.f;
    for (int k0 = 0; k0 < kend; k0 += chunk) {
        const int n = min(chunk, kend - k0);
        const int dbase = i0 - k0 - (n - 1);
        const int span = n + kPpRows - 1;
        for (int u = threadIdx.x; u < span; u += kPpThreads) {
            const int d = dbase + u;
            if (u < n) sa[u] = ah[k0 + u] * kLog2e;
            sr[u] = (d >= 0 && d < T) ? rh[d] * kLog2e : kNegInf;
        }
        __syncthreads();
        const int per = ((n + 8 * kPpWarps - 1) / (8 * kPpWarps)) * 8;
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
    sh.pm[warp][lane] = m;
    sh.ps[warp][lane] = s;
    __syncthreads();
    float M = kLnFloor;
#pragma unroll
    for (int w = 0; w < kPpWarps; ++w) M = fmaxf(M, sh.pm[w][lane]);
    float S = 0.f;
#pragma unroll
    for (int w = 0; w < kPpWarps; ++w) S += sh.ps[w][lane] * exp2f(sh.pm[w][lane] - M);
    __syncthreads();
    return (S > 0.f) ? (M + log2f(S)) * kLn2 : kNegInf;
}

// Tile t (rows 32t .. 32t + 31) of replaced slot `slot`, by the block's 256
// threads (every thread of the block calls it).
__device__ void pattern_tile(const PatternJob& J, int slot, int t, float* dyn, PatternShared& sh) {
    const int T = J.T, h = J.hl.heads[slot];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float* ah = J.a + (size_t)h * T;
    const float* rh = J.r + (size_t)h * T;
    // the head's max a, min a (over finite values), max r; eight loads of
    // each vector in flight per thread
    float4 v = make_float4(kNegInf, -kNegInf, kNegInf, 0.f);
    for (int k0 = 0; k0 < T; k0 += 8 * kPpThreads) {
        float av[8], rv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int k = k0 + e * kPpThreads + tid;
            av[e] = k < T ? ah[k] : kNegInf;
            rv[e] = k < T ? rh[k] : kNegInf;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            v.x = fmaxf(v.x, av[e]);
            if (av[e] != kNegInf) v.y = fminf(v.y, av[e]);
            v.z = fmaxf(v.z, rv[e]);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        v.x = fmaxf(v.x, __shfl_xor_sync(0xffffffffu, v.x, off));
        v.y = fminf(v.y, __shfl_xor_sync(0xffffffffu, v.y, off));
        v.z = fmaxf(v.z, __shfl_xor_sync(0xffffffffu, v.z, off));
    }
    if (lane == 0) sh.red[warp] = v;
    __syncthreads();
    v = sh.red[0];
#pragma unroll
    for (int w = 1; w < kPpWarps; ++w) {
        v.x = fmaxf(v.x, sh.red[w].x);
        v.y = fminf(v.y, sh.red[w].y);
        v.z = fmaxf(v.z, sh.red[w].z);
    }
    const float amin = v.y;
    const float A = (v.x == kNegInf) ? 0.f : v.x;
    const float R = (v.z == kNegInf) ? 0.f : v.z;
    const int i0 = t * kPpRows, i = i0 + lane;

    float lz = kNegInf;
    if (J.logz_in) {
        if (i < T) lz = J.logz_in[(size_t)h * T + i];
    } else {
        // S(i) = sum_{k<=i} c_k E[i-k]: per chunk, sc[u] = c_{k0+u} and sE[q] =
        // E[dbase + q] (0 outside [0, T)); every load of a chunk in flight
        // before the exps and stores
        float* sc = dyn;
        float* sE = dyn + J.chunk;
        const int kend = min(i0 + kPpRows, T);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k0 = 0; k0 < kend; k0 += J.chunk) {
            const int n = min(J.chunk, kend - k0);
            const int dbase = i0 - k0 - (n - 1);
            const int span = n + kPpRows - 1;
            constexpr int kPer = (kPpChunk + kPpRows) / kPpThreads + 1;
            float va[kPer], vr[kPer];
#pragma unroll
            for (int e = 0; e < kPer; ++e) {
                const int u = tid + e * kPpThreads;
                const int d = dbase + u;
                va[e] = u < n ? ah[k0 + u] : kNegInf;
                vr[e] = (u < span && d >= 0 && d < T) ? rh[d] : kNegInf;
            }
#pragma unroll
            for (int e = 0; e < kPer; ++e) {
                const int u = tid + e * kPpThreads;
                if (u < n) sc[u] = tc::ex2((va[e] - A) * kLog2e);
                if (u < span) sE[u] = tc::ex2((vr[e] - R) * kLog2e);
            }
            __syncthreads();
            // warp w takes k in [w * per, (w + 1) * per) of the chunk (per a
            // multiple of 8; keys past the chunk read sc = 0 beyond n, below);
            // row i = i0 + lane, k = k0 + u: d - dbase = lane + (n - 1) - u
            const int per = ((n + 8 * kPpWarps - 1) / (8 * kPpWarps)) * 8;
            const int ub = warp * per, ue = min(n, ub + per);
            for (int u0 = ub; u0 < ue; u0 += 8) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int u = u0 + e;
                    if (u < ue) acc[e & 3] = fmaf(sc[u], sE[lane + (n - 1) - u], acc[e & 3]);
                }
            }
            __syncthreads();
        }
        sh.ps[warp][lane] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        __syncthreads();
        float S = 0.f;
#pragma unroll
        for (int w = 0; w < kPpWarps; ++w) S += sh.ps[w][lane];
        const bool small = i < T && !(S >= kSafeSum);
        if (__syncthreads_or(small)) lz = exact_tile(ah, rh, T, i0, J.chunk, dyn, sh);
        else if (i < T) lz = A + R + logf(S);
    }
    if (J.logz_out && warp == 0 && i < T) J.logz_out[(size_t)h * T + i] = lz;
    if (!J.w.epair) return;

    const ReplacedWs& w = J.w;
    const int Tp = w.Tp, Lp = w.Lp;
    const bool last = t == J.ntiles - 1;
    if (warp == 0) {
        // r_i, and the tile's flag: a lost term can reach r_i e^-87 =
        // exp(A + R - log Z(i) - 87) of P, so rows with A + R - log Z(i) > 50
        // need the per-element path; so does a c_j below e^-80 (A - a_j > 80,
        // which the backward divides out)
        if (i < Tp) w.rsc[(size_t)slot * Tp + i] = (i < T && lz != kNegInf) ? tc::ex2((A + R - lz) * kLog2e) : 0.f;
        const bool far = i < T && lz != kNegInf && A + R - lz > 50.f;
        const bool any = __any_sync(0xffffffffu, far);
        if (lane == 0)
            w.tflag[(size_t)slot * w.ntiles + t] = (any || (amin != -kNegInf && A - amin > 80.f)) ? 1 : 0;
        if (last)  // r_i past the last tile
            for (int ii = J.ntiles * kPpRows + lane; ii < Tp; ii += 32) w.rsc[(size_t)slot * Tp + ii] = 0.f;
    } else {
        const int wt = tid - 32, wn = kPpThreads - 32;
        const int x_lo = t == 0 ? -128 : i0;
        const int x_hi = last ? Tp + 128 : i0 + kPpRows;
        uint32_t* ep = w.epair + (size_t)slot * Lp;
        float* efs = w.ef + (size_t)slot * Lp;
        for (int x = x_lo + wt; x < x_hi; x += wn) {
            const float e0 = (x >= 0 && x < T) ? tc::ex2((rh[x] - R) * kLog2e) : 0.f;
            const float e1 = (x - 1 >= 0 && x - 1 < T) ? tc::ex2((rh[x - 1] - R) * kLog2e) : 0.f;
            __nv_bfloat162 pr = __floats2bfloat162_rn(e0, e1);
            ep[x + 128] = *reinterpret_cast<uint32_t*>(&pr);
            efs[x + 128] = e0;
        }
        // c pairs m of this tile (the last tile runs on to Tp)
        const int m_lo = i0 / 2, m_hi = last ? Tp / 2 : (i0 + kPpRows) / 2;
        uint32_t* cp = w.cpair + (size_t)slot * (Tp / 2);
        float* cfs = w.cf + (size_t)slot * Tp;
        for (int mm = m_lo + wt; mm < m_hi; mm += wn) {
            const int j = 2 * mm;
            const float c0 = j < T ? tc::ex2((ah[j] - A) * kLog2e) : 0.f;
            const float c1 = j + 1 < T ? tc::ex2((ah[j + 1] - A) * kLog2e) : 0.f;
            __nv_bfloat162 pr = __floats2bfloat162_rn(c0, c1);
            cp[mm] = *reinterpret_cast<uint32_t*>(&pr);
            cfs[j] = c0;
            cfs[j + 1] = c1;
        }
    }
}

// The pattern preparation alone: grid (ntiles, replaced heads), tiles with
// the most keys first.
__global__ void __launch_bounds__(kPpThreads) pattern_kernel(const PatternJob J) {
    extern __shared__ float pp_smem[];
    __shared__ PatternShared sh;
    // the forward kernel that follows waits for this grid only where it reads
    // what this grid writes: it may start now
    tc::griddep_launch_dependents();
    pattern_tile(J, blockIdx.y, J.ntiles - 1 - blockIdx.x, pp_smem, sh);
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

// Backward preprocessing, one launch: rows of [BH, Tp] get -lse2 = -lse*log2(e)
// (-inf past T) and D = rowsum(dO o O) (0 past T), the dQ accumulator rows
// are zeroed (8 threads per row); the first
// `pattern_blocks` blocks instead prepare the replaced heads' patterns
// (pattern_tile; tiles with the most keys first).
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ dout,
                                                      const float* __restrict__ lse, int T, int Tp, int64_t rows,
                                                      float* __restrict__ nlse2p, float* __restrict__ dvecp,
                                                      float* __restrict__ dqacc, const PatternJob J,
                                                      int pattern_blocks) {
    if ((int)blockIdx.x < pattern_blocks) {
        extern __shared__ float pp_smem[];
        __shared__ PatternShared sh;
        const int slot = blockIdx.x / J.ntiles;
        pattern_tile(J, slot, J.ntiles - 1 - (blockIdx.x - slot * J.ntiles), pp_smem, sh);
        return;
    }
    const int64_t rr = (int64_t)(blockIdx.x - pattern_blocks) * 32 + (threadIdx.x >> 3);
    const int part = threadIdx.x & 7;
    if (rr >= rows) return;
    const int64_t bh = rr / Tp;
    const int i = (int)(rr - bh * Tp);
    float acc = 0.f;
    if (i < T) {
        const int64_t row = bh * T + i;
        const uint4 ov = *reinterpret_cast<const uint4*>(o + row * kHeadDim + part * 8);
        const uint4 dv = *reinterpret_cast<const uint4*>(dout + row * kHeadDim + part * 8);
        const __nv_bfloat162* op = reinterpret_cast<const __nv_bfloat162*>(&ov);
        const __nv_bfloat162* dp = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 x = __bfloat1622float2(op[e]), y = __bfloat1622float2(dp[e]);
            acc = fmaf(x.x, y.x, acc);
            acc = fmaf(x.y, y.y, acc);
        }
        float4* z = reinterpret_cast<float4*>(dqacc + row * kHeadDim + part * 8);
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    if (part == 0) {
        dvecp[rr] = i < T ? acc : 0.f;
        nlse2p[rr] = i < T ? -lse[bh * T + i] * kLog2e : kNegInf;
    }
}

PatternJob make_job(const float* a, const float* r, const float* logz_in, float* logz_out, const HeadList& hl,
                    int T, const ReplacedWs* w) {
    PatternJob J;
    J.a = a;
    J.r = r;
    J.logz_in = logz_in;
    J.logz_out = logz_out;
    if (w) {
        J.w = *w;
    } else {
        memset(&J.w, 0, sizeof(J.w));
    }
    J.hl = hl;
    J.T = T;
    J.ntiles = (T + kPpRows - 1) / kPpRows;
    J.chunk = std::min(T, kPpChunk);
    return J;
}

}  // namespace

cudaError_t launch_pattern(const float* a, const float* r, const float* logz_in, float* logz_out, const HeadList& hl,
                           int T, const ReplacedWs* w, cudaStream_t stream) {
    if (hl.n == 0 || T == 0) return cudaSuccess;
    const PatternJob J = make_job(a, r, logz_in, logz_out, hl, T, w);
    launch_begin(KID_PATTERN, stream);
    pattern_kernel<<<dim3(J.ntiles, hl.n), kPpThreads, pattern_smem_bytes(J.chunk), stream>>>(J);
    launch_end(KID_PATTERN, stream);
    return cudaGetLastError();
}

cudaError_t launch_lognorm(const float* a, const float* r, const HeadList& hl, int T, float* logz,
                           cudaStream_t stream) {
    return launch_pattern(a, r, nullptr, logz, hl, T, nullptr, stream);
}

cudaError_t launch_bwd_pre(const __nv_bfloat16* o, const __nv_bfloat16* dout, const float* lse, int BH, int T,
                           float* nlse2p, float* dvecp, float* dqacc, const float* a, const float* r,
                           const float* logz_in, float* logz_out, const HeadList& hl, const ReplacedWs& w,
                           cudaStream_t stream) {
    const int Tp = round_up128(T);
    const int64_t rows = (int64_t)BH * Tp;
    if (rows == 0) return cudaSuccess;
    const PatternJob J = make_job(a, r, logz_in, logz_out, hl, T, &w);
    const int pattern_blocks = hl.n > 0 ? J.ntiles * hl.n : 0;
    const int smem = hl.n > 0 ? pattern_smem_bytes(J.chunk) : 0;
    launch_begin(KID_BWD_PRE, stream);
    bwd_pre_kernel<<<(unsigned)(pattern_blocks + (rows + 31) / 32), 256, smem, stream>>>(
        o, dout, lse, T, Tp, rows, nlse2p, dvecp, dqacc, J, pattern_blocks);
    launch_end(KID_BWD_PRE, stream);
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
