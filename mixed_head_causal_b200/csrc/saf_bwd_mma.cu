// Mixed-head causal attention backward, warp-level mma.sync path.
//
// Two kernels, each recomputing the attention probabilities from the saved
// row log-sum-exp (no T x T matrix is ever stored):
//
//  * dkdv_kernel: one CTA per 64-key block, walking the query blocks at and
//    below the diagonal.  Ordinary heads:  P^T = exp(K Q^T s - lse),
//    dV += P^T dO,  dP^T = V dO^T,  dS^T = P^T o (dP^T - D),  dK += dS^T Q s.
//    Replaced heads: P^T is the fixed pattern of Eq. (3) ("When Can Attention
//    Heads Be Statically Defined?", section 二.3) and only dV = P^T dO is
//    formed (section 二.4); dK is written as zeros.
//  * dq_kernel: one CTA per 64-query block, walking key blocks up to the
//    diagonal: dQ += dS K s.  Replaced heads write zeros.
//
// D[i] = sum_c dO[i,c] O[i,c] comes from the dot kernel (saf_prep.cu).
#include "mma_util.cuh"
#include "saf_common.cuh"

namespace saf {
namespace {

using namespace mma;

constexpr int BK = 64;   // keys per CTA (dkdv) / per block (dq)
constexpr int BQ = 64;   // queries per block (dkdv) / per CTA (dq)
constexpr int NT = 128;  // 4 warps x 16 rows

struct BwdParams {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const __nv_bfloat16* dout;
    const float* lse;
    const float* dvec;
    const float* a;
    const float* r;
    const float* logz;
    void* dq;
    void* dk;
    void* dv;
    HeadList hl;
    int H, T, grad_fp32;
    float scale;       // 1/sqrt(d_h)
    float scale_log2;  // log2(e)/sqrt(d_h)
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

// Writes a 16 x 64 fp32 accumulator block (C-fragment layout) scaled by `mul`.
__device__ __forceinline__ void store_rows(void* base, int grad_fp32, int row_lo, int row_hi, int T,
                                           const float (&acc)[8][4], float mul, int t) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        const int c = nt * 8 + 2 * t;
        if (grad_fp32) {
            float* g = reinterpret_cast<float*>(base);
            if (row_lo < T) *reinterpret_cast<float2*>(g + (size_t)row_lo * kHeadDim + c) = make_float2(acc[nt][0] * mul, acc[nt][1] * mul);
            if (row_hi < T) *reinterpret_cast<float2*>(g + (size_t)row_hi * kHeadDim + c) = make_float2(acc[nt][2] * mul, acc[nt][3] * mul);
        } else {
            __nv_bfloat16* g = reinterpret_cast<__nv_bfloat16*>(base);
            if (row_lo < T) *reinterpret_cast<__nv_bfloat162*>(g + (size_t)row_lo * kHeadDim + c) = __floats2bfloat162_rn(acc[nt][0] * mul, acc[nt][1] * mul);
            if (row_hi < T) *reinterpret_cast<__nv_bfloat162*>(g + (size_t)row_hi * kHeadDim + c) = __floats2bfloat162_rn(acc[nt][2] * mul, acc[nt][3] * mul);
        }
    }
}

__device__ __forceinline__ void zero_acc(float (&acc)[8][4]) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
}

__global__ void __launch_bounds__(NT) dkdv_kernel(const BwdParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sK = smem_u32(smem);     // 64 x 64
    const uint32_t sV = sK + BK * 128;      // 64 x 64
    const uint32_t sQ = sV + BK * 128;      // 2 x 64 x 64
    const uint32_t sO = sQ + 2 * BQ * 128;  // dO: 2 x 64 x 64
    float* sL = reinterpret_cast<float*>(smem + 2 * BK * 128 + 4 * BQ * 128);  // 2 x 64 lse*log2e
    float* sD = sL + 2 * BQ;                                                   // 2 x 64 D

    const int T = p.T;
    const int kb = blockIdx.y;  // key block 0 has the most query blocks: run first
    const int bh = blockIdx.x;
    const int h = bh % p.H;
    const bool rep = p.hl.replaced[h] != 0;
    const size_t base = (size_t)bh * T * kHeadDim;
    const __nv_bfloat16* Qg = p.q + base;
    const __nv_bfloat16* Kg = p.k + base;
    const __nv_bfloat16* Vg = p.v + base;
    const __nv_bfloat16* Og = p.dout + base;
    const float* Lg = p.lse + (size_t)bh * T;
    const float* Dg = p.dvec + (size_t)bh * T;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int k0 = kb * BK;
    const int key_lo = k0 + warp * 16 + g, key_hi = key_lo + 8;
    const int qb_first = k0 / BQ;
    const int nqb = (T + BQ - 1) / BQ;

    if (!rep) load_tile_async(sK, Kg, k0, T, BK, tid, NT);
    if (!rep) load_tile_async(sV, Vg, k0, T, BK, tid, NT);
    auto load_q_block = [&](int qb, int buf) {
        const int q0 = qb * BQ;
        if (!rep) load_tile_async(sQ + buf * BQ * 128, Qg, q0, T, BQ, tid, NT);
        load_tile_async(sO + buf * BQ * 128, Og, q0, T, BQ, tid, NT);
        if (tid < BQ) {
            const int i = q0 + tid;
            float lv = 0.f, dv = 0.f;
            if (i < T) {
                lv = rep ? p.logz[(size_t)h * T + i] * kLog2e : Lg[i] * kLog2e;
                dv = rep ? 0.f : Dg[i];
            }
            sL[buf * BQ + tid] = lv;
            sD[buf * BQ + tid] = dv;
        }
    };
    load_q_block(qb_first, 0);
    cp_async_commit();

    const float* ah = p.a + (size_t)h * T;
    const float* rh = p.r + (size_t)h * T;
    float a2_lo[1], a2_hi[1];
    a2_lo[0] = (rep && key_lo < T) ? __ldg(ah + key_lo) * kLog2e : 0.f;
    a2_hi[0] = (rep && key_hi < T) ? __ldg(ah + key_hi) * kLog2e : 0.f;

    uint32_t kf[4][4], vf[4][4];
    float dvacc[8][4], dkacc[8][4];
    zero_acc(dvacc);
    zero_acc(dkacc);

    for (int qb = qb_first; qb < nqb; ++qb) {
        const int buf = (qb - qb_first) & 1;
        if (qb + 1 < nqb) {
            load_q_block(qb + 1, buf ^ 1);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        if (qb == qb_first && !rep) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                load_a_frag(kf[ks], sK, warp * 16, ks * 16, lane);
                load_a_frag(vf[ks], sV, warp * 16, ks * 16, lane);
            }
        }
        const int q0 = qb * BQ;
        const uint32_t sQb = sQ + buf * BQ * 128;
        const uint32_t sOb = sO + buf * BQ * 128;
        const float* sLb = sL + buf * BQ;
        const float* sDb = sD + buf * BQ;
        if (q0 + BQ - 1 >= k0 + warp * 16) {  // some query of the block sees this warp's keys
            float s[8][4];  // P^T: rows = keys (lo/hi), cols = queries
            if (!rep) {
                zero_acc(s);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
                    for (int np = 0; np < 4; ++np) {
                        uint32_t b[4];
                        load_b_frag_nk(b, sQb, np * 16, ks * 16, lane);
                        mma_bf16(s[2 * np], kf[ks], b[0], b[1]);
                        mma_bf16(s[2 * np + 1], kf[ks], b[2], b[3]);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int il = nt * 8 + 2 * t + (e & 1);
                        const int i = q0 + il;
                        const int j = (e < 2) ? key_lo : key_hi;
                        s[nt][e] = (i >= j && i < T && j < T) ? ex2(s[nt][e] * p.scale_log2 - sLb[il]) : 0.f;
                    }
                }
            } else {
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int il = nt * 8 + 2 * t + (e & 1);
                        const int i = q0 + il;
                        const int j = (e < 2) ? key_lo : key_hi;
                        const float a2 = (e < 2) ? a2_lo[0] : a2_hi[0];
                        float pv = 0.f;
                        if (i >= j && i < T && j < T && sLb[il] != kNegInf)
                            pv = ex2(a2 + __ldg(rh + (i - j)) * kLog2e - sLb[il]);
                        s[nt][e] = pv;
                    }
                }
            }
            // dV += P^T dO   (k = queries, n = head dim).  Replaced heads use
            // a hi + lo bf16 split of P^T: a column of a fixed pattern (a
            // sink, say) can hold large weights over many rows, and bf16
            // rounding of each would add up in dV.
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t pf[4], pl[4];
                if (!rep) {
                    pf[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
                    pf[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
                    pf[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
                    pf[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
                } else {
                    pack_bf16_split(s[2 * kk][0], s[2 * kk][1], pf[0], pl[0]);
                    pack_bf16_split(s[2 * kk][2], s[2 * kk][3], pf[1], pl[1]);
                    pack_bf16_split(s[2 * kk + 1][0], s[2 * kk + 1][1], pf[2], pl[2]);
                    pack_bf16_split(s[2 * kk + 1][2], s[2 * kk + 1][3], pf[3], pl[3]);
                }
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b[4];
                    load_b_frag_kn(b, sOb, np * 16, kk * 16, lane);
                    mma_bf16(dvacc[2 * np], pf, b[0], b[1]);
                    mma_bf16(dvacc[2 * np + 1], pf, b[2], b[3]);
                    if (rep) {
                        mma_bf16(dvacc[2 * np], pl, b[0], b[1]);
                        mma_bf16(dvacc[2 * np + 1], pl, b[2], b[3]);
                    }
                }
            }
            if (!rep) {
                // dP^T = V dO^T  (rows = keys, cols = queries)
                float dp[8][4];
                zero_acc(dp);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
                    for (int np = 0; np < 4; ++np) {
                        uint32_t b[4];
                        load_b_frag_nk(b, sOb, np * 16, ks * 16, lane);
                        mma_bf16(dp[2 * np], vf[ks], b[0], b[1]);
                        mma_bf16(dp[2 * np + 1], vf[ks], b[2], b[3]);
                    }
                }
                // dS^T = P^T o (dP^T - D[query]);  dK += dS^T Q
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    uint32_t df[4];
                    float d0 = sDb[kk * 16 + 2 * t], d1 = sDb[kk * 16 + 2 * t + 1];
                    float d8 = sDb[kk * 16 + 8 + 2 * t], d9 = sDb[kk * 16 + 8 + 2 * t + 1];
                    df[0] = pack_bf16(s[2 * kk][0] * (dp[2 * kk][0] - d0), s[2 * kk][1] * (dp[2 * kk][1] - d1));
                    df[1] = pack_bf16(s[2 * kk][2] * (dp[2 * kk][2] - d0), s[2 * kk][3] * (dp[2 * kk][3] - d1));
                    df[2] = pack_bf16(s[2 * kk + 1][0] * (dp[2 * kk + 1][0] - d8), s[2 * kk + 1][1] * (dp[2 * kk + 1][1] - d9));
                    df[3] = pack_bf16(s[2 * kk + 1][2] * (dp[2 * kk + 1][2] - d8), s[2 * kk + 1][3] * (dp[2 * kk + 1][3] - d9));
#pragma unroll
                    for (int np = 0; np < 4; ++np) {
                        uint32_t b[4];
                        load_b_frag_kn(b, sQb, np * 16, kk * 16, lane);
                        mma_bf16(dkacc[2 * np], df, b[0], b[1]);
                        mma_bf16(dkacc[2 * np + 1], df, b[2], b[3]);
                    }
                }
            }
        }
        __syncthreads();
    }
    store_rows(reinterpret_cast<char*>(p.dv) + base * (p.grad_fp32 ? 4 : 2), p.grad_fp32, key_lo, key_hi, T, dvacc, 1.f, t);
    store_rows(reinterpret_cast<char*>(p.dk) + base * (p.grad_fp32 ? 4 : 2), p.grad_fp32, key_lo, key_hi, T, dkacc, p.scale, t);
}

__global__ void __launch_bounds__(NT) dq_kernel(const BwdParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sQ = smem_u32(smem);     // 64 x 64 (Q, then reused for nothing)
    const uint32_t sO = sQ + BQ * 128;      // dO 64 x 64
    const uint32_t sK = sO + BQ * 128;      // 2 x 64 x 64
    const uint32_t sV = sK + 2 * BK * 128;  // 2 x 64 x 64

    const int T = p.T;
    const int nqb = (T + BQ - 1) / BQ;
    const int qb = nqb - 1 - (int)blockIdx.y;
    const int bh = blockIdx.x;
    const int h = bh % p.H;
    const bool rep = p.hl.replaced[h] != 0;
    const size_t base = (size_t)bh * T * kHeadDim;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int q0 = qb * BQ;
    const int wr0 = q0 + warp * 16;
    const int row_lo = wr0 + g, row_hi = row_lo + 8;
    float acc[8][4];
    zero_acc(acc);
    char* dqbase = reinterpret_cast<char*>(p.dq) + base * (p.grad_fp32 ? 4 : 2);
    if (rep) {  // no query path: dQ = 0
        store_rows(dqbase, p.grad_fp32, row_lo, row_hi, T, acc, 0.f, t);
        return;
    }
    const __nv_bfloat16* Qg = p.q + base;
    const __nv_bfloat16* Kg = p.k + base;
    const __nv_bfloat16* Vg = p.v + base;
    const __nv_bfloat16* Og = p.dout + base;
    const float l2_lo = row_lo < T ? p.lse[(size_t)bh * T + row_lo] * kLog2e : 0.f;
    const float l2_hi = row_hi < T ? p.lse[(size_t)bh * T + row_hi] * kLog2e : 0.f;
    const float D_lo = row_lo < T ? p.dvec[(size_t)bh * T + row_lo] : 0.f;
    const float D_hi = row_hi < T ? p.dvec[(size_t)bh * T + row_hi] : 0.f;

    const int kend = min(q0 + BQ, T);
    const int nkb = (kend + BK - 1) / BK;
    load_tile_async(sQ, Qg, q0, T, BQ, tid, NT);
    load_tile_async(sO, Og, q0, T, BQ, tid, NT);
    load_tile_async(sK, Kg, 0, T, BK, tid, NT);
    load_tile_async(sV, Vg, 0, T, BK, tid, NT);
    cp_async_commit();
    uint32_t qf[4][4], of[4][4];
    for (int kb = 0; kb < nkb; ++kb) {
        const int buf = kb & 1;
        if (kb + 1 < nkb) {
            load_tile_async(sK + (buf ^ 1) * BK * 128, Kg, (kb + 1) * BK, T, BK, tid, NT);
            load_tile_async(sV + (buf ^ 1) * BK * 128, Vg, (kb + 1) * BK, T, BK, tid, NT);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        if (kb == 0) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                load_a_frag(qf[ks], sQ, warp * 16, ks * 16, lane);
                load_a_frag(of[ks], sO, warp * 16, ks * 16, lane);
            }
        }
        const int k0 = kb * BK;
        if (k0 <= wr0 + 15) {
            const uint32_t sKb = sK + buf * BK * 128;
            const uint32_t sVb = sV + buf * BK * 128;
            float s[8][4], dp[8][4];
            zero_acc(s);
            zero_acc(dp);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b[4];
                    load_b_frag_nk(b, sKb, np * 16, ks * 16, lane);
                    mma_bf16(s[2 * np], qf[ks], b[0], b[1]);
                    mma_bf16(s[2 * np + 1], qf[ks], b[2], b[3]);
                    load_b_frag_nk(b, sVb, np * 16, ks * 16, lane);
                    mma_bf16(dp[2 * np], of[ks], b[0], b[1]);
                    mma_bf16(dp[2 * np + 1], of[ks], b[2], b[3]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = k0 + nt * 8 + 2 * t + (e & 1);
                    const int i = (e < 2) ? row_lo : row_hi;
                    const float l2 = (e < 2) ? l2_lo : l2_hi;
                    const float D = (e < 2) ? D_lo : D_hi;
                    const float pv = (j <= i && j < T && i < T) ? ex2(s[nt][e] * p.scale_log2 - l2) : 0.f;
                    s[nt][e] = pv * (dp[nt][e] - D);  // dS
                }
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t af[4];
                af[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
                af[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
                af[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
                af[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b[4];
                    load_b_frag_kn(b, sKb, np * 16, kk * 16, lane);
                    mma_bf16(acc[2 * np], af, b[0], b[1]);
                    mma_bf16(acc[2 * np + 1], af, b[2], b[3]);
                }
            }
        }
        __syncthreads();
    }
    store_rows(dqbase, p.grad_fp32, row_lo, row_hi, T, acc, p.scale, t);
}

}  // namespace

cudaError_t launch_bwd_mma(const __nv_bfloat16* q, const __nv_bfloat16* k,
                           const __nv_bfloat16* v, const __nv_bfloat16* dout,
                           const float* lse, const float* dvec,
                           const float* a, const float* r, const float* logz,
                           const HeadList& hl, int B, int H, int T,
                           void* dq, void* dk, void* dv, int grad_fp32, cudaStream_t stream) {
    BwdParams p{q, k, v, dout, lse, dvec, a, r, logz, dq, dk, dv, hl, H, T, grad_fp32,
                0.125f, kLog2e * 0.125f};
    const int gx = B * H;
    if (gx == 0) return cudaSuccess;
    const int smem1 = 2 * BK * 128 + 4 * BQ * 128 + 4 * BQ * (int)sizeof(float);
    const int smem2 = 2 * BQ * 128 + 4 * BK * 128;
    cudaError_t e = cudaFuncSetAttribute(dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2);
    if (e != cudaSuccess) return e;
    launch_begin(KID_DKDV_MMA, stream);
    dkdv_kernel<<<dim3(gx, (T + BK - 1) / BK), NT, smem1, stream>>>(p);
    launch_end(KID_DKDV_MMA, stream);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    launch_begin(KID_DQ_MMA, stream);
    dq_kernel<<<dim3(gx, (T + BQ - 1) / BQ), NT, smem2, stream>>>(p);
    launch_end(KID_DQ_MMA, stream);
    return cudaGetLastError();
}

}  // namespace saf
