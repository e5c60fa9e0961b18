// Mixed-head causal attention forward, warp-level mma.sync path.
//
// One CTA computes one 128-row query block of one (batch, head) slice with
// eight warps of 16 rows each, walking 64-key blocks from key 0 up to the
// diagonal (causal tile skipping: blocks entirely above the diagonal are
// never visited; the diagonal block is masked element-wise).
//
//  * Ordinary heads: S = Q K^T / sqrt(d_h) with an online softmax (running
//    row max and sum, FlashAttention-2 style), O = P V / l, and the row
//    log-sum-exp as lse.
//  * Replaced heads: the fixed pattern of Eq. (3) ("When Can Attention Heads
//    Be Statically Defined?", section 二.3) is rebuilt tile by tile in
//    registers, P(i,j) = exp(a[j] + r[i-j] - log Z(i)), and multiplied with
//    the current V; no scores, no softmax, Q and K are never read (section
//    二.4 and Fig. 2).  lse is log Z.
#include "mma_util.cuh"
#include "saf_common.cuh"

namespace saf {
namespace {

using namespace mma;

constexpr int BM = 128;  // query rows per CTA
constexpr int BN = 64;   // keys per block
constexpr int NT = 256;  // threads

struct FwdParams {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    __nv_bfloat16* o;
    float* lse;
    const float* a;
    const float* r;
    const float* logz;
    HeadList hl;
    int H, T;
    float scale_log2;  // log2(e) / sqrt(d_h)
};

__global__ void __launch_bounds__(NT) fwd_mma_kernel(const FwdParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sQ = smem_u32(smem);                  // 128 x 64 bf16
    const uint32_t sK = sQ + BM * 128;                   // 2 x 64 x 64
    const uint32_t sV = sK + 2 * BN * 128;               // 2 x 64 x 64

    const int T = p.T;
    const int nqb = (T + BM - 1) / BM;
    const int qb = nqb - 1 - (int)blockIdx.y;  // longest rows first
    const int bh = blockIdx.x;
    const int h = bh % p.H;
    const bool rep = p.hl.replaced[h] != 0;
    const size_t base = (size_t)bh * T * kHeadDim;
    const __nv_bfloat16* Qg = p.q + base;
    const __nv_bfloat16* Kg = p.k + base;
    const __nv_bfloat16* Vg = p.v + base;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int q0 = qb * BM;
    const int wr0 = q0 + warp * 16;              // first row of this warp
    const int row_lo = wr0 + g, row_hi = wr0 + g + 8;
    const int kend = min(q0 + BM, T);            // keys [0, kend) are needed
    const int nkb = (kend + BN - 1) / BN;

    if (!rep) load_tile_async(sQ, Qg, q0, T, BM, tid, NT);
    if (!rep) load_tile_async(sK, Kg, 0, T, BN, tid, NT);
    load_tile_async(sV, Vg, 0, T, BN, tid, NT);
    cp_async_commit();

    const float* ah = p.a + (size_t)h * T;
    const float* rh = p.r + (size_t)h * T;
    float lz_lo = 0.f, lz_hi = 0.f;
    if (rep) {
        const float* lz = p.logz + (size_t)h * T;
        lz_lo = row_lo < T ? lz[row_lo] : 0.f;
        lz_hi = row_hi < T ? lz[row_hi] : 0.f;
    }
    const float lz2_lo = lz_lo * kLog2e, lz2_hi = lz_hi * kLog2e;

    uint32_t qf[4][4];
    float oacc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[i][e] = 0.f;
    float m_lo = kNegInf, m_hi = kNegInf, l_lo = 0.f, l_hi = 0.f;

    for (int kb = 0; kb < nkb; ++kb) {
        const int buf = kb & 1;
        if (kb + 1 < nkb) {
            const int nb = buf ^ 1;
            if (!rep) load_tile_async(sK + nb * BN * 128, Kg, (kb + 1) * BN, T, BN, tid, NT);
            load_tile_async(sV + nb * BN * 128, Vg, (kb + 1) * BN, T, BN, tid, NT);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        if (kb == 0 && !rep) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) load_a_frag(qf[ks], sQ, warp * 16, ks * 16, lane);
        }
        const int k0 = kb * BN;
        if (k0 <= wr0 + 15) {  // some key of this block is visible to this warp
            float s[8][4];
            const uint32_t sKb = sK + buf * BN * 128;
            const uint32_t sVb = sV + buf * BN * 128;
            if (!rep) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int e = 0; e < 4; ++e) s[i][e] = 0.f;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
                    for (int np = 0; np < 4; ++np) {
                        uint32_t b[4];
                        load_b_frag_nk(b, sKb, np * 16, ks * 16, lane);
                        mma_bf16(s[2 * np], qf[ks], b[0], b[1]);
                        mma_bf16(s[2 * np + 1], qf[ks], b[2], b[3]);
                    }
                }
                // scale, causal + tail mask, online softmax
                float mx_lo = m_lo, mx_hi = m_hi;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = k0 + nt * 8 + 2 * t + (e & 1);
                        const int i = (e < 2) ? row_lo : row_hi;
                        float x = s[nt][e] * p.scale_log2;
                        if (j > i || j >= T) x = kNegInf;
                        s[nt][e] = x;
                        if (e < 2) mx_lo = fmaxf(mx_lo, x); else mx_hi = fmaxf(mx_hi, x);
                    }
                }
                mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
                mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
                mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
                mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
                const float c_lo = (m_lo == kNegInf) ? 0.f : exp2f(m_lo - mx_lo);
                const float c_hi = (m_hi == kNegInf) ? 0.f : exp2f(m_hi - mx_hi);
                m_lo = mx_lo;
                m_hi = mx_hi;
                l_lo *= c_lo;
                l_hi *= c_hi;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    oacc[nt][0] *= c_lo; oacc[nt][1] *= c_lo;
                    oacc[nt][2] *= c_hi; oacc[nt][3] *= c_hi;
                }
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float mm = (e < 2) ? mx_lo : mx_hi;
                        const float pv = (s[nt][e] == kNegInf) ? 0.f : exp2f(s[nt][e] - mm);
                        s[nt][e] = pv;
                        if (e < 2) l_lo += pv; else l_hi += pv;
                    }
                }
            } else {
                // P(i,j) = exp(a[j] + r[i-j] - log Z(i)) for j <= i < T
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = k0 + nt * 8 + 2 * t + (e & 1);
                        const int i = (e < 2) ? row_lo : row_hi;
                        const float lz2 = (e < 2) ? lz2_lo : lz2_hi;
                        float pv = 0.f;
                        if (j <= i && i < T && lz2 != kNegInf)
                            pv = exp2f((__ldg(ah + j) + __ldg(rh + (i - j))) * kLog2e - lz2);
                        s[nt][e] = pv;
                    }
                }
            }
            // O += P V.  A replaced head's P enters as a hi + lo bf16 pair:
            // its weights are not renormalised by an online softmax, so their
            // rounding would otherwise reach the output at full size.
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t af[4], al[4];
                if (!rep) {
                    af[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
                    af[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
                    af[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
                    af[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
                } else {
                    pack_bf16_split(s[2 * kk][0], s[2 * kk][1], af[0], al[0]);
                    pack_bf16_split(s[2 * kk][2], s[2 * kk][3], af[1], al[1]);
                    pack_bf16_split(s[2 * kk + 1][0], s[2 * kk + 1][1], af[2], al[2]);
                    pack_bf16_split(s[2 * kk + 1][2], s[2 * kk + 1][3], af[3], al[3]);
                }
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b[4];
                    load_b_frag_kn(b, sVb, np * 16, kk * 16, lane);
                    mma_bf16(oacc[2 * np], af, b[0], b[1]);
                    mma_bf16(oacc[2 * np + 1], af, b[2], b[3]);
                    if (rep) {
                        mma_bf16(oacc[2 * np], al, b[0], b[1]);
                        mma_bf16(oacc[2 * np + 1], al, b[2], b[3]);
                    }
                }
            }
        }
        __syncthreads();
    }

    // epilogue
    float inv_lo = 1.f, inv_hi = 1.f, lse_lo, lse_hi;
    if (!rep) {
        l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
        l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
        l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
        l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
        inv_lo = l_lo > 0.f ? 1.f / l_lo : 0.f;
        inv_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
        lse_lo = (m_lo + log2f(l_lo)) * kLn2;
        lse_hi = (m_hi + log2f(l_hi)) * kLn2;
    } else {
        lse_lo = lz_lo;
        lse_hi = lz_hi;
    }
    __nv_bfloat16* Og = p.o + base;
    float* Lg = p.lse + (size_t)bh * T;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        const int c = nt * 8 + 2 * t;
        if (row_lo < T)
            *reinterpret_cast<__nv_bfloat162*>(Og + (size_t)row_lo * kHeadDim + c) =
                __floats2bfloat162_rn(oacc[nt][0] * inv_lo, oacc[nt][1] * inv_lo);
        if (row_hi < T)
            *reinterpret_cast<__nv_bfloat162*>(Og + (size_t)row_hi * kHeadDim + c) =
                __floats2bfloat162_rn(oacc[nt][2] * inv_hi, oacc[nt][3] * inv_hi);
    }
    if (t == 0) {
        if (row_lo < T) Lg[row_lo] = lse_lo;
        if (row_hi < T) Lg[row_hi] = lse_hi;
    }
}

}  // namespace

cudaError_t launch_fwd_mma(const __nv_bfloat16* q, const __nv_bfloat16* k,
                           const __nv_bfloat16* v, __nv_bfloat16* o, float* lse,
                           const float* a, const float* r, const float* logz,
                           const HeadList& hl, int B, int H, int T, cudaStream_t stream) {
    FwdParams p{q, k, v, o, lse, a, r, logz, hl, H, T, kLog2e / 8.0f};
    const int smem = BM * 128 + 4 * BN * 128;
    cudaError_t e = cudaFuncSetAttribute(fwd_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(B * H, (T + BM - 1) / BM);
    if (grid.x == 0) return cudaSuccess;
    launch_begin(KID_FWD_MMA, stream);
    fwd_mma_kernel<<<grid, NT, smem, stream>>>(p);
    launch_end(KID_FWD_MMA, stream);
    return cudaGetLastError();
}

}  // namespace saf
