// Trainable pattern: gradients of the replaced heads' pattern vectors.
//
// In the variant of "When Can Attention Heads Be Statically Defined?" where
// alpha and rho are trained (Table 14, "trainable"), the loss reaches them
// through Eq. (3): P is the row softmax of the logits alpha[j] + rho[i-j], so
// with dP = dO V^T and D(i) = sum_j P(i,j) dP(i,j),
//   dS(i,j) = P(i,j) (dP(i,j) - D(i)),
//   dalpha[j] = sum_{b,i} dS(i,j),   drho[d] = sum_{b, i-j=d} dS(i,j)
// (alpha and rho are per head, so the batch sums in).
//
// One CTA per (batch, replaced head, 64-row query block), four warps of 16
// query rows, warp-level bf16 MMAs (m16n8k16, fp32 accumulators) for dP over
// 64-key blocks; P from Eq. (3) with one fp32 exp per element.  Two passes
// over the key blocks: the first accumulates D(i) exactly as defined, the
// second forms dS, stages the 64 x 64 tile in shared memory and sums its
// columns (one thread per key) and diagonals (one thread per distance i - j),
// added to dalpha / drho with one global atomic per key and per distance.
#include "mma_util.cuh"
#include "saf_common.cuh"

namespace saf {
namespace {

using namespace mma;

constexpr int PG_BM = 64;   // query rows per CTA
constexpr int PG_BN = 64;   // keys per block
constexpr int PG_NT = 128;  // 4 warps x 16 rows
constexpr int PG_BINS = PG_BM + PG_BN - 1;  // distances i - j met in one tile
constexpr int PG_LD = PG_BN + 1;            // dS tile row stride (floats): rows and diagonals hit distinct banks

struct PgParams {
    const __nv_bfloat16* v;
    const __nv_bfloat16* dout;
    const float* a;
    const float* r;
    const float* logz;
    float* da;
    float* dr;
    HeadList hl;
    int H, T;
};

__global__ void __launch_bounds__(PG_NT) pattern_grad_kernel(const PgParams p) {
    __shared__ __align__(128) uint8_t sDOb[PG_BM * 128];
    __shared__ __align__(128) uint8_t sVb[PG_BN * 128];
    __shared__ float sDS[PG_BM * PG_LD];
    const uint32_t sDO = smem_u32(sDOb), sV = smem_u32(sVb);

    const int T = p.T;
    const int nqb = (T + PG_BM - 1) / PG_BM;
    const int qb = nqb - 1 - (int)blockIdx.y;  // longest rows first
    const int slot = (int)(blockIdx.x % (unsigned)p.hl.n);
    const int b = (int)(blockIdx.x / (unsigned)p.hl.n);
    const int h = p.hl.heads[slot];
    const size_t base = ((size_t)b * p.H + h) * (size_t)T * kHeadDim;
    const float* ah = p.a + (size_t)h * T;
    const float* rh = p.r + (size_t)h * T;
    const float* lzh = p.logz + (size_t)h * T;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int i0 = qb * PG_BM;
    const int row_lo = i0 + warp * 16 + g, row_hi = row_lo + 8;
    const float lz_lo = row_lo < T ? lzh[row_lo] : kNegInf;
    const float lz_hi = row_hi < T ? lzh[row_hi] : kNegInf;

    load_tile_async(sDO, p.dout + base, i0, T, PG_BM, tid, PG_NT);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    uint32_t af[4][4];  // dO rows of this warp, k = 0..63
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) load_a_frag(af[ks], sDO, warp * 16, ks * 16, lane);

    float D_lo = 0.f, D_hi = 0.f;
    for (int pass = 0; pass < 2; ++pass) {
        for (int kb = 0; kb <= qb; ++kb) {
            const int k0 = kb * PG_BN;
            __syncthreads();  // the previous block's V tile and sums are consumed
            load_tile_async(sV, p.v + base, k0, T, PG_BN, tid, PG_NT);
            cp_async_commit();
            cp_async_wait<0>();
            __syncthreads();
            // dP = dO V^T for this warp's 16 rows x 64 keys
            float dp[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) dp[nt][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t bf[4];
                    load_b_frag_nk(bf, sV, np * 16, ks * 16, lane);
                    mma_bf16(dp[2 * np], af[ks], bf[0], bf[1]);
                    mma_bf16(dp[2 * np + 1], af[ks], bf[2], bf[3]);
                }
            }
            // element (nt, e): row i = e < 2 ? row_lo : row_hi, key j = k0 + nt*8 + 2t + (e & 1)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = k0 + nt * 8 + 2 * t + (e & 1);
                    const int i = (e < 2) ? row_lo : row_hi;
                    const float lz = (e < 2) ? lz_lo : lz_hi;
                    float pv = 0.f;
                    if (j <= i && i < T && lz != kNegInf) pv = __expf(__ldg(ah + j) + __ldg(rh + (i - j)) - lz);
                    if (pass == 0) {
                        if (e < 2) D_lo += pv * dp[nt][e];
                        else D_hi += pv * dp[nt][e];
                    } else {
                        sDS[(i - i0) * PG_LD + (j - k0)] = pv * (dp[nt][e] - ((e < 2) ? D_lo : D_hi));
                    }
                }
            }
            if (pass == 1) {
                __syncthreads();
                // column sums (thread u: key k0 + u) and diagonal sums (thread u:
                // distance i - j = i0 - k0 + u - (PG_BN - 1), i.e. row - col = u - 63)
                if (tid < PG_BN && k0 + tid < T) {
                    float s = 0.f;
                    for (int rr = 0; rr < PG_BM; ++rr) s += sDS[rr * PG_LD + tid];
                    if (s != 0.f) atomicAdd(p.da + (size_t)h * T + k0 + tid, s);
                }
                if (tid < PG_BINS) {
                    const int off = tid - (PG_BN - 1);  // row - col
                    const int d = i0 - k0 + off;
                    if (d >= 0 && d < T) {
                        float s = 0.f;
                        const int c_lo = off < 0 ? -off : 0, c_hi = off < 0 ? PG_BN : PG_BM - off;
                        for (int c = c_lo; c < c_hi; ++c) s += sDS[(c + off) * PG_LD + c];
                        if (s != 0.f) atomicAdd(p.dr + (size_t)h * T + d, s);
                    }
                }
            }
        }
        if (pass == 0) {
            // D(i): the four lanes t of a row hold disjoint keys
            D_lo += __shfl_xor_sync(0xffffffffu, D_lo, 1);
            D_lo += __shfl_xor_sync(0xffffffffu, D_lo, 2);
            D_hi += __shfl_xor_sync(0xffffffffu, D_hi, 1);
            D_hi += __shfl_xor_sync(0xffffffffu, D_hi, 2);
        }
    }
}

}  // namespace

cudaError_t launch_pattern_grad(const __nv_bfloat16* v, const __nv_bfloat16* dout, const float* a, const float* r,
                                const float* logz, const HeadList& hl, int B, int H, int T, float* da, float* dr,
                                cudaStream_t stream) {
    if (hl.n == 0 || B == 0 || T == 0) return cudaSuccess;
    PgParams p{v, dout, a, r, logz, da, dr, hl, H, T};
    dim3 grid((unsigned)(B * hl.n), (unsigned)((T + PG_BM - 1) / PG_BM));
    launch_begin(KID_PATTERN_GRAD, stream);
    pattern_grad_kernel<<<grid, PG_NT, 0, stream>>>(p);
    launch_end(KID_PATTERN_GRAD, stream);
    return cudaGetLastError();
}

}  // namespace saf
