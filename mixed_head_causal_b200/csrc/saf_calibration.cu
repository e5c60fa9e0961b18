// Calibration statistics of attention heads (section 二.1 of the reading notes
// for "When Can Attention Heads Be Statically Defined?"): over N calibration
// sequences, the sample mean of each head's causal softmax attention matrix,
//   A_hat = (1/N) sum_n A^(n),
// and its reconstruction error, Eq. (1),
//   s_var = sum_n ||A^(n) - A_hat||_F^2 / ((N - 1) T^2).
//
// One CTA per (64 x 64 tile of A, head); it walks the N samples twice with the
// tile's scores recomputed each time (S = Q K^T on warp-level bf16 MMAs, P =
// exp(S / sqrt(d) - lse) with the lse of the forward pass), so no per-sample
// T x T matrix is ever stored: the first walk sums P into the mean tile held in
// registers, the second sums (P - A_hat)^2.  Each tile writes its part of
// A_hat and one partial error; a second kernel adds the partials of a head in
// a fixed order (deterministic).
#include "mma_util.cuh"
#include "saf_common.cuh"

namespace saf {
namespace {

using namespace mma;

constexpr int CB_T = 64;    // tile rows (queries) and columns (keys)
constexpr int CB_NT = 128;  // 4 warps x 16 rows

struct CalParams {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const float* lse;
    float* a_hat;    // [H, T, T]
    float* partial;  // [H, ntile * ntile] squared-error partial sums
    int N, H, T;
    float scale;
};

__global__ void __launch_bounds__(CB_NT) calibration_tile_kernel(const CalParams p) {
    __shared__ __align__(128) uint8_t sQb[CB_T * 128];
    __shared__ __align__(128) uint8_t sKb[CB_T * 128];
    __shared__ float sRed[CB_NT / 32];
    const uint32_t sQ = smem_u32(sQb), sK = smem_u32(sKb);
    const int T = p.T;
    const int nt = (T + CB_T - 1) / CB_T;
    const int qb = (int)blockIdx.x / nt, kb = (int)blockIdx.x % nt;
    const int h = (int)blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int i0 = qb * CB_T, j0 = kb * CB_T;
    const int row_lo = i0 + warp * 16 + g, row_hi = row_lo + 8;
    float* out = p.a_hat + (size_t)h * T * T;

    if (kb > qb) {  // strictly above the diagonal: A is zero there
        for (int e = tid; e < CB_T * CB_T; e += CB_NT) {
            const int i = i0 + e / CB_T, j = j0 + e % CB_T;
            if (i < T && j < T) out[(size_t)i * T + j] = 0.f;
        }
        if (tid == 0) p.partial[(size_t)h * nt * nt + blockIdx.x] = 0.f;
        return;
    }

    float mean[8][4];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int e = 0; e < 4; ++e) mean[a][e] = 0.f;
    float err = 0.f;
    for (int pass = 0; pass < 2; ++pass) {
        for (int n = 0; n < p.N; ++n) {
            const size_t base = ((size_t)n * p.H + h) * (size_t)T * kHeadDim;
            __syncthreads();  // the previous sample's tiles are consumed
            load_tile_async(sQ, p.q + base, i0, T, CB_T, tid, CB_NT);
            load_tile_async(sK, p.k + base, j0, T, CB_T, tid, CB_NT);
            cp_async_commit();
            cp_async_wait<0>();
            __syncthreads();
            const float* lse = p.lse + ((size_t)n * p.H + h) * T;
            const float l_lo = row_lo < T ? lse[row_lo] : 0.f;
            const float l_hi = row_hi < T ? lse[row_hi] : 0.f;
            float s[8][4];
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[a][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t af[4];
                load_a_frag(af, sQ, warp * 16, ks * 16, lane);
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t bf[4];
                    load_b_frag_nk(bf, sK, np * 16, ks * 16, lane);
                    mma_bf16(s[2 * np], af, bf[0], bf[1]);
                    mma_bf16(s[2 * np + 1], af, bf[2], bf[3]);
                }
            }
            // element (a, e): row i = e < 2 ? row_lo : row_hi, key j = j0 + a*8 + 2t + (e & 1)
#pragma unroll
            for (int a = 0; a < 8; ++a) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = j0 + a * 8 + 2 * t + (e & 1);
                    const int i = (e < 2) ? row_lo : row_hi;
                    const float pv = (j <= i && i < T && j < T) ? expf(s[a][e] * p.scale - ((e < 2) ? l_lo : l_hi))
                                                                : 0.f;
                    if (pass == 0) {
                        mean[a][e] += pv;
                    } else {
                        const float x = pv - mean[a][e];
                        err += x * x;
                    }
                }
            }
        }
        if (pass == 0) {
            const float inv = 1.f / (float)p.N;
#pragma unroll
            for (int a = 0; a < 8; ++a) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    mean[a][e] *= inv;
                    const int j = j0 + a * 8 + 2 * t + (e & 1);
                    const int i = (e < 2) ? row_lo : row_hi;
                    if (i < T && j < T) out[(size_t)i * T + j] = mean[a][e];
                }
            }
        }
    }
    // the tile's squared error: warp shuffle, then the four warps in order
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) err += __shfl_xor_sync(0xffffffffu, err, off);
    if (lane == 0) sRed[warp] = err;
    __syncthreads();
    if (tid == 0) {
        float tot = 0.f;
        for (int w = 0; w < CB_NT / 32; ++w) tot += sRed[w];
        p.partial[(size_t)h * nt * nt + blockIdx.x] = tot;
    }
}

// s_var[h] = sum of the head's tile partials (fixed order) / ((N - 1) T^2).
__global__ void __launch_bounds__(256) calibration_finish_kernel(const float* __restrict__ partial, int ntiles,
                                                                 int N, int T, float* __restrict__ svar) {
    __shared__ double red[256];
    const int h = blockIdx.x;
    double s = 0.0;
    for (int u = threadIdx.x; u < ntiles; u += blockDim.x) s += (double)partial[(size_t)h * ntiles + u];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) svar[h] = (float)(red[0] / ((double)(N - 1) * (double)T * (double)T));
}

}  // namespace

size_t calibration_partial_floats(int H, int T) {
    const size_t nt = (size_t)(T + CB_T - 1) / CB_T;
    return (size_t)H * nt * nt;
}

cudaError_t launch_calibration(const __nv_bfloat16* q, const __nv_bfloat16* k, const float* lse, int N, int H,
                               int T, float* a_hat, float* svar, float* partial, cudaStream_t stream) {
    if (H == 0 || T == 0) return cudaSuccess;
    const int nt = (T + CB_T - 1) / CB_T;
    CalParams p{q, k, lse, a_hat, partial, N, H, T, 0.125f};
    launch_begin(KID_CALIBRATION, stream);
    calibration_tile_kernel<<<dim3((unsigned)(nt * nt), (unsigned)H), CB_NT, 0, stream>>>(p);
    launch_end(KID_CALIBRATION, stream);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    launch_begin(KID_CALIBRATION, stream);
    calibration_finish_kernel<<<(unsigned)H, 256, 0, stream>>>(partial, nt * nt, N, T, svar);
    launch_end(KID_CALIBRATION, stream);
    return cudaGetLastError();
}

}  // namespace saf
