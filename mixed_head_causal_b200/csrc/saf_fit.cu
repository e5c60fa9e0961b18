// Pattern fitting: the compact form of Eq. (3) fitted to a target pattern
// ("When Can Attention Heads Be Statically Defined?", reading notes section
// 二.3: row-wise cross-entropy to the target, whose column (absolute
// position) and distance marginals are the sufficient statistics, Eq. (4);
// 400 Adam steps per head, accepted at a mean row KL of at most 0.2 nat).
//
// With m[j] = sum_i A(i,j), n[d] = sum_i A(i,i-d) of a target A with unit row
// sums, the loss is L = -(1/T) (sum_j alpha_j m_j + sum_d rho_d n_d -
// sum_i log Z(i)), so one Adam step needs log Z (the log-normaliser kernel)
// and the fitted pattern's own column and distance sums,
//   cs[j] = sum_{u>=0} exp(alpha_j + rho_u - log Z(j+u)),
//   ds[d] = sum_{u>=0} exp(alpha_u + rho_d - log Z(u+d)),
// every term a probability (no overflow, underflow only of negligible terms).
// The gradient is dL/dalpha = -(m - cs) / T, dL/drho = -(n - ds) / T.
#include <algorithm>
#include <cstring>

#include "saf_common.cuh"
#include "tc_util.cuh"

namespace saf {
namespace {

constexpr int kFitLanes = 32, kFitWarps = 8;

// Column sums m, distance sums n and sum A log A of each target [slot, T, T].
// Block (slot, 256 outputs): thread k owns column k and distance k.
__global__ void __launch_bounds__(256) fit_stats_kernel(const float* __restrict__ target, int T,
                                                        float* __restrict__ m, float* __restrict__ n,
                                                        double* __restrict__ ent) {
    __shared__ double red[256];
    const int slot = blockIdx.y;
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    const float* A = target + (size_t)slot * T * T;
    double e = 0.0;
    if (k < T) {
        float cm = 0.f, dn = 0.f;
        for (int i = k; i < T; ++i) {
            const float x = A[(size_t)i * T + k];  // column k
            cm += x;
            if (x > 0.f) e += (double)x * log((double)x);
            dn += A[(size_t)i * T + (i - k)];  // distance k
        }
        m[(size_t)slot * T + k] = cm;
        n[(size_t)slot * T + k] = dn;
    }
    red[threadIdx.x] = e;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) atomicAdd(ent + slot, red[0]);
}

// cs (blockIdx.z = 0) or ds (blockIdx.z = 1) for 32 outputs of one slot: lane
// = output index, the 8 warps split the u range; a, r, log Z staged in
// shared memory (3 T floats).
__global__ void __launch_bounds__(kFitLanes * kFitWarps) fit_sums_kernel(const float* __restrict__ alpha,
                                                                         const float* __restrict__ rho,
                                                                         const float* __restrict__ logz, int T,
                                                                         float* __restrict__ cs,
                                                                         float* __restrict__ ds) {
    extern __shared__ float fit_smem[];
    float* sa = fit_smem;
    float* sr = fit_smem + T;
    float* sl = fit_smem + 2 * T;
    __shared__ float part[kFitWarps][kFitLanes];
    const int slot = blockIdx.y;
    const bool diag = blockIdx.z == 1;
    for (int u = threadIdx.x; u < T; u += blockDim.x) {
        sa[u] = alpha[(size_t)slot * T + u];
        sr[u] = rho[(size_t)slot * T + u];
        sl[u] = logz[(size_t)slot * T + u];
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int o = blockIdx.x * kFitLanes + lane;  // output: column j (cs) or distance d (ds)
    const int len = o < T ? T - o : 0;            // u in [0, len)
    const int maxlen = T - blockIdx.x * kFitLanes;
    const int per = (maxlen + kFitWarps - 1) / kFitWarps;
    const int u0 = warp * per, u1 = min(maxlen, u0 + per);
    float s = 0.f;
    for (int u = u0; u < u1; ++u) {
        if (u < len) {
            const float x = diag ? sa[u] + sr[o] - sl[u + o] : sa[o] + sr[u] - sl[o + u];
            s += tc::ex2(x * kLog2e);
        }
    }
    part[warp][lane] = s;
    __syncthreads();
    if (warp == 0 && o < T) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < kFitWarps; ++w) t += part[w][lane];
        (diag ? ds : cs)[(size_t)slot * T + o] = t;
    }
}

// One bias-corrected Adam step on (alpha, rho) of every slot.
__global__ void __launch_bounds__(256) fit_adam_kernel(float* __restrict__ alpha, float* __restrict__ rho,
                                                       const float* __restrict__ m, const float* __restrict__ n,
                                                       const float* __restrict__ cs, const float* __restrict__ ds,
                                                       float* __restrict__ m1, float* __restrict__ m2, int T,
                                                       int nslots, float lr, float c1, float c2) {
    const int64_t total = (int64_t)nslots * 2 * T;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t slot = idx / (2 * T);
        const int e = (int)(idx - slot * 2 * T);
        const bool is_a = e < T;
        const int k = is_a ? e : e - T;
        const size_t at = (size_t)slot * T + k;
        const float g = is_a ? -(m[at] - cs[at]) / (float)T : -(n[at] - ds[at]) / (float)T;
        const float a1 = 0.9f * m1[idx] + 0.1f * g;
        const float a2 = 0.999f * m2[idx] + 0.001f * g * g;
        m1[idx] = a1;
        m2[idx] = a2;
        const float step = lr * (a1 / c1) / (sqrtf(a2 / c2) + 1e-8f);
        if (is_a) alpha[at] -= step;
        else rho[at] -= step;
    }
}

// kl[slot] = (-(sum_j alpha_j m_j + sum_d rho_d n_d - sum_i log Z(i)) + sum A log A) / T
__global__ void __launch_bounds__(256) fit_kl_kernel(const float* __restrict__ alpha, const float* __restrict__ rho,
                                                     const float* __restrict__ logz, const float* __restrict__ m,
                                                     const float* __restrict__ n, const double* __restrict__ ent,
                                                     int T, float* __restrict__ kl) {
    __shared__ double red[256];
    const int slot = blockIdx.x;
    double s = 0.0;
    for (int k = threadIdx.x; k < T; k += blockDim.x) {
        const size_t at = (size_t)slot * T + k;
        s += (double)alpha[at] * m[at] + (double)rho[at] * n[at] - (double)logz[at];
    }
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) kl[slot] = (float)((-red[0] + ent[slot]) / T);
}

}  // namespace

size_t fit_workspace_bytes(int nslots, int T) {
    const size_t nt = (size_t)nslots * T;
    return align256(sizeof(double) * nslots) + 9 * align256(sizeof(float) * nt);
}

cudaError_t launch_fit(const float* target, int nslots, int T, int steps, float lr, float* alpha, float* rho,
                       float* kl, void* ws, cudaStream_t stream) {
    if (nslots == 0 || T == 0) return cudaSuccess;
    const size_t nt = (size_t)nslots * T;
    char* w = static_cast<char*>(ws);
    double* ent = reinterpret_cast<double*>(w);
    w += align256(sizeof(double) * nslots);
    auto take = [&](size_t floats) {
        float* p = reinterpret_cast<float*>(w);
        w += align256(sizeof(float) * floats);
        return p;
    };
    float* m = take(nt);
    float* n = take(nt);
    float* lz = take(nt);
    float* cs = take(nt);
    float* ds = take(nt);
    float* m1 = take(2 * nt);
    float* m2 = take(2 * nt);
    cudaError_t e;
    if ((e = cudaMemsetAsync(ent, 0, sizeof(double) * nslots, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(alpha, 0, sizeof(float) * nt, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(rho, 0, sizeof(float) * nt, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(m1, 0, sizeof(float) * 2 * nt, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(m2, 0, sizeof(float) * 2 * nt, stream)) != cudaSuccess) return e;
    launch_begin(KID_FIT, stream);
    fit_stats_kernel<<<dim3((unsigned)((T + 255) / 256), (unsigned)nslots), 256, 0, stream>>>(target, T, m, n, ent);
    launch_end(KID_FIT, stream);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    HeadList hl;
    memset(&hl, 0, sizeof(hl));
    hl.n = nslots;
    for (int s = 0; s < nslots; ++s) {
        hl.heads[s] = (int16_t)s;
        hl.replaced[s] = 1;
    }
    const int smem = (int)sizeof(float) * 3 * T;  // plus 1 KB of static shared memory
    if ((e = cudaFuncSetAttribute(fit_sums_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
        return e;
    const dim3 sums_grid((unsigned)((T + kFitLanes - 1) / kFitLanes), (unsigned)nslots, 2);
    const int adam_blocks = (int)std::min<int64_t>(148 * 8, ((int64_t)2 * nt + 255) / 256);
    double p1 = 1.0, p2 = 1.0;
    for (int it = 0; it < steps; ++it) {
        if ((e = launch_lognorm(alpha, rho, hl, T, lz, stream)) != cudaSuccess) return e;
        launch_begin(KID_FIT, stream);
        fit_sums_kernel<<<sums_grid, kFitLanes * kFitWarps, smem, stream>>>(alpha, rho, lz, T, cs, ds);
        launch_end(KID_FIT, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        p1 *= 0.9;
        p2 *= 0.999;
        launch_begin(KID_FIT, stream);
        fit_adam_kernel<<<adam_blocks, 256, 0, stream>>>(alpha, rho, m, n, cs, ds, m1, m2, T, nslots, lr,
                                                          (float)(1.0 - p1), (float)(1.0 - p2));
        launch_end(KID_FIT, stream);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if ((e = launch_lognorm(alpha, rho, hl, T, lz, stream)) != cudaSuccess) return e;
    launch_begin(KID_FIT, stream);
    fit_kl_kernel<<<(unsigned)nslots, 256, 0, stream>>>(alpha, rho, lz, m, n, ent, T, kl);
    launch_end(KID_FIT, stream);
    return cudaGetLastError();
}

}  // namespace saf
