// Warp-level helpers for the mma.sync (m16n8k16, bf16 -> fp32) kernels:
// swizzled shared-memory tiles of 64 bf16 columns, cp.async tile loads and
// ldmatrix fragment loads.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace saf {
namespace mma {

// Byte offset of element (row, col) in a [rows][64] bf16 tile whose 16-byte
// chunks are XOR-swizzled by (row % 8), so that the eight rows an ldmatrix
// phase reads fall in eight different bank groups.
__device__ __forceinline__ uint32_t swz(int row, int col) {
    return (uint32_t)(row * 128 + ((((col >> 3) ^ (row & 7))) << 4) + (col & 7) * 2);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Copies rows [row0, row0 + nrows) of a [T][64] bf16 matrix into a swizzled
// tile; rows at or beyond T are zero-filled (no bytes are read for them).
__device__ __forceinline__ void load_tile_async(uint32_t sbase, const __nv_bfloat16* g, int row0,
                                                int T, int nrows, int tid, int nthreads) {
    for (int idx = tid; idx < nrows * 8; idx += nthreads) {
        const int r = idx >> 3, c = idx & 7;
        const int row = row0 + r;
        const int src_row = row < T ? row : (T - 1);
        const __nv_bfloat16* src = g + (size_t)src_row * 64 + c * 8;
        const uint32_t bytes = row < T ? 16u : 0u;
        const uint32_t dst = sbase + (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(bytes));
    }
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// x ~= hi + lo with hi = bf16(x), lo = bf16(x - hi): a two-term bf16 split
// whose sum carries about 16 significant bits instead of 8.
__device__ __forceinline__ void pack_bf16_split(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    float2 hf = __bfloat1622float2(h);
    __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<uint32_t*>(&h);
    lo = *reinterpret_cast<uint32_t*>(&l);
}

// A fragment (16 rows x 16 k) of a swizzled tile: rows r0.., k columns k0...
__device__ __forceinline__ void load_a_frag(uint32_t* a, uint32_t sbase, int r0, int k0, int lane) {
    const int row = r0 + (lane & 7) + ((lane >> 3) & 1) * 8;
    const int col = k0 + (lane >> 4) * 8;
    ldsm_x4(a[0], a[1], a[2], a[3], sbase + swz(row, col));
}

// B fragments of two n8 tiles (n0.., n0+8..) for k-step k0 from a tile stored
// [n][k] (k contiguous, e.g. K for Q K^T).  b[0..1]: tile n0, b[2..3]: n0+8.
__device__ __forceinline__ void load_b_frag_nk(uint32_t* b, uint32_t sbase, int n0, int k0, int lane) {
    const int n = n0 + (lane & 7) + ((lane >> 4) << 3);
    const int k = k0 + ((lane >> 3) & 1) * 8;
    ldsm_x4(b[0], b[1], b[2], b[3], sbase + swz(n, k));
}

// Same, from a tile stored [k][n] (n contiguous, e.g. V for P V).
__device__ __forceinline__ void load_b_frag_kn(uint32_t* b, uint32_t sbase, int n0, int k0, int lane) {
    const int k = k0 + (lane & 7) + ((lane >> 3) & 1) * 8;
    const int n = n0 + (lane >> 4) * 8;
    ldsm_x4_t(b[0], b[1], b[2], b[3], sbase + swz(k, n));
}

}  // namespace mma
}  // namespace saf
