// Mixed-head causal attention backward on the 5th-generation tensor cores.
//
// A work item is one 128-key block J of one (batch, head) slice; it walks the
// query blocks I >= J (causal tile skipping; the diagonal block is masked).
// dK and dV accumulate in TMEM for the whole walk; each tile's dQ
// contribution is reduced into an fp32 accumulator in global memory with a
// TMA reduce-add.  The kernel is persistent: one CTA per SM pulls items,
// longest first, from a counter in the workspace header (reset by the last
// CTA), so K/V of the next item load while this one runs and the next item's
// first MMAs overlap this one's dK/dV read-out.  Warp roles:
//   warp 0      TMA producer: work items; K (two stages), V per item; Q, dO
//               and the per-query vectors of each query block through an
//               NQS-stage ring that runs on across items
//   warp 1      TMEM owner and MMA issuer (one elected lane)
//   warps 2..9  key rows, two warps per row quarter (query columns 0..63 and
//               64..127 of each tile): P^T, dS^T, and the dK/dV epilogue
//   warps 10..13 one query row per thread: dQ tile TMEM -> smem -> reduce-add
//
// Ordinary head, per tile (rows = keys j, columns = queries i; the textbook
// softmax-attention gradients, section 二.4 of the reading notes):
//   S^T  = K Q^T            SS MMA            P^T = exp2(S^T s log2e - lse2_i)
//   dP^T = V dO^T           SS MMA            dS^T = P^T o (dP^T - D_i)
//   dV  += P^T dO           TS MMA (P^T as bf16 in TMEM, aliasing S^T)
//   dK  += dS^T Q           TS MMA (dS^T as bf16 in TMEM, aliasing dP^T)
//   dQ_I = dS K             SS MMA (dS^T in smem read as an MN-major A)
// Replaced head: only dV = P^T dO (section 二.4), with P in the factored
// form of Eq. (3): P^T(j,i) = c_j * W(j,i), W(j,i) = E[i-j] r_i in fp32,
// fed to the tensor cores as a hi + lo bf16 pair (two TS MMAs) so that a
// column with large weights over many rows (a sink) keeps its precision;
// c_j is applied in the epilogue.  dK = 0 there, and dQ gets no contribution.
// A replaced head whose factors would leave fp32 range (flag set by the prep
// kernel) uses P^T itself, one exp per element, and no c_j.
#include "saf_common.cuh"
#include "tc_util.cuh"

namespace saf {
namespace {

using namespace tc;

constexpr int BM = 128;  // queries per block
constexpr int BN = 128;  // keys per CTA
constexpr int NTHREADS = 448;  // producer, MMA, 8 key-row warps, 4 dQ warps
constexpr uint32_t TILE = 128 * 64 * 2;  // 16 KB bf16 tile
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t C_S = 0, C_DP = 128, C_DV = 256, C_DK = 320, C_DQ0 = 384, C_DQ1 = 448;
constexpr long long kWaitLimit = 1ll << 31;

// K in two stages (its last reader, dQ = dS K, closes an item); V in one,
// free once the item's last dP^T MMA is done, about a tile before the item ends
constexpr uint32_t SM_K = 0;
constexpr uint32_t SM_V = SM_K + 2 * TILE;
// Q/dO ring depth: a TMA round trip from L2 takes several tiles' worth of
// MMA time, so the ring keeps NQS query blocks in flight
constexpr int NQS = 3;
constexpr uint32_t SM_Q = SM_V + TILE;          // NQS stages
constexpr uint32_t SM_DO = SM_Q + NQS * TILE;   // NQS stages
constexpr uint32_t SM_DS = SM_DO + NQS * TILE;  // 32 KB: dS^T as two 64-query atoms
// dQ staging, 32 KB: per dQ warp two [32][32] fp32 boxes (its 32 query rows,
// columns 0..31 and 32..63) with the 128-byte swizzle of the reduce map
constexpr uint32_t SM_DQ = SM_DS + 2 * TILE;
constexpr uint32_t SM_VEC1 = SM_DQ + 2 * TILE;        // NQS x 512 B: -lse2 (ordinary) / r (replaced)
constexpr uint32_t SM_VEC2 = SM_VEC1 + 512 * NQS;  // NQS x 512 B: D
constexpr uint32_t SM_BAR = SM_VEC2 + 512 * NQS;
// (SM_BAR + 256: the two work-item slots, 16 bytes each)
constexpr uint32_t SM_DFL = SM_BAR + 512;  // per replaced slot: 1 = per-element path
constexpr uint32_t SM_TOTAL = SM_DFL + 256;

struct BwdTcParams {
    const float* nlse2p;
    const float* dvecp;
    const float* a;  // [H, T] pattern vectors and log Z (read for flag-1 replaced heads only)
    const float* r;
    const float* logz;
    ReplacedWs w;
    void* dk;
    void* dv;
    unsigned int* err;
    int16_t slot_of_head[kMaxHeads];
    int H, Hkv, BH, T, Tp, nqb, grad_fp32;  // Hkv: K/V heads (H / Hkv query heads share one)
    int tma_grads;  // bf16 dK, dV written by TMA stores of 32-row boxes (else per-thread row stores)
    int nslots;  // replaced heads
    float scale, scale_log2;
};

__device__ __forceinline__ void report(unsigned int* err, unsigned int code) {
    atomicOr(err, 1u);
    atomicCAS(err + 1, 0u, code);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// TMEM column (relative to its fp32 region) of the bf16 pairs of query chunk
// c: queries 0..63 pack into columns 0..31, queries 64..127 into 64..95, so
// each half of a row only ever overwrites columns it has already read itself.
__device__ __forceinline__ uint32_t packed_col(int c) { return c < 2 ? 16 * c : 64 + 16 * (c - 2); }
// A-operand column of MMA k-step k (16 queries) in that packing.
__device__ __forceinline__ uint32_t packed_kcol(int k) { return k < 4 ? 8 * k : 64 + 8 * (k - 4); }

// P^T for this warp's 64 queries [64 half, 64 half + 64) of key row jl:
// exp2(S^T * scale - lse2), as bf16 pairs over the S^T columns already read
// (the 32-query chunk c goes to packed_col(c)).  Shared memory at nlse2 holds
// -lse2 per query (read as pairs, 16 bytes at a time); the scale-and-shift
// runs on paired fp32 FMAs.  Four 16-query steps whose TMEM loads are double
// buffered: the load of step k + 1 is in flight while step k is computed.
// MASK: zero where the query precedes the key on the diagonal tile, or where
// the key lies past T.
template <bool MASK>
__device__ __forceinline__ void p_half(uint32_t tS, int half, uint32_t nlse2, float scale, int jl, bool diag,
                                       bool key_ok, uint32_t (&pw)[2][16]) {
    const uint64_t sc2 = f32x2(scale, scale);
    uint32_t va[16], vb[16];
    tmem_ld16(tS + 64 * half, va);
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t(&cur)[16] = (k & 1) ? vb : va;
        uint32_t(&nxt)[16] = (k & 1) ? va : vb;
        if (k < 3) tmem_ld16(tS + 64 * half + 16 * (k + 1), nxt);
        const int q0 = 64 * half + 16 * k;  // first query of the step
        uint64_t nl[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) ld_shared_2x64(nlse2 + 4 * q0 + 16 * q, nl[2 * q], nl[2 * q + 1]);
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
            const int ql = q0 + e;
            const float2 x =
                split_f32x2(fma_f32x2(f32x2(__uint_as_float(cur[e]), __uint_as_float(cur[e + 1])), sc2, nl[e / 2]));
            float p0 = ex2(x.x), p1 = ex2(x.y);
            if (MASK) {
                if (!key_ok || (diag && ql < jl)) p0 = 0.f;
                if (!key_ok || (diag && ql + 1 < jl)) p1 = 0.f;
            }
            pw[k >> 1][8 * (k & 1) + e / 2] = pack_bf16x2(p0, p1);
        }
        if (k & 1) tmem_st16(tS + packed_col(2 * half + (k >> 1)), pw[k >> 1]);
        if (k < 3) tmem_wait_ld();
    }
}

// Stores one 64-wide row of an fp32 accumulator (already scaled) as bf16 or fp32.
__device__ __forceinline__ void store_row(void* base, int grad_fp32, size_t row, const float* v) {
    if (grad_fp32) {
        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + row * kHeadDim);
#pragma unroll
        for (int e = 0; e < 16; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
    } else {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(base) + row * kHeadDim);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            dst[e] = make_uint4(pack_bf16x2(v[8 * e], v[8 * e + 1]), pack_bf16x2(v[8 * e + 2], v[8 * e + 3]),
                                pack_bf16x2(v[8 * e + 4], v[8 * e + 5]), pack_bf16x2(v[8 * e + 6], v[8 * e + 7]));
    }
}

// P^T(j, i) = exp(a[j] + r[i-j] - log Z(i)) of a replaced head straight from
// Eq. (3) (aj = a[j], -inf past T); 0 before the key, past T, or where log Z
// is -inf.
__device__ __forceinline__ float direct_pt(const BwdTcParams& p, int h, int T, float aj, int j, int i) {
    if (i < j || i >= T) return 0.f;
    const float lz = __ldg(p.logz + (size_t)h * T + i);
    if (lz == kNegInf) return 0.f;
    return ex2((aj + __ldg(p.r + (size_t)h * T + (i - j)) - lz) * kLog2e);
}

// The direct P^T for query columns [64 half, 64 half + 64) of this thread's
// key row, as hi + lo bf16 pairs into the W buffer at tW (kept out of line:
// the path is rare).
__device__ __noinline__ void direct_pt_half(const BwdTcParams& p, int h, int T, float aj, int j, int qbase, int half,
                                            uint32_t tW) {
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * half + cc;
        uint32_t hw[16], lw[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
            const float w0 = direct_pt(p, h, T, aj, j, qbase + 32 * c + e);
            const float w1 = direct_pt(p, h, T, aj, j, qbase + 32 * c + e + 1);
            const uint32_t hb = pack_bf16x2(w0, w1);
            const float2 hf = unpack_bf16x2(hb);
            hw[e / 2] = hb;
            lw[e / 2] = pack_bf16x2(w0 - hf.x, w1 - hf.y);
        }
        tmem_st16(tW + 16 * c, hw);
        tmem_st16(tW + 64 + 16 * c, lw);
    }
}

__global__ void __launch_bounds__(NTHREADS, 1)
bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
              const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmDK,
              const __grid_constant__ CUtensorMap tmDV, const BwdTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sb = smem_addr(smem);
    const uint32_t bar_itf = sb + SM_BAR;       // [2] work item slot full
    const uint32_t bar_ite = bar_itf + 16;      // [2] work item slot read (13 warp arrivals)
    const uint32_t bar_kf = bar_ite + 16;       // [2] K stage full
    const uint32_t bar_ke = bar_kf + 16;        // [2] K stage free (the MMAs of its item done)
    const uint32_t bar_vf = bar_ke + 16;        // V full
    const uint32_t bar_ve = bar_vf + 8;         // V free (the item's last dP^T MMA done)
    const uint32_t bar_qf = bar_ve + 8;         // [NQS]
    const uint32_t bar_qe = bar_qf + 8 * NQS;   // [NQS]
    const uint32_t bar_s = bar_qe + 8 * NQS;
    const uint32_t bar_dp = bar_s + 8;
    const uint32_t bar_p = bar_dp + 8;      // 256 arrivals
    const uint32_t bar_ds = bar_p + 8;      // 256 arrivals
    const uint32_t bar_dqf = bar_ds + 8;    // [2]
    const uint32_t bar_dqe = bar_dqf + 16;  // [2] 128 arrivals
    const uint32_t bar_acc = bar_dqe + 16;  // an item's dK, dV complete in TMEM
    const uint32_t bar_acr = bar_acc + 8;   // an item's dK, dV read out of TMEM (8 warp arrivals)
    const uint32_t bar_wb = bar_acr + 8;    // [2] replaced head: W buffer b consumed
    const uint32_t bar_pb = bar_wb + 16;    // [2] replaced head: W buffer b written (256 arrivals)
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SM_BAR + 240);
    // [2] work item n & 1, decoded by the producer: {word (-1: none left), bh, J, h}
    const uint32_t item_slot = sb + SM_BAR + 256;
    static_assert(80 + 16 * NQS + 112 <= 240, "barrier area");

    const int T = p.T;
    const int total = p.BH * p.nqb;  // work items: one key block of one (b, h) slice
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_itf + 8 * b, 1);
            mbar_init(bar_ite + 8 * b, 13);
            mbar_init(bar_kf + 8 * b, 1);
            mbar_init(bar_ke + 8 * b, 1);
            mbar_init(bar_dqf + 8 * b, 1);
            mbar_init(bar_dqe + 8 * b, 128);
            mbar_init(bar_wb + 8 * b, 1);
            mbar_init(bar_pb + 8 * b, 256);
        }
        for (int s = 0; s < NQS; ++s) {
            mbar_init(bar_qf + 8 * s, 1);
            mbar_init(bar_qe + 8 * s, 1);
        }
        mbar_init(bar_vf, 1);
        mbar_init(bar_ve, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_dp, 1);
        mbar_init(bar_p, 256);
        mbar_init(bar_ds, 256);
        mbar_init(bar_acc, 1);
        mbar_init(bar_acr, 8);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_holder), TMEM_COLS);
        tmem_relinquish();
    }
    uint8_t* dfl = smem + SM_DFL;
    if (warp == 0) slot_flags(p.w, p.nslots, dfl);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    // Work item n of this CTA (-1: none left), published by the producer
    // through a 2-slot ring; every consumer warp acknowledges it.
    // (b, h) slice and key block of an item, grouped longest-first order (key
    // block J walks nqb - J query blocks; a group's Q/dO tiles and dQ
    // accumulator rows stay in L2)
    struct Item {
        int bh, bhkv, J, h, slot, ntiles;  // query slice, its K/V slice, key block, head, replaced slot, tiles
        bool rep, direct, ragged;
    };
    // the published item word carries the head's per-element flag in bit 30
    // (set by the producer from the per-slot flags)
    auto decode = [&](int word) {
        const int item = word & 0x3fffffff;
        Item it;
        grouped_order((unsigned)item, p.BH, p.nqb, it.bh, it.J);
        it.h = it.bh % p.H;
        it.bhkv = (it.bh / p.H) * p.Hkv + it.h / (p.H / p.Hkv);  // the K/V slice this query head reads
        it.slot = p.slot_of_head[it.h];
        it.rep = it.slot >= 0;
        // a replaced head whose factors would leave fp32 range takes P^T itself
        // (one exp per element) in place of W^T, and its dV rows need no c_j
        it.direct = it.rep && ((word >> 30) & 1) != 0;
        it.ntiles = p.nqb - it.J;
        it.ragged = (it.J + 1) * BN > T;  // the key block runs past T
        return it;
    };
    // Work item n of this CTA (-1: none left), published by the producer,
    // already decoded, through a 2-slot ring; every consumer warp acknowledges
    // it.
    auto take_item = [&](int n, int& item, Item& it) -> bool {
        if (!mbar_wait(bar_itf + 8 * (n & 1), (n >> 1) & 1, kWaitLimit)) return false;
        const uint4 w = ld_shared_u4(item_slot + 16 * (n & 1));
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_ite + 8 * (n & 1));
        item = (int)w.x;
        it.bh = (int)w.y;
        it.J = (int)w.z;
        it.h = (int)w.w;
        it.bhkv = -1;  // the producer's alone
        it.slot = item >= 0 ? p.slot_of_head[it.h] : -1;
        it.rep = it.slot >= 0;
        it.direct = it.rep && ((item >> 30) & 1) != 0;
        it.ntiles = p.nqb - it.J;
        it.ragged = (it.J + 1) * BN > T;
        return true;
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmDO);
            int s = 0, u = 0, nk = 0;  // ring stage and pass of the next query block; ordinary items so far
            bool ok = true;
            for (int n = 0; ok; ++n) {
                const int w = (int)atomicAdd(p.err + kCtrBwdNext, 1u);
                int item = w < total ? w : -1;
                Item it{};
                if (item >= 0) {
                    it = decode(item);
                    if (!SAF_CHECKED_OK(p.err,
                                        it.bh >= 0 && it.bh < p.BH && it.J >= 0 && it.J < p.nqb && it.h >= 0 &&
                                            it.h < p.H && it.slot < p.nslots && it.bhkv >= 0 &&
                                            it.bhkv < (p.BH / p.H) * p.Hkv,
                                        0x9201u)) {
                        ok = false;
                        break;
                    }
                    if (it.rep && dfl[it.slot]) {
                        item |= 1 << 30;
                        it.direct = true;
                    }
                }
                if (!mbar_wait(bar_ite + 8 * (n & 1), ((n >> 1) & 1) ^ 1, kWaitLimit)) { ok = false; break; }
                st_shared_v4(item_slot + 16 * (n & 1), (uint32_t)item, (uint32_t)it.bh, (uint32_t)it.J, (uint32_t)it.h);
                mbar_arrive(bar_itf + 8 * (n & 1));
                if (item < 0) break;
                if (!it.rep) {
                    // K of the key block into stage nk & 1, once the MMAs of the
                    // ordinary item two before (the stage's last user) are done;
                    // this overlaps the load with the current item's tiles.  V goes
                    // to L2 now and to shared memory after the first query block
                    // (its buffer frees up only late in the previous item).
                    const int kb = nk & 1;
                    if (!mbar_wait(bar_ke + 8 * kb, ((nk >> 1) & 1) ^ 1, kWaitLimit)) { ok = false; break; }
                    mbar_expect_tx(bar_kf + 8 * kb, TILE);
                    tma_load_3d(sb + SM_K + kb * TILE, &tmK, bar_kf + 8 * kb, 0, it.J * BN, it.bhkv);
                    tma_prefetch_l2_3d(&tmV, 0, it.J * BN, it.bhkv);
                }
                for (int t = 0; t < it.ntiles; ++t) {
                    const int I = it.J + t;
                    if (!mbar_wait(bar_qe + 8 * s, (u & 1) ^ 1, kWaitLimit)) { ok = false; break; }
                    const uint32_t bq = bar_qf + 8 * s;
                    if (!it.rep) {
                        mbar_expect_tx(bq, 2 * TILE + 1024);
                        tma_load_3d(sb + SM_Q + s * TILE, &tmQ, bq, 0, I * BM, it.bh);
                        tma_load_3d(sb + SM_DO + s * TILE, &tmDO, bq, 0, I * BM, it.bh);
                        if (!SAF_CHECKED_OK(p.err, I < p.nqb && (size_t)I * BM + BM <= (size_t)p.Tp, 0x9202u)) {
                            ok = false;
                            break;
                        }
                        bulk_load(sb + SM_VEC1 + 512 * s, p.nlse2p + (size_t)it.bh * p.Tp + I * BM, 512, bq);
                        bulk_load(sb + SM_VEC2 + 512 * s, p.dvecp + (size_t)it.bh * p.Tp + I * BM, 512, bq);
                        if (t == 0) {
                            // V of ordinary item nk: the previous one's last dP^T read V
                            if (!mbar_wait(bar_ve, (nk & 1) ^ 1, kWaitLimit)) { ok = false; break; }
                            mbar_expect_tx(bar_vf, TILE);
                            tma_load_3d(sb + SM_V, &tmV, bar_vf, 0, it.J * BN, it.bhkv);
                        }
                    } else {
                        mbar_expect_tx(bq, TILE + 512);
                        tma_load_3d(sb + SM_DO + s * TILE, &tmDO, bq, 0, I * BM, it.bh);
                        if (!SAF_CHECKED_OK(p.err, it.slot >= 0 && I < p.nqb && (size_t)I * BM + BM <= (size_t)p.w.Tp,
                                            0x9203u)) {
                            ok = false;
                            break;
                        }
                        bulk_load(sb + SM_VEC1 + 512 * s, p.w.rsc + (size_t)it.slot * p.w.Tp + I * BM, 512, bq);
                    }
                    if (++s == NQS) {
                        s = 0;
                        ++u;
                    }
                }
                if (!it.rep) ++nk;
            }
            if (!ok) report(p.err, 0x1101);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        const uint32_t idSS = idesc_bf16(128, 128, 0, 0);  // K-major x K-major, 128 x 128
        const uint32_t idTS = idesc_bf16(128, 64, 0, 1);   // TMEM A x MN-major B, 128 x 64
        const uint32_t idDQ = idesc_bf16(128, 64, 1, 1);   // MN-major A x MN-major B
        // descriptors of the tiles: one base plus (byte offset / 16); ring
        // stages and their descriptors advance incrementally (the issuing
        // thread keeps its scalar work small: the pipe stalls while it computes)
        constexpr uint64_t kStage = TILE >> 4;
        const uint64_t d0 = sw128_desc(sb);
        const uint64_t dK0 = d0 + (SM_K >> 4), dVd = d0 + (SM_V >> 4);
        const uint64_t dQ0 = d0 + (SM_Q >> 4), dDO0 = d0 + (SM_DO >> 4);
        const uint64_t dDS = sw128_desc(sb + SM_DS, 16384);
        int s = 0, ph = 0;           // ring stage of the next query block and its phase parity
        int go = 0, gr = 0, nk = 0;  // ordinary tiles, replaced tiles, ordinary items so far
        bool ok = true;
        for (int n = 0; ok; ++n) {
            int item;
            Item it;
            ok = __all_sync(0xffffffffu, take_item(n, item, it));
            if (!ok) {
                if (lane == 0) report(p.err, 0x1208);
                break;
            }
            if (item < 0) break;
            int okl = 1;
            // The whole warp runs the schedule (its waits give one answer for
            // all lanes) and one elected lane issues each group of MMAs and their
            // commits (always the same lane, so a commit covers all its MMAs).
            if (!it.rep) {
                // Ordinary heads run one tile ahead: S^T of tile t+1 is issued
                // right after dV_t (the last reader of the P^T columns it
                // overwrites) and dP^T of tile t+1 right after dQ_t, so the tensor
                // cores work on the next tile while the row threads finish this
                // one; an item's first S^T and dP^T go in while the row threads
                // still read out the previous item's dK, dV.  The tensor pipe
                // executes one thread's MMAs in order, which orders those reuses.
                const int kb = nk & 1;
                const uint64_t dK = dK0 + (uint64_t)kb * kStage;
                auto issue_s = [&](uint64_t dQn) {
                    if (elect_one()) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) mma_ss(tmem + C_S, dK + 2 * k, dQn + 2 * k, idSS, k > 0);
                        mma_commit(bar_s);
                    }
                    __syncwarp();
                };
                // dP^T of the item's last tile is V's last reader: V's buffer is
                // released with it
                auto issue_dp = [&](uint64_t dDOn, bool last) {
                    if (elect_one()) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) mma_ss(tmem + C_DP, dVd + 2 * k, dDOn + 2 * k, idSS, k > 0);
                        mma_commit(bar_dp);
                        if (last) mma_commit(bar_ve);
                    }
                    __syncwarp();
                };
                if (!mbar_wait_warp(bar_kf + 8 * kb, (nk >> 1) & 1, kWaitLimit) ||
                    !mbar_wait_warp(bar_qf + 8 * s, ph, kWaitLimit)) {
                    report(p.err, 0x1201);
                    okl = 0;
                } else {
                    tc_fence_after();
                    issue_s(dQ0 + (uint64_t)s * kStage);
                    if (!mbar_wait_warp(bar_vf, nk & 1, kWaitLimit)) {
                        report(p.err, 0x120a);
                        okl = 0;
                    } else {
                        tc_fence_after();
                        issue_dp(dDO0 + (uint64_t)s * kStage, it.ntiles == 1);
                    }
                }
                for (int t = 0; okl && t < it.ntiles; ++t) {
                    const bool wrap = (s + 1 == NQS);
                    const int s1 = wrap ? 0 : s + 1, ph1 = wrap ? ph ^ 1 : ph;  // tile t + 1
                    const uint64_t dQs = dQ0 + (uint64_t)s * kStage, dDOs = dDO0 + (uint64_t)s * kStage;
                    const uint32_t acc = t > 0 ? 1u : 0u;
                    if (!mbar_wait_warp(bar_p, go & 1, kWaitLimit)) { report(p.err, 0x1203); okl = 0; break; }
                    // dV, dK start over: the previous item's must have been read out
                    // (already implied: the row warps read them out before writing
                    // this P^T; the wait is a cheap safeguard)
                    if (t == 0 && n > 0 && !mbar_wait_warp(bar_acr, (n - 1) & 1, kWaitLimit)) {
                        report(p.err, 0x1209);
                        okl = 0;
                        break;
                    }
                    tc_fence_after();
                    if (elect_one()) {
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_ts(tmem + C_DV, tmem + C_S + packed_kcol(k), dDOs + 128 * k, idTS, k > 0 ? 1u : acc);
                    }
                    __syncwarp();
                    const bool more = t + 1 < it.ntiles;
                    if (more) {
                        if (!mbar_wait_warp(bar_qf + 8 * s1, ph1, kWaitLimit)) { report(p.err, 0x1207); okl = 0; break; }
                        tc_fence_after();
                        issue_s(dQ0 + (uint64_t)s1 * kStage);
                    }
                    if (!mbar_wait_warp(bar_ds, go & 1, kWaitLimit)) { report(p.err, 0x1204); okl = 0; break; }
                    tc_fence_after();
                    if (elect_one()) {
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_ts(tmem + C_DK, tmem + C_DP + packed_kcol(k), dQs + 128 * k, idTS, k > 0 ? 1u : acc);
                    }
                    __syncwarp();
                    const int b = go & 1;
                    if (!mbar_wait_warp(bar_dqe + 8 * b, ((go >> 1) & 1) ^ 1, kWaitLimit)) {
                        report(p.err, 0x1205);
                        okl = 0;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t cdq = b ? C_DQ1 : C_DQ0;
                    if (elect_one()) {
#pragma unroll
                        for (int k = 0; k < 8; ++k) mma_ss(tmem + cdq, dDS + 128 * k, dK + 128 * k, idDQ, k > 0);
                        mma_commit(bar_dqf + 8 * b);
                    }
                    __syncwarp();
                    if (more) issue_dp(dDO0 + (uint64_t)s1 * kStage, t + 2 == it.ntiles);
                    if (elect_one()) mma_commit(bar_qe + 8 * s);
                    __syncwarp();
                    s = s1;
                    ph = ph1;
                    ++go;
                }
                if (okl) {
                    if (elect_one()) {
                        mma_commit(bar_acc);
                        mma_commit(bar_ke + 8 * kb);
                    }
                    __syncwarp();
                }
                ++nk;
            } else {
                for (int t = 0; okl && t < it.ntiles; ++t) {
                    const bool wrap = (s + 1 == NQS);
                    const int s1 = wrap ? 0 : s + 1, ph1 = wrap ? ph ^ 1 : ph;
                    const uint64_t dDOs = dDO0 + (uint64_t)s * kStage;
                    const uint32_t acc = t > 0 ? 1u : 0u;
                    if (!mbar_wait_warp(bar_qf + 8 * s, ph, kWaitLimit)) { report(p.err, 0x1202); okl = 0; break; }
                    if (!mbar_wait_warp(bar_pb + 8 * (gr & 1), (gr >> 1) & 1, kWaitLimit)) {
                        report(p.err, 0x1206);
                        okl = 0;
                        break;
                    }
                    if (t == 0 && n > 0 && !mbar_wait_warp(bar_acr, (n - 1) & 1, kWaitLimit)) {
                        report(p.err, 0x1209);
                        okl = 0;
                        break;
                    }
                    tc_fence_after();
                    // W of this tile sits in buffer gr & 1 (the S^T or the dP^T
                    // columns, both unused by a replaced head): hi, then lo
                    const uint32_t wcol = C_S + 128 * (gr & 1);
                    if (elect_one()) {
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_ts(tmem + C_DV, tmem + wcol + 8 * k, dDOs + 128 * k, idTS, k > 0 ? 1u : acc);
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            mma_ts(tmem + C_DV, tmem + wcol + 64 + 8 * k, dDOs + 128 * k, idTS, 1u);
                        mma_commit(bar_wb + 8 * (gr & 1));
                        mma_commit(bar_qe + 8 * s);
                    }
                    __syncwarp();
                    s = s1;
                    ph = ph1;
                    ++gr;
                }
                if (okl) {
                    if (elect_one()) mma_commit(bar_acc);
                    __syncwarp();
                }
            }
            ok = okl != 0;  // the same in every lane
        }
    } else if (warp < 10) {
        // ------------------------------------------------ key rows
        // two warps per TMEM lane quarter: `half` 0 takes query columns 0..63,
        // half 1 columns 64..127 (all the work on a 32-column chunk is local)
        const int quarter = warp & 3;
        const int half = (warp - 2) >> 2;
        const int jl = quarter * 32 + lane;  // key within the block = TMEM lane
        const uint32_t lo = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + lo + C_S, tDP = tmem + lo + C_DP;
        const uint32_t vec1 = sb + SM_VEC1, vec2 = sb + SM_VEC2;  // shared addresses
        int s = 0, u = 0, go = 0, gr = 0;  // ring stage and pass; ordinary, replaced tiles so far
        bool ok = true;
        for (int n = 0; ok; ++n) {
            int item;
            Item it;
            ok = __all_sync(0xffffffffu, take_item(n, item, it));
            if (!ok) {
                report(p.err, 0x1306);
                break;
            }
            if (item < 0) break;
            const int j = it.J * BN + jl;
            const float aj = (it.direct && j < T) ? p.a[(size_t)it.h * T + j] : kNegInf;
            for (int t = 0; t < it.ntiles; ++t) {
                const int I = it.J + t;
                ok = __all_sync(0xffffffffu, mbar_wait(bar_qf + 8 * s, u & 1, kWaitLimit));
                if (!ok) { report(p.err, 0x1301); break; }
                const uint32_t v1 = vec1 + 512 * s;
                if (!it.rep) {
                    const uint32_t v2 = vec2 + 512 * s;
                    ok = __all_sync(0xffffffffu, mbar_wait(bar_s, go & 1, kWaitLimit));
                    if (!ok) { report(p.err, 0x1302); break; }
                    tc_fence_after();
                    // P^T, 32 queries at a time: bf16 pairs written over the S^T
                    // columns already read (chunk c -> columns [16c, 16c + 16)).
                    // Masks only on the diagonal tile and in a ragged last key
                    // block (a warp-uniform choice: the TMEM ops are collective).
                    // P^T stays in registers for dS^T: the S^T columns are reused by
                    // the next tile's S^T as soon as dV has read them.
                    uint32_t pw[2][16];
                    if (t == 0 || it.ragged)
                        p_half<true>(tS, half, v1, p.scale_log2, jl, t == 0, j < T, pw);
                    else
                        p_half<false>(tS, half, v1, p.scale_log2, jl, false, true, pw);
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar_p);
                    // dS^T = P^T o (dP^T - D), P^T from registers; dS^T goes over the
                    // dP^T columns this warp has read and, as row jl of the MN-major
                    // A operand of dQ = dS K, into shared memory
                    ok = __all_sync(0xffffffffu, mbar_wait(bar_dp, go & 1, kWaitLimit));
                    if (!ok) { report(p.err, 0x1303); break; }
                    tc_fence_after();
                    if (t == 0 && p.tma_grads) {  // this warp's last dK/dV box has been read
                        if (lane == 0) bulk_wait_read0();
                        __syncwarp();
                    }
                    // 16 queries per step, the TMEM load of the next step in flight
                    uint32_t va[16], vb[16];
                    tmem_ld16(tDP + 64 * half, va);
                    tmem_wait_ld();
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int c = 2 * half + cc;
                        uint32_t dsw[16];
#pragma unroll
                        for (int k2 = 0; k2 < 2; ++k2) {
                            const int k = 2 * cc + k2;
                            uint32_t(&cur)[16] = (k & 1) ? vb : va;
                            uint32_t(&nxt)[16] = (k & 1) ? va : vb;
                            if (k < 3) tmem_ld16(tDP + 64 * half + 16 * (k + 1), nxt);
                            uint64_t d2[8];
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                ld_shared_2x64(v2 + 4 * (64 * half + 16 * k) + 16 * q, d2[2 * q], d2[2 * q + 1]);
#pragma unroll
                            for (int e = 0; e < 16; e += 2) {
                                // (dP - D) paired, times P (bf16, widened), one rounding
                                const float2 pf = unpack_bf16x2(pw[cc][8 * k2 + e / 2]);
                                const uint64_t g =
                                    sub_f32x2(f32x2(__uint_as_float(cur[e]), __uint_as_float(cur[e + 1])), d2[e / 2]);
                                const float2 ds = split_f32x2(mul_f32x2(f32x2(pf.x, pf.y), g));
                                dsw[8 * k2 + e / 2] = pack_bf16x2(ds.x, ds.y);
                            }
                            if (k < 3) tmem_wait_ld();
                        }
                        tmem_st16(tDP + packed_col(c), dsw);
                        // queries [64 half, 64 half + 64) form the MN atom `half`
                        const uint32_t blk = sb + SM_DS + half * 16384 + (jl >> 3) * 1024 + (jl & 7) * 128;
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const int ch = cc * 4 + q4;
                            st_shared_v4(blk + ((ch ^ (jl & 7)) << 4), dsw[4 * q4], dsw[4 * q4 + 1],
                                         dsw[4 * q4 + 2], dsw[4 * q4 + 3]);
                        }
                    }
                    fence_proxy_async_smem();
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar_ds);
                    ++go;
                } else {
                    // W^T(j, i) = E[i-j] r_i, hi + lo bf16, into buffer gr & 1; that
                    // buffer was last read by the MMAs of replaced tile gr - 2 (one
                    // barrier per buffer, so neither can run two phases ahead of this
                    // wait); MMAs of any ordinary item in between finished before this
                    // item started (its dK, dV read-out waited for them)
                    const uint32_t tW = tmem + lo + C_S + 128 * (gr & 1);
                    if (gr >= 2) {
                        ok = __all_sync(0xffffffffu,
                                        mbar_wait(bar_wb + 8 * (gr & 1), ((gr >> 1) & 1) ^ 1, kWaitLimit));
                        if (!ok) { report(p.err, 0x1304); break; }
                    }
                    tc_fence_after();
                    if (!it.direct) {
                        const float* ef = p.w.ef + (size_t)it.slot * p.w.Lp + 128 + (I - it.J) * BM - jl;
                        // the 64 entries this thread reads lie inside the slot's padded array
                        [[maybe_unused]] const int e_lo = 128 + (I - it.J) * BM - jl + 64 * half;
                        const bool win_ok = SAF_CHECKED_OK(p.err, e_lo >= 0 && e_lo + 64 <= p.w.Lp, 0x9204u);
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            const int c = 2 * half + cc;
                            uint32_t hw[16], lw[16];
#pragma unroll
                            for (int e = 0; e < 32; e += 4) {
                                const int ql = 32 * c + e;
                                const float4 r4 = ld_shared_f4(v1 + 4 * ql);
                                const float rr[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
                                for (int u = 0; u < 4; u += 2) {
                                    const float w0 = win_ok ? __ldg(ef + ql + u) * rr[u] : 0.f;
                                    const float w1 = win_ok ? __ldg(ef + ql + u + 1) * rr[u + 1] : 0.f;
                                    const uint32_t hb = pack_bf16x2(w0, w1);
                                    const float2 hf = unpack_bf16x2(hb);
                                    hw[(e + u) / 2] = hb;
                                    lw[(e + u) / 2] = pack_bf16x2(w0 - hf.x, w1 - hf.y);
                                }
                            }
                            tmem_st16(tW + 16 * c, hw);
                            tmem_st16(tW + 64 + 16 * c, lw);
                        }
                    } else {
                        direct_pt_half(p, it.h, T, aj, j, I * BM, half, tW);
                    }
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar_pb + 8 * (gr & 1));
                    ++gr;
                }
                if (++s == NQS) {
                    s = 0;
                    ++u;
                }
            }
            if (!ok) break;
            // the item's dK, dV: half 0 writes the dV row (times c_j for a replaced
            // head), half 1 the dK row (times 1/sqrt(d); zero for a replaced head)
            ok = __all_sync(0xffffffffu, mbar_wait(bar_acc, n & 1, kWaitLimit));
            if (!ok) {
                report(p.err, 0x1305);
                break;
            }
            tc_fence_after();
            float vals[64];
            float mul;
            if (half == 0) mul = (it.rep && !it.direct && j < T) ? p.w.cf[(size_t)it.slot * p.w.Tp + j] : 1.f;
            else mul = it.rep ? 0.f : p.scale;
            const uint32_t col = half == 0 ? C_DV : C_DK;
            // a replaced head's dK columns were never written by this item (TMEM
            // holds whatever came before): its rows are zeros, not 0 x that
            const bool zero = half == 1 && it.rep;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + lo + col + 32 * c, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) vals[32 * c + e] = zero ? 0.f : __uint_as_float(v[e]) * mul;
            }
            tc_fence_before();
            mbar_arrive_warp(bar_acr);
            if (p.tma_grads) {
                // bf16: the warp's 32 rows as one TMA box, staged in the warp's own
                // 4 KB of the dS^T area (row `lane`, 16-byte chunks in the 128-byte
                // swizzle of the store map), where this warp alone writes its dS^T
                // rows.  The area is idle here: the item's last dQ MMA, its last
                // reader, completed before bar_acc.  The warp moves on once the
                // store is issued; 32 per-thread row stores instead block its next
                // shared-memory and barrier operations for thousands of cycles.
                const uint32_t box = sb + SM_DS + half * 16384 + quarter * 4096;
                if (lane == 0) bulk_wait_read0();  // the previous box has been read
                __syncwarp();
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    st_shared_v4(box + lane * 128 + ((k ^ (lane & 7)) << 4), pack_bf16x2(vals[8 * k], vals[8 * k + 1]),
                                 pack_bf16x2(vals[8 * k + 2], vals[8 * k + 3]),
                                 pack_bf16x2(vals[8 * k + 4], vals[8 * k + 5]),
                                 pack_bf16x2(vals[8 * k + 6], vals[8 * k + 7]));
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(half == 0 ? &tmDV : &tmDK, box, 0, it.J * BN + quarter * 32, it.bh);
                    bulk_commit();
                }
            } else if (j < T) {
                store_row(half == 0 ? p.dv : p.dk, p.grad_fp32, (size_t)it.bh * T + j, vals);
            }
        }
        if (lane == 0) bulk_wait0();  // the dK/dV stores complete before the CTA ends
    } else {
        // ------------------------------------------------ dQ tiles -> global accumulator
        // Each warp moves its own 32 query rows: TMEM -> two 4 KB swizzled boxes
        // of its own (columns 0..31, 32..63) -> TMA reduce-add (no cross-warp sync).
        const int quarter = warp & 3;
        const int ql = quarter * 32 + lane;
        const uint32_t lo = (uint32_t)(quarter * 32) << 16;
        const uint32_t box = sb + SM_DQ + quarter * 8192;
        const uint32_t stg = box + lane * 128;
        int go = 0;
        bool ok = true;
        for (int n = 0; ok; ++n) {
            int item;
            Item it;
            ok = __all_sync(0xffffffffu, take_item(n, item, it));
            if (!ok) {
                report(p.err, 0x1402);
                break;
            }
            if (item < 0) break;
            if (it.rep) continue;  // a replaced head adds nothing to dQ
            for (int t = 0; t < it.ntiles; ++t, ++go) {
                const int I = it.J + t, b = go & 1;
                ok = __all_sync(0xffffffffu, mbar_wait(bar_dqf + 8 * b, (go >> 1) & 1, kWaitLimit));
                if (!ok) { report(p.err, 0x1401); break; }
                tc_fence_after();
                uint32_t v0[32], v1[32];
                tmem_ld32(tmem + lo + (b ? C_DQ1 : C_DQ0), v0);
                tmem_ld32(tmem + lo + (b ? C_DQ1 : C_DQ0) + 32, v1);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(bar_dqe + 8 * b);
                // the boxes must have been read by the previous tile's reduces
                if (lane == 0) bulk_wait_read0();
                __syncwarp();
                // row `lane` of each [32][32] fp32 box, 16-byte chunks XOR-swizzled
                // by row (the reduce map's 128-byte swizzle; conflict-free stores)
#pragma unroll
                for (int c4 = 0; c4 < 8; ++c4) {
                    const uint32_t off = (uint32_t)((c4 ^ (ql & 7)) << 4);
                    st_shared_v4(stg + off, v0[4 * c4], v0[4 * c4 + 1], v0[4 * c4 + 2], v0[4 * c4 + 3]);
                    st_shared_v4(stg + 4096 + off, v1[4 * c4], v1[4 * c4 + 1], v1[4 * c4 + 2], v1[4 * c4 + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_reduce_add_3d(&tmDQ, box, 0, I * BM + quarter * 32, it.bh);
                    tma_reduce_add_3d(&tmDQ, box + 4096, 32, I * BM + quarter * 32, it.bh);
                    bulk_commit();
                }
            }
        }
        if (lane == 0) bulk_wait0();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
    // the last CTA to finish resets the work counters for the next launch
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(p.err + kCtrBwdDone, 1u) == gridDim.x - 1) {
            atomicExch(p.err + kCtrBwdNext, 0u);
            atomicExch(p.err + kCtrBwdDone, 0u);
        }
    }
}

// Shared K/V (Hkv < H): dK[b, g] = sum over the H / Hkv query heads h of group
// g of the per-query-head fp32 rows, written in the output dtype (the
// gradient of a shared input is the sum of its uses).  Four floats a thread.
__global__ void __launch_bounds__(256) group_sum_kernel(const float* __restrict__ src, void* __restrict__ dst,
                                                        int B, int H, int Hkv, int64_t rows_T, int grad_fp32) {
    const int G = H / Hkv;
    const int64_t per_head = rows_T * (kHeadDim / 4);  // float4s of one [T, 64] slice
    const int64_t n = (int64_t)B * Hkv * per_head;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t bg = idx / per_head, off = idx - bg * per_head;
        const int64_t b = bg / Hkv, g = bg - b * Hkv;
        const float4* s0 = reinterpret_cast<const float4*>(src) + ((b * H + g * G) * per_head + off);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int u = 0; u < G; ++u) {
            const float4 x = s0[(int64_t)u * per_head];
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
        if (grad_fp32) {
            reinterpret_cast<float4*>(dst)[idx] = acc;
        } else {
            uint2 o;
            o.x = pack_bf16x2(acc.x, acc.y);
            o.y = pack_bf16x2(acc.z, acc.w);
            reinterpret_cast<uint2*>(dst)[idx] = o;
        }
    }
}

__global__ void __launch_bounds__(256) dq_convert_kernel(const float* __restrict__ acc, void* __restrict__ dq,
                                                         int64_t n4, int grad_fp32, float scale) {
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n4;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const float4 a = reinterpret_cast<const float4*>(acc)[idx];
        if (grad_fp32) {
            reinterpret_cast<float4*>(dq)[idx] = make_float4(a.x * scale, a.y * scale, a.z * scale, a.w * scale);
        } else {
            reinterpret_cast<uint2*>(dq)[idx] =
                make_uint2(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale));
        }
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

}  // namespace

// [BH, T, 64] fp32 as a 3-D tensor (d, t, bh); 32 x 32 boxes (32 rows of 128
// bytes) with the 128-byte swizzle.
bool make_tmap_bhtd_f32(const void* base, int BH, int T, CUtensorMap* out) {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    if (!fn) return false;
    cuuint64_t dims[3] = {64, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {64 * 4, (cuuint64_t)T * 64 * 4};
    cuuint32_t box[3] = {32, 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_dq_convert(const float* dqacc, void* dq, int64_t rows, int grad_fp32, cudaStream_t stream) {
    const int64_t n4 = rows * kHeadDim / 4;
    if (n4 == 0) return cudaSuccess;
    const int64_t blocks = (n4 + 255) / 256;
    launch_begin(KID_DQ_CONVERT, stream);
    dq_convert_kernel<<<(unsigned)(blocks < 148 * 16 ? blocks : 148 * 16), 256, 0, stream>>>(dqacc, dq, n4,
                                                                                            grad_fp32, 0.125f);
    launch_end(KID_DQ_CONVERT, stream);
    return cudaGetLastError();
}

cudaError_t launch_group_sum(const float* src, void* dst, int B, int H, int Hkv, int T, int grad_fp32,
                             cudaStream_t stream) {
    const int64_t n4 = (int64_t)B * Hkv * T * (kHeadDim / 4);
    if (n4 == 0) return cudaSuccess;
    const int64_t blocks = (n4 + 255) / 256;
    launch_begin(KID_GROUP_SUM, stream);
    group_sum_kernel<<<(unsigned)(blocks < 148 * 16 ? blocks : 148 * 16), 256, 0, stream>>>(src, dst, B, H, Hkv,
                                                                                          (int64_t)T, grad_fp32);
    launch_end(KID_GROUP_SUM, stream);
    return cudaGetLastError();
}

cudaError_t launch_bwd_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                          const __nv_bfloat16* dout, const float* nlse2p, const float* dvecp, float* dqacc,
                          const float* a, const float* r, const float* logz, const HeadList& hl,
                          const ReplacedWs& w, int B, int H, int Hkv, int T, void* dk, void* dv, int grad_fp32,
                          unsigned int* err, cudaStream_t stream) {
    const int BH = B * H;
    CUtensorMap mq, mk, mv, mdo, mdq, mdk, mdv;
    if (!make_tmap_bhtd(q, BH, T, &mq) || !make_tmap_bhtd(k, B * Hkv, T, &mk) ||
        !make_tmap_bhtd(v, B * Hkv, T, &mv) ||
        !make_tmap_bhtd(dout, BH, T, &mdo) || !make_tmap_bhtd_f32(dqacc, BH, T, &mdq))
        return cudaErrorNotSupported;
    // bf16 dK, dV [BH, T, 64] by 32-row TMA stores when their maps encode (a
    // base the encoder rejects, e.g. not 16-byte aligned, takes the row stores)
    const bool tma_grads = !grad_fp32 && make_tmap_bhtd(dk, BH, T, &mdk, 32) && make_tmap_bhtd(dv, BH, T, &mdv, 32);
    if (!tma_grads) mdk = mdv = mq;  // not read
    BwdTcParams p;
    p.nlse2p = nlse2p;
    p.dvecp = dvecp;
    p.a = a;
    p.r = r;
    p.logz = logz;
    p.w = w;
    p.dk = dk;
    p.dv = dv;
    p.err = err;
    int slot = 0;
    for (int hh = 0; hh < kMaxHeads; ++hh) p.slot_of_head[hh] = -1;
    for (int hh = 0; hh < H; ++hh)
        if (hl.replaced[hh]) p.slot_of_head[hh] = (int16_t)(slot++);
    p.nslots = slot;
    p.H = H;
    p.Hkv = Hkv;
    p.BH = BH;
    p.T = T;
    p.Tp = round_up128(T);
    p.nqb = (T + BM - 1) / BM;
    if ((int64_t)BH * p.nqb >= (int64_t)1 << 30) return cudaErrorNotSupported;  // item words hold 30 bits
    p.grad_fp32 = grad_fp32;
    p.tma_grads = tma_grads ? 1 : 0;
    p.scale = 0.125f;
    p.scale_log2 = kLog2e * 0.125f;
    const int smem = SM_TOTAL + 1024;
    cudaError_t e = cudaFuncSetAttribute(bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM (TMEM and shared memory allow one), at most one per item
    const int items = BH * p.nqb;
    const int grid = items < sm_count() ? items : sm_count();
    launch_begin(KID_BWD_TC, stream);
    bwd_tc_kernel<<<dim3((unsigned)grid), NTHREADS, smem, stream>>>(mq, mk, mv, mdo, mdq, mdk, mdv, p);
    launch_end(KID_BWD_TC, stream);
    return cudaGetLastError();
}

}  // namespace saf
