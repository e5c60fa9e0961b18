// Mixed-head causal attention forward on the 5th-generation tensor cores
// (tcgen05, accumulators in TMEM, operands staged by TMA).
//
// A work item is one 128-row query block of one (batch, head) slice; both
// head kinds share the item stream.  The kernel is persistent: two CTAs per SM
// pull items from a counter in the workspace header (reset by the last CTA),
// in groups of slices with the longest rows first inside a group.  Warp roles:
//   warp 0      TMA producer: work items (decoded, through a two-slot ring);
//               Q per item (two buffers: this item and the next), then K and
//               V tiles of 128 keys through separate rings (2 K stages, 2 V
//               stages), K one block ahead of V (K is skipped for replaced
//               heads, whose blocks' W inputs come through a two-stage ring)
//   warp 1      TMEM owner and MMA issuer (one elected lane)
//   warps 2..5  one query row per thread: softmax / pattern builder, epilogue
//
// Ordinary head, per key block j (FlashAttention-style online softmax, the
// "FlashAttention-2 online softmax tile" of the reading notes, section 二.4):
//   S = Q K_j^T             tcgen05 SS MMA, 128x128, fp32 in TMEM
//   P = exp2(S*log2e/sqrt(d) - m), row max m kept lazily (the O rescale is
//       skipped unless m grows by more than 8 in log2 units), P as bf16 into TMEM
//   O += P V_j              tcgen05 TS MMA (A = P from TMEM), fp32 in TMEM
// The row threads copy S_j to registers and release its TMEM columns at once,
// so the MMA warp issues S_{j+1} while they still work on block j; the MMA
// order is S_0, S_1, PV_0, S_2, PV_1, ...
// Replaced head (Eq. (3), section 二.3, in factored form): the tile
//   W(i,j) = E[i-j] c_j     (bf16 pairs multiplied in registers, no exp)
// is written to TMEM and O += W V_j; a second MMA against a tile of ones
// accumulates the row sums of the same bf16 W, and the epilogue divides row i
// by its sum.  Eq. (3) gives W(i,j) / sum_j W(i,j) = exp(a[j] + r[i-j] - log Z(i))
// (the factors E, c and r_i cancel), so
//   O_i = sum_j exp(a[j] + r[i-j] - log Z(i)) V_j,
// and normalising by the sum of the rounded weights, as an ordinary head
// normalises by the sum of its probabilities, reproduces a dominant term's V
// exactly instead of scaling it by the rounding of its weight.
// A replaced head whose factors would leave fp32 range (flag set by the prep
// kernel) takes the pattern itself, one exp per element, in the same slot.
// Causal tile skipping: key blocks past the diagonal are never visited; the
// diagonal block is masked (ordinary) or zero by construction (E[d<0] = 0).
#include <algorithm>

#include "saf_common.cuh"
#include "tc_util.cuh"

namespace saf {
namespace {

using namespace tc;

constexpr int BM = 128;          // query rows per CTA
constexpr int BN = 128;          // keys per block
constexpr int NSK = 2;           // K ring stages
constexpr int NSV = 2;           // V ring stages
constexpr int NTHREADS = 192;
constexpr uint32_t TILE_BYTES = 128 * 64 * 2;  // one 128 x 64 bf16 tile
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t TS_COL = 0, TO_COL = 128, TP_COL = 192;  // S, O, P regions
// replaced heads: row sums of W in the (then unused) P columns 192..207
constexpr uint32_t TSUM_COL = TP_COL;
constexpr long long kWaitLimit = 1ll << 31;                 // cycles

// shared memory map (offsets from a 1024-aligned base)
constexpr uint32_t SM_Q = 0;
constexpr uint32_t SM_K = SM_Q + 2 * TILE_BYTES;  // Q: two buffers (this item, next item)
constexpr uint32_t SM_V = SM_K + NSK * TILE_BYTES;
// 16 rows x 128 bytes of bf16 ones: the B operand (N = 16, K-major) of the
// row-sum MMA of replaced heads (every element is 1, so each 16-key step
// reads the same atom)
constexpr uint32_t SM_ONES = SM_V + NSV * TILE_BYTES;
constexpr uint32_t SM_BAR = SM_ONES + 2048;
// replaced heads: what block g's W is built from, in stage g & 1: the 256 E
// pairs [128 (I - j), + 256) of the padded array (1 KB), then the 64 c pairs
// of the key block (256 B)
constexpr uint32_t WST_E = 1024, WST_BYTES = 1280;
constexpr uint32_t SM_WST = SM_BAR + 512;  // (SM_BAR + 256: the two work-item slots, 16 bytes each)
// O staging: per row warp a 2 KB box (its 32 rows x 32 columns of bf16, the
// 64-byte swizzle of the store map), stored to global by TMA twice per item
constexpr uint32_t SM_OST = (SM_WST + 2 * WST_BYTES + 1023) & ~1023u;
constexpr uint32_t SM_TOTAL = SM_OST + 4 * 2048;

struct FwdTcParams {
    __nv_bfloat16* o;
    float* lse;
    const float* a;  // [H, T] pattern vectors (read for flag-1 replaced heads only)
    const float* r;
    const float* logz;
    ReplacedWs w;
    unsigned int* err;
    int16_t slot_of_head[kMaxHeads];
    int H, Hkv, BH, T, nqb;  // query heads, K/V heads (H / Hkv query heads share one)
    int nslots;  // replaced heads
    int tma_o;   // O written by TMA stores of 32 x 32 boxes (else per-thread row stores)
    float scale_log2;
};

__device__ __forceinline__ void report(unsigned int* err, unsigned int code) {
    atomicOr(err, 1u);
    atomicCAS(err + 1, 0u, code);
}

// The 128 raw scores of this thread's row of S, TMEM -> registers.
__device__ __forceinline__ void load_s_row(uint32_t tS, uint32_t (&v)[128]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
    tmem_wait_ld();
}

// Row max of one 128-key block of raw scores.  Three-input max, four
// independent chains.
__device__ __forceinline__ float row_max(const uint32_t (&v)[128]) {
    float mx[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
#pragma unroll
    for (int e = 0; e < 128; e += 2)
        mx[(e >> 1) & 3] = max3(mx[(e >> 1) & 3], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
    return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
}

// P = exp2(s * scale - m) for keys [32 Q, 32 Q + 32) of the block (Q = 0..3)
// as 16 bf16 pairs; the (unrounded) probabilities are added to the paired
// sums l2.  The scale-and-shift (sc2 = scale, nm2 = -m, paired) and the sums
// use the paired fp32 instructions (same rounding as the scalar ones).
template <int Q>
__device__ __forceinline__ void exp_quarter(const uint32_t (&v)[128], uint64_t sc2, uint64_t nm2, uint64_t (&l2)[4],
                                            uint32_t (&pw)[16]) {
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        const float2 x = split_f32x2(
            fma_f32x2(f32x2(__uint_as_float(v[32 * Q + e]), __uint_as_float(v[32 * Q + e + 1])), sc2, nm2));
        const float p0 = ex2(x.x), p1 = ex2(x.y);
        l2[(e >> 1) & 3] = add_f32x2(l2[(e >> 1) & 3], f32x2(p0, p1));
        pw[e >> 1] = pack_bf16x2(p0, p1);
    }
}

// Rescales this warp's 32 O rows by f (a whole-warp TMEM round trip, taken
// when any row of the warp needs it).
__device__ __forceinline__ void rescale_o(uint32_t tO, float f) {
    if (__any_sync(0xffffffffu, f != 1.f)) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint32_t ov[32];
            tmem_ld32(tO + 32 * c, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * f);
            tmem_st32(tO + 32 * c, ov);
        }
    }
}

// The running max m moves only when a block's max mx exceeds it by more than
// 8 (log2 units), so P stays below 2^8 and O is rarely rescaled; returns the
// factor f for l and O (1 when m stays).
__device__ __forceinline__ float update_max(float mx, float& m, float& l) {
    float f = 1.f;
    if (m == kNegInf) {
        m = mx;
    } else if (mx > m + 8.f) {
        f = ex2(m - mx);
        l *= f;
        m = mx;
    }
    return f;
}

// The diagonal block of an item (query block I, key block I; key e and row r
// counted from the same start, BN = BM) keeps key e of row r when e <= r.  It
// runs once per item, so its code is short and out of line (loops over
// 32-key chunks, S read from TMEM in each pass) where the other blocks' is
// unrolled: a cold unrolled copy, fetched once per item, costs several times
// its arithmetic.  Rows of lane quarter q see every key of chunks c < q, part
// of chunk q and none past it.  No key of a stored row lies past T
// (key <= row < T); rows past T see zero-filled keys.  S stays in TMEM until
// P is handed over (the next S, the next item's first, is issued after this
// block's P.V).  Waits for P.V_{j-1} (parity o_par) unless j = 0, rescales O,
// writes P (zeros past the row) to the P columns; m and l in ml (x, y) are
// updated.  False when the wait gave up.
__device__ __noinline__ bool diag_block(uint32_t tS, uint32_t tO, uint32_t tP, int quarter, int row, float scale,
                                        bool first, uint32_t bar_o, uint32_t o_par, float2& ml) {
    float m = ml.x, l = ml.y;
    float mx2[2] = {kNegInf, kNegInf};
#pragma unroll 1
    for (int c = 0; c <= quarter; ++c) {
        uint32_t v[32];
        tmem_ld32(tS + 32 * c, v);
        tmem_wait_ld();
        const int lim = row - 32 * c;
#pragma unroll
        for (int e = 0; e < 32; e += 2)
            mx2[(e >> 1) & 1] = max3(mx2[(e >> 1) & 1], e > lim ? kNegInf : __uint_as_float(v[e]),
                                     e + 1 > lim ? kNegInf : __uint_as_float(v[e + 1]));
    }
    const float f = update_max(fmaxf(mx2[0], mx2[1]) * scale, m, l);
    if (!first) {
        if (!__all_sync(0xffffffffu, mbar_wait(bar_o, o_par, kWaitLimit))) return false;
        tc_fence_after();
    }
    rescale_o(tO, f);
    const uint64_t sc2 = f32x2(scale, scale), nm2 = f32x2(-m, -m);
    uint64_t l2[2] = {0, 0};
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        uint32_t pw[16];
        if (c <= quarter) {
            uint32_t v[32];
            tmem_ld32(tS + 32 * c, v);
            tmem_wait_ld();
            const int lim = row - 32 * c;
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                const float2 x =
                    split_f32x2(fma_f32x2(f32x2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), sc2, nm2));
                const float p0 = e > lim ? 0.f : ex2(x.x), p1 = e + 1 > lim ? 0.f : ex2(x.y);
                l2[(e >> 1) & 1] = add_f32x2(l2[(e >> 1) & 1], f32x2(p0, p1));
                pw[e >> 1] = pack_bf16x2(p0, p1);
            }
        } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) pw[e] = 0u;
        }
        tmem_st16(tP + 16 * c, pw);
    }
    const float2 a = split_f32x2(add_f32x2(l2[0], l2[1]));
    ml = make_float2(m, l + (a.x + a.y));
    return true;
}

// W(i, j) = E[i-j] c_j for 64 keys (q0 = 0 or 8 selects the half): bf16 pair
// products of the E pairs (walking down from row i; shared address e_row)
// and the c pairs (shared address c0), both staged in shared memory.
__device__ __forceinline__ void build_w_half(uint32_t e_row, uint32_t c0, int q0, uint32_t (&pw)[32]) {
#pragma unroll
    for (int q4 = 0; q4 < 8; ++q4) {
        const uint4 c4 = ld_shared_u4(c0 + 16 * (q0 + q4));
        const uint32_t cw[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int mm = 4 * (q0 + q4) + u;  // key pair (2mm, 2mm+1)
            const uint32_t e2 = ld_shared_u32(e_row - 8 * mm);
            __nv_bfloat162 prod = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&e2),
                                          *reinterpret_cast<const __nv_bfloat162*>(&cw[u]));
            pw[4 * q4 + u] = *reinterpret_cast<uint32_t*>(&prod);
        }
    }
}

// A replaced head whose factored form would leave fp32 range: row i of the
// pattern for keys [k0, k0 + 128) straight from Eq. (3), one exp per element,
// P = exp(a[k] + r[i-k] - log Z(i)) (0 past the row, past T, or where log Z is
// -inf), as 64 bf16 pairs stored to the W buffer at tW; the epilogue then
// needs no row scale.  Kept out of line: the path is rare.
__device__ __noinline__ void direct_p_row(const float* ah, const float* rh, const float* logz, int h, int T, int i,
                                          int k0, uint32_t tW) {
    const float lz = i < T ? logz[(size_t)h * T + i] : kNegInf;
    const bool row_ok = lz != kNegInf;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        uint32_t pw[32];
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
            float pr[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int k = k0 + 64 * c + e + u;
                pr[u] = (row_ok && k <= i && k < T) ? ex2((__ldg(ah + k) + __ldg(rh + (i - k)) - lz) * kLog2e) : 0.f;
            }
            pw[e >> 1] = pack_bf16x2(pr[0], pr[1]);
        }
        tmem_st32(tW + 32 * c, pw);
    }
}

// Whether replaced slot s takes the per-element path: any of its tiles' range
// flags (a warp-wide OR).  Out of line: it runs once per replaced item and
// keeps its registers out of the row loop's allocation.
__device__ __noinline__ bool head_direct(const ReplacedWs& w, int s) {
    int any = 0;
    for (int t = threadIdx.x & 31; t < w.ntiles; t += 32) any |= w.tflag[(size_t)s * w.ntiles + t];
    return __any_sync(0xffffffffu, any != 0);
}

__global__ void __launch_bounds__(NTHREADS, 2)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
              const FwdTcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t bar_itf = sbase + SM_BAR;      // [2] work item slot full
    const uint32_t bar_ite = bar_itf + 16;        // [2] work item slot read (5 arrivals)
    const uint32_t bar_qf = bar_ite + 16;         // [2] Q buffer full
    const uint32_t bar_qe = bar_qf + 16;          // [2] Q buffer free (last S MMA of its item done)
    const uint32_t bar_kf = bar_qe + 16;          // [NSK] K stage full
    const uint32_t bar_ke = bar_kf + 8 * NSK;     // [NSK] K stage free (S MMA done)
    const uint32_t bar_vf = bar_ke + 8 * NSK;     // [NSV] V stage full
    const uint32_t bar_ve = bar_vf + 8 * NSV;     // [NSV] V stage free (P.V MMA done)
    const uint32_t bar_s = bar_ve + 8 * NSV;      // S ready
    const uint32_t bar_sf = bar_s + 8;            // S copied out by the rows (4 warp arrivals)
    const uint32_t bar_p = bar_sf + 8;            // P written (4 warp arrivals)
    const uint32_t bar_o = bar_p + 8;             // P.V done (ordinary head)
    const uint32_t bar_ob = bar_o + 8;            // [2] P.V of W buffer b done (replaced head)
    const uint32_t bar_pb = bar_ob + 16;          // [2] W buffer b written (replaced head, 4 warp arrivals)
    const uint32_t bar_wf = bar_pb + 16;          // [2] W inputs of stage b landed (replaced head)
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SM_BAR + 232);
    // [2] work item n & 1, decoded by the producer: {item (-1: none left), bh, I, h}
    const uint32_t item_slot = sbase + SM_BAR + 256;
    static_assert(16 * 4 + 16 * NSK + 16 * NSV + 32 + 48 <= 232, "barrier area");

    const int T = p.T;
    const int total = p.BH * p.nqb;  // work items: one query block of one (b, h) slice
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_itf + 8 * b, 1);
            mbar_init(bar_ite + 8 * b, 5);
            mbar_init(bar_qf + 8 * b, 1);
            mbar_init(bar_qe + 8 * b, 1);
            mbar_init(bar_ob + 8 * b, 1);
            mbar_init(bar_pb + 8 * b, 4);
            mbar_init(bar_wf + 8 * b, 1);
        }
        for (int s = 0; s < NSK; ++s) {
            mbar_init(bar_kf + 8 * s, 1);
            mbar_init(bar_ke + 8 * s, 1);
        }
        for (int s = 0; s < NSV; ++s) {
            mbar_init(bar_vf + 8 * s, 1);
            mbar_init(bar_ve + 8 * s, 1);
        }
        mbar_init(bar_s, 1);
        mbar_init(bar_sf, 4);
        mbar_init(bar_p, 4);
        mbar_init(bar_o, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_holder), TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0) {  // the ones tile (2 KB), 64 bytes per lane of the producer warp
        const uint32_t one2 = 0x3F803F80u;  // two bf16 1.0
#pragma unroll
        for (int u = 0; u < 4; ++u) st_shared_v4(sbase + SM_ONES + (u * 32 + lane) * 16, one2, one2, one2, one2);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    // (b, h) slice and query block of an item, grouped longest-first order
    // (query block I visits I + 1 key blocks)
    struct Item {
        int bh, bhkv, I, h, slot;  // query slice, its K/V slice, query block, head, replaced slot
        bool rep;
    };
    auto decode = [&](int item) {
        Item it;
        int rank;
        grouped_order((unsigned)item, p.BH, p.nqb, it.bh, rank);
        it.I = p.nqb - 1 - rank;
        it.h = it.bh % p.H;
        it.bhkv = (it.bh / p.H) * p.Hkv + it.h / (p.H / p.Hkv);
        it.slot = p.slot_of_head[it.h];
        it.rep = it.slot >= 0;
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
        it.I = (int)w.z;
        it.h = (int)w.w;
        it.bhkv = -1;  // the producer's alone
        it.slot = item >= 0 ? p.slot_of_head[it.h] : -1;
        it.rep = it.slot >= 0;
        return true;
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            int gk = 0, gv = 0, gr = 0, nq = 0;  // K, V, replaced blocks; ordinary items so far
            bool ok = true, waited = false;
            for (int n = 0; ok; ++n) {
                const int w = (int)atomicAdd(p.err + kCtrFwdNext, 1u);
                const int item = w < total ? w : -1;
                const Item it = item >= 0 ? decode(item) : Item{0, 0, 0, 0, -1, false};
                if (item >= 0 && !SAF_CHECKED_OK(p.err,
                                                 it.bh >= 0 && it.bh < p.BH && it.I >= 0 && it.I < p.nqb && it.h >= 0 &&
                                                     it.h < p.H && it.slot < p.nslots,
                                                 0x9101u)) {
                    ok = false;
                    break;
                }
                if (!mbar_wait(bar_ite + 8 * (n & 1), ((n >> 1) & 1) ^ 1, kWaitLimit)) { ok = false; break; }
                st_shared_v4(item_slot + 16 * (n & 1), (uint32_t)item, (uint32_t)it.bh, (uint32_t)it.I, (uint32_t)it.h);
                mbar_arrive(bar_itf + 8 * (n & 1));
                if (item < 0) break;
                const int nkb = it.I + 1;
                if (!it.rep) {
                    const int b = nq & 1;
                    if (!mbar_wait(bar_qe + 8 * b, ((nq >> 1) & 1) ^ 1, kWaitLimit)) { ok = false; break; }
                    mbar_expect_tx(bar_qf + 8 * b, TILE_BYTES);
                    tma_load_3d(sbase + SM_Q + b * TILE_BYTES, &tmQ, bar_qf + 8 * b, 0, it.I * BM, it.bh);
                    ++nq;
                }
                // K_j is consumed by S_j, which runs a block ahead of P.V_j: the
                // K loads go one block ahead of the V loads
                auto load_k = [&](int j) -> bool {
                    const int g = gk + j, s = g % NSK, u = g / NSK;
                    if (!mbar_wait(bar_ke + 8 * s, (u & 1) ^ 1, kWaitLimit)) return false;
                    mbar_expect_tx(bar_kf + 8 * s, TILE_BYTES);
                    tma_load_3d(sbase + SM_K + s * TILE_BYTES, &tmK, bar_kf + 8 * s, 0, j * BN, it.bhkv);
                    return true;
                };
                if (!it.rep && !load_k(0)) { ok = false; break; }
                for (int j = 0; j < nkb; ++j) {
                    if (!it.rep && j + 1 < nkb && !load_k(j + 1)) { ok = false; break; }
                    if (it.rep) {
                        // the W inputs of replaced block g into stage g & 1, once the
                        // rows have built block g - 2's W from it; the arrays come
                        // from the pattern preparation, which a programmatic launch
                        // may still be running: wait for it once
                        const int g = gr + j, b = g & 1;
                        if (!waited) {
                            griddep_wait();
                            waited = true;
                        }
                        if (g >= 2 && !mbar_wait(bar_pb + 8 * b, ((g >> 1) & 1) ^ 1, kWaitLimit)) { ok = false; break; }
                        const uint32_t st = sbase + SM_WST + b * WST_BYTES;
                        if (!SAF_CHECKED_OK(p.err,
                                            (size_t)(it.I - j) * BN + 256 <= (size_t)p.w.Lp &&
                                                (size_t)j * 64 + 64 <= (size_t)p.w.Tp / 2,
                                            0x9102u)) {
                            ok = false;
                            break;
                        }
                        mbar_expect_tx(bar_wf + 8 * b, WST_BYTES);
                        bulk_load(st, p.w.epair + (size_t)it.slot * p.w.Lp + (size_t)(it.I - j) * BN, WST_E, bar_wf + 8 * b);
                        bulk_load(st + WST_E, p.w.cpair + (size_t)it.slot * (p.w.Tp / 2) + (size_t)j * 64,
                                  WST_BYTES - WST_E, bar_wf + 8 * b);
                    }
                    const int g = gv + j, s = g % NSV, u = g / NSV;
                    if (!mbar_wait(bar_ve + 8 * s, (u & 1) ^ 1, kWaitLimit)) { ok = false; break; }
                    mbar_expect_tx(bar_vf + 8 * s, TILE_BYTES);
                    tma_load_3d(sbase + SM_V + s * TILE_BYTES, &tmV, bar_vf + 8 * s, 0, j * BN, it.bhkv);
                }
                if (it.rep) gr += nkb;
                else gk += nkb;
                gv += nkb;
            }
            if (!ok) report(p.err, 0x101);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        const uint32_t idS = idesc_bf16(128, 128, 0, 0);  // Q (K-major) x K (K-major)
        const uint32_t idO = idesc_bf16(128, 64, 0, 1);   // P (TMEM) x V (MN-major)
        const uint32_t idSum = idesc_bf16(128, 16, 0, 0); // W (TMEM) x ones (K-major)
        const uint64_t dOnes = sw128_desc(sbase + SM_ONES);
        // descriptors advance by stage (TILE_BYTES = TILE_BYTES / 16 units):
        // the issuing thread keeps its scalar work small, the pipe waits on it
        constexpr uint64_t kStage = TILE_BYTES >> 4;
        const uint64_t dQ0 = sw128_desc(sbase + SM_Q), dK0 = sw128_desc(sbase + SM_K);
        const uint64_t dV0 = sw128_desc(sbase + SM_V);
        int gk = 0, gv = 0, go = 0, gr = 0, nq = 0;  // K, V, ordinary, replaced blocks; ordinary items
        bool ok = true;
        for (int n = 0; ok; ++n) {
            int item;
            Item it;
            ok = __all_sync(0xffffffffu, take_item(n, item, it));
            if (!ok) { if (lane == 0) report(p.err, 0x205); break; }
            if (item < 0) break;
            const int nkb = it.I + 1;
            // The whole warp runs the schedule (its waits give one answer for
            // all lanes) and one elected lane issues each group of MMAs and their
            // commits (always the same lane, so a commit covers all its MMAs).
            {
                const int b = nq & 1;
                const uint64_t dq = dQ0 + (uint64_t)b * kStage;
                // S_j = Q K_j^T into the S columns; frees K stage j when done,
                // and the Q buffer after the item's last block
                auto issue_s = [&](int j) -> bool {
                    const int g = gk + j, s = g % NSK, u = g / NSK;
                    if (!mbar_wait_warp(bar_kf + 8 * s, u & 1, kWaitLimit)) return false;
                    tc_fence_after();
                    const uint64_t dk = dK0 + (uint64_t)s * kStage;
                    if (elect_one()) {
#pragma unroll
                        for (int k = 0; k < 4; ++k)  // K = 64 in steps of 16 (32 bytes)
                            mma_ss(tmem + TS_COL, dq + 2 * k, dk + 2 * k, idS, k > 0 ? 1u : 0u);
                        mma_commit(bar_s);
                        mma_commit(bar_ke + 8 * s);
                        if (j == nkb - 1) mma_commit(bar_qe + 8 * b);
                    }
                    __syncwarp();
                    return true;
                };
                if (!it.rep) ok = mbar_wait_warp(bar_qf + 8 * b, (nq >> 1) & 1, kWaitLimit) && issue_s(0);
                if (!ok) report(p.err, 0x201);
                for (int j = 0; ok && j < nkb; ++j) {
                    if (!it.rep && j + 1 < nkb) {
                        // S_{j+1} once the rows have copied S_j out of TMEM
                        if (!mbar_wait_warp(bar_sf, (go + j) & 1, kWaitLimit) || !issue_s(j + 1)) {
                            report(p.err, 0x202);
                            ok = false;
                            break;
                        }
                    }
                    const int g = gv + j, s = g % NSV, u = g / NSV;
                    if (!mbar_wait_warp(bar_vf + 8 * s, u & 1, kWaitLimit)) { report(p.err, 0x203); ok = false; break; }
                    const int wb = (gr + j) & 1;
                    if (!(it.rep ? mbar_wait_warp(bar_pb + 8 * wb, ((gr + j) >> 1) & 1, kWaitLimit)
                                 : mbar_wait_warp(bar_p, (go + j) & 1, kWaitLimit))) {
                        report(p.err, 0x204);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t dv = dV0 + (uint64_t)s * kStage;
                    // a replaced head's W alternates between two buffers in the S
                    // columns (unused there), so building W_{j+1} overlaps this MMA
                    const uint32_t acol = it.rep ? 64 * wb : TP_COL;
                    if (elect_one()) {
#pragma unroll
                        for (int k = 0; k < 8; ++k)  // K = 128 keys in steps of 16 (16 rows x 128 B)
                            mma_ts(tmem + TO_COL, tmem + acol + 8 * k, dv + 128 * k, idO, (j > 0 || k > 0) ? 1u : 0u);
                        if (it.rep) {
#pragma unroll
                            for (int k = 0; k < 8; ++k)  // row sums of the same W
                                mma_ts(tmem + TSUM_COL, tmem + acol + 8 * k, dOnes + 2 * (k & 3), idSum,
                                       (j > 0 || k > 0) ? 1u : 0u);
                        }
                        mma_commit(it.rep ? bar_ob + 8 * wb : bar_o);
                        mma_commit(bar_ve + 8 * s);
                    }
                    __syncwarp();
                }
            }
            if (it.rep) {
                gr += nkb;
            } else {
                gk += nkb;
                go += nkb;
                ++nq;
            }
            gv += nkb;
        }
    } else {
        // ------------------------------------------------ row threads
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;  // TMEM lane = query row within the block
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_off + TS_COL;
        const uint32_t tO = tmem + lane_off + TO_COL;
        const uint32_t tP = tmem + lane_off + TP_COL;
        int go = 0, gr = 0;  // ordinary and replaced blocks so far
        // Replaced heads read what the pattern preparation writes (the factored
        // arrays, their range flags, log Z); with a programmatic launch this
        // kernel may start before that grid ends, so the row warps wait for it
        // at their first replaced item.  A head's per-element flag (any of its
        // tiles' range flags) is read at each of its items.
        bool waited = false;
        bool ok = true;
        for (int n = 0; ok; ++n) {
            int item, I, slot, h, bh;
            bool rep, direct = false;
            {
                Item it;
                ok = __all_sync(0xffffffffu, take_item(n, item, it));
                I = it.I;
                slot = it.slot;
                h = it.h;
                bh = it.bh;
                rep = it.rep;
            }
            if (!ok) { report(p.err, 0x305); break; }
            if (item < 0) break;
            if (rep) {
                if (!waited) {
                    griddep_wait();
                    waited = true;
                }
                direct = head_direct(p.w, slot);  // per-element exps instead of the factored form
            }
            const int nkb = I + 1;
            const int i = I * BM + row;
            float m = kNegInf, l = 0.f;
            for (int j = 0; j < nkb; ++j) {
                if (!rep) {
                    ok = __all_sync(0xffffffffu, mbar_wait(bar_s, (go + j) & 1, kWaitLimit));
                    if (!ok) { report(p.err, 0x301); break; }
                    tc_fence_after();
                    if (j == I) {
                        float2 ml = make_float2(m, l);
                        ok = diag_block(tS, tO, tP, quarter, row, p.scale_log2, j == 0, bar_o, (go + j - 1) & 1, ml);
                        if (!ok) { report(p.err, 0x302); break; }
                        m = ml.x;
                        l = ml.y;
                        tc_fence_before();
                        mbar_arrive_warp(bar_sf);
                    } else {
                        uint32_t v[128];
                        load_s_row(tS, v);
                        tc_fence_before();
                        mbar_arrive_warp(bar_sf);  // the MMA warp may now overwrite S
                        // row max of the block (the scale is positive); every row of
                        // a visited block has a visible key, so it is finite
                        const float f = update_max(row_max(v) * p.scale_log2, m, l);
                        // P_j replaces P_{j-1} in TMEM once P.V_{j-1} has read it (the
                        // previous item's last P.V was waited for by its epilogue), which
                        // is done by now as a rule.  P then goes to TMEM 32 keys at a time,
                        // so only a quarter of it is held in registers; the O rows are rescaled
                        // after (that P.V has landed in O; P.V_j waits for this warp)
                        if (j > 0) {
                            ok = __all_sync(0xffffffffu, mbar_wait(bar_o, (go + j - 1) & 1, kWaitLimit));
                            if (!ok) { report(p.err, 0x302); break; }
                            tc_fence_after();
                        }
                        const uint64_t sc2 = f32x2(p.scale_log2, p.scale_log2), nm2 = f32x2(-m, -m);
                        uint64_t l2[4] = {0, 0, 0, 0};
                        {
                            uint32_t pw[16];  // P as bf16 pairs, keys 0..31
                            exp_quarter<0>(v, sc2, nm2, l2, pw);
                            tmem_st16(tP, pw);
                        }
                        {
                            uint32_t pw[16];
                            exp_quarter<1>(v, sc2, nm2, l2, pw);
                            tmem_st16(tP + 16, pw);
                        }
                        {
                            uint32_t pw[16];
                            exp_quarter<2>(v, sc2, nm2, l2, pw);
                            tmem_st16(tP + 32, pw);
                        }
                        {
                            uint32_t pw[16];
                            exp_quarter<3>(v, sc2, nm2, l2, pw);
                            tmem_st16(tP + 48, pw);
                        }
                        const float2 ls = split_f32x2(add_f32x2(add_f32x2(l2[0], l2[1]), add_f32x2(l2[2], l2[3])));
                        l += ls.x + ls.y;
                        rescale_o(tO, f);
                    }
                } else {
                    // W(i,j) = E[i-j] c_j, bf16 pairs, into buffer g & 1 (g counts
                    // replaced blocks), last read by the P.V of block g - 2 (one
                    // barrier per buffer, so neither runs two phases ahead)
                    const int g = gr + j;
                    if (g >= 2) {
                        ok = __all_sync(0xffffffffu,
                                        mbar_wait(bar_ob + 8 * (g & 1), ((g >> 1) & 1) ^ 1, kWaitLimit));
                        if (!ok) { report(p.err, 0x303); break; }
                    }
                    // its inputs, staged by the producer
                    ok = __all_sync(0xffffffffu, mbar_wait(bar_wf + 8 * (g & 1), (g >> 1) & 1, kWaitLimit));
                    if (!ok) { report(p.err, 0x306); break; }
                    tc_fence_after();
                    if (!direct) {
                        uint32_t pw0[32], pw1[32];
                        // E pair 128 + (I - j) BN + row - 2mm of the padded array is entry
                        // 128 + row - 2mm of the staged window
                        const uint32_t st = sbase + SM_WST + (g & 1) * WST_BYTES;
                        build_w_half(st + 4 * (128 + row), st + WST_E, 0, pw0);
                        build_w_half(st + 4 * (128 + row), st + WST_E, 8, pw1);
                        tmem_st32(tS + 64 * (g & 1), pw0);
                        tmem_st32(tS + 64 * (g & 1) + 32, pw1);
                    } else {
                        direct_p_row(p.a + (size_t)h * T, p.r + (size_t)h * T, p.logz, h, T, i, j * BN,
                                     tS + 64 * (g & 1));
                    }
                }
                // hand P (or W) to the MMA warp
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive_warp(rep ? bar_pb + 8 * ((gr + j) & 1) : bar_p);
            }
            // epilogue (TMEM reads by whole warps; rows past T are not stored)
            if (ok) {
                const int gl = (rep ? gr : go) + nkb - 1;  // the last P.V (MMAs complete in order)
                ok = __all_sync(0xffffffffu, rep ? mbar_wait(bar_ob + 8 * (gl & 1), (gl >> 1) & 1, kWaitLimit)
                                                 : mbar_wait(bar_o, gl & 1, kWaitLimit));
                if (!ok) report(p.err, 0x304);
            }
            tc_fence_after();
            if (ok) {
                float scale = 0.f, lse_v = kNegInf;
                if (i < T) {
                    if (!rep) {
                        scale = l > 0.f ? 1.f / l : 0.f;
                        lse_v = (m == kNegInf || l <= 0.f) ? kNegInf : (m + log2f(l)) * kLn2;
                    } else {
                        lse_v = p.logz[(size_t)h * T + i];
                    }
                }
                if (rep) {  // every row reads its W sum (a warp-wide TMEM load)
                    const float sum = __uint_as_float(tmem_ld1(tmem + lane_off + TSUM_COL));
                    tmem_wait_ld();
                    scale = (i < T && sum > 0.f) ? 1.f / sum : 0.f;
                }
                __nv_bfloat16* orow = p.o + ((size_t)bh * T + (i < T ? i : 0)) * kHeadDim;
                // The warp's 32 rows go out as two 32-column TMA boxes through its
                // 2 KB staging area (row `lane` at lane * 64, 16-byte chunks in the
                // 64-byte swizzle); the warp moves on once a store is issued, where
                // 32 per-thread row stores would block its next barrier waits.
                // Rows past T are clipped by the store.
                const uint32_t ost = sbase + SM_OST + quarter * 2048 + lane * 64;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tO + 32 * c, v);
                    tmem_wait_ld();
                    uint32_t packed[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        packed[e] =
                            pack_bf16x2(__uint_as_float(v[2 * e]) * scale, __uint_as_float(v[2 * e + 1]) * scale);
                    if (p.tma_o) {
                        if (lane == 0) bulk_wait_read0();  // the previous box has been read
                        __syncwarp();
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            st_shared_v4(ost + ((k ^ ((lane >> 1) & 3)) << 4), packed[4 * k], packed[4 * k + 1],
                                         packed[4 * k + 2], packed[4 * k + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_3d(&tmO, sbase + SM_OST + quarter * 2048, 32 * c, I * BM + quarter * 32, bh);
                            bulk_commit();
                        }
                    } else if (i < T) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] =
                                make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
                    }
                }
                if (i < T) p.lse[(size_t)bh * T + i] = lse_v;
            } else if (i < T) {
                p.lse[(size_t)bh * T + i] = __int_as_float(0x7fc00000);  // NaN marks the failed rows
            }
            if (rep) gr += nkb;
            else go += nkb;
        }
        if (lane == 0) bulk_wait0();  // the O stores complete before the CTA ends
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
        if (atomicAdd(p.err + kCtrFwdDone, 1u) == gridDim.x - 1) {
            atomicExch(p.err + kCtrFwdNext, 0u);
            atomicExch(p.err + kCtrFwdDone, 0u);
        }
    }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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
    return fn;
}

}  // namespace

int sm_count() {
    constexpr int kMaxDev = 64;
    static int cached[kMaxDev] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

// [BH, T, 64] bf16 viewed as a 3-D tensor (d, t, bh); 128 x 64 boxes with the
// 128-byte swizzle; rows past T read as zeros.
bool make_tmap_bhtd(const void* base, int BH, int T, CUtensorMap* out, int box_rows, int box_cols) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || (box_cols != 64 && box_cols != 32)) return false;
    cuuint64_t dims[3] = {64, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {64 * 2, (cuuint64_t)T * 64 * 2};
    cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_fwd_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                          __nv_bfloat16* o, float* lse, const float* a, const float* r, const float* logz,
                          const HeadList& hl, const ReplacedWs& w, int B, int H, int Hkv, int T, unsigned int* err,
                          bool after_pattern, cudaStream_t stream) {
    CUtensorMap mq, mk, mv, mo;
    const int BH = B * H;
    if (!make_tmap_bhtd(q, BH, T, &mq) || !make_tmap_bhtd(k, B * Hkv, T, &mk) ||
        !make_tmap_bhtd(v, B * Hkv, T, &mv))
        return cudaErrorNotSupported;
    FwdTcParams p;
    // O by 32 x 32 TMA stores when its map encodes (a base the encoder
    // rejects, e.g. not 16-byte aligned, takes the row stores)
    p.tma_o = make_tmap_bhtd(o, BH, T, &mo, 32, 32) ? 1 : 0;
    if (!p.tma_o) mo = mq;  // not read
    p.o = o;
    p.lse = lse;
    p.a = a;
    p.r = r;
    p.logz = logz;
    p.w = w;
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
    p.nqb = (T + BM - 1) / BM;
    if ((int64_t)BH * p.nqb >= (int64_t)1 << 30) return cudaErrorNotSupported;  // item words hold 30 bits
    p.scale_log2 = kLog2e / 8.0f;
    const int smem = SM_TOTAL + 1024;
    cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // persistent: two CTAs per SM pull work items from a counter in the
    // workspace header
    const int items = BH * p.nqb;
    const int grid = std::min(items, 2 * sm_count());
    launch_begin(KID_FWD_TC, stream);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    // after the pattern preparation of this call (after_pattern), the kernel
    // may start while that grid runs: its ordinary items do not depend on it
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_pattern ? 1 : 0;
    cudaError_t le = cudaLaunchKernelEx(&cfg, fwd_tc_kernel, mq, mk, mv, mo, p);
    launch_end(KID_FWD_TC, stream);
    if (le != cudaSuccess) return le;
    return cudaGetLastError();
}

}  // namespace saf
