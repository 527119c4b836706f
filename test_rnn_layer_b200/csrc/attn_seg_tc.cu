// Segment-local multi-head attention on the tcgen05 tensor cores (head dim
// 64, bf16 Q/K/V, fp32 accumulation), with the sublayer's residual add in the
// epilogue:
//   Out[t, h] = Xres[t, h] + sum_{u in seg(t)} softmax_u(q_t . k_u / 8) v_u
// where seg(t) is the segment [s L, min((s+1) L, T)) holding token t.
//
// Source: One-Minute Video Generation with Test-Time Training, paper notes
// page, "方法详解 / 整体框架": the backbone's self-attention spans only the
// tokens of one 3-second segment; the TTT layer after it spans the sequence.
//
// Work: an item is 256 query rows (tiles A and B of 128) of one head inside
// one segment; a persistent grid walks the items in the order (segment, head,
// rows), so CTAs that run at the same time read the same head's keys and
// values from L2.  For each key tile j of 128 keys of the segment:
//   S_X = Q_X K_j^T             tensor cores, 4 MMAs of K = 16, fp32 in tensor memory
//   P_X = exp2(S_X c - m_X)     one thread per query row, c = log2(e) / 8
//   O_X += P_X V_j              P_X from tensor memory as bf16 pairs, V_j from shared memory
// The running maximum m_X of a row is raised only when a tile's maximum passes
// it by more than 8 (then the row sum and O_X are scaled by 2^(m_old - m_new));
// otherwise the exponents stay below 2^8 and nothing is rescaled.  This is the
// online softmax with a lazily raised maximum: the quotient O_X / l_X is the
// same for any reference value, only overflow has to be excluded.
//
// Roles (352 threads): warps 0-3 the softmax of tile A, warps 4-7 that of
// tile B (a thread per query row, i.e. per tensor-memory lane), warp 8 the TMA
// producer, warps 9 and 10 the MMA issuers of tiles A and B (one each, so that
// neither tile's products queue behind the other's waits).  While one softmax
// group works on the exponential unit, the tensor cores run the other's products.
//
// Tensor memory (512 columns): S_A 0, S_B 128 (fp32 128 x 128); O_A 256,
// O_B 320 (fp32 128 x 64); P_A 384, P_B 448 (128 x 128 bf16, two per column).
// Shared memory: Q_A, Q_B (16 KB each) and NST stages of a K and a V tile
// (16 KB each), all in the 128-byte swizzle TMA writes: rows of 64 bf16, so
// Q and K are K-major operands of S and V is the MN-major B operand of P V.
// Every wait is bounded; on a timeout the CTA sets the status word, lets its
// copies and products in flight land and returns.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "fma_exp2.cuh"
#include "internal.h"
#include "tc_prims.cuh"

namespace ttt {
namespace {

#ifndef TTT_ATTN_NST
#define TTT_ATTN_NST 4
#endif
constexpr int DH = 64, BQ = 128, BKV = 128, ROWS = 2 * BQ, NST = TTT_ATTN_NST, THREADS = 352;
constexpr int TILE = BQ * DH * 2;                 // 16 KB: a 128 x 64 bf16 tile
constexpr int OFF_Q = 0;                          // Q_A, Q_B
constexpr int OFF_KV = 2 * TILE;                  // stage s: K at OFF_KV + 2 s TILE, V after it
constexpr int OFF_BAR = OFF_KV + NST * 2 * TILE;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TM_S = 0, TM_O = 256, TM_P = 384;   // + 128 X (S), + 64 X (O, P) for tile X
constexpr float kLazy = 8.0f;                     // log2 of the largest unscaled exponential
// Pairs of every 8 whose exponentials run as a polynomial on the FMA pipe
// (the exponential unit, 16 results per cycle per SM, is the softmax's bound).
#ifndef TTT_ATTN_EMU
#define TTT_ATTN_EMU 1
#endif
constexpr int EMU = TTT_ATTN_EMU;


// Barrier slots (8 bytes each) from OFF_BAR.
enum : int {
    B_QF = 0,              // Q_A, Q_B landed (TMA bytes)
    B_QE = 1,              // the item's last S products of both tiles are done: Q may be reloaded (2 MMA commits)
    B_KF = 2,              // [NST] K tile landed
    B_VF = 2 + NST,        // [NST] V tile landed
    B_KVE = 2 + 2 * NST,   // [NST] both tiles' P V products of the stage are done (2 MMA commits)
    B_SF = 2 + 3 * NST,    // [2] S_X is in tensor memory (MMA commit)
    B_SR = B_SF + 2,       // [2] the softmax group has read S_X (4 warp arrivals)
    B_PF = B_SR + 2,       // [2] P_X written, O_X rescaled (4 warp arrivals)
    B_PV = B_PF + 2,       // [2] O_X += P_X V done (MMA commit)
    B_SLOT = B_PV + 2      // tensor memory address (u32) and the abort flag (int)
};
static_assert(B_SLOT * 8 + 8 <= 256, "barrier area");
static_assert(SMEM_BYTES <= 232448, "shared memory");

// Rows [q0, q1) of one segment whose keys are [kv0, kv1); `pairs` items of
// 256 rows per head, items item0 .. item0 + H pairs - 1 (head-major).
struct AttnGroup {
    int q0, q1, kv0, kv1, pairs, item0;
};
constexpr int kMaxGroups = 64;

struct AttnArgs {
    CUtensorMap mapQ, mapK, mapV;   // bf16 [T rows x H*64 columns], 64 x 128 boxes
    const __nv_bfloat16* xres;      // optional residual (null: none)
    long long ld_res;
    __nv_bfloat16* out;
    long long ld_out;
    int T, H, n_groups, n_items;
    float c;                        // log2(e) / sqrt(64)
    int* status;
    AttnGroup g[kMaxGroups];
};

#ifdef TTT_DEBUG_STAGES
// Debug builds only: cycles between stage boundaries seen in CTA 0 by thread 0
// (tile A's softmax, slots 0-7), thread 128 (tile B's, 8-15) and the MMA
// issuer (16-23).
__device__ long long* g_dbg_attn = nullptr;   // 40 slots
#define STAMPA(k)                                                   \
    do {                                                            \
        if (stamper) {                                              \
            const long long now_ = clock64();                       \
            stamp_acc[k] += now_ - stamp_last;                      \
            stamp_last = now_;                                      \
        }                                                           \
    } while (0)
#else
#define STAMPA(k) \
    do {          \
    } while (0)
#endif

__device__ __forceinline__ void item_of(const AttnArgs& p, int w, int& gi, int& h, int& pr) {
    gi = 0;
    while (gi + 1 < p.n_groups && p.g[gi + 1].item0 <= w) ++gi;
    const int r = w - p.g[gi].item0;
    h = r / p.g[gi].pairs;
    pr = r - h * p.g[gi].pairs;
}

__device__ __forceinline__ float ex2(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// max that returns NaN if an operand is NaN (fmaxf would drop it); two- and three-input forms
__device__ __forceinline__ float max_nan(float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
    float r;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Pairs of fp32 values in one 64-bit register pair, for the packed f32x2 arithmetic of sm_100
// (one instruction for two elements).
__device__ __forceinline__ uint64_t f2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// 2^x0, 2^x1 on the FMA pipe: fma_exp2.cuh's cubic (relative error 7.6e-5, 25 times below the bf16
// rounding P gets) on a pair, with the packed f32x2 arithmetic.  x <= 8 here; below -125 it returns about
// 2^-125, which next to a row maximum of at least 2^-8 is far below fp32 resolution.
__device__ __forceinline__ void ex2_poly2(uint64_t x, float& p0, float& p1) {
    float x0, x1;
    f2_split(x, x0, x1);
    x = f2(max_nan(x0, -125.0f), max_nan(x1, -125.0f));   // as fexp::clamp_low; NaN stays NaN
    using namespace fexp;
    const uint64_t shift = f2(kShift, kShift);
    const uint64_t t = f2_add(x, shift);
    const uint64_t f = f2_sub(x, f2_sub(t, shift));
    uint64_t p = f2_fma(f2(kC3_3, kC3_3), f, f2(kC3_2, kC3_2));
    p = f2_fma(p, f, f2(kC3_1, kC3_1));
    p = f2_fma(p, f, f2(kC3_0, kC3_0));
    float t0, t1, q0, q1;
    f2_split(t, t0, t1);
    f2_split(p, q0, q1);
    p0 = scale_by_rint(q0, t0);
    p1 = scale_by_rint(q1, t1);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ uint64_t kmajor_desc(const uint8_t* p) { return tc::smem_desc(tc::smem_u32(p), 16, 1024); }
// MN-major (V): one 64-wide block, 8-row groups 1 KB apart; K step of 16 keys = 2048 bytes.
__device__ __forceinline__ uint64_t mnmajor_desc(const uint8_t* p) { return tc::smem_desc(tc::smem_u32(p), 16384, 1024); }

__global__ void __launch_bounds__(THREADS, 1) attn_seg_kernel(const __grid_constant__ AttnArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_SLOT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        tc::mbar_init(bars + B_QF, 1);
        tc::mbar_init(bars + B_QE, 2);
        for (int s = 0; s < NST; ++s) {
            tc::mbar_init(bars + B_KF + s, 1);
            tc::mbar_init(bars + B_VF + s, 1);
            tc::mbar_init(bars + B_KVE + s, 2);
        }
        for (int x = 0; x < 2; ++x) {
            tc::mbar_init(bars + B_SF + x, 1);
            tc::mbar_init(bars + B_SR + x, 4);
            tc::mbar_init(bars + B_PF + x, 4);
            tc::mbar_init(bars + B_PV + x, 1);
        }
        *abort_flag = 0;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&p.mapQ);
        tc::tma_prefetch_desc(&p.mapK);
        tc::tma_prefetch_desc(&p.mapV);
    }
    if (warp == 9) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tm = *tmem_slot;

    auto give_up = [&]() {
        *abort_flag = 1;
        atomicOr(p.status, kStatusTimeout);
    };
#ifdef TTT_DEBUG_STAGES
    const bool stamper = blockIdx.x == 0 && (tid == 0 || tid == 128 || tid == 288 || tid == 320 || tid == 256);
    long long stamp_acc[8] = {};
    long long stamp_last = clock64();
#endif

    if (warp == 8) {
        // ---------------- TMA producer: the item's Q tiles, then its K and V tiles through the ring
        if (tc::elect_one()) {
            int gkv = 0, it = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < p.n_items && ok && !*abort_flag; w += gridDim.x, ++it) {
                int gi, h, pr;
                item_of(p, w, gi, h, pr);
                const AttnGroup& G = p.g[gi];
                const int q_lo = G.q0 + ROWS * pr, x = h * DH;
                const int nkv = (G.kv1 - G.kv0 + BKV - 1) / BKV;
                STAMPA(3);
                if (it > 0 && !tc::mbar_wait(bars + B_QE, (it - 1) & 1, abort_flag)) { ok = false; break; }
                STAMPA(2);
                tc::mbar_arrive_expect_tx(bars + B_QF, 2 * TILE);
                tc::tma_load_2d(sm + OFF_Q, &p.mapQ, x, q_lo, bars + B_QF);
                // tile B past the last token: load tile A's rows again (its rows are never stored)
                tc::tma_load_2d(sm + OFF_Q + TILE, &p.mapQ, x, q_lo + BQ < p.T ? q_lo + BQ : q_lo, bars + B_QF);
                for (int j = 0; j < nkv; ++j, ++gkv) {
                    const int s = gkv % NST, use = gkv / NST;
                    STAMPA(3);
                    if (use > 0 && !tc::mbar_wait(bars + B_KVE + s, (use - 1) & 1, abort_flag)) { ok = false; break; }
                    STAMPA(0);
                    uint8_t* kt = sm + OFF_KV + s * 2 * TILE;
                    tc::mbar_arrive_expect_tx(bars + B_KF + s, TILE);
                    tc::tma_load_2d(kt, &p.mapK, x, G.kv0 + BKV * j, bars + B_KF + s);
                    tc::mbar_arrive_expect_tx(bars + B_VF + s, TILE);
                    tc::tma_load_2d(kt + TILE, &p.mapV, x, G.kv0 + BKV * j, bars + B_VF + s);
                    STAMPA(1);
                }
            }
            if (!ok) give_up();
        }
    } else if (warp >= 9) {
        // ---------------- MMA issuers, one per tile (warp 9: A, warp 10: B), so that neither tile's products
        // wait behind the other's.  Step n = (item, key tile j) in the CTA's order; at iteration j the issuer
        // of tile X issues S_X of step j (once its group has read S_X of the step before), then P_X V of
        // step j - 1.  A stage of the ring and the Q tiles are released when both issuers' products are done.
        const int X = warp - 9;
        if (tc::elect_one()) {
            constexpr uint32_t ID_S = tc::instr_desc(1, BQ, BKV, 0, 0);   // bf16, both K-major
            constexpr uint32_t ID_PV = tc::instr_desc(1, BQ, DH, 0, 1);   // bf16, A in tensor memory, V MN-major
            const uint64_t dQ = kmajor_desc(sm + OFF_Q + X * TILE);
            int gkv = 0, gs = 0, it = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < p.n_items && ok && !*abort_flag; w += gridDim.x, ++it) {
                int gi, h, pr;
                item_of(p, w, gi, h, pr);
                const int nkv = (p.g[gi].kv1 - p.g[gi].kv0 + BKV - 1) / BKV;
                if (!tc::mbar_wait(bars + B_QF, it & 1, abort_flag)) { ok = false; break; }
                tc::tc_fence_after();
                STAMPA(5);
                for (int j = 0; j <= nkv && ok; ++j) {
                    if (j < nkv) {
                        const int n = gs + j, s = (gkv + j) % NST, use = (gkv + j) / NST;
#ifdef TTT_DEBUG_STAGES
                        if (stamper && tc::mbar_try_wait(bars + B_KF + s, use & 1)) stamp_acc[6] += 1;
#endif
                        if (!tc::mbar_wait(bars + B_KF + s, use & 1, abort_flag)) { ok = false; break; }
                        STAMPA(0);
                        if (n > 0 && !tc::mbar_wait(bars + B_SR + X, (n - 1) & 1, abort_flag)) { ok = false; break; }
                        tc::tc_fence_after();
                        const uint64_t dK = kmajor_desc(sm + OFF_KV + s * 2 * TILE);
#pragma unroll
                        for (int kk = 0; kk < DH / 16; ++kk)
                            tc::mma_f16_ss(tm + TM_S + 128 * X, dQ + 2 * kk, dK + 2 * kk, ID_S, kk > 0);
                        tc::mma_commit(bars + B_SF + X);
                        if (j == nkv - 1) tc::mma_commit(bars + B_QE);
                        STAMPA(1);
                    }
                    if (j > 0) {
                        const int n = gs + j - 1, s = (gkv + j - 1) % NST, use = (gkv + j - 1) / NST;
                        if (!tc::mbar_wait(bars + B_VF + s, use & 1, abort_flag)) { ok = false; break; }
                        if (!tc::mbar_wait(bars + B_PF + X, n & 1, abort_flag)) { ok = false; break; }
                        tc::tc_fence_after();
                        STAMPA(2);
                        const uint64_t dV = mnmajor_desc(sm + OFF_KV + s * 2 * TILE + TILE);
#pragma unroll
                        for (int kk = 0; kk < BKV / 16; ++kk)
                            tc::mma_f16_ts(tm + TM_O + 64 * X, tm + TM_P + 64 * X + 8 * kk, dV + (uint64_t)(kk * 128),
                                           ID_PV, (j > 1 || kk > 0) ? 1u : 0u);
                        tc::mma_commit(bars + B_PV + X);
                        tc::mma_commit(bars + B_KVE + s);
                        STAMPA(3);
                    }
                }
                gs += nkv;
                gkv += nkv;
            }
            if (!ok) give_up();
        }
    } else {
        // ---------------- softmax groups: warps 0-3 tile A, 4-7 tile B; thread = query row r of its tile
        const int X = warp >> 2, qd = warp & 3, r = 32 * qd + lane;
        const uint32_t lanes = (uint32_t)(32 * qd) << 16;
        const uint32_t tS = tm + lanes + TM_S + 128 * X, tO = tm + lanes + TM_O + 64 * X, tP = tm + lanes + TM_P + 64 * X;
        const float c = p.c;
        int gs = 0, nonfinite = 0;
        bool ok = true;
        // every branch below is uniform over the warp (the item, the key tile, the waits' outcome)
        auto wait_all = [&](uint64_t* bar, uint32_t parity) {
            const bool got = tc::mbar_wait(bar, parity, abort_flag);
            return __all_sync(0xffffffffu, got);
        };
        for (int w = blockIdx.x; w < p.n_items && ok && !*abort_flag; w += gridDim.x) {
            int gi, h, pr;
            item_of(p, w, gi, h, pr);
            const AttnGroup& G = p.g[gi];
            const int q_lo = G.q0 + ROWS * pr;
            const int nkv = (G.kv1 - G.kv0 + BKV - 1) / BKV;
            float m_run = -INFINITY, l = 0.f;
            for (int j = 0; j < nkv; ++j, ++gs) {
                if (!wait_all(bars + B_SF + X, gs & 1)) { ok = false; break; }
                tc::tc_fence_after();
                STAMPA(0);
                uint32_t s[BKV];
                tc::tmem_ld_32x32b_x32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(s + 0));
                tc::tmem_ld_32x32b_x32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(s + 32));
                tc::tmem_ld_32x32b_x32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(s + 64));
                tc::tmem_ld_32x32b_x32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(s + 96));
                tc::tmem_wait_ld();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bars + B_SR + X);   // S_X may be overwritten
                STAMPA(1);
                const int valid = G.kv1 - (G.kv0 + BKV * j);
                if (valid < BKV) {   // the segment's last key tile: keys past its end do not take part
#pragma unroll
                    for (int k = 0; k < BKV; ++k)
                        if (k >= valid) s[k] = 0xff800000u;   // -inf
                }
                // the tile's row maximum in eight independent chains of three-input maxima (a NaN anywhere
                // makes it NaN, so a non-finite input spoils the whole row and reaches the output check)
                float m8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) m8[i] = max_nan(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1]));
#pragma unroll
                for (int k = 16; k < BKV; k += 16) {
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        m8[i] = max3_nan(m8[i], __uint_as_float(s[k + 2 * i]), __uint_as_float(s[k + 2 * i + 1]));
                }
                float mt = max3_nan(max3_nan(m8[0], m8[1], m8[2]), max3_nan(m8[3], m8[4], m8[5]), max_nan(m8[6], m8[7]));
                mt *= c;
                STAMPA(2);
                float f = 1.f;
                bool rescale = false;
                if (mt > m_run + kLazy) {   // raise the reference maximum (always on the item's first tile)
                    f = ex2(m_run - mt);
                    rescale = j > 0;
                    m_run = mt;
                    l *= f;
                }
                // P as bf16 pairs, packed into the front of s (pair k2 lands in s[k2] after s[2 k2], s[2 k2 + 1] are read)
                // x = s c - m two at a time; EMU of every 8 pairs take 2^x on the FMA pipe, the rest on the
                // exponential unit; row sums in four packed partial sums
                const uint64_t c2 = f2(c, c), nm2 = f2(-m_run, -m_run);
                uint64_t ls[4] = {0, 0, 0, 0};
#pragma unroll
                for (int k2 = 0; k2 < BKV / 2; ++k2) {
                    const uint64_t x = f2_fma(f2(__uint_as_float(s[2 * k2]), __uint_as_float(s[2 * k2 + 1])), c2, nm2);
                    float p0, p1;
                    if ((k2 & 7) >= 8 - EMU) {
                        ex2_poly2(x, p0, p1);
                    } else {
                        float x0, x1;
                        f2_split(x, x0, x1);
                        p0 = ex2(x0);
                        p1 = ex2(x1);
                    }
                    const uint64_t pp = f2(p0, p1);
                    ls[k2 & 3] = f2_add(ls[k2 & 3], pp);
                    s[k2] = pack_bf16(p0, p1);
                }
                {
                    float a0, a1, b0, b1;
                    f2_split(f2_add(f2_add(ls[0], ls[1]), f2_add(ls[2], ls[3])), a0, a1);
                    (void)b0;
                    (void)b1;
                    l += a0 + a1;
                }
                STAMPA(3);
                // the previous step's P V is done: P_X may be rewritten and O_X is stable
                if (gs > 0) {
                    if (!wait_all(bars + B_PV + X, (gs - 1) & 1)) { ok = false; break; }
                    tc::tc_fence_after();
                }
                STAMPA(4);
                if (__any_sync(0xffffffffu, rescale)) {
                    const float g = rescale ? f : 1.f;
                    uint32_t o[32];
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        tc::tmem_ld_32x32b_x32(tO + 32 * half, o);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * g);
                        tc::tmem_st_32x32b_x32(tO + 32 * half, o);
                    }
                }
                tc::tmem_st_32x32b_x32(tP + 0, *reinterpret_cast<uint32_t(*)[32]>(s + 0));
                tc::tmem_st_32x32b_x32(tP + 32, *reinterpret_cast<uint32_t(*)[32]>(s + 32));
                tc::tmem_wait_st();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bars + B_PF + X);
                STAMPA(5);
            }
            if (!ok) break;
            // ---- epilogue: O_X / l (+ residual) as bf16, row q_lo + 128 X + r if it belongs to the item
            if (!wait_all(bars + B_PV + X, (gs - 1) & 1)) { ok = false; break; }
            tc::tc_fence_after();
            uint32_t o[64];
            tc::tmem_ld_32x32b_x32(tO + 0, *reinterpret_cast<uint32_t(*)[32]>(o + 0));
            tc::tmem_ld_32x32b_x32(tO + 32, *reinterpret_cast<uint32_t(*)[32]>(o + 32));
            tc::tmem_wait_ld();
            const int t = q_lo + BQ * X + r;
            if (t < G.q1) {
                const float inv = 1.0f / l;
                const long long col = (long long)h * DH;
                const uint4* xr = p.xres ? reinterpret_cast<const uint4*>(p.xres + t * p.ld_res + col) : nullptr;
                uint4* dst = reinterpret_cast<uint4*>(p.out + t * p.ld_out + col);
#pragma unroll
                for (int c8 = 0; c8 < DH / 8; ++c8) {
                    float v[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(o[8 * c8 + e]) * inv;
                    if (xr) {
                        const uint4 xv = xr[c8];
                        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&xw[e]);
                            v[2 * e] += __low2float(b2);
                            v[2 * e + 1] += __high2float(b2);
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) nonfinite |= !isfinite(v[e]);
                    dst[c8] = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                                         pack_bf16(v[6], v[7]));
                }
            }
        }
        if (!ok) {
            if (lane == 0) give_up();
        }
        if (__any_sync(0xffffffffu, nonfinite) && lane == 0) atomicOr(p.status, kStatusNonFinite);
    }

#ifdef TTT_DEBUG_STAGES
    if (stamper && g_dbg_attn) {
        const int role = tid == 0 ? 0 : tid == 128 ? 1 : tid == 288 ? 2 : tid == 320 ? 3 : 4;
        for (int k = 0; k < 8; ++k) g_dbg_attn[8 * role + k] = stamp_acc[k];
    }
#endif
    if (*abort_flag) {
        // let copies and products already in flight land before the CTA's memory goes away
        const uint64_t t0 = tc::globaltimer_ns();
        while (tc::globaltimer_ns() - t0 < 1000000ull) __nanosleep(1000);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tm, 512);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// bf16 [T rows x cols columns], row stride ld elements; boxes of 64 columns x 128 rows, 128-byte swizzle
// (rows past T read as zero).
bool make_map(CUtensorMap* m, const void* base, int T, int cols, long long ld) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)T};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    cuuint32_t box[2] = {DH, BQ};
    cuuint32_t es[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

#ifdef TTT_DEBUG_STAGES
extern "C" __attribute__((visibility("default"))) int ttt_debug_set_dump_attn(long long* p) {
    return (int)cudaMemcpyToSymbol(g_dbg_attn, &p, sizeof(p));
}
#endif

bool attn_seg_supported(int d) { return d == DH; }

long long attn_seg_items(int T, int H, int L, int row0, int row1) {
    long long n = 0;
    for (int s0 = (row0 / L) * L; s0 < row1; s0 += L) {
        const int q0 = std::max(row0, s0), q1 = std::min(row1, std::min(s0 + L, T));
        if (q1 > q0) n += (long long)H * ((q1 - q0 + ROWS - 1) / ROWS);
    }
    return n;
}

cudaError_t launch_attn_seg(const void* Q, const void* K, const void* V, long long ld_qkv, const void* Xres,
                            long long ld_res, void* Out, long long ld_out, int T, int H, int L, int row0, int row1,
                            int* status, int max_ctas, cudaStream_t s) {
    if (row1 <= row0) return cudaSuccess;
    AttnArgs p{};
    const int cols = H * DH;
    if (!make_map(&p.mapQ, Q, T, cols, ld_qkv) || !make_map(&p.mapK, K, T, cols, ld_qkv) ||
        !make_map(&p.mapV, V, T, cols, ld_qkv))
        return cudaErrorInvalidValue;
    p.xres = static_cast<const __nv_bfloat16*>(Xres);
    p.ld_res = ld_res;
    p.out = static_cast<__nv_bfloat16*>(Out);
    p.ld_out = ld_out;
    p.T = T;
    p.H = H;
    p.c = 1.4426950408889634f / 8.0f;   // log2(e) / sqrt(64)
    p.status = status;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e = cudaFuncSetAttribute(attn_seg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // the segments that meet [row0, row1), at most kMaxGroups per launch
    std::vector<AttnGroup> groups;
    for (int s0 = (row0 / L) * L; s0 < row1; s0 += L) {
        AttnGroup g{};
        g.q0 = std::max(row0, s0);
        g.q1 = std::min(row1, std::min(s0 + L, T));
        g.kv0 = s0;
        g.kv1 = std::min(s0 + L, T);
        g.pairs = (g.q1 - g.q0 + ROWS - 1) / ROWS;
        if (g.q1 > g.q0) groups.push_back(g);
    }
    for (size_t b0 = 0; b0 < groups.size(); b0 += kMaxGroups) {
        const int ng = (int)std::min(groups.size() - b0, (size_t)kMaxGroups);
        int items = 0;
        for (int k = 0; k < ng; ++k) {
            p.g[k] = groups[b0 + k];
            p.g[k].item0 = items;
            items += H * p.g[k].pairs;
        }
        p.n_groups = ng;
        p.n_items = items;
        int grid = std::min(items, sms);
        if (max_ctas > 0 && grid > max_ctas) grid = max_ctas;
        LaunchScope scope("attn_seg_tc", s);
        attn_seg_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace ttt
