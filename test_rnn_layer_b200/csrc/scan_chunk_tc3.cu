// Chunked TTT-MLP scan on the tcgen05 tensor cores, each head split over a
// cluster of two CTAs and each CTA split into two warp groups that work on
// different chunks at the same time (d = 64, m = 256, b <= 64).
//
// The per-chunk work has two branches (paper notes page, "关键设计 / TTT-MLP 层";
// chunk c of b tokens, W1, W2 the state at the chunk start, all gradients at
// that state, token t read with the prefix state):
//   state branch:  A^T = W1 K^T, G = GELU(A), Y^T = W2 G^T, D2' = -2 eta (Y - V),
//                  P^T = W2^T D2'^T, Dl = P * GELU'(A), W1 += Dl^T K, W2^T += G^T D2'
//   output branch: Aq^T = W1 Q^T + Dl^T M^T (M[t,s] = q_t.k_s, s not after t),
//                  Gq = GELU(Aq), z_t = W2_t GELU(Aq_t).
// Only the state branch feeds the next chunk, so warps 0-7 (the state group)
// walk the state chain while warps 8-15 (the output group) finish the output
// branch of the chunk before.  The output group reads z with the state at the
// END of its chunk and removes the later tokens' updates:
//   [Z1^T; N] = [W2_{c+1}; G] Gq^T,  Z^T = Z1^T - D2'^T Npost^T,
//   Npost[t,s] = N[s,t] = g_s.gq_t for s after t,
// so it needs the W2 copy the state group makes for the next chunk anyway.
//
// CTA r of the pair owns hidden units [128 r, 128 r + 128): its rows of W1 and
// W2^T live in tensor memory as fp32 accumulators for the whole sequence.  The
// two contractions over hidden units (Y^T and [Z1^T; N]) are split between the
// pair; the Y^T partials cross through distributed shared memory on the state
// chain, and each CTA finishes the z of 32 of the 64 tokens from the two z
// partials (the masked correction is linear in N, so each CTA corrects its own
// partial).  All partials travel as asynchronous 16-byte stores that complete
// bytes on a receive barrier of the peer, one barrier per sending/receiving
// warp pair and per buffer parity (the receive buffers alternate by chunk).
//
// Precision: the contractions that read the fp32 state from tensor memory
// (W1 K^T, W1 Q^T, W2^T D2'^T) and Q K^T take tf32 operands; every operand the
// threads produce (G, Gq, the W2 copy, K^T, D2'^T, Dl, G^T, the masks) is
// stored as fp16 and those contractions run as kind::f16 -- fp16 has the same
// 10-bit mantissa as tf32 (and is rounded, not truncated), its range covers
// these operands (|values| < 1e3; the smallest, Dl and D2', lose only an
// absolute 3e-8 at the subnormal floor), and it halves their shared memory
// and tensor time.  Accumulation is fp32 throughout.
//
// Ordering between the groups (mbarriers; a barrier that may be waited on two
// chunks late alternates with a second one, so no wait lags its barrier by two
// phases):
//   state -> output   bar_aq[c&1]: Aq of chunk c is final (the Dl^T M^T MMA)
//                     bar_w2r[c&1]: the W2 copy beside G_c holds W2_{c+1}
//   output -> state   bar_zn[c&1]: the [Z1; N] MMA of chunk c is done (its Aq
//                     buffer, G_c and W2 copy may be rewritten, at chunk c+2)
//                     bar_zd[c&1]: chunk c's output is done (its D2'^T buffer and
//                     z receive buffer may be rewritten, at chunk c+2)
// Every wait is bounded; a timeout sets the status word and an abort flag that
// both groups turn into a uniform exit at their next group barrier.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc_prims.cuh"

namespace ttt {
namespace {

constexpr int BT = 64, DH = 64, MH = 256, MLOC = 128, THREADS = 512, NG = 256;

// Shared memory (bytes from a 1024-aligned base).  fp32 tiles: 128-byte
// swizzled atoms of 8 rows x 32 columns, the two 32-column halves 8 KB apart
// (TMA layout).  fp16 operands, 128-byte swizzle, 64 values per 128-byte row:
// K-major ones hold a row per M/N index; MN-major ones a row per K index, in
// blocks of 64 M/N values 16 KB apart (the descriptor's leading offset) and
// 8-row groups 1 KB apart (its stride offset), so that a thread that owns one
// K index (a tensor-memory lane) writes its row with 16-byte stores.
constexpr int OFF_W2G = 0;          // [2] x 32 KB, MN-major over K = i: block 0 the W2 copy [i][j], block 1 G [i][t]
constexpr int OFF_GQ = 65536;       // 16 KB: Gq, MN-major [i][t]
constexpr int OFF_Q = 81920;        // 16 KB fp32 Q [t][j] (TMA)
constexpr int OFF_K = 98304;        // 16 KB fp32 K [t][j] (TMA)
constexpr int OFF_V = 114688;       // 16 KB fp32 V [t][j] (TMA)
constexpr int OFF_X1 = 131072;      // 8 KB: K fp16, MN-major over K = t: [t][j]
constexpr int OFF_X2 = 139264;      // 8 KB: M [t][s] fp16 (prefix mask of Q K^T)
constexpr int OFF_X3 = 147456;      // [2] x 8 KB: D2'^T [j][t] fp16 (a 128-row read of either stays inside X3, X4)
constexpr int OFF_X4 = 163840;      // 8 KB: -Npost, MN-major over K = s: [s][t] fp16
constexpr int OFF_RY = 172032;      // [2] x 16 KB: the peer's Y^T partial [j][t] fp32
constexpr int OFF_RZ = 204800;      // [2] x 8 KB: the peer's z partial for my tokens [j][t_own] fp32, then my z
constexpr int OFF_XS = 221184;      // 8 KB: the gate's x of my 32 tokens [t][j] (bf16 or fp32, by cp.async)
constexpr int OFF_BAR = 229376;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr int ST64 = 8192;
constexpr uint32_t RY_WARP_BYTES = 4096, RZ_WARP_BYTES = 4096;

// Tensor memory (128 lanes x 512 32-bit columns).
constexpr uint32_t TM_W1 = 0;       // my W1 rows [i][j] fp32
constexpr uint32_t TM_W2T = 64;     // my W2^T rows [i][j] fp32
constexpr uint32_t TM_R1 = 128;     // A^T [i][t], then the Y^T partial [j][t]
constexpr uint32_t TM_R2 = 192;     // S [t][s], then P^T [i][t]
constexpr uint32_t TM_GT = 256;     // G^T [i][t] fp16 pairs
constexpr uint32_t TM_DL = 288;     // Dl^T [i][t] fp16 pairs
constexpr uint32_t TM_AQ = 320;     // [2] x 64: Aq^T [i][t] fp32
constexpr uint32_t TM_ZN = 448;     // [Z1^T; N] partial [j | s][t] fp32

// Barrier slots (8 bytes each) from OFF_BAR.
enum : int {
    B_A = 0, B_S, B_Y, B_P, B_U, B_K, B_Q, B_V, B_CORR, B_NEVER,
    B_AQ = 10,     // [2]
    B_W2R = 12,    // [2]
    B_ZN = 14,     // [2]
    B_ZD = 16,     // [2]
    B_RY = 18,     // [2][4]
    B_RZ = 26,     // [2][2]
    B_SLOT = 30    // tensor memory address (u32) and the abort flag (int)
};

#ifdef TTT_DEBUG_STAGES
// Debug builds only: cycles between stage boundaries seen by thread 0 (state
// group, slots 0-15) and thread 256 (output group, slots 16-31) of CTA 0.
__device__ float* g_dbg3 = nullptr;
#define STAMP3(k)                                                   \
    do {                                                            \
        if ((tid == 0 || tid == NG) && blockIdx.x == 0) {           \
            const long long now_ = clock64();                       \
            stamp_acc[k] += now_ - stamp_last;                      \
            stamp_last = now_;                                      \
        }                                                           \
    } while (0)
#else
#define STAMP3(k) \
    do {          \
    } while (0)
#endif

struct ScanTc3Args {
    CUtensorMap mapQ, mapK, mapV;
    ScanArgs a;
    int full;
};

__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float ex2_approx(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// erf-GELU and GELU' with erf from Abramowitz & Stegun, Handbook of
// Mathematical Functions, formula 7.1.26 (|error| <= 1.5e-7, far below the
// fp16/tf32 rounding the results get); GELU and GELU' share one exponential.
__device__ __forceinline__ void gelu_as(float a, float& g, float& gp, bool want_prime) {
    const float u = rcp_approx(fmaf(0.3275911f * 0.70710678118654752f, fabsf(a), 1.0f));
    const float e = ex2_approx(a * (a * -0.72134752044448170f));   // exp(-a^2 / 2)
    float poly = fmaf(1.061405429f, u, -1.453152027f);
    poly = fmaf(poly, u, 1.421413741f);
    poly = fmaf(poly, u, -0.284496736f);
    poly = fmaf(poly, u, 0.254829592f);
    poly *= u;
    const float erf_abs = 1.0f - poly * e;
    const float Phi = 0.5f + 0.5f * copysignf(erf_abs, a);
    g = a * Phi;
    if (want_prime) gp = fmaf(a * 0.39894228040143268f, e, Phi);
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(tc::smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(tc::smem_u32(bar))
        : "memory");
}

// A K-major operand descriptor advanced to K-step kk (32 bytes per step: 8
// tf32 or 16 fp16 values), `stride` bytes between 128-byte column blocks.
__device__ __forceinline__ uint64_t kstep(uint64_t d0, int kk, uint32_t stride) {
    return d0 + (uint64_t)(((kk >> 2) * stride + (kk & 3) * 32) >> 4);
}

// Byte offset of fp32 element (R, c) of a swizzled tile (32 columns per block).
__device__ __forceinline__ uint32_t f32_off(int R, int c, int stride) {
    return (uint32_t)((c >> 5) * stride + (R >> 3) * 1024 + (R & 7) * 128 + ((((c & 31) >> 2) ^ (R & 7)) << 4) +
                      (c & 3) * 4);
}

// Byte offset of the 16-byte chunk holding fp16 values mn .. mn+7 (mn % 8 == 0)
// of K index k in an MN-major operand (blocks of 64 values `blk` bytes apart).
__device__ __forceinline__ uint32_t mn_chunk(int k, int mn, int blk) {
    return (uint32_t)((mn >> 6) * blk + (k >> 3) * 1024 + (k & 7) * 128 + ((((mn & 63) >> 3) ^ (k & 7)) << 4));
}

// 32 fp16 values (from 16 packed pairs) as four 16-byte stores at MN-major row k, values mn0 .. mn0+31.
__device__ __forceinline__ void st_row32(uint8_t* base, int k, int mn0, int blk, const uint32_t (&u)[16]) {
#pragma unroll
    for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(base + mn_chunk(k, mn0 + 8 * c, blk)) =
            make_uint4(u[4 * c], u[4 * c + 1], u[4 * c + 2], u[4 * c + 3]);
}

// An MN-major operand descriptor advanced to K-step kk (16 K indices = 2048 bytes).
__device__ __forceinline__ uint64_t kstep_mn(uint64_t d0, int kk) { return d0 + (uint64_t)((kk * 2048) >> 4); }

// Byte offset of the 16-byte chunk holding fp16 columns k .. k+7 (k % 8 == 0) of row R.
__device__ __forceinline__ uint32_t h_chunk(int R, int k, int stride) {
    return (uint32_t)((k >> 6) * stride + (R >> 3) * 1024 + (R & 7) * 128 + ((((k & 63) >> 3) ^ (R & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Receive buffers: rows of 16-byte chunks, chunk index XOR-ed with the row.
__device__ __forceinline__ uint32_t ry_off(int j, int t) { return (uint32_t)(j * 256 + (((t >> 2) ^ (j & 15)) << 4)); }
__device__ __forceinline__ uint32_t rz_off(int j, int t) { return (uint32_t)(j * 128 + (((t >> 2) ^ (j & 7)) << 4)); }

__global__ void __launch_bounds__(THREADS, 1) scan_tc3_kernel(const __grid_constant__ ScanTc3Args P) {
    const ScanArgs& a = P.a;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_SLOT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool state_group = warp < 8;
    const int q = warp & 3, gh = (warp >> 2) & 1;   // TMEM lane quarter; token half (32 tokens)
    const int i_loc = 32 * q + lane;
    const int t0 = 32 * gh;
    const uint32_t r_cta = tc::cluster_ctarank();
    const uint32_t r_peer = r_cta ^ 1u;
    const int h = blockIdx.x >> 1;
    const int T = a.T, b = a.b;
    const int nchunks = (T + b - 1) / b;
    const int c_first = a.c_begin, c_last = a.c_end > 0 ? min(a.c_end, nchunks) : nchunks;
    const int nloc = c_last - c_first;
    const float eta = a.eta;

    if (tid == 0) {
        for (int k = 0; k < B_SLOT; ++k) tc::mbar_init(bars + k, 1);
        *abort_flag = 0;
        for (int p = 0; p < 2; ++p) {   // arm phase 0 of every receive barrier (the peer's stores complete it)
            for (int w = 0; w < 4; ++w) tc::mbar_arrive_expect_tx(bars + B_RY + 4 * p + w, RY_WARP_BYTES);
            for (int w = 0; w < 2; ++w) tc::mbar_arrive_expect_tx(bars + B_RZ + 2 * p + w, RZ_WARP_BYTES);
        }
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    tc::cluster_sync();   // both CTAs' barriers exist before either arrives remotely
    tc::tc_fence_after();
    const uint32_t tm = *tmem_slot;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;

    auto give_up = [&]() {
        *abort_flag = 1;
        atomicOr(a.status, kStatusTimeout);
    };
    auto wait_bar = [&](int k, uint32_t parity) {
        if (!tc::mbar_wait(bars + k, parity, abort_flag)) give_up();
    };
    auto chunk_rows = [&](int c, int& y0, int& bc) {
        bc = min(b, T - c * b);
        y0 = a.reverse ? (T - c * b - bc) : c * b;
    };
    auto load_tile = [&](const CUtensorMap* map, uint32_t dst_off, int k, int y0) {
        tc::mbar_arrive_expect_tx(bars + k, BT * DH * 4);
        for (int half = 0; half < 2; ++half) {
            if (P.full) tma_load_3d(sm + dst_off + half * ST64, map, half * 32, h, y0, bars + k);
            else tma_load_3d(sm + dst_off + half * ST64, map, half * 32, y0, h, bars + k);
        }
    };
    auto after = [&](int s, int t) -> bool { return a.reverse ? (s < t) : (s > t); };

    constexpr uint32_t ID_TF32 = tc::instr_desc(2, 128, 64, 0, 0);
    constexpr uint32_t ID_F16 = tc::instr_desc(0, 128, 64, 0, 0);       // both operands K-major
    constexpr uint32_t ID_F16_MM = tc::instr_desc(0, 128, 64, 1, 1);    // both MN-major
    constexpr uint32_t ID_F16_KM = tc::instr_desc(0, 128, 64, 0, 1);    // A K-major (or in tensor memory), B MN-major
    const uint32_t s_base = tc::smem_u32(sm);
    const uint64_t dQ = tc::smem_desc(s_base + OFF_Q, 16, 1024), dK = tc::smem_desc(s_base + OFF_K, 16, 1024);
    const uint64_t dX1 = tc::smem_desc(s_base + OFF_X1, 16384, 1024), dX2 = tc::smem_desc(s_base + OFF_X2, 16, 1024);
    const uint64_t dX4 = tc::smem_desc(s_base + OFF_X4, 16384, 1024), dGQ = tc::smem_desc(s_base + OFF_GQ, 16384, 1024);
    auto dW2G = [&](int p) { return tc::smem_desc(s_base + OFF_W2G + p * 32768, 16384, 1024); };
    auto dG = [&](int p) { return tc::smem_desc(s_base + OFF_W2G + p * 32768 + 16384, 16384, 1024); };
    auto dX3 = [&](int p) { return tc::smem_desc(s_base + OFF_X3 + p * 8192, 16, 1024); };
    auto dX3mn = [&](int p) { return tc::smem_desc(s_base + OFF_X3 + p * 8192, 16384, 1024); };   // read MN-major
    auto dW2k = [&](int p) { return tc::smem_desc(s_base + OFF_W2G + p * 32768, 16, 1024); };     // W2 copy, K-major

    if (a.inject_timeout && warp == 0) {   // tests: a bounded wait that expires (1 ms)
        if (!tc::mbar_wait(bars + B_NEVER, 0, nullptr, 1000000ull) && lane == 0) give_up();
    }
#ifdef TTT_DEBUG_STAGES
    long long stamp_acc[32] = {};
    long long stamp_last = clock64();
#endif

    if (state_group) {
        // =====================================================================================
        // state group: warps 0-7.  Thread (q, gh, lane) owns hidden row i_loc of the i-tiles
        // and tokens t0 .. t0 + 31 of the token tiles.
        // =====================================================================================
        {   // initial state: my rows of W1 and W2^T -> tensor memory
            const int ig = (int)r_cta * MLOC + i_loc;
            const float* w1 = a.W1_0 + ((long long)h * MH + ig) * DH + t0;
            const float* w2 = a.W2_0 + (long long)h * DH * MH + ig;   // W2[j][i] at j * MH + i
            int bad = 0;
            for (int half = 0; half < 2; ++half) {
                uint32_t r1[16], r2[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    r1[k] = __float_as_uint(w1[16 * half + k]);
                    r2[k] = __float_as_uint(w2[(long long)(t0 + 16 * half + k) * MH]);
                    bad |= ((r1[k] & 0x7f800000u) == 0x7f800000u) | ((r2[k] & 0x7f800000u) == 0x7f800000u);
                }
                tc::tmem_st_32x32b_x16(tm + lane_base + TM_W1 + t0 + 16 * half, r1);
                tc::tmem_st_32x32b_x16(tm + lane_base + TM_W2T + t0 + 16 * half, r2);
            }
            if (bad) atomicOr(a.status, kStatusNonFinite);
            tc::tmem_wait_st();
        }
        if (tid == 0 && nloc > 0) {
            int y0, bc;
            chunk_rows(c_first, y0, bc);
            load_tile(&P.mapK, OFF_K, B_K, y0);
            load_tile(&P.mapQ, OFF_Q, B_Q, y0);
            load_tile(&P.mapV, OFF_V, B_V, y0);
        }
        // W2 copy (fp16 [j][i]) of my W2^T rows into the W2 rows of the listed buffers.
        auto refresh_w2 = [&](int pa, int pb) {   // my row i of the W2 copy block: j = t0 .. t0 + 31
            uint32_t u[16];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t r[16];
                tc::tmem_ld_32x32b_x16(tm + lane_base + TM_W2T + t0 + 16 * half, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int k2 = 0; k2 < 8; ++k2)
                    u[8 * half + k2] = pack_h2(__uint_as_float(r[2 * k2]), __uint_as_float(r[2 * k2 + 1]));
            }
            st_row32(sm + OFF_W2G + pa * 32768, i_loc, t0, 16384, u);
            if (pb >= 0) st_row32(sm + OFF_W2G + pb * 32768, i_loc, t0, 16384, u);
        };
        auto group_sync = [&]() -> bool {   // state warps; true if some thread saw an abort
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            const bool ab = tc::bar_sync_or(1, NG, *abort_flag != 0);
            tc::tc_fence_after();
            return ab;
        };
        uint32_t ph_a = 0, ph_s = 0, ph_y = 0, ph_p = 0, ph_u = 0, ph_k = 0, ph_q = 0, ph_v = 0;
        bool aborted = group_sync();   // the initial state is in tensor memory for the first refresh

        for (int n = 0; n < nloc && !aborted; ++n) {
            const int c = c_first + n, p = n & 1;
            int y0, bc;
            chunk_rows(c, y0, bc);
            // ---- A: A^T = W1 K^T; S = Q K^T and Aq0^T = W1 Q^T into Aq[p].  Meanwhile: W2_c into the W2
            //      rows of buffer p (for Y_c) and 1-p (for the output of chunk c-1), K^T (fp16) into X1.
            STAMP3(15);
            wait_bar(B_K, ph_k); ph_k ^= 1;
            wait_bar(B_Q, ph_q); ph_q ^= 1;
            STAMP3(0);
            if (n >= 2) wait_bar(B_ZN + p, ((n - 2) >> 1) & 1);   // output of chunk c-2 read Aq[p], W2G[p]
            STAMP3(1);
            if (bc < BT) {   // rows beyond the chunk hold other tokens (or zero fill): clear them
                float* fK = reinterpret_cast<float*>(sm + OFF_K);
                float* fQ = reinterpret_cast<float*>(sm + OFF_Q);
                for (int idx = tid; idx < (BT - bc) * DH; idx += NG) {
                    const int rr = bc + idx / DH, j = idx % DH;
                    const uint32_t o = f32_off(rr, j, ST64);
                    fK[o / 4] = 0.f;
                    fQ[o / 4] = 0.f;
                }
                if (group_sync()) break;
            }
            tc::tc_fence_after();
            // A^T first (it is on the chain), then S and Aq0 behind it on the tensor pipe: warp 1
            // issues only after warp 0 has (a barrier of the two warps orders the issue)
            if (tid == 0) {
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_tf32_ts(tm + TM_R1, tm + TM_W1 + kk * 8, kstep(dK, kk, ST64), ID_TF32, kk > 0);
                tc::mma_commit(bars + B_A);
            }
            if (warp < 2) asm volatile("bar.sync 3, 64;" ::: "memory");
            if (tid == 32) {
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_tf32_ss(tm + TM_R2, kstep(dQ, kk, ST64), kstep(dK, kk, ST64), ID_TF32, kk > 0);
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_tf32_ts(tm + TM_AQ + 64 * p, tm + TM_W1 + kk * 8, kstep(dQ, kk, ST64), ID_TF32, kk > 0);
                tc::mma_commit(bars + B_S);
            }
            STAMP3(2);
            refresh_w2(p, n >= 1 ? 1 - p : -1);
            {   // K as fp16 [t][j]: thread (t, 16 values of j): four 16-byte reads, two 16-byte writes
                const int t = tid >> 2, jb = 16 * (tid & 3);
                float v[16];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float4 f = *reinterpret_cast<const float4*>(sm + OFF_K + f32_off(t, jb + 4 * c, ST64));
                    v[4 * c] = f.x; v[4 * c + 1] = f.y; v[4 * c + 2] = f.z; v[4 * c + 3] = f.w;
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    *reinterpret_cast<uint4*>(sm + OFF_X1 + mn_chunk(t, jb + 8 * hh, 16384)) =
                        make_uint4(pack_h2(v[8 * hh], v[8 * hh + 1]), pack_h2(v[8 * hh + 2], v[8 * hh + 3]),
                                   pack_h2(v[8 * hh + 4], v[8 * hh + 5]), pack_h2(v[8 * hh + 6], v[8 * hh + 7]));
            }
            STAMP3(3);
            wait_bar(B_A, ph_a); ph_a ^= 1;
            tc::tc_fence_after();
            STAMP3(4);

            // ---- B: G = GELU(A) (fp16 into the G rows of buffer p, fp16 pairs into tensor memory as G^T);
            //      G' kept in registers
            __half2 gp[16];
            {
                uint32_t gt[16];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[16];
                    tc::tmem_ld_32x32b_x16(tm + lane_base + TM_R1 + t0 + 16 * half, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int k2 = 0; k2 < 8; ++k2) {
                        float g0, g1, d0, d1;
                        gelu_as(__uint_as_float(r[2 * k2]), g0, d0, true);
                        gelu_as(__uint_as_float(r[2 * k2 + 1]), g1, d1, true);
                        gp[8 * half + k2] = __floats2half2_rn(d0, d1);
                        gt[8 * half + k2] = pack_h2(g0, g1);
                    }
                }
                st_row32(sm + OFF_W2G + p * 32768 + 16384, i_loc, t0, 16384, gt);   // G block: row i, t0 .. t0 + 31
                tc::tmem_st_32x32b_x16(tm + lane_base + TM_GT + 16 * gh, gt);
                tc::tmem_wait_st();
            }
            STAMP3(5);
            if (group_sync()) break;
            STAMP3(6);

            // ---- C: my Y^T partial = W2_c[:, mine] G[:, mine]^T (rows 64.. of the A operand are G: unused);
            //      meanwhile the prefix mask M from S into X2 (after the Aq update of chunk c-1 read it)
            if (tid == 0) {
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16_ss(tm + TM_R1, kstep_mn(dW2G(p), kk), kstep_mn(dG(p), kk), ID_F16_MM, kk > 0);
                tc::mma_commit(bars + B_Y);
                // the output of chunk c-1 may now read W2_c beside its G: its [Z1; N] MMA queues behind Y^T
                if (n >= 1) tc::mbar_arrive(bars + B_W2R + (1 - p));
            }
            wait_bar(B_S, ph_s); ph_s ^= 1;
            if (n >= 1) wait_bar(B_AQ + (1 - p), ((n - 1) >> 1) & 1);
            tc::tc_fence_after();
            if (tid == 0 && n + 1 < nloc) {   // Q and K are free (K was converted before stage B): the next
                int ny0, nbc;                 // chunk's queries and keys
                chunk_rows(c + 1, ny0, nbc);
                load_tile(&P.mapQ, OFF_Q, B_Q, ny0);
                load_tile(&P.mapK, OFF_K, B_K, ny0);
            }
            if (q < 2) {   // M[t][s] = S[t][s] for s not after t: thread (t, 32 s)
                const int t = 32 * q + lane;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[16];
                    tc::tmem_ld_32x32b_x16(tm + lane_base + TM_R2 + t0 + 16 * half, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int c8 = 0; c8 < 2; ++c8) {
                        uint32_t u[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int s0 = t0 + 16 * half + 8 * c8 + 2 * e;
                            u[e] = pack_h2(after(s0, t) ? 0.f : __uint_as_float(r[8 * c8 + 2 * e]),
                                           after(s0 + 1, t) ? 0.f : __uint_as_float(r[8 * c8 + 2 * e + 1]));
                        }
                        *reinterpret_cast<uint4*>(sm + OFF_X2 + h_chunk(t, t0 + 16 * half + 8 * c8, 0)) =
                            make_uint4(u[0], u[1], u[2], u[3]);
                    }
                }
            }
            STAMP3(7);
            wait_bar(B_Y, ph_y); ph_y ^= 1;
            tc::tc_fence_after();
            STAMP3(8);

            // ---- D: exchange the Y^T partials; D2' = -2 eta (Y - V) as fp16 [j][t] (X3[p])
            if (n >= 2) wait_bar(B_ZD + p, ((n - 2) >> 1) & 1);   // output of chunk c-2 done with X3[p] and RZ[p]
            wait_bar(B_V, ph_v); ph_v ^= 1;                      // V is read here only
            STAMP3(9);
            if (q < 2) {
                const int j = 32 * q + lane, wx = 2 * gh + q;
                const uint32_t peer_ry = tc::mapa_shared(s_base + OFF_RY + p * 16384, r_peer);
                const uint32_t peer_bar = tc::mapa_shared(tc::smem_u32(bars + B_RY + 4 * p + wx), r_peer);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[16];
                    tc::tmem_ld_32x32b_x16(tm + lane_base + TM_R1 + t0 + 16 * half, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4)
                        tc::st_async_v4(peer_ry + ry_off(j, t0 + 16 * half + 4 * c4), r[4 * c4], r[4 * c4 + 1],
                                        r[4 * c4 + 2], r[4 * c4 + 3], peer_bar);
                }
                STAMP3(10);
                if (!tc::mbar_wait_cluster_abort(bars + B_RY + 4 * p + wx, (n >> 1) & 1, abort_flag)) give_up();
                if (lane == 0) tc::mbar_arrive_expect_tx(bars + B_RY + 4 * p + wx, RY_WARP_BYTES);   // arm chunk c+2
                STAMP3(11);
                const uint8_t* ry = sm + OFF_RY + p * 16384;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int tb = t0 + 16 * half;
                    uint32_t r[16];
                    tc::tmem_ld_32x32b_x16(tm + lane_base + TM_R1 + tb, r);
                    float d2[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) d2[k] = *reinterpret_cast<const float*>(sm + OFF_V + f32_off(tb + k, j, ST64));
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const float4 v4 = *reinterpret_cast<const float4*>(ry + ry_off(j, tb + 4 * c4));
                        const float yy[4] = {__uint_as_float(r[4 * c4]) + v4.x, __uint_as_float(r[4 * c4 + 1]) + v4.y,
                                             __uint_as_float(r[4 * c4 + 2]) + v4.z, __uint_as_float(r[4 * c4 + 3]) + v4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int k = 4 * c4 + e;
                            d2[k] = (tb + k < bc) ? -2.0f * eta * (yy[e] - d2[k]) : 0.f;
                        }
                    }
#pragma unroll
                    for (int c8 = 0; c8 < 2; ++c8)
                        *reinterpret_cast<uint4*>(sm + OFF_X3 + p * 8192 + h_chunk(j, tb + 8 * c8, 0)) =
                            make_uint4(pack_h2(d2[8 * c8], d2[8 * c8 + 1]), pack_h2(d2[8 * c8 + 2], d2[8 * c8 + 3]),
                                       pack_h2(d2[8 * c8 + 4], d2[8 * c8 + 5]), pack_h2(d2[8 * c8 + 6], d2[8 * c8 + 7]));
                }
            }
            if (group_sync()) break;
            STAMP3(12);

            // ---- E: P^T = W2^T D2'^T (my rows), fp16: the W2 copy read K-major (M = i, K = j), D2'^T MN-major
            if (tid == 0) {
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16_ss(tm + TM_R2, kstep(dW2k(p), kk, 0), kstep_mn(dX3mn(p), kk), ID_F16_KM, kk > 0);
                tc::mma_commit(bars + B_P);
                if (n + 1 < nloc) {   // V is free: fetch the next chunk's values
                    int ny0, nbc;
                    chunk_rows(c + 1, ny0, nbc);
                    load_tile(&P.mapV, OFF_V, B_V, ny0);
                }
            }
            wait_bar(B_P, ph_p); ph_p ^= 1;
            tc::tc_fence_after();
            STAMP3(13);

            // ---- F: Dl = P * G' (fp16 pairs into tensor memory as Dl^T)
            {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[16], dl[8];
                    tc::tmem_ld_32x32b_x16(tm + lane_base + TM_R2 + t0 + 16 * half, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int k2 = 0; k2 < 8; ++k2) {
                        const float2 d = __half22float2(gp[8 * half + k2]);
                        dl[k2] = pack_h2(__uint_as_float(r[2 * k2]) * d.x, __uint_as_float(r[2 * k2 + 1]) * d.y);
                    }
                    tc::tmem_st_32x32b_x8(tm + lane_base + TM_DL + 16 * gh + 8 * half, dl);
                }
                tc::tmem_wait_st();
            }
            if (group_sync()) break;

            // ---- G: W1 += Dl^T K, W2^T += G^T D2' (bar U); Aq[p]^T += Dl^T M^T (bar AQ[p], for the output group)
            if (tid == 0) {   // the state updates first (on the chain), then the output's Aq behind them
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16_ts(tm + TM_W1, tm + TM_DL + kk * 8, kstep_mn(dX1, kk), ID_F16_KM, 1);
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16_ts(tm + TM_W2T, tm + TM_GT + kk * 8, kstep(dX3(p), kk, 0), ID_F16, 1);
                tc::mma_commit(bars + B_U);
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16_ts(tm + TM_AQ + 64 * p, tm + TM_DL + kk * 8, kstep(dX2, kk, 0), ID_F16, 1);
                tc::mma_commit(bars + B_AQ + p);
            }
            STAMP3(14);
            wait_bar(B_U, ph_u); ph_u ^= 1;
            tc::tc_fence_after();
        }

        // the last chunk's output reads the final W2 beside its G
        aborted = tc::bar_sync_or(1, NG, *abort_flag != 0);
        if (!aborted && nloc > 0) {
            const int p = (nloc - 1) & 1;
            refresh_w2(p, -1);   // W2G[p] held W2 of the last chunk for its Y (done)
            if (!group_sync() && tid == 0) tc::mbar_arrive(bars + B_W2R + p);
        }
        if (!*abort_flag) {   // final state
            const int ig = (int)r_cta * MLOC + i_loc;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                const int jb = t0 + 16 * half;
                uint32_t w[16], v[16];
                tc::tmem_ld_32x32b_x16(tm + lane_base + TM_W1 + jb, w);
                tc::tmem_ld_32x32b_x16(tm + lane_base + TM_W2T + jb, v);
                tc::tmem_wait_ld();
                if (a.W1_T) {
                    float* dst = a.W1_T + ((long long)h * MH + ig) * DH + jb;
#pragma unroll
                    for (int k = 0; k < 16; ++k) dst[k] = __uint_as_float(w[k]);
                }
                if (a.W2_T) {
                    float* dst = a.W2_T + (long long)h * DH * MH + ig;
#pragma unroll
                    for (int k = 0; k < 16; ++k) dst[(long long)(jb + k) * MH] = __uint_as_float(v[k]);
                }
            }
        }
    } else {
        // =====================================================================================
        // output group: warps 8-15, the output branch of each chunk after the state group's
        // update of that chunk.  Thread (q, gh, lane) as in the state group.
        // =====================================================================================
        const int ztid = tid - NG;
        auto group_sync = [&]() -> bool {
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            const bool ab = tc::bar_sync_or(2, NG, *abort_flag != 0);
            tc::tc_fence_after();
            return ab;
        };
        uint32_t ph_corr = 0;
        // the gate: thread (token gr of my 32, channels gj .. gj + 7)
        const int gr = ztid >> 3, gj = 8 * (ztid & 7);
        float tan_a[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) tan_a[e] = a.fuse_gate ? tanhf(a.alpha[h * DH + gj + e]) : 0.f;
        int nonfinite = 0;
        for (int n = 0; n < nloc; ++n) {
            const int c = c_first + n, p = n & 1;
            int y0, bc;
            chunk_rows(c, y0, bc);
            // ---- Z1: Gq = GELU(Aq) (fp16 [t][i]); meanwhile the gate's x of my tokens -> shared memory
            if (a.fuse_gate) {   // rows y0 + 32 r .. of Xin, 64 channels of head h, 16 bytes per copy
                const int esz = a.xin_bf16 ? 2 : 4, per_row = DH * esz / 16;
                const int t_own = 32 * (int)r_cta;
                const char* xb = static_cast<const char*>(a.Xin);
                for (int u = ztid; u < 32 * per_row; u += NG) {
                    const int tr = u / per_row, piece = u % per_row;
                    if (t_own + tr < bc) {
                        const long long e0 = (long long)h * a.x_hs + (long long)(y0 + t_own + tr) * a.x_ts;
                        const uint32_t dst = s_base + OFF_XS + tr * DH * esz + piece * 16;
                        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst),
                                     "l"(xb + e0 * esz + piece * 16)
                                     : "memory");
                    }
                }
                asm volatile("cp.async.commit_group;" ::: "memory");
            }
            STAMP3(31);
            wait_bar(B_AQ + p, (n >> 1) & 1);
            tc::tc_fence_after();
            STAMP3(16);
            {
                uint32_t u[16];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[16];
                    tc::tmem_ld_32x32b_x16(tm + lane_base + TM_AQ + 64 * p + t0 + 16 * half, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int k2 = 0; k2 < 8; ++k2) {
                        float g0, g1, unused;
                        gelu_as(__uint_as_float(r[2 * k2]), g0, unused, false);
                        gelu_as(__uint_as_float(r[2 * k2 + 1]), g1, unused, false);
                        u[8 * half + k2] = pack_h2(g0, g1);
                    }
                }
                st_row32(sm + OFF_GQ, i_loc, t0, 16384, u);   // row i, t0 .. t0 + 31
            }
            STAMP3(17);
            if (group_sync()) break;
            STAMP3(18);
            // ---- Z2: my [Z1^T; N] partial = [W2_{c+1}; G_c][:, mine] Gq[:, mine]^T
            wait_bar(B_W2R + p, (n >> 1) & 1);
            tc::tc_fence_after();
            STAMP3(19);
            if (ztid == 0) {
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_f16_ss(tm + TM_ZN, kstep_mn(dW2G(p), kk), kstep_mn(dGQ, kk), ID_F16_MM, kk > 0);
                tc::mma_commit(bars + B_ZN + p);
            }
            wait_bar(B_ZN + p, (n >> 1) & 1);
            tc::tc_fence_after();
            STAMP3(20);
            // ---- Z3: -Npost[t][s] = -N[s][t] for s after t, from my partial N (lanes 64-127), into X4
            if (q >= 2) {   // row s, t0 .. t0 + 31
                const int s = i_loc - 64;
                uint32_t u[16];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int tb = t0 + 16 * half;
                    uint32_t r[16];
                    tc::tmem_ld_32x32b_x16(tm + lane_base + TM_ZN + tb, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int k2 = 0; k2 < 8; ++k2)
                        u[8 * half + k2] = pack_h2(after(s, tb + 2 * k2) ? -__uint_as_float(r[2 * k2]) : 0.f,
                                                   after(s, tb + 2 * k2 + 1) ? -__uint_as_float(r[2 * k2 + 1]) : 0.f);
                }
                st_row32(sm + OFF_X4, s, t0, 16384, u);
            }
            if (group_sync()) break;
            // ---- Z4: my z partial Z^T = Z1^T + D2'^T (-Npost)^T (rows 64.. of the A operand are unused and land
            //      on the consumed N rows)
            if (ztid == 0) {
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16_ss(tm + TM_ZN, kstep(dX3(p), kk, 0), kstep_mn(dX4, kk), ID_F16_KM, 1);
                tc::mma_commit(bars + B_CORR);
            }
            STAMP3(21);
            if (a.fuse_gate) asm volatile("cp.async.wait_all;" ::: "memory");   // my copies of x have landed
            wait_bar(B_CORR, ph_corr); ph_corr ^= 1;
            tc::tc_fence_after();
            if (a.fuse_gate && tc::bar_sync_or(2, NG, *abort_flag != 0)) break;   // everyone's x is visible
            STAMP3(22);
            // ---- Z5: z of the peer's tokens -> the peer; the peer's partial + mine for my tokens -> z
            if (q < 2) {
                const int j = 32 * q + lane;
                if (gh != (int)r_cta) {   // the peer's tokens
                    const uint32_t peer_rz = tc::mapa_shared(s_base + OFF_RZ + p * 8192, r_peer);
                    const uint32_t peer_bar = tc::mapa_shared(tc::smem_u32(bars + B_RZ + 2 * p + q), r_peer);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t r[16];
                        tc::tmem_ld_32x32b_x16(tm + lane_base + TM_ZN + t0 + 16 * half, r);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4)
                            tc::st_async_v4(peer_rz + rz_off(j, 16 * half + 4 * c4), r[4 * c4], r[4 * c4 + 1],
                                            r[4 * c4 + 2], r[4 * c4 + 3], peer_bar);
                    }
                } else if (tc::mbar_wait_cluster_abort(bars + B_RZ + 2 * p + q, (n >> 1) & 1, abort_flag)) {
                    if (lane == 0) tc::mbar_arrive_expect_tx(bars + B_RZ + 2 * p + q, RZ_WARP_BYTES);   // chunk c+2
                    uint8_t* rz = sm + OFF_RZ + p * 8192;
                    const long long base = (long long)h * a.x_hs + (long long)y0 * a.x_ts + j;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t r[16];
                        tc::tmem_ld_32x32b_x16(tm + lane_base + TM_ZN + t0 + 16 * half, r);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4) {
                            float4* slot = reinterpret_cast<float4*>(rz + rz_off(j, 16 * half + 4 * c4));
                            const float4 v4 = *slot;
                            const float4 zz = make_float4(__uint_as_float(r[4 * c4]) + v4.x,
                                                          __uint_as_float(r[4 * c4 + 1]) + v4.y,
                                                          __uint_as_float(r[4 * c4 + 2]) + v4.z,
                                                          __uint_as_float(r[4 * c4 + 3]) + v4.w);
                            if (a.fuse_gate) {   // my z, for the whole group's gate below
                                *slot = zz;
                                continue;
                            }
                            const float zv[4] = {zz.x, zz.y, zz.z, zz.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int t = t0 + 16 * half + 4 * c4 + e;
                                if (t < bc) a.Zscan[base + (long long)t * a.x_ts] = zv[e];
                            }
                        }
                    }
                } else {
                    give_up();
                }
            }
            STAMP3(23);
            if (group_sync()) break;
            if (a.fuse_gate && 32 * (int)r_cta + gr < bc) {
                // the gate out = x + tanh(alpha) z (paper notes page, "关键设计 / 门控 + 双向机制") over my 32
                // tokens, eight channels per thread with 16-byte loads and stores
                const uint8_t* rz = sm + OFF_RZ + p * 8192;
                float zv[8], xv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    zv[e] = *reinterpret_cast<const float*>(rz + rz_off(gj + e, gr & ~3) + (gr & 3) * 4);
                if (a.xin_bf16) {
                    const uint4 u = *reinterpret_cast<const uint4*>(sm + OFF_XS + (gr * DH + gj) * 2);
                    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
                        xv[2 * e] = f.x;
                        xv[2 * e + 1] = f.y;
                    }
                } else {
                    const float4* src = reinterpret_cast<const float4*>(sm + OFF_XS + (gr * DH + gj) * 4);
                    const float4 f0 = src[0], f1 = src[1];
                    xv[0] = f0.x; xv[1] = f0.y; xv[2] = f0.z; xv[3] = f0.w;
                    xv[4] = f1.x; xv[5] = f1.y; xv[6] = f1.z; xv[7] = f1.w;
                }
                float o[8], dz[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    dz[e] = tan_a[e] * zv[e];
                    o[e] = xv[e] + dz[e];
                    nonfinite |= !(isfinite(xv[e]) && isfinite(zv[e]));
                }
                const long long idx = (long long)h * a.x_hs + (long long)(y0 + 32 * (int)r_cta + gr) * a.x_ts + gj;
                auto bf2 = [](float lo, float hi) {
                    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
                    return *reinterpret_cast<const uint32_t*>(&v);
                };
                if (a.out_bf16) {
                    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.Out) + idx) =
                        make_uint4(bf2(o[0], o[1]), bf2(o[2], o[3]), bf2(o[4], o[5]), bf2(o[6], o[7]));
                } else {
                    float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.Out) + idx);
                    dst[0] = make_float4(o[0], o[1], o[2], o[3]);
                    dst[1] = make_float4(o[4], o[5], o[6], o[7]);
                }
                if (a.Delta)
                    *reinterpret_cast<uint4*>(a.Delta + idx) =
                        make_uint4(bf2(dz[0], dz[1]), bf2(dz[2], dz[3]), bf2(dz[4], dz[5]), bf2(dz[6], dz[7]));
                if (a.Zdbg) {
                    float4* dst = reinterpret_cast<float4*>(a.Zdbg + idx);
                    dst[0] = make_float4(zv[0], zv[1], zv[2], zv[3]);
                    dst[1] = make_float4(zv[4], zv[5], zv[6], zv[7]);
                }
            }
            if (a.fuse_gate && group_sync()) break;   // RZ[p] and XS are read before they are reused
            if (ztid == 0) tc::mbar_arrive(bars + B_ZD + p);
            STAMP3(24);
        }
        if (nonfinite) atomicOr(a.status, kStatusNonFinite);
    }

#ifdef TTT_DEBUG_STAGES
    if ((tid == 0 || tid == NG) && blockIdx.x == 0 && g_dbg3) {
        for (int k = (tid == 0 ? 0 : 16); k < (tid == 0 ? 16 : 32); ++k) g_dbg3[k] = (float)stamp_acc[k];
        if (tid == 0) g_dbg3[40] = (float)nloc;
    }
#endif
    // ---- both groups: leave together
    tc::tc_fence_before();
    __syncthreads();
    if (*abort_flag) {   // let copies and MMAs in flight land before the memory goes away
        const uint64_t tw = tc::globaltimer_ns();
        while (tc::globaltimer_ns() - tw < 1000000ull) __nanosleep(1000);
    }
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tm, 512);
    }
    tc::cluster_sync();   // neither CTA leaves while the peer may still write into its shared memory
}

bool make_stream_map(CUtensorMap* m, const float* base, const ScanArgs& a, bool full) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &qr) != cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
        return false;
    auto fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    cuuint64_t dims[3];
    cuuint64_t strides[2];
    cuuint32_t box[3];
    if (full) {   // element (j, h, t) at t * D + h * d + j
        dims[0] = DH; dims[1] = a.H; dims[2] = a.T;
        strides[0] = DH * 4; strides[1] = (cuuint64_t)a.qkv_ts * 4;
        box[0] = 32; box[1] = 1; box[2] = BT;
    } else {      // element (j, t, h) at (h * T + t) * d + j
        dims[0] = DH; dims[1] = a.T; dims[2] = a.H;
        strides[0] = DH * 4; strides[1] = (cuuint64_t)a.qkv_hs * 4;
        box[0] = 32; box[1] = BT; box[2] = 1;
    }
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

#ifdef TTT_DEBUG_STAGES
extern "C" __attribute__((visibility("default"))) int ttt_debug_set_dump3(float* p) {
    return (int)cudaMemcpyToSymbol(g_dbg3, &p, sizeof(p));
}
#endif

cudaError_t launch_scan_chunk_tc3(const ScanArgs& a, cudaStream_t s) {
    const int nchunks = (a.T + a.b - 1) / a.b;
    const int c_end = a.c_end > 0 ? a.c_end : nchunks;
    if (a.c_begin < 0 || c_end > nchunks || a.c_begin >= c_end) return cudaErrorInvalidValue;
    ScanTc3Args P{};
    P.a = a;
    P.full = (a.qkv_ts != DH) ? 1 : 0;
    if (!make_stream_map(&P.mapQ, a.Q, a, P.full) || !make_stream_map(&P.mapK, a.K, a, P.full) ||
        !make_stream_map(&P.mapV, a.V, a, P.full))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(scan_tc3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * a.H);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    LaunchScope scope("scan_chunk_tc3", s);
    e = cudaLaunchKernelEx(&cfg, scan_tc3_kernel, P);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace ttt
