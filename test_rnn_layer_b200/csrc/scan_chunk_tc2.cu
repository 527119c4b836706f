// Chunked TTT-MLP scan on the tcgen05 tensor cores with each head split over
// a cluster of two CTAs (d = 64, m = 256, b <= 64).
//
// CTA r of the pair owns hidden units i in [128 r, 128 r + 128): its halves of
// W1 [i][j] and W2^T [i][j] live in its tensor memory as fp32 accumulators for
// the whole sequence (A operands of the MMAs that multiply by them, updated by
// accumulate-MMAs), with a K-major copy of its W2 columns [j][i] in shared
// memory.  Every product whose contraction runs over j or over the chunk's
// tokens stays inside the CTA; the two that run over i are split and their
// partial sums exchanged through distributed shared memory:
//   Y^T  = W2 G^T           both CTAs receive the peer's [64 x 64] partial,
//                           so both form the same D2' (fp32 a + b == b + a);
//   [Z1^T; N] = [W2; G] Gq^T  kept as partials (see below); each CTA owns 32 of
//                           the 64 tokens of z and receives the peer's partial
//                           z for those columns only.
// The final z is also a sum over the pair: the masked correction is linear in N,
// so each CTA adds D2'^T Np_r^T built from its own partial N_r to its own Z1
// partial, and only the z partials for the peer's tokens cross (8 KB).  No
// later stage depends on z, so the peer's half is received and stored while
// the next chunk's first MMAs run.
// The algebra per chunk (tokens t, s of the chunk in walking order; see the
// one-CTA kernel for the derivation; paper notes page, "关键设计 / TTT-MLP 层"):
//   A^T = W1 K^T, G = GELU(A), Y^T = W2 G^T, D2' = -2 eta (Y - V),
//   P^T = W2^T D2'^T, Dl = P * GELU'(A), W1 += Dl^T K, W2^T += G^T D2',
//   Aq^T = W1_old Q^T + Dl^T M^T (M[t,s] = q_t.k_s, s not after t), Gq = GELU(Aq),
//   [Z1^T; N] = [W2_old; G] Gq^T, Z^T = Z1^T + D2'^T Np^T (Np[t,s] = N[s,t], s not after t):
//   token t sees W2_old plus the updates of the tokens up to and including t.
// The MMAs a later stage does not need at once are committed separately (the
// first stage's Aq0 and S, the update stage's W1 and W2^T), independent
// accumulators are issued by different threads, the z correction MMA is issued
// behind a barrier of only the warps that build its operand, and the shared
// copy of the updated W2 is refreshed off the chain (lanes 0-63 in the stage
// after [Z1; N], lanes 64-127 during the next chunk's first MMAs).
// The kernel stores z; the gate out = x + tanh(alpha) z is a separate
// bandwidth-bound kernel, keeping global loads off the scan's dependent chain.
// All contractions are kind::tf32 MMAs (fp32 accumulate) on K-major
// shared-memory operands with the 128-byte swizzle.  Waits are bounded.
//
// The partials travel as asynchronous 16-byte stores into the peer's shared
// memory that complete bytes on a receive barrier of the peer.  Each receiving
// warp reads exactly what one sending warp of the peer wrote, so every warp
// pair has a barrier of its own (2 KB per phase, armed by the receiving warp's
// lane 0 right after the previous phase completed).
// Ordering of the exchange buffers (no handshake needed): the peer writes my
// RY for chunk c+1 only after it received my z partial of chunk c (before a
// block barrier that precedes its Y send), which I send after I have read RY
// of chunk c; it writes my RZ for chunk c+1 only after it received my Y
// partial of chunk c+1, which I send after I have read RZ of chunk c.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc_prims.cuh"

namespace ttt {
namespace {

constexpr int BT = 64, DH = 64, MH = 256, MLOC = 128, THREADS = 512;

// Shared memory (bytes from a 1024-aligned base), 128-byte-swizzled atoms of
// 8 rows x 32 fp32 columns (atoms down the rows 1024 B apart).  A 64-row tile
// read as a 128-row MMA operand spills into the next 16 KB, hence the order.
constexpr int OFF_W2G = 0;        // 128 x 128: rows 0-63 my W2 columns [j][i], rows 64-127 G [t][i]; stride 16384
constexpr int OFF_GQ = 65536;     // 64 x 128: Gq [t][i]; stride 8192
constexpr int OFF_Q = 98304;      // 64 x 64: Q [t][j] (TMA)
constexpr int OFF_K = 114688;     // 64 x 64: K [t][j] (TMA); then D2' [t][j]
constexpr int OFF_X3 = 131072;    // 64 x 64: D2'^T [j][t]
constexpr int OFF_X1 = 147456;    // 64 x 64: K^T [j][t]; then Np [t_own][s] (32 rows)
constexpr int OFF_X2 = 163840;    // 64 x 64: M [t][s] (prefix mask)
constexpr int OFF_V = 180224;     // 64 x 64: V [t][j] (TMA)
constexpr int OFF_RY = 196608;    // 64 x 64 fp32 [j][t]: the peer's Y^T partial (ry_off)
constexpr int OFF_RZ = 212992;    // 64 x 32 fp32 [j][t_own]: the peer's z partial for my tokens (rz_off)
constexpr uint32_t XCHG_WARP_BYTES = 2048;   // each exchange: 8 warps x 2 KB each way
constexpr int OFF_BAR = 229376;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr int ST64 = 8192;

// Tensor memory (128 lanes x 32-bit columns).
constexpr uint32_t TM_W1 = 0;     // my W1 rows: [i][j]
constexpr uint32_t TM_W2T = 64;   // my W2^T rows: [i][j]
constexpr uint32_t TM_X = 128;    // A^T -> G^T: [i][t]
constexpr uint32_t TM_S = 192;    // S[t][s] (lanes t < 64)
constexpr uint32_t TM_Y = 256;    // my Y^T partial [j][t] (lanes j < 64)
constexpr uint32_t TM_P = 320;    // P^T -> Dl^T: [i][t]
constexpr uint32_t TM_ZN = 384;   // [Z1^T; N] partial: [j | s][t]
constexpr uint32_t TM_AQ = 448;   // Aq^T: [i][t]

#ifdef TTT_DEBUG_STAGES
// Debug builds only: cycles thread 0 of CTA TTT_STAMP_CTA spends between stage boundaries.
#ifndef TTT_STAMP_CTA
#define TTT_STAMP_CTA 0
#endif
__device__ float* g_dbg2 = nullptr;
#define STAMP(k)                                                      \
    do {                                                              \
        if (tid == 0 && blockIdx.x == TTT_STAMP_CTA) {                \
            const long long now_ = clock64();                         \
            stamp_acc[k] += now_ - stamp_last;                        \
            stamp_last = now_;                                        \
        }                                                             \
    } while (0)
#else
#define STAMP(k) \
    do {         \
    } while (0)
#endif

struct ScanTc2Args {
    CUtensorMap mapQ, mapK, mapV;
    ScanArgs a;
    int full;
};

// Round to the nearest tf32 value, ties away from zero: add half a unit of the
// 13 dropped mantissa bits, then clear them (a carry into the exponent is the
// correct result, infinities stay infinite).  Two integer operations.  A NaN
// may come out as zero (the GPU's NaN 0x7fffffff carries into the sign bit), so
// non-finite values are detected where they enter instead: the projections
// check Q, K, V, this kernel checks W1_0 and W2_0, the gate checks x and z.
__device__ __forceinline__ float tf32r(float x) {
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xffffe000u);
}

__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// erf-GELU (and GELU') with erf from Abramowitz & Stegun, Handbook of
// Mathematical Functions, formula 7.1.26: |error| <= 1.5e-7, far below the
// tf32 rounding the results get; GELU and GELU' share one exponential.
__device__ __forceinline__ float ex2_approx(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ void gelu_as(float a, float& g, float& gp, bool want_prime) {
    // u = 1 / (1 + p |a| / sqrt 2), the two constants folded into one
    const float u = rcp_approx(fmaf(0.3275911f * 0.70710678118654752f, fabsf(a), 1.0f));   // argument >= 1
    const float e = ex2_approx(a * (a * -0.72134752044448170f));   // exp(-a^2 / 2) = 2^(-a^2 log2(e) / 2)
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

// A K-major operand descriptor advanced to K-step kk (8 tf32 = 32 bytes per step).
__device__ __forceinline__ uint64_t kstep(uint64_t d0, int kk, uint32_t stride) {
    return d0 + (uint64_t)(((kk >> 2) * stride + (kk & 3) * 32) >> 4);
}

// Column-fixed swizzled addressing: element (R, c) at ph[R & 7] + (R >> 3) * 1024.
__device__ __forceinline__ void col_phases(int c, int stride, uint32_t (&ph)[8]) {
    const uint32_t base = (uint32_t)((c >> 5) * stride + (c & 3) * 4);
    const uint32_t cq = (uint32_t)((c & 31) >> 2);
#pragma unroll
    for (int r = 0; r < 8; ++r) ph[r] = base + r * 128 + ((cq ^ r) << 4);
}

// Byte offset of the 16-byte chunk holding columns c .. c+3 (c a multiple of 4) of row R.
__device__ __forceinline__ uint32_t row4_off(int R, int c, int stride) {
    return (uint32_t)((c >> 5) * stride + (R >> 3) * 1024 + (R & 7) * 128 + ((((c & 31) >> 2) ^ (R & 7)) << 4));
}

// Receive buffers: rows of 16-byte chunks, chunk index XOR-ed with the row so
// that 32 threads on consecutive rows hit distinct banks.  t a multiple of 4.
__device__ __forceinline__ uint32_t ry_off(int j, int t) { return (uint32_t)(j * 256 + (((t >> 2) ^ (j & 15)) << 4)); }
__device__ __forceinline__ uint32_t rz_off(int j, int t) { return (uint32_t)(j * 128 + (((t >> 2) ^ (j & 7)) << 4)); }

__device__ __forceinline__ void st4(uint8_t* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}

__global__ void __launch_bounds__(THREADS, 1) scan_tc2_kernel(const __grid_constant__ ScanTc2Args P) {
    const ScanArgs& a = P.a;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar_mma = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint64_t* bar_k = bar_mma + 1;
    uint64_t* bar_q = bar_mma + 2;
    uint64_t* bar_v = bar_mma + 3;
    uint64_t* bar_ryw = bar_mma + 10;   // [8] a peer warp's part of the Y^T partial has landed in RY
    uint64_t* bar_rzw = bar_mma + 18;   // [4] a peer warp's part of the z partial has landed in RZ
    uint64_t* bar_l = bar_mma + 26;     // the z correction MMA of the previous chunk
    uint64_t* bar_never = bar_mma + 6;   // fault injection: nothing ever arrives here
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma + 7);
    uint64_t* bar_a2 = bar_mma + 8;      // the first stage's second group (Aq0, S)
    uint64_t* bar_g2 = bar_mma + 9;      // the update stage's second group (W1, W2^T)
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, g = warp >> 2;       // TMEM lane quarter; token group (16 tokens)
    const uint32_t r_cta = tc::cluster_ctarank();
    const uint32_t r_peer = r_cta ^ 1u;
    const int i_loc = 32 * q + lane;             // my hidden row in the i-lane tiles
    const int h = blockIdx.x >> 1;
    const int T = a.T, b = a.b;
    const int nchunks = (T + b - 1) / b;
    const int c_first = a.c_begin, c_last = a.c_end > 0 ? min(a.c_end, nchunks) : nchunks;
    const float eta = a.eta;
    const bool my_tokens = (g >> 1) == (int)r_cta;   // tokens 16g .. 16g+15 belong to this CTA

    const uint32_t sW2G = tc::smem_u32(sm + OFF_W2G), sGQ = tc::smem_u32(sm + OFF_GQ);
    const uint32_t sQ = tc::smem_u32(sm + OFF_Q), sK = tc::smem_u32(sm + OFF_K);
    const uint32_t sX1 = tc::smem_u32(sm + OFF_X1), sX2 = tc::smem_u32(sm + OFF_X2);
    const uint32_t sX3 = tc::smem_u32(sm + OFF_X3);
    // the peer's receive buffers and barriers
    const uint32_t peer_ry = tc::mapa_shared(tc::smem_u32(sm + OFF_RY), r_peer);
    const uint32_t peer_rz = tc::mapa_shared(tc::smem_u32(sm + OFF_RZ), r_peer);
    // exchange warp pairs: both exchanges pair q < 2 warps (Y: all token groups, z: one token half)
    const int wx_y = 2 * g + (q & 1), wx_z = 2 * (g & 1) + (q & 1);
    const uint32_t peer_bar_ry = tc::mapa_shared(tc::smem_u32(bar_ryw + wx_y), r_peer);
    const uint32_t peer_bar_rz = tc::mapa_shared(tc::smem_u32(bar_rzw + wx_z), r_peer);

    if (tid == 0) {
        tc::mbar_init(bar_mma, 1);
        tc::mbar_init(bar_k, 1);
        tc::mbar_init(bar_q, 1);
        tc::mbar_init(bar_v, 1);
        for (int w = 0; w < 8; ++w) {   // one local arrival with expect_tx; the peer's stores complete the bytes
            tc::mbar_init(bar_ryw + w, 1);
            if (w < 4) tc::mbar_init(bar_rzw + w, 1);
        }
        tc::mbar_init(bar_never, 1);
        tc::mbar_init(bar_a2, 2);   // two issuing threads commit to each
        tc::mbar_init(bar_g2, 2);
        tc::mbar_init(bar_l, 1);
        *abort_flag = 0;
        for (int w = 0; w < 8; ++w) {   // arm phase 0 of the receive barriers
            tc::mbar_arrive_expect_tx(bar_ryw + w, XCHG_WARP_BYTES);
            if (w < 4) tc::mbar_arrive_expect_tx(bar_rzw + w, XCHG_WARP_BYTES);
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

    auto chunk_rows = [&](int c, int& y0, int& bc) {
        bc = min(b, T - c * b);
        y0 = a.reverse ? (T - c * b - bc) : c * b;
    };
    auto load_tile = [&](const CUtensorMap* map, uint32_t dst_off, uint64_t* bar, int y0) {
        tc::mbar_arrive_expect_tx(bar, BT * DH * 4);
        for (int half = 0; half < 2; ++half) {
            if (P.full) tma_load_3d(sm + dst_off + half * ST64, map, half * 32, h, y0, bar);
            else tma_load_3d(sm + dst_off + half * ST64, map, half * 32, y0, h, bar);
        }
    };
    auto after = [&](int s, int t) -> bool { return a.reverse ? (s < t) : (s > t); };

    // ---- initial state: my rows of W1 and W2^T -> tensor memory
    {
        const int j0 = 16 * g;
        const int ig = (int)r_cta * MLOC + i_loc;
        const float* w1 = a.W1_0 + ((long long)h * MH + ig) * DH + j0;
        const float* w2 = a.W2_0 + (long long)h * DH * MH + ig;   // W2[j][i] at j * MH + i
        uint32_t r1[16], r2[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            r1[k] = __float_as_uint(w1[k]);
            r2[k] = __float_as_uint(w2[(long long)(j0 + k) * MH]);
        }
        int bad = 0;
#pragma unroll
        for (int k = 0; k < 16; ++k)
            bad |= ((r1[k] & 0x7f800000u) == 0x7f800000u) | ((r2[k] & 0x7f800000u) == 0x7f800000u);
        if (bad) atomicOr(a.status, kStatusNonFinite);
        tc::tmem_st_32x32b_x16(tm + lane_base + TM_W1 + j0, r1);
        tc::tmem_st_32x32b_x16(tm + lane_base + TM_W2T + j0, r2);
        tc::tmem_wait_st();
    }
    if (tid == 0) {
        int y0, bc;
        chunk_rows(c_first, y0, bc);
        load_tile(&P.mapK, OFF_K, bar_k, y0);
        load_tile(&P.mapQ, OFF_Q, bar_q, y0);
        load_tile(&P.mapV, OFF_V, bar_v, y0);
    }

    uint32_t ph_mma = 0, ph_k = 0, ph_q = 0, ph_v = 0, ph_ry = 0, ph_rz = 0, ph_a2 = 0, ph_g2 = 0, ph_l = 0;

    constexpr uint32_t ID64 = tc::instr_desc(2, 128, 64, 0, 0);
    const uint64_t dK = tc::smem_desc(sK, 16, 1024), dQ = tc::smem_desc(sQ, 16, 1024);
    const uint64_t dW2 = tc::smem_desc(sW2G, 16, 1024), dG = tc::smem_desc(sW2G + 8192, 16, 1024);
    const uint64_t dX1 = tc::smem_desc(sX1, 16, 1024), dX2 = tc::smem_desc(sX2, 16, 1024);
    const uint64_t dX3 = tc::smem_desc(sX3, 16, 1024), dGQ = tc::smem_desc(sGQ, 16, 1024);

    // W2 [j][i] (tf32 copy, K-major) from my W2^T rows in tensor memory.
    auto refresh_w2 = [&]() {
        const int j0 = 16 * g;
        uint32_t ph[8], r[16];
        tc::tmem_ld_32x32b_x16(tm + lane_base + TM_W2T + j0, r);
        col_phases(i_loc, 16384, ph);
        uint8_t* p = sm + OFF_W2G + (j0 >> 3) * 1024;
        tc::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k)
            *reinterpret_cast<float*>(p + ph[k & 7] + (k >> 3) * 1024) = tf32r(__uint_as_float(r[k]));
    };
    refresh_w2();

#ifdef TTT_DEBUG_STAGES
    long long stamp_acc[28] = {};
    long long stamp_last = clock64();
#endif
    auto give_up = [&]() {
        *abort_flag = 1;
        atomicOr(a.status, kStatusTimeout);
    };
    // Every thread waits for an MMA group itself (no block barrier after the
    // MMAs); a thread whose wait expires raises the abort flag, which the next
    // stage's leading barrier turns into a uniform exit.
    auto wait_mma = [&](uint64_t* bar, uint32_t& ph) {
        if (!tc::mbar_wait(bar, ph, abort_flag)) give_up();
        ph ^= 1;
        tc::tc_fence_after();
    };
    // One MMA stage: all threads' operand writes become visible, the issuing
    // threads issue (and commit: the group the stage waits for goes to
    // bar_mma), `work` (touching nothing the MMAs read or write) runs meanwhile.
    // Accumulators that do not depend on one another are issued by different
    // threads (lane 0 of warps 0, 1, 2) so that their issue overlaps.
    auto mma_stage_with = [&](auto issue, auto work) -> bool {
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        if (__syncthreads_or(*abort_flag)) return false;
        tc::tc_fence_after();
        issue();
        work();
        wait_mma(bar_mma, ph_mma);
        return true;
    };
    auto mma_stage = [&](auto issue) -> bool { return mma_stage_with(issue, [] {}); };
    // A finished chunk's z for my tokens (rows y0c .. y0c + bcc - 1): my partial
    // from tensor memory plus the peer's from RZ, stored to global memory; no
    // global loads on this path (the gate x + tanh(alpha) z runs afterwards as a
    // separate elementwise kernel).  Called by all threads.
    auto store_z_chunk = [&](int y0c, int bcc) {
        if (q < 2 && my_tokens) {
            const int j = 32 * q + lane, t0 = 16 * g, tl0 = t0 - 32 * (int)r_cta;
            uint32_t r[16];
            tc::tmem_ld_32x32b_x16(tm + lane_base + TM_ZN + t0, r);
            tc::tmem_wait_ld();
            if (tc::mbar_wait_cluster(bar_rzw + wx_z, ph_rz)) {
                if (lane == 0) tc::mbar_arrive_expect_tx(bar_rzw + wx_z, XCHG_WARP_BYTES);   // arm the next phase
                float v[16];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const float4 v4 = *reinterpret_cast<const float4*>(sm + OFF_RZ + rz_off(j, tl0 + 4 * c4));
                    v[4 * c4] = __uint_as_float(r[4 * c4]) + v4.x;
                    v[4 * c4 + 1] = __uint_as_float(r[4 * c4 + 1]) + v4.y;
                    v[4 * c4 + 2] = __uint_as_float(r[4 * c4 + 2]) + v4.z;
                    v[4 * c4 + 3] = __uint_as_float(r[4 * c4 + 3]) + v4.w;
                }
                float* zrow = a.Zscan + (long long)h * a.x_hs + (long long)y0c * a.x_ts + j;
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    if (t0 + k < bcc) zrow[(long long)(t0 + k) * a.x_ts] = v[k];
            } else {
                give_up();
            }
        }
        ph_rz ^= 1;
    };
    // My partial z for the peer's tokens -> the peer's RZ (right after the chunk's last MMA).
    auto send_z_chunk = [&]() {
        if (q < 2 && !my_tokens) {
            const int j = 32 * q + lane, t0 = 16 * g, tl0 = t0 - 32 * (int)r_peer;
            uint32_t r[16];
            tc::tmem_ld_32x32b_x16(tm + lane_base + TM_ZN + t0, r);
            tc::tmem_wait_ld();
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
                tc::st_async_v4(peer_rz + rz_off(j, tl0 + 4 * c4), r[4 * c4], r[4 * c4 + 1], r[4 * c4 + 2],
                                r[4 * c4 + 3], peer_bar_rz);
        }
    };
    int prev_y0 = 0, prev_bc = 0;   // the chunk whose z is still to be stored (prev_bc == 0: none)

    if (a.inject_timeout && warp == 0) {   // tests: a bounded wait that expires (1 ms)
        if (!tc::mbar_wait(bar_never, 0, nullptr, 1000000ull) && lane == 0) give_up();
    }

    for (int c = c_first; c < c_last; ++c) {
        int y0, bc;
        chunk_rows(c, y0, bc);
        STAMP(13);
        if (warp == 0) {
            const bool ok = tc::mbar_wait(bar_k, ph_k, nullptr) && tc::mbar_wait(bar_q, ph_q, nullptr) &&
                            tc::mbar_wait(bar_v, ph_v, nullptr);
            if (!ok && lane == 0) give_up();
        }
        ph_k ^= 1;
        ph_q ^= 1;
        ph_v ^= 1;
        if (bc < BT) {   // rows beyond the chunk hold other tokens (or zero fill): clear them
            __syncthreads();
            float* fK = reinterpret_cast<float*>(sm + OFF_K);
            float* fQ = reinterpret_cast<float*>(sm + OFF_Q);
            for (int idx = tid; idx < (BT - bc) * DH; idx += THREADS) {
                const int rr = bc + idx / DH, j = idx % DH;
                const uint32_t o = row4_off(rr, j & ~3, ST64) + (j & 3) * 4;
                fK[o / 4] = 0.f;
                fQ[o / 4] = 0.f;
            }
        }

        STAMP(0);
        // ---- A: A^T = W1 K^T (my rows); then Aq0^T = W1 Q^T, S = Q K^T (bar_a2).  Meanwhile:
        //      the previous chunk's z out, K^T into X1 (nothing later in the chunk writes K or X1
        //      before a block barrier)
        if (!mma_stage_with(
                [&] {
                    if (tid == 0) {
                        for (int kk = 0; kk < 8; ++kk)
                            tc::mma_tf32_ts(tm + TM_X, tm + TM_W1 + kk * 8, kstep(dK, kk, ST64), ID64, kk > 0);
                        tc::mma_commit(bar_mma);
                        STAMP(14);
                    } else if (tid == 32) {
                        for (int kk = 0; kk < 8; ++kk)
                            tc::mma_tf32_ts(tm + TM_AQ, tm + TM_W1 + kk * 8, kstep(dQ, kk, ST64), ID64, kk > 0);
                        tc::mma_commit(bar_a2);
                    } else if (tid == 64) {
                        for (int kk = 0; kk < 8; ++kk)
                            tc::mma_tf32_ss(tm + TM_S, kstep(dQ, kk, ST64), kstep(dK, kk, ST64), ID64, kk > 0);
                        tc::mma_commit(bar_a2);
                    }
                },
                [&] {
                    if (prev_bc) {   // the previous chunk's z correction has run: send the peer its half
                        wait_mma(bar_l, ph_l);
                        send_z_chunk();
                    }
                    {   // K^T: thread (j, 8 tokens): column reads of K, two 16-byte row writes of K^T
                        const int j = tid & 63, tb = tid >> 6;
                        uint32_t ph[8];
                        col_phases(j, ST64, ph);
                        const uint8_t* src = sm + OFF_K + tb * 1024;
                        float v[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) v[e] = *reinterpret_cast<const float*>(src + ph[e]);
                        st4(sm + OFF_X1 + row4_off(j, 8 * tb, ST64), v[0], v[1], v[2], v[3]);
                        st4(sm + OFF_X1 + row4_off(j, 8 * tb + 4, ST64), v[4], v[5], v[6], v[7]);
                    }
                    if (q >= 2) refresh_w2();   // the other half of the W2 copy (lanes 0-63 refreshed in K)
                    if (prev_bc) store_z_chunk(prev_y0, prev_bc);   // + the peer's half, for my tokens
                }))
            break;
        prev_bc = 0;

        STAMP(1);
        // ---- B: G = GELU(A) to shared [t][i] and in place (G^T); G' kept
        __half2 gp[8];
        {
            const int t0 = 16 * g;
            uint32_t ph[8], r[16];
            const uint32_t addr = tm + lane_base + TM_X + t0;
            tc::tmem_ld_32x32b_x16(addr, r);
            col_phases(i_loc, 16384, ph);
            uint8_t* p = sm + OFF_W2G + ((64 + t0) >> 3) * 1024;
            tc::tmem_wait_ld();
#pragma unroll
            for (int k2 = 0; k2 < 8; ++k2) {
                const int k = 2 * k2;
                float g0, g1, d0, d1;
                gelu_as(__uint_as_float(r[k]), g0, d0, true);
                gelu_as(__uint_as_float(r[k + 1]), g1, d1, true);
                gp[k2] = __floats2half2_rn(d0, d1);
                g0 = tf32r(g0);
                g1 = tf32r(g1);
                *reinterpret_cast<float*>(p + ph[k & 7] + (k >> 3) * 1024) = g0;
                *reinterpret_cast<float*>(p + ph[(k + 1) & 7] + ((k + 1) >> 3) * 1024) = g1;
                r[k] = __float_as_uint(g0);
                r[k + 1] = __float_as_uint(g1);
            }
            tc::tmem_st_32x32b_x16(addr, r);
        }
        tc::tmem_wait_st();

        STAMP(2);
        // ---- C: my Y^T partial = W2[:, mine] G[:, mine]^T  (rows 64.. of the A operand are unused);
        //      meanwhile the prefix mask M from S (the next stage writes neither S nor X2)
        if (!mma_stage_with(
                [&] {
                    if (tid == 0) {
                        for (int kk = 0; kk < 16; ++kk)
                            tc::mma_tf32_ss(tm + TM_Y, kstep(dW2, kk, 16384), kstep(dG, kk, 16384), ID64, kk > 0);
                        tc::mma_commit(bar_mma);
                        STAMP(15);
                    }
                },
                [&] {
                    wait_mma(bar_a2, ph_a2);   // S is ready; Q and K are no longer read
                    if (tid == 0 && c + 1 < c_last) {   // Q is free: fetch the next chunk's queries
                        int ny0, nbc;
                        chunk_rows(c + 1, ny0, nbc);
                        load_tile(&P.mapQ, OFF_Q, bar_q, ny0);
                    }
                    if (q < 2) {   // M[t][s] = S[t][s] for s not after t (prefix)
                        const int t = 32 * q + lane, s0 = 16 * g;
                        uint32_t r[16];
                        tc::tmem_ld_32x32b_x16(tm + lane_base + TM_S + s0, r);
                        tc::tmem_wait_ld();
                        float m[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k) m[k] = after(s0 + k, t) ? 0.f : tf32r(__uint_as_float(r[k]));
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4)
                            st4(sm + OFF_X2 + row4_off(t, s0 + 4 * c4, ST64), m[4 * c4], m[4 * c4 + 1], m[4 * c4 + 2],
                                m[4 * c4 + 3]);
                    }
                }))
            break;

        STAMP(3);
        // ---- D: exchange the Y^T partials; D2' = -2 eta (Y - V) as [t][j] (over K) and [j][t]
        if (q < 2) {
            const int j = 32 * q + lane, t0 = 16 * g;
            uint32_t r[16], ph[8];
            tc::tmem_ld_32x32b_x16(tm + lane_base + TM_Y + t0, r);
            tc::tmem_wait_ld();
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
                tc::st_async_v4(peer_ry + ry_off(j, t0 + 4 * c4), r[4 * c4], r[4 * c4 + 1], r[4 * c4 + 2], r[4 * c4 + 3],
                                peer_bar_ry);
            col_phases(j, ST64, ph);
            const uint32_t rg = (t0 >> 3) * 1024;
            STAMP(20);
            float vv[16];   // V first: no load waits behind a store below
#pragma unroll
            for (int k = 0; k < 16; ++k)
                vv[k] = *reinterpret_cast<const float*>(sm + OFF_V + rg + ph[k & 7] + (k >> 3) * 1024);
            if (!tc::mbar_wait_cluster(bar_ryw + wx_y, ph_ry)) give_up();
            STAMP(21);
            if (lane == 0) tc::mbar_arrive_expect_tx(bar_ryw + wx_y, XCHG_WARP_BYTES);   // arm the next phase
            STAMP(24);
            float ry[16];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const float4 v4 = *reinterpret_cast<const float4*>(sm + OFF_RY + ry_off(j, t0 + 4 * c4));
                ry[4 * c4] = v4.x;
                ry[4 * c4 + 1] = v4.y;
                ry[4 * c4 + 2] = v4.z;
                ry[4 * c4 + 3] = v4.w;
            }
            STAMP(25);
            float d2[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float y = __uint_as_float(r[k]) + ry[k];
                d2[k] = (t0 + k < bc) ? tf32r(-2.0f * eta * (y - vv[k])) : 0.f;
            }
#pragma unroll
            for (int k = 0; k < 16; ++k)
                *reinterpret_cast<float*>(sm + OFF_K + rg + ph[k & 7] + (k >> 3) * 1024) = d2[k];
            STAMP(26);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
                st4(sm + OFF_X3 + row4_off(j, t0 + 4 * c4, ST64), d2[4 * c4], d2[4 * c4 + 1], d2[4 * c4 + 2],
                    d2[4 * c4 + 3]);
        }
        ph_ry ^= 1;

        STAMP(4);
        // ---- E: P^T = W2^T D2'^T (my rows)
        if (!mma_stage([&] {
                if (tid == 0) {
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ts(tm + TM_P, tm + TM_W2T + kk * 8, kstep(dK, kk, ST64), ID64, kk > 0);
                    tc::mma_commit(bar_mma);
                    STAMP(16);
                }
            }))
            break;
        if (tid == 0 && c + 1 < c_last) {   // K and V buffers are free: fetch the next chunk's tiles
            int ny0, nbc;
            chunk_rows(c + 1, ny0, nbc);
            load_tile(&P.mapK, OFF_K, bar_k, ny0);
            load_tile(&P.mapV, OFF_V, bar_v, ny0);
        }

        STAMP(5);
        // ---- F: Dl = P * G' in place
        {
            const uint32_t addr = tm + lane_base + TM_P + 16 * g;
            uint32_t r[16];
            tc::tmem_ld_32x32b_x16(addr, r);
            tc::tmem_wait_ld();
#pragma unroll
            for (int k2 = 0; k2 < 8; ++k2) {
                const float2 d = __half22float2(gp[k2]);
                r[2 * k2] = __float_as_uint(tf32r(__uint_as_float(r[2 * k2]) * d.x));
                r[2 * k2 + 1] = __float_as_uint(tf32r(__uint_as_float(r[2 * k2 + 1]) * d.y));
            }
            tc::tmem_st_32x32b_x16(addr, r);
            tc::tmem_wait_st();
        }

        STAMP(6);
        // ---- G: Aq^T += Dl^T M^T (waited for); then W1 += Dl^T K, W2^T += G^T D2' (bar_g2)
        if (!mma_stage([&] {
                if (tid == 0) {
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ts(tm + TM_AQ, tm + TM_P + kk * 8, kstep(dX2, kk, ST64), ID64, 1);
                    tc::mma_commit(bar_mma);
                    STAMP(17);
                } else if (tid == 32) {
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ts(tm + TM_W1, tm + TM_P + kk * 8, kstep(dX1, kk, ST64), ID64, 1);
                    tc::mma_commit(bar_g2);
                } else if (tid == 64) {
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ts(tm + TM_W2T, tm + TM_X + kk * 8, kstep(dX3, kk, ST64), ID64, 1);
                    tc::mma_commit(bar_g2);
                }
            }))
            break;

        STAMP(8);
        // ---- I: Gq = GELU(Aq) to shared [t][i]
        {
            const int t0 = 16 * g;
            uint32_t ph[8], r[16];
            tc::tmem_ld_32x32b_x16(tm + lane_base + TM_AQ + t0, r);
            col_phases(i_loc, ST64, ph);
            uint8_t* p = sm + OFF_GQ + (t0 >> 3) * 1024;
            tc::tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                float gg, unused;
                gelu_as(__uint_as_float(r[k]), gg, unused, false);
                *reinterpret_cast<float*>(p + ph[k & 7] + (k >> 3) * 1024) = tf32r(gg);
            }
        }

        STAMP(9);
        // ---- J: my [Z1^T; N] partial = [W2; G][:, mine] Gq[:, mine]^T
        //      meanwhile: the W1 and W2^T updates have landed (X1 is rewritten next, W2^T read in L)
        if (!mma_stage_with(
                [&] {
                    if (tid == 0) {
                        for (int kk = 0; kk < 16; ++kk)
                            tc::mma_tf32_ss(tm + TM_ZN, kstep(dW2, kk, 16384), kstep(dGQ, kk, ST64), ID64, kk > 0);
                        tc::mma_commit(bar_mma);
                        STAMP(18);
                    }
                },
                [&] { wait_mma(bar_g2, ph_g2); }))
            break;

        STAMP(10);
        // ---- K: Np_r[t][s] = N_r[s][t] for s not after t, from my partial N_r (rows 64-127), all
        //      tokens, into X2 (M is consumed).  Then the z correction, my partial Z^T += D2'^T Np_r^T
        //      (rows 64.. of the A operand are unused and land on the consumed N rows), is issued by
        //      one of these warps after a barrier of the eight alone: no later stage of the chain
        //      needs z, so the block moves on to the next chunk while it runs (bar_l).
        if (q < 2) {
            refresh_w2();   // my lanes' part of the W2 update (landed, see J) into the copy stage C reads
        } else {
            const int t0 = 16 * g, s = i_loc - 64;
            uint32_t r[16], ph[8];
            tc::tmem_ld_32x32b_x16(tm + lane_base + TM_ZN + t0, r);
            col_phases(s, ST64, ph);
            uint8_t* p = sm + OFF_X2 + (t0 >> 3) * 1024;
            tc::tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k)
                *reinterpret_cast<float*>(p + ph[k & 7] + (k >> 3) * 1024) =
                    after(s, t0 + k) ? 0.f : tf32r(__uint_as_float(r[k]));
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            asm volatile("bar.sync 1, 256;" ::: "memory");   // the eight q >= 2 warps
            if (tid == 64) {
                tc::tc_fence_after();
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_tf32_ss(tm + TM_ZN, kstep(dX3, kk, ST64), kstep(dX2, kk, ST64), ID64, 1);
                tc::mma_commit(bar_l);
            }
        }
        STAMP(11);
        prev_y0 = y0;
        prev_bc = bc;

        STAMP(12);
    }

    if (prev_bc && !*abort_flag) {   // the last chunk's z
        wait_mma(bar_l, ph_l);
        send_z_chunk();
        store_z_chunk(prev_y0, prev_bc);
    }

#ifdef TTT_DEBUG_STAGES
    if (tid == 0 && blockIdx.x == TTT_STAMP_CTA && g_dbg2) {
        for (int k = 0; k < 28; ++k) g_dbg2[k] = (float)stamp_acc[k];
        g_dbg2[30] = (float)(c_last - c_first);
    }
#endif
    if (*abort_flag) {
        const uint64_t t0 = tc::globaltimer_ns();
        while (tc::globaltimer_ns() - t0 < 1000000ull) __nanosleep(1000);
    } else {
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
        const int j0 = 16 * g;
        const int ig = (int)r_cta * MLOC + i_loc;
        uint32_t w[16], v[16];
        tc::tmem_ld_32x32b_x16(tm + lane_base + TM_W1 + j0, w);
        tc::tmem_ld_32x32b_x16(tm + lane_base + TM_W2T + j0, v);
        tc::tmem_wait_ld();
        if (a.W1_T) {
            float* dst = a.W1_T + ((long long)h * MH + ig) * DH + j0;
#pragma unroll
            for (int k = 0; k < 16; ++k) dst[k] = __uint_as_float(w[k]);
        }
        if (a.W2_T) {
            float* dst = a.W2_T + (long long)h * DH * MH + ig;
#pragma unroll
            for (int k = 0; k < 16; ++k) dst[(long long)(j0 + k) * MH] = __uint_as_float(v[k]);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
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
extern "C" __attribute__((visibility("default"))) int ttt_debug_set_dump2(float* p) {
    return (int)cudaMemcpyToSymbol(g_dbg2, &p, sizeof(p));
}
#endif

cudaError_t launch_scan_chunk_tc2(const ScanArgs& a, cudaStream_t s) {
    const int nchunks = (a.T + a.b - 1) / a.b;
    const int c_end = a.c_end > 0 ? a.c_end : nchunks;
    if (a.c_begin < 0 || c_end > nchunks || a.c_begin >= c_end) return cudaErrorInvalidValue;
    ScanTc2Args P{};
    P.a = a;
    P.full = (a.qkv_ts != DH) ? 1 : 0;
    if (!make_stream_map(&P.mapQ, a.Q, a, P.full) || !make_stream_map(&P.mapK, a.K, a, P.full) ||
        !make_stream_map(&P.mapV, a.V, a, P.full))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(scan_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
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
    LaunchScope scope("scan_chunk_tc2", s);
    e = cudaLaunchKernelEx(&cfg, scan_tc2_kernel, P);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace ttt
