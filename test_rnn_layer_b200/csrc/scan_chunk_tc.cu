// Chunked TTT-MLP scan on the tcgen05 tensor cores (d = 64, m = 256, b <= 64).
//
// One CTA (16 warps) per head.  The hidden state stays on chip for the whole
// sequence, in tensor memory as fp32 accumulators: W1 [i][j] and W2^T [i][j]
// (i: hidden unit, 256 lanes in two halves; j: head channel).  Both serve
// directly as the A operand of the MMAs that multiply by them, and the state
// updates are accumulate-MMAs into them.  A K-major copy of W2 [j][i] in
// shared memory (refreshed each chunk) is the A operand of W2 x products.
//
// Each chunk of bc <= b tokens is a 64-row tile (rows beyond bc are zero and
// contribute nothing).  Every gradient is taken at the chunk-start state and
// token t is read with the prefix state (paper notes page, "关键设计 / TTT-MLP
// 层", mini-batch reading).  With t, s tokens of the chunk in walking order:
//   A^T  = W1 K^T,  G = GELU(A),  G' = GELU'(A)
//   Y^T  = W2 G^T,  D2' = -2 eta (Y - V)                    (-eta dl/dy)
//   P^T  = W2^T D2'^T,  Dl = P * G'                         (-eta delta)
//   W1  += Dl^T K,   W2^T += G^T D2'                        (state update)
//   Aq^T = W1_new Q^T + Dl^T M^T,   M[t,s] = -q_t.k_s for s after t
//   [Z1^T; N] = [W2_new; G] Gq^T,   Gq = GELU(Aq)            (one M = 128 MMA)
//   Z^T  = Z1^T + D2'^T Nm^T,       Nm[t,s] = -N[s,t] for s after t
// (W_new minus the contributions of the tokens after t is the prefix state
// W_t).  All contractions are kind::tf32 MMAs with fp32 accumulation; every
// shared-memory operand is K-major with the 128-byte swizzle; operands the
// threads write are rounded to tf32 first.  The gate x + tanh(alpha) z is
// applied in the final store.
//
// Stages are bulk-synchronous: threads write operands, one thread issues the
// MMAs and commits them to an mbarrier, all threads wait (bounded) and read
// the results from tensor memory.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc_prims.cuh"

namespace ttt {
namespace {

constexpr int BT = 64, DH = 64, MH = 256, THREADS = 512;

// Shared memory (bytes from a 1024-aligned base).  Every matrix is stored as
// 128-byte-swizzled atoms of 8 rows x 32 fp32 columns; atoms down the rows are
// 1024 B apart, atom columns `stride` bytes apart.  The order matters where a
// 64-row operand is read as a 128-row one (the extra rows then fall inside
// the next buffer and only produce unused output rows).
constexpr int OFF_W2G = 0;        // 128 x 256: rows 0-63 W2 [j][i] (tf32 copy), rows 64-127 G [t][i]; stride 16384
constexpr int OFF_GQ = 131072;    // 32 x 256: half of Gq [t][i], stride 4096 (stages I/J); it spans:
constexpr int OFF_V = 131072;     //   64 x 64: V [t][j] (TMA, prefetched a chunk ahead; dead after stage D)
constexpr int OFF_X2 = 147456;    //   64 x 64: M [t][s] (dead after stage H)
constexpr int OFF_Q = 163840;     // 64 x 64: Q [t][j] (TMA); read as 128 rows -> needs the next 16 KB
constexpr int OFF_K = 180224;     // 64 x 64: K [t][j] (TMA); then D2' [t][j]
constexpr int OFF_X3 = 196608;    // 64 x 64: D2'^T [j][t]; read as 128 rows -> needs the next 16 KB
constexpr int OFF_X1 = 212992;    // 64 x 64: K^T [j][t]; then Nm [t][s]
constexpr int OFF_BAR = 229376;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr int ST64 = 8192;        // atom-column stride of the 64 x 64 tiles

// Tensor-memory columns (128 lanes each).
constexpr uint32_t TM_W1 = 0;     // W1 half h: cols h*64 + j
constexpr uint32_t TM_W2T = 128;  // W2^T half h: cols 128 + h*64 + j
constexpr uint32_t TM_X = 256;    // A^T -> G^T -> Aq^T: half h at 256 + h*64 + t
constexpr uint32_t TM_S = 384;    // S[t][s] (lanes t < 64)
constexpr uint32_t TM_Y = 448;    // Y^T[j][t] (lanes j < 64)
constexpr uint32_t TM_P = 384;    // P^T -> Dl^T: half h at 384 + h*64 + t
constexpr uint32_t TM_ZN = 384;   // [Z1^T; N] at 384 + t

struct ScanTcArgs {
    CUtensorMap mapQ, mapK, mapV;
    ScanArgs a;
    int full;   // 1: streams are [T, H*d]; 0: [H, T, d]
};

__device__ __forceinline__ uint32_t sw_off(int R, int c, int stride) {
    return (uint32_t)((c >> 5) * stride + (R >> 3) * 1024 + (R & 7) * 128 + ((((c & 31) >> 2) ^ (R & 7)) << 4) +
                      ((c & 3) << 2));
}

#if defined(TTT_DEBUG_DUMP) || defined(TTT_DEBUG_STAGES)
// Debug builds only: TTT_DEBUG_DUMP copies head 0, chunk 0 intermediates to
// g_dbg (regions of 16384 floats, row-major); TTT_DEBUG_STAGES accumulates the
// cycles thread 0 of CTA 0 spends between stage boundaries.
__device__ float* g_dbg = nullptr;
#endif
#ifdef TTT_DEBUG_DUMP
enum { DBG_AT = 0, DBG_S, DBG_YT, DBG_PT, DBG_W1, DBG_DW2T, DBG_AQT, DBG_ZN, DBG_Z, DBG_D2T, DBG_G, DBG_N };
#define DBG(region, row, col, ncol, val)                                                                       \
    do {                                                                                                       \
        if (g_dbg && blockIdx.x == 0 && c == 0) g_dbg[(region) * 16384 + (row) * (ncol) + (col)] = (val);     \
    } while (0)
#else
#define DBG(region, row, col, ncol, val) \
    do {                                 \
    } while (0)
#endif
#ifdef TTT_DEBUG_STAGES
#define STAMP(k)                                                      \
    do {                                                              \
        if (tid == 0 && blockIdx.x == 0) {                            \
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

// Round to the nearest tf32 value, ties away from zero: add half a unit of the
// 13 dropped mantissa bits, then clear them (a carry into the exponent is the
// correct result, infinities stay infinite).  NaN is passed through as it is:
// the GPU's NaN 0x7fffffff would carry into the sign bit.
__device__ __forceinline__ float tf32r(float x) {
    const float r = __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xffffe000u);
    return x != x ? x : r;
}

__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// erf-GELU and its derivative with erf from Abramowitz & Stegun, Handbook of
// Mathematical Functions, formula 7.1.26 (after Hastings): for x >= 0,
// erf(x) = 1 - (a1 u + a2 u^2 + a3 u^3 + a4 u^4 + a5 u^5) exp(-x^2), u = 1/(1 + p x),
// |error| <= 1.5e-7 -- far below the tf32 rounding (2^-11) the results get.
// With x = |a|/sqrt(2), exp(-x^2) = exp(-a^2/2) is also the normal density's
// exponential, so GELU and GELU' share one exponential and one reciprocal.
__device__ __forceinline__ void gelu_as(float a, float& g, float& gp, bool want_prime) {
    const float x = fabsf(a) * 0.70710678118654752f;
    const float u = rcp_approx(fmaf(0.3275911f, x, 1.0f));   // argument >= 1
    const float e = __expf(-0.5f * a * a);
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

// A K-major operand descriptor advanced to K-step kk (8 tf32 = 32 bytes per step): only the start-address field (low
// bits, 16-byte units) changes, and it cannot carry out of its 14 bits.
__device__ __forceinline__ uint64_t kstep(uint64_t d0, int kk, uint32_t stride) {
    return d0 + (uint64_t)(((kk >> 2) * stride + (kk & 3) * 32) >> 4);
}

// Swizzled addressing for a thread that owns one column c and walks down the
// rows: element (R, c) sits at ph[R & 7] + (R >> 3) * 1024, so the eight row
// phases are computed once instead of per element.
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

__device__ __forceinline__ void st4(uint8_t* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}

__global__ void __launch_bounds__(THREADS, 1) scan_tc_kernel(const __grid_constant__ ScanTcArgs P) {
    const ScanArgs& a = P.a;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* fK = reinterpret_cast<float*>(sm + OFF_K);
    float* fQ = reinterpret_cast<float*>(sm + OFF_Q);
    uint64_t* bar_mma = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint64_t* bar_k = bar_mma + 1;
    uint64_t* bar_q = bar_mma + 2;
    uint64_t* bar_v = bar_mma + 3;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, g = warp >> 2;   // TMEM lane quarter; group of 4 warps
    const int hh = g >> 1;                   // hidden half handled in the i-lane stages
    const int i_row = hh * 128 + 32 * q + lane;
    const int h = blockIdx.x;
    const int T = a.T, b = a.b;
    const int nchunks = (T + b - 1) / b;
    const float eta = a.eta;

    const uint32_t sW2G = tc::smem_u32(sm + OFF_W2G), sGQ = tc::smem_u32(sm + OFF_GQ);
    const uint32_t sQ = tc::smem_u32(sm + OFF_Q), sK = tc::smem_u32(sm + OFF_K);
    const uint32_t sX1 = tc::smem_u32(sm + OFF_X1), sX2 = tc::smem_u32(sm + OFF_X2);
    const uint32_t sX3 = tc::smem_u32(sm + OFF_X3);

    if (tid == 0) {
        tc::mbar_init(bar_mma, 1);
        tc::mbar_init(bar_k, 1);
        tc::mbar_init(bar_q, 1);
        tc::mbar_init(bar_v, 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
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
    // s comes after t in walking order (rows are natural token order)
    auto after = [&](int s, int t) -> bool { return a.reverse ? (s < t) : (s > t); };

    // ---- initial state: W1, W2^T -> tensor memory
    {
        const int j0 = 32 * (g & 1);
        const float* w1 = a.W1_0 + ((long long)h * MH + i_row) * DH + j0;
        const float* w2 = a.W2_0 + (long long)h * DH * MH + i_row;   // W2[j][i] at j * MH + i
        for (int part = 0; part < 2; ++part) {
            uint32_t r1[16], r2[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                r1[k] = __float_as_uint(w1[part * 16 + k]);
                r2[k] = __float_as_uint(w2[(long long)(j0 + part * 16 + k) * MH]);
            }
            tc::tmem_st_32x32b_x16(tm + lane_base + TM_W1 + hh * 64 + j0 + part * 16, r1);
            tc::tmem_st_32x32b_x16(tm + lane_base + TM_W2T + hh * 64 + j0 + part * 16, r2);
        }
        tc::tmem_wait_st();
    }
    if (tid == 0) {
        int y0, bc;
        chunk_rows(0, y0, bc);
        load_tile(&P.mapK, OFF_K, bar_k, y0);
        load_tile(&P.mapQ, OFF_Q, bar_q, y0);
        load_tile(&P.mapV, OFF_V, bar_v, y0);
    }

    float tanh_a = 0.f;
    if (q < 2) tanh_a = tanhf(a.alpha[h * DH + 32 * q + lane]);
    int nonfinite = 0;
    uint32_t ph_mma = 0, ph_k = 0, ph_q = 0, ph_v = 0;

    constexpr uint32_t ID64 = tc::instr_desc(2, 128, 64, 0, 0);
    const uint64_t dK = tc::smem_desc(sK, 16, 1024), dQ = tc::smem_desc(sQ, 16, 1024);
    const uint64_t dW2 = tc::smem_desc(sW2G, 16, 1024), dG = tc::smem_desc(sW2G + 8192, 16, 1024);
    const uint64_t dX1 = tc::smem_desc(sX1, 16, 1024), dX2 = tc::smem_desc(sX2, 16, 1024);
    const uint64_t dX3 = tc::smem_desc(sX3, 16, 1024), dGQ = tc::smem_desc(sGQ, 16, 1024);
    constexpr uint32_t ID32 = tc::instr_desc(2, 128, 32, 0, 0);

    // W2 [j][i] (tf32 copy, K-major) from the W2^T master in tensor memory.
    auto refresh_w2 = [&]() {
        const int j0 = 32 * (g & 1);
        uint32_t ph[8];
        col_phases(i_row, 16384, ph);
        uint8_t* p = sm + OFF_W2G + (j0 >> 3) * 1024;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            uint32_t r[16];
            tc::tmem_ld_32x32b_x16(tm + lane_base + TM_W2T + hh * 64 + j0 + 16 * hf, r);
            tc::tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int kk = 16 * hf + k;
                *reinterpret_cast<float*>(p + ph[kk & 7] + (kk >> 3) * 1024) = tf32r(__uint_as_float(r[k]));
            }
        }
    };
    refresh_w2();

#ifdef TTT_DEBUG_STAGES
    long long stamp_acc[20] = {};
    long long stamp_last = clock64();
#endif
    // One bulk-synchronous MMA stage.  Returns false (uniformly) once a wait has expired.
    auto mma_stage = [&](auto issue) -> bool {
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
#ifdef TTT_DEBUG_STAGES
        long long t_a = clock64();
#endif
        if (__syncthreads_or(*abort_flag)) return false;
#ifdef TTT_DEBUG_STAGES
        long long t_b = clock64();
#endif
        // Only warp 0 issues and waits; the other warps park in the hardware
        // barrier below instead of spinning on the mbarrier (spinning warps
        // starve the issue slots and the load/store pipe of the working ones).
        if (warp == 0) {
            if (lane == 0) {
                tc::tc_fence_after();
                issue();
                tc::mma_commit(bar_mma);
            }
            __syncwarp();
#ifdef TTT_DEBUG_STAGES
            long long t_c = clock64();
#endif
            const bool waited = tc::mbar_wait(bar_mma, ph_mma, nullptr);
#ifdef TTT_DEBUG_STAGES
            if (tid == 0 && blockIdx.x == 0) {
                const long long t_d = clock64();
                stamp_acc[16] += t_b - t_a;
                stamp_acc[17] += t_c - t_b;
                stamp_acc[18] += t_d - t_c;
            }
#endif
            if (!waited && lane == 0) {
                *abort_flag = 1;
                atomicOr(a.status, kStatusTimeout);
            }
        }
        ph_mma ^= 1;
        const int stop = __syncthreads_or(*abort_flag);
        tc::tc_fence_after();
        return !stop;
    };

    for (int c = 0; c < nchunks; ++c) {
        int y0, bc;
        chunk_rows(c, y0, bc);
        STAMP(14);
        if (warp == 0) {   // the tiles' arrival is published to the other warps by the next barrier
            const bool ok = tc::mbar_wait(bar_k, ph_k, nullptr) && tc::mbar_wait(bar_q, ph_q, nullptr) &&
                            tc::mbar_wait(bar_v, ph_v, nullptr);
            if (!ok && lane == 0) {
                *abort_flag = 1;
                atomicOr(a.status, kStatusTimeout);
            }
        }
        ph_k ^= 1;
        ph_q ^= 1;
        ph_v ^= 1;
        STAMP(15);
        if (bc < BT) {   // rows beyond the chunk hold other tokens (or zero fill): clear them
            __syncthreads();
            for (int idx = tid; idx < (BT - bc) * DH; idx += THREADS) {
                const int r = bc + idx / DH, j = idx % DH;
                fK[sw_off(r, j, ST64) / 4] = 0.f;
                fQ[sw_off(r, j, ST64) / 4] = 0.f;
            }
        }

        STAMP(0);
        // ---- stage A: A^T = W1 K^T;  S = Q K^T
        if (!mma_stage([&] {
                for (int x = 0; x < 2; ++x)
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ts(tm + TM_X + x * 64, tm + TM_W1 + x * 64 + kk * 8, kstep(dK, kk, ST64), ID64,
                                        kk > 0);
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_tf32_ss(tm + TM_S, kstep(dQ, kk, ST64), kstep(dK, kk, ST64), ID64, kk > 0);
            }))
            break;

        STAMP(1);
        // ---- stage B (threads): G = GELU(A) to shared [t][i] and to tensor memory (G^T), keep G';
        //      K^T copy; M[t][s] = -S[t][s] for s after t
        __half2 gp[16];   // GELU'(A): |values| < 1.2, kept at fp16 (the same 11-bit significand as tf32)
        {
            const int t0 = 32 * (g & 1);
            uint32_t ph[8];
            col_phases(i_row, 16384, ph);
            uint8_t* p = sm + OFF_W2G + ((64 + t0) >> 3) * 1024;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint32_t addr = tm + lane_base + TM_X + hh * 64 + t0 + 16 * hf;
                uint32_t r[16];
                tc::tmem_ld_32x32b_x16(addr, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int k2 = 0; k2 < 8; ++k2) {
                    const int k = 16 * hf + 2 * k2;
                    DBG(DBG_AT, i_row, t0 + k, 64, __uint_as_float(r[2 * k2]));
                    DBG(DBG_AT, i_row, t0 + k + 1, 64, __uint_as_float(r[2 * k2 + 1]));
                    float g0, g1, d0, d1;
                    gelu_as(__uint_as_float(r[2 * k2]), g0, d0, true);
                    gelu_as(__uint_as_float(r[2 * k2 + 1]), g1, d1, true);
                    gp[8 * hf + k2] = __floats2half2_rn(d0, d1);
                    g0 = tf32r(g0);
                    g1 = tf32r(g1);
                    *reinterpret_cast<float*>(p + ph[k & 7] + (k >> 3) * 1024) = g0;
                    *reinterpret_cast<float*>(p + ph[(k + 1) & 7] + ((k + 1) >> 3) * 1024) = g1;
                    r[2 * k2] = __float_as_uint(g0);
                    r[2 * k2 + 1] = __float_as_uint(g1);
                }
                tc::tmem_st_32x32b_x16(addr, r);   // G^T in place: A operand of the W2^T update
            }
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
        if (q < 2) {
            const int t = 32 * q + lane, s0 = 16 * g;
            uint32_t r[16];
            tc::tmem_ld_32x32b_x16(tm + lane_base + TM_S + s0, r);
            tc::tmem_wait_ld();
            float m[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int s = s0 + k;
                DBG(DBG_S, t, s, 64, __uint_as_float(r[k]));
                m[k] = after(s, t) ? tf32r(-__uint_as_float(r[k])) : 0.f;
            }
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
                st4(sm + OFF_X2 + row4_off(t, s0 + 4 * c4, ST64), m[4 * c4], m[4 * c4 + 1], m[4 * c4 + 2],
                    m[4 * c4 + 3]);
        }
        tc::tmem_wait_st();

        STAMP(2);
        // ---- stage C: Y^T = W2 G^T  (A = rows 0..127 of W2G; rows 64.. give unused output rows)
        if (!mma_stage([&] {
                for (int kk = 0; kk < 32; ++kk)
                    tc::mma_tf32_ss(tm + TM_Y, kstep(dW2, kk, 16384), kstep(dG, kk, 16384), ID64, kk > 0);
            }))
            break;

        STAMP(3);
        // ---- stage D (threads): D2' = -2 eta (Y - V) as [t][j] (over K) and [j][t]
        if (q < 2) {
            const int j = 32 * q + lane, t0 = 16 * g;
            uint32_t r[16], ph[8];
            tc::tmem_ld_32x32b_x16(tm + lane_base + TM_Y + t0, r);
            col_phases(j, ST64, ph);
            const uint32_t rg = (t0 >> 3) * 1024;
            tc::tmem_wait_ld();
            float d2[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int t = t0 + k;
                DBG(DBG_YT, j, t, 64, __uint_as_float(r[k]));
                const uint32_t off = rg + ph[k & 7] + (k >> 3) * 1024;
                const float v = *reinterpret_cast<const float*>(sm + OFF_V + off);
                d2[k] = (t < bc) ? tf32r(-2.0f * eta * (__uint_as_float(r[k]) - v)) : 0.f;
                *reinterpret_cast<float*>(sm + OFF_K + off) = d2[k];
            }
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
                st4(sm + OFF_X3 + row4_off(j, t0 + 4 * c4, ST64), d2[4 * c4], d2[4 * c4 + 1], d2[4 * c4 + 2],
                    d2[4 * c4 + 3]);
        }

        STAMP(4);
        // ---- stage E: P^T = W2^T D2'^T  (W2^T from tensor memory)
        if (!mma_stage([&] {
                for (int x = 0; x < 2; ++x)
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ts(tm + TM_P + x * 64, tm + TM_W2T + x * 64 + kk * 8, kstep(dK, kk, ST64), ID64,
                                        kk > 0);
            }))
            break;
        if (tid == 0 && c + 1 < nchunks) {   // the K buffer is free: fetch the next chunk's keys
            int ny0, nbc;
            chunk_rows(c + 1, ny0, nbc);
            load_tile(&P.mapK, OFF_K, bar_k, ny0);
        }

        STAMP(5);
        // ---- stage F (threads): Dl = P * G', written back in place (A operand of stage G)
        {
            const int t0 = 32 * (g & 1);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint32_t addr = tm + lane_base + TM_P + hh * 64 + t0 + 16 * hf;
                uint32_t r[16];
                tc::tmem_ld_32x32b_x16(addr, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int k2 = 0; k2 < 8; ++k2) {
                    DBG(DBG_PT, i_row, t0 + 16 * hf + 2 * k2, 64, __uint_as_float(r[2 * k2]));
                    DBG(DBG_PT, i_row, t0 + 16 * hf + 2 * k2 + 1, 64, __uint_as_float(r[2 * k2 + 1]));
                    const float2 d = __half22float2(gp[8 * hf + k2]);
                    r[2 * k2] = __float_as_uint(tf32r(__uint_as_float(r[2 * k2]) * d.x));
                    r[2 * k2 + 1] = __float_as_uint(tf32r(__uint_as_float(r[2 * k2 + 1]) * d.y));
                }
                tc::tmem_st_32x32b_x16(addr, r);
            }
            tc::tmem_wait_st();
        }

        // ---- stage G: W1 += Dl^T K;  W2^T += G^T D2'
        if (!mma_stage([&] {
                for (int x = 0; x < 2; ++x) {
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ts(tm + TM_W1 + x * 64, tm + TM_P + x * 64 + kk * 8, kstep(dX1, kk, ST64), ID64,
                                        1);
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ts(tm + TM_W2T + x * 64, tm + TM_X + x * 64 + kk * 8, kstep(dX3, kk, ST64),
                                        ID64, 1);
                }
            }))
            break;

        STAMP(7);
        // ---- stage H: Aq^T = W1_new Q^T + Dl^T M^T
        if (!mma_stage([&] {
                for (int x = 0; x < 2; ++x) {
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ts(tm + TM_X + x * 64, tm + TM_W1 + x * 64 + kk * 8, kstep(dQ, kk, ST64), ID64,
                                        kk > 0);
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ts(tm + TM_X + x * 64, tm + TM_P + x * 64 + kk * 8, kstep(dX2, kk, ST64), ID64,
                                        1);
                }
            }))
            break;
        if (tid == 0 && c + 1 < nchunks) {   // Q is free: fetch the next chunk's queries
            int ny0, nbc;
            chunk_rows(c + 1, ny0, nbc);
            load_tile(&P.mapQ, OFF_Q, bar_q, ny0);
        }

        STAMP(8);
        // ---- stages I/J: W2 copy from the updated master; then, per 16 tokens,
        //      Gq = GELU(Aq) and [Z1^T; N] = [W2_new; G] Gq^T
        refresh_w2();
#ifdef TTT_DEBUG_DUMP
        {
            const int j0 = 32 * (g & 1);
            uint32_t w[32], v[32];
            tc::tmem_ld_32x32b_x32(tm + lane_base + TM_W1 + hh * 64 + j0, w);
            tc::tmem_ld_32x32b_x32(tm + lane_base + TM_W2T + hh * 64 + j0, v);
            tc::tmem_wait_ld();
            for (int k = 0; k < 32; ++k) {
                DBG(DBG_W1, i_row, j0 + k, 64, __uint_as_float(w[k]));
                DBG(DBG_DW2T, i_row, j0 + k, 64, __uint_as_float(v[k]));
            }
        }
#endif
        STAMP(9);
        bool stopped = false;
        for (int u = 0; u < 2 && !stopped; ++u) {
            {
                const int t0 = 32 * u + 16 * (g & 1);
                uint32_t r[16], ph[8];
                tc::tmem_ld_32x32b_x16(tm + lane_base + TM_X + hh * 64 + t0, r);
                col_phases(i_row, 4096, ph);
                uint8_t* p = sm + OFF_GQ + 2 * (g & 1) * 1024;
                tc::tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    DBG(DBG_AQT, i_row, t0 + k, 64, __uint_as_float(r[k]));
                    float gg, unused;
                    gelu_as(__uint_as_float(r[k]), gg, unused, false);
                    *reinterpret_cast<float*>(p + ph[k & 7] + (k >> 3) * 1024) = tf32r(gg);
                }
            }
            if (!mma_stage([&] {
                    for (int kk = 0; kk < 32; ++kk)
                        tc::mma_tf32_ss(tm + TM_ZN + 32 * u, kstep(dW2, kk, 16384), kstep(dGQ, kk, 4096), ID32,
                                        kk > 0);
                }))
                stopped = true;
        }
        if (stopped) break;
        if (tid == 0 && c + 1 < nchunks) {   // the Gq buffer is free: fetch the next chunk's values
            int ny0, nbc;
            chunk_rows(c + 1, ny0, nbc);
            load_tile(&P.mapV, OFF_V, bar_v, ny0);
        }

        STAMP(10);
        // ---- stage K (threads): Nm[t][s] = -N[s][t] for s after t  (into X1: K^T is dead)
        if (q >= 2) {
            const int s = 32 * (q - 2) + lane, t0 = 16 * g;
            uint32_t r[16], ph[8];
            tc::tmem_ld_32x32b_x16(tm + lane_base + TM_ZN + t0, r);
            col_phases(s, ST64, ph);
            uint8_t* p = sm + OFF_X1 + (t0 >> 3) * 1024;
            tc::tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int t = t0 + k;
                DBG(DBG_N, s, t, 64, __uint_as_float(r[k]));
                *reinterpret_cast<float*>(p + ph[k & 7] + (k >> 3) * 1024) =
                    after(s, t) ? tf32r(-__uint_as_float(r[k])) : 0.f;
            }
        }

        STAMP(11);
        // ---- stage L: Z^T += D2'^T Nm^T
        if (!mma_stage([&] {
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_tf32_ss(tm + TM_ZN, kstep(dX3, kk, ST64), kstep(dX1, kk, ST64), ID64, 1);
            }))
            break;

        STAMP(12);
        // ---- stage M (threads): gate and stores
        if (q < 2) {
            const int j = 32 * q + lane, t0 = 16 * g;
            uint32_t r[16];
            tc::tmem_ld_32x32b_x16(tm + lane_base + TM_ZN + t0, r);
            tc::tmem_wait_ld();
            STAMP(13);
            // All 16 loads are issued before any is used: one dtype branch around
            // the whole batch (a per-element branch would wait on each load).
            float xv[16];
            const long long xrow = (long long)h * a.x_hs + (long long)y0 * a.x_ts + j;
            if (a.xin_bf16) {
                const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(a.Xin) + xrow;
                __nv_bfloat16 raw[16];
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    raw[k] = (t0 + k < bc) ? xb[(long long)(t0 + k) * a.x_ts] : __float2bfloat16_rn(0.f);
#pragma unroll
                for (int k = 0; k < 16; ++k) xv[k] = __bfloat162float(raw[k]);
            } else {
                const float* xf = reinterpret_cast<const float*>(a.Xin) + xrow;
#pragma unroll
                for (int k = 0; k < 16; ++k) xv[k] = (t0 + k < bc) ? xf[(long long)(t0 + k) * a.x_ts] : 0.f;
            }
#ifdef TTT_DEBUG_STAGES
            {
                float sum = 0.f;
                for (int k = 0; k < 16; ++k) sum += xv[k];
                asm volatile("" ::"f"(sum));
            }
            STAMP(19);
#endif
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int t = t0 + k;
                DBG(DBG_Z, j, t, 64, __uint_as_float(r[k]));
                if (t < bc) {
                    const float z = __uint_as_float(r[k]);
                    const long long xo = (long long)h * a.x_hs + (long long)(y0 + t) * a.x_ts + j;
                    const float dz = tanh_a * z;
                    store_elem(a.Out, xo, a.out_bf16, xv[k] + dz);
                    if (a.Delta) a.Delta[xo] = __float2bfloat16_rn(dz);
                    if (a.Zdbg) a.Zdbg[xo] = z;
                    nonfinite |= !isfinite(z);
                }
            }
        }
    }

#ifdef TTT_DEBUG_STAGES
    if (tid == 0 && blockIdx.x == 0 && g_dbg) {
        STAMP(13);
        for (int k = 0; k < 20; ++k) g_dbg[11 * 16384 + 16000 + k] = (float)stamp_acc[k];
        g_dbg[11 * 16384 + 16030] = (float)nchunks;
    }
#endif
    if (*abort_flag) {
        // let copies and MMAs already in flight land before the CTA's memory goes away
        const uint64_t t0 = tc::globaltimer_ns();
        while (tc::globaltimer_ns() - t0 < 1000000ull) __nanosleep(1000);
    } else {
        tc::tc_fence_before();
        __syncthreads();
        tc::tc_fence_after();
        const int j0 = 32 * (g & 1);
        uint32_t w[32], v[32];
        tc::tmem_ld_32x32b_x32(tm + lane_base + TM_W1 + hh * 64 + j0, w);
        tc::tmem_ld_32x32b_x32(tm + lane_base + TM_W2T + hh * 64 + j0, v);
        tc::tmem_wait_ld();
        if (a.W1_T) {
            float* dst = a.W1_T + ((long long)h * MH + i_row) * DH + j0;
#pragma unroll
            for (int k = 0; k < 32; ++k) dst[k] = __uint_as_float(w[k]);
        }
        if (a.W2_T) {
            float* dst = a.W2_T + (long long)h * DH * MH + i_row;
#pragma unroll
            for (int k = 0; k < 32; ++k) dst[(long long)(j0 + k) * MH] = __uint_as_float(v[k]);
        }
    }
    if (nonfinite) atomicOr(a.status, kStatusNonFinite);
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tm, 512);
    }
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

#if defined(TTT_DEBUG_DUMP) || defined(TTT_DEBUG_STAGES)
extern "C" __attribute__((visibility("default"))) int ttt_debug_set_dump(float* p) {
    return (int)cudaMemcpyToSymbol(g_dbg, &p, sizeof(p));
}
#endif

bool scan_chunk_tc_supported(int d, int b) { return d == DH && b >= 2 && b <= BT; }

cudaError_t launch_scan_chunk_tc(const ScanArgs& a, cudaStream_t s) {
    ScanTcArgs P{};
    P.a = a;
    P.full = (a.qkv_ts != DH) ? 1 : 0;
    if (!make_stream_map(&P.mapQ, a.Q, a, P.full) || !make_stream_map(&P.mapK, a.K, a, P.full) ||
        !make_stream_map(&P.mapV, a.V, a, P.full))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    LaunchScope scope("scan_chunk_tc", s);
    scan_tc_kernel<<<a.H, THREADS, SMEM_BYTES, s>>>(P);
    return cudaGetLastError();
}

}  // namespace ttt
