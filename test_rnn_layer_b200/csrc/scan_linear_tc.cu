// TTT-Linear scan on the tcgen05 tensor cores (d = 64, 2 <= b <= 64), one CTA
// per head.  The chunk of the linear layer (paper notes page, "实验关键数据 /
// 消融实验": TTT-Linear; mini-batch reading of "关键设计 / TTT-MLP 层") in
// matrix form, t, s tokens of the chunk in walking order, W_c the chunk-start
// state [i][j]:
//   E'^T = -2 eta (W_c K^T - V^T)                  (-eta dl/dz per token, [i][t])
//   W_{c+1} = W_c + E'^T K                         (the chunk's update)
//   Z^T  = W_{c+1} Q^T - E'^T Npost^T,  Npost[t,s] = q_t.k_s for s after t
// which is token t read with the prefix state W_c + sum_{s<=t} E'_s k_s^T: the
// output is read with the state at the chunk's END, less the later tokens'
// updates.  So W_{c+1} Q_c^T and the next chunk's W_{c+1} K_{c+1}^T share
// their A operand and run as one N = 128 product over [K_{c+1}; Q_c], and no
// product that reads W is ever in flight while the update writes it.
//
// Per chunk the dependent chain is: [W K^T | W Q_prev^T] (tf32, W the A operand
// from tensor memory), the E' thread stage (fp16 pairs into tensor memory), the
// update (kind::f16 on K as fp16).  Off the chain: S = Q K^T (tf32, issued by
// warp 2), the previous chunk's correction (kind::f16), the mask -Npost as
// fp16, the z stores, K as fp16, and the tile loads (warp 3) a chunk ahead.
// fp16 holds the thread-produced operands (E', K, the mask): the same 10-bit
// mantissa as tf32, rounded rather than truncated.  Every wait is bounded.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc_prims.cuh"

namespace ttt {
namespace {

constexpr int BT = 64, DH = 64, THREADS = 512;

// Shared memory (bytes from a 1024-aligned base).  fp32 tiles are 128-byte
// swizzled atoms (8 rows x 32 columns, atom rows 1024 B apart).  K and Q share
// two 32 KB regions: region r holds K of chunk parity r at +0 (columns 0-31) /
// +16 KB (columns 32-63) and Q of parity 1-r at +8 KB / +24 KB, so that rows
// 0-127 of a region are [K_c; Q_{c-1}] with 16 KB between the column halves.
// A 128-row read of Q as an A operand runs into the next 8 KB (unused rows).
constexpr int OFF_REG = 0;          // [2] x 32 KB: K / Q regions
constexpr int REG = 32768;
constexpr int QSLOT = 8192;         // Q's rows within a region
constexpr int KQ_HALF = 16384;      // column-half stride of K and Q
constexpr int OFF_V = 65536;        // [2] x 16 KB: V [t][j], column halves 8 KB apart
constexpr int V_HALF = 8192;
constexpr int OFF_X1 = 98304;       // 8 KB: K fp16 [t][j], MN-major (row per K index t)
constexpr int OFF_X2 = 106496;      // [2] x 8 KB: -Npost fp16 [t][s], K-major (row per t)
constexpr int OFF_BAR = 122880;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;

// Tensor memory (128 lanes x 512 columns; lanes 0-63 are the head's rows, 64-127 unused).
constexpr uint32_t TM_W = 0;        // W [i][j]
constexpr uint32_t TM_B = 64;       // [2] x 128: [E^T of chunk c | Z^T of chunk c-1], block of parity c
constexpr uint32_t TM_S = 320;      // S [t][s]
constexpr uint32_t TM_PK = 384;     // [2] x 32: E'^T [i][t] as fp16 pairs (the A operand)

#ifdef TTT_DEBUG_STAGES
// Debug builds only: cycles between stage boundaries seen by thread 0 of CTA 0.
__device__ float* g_dbg_lin = nullptr;
#define STAMPL(k)                                         \
    do {                                                  \
        if (tid == 0 && blockIdx.x == 0) {                \
            const long long now_ = clock64();             \
            stamp_acc[k] += now_ - stamp_last;            \
            stamp_last = now_;                            \
        }                                                 \
    } while (0)
#else
#define STAMPL(k) \
    do {          \
    } while (0)
#endif

struct LinTcArgs {
    CUtensorMap mapQ, mapK, mapV;
    LinearScanArgs a;
    int full;
};

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(tc::smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(tc::smem_u32(bar))
        : "memory");
}

// K-step kk (8 tf32 = 32 B) of a 64-wide fp32 tile whose column halves are `half` bytes apart.
__device__ __forceinline__ uint64_t kstep(uint64_t d0, int kk, int half) {
    return d0 + (uint64_t)(((kk >> 2) * half + (kk & 3) * 32) >> 4);
}
// K-step kk (16 fp16 = 32 B) of a K-major fp16 operand (64 K values per 128-byte row).
__device__ __forceinline__ uint64_t kstep_h(uint64_t d0, int kk) { return d0 + (uint64_t)((kk * 32) >> 4); }
// K-step kk (16 K rows = 2 KB) of an MN-major fp16 operand.
__device__ __forceinline__ uint64_t kstep_mn(uint64_t d0, int kk) { return d0 + (uint64_t)((kk * 2048) >> 4); }

// 16-byte chunk of fp32 columns c..c+3 of row R (column halves `half` bytes apart).
__device__ __forceinline__ uint32_t row4_off(int R, int c, int half) {
    return (uint32_t)((c >> 5) * half + (R >> 3) * 1024 + (R & 7) * 128 + ((((c & 31) >> 2) ^ (R & 7)) << 4));
}

// 16-byte chunk of fp16 values c..c+7 (c % 8 == 0, c < 64) of 128-byte row R, 128-byte swizzle.
__device__ __forceinline__ uint32_t h_chunk(int R, int c) {
    return (uint32_t)((R >> 3) * 1024 + (R & 7) * 128 + (((c >> 3) ^ (R & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(THREADS, 1) scan_linear_tc_kernel(const __grid_constant__ LinTcArgs P) {
    const LinearScanArgs& a = P.a;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint64_t* bar_g = bars + 0;    // [W K^T | W Q_prev^T] of the chunk
    uint64_t* bar_u = bars + 1;    // the update
    uint64_t* bar_c = bars + 2;    // the previous chunk's correction (and the last chunk's output products)
    uint64_t* bar_s = bars + 3;    // S = Q K^T
    uint64_t* bar_ld = bars + 4;   // [2]: a chunk's Q, K, V tiles, by chunk parity
    uint64_t* bar_go = bars + 6;   // a chunk has started: its first product is issued, the chunk before is done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 7);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, g = warp >> 2;   // TMEM lane quarter; token group of 16
    const int h = blockIdx.x;
    const int T = a.T, b = a.b;
    const int nchunks = (T + b - 1) / b;
    const int c_first = a.c_begin, c_last = a.c_end > 0 ? min(a.c_end, nchunks) : nchunks;
    const int nloc = c_last - c_first;
    const float m2eta = -2.0f * a.eta;

    if (tid == 0) {
        for (int k = 0; k < 7; ++k) tc::mbar_init(bars + k, 1);
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

    auto give_up = [&]() {
        *abort_flag = 1;
        atomicOr(a.status, kStatusTimeout);
    };
    auto wait_ok = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (tc::mbar_wait(bar, parity, abort_flag)) return true;
        give_up();
        return false;
    };
    auto chunk_rows = [&](int c, int& y0, int& bc) {
        bc = min(b, T - c * b);
        y0 = a.reverse ? (T - c * b - bc) : c * b;
    };
    // where the tiles of local chunk n live
    auto k_tile = [&](int n) { return sm + OFF_REG + (n & 1) * REG; };
    auto q_tile = [&](int n) { return sm + OFF_REG + ((n & 1) ^ 1) * REG + QSLOT; };
    auto v_tile = [&](int n) { return sm + OFF_V + (n & 1) * 16384; };
    auto load_tiles = [&](int n) {   // thread 96: local chunk n's Q, K, V
        int y0, bc;
        chunk_rows(c_first + n, y0, bc);
        uint64_t* bl = bar_ld + (n & 1);
        tc::mbar_arrive_expect_tx(bl, 3 * BT * DH * 4);
        const CUtensorMap* maps[3] = {&P.mapQ, &P.mapK, &P.mapV};
        uint8_t* dst[3] = {q_tile(n), k_tile(n), v_tile(n)};
        const int half[3] = {KQ_HALF, KQ_HALF, V_HALF};
        for (int w = 0; w < 3; ++w)
            for (int hf = 0; hf < 2; ++hf) {
                uint8_t* d = dst[w] + hf * half[w];
                if (P.full) tma_load_3d(d, maps[w], hf * 32, h, y0, bl);
                else tma_load_3d(d, maps[w], hf * 32, y0, h, bl);
            }
    };

    // ---- initial state: W rows 0-63 (lanes of quarters 0, 1); unused rows 64-127 zero
    {
        const int i = 32 * q + lane, j0 = 16 * g;
        uint32_t r[16];
        int bad = 0;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float v = (q < 2) ? a.W_0[((long long)h * DH + i) * DH + j0 + k] : 0.f;
            bad |= !isfinite(v);
            r[k] = __float_as_uint(v);
        }
        if (bad) atomicOr(a.status, kStatusNonFinite);
        tc::tmem_st_32x32b_x16(tm + lane_base + TM_W + j0, r);
        tc::tmem_wait_st();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    constexpr uint32_t ID64 = tc::instr_desc(2, 128, 64, 0, 0);
    constexpr uint32_t ID128 = tc::instr_desc(2, 128, 128, 0, 0);
    constexpr uint32_t ID_F16 = tc::instr_desc(0, 128, 64, 0, 0);      // A in tensor memory, B K-major
    constexpr uint32_t ID_F16_MN = tc::instr_desc(0, 128, 64, 0, 1);   // A in tensor memory, B MN-major
    auto dsc = [&](const uint8_t* p, uint32_t lbo) { return tc::smem_desc(tc::smem_u32(p), lbo, 1024); };
    const uint64_t dX1 = dsc(sm + OFF_X1, 16384);   // K fp16 [t][j], MN-major (one 64-wide block)
    auto dX2 = [&](int n) { return dsc(sm + OFF_X2 + (n & 1) * 8192, 16); };
    auto tb_of = [](int n) { return TM_B + 128u * (uint32_t)(n & 1); };
    auto pk_of = [](int n) { return TM_PK + 32u * (uint32_t)(n & 1); };
#ifdef TTT_DEBUG_STAGES
    long long stamp_acc[8] = {};
    long long stamp_last = clock64();
#endif

    if (q < 2) {
        // =====================================================================================
        // E warps (0, 1, 4, 5, 8, 9, 12, 13): the chain.  Thread (q, g, lane) owns row i = 32 q + lane of
        // the [i][t] tiles and tokens 16 g .. 16 g + 15; thread 0 issues the chain's products.
        // =====================================================================================
        const int et = (g * 2 + q) * 32 + lane;   // 0 .. 255 over the E warps
        auto esync = [&]() -> bool {                // the E warps; true if some thread saw an abort
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            const bool ab = tc::bar_sync_or(1, 256, *abort_flag != 0);
            tc::tc_fence_after();
            return ab;
        };
        auto wait_mma = [&](uint64_t* bar, uint32_t& ph) {
            wait_ok(bar, ph);
            ph ^= 1;
            tc::tc_fence_after();
        };
        // z of a finished chunk (16 tokens of row i per thread) to global memory
        auto store_z = [&](uint32_t tz, int y0c, int bcc) {
            const int i = 32 * q + lane, t0 = 16 * g;
            uint32_t r[16];
            tc::tmem_ld_32x32b_x16(tm + lane_base + tz + t0, r);
            tc::tmem_wait_ld();
            float* zrow = a.Z + (long long)h * a.x_hs + (long long)y0c * a.x_ts + i;
#pragma unroll
            for (int k = 0; k < 16; ++k)
                if (t0 + k < bcc) zrow[(long long)(t0 + k) * a.x_ts] = __uint_as_float(r[k]);
        };
        uint32_t ph_g = 0, ph_u = 0, ph_c = 0, ph_s = 0;
        int prev_y0 = 0, prev_bc = 0;
        bool aborted = false;
        for (int n = 0; n < nloc; ++n) {
            int y0, bc;
            chunk_rows(c_first + n, y0, bc);
            const uint32_t tb = tb_of(n), pk = pk_of(n);
            STAMPL(0);
            // ---- 0: the chunk's tiles (rows beyond a short chunk cleared in K and Q), then the first
            //      product [E^T_c | Z'^T_{c-1}] = W_c [K_c; Q_{c-1}]^T (the B rows 64.. are Q_{c-1})
            if (tid == 0) wait_ok(bar_ld + (n & 1), (uint32_t)(n >> 1) & 1u);
            if ((aborted = esync())) break;
            if (bc < BT) {
                float* fK = reinterpret_cast<float*>(k_tile(n));
                float* fQ = reinterpret_cast<float*>(q_tile(n));
                for (int idx = et; idx < (BT - bc) * DH; idx += 256) {
                    const int rr = bc + idx / DH, j = idx % DH;
                    const uint32_t o = row4_off(rr, j & ~3, KQ_HALF) + (j & 3) * 4;
                    fK[o / 4] = 0.f;
                    fQ[o / 4] = 0.f;
                }
                if ((aborted = esync())) break;
            }
            if (tid == 0) {
                const uint64_t d = dsc(k_tile(n), 16);
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_tf32_ts(tm + tb, tm + TM_W + kk * 8, kstep(d, kk, KQ_HALF), ID128, kk > 0);
                tc::mma_commit(bar_g);
                tc::mbar_arrive(bar_go);
            }
            // ---- 1: K as fp16 [t][j] into X1 (the update of chunk c-1 has read it): thread (t, 16 j)
            {
                const int t = et >> 2, j0 = 16 * (et & 3);
                const uint8_t* kt = k_tile(n);
                float v[16];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const float4 f = *reinterpret_cast<const float4*>(kt + row4_off(t, j0 + 4 * c4, KQ_HALF));
                    v[4 * c4] = f.x;
                    v[4 * c4 + 1] = f.y;
                    v[4 * c4 + 2] = f.z;
                    v[4 * c4 + 3] = f.w;
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    *reinterpret_cast<uint4*>(sm + OFF_X1 + h_chunk(t, j0 + 8 * hh)) =
                        make_uint4(pack_h2(v[8 * hh], v[8 * hh + 1]), pack_h2(v[8 * hh + 2], v[8 * hh + 3]),
                                   pack_h2(v[8 * hh + 4], v[8 * hh + 5]), pack_h2(v[8 * hh + 6], v[8 * hh + 7]));
            }
            // ---- 2: E'^T = -2 eta (E^T - V^T) as fp16 pairs (zero beyond the chunk)
            wait_mma(bar_g, ph_g);
            STAMPL(1);
            {
                const int i = 32 * q + lane, t0 = 16 * g;
                uint32_t r[16], pr[8];
                tc::tmem_ld_32x32b_x16(tm + lane_base + tb + t0, r);
                const uint8_t* vt = v_tile(n);
                float vv[16];
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    vv[k] = *reinterpret_cast<const float*>(vt + row4_off(t0 + k, i & ~3, V_HALF) + (i & 3) * 4);
                tc::tmem_wait_ld();
#pragma unroll
                for (int k2 = 0; k2 < 8; ++k2) {
                    const int k = 2 * k2;
                    pr[k2] = pack_h2((t0 + k < bc) ? m2eta * (__uint_as_float(r[k]) - vv[k]) : 0.f,
                                     (t0 + k + 1 < bc) ? m2eta * (__uint_as_float(r[k + 1]) - vv[k + 1]) : 0.f);
                }
                tc::tmem_st_32x32b_x8(tm + lane_base + pk + 8 * g, pr);
                tc::tmem_wait_st();
            }
            if ((aborted = esync())) break;
            STAMPL(2);
            // ---- 3: W += E'^T K (the chain), then the previous chunk's correction
            //      Z^T_{c-1} += E'^T_{c-1} (-Npost_{c-1})^T into the Z'_{c-1} the first product left here
            if (tid == 0) {
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16_ts(tm + TM_W, tm + pk + kk * 8, kstep_mn(dX1, kk), ID_F16_MN, 1);
                tc::mma_commit(bar_u);
                if (n > 0) {
                    for (int kk = 0; kk < 4; ++kk)
                        tc::mma_f16_ts(tm + tb + 64, tm + pk_of(n - 1) + kk * 8, kstep_h(dX2(n - 1), kk), ID_F16, 1);
                    tc::mma_commit(bar_c);
                }
            }
            //      meanwhile -Npost of chunk c (fp16, K-major row t) once S is done: thread (t, 16 s)
            wait_mma(bar_s, ph_s);
            {
                const int t = 32 * q + lane, s0 = 16 * g;
                uint32_t r[16], u[8];
                tc::tmem_ld_32x32b_x16(tm + lane_base + TM_S + s0, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int k2 = 0; k2 < 8; ++k2) {
                    const int s = s0 + 2 * k2;
                    const bool l0 = a.reverse ? (s < t) : (s > t), l1 = a.reverse ? (s + 1 < t) : (s + 1 > t);
                    u[k2] = pack_h2(l0 ? -__uint_as_float(r[2 * k2]) : 0.f, l1 ? -__uint_as_float(r[2 * k2 + 1]) : 0.f);
                }
                uint8_t* x2 = sm + OFF_X2 + (n & 1) * 8192;
                *reinterpret_cast<uint4*>(x2 + h_chunk(t, s0)) = make_uint4(u[0], u[1], u[2], u[3]);
                *reinterpret_cast<uint4*>(x2 + h_chunk(t, s0 + 8)) = make_uint4(u[4], u[5], u[6], u[7]);
            }
            //      and the previous chunk's z once its correction is done
            if (n > 0) {
                wait_mma(bar_c, ph_c);
                store_z(tb + 64, prev_y0, prev_bc);
            }
            wait_mma(bar_u, ph_u);
            STAMPL(3);
            prev_y0 = y0;
            prev_bc = bc;
            if ((aborted = esync())) break;   // the mask, the z and W are done: the next chunk may start
        }
        if (!aborted && nloc > 0) {   // the last chunk's output: Z'^T = W_{c+1} Q^T, then its correction
            const int nl = nloc - 1;
            const uint32_t tz = tb_of(nl + 1) + 64;
            if (tid == 0) {
                const uint64_t d = dsc(q_tile(nl), 16);
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_tf32_ts(tm + tz, tm + TM_W + kk * 8, kstep(d, kk, KQ_HALF), ID64, kk > 0);
                tc::mma_commit(bar_c);
            }
            wait_mma(bar_c, ph_c);
            if (tid == 0) {
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_f16_ts(tm + tz, tm + pk_of(nl) + kk * 8, kstep_h(dX2(nl), kk), ID_F16, 1);
                tc::mma_commit(bar_c);
            }
            wait_mma(bar_c, ph_c);
            store_z(tz, prev_y0, prev_bc);
        }
    } else if (warp == 2) {
        // S = Q_c K_c^T once the chunk's first product is issued (A: 128 rows from Q; rows 64.. unused)
        for (int n = 0; n < nloc; ++n) {
            int ok = 1;
            if (lane == 0) {
                ok = wait_ok(bar_go, (uint32_t)n & 1u);
                tc::tc_fence_after();
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            if (lane == 0) {
                const uint64_t dq = dsc(q_tile(n), 16), dk = dsc(k_tile(n), 16);
                for (int kk = 0; kk < 8; ++kk)
                    tc::mma_tf32_ss(tm + TM_S, kstep(dq, kk, KQ_HALF), kstep(dk, kk, KQ_HALF), ID64, kk > 0);
                tc::mma_commit(bar_s);
            }
            __syncwarp();
        }
    } else if (warp == 3) {
        // the tiles, a chunk ahead: chunk n+1's go where chunk n-1's were, once chunk n's first
        // product (the last reader of Q_{n-1}) is done
        if (lane == 0 && nloc > 0) load_tiles(0);
        for (int n = 0; n + 1 < nloc; ++n) {
            int ok = 1;
            if (lane == 0) ok = wait_ok(bar_g, (uint32_t)n & 1u);
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            if (lane == 0) load_tiles(n + 1);
            __syncwarp();
        }
    }

#ifdef TTT_DEBUG_STAGES
    if (tid == 0 && blockIdx.x == 0 && g_dbg_lin) {
        for (int k = 0; k < 8; ++k) g_dbg_lin[k] = (float)stamp_acc[k];
        g_dbg_lin[8] = (float)nloc;
    }
#endif
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (*abort_flag) {   // let copies and MMAs in flight land before the memory goes away
        const uint64_t t0 = tc::globaltimer_ns();
        while (tc::globaltimer_ns() - t0 < 1000000ull) __nanosleep(1000);
    } else if (a.W_T && q < 2) {
        const int i = 32 * q + lane, j0 = 16 * g;
        uint32_t r[16];
        tc::tmem_ld_32x32b_x16(tm + lane_base + TM_W + j0, r);
        tc::tmem_wait_ld();
        float* dst = a.W_T + ((long long)h * DH + i) * DH + j0;
#pragma unroll
        for (int k = 0; k < 16; ++k) dst[k] = __uint_as_float(r[k]);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tm, 512);
    }
}

bool make_map(CUtensorMap* m, const float* base, const LinearScanArgs& a, bool full) {
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
extern "C" __attribute__((visibility("default"))) int ttt_debug_set_dump_lin(float* p) {
    return (int)cudaMemcpyToSymbol(g_dbg_lin, &p, sizeof(p));
}
#endif

bool scan_linear_tc_supported(int d, int b) { return d == DH && b >= 2 && b <= BT; }

cudaError_t launch_scan_linear_tc(const LinearScanArgs& a, cudaStream_t s) {
    if (!scan_linear_tc_supported(a.d, a.b)) return cudaErrorInvalidValue;
    const int nchunks = (a.T + a.b - 1) / a.b;
    const int c_end = a.c_end > 0 ? a.c_end : nchunks;
    if (a.c_begin < 0 || c_end > nchunks || a.c_begin >= c_end) return cudaErrorInvalidValue;
    LinTcArgs P{};
    P.a = a;
    P.full = (a.qkv_ts != DH) ? 1 : 0;
    if (!make_map(&P.mapQ, a.Q, a, P.full) || !make_map(&P.mapK, a.K, a, P.full) || !make_map(&P.mapV, a.V, a, P.full))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(scan_linear_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM_BYTES);
    if (e != cudaSuccess) return e;
    LaunchScope scope("scan_linear_tc", s);
    scan_linear_tc_kernel<<<a.H, THREADS, SMEM_BYTES, s>>>(P);
    return cudaGetLastError();
}

}  // namespace ttt
