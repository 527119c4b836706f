// TTT-Linear scan on the tcgen05 tensor cores (d = 64, 2 <= b <= 64), one CTA
// per head.  The chunk of the linear layer (paper notes page, "实验关键数据 /
// 消融实验": TTT-Linear; mini-batch reading of "关键设计 / TTT-MLP 层") in
// matrix form, t, s tokens of the chunk in walking order, W the chunk-start
// state [i][j]:
//   E'^T = -2 eta (W K^T - V^T)                      (-eta dl/dz per token, [i][t])
//   Z^T  = W Q^T + E'^T M^T,  M[t,s] = q_t.k_s for s not after t
//   W   += E'^T K                                     (the chunk's update)
// which is token t read with the prefix state W + sum_{s<=t} E'_s k_s^T.
// W lives in tensor memory as an fp32 accumulator (lanes i) for the whole
// sequence and is the A operand of W K^T and W Q^T; E'^T (tensor memory) is the
// A operand of the two products that use it.  Q, K, V arrive by TMA (3-D maps,
// 128-byte swizzle) a chunk ahead.  Per chunk the dependent chain is one MMA
// stage (W K^T), one thread stage (E'), one MMA stage (the correction and the
// update); S = Q K^T and W Q^T run behind the first, the z store of the
// previous chunk, K^T and the prefix mask overlap the MMAs.  All contractions
// are kind::tf32 (fp32 accumulate) on K-major operands; every wait is bounded.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc_prims.cuh"

namespace ttt {
namespace {

constexpr int BT = 64, DH = 64, THREADS = 512;

// Shared memory (bytes from a 1024-aligned base): 64 x 64 fp32 tiles as
// 128-byte-swizzled atoms (8 rows x 32 columns; atom rows 1024 B apart, atom
// columns 8192 B apart).  Q is read as a 128-row A operand: its extra rows fall
// in K (unused output rows).
constexpr int OFF_Q = 0;         // Q [t][j] (TMA)
constexpr int OFF_K = 16384;     // K [t][j] (TMA)
constexpr int OFF_V = 32768;     // V [t][j] (TMA)
constexpr int OFF_X1 = 49152;    // K^T [j][t]
constexpr int OFF_X2 = 65536;    // M [t][s]
constexpr int OFF_BAR = 81920;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr int ST64 = 8192;

// Tensor memory columns (lanes 0-63 hold the head's 64 rows; 64-127 are unused rows).
constexpr uint32_t TM_W = 0;     // W [i][j]
constexpr uint32_t TM_E = 64;    // E^T -> E'^T [i][t]
constexpr uint32_t TM_S = 128;   // S [t][s]
constexpr uint32_t TM_Z = 192;   // Z^T [i][t], two buffers (chunk parity) at 192 and 256

struct LinTcArgs {
    CUtensorMap mapQ, mapK, mapV;
    LinearScanArgs a;
    int full;
};

__device__ __forceinline__ float tf32r(float x) {   // nearest tf32, ties away (finite inputs)
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xffffe000u);
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(tc::smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(tc::smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ uint64_t kstep(uint64_t d0, int kk) {   // K-step kk (8 tf32 = 32 B) of a 64-wide tile
    return d0 + (uint64_t)(((kk >> 2) * ST64 + (kk & 3) * 32) >> 4);
}

// Column-fixed swizzled addressing: element (R, c) at ph[R & 7] + (R >> 3) * 1024.
__device__ __forceinline__ void col_phases(int c, uint32_t (&ph)[8]) {
    const uint32_t base = (uint32_t)((c >> 5) * ST64 + (c & 3) * 4);
    const uint32_t cq = (uint32_t)((c & 31) >> 2);
#pragma unroll
    for (int r = 0; r < 8; ++r) ph[r] = base + r * 128 + ((cq ^ r) << 4);
}

__device__ __forceinline__ uint32_t row4_off(int R, int c) {   // 16-byte chunk of columns c..c+3 of row R
    return (uint32_t)((c >> 5) * ST64 + (R >> 3) * 1024 + (R & 7) * 128 + ((((c & 31) >> 2) ^ (R & 7)) << 4));
}

__global__ void __launch_bounds__(THREADS, 1) scan_linear_tc_kernel(const __grid_constant__ LinTcArgs P) {
    const LinearScanArgs& a = P.a;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar_mma = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint64_t* bar_a2 = bar_mma + 1;     // S and W Q^T
    uint64_t* bar_ld = bar_mma + 2;     // the chunk's Q, K, V tiles
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_mma + 3);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3, g = warp >> 2;   // TMEM lane quarter; token group of 16
    const int h = blockIdx.x;
    const int T = a.T, b = a.b;
    const int nchunks = (T + b - 1) / b;
    const int c_first = a.c_begin, c_last = a.c_end > 0 ? min(a.c_end, nchunks) : nchunks;
    const float m2eta = -2.0f * a.eta;

    if (tid == 0) {
        tc::mbar_init(bar_mma, 1);
        tc::mbar_init(bar_a2, 1);
        tc::mbar_init(bar_ld, 1);
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
    auto chunk_rows = [&](int c, int& y0, int& bc) {
        bc = min(b, T - c * b);
        y0 = a.reverse ? (T - c * b - bc) : c * b;
    };
    auto load_tiles = [&](int y0) {   // thread 0
        tc::mbar_arrive_expect_tx(bar_ld, 3 * BT * DH * 4);
        const CUtensorMap* maps[3] = {&P.mapQ, &P.mapK, &P.mapV};
        const int offs[3] = {OFF_Q, OFF_K, OFF_V};
        for (int w = 0; w < 3; ++w)
            for (int half = 0; half < 2; ++half) {
                if (P.full) tma_load_3d(sm + offs[w] + half * ST64, maps[w], half * 32, h, y0, bar_ld);
                else tma_load_3d(sm + offs[w] + half * ST64, maps[w], half * 32, y0, h, bar_ld);
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
    if (tid == 0) {
        int y0, bc;
        chunk_rows(c_first, y0, bc);
        load_tiles(y0);
    }

    uint32_t ph_mma = 0, ph_a2 = 0, ph_ld = 0;
    constexpr uint32_t ID64 = tc::instr_desc(2, 128, 64, 0, 0);
    const uint64_t dQ = tc::smem_desc(tc::smem_u32(sm + OFF_Q), 16, 1024);
    const uint64_t dK = tc::smem_desc(tc::smem_u32(sm + OFF_K), 16, 1024);
    const uint64_t dX1 = tc::smem_desc(tc::smem_u32(sm + OFF_X1), 16, 1024);
    const uint64_t dX2 = tc::smem_desc(tc::smem_u32(sm + OFF_X2), 16, 1024);

    auto wait_mma = [&](uint64_t* bar, uint32_t& ph) {
        if (!tc::mbar_wait(bar, ph, abort_flag)) give_up();
        ph ^= 1;
        tc::tc_fence_after();
    };
    auto mma_stage_with = [&](auto issue, auto work) -> bool {
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        if (__syncthreads_or(*abort_flag)) return false;
        tc::tc_fence_after();
        if (tid == 0) issue();
        work();
        wait_mma(bar_mma, ph_mma);
        return true;
    };
    // z of a finished chunk (rows i of quarters 0, 1; 16 tokens per thread) to global memory.
    auto store_z = [&](uint32_t tz, int y0c, int bcc) {
        if (q < 2) {
            const int i = 32 * q + lane, t0 = 16 * g;
            uint32_t r[16];
            tc::tmem_ld_32x32b_x16(tm + lane_base + tz + t0, r);
            tc::tmem_wait_ld();
            float* zrow = a.Z + (long long)h * a.x_hs + (long long)y0c * a.x_ts + i;
#pragma unroll
            for (int k = 0; k < 16; ++k)
                if (t0 + k < bcc) zrow[(long long)(t0 + k) * a.x_ts] = __uint_as_float(r[k]);
        }
    };
    int prev_y0 = 0, prev_bc = 0;

    for (int c = c_first; c < c_last; ++c) {
        int y0, bc;
        chunk_rows(c, y0, bc);
        const uint32_t tz = TM_Z + 64 * (c & 1);
        if (warp == 0) {
            if (!tc::mbar_wait(bar_ld, ph_ld, nullptr) && lane == 0) give_up();
        }
        ph_ld ^= 1;
        if (bc < BT) {   // rows beyond the chunk: zero in K and Q (they then add nothing)
            __syncthreads();
            float* fK = reinterpret_cast<float*>(sm + OFF_K);
            float* fQ = reinterpret_cast<float*>(sm + OFF_Q);
            for (int idx = tid; idx < (BT - bc) * DH; idx += THREADS) {
                const int rr = bc + idx / DH, j = idx % DH;
                const uint32_t o = row4_off(rr, j & ~3) + (j & 3) * 4;
                fK[o / 4] = 0.f;
                fQ[o / 4] = 0.f;
            }
        }

        // ---- 1: E^T = W K^T (waited for); then S = Q K^T, Z^T = W Q^T (bar_a2).
        //      Meanwhile: the previous chunk's z out, K^T into X1.
        if (!mma_stage_with(
                [&] {
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ts(tm + TM_E, tm + TM_W + kk * 8, kstep(dK, kk), ID64, kk > 0);
                    tc::mma_commit(bar_mma);
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ss(tm + TM_S, kstep(dQ, kk), kstep(dK, kk), ID64, kk > 0);
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ts(tm + tz, tm + TM_W + kk * 8, kstep(dQ, kk), ID64, kk > 0);
                    tc::mma_commit(bar_a2);
                },
                [&] {
                    if (prev_bc) store_z(TM_Z + 64 * ((c - 1) & 1), prev_y0, prev_bc);
                    {   // K^T: thread (j, 8 tokens): column reads of K, two 16-byte row writes of K^T
                        const int j = tid & 63, tb = tid >> 6;
                        uint32_t ph[8];
                        col_phases(j, ph);
                        const uint8_t* src = sm + OFF_K + tb * 1024;
                        float v[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) v[e] = *reinterpret_cast<const float*>(src + ph[e]);
                        *reinterpret_cast<float4*>(sm + OFF_X1 + row4_off(j, 8 * tb)) =
                            make_float4(v[0], v[1], v[2], v[3]);
                        *reinterpret_cast<float4*>(sm + OFF_X1 + row4_off(j, 8 * tb + 4)) =
                            make_float4(v[4], v[5], v[6], v[7]);
                    }
                }))
            break;
        prev_bc = 0;

        // ---- 2 (threads): E'^T = -2 eta (E^T - V^T) in place (zero beyond the chunk); then the
        //      prefix mask M from S once bar_a2 is done.  Rows of quarters 0, 1 only.
        if (q < 2) {
            const int i = 32 * q + lane, t0 = 16 * g;
            const uint32_t addr = tm + lane_base + TM_E + t0;
            uint32_t r[16], ph[8];
            tc::tmem_ld_32x32b_x16(addr, r);
            col_phases(i, ph);
            const uint8_t* vrow = sm + OFF_V + (t0 >> 3) * 1024;
            float vv[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) vv[k] = *reinterpret_cast<const float*>(vrow + ph[k & 7] + (k >> 3) * 1024);
            tc::tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k)
                r[k] = __float_as_uint((t0 + k < bc) ? tf32r(m2eta * (__uint_as_float(r[k]) - vv[k])) : 0.f);
            tc::tmem_st_32x32b_x16(addr, r);
        }
        wait_mma(bar_a2, ph_a2);
        if (q < 2) {   // M[t][s] = S[t][s] for s not after t
            const int t = 32 * q + lane, s0 = 16 * g;
            uint32_t r[16];
            tc::tmem_ld_32x32b_x16(tm + lane_base + TM_S + s0, r);
            tc::tmem_wait_ld();
            float m[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const bool later = a.reverse ? (s0 + k < t) : (s0 + k > t);
                m[k] = later ? 0.f : tf32r(__uint_as_float(r[k]));
            }
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
                *reinterpret_cast<float4*>(sm + OFF_X2 + row4_off(t, s0 + 4 * c4)) =
                    make_float4(m[4 * c4], m[4 * c4 + 1], m[4 * c4 + 2], m[4 * c4 + 3]);
        }
        tc::tmem_wait_st();

        // ---- 3: Z^T += E'^T M^T;  W += E'^T K.  Q, K, V are free: fetch the next chunk's tiles.
        if (!mma_stage_with(
                [&] {
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ts(tm + tz, tm + TM_E + kk * 8, kstep(dX2, kk), ID64, 1);
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_tf32_ts(tm + TM_W, tm + TM_E + kk * 8, kstep(dX1, kk), ID64, 1);
                    tc::mma_commit(bar_mma);
                    if (c + 1 < c_last) {
                        int ny0, nbc;
                        chunk_rows(c + 1, ny0, nbc);
                        load_tiles(ny0);
                    }
                },
                [] {}))
            break;
        prev_y0 = y0;
        prev_bc = bc;
    }
    if (prev_bc && !*abort_flag) store_z(TM_Z + 64 * ((c_last - 1) & 1), prev_y0, prev_bc);

    if (*abort_flag) {
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
