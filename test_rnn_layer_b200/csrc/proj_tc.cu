// theta_Q / theta_K / theta_V projections of the full layer on the tcgen05
// tensor cores: C_w[t, n] (+)= sum_c A[t, c] Theta_w[n, c], A and Theta bf16,
// fp32 accumulation in TMEM, fp32 output (paper notes page, "关键设计 /
// TTT-MLP 层": the outer-loop key/value/query projections).
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles (M = 128 tokens,
// N = 256 features of one projection), K consumed in 64-wide blocks:
//   warp 0      TMA producer: A and Theta tiles into a 4-stage ring (128-byte swizzle)
//   warp 1      allocates TMEM; one lane issues tcgen05.mma (M128 N256 K16) and commits
//   warps 2..5  epilogue: TMEM -> registers -> swizzled shared staging -> TMA store
//               (or TMA reduce-add when accumulating onto C)
// Two TMEM accumulators (2 x 256 columns) let the epilogue of one tile overlap
// the main loop of the next.  Every wait is bounded; on expiry the CTA records
// kStatusTimeout, drains and exits.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_prims.cuh"

namespace ttt {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;          // 16 KB
constexpr int B_BYTES = BN * BK * 2;          // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int EPI_WARPS = 4;
constexpr int EPI_BUF = 32 * 32 * 4;          // one 32 x 32 fp32 box
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_WARPS * 2 * EPI_BUF + 256;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr uint32_t TMEM_COLS = 512;
// Tile order: groups of GROUP_M row tiles, and within a group every column tile over the group's row
// tiles before the next column tile.  A theta panel (256 rows, the whole reduction) is then read by
// GROUP_M row tiles in a row while the group's X tiles (GROUP_M x 768 KB) stay in L2, instead of
// cycling through all of theta for every row tile next to the scan's streams.
#ifndef TTT_PROJ_GROUP_M
#define TTT_PROJ_GROUP_M 32
#endif
constexpr int GROUP_M = TTT_PROJ_GROUP_M;

// Up to 3 outputs C_w (+)= sum over segments s of A_{w,s} B_{w,s}^T, every segment the same reduction
// length K: the projections pass one A for all three outputs and one segment; the projection gradients
// pass several (the high and low bf16 halves of an fp32 operand, two sources).
constexpr int kMaxSeg = 4;
struct ProjTcArgs {
    CUtensorMap mapA[3][kMaxSeg];
    CUtensorMap mapB[3][kMaxSeg];
    CUtensorMap mapC[3];
    int K;                 // reduction length of one segment
    int nseg;              // segments along the reduction
    int a_mn, b_mn;        // 1: that operand is MN-major in memory (rows = K), 0: K-major (rows = M or N)
    int N;                 // output columns of each output (a multiple of 64; the last tile may be partial)
    int m_tiles, n_tiles_per, nw, tiles;
    int accumulate;
    int* status;
};

// Row tile and column tile of linear tile index `tile` (see GROUP_M).
__device__ __forceinline__ void tile_of(int tile, int m_tiles, int n_tiles, int& mt, int& nt) {
    const int per_group = GROUP_M * n_tiles;
    const int g = tile / per_group, local = tile - g * per_group;
    const int gm = min(GROUP_M, m_tiles - g * GROUP_M);   // row tiles in this (possibly last, short) group
    nt = local / gm;
    mt = g * GROUP_M + (local - nt * gm);
}

__global__ void __launch_bounds__(THREADS, 1) proj_tc_kernel(const __grid_constant__ ProjTcArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stage_base = smem;
    uint8_t* epi_base = smem + STAGES * STAGE_BYTES;
    uint64_t* full = reinterpret_cast<uint64_t*>(epi_base + EPI_WARPS * 2 * EPI_BUF);
    uint64_t* empty = full + STAGES;
    uint64_t* tmem_full = empty + STAGES;
    uint64_t* tmem_empty = tmem_full + 2;
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(tmem_empty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { tc::mbar_init(&full[s], 1); tc::mbar_init(&empty[s], 1); }
        for (int a = 0; a < 2; ++a) { tc::mbar_init(&tmem_full[a], 1); tc::mbar_init(&tmem_empty[a], EPI_WARPS); }
        *abort_flag = 0;
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&p.mapA[0][0]);
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_base_slot, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_base_slot;
    const int KB = (p.K + BK - 1) / BK;   // per segment; operand columns or rows past K read as zero
    const int n_tiles = p.nw * p.n_tiles_per;

    auto give_up = [&]() {
        *abort_flag = 1;
        atomicOr(p.status, kStatusTimeout);
    };

    if (warp == 0) {
        // ---------------- TMA producer
        if (tc::elect_one()) {
            int s = 0;
            uint32_t phase = 0;
            // theta is read by every M tile: keep it in L2 ahead of the streaming output
            const uint64_t keep = tc::l2_policy_evict_last();
            for (int tile = blockIdx.x; tile < p.tiles && !*abort_flag; tile += gridDim.x) {
                int mt, nt;
                tile_of(tile, p.m_tiles, n_tiles, mt, nt);
                const int which = nt / p.n_tiles_per;
                const int n0 = (nt % p.n_tiles_per) * BN;
                for (int kb = 0; kb < KB * p.nseg; ++kb) {
                    if (!tc::mbar_wait(&empty[s], phase ^ 1, abort_flag)) { give_up(); break; }
                    uint8_t* st = stage_base + s * STAGE_BYTES;
                    const int seg = kb / KB, k0 = (kb - seg * KB) * BK;
                    const CUtensorMap* ma = &p.mapA[which][seg];
                    const CUtensorMap* mb = &p.mapB[which][seg];
                    tc::mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
                    // K-major: one box of BK columns; MN-major: boxes of 64 M/N columns x BK rows, 8 KB apart
                    if (!p.a_mn) tc::tma_load_2d(st, ma, k0, mt * BM, &full[s]);
                    else
                        for (int i = 0; i < BM / 64; ++i) tc::tma_load_2d(st + i * 8192, ma, mt * BM + 64 * i, k0, &full[s]);
                    if (!p.b_mn) tc::tma_load_2d_hint(st + A_BYTES, mb, k0, n0, &full[s], keep);
                    else
                        for (int i = 0; i < BN / 64; ++i)
                            tc::tma_load_2d_hint(st + A_BYTES + i * 8192, mb, n0 + 64 * i, k0, &full[s], keep);
                    if (++s == STAGES) { s = 0; phase ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (tc::elect_one()) {
            const uint32_t idesc = tc::instr_desc(1, BM, BN, p.a_mn, p.b_mn);
            // K step of 16: K-major +32 bytes inside the 128-byte row; MN-major +16 rows (2 KB), the 64-wide
            // M/N blocks 8 KB apart (leading offset), 8-row groups 1 KB apart (stride offset)
            const uint32_t a_step = p.a_mn ? 2048 : 32, b_step = p.b_mn ? 2048 : 32;
            const uint32_t a_lbo = p.a_mn ? 8192 : 16, b_lbo = p.b_mn ? 8192 : 16;
            int s = 0;
            uint32_t phase = 0;
            int it = 0;
            for (int tile = blockIdx.x; tile < p.tiles && !*abort_flag; tile += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t acc_phase = (it >> 1) & 1;
                if (!tc::mbar_wait(&tmem_empty[acc], acc_phase ^ 1, abort_flag)) { give_up(); break; }
                tc::tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                bool ok = true;
                for (int kb = 0; kb < KB * p.nseg; ++kb) {
                    if (!tc::mbar_wait(&full[s], phase, abort_flag)) { ok = false; break; }
                    tc::tc_fence_after();
                    const uint32_t a_addr = tc::smem_u32(stage_base + s * STAGE_BYTES);
                    const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        const uint64_t ad = tc::smem_desc(a_addr + k * a_step, a_lbo, 1024);
                        const uint64_t bd = tc::smem_desc(b_addr + k * b_step, b_lbo, 1024);
                        tc::mma_f16_ss(d_tmem, ad, bd, idesc, (kb | k) != 0);
                    }
                    tc::mma_commit(&empty[s]);
                    if (++s == STAGES) { s = 0; phase ^= 1; }
                }
                if (!ok) { give_up(); break; }
                tc::mma_commit(&tmem_full[acc]);
            }
        }
    } else {
        // ---------------- epilogue (warps 2..5 -> TMEM lane quarters 2, 3, 0, 1)
        const int q = warp % 4;
        uint8_t* bufs = epi_base + (warp - 2) * 2 * EPI_BUF;
        int it = 0, nbuf = 0, nonfinite = 0;
        const uint64_t stream_out = tc::l2_policy_evict_first();
        for (int tile = blockIdx.x; tile < p.tiles && !*abort_flag; tile += gridDim.x, ++it) {
            const int acc = it & 1;
            const uint32_t acc_phase = (it >> 1) & 1;
            int mt, nt;
            tile_of(tile, p.m_tiles, n_tiles, mt, nt);
            const int which = nt / p.n_tiles_per;
            const int n0 = (nt % p.n_tiles_per) * BN;
            // the whole warp leaves together (it meets __syncwarp below and __any_sync after the loop)
            const bool got = tc::mbar_wait(&tmem_full[acc], acc_phase, abort_flag);
            if (!__all_sync(0xffffffffu, got)) {
                if (lane == 0) give_up();
                break;
            }
            tc::tc_fence_after();
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tc::tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(32 * q) << 16) + acc * BN + c * 32, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) nonfinite |= (r[j] & 0x7f800000u) == 0x7f800000u;
                uint8_t* buf = bufs + nbuf * EPI_BUF;
                if (lane == 0) tc::bulk_wait_group_read<1>();   // the store that last used `buf` has read it
                __syncwarp();
                // row `lane` of a 32 x 32 fp32 box, 128-byte swizzle: 16-byte chunk j at (j ^ (row & 7))
                uint4* row = reinterpret_cast<uint4*>(buf + lane * 128);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    row[j ^ (lane & 7)] = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
                tc::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int x = n0 + c * 32, y = mt * BM + 32 * q;
                    if (x < p.N) {   // columns of a partial last tile beyond N are zero (theta rows read as fill)
                        // the output streams through L2 once: first to be evicted
                        if (p.accumulate) tc::tma_reduce_add_2d_hint(&p.mapC[which], buf, x, y, stream_out);
                        else tc::tma_store_2d_hint(&p.mapC[which], buf, x, y, stream_out);
                    }
                    tc::bulk_commit_group();
                }
                nbuf ^= 1;
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&tmem_empty[acc]);
        }
        if (lane == 0) tc::bulk_wait_group<0>();
        // a non-finite input (X, theta or the increment) reaches the projections
        if (__any_sync(0xffffffffu, nonfinite) && lane == 0) atomicOr(p.status, kStatusNonFinite);
    }

    if (*abort_flag) {
        // let copies and MMAs already in flight land before the CTA's memory goes away
        const uint64_t t0 = tc::globaltimer_ns();
        while (tc::globaltimer_ns() - t0 < 1000000ull) __nanosleep(1000);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, TMEM_COLS);
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

bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t es[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// N: whole 32-column boxes of the epilogue (64 keeps every box either inside or past N); the B loads of a
// partial last tile read theta rows beyond N as zero fill.
bool proj_full_tc_supported(int N, int K) { return N % 64 == 0 && K % BK == 0 && N > 0 && K > 0; }

cudaError_t launch_gemm_tc(const GemmTc& g, cudaStream_t s) {
    if (g.nw < 1 || g.nw > 3 || g.nseg < 1 || g.nseg > kMaxSeg || g.M < 1 || g.N < 1 || g.K < 1 || g.N % 64 != 0)
        return cudaErrorInvalidValue;
    ProjTcArgs p{};
    bool ok = true;
    for (int w = 0; w < g.nw && ok; ++w) {
        for (int sg = 0; sg < g.nseg && ok; ++sg) {
            const GemmTcOperand& a = g.A[w][sg];
            const GemmTcOperand& b = g.B[w][sg];
            ok = (g.a_mn ? make_map(&p.mapA[w][sg], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.ptr, g.M, g.K, a.ld * 2, 64, BK)
                         : make_map(&p.mapA[w][sg], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.ptr, g.K, g.M, a.ld * 2, BK, BM)) &&
                 (g.b_mn ? make_map(&p.mapB[w][sg], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, b.ptr, g.N, g.K, b.ld * 2, 64, BK)
                         : make_map(&p.mapB[w][sg], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, b.ptr, g.K, g.N, b.ld * 2, BK, BN));
        }
        ok = ok && make_map(&p.mapC[w], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.C[w], g.N, g.M, (uint64_t)g.ldc * 4, 32, 32);
    }
    if (!ok) return cudaErrorInvalidValue;
    p.K = g.K;
    p.nseg = g.nseg;
    p.a_mn = g.a_mn;
    p.b_mn = g.b_mn;
    p.N = g.N;
    p.m_tiles = (g.M + BM - 1) / BM;
    p.n_tiles_per = (g.N + BN - 1) / BN;
    p.nw = g.nw;
    p.tiles = p.m_tiles * g.nw * p.n_tiles_per;
    p.accumulate = g.accumulate;
    p.status = g.status;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e = cudaFuncSetAttribute(proj_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    LaunchScope scope(g.name ? g.name : "gemm_tc", s);
    int grid = p.tiles < sms ? p.tiles : sms;
    if (g.max_ctas > 0 && grid > g.max_ctas) grid = g.max_ctas;
    proj_tc_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_proj_full_tc(const void* A, const void* const theta[3], float* const out[3], int T, int N, int K,
                                int accumulate, int* status, int max_ctas, cudaStream_t s) {
    GemmTc g{};
    g.nw = 3;
    g.nseg = 1;
    g.M = T;
    g.N = N;
    g.K = K;
    for (int w = 0; w < 3; ++w) {
        g.A[w][0] = {A, K};
        g.B[w][0] = {theta[w], K};
        g.C[w] = out[w];
    }
    g.ldc = N;
    g.accumulate = accumulate;
    g.status = status;
    g.max_ctas = max_ctas;
    g.name = "proj_full_tc";
    return launch_gemm_tc(g, s);
}

}  // namespace ttt
