// Per-token (b = 1) TTT-MLP scan, d = 64, with each head's state sharded over
// a cluster of four CTAs (the state resident on chip for the whole sequence).
//
// Per token (paper notes page, "关键设计 / TTT-MLP 层"):
//   a = W1 k, g = GELU(a), e' = -2 eta (W2 g - v),
//   W2 <- W2 + e' g^T,  W1 <- W1 + ((W2_old^T e') * GELU'(a)) k^T,
//   z = W2 GELU(W1 q)  with the updated state;  out = x + tanh(alpha) z.
//
// CTA r of a head's cluster owns hidden units [64 r, 64 r + 64); thread
// (i, qd) of its 256 holds a quarter of row i of W1 (columns 16 qd .. +15) and
// of column i of W2 (rows 16 qd .. +15) in registers.  So W1 u and W2^T e' are
// 16 products and two shuffles, the rank-1 updates are thread-local, and the
// sums over hidden units (W2 g for the token's y, W2 g_q for the previous
// token's z) are a shuffle reduce-scatter inside a warp, a sum over the 8
// warps in shared memory, and a sum over the 4 CTAs whose partials cross
// distributed shared memory as 16-byte asynchronous stores that complete bytes
// on the receiver's barrier.  The previous token's z is summed together with
// the current token's y (both read the same state), so each token costs one
// exchange.  The receive buffers and barriers alternate by token parity: a CTA
// sends token n + 2's partials only after it received every peer's token n + 1
// partials, which each peer sends only after it read its buffer for token n.
#include "common.cuh"
#include "internal.h"
#include "tc_prims.cuh"

namespace ttt {
namespace {

constexpr int DT = 64, MLOC = 64, NCTA = 4, NT = 256, TOKB = 32;

#ifdef TTT_DEBUG_STAGES
// Debug builds only: cycles between phase boundaries seen by thread 0 of CTA 0.
__device__ float* g_dbg_tok = nullptr;
#define STAMPT(k)                                         \
    do {                                                  \
        if (tid == 0 && blockIdx.x == 0) {                \
            const long long now_ = clock64();             \
            stamp_acc[k] += now_ - stamp_last;            \
            stamp_last = now_;                            \
        }                                                 \
    } while (0)
#else
#define STAMPT(k) \
    do {          \
    } while (0)
#endif

// Sum of p[0..15] over the 8 lanes of a warp that share lane bits 0-1 (the
// quarter qd); afterwards the lane holds the sums for rows base, base + 1 of
// its quarter's 16.
__device__ __forceinline__ void reduce8(float (&p)[16], int lane, float& s0, float& s1, int& base) {
    float v[8];
    const bool u16 = lane & 16;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float send = u16 ? p[k] : p[k + 8];
        const float keep = u16 ? p[k + 8] : p[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    base = u16 ? 8 : 0;
    const bool u8 = lane & 8;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float send = u8 ? v[k] : v[k + 4];
        const float keep = u8 ? v[k + 4] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    base += u8 ? 4 : 0;
    const bool u4 = lane & 4;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float send = u4 ? v[k] : v[k + 2];
        const float keep = u4 ? v[k + 2] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    base += u4 ? 2 : 0;
    s0 = v[0];
    s1 = v[1];
}

__global__ void __launch_bounds__(NT, 1) scan_token_cluster_kernel(ScanArgs a) {
    __shared__ __align__(16) float sK[TOKB][DT], sQ[TOKB][DT], sV[TOKB][DT], sX[TOKB][DT];
    __shared__ __align__(16) float sY[NT / 32][DT], sZ[NT / 32][DT];
    __shared__ __align__(16) float rcv[2][NCTA][2 * DT];   // [token parity][sender][y partial | z partial]
    __shared__ __align__(16) float sE[DT];   // 16-byte loads of sK, sQ, sE rows
    __shared__ __align__(8) uint64_t rcvbar[2];   // the peers' partials of a token parity have landed
    __shared__ int abort_flag;

    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int il = tid >> 2, qd = tid & 3;
    const uint32_t r_cta = tc::cluster_ctarank();
    const int h = blockIdx.x / NCTA;
    const int i = (int)r_cta * MLOC + il;   // my hidden unit
    const int T = a.T, M = a.m;
    const float m2eta = -2.0f * a.eta;

    float w1[16], w2[16], qprev[16];
    {
        const float* W1 = a.W1_0 + ((long long)h * M + i) * DT + 16 * qd;
        const float* W2 = a.W2_0 + (long long)h * DT * M + (long long)(16 * qd) * M + i;
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
            w1[jj] = W1[jj];
            w2[jj] = W2[(long long)jj * M];
            qprev[jj] = 0.f;
        }
    }
    const int jout = tid - DT;   // threads 64..127 finish z for channel jout
    float tanh_a = 0.f;
    if (jout >= 0 && jout < DT) tanh_a = tanhf(a.alpha[h * DT + jout]);
    int nonfinite = 0;
    const uint32_t rcv_base = tc::smem_u32(&rcv[0][0][0]);
    constexpr uint32_t kPeerBytes = (NCTA - 1) * 32 * 16;   // three peers x 32 x 16-byte stores per token
    if (tid == 0) {
        tc::mbar_init(&rcvbar[0], 1);
        tc::mbar_init(&rcvbar[1], 1);
        abort_flag = 0;
        tc::fence_mbar_init();
        tc::mbar_arrive_expect_tx(&rcvbar[0], kPeerBytes);   // tokens 0 and 1
        tc::mbar_arrive_expect_tx(&rcvbar[1], kPeerBytes);
    }
    tc::cluster_sync();   // every CTA of the cluster runs, its barriers armed, before any distributed store

#ifdef TTT_DEBUG_STAGES
    long long stamp_acc[12] = {};
    long long stamp_last = clock64();
#endif
    float g = 0.f, gp = 0.f, xprev = 0.f;   // xprev: the gate's x of the previous token, my channel
    float kk[16], qcur[16];
    for (int n = 0; n <= T; ++n) {   // n = T: only the last token's z
        const bool tok = n < T, prev = n > 0;
        const int r = n % TOKB;
        if (tok && r == 0) {   // the next 32 tokens' q, k, v
            __syncthreads();
            const int nb = min(TOKB, T - n);
            for (int idx = tid; idx < nb * DT; idx += NT) {
                const int rr = idx / DT, j = idx % DT;
                const int t = a.reverse ? (T - 1 - (n + rr)) : (n + rr);
                const long long off = (long long)h * a.qkv_hs + (long long)t * a.qkv_ts + j;
                sK[rr][j] = a.K[off];
                sQ[rr][j] = a.Q[off];
                sV[rr][j] = a.V[off];
                sX[rr][j] = load_elem(a.Xin, (long long)h * a.x_hs + (long long)t * a.x_ts + j, a.xin_bf16);
            }
            __syncthreads();
        }
        STAMPT(0);
        // ---- A: y partial of token n and z partial of token n-1, both with the current state (the
        //      two chains interleaved; for n = T or n = 0 one of them is computed and not used)
        {
            const float4* k4 = reinterpret_cast<const float4*>(&sK[r][16 * qd]);
            const float4* q4 = reinterpret_cast<const float4*>(&sQ[r][16 * qd]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float4 f = k4[c], fq = q4[c];
                kk[4 * c] = f.x; kk[4 * c + 1] = f.y; kk[4 * c + 2] = f.z; kk[4 * c + 3] = f.w;
                qcur[4 * c] = fq.x; qcur[4 * c + 1] = fq.y; qcur[4 * c + 2] = fq.z; qcur[4 * c + 3] = fq.w;
            }
            float ak[4] = {0.f, 0.f, 0.f, 0.f}, aq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                ak[jj & 3] = fmaf(w1[jj], kk[jj], ak[jj & 3]);
                aq[jj & 3] = fmaf(w1[jj], qprev[jj], aq[jj & 3]);
            }
            float xa = (ak[0] + ak[1]) + (ak[2] + ak[3]), xq = (aq[0] + aq[1]) + (aq[2] + aq[3]);
            xa += __shfl_xor_sync(0xffffffffu, xa, 1);
            xq += __shfl_xor_sync(0xffffffffu, xq, 1);
            xa += __shfl_xor_sync(0xffffffffu, xa, 2);
            xq += __shfl_xor_sync(0xffffffffu, xq, 2);
            gelu_and_prime(xa, g, gp);
            const float gq = gelu(xq);
            float py[16], pz[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                py[jj] = w2[jj] * g;
                pz[jj] = w2[jj] * gq;
            }
            int by, bz;
            float y0, y1, z0, z1;
            reduce8(py, lane, y0, y1, by);
            reduce8(pz, lane, z0, z1, bz);
            sY[w][16 * qd + by] = y0;
            sY[w][16 * qd + by + 1] = y1;
            sZ[w][16 * qd + bz] = z0;
            sZ[w][16 * qd + bz + 1] = z1;
        }
        STAMPT(1);
        __syncthreads();
        STAMPT(2);
        // ---- B: this CTA's partials (warp 0: 4 consecutive sums per lane) into its own slot of every
        //      CTA's receive buffer: a plain store here, 16-byte stores that complete bytes on the receive
        //      barrier of the three peers
        const int par = n & 1;
        if (w == 0) {
            const int k0 = 4 * lane;   // y sums 0..63, z sums 64..127
            const bool isy = k0 < DT;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (isy ? tok : prev) {
#pragma unroll
                for (int ww = 0; ww < NT / 32; ++ww) {
                    const float4 f = *reinterpret_cast<const float4*>(isy ? &sY[ww][k0] : &sZ[ww][k0 - DT]);
                    v.x += f.x; v.y += f.y; v.z += f.z; v.w += f.w;
                }
            }
            *reinterpret_cast<float4*>(&rcv[par][r_cta][k0]) = v;
            const uint32_t off = (uint32_t)(((par * NCTA + (int)r_cta) * 2 * DT + k0) * 4);
            const uint32_t bar = tc::smem_u32(&rcvbar[par]);
#pragma unroll
            for (int d1 = 1; d1 < NCTA; ++d1) {
                const uint32_t dst = (r_cta + (uint32_t)d1) % NCTA;
                tc::st_async_v4(tc::mapa_shared(rcv_base + off, dst), __float_as_uint(v.x), __float_as_uint(v.y),
                                __float_as_uint(v.z), __float_as_uint(v.w), tc::mapa_shared(bar, dst));
            }
        }
        STAMPT(3);
        __syncthreads();   // my own partials are visible
        if (tid < 2 * DT) {   // the peers' partials of this token have landed (bounded wait)
            if (!tc::mbar_wait_cluster_abort(&rcvbar[par], (uint32_t)(n >> 1) & 1u, &abort_flag)) {
                abort_flag = 1;
                atomicOr(a.status, kStatusTimeout);
            }
            // arm the barrier for token n + 2 (its bytes come only after this CTA's token n + 1 partials)
            if (tid == 0) tc::mbar_arrive_expect_tx(&rcvbar[par], kPeerBytes);
        }
        STAMPT(4);
        // ---- C: e' of token n; z and the gate of token n-1 (each CTA stores 16 of the 64 channels)
        if (tid < DT) {
            if (tok) {
                float y = 0.f;
#pragma unroll
                for (int src = 0; src < NCTA; ++src) y += rcv[par][src][tid];
                sE[tid] = m2eta * (y - sV[r][tid]);
            }
        } else if (jout < DT && prev && (jout >> 4) == (int)r_cta) {
            float z = 0.f;
#pragma unroll
            for (int src = 0; src < NCTA; ++src) z += rcv[par][src][DT + jout];
            const int t = a.reverse ? (T - n) : (n - 1);
            const long long xo = (long long)h * a.x_hs + (long long)t * a.x_ts + jout;
            const float dz = tanh_a * z;
            store_elem(a.Out, xo, a.out_bf16, xprev + dz);
            if (a.Delta) a.Delta[xo] = __float2bfloat16_rn(dz);
            if (a.Zdbg) a.Zdbg[xo] = z;
            nonfinite |= !isfinite(z);
        }
        STAMPT(5);
        if (__syncthreads_or(abort_flag)) break;
        STAMPT(6);
        // ---- D: the update with e' (W2^T e' read before W2 changes)
        if (tok) {
            float ee[16];
            const float4* e4 = reinterpret_cast<const float4*>(&sE[16 * qd]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float4 f = e4[c];
                ee[4 * c] = f.x; ee[4 * c + 1] = f.y; ee[4 * c + 2] = f.z; ee[4 * c + 3] = f.w;
            }
            STAMPT(8);
            float bk[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) bk[jj & 3] = fmaf(w2[jj], ee[jj], bk[jj & 3]);
            float back = (bk[0] + bk[1]) + (bk[2] + bk[3]);
            back += __shfl_xor_sync(0xffffffffu, back, 1);
            back += __shfl_xor_sync(0xffffffffu, back, 2);
            const float dl = back * gp;
            STAMPT(9);
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                w1[jj] = fmaf(dl, kk[jj], w1[jj]);
                w2[jj] = fmaf(ee[jj], g, w2[jj]);
                qprev[jj] = qcur[jj];
            }
            if (jout >= 0 && jout < DT) xprev = sX[r][jout];
        }
        STAMPT(7);
    }
    if (a.W1_T) {
        float* W1 = a.W1_T + ((long long)h * M + i) * DT + 16 * qd;
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) W1[jj] = w1[jj];
    }
    if (a.W2_T) {
        float* W2 = a.W2_T + (long long)h * DT * M + (long long)(16 * qd) * M + i;
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) W2[(long long)jj * M] = w2[jj];
    }
    if (nonfinite) atomicOr(a.status, kStatusNonFinite);
#ifdef TTT_DEBUG_STAGES
    if (tid == 0 && blockIdx.x == 0 && g_dbg_tok) {
        for (int k = 0; k < 12; ++k) g_dbg_tok[k] = (float)stamp_acc[k];
        g_dbg_tok[12] = (float)T;
    }
#endif
    if (abort_flag) {   // let a peer's stores already in flight land before the memory goes away
        const uint64_t t0 = tc::globaltimer_ns();
        while (tc::globaltimer_ns() - t0 < 1000000ull) __nanosleep(1000);
    }
    tc::cluster_sync();   // no CTA leaves while a peer may still address its shared memory
}

}  // namespace

#ifdef TTT_DEBUG_STAGES
extern "C" __attribute__((visibility("default"))) int ttt_debug_set_dump_tok(float* p) {
    return (int)cudaMemcpyToSymbol(g_dbg_tok, &p, sizeof(p));
}
#endif

bool scan_token_cluster_supported(int d) { return d == DT; }

cudaError_t launch_scan_token_cluster(const ScanArgs& a, cudaStream_t s) {
    if (!scan_token_cluster_supported(a.d) || a.m != 4 * DT) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(NCTA * a.H);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = NCTA;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    LaunchScope scope("scan_token_cluster", s);
    cudaError_t e = cudaLaunchKernelEx(&cfg, scan_token_cluster_kernel, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace ttt
