// TTT-Linear scan: the layer with a linear hidden state f(u; W) = W u,
// W [d x d] per head (paper notes page, "实验关键数据 / 消融实验": TTT-Linear;
// loss, update rule and prefix reading as in "关键设计 / TTT-MLP 层").  For
// the loss ||W k - v||^2 the gradient is 2 (W k - v) k^T, so with e = W_c k - v
// (W_c the chunk-start state) a token's step is the rank-1 update
//     W <- W - 2 eta e k^T,
// and token t is read with the running state after its own update: z_t = W q_t.
//
// Rows of W are independent (row i needs only its own e_i and the shared k, q),
// so a head is split over CTAs of R rows with no communication; thread (i, c)
// holds columns [c d/4, (c+1) d/4) of row i of both the chunk-start and the
// running state in registers, and the row sums are reductions over the four
// threads of a quad.  Tokens stream through shared memory in tiles of 64 (in
// walking order; the reverse direction walks t = T-1 .. 0): first e for every
// token of the tile (one state, independent sums), then the running updates and
// the z reads token by token.  The next tile streams in by asynchronous copies
// into a second buffer while one is computed.  fp32 throughout; z goes to a
// buffer in X's layout, the gate runs afterwards as its own kernel.
#include "common.cuh"
#include "internal.h"

namespace ttt {
namespace {

constexpr int TT = 64;   // tokens per shared-memory tile
constexpr int R = 16;    // rows of W per CTA

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
                 "l"(gmem)
                 : "memory");
}

template <int D>
__global__ void __launch_bounds__(4 * R) scan_linear_kernel(LinearScanArgs a) {
    constexpr int JD = D / 4;
    constexpr int BUF = 2 * TT * D + TT * R;   // one tile: Q, K [TT][D], V [TT][R] (my rows)
    extern __shared__ __align__(16) float smf[];
    float* Es = smf + 2 * BUF;   // [TT][R]
    float* Zs = Es + TT * R;     // [TT][R]
    const int cta_per_head = D / R;
    const int h = blockIdx.x / cta_per_head, r0 = (blockIdx.x % cta_per_head) * R;
    const int tid = threadIdx.x, il = tid >> 2, c = tid & 3, i = r0 + il;
    const int T = a.T, b = a.b;
    const float two_eta = 2.0f * a.eta;

    float wc[JD], wr[JD];
    {
        const float* w0 = a.W_0 + ((long long)h * D + i) * D + c * JD;
        int bad = 0;
#pragma unroll
        for (int jj = 0; jj < JD; ++jj) {
            wc[jj] = wr[jj] = w0[jj];
            bad |= !isfinite(w0[jj]);
        }
        if (bad) atomicOr(a.status, kStatusNonFinite);
    }

    auto token = [&](int n) { return a.reverse ? T - 1 - n : n; };
    // Tiles of at most TT tokens in walking order that never straddle a chunk
    // (b == 1: every token is a chunk of its own and is handled inline).
    const int CL = (b == 1) ? T : b;
    int it_s0 = 0, it_p0 = 0;
    auto next_tile = [&](int& n0, int& nt, int& chunk_end) -> bool {
        if (it_s0 >= T) return false;
        const int bc = min(CL, T - it_s0);
        n0 = it_s0 + it_p0;
        nt = min(TT, bc - it_p0);
        it_p0 += nt;
        chunk_end = it_p0 >= bc;
        if (chunk_end) { it_s0 += CL; it_p0 = 0; }
        return true;
    };
    // Asynchronous 16-byte copies of a tile into buffer `buf` (one commit group).
    auto issue_load = [&](int buf, int n0, int nt) {
        float* Qs = smf + buf * BUF;
        float* Ks = Qs + TT * D;
        float* Vs = Ks + TT * D;
        for (int p = tid; p < nt * (D / 4); p += 4 * R) {
            const int u = p / (D / 4), q4 = p % (D / 4);
            const long long off = (long long)h * a.qkv_hs + (long long)token(n0 + u) * a.qkv_ts + 4 * q4;
            cp_async16(Qs + u * D + 4 * q4, a.Q + off);
            cp_async16(Ks + u * D + 4 * q4, a.K + off);
        }
        for (int p = tid; p < nt * (R / 4); p += 4 * R) {
            const int u = p / (R / 4), q4 = p % (R / 4);
            const long long off = (long long)h * a.qkv_hs + (long long)token(n0 + u) * a.qkv_ts + r0 + 4 * q4;
            cp_async16(Vs + u * R + 4 * q4, a.V + off);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    auto quad_sum = [](float s) {
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        return s;
    };

    int n0 = 0, nt = 0, ce = 0, buf = 0;
    bool have = next_tile(n0, nt, ce);
    if (have) issue_load(0, n0, nt);
    while (have) {
        int n0n = 0, ntn = 0, cen = 0;
        const bool haven = next_tile(n0n, ntn, cen);
        if (haven) {   // the other buffer was released by the barrier that ended the previous tile
            issue_load(buf ^ 1, n0n, ntn);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();   // this tile's copies (every thread's) have landed
        const float* Qs = smf + buf * BUF;
        const float* Ks = Qs + TT * D;
        const float* Vs = Ks + TT * D;
        // Running update with e (the full row value) and the z read of token u.
        auto step = [&](int u, float e) {
            const float* k = Ks + u * D + c * JD;
            const float* q = Qs + u * D + c * JD;
            float z0 = 0.f, z1 = 0.f;
#pragma unroll
            for (int jj = 0; jj < JD; jj += 2) {
                wr[jj] = fmaf(-two_eta * e, k[jj], wr[jj]);
                wr[jj + 1] = fmaf(-two_eta * e, k[jj + 1], wr[jj + 1]);
                z0 = fmaf(wr[jj], q[jj], z0);
                z1 = fmaf(wr[jj + 1], q[jj + 1], z1);
            }
            const float z = quad_sum(z0 + z1);
            if (c == 0) Zs[u * R + il] = z;
        };
        if (b == 1) {   // e from the running state, then the step, token by token
            for (int u = 0; u < nt; ++u) {
                const float* k = Ks + u * D + c * JD;
                float s0 = 0.f, s1 = 0.f;
#pragma unroll
                for (int jj = 0; jj < JD; jj += 2) {
                    s0 = fmaf(wr[jj], k[jj], s0);
                    s1 = fmaf(wr[jj + 1], k[jj + 1], s1);
                }
                step(u, quad_sum(s0 + s1) - Vs[u * R + il]);
            }
        } else {
            // e of every token of the tile at the chunk-start state
            for (int u = 0; u < nt; ++u) {
                const float* k = Ks + u * D + c * JD;
                float e0 = 0.f, e1 = 0.f;
#pragma unroll
                for (int jj = 0; jj < JD; jj += 2) {
                    e0 = fmaf(wc[jj], k[jj], e0);
                    e1 = fmaf(wc[jj + 1], k[jj + 1], e1);
                }
                const float e = quad_sum(e0 + e1);
                if (c == 0) Es[u * R + il] = e - Vs[u * R + il];
            }
            __syncwarp();   // a quad's Es entry is written and read within one warp
            for (int u = 0; u < nt; ++u) step(u, Es[u * R + il]);
            if (ce) {
#pragma unroll
                for (int jj = 0; jj < JD; ++jj) wc[jj] = wr[jj];   // the next chunk's gradients at this state
            }
        }
        __syncthreads();   // Zs complete
        for (int p = tid; p < nt * (R / 4); p += 4 * R) {
            const int u = p / (R / 4), q4 = p % (R / 4);
            const long long off = (long long)h * a.x_hs + (long long)token(n0 + u) * a.x_ts + r0 + 4 * q4;
            *reinterpret_cast<float4*>(a.Z + off) = reinterpret_cast<const float4*>(Zs + u * R)[q4];
        }
        __syncthreads();   // Zs and this tile's buffer are free again
        n0 = n0n; nt = ntn; ce = cen; have = haven; buf ^= 1;
    }

    if (a.W_T) {
        float* wt = a.W_T + ((long long)h * D + i) * D + c * JD;
#pragma unroll
        for (int jj = 0; jj < JD; ++jj) wt[jj] = wr[jj];
    }
}

template <int D>
cudaError_t launch_d(const LinearScanArgs& a, cudaStream_t s) {
    const size_t smem = sizeof(float) * (2 * ((size_t)2 * TT * D + TT * R) + 2 * TT * R);
    cudaError_t e = cudaFuncSetAttribute(scan_linear_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    LaunchScope scope("scan_linear", s);
    scan_linear_kernel<D><<<a.H * (D / R), 4 * R, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool scan_linear_supported(int d) { return d == 16 || d == 32 || d == 64; }

cudaError_t launch_scan_linear(const LinearScanArgs& a, cudaStream_t s) {
    switch (a.d) {
        case 16: return launch_d<16>(a, s);
        case 32: return launch_d<32>(a, s);
        case 64: return launch_d<64>(a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ttt
