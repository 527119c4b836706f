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
// the z reads token by token.  fp32 throughout; z goes to a buffer in X's
// layout, the gate runs afterwards as its own kernel.
#include "common.cuh"
#include "internal.h"

namespace ttt {
namespace {

constexpr int TT = 64;   // tokens per shared-memory tile
constexpr int R = 16;    // rows of W per CTA

template <int D>
__global__ void __launch_bounds__(4 * R) scan_linear_kernel(LinearScanArgs a) {
    constexpr int JD = D / 4;
    extern __shared__ float smf[];
    float* Qs = smf;             // [TT][D]
    float* Ks = Qs + TT * D;     // [TT][D]
    float* Vs = Ks + TT * D;     // [TT][R]: my rows only
    float* Es = Vs + TT * R;     // [TT][R]
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
    // Tile of tokens [n0, n0 + nt) in walking order into shared memory.
    auto load_tile = [&](int n0, int nt) {
        __syncthreads();   // the previous tile's Zs is written out and nothing reads Qs/Ks/Vs
        for (int p = tid; p < nt * (D / 4); p += 4 * R) {
            const int u = p / (D / 4), q4 = p % (D / 4);
            const long long off = (long long)h * a.qkv_hs + (long long)token(n0 + u) * a.qkv_ts + 4 * q4;
            reinterpret_cast<float4*>(Qs + u * D)[q4] = *reinterpret_cast<const float4*>(a.Q + off);
            reinterpret_cast<float4*>(Ks + u * D)[q4] = *reinterpret_cast<const float4*>(a.K + off);
        }
        for (int p = tid; p < nt * (R / 4); p += 4 * R) {
            const int u = p / (R / 4), q4 = p % (R / 4);
            const long long off = (long long)h * a.qkv_hs + (long long)token(n0 + u) * a.qkv_ts + r0 + 4 * q4;
            reinterpret_cast<float4*>(Vs + u * R)[q4] = *reinterpret_cast<const float4*>(a.V + off);
        }
        __syncthreads();
    };
    auto store_tile = [&](int n0, int nt) {
        __syncthreads();
        for (int p = tid; p < nt * (R / 4); p += 4 * R) {
            const int u = p / (R / 4), q4 = p % (R / 4);
            const long long off = (long long)h * a.x_hs + (long long)token(n0 + u) * a.x_ts + r0 + 4 * q4;
            *reinterpret_cast<float4*>(a.Z + off) = reinterpret_cast<const float4*>(Zs + u * R)[q4];
        }
    };
    auto quad_sum = [](float s) {
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        return s;
    };
    // Running update with e (already the full row value) and the z read of token u of the tile.
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

    if (b == 1) {
        // every token is its own chunk: e from the running state, then the step
        for (int n0 = 0; n0 < T; n0 += TT) {
            const int nt = min(TT, T - n0);
            load_tile(n0, nt);
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
            store_tile(n0, nt);
        }
    } else {
        for (int s0 = 0; s0 < T; s0 += b) {
            const int bc = min(b, T - s0);
            for (int p0 = 0; p0 < bc; p0 += TT) {
                const int nt = min(TT, bc - p0);
                load_tile(s0 + p0, nt);
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
                store_tile(s0 + p0, nt);
            }
#pragma unroll
            for (int jj = 0; jj < JD; ++jj) wc[jj] = wr[jj];   // the next chunk's gradients at this state
        }
    }

    if (a.W_T) {
        float* wt = a.W_T + ((long long)h * D + i) * D + c * JD;
#pragma unroll
        for (int jj = 0; jj < JD; ++jj) wt[jj] = wr[jj];
    }
}

template <int D>
cudaError_t launch_d(const LinearScanArgs& a, cudaStream_t s) {
    const size_t smem = sizeof(float) * ((size_t)2 * TT * D + 3 * TT * R);
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
