// theta_Q / theta_K / theta_V projections on the FP32 SIMT pipe.
//
// Per-head mode: q_t = theta_Q[h] x_t for every head and token (a d x d
// matrix-vector product per token); full mode: U = X Theta^T with X [T, Dm]
// and Theta [N, Dm] (the nn.Linear layout), fp32 accumulation and output.
// Paper notes page, "关键设计 / TTT-MLP 层": theta_K, theta_V, theta_Q are the
// outer-loop key/value/query projections.
#include "common.cuh"
#include "internal.h"

namespace ttt {
namespace {

constexpr int kPhTok = 256;      // tokens per CTA, per-head projection (theta loaded once per 256 tokens)
constexpr int kPhThreads = 256;

// One head, 256 tokens: U [tokens x 3d] = X [tokens x d] Theta^T [d x 3d] with
// Theta = [theta_Q; theta_K; theta_V] of the head, both operands in shared
// memory (x rows padded to d + 1), 64 x 64 output blocks, 4 x 4 per thread.
template <int D>
__global__ void __launch_bounds__(kPhThreads)
proj_per_head_kernel(const void* X, int x_bf16, const void* thq, const void* thk, const void* thv,
                     int th_bf16, float* oq, float* ok, float* ov, int T, int* status) {
    constexpr int N3 = 3 * D, XP = D + 1;
    extern __shared__ float sm[];
    float* thT = sm;                    // [D][3D]: thT[j][w D + e] = theta_w[h][e][j]
    float* xs = sm + D * N3;            // [kPhTok][D + 1]
    const int h = blockIdx.y;
    const int t0 = blockIdx.x * kPhTok;
    const int nt = min(kPhTok, T - t0);
    const void* ths[3] = {thq, thk, thv};
    const int tid = threadIdx.x;
    for (int p = tid; p < 3 * D * D; p += kPhThreads) {
        const int w = p / (D * D), q = p % (D * D), e = q / D, j = q % D;
        thT[j * N3 + w * D + e] = load_elem(ths[w], (long long)h * D * D + q, th_bf16);
    }
    for (int p = tid; p < nt * D; p += kPhThreads)
        xs[(p / D) * XP + p % D] = load_elem(X, ((long long)h * T + t0) * D + p, x_bf16);
    __syncthreads();
    float* outs[3] = {oq, ok, ov};
    const int tr = tid / 16, tc = tid % 16;
    int bad = 0;   // a non-finite input reaches every projection of its token
    for (int r0 = 0; r0 < nt; r0 += 64) {
        for (int n0 = 0; n0 < N3; n0 += 64) {
            float acc[4][4] = {};
#pragma unroll 4
            for (int j = 0; j < D; ++j) {
                float av[4], bv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) av[i] = xs[(r0 + tr + 16 * i) * XP + j];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int n = n0 + tc + 16 * k;
                    bv[k] = n < N3 ? thT[j * N3 + n] : 0.f;
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int k = 0; k < 4; ++k) acc[i][k] = fmaf(av[i], bv[k], acc[i][k]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = r0 + tr + 16 * i;
                if (r >= nt) continue;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int n = n0 + tc + 16 * k;
                    if (n >= N3) continue;
                    outs[n / D][((long long)h * T + t0 + r) * D + n % D] = acc[i][k];
                    bad |= !isfinite(acc[i][k]);
                }
            }
        }
    }
    if (__syncthreads_or(bad) && tid == 0) atomicOr(status, kStatusNonFinite);
}

// C[t, n] (+)= sum_c A[t, c] B[n, c]; 64 x 64 tile, 16-deep k steps, 4 x 4 per thread.
constexpr int kGT = 64, kGK = 16;

__global__ void __launch_bounds__(256)
proj_full_simt_kernel(const void* A, int a_bf16, const void* B0, const void* B1, const void* B2, int b_bf16,
                      float* C0, float* C1, float* C2, int T, int N, int Dm, int accumulate, int* status) {
    __shared__ float As[kGK][kGT + 4];
    __shared__ float Bs[kGK][kGT + 4];
    const void* B = blockIdx.z == 0 ? B0 : (blockIdx.z == 1 ? B1 : B2);
    float* C = blockIdx.z == 0 ? C0 : (blockIdx.z == 1 ? C1 : C2);
    const int n0 = blockIdx.x * kGT, t0 = blockIdx.y * kGT;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4] = {};
    for (int c0 = 0; c0 < Dm; c0 += kGK) {
        for (int p = threadIdx.x; p < kGT * kGK; p += 256) {
            const int r = p / kGK, c = p % kGK;
            const int t = t0 + r, n = n0 + r, cc = c0 + c;
            As[c][r] = (t < T && cc < Dm) ? load_elem(A, (long long)t * Dm + cc, a_bf16) : 0.f;
            Bs[c][r] = (n < N && cc < Dm) ? load_elem(B, (long long)n * Dm + cc, b_bf16) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < kGK; ++c) {
            float av[4], bv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) { av[u] = As[c][ty * 4 + u]; bv[u] = Bs[c][tx * 4 + u]; }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
        }
        __syncthreads();
    }
    int bad = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int t = t0 + ty * 4 + u;
        if (t >= T) continue;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int n = n0 + tx * 4 + v;
            if (n >= N) continue;
            float* dst = C + (long long)t * N + n;
            *dst = accumulate ? *dst + acc[u][v] : acc[u][v];
            bad |= !isfinite(acc[u][v]);
        }
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(status, kStatusNonFinite);
}

}  // namespace

cudaError_t launch_proj_per_head(const void* X, int x_bf16, const void* const theta[3], int th_bf16,
                                 float* const out[3], int T, int H, int d, int* status, cudaStream_t s) {
    auto run = [&](auto kernel, int D) -> cudaError_t {
        const size_t smem = sizeof(float) * (3 * (size_t)D * D + (size_t)kPhTok * (D + 1));
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        LaunchScope scope("proj_per_head", s);
        dim3 grid((T + kPhTok - 1) / kPhTok, H);
        kernel<<<grid, kPhThreads, smem, s>>>(X, x_bf16, theta[0], theta[1], theta[2], th_bf16, out[0], out[1],
                                              out[2], T, status);
        return cudaGetLastError();
    };
    switch (d) {
        case 16: return run(proj_per_head_kernel<16>, 16);
        case 32: return run(proj_per_head_kernel<32>, 32);
        case 64: return run(proj_per_head_kernel<64>, 64);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_proj_full_simt(const void* A, int a_bf16, const void* const theta[3], int th_bf16,
                                  float* const out[3], int T, int N, int Dm, int accumulate, int* status,
                                  cudaStream_t s) {
    LaunchScope scope("proj_full_simt", s);
    dim3 grid((N + kGT - 1) / kGT, (T + kGT - 1) / kGT, 3);
    proj_full_simt_kernel<<<grid, 256, 0, s>>>(A, a_bf16, theta[0], theta[1], theta[2], th_bf16, out[0], out[1],
                                                out[2], T, N, Dm, accumulate, status);
    return cudaGetLastError();
}

}  // namespace ttt
