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

// d = 64: one head, 512 tokens per CTA in tiles of 128.  U [128 x 192] =
// X [128 x 64] Theta^T [64 x 192] with both operands transposed in shared
// memory (k-major rows, so that a thread's 8 tokens and its 4-wide output
// groups are 16-byte loads) and 8 x 12 outputs per thread: 5 shared loads per
// 96 FMAs.  Thread (ty, tx) computes tokens 8 ty .. 8 ty + 7 and, for each of
// Q, K, V, channels 4 tx .. 4 tx + 3, so 16 threads store one 256-byte row of
// an output with float4 stores.
constexpr int kP64Tile = 128, kP64Tok = 512, kP64XS = kP64Tile + 4, kP64TS = 3 * 64 + 4;

__global__ void __launch_bounds__(256, 2)
proj_per_head64_kernel(const void* X, int x_bf16, const void* thq, const void* thk, const void* thv, int th_bf16,
                       float* oq, float* ok, float* ov, int T, int* status) {
    extern __shared__ __align__(16) float sm64[];
    float* thT = sm64;                  // [64][kP64TS]: thT[k][w 64 + e] = theta_w[h][e][k]
    float* xT = sm64 + 64 * kP64TS;     // [64][kP64XS]: xT[k][r] = x[h][t0 + r][k]
    const int h = blockIdx.y, tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const void* ths[3] = {thq, thk, thv};
    float* outs[3] = {oq, ok, ov};
    for (int p = tid; p < 3 * 64 * 64; p += 256) {   // consecutive threads read consecutive k of a row e
        const int w = p >> 12, e = (p >> 6) & 63, k = p & 63;
        thT[k * kP64TS + w * 64 + e] = load_elem(ths[w], (long long)h * 4096 + e * 64 + k, th_bf16);
    }
    int bad = 0;
    for (int t0 = blockIdx.x * kP64Tok; t0 < min(T, (int)(blockIdx.x + 1) * kP64Tok); t0 += kP64Tile) {
        const int nt = min(kP64Tile, T - t0);
        __syncthreads();   // the previous tile's xT reads are done (and theta is in place)
        for (int p = tid; p < kP64Tile * 64; p += 256) {
            const int r = p >> 6, k = p & 63;
            xT[k * kP64XS + r] = r < nt ? load_elem(X, ((long long)h * T + t0 + r) * 64 + k, x_bf16) : 0.f;
        }
        __syncthreads();
        float acc[8][12];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int c = 0; c < 12; ++c) acc[i][c] = 0.f;
#pragma unroll 2
        for (int k = 0; k < 64; ++k) {
            const float4 x0 = *reinterpret_cast<const float4*>(xT + k * kP64XS + 8 * ty);
            const float4 x1 = *reinterpret_cast<const float4*>(xT + k * kP64XS + 8 * ty + 4);
            const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
            float tv[12];
#pragma unroll
            for (int g = 0; g < 3; ++g) {
                const float4 f = *reinterpret_cast<const float4*>(thT + k * kP64TS + 64 * g + 4 * tx);
                tv[4 * g] = f.x; tv[4 * g + 1] = f.y; tv[4 * g + 2] = f.z; tv[4 * g + 3] = f.w;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int c = 0; c < 12; ++c) acc[i][c] = fmaf(xv[i], tv[c], acc[i][c]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = 8 * ty + i;
            if (r >= nt) continue;
#pragma unroll
            for (int g = 0; g < 3; ++g) {
                const float4 v = make_float4(acc[i][4 * g], acc[i][4 * g + 1], acc[i][4 * g + 2], acc[i][4 * g + 3]);
                bad |= !(isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w));
                *reinterpret_cast<float4*>(outs[g] + ((long long)h * T + t0 + r) * 64 + 4 * tx) = v;
            }
        }
    }
    if (__syncthreads_or(bad) && tid == 0) atomicOr(status, kStatusNonFinite);
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
    if (d == 64) {   // the register-tiled kernel
        const size_t smem = sizeof(float) * (64 * (size_t)kP64TS + 64 * (size_t)kP64XS);
        cudaError_t e = cudaFuncSetAttribute(proj_per_head64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        LaunchScope scope("proj_per_head", s);
        dim3 grid((T + kP64Tok - 1) / kP64Tok, H);
        proj_per_head64_kernel<<<grid, 256, smem, s>>>(X, x_bf16, theta[0], theta[1], theta[2], th_bf16, out[0],
                                                        out[1], out[2], T, status);
        return cudaGetLastError();
    }
    switch (d) {
        case 16: return run(proj_per_head_kernel<16>, 16);
        case 32: return run(proj_per_head_kernel<32>, 32);
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
