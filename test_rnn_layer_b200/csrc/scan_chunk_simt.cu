// Chunked (mini-batch) TTT-MLP scan on the FP32 SIMT pipe: the reference
// CUDA kernel for every (d, b) the library accepts, and the fallback for
// shapes the tensor-core kernel does not take.
//
// One CTA per head.  The hidden state W1 [m x d], W2 [d x m] stays in shared
// memory for the whole sequence; the per-chunk intermediates live in a
// per-head scratch slice of the workspace (L2-resident).
//
// Per chunk of bc <= b tokens (rows r in walking order), with every gradient
// taken at the chunk-start state and token r read with the prefix state
// (paper notes page, "关键设计 / TTT-MLP 层", mini-batch reading), the chunk in
// matrix form is
//   A  = K W1^T,  G = GELU(A),  Gp = GELU'(A)
//   D2 = -2 eta (G W2^T - V)                     (= -eta dl/dy per token)
//   Dl = (D2 W2) * Gp                            (= -eta delta per token)
//   Aq = Q W1^T + tril(Q K^T) Dl,   Gq = GELU(Aq)
//   Z  = Gq W2^T + tril(Gq G^T) D2
//   W1 += Dl^T K,   W2 += D2^T G
// where tril keeps s <= r.  For bc = 1 this is the per-token rule.
#include "common.cuh"
#include "internal.h"

namespace ttt {
namespace {

constexpr int kThreads = 512;

// C[i, j] = alpha * sum_k A(i, k) B(k, j) (+ C[i, j] if acc).  A(i, k) at
// A[i * sai + k * sak], B(k, j) at B[k * sbk + j * sbj], C row-major with ldc.
// Element (i, j) is always computed by the same thread for a given (M, N),
// so two calls accumulating into the same C need no barrier in between.
__device__ void block_mm(int M, int N, int K, const float* A, int sai, int sak, const float* B,
                         int sbk, int sbj, float* C, int ldc, bool acc) {
    for (int idx = threadIdx.x; idx < M * N; idx += blockDim.x) {
        const int i = idx / N, j = idx % N;
        float s = 0.f;
        for (int k = 0; k < K; ++k) s = fmaf(A[i * sai + k * sak], B[k * sbk + j * sbj], s);
        C[i * ldc + j] = acc ? C[i * ldc + j] + s : s;
    }
}

// tril(P P2^T): S[r, s] = sum_k P[r, k] P2[s, k] for s <= r, else 0.
__device__ void block_tril_gram(int n, int K, const float* P, const float* P2, float* S) {
    for (int idx = threadIdx.x; idx < n * n; idx += blockDim.x) {
        const int r = idx / n, s = idx % n;
        float acc = 0.f;
        if (s <= r)
            for (int k = 0; k < K; ++k) acc = fmaf(P[r * K + k], P2[s * K + k], acc);
        S[idx] = acc;
    }
}

__global__ void __launch_bounds__(kThreads) scan_chunk_simt_kernel(ScanArgs a) {
    extern __shared__ float smem[];
    const int d = a.d, m = a.m, b = a.b, T = a.T;
    const int h = blockIdx.x;
    float* W1 = smem;              // [m][d]
    float* W2 = smem + m * d;      // [d][m]

    float* sc = a.scratch + (long long)h * a.scratch_per_head;
    float* Kc = sc;  sc += b * d;
    float* Qc = sc;  sc += b * d;
    float* Vc = sc;  sc += b * d;
    float* G = sc;   sc += b * m;
    float* Gp = sc;  sc += b * m;
    float* Dl = sc;  sc += b * m;
    float* Gq = sc;  sc += b * m;
    float* D2 = sc;  sc += b * d;
    float* Zc = sc;  sc += b * d;
    float* S = sc;   sc += b * b;

    for (int p = threadIdx.x; p < m * d; p += blockDim.x) {
        W1[p] = a.W1_0[(long long)h * m * d + p];
        W2[p] = a.W2_0[(long long)h * m * d + p];
    }
    const float eta = a.eta;
    int nonfinite = 0;
    __syncthreads();

    for (int n0 = 0; n0 < T; n0 += b) {
        const int bc = min(b, T - n0);
        for (int idx = threadIdx.x; idx < bc * d; idx += blockDim.x) {
            const int r = idx / d, j = idx % d;
            const int t = a.reverse ? (T - 1 - (n0 + r)) : (n0 + r);
            const long long off = (long long)h * a.qkv_hs + (long long)t * a.qkv_ts + j;
            Kc[idx] = a.K[off];
            Qc[idx] = a.Q[off];
            Vc[idx] = a.V[off];
        }
        __syncthreads();
        // A = K W1^T  (into G), then G = GELU(A), Gp = GELU'(A)
        block_mm(bc, m, d, Kc, d, 1, W1, 1, d, G, m, false);
        __syncthreads();
        for (int idx = threadIdx.x; idx < bc * m; idx += blockDim.x) {
            float g, gp;
            gelu_and_prime(G[idx], g, gp);
            G[idx] = g;
            Gp[idx] = gp;
        }
        __syncthreads();
        // D2 = -2 eta (G W2^T - V)
        block_mm(bc, d, m, G, m, 1, W2, 1, m, D2, d, false);
        __syncthreads();
        for (int idx = threadIdx.x; idx < bc * d; idx += blockDim.x)
            D2[idx] = -2.0f * eta * (D2[idx] - Vc[idx]);
        __syncthreads();
        // Dl = (D2 W2) * Gp;  S = tril(Q K^T)
        block_mm(bc, m, d, D2, d, 1, W2, m, 1, Dl, m, false);
        block_tril_gram(bc, d, Qc, Kc, S);
        __syncthreads();
        for (int idx = threadIdx.x; idx < bc * m; idx += blockDim.x) Dl[idx] *= Gp[idx];
        __syncthreads();
        // Aq = Q W1^T + S Dl;  Gq = GELU(Aq)
        block_mm(bc, m, d, Qc, d, 1, W1, 1, d, Gq, m, false);
        block_mm(bc, m, bc, S, bc, 1, Dl, m, 1, Gq, m, true);
        __syncthreads();
        for (int idx = threadIdx.x; idx < bc * m; idx += blockDim.x) Gq[idx] = gelu(Gq[idx]);
        __syncthreads();
        // Z = Gq W2^T + tril(Gq G^T) D2
        block_tril_gram(bc, m, Gq, G, S);
        block_mm(bc, d, m, Gq, m, 1, W2, 1, m, Zc, d, false);
        __syncthreads();
        block_mm(bc, d, bc, S, bc, 1, D2, d, 1, Zc, d, true);
        __syncthreads();
        // gate and stores
        for (int idx = threadIdx.x; idx < bc * d; idx += blockDim.x) {
            const int r = idx / d, j = idx % d;
            const int t = a.reverse ? (T - 1 - (n0 + r)) : (n0 + r);
            const long long xo = (long long)h * a.x_hs + (long long)t * a.x_ts + j;
            const float z = Zc[idx];
            const float dz = tanhf(a.alpha[h * d + j]) * z;
            store_elem(a.Out, xo, a.out_bf16, load_elem(a.Xin, xo, a.xin_bf16) + dz);
            if (a.Delta) a.Delta[xo] = __float2bfloat16_rn(dz);
            if (a.Zdbg) a.Zdbg[xo] = z;
            nonfinite |= !isfinite(z);
        }
        // state update: W1 += Dl^T K, W2 += D2^T G
        block_mm(m, d, bc, Dl, 1, m, Kc, d, 1, W1, d, true);
        block_mm(d, m, bc, D2, 1, d, G, m, 1, W2, m, true);
        __syncthreads();
    }
    for (int p = threadIdx.x; p < m * d; p += blockDim.x) {
        if (a.W1_T) a.W1_T[(long long)h * m * d + p] = W1[p];
        if (a.W2_T) a.W2_T[(long long)h * m * d + p] = W2[p];
    }
    if (nonfinite) atomicOr(a.status, kStatusNonFinite);
}

}  // namespace

long long scan_chunk_simt_scratch_floats(int d, int m, int b) {
    return (long long)b * (5LL * d + 4LL * m + b);
}

cudaError_t launch_scan_chunk_simt(const ScanArgs& a, cudaStream_t s) {
    const size_t smem = sizeof(float) * 2 * (size_t)a.m * a.d;
    cudaError_t e = cudaFuncSetAttribute(scan_chunk_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    LaunchScope scope("scan_chunk_simt", s);
    scan_chunk_simt_kernel<<<a.H, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace ttt
