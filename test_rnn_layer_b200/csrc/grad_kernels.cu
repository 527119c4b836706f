// Gradient kernels around the scan's backward pass (fp32 SIMT):
//   * the gate out = x + tanh(alpha) z (paper notes page, "关键设计 / 门控 + 双向机制")
//     backward: dz = tanh(alpha) g and dalpha_c += (1 - tanh^2 alpha_c) sum_t g_tc z_tc,
//     g the gradient with respect to the gate's output (its x-path gradient is g
//     itself, which the caller keeps);
//   * a batched, split-K GEMM C (+)= A B for the projections' gradients
//     (dX += dU theta and dtheta += dU^T X, per head or over the full width),
//     reading bf16 or fp32 operands through row/column strides.
#include "common.cuh"
#include "internal.h"

namespace ttt {
namespace {

// One thread per channel; blockIdx.y covers a range of tokens.
__global__ void __launch_bounds__(256) gate_bwd_kernel(const float* g, const float* z, const float* alpha, float* dz,
                                                       float* dalpha, int T, int H, int d, int per_head,
                                                       int tok_per_block) {
    const int D = H * d;
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= D) return;
    const int h = c / d, j = c % d;
    const float ta = tanhf(alpha[c]);
    const int t0 = blockIdx.y * tok_per_block, t1 = min(T, t0 + tok_per_block);
    float acc = 0.f;
    for (int t = t0; t < t1; ++t) {
        const long long i = per_head ? ((long long)h * T + t) * d + j : (long long)t * D + c;
        const float gv = g[i];
        acc = fmaf(gv, z[i], acc);
        dz[i] = ta * gv;
    }
    atomicAdd(dalpha + c, (1.0f - ta * ta) * acc);
}

constexpr int GM = 64, GN = 64, GK = 16, GT = 256;

struct GemmOp {
    const void* p;
    int bf16;
    long long rs, cs, bs;   // element (b, r, c) at p[b * bs + r * rs + c * cs]
    __device__ float at(int b, long long r, long long c) const {
        const long long i = (long long)b * bs + r * rs + c * cs;
        return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i])
                    : reinterpret_cast<const float*>(p)[i];
    }
};

// C[b] (+)= A[b] [M x K] B[b] [K x N]; C fp32 row-major (ldc, batch stride cbs).
// blockIdx.z = batch * ksplit + kpart; with ksplit > 1 the parts are added with atomics.
__global__ void __launch_bounds__(GT) gemm_kernel(float* C, long long ldc, long long cbs, GemmOp A, GemmOp B, int M,
                                                  int N, long long K, int ksplit, int accumulate) {
    __shared__ float sA[GK][GM + 1], sB[GK][GN + 1];
    const int bz = blockIdx.z / ksplit, kp = blockIdx.z % ksplit;
    const int m0 = blockIdx.y * GM, n0 = blockIdx.x * GN;
    const long long kchunk = (K + ksplit - 1) / ksplit;
    const long long k_lo = kp * kchunk, k_hi = min(K, k_lo + kchunk);
    const int tid = threadIdx.x, tr = tid / 16, tc = tid % 16;   // 16 x 16 threads, 4 x 4 outputs each
    float acc[4][4] = {};
    for (long long k0 = k_lo; k0 < k_hi; k0 += GK) {
        __syncthreads();
        // consecutive threads walk the operand's contiguous dimension (coalesced loads)
        for (int idx = tid; idx < GK * GM; idx += GT) {
            const int kk = A.cs == 1 ? idx % GK : idx / GM, mm = A.cs == 1 ? idx / GK : idx % GM;
            sA[kk][mm] = (m0 + mm < M && k0 + kk < k_hi) ? A.at(bz, m0 + mm, k0 + kk) : 0.f;
        }
        for (int idx = tid; idx < GK * GN; idx += GT) {
            const int kk = B.rs == 1 ? idx % GK : idx / GN, nn = B.rs == 1 ? idx / GK : idx % GN;
            sB[kk][nn] = (n0 + nn < N && k0 + kk < k_hi) ? B.at(bz, k0 + kk, n0 + nn) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < GK; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) av[i] = sA[kk][tr + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bv[j] = sB[kk][tc + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = m0 + tr + 16 * i, c = n0 + tc + 16 * j;
            if (r >= M || c >= N) continue;
            float* dst = C + (long long)bz * cbs + (long long)r * ldc + c;
            if (ksplit > 1) atomicAdd(dst, acc[i][j]);
            else *dst = accumulate ? *dst + acc[i][j] : acc[i][j];
        }
}

// hi = bf16(x) (nearest), lo = bf16(x - hi): the pair carries 16 bits of x's 24-bit significand, so a
// product with a bf16 operand formed as hi b + lo b keeps about 2^-16 relative; four elements per thread.
__global__ void __launch_bounds__(256) split_bf16_kernel(const float4* x, uint2* hi, uint2* lo, long long n4) {
    for (long long i = blockIdx.x * 256LL + threadIdx.x; i < n4; i += (long long)gridDim.x * 256) {
        const float4 v = x[i];
        const __nv_bfloat162 h01 = __floats2bfloat162_rn(v.x, v.y), h23 = __floats2bfloat162_rn(v.z, v.w);
        const __nv_bfloat162 l01 = __floats2bfloat162_rn(v.x - __low2float(h01), v.y - __high2float(h01));
        const __nv_bfloat162 l23 = __floats2bfloat162_rn(v.z - __low2float(h23), v.w - __high2float(h23));
        hi[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
        lo[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&l01), *reinterpret_cast<const uint32_t*>(&l23));
    }
}

}  // namespace

cudaError_t launch_split_bf16(const float* x, __nv_bfloat16* hi, __nv_bfloat16* lo, long long n, cudaStream_t s) {
    if (n % 4 != 0) return cudaErrorInvalidValue;
    const long long n4 = n / 4;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long want = (n4 + 255) / 256;
    const int grid = (int)(want < 8LL * sms ? want : 8LL * sms);
    LaunchScope scope("split_bf16", s);
    split_bf16_kernel<<<grid > 0 ? grid : 1, 256, 0, s>>>(reinterpret_cast<const float4*>(x),
                                                           reinterpret_cast<uint2*>(hi), reinterpret_cast<uint2*>(lo),
                                                           n4);
    return cudaGetLastError();
}

cudaError_t launch_gate_backward(const float* g, const float* z, const float* alpha, float* dz, float* dalpha, int T,
                                 int H, int d, int per_head, cudaStream_t s) {
    const int D = H * d;
    const int tok = 2048;
    dim3 grid((D + 255) / 256, (T + tok - 1) / tok);
    LaunchScope scope("gate_backward", s);
    gate_bwd_kernel<<<grid, 256, 0, s>>>(g, z, alpha, dz, dalpha, T, H, d, per_head, tok);
    return cudaGetLastError();
}

cudaError_t launch_grad_gemm(float* C, long long ldc, long long cbs, const void* A, int a_bf16, long long a_rs,
                             long long a_cs, long long a_bs, const void* B, int b_bf16, long long b_rs, long long b_cs,
                             long long b_bs, int batch, int M, int N, long long K, int accumulate, cudaStream_t s) {
    // split K when the output has few tiles (the weight gradients: K = tokens)
    const long long tiles = (long long)((N + GN - 1) / GN) * ((M + GM - 1) / GM) * batch;
    int ksplit = 1;
    while (tiles * ksplit < 1184 && K / (ksplit * 2) >= 512 && ksplit < 1024) ksplit *= 2;
    if (ksplit > 1 && !accumulate) {
        const cudaError_t e = cudaMemsetAsync(C, 0, sizeof(float) * (size_t)batch * cbs, s);
        if (e != cudaSuccess) return e;
    }
    dim3 grid((N + GN - 1) / GN, (M + GM - 1) / GM, batch * ksplit);
    if (grid.y > 65535 || grid.z > 65535) return cudaErrorInvalidValue;
    LaunchScope scope("grad_gemm", s);
    gemm_kernel<<<grid, GT, 0, s>>>(C, ldc, cbs, GemmOp{A, a_bf16, a_rs, a_cs, a_bs}, GemmOp{B, b_bf16, b_rs, b_cs, b_bs},
                                    M, N, K, ksplit, accumulate);
    return cudaGetLastError();
}

}  // namespace ttt
