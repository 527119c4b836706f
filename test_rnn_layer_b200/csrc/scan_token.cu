// Per-token (b = 1) TTT-MLP scan with the hidden state resident in registers.
//
// One CTA per head, m = 4 d threads.  Thread i owns row i of W1 (d values)
// and column i of W2 (d values) for the whole sequence, so W1 u, W2^T e and
// both rank-1 updates are thread-local; only y = W2 g and z = W2 g_q are sums
// over the hidden units, done as a warp-shuffle reduce-scatter followed by a
// cross-warp sum in shared memory.
//
// Per token (paper notes page, "关键设计 / TTT-MLP 层"):
//   a = W1 k, g = GELU(a), e = W2 g - v,
//   W2 <- W2 - eta 2 e g^T,  W1 <- W1 - eta ((W2_old^T 2e) * GELU'(a)) k^T,
//   z = W2 GELU(W1 q)  with the updated state;  out = x + tanh(alpha) z.
#include "common.cuh"
#include "internal.h"

namespace ttt {
namespace {

constexpr int kTokBlock = 32;   // tokens staged in shared memory at a time

// Sum over the 32 lanes of the d values p_j = w2[j] * g.  Afterwards the lane
// holds kOut = max(D / 32, 1) sums for j = base + k and writes them to row[].
template <int D>
__device__ __forceinline__ void reduce_scatter_store(const float (&w2)[D], float g, float* row, int lane) {
    constexpr int H0 = D / 2;
    float v[H0];
    const bool up = lane & 16;
#pragma unroll
    for (int k = 0; k < H0; ++k) {
        const float lo = w2[k] * g, hi = w2[k + H0] * g;
        const float send = up ? lo : hi;
        const float keep = up ? hi : lo;
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    int base = up ? H0 : 0;
    int live = H0;   // values still held per lane
#pragma unroll
    for (int s = 8; s >= 1; s >>= 1) {
        if (live >= 2) {
            const int half = live / 2;
            const bool u = lane & s;
#pragma unroll
            for (int k = 0; k < H0 / 2; ++k) {
                if (k < half) {
                    const float send = u ? v[k] : v[k + half];
                    const float keep = u ? v[k + half] : v[k];
                    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, s);
                }
            }
            if (u) base += half;
            live = half;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], s);
        }
    }
    // D >= 32: live values per lane, distinct j.  D < 32: lanes sharing j hold
    // the same sum; the one with the low (32/D - 1) bits clear writes it.
    if (D >= 32) {
#pragma unroll
        for (int k = 0; k < (D >= 32 ? D / 32 : 1); ++k) row[base + k] = v[k];
    } else {
        if ((lane & (32 / D - 1)) == 0) row[base] = v[0];
    }
}

template <int D>
__global__ void __launch_bounds__(4 * D) scan_token_kernel(ScanArgs a) {
    constexpr int M = 4 * D;
    constexpr int NW = M / 32;
    __shared__ float sK[kTokBlock][D], sQ[kTokBlock][D], sV[kTokBlock][D];
    __shared__ float sRedY[NW][D], sRedZ[NW][D];
    __shared__ float sE[D];

    const int h = blockIdx.x;
    const int i = threadIdx.x;
    const int lane = i & 31, w = i >> 5;
    const int T = a.T;

    float w1[D], w2[D];
    {
        const float* W1 = a.W1_0 + (long long)h * M * D + (long long)i * D;
        const float* W2 = a.W2_0 + (long long)h * D * M + i;
#pragma unroll
        for (int j = 0; j < D; ++j) { w1[j] = W1[j]; w2[j] = W2[(long long)j * M]; }
    }
    const float eta = a.eta;
    float tanh_alpha = 0.f;
    if (i < D) tanh_alpha = tanhf(a.alpha[h * D + i]);
    int nonfinite = 0;

    for (int n0 = 0; n0 < T; n0 += kTokBlock) {
        const int nb = min(kTokBlock, T - n0);
        __syncthreads();
        for (int idx = i; idx < nb * D; idx += M) {
            const int r = idx / D, j = idx % D;
            const int t = a.reverse ? (T - 1 - (n0 + r)) : (n0 + r);
            const long long off = (long long)h * a.qkv_hs + (long long)t * a.qkv_ts + j;
            sK[r][j] = a.K[off];
            sQ[r][j] = a.Q[off];
            sV[r][j] = a.V[off];
        }
        __syncthreads();
        for (int r = 0; r < nb; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < D; ++j) acc = fmaf(w1[j], sK[r][j], acc);
            float g, gp;
            gelu_and_prime(acc, g, gp);
            reduce_scatter_store<D>(w2, g, sRedY[w], lane);
            __syncthreads();
            if (i < D) {
                float y = 0.f;
#pragma unroll
                for (int q = 0; q < NW; ++q) y += sRedY[q][i];
                sE[i] = -2.0f * eta * (y - sV[r][i]);   // -eta * dl/dy
            }
            __syncthreads();
            float back = 0.f;
#pragma unroll
            for (int j = 0; j < D; ++j) back = fmaf(w2[j], sE[j], back);
            const float dl = back * gp;                  // -eta * delta_i
#pragma unroll
            for (int j = 0; j < D; ++j) {
                w1[j] = fmaf(dl, sK[r][j], w1[j]);
                w2[j] = fmaf(sE[j], g, w2[j]);
            }
            float aq = 0.f;
#pragma unroll
            for (int j = 0; j < D; ++j) aq = fmaf(w1[j], sQ[r][j], aq);
            const float gq = gelu(aq);
            reduce_scatter_store<D>(w2, gq, sRedZ[w], lane);
            __syncthreads();
            if (i < D) {
                float z = 0.f;
#pragma unroll
                for (int q = 0; q < NW; ++q) z += sRedZ[q][i];
                const int t = a.reverse ? (T - 1 - (n0 + r)) : (n0 + r);
                const long long xo = (long long)h * a.x_hs + (long long)t * a.x_ts + i;
                const float x = load_elem(a.Xin, xo, a.xin_bf16);
                const float dz = tanh_alpha * z;
                store_elem(a.Out, xo, a.out_bf16, x + dz);
                if (a.Delta) a.Delta[xo] = __float2bfloat16_rn(dz);
                if (a.Zdbg) a.Zdbg[xo] = z;
                nonfinite |= !isfinite(z);
            }
        }
    }
    if (a.W1_T) {
        float* W1 = a.W1_T + (long long)h * M * D + (long long)i * D;
#pragma unroll
        for (int j = 0; j < D; ++j) W1[j] = w1[j];
    }
    if (a.W2_T) {
        float* W2 = a.W2_T + (long long)h * D * M + i;
#pragma unroll
        for (int j = 0; j < D; ++j) W2[(long long)j * M] = w2[j];
    }
    if (nonfinite) atomicOr(a.status, kStatusNonFinite);
}

}  // namespace

cudaError_t launch_scan_token(const ScanArgs& a, cudaStream_t s) {
    LaunchScope scope("scan_token", s);
    switch (a.d) {
        case 16: scan_token_kernel<16><<<a.H, 64, 0, s>>>(a); break;
        case 32: scan_token_kernel<32><<<a.H, 128, 0, s>>>(a); break;
        case 64: scan_token_kernel<64><<<a.H, 256, 0, s>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace ttt
