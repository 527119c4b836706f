// The gate out = x + tanh(alpha) * z over a whole direction's outputs
// (paper notes page, "关键设计 / 门控 + 双向机制"), with the optional bf16
// increment tanh(alpha) * z that the full layer's reverse projection uses, and
// the non-finite check of x and z.  Bandwidth-bound: four elements per thread,
// two grid-stride steps per iteration with all their loads issued before any
// store (bytes in flight are what limit a launch capped to a few SMs), over the
// flat arrays (all in X's layout).
#include "common.cuh"
#include "internal.h"

namespace ttt {
namespace {

struct GateArgs {
    const void* X;
    int x_bf16;
    const float* Z;
    const float* alpha;     // [H d]
    void* Out;
    int out_bf16;
    __nv_bfloat16* Delta;   // optional
    int* status;
    long long n;            // elements (a multiple of 4)
    int per_head;           // 1: [H, T, d] layout; 0: [T, D]
    long long Td;           // T * d (per-head layout)
    int d, D;
};

__device__ __forceinline__ float4 load4(const void* p, long long i, int bf16) {
    if (bf16) {
        const uint2 raw = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(p) + i);
        const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
        const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
        const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
        return make_float4(a.x, a.y, b.x, b.y);
    }
    return *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i);
}

__device__ __forceinline__ void store4(void* p, long long i, int bf16, float4 v) {
    if (bf16) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
        uint2 raw;
        raw.x = *reinterpret_cast<uint32_t*>(&lo);
        raw.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p) + i) = raw;
    } else {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(p) + i) = v;
    }
}

__global__ void __launch_bounds__(256) gate_kernel(GateArgs g) {
    constexpr int U = 2;
    int nonfinite = 0;
    const long long stride = (long long)gridDim.x * blockDim.x * 4;
    for (long long i0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4; i0 < g.n; i0 += U * stride) {
        float4 x[U], z[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long i = i0 + u * stride;
            if (i < g.n) {
                x[u] = load4(g.X, i, g.x_bf16);
                z[u] = *reinterpret_cast<const float4*>(g.Z + i);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long i = i0 + u * stride;
            if (i >= g.n) break;
            // channel of element i (4 consecutive elements share the row; d is a multiple of 4)
            const long long ch = g.per_head ? (i / g.Td) * g.d + (i % g.d) : (i % g.D);
            const float4 al = *reinterpret_cast<const float4*>(g.alpha + ch);
            const float4 zz = z[u], xx = x[u];
            const float4 dz =
                make_float4(tanhf(al.x) * zz.x, tanhf(al.y) * zz.y, tanhf(al.z) * zz.z, tanhf(al.w) * zz.w);
            store4(g.Out, i, g.out_bf16, make_float4(xx.x + dz.x, xx.y + dz.y, xx.z + dz.z, xx.w + dz.w));
            if (g.Delta) store4(g.Delta, i, 1, dz);
            nonfinite |= !(isfinite(zz.x) && isfinite(zz.y) && isfinite(zz.z) && isfinite(zz.w) && isfinite(xx.x) &&
                           isfinite(xx.y) && isfinite(xx.z) && isfinite(xx.w));
        }
    }
    if (__syncthreads_or(nonfinite) && threadIdx.x == 0) atomicOr(g.status, kStatusNonFinite);
}

}  // namespace

cudaError_t launch_gate(const void* X, int x_bf16, const float* Z, const float* alpha, void* Out, int out_bf16,
                        __nv_bfloat16* Delta, int* status, int T, int H, int d, int per_head, int max_blocks,
                        cudaStream_t s) {
    GateArgs g{};
    g.X = X; g.x_bf16 = x_bf16; g.Z = Z; g.alpha = alpha; g.Out = Out; g.out_bf16 = out_bf16;
    g.Delta = Delta; g.status = status;
    g.n = (long long)T * H * d;
    g.per_head = per_head; g.Td = (long long)T * d; g.d = d; g.D = H * d;
    if (g.n % 4 != 0 || d % 4 != 0) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    long long blocks = (g.n / 4 + 255) / 256;
    if (blocks > (long long)sms * 6) blocks = (long long)sms * 6;
    if (max_blocks > 0 && blocks > max_blocks) blocks = max_blocks;
    LaunchScope scope("gate", s);
    gate_kernel<<<(unsigned)blocks, 256, 0, s>>>(g);
    return cudaGetLastError();
}

}  // namespace ttt
