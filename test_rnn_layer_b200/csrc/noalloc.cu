// ttt_mlp_forward_noalloc: the layer for callers that cannot allocate device
// memory themselves.
//
// Some callers have no way to obtain a device workspace: code running inside a
// host framework whose allocator it does not own, plug-ins that may not call
// cudaMalloc, or environments that forbid allocation after start-up.  This
// entry point runs the same kernels as ttt_mlp_forward, but its scratch (the
// Q/K/V streams, X', the chunk intermediates and the status word) lives in one
// fixed-size array in the library's own device memory instead of a
// caller-provided workspace.  Every GPU that loads the library holds that
// array (kNoAllocBytes) until the process exits.  Every kernel runs on the
// caller's stream (never the chunk-segment schedule on the library's own
// streams), so a call creates no streams or events either.
#include <mutex>

#include "../../include/tttmlp.h"
#include "internal.h"

namespace {

constexpr size_t kNoAllocBytes = size_t(32) << 20;   // 32 MiB
constexpr int kMaxDevices = 64;

// The shared scratch.  In host code this name is only a stand-in for the
// device symbol, not a device address: its address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

std::mutex g_mu;
void* g_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and kept for the life of the process.
ttt_status scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return ttt::set_error(TTT_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return ttt::set_error(TTT_ERR_UNSUPPORTED, "device index %d too large", dev);
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return ttt::set_error(TTT_ERR_CUDA, "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
        g_ptr[dev] = p;
    }
    *out = g_ptr[dev];
    return TTT_OK;
}

}  // namespace

extern "C" TTT_API ttt_status ttt_mlp_forward_noalloc(const ttt_mlp_desc* desc, const void* X, const void* theta_q,
                                                      const void* theta_k, const void* theta_v, const float* W1_0,
                                                      const float* W2_0, float eta, int b, ttt_direction dir,
                                                      const float* alpha_f, const float* alpha_r, void* Y,
                                                      float* Z_out, float* W1_T, float* W2_T, ttt_stream_t stream) {
    const size_t need = ttt_mlp_workspace_size(desc, b, dir);
    if (need == 0) return TTT_ERR_INVALID_ARG;   // ttt_last_error() already says why
    if (need > kNoAllocBytes) {
        return ttt::set_error(TTT_ERR_UNSUPPORTED,
                              "ttt_mlp_forward_noalloc: this shape needs %zu bytes of scratch, more than the "
                              "library's fixed %zu bytes; use ttt_mlp_forward with a caller workspace",
                              need, kNoAllocBytes);
    }
    void* ws = nullptr;
    const ttt_status st = scratch_address(&ws);
    if (st != TTT_OK) return st;
    return ttt::forward_single_stream(desc, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, dir, alpha_f, alpha_r,
                                      Y, Z_out, W1_T, W2_T, ws, kNoAllocBytes, stream);
}

extern "C" TTT_API ttt_status ttt_mlp_noalloc_status(ttt_stream_t stream) {
    void* ws = nullptr;
    const ttt_status st = scratch_address(&ws);
    if (st != TTT_OK) return st;
    return ttt_mlp_status(ws, stream);
}
