// Internal launcher interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tttmlp.h"

namespace ttt {

// Status bits a kernel may set in the workspace status word.
enum : int { kStatusNonFinite = 1, kStatusTimeout = 2 };

// Token-stream and gate arguments of one direction's scan.  Element (h, t, j)
// of a [H, T, d]-style stream lives at base + h * hs + t * ts + j; the same
// (hs, ts) pair describes both the per-head layout [H, T, d] (hs = T d,
// ts = d) and the concatenated-heads layout [T, H d] (hs = d, ts = H d).
struct ScanArgs {
    const float* Q;
    const float* K;
    const float* V;
    long long qkv_hs, qkv_ts;
    const void* Xin;        // gate residual input
    int xin_bf16;
    long long x_hs, x_ts;   // layout of Xin, Out, Delta and Zdbg
    const float* alpha;     // [H d], channel (h, j) = alpha[h d + j]
    void* Out;              // gate output: x + tanh(alpha) z
    int out_bf16;
    __nv_bfloat16* Delta;   // optional: bf16(tanh(alpha) z), same layout
    float* Zdbg;            // optional: pre-gate z (fp32)
    const float* W1_0;      // [H, m, d]
    const float* W2_0;      // [H, d, m]
    float* W1_T;            // optional [H, m, d]
    float* W2_T;            // optional [H, d, m]
    int T, H, d, m, b, reverse;
    float eta;
    int* status;            // OR-ed status bits
    float* scratch;         // per-head scratch (chunk SIMT kernel)
    int inject_timeout;     // tests: make the first bounded wait expire (cluster scan)
    float* Zscan;           // cluster scan: where it stores z (the gate runs as its own kernel)
    int c_begin, c_end;     // cluster scan: chunks [c_begin, c_end) of the walk (c_end 0: to the end);
                            // state from W1_0/W2_0, final state to W1_T/W2_T
    long long scratch_per_head;  // floats
    int fuse_gate;          // split-group cluster scan: apply the gate itself (Out, Delta, Zdbg; no Zscan)
};

// Scan kernels.  Each returns a cudaError_t from the launch.
cudaError_t launch_scan_token(const ScanArgs& a, cudaStream_t s);        // b == 1, one CTA per head
// b == 1, d = 64: a head's state sharded over a cluster of four CTAs
bool scan_token_cluster_supported(int d);
cudaError_t launch_scan_token_cluster(const ScanArgs& a, cudaStream_t s);
cudaError_t launch_scan_chunk_simt(const ScanArgs& a, cudaStream_t s);   // any b
long long scan_chunk_simt_scratch_floats(int d, int m, int b);
// tcgen05 chunk scan: d = 64, 2 <= b <= 64, tf32 contractions with fp32 accumulation.
bool scan_chunk_tc_supported(int d, int b);
cudaError_t launch_scan_chunk_tc(const ScanArgs& a, cudaStream_t s);    // one CTA per head
cudaError_t launch_scan_chunk_tc2(const ScanArgs& a, cudaStream_t s);   // a cluster of two CTAs per head
// A cluster of two CTAs per head, each split into a state warp group and an
// output warp group that run one chunk apart (fp16 operands for the products
// of thread-produced values, tf32 for those that read the fp32 state).
cudaError_t launch_scan_chunk_tc3(const ScanArgs& a, cudaStream_t s);

// TTT-Linear scan (f(u; W) = W u, W [d x d] per head): z of one direction into Z
// (X's layout); state from W_0 [H, d, d], final state to W_T (optional).
struct LinearScanArgs {
    const float* Q;
    const float* K;
    const float* V;
    long long qkv_hs, qkv_ts;
    float* Z;
    long long x_hs, x_ts;
    const float* W_0;
    float* W_T;
    int T, H, d, b, reverse;
    float eta;
    int* status;
    int c_begin, c_end;   // tensor-core kernel: chunks [c_begin, c_end) of the walk (c_end 0: to the end)
};
bool scan_linear_supported(int d);
cudaError_t launch_scan_linear(const LinearScanArgs& a, cudaStream_t s);   // fp32 SIMT, any b
// tcgen05 chunk form (tf32 contractions, fp32 state): d = 64, 2 <= b <= 64.
bool scan_linear_tc_supported(int d, int b);
cudaError_t launch_scan_linear_tc(const LinearScanArgs& a, cudaStream_t s);

// Per-head projections: U[which][h, t, e] = sum_j theta_which[h][e][j] x[h, t, j].
cudaError_t launch_proj_per_head(const void* X, int x_bf16, const void* const theta[3], int th_bf16,
                                 float* const out[3], int T, int H, int d, int* status, cudaStream_t s);

// Full-mode projections: C_which[t, n] (+)= sum_c A[t, c] Theta_which[n, c],
// A [T, Dm] row-major, Theta [N, Dm] row-major, C [T, N] fp32.
cudaError_t launch_proj_full_simt(const void* A, int a_bf16, const void* const theta[3], int th_bf16,
                                  float* const out[3], int T, int N, int Dm, int accumulate, int* status,
                                  cudaStream_t s);

// tcgen05 projections (bf16 A and Theta, N % 256 == 0, K % 64 == 0), same contract.
bool proj_full_tc_supported(int N, int K);
cudaError_t launch_proj_full_tc(const void* A, const void* const theta[3], float* const out[3], int T, int N, int K,
                                int accumulate, int* status, int max_ctas, cudaStream_t s);

// The same tcgen05 kernel as a general bf16 GEMM: up to 3 outputs
//   C_w[M x N] (+)= sum_{s < nseg} A_{w,s} B_{w,s}^T   (fp32 accumulate, fp32 C, row stride ldc)
// with every operand bf16 and row-major in memory: K-major (a_mn / b_mn = 0) means A is [M x K] and B is
// [N x K]; MN-major (= 1) means A is [K x M] and B is [K x N], K the row index.  N must be a multiple
// of 64; operand rows or columns past M, N or K read as zero.  ld: the operand's row stride (elements,
// a multiple of 8).
struct GemmTcOperand {
    const void* ptr;
    long long ld;
};
struct GemmTc {
    int nw, nseg, a_mn, b_mn;
    int M, N, K;   // K: the reduction length of every segment
    GemmTcOperand A[3][4], B[3][4];
    float* C[3];
    long long ldc;
    int accumulate;
    int* status;
    int max_ctas;      // 0: one CTA per SM
    const char* name;  // for the launch timing ("gemm_tc" if null)
};
cudaError_t launch_gemm_tc(const GemmTc& g, cudaStream_t s);
// hi = bf16(x), lo = bf16(x - hi): x = hi + lo to about 2^-16 relative (n elements, 16-byte aligned).
cudaError_t launch_split_bf16(const float* x, __nv_bfloat16* hi, __nv_bfloat16* lo, long long n, cudaStream_t s);

// Segment-local attention (d = 64, bf16) with a residual add, tcgen05:
// rows [row0, row1) of Out = Xres + softmax(Q K^T / 8) V inside segments of L
// tokens.  Q, K, V share the row stride ld_qkv; Xres (optional) and Out share
// ld_out / ld_res.  max_ctas > 0 caps the persistent grid.
bool attn_seg_supported(int d);
long long attn_seg_items(int T, int H, int L, int row0, int row1);
cudaError_t launch_attn_seg(const void* Q, const void* K, const void* V, long long ld_qkv, const void* Xres,
                            long long ld_res, void* Out, long long ld_out, int T, int H, int L, int row0, int row1,
                            int* status, int max_ctas, cudaStream_t s);

// out = x + tanh(alpha) z (+ bf16 increment, + non-finite check) over one direction.
cudaError_t launch_gate(const void* X, int x_bf16, const float* Z, const float* alpha, void* Out, int out_bf16,
                        __nv_bfloat16* Delta, int* status, int T, int H, int d, int per_head, int max_blocks,
                        cudaStream_t s);

// ttt_mlp_forward with every kernel on `stream` itself: the same kernels and
// arithmetic, but never the chunk-segment schedule on the library's own
// streams, so that the call creates no streams or events.
ttt_status forward_single_stream(const ttt_mlp_desc* desc, const void* X, const void* theta_q, const void* theta_k,
                                 const void* theta_v, const float* W1_0, const float* W2_0, float eta, int b,
                                 ttt_direction dir, const float* alpha_f, const float* alpha_r, void* Y, float* Z_out,
                                 float* W1_T, float* W2_T, void* workspace, size_t workspace_bytes,
                                 ttt_stream_t stream);

// Backward pass of one direction of the scan (fp32 state, b <= 64, d = 16/32/64):
// dQ, dK, dV (qkv layout) from dZ (X layout); dW1, dW2 [H, m, d] / [H, d, m]
// accumulated; scratch of H * scan_backward_scratch_floats(d, b, T) floats.
// split_tf32: products on tf32 tensor cores in the split form (fp32-accurate);
// 0: single tf32 products (the precision of the bf16 layer's forward products).
long long scan_backward_scratch_floats(int d, int b, int T);
cudaError_t launch_scan_backward(const float* Q, const float* K, const float* V, long long qkv_hs, long long qkv_ts,
                                 const float* dZ, long long x_hs, long long x_ts, const float* W1_0,
                                 const float* W2_0, float* dQ, float* dK, float* dV, float* dW1, float* dW2,
                                 float* scratch, int T, int H, int d, int b, int reverse, float eta, int split_tf32,
                                 cudaStream_t s);
// CTAs per head of launch_scan_backward (process-wide): 0 automatic, 1 or 2.
void set_scan_backward_ctas(int ctas);
// Gate backward: dz = tanh(alpha) g, dalpha += (1 - tanh^2 alpha) sum_t g z (per channel).
cudaError_t launch_gate_backward(const float* g, const float* z, const float* alpha, float* dz, float* dalpha, int T,
                                 int H, int d, int per_head, cudaStream_t s);
// Batched GEMM C[b] (+)= A[b] [M x K] B[b] [K x N] (fp32 C row-major; A, B bf16 or fp32 via strides).
cudaError_t launch_grad_gemm(float* C, long long ldc, long long cbs, const void* A, int a_bf16, long long a_rs,
                             long long a_cs, long long a_bs, const void* B, int b_bf16, long long b_rs, long long b_cs,
                             long long b_bs, int batch, int M, int N, long long K, int accumulate, cudaStream_t s);

// Records a message for ttt_last_error() on this thread and returns `code`.
ttt_status set_error(ttt_status code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));

// Counts a kernel launch and, while kernel timing is on, brackets it with
// CUDA events recorded on its stream.  Construct right before the launch.
class LaunchScope {
  public:
    LaunchScope(const char* name, cudaStream_t s);
    ~LaunchScope();
    LaunchScope(const LaunchScope&) = delete;
    LaunchScope& operator=(const LaunchScope&) = delete;

  private:
    const char* name_;
    cudaStream_t s_;
    cudaEvent_t start_ = nullptr;
};

}  // namespace ttt
