// C ABI of the TTT-MLP layer: argument checks, workspace carving and the
// direction driver.  Every step of the computation runs in this library's
// kernels; this file only sequences them on the caller's stream.
//
// Bidirectional composition (paper notes page, "关键设计 / 门控 + 双向机制"):
// the forward scan runs on X and its gate writes X' = X + tanh(alpha_f) z_f;
// the reverse scan runs on X' (same theta, same W_0) and its gate writes
// Y = X' + tanh(alpha_r) z_r.
#include <algorithm>
#include <atomic>
#include <functional>
#include <map>
#include <memory>
#include <cstdarg>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/tttmlp.h"
#include "internal.h"

namespace ttt {

static std::atomic<uint64_t> g_launches{0};

// Per-kernel timing: while on, each launch is bracketed by two CUDA events on
// its own stream; ttt_kernel_times sums the elapsed times per kernel name.
struct TimedLaunch {
    const char* name;
    cudaEvent_t start, stop;
};
static std::mutex g_timing_mu;
static std::atomic<bool> g_timing_on{false};
static std::vector<TimedLaunch> g_timed;

LaunchScope::LaunchScope(const char* name, cudaStream_t s) : name_(name), s_(s) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (g_timing_on.load(std::memory_order_relaxed)) {
        if (cudaEventCreate(&start_) == cudaSuccess) cudaEventRecord(start_, s_);
        else start_ = nullptr;
    }
}

LaunchScope::~LaunchScope() {
    if (!start_) return;
    cudaEvent_t stop = nullptr;
    if (cudaEventCreate(&stop) != cudaSuccess) { cudaEventDestroy(start_); return; }
    cudaEventRecord(stop, s_);
    std::lock_guard<std::mutex> lk(g_timing_mu);
    g_timed.push_back({name_, start_, stop});
}

static std::atomic<int> g_scan_impl{0}, g_proj_impl{0};

// The split-group cluster scan applies the gate in its output group (1) or
// leaves it to the separate gate kernel (0).
#ifndef TTT_SPLIT_SCAN_GATES
#define TTT_SPLIT_SCAN_GATES 1
#endif
constexpr bool kSplitScanGates = TTT_SPLIT_SCAN_GATES != 0;
static std::atomic<int> g_inject_timeout{0};
// The block's schedule: -1 = the whole attention first; p >= 0 = each segment's attention just before its
// projection, with the first p% of the first direction's chunks on the whole GPU before its scan starts.
static std::atomic<int> g_block_front{-1};

}  // namespace ttt

using namespace ttt;

namespace {

thread_local std::string t_err;

ttt_status fail(ttt_status code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
ttt_status fail(ttt_status code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_err = buf;
    return code;
}

}  // namespace

ttt_status ttt::set_error(ttt_status code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_err = buf;
    return code;
}

namespace {

#define CUDA_TRY(expr)                                                                           \
    do {                                                                                         \
        cudaError_t e_ = (expr);                                                                 \
        if (e_ != cudaSuccess) return fail(TTT_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_)); \
    } while (0)

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_size(ttt_dtype t) { return t == TTT_BF16 ? 2 : 4; }

ttt_status check_desc(const ttt_mlp_desc* desc, int b, ttt_direction dir) {
    if (!desc) return fail(TTT_ERR_INVALID_ARG, "desc is NULL");
    const ttt_mlp_desc& q = *desc;
    if (q.T < 1 || q.H < 1) return fail(TTT_ERR_INVALID_ARG, "T=%d and H=%d must be >= 1", q.T, q.H);
    if (q.d < 1 || q.m != 4 * q.d)
        return fail(TTT_ERR_INVALID_ARG, "m=%d must be 4*d (d=%d)", q.m, q.d);
    if ((long long)q.D != (long long)q.H * q.d)
        return fail(TTT_ERR_INVALID_ARG, "D=%d must equal H*d=%lld", q.D, (long long)q.H * q.d);
    if (q.per_head_input != 0 && q.per_head_input != 1)
        return fail(TTT_ERR_INVALID_ARG, "per_head_input must be 0 or 1");
    if (q.x_dtype != TTT_F32 && q.x_dtype != TTT_BF16) return fail(TTT_ERR_INVALID_ARG, "bad x_dtype");
    if (dir != TTT_FWD && dir != TTT_REV && dir != TTT_BIDIR) return fail(TTT_ERR_INVALID_ARG, "bad direction");
    if (b < 1 || b > 256) return fail(TTT_ERR_INVALID_ARG, "b=%d outside [1, 256]", b);
    if (q.d != 16 && q.d != 32 && q.d != 64)
        return fail(TTT_ERR_UNSUPPORTED, "head dim d=%d not supported (16, 32, 64)", q.d);
    if ((long long)q.T * q.D > (1LL << 40)) return fail(TTT_ERR_INVALID_ARG, "T*D too large");
    return TTT_OK;
}

struct Layout {
    size_t status, qkv[3], xp, delta, scratch, zbuf, state, total;
    long long scratch_per_head;
    bool split_reverse;   // reverse projection as theta X + theta bf16(X' - X)
};

Layout plan(const ttt_mlp_desc& q, int b, ttt_direction dir) {
    Layout L{};
    const size_t n = (size_t)q.T * q.D;
    size_t off = 0;
    L.status = off; off += kAlign;
    for (int w = 0; w < 3; ++w) { L.qkv[w] = off; off = align_up(off + n * sizeof(float)); }
    L.split_reverse = (dir == TTT_BIDIR) && !q.per_head_input && q.x_dtype == TTT_BF16;
    L.xp = off;
    if (dir == TTT_BIDIR) off = align_up(off + n * sizeof(float));
    L.delta = off;
    if (L.split_reverse) off = align_up(off + n * 2);
    L.scratch = off;
    // the SIMT chunk kernel may run for any b (it is selectable for b = 1 too)
    L.scratch_per_head = scan_chunk_simt_scratch_floats(q.d, q.m, b);
    off = align_up(off + (size_t)q.H * L.scratch_per_head * sizeof(float));
    // z of one direction for the cluster tensor-core scan, whose gate runs separately
    L.zbuf = off;
    if (scan_chunk_tc_supported(q.d, b)) off = align_up(off + n * sizeof(float));
    // W1 and W2 of every head between two segments of a pipelined direction
    L.state = off;
    if (scan_chunk_tc_supported(q.d, b)) off = align_up(off + 2 * (size_t)q.H * q.m * q.d * sizeof(float));
    L.total = off;
    return L;
}

struct Dir {
    int reverse;
    const void* xin;
    int xin_bf16;
    const float* alpha;
    void* out;
    int out_bf16;
    __nv_bfloat16* delta;
    float* zdbg;
    float* w1t;
    float* w2t;
};

ttt_status project(const ttt_mlp_desc& q, const void* src, int src_bf16, const void* const th[3],
                   float* const out[3], int accumulate, int* status, cudaStream_t s) {
    const int th_bf16 = q.x_dtype == TTT_BF16;
    if (q.per_head_input) {
        if (accumulate) return fail(TTT_ERR_UNSUPPORTED, "internal: accumulate in per-head projection");
        CUDA_TRY(launch_proj_per_head(src, src_bf16, th, th_bf16, out, q.T, q.H, q.d, status, s));
        return TTT_OK;
    }
    const int impl = g_proj_impl.load();
    const bool tc_ok = src_bf16 && th_bf16 && proj_full_tc_supported(q.D, q.D);
    if (impl == 2 && !tc_ok)
        return fail(TTT_ERR_UNSUPPORTED, "tensor-core projection needs bf16 inputs, D %% 256 == 0");
    if (tc_ok && impl != 1) {
        CUDA_TRY(launch_proj_full_tc(src, th, out, q.T, q.D, q.D, accumulate, status, 0, s));
    } else {
        CUDA_TRY(launch_proj_full_simt(src, src_bf16, th, th_bf16, out, q.T, q.D, q.D, accumulate, status, s));
    }
    return TTT_OK;
}

ScanArgs scan_args(const ttt_mlp_desc& q, const Layout& L, char* ws, const float* W1_0, const float* W2_0,
                   float eta, int b, const Dir& dd) {
    ScanArgs a{};
    a.Q = reinterpret_cast<const float*>(ws + L.qkv[0]);
    a.K = reinterpret_cast<const float*>(ws + L.qkv[1]);
    a.V = reinterpret_cast<const float*>(ws + L.qkv[2]);
    if (q.per_head_input) { a.qkv_hs = (long long)q.T * q.d; a.qkv_ts = q.d; }
    else { a.qkv_hs = q.d; a.qkv_ts = q.D; }
    a.x_hs = a.qkv_hs; a.x_ts = a.qkv_ts;
    a.Xin = dd.xin; a.xin_bf16 = dd.xin_bf16;
    a.alpha = dd.alpha;
    a.Out = dd.out; a.out_bf16 = dd.out_bf16;
    a.Delta = dd.delta; a.Zdbg = dd.zdbg;
    a.W1_0 = W1_0; a.W2_0 = W2_0; a.W1_T = dd.w1t; a.W2_T = dd.w2t;
    a.T = q.T; a.H = q.H; a.d = q.d; a.m = q.m; a.b = b; a.reverse = dd.reverse;
    a.eta = eta;
    a.status = reinterpret_cast<int*>(ws + L.status);
    a.scratch = reinterpret_cast<float*>(ws + L.scratch);
    a.scratch_per_head = L.scratch_per_head;
    a.inject_timeout = g_inject_timeout.load();
    return a;
}

ttt_status scan(const ttt_mlp_desc& q, const Layout& L, char* ws, const float* W1_0, const float* W2_0,
                float eta, int b, const Dir& dd, cudaStream_t s) {
    ScanArgs a = scan_args(q, L, ws, W1_0, W2_0, eta, b, dd);
    // Kernel choice: the tensor-core scan (the split-group cluster kernel)
    // serves bf16-input layers (whose tolerance is 2e-2); fp32-input layers
    // keep the fp32 kernels unless a tensor-core kernel is requested explicitly.
    const int impl = g_scan_impl.load();
    const bool tc_ok = scan_chunk_tc_supported(q.d, b);
    if (impl == 2 && !tc_ok) return fail(TTT_ERR_UNSUPPORTED, "tensor-core scan needs d = 64 and 2 <= b <= 64");
    if (impl == 3) {   // one CTA per head
        if (b == 1) {
            CUDA_TRY(launch_scan_token(a, s));
            return TTT_OK;
        }
        if (!tc_ok) return fail(TTT_ERR_UNSUPPORTED, "tensor-core scan needs d = 64 and 2 <= b <= 64");
        CUDA_TRY(launch_scan_chunk_tc(a, s));
    } else if (impl == 2 || impl == 4 || (impl == 0 && tc_ok && q.x_dtype == TTT_BF16)) {
        if (impl == 4 && !tc_ok) return fail(TTT_ERR_UNSUPPORTED, "tensor-core scan needs d = 64 and 2 <= b <= 64");
        const bool split = impl != 2;   // automatic: the split-group cluster scan
        a.Zscan = dd.zdbg ? dd.zdbg : reinterpret_cast<float*>(ws + L.zbuf);
        if (split && kSplitScanGates) {   // the split-group scan applies the gate itself
            a.fuse_gate = 1;
            CUDA_TRY(launch_scan_chunk_tc3(a, s));
        } else {
            if (split) CUDA_TRY(launch_scan_chunk_tc3(a, s));
            else CUDA_TRY(launch_scan_chunk_tc2(a, s));
            CUDA_TRY(launch_gate(dd.xin, dd.xin_bf16, a.Zscan, dd.alpha, dd.out, dd.out_bf16, dd.delta, a.status,
                                 q.T, q.H, q.d, q.per_head_input, 0, s));
        }
    } else if (b == 1 && impl != 1) {   // per token: a head's state over a four-CTA cluster where it fits
        if (scan_token_cluster_supported(q.d)) CUDA_TRY(launch_scan_token_cluster(a, s));
        else CUDA_TRY(launch_scan_token(a, s));
    } else {
        CUDA_TRY(launch_scan_chunk_simt(a, s));
    }
    return TTT_OK;
}

// ---------------------------------------------------------------- pipelined full layer
// With the full-width projection on the tensor cores and the cluster scan, a
// direction runs as a sequence of chunk segments so that the projection and
// the gate use the SMs the scan leaves free (the scan holds two SMs per head):
//   side stream : proj(seg 0), proj(seg 1), ...  then, after scan(seg k), gate(seg k)
//   scan stream : after proj(seg k), scan(seg k) -- the state W1, W2 is carried
//                 from one segment to the next in the workspace
// Only stream order and events connect the two streams (no kernel waits on
// another).  Projection and gate launches next to a running scan are capped
// to the free SMs less a margin, so that every CTA pair of the next scan
// segment finds room; the scan stream has the higher priority.  Each (device,
// caller stream) pair has its own set of library streams and events, so calls
// on different caller streams neither wait on each other nor share events;
// calls on one caller stream take turns while they enqueue.
struct Pipe {
    cudaStream_t scan = nullptr, side = nullptr, copy = nullptr;
    std::vector<cudaEvent_t> ev;
    int sms = 0;
    std::mutex mu;
};
std::mutex g_pipe_mu;   // guards g_pipes (not the enqueue)
std::map<std::pair<int, cudaStream_t>, std::unique_ptr<Pipe>> g_pipes;

Pipe& pipe_for(int dev, cudaStream_t caller) {
    std::lock_guard<std::mutex> lk(g_pipe_mu);
    std::unique_ptr<Pipe>& p = g_pipes[{dev, caller}];
    if (!p) p.reset(new Pipe());
    return *p;
}

constexpr int kPipeMinSegChunks = 16;
#ifndef TTT_PIPE_SM_MARGIN
#define TTT_PIPE_SM_MARGIN 4
#endif
constexpr int kPipeSmMargin = TTT_PIPE_SM_MARGIN;
// When the scan applies the gate itself, the projections of the segments that
// cover the first kPipeFrontPercent of a direction's chunks run on the whole
// GPU before that direction's scan starts (a head start: the scan then walks
// faster than the projection can follow on the SMs the scan leaves free).
#ifndef TTT_PIPE_FRONT_PERCENT
#define TTT_PIPE_FRONT_PERCENT 15
#endif
constexpr int kPipeFrontPercent = TTT_PIPE_FRONT_PERCENT;

// Chunk ranges [begin, end) of a walk over `nchunks` chunks: segments grow
// by 3/2 from 16 chunks at both ends (short exposed head and tail: 16, 24,
// 36, ... and ..., 36, 24, 16), with equal pieces of at most
// max(16, ceil(nchunks / TTT_PIPE_SEG_DIV)) chunks in between.
#ifndef TTT_PIPE_SEG_DIV
#define TTT_PIPE_SEG_DIV 16
#endif
std::vector<std::pair<int, int>> pipe_segments(int nchunks) {
    const int cap = std::max(kPipeMinSegChunks, (nchunks + TTT_PIPE_SEG_DIV - 1) / TTT_PIPE_SEG_DIV);
    std::vector<int> front, back;
    int rem = nchunks;
    for (int sz = kPipeMinSegChunks; sz < cap && rem > 0; sz = sz * 3 / 2) {
        int t = std::min(sz, rem);
        front.push_back(t);
        rem -= t;
        if (rem <= 0) break;
        t = std::min(sz, rem);
        back.push_back(t);
        rem -= t;
    }
    if (rem > 0) {   // the middle in equal pieces (no short leftover segment)
        const int n = (rem + cap - 1) / cap;
        for (int k = 0; k < n; ++k) front.push_back(rem / n + (k < rem % n ? 1 : 0));
    }
    front.insert(front.end(), back.rbegin(), back.rend());
    std::vector<std::pair<int, int>> out;
    int c = 0;
    for (int sz : front) {
        out.emplace_back(c, c + sz);
        c += sz;
    }
    return out;
}

// SMs the projection and gate may use next to a running scan that holds
// `scan_sms_per_head` SMs per head (0: no pipelining).
int pipe_side_sms(const ttt_mlp_desc& q, int scan_sms_per_head) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    const int side = sms - scan_sms_per_head * q.H - kPipeSmMargin;
    return side >= 16 ? side : 0;
}

bool pipe_eligible(const ttt_mlp_desc& q, const Layout& L, int b, ttt_direction dir) {
    const int si = g_scan_impl.load(), pi = g_proj_impl.load();
    if (q.per_head_input || q.x_dtype != TTT_BF16) return false;
    if (!(si == 0 || si == 2 || si == 4) || !scan_chunk_tc_supported(q.d, b)) return false;
    if (pi == 1 || !proj_full_tc_supported(q.D, q.D)) return false;
    if (dir == TTT_BIDIR && !L.split_reverse) return false;
    return pipe_side_sms(q, 2) > 0;
}

// Workspace buffers the pipeline uses (layer-independent).
struct PipeBufs {
    int* status;
    float* xp;              // X' (fp32) between the directions
    __nv_bfloat16* delta;   // bf16 gate increment (reverse projection input)
    float* zbuf;            // z of one direction when the caller wants none
};
// Launches the scan over chunks [c_begin, c_end) of direction `di` (first/last:
// the segment starts from W_0 / leaves the final state for the caller).
using SegScan = std::function<cudaError_t(int di, const struct Dir& dd, int c_begin, int c_end, bool first,
                                          bool last, float* zscan, cudaStream_t s)>;
// Work that produces rows [r0, r1) of X, enqueued on the side stream just before the first direction's
// projection of those rows (max_ctas: the SM cap of that projection, 0 = whole GPU).
using RowsHook = std::function<cudaError_t(int r0, int r1, int max_ctas, cudaStream_t s)>;

ttt_status forward_pipelined(const ttt_mlp_desc& q, const PipeBufs& B, int scan_sms_per_head, const SegScan& seg_scan,
                             const void* X, const void* const th[3], float* const qkv[3], int b, ttt_direction dir,
                             const float* alpha_f, const float* alpha_r, void* Y, float* Z_out, cudaStream_t s,
                             const void* X_host, void* Y_host, bool scan_gates = false,
                             const RowsHook* pre_rows = nullptr, int first_front_percent = -1) {
    int dev = 0;
    CUDA_TRY(cudaGetDevice(&dev));
    Pipe& P = pipe_for(dev, s);
    std::lock_guard<std::mutex> lk(P.mu);
    if (!P.scan) {
        int lo = 0, hi = 0;
        CUDA_TRY(cudaDeviceGetStreamPriorityRange(&lo, &hi));
        CUDA_TRY(cudaStreamCreateWithPriority(&P.scan, cudaStreamNonBlocking, hi));
        CUDA_TRY(cudaStreamCreateWithPriority(&P.side, cudaStreamNonBlocking, lo));
        CUDA_TRY(cudaStreamCreateWithPriority(&P.copy, cudaStreamNonBlocking, lo));
    }
    const int side_sms = pipe_side_sms(q, scan_sms_per_head);
    const int nch = (q.T + b - 1) / b;
    const auto seg = pipe_segments(nch);
    const int ns = (int)seg.size();
    const int ndir = dir == TTT_BIDIR ? 2 : 1;
    const size_t need_ev = 4 + (size_t)ndir * 4 * ns;
    while (P.ev.size() < need_ev) {
        cudaEvent_t e;
        CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
        P.ev.push_back(e);
    }
    size_t next_ev = 0;
    auto new_ev = [&]() { return P.ev[next_ev++]; };

    cudaEvent_t fork = new_ev();
    CUDA_TRY(cudaEventRecord(fork, s));
    CUDA_TRY(cudaStreamWaitEvent(P.scan, fork, 0));
    CUDA_TRY(cudaStreamWaitEvent(P.side, fork, 0));
    CUDA_TRY(cudaStreamWaitEvent(P.copy, fork, 0));

    auto enqueue = [&]() -> ttt_status {
        const size_t n = (size_t)q.T * q.D;
        const int D = q.D;
        cudaEvent_t prev_dir_done = nullptr;   // the previous direction's last scan segment
        float* xp = B.xp;
        __nv_bfloat16* delta = B.delta;
        int* status = B.status;

        for (int di = 0; di < ndir; ++di) {
            Dir dd{};
            dd.reverse = (dir == TTT_REV || di == 1) ? 1 : 0;
            const bool second = di == 1;
            dd.xin = second ? static_cast<const void*>(xp) : X;
            dd.xin_bf16 = second ? 0 : 1;
            dd.alpha = dd.reverse ? alpha_r : alpha_f;
            if (dir == TTT_BIDIR && !second) { dd.out = xp; dd.out_bf16 = 0; dd.delta = delta; }
            else { dd.out = Y; dd.out_bf16 = 1; dd.delta = nullptr; }
            dd.zdbg = Z_out ? Z_out + di * n : nullptr;
            const void* psrc = second ? static_cast<const void*>(delta) : X;   // both bf16
            const int pacc = second ? 1 : 0;
            float* zscan = Z_out ? Z_out + di * n : B.zbuf;

            std::vector<cudaEvent_t> ev_proj(ns), ev_scan(ns), ev_h2d(ns), ev_gate(ns);
            for (int k = 0; k < ns; ++k) { ev_proj[k] = new_ev(); ev_scan[k] = new_ev(); ev_h2d[k] = new_ev(); ev_gate[k] = new_ev(); }
            const bool copy_in = X_host && di == 0;           // X arrives segment by segment
            const bool copy_out = Y_host && di == ndir - 1;   // Y leaves segment by segment
            auto rows = [&](int k, int& r0, int& r1) {
                const int lo = seg[k].first * b, hi = std::min(seg[k].second * b, q.T);
                if (dd.reverse) { r0 = q.T - hi; r1 = q.T - lo; }
                else { r0 = lo; r1 = hi; }
            };
            if (copy_in) {
                for (int k = 0; k < ns; ++k) {
                    int r0, r1;
                    rows(k, r0, r1);
                    const size_t o = (size_t)r0 * D * 2, nb = (size_t)(r1 - r0) * D * 2;
                    CUDA_TRY(cudaMemcpyAsync(const_cast<char*>(static_cast<const char*>(X)) + o,
                                             static_cast<const char*>(X_host) + o, nb, cudaMemcpyHostToDevice, P.copy));
                    CUDA_TRY(cudaEventRecord(ev_h2d[k], P.copy));
                }
            }
            // projections: the first runs alone on the whole GPU (with a gating scan, the segments of the
            // first kPipeFrontPercent of the chunks); the reverse ones after the forward scan wrote X'
            if (prev_dir_done) CUDA_TRY(cudaStreamWaitEvent(P.side, prev_dir_done, 0));
            const int front_pct = (di == 0 && first_front_percent >= 0) ? first_front_percent : kPipeFrontPercent;
            const int front_chunks = scan_gates ? (int)((long long)nch * front_pct / 100) : 0;
            int last_front = 0;   // the first scan segment waits for the projections of the head start
            for (int k = 0; k < ns; ++k)
                if (seg[k].second <= front_chunks) last_front = k;
            for (int k = 0; k < ns; ++k) {
                int r0, r1;
                rows(k, r0, r1);
                if (copy_in) CUDA_TRY(cudaStreamWaitEvent(P.side, ev_h2d[k], 0));
                const void* a = static_cast<const char*>(psrc) + (size_t)r0 * D * 2;
                float* out[3] = {qkv[0] + (size_t)r0 * D, qkv[1] + (size_t)r0 * D, qkv[2] + (size_t)r0 * D};
                const bool whole_gpu = k == 0 || seg[k].second <= front_chunks;
                if (pre_rows && di == 0) CUDA_TRY((*pre_rows)(r0, r1, whole_gpu ? 0 : side_sms, P.side));
                CUDA_TRY(launch_proj_full_tc(a, th, out, r1 - r0, D, D, pacc, status, whole_gpu ? 0 : side_sms, P.side));
                CUDA_TRY(cudaEventRecord(ev_proj[k], P.side));
            }
            // scan segments, the state carried by the launcher
            for (int k = 0; k < ns; ++k) {
                CUDA_TRY(cudaStreamWaitEvent(P.scan, ev_proj[k == 0 ? last_front : k], 0));
                CUDA_TRY(seg_scan(di, dd, seg[k].first, seg[k].second, k == 0, k == ns - 1, zscan, P.scan));
                CUDA_TRY(cudaEventRecord(ev_scan[k], P.scan));
            }
            prev_dir_done = ev_scan[ns - 1];
            // gates, each after its segment's scan (or in the scan itself)
            for (int k = 0; k < ns; ++k) {
                int r0, r1;
                rows(k, r0, r1);
                const size_t o = (size_t)r0 * D;
                if (scan_gates) {
                    if (copy_out) {
                        CUDA_TRY(cudaStreamWaitEvent(P.copy, ev_scan[k], 0));
                        CUDA_TRY(cudaMemcpyAsync(static_cast<char*>(Y_host) + o * 2,
                                                 static_cast<const char*>(Y) + o * 2, (size_t)(r1 - r0) * D * 2,
                                                 cudaMemcpyDeviceToHost, P.copy));
                    }
                    continue;
                }
                CUDA_TRY(cudaStreamWaitEvent(P.side, ev_scan[k], 0));
                const void* xin = static_cast<const char*>(dd.xin) + o * (dd.xin_bf16 ? 2 : 4);
                void* out = static_cast<char*>(dd.out) + o * (dd.out_bf16 ? 2 : 4);
                const bool last = k == ns - 1;
                CUDA_TRY(launch_gate(xin, dd.xin_bf16, zscan + o, dd.alpha, out, dd.out_bf16,
                                     dd.delta ? dd.delta + o : nullptr, status, r1 - r0, q.H, q.d, 0,
                                     last ? 0 : side_sms * 6, P.side));
                if (copy_out) {
                    CUDA_TRY(cudaEventRecord(ev_gate[k], P.side));
                    CUDA_TRY(cudaStreamWaitEvent(P.copy, ev_gate[k], 0));
                    CUDA_TRY(cudaMemcpyAsync(static_cast<char*>(Y_host) + o * 2, static_cast<const char*>(Y) + o * 2,
                                             (size_t)(r1 - r0) * D * 2, cudaMemcpyDeviceToHost, P.copy));
                }
            }
        }
        return TTT_OK;
    };
    const ttt_status st = enqueue();
    // Join the library's streams back into the caller's stream, after a failed
    // enqueue too: nothing launched on them may outlive the caller's view of the call.
    cudaEvent_t j1 = new_ev(), j2 = new_ev(), j3 = new_ev();
    const cudaError_t je[6] = {cudaEventRecord(j1, P.scan), cudaEventRecord(j2, P.side), cudaEventRecord(j3, P.copy),
                               cudaStreamWaitEvent(s, j1, 0), cudaStreamWaitEvent(s, j2, 0),
                               cudaStreamWaitEvent(s, j3, 0)};
    if (st != TTT_OK) return st;
    for (cudaError_t e : je)
        if (e != cudaSuccess) return fail(TTT_ERR_CUDA, "joining the library's streams: %s", cudaGetErrorString(e));
    return TTT_OK;
}

ttt_status check_ptrs(const ttt_mlp_desc& q, const void* X, const void* tq, const void* tk, const void* tv,
                      const float* W1_0, const float* W2_0, float eta, ttt_direction dir,
                      const float* alpha_f, const float* alpha_r) {
    if (!X || !tq || !tk || !tv || !W1_0 || !W2_0)
        return fail(TTT_ERR_INVALID_ARG, "X, theta_q/k/v, W1_0 and W2_0 must be non-NULL");
    if ((dir == TTT_FWD || dir == TTT_BIDIR) && !alpha_f)
        return fail(TTT_ERR_INVALID_ARG, "alpha_f is required for this direction");
    if ((dir == TTT_REV || dir == TTT_BIDIR) && !alpha_r)
        return fail(TTT_ERR_INVALID_ARG, "alpha_r is required for this direction");
    if (!std::isfinite(eta) || eta < 0.f) return fail(TTT_ERR_INVALID_ARG, "eta must be finite and >= 0");
    const void* ps[] = {X, tq, tk, tv, W1_0, W2_0, alpha_f, alpha_r};
    for (const void* p : ps)
        if (p && !aligned16(p)) return fail(TTT_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", p);
    (void)q;
    return TTT_OK;
}

}  // namespace

namespace {

// The layer on device buffers; with X_host / Y_host (host buffers) X is first
// copied into the device buffer X and Y copied back out, overlapped with the
// computation on the pipelined path.
// Arguments of the segment attention (and of the block's attention step): Out must not overlap Q, K, V
// (it may be Xres itself: each element is read before the same thread writes it).
ttt_status check_attention(int T, int H, int d, int L, const void* Q, const void* K, const void* V, int ld_qkv,
                           const void* Xres, const void* Out, int ld_out) {
    if (!attn_seg_supported(d)) return fail(TTT_ERR_UNSUPPORTED, "segment attention needs d = 64 (got %d)", d);
    if (T < 1 || H < 1 || L < 1) return fail(TTT_ERR_INVALID_ARG, "T, H and the segment length must be positive");
    const long long cols = (long long)H * d;
    if (ld_qkv < cols || ld_out < cols || ld_qkv % 8 != 0 || ld_out % 8 != 0)
        return fail(TTT_ERR_INVALID_ARG, "row strides (%d, %d) must hold %lld columns and be multiples of 8", ld_qkv,
                    ld_out, cols);
    if (!Q || !K || !V || !Out) return fail(TTT_ERR_INVALID_ARG, "Q, K, V and Out must be non-NULL");
    const void* ps[] = {Q, K, V, Xres, Out};
    for (const void* p : ps)
        if (p && !aligned16(p)) return fail(TTT_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", p);
    const size_t in_bytes = ((size_t)(T - 1) * ld_qkv + cols) * 2, out_bytes = ((size_t)(T - 1) * ld_out + cols) * 2;
    const char* o = static_cast<const char*>(Out);
    for (const void* p : {Q, K, V}) {
        const char* c = static_cast<const char*>(p);
        if (o < c + in_bytes && c < o + out_bytes) return fail(TTT_ERR_INVALID_ARG, "Out must not overlap Q, K or V");
    }
    return TTT_OK;
}

ttt_status forward_impl(const ttt_mlp_desc* desc, const void* X, const void* theta_q, const void* theta_k,
                        const void* theta_v, const float* W1_0, const float* W2_0, float eta, int b,
                        ttt_direction dir, const float* alpha_f, const float* alpha_r, void* Y, float* Z_out,
                        float* W1_T, float* W2_T, void* workspace, size_t workspace_bytes, ttt_stream_t stream_,
                        const void* X_host, void* Y_host, bool allow_pipeline = true,
                        const RowsHook* pre_rows = nullptr, int first_front_percent = -1) {
    ttt_status st = check_desc(desc, b, dir);
    if (st != TTT_OK) return st;
    const ttt_mlp_desc& q = *desc;
    st = check_ptrs(q, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, dir, alpha_f, alpha_r);
    if (st != TTT_OK) return st;
    if (!Y || !workspace) return fail(TTT_ERR_INVALID_ARG, "Y and workspace must be non-NULL");
    const void* outs[] = {Y, Z_out, W1_T, W2_T};
    for (const void* p : outs)
        if (p && !aligned16(p)) return fail(TTT_ERR_INVALID_ARG, "output pointer %p is not 16-byte aligned", p);
    if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
        return fail(TTT_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const size_t xbytes = (size_t)q.T * q.D * elem_size(q.x_dtype);
    {
        const char* xs = static_cast<const char*>(X);
        const char* ys = static_cast<const char*>(Y);
        if (xs < ys + xbytes && ys < xs + xbytes) return fail(TTT_ERR_INVALID_ARG, "Y must not alias X");
    }
    const Layout L = plan(q, b, dir);
    if (workspace_bytes < L.total)
        return fail(TTT_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, L.total);

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
    char* ws = static_cast<char*>(workspace);
    CUDA_TRY(cudaMemsetAsync(ws + L.status, 0, 16, s));
    const int x_bf16 = q.x_dtype == TTT_BF16;
    const void* th[3] = {theta_q, theta_k, theta_v};
    float* qkv[3] = {reinterpret_cast<float*>(ws + L.qkv[0]), reinterpret_cast<float*>(ws + L.qkv[1]),
                     reinterpret_cast<float*>(ws + L.qkv[2])};
    const size_t n = (size_t)q.T * q.D;
    const size_t nW = (size_t)q.H * q.m * q.d;
    float* xp = reinterpret_cast<float*>(ws + L.xp);
    int* status = reinterpret_cast<int*>(ws + L.status);

    if (allow_pipeline && pipe_eligible(q, L, b, dir)) {
        // the cluster scan, the state W1, W2 carried between segments through the workspace
        const size_t nW = (size_t)q.H * q.m * q.d;
        float* st1 = reinterpret_cast<float*>(ws + L.state);
        float* st2 = st1 + nW;
        const bool split_groups = g_scan_impl.load() != 2;   // automatic: the split-group cluster scan
        const SegScan seg_scan = [&](int di, const Dir& dd, int cb, int ce, bool first, bool last, float* zscan,
                                     cudaStream_t ss) {
            ScanArgs a = scan_args(q, L, ws, first ? W1_0 : st1, first ? W2_0 : st2, eta, b, dd);
            a.Zscan = zscan;
            a.c_begin = cb;
            a.c_end = ce;
            a.W1_T = last ? (W1_T ? W1_T + di * nW : nullptr) : st1;
            a.W2_T = last ? (W2_T ? W2_T + di * nW : nullptr) : st2;
            if (split_groups) {
                a.fuse_gate = kSplitScanGates ? 1 : 0;
                return launch_scan_chunk_tc3(a, ss);
            }
            return launch_scan_chunk_tc2(a, ss);
        };
        const PipeBufs bufs{status, xp, reinterpret_cast<__nv_bfloat16*>(ws + L.delta),
                            reinterpret_cast<float*>(ws + L.zbuf)};
        return forward_pipelined(q, bufs, 2, seg_scan, X, th, qkv, b, dir, alpha_f, alpha_r, Y, Z_out, s, X_host,
                                 Y_host, split_groups && kSplitScanGates, pre_rows, first_front_percent);
    }
    if (pre_rows) CUDA_TRY((*pre_rows)(0, q.T, 0, s));   // X's producer, then the layer on one stream
    if (X_host) CUDA_TRY(cudaMemcpyAsync(const_cast<void*>(X), X_host, xbytes, cudaMemcpyHostToDevice, s));
    auto finish = [&]() -> ttt_status {
        if (Y_host) CUDA_TRY(cudaMemcpyAsync(Y_host, Y, xbytes, cudaMemcpyDeviceToHost, s));
        return TTT_OK;
    };

    // first (or only) direction
    Dir d0{};
    d0.reverse = dir == TTT_REV;
    d0.xin = X; d0.xin_bf16 = x_bf16;
    d0.alpha = (dir == TTT_REV) ? alpha_r : alpha_f;
    if (dir == TTT_BIDIR) { d0.out = xp; d0.out_bf16 = 0; }
    else { d0.out = Y; d0.out_bf16 = x_bf16; }
    d0.delta = L.split_reverse ? reinterpret_cast<__nv_bfloat16*>(ws + L.delta) : nullptr;
    d0.zdbg = Z_out; d0.w1t = W1_T; d0.w2t = W2_T;
    st = project(q, X, x_bf16, th, qkv, 0, status, s);
    if (st != TTT_OK) return st;
    st = scan(q, L, ws, W1_0, W2_0, eta, b, d0, s);
    if (st != TTT_OK) return st;
    if (dir != TTT_BIDIR) return finish();

    // reverse direction on X' = X + tanh(alpha_f) z_f
    if (L.split_reverse) {
        // theta X' = theta X + theta (X' - X): add the projection of the bf16
        // gate increment onto the forward projections already in place.
        st = project(q, ws + L.delta, 1, th, qkv, 1, status, s);
    } else {
        st = project(q, xp, 0, th, qkv, 0, status, s);
    }
    if (st != TTT_OK) return st;
    Dir d1{};
    d1.reverse = 1;
    d1.xin = xp; d1.xin_bf16 = 0;
    d1.alpha = alpha_r;
    d1.out = Y; d1.out_bf16 = x_bf16;
    d1.zdbg = Z_out ? Z_out + n : nullptr;
    d1.w1t = W1_T ? W1_T + nW : nullptr;
    d1.w2t = W2_T ? W2_T + nW : nullptr;
    st = scan(q, L, ws, W1_0, W2_0, eta, b, d1, s);
    if (st != TTT_OK) return st;
    return finish();
}

}  // namespace

ttt_status ttt::forward_single_stream(const ttt_mlp_desc* desc, const void* X, const void* theta_q,
                                      const void* theta_k, const void* theta_v, const float* W1_0, const float* W2_0,
                                      float eta, int b, ttt_direction dir, const float* alpha_f,
                                      const float* alpha_r, void* Y, float* Z_out, float* W1_T, float* W2_T,
                                      void* workspace, size_t workspace_bytes, ttt_stream_t stream) {
    return forward_impl(desc, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, dir, alpha_f, alpha_r, Y, Z_out, W1_T,
                        W2_T, workspace, workspace_bytes, stream, nullptr, nullptr, false);
}

namespace {

// ---------------------------------------------------------------- backward pass
struct BwdLayout {
    size_t fwd, y, zs, xp, u[3], du[3], g, dz, scratch, total;
};

BwdLayout plan_backward(const ttt_mlp_desc& q, int b, ttt_direction dir) {
    BwdLayout L{};
    const size_t n = (size_t)q.T * q.D;
    const int nd = dir == TTT_BIDIR ? 2 : 1;
    size_t off = 0;
    L.fwd = off; off = align_up(off + plan(q, b, dir).total);
    L.y = off; off = align_up(off + n * elem_size(q.x_dtype));
    L.zs = off; off = align_up(off + nd * n * sizeof(float));
    L.xp = off; if (dir == TTT_BIDIR) off = align_up(off + n * sizeof(float));
    for (int w = 0; w < 3; ++w) { L.u[w] = off; off = align_up(off + n * sizeof(float)); }
    for (int w = 0; w < 3; ++w) { L.du[w] = off; off = align_up(off + n * sizeof(float)); }
    L.g = off; off = align_up(off + n * sizeof(float));
    L.dz = off; off = align_up(off + n * sizeof(float));
    L.scratch = off; off = align_up(off + (size_t)q.H * scan_backward_scratch_floats(q.d, b, q.T) * sizeof(float));
    L.total = off;
    return L;
}

// dX += dU theta (X layout) and dtheta += dU^T src, for one projection.
// Full-width bf16 layer: the projections' gradients on the tensor cores (the projection kernel as a
// general GEMM).  Each fp32 dU_w is split into bf16 halves hi + lo (stored in U_w, free once the scan's
// backward has read it), so every product keeps about 16 significand bits of dU; theta and the sources
// are bf16 already.
//   dX (in G):  G[t, c] += sum_w sum_j (hi_w + lo_w)[t, j] theta_w[j, c]     (theta read MN-major)
//   dtheta_w:   dtheta_w[j, c] += sum_t (hi_w + lo_w)[t, j] src[t, c]        (both read MN-major)
// with src = X, and for the reverse pass of the bidirectional layer src = X + bf16 increment, the two
// bf16 arrays the forward pass projected.
ttt_status projection_grads_tc(const ttt_mlp_desc& q, float* const dU[3], const void* const th[3], const void* X,
                               const __nv_bfloat16* delta, float* const U[3], float* G, float* const dth[3],
                               int* status, cudaStream_t s) {
    const long long T = q.T, D = q.D, n = T * D;
    __nv_bfloat16* hi[3];
    __nv_bfloat16* lo[3];
    for (int w = 0; w < 3; ++w) {
        hi[w] = reinterpret_cast<__nv_bfloat16*>(U[w]);
        lo[w] = hi[w] + n;
        CUDA_TRY(launch_split_bf16(dU[w], hi[w], lo[w], n, s));
    }
    for (int part = 0; part < 2; ++part) {   // dX from the high halves, then the low halves
        GemmTc g{};
        g.nw = 1;
        g.nseg = 3;
        g.a_mn = 0;
        g.b_mn = 1;
        g.M = (int)T;
        g.N = (int)D;
        g.K = (int)D;
        for (int w = 0; w < 3; ++w) {
            g.A[0][w] = {part ? lo[w] : hi[w], D};
            g.B[0][w] = {th[w], D};
        }
        g.C[0] = G;
        g.ldc = D;
        g.accumulate = 1;
        g.status = status;
        g.name = "grad_gemm_tc";
        CUDA_TRY(launch_gemm_tc(g, s));
    }
    const void* srcs[2] = {X, delta};
    const int nsrc = delta ? 2 : 1;
    GemmTc g{};
    g.nw = 3;
    g.nseg = 2 * nsrc;
    g.a_mn = 1;
    g.b_mn = 1;
    g.M = (int)D;
    g.N = (int)D;
    g.K = (int)T;
    for (int w = 0; w < 3; ++w) {
        int sg = 0;
        for (int k = 0; k < nsrc; ++k)
            for (int part = 0; part < 2; ++part) {
                g.A[w][sg] = {part ? lo[w] : hi[w], D};
                g.B[w][sg] = {srcs[k], D};
                ++sg;
            }
        g.C[w] = dth[w];
    }
    g.ldc = D;
    g.accumulate = 1;
    g.status = status;
    g.name = "grad_gemm_tc";
    CUDA_TRY(launch_gemm_tc(g, s));
    return TTT_OK;
}

ttt_status projection_grads(const ttt_mlp_desc& q, const float* dU, const void* theta, int th_bf16, const void* src,
                            int src_bf16, float* G, float* dtheta, cudaStream_t s) {
    const long long T = q.T, D = q.D, d = q.d;
    if (q.per_head_input) {   // per head: U[h] [T x d] = X[h] theta[h]^T
        CUDA_TRY(launch_grad_gemm(G, d, T * d, dU, 0, d, 1, T * d, theta, th_bf16, d, 1, d * d, q.H, (int)T, (int)d, d,
                                  1, s));
        CUDA_TRY(launch_grad_gemm(dtheta, d, d * d, dU, 0, 1, d, T * d, src, src_bf16, d, 1, T * d, q.H, (int)d,
                                  (int)d, T, 1, s));
    } else {                  // full width: U [T x D] = X theta^T, theta [D x D]
        CUDA_TRY(launch_grad_gemm(G, D, 0, dU, 0, D, 1, 0, theta, th_bf16, D, 1, 0, 1, (int)T, (int)D, D, 1, s));
        CUDA_TRY(launch_grad_gemm(dtheta, D, 0, dU, 0, 1, D, 0, src, src_bf16, D, 1, 0, 1, (int)D, (int)D, T, 1, s));
    }
    return TTT_OK;
}

}  // namespace

namespace {

// ---------------------------------------------------------------- TTT-Linear
ttt_status check_desc_linear(const ttt_mlp_desc* desc, int b, ttt_direction dir) {
    if (!desc) return fail(TTT_ERR_INVALID_ARG, "desc is NULL");
    ttt_mlp_desc q = *desc;
    q.m = 4 * q.d;   // not used by the linear layer
    return check_desc(&q, b, dir);
}

struct LinearLayout {
    size_t status, qkv[3], xp, delta, zbuf, state, total;
    bool split_reverse;
};

LinearLayout plan_linear(const ttt_mlp_desc& q, ttt_direction dir) {
    LinearLayout L{};
    const size_t n = (size_t)q.T * q.D;
    size_t off = 0;
    L.status = off; off += kAlign;
    for (int w = 0; w < 3; ++w) { L.qkv[w] = off; off = align_up(off + n * sizeof(float)); }
    L.split_reverse = (dir == TTT_BIDIR) && !q.per_head_input && q.x_dtype == TTT_BF16;
    L.xp = off;
    if (dir == TTT_BIDIR) off = align_up(off + n * sizeof(float));
    L.delta = off;
    if (L.split_reverse) off = align_up(off + n * 2);
    L.zbuf = off;
    off = align_up(off + n * sizeof(float));
    L.state = off;   // W of every head between two segments of a pipelined direction
    off = align_up(off + (size_t)q.H * q.d * q.d * sizeof(float));
    L.total = off;
    return L;
}

ttt_status linear_direction(const ttt_mlp_desc& q, const LinearLayout& L, char* ws, const void* xin, int xin_bf16,
                            const void* src, int src_bf16, int accumulate, const void* const th[3],
                            const float* W_0, float eta, int b, int reverse, const float* alpha, void* out,
                            int out_bf16, __nv_bfloat16* delta, float* z_out, float* w_t, cudaStream_t s) {
    int* status = reinterpret_cast<int*>(ws + L.status);
    float* qkv[3] = {reinterpret_cast<float*>(ws + L.qkv[0]), reinterpret_cast<float*>(ws + L.qkv[1]),
                     reinterpret_cast<float*>(ws + L.qkv[2])};
    ttt_status st = project(q, src, src_bf16, th, qkv, accumulate, status, s);
    if (st != TTT_OK) return st;
    LinearScanArgs a{};
    a.Q = qkv[0]; a.K = qkv[1]; a.V = qkv[2];
    if (q.per_head_input) { a.qkv_hs = (long long)q.T * q.d; a.qkv_ts = q.d; }
    else { a.qkv_hs = q.d; a.qkv_ts = q.D; }
    a.x_hs = a.qkv_hs; a.x_ts = a.qkv_ts;
    a.Z = z_out ? z_out : reinterpret_cast<float*>(ws + L.zbuf);
    a.W_0 = W_0; a.W_T = w_t;
    a.T = q.T; a.H = q.H; a.d = q.d; a.b = b; a.reverse = reverse; a.eta = eta;
    a.status = status;
    // bf16-input layers (tolerance 2e-2) take the tensor-core chunk form; fp32 inputs, b = 1 and
    // ttt_mlp_select_kernels(1, .) keep the fp32 SIMT scan
    if (g_scan_impl.load() != 1 && q.x_dtype == TTT_BF16 && scan_linear_tc_supported(q.d, b))
        CUDA_TRY(launch_scan_linear_tc(a, s));
    else
        CUDA_TRY(launch_scan_linear(a, s));
    CUDA_TRY(launch_gate(xin, xin_bf16, a.Z, alpha, out, out_bf16, delta, status, q.T, q.H, q.d,
                         q.per_head_input, 0, s));
    return TTT_OK;
}

}  // namespace

extern "C" {

size_t ttt_mlp_workspace_size(const ttt_mlp_desc* desc, int b, ttt_direction dir) {
    if (check_desc(desc, b, dir) != TTT_OK) return 0;
    return plan(*desc, b, dir).total;
}

size_t ttt_mlp_host_io_workspace_size(const ttt_mlp_desc* desc, int b, ttt_direction dir) {
    if (check_desc(desc, b, dir) != TTT_OK) return 0;
    const size_t io = align_up((size_t)desc->T * desc->D * elem_size(desc->x_dtype));
    return plan(*desc, b, dir).total + 2 * io;
}

ttt_status ttt_mlp_forward(const ttt_mlp_desc* desc, const void* X, const void* theta_q, const void* theta_k,
                           const void* theta_v, const float* W1_0, const float* W2_0, float eta, int b,
                           ttt_direction dir, const float* alpha_f, const float* alpha_r, void* Y, float* Z_out,
                           float* W1_T, float* W2_T, void* workspace, size_t workspace_bytes,
                           ttt_stream_t stream_) {
    return forward_impl(desc, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, dir, alpha_f, alpha_r, Y, Z_out, W1_T,
                        W2_T, workspace, workspace_bytes, stream_, nullptr, nullptr);
}

size_t ttt_linear_workspace_size(const ttt_mlp_desc* desc, int b, ttt_direction dir) {
    if (check_desc_linear(desc, b, dir) != TTT_OK) return 0;
    return plan_linear(*desc, dir).total;
}

}  // extern "C"

namespace {
// ttt_linear_forward; with X_host / Y_host set, X is copied in from X_host and Y out to Y_host (segment by
// segment on the pipelined path, whole otherwise) and X, Y are the device staging arrays.
ttt_status linear_impl(const ttt_mlp_desc* desc, const void* X, const void* theta_q, const void* theta_k,
                       const void* theta_v, const float* W_0, float eta, int b, ttt_direction dir,
                       const float* alpha_f, const float* alpha_r, void* Y, float* Z_out, float* W_T,
                       void* workspace, size_t workspace_bytes, ttt_stream_t stream_, const void* X_host,
                       void* Y_host) {
    ttt_status st = check_desc_linear(desc, b, dir);
    if (st != TTT_OK) return st;
    const ttt_mlp_desc& q = *desc;
    if (!scan_linear_supported(q.d)) return fail(TTT_ERR_UNSUPPORTED, "head dim d=%d not supported (16, 32, 64)", q.d);
    st = check_ptrs(q, X, theta_q, theta_k, theta_v, W_0, W_0, eta, dir, alpha_f, alpha_r);
    if (st != TTT_OK) return st;
    if (!Y || !workspace) return fail(TTT_ERR_INVALID_ARG, "Y and workspace must be non-NULL");
    const void* outs[] = {Y, Z_out, W_T};
    for (const void* p : outs)
        if (p && !aligned16(p)) return fail(TTT_ERR_INVALID_ARG, "output pointer %p is not 16-byte aligned", p);
    if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
        return fail(TTT_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const size_t xbytes = (size_t)q.T * q.D * elem_size(q.x_dtype);
    {
        const char* xs = static_cast<const char*>(X);
        const char* ys = static_cast<const char*>(Y);
        if (xs < ys + xbytes && ys < xs + xbytes) return fail(TTT_ERR_INVALID_ARG, "Y must not alias X");
    }
    const LinearLayout L = plan_linear(q, dir);
    if (workspace_bytes < L.total)
        return fail(TTT_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, L.total);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
    char* ws = static_cast<char*>(workspace);
    CUDA_TRY(cudaMemsetAsync(ws + L.status, 0, 16, s));
    const int x_bf16 = q.x_dtype == TTT_BF16;
    const void* th[3] = {theta_q, theta_k, theta_v};
    const size_t n = (size_t)q.T * q.D, nW = (size_t)q.H * q.d * q.d;
    float* xp = reinterpret_cast<float*>(ws + L.xp);
    __nv_bfloat16* delta = L.split_reverse ? reinterpret_cast<__nv_bfloat16*>(ws + L.delta) : nullptr;
    // the full-width bf16 layer on the tensor cores: chunk segments on two streams, as for the MLP layer
    if (!q.per_head_input && x_bf16 && g_scan_impl.load() != 1 && scan_linear_tc_supported(q.d, b) &&
        g_proj_impl.load() != 1 && proj_full_tc_supported(q.D, q.D) && (dir != TTT_BIDIR || L.split_reverse) &&
        pipe_side_sms(q, 1) > 0) {
        float* stW = reinterpret_cast<float*>(ws + L.state);
        int* status = reinterpret_cast<int*>(ws + L.status);
        float* qkv[3] = {reinterpret_cast<float*>(ws + L.qkv[0]), reinterpret_cast<float*>(ws + L.qkv[1]),
                         reinterpret_cast<float*>(ws + L.qkv[2])};
        const SegScan seg_scan = [&](int di, const Dir& dd, int cb, int ce, bool first, bool last, float* zscan,
                                     cudaStream_t ss) {
            LinearScanArgs a{};
            a.Q = qkv[0]; a.K = qkv[1]; a.V = qkv[2];
            a.qkv_hs = q.d; a.qkv_ts = q.D; a.x_hs = q.d; a.x_ts = q.D;
            a.Z = zscan;
            a.W_0 = first ? W_0 : stW;
            a.W_T = last ? (W_T ? W_T + di * nW : nullptr) : stW;
            a.T = q.T; a.H = q.H; a.d = q.d; a.b = b; a.reverse = dd.reverse; a.eta = eta;
            a.status = status;
            a.c_begin = cb;
            a.c_end = ce;
            return launch_scan_linear_tc(a, ss);
        };
        const PipeBufs bufs{status, xp, delta, reinterpret_cast<float*>(ws + L.zbuf)};
        return forward_pipelined(q, bufs, 1, seg_scan, X, th, qkv, b, dir, alpha_f, alpha_r, Y, Z_out, s, X_host,
                                 Y_host);
    }
    if (X_host) CUDA_TRY(cudaMemcpyAsync(const_cast<void*>(X), X_host, xbytes, cudaMemcpyHostToDevice, s));
    if (dir != TTT_BIDIR) {
        st = linear_direction(q, L, ws, X, x_bf16, X, x_bf16, 0, th, W_0, eta, b, dir == TTT_REV,
                              dir == TTT_REV ? alpha_r : alpha_f, Y, x_bf16, nullptr, Z_out, W_T, s);
    } else {
        st = linear_direction(q, L, ws, X, x_bf16, X, x_bf16, 0, th, W_0, eta, b, 0, alpha_f, xp, 0, delta, Z_out,
                              W_T, s);
        if (st != TTT_OK) return st;
        // reverse on X' = X + tanh(alpha_f) z_f; theta X' = theta X + theta bf16(X' - X) where X is bf16 and full
        // width
        st = linear_direction(q, L, ws, xp, 0, L.split_reverse ? static_cast<const void*>(delta) : xp,
                              L.split_reverse ? 1 : 0, L.split_reverse ? 1 : 0, th, W_0, eta, b, 1, alpha_r, Y,
                              x_bf16, nullptr, Z_out ? Z_out + n : nullptr, W_T ? W_T + nW : nullptr, s);
    }
    if (st != TTT_OK) return st;
    if (Y_host) CUDA_TRY(cudaMemcpyAsync(Y_host, Y, xbytes, cudaMemcpyDeviceToHost, s));
    return TTT_OK;
}
}  // namespace

extern "C" {

ttt_status ttt_linear_forward(const ttt_mlp_desc* desc, const void* X, const void* theta_q, const void* theta_k,
                              const void* theta_v, const float* W_0, float eta, int b, ttt_direction dir,
                              const float* alpha_f, const float* alpha_r, void* Y, float* Z_out, float* W_T,
                              void* workspace, size_t workspace_bytes, ttt_stream_t stream) {
    return linear_impl(desc, X, theta_q, theta_k, theta_v, W_0, eta, b, dir, alpha_f, alpha_r, Y, Z_out, W_T,
                       workspace, workspace_bytes, stream, nullptr, nullptr);
}

size_t ttt_linear_host_io_workspace_size(const ttt_mlp_desc* desc, int b, ttt_direction dir) {
    if (check_desc_linear(desc, b, dir) != TTT_OK) return 0;
    const size_t io = align_up((size_t)desc->T * desc->D * elem_size(desc->x_dtype));
    return plan_linear(*desc, dir).total + 2 * io;
}

ttt_status ttt_linear_forward_host(const ttt_mlp_desc* desc, const void* X_host, const void* theta_q,
                                   const void* theta_k, const void* theta_v, const float* W_0, float eta, int b,
                                   ttt_direction dir, const float* alpha_f, const float* alpha_r, void* Y_host,
                                   void* workspace, size_t workspace_bytes, ttt_stream_t stream) {
    ttt_status st = check_desc_linear(desc, b, dir);
    if (st != TTT_OK) return st;
    if (!X_host || !Y_host || !workspace) return fail(TTT_ERR_INVALID_ARG, "X_host, Y_host, workspace must be non-NULL");
    const size_t need = ttt_linear_host_io_workspace_size(desc, b, dir);
    if (workspace_bytes < need)
        return fail(TTT_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
    const LinearLayout L = plan_linear(*desc, dir);
    const size_t xbytes = (size_t)desc->T * desc->D * elem_size(desc->x_dtype);
    char* ws = static_cast<char*>(workspace);
    void* Xd = ws + L.total;
    void* Yd = ws + L.total + align_up(xbytes);
    st = linear_impl(desc, Xd, theta_q, theta_k, theta_v, W_0, eta, b, dir, alpha_f, alpha_r, Yd, nullptr, nullptr,
                     workspace, L.total, stream, X_host, Y_host);
    if (st != TTT_OK) return st;
    return ttt_mlp_status(workspace, stream);
}

size_t ttt_mlp_backward_workspace_size(const ttt_mlp_desc* desc, int b, ttt_direction dir) {
    if (check_desc(desc, b, dir) != TTT_OK) return 0;
    if (b > 64) {
        fail(TTT_ERR_UNSUPPORTED, "backward pass: chunk size b=%d above 64", b);
        return 0;
    }
    return plan_backward(*desc, b, dir).total;
}

ttt_status ttt_mlp_backward(const ttt_mlp_desc* desc, const void* X, const void* theta_q, const void* theta_k,
                            const void* theta_v, const float* W1_0, const float* W2_0, float eta, int b,
                            ttt_direction dir, const float* alpha_f, const float* alpha_r, const float* dY, float* dX,
                            float* dtheta_q, float* dtheta_k, float* dtheta_v, float* dW1_0, float* dW2_0,
                            float* dalpha_f, float* dalpha_r, void* workspace, size_t workspace_bytes,
                            ttt_stream_t stream_) {
    ttt_status st = check_desc(desc, b, dir);
    if (st != TTT_OK) return st;
    const ttt_mlp_desc& q = *desc;
    if (b > 64) return fail(TTT_ERR_UNSUPPORTED, "backward pass: chunk size b=%d above 64", b);
    st = check_ptrs(q, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, dir, alpha_f, alpha_r);
    if (st != TTT_OK) return st;
    const bool uses_f = dir != TTT_REV, uses_r = dir != TTT_FWD;
    if (!dY || !dX || !dtheta_q || !dtheta_k || !dtheta_v || !dW1_0 || !dW2_0 || (uses_f && !dalpha_f) ||
        (uses_r && !dalpha_r) || !workspace)
        return fail(TTT_ERR_INVALID_ARG, "dY, every gradient output of this direction and workspace must be non-NULL");
    const void* ps[] = {dY, dX, dtheta_q, dtheta_k, dtheta_v, dW1_0, dW2_0, dalpha_f, dalpha_r};
    for (const void* p : ps)
        if (p && !aligned16(p)) return fail(TTT_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", p);
    if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
        return fail(TTT_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const BwdLayout B = plan_backward(q, b, dir);
    if (workspace_bytes < B.total)
        return fail(TTT_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, B.total);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
    char* ws = static_cast<char*>(workspace);
    const size_t n = (size_t)q.T * q.D;
    const int x_bf16 = q.x_dtype == TTT_BF16;
    float* zs = reinterpret_cast<float*>(ws + B.zs);

    // the forward pass, keeping each direction's z (its status word lands at the workspace start)
    st = forward_impl(desc, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, dir, alpha_f, alpha_r, ws + B.y, zs,
                      nullptr, nullptr, ws + B.fwd, plan(q, b, dir).total, stream_, nullptr, nullptr);
    if (st != TTT_OK) return st;
    int* status = reinterpret_cast<int*>(ws + B.fwd);
    const size_t th_elems = q.per_head_input ? (size_t)q.H * q.d * q.d : (size_t)q.D * q.D;
    const size_t w_elems = (size_t)q.H * q.m * q.d;
    float* dth[3] = {dtheta_q, dtheta_k, dtheta_v};
    for (float* p : dth) CUDA_TRY(cudaMemsetAsync(p, 0, th_elems * sizeof(float), s));
    CUDA_TRY(cudaMemsetAsync(dW1_0, 0, w_elems * sizeof(float), s));
    CUDA_TRY(cudaMemsetAsync(dW2_0, 0, w_elems * sizeof(float), s));
    if (dalpha_f && uses_f) CUDA_TRY(cudaMemsetAsync(dalpha_f, 0, q.D * sizeof(float), s));
    if (dalpha_r && uses_r) CUDA_TRY(cudaMemsetAsync(dalpha_r, 0, q.D * sizeof(float), s));
    float* G = reinterpret_cast<float*>(ws + B.g);   // gradient with respect to the current gate's output
    CUDA_TRY(cudaMemcpyAsync(G, dY, n * sizeof(float), cudaMemcpyDeviceToDevice, s));
    float* xp = reinterpret_cast<float*>(ws + B.xp);
    // the full-width bf16 layer takes its projection gradients on the tensor cores, and (as its forward pass
    // does) projects the reverse direction's input as X plus the bf16 gate increment, kept where Y was
    const bool tc_grads = !q.per_head_input && x_bf16 && proj_full_tc_supported(q.D, q.D) && g_proj_impl.load() != 1;
    __nv_bfloat16* delta = tc_grads && dir == TTT_BIDIR ? reinterpret_cast<__nv_bfloat16*>(ws + B.y) : nullptr;
    if (dir == TTT_BIDIR)   // X' = X + tanh(alpha_f) z_f, the reverse direction's input
        CUDA_TRY(launch_gate(X, x_bf16, zs, alpha_f, xp, 0, delta, status, q.T, q.H, q.d, q.per_head_input, 0, s));
    const void* th[3] = {theta_q, theta_k, theta_v};
    float* U[3] = {reinterpret_cast<float*>(ws + B.u[0]), reinterpret_cast<float*>(ws + B.u[1]),
                   reinterpret_cast<float*>(ws + B.u[2])};
    float* dU[3] = {reinterpret_cast<float*>(ws + B.du[0]), reinterpret_cast<float*>(ws + B.du[1]),
                    reinterpret_cast<float*>(ws + B.du[2])};
    float* dz = reinterpret_cast<float*>(ws + B.dz);
    const long long qkv_hs = q.per_head_input ? (long long)q.T * q.d : q.d;
    const long long qkv_ts = q.per_head_input ? q.d : q.D;
    // directions from the last to the first
    const int ndir = dir == TTT_BIDIR ? 2 : 1;
    for (int k = ndir - 1; k >= 0; --k) {
        const bool reverse = dir == TTT_REV || k == 1;
        const bool on_xp = dir == TTT_BIDIR && k == 1;
        const void* src = on_xp ? static_cast<const void*>(xp) : X;
        const int src_bf16 = on_xp ? 0 : x_bf16;
        CUDA_TRY(launch_gate_backward(G, zs + k * n, reverse ? alpha_r : alpha_f, dz, reverse ? dalpha_r : dalpha_f,
                                      q.T, q.H, q.d, q.per_head_input, s));
        if (on_xp && delta) {
            st = project(q, X, 1, th, U, 0, status, s);
            if (st == TTT_OK) st = project(q, delta, 1, th, U, 1, status, s);
        } else {
            st = project(q, src, src_bf16, th, U, 0, status, s);
        }
        if (st != TTT_OK) return st;
        CUDA_TRY(launch_scan_backward(U[0], U[1], U[2], qkv_hs, qkv_ts, dz, qkv_hs, qkv_ts, W1_0, W2_0, dU[0], dU[1],
                                      dU[2], dW1_0, dW2_0, reinterpret_cast<float*>(ws + B.scratch), q.T, q.H, q.d, b,
                                      reverse ? 1 : 0, eta, x_bf16 ? 0 : 1, s));
        if (tc_grads) {   // the gate's x path keeps G; the projections add theta's share
            st = projection_grads_tc(q, dU, th, X, on_xp ? delta : nullptr, U, G, dth, status, s);
            if (st != TTT_OK) return st;
        } else {
            for (int w = 0; w < 3; ++w) {
                st = projection_grads(q, dU[w], th[w], x_bf16, src, src_bf16, G, dth[w], s);
                if (st != TTT_OK) return st;
            }
        }
    }
    CUDA_TRY(cudaMemcpyAsync(dX, G, n * sizeof(float), cudaMemcpyDeviceToDevice, s));
    return TTT_OK;
}

ttt_status ttt_mlp_status(void* workspace, ttt_stream_t stream_) {
    if (!workspace) return fail(TTT_ERR_INVALID_ARG, "workspace is NULL");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
    CUDA_TRY(cudaStreamSynchronize(s));
    int word = 0;
    CUDA_TRY(cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost));
    CUDA_TRY(cudaMemset(workspace, 0, sizeof(int)));
    if (word & kStatusTimeout) return fail(TTT_ERR_TIMEOUT, "a bounded wait inside a scan kernel expired");
    if (word & kStatusNonFinite)
        return fail(TTT_ERR_NONFINITE, "non-finite values in the inputs, projections or outputs");
    return TTT_OK;
}

// ---------------------------------------------------------------- one rank's heads
size_t ttt_mlp_heads_workspace_size(const ttt_mlp_desc* desc, int hn, int b) {
    if (check_desc(desc, b, TTT_BIDIR) != TTT_OK || hn < 1 || hn > desc->H) return 0;
    const size_t nl = (size_t)desc->T * hn * desc->d;
    return kAlign + 3 * align_up(nl * sizeof(float));
}

ttt_status ttt_mlp_forward_heads(const ttt_mlp_desc* desc, int h0, int hn, ttt_phase phase, const void* X,
                                 const void* theta_q, const void* theta_k, const void* theta_v, const float* W1_0,
                                 const float* W2_0, float eta, int b, const float* alpha, const void* delta_all,
                                 float* Xp, void* delta_or_y, void* workspace, size_t workspace_bytes,
                                 ttt_stream_t stream_) {
    ttt_status st = check_desc(desc, b, TTT_BIDIR);
    if (st != TTT_OK) return st;
    const ttt_mlp_desc& q = *desc;
    if (q.per_head_input || q.x_dtype != TTT_BF16)
        return fail(TTT_ERR_UNSUPPORTED, "head phases need a full-width bf16 layer");
    if (!scan_chunk_tc_supported(q.d, b) || !proj_full_tc_supported(q.d, q.D))
        return fail(TTT_ERR_UNSUPPORTED, "head phases need d = 64, 2 <= b <= 64 and D %% 64 == 0");
    if (phase != TTT_PHASE_FWD && phase != TTT_PHASE_REV) return fail(TTT_ERR_INVALID_ARG, "bad phase");
    if (h0 < 0 || hn < 1 || h0 + hn > q.H)
        return fail(TTT_ERR_INVALID_ARG, "heads [%d, %d) outside [0, %d)", h0, h0 + hn, q.H);
    const bool rev = phase == TTT_PHASE_REV;
    st = check_ptrs(q, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, TTT_FWD, alpha, alpha);
    if (st != TTT_OK) return st;
    if (!Xp || !delta_or_y || !workspace || (rev && !delta_all))
        return fail(TTT_ERR_INVALID_ARG, "Xp, delta_or_y, workspace (and delta_all for the reverse phase) needed");
    const void* ps[] = {Xp, delta_or_y, delta_all};
    for (const void* p : ps)
        if (p && !aligned16(p)) return fail(TTT_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", p);
    if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
        return fail(TTT_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const size_t need = ttt_mlp_heads_workspace_size(desc, hn, b);
    if (workspace_bytes < need)
        return fail(TTT_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, need);

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
    char* ws = static_cast<char*>(workspace);
    int* status = reinterpret_cast<int*>(ws);
    CUDA_TRY(cudaMemsetAsync(ws, 0, 16, s));
    const int N = hn * q.d;
    const size_t nl = (size_t)q.T * N;
    float* qkv[3];
    for (int w = 0; w < 3; ++w) qkv[w] = reinterpret_cast<float*>(ws + kAlign + w * align_up(nl * sizeof(float)));
    // the heads' rows of theta: Q, K, V [T, hn d] from X (and, reverse, the gate increment of every head)
    const size_t row0 = (size_t)h0 * q.d * q.D;
    const void* th[3] = {static_cast<const __nv_bfloat16*>(theta_q) + row0,
                         static_cast<const __nv_bfloat16*>(theta_k) + row0,
                         static_cast<const __nv_bfloat16*>(theta_v) + row0};
    CUDA_TRY(launch_proj_full_tc(X, th, qkv, q.T, N, q.D, 0, status, 0, s));
    if (rev) CUDA_TRY(launch_proj_full_tc(delta_all, th, qkv, q.T, N, q.D, 1, status, 0, s));

    ScanArgs a{};
    a.Q = qkv[0]; a.K = qkv[1]; a.V = qkv[2];
    a.qkv_hs = q.d; a.qkv_ts = N;
    a.x_hs = q.d; a.x_ts = q.D;   // X, X', the increment and Y: [T, D], these heads' columns
    const size_t col0 = (size_t)h0 * q.d;
    __nv_bfloat16* dy = static_cast<__nv_bfloat16*>(delta_or_y) + col0;
    if (rev) {
        a.Xin = Xp + col0; a.xin_bf16 = 0;
        a.Out = dy; a.out_bf16 = 1; a.Delta = nullptr;
    } else {
        a.Xin = static_cast<const __nv_bfloat16*>(X) + col0; a.xin_bf16 = 1;
        a.Out = Xp + col0; a.out_bf16 = 0; a.Delta = dy;
    }
    a.alpha = alpha + col0;
    a.W1_0 = W1_0 + (size_t)h0 * q.m * q.d;
    a.W2_0 = W2_0 + (size_t)h0 * q.d * q.m;
    a.T = q.T; a.H = hn; a.d = q.d; a.m = q.m; a.b = b; a.reverse = rev ? 1 : 0;
    a.eta = eta;
    a.status = status;
    a.inject_timeout = g_inject_timeout.load();
    a.fuse_gate = 1;
    CUDA_TRY(launch_scan_chunk_tc3(a, s));
    return TTT_OK;
}

// ---------------------------------------------------------------- segment-local attention, the block
size_t ttt_seg_attention_workspace_size(void) { return kAlign; }

ttt_status ttt_seg_attention(int T, int H, int d, int L, const void* Q, const void* K, const void* V, int ld_qkv,
                             const void* Xres, void* Out, int ld_out, int row0, int row1, void* workspace,
                             size_t workspace_bytes, ttt_stream_t stream_) {
    ttt_status st = check_attention(T, H, d, L, Q, K, V, ld_qkv, Xres, Out, ld_out);
    if (st != TTT_OK) return st;
    if (row0 < 0 || row1 < row0 || row1 > T)
        return fail(TTT_ERR_INVALID_ARG, "rows [%d, %d) outside [0, %d]", row0, row1, T);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 || workspace_bytes < kAlign)
        return fail(TTT_ERR_INVALID_ARG, "workspace must be %zu bytes, 256-byte aligned", kAlign);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_);
    int* status = static_cast<int*>(workspace);
    CUDA_TRY(cudaMemsetAsync(status, 0, 16, s));
    CUDA_TRY(launch_attn_seg(Q, K, V, ld_qkv, Xres, ld_out, Out, ld_out, T, H, L, row0, row1, status, 0, s));
    return TTT_OK;
}

size_t ttt_block_workspace_size(const ttt_mlp_desc* desc, int b) { return ttt_mlp_workspace_size(desc, b, TTT_BIDIR); }

ttt_status ttt_block_forward(const ttt_mlp_desc* desc, int seg_len, const void* Qa, const void* Ka, const void* Va,
                             int ld_qkv, const void* Xres, void* X, const void* theta_q, const void* theta_k,
                             const void* theta_v, const float* W1_0, const float* W2_0, float eta, int b,
                             const float* alpha_f, const float* alpha_r, void* Y, void* workspace,
                             size_t workspace_bytes, ttt_stream_t stream) {
    ttt_status st = check_desc(desc, b, TTT_BIDIR);
    if (st != TTT_OK) return st;
    const ttt_mlp_desc& q = *desc;
    if (q.per_head_input || q.x_dtype != TTT_BF16 || q.D != q.H * q.d)
        return fail(TTT_ERR_UNSUPPORTED, "the block needs a full-width bf16 layer with D = H * d");
    st = check_attention(q.T, q.H, q.d, seg_len, Qa, Ka, Va, ld_qkv, Xres, X, q.D);
    if (st != TTT_OK) return st;
    if (workspace_bytes < ttt_block_workspace_size(desc, b) || !workspace)
        return fail(TTT_ERR_INVALID_ARG, "workspace too small");
    int* status = reinterpret_cast<int*>(static_cast<char*>(workspace) + plan(q, b, TTT_BIDIR).status);
    // Default: the attention of every row as one launch on the whole GPU, ahead of the first projection, then
    // the layer's own schedule.  The layer's projections and scan already occupy every SM (the scan's CTA
    // pairs, the projections the rest), so attention beside them only takes SMs from the projections; with a
    // head start p >= 0 set (ttt_debug_set_block_front), each segment's rows are attended to just before
    // that segment's projection instead.
    const int front = g_block_front.load();
    const bool interleave = front >= 0;
    const RowsHook attention = [&](int r0, int r1, int max_ctas, cudaStream_t ss) -> cudaError_t {
        if (!interleave) {
            if (r0 != 0) return cudaSuccess;
            r1 = q.T;
            max_ctas = 0;
        }
        return launch_attn_seg(Qa, Ka, Va, ld_qkv, Xres, q.D, X, q.D, q.T, q.H, seg_len, r0, r1, status, max_ctas,
                               ss);
    };
    return forward_impl(desc, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, TTT_BIDIR, alpha_f, alpha_r, Y,
                        nullptr, nullptr, nullptr, workspace, workspace_bytes, stream, nullptr, nullptr, true,
                        &attention, interleave ? front : -1);
}

ttt_status ttt_mlp_forward_host(const ttt_mlp_desc* desc, const void* X_host, const void* theta_q,
                                const void* theta_k, const void* theta_v, const float* W1_0, const float* W2_0,
                                float eta, int b, ttt_direction dir, const float* alpha_f, const float* alpha_r,
                                void* Y_host, void* workspace, size_t workspace_bytes, ttt_stream_t stream_) {
    ttt_status st = check_desc(desc, b, dir);
    if (st != TTT_OK) return st;
    if (!X_host || !Y_host || !workspace) return fail(TTT_ERR_INVALID_ARG, "X_host, Y_host, workspace must be non-NULL");
    const ttt_mlp_desc& q = *desc;
    const size_t need = ttt_mlp_host_io_workspace_size(desc, b, dir);
    if (workspace_bytes < need)
        return fail(TTT_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
    const Layout L = plan(q, b, dir);
    const size_t xbytes = (size_t)q.T * q.D * elem_size(q.x_dtype);
    char* ws = static_cast<char*>(workspace);
    void* Xd = ws + L.total;
    void* Yd = ws + L.total + align_up(xbytes);
    st = forward_impl(desc, Xd, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, dir, alpha_f, alpha_r, Yd, nullptr,
                      nullptr, nullptr, workspace, L.total, stream_, X_host, Y_host);
    if (st != TTT_OK) return st;
    return ttt_mlp_status(workspace, stream_);
}

ttt_status ttt_mlp_select_kernels(int scan_impl, int proj_impl) {
    if (scan_impl < 0 || scan_impl > 4 || proj_impl < 0 || proj_impl > 2)
        return fail(TTT_ERR_INVALID_ARG,
                    "kernel selector must be 0 (auto), 1 (SIMT), 2 (tensor core) or, for the scan, 3 (tensor core, "
                    "one CTA per head) or 4 (tensor core, two warp groups per CTA)");
    g_scan_impl.store(scan_impl);
    g_proj_impl.store(proj_impl);
    return TTT_OK;
}

ttt_status ttt_kernel_timing(int enable) {
    std::lock_guard<std::mutex> lk(g_timing_mu);
    if (enable) {
        for (auto& r : g_timed) { cudaEventDestroy(r.start); cudaEventDestroy(r.stop); }
        g_timed.clear();
    }
    g_timing_on.store(enable != 0);
    return TTT_OK;
}

int ttt_kernel_times(int max_kernels, char* names, size_t names_cap, double* total_ms, uint64_t* launches) {
    std::lock_guard<std::mutex> lk(g_timing_mu);
    std::vector<std::string> keys;
    std::vector<double> ms;
    std::vector<uint64_t> cnt;
    for (auto& r : g_timed) {
        if (cudaEventSynchronize(r.stop) != cudaSuccess) return -1;
        float e = 0.f;
        if (cudaEventElapsedTime(&e, r.start, r.stop) != cudaSuccess) return -1;
        size_t k = 0;
        while (k < keys.size() && keys[k] != r.name) ++k;
        if (k == keys.size()) { keys.emplace_back(r.name); ms.push_back(0.0); cnt.push_back(0); }
        ms[k] += e;
        cnt[k] += 1;
    }
    std::string csv;
    const int n = (int)keys.size() < max_kernels ? (int)keys.size() : max_kernels;
    for (int k = 0; k < n; ++k) {
        if (total_ms) total_ms[k] = ms[k];
        if (launches) launches[k] = cnt[k];
        csv += keys[k];
        csv += '\n';
    }
    if (names && names_cap) {
        std::strncpy(names, csv.c_str(), names_cap - 1);
        names[names_cap - 1] = '\0';
    }
    return (int)keys.size();
}

int ttt_debug_pipe_segments(int nchunks, int* out, int max_segments) {
    if (nchunks < 1) return -1;
    const auto seg = pipe_segments(nchunks);
    for (int k = 0; k < (int)seg.size() && k < max_segments && out; ++k) {
        out[2 * k] = seg[k].first;
        out[2 * k + 1] = seg[k].second;
    }
    return (int)seg.size();
}

ttt_status ttt_debug_set_block_front(int percent) {
    if (percent < -1 || percent > 100) return fail(TTT_ERR_INVALID_ARG, "percent must be -1 (default) or 0..100");
    g_block_front.store(percent);
    return TTT_OK;
}

ttt_status ttt_debug_set_backward_ctas(int ctas) {
    if (ctas < 0 || ctas > 2) return fail(TTT_ERR_INVALID_ARG, "ctas must be 0 (automatic), 1 or 2");
    set_scan_backward_ctas(ctas);
    return TTT_OK;
}

ttt_status ttt_debug_inject_wait_timeout(int enable) {
    g_inject_timeout.store(enable ? 1 : 0);
    return TTT_OK;
}

const char* ttt_last_error(void) { return t_err.c_str(); }

uint64_t ttt_launch_count(void) { return g_launches.load(); }

}  // extern "C"
