"""Python binding of libtttmlp.so (the C ABI in include/tttmlp.h).

Argument marshalling only: every function forwards to the C entry point of
the same name; all arithmetic runs in the library's CUDA kernels.  PyTorch
is used for device memory and streams.  There is no fallback: if the
library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtttmlp.so")
_lib = None

TTT_OK, TTT_ERR_INVALID_ARG, TTT_ERR_UNSUPPORTED, TTT_ERR_CUDA, TTT_ERR_NONFINITE, TTT_ERR_TIMEOUT = range(6)
STATUS_NAMES = {0: "TTT_OK", 1: "TTT_ERR_INVALID_ARG", 2: "TTT_ERR_UNSUPPORTED", 3: "TTT_ERR_CUDA",
                4: "TTT_ERR_NONFINITE", 5: "TTT_ERR_TIMEOUT"}
TTT_FWD, TTT_REV, TTT_BIDIR = 0, 1, 2
TTT_F32, TTT_BF16 = 0, 1
TTT_PHASE_FWD, TTT_PHASE_REV = 0, 1
DIRS = {"fwd": TTT_FWD, "rev": TTT_REV, "bidir": TTT_BIDIR}

EXPORTED = ["ttt_mlp_workspace_size", "ttt_mlp_forward", "ttt_mlp_status", "ttt_mlp_host_io_workspace_size",
            "ttt_mlp_forward_host", "ttt_mlp_select_kernels", "ttt_last_error", "ttt_launch_count",
            "ttt_kernel_timing", "ttt_kernel_times", "ttt_mlp_forward_noalloc", "ttt_mlp_noalloc_status", "ttt_debug_inject_wait_timeout",
            "ttt_linear_workspace_size", "ttt_linear_forward", "ttt_debug_pipe_segments",
            "ttt_mlp_backward_workspace_size", "ttt_mlp_backward", "ttt_mlp_heads_workspace_size",
            "ttt_mlp_forward_heads", "ttt_seg_attention_workspace_size", "ttt_seg_attention",
            "ttt_block_workspace_size", "ttt_block_forward", "ttt_debug_set_block_front",
            "ttt_linear_host_io_workspace_size", "ttt_linear_forward_host", "ttt_debug_set_backward_ctas"]


class TTTError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {ttt_last_error()}")


class ttt_mlp_desc(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int), ("m", ctypes.c_int),
                ("D", ctypes.c_int), ("per_head_input", ctypes.c_int), ("x_dtype", ctypes.c_int)]


def make_desc(T: int, H: int, d: int, per_head: bool, bf16: bool) -> ttt_mlp_desc:
    return ttt_mlp_desc(T, H, d, 4 * d, H * d, 1 if per_head else 0, TTT_BF16 if bf16 else TTT_F32)


def library_path() -> str:
    return _LIB_PATH


def lib():
    """Load libtttmlp.so (raises if it is missing: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with python -m test_rnn_layer_b200.build")
        L = ctypes.CDLL(_LIB_PATH)
        vp, sz, i, f = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
        dp = ctypes.POINTER(ttt_mlp_desc)
        L.ttt_mlp_workspace_size.restype = sz
        L.ttt_mlp_workspace_size.argtypes = [dp, i, i]
        L.ttt_mlp_host_io_workspace_size.restype = sz
        L.ttt_mlp_host_io_workspace_size.argtypes = [dp, i, i]
        L.ttt_mlp_forward.restype = i
        L.ttt_mlp_forward.argtypes = [dp, vp, vp, vp, vp, vp, vp, f, i, i, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.ttt_mlp_forward_host.restype = i
        L.ttt_mlp_forward_host.argtypes = [dp, vp, vp, vp, vp, vp, vp, f, i, i, vp, vp, vp, vp, sz, vp]
        L.ttt_mlp_forward_noalloc.restype = i
        L.ttt_mlp_forward_noalloc.argtypes = [dp, vp, vp, vp, vp, vp, vp, f, i, i, vp, vp, vp, vp, vp, vp, vp]
        L.ttt_mlp_backward_workspace_size.restype = sz
        L.ttt_mlp_backward_workspace_size.argtypes = [dp, i, i]
        L.ttt_mlp_backward.restype = i
        L.ttt_mlp_backward.argtypes = [dp, vp, vp, vp, vp, vp, vp, f, i, i, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                       vp, sz, vp]
        L.ttt_mlp_heads_workspace_size.restype = sz
        L.ttt_mlp_heads_workspace_size.argtypes = [dp, i, i]
        L.ttt_mlp_forward_heads.restype = i
        L.ttt_mlp_forward_heads.argtypes = [dp, i, i, i, vp, vp, vp, vp, vp, vp, f, i, vp, vp, vp, vp, vp, sz, vp]
        L.ttt_seg_attention_workspace_size.restype = sz
        L.ttt_seg_attention_workspace_size.argtypes = []
        L.ttt_seg_attention.restype = i
        L.ttt_seg_attention.argtypes = [i, i, i, i, vp, vp, vp, i, vp, vp, i, i, i, vp, sz, vp]
        L.ttt_block_workspace_size.restype = sz
        L.ttt_block_workspace_size.argtypes = [dp, i]
        L.ttt_block_forward.restype = i
        L.ttt_block_forward.argtypes = [dp, i, vp, vp, vp, i, vp, vp, vp, vp, vp, vp, vp, f, i, vp, vp, vp, vp, sz, vp]
        L.ttt_debug_set_block_front.restype = i
        L.ttt_debug_set_block_front.argtypes = [i]
        L.ttt_debug_set_backward_ctas.restype = i
        L.ttt_debug_set_backward_ctas.argtypes = [i]
        L.ttt_mlp_noalloc_status.restype = i
        L.ttt_mlp_noalloc_status.argtypes = [vp]
        L.ttt_linear_workspace_size.restype = sz
        L.ttt_linear_workspace_size.argtypes = [dp, i, i]
        L.ttt_linear_host_io_workspace_size.restype = sz
        L.ttt_linear_host_io_workspace_size.argtypes = [dp, i, i]
        L.ttt_linear_forward_host.restype = i
        L.ttt_linear_forward_host.argtypes = [dp, vp, vp, vp, vp, vp, f, i, i, vp, vp, vp, vp, sz, vp]
        L.ttt_linear_forward.restype = i
        L.ttt_linear_forward.argtypes = [dp, vp, vp, vp, vp, vp, f, i, i, vp, vp, vp, vp, vp, vp, sz, vp]
        L.ttt_mlp_status.restype = i
        L.ttt_mlp_status.argtypes = [vp, vp]
        L.ttt_mlp_select_kernels.restype = i
        L.ttt_mlp_select_kernels.argtypes = [i, i]
        L.ttt_last_error.restype = ctypes.c_char_p
        L.ttt_last_error.argtypes = []
        L.ttt_launch_count.restype = ctypes.c_uint64
        L.ttt_launch_count.argtypes = []
        L.ttt_debug_pipe_segments.restype = i
        L.ttt_debug_pipe_segments.argtypes = [i, ctypes.POINTER(ctypes.c_int), i]
        L.ttt_debug_inject_wait_timeout.restype = i
        L.ttt_debug_inject_wait_timeout.argtypes = [i]
        L.ttt_kernel_timing.restype = i
        L.ttt_kernel_timing.argtypes = [i]
        L.ttt_kernel_times.restype = i
        L.ttt_kernel_times.argtypes = [i, ctypes.c_char_p, sz, ctypes.POINTER(ctypes.c_double),
                                       ctypes.POINTER(ctypes.c_uint64)]
        _lib = L
    return _lib


def _p(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return ctypes.c_void_p(x.data_ptr())
    return ctypes.c_void_p(int(x))


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


# ------------------------------------------------------------------ the C entry points
def ttt_last_error() -> str:
    return lib().ttt_last_error().decode()


def ttt_launch_count() -> int:
    return int(lib().ttt_launch_count())


def ttt_debug_inject_wait_timeout(enable: bool) -> int:
    return int(lib().ttt_debug_inject_wait_timeout(1 if enable else 0))


def ttt_debug_pipe_segments(nchunks: int, max_segments: int = 256) -> list:
    """Chunk segments [(begin, end), ...] of the pipelined full-width layer (tests)."""
    buf = (ctypes.c_int * (2 * max_segments))()
    n = int(lib().ttt_debug_pipe_segments(int(nchunks), buf, max_segments))
    if n < 0:
        raise TTTError(TTT_ERR_INVALID_ARG, "ttt_debug_pipe_segments")
    return [(buf[2 * k], buf[2 * k + 1]) for k in range(min(n, max_segments))]


def ttt_kernel_timing(enable: bool) -> int:
    return int(lib().ttt_kernel_timing(1 if enable else 0))


def ttt_kernel_times(max_kernels: int = 32) -> dict:
    """{kernel name: (total ms, launches)} recorded since ttt_kernel_timing(True)."""
    names = ctypes.create_string_buffer(4096)
    ms = (ctypes.c_double * max_kernels)()
    cnt = (ctypes.c_uint64 * max_kernels)()
    n = lib().ttt_kernel_times(max_kernels, names, 4096, ms, cnt)
    if n < 0:
        raise TTTError(TTT_ERR_CUDA, "ttt_kernel_times")
    keys = names.value.decode().split("\n")[:min(n, max_kernels)]
    return {k: (ms[i], int(cnt[i])) for i, k in enumerate(keys)}


def ttt_mlp_workspace_size(desc: ttt_mlp_desc, b: int, direction: int) -> int:
    return int(lib().ttt_mlp_workspace_size(ctypes.byref(desc), b, direction))


def ttt_mlp_host_io_workspace_size(desc: ttt_mlp_desc, b: int, direction: int) -> int:
    return int(lib().ttt_mlp_host_io_workspace_size(ctypes.byref(desc), b, direction))


def ttt_mlp_select_kernels(scan_impl: int, proj_impl: int) -> int:
    return int(lib().ttt_mlp_select_kernels(scan_impl, proj_impl))


def ttt_mlp_forward(desc, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, direction, alpha_f, alpha_r, Y,
                    Z_out, W1_T, W2_T, workspace, workspace_bytes, stream=None) -> int:
    return int(lib().ttt_mlp_forward(ctypes.byref(desc), _p(X), _p(theta_q), _p(theta_k), _p(theta_v), _p(W1_0),
                                     _p(W2_0), float(eta), int(b), int(direction), _p(alpha_f), _p(alpha_r), _p(Y),
                                     _p(Z_out), _p(W1_T), _p(W2_T), _p(workspace), int(workspace_bytes),
                                     _stream(stream)))


def ttt_mlp_forward_host(desc, X_host, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, direction, alpha_f, alpha_r,
                         Y_host, workspace, workspace_bytes, stream=None) -> int:
    return int(lib().ttt_mlp_forward_host(ctypes.byref(desc), _p(X_host), _p(theta_q), _p(theta_k), _p(theta_v),
                                          _p(W1_0), _p(W2_0), float(eta), int(b), int(direction), _p(alpha_f),
                                          _p(alpha_r), _p(Y_host), _p(workspace), int(workspace_bytes),
                                          _stream(stream)))


def ttt_mlp_forward_noalloc(desc, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, direction, alpha_f, alpha_r,
                            Y, Z_out, W1_T, W2_T, stream=None) -> int:
    """ttt_mlp_forward without a workspace argument: for callers that cannot
    allocate device memory (the library uses its own fixed 32 MiB scratch)."""
    return int(lib().ttt_mlp_forward_noalloc(ctypes.byref(desc), _p(X), _p(theta_q), _p(theta_k), _p(theta_v),
                                             _p(W1_0), _p(W2_0), float(eta), int(b), int(direction), _p(alpha_f),
                                             _p(alpha_r), _p(Y), _p(Z_out), _p(W1_T), _p(W2_T), _stream(stream)))


def ttt_mlp_backward_workspace_size(desc: ttt_mlp_desc, b: int, direction: int) -> int:
    return int(lib().ttt_mlp_backward_workspace_size(ctypes.byref(desc), b, direction))


def ttt_mlp_backward(desc, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, direction, alpha_f, alpha_r, dY, dX,
                     dtheta_q, dtheta_k, dtheta_v, dW1_0, dW2_0, dalpha_f, dalpha_r, workspace, workspace_bytes,
                     stream=None) -> int:
    return int(lib().ttt_mlp_backward(ctypes.byref(desc), _p(X), _p(theta_q), _p(theta_k), _p(theta_v), _p(W1_0),
                                      _p(W2_0), float(eta), int(b), int(direction), _p(alpha_f), _p(alpha_r), _p(dY),
                                      _p(dX), _p(dtheta_q), _p(dtheta_k), _p(dtheta_v), _p(dW1_0), _p(dW2_0),
                                      _p(dalpha_f), _p(dalpha_r), _p(workspace), int(workspace_bytes),
                                      _stream(stream)))


def layer_backward(X, theta_q, theta_k, theta_v, W1_0, W2_0, eta: float, b: int, dirs: str, alpha_f, alpha_r, dY,
                   per_head: bool = True, workspace: torch.Tensor | None = None, check_status: bool = True,
                   stream=None) -> dict:
    """Allocate gradient outputs (fp32, on X's device) and call ttt_mlp_backward once."""
    dev = X.device
    if per_head:
        H, T, d = X.shape
    else:
        T, _ = X.shape
        H, d = W1_0.shape[0], W1_0.shape[2]
    desc = make_desc(T, H, d, per_head, X.dtype == torch.bfloat16)
    direction = DIRS[dirs]
    if workspace is None:
        n = ttt_mlp_backward_workspace_size(desc, b, direction)
        if n == 0:
            raise TTTError(TTT_ERR_INVALID_ARG, "backward workspace size")
        workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"dX": torch.empty(X.shape, **f32), "dtheta_q": torch.empty(theta_q.shape, **f32),
           "dtheta_k": torch.empty(theta_k.shape, **f32), "dtheta_v": torch.empty(theta_v.shape, **f32),
           "dW1_0": torch.empty(W1_0.shape, **f32), "dW2_0": torch.empty(W2_0.shape, **f32),
           "dalpha_f": torch.zeros(alpha_f.shape, **f32), "dalpha_r": torch.zeros(alpha_r.shape, **f32)}
    st = ttt_mlp_backward(desc, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, direction, alpha_f, alpha_r,
                          dY.float().contiguous(), out["dX"], out["dtheta_q"], out["dtheta_k"], out["dtheta_v"],
                          out["dW1_0"], out["dW2_0"], out["dalpha_f"], out["dalpha_r"], workspace, workspace.numel(),
                          stream)
    check(st, "ttt_mlp_backward")
    if check_status:
        check(ttt_mlp_status(workspace, stream), "ttt_mlp_status")
    out["workspace"] = workspace
    return out


def ttt_mlp_heads_workspace_size(desc: ttt_mlp_desc, hn: int, b: int) -> int:
    return int(lib().ttt_mlp_heads_workspace_size(ctypes.byref(desc), hn, b))


def ttt_mlp_forward_heads(desc, h0, hn, phase, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, alpha, delta_all,
                          Xp, delta_or_y, workspace, workspace_bytes, stream=None) -> int:
    return int(lib().ttt_mlp_forward_heads(ctypes.byref(desc), h0, hn, phase, _p(X), _p(theta_q), _p(theta_k),
                                           _p(theta_v), _p(W1_0), _p(W2_0), float(eta), b, _p(alpha),
                                           _p(delta_all), _p(Xp), _p(delta_or_y), _p(workspace), workspace_bytes,
                                           _stream(stream)))


def ttt_seg_attention_workspace_size() -> int:
    return int(lib().ttt_seg_attention_workspace_size())


def ttt_seg_attention(T, H, d, L, Q, K, V, ld_qkv, Xres, Out, ld_out, row0, row1, workspace, workspace_bytes,
                      stream=None) -> int:
    return int(lib().ttt_seg_attention(T, H, d, L, _p(Q), _p(K), _p(V), ld_qkv, _p(Xres), _p(Out), ld_out, row0,
                                       row1, _p(workspace), workspace_bytes, _stream(stream)))


def ttt_block_workspace_size(desc: ttt_mlp_desc, b: int) -> int:
    return int(lib().ttt_block_workspace_size(ctypes.byref(desc), b))


def ttt_block_forward(desc, seg_len, Qa, Ka, Va, ld_qkv, Xres, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b,
                      alpha_f, alpha_r, Y, workspace, workspace_bytes, stream=None) -> int:
    return int(lib().ttt_block_forward(ctypes.byref(desc), seg_len, _p(Qa), _p(Ka), _p(Va), ld_qkv, _p(Xres), _p(X),
                                       _p(theta_q), _p(theta_k), _p(theta_v), _p(W1_0), _p(W2_0), float(eta), b,
                                       _p(alpha_f), _p(alpha_r), _p(Y), _p(workspace), workspace_bytes,
                                       _stream(stream)))


def ttt_debug_set_block_front(percent: int) -> int:
    return int(lib().ttt_debug_set_block_front(percent))


def ttt_debug_set_backward_ctas(ctas: int) -> int:
    return int(lib().ttt_debug_set_backward_ctas(ctas))


def ttt_mlp_noalloc_status(stream=None) -> int:
    """ttt_mlp_status for the no-alloc entry point (its status word lives in
    the library's fixed scratch array on the current device)."""
    return int(lib().ttt_mlp_noalloc_status(_stream(stream)))


def ttt_linear_workspace_size(desc: ttt_mlp_desc, b: int, direction: int) -> int:
    return int(lib().ttt_linear_workspace_size(ctypes.byref(desc), b, direction))


def ttt_linear_host_io_workspace_size(desc: ttt_mlp_desc, b: int, direction: int) -> int:
    return int(lib().ttt_linear_host_io_workspace_size(ctypes.byref(desc), b, direction))


def ttt_linear_forward_host(desc, X_host, theta_q, theta_k, theta_v, W_0, eta, b, direction, alpha_f, alpha_r,
                            Y_host, workspace, workspace_bytes, stream=None) -> int:
    return int(lib().ttt_linear_forward_host(ctypes.byref(desc), _p(X_host), _p(theta_q), _p(theta_k), _p(theta_v),
                                             _p(W_0), float(eta), b, direction, _p(alpha_f), _p(alpha_r),
                                             _p(Y_host), _p(workspace), workspace_bytes, _stream(stream)))


def ttt_linear_forward(desc, X, theta_q, theta_k, theta_v, W_0, eta, b, direction, alpha_f, alpha_r, Y, Z_out,
                       W_T, workspace, workspace_bytes, stream=None) -> int:
    return int(lib().ttt_linear_forward(ctypes.byref(desc), _p(X), _p(theta_q), _p(theta_k), _p(theta_v), _p(W_0),
                                        float(eta), int(b), int(direction), _p(alpha_f), _p(alpha_r), _p(Y),
                                        _p(Z_out), _p(W_T), _p(workspace), int(workspace_bytes), _stream(stream)))


def ttt_mlp_status(workspace, stream=None) -> int:
    return int(lib().ttt_mlp_status(_p(workspace), _stream(stream)))


# ------------------------------------------------------------------ tensor-level convenience
def check(status: int, where: str) -> None:
    if status != TTT_OK:
        raise TTTError(status, where)


def alloc_workspace(desc: ttt_mlp_desc, b: int, direction: int, device, host_io: bool = False) -> torch.Tensor:
    n = (ttt_mlp_host_io_workspace_size if host_io else ttt_mlp_workspace_size)(desc, b, direction)
    if n == 0:
        raise TTTError(TTT_ERR_INVALID_ARG, "workspace size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def layer_forward(X, theta_q, theta_k, theta_v, W1_0, W2_0, eta: float, b: int, dirs: str, alpha_f=None,
                  alpha_r=None, per_head: bool = True, want_z: bool = False, want_state: bool = False,
                  workspace: torch.Tensor | None = None, check_status: bool = True, stream=None) -> dict:
    """Allocate outputs (torch, on X's device) and call ttt_mlp_forward once."""
    dev = X.device
    if per_head:
        H, T, d = X.shape
    else:
        T, D = X.shape
        d = W1_0.shape[2]
        H = W1_0.shape[0]
    desc = make_desc(T, H, d, per_head, X.dtype == torch.bfloat16)
    direction = DIRS[dirs]
    nd = 2 if dirs == "bidir" else 1
    ws = workspace if workspace is not None else alloc_workspace(desc, b, direction, dev)
    Y = torch.empty_like(X)
    Z = torch.empty((nd,) + tuple(X.shape), dtype=torch.float32, device=dev) if want_z else None
    W1T = torch.empty((nd,) + tuple(W1_0.shape), dtype=torch.float32, device=dev) if want_state else None
    W2T = torch.empty((nd,) + tuple(W2_0.shape), dtype=torch.float32, device=dev) if want_state else None
    st = ttt_mlp_forward(desc, X, theta_q, theta_k, theta_v, W1_0, W2_0, eta, b, direction, alpha_f, alpha_r, Y, Z,
                         W1T, W2T, ws, ws.numel(), stream)
    check(st, "ttt_mlp_forward")
    out = {"Y": Y, "Z": Z, "W1_T": W1T, "W2_T": W2T, "workspace": ws}
    if check_status:
        st = ttt_mlp_status(ws, stream)
        out["status"] = st
        check(st, "ttt_mlp_status")
    return out


def linear_layer_forward(X, theta_q, theta_k, theta_v, W_0, eta: float, b: int, dirs: str, alpha_f=None,
                         alpha_r=None, per_head: bool = True, want_z: bool = False, want_state: bool = False,
                         workspace: torch.Tensor | None = None, check_status: bool = True, stream=None) -> dict:
    """Allocate outputs (torch, on X's device) and call ttt_linear_forward once."""
    dev = X.device
    if per_head:
        H, T, d = X.shape
    else:
        T, _ = X.shape
        H, d = W_0.shape[0], W_0.shape[2]
    desc = make_desc(T, H, d, per_head, X.dtype == torch.bfloat16)
    direction = DIRS[dirs]
    nd = 2 if dirs == "bidir" else 1
    if workspace is None:
        n = ttt_linear_workspace_size(desc, b, direction)
        if n == 0:
            raise TTTError(TTT_ERR_INVALID_ARG, "workspace size")
        workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    Y = torch.empty_like(X)
    Z = torch.empty((nd,) + tuple(X.shape), dtype=torch.float32, device=dev) if want_z else None
    WT = torch.empty((nd,) + tuple(W_0.shape), dtype=torch.float32, device=dev) if want_state else None
    st = ttt_linear_forward(desc, X, theta_q, theta_k, theta_v, W_0, eta, b, direction, alpha_f, alpha_r, Y, Z, WT,
                            workspace, workspace.numel(), stream)
    check(st, "ttt_linear_forward")
    out = {"Y": Y, "Z": Z, "W_T": WT, "workspace": workspace}
    if check_status:
        st = ttt_mlp_status(workspace, stream)
        out["status"] = st
        check(st, "ttt_mlp_status")
    return out
