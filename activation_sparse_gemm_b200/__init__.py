"""RT-Lynx activation-sparse linear layer for NVIDIA B200 (sm_100a).

Python binding of ``librtlynx.so`` (argument marshalling only; every step of
the layer runs in the library's CUDA kernels).  The C ABI is declared in
``include/rtlynx.h``; the functions below carry the same names and take
device pointers as ints, or torch tensors (their ``data_ptr()``), and a CUDA
stream handle (int) or a ``torch.cuda.Stream``.

    Y = S(X) W^T + X (L_A L_B)^T        mode = MODE_SPARSE
    Y = X W^T                           mode = MODE_DENSE_SKIP
    H = GELU(up(X)), Y = down(H)        rtlynx_mlp_block (two such layers)

(RT-Lynx summary page, four-step pipeline paragraph, steps 1-3.)

The library is built in-tree with ``python -m activation_sparse_gemm_b200.build``.
There is no fallback: if the library is missing every call raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "librtlynx.so")

MODE_SPARSE = 0
MODE_DENSE_SKIP = 1

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_CUDA = 3
ERR_OOM = 4
ERR_DEVICE_TIMEOUT = 5

# Every symbol include/rtlynx.h declares.
ABI_SYMBOLS = (
    "rtlynx_linear", "rtlynx_workspace_size", "rtlynx_linear_ws", "rtlynx_linear_ws_events",
    "rtlynx_workspace_layout",
    "rtlynx_sparsify_debug", "rtlynx_linear_host", "rtlynx_mlp_block", "rtlynx_linear_noalloc",
    "rtlynx_kernel_launches", "rtlynx_schedule_info",
    "rtlynx_quantize_weight_fp8", "rtlynx_linear_fp8", "rtlynx_linear_fp8_events", "rtlynx_sparsify_fp8_debug",
    "rtlynx_wait_selftest", "rtlynx_stream_status", "rtlynx_status_string", "rtlynx_release",
)

NOALLOC_MAX_BYTES = 32 << 20

_lib = None


class RtlynxError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {rtlynx_status_string(status)} (status {status})")


class WsLayout(ctypes.Structure):
    _fields_ = [("M_pad", ctypes.c_int64), ("Kc_pad", ctypes.c_int64), ("k_chunks", ctypes.c_int64),
                ("R_pad", ctypes.c_int64), ("vals", ctypes.c_size_t), ("meta", ctypes.c_size_t),
                ("s", ctypes.c_size_t), ("T", ctypes.c_size_t), ("total", ctypes.c_size_t)]


class Schedule(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "prologue_ctas", "prologue_tiles", "prologue_max_segs", "row_blocks", "k_tiles_per_block",
        "gemm_pairs", "gemm_tiles", "tail_full", "tail_split", "tail_units", "k_stages", "lora_stages",
        "small_path")]


def lib() -> ctypes.CDLL:
    """Loads librtlynx.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m activation_sparse_gemm_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        p, i64, i = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.rtlynx_linear.argtypes = [p, p, p, p, p, i64, i64, i64, i64, i, p]
        L.rtlynx_linear.restype = i
        L.rtlynx_workspace_size.argtypes = [i64, i64, i64, i64, i]
        L.rtlynx_workspace_size.restype = ctypes.c_size_t
        L.rtlynx_linear_ws.argtypes = [p, p, p, p, p, i64, i64, i64, i64, i, p, ctypes.c_size_t, p]
        L.rtlynx_linear_ws.restype = i
        L.rtlynx_linear_ws_events.argtypes = [p, p, p, p, p, i64, i64, i64, i64, i, p, ctypes.c_size_t, p, p, p,
                                               p]
        L.rtlynx_linear_ws_events.restype = i
        L.rtlynx_workspace_layout.argtypes = [i64, i64, i64, i64, ctypes.POINTER(WsLayout)]
        L.rtlynx_workspace_layout.restype = i
        L.rtlynx_sparsify_debug.argtypes = [p, p, i64, i64, i64, p, p, p, p, p]
        L.rtlynx_sparsify_debug.restype = i
        L.rtlynx_linear_host.argtypes = [p, p, p, p, p, i64, i64, i64, i64, i, p, p, p]
        L.rtlynx_linear_host.restype = i
        L.rtlynx_mlp_block.argtypes = [p, p, p, p, p, p, p, p, p, i64, i64, i64, i64, i, i, p]
        L.rtlynx_mlp_block.restype = i
        L.rtlynx_linear_noalloc.argtypes = [p, p, p, p, p, i64, i64, i64, i64, i, p, p]
        L.rtlynx_linear_noalloc.restype = i
        L.rtlynx_quantize_weight_fp8.argtypes = [p, p, p, p, p, i64, i64, i64, p]
        L.rtlynx_quantize_weight_fp8.restype = i
        L.rtlynx_linear_fp8.argtypes = [p, p, p, p, p, p, i64, i64, i64, i64, p]
        L.rtlynx_linear_fp8.restype = i
        L.rtlynx_linear_fp8_events.argtypes = [p, p, p, p, p, p, i64, i64, i64, i64, p, p, p, p]
        L.rtlynx_linear_fp8_events.restype = i
        L.rtlynx_sparsify_fp8_debug.argtypes = [p, i64, i64, p, p, p, p]
        L.rtlynx_sparsify_fp8_debug.restype = i
        L.rtlynx_kernel_launches.argtypes = [i64, i64, i64, i64, i]
        L.rtlynx_kernel_launches.restype = i
        L.rtlynx_schedule_info.argtypes = [i64, i64, i64, i64, i, ctypes.POINTER(Schedule)]
        L.rtlynx_schedule_info.restype = i
        L.rtlynx_wait_selftest.argtypes = [i64, p]
        L.rtlynx_wait_selftest.restype = i
        L.rtlynx_stream_status.argtypes = [p]
        L.rtlynx_stream_status.restype = i
        L.rtlynx_status_string.argtypes = [i]
        L.rtlynx_status_string.restype = ctypes.c_char_p
        L.rtlynx_release.argtypes = []
        L.rtlynx_release.restype = None
        _lib = L
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _stream(s):
    if s is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)


def _check(status: int, what: str) -> int:
    if status != OK:
        raise RtlynxError(status, what)
    return status


# ------------------------------------------------------------------ the ABI, one to one
def rtlynx_linear(X, W, L_A, L_B, Y, M, D_in, D_out, R, mode, stream=None) -> int:
    return _check(lib().rtlynx_linear(_ptr(X), _ptr(W), _ptr(L_A), _ptr(L_B), _ptr(Y), M, D_in, D_out, R,
                                      mode, _stream(stream)), "rtlynx_linear")


def rtlynx_mlp_block(X, W_up, LA_up, LB_up, W_down, LA_down, LB_down, H, Y, M, D, D_ff, R, mode_up=MODE_SPARSE,
                     mode_down=MODE_SPARSE, stream=None) -> int:
    """H = GELU(layer_up(X)) [M, D_ff], Y = layer_down(H) [M, D]; see include/rtlynx.h."""
    return _check(lib().rtlynx_mlp_block(_ptr(X), _ptr(W_up), _ptr(LA_up), _ptr(LB_up), _ptr(W_down), _ptr(LA_down),
                                         _ptr(LB_down), _ptr(H), _ptr(Y), M, D, D_ff, R, mode_up, mode_down,
                                         _stream(stream)), "rtlynx_mlp_block")


def rtlynx_workspace_size(M, D_in, D_out, R, mode) -> int:
    return int(lib().rtlynx_workspace_size(M, D_in, D_out, R, mode))


def rtlynx_linear_ws(X, W, L_A, L_B, Y, M, D_in, D_out, R, mode, workspace, ws_bytes, stream=None) -> int:
    return _check(lib().rtlynx_linear_ws(_ptr(X), _ptr(W), _ptr(L_A), _ptr(L_B), _ptr(Y), M, D_in, D_out, R,
                                         mode, _ptr(workspace), ws_bytes, _stream(stream)), "rtlynx_linear_ws")


def _event(ev):
    if ev is None or isinstance(ev, int):
        return ev
    return int(ev.cuda_event)


def rtlynx_linear_ws_events(X, W, L_A, L_B, Y, M, D_in, D_out, R, mode, workspace, ws_bytes, ev_start, ev_mid,
                            ev_end, stream=None) -> int:
    """Events may be raw cudaEvent_t ints or torch.cuda.Event objects that were recorded once already."""
    return _check(lib().rtlynx_linear_ws_events(_ptr(X), _ptr(W), _ptr(L_A), _ptr(L_B), _ptr(Y), M, D_in, D_out,
                                                R, mode, _ptr(workspace), ws_bytes, _event(ev_start),
                                                _event(ev_mid), _event(ev_end), _stream(stream)),
                  "rtlynx_linear_ws_events")


def rtlynx_workspace_layout(M, D_in, D_out, R) -> WsLayout:
    out = WsLayout()
    _check(lib().rtlynx_workspace_layout(M, D_in, D_out, R, ctypes.byref(out)), "rtlynx_workspace_layout")
    return out


def rtlynx_sparsify_debug(X, L_B, M, D_in, R, vals, meta, s, T, stream=None) -> int:
    return _check(lib().rtlynx_sparsify_debug(_ptr(X), _ptr(L_B), M, D_in, R, _ptr(vals), _ptr(meta), _ptr(s),
                                              _ptr(T), _stream(stream)), "rtlynx_sparsify_debug")


def rtlynx_linear_host(X_host, W, L_A, L_B, Y_host, M, D_in, D_out, R, mode, X_dev, Y_dev, stream=None) -> int:
    return _check(lib().rtlynx_linear_host(_ptr(X_host), _ptr(W), _ptr(L_A), _ptr(L_B), _ptr(Y_host), M, D_in,
                                           D_out, R, mode, _ptr(X_dev), _ptr(Y_dev), _stream(stream)),
                  "rtlynx_linear_host")


def rtlynx_linear_noalloc(X, W, L_A, L_B, Y, M, D_in, D_out, R, mode, dev_status=None, stream=None) -> int:
    """rtlynx_linear without any device allocation: for callers that cannot call
    cudaMalloc (their memory belongs to another pool, or the call sits on a path
    that must not synchronize).  The workspace is a static device array of
    NOALLOC_MAX_BYTES shared by all calls on a device; calls that overlap on the
    GPU race on it.  dev_status: optional device int32 that receives the
    device-side timeout code; without it a timeout goes to the library's error
    word, which rtlynx_stream_status reports."""
    return _check(lib().rtlynx_linear_noalloc(_ptr(X), _ptr(W), _ptr(L_A), _ptr(L_B), _ptr(Y), M, D_in, D_out, R,
                                              mode, _ptr(dev_status), _stream(stream)), "rtlynx_linear_noalloc")


def rtlynx_quantize_weight_fp8(W, L_A, W8, qw, L_A8, D_out, D_in, R, stream=None) -> int:
    return _check(lib().rtlynx_quantize_weight_fp8(_ptr(W), _ptr(L_A), _ptr(W8), _ptr(qw), _ptr(L_A8), D_out, D_in,
                                                   R, _stream(stream)), "rtlynx_quantize_weight_fp8")


def rtlynx_linear_fp8(X, W8, qw, L_A8, L_B, Y, M, D_in, D_out, R, stream=None) -> int:
    return _check(lib().rtlynx_linear_fp8(_ptr(X), _ptr(W8), _ptr(qw), _ptr(L_A8), _ptr(L_B), _ptr(Y), M, D_in,
                                          D_out, R, _stream(stream)), "rtlynx_linear_fp8")


def rtlynx_linear_fp8_events(X, W8, qw, L_A8, L_B, Y, M, D_in, D_out, R, ev_start, ev_mid, ev_end,
                             stream=None) -> int:
    """Events are torch.cuda.Event objects (or raw handles), any may be None."""
    def h(e):
        return None if e is None else (e if isinstance(e, int) else int(e.cuda_event))
    return _check(lib().rtlynx_linear_fp8_events(_ptr(X), _ptr(W8), _ptr(qw), _ptr(L_A8), _ptr(L_B), _ptr(Y), M,
                                                 D_in, D_out, R, h(ev_start), h(ev_mid), h(ev_end),
                                                 _stream(stream)), "rtlynx_linear_fp8_events")


def rtlynx_sparsify_fp8_debug(X, M, D_in, codes, meta, qx, stream=None) -> int:
    return _check(lib().rtlynx_sparsify_fp8_debug(_ptr(X), M, D_in, _ptr(codes), _ptr(meta), _ptr(qx),
                                                  _stream(stream)), "rtlynx_sparsify_fp8_debug")


def rtlynx_kernel_launches(M, D_in, D_out, R, mode) -> int:
    return int(lib().rtlynx_kernel_launches(M, D_in, D_out, R, mode))


def rtlynx_schedule_info(M, D_in, D_out, R, num_sms) -> Schedule:
    """The work split of a sparse-mode call on a GPU with num_sms SMs (host only)."""
    out = Schedule()
    _check(lib().rtlynx_schedule_info(M, D_in, D_out, R, num_sms, ctypes.byref(out)), "rtlynx_schedule_info")
    return out


def rtlynx_wait_selftest(limit_ns, stream=None) -> int:
    return _check(lib().rtlynx_wait_selftest(int(limit_ns), _stream(stream)), "rtlynx_wait_selftest")


def rtlynx_stream_status(stream=None) -> int:
    return int(lib().rtlynx_stream_status(_stream(stream)))


def rtlynx_status_string(status: int) -> str:
    try:
        return lib().rtlynx_status_string(int(status)).decode()
    except RuntimeError:
        return f"status {status}"


def rtlynx_release() -> None:
    lib().rtlynx_release()


# ------------------------------------------------------------------ torch convenience (marshalling only)
def linear(X, W, L_A=None, L_B=None, mode: int = MODE_SPARSE, out=None, stream=None):
    """Y for torch bf16 CUDA tensors X [M,D_in], W [D_out,D_in], L_A [D_out,R], L_B [R,D_in]."""
    import torch
    M, D_in = X.shape
    D_out = W.shape[0]
    R = 0 if (L_A is None or L_B is None or mode == MODE_DENSE_SKIP) else L_B.shape[0]
    for t in (X, W, L_A, L_B):
        if t is not None and (t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous()):
            raise ValueError("inputs must be contiguous bf16 CUDA tensors")
    Y = out if out is not None else torch.empty((M, D_out), dtype=torch.bfloat16, device=X.device)
    rtlynx_linear(X, W, L_A if R else None, L_B if R else None, Y, M, D_in, D_out, R, mode, stream)
    return Y
