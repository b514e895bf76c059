"""CPU oracle for the RT-Lynx activation-sparse linear layer (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA product path never does.

The arithmetic lives in ``rtlynx_oracle.c`` (plain C, double precision, plain
triple-loop GEMMs, OpenMP over tokens).  It follows the four-step pipeline
paragraph of the RT-Lynx summary page (paper.rainbus.top, arXiv 2605.26632),
steps 1-3: Top-K 2-of-4 mask, norm-compensating scale s, LoRA branch on the
dense X, and the dense path for skipped layers; plus the feed-forward block of
two such layers joined by GELU (erf form), and the layer's FP8 form (E4M3
codes for W per output channel and for S(X) per token; the reading is in the
C source).  This module only compiles the
C file with gcc and marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rtlynx_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lib = None

MODE_SPARSE = 0
MODE_DENSE_SKIP = 1


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle C source into a shared library (gcc, OpenMP)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns as numpy uint16")
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """ctypes view of one compiled oracle library."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.oracle_sparsify.argtypes = [p, i64, i64, p, p, p]
        lib.oracle_sparsify.restype = ctypes.c_int
        lib.oracle_linear_rows.argtypes = [p, p, p, p, i64, i64, i64, i64, ctypes.c_int, p, i64, p, p]
        lib.oracle_linear_rows.restype = ctypes.c_int
        lib.oracle_bf16_from_double.argtypes = [ctypes.c_double]
        lib.oracle_bf16_from_double.restype = ctypes.c_uint16
        lib.oracle_gelu_bf16.argtypes = [p, i64, p]
        lib.oracle_gelu_bf16.restype = ctypes.c_int
        lib.oracle_gelu.argtypes = [ctypes.c_double]
        lib.oracle_gelu.restype = ctypes.c_double
        lib.oracle_e4m3_from_float.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_from_float.restype = ctypes.c_uint8
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_double.restype = ctypes.c_double
        lib.oracle_quantize_weight_fp8.argtypes = [p, i64, i64, p, p]
        lib.oracle_quantize_weight_fp8.restype = ctypes.c_int
        lib.oracle_sparsify_fp8.argtypes = [p, i64, i64, p, p, p, p]
        lib.oracle_sparsify_fp8.restype = ctypes.c_int
        lib.oracle_linear_fp8_rows.argtypes = [p, p, p, p, p, i64, i64, i64, i64, p, i64, p]
        lib.oracle_linear_fp8_rows.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        self.lib = lib

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def bf16_round(self, v: float) -> int:
        """bf16 bits of the double v, rounded to nearest, ties to even."""
        return int(self.lib.oracle_bf16_from_double(float(v)))

    def sparsify(self, X: np.ndarray):
        """Step 1 per token: (meta [M,K/4] uint8, vals [M,K/2] bf16 bits, s [M] float32)."""
        X = _u16(X)
        M, K = X.shape
        meta = np.empty((M, K // 4), np.uint8)
        vals = np.empty((M, K // 2), np.uint16)
        s = np.empty((M,), np.float32)
        rc = self.lib.oracle_sparsify(_ptr(X), M, K, _ptr(meta), _ptr(vals), _ptr(s))
        if rc:
            raise ValueError("oracle_sparsify rejected its arguments")
        return meta, vals, s

    def linear(self, X, W, L_A=None, L_B=None, mode: int = MODE_SPARSE, rows=None, want_T: bool = False):
        """Y (float64) for the listed rows (all rows when rows is None); also T when want_T."""
        X = _u16(X)
        W = _u16(W)
        M, K = X.shape
        N = W.shape[0]
        if W.shape[1] != K:
            raise ValueError("W must be [D_out, D_in]")
        R = 0
        if L_A is not None and L_B is not None:
            L_A = _u16(L_A)
            L_B = _u16(L_B)
            R = L_B.shape[0]
            if L_A.shape != (N, R) or L_B.shape != (R, K):
                raise ValueError("L_A must be [D_out,R] and L_B [R,D_in]")
        else:
            L_A = L_B = None
        if rows is None:
            rows_arr = None
            nrows = M
        else:
            rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
            nrows = rows_arr.shape[0]
        Y = np.empty((nrows, N), np.float64)
        T = np.empty((nrows, max(R, 1)), np.float64) if want_T else None
        rc = self.lib.oracle_linear_rows(_ptr(X), _ptr(W), _ptr(L_A), _ptr(L_B), M, K, N, R, int(mode),
                                         _ptr(rows_arr), nrows, _ptr(Y), _ptr(T))
        if rc:
            raise ValueError("oracle_linear_rows rejected its arguments")
        if want_T:
            return Y, T[:, :R]
        return Y


    def gelu(self, y: float) -> float:
        """GELU (erf form) of one double, in double."""
        return float(self.lib.oracle_gelu(float(y)))

    def gelu_bf16(self, Y: np.ndarray) -> np.ndarray:
        """bf16 bits of GELU(Y) (erf form, double, one rounding), same shape as Y."""
        Y = np.ascontiguousarray(Y, dtype=np.float64)
        H = np.empty(Y.shape, np.uint16)
        if self.lib.oracle_gelu_bf16(_ptr(Y), Y.size, _ptr(H)):
            raise ValueError("oracle_gelu_bf16 rejected its arguments")
        return H

    def mlp_block(self, X, W_up, LA_up, LB_up, W_down, LA_down, LB_down, mode_up: int = MODE_SPARSE,
                  mode_down: int = MODE_SPARSE, rows=None):
        """The DiT feed-forward block of two layers: H = bf16(GELU(layer_up(X))) and
        Y = layer_down(H), for the listed tokens (all when rows is None; tokens are
        independent).  Returns (Y_up float64, H bf16 bits, Y float64)."""
        Y_up = self.linear(X, W_up, LA_up, LB_up, mode=mode_up, rows=rows)
        H = self.gelu_bf16(Y_up)
        Y = self.linear(H, W_down, LA_down, LB_down, mode=mode_down)
        return Y_up, H, Y

    # ------------------------------------------------------------------ FP8 form
    def e4m3(self, v: float) -> int:
        """E4M3 code of the float32 value v (nearest, ties to even; saturates at 448)."""
        return int(self.lib.oracle_e4m3_from_float(float(v)))

    def e4m3_value(self, code: int) -> float:
        return float(self.lib.oracle_e4m3_to_double(int(code) & 0xFF))

    def quantize_weight_fp8(self, W):
        """(W8 [N,K] E4M3 codes, q_w [N] float32) for W [N,K] bf16 bits."""
        W = _u16(W)
        N, K = W.shape
        W8 = np.empty((N, K), np.uint8)
        qw = np.empty((N,), np.float32)
        if self.lib.oracle_quantize_weight_fp8(_ptr(W), N, K, _ptr(W8), _ptr(qw)):
            raise ValueError("oracle_quantize_weight_fp8 rejected its arguments")
        return W8, qw

    def sparsify_fp8(self, X):
        """Step 1 in FP8: (meta [M,K/4], x8 [M,K/2] E4M3 codes of the kept entries,
        s [M] float32, q_x [M] float64)."""
        X = _u16(X)
        M, K = X.shape
        meta = np.empty((M, K // 4), np.uint8)
        x8 = np.empty((M, K // 2), np.uint8)
        s = np.empty((M,), np.float32)
        qx = np.empty((M,), np.float64)
        if self.lib.oracle_sparsify_fp8(_ptr(X), M, K, _ptr(meta), _ptr(x8), _ptr(s), _ptr(qx)):
            raise ValueError("oracle_sparsify_fp8 rejected its arguments")
        return meta, x8, s, qx

    def linear_fp8(self, X, W8, qw, L_A=None, L_B=None, rows=None):
        """Y (float64) of the FP8 form for the listed rows (all when rows is None)."""
        X = _u16(X)
        W8 = np.ascontiguousarray(W8, dtype=np.uint8)
        qw = np.ascontiguousarray(qw, dtype=np.float32)
        M, K = X.shape
        N = W8.shape[0]
        R = 0
        if L_A is not None and L_B is not None:
            L_A = _u16(L_A)
            L_B = _u16(L_B)
            R = L_B.shape[0]
        else:
            L_A = L_B = None
        rows_arr = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nrows = M if rows is None else rows_arr.shape[0]
        Y = np.empty((nrows, N), np.float64)
        if self.lib.oracle_linear_fp8_rows(_ptr(X), _ptr(W8), _ptr(qw), _ptr(L_A), _ptr(L_B), M, K, N, R,
                                           _ptr(rows_arr), nrows, _ptr(Y)):
            raise ValueError("oracle_linear_fp8_rows rejected its arguments")
        return Y


def _default() -> Oracle:
    global _lib
    if _lib is None:
        _lib = Oracle(build())
    return _lib


def num_threads() -> int:
    return _default().num_threads()


def bf16_round(v: float) -> int:
    return _default().bf16_round(v)


def sparsify(X):
    return _default().sparsify(X)


def linear(X, W, L_A=None, L_B=None, mode: int = MODE_SPARSE, rows=None, want_T: bool = False):
    return _default().linear(X, W, L_A, L_B, mode=mode, rows=rows, want_T=want_T)


def gelu(y: float) -> float:
    return _default().gelu(y)


def gelu_bf16(Y):
    return _default().gelu_bf16(Y)


def mlp_block(X, W_up, LA_up, LB_up, W_down, LA_down, LB_down, mode_up: int = MODE_SPARSE,
              mode_down: int = MODE_SPARSE, rows=None):
    return _default().mlp_block(X, W_up, LA_up, LB_up, W_down, LA_down, LB_down, mode_up=mode_up,
                                mode_down=mode_down, rows=rows)


def e4m3(v: float) -> int:
    return _default().e4m3(v)


def e4m3_value(code: int) -> float:
    return _default().e4m3_value(code)


def quantize_weight_fp8(W):
    return _default().quantize_weight_fp8(W)


def sparsify_fp8(X):
    return _default().sparsify_fp8(X)


def linear_fp8(X, W8, qw, L_A=None, L_B=None, rows=None):
    return _default().linear_fp8(X, W8, qw, L_A, L_B, rows=rows)


# ------------------------------------------------------------------ LoRA fit (closed form)
def reduced_rank_fit(X: np.ndarray, E: np.ndarray, R: int):
    """Reduced-rank regression: the rank-R C [N, K] minimising ||X C^T - E||_F,
    for X [M, K] of full column rank and E [M, N], all float64.

    Least squares B0 = argmin ||X B - E|| (numpy lstsq), the fit Yhat = X B0,
    its top-R right singular vectors V_R [N, R]; then C^T = B0 V_R V_R^T.
    Returned as the LoRA factors L_A = V_R [N, R] and L_B = (B0 V_R)^T [R, K]
    (C = L_A L_B), with the singular values of Yhat."""
    X = np.asarray(X, np.float64)
    E = np.asarray(E, np.float64)
    B0 = np.linalg.lstsq(X, E, rcond=None)[0]
    _, sig, Vt = np.linalg.svd(X @ B0, full_matrices=False)
    V = Vt[:R].T
    return V, (B0 @ V).T, sig


def lora_fit(X, W, R: int):
    """The LoRA of the RT-Lynx summary page's step 2 fitted in closed form on the
    calibration tokens X (bf16 bits [M, K]): it minimises
    ||X W^T - S(X) W^T - X (L_A L_B)^T||_F^2, whose target is the residual
    E = X W^T - S(X) W^T of the dense layer minus the sparse one (both exact,
    from this oracle).  Returns (L_A float64 [N, R], L_B float64 [R, K], E)."""
    Yd = linear(X, W, mode=MODE_DENSE_SKIP)
    Ys = linear(X, W, mode=MODE_SPARSE)
    E = Yd - Ys
    L_A, L_B, _ = reduced_rank_fit(bf16_to_f64(X), E, R)
    return L_A, L_B, E


def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) to float64, exactly."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
