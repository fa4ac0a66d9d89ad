"""CPU oracle for the SmoothQuant W8A8 path and the LLM.int8() decomposition.

TEST INFRASTRUCTURE ONLY. Tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package; the product package
never does. The arithmetic lives in ``sq_oracle.c`` (plain loops, fp64/int64
where the method has an exact definition, correctly rounded fp32 where a
quantised code is decided). This module only marshals numpy arrays.

Functions whose exact fp32 bits depend on the reduction order convention
(the normalisation sums) are marked "parity unpinned" in ``sq_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (strict IEEE flags)."""
    hdr = os.path.join(_HERE, "sq_oracle.h")
    fresh = os.path.exists(_LIB) and os.path.getmtime(_LIB) >= max(
        os.path.getmtime(_SRC), os.path.getmtime(hdr))
    if force or not fresh:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_i = ctypes.c_int
_f = ctypes.c_float
_d = ctypes.c_double


def _declare(L):
    L.or_col_absmax.argtypes = [_p, _i64, _i64, _i64, _p]
    L.or_smooth_scales.argtypes = [_p, _p, _i64, _d, _p]
    L.or_fold_weight.argtypes = [_p, _i64, _i64, _p, _i, _p]
    L.or_fold_norm.argtypes = [_p, _p, _p, _i64, _i, _p, _p]
    L.or_fold_prev_linear.argtypes = [_p, _i64, _i64, _p, _p, _i, _p, _p]
    L.or_e4m3_round.argtypes = [_f]
    L.or_e4m3_round.restype = _f
    L.or_e4m3_bits.argtypes = [_f]
    L.or_e4m3_bits.restype = ctypes.c_uint8
    L.or_e4m3_value.argtypes = [ctypes.c_uint8]
    L.or_e4m3_value.restype = _d
    L.or_quantize_fp8.argtypes = [_p, _i64, _i64, _i64, _p, _i, _i, _p, _p, _p]
    L.or_gemm_fp8.argtypes = [_p, _p, _i64, _i64, _i64, _i64, _i64, _p]
    L.or_dequant_f64.argtypes = [_p, _i64, _i64, _i64, _p, _i, _p, _i, _p, _p]
    L.or_expf_array.argtypes = [_p, _i64, _p]
    L.or_silu_array.argtypes = [_p, _i64, _p]
    L.or_gelu_array.argtypes = [_p, _i64, _p]
    L.or_act_quant.argtypes = [_p, _i64, _i64, _i64, _i, _i, _p, _p, _p, _p, _p]
    L.or_quantize_weight.argtypes = [_p, _i64, _i64, _i, _p, _p]
    L.or_quantize_act.argtypes = [_p, _i64, _i64, _i64, _p, _i, _p, _p, _p]
    L.or_scale_from_absmax.argtypes = [_p, _i64]
    L.or_scale_from_absmax.restype = _f
    L.or_norm_smooth_quant.argtypes = [_p, _i64, _i64, _i64, _i, _p, _p, _f, _i, _p, _p, _p, _p, _p]
    L.or_norm_f64.argtypes = [_p, _i64, _i64, _i, _p, _p, _d, _p]
    L.or_gemm_i8.argtypes = [_p, _p, _i64, _i64, _i64, _i64, _i64, _p]
    L.or_dequant.argtypes = [_p, _i64, _i64, _i64, _p, _i, _p, _i, _p, _p]
    L.or_round_bf16.argtypes = [_d]
    L.or_round_bf16.restype = ctypes.c_uint16
    L.or_round_fp16.argtypes = [_d]
    L.or_round_fp16.restype = ctypes.c_uint16
    L.or_round_bf16_array.argtypes = [_p, _i64, _p]
    L.or_round_fp16_array.argtypes = [_p, _i64, _p]
    L.or_llmint8_outliers.argtypes = [_p, _i64, _i64, _i64, _f, _d, _p]
    L.or_llmint8_outliers.restype = _i64
    L.or_llmint8_quant_rows.argtypes = [_p, _i64, _i64, _i64, _p, _i64, _p, _p]
    L.or_llmint8_quant_weight.argtypes = [_p, _i64, _i64, _p, _i64, _p, _p]
    L.or_llmint8_combine.argtypes = [_p, _i64, _i64, _i64, _i64, _p, _p, _p, _i64, _p, _p, _i64, _p]


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def f32(a):
    """fp32 image of an array-like (exact for fp16/bf16 sources)."""
    try:
        import torch

        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu", torch.float32).contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return _c(a, np.float32)


# ---------------------------------------------------------------- calibration absmax
def col_absmax(X, running=None):
    X = f32(X)
    M, K = X.shape
    io = np.zeros(K, np.float32) if running is None else _c(running, np.float32).copy()
    lib().or_col_absmax(_ptr(X), M, K, K, _ptr(io))
    return io


# ---------------------------------------------------------------- smoothing factors and folds
def smooth_scales(x, w, alpha):
    x, w = f32(x), f32(w)
    s = np.empty_like(x)
    lib().or_smooth_scales(_ptr(x), _ptr(w), x.size, float(alpha), _ptr(s))
    return s


def fold_weight(W, s, round_f32=True):
    W = _c(f32(W) if round_f32 else W, np.float64)
    s = _c(s, np.float64)
    N, K = W.shape
    out = np.empty_like(W)
    lib().or_fold_weight(_ptr(W), N, K, _ptr(s), int(round_f32), _ptr(out))
    return out.astype(np.float32) if round_f32 else out


def fold_norm(gamma, beta, s, round_f32=True):
    g = _c(gamma, np.float64)
    b = None if beta is None else _c(beta, np.float64)
    s = _c(s, np.float64)
    go = np.empty_like(g)
    bo = None if b is None else np.empty_like(b)
    lib().or_fold_norm(_ptr(g), _ptr(b), _ptr(s), g.size, int(round_f32), _ptr(go), _ptr(bo))
    if round_f32:
        return go.astype(np.float32), (None if bo is None else bo.astype(np.float32))
    return go, bo


# ---------------------------------------------------------------- fold into the previous linear
def fold_prev_linear(W, s, bias=None, round_f32=True):
    """Output channel n of the previous layer (row n, bias_n) divided by s_n."""
    W = _c(f32(W) if round_f32 else W, np.float64)
    s = _c(s, np.float64)
    b = None if bias is None else _c(f32(bias) if round_f32 else bias, np.float64)
    N, K = W.shape
    out = np.empty_like(W)
    bo = None if b is None else np.empty_like(b)
    lib().or_fold_prev_linear(_ptr(W), N, K, _ptr(b), _ptr(s), int(round_f32), _ptr(out), _ptr(bo))
    if round_f32:
        return out.astype(np.float32), (None if bo is None else bo.astype(np.float32))
    return out, bo


# ---------------------------------------------------------------- MLP activation + int8
SWIGLU, RELU, GELU = 0, 1, 2


def expf(x):
    x = f32(np.atleast_1d(x))
    out = np.empty_like(x)
    lib().or_expf_array(_ptr(x), x.size, _ptr(out))
    return out


def silu(x):
    x = f32(np.atleast_1d(x))
    out = np.empty_like(x)
    lib().or_silu_array(_ptr(x), x.size, _ptr(out))
    return out


def gelu(x):
    x = f32(np.atleast_1d(x))
    out = np.empty_like(x)
    lib().or_gelu_array(_ptr(x), x.size, _ptr(out))
    return out


def act_quant(A, act, per_token=True, static_qs=None, quantize=True, absmax=None, want_h=False):
    """SwiGLU (A = [gate | up], [M, 2I]), ReLU or GELU (A = [M, I]) then int8."""
    A = f32(A)
    M, W = A.shape
    I = W // 2 if act == SWIGLU else W
    st = None if static_qs is None else np.array([static_qs], np.float32)
    Xq = np.empty((M, I), np.int8) if quantize else None
    qs = np.empty(M if per_token else 1, np.float32) if quantize else None
    am = None if absmax is None else _c(absmax, np.float32).copy()
    H = np.empty((M, I), np.float32) if want_h else None
    lib().or_act_quant(_ptr(A), M, I, W, int(act), int(per_token), _ptr(st), _ptr(Xq), _ptr(qs), _ptr(am),
                       _ptr(H))
    return {"Xq": Xq, "qs": qs, "absmax": am, "H": H}


# ---------------------------------------------------------------- FP8 variant
def e4m3_round(x):
    return np.float32(lib().or_e4m3_round(float(x)))


def e4m3_bits(v):
    return int(lib().or_e4m3_bits(float(v)))


def e4m3_value(b):
    return float(lib().or_e4m3_value(int(b)))


def quantize_fp8(X, s=None, s_div=False, per_row=True, static_qs=None):
    """E4M3 codes (uint8) and scales of fp32(X) (* s or / s per column)."""
    X = f32(X)
    M, K = X.shape
    sv = None if s is None else f32(s)
    st = None if static_qs is None else np.array([static_qs], np.float32)
    Q = np.empty((M, K), np.uint8)
    qs = np.empty(M if per_row else 1, np.float32)
    lib().or_quantize_fp8(_ptr(X), M, K, K, _ptr(sv), int(s_div), int(per_row), _ptr(st), _ptr(Q), _ptr(qs))
    return Q, qs


def gemm_fp8(A, B, rows=None):
    """fp64 sums of the decoded E4M3 products (rows: optional row subset)."""
    A, B = _c(A, np.uint8), _c(B, np.uint8)
    M, K = A.shape
    N = B.shape[0]
    if rows is None:
        acc = np.empty((M, N), np.float64)
        lib().or_gemm_fp8(_ptr(A), _ptr(B), M, N, K, 0, M, _ptr(acc))
        return acc
    out = np.empty((len(rows), N), np.float64)
    for n, r in enumerate(rows):
        lib().or_gemm_fp8(_ptr(A), _ptr(B), M, N, K, int(r), int(r) + 1, _ptr(out[n:n + 1]))
    return out


def dequant_f64(acc, qs_x, qs_w, bias=None, rows=None):
    acc = _c(acc, np.float64)
    R, N = acc.shape
    qx, qw = f32(qs_x), f32(qs_w)
    if rows is not None:
        qx = f32(np.asarray(qs_x)[list(rows)]) if qx.size > 1 else qx
    b = None if bias is None else f32(bias)
    y = np.empty_like(acc)
    lib().or_dequant_f64(_ptr(acc), 0, R, N, _ptr(qx), int(qx.size > 1), _ptr(qw), int(qw.size > 1), _ptr(b), _ptr(y))
    return y


# ---------------------------------------------------------------- weight quantisation
def quantize_weight(Wp, per_channel=True):
    Wp = f32(Wp)
    N, K = Wp.shape
    Wq = np.empty((N, K), np.int8)
    qs = np.empty(N if per_channel else 1, np.float32)
    lib().or_quantize_weight(_ptr(Wp), N, K, int(per_channel), _ptr(Wq), _ptr(qs))
    return Wq, qs


# ---------------------------------------------------------------- activation quantisation without a norm
def quantize_act(X, s=None, per_token=True, static_qs=None):
    X = f32(X)
    M, K = X.shape
    s = None if s is None else f32(s)
    st = None if static_qs is None else np.array([static_qs], np.float32)
    Xq = np.empty((M, K), np.int8)
    qs = np.empty(M if per_token else 1, np.float32)
    lib().or_quantize_act(_ptr(X), M, K, K, _ptr(s), int(per_token), _ptr(st), _ptr(Xq), _ptr(qs))
    return Xq, qs


def scale_from_absmax(absmax):
    a = f32(absmax).ravel()
    return np.float32(lib().or_scale_from_absmax(_ptr(a), a.size))


# ---------------------------------------------------------------- fused norm + smoothing + int8
LAYERNORM, RMSNORM = 0, 1


def norm_smooth_quant(H, norm, gamma, beta=None, eps=1e-5, per_token=True, static_qs=None,
                      quantize=True, absmax=None, want_v=False):
    H = f32(H)
    M, K = H.shape
    g = f32(gamma)
    b = None if beta is None else f32(beta)
    st = None if static_qs is None else np.array([static_qs], np.float32)
    Xq = np.empty((M, K), np.int8) if quantize else None
    qs = np.empty(M if per_token else 1, np.float32) if quantize else None
    am = None if absmax is None else _c(absmax, np.float32).copy()
    V = np.empty((M, K), np.float32) if want_v else None
    lib().or_norm_smooth_quant(_ptr(H), M, K, K, int(norm), _ptr(g), _ptr(b), float(eps),
                               int(per_token), _ptr(st), _ptr(Xq), _ptr(qs), _ptr(am), _ptr(V))
    return {"Xq": Xq, "qs": qs, "absmax": am, "V": V}


def norm_f64(H, norm, gamma, beta=None, eps=1e-5):
    H = _c(H, np.float64)
    M, K = H.shape
    g = _c(gamma, np.float64)
    b = None if beta is None else _c(beta, np.float64)
    V = np.empty((M, K), np.float64)
    lib().or_norm_f64(_ptr(H), M, K, int(norm), _ptr(g), _ptr(b), float(eps), _ptr(V))
    return V


# ---------------------------------------------------------------- int8 GEMM
def gemm_i8(Xq, Wq, rows=None):
    Xq, Wq = _c(Xq, np.int8), _c(Wq, np.int8)
    M, K = Xq.shape
    N = Wq.shape[0]
    r0, r1 = (0, M) if rows is None else rows
    acc = np.empty((r1 - r0, N), np.int64)
    lib().or_gemm_i8(_ptr(Xq), _ptr(Wq), M, N, K, r0, r1, _ptr(acc))
    return acc


def dequant(acc, qs_x, qs_w, bias=None, rows=None):
    acc = _c(acc, np.int64)
    qs_x, qs_w = _c(qs_x, np.float32).ravel(), _c(qs_w, np.float32).ravel()
    n_rows, N = acc.shape
    r0 = 0 if rows is None else rows[0]
    b = None if bias is None else _c(f32(bias), np.float64)
    y = np.empty((n_rows, N), np.float64)
    # qs_x is the full per-token vector (indexed by absolute row) or one scale
    lib().or_dequant(_ptr(acc), r0, r0 + n_rows, N, _ptr(qs_x), int(qs_x.size > 1), _ptr(qs_w),
                     int(qs_w.size > 1), _ptr(b), _ptr(y))
    return y


def round_bf16_bits(y):
    """Bits of the bf16 nearest to each fp64 value (ties to even)."""
    y = _c(y, np.float64)
    out = np.empty(y.shape, np.uint16)
    lib().or_round_bf16_array(_ptr(y), y.size, _ptr(out))
    return out


def round_fp16_bits(y):
    """Bits of the fp16 nearest to each fp64 value (ties to even)."""
    y = _c(y, np.float64)
    out = np.empty(y.shape, np.uint16)
    lib().or_round_fp16_array(_ptr(y), y.size, _ptr(out))
    return out


# ---------------------------------------------------------------- batched int8 GEMM (attention)
def bmm_i8(A, B, rows=None):
    """Per problem b: the int64 product A[b] B[b]^T (the plain GEMM, problem by
    problem: the batched product is nothing more); rows: a list of rows of
    every A[b] to compute."""
    A, B = _c(A, np.int8), _c(B, np.int8)
    pick = (lambda a: a) if rows is None else (lambda a: np.ascontiguousarray(a[list(rows)]))
    return np.stack([gemm_i8(pick(A[i]), B[i]) for i in range(A.shape[0])])


def bmm_dequant(acc, qs_a, qs_b, rows=None):
    """fp64 acc / (qs_a[b, i] * qs_b[b, j]) per problem b."""
    out = []
    for i in range(acc.shape[0]):
        qa = np.asarray(qs_a[i])
        qa = qa[list(rows)] if (rows is not None and qa.size > 1) else qa
        out.append(dequant(acc[i], qa, np.asarray(qs_b[i])))
    return np.stack(out)


# ---------------------------------------------------------------- LLM.int8() decomposition
def llmint8_outliers(X, thr=6.0, min_ratio=0.0):
    X = f32(X)
    M, K = X.shape
    idx = np.empty(max(K, 1), np.int32)
    n = lib().or_llmint8_outliers(_ptr(X), M, K, K, float(thr), float(min_ratio), _ptr(idx))
    return idx[:n].copy()


def llmint8_quant_rows(X, idx):
    X = f32(X)
    M, K = X.shape
    idx = _c(idx, np.int32)
    Xq = np.empty((M, K), np.int8)
    qs = np.empty(M, np.float32)
    lib().or_llmint8_quant_rows(_ptr(X), M, K, K, _ptr(idx), idx.size, _ptr(Xq), _ptr(qs))
    return Xq, qs


def llmint8_quant_weight(W, idx):
    W = f32(W)
    N, K = W.shape
    idx = _c(idx, np.int32)
    Wq = np.empty((N, K), np.int8)
    qs = np.empty(N, np.float32)
    lib().or_llmint8_quant_weight(_ptr(W), N, K, _ptr(idx), idx.size, _ptr(Wq), _ptr(qs))
    return Wq, qs


def llmint8_combine(acc, qs_x, qs_w, X, W, idx, rows=None):
    acc = _c(acc, np.int64)
    X, W = f32(X), f32(W)
    M, K = X.shape
    N = W.shape[0]
    idx = _c(idx, np.int32)
    n_rows = acc.shape[0]
    r0 = 0 if rows is None else rows[0]
    y = np.empty((n_rows, N), np.float64)
    lib().or_llmint8_combine(_ptr(acc), r0, r0 + n_rows, N, K, _ptr(_c(qs_x, np.float32)),
                             _ptr(_c(qs_w, np.float32)), _ptr(X), K, _ptr(W), _ptr(idx), idx.size, _ptr(y))
    return y


def llmint8_matmul(X, W, thr=6.0, min_ratio=0.0, rows=None):
    """Whole decomposition: returns (y fp64, idx, Xq, qs_x, Wq, qs_w)."""
    idx = llmint8_outliers(X, thr, min_ratio)
    Xq, qs_x = llmint8_quant_rows(X, idx)
    Wq, qs_w = llmint8_quant_weight(W, idx)
    acc = gemm_i8(Xq, Wq, rows)
    y = llmint8_combine(acc, qs_x, qs_w, X, W, idx, rows)
    return y, idx, Xq, qs_x, Wq, qs_w
