"""ctypes binding of libsq_b200.so: argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
tensors that already live on the GPU (torch provides device memory and the
current stream), checks dtype/contiguity, passes raw pointers and sizes, and
raises SqError when the call returns a non-zero status. No arithmetic of the
method happens in Python, and there is no fallback: if the shared library is
missing or cannot be loaded, the first call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsq_b200.so")

SQ_F32, SQ_F16, SQ_BF16, SQ_I32, SQ_I8 = 0, 1, 2, 3, 4
SQ_LAYERNORM, SQ_RMSNORM = 0, 1
SQ_ACT_SWIGLU, SQ_ACT_RELU, SQ_ACT_GELU = 0, 1, 2
SQ_OP_GEMM, SQ_OP_QUANT_ACT, SQ_OP_QUANT_WEIGHT, SQ_OP_LLMINT8_DETECT, SQ_OP_LLMINT8 = 0, 1, 2, 3, 4

STATUS = {0: "SQ_OK", 1: "SQ_ERR_INVALID_ARG", 2: "SQ_ERR_UNSUPPORTED_SHAPE", 3: "SQ_ERR_ALIGNMENT",
          4: "SQ_ERR_CUDA", 5: "SQ_ERR_TIMEOUT"}

_DT = {torch.float32: SQ_F32, torch.float16: SQ_F16, torch.bfloat16: SQ_BF16, torch.int32: SQ_I32,
       torch.int8: SQ_I8}


class SqError(RuntimeError):
    def __init__(self, name, status, msg):
        super().__init__(f"{name}: {STATUS.get(status, status)}: {msg}")
        self.status = status


class LLMInt8Weight(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("N", ctypes.c_int64), ("Wq", ctypes.c_void_p),
                ("qs_w", ctypes.c_void_p), ("cached_idx", ctypes.c_void_p), ("cached_n", ctypes.c_void_p),
                ("wo", ctypes.c_void_p)]


_p, _i64, _i, _f, _d, _sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double,
                             ctypes.c_size_t)

SIGNATURES = {
    "sq_workspace_size": ([_i, _i64, _i64, _i64], _sz),
    "sq_last_error_string": ([], ctypes.c_char_p),
    "sq_workspace_status": ([_p, _p], _i),
    "sq_version": ([], _i),
    "sq_selftest_wait_timeout": ([_p, _sz, ctypes.c_uint64, _p], _i),
    "sq_calib_absmax": ([_p, _i, _i64, _i64, _i64, _p, _p], _i),
    "sq_weight_absmax": ([_p, _i, _i64, _i64, _i64, _p, _p], _i),
    "sq_smooth_scales": ([_p, _p, _i64, _d, _p, _p], _i),
    "sq_fold_weight": ([_p, _i, _i64, _i64, _p, _p, _p], _i),
    "sq_quantize_weight_fold_prev": ([_p, _i, _i64, _i64, _p, _p, _p, _p, _p], _i),
    "sq_fold_norm": ([_p, _p, _p, _i64, _p, _p, _p], _i),
    "sq_smooth_fold_norm": ([_p, _p, _i64, _d, _p, _p, _p, _p, _p, _p], _i),
    "sq_fold_prev_linear": ([_p, _i, _i64, _i64, _p, _p, _p, _p, _p], _i),
    "sq_quantize_weight": ([_p, _i, _i64, _i64, _p, _i, _p, _p, _p, _sz, _p], _i),
    "sq_quantize_act": ([_p, _i, _i64, _i64, _i64, _p, _i, _p, _p, _p, _p, _sz, _p], _i),
    "sq_scale_from_absmax": ([_p, _i64, _p, _p], _i),
    "sq_norm_smooth_quant": ([_p, _i, _i64, _i64, _i64, _i, _p, _p, _f, _i, _p, _p, _p, _p, _p, _p], _i),
    "sq_bmm_w8a8": ([_p, _p, _i64, _i64, _i64, _i64, _p, _i, _p, _i, _i, _p, _i64, _p, _sz, _p], _i),
    "sq_quantize_weight_fp8": ([_p, _i, _i64, _i64, _p, _i, _p, _p, _p, _sz, _p], _i),
    "sq_quantize_act_fp8": ([_p, _i, _i64, _i64, _i64, _p, _i, _p, _p, _p, _p, _sz, _p], _i),
    "sq_gemm_fp8": ([_p, _p, _i64, _i64, _i64, _p, _i, _p, _i, _p, _i, _p, _i64, _p, _sz, _p], _i),
    "sq_act_quant": ([_p, _i, _i64, _i64, _i64, _i, _i, _p, _p, _p, _p, _p, _p], _i),
    "sq_gemm_w8a8": ([_p, _p, _i64, _i64, _i64, _p, _i, _p, _i, _p, _i, _p, _i64, _p, _sz, _p], _i),
    "sq_gemm_w8a8_act": ([_p, _p, _i64, _i64, _i64, _p, _i, _p, _i, _p, _i, _p, _i, _p, _i64, _p, _sz, _p], _i),
    "sq_llmint8_detect": ([_p, _i, _i64, _i64, _i64, _f, _d, _p, _p, _p, _sz, _p], _i),
    "sq_llmint8_detect_noalloc": ([_p, _i, _i64, _i64, _i64, _f, _d, _p, _p, _p], _i),
    "sq_llmint8_quant_rows": ([_p, _i, _i64, _i64, _i64, _p, _p, _p, _p, _p], _i),
    "sq_llmint8_quant_weight": ([_p, _i, _i64, _i64, _p, _p, _p, _p, _p], _i),
    "sq_llmint8_matmul": ([_p, _i, _i64, _i64, _i64, ctypes.POINTER(LLMInt8Weight), _f, _d, _p, _i64, _p, _p, _p,
                           _sz, _p], _i),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libsq_b200.so (once). Raises if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -m w8a8_post_quantization_sq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(name, status):
    if status != 0:
        raise SqError(name, status, lib().sq_last_error_string().decode())


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if t.device.index is not None and t.device.index != torch.cuda.current_device():
        raise ValueError(f"tensor on {t.device}, but the current device is cuda:{torch.cuda.current_device()}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dt(t):
    return _DT[t.dtype]


def _ld(t):
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit inner stride")
    return t.stride(0)


def _need(ok, msg):
    if not ok:
        raise ValueError(msg)


def _out(t, dtype, n, what):
    """An output the library writes n elements of, back to back."""
    _need(t.dtype == dtype and t.is_contiguous() and t.numel() >= n,
          f"{what} must be a contiguous {dtype} tensor of at least {n} elements")


def _scales(t, n, what):
    """One scale, or one per row/column: the library reads n entries whenever
    the tensor holds more than one."""
    _need(t is None or t.numel() == 1 or t.numel() >= n, f"{what} must hold 1 or at least {n} scales")


def _vec(t, dtype, n=None):
    if t is None:
        return None
    if t.dtype != dtype or not t.is_contiguous() or (n is not None and t.numel() != n):
        raise ValueError(f"expected a contiguous {dtype} tensor of {n} elements")
    return _ptr(t)


# ---------------------------------------------------------------- workspace
def sq_workspace_size(op, M, N, K):
    return int(lib().sq_workspace_size(op, M, N, K))


def workspace(op, M, N, K, device=None):
    """A zeroed workspace tensor sized for `op` (allocated by torch)."""
    n = max(sq_workspace_size(op, M, N, K), 256)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def sq_workspace_status(ws, stream=None):
    _check("sq_workspace_status", lib().sq_workspace_status(_ptr(ws), _stream(stream)))


def sq_selftest_wait_timeout(ws, timeout_ns, stream=None):
    _check("sq_selftest_wait_timeout", lib().sq_selftest_wait_timeout(_ptr(ws), ws.numel(), int(timeout_ns),
                                                                      _stream(stream)))


def sq_version():
    return int(lib().sq_version())


# ---------------------------------------------------------------- calibration absmax
def sq_calib_absmax(X, xmax, stream=None):
    _check("sq_calib_absmax", lib().sq_calib_absmax(_ptr(X), _dt(X), X.shape[0], X.shape[1], _ld(X),
                                                    _vec(xmax, torch.float32, X.shape[1]), _stream(stream)))


def sq_weight_absmax(W, wmax, stream=None):
    _check("sq_weight_absmax", lib().sq_weight_absmax(_ptr(W), _dt(W), W.shape[0], W.shape[1], _ld(W),
                                                      _vec(wmax, torch.float32, W.shape[1]), _stream(stream)))


# ---------------------------------------------------------------- smoothing factors and folds
def sq_smooth_scales(xmax, wmax, alpha, s_out, stream=None):
    K = xmax.numel()
    _check("sq_smooth_scales", lib().sq_smooth_scales(_vec(xmax, torch.float32, K), _vec(wmax, torch.float32, K), K,
                                                      float(alpha), _vec(s_out, torch.float32, K), _stream(stream)))


def sq_fold_weight(W, s, Wp_out, stream=None):
    N, K = W.shape
    _need(W.is_contiguous(), "W must be contiguous")
    _out(Wp_out, torch.float32, N * K, "Wp_out")
    _check("sq_fold_weight", lib().sq_fold_weight(_ptr(W), _dt(W), N, K, _vec(s, torch.float32, K), _ptr(Wp_out),
                                                  _stream(stream)))


def sq_fold_norm(gamma, beta, s, gamma_out, beta_out=None, stream=None):
    K = gamma.numel()
    _check("sq_fold_norm", lib().sq_fold_norm(_vec(gamma, torch.float32, K), _vec(beta, torch.float32, K),
                                              _vec(s, torch.float32, K), K, _vec(gamma_out, torch.float32, K),
                                              _vec(beta_out, torch.float32, K), _stream(stream)))


def sq_quantize_weight_fold_prev(W, s_next, s, Wq, qs_w, stream=None):
    N, K = W.shape
    _need(W.is_contiguous(), "W must be contiguous")
    _out(Wq, torch.int8, N * K, "Wq")
    _check("sq_quantize_weight_fold_prev", lib().sq_quantize_weight_fold_prev(
        _ptr(W), _dt(W), N, K, _vec(s_next, torch.float32, N), _vec(s, torch.float32, K), _ptr(Wq),
        _vec(qs_w, torch.float32, N), _stream(stream)))


def sq_smooth_fold_norm(xmax, wmax, alpha, gamma, beta, s_out, gamma_out, beta_out=None, stream=None):
    K = xmax.numel()
    _check("sq_smooth_fold_norm", lib().sq_smooth_fold_norm(
        _vec(xmax, torch.float32, K), _vec(wmax, torch.float32, K), K, float(alpha), _vec(gamma, torch.float32, K),
        _vec(beta, torch.float32, K), _vec(s_out, torch.float32, K), _vec(gamma_out, torch.float32, K),
        _vec(beta_out, torch.float32, K), _stream(stream)))


def sq_fold_prev_linear(W, s, Wp_out, bias=None, bias_out=None, stream=None):
    N, K = W.shape
    _need(W.is_contiguous(), "W must be contiguous")
    _out(Wp_out, torch.float32, N * K, "Wp_out")
    _check("sq_fold_prev_linear", lib().sq_fold_prev_linear(
        _ptr(W), _dt(W), N, K, _vec(bias, torch.float32, N), _vec(s, torch.float32, N), _ptr(Wp_out),
        _vec(bias_out, torch.float32, N), _stream(stream)))


# ---------------------------------------------------------------- weight quantisation
def sq_quantize_weight(W, s, per_channel, Wq, qs_w, ws=None, stream=None):
    N, K = W.shape
    _need(W.is_contiguous(), "W must be contiguous")
    _out(Wq, torch.int8, N * K, "Wq")
    _check("sq_quantize_weight", lib().sq_quantize_weight(
        _ptr(W), _dt(W), N, K, _vec(s, torch.float32, K), int(per_channel), _ptr(Wq),
        _vec(qs_w, torch.float32, N if per_channel else 1), _ptr(ws), 0 if ws is None else ws.numel(),
        _stream(stream)))


# ---------------------------------------------------------------- activation quantisation without a norm
def sq_quantize_act(X, s, per_token, static_qs, Xq, qs_x, ws=None, stream=None):
    M, K = X.shape
    _out(Xq, torch.int8, M * K, "Xq")
    _check("sq_quantize_act", lib().sq_quantize_act(
        _ptr(X), _dt(X), M, K, _ld(X), _vec(s, torch.float32, K), int(per_token), _vec(static_qs, torch.float32, 1),
        _ptr(Xq), _vec(qs_x, torch.float32, M if per_token else 1), _ptr(ws), 0 if ws is None else ws.numel(),
        _stream(stream)))


def sq_scale_from_absmax(absmax, qs_out, stream=None):
    _check("sq_scale_from_absmax", lib().sq_scale_from_absmax(_vec(absmax, torch.float32), absmax.numel(),
                                                              _vec(qs_out, torch.float32, 1), _stream(stream)))


# ---------------------------------------------------------------- fused norm + smoothing + int8
def sq_norm_smooth_quant(H, norm, gamma, beta, eps, per_token, static_qs, Xq, qs_x, absmax=None, V=None,
                         stream=None):
    M, K = H.shape
    if Xq is not None:
        _out(Xq, torch.int8, M * K, "Xq")
        _need(qs_x is not None and qs_x.numel() >= (M if per_token else 1),
              f"qs_x must hold {M if per_token else 1} scales")
    if V is not None:
        _out(V, H.dtype, M * K, "V")
    _check("sq_norm_smooth_quant", lib().sq_norm_smooth_quant(
        _ptr(H), _dt(H), M, K, _ld(H), int(norm), _vec(gamma, torch.float32, K), _vec(beta, torch.float32, K),
        float(eps), int(per_token), _vec(static_qs, torch.float32, 1), _ptr(Xq),
        None if qs_x is None else _vec(qs_x, torch.float32), _vec(absmax, torch.float32, K), _ptr(V),
        _stream(stream)))


# ---------------------------------------------------------------- batched int8 GEMM (attention)
def sq_bmm_w8a8(Aq, Bq, qs_a, qs_b, Y, ws, stream=None):
    """Aq [batch, M, K], Bq [batch, N, K] int8; qs_a [batch, M] or [batch];
    qs_b [batch, N] or [batch]; Y [batch, M, N] (inner stride 1)."""
    b, M, K = Aq.shape
    N = Bq.shape[1]
    if Aq.dtype != torch.int8 or Bq.dtype != torch.int8 or not Aq.is_contiguous() or not Bq.is_contiguous():
        raise ValueError("Aq and Bq must be contiguous int8")
    if Bq.shape[0] != b or Bq.shape[2] != K or tuple(Y.shape[:2]) != (b, M) or Y.shape[2] != N:
        raise ValueError("shape mismatch")
    if Y.stride(2) != 1 or Y.stride(0) != M * Y.stride(1):
        raise ValueError("Y must be [batch, M, ldy] with batches back to back")
    _need(qs_a is None or qs_a.numel() >= b, f"qs_a must hold one scale per problem ({b}) or per row")
    _need(qs_b is None or qs_b.numel() >= b, f"qs_b must hold one scale per problem ({b}) or per row")
    _check("sq_bmm_w8a8", lib().sq_bmm_w8a8(
        _ptr(Aq), _ptr(Bq), b, M, N, K, _vec(qs_a, torch.float32), int(qs_a is not None and qs_a.numel() == b * M),
        _vec(qs_b, torch.float32), int(qs_b is not None and qs_b.numel() == b * N), _dt(Y), _ptr(Y), Y.stride(1),
        _ptr(ws), ws.numel(), _stream(stream)))


# ---------------------------------------------------------------- FP8 variant
def sq_quantize_weight_fp8(W, s, per_channel, Wq, qs_w, ws=None, stream=None):
    N, K = W.shape
    _need(W.is_contiguous(), "W must be contiguous")
    _out(Wq, torch.uint8, N * K, "Wq (E4M3 codes)")
    _check("sq_quantize_weight_fp8", lib().sq_quantize_weight_fp8(
        _ptr(W), _dt(W), N, K, _vec(s, torch.float32, K), int(per_channel), _ptr(Wq),
        _vec(qs_w, torch.float32, N if per_channel else 1), _ptr(ws), 0 if ws is None else ws.numel(),
        _stream(stream)))


def sq_quantize_act_fp8(X, s, per_token, static_qs, Xq, qs_x, ws=None, stream=None):
    M, K = X.shape
    _out(Xq, torch.uint8, M * K, "Xq (E4M3 codes)")
    _check("sq_quantize_act_fp8", lib().sq_quantize_act_fp8(
        _ptr(X), _dt(X), M, K, _ld(X), _vec(s, torch.float32, K), int(per_token), _vec(static_qs, torch.float32, 1),
        _ptr(Xq), _vec(qs_x, torch.float32, M if per_token else 1), _ptr(ws), 0 if ws is None else ws.numel(),
        _stream(stream)))


def sq_gemm_fp8(Xq, Wq, qs_x, qs_w, bias, Y, ws, stream=None):
    M, K = Xq.shape
    N = Wq.shape[0]
    if Xq.dtype != torch.uint8 or Wq.dtype != torch.uint8 or not Xq.is_contiguous() or not Wq.is_contiguous():
        raise ValueError("Xq and Wq must be contiguous uint8 (E4M3 codes)")
    if Wq.shape[1] != K or Y.shape[0] != M or Y.shape[1] != N:
        raise ValueError("shape mismatch")
    _scales(qs_x, M, "qs_x")
    _scales(qs_w, N, "qs_w")
    _check("sq_gemm_fp8", lib().sq_gemm_fp8(
        _ptr(Xq), _ptr(Wq), M, N, K, _vec(qs_x, torch.float32), int(qs_x.numel() > 1), _vec(qs_w, torch.float32),
        int(qs_w.numel() > 1), _vec(bias, torch.float32, N), _dt(Y), _ptr(Y), _ld(Y), _ptr(ws), ws.numel(),
        _stream(stream)))


# ---------------------------------------------------------------- MLP activation + int8
def sq_act_quant(A, act, per_token, static_qs, Xq, qs_x, absmax=None, H=None, stream=None):
    """A: [M, 2I] ([gate | up], SQ_ACT_SWIGLU) or [M, I] (SQ_ACT_RELU, SQ_ACT_GELU)."""
    M, W = A.shape
    I = W // 2 if act == SQ_ACT_SWIGLU else W
    if Xq is not None:
        _out(Xq, torch.int8, M * I, "Xq")
        _need(qs_x is not None and qs_x.numel() >= (M if per_token else 1),
              f"qs_x must hold {M if per_token else 1} scales")
    if H is not None:
        _out(H, A.dtype, M * I, "H")
    _check("sq_act_quant", lib().sq_act_quant(
        _ptr(A), _dt(A), M, I, _ld(A), int(act), int(per_token), _vec(static_qs, torch.float32, 1), _ptr(Xq),
        None if qs_x is None else _vec(qs_x, torch.float32), _vec(absmax, torch.float32, I), _ptr(H),
        _stream(stream)))


# ---------------------------------------------------------------- int8 GEMM
def sq_gemm_w8a8(Xq, Wq, qs_x, qs_w, bias, Y, ws, stream=None):
    M, K = Xq.shape
    N = Wq.shape[0]
    if Xq.dtype != torch.int8 or Wq.dtype != torch.int8 or not Xq.is_contiguous() or not Wq.is_contiguous():
        raise ValueError("Xq and Wq must be contiguous int8")
    if Wq.shape[1] != K or Y.shape[0] != M or Y.shape[1] != N:
        raise ValueError("shape mismatch")
    _scales(qs_x, M, "qs_x")
    _scales(qs_w, N, "qs_w")
    _check("sq_gemm_w8a8", lib().sq_gemm_w8a8(
        _ptr(Xq), _ptr(Wq), M, N, K, _vec(qs_x, torch.float32), int(qs_x is not None and qs_x.numel() > 1),
        _vec(qs_w, torch.float32), int(qs_w is not None and qs_w.numel() > 1), _vec(bias, torch.float32, N),
        _dt(Y), _ptr(Y), _ld(Y), _ptr(ws), ws.numel(), _stream(stream)))


def sq_gemm_w8a8_act(Xq, Wq, qs_x, qs_w, bias, act, H, ws, static_qs=None, out_dtype=None, stream=None):
    """The int8 GEMM with the MLP activation in its epilogue: H [M, N/2]
    (SwiGLU over interleaved gate/up channel pairs) or [M, N] (ReLU, GELU).
    Without static_qs H is 16-bit (its dtype is the dtype the GEMM rounds Y
    to); with a static scale H is int8 codes and out_dtype gives Y's dtype."""
    M, K = Xq.shape
    N = Wq.shape[0]
    if Xq.dtype != torch.int8 or Wq.dtype != torch.int8 or not Xq.is_contiguous() or not Wq.is_contiguous():
        raise ValueError("Xq and Wq must be contiguous int8")
    width = N // 2 if act == SQ_ACT_SWIGLU else N
    if Wq.shape[1] != K or H.shape[0] != M or H.shape[1] != width:
        raise ValueError(f"shape mismatch: H must be [{M}, {width}]")
    if static_qs is None:
        _need(H.dtype in (torch.float16, torch.bfloat16), "H must be fp16 or bf16")
        ydt = _dt(H)
    else:
        _need(H.dtype == torch.int8, "with a static scale H must be int8")
        _need(out_dtype in (torch.float16, torch.bfloat16), "out_dtype (Y's dtype) must be fp16 or bf16")
        ydt = SQ_F16 if out_dtype == torch.float16 else SQ_BF16
    _scales(qs_x, M, "qs_x")
    _scales(qs_w, N, "qs_w")
    _check("sq_gemm_w8a8_act", lib().sq_gemm_w8a8_act(
        _ptr(Xq), _ptr(Wq), M, N, K, _vec(qs_x, torch.float32), int(qs_x.numel() > 1), _vec(qs_w, torch.float32),
        int(qs_w.numel() > 1), _vec(bias, torch.float32, N), int(act), _vec(static_qs, torch.float32, 1), ydt,
        _ptr(H), _ld(H), _ptr(ws), ws.numel(), _stream(stream)))


# ---------------------------------------------------------------- LLM.int8() decomposition
def sq_llmint8_detect(X, threshold, min_ratio, idx, n, ws, stream=None):
    M, K = X.shape
    _check("sq_llmint8_detect", lib().sq_llmint8_detect(
        _ptr(X), _dt(X), M, K, _ld(X), float(threshold), float(min_ratio), _vec(idx, torch.int32, K),
        _vec(n, torch.int32, 1), _ptr(ws), ws.numel(), _stream(stream)))


def sq_llmint8_detect_noalloc(X, threshold, min_ratio, idx, n, stream=None):
    """sq_llmint8_detect with the library's own fixed scratch (no workspace)."""
    M, K = X.shape
    _check("sq_llmint8_detect_noalloc", lib().sq_llmint8_detect_noalloc(
        _ptr(X), _dt(X), M, K, _ld(X), float(threshold), float(min_ratio), _vec(idx, torch.int32, K),
        _vec(n, torch.int32, 1), _stream(stream)))


def sq_llmint8_quant_rows(X, idx, n, Xq, qs_x, stream=None):
    M, K = X.shape
    _out(Xq, torch.int8, M * K, "Xq")
    _check("sq_llmint8_quant_rows", lib().sq_llmint8_quant_rows(
        _ptr(X), _dt(X), M, K, _ld(X), _vec(idx, torch.int32), _vec(n, torch.int32, 1), _ptr(Xq),
        _vec(qs_x, torch.float32, M), _stream(stream)))


def sq_llmint8_quant_weight(W, idx, n, Wq, qs_w, stream=None):
    N, K = W.shape
    _need(W.is_contiguous(), "W must be contiguous")
    _out(Wq, torch.int8, N * K, "Wq")
    _check("sq_llmint8_quant_weight", lib().sq_llmint8_quant_weight(
        _ptr(W), _dt(W), N, K, _vec(idx, torch.int32), _vec(n, torch.int32, 1), _ptr(Wq),
        _vec(qs_w, torch.float32, N), _stream(stream)))


def llmint8_weight_state(W, keep_wo=True):
    """Device buffers of the int8 weight cache for sq_llmint8_matmul (torch
    allocates them; cached_n = -1 marks the cache empty). keep_wo: also keep
    the fp32 outlier channels of W (32 x N rounded up to 256) in the state."""
    N, K = W.shape
    st = {"W": W, "Wq": torch.empty((N, K), dtype=torch.int8, device=W.device),
          "qs_w": torch.empty(N, dtype=torch.float32, device=W.device),
          "cached_idx": torch.zeros(K, dtype=torch.int32, device=W.device),
          "cached_n": torch.full((1,), -1, dtype=torch.int32, device=W.device),
          "wo": torch.zeros((32, (N + 255) // 256 * 256), dtype=torch.float32, device=W.device) if keep_wo else None}
    st["c"] = LLMInt8Weight(W.data_ptr(), N, st["Wq"].data_ptr(), st["qs_w"].data_ptr(),
                            st["cached_idx"].data_ptr(), st["cached_n"].data_ptr(),
                            st["wo"].data_ptr() if keep_wo else None)
    return st


def sq_llmint8_matmul(X, wstate, threshold, min_ratio, Y, idx, n, ws, stream=None):
    M, K = X.shape
    W = wstate["W"]
    _need(W.dtype == X.dtype and W.dim() == 2 and W.shape[1] == K, "the weight state's W must be [N, K] of X's dtype")
    _need(Y.dtype == X.dtype and tuple(Y.shape) == (M, W.shape[0]), "Y must be [M, N] of X's dtype")
    _check("sq_llmint8_matmul", lib().sq_llmint8_matmul(
        _ptr(X), _dt(X), M, K, _ld(X), ctypes.byref(wstate["c"]), float(threshold), float(min_ratio), _ptr(Y),
        _ld(Y), _vec(idx, torch.int32, K), _vec(n, torch.int32, 1), _ptr(ws), ws.numel(), _stream(stream)))
