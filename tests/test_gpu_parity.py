"""GPU parity: every hot-path step through the C ABI against the CPU oracle.

Bit-exact for int8 codes, scales, int32 accumulators, calibration maxima,
smoothing factors and outlier sets. Dequantised outputs:
  fp32  |gpu - y| <= 1e-6 * (|acc/(qx qw)| + |h| + |bias|)   (y = oracle fp64)
  16-bit  within 1 ulp of RN16(y), plus the same fp32 allowance where terms
          cancel (bias or the LLM.int8 outlier term).
The fp32 epilogue computes acc * ((1/qx) * (1/qw)) with four roundings, at most
about 3e-7 relative, so 1e-6 is the bound the arithmetic gives.
"""
import numpy as np
import pytest
import torch

import oracle
import w8a8_post_quantization_sq_b200 as sq
from w8a8_post_quantization_sq_b200 import inputs
from parity_helpers import assert_close_16, assert_close_f32, npf, npu16, ord16, ulp16  # noqa: F401

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sq.lib()
    oracle.lib()


def rnd(shape, seed, dtype=torch.float32, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(dtype)


# ---------------------------------------------------------------- calibration absmax
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("M,K", [(1, 8), (37, 1000), (300, 2056), (1029, 4104)])
def test_calib_absmax(dtype, M, K):
    if dtype == torch.float32 and K % 4:
        pytest.skip()
    X1 = rnd((M, K), 1, dtype, 3.0)
    X2 = rnd((M + 5, K), 2, dtype, 3.0)
    X2[:, K // 3] *= 100
    xmax = torch.zeros(K, device=DEV)
    sq.sq_calib_absmax(X1.to(DEV), xmax)
    sq.sq_calib_absmax(X2.to(DEV), xmax)
    ref = oracle.col_absmax(X2, oracle.col_absmax(X1))
    assert np.array_equal(npf(xmax), ref)


@pytest.mark.parametrize("dtype,M,K,ld", [(torch.bfloat16, 2061, 5128, 5128), (torch.float16, 1531, 6144, 6160),
                                           (torch.float32, 1203, 4100, 4100)])
def test_calib_absmax_bulk(dtype, M, K, ld):
    """Inputs of 16 MB and more take the bulk-staged kernel: ragged row bands,
    a short last column block, a row stride wider than K."""
    X = rnd((M, ld), 11, dtype, 2.0)
    X[M // 2, K - 1] = 500.0
    X[M - 1, 7] = -300.0
    xmax = torch.full((K,), 0.25, device=DEV)  # running max: entries above the data survive
    xmax[5] = 1000.0
    view = X.to(DEV)[:, :K]
    assert view.numel() * view.element_size() >= 16 * 2**20
    sq.sq_calib_absmax(view, xmax)
    prev = np.full(K, 0.25, dtype=np.float32)
    prev[5] = 1000.0
    assert np.array_equal(npf(xmax), oracle.col_absmax(X[:, :K], prev))


def test_calib_absmax_strided_and_weight():
    X = rnd((64, 1024), 3, torch.bfloat16)
    view = X.to(DEV)[:, 256:768]  # ld = 1024, K = 512
    xmax = torch.zeros(512, device=DEV)
    sq.sq_calib_absmax(view, xmax)
    assert np.array_equal(npf(xmax), oracle.col_absmax(X[:, 256:768]))
    W = rnd((3000, 520), 4, torch.float32, 0.02)
    wmax = torch.zeros(520, device=DEV)
    sq.sq_weight_absmax(W.to(DEV), wmax)
    assert np.array_equal(npf(wmax), oracle.col_absmax(W))


# ---------------------------------------------------------------- smoothing factors and folds
@pytest.mark.parametrize("alpha", [0.0, 0.4, 0.5, 0.6, 0.75, 1.0])
def test_smooth_scales(alpha):
    K = 12288
    g = torch.Generator().manual_seed(5)
    x = torch.rand(K, generator=g) * 200
    w = torch.rand(K, generator=g) * 0.3
    x[:7] = torch.tensor([0.0, 1e-7, 1e-5, 1.0, 4.0, 100.0, 32.0])
    w[:7] = torch.tensor([0.0, 1.0, 1e-5, 0.0, 4.0, 0.01, 32.0])
    s = torch.empty(K, device=DEV)
    sq.sq_smooth_scales(x.to(DEV), w.to(DEV), alpha, s)
    ref = oracle.smooth_scales(x, w, alpha)
    got = npf(s)
    mism = np.nonzero(got != ref)[0]
    assert mism.size == 0, f"alpha={alpha}: {mism.size} mismatches, e.g. {mism[:3]} {got[mism[:3]]} {ref[mism[:3]]}"


def test_fold_weight_and_norm():
    N, K = 333, 1032
    for dtype in (torch.float16, torch.bfloat16, torch.float32):
        W = rnd((N, K), 6, dtype, 0.03)
        s = (torch.rand(K, generator=torch.Generator().manual_seed(7)) * 20 + 0.01)
        Wp = torch.empty((N, K), device=DEV)
        sq.sq_fold_weight(W.to(DEV), s.to(DEV), Wp)
        assert np.array_equal(npf(Wp), oracle.fold_weight(W.float().numpy(), s.numpy(), round_f32=True))
    gamma = 1 + 0.1 * rnd(K, 8)
    beta = 0.1 * rnd(K, 9)
    go = torch.empty(K, device=DEV)
    bo = torch.empty(K, device=DEV)
    sq.sq_fold_norm(gamma.to(DEV), beta.to(DEV), s.to(DEV), go, bo)
    rg, rb = oracle.fold_norm(gamma.numpy(), beta.numpy(), s.numpy(), round_f32=True)
    assert np.array_equal(npf(go), rg) and np.array_equal(npf(bo), rb)


@pytest.mark.parametrize("alpha", [0.5, 0.4, 0.0, 1.0])
@pytest.mark.parametrize("with_beta", [True, False])
def test_smooth_fold_norm(alpha, with_beta):
    """The one-launch smoothing + norm fold against the oracle's two steps."""
    K = 4104
    g = torch.Generator().manual_seed(17)
    xmax = torch.rand(K, generator=g) * 80
    wmax = torch.rand(K, generator=g) * 0.3
    xmax[:5] = 0.0  # the clamp at 1e-5
    gamma = 1 + 0.1 * rnd(K, 18)
    beta = 0.1 * rnd(K, 19) if with_beta else None
    s = torch.empty(K, device=DEV)
    go = torch.empty(K, device=DEV)
    bo = torch.empty(K, device=DEV) if with_beta else None
    sq.sq_smooth_fold_norm(xmax.to(DEV), wmax.to(DEV), alpha, gamma.to(DEV), None if beta is None else beta.to(DEV),
                           s, go, bo)
    rs = oracle.smooth_scales(xmax.numpy(), wmax.numpy(), alpha)
    assert np.array_equal(npf(s), rs)
    rg, rb = oracle.fold_norm(gamma.numpy(), None if beta is None else beta.numpy(), rs, round_f32=True)
    assert np.array_equal(npf(go), rg)
    if with_beta:
        assert np.array_equal(npf(bo), rb)
    with pytest.raises(sq.SqError):
        sq.sq_smooth_fold_norm(xmax.to(DEV), wmax.to(DEV), 1.5, gamma.to(DEV), None, s, go)


# ---------------------------------------------------------------- fold into the previous linear
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("N,K", [(333, 1024), (3072, 1040), (200, 3072), (96, 8208)])
def test_quantize_weight_fold_prev(dtype, N, K):
    """The fold of 1/s_next into the output channels and the int8 quantisation
    in one pass against the oracle's fold, smoothing fold and quantisation."""
    W = rnd((N, K), N + K, dtype, 0.03)
    g = torch.Generator().manual_seed(N)
    s_next = torch.rand(N, generator=g) * 20 + 0.01
    s = torch.rand(K, generator=g) * 5 + 0.05
    Wq = torch.empty((N, K), dtype=torch.int8, device=DEV)
    qw = torch.empty(N, device=DEV)
    sq.sq_quantize_weight_fold_prev(W.to(DEV), s_next.to(DEV), s.to(DEV), Wq, qw)
    up_f, _ = oracle.fold_prev_linear(W.float().numpy(), s_next.numpy())
    rq, rqs = oracle.quantize_weight(oracle.fold_weight(up_f, s.numpy()), True)
    assert np.array_equal(Wq.cpu().numpy(), rq)
    assert np.array_equal(npf(qw), rqs)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("with_bias", [True, False])
def test_fold_prev_linear(dtype, with_bias):
    N, K = 333, 1032
    W = rnd((N, K), 12, dtype, 0.03)
    s = torch.rand(N, generator=torch.Generator().manual_seed(13)) * 20 + 0.01
    b = rnd(N, 14) if with_bias else None
    Wp = torch.empty((N, K), device=DEV)
    bo = torch.empty(N, device=DEV) if with_bias else None
    sq.sq_fold_prev_linear(W.to(DEV), s.to(DEV), Wp, None if b is None else b.to(DEV), bo)
    rW, rb = oracle.fold_prev_linear(W.float().numpy(), s.numpy(), None if b is None else b.numpy())
    assert np.array_equal(npf(Wp), rW)
    if with_bias:
        assert np.array_equal(npf(bo), rb)


# ---------------------------------------------------------------- MLP activation + int8
def _act_input(M, I, act, dtype, seed, extra_cols=0):
    """Gate/up (or fc1) outputs: N(0, 2), with exp-range edge values planted."""
    width = (2 * I if act == sq.SQ_ACT_SWIGLU else I) + extra_cols
    A = rnd((M, width), seed, torch.float32, 2.0)
    A[0, :8] = torch.tensor([0.0, -0.0, 88.5, -88.5, 87.0, -87.0, 30.0, -30.0])
    A[min(1, M - 1), 3] = 200.0
    if act == sq.SQ_ACT_GELU:
        A[min(1, M - 1), :8] = torch.tensor([-10.0, -10.5, -4.0, 1e-20, -1e-20, 5e3, -5e3, 3.0])  # exp's edges
    if act == sq.SQ_ACT_RELU and M > 2:
        A[2] = -A[2].abs()  # an all-zero h row: scale from the 1e-8 floor
    return A.to(dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("act", [0, 1, 2])
@pytest.mark.parametrize("I,M", [(8, 5), (1000, 67), (3072, 300), (8192, 33), (9000, 21), (28672, 9)])
def test_act_quant(dtype, act, I, M):
    """Codes, scales, the 16-bit h and the calibration maxima bit for bit; a
    row stride wider than the row."""
    A = _act_input(M, I, act, dtype, I + act, extra_cols=8)
    width = 2 * I if act == sq.SQ_ACT_SWIGLU else I
    Ad = A.to(DEV)[:, :width]
    Xq = torch.empty((M, I), dtype=torch.int8, device=DEV)
    qs = torch.empty(M, device=DEV)
    H = torch.empty((M, I), dtype=dtype, device=DEV)
    am = torch.full((I,), 0.5, device=DEV)
    sq.sq_act_quant(Ad, act, True, None, Xq, qs, am, H)
    r = oracle.act_quant(A[:, :width].float().numpy(), act, want_h=True, absmax=np.full(I, 0.5, np.float32))
    assert np.array_equal(npf(qs), r["qs"])
    assert np.array_equal(Xq.cpu().numpy(), r["Xq"])
    assert np.array_equal(npu16(H), npu16(torch.from_numpy(r["H"]).to(dtype)))
    assert np.array_equal(npf(am), r["absmax"])
    # static per-tensor scale: values beyond the range clip
    qst = torch.tensor([11.0], device=DEV)
    qx = torch.empty(1, device=DEV)
    sq.sq_act_quant(Ad, act, False, qst, Xq, qx)
    rs = oracle.act_quant(A[:, :width].float().numpy(), act, per_token=False, static_qs=11.0)
    assert np.array_equal(Xq.cpu().numpy(), rs["Xq"])
    assert npf(qx)[0] == np.float32(11.0)


def test_act_quant_errors():
    A = torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV)
    Xq = torch.empty((4, 32), dtype=torch.int8, device=DEV)
    with pytest.raises(sq.SqError):
        sq.sq_act_quant(A, sq.SQ_ACT_SWIGLU, False, None, Xq, torch.empty(1, device=DEV))  # no static scale
    with pytest.raises(sq.SqError):
        sq.sq_act_quant(A[:, :60], sq.SQ_ACT_RELU, True, None, torch.empty((4, 60), dtype=torch.int8, device=DEV),
                        torch.empty(4, device=DEV))  # I % 8 != 0
    sq.sq_act_quant(A[:0], sq.SQ_ACT_SWIGLU, True, None, Xq[:0], torch.empty(0, device=DEV))  # M = 0


# ---------------------------------------------------------------- weight quantisation
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("per_channel", [True, False])
@pytest.mark.parametrize("with_s", [True, False])
@pytest.mark.parametrize("K", [1024, 2064, 11008, 12288, 20480, 49152])
def test_quantize_weight(dtype, per_channel, with_s, K):
    """Every row kernel: warp-held rows, block-held rows (six chunks per
    thread up to K = 12288, ragged at 11008), and rows read twice by a block
    (K = 20480, 49152; at 49152, 1100 rows: more than the grid, which is capped
    by the rows in flight, so blocks take several)."""
    if K == 49152 and not per_channel:
        pytest.skip("per-tensor scales at K = 49152 add nothing the per-channel case does not cover")
    N = 517 if K <= 2064 else (1100 if K == 49152 else 131)
    W = rnd((N, K), 10, dtype, 0.02)
    s = torch.rand(K, generator=torch.Generator().manual_seed(11)) * 30 + 0.05 if with_s else None
    Wq = torch.empty((N, K), dtype=torch.int8, device=DEV)
    qs = torch.empty(N if per_channel else 1, device=DEV)
    ws = sq.workspace(sq.SQ_OP_QUANT_WEIGHT, 0, N, K)
    sq.sq_quantize_weight(W.to(DEV), None if s is None else s.to(DEV), per_channel, Wq, qs, ws)
    Wp = oracle.fold_weight(W.float().numpy(), s.numpy(), True) if with_s else W.float().numpy()
    rq, rs = oracle.quantize_weight(Wp, per_channel)
    assert np.array_equal(npf(qs), rs)
    assert np.array_equal(Wq.cpu().numpy(), rq)


# ---------------------------------------------------------------- activation quantisation without a norm
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("mode", ["token", "tensor_dynamic", "tensor_static"])
@pytest.mark.parametrize("K", [256, 1040, 4096, 16400])
def test_quantize_act(dtype, mode, K):
    M = 77
    X = rnd((M, K), 12, dtype)
    X[:, 5] *= 50
    s = torch.rand(K, generator=torch.Generator().manual_seed(13)) * 8 + 0.1
    per_token = mode == "token"
    static = torch.tensor([3.7]) if mode == "tensor_static" else None
    Xq = torch.empty((M, K), dtype=torch.int8, device=DEV)
    qs = torch.empty(M if per_token else 1, device=DEV)
    ws = sq.workspace(sq.SQ_OP_QUANT_ACT, M, 0, K)
    sq.sq_quantize_act(X.to(DEV), s.to(DEV), per_token, None if static is None else static.to(DEV), Xq, qs, ws)
    rq, rs = oracle.quantize_act(X, s.numpy(), per_token, None if static is None else 3.7)
    assert np.array_equal(npf(qs), rs)
    assert np.array_equal(Xq.cpu().numpy(), rq)


def test_quantize_act_config1_worked_path():
    """Single linear, p4 toy shapes: X [16,1024] ch0 x50, per-tensor, s from X itself."""
    d = inputs.c1_single_linear()
    X, W = d["X"], d["W"]
    xmax = torch.zeros(1024, device=DEV)
    wmax = torch.zeros(1024, device=DEV)
    sq.sq_calib_absmax(X.to(DEV), xmax)
    sq.sq_weight_absmax(W.to(DEV), wmax)
    s = torch.empty(1024, device=DEV)
    sq.sq_smooth_scales(xmax, wmax, 0.5, s)
    rs = oracle.smooth_scales(oracle.col_absmax(X), oracle.col_absmax(W), 0.5)
    assert np.array_equal(npf(s), rs)
    Xq = torch.empty((16, 1024), dtype=torch.int8, device=DEV)
    qx = torch.empty(1, device=DEV)
    ws = sq.workspace(sq.SQ_OP_QUANT_ACT, 16, 0, 1024)
    sq.sq_quantize_act(X.to(DEV), s, False, None, Xq, qx, ws)
    rq, rqs = oracle.quantize_act(X, rs, False)
    assert np.array_equal(Xq.cpu().numpy(), rq) and np.array_equal(npf(qx), rqs)


# ---------------------------------------------------------------- fused norm + smoothing + int8
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("norm", ["ln", "rms"])
@pytest.mark.parametrize("K", [8, 1000, 1024, 3072, 7168, 12288, 16384])
def test_norm_smooth_quant_per_token(dtype, norm, K):
    M = 37 if K >= 7168 else 129
    H = rnd((M, K), K, dtype)
    H[:, K // 5] *= 60
    gamma = 1 + 0.1 * rnd(K, 1)
    beta = 0.1 * rnd(K, 2) if norm == "ln" else None
    eps = 1e-5 if norm == "ln" else 1e-6
    nt = sq.SQ_LAYERNORM if norm == "ln" else sq.SQ_RMSNORM
    Xq = torch.empty((M, K), dtype=torch.int8, device=DEV)
    qs = torch.empty(M, device=DEV)
    V = torch.empty((M, K), dtype=dtype, device=DEV)
    sq.sq_norm_smooth_quant(H.to(DEV), nt, gamma.to(DEV), None if beta is None else beta.to(DEV), eps, True, None,
                            Xq, qs, None, V)
    r = oracle.norm_smooth_quant(H, oracle.LAYERNORM if norm == "ln" else oracle.RMSNORM, gamma.numpy(),
                                 None if beta is None else beta.numpy(), eps, True, want_v=True)
    assert np.array_equal(npf(qs), r["qs"])
    assert np.array_equal(Xq.cpu().numpy(), r["Xq"])
    assert np.array_equal(npu16(V), npu16(torch.from_numpy(r["V"]).to(dtype)))


@pytest.mark.parametrize("norm", ["ln", "rms"])
@pytest.mark.parametrize("K,M,dtype", [(5000, 300, torch.bfloat16), (8192, 300, torch.float16),
                                       (8192, 301, torch.bfloat16), (11008, 300, torch.float16),
                                       (12288, 2500, torch.bfloat16), (12288, 2501, torch.float16),
                                       (12288, 1, torch.bfloat16), (13000, 300, torch.bfloat16),
                                       (16384, 700, torch.float16)])
def test_norm_quant_only(norm, K, M, dtype):
    """Codes and scales without the V output, per token and with a static scale:
    the quantise-only kernels, with full and ragged chunk sets; at M = 2500
    every block of the grid cycles its ring of staged rows more than once; odd
    M and a single row leave some blocks fewer rows than the others."""
    H = rnd((M, K), K + 7, dtype)
    H[:, K // 3] *= 50
    gamma = 1 + 0.1 * rnd(K, 5)
    beta = 0.1 * rnd(K, 6) if norm == "ln" else None
    eps = 1e-5 if norm == "ln" else 1e-6
    nt = sq.SQ_LAYERNORM if norm == "ln" else sq.SQ_RMSNORM
    on = oracle.LAYERNORM if norm == "ln" else oracle.RMSNORM
    bd = None if beta is None else beta.to(DEV)
    Hd = H.to(DEV)
    Xq = torch.empty((M, K), dtype=torch.int8, device=DEV)
    qs = torch.empty(M, device=DEV)
    sq.sq_norm_smooth_quant(Hd, nt, gamma.to(DEV), bd, eps, True, None, Xq, qs, None, None)
    r = oracle.norm_smooth_quant(H, on, gamma.numpy(), None if beta is None else beta.numpy(), eps, True)
    assert np.array_equal(npf(qs), r["qs"])
    assert np.array_equal(Xq.cpu().numpy(), r["Xq"])
    qst = torch.tensor([21.5], device=DEV)
    qx = torch.empty(1, device=DEV)
    sq.sq_norm_smooth_quant(Hd, nt, gamma.to(DEV), bd, eps, False, qst, Xq, qx, None, None)
    r = oracle.norm_smooth_quant(H, on, gamma.numpy(), None if beta is None else beta.numpy(), eps,
                                 per_token=False, static_qs=21.5)
    assert np.array_equal(Xq.cpu().numpy(), r["Xq"])
    assert npf(qx)[0] == np.float32(21.5)


@pytest.mark.parametrize("norm", ["ln", "rms"])
@pytest.mark.parametrize("K", [1024, 7168, 8192, 12288])
def test_norm_static_and_calibration(norm, K):
    """Calibration mode (running per-channel max of |v| over batches) and the
    static per-tensor scale taken from it, the OPT-30B-style path (K = 7168
    and 8192: the maxima held in registers, ragged and full chunk sets)."""
    M = 200
    nt = sq.SQ_LAYERNORM if norm == "ln" else sq.SQ_RMSNORM
    on = oracle.LAYERNORM if norm == "ln" else oracle.RMSNORM
    gamma = 1 + 0.1 * rnd(K, 3)
    beta = 0.1 * rnd(K, 4) if norm == "ln" else None
    am = torch.zeros(K, device=DEV)
    ram = np.zeros(K, np.float32)
    for b in range(3):
        H = rnd((M, K), 20 + b, torch.float16)
        H[:, 11] *= 60
        sq.sq_norm_smooth_quant(H.to(DEV), nt, gamma.to(DEV), None if beta is None else beta.to(DEV), 1e-5, True,
                                None, None, None, am, None)
        ram = oracle.norm_smooth_quant(H, on, gamma.numpy(), None if beta is None else beta.numpy(), 1e-5,
                                       quantize=False, absmax=ram)["absmax"]
    assert np.array_equal(npf(am), ram)
    qs_static = torch.empty(1, device=DEV)
    sq.sq_scale_from_absmax(am, qs_static)
    rqs = oracle.scale_from_absmax(ram)
    assert npf(qs_static)[0] == rqs
    H = rnd((M, K), 99, torch.float16, 1.3)  # values beyond the calibrated range clip
    H[:, 11] *= 80
    Xq = torch.empty((M, K), dtype=torch.int8, device=DEV)
    qx = torch.empty(1, device=DEV)
    sq.sq_norm_smooth_quant(H.to(DEV), nt, gamma.to(DEV), None if beta is None else beta.to(DEV), 1e-5, False,
                            qs_static, Xq, qx, None, None)
    r = oracle.norm_smooth_quant(H, on, gamma.numpy(), None if beta is None else beta.numpy(), 1e-5,
                                 per_token=False, static_qs=float(rqs))
    assert np.array_equal(Xq.cpu().numpy(), r["Xq"])
    assert npf(qx)[0] == rqs


# ---------------------------------------------------------------- int8 GEMM
GEMM_SHAPES = [(1, 16, 16), (16, 1024, 1024), (200, 300, 272), (257, 513, 1040), (128, 256, 128),
               (640, 2048, 384), (129, 4096, 1024)]


def rand_i8(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(-127, 128, shape, generator=g, dtype=torch.int32).to(torch.int8)


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_int32_exact(M, N, K):
    Xq, Wq = rand_i8((M, K), M + 1), rand_i8((N, K), N + 2)
    Y = torch.empty((M, N), dtype=torch.int32, device=DEV)
    ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K)
    sq.sq_gemm_w8a8(Xq.to(DEV), Wq.to(DEV), None, None, None, Y, ws)
    torch.cuda.synchronize()
    sq.sq_workspace_status(ws)
    ref = oracle.gemm_i8(Xq.numpy(), Wq.numpy())
    assert np.all(np.abs(ref) < 2 ** 31)
    assert np.array_equal(Y.cpu().numpy().astype(np.int64), ref)


def test_gemm_int32_extremes():
    """All-127 operands at the largest K of the workloads: no overflow."""
    K = 49152
    Xq = torch.full((130, K), 127, dtype=torch.int8)
    Xq[1::2] = -127
    Wq = torch.full((260, K), 127, dtype=torch.int8)
    Wq[5] = -127
    Y = torch.empty((130, 260), dtype=torch.int32, device=DEV)
    sq.sq_gemm_w8a8(Xq.to(DEV), Wq.to(DEV), None, None, None, Y, sq.workspace(0, 130, 260, K))
    y = Y.cpu().numpy().astype(np.int64)
    expect = np.where((np.arange(130)[:, None] % 2 == 1) ^ (np.arange(260)[None, :] == 5), -1, 1) * 792_772_608
    assert np.array_equal(y, expect)


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("per_token,per_channel,with_bias", [(True, True, False), (False, False, False),
                                                             (True, False, True), (False, True, True)])
def test_gemm_dequant(out_dtype, per_token, per_channel, with_bias):
    M, N, K = 300, 520, 1040
    Xq, Wq = rand_i8((M, K), 31), rand_i8((N, K), 32)
    g = torch.Generator().manual_seed(33)
    qx = torch.rand(M if per_token else 1, generator=g) * 100 + 1
    qw = torch.rand(N if per_channel else 1, generator=g) * 5000 + 100
    bias = torch.randn(N, generator=g) if with_bias else None
    Y = torch.empty((M, N), dtype=out_dtype, device=DEV)
    sq.sq_gemm_w8a8(Xq.to(DEV), Wq.to(DEV), qx.to(DEV), qw.to(DEV), None if bias is None else bias.to(DEV), Y,
                    sq.workspace(0, M, N, K))
    acc = oracle.gemm_i8(Xq.numpy(), Wq.numpy())
    y = oracle.dequant(acc, qx.numpy(), qw.numpy(), None if bias is None else bias.numpy())
    terms = np.abs(oracle.dequant(acc, qx.numpy(), qw.numpy()))
    if bias is not None:
        terms = terms + np.abs(bias.numpy().astype(np.float64))[None, :]
    if out_dtype == torch.float32:
        assert_close_f32(Y, y, terms)
    else:
        assert_close_16(Y, y, out_dtype, terms if bias is not None else None)


def test_gemm_strided_output_untouched_tail():
    """Outputs beyond N (ldy > N) keep their contents; rows past M are never written."""
    M, N, K = 131, 200, 256
    Xq, Wq = rand_i8((M, K), 41), rand_i8((N, K), 42)
    big = torch.full((M + 3, 264), 7.0, dtype=torch.bfloat16, device=DEV)
    Y = big[:M, :N]
    qx = torch.full((M,), 50.0, device=DEV)
    qw = torch.full((N,), 400.0, device=DEV)
    sq.sq_gemm_w8a8(Xq.to(DEV), Wq.to(DEV), qx, qw, None, Y, sq.workspace(0, M, N, K))
    b = big.cpu()
    assert torch.all(b[:, N:] == 7.0) and torch.all(b[M:] == 7.0)
    y = oracle.dequant(oracle.gemm_i8(Xq.numpy(), Wq.numpy()), np.full(M, 50, np.float32), np.full(N, 400, np.float32))
    assert_close_16(b[:M, :N].contiguous(), y, torch.bfloat16)


def test_gemm_deterministic():
    M, N, K = 1024, 2048, 2048
    Xq, Wq = rand_i8((M, K), 51).to(DEV), rand_i8((N, K), 52).to(DEV)
    qx = torch.rand(M, device=DEV) + 1
    qw = torch.rand(N, device=DEV) + 100
    ws = sq.workspace(0, M, N, K)
    outs = []
    for _ in range(2):
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
        sq.sq_gemm_w8a8(Xq, Wq, qx, qw, None, Y, ws)
        outs.append(Y)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))


# shapes whose last wave of whole tiles is at most three quarters full, with
# k-loops of 128 blocks or more: that wave is cut by k-blocks (ragged M and K;
# pieces of 4 to 100 k-blocks)
# stream-K plans on 148 SMs: last waves of 104 tiles (129 and 57 k-blocks),
# of 24 tiles (128 k-blocks), and of 104 tiles with the waves 90 % busy
# (64 k-blocks)
SK_SHAPES = [(1029, 7168, 16400), (1029, 7168, 7200), (2560, 4096, 16384), (2048, 6400, 8192)]


@pytest.mark.parametrize("M,N,K", SK_SHAPES)
def test_gemm_stream_k(M, N, K, monkeypatch):
    # stream-K runs on single-CTA tiles: keep the plan off CTA pairs
    monkeypatch.setenv("SQ_GEMM_CTA_PAIRS", "0")
    assert sq.sq_workspace_size(sq.SQ_OP_GEMM, M, N, K) > 256, "the plan was expected to cut this shape"
    Xq, Wq = rand_i8((M, K), M + 3), rand_i8((N, K), N + 4)
    Xd, Wd = Xq.to(DEV), Wq.to(DEV)
    ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K)
    Y = torch.empty((M, N), dtype=torch.int32, device=DEV)
    sq.sq_gemm_w8a8(Xd, Wd, None, None, None, Y, ws)
    sq.sq_workspace_status(ws)
    # whole tiles (a workspace with no room for the split) agree bit for bit
    Yw = torch.empty_like(Y)
    sq.sq_gemm_w8a8(Xd, Wd, None, None, None, Yw, torch.zeros(256, dtype=torch.uint8, device=DEV))
    assert torch.equal(Y, Yw)
    Np = (N + 7) // 8 * 8
    Wp = torch.zeros((Np, K), dtype=torch.int8, device=DEV)
    Wp[:N] = Wd
    assert torch.equal(Y, torch._int_mm(Xd, Wp.t())[:, :N])
    rows = sorted({0, 127, 128, M // 2, M - 1})
    acc = oracle.gemm_i8(Xq[rows].numpy(), Wq.numpy())
    assert np.array_equal(Y[rows].cpu().numpy().astype(np.int64), acc)
    # the counters are back at zero: a second call on the same workspace agrees
    Y2 = torch.empty_like(Y)
    sq.sq_gemm_w8a8(Xd, Wd, None, None, None, Y2, ws)
    assert torch.equal(Y, Y2)
    # dequantised bf16 with per-token and per-channel scales and a bias
    g = torch.Generator().manual_seed(M + N + K)
    qx = torch.rand(M, generator=g) * 100 + 1
    qw = torch.rand(N, generator=g) * 5000 + 100
    bias = torch.randn(N, generator=g)
    Yb = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    sq.sq_gemm_w8a8(Xd, Wd, qx.to(DEV), qw.to(DEV), bias.to(DEV), Yb, ws)
    y = oracle.dequant(acc, qx.numpy()[rows], qw.numpy(), bias.numpy())
    terms = np.abs(oracle.dequant(acc, qx.numpy()[rows], qw.numpy())) + np.abs(bias.numpy().astype(np.float64))[None]
    assert_close_16(Yb[rows].contiguous(), y, torch.bfloat16, terms)


def test_stream_k_workspace_recovers_after_a_timeout(monkeypatch):
    """A stream-K GEMM that gave up part-way leaves its arrival counters
    counted in. The failure is made on the host (no GPU fault): after a
    normal call, garbage counts and a timeout code are written into the
    workspace; sq_workspace_status reports the timeout and clears the
    counters, and the next call on the same workspace is exact."""
    monkeypatch.setenv("SQ_GEMM_CTA_PAIRS", "0")
    M, N, K = 1029, 7168, 7200
    Xq, Wq = rand_i8((M, K), 91), rand_i8((N, K), 92)
    Xd, Wd = Xq.to(DEV), Wq.to(DEV)
    ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K)
    Y = torch.empty((M, N), dtype=torch.int32, device=DEV)
    sq.sq_gemm_w8a8(Xd, Wd, None, None, None, Y, ws)
    sq.sq_workspace_status(ws)
    hdr = ws[:256].view(torch.int32)
    cnt_bytes = int(hdr[3].item())
    assert cnt_bytes > 0 and cnt_bytes % 256 == 0  # the counters' region was recorded
    ws[256:256 + cnt_bytes].view(torch.int32).fill_(3)  # pieces counted in, never completed
    hdr[0] = 0x6E1
    with pytest.raises(sq.SqError):
        sq.sq_workspace_status(ws)
    assert int(ws[256:256 + cnt_bytes].view(torch.int32).abs().sum().item()) == 0
    assert int(hdr[0].item()) == 0
    Y2 = torch.empty_like(Y)
    sq.sq_gemm_w8a8(Xd, Wd, None, None, None, Y2, ws)
    sq.sq_workspace_status(ws)
    assert torch.equal(Y, Y2)
    rows = [0, 511, 1028]
    assert np.array_equal(Y2[rows].cpu().numpy().astype(np.int64), oracle.gemm_i8(Xq[rows].numpy(), Wq.numpy()))


def test_bounded_wait_timeout():
    """A wait that nothing completes gives up after its limit, the status word
    says so (SQ_ERR_TIMEOUT on the host), and the context stays usable."""
    ws = sq.workspace(sq.SQ_OP_GEMM, 1, 16, 16)
    sq.sq_selftest_wait_timeout(ws, 20_000_000)  # 20 ms
    with pytest.raises(sq.SqError) as e:
        sq.sq_workspace_status(ws)
    assert e.value.status == 5
    sq.sq_workspace_status(ws)  # read and cleared
    Xq, Wq = rand_i8((130, 256), 7), rand_i8((200, 256), 8)
    Y = torch.empty((130, 200), dtype=torch.int32, device=DEV)
    sq.sq_gemm_w8a8(Xq.to(DEV), Wq.to(DEV), None, None, None, Y, ws)
    assert np.array_equal(Y.cpu().numpy().astype(np.int64), oracle.gemm_i8(Xq.numpy(), Wq.numpy()))


@pytest.mark.parametrize("M,N,K", [(4096, 36864, 12288), (1024, 28672, 7168), (2048, 16384, 4096),
                                   (1024, 7168, 28672)])
@pytest.mark.parametrize("pairs", ["", "0"])
def test_gemm_full_size_sampled(M, N, K, pairs, monkeypatch):
    """Full-size shapes in the launch configuration the benchmark times (and
    on single-CTA tiles): all outputs against torch._int_mm (a library
    cross-check, test only) and sampled rows against the oracle."""
    if pairs:
        monkeypatch.setenv("SQ_GEMM_CTA_PAIRS", pairs)
    else:
        monkeypatch.delenv("SQ_GEMM_CTA_PAIRS", raising=False)
    g = torch.Generator(device=DEV).manual_seed(M + N)
    Xq = torch.randint(-127, 128, (M, K), generator=g, device=DEV, dtype=torch.int8)
    Wq = torch.randint(-127, 128, (N, K), generator=g, device=DEV, dtype=torch.int8)
    Y = torch.empty((M, N), dtype=torch.int32, device=DEV)
    ws = sq.workspace(0, M, N, K)
    sq.sq_gemm_w8a8(Xq, Wq, None, None, None, Y, ws)
    ref = torch._int_mm(Xq, Wq.t())
    assert torch.equal(Y, ref)
    rows = [0, 1, 127, 128, M // 2 + 3, M - 1]
    Xs = Xq[rows].cpu().numpy()
    acc = oracle.gemm_i8(Xs, Wq.cpu().numpy())
    assert np.array_equal(Y[rows].cpu().numpy().astype(np.int64), acc)
    del Xq, Wq, Y, ref
    torch.cuda.empty_cache()


# ---------------------------------------------------------------- LLM.int8() decomposition
def _llm_case(M, K, N, n_out, seed, dtype=torch.float16):
    d = inputs.c4_llmint8(device="cpu", M=M, K=K, N=N, n_out=n_out, seed=seed)
    return d["X"].to(dtype), d["W"].to(dtype), d["dims"]


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("M,K,N,n_out", [(256, 512, 384, 3), (300, 1024, 520, 6), (64, 256, 128, 0)])
def test_llmint8_steps_and_matmul(dtype, M, K, N, n_out):
    X, W, dims = _llm_case(M, K, N, n_out, seed=M + n_out, dtype=dtype)
    Xd, Wd = X.to(DEV), W.to(DEV)
    idx = torch.empty(K, dtype=torch.int32, device=DEV)
    n = torch.empty(1, dtype=torch.int32, device=DEV)
    wsd = sq.workspace(sq.SQ_OP_LLMINT8_DETECT, M, N, K)
    sq.sq_llmint8_detect(Xd, 6.0, 0.0, idx, n, wsd)
    ridx = oracle.llmint8_outliers(X, 6.0, 0.0)
    assert ridx.tolist() == dims.tolist()
    nn_ = int(n.item())
    assert nn_ == ridx.size and idx[:nn_].cpu().numpy().tolist() == ridx.tolist()
    Xq = torch.empty((M, K), dtype=torch.int8, device=DEV)
    qx = torch.empty(M, device=DEV)
    sq.sq_llmint8_quant_rows(Xd, idx, n, Xq, qx)
    rXq, rqx = oracle.llmint8_quant_rows(X, ridx)
    assert np.array_equal(Xq.cpu().numpy(), rXq) and np.array_equal(npf(qx), rqx)
    Wq = torch.empty((N, K), dtype=torch.int8, device=DEV)
    qw = torch.empty(N, device=DEV)
    sq.sq_llmint8_quant_weight(Wd, idx, n, Wq, qw)
    rWq, rqw = oracle.llmint8_quant_weight(W, ridx)
    assert np.array_equal(Wq.cpu().numpy(), rWq) and np.array_equal(npf(qw), rqw)
    # the fused call
    st = sq.llmint8_weight_state(Wd)
    Y = torch.empty((M, N), dtype=dtype, device=DEV)
    idx2 = torch.empty(K, dtype=torch.int32, device=DEV)
    n2 = torch.empty(1, dtype=torch.int32, device=DEV)
    ws = sq.workspace(sq.SQ_OP_LLMINT8, M, N, K)
    sq.sq_llmint8_matmul(Xd, st, 6.0, 0.0, Y, idx2, n2, ws)
    torch.cuda.synchronize()
    sq.sq_workspace_status(ws)
    assert int(n2.item()) == ridx.size and idx2[:ridx.size].cpu().numpy().tolist() == ridx.tolist()
    assert np.array_equal(st["Wq"].cpu().numpy(), rWq) and np.array_equal(npf(st["qs_w"]), rqw)
    acc = oracle.gemm_i8(rXq, rWq)
    y = oracle.llmint8_combine(acc, rqx, rqw, X, W, ridx)
    Xf, Wf = npf(X).astype(np.float64), npf(W).astype(np.float64)
    terms = np.abs(oracle.dequant(acc, rqx, rqw)) + np.abs(Xf[:, ridx]) @ np.abs(Wf[:, ridx]).T
    assert_close_16(Y, y, dtype, terms)
    # second call, same O: the cached weight is reused and the result repeats
    Y2 = torch.empty_like(Y)
    sq.sq_llmint8_matmul(Xd, st, 6.0, 0.0, Y2, idx2, n2, ws)
    assert int(ws[4:8].view(torch.int32).item()) == 0  # O unchanged
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))


@pytest.mark.parametrize("keep_wo", [True, False])
def test_llmint8_cache_follows_outlier_set(keep_wo):
    """The cached int8 weight (and, when the state keeps it, the gathered fp32
    outlier channels of W) follows O as it changes from call to call."""
    M, K, N = 128, 512, 256
    X1, W, _ = _llm_case(M, K, N, 3, seed=1)
    X2, _, _ = _llm_case(M, K, N, 5, seed=2)
    Wd = W.to(DEV)
    st = sq.llmint8_weight_state(Wd, keep_wo=keep_wo)
    ws = sq.workspace(sq.SQ_OP_LLMINT8, M, N, K)
    idx = torch.empty(K, dtype=torch.int32, device=DEV)
    n = torch.empty(1, dtype=torch.int32, device=DEV)
    for X in (X1, X2, X1):
        Y = torch.empty((M, N), dtype=torch.float16, device=DEV)
        sq.sq_llmint8_matmul(X.to(DEV), st, 6.0, 0.0, Y, idx, n, ws)
        ridx = oracle.llmint8_outliers(X, 6.0, 0.0)
        assert int(ws[4:8].view(torch.int32).item()) == 1  # O changed each time
        rWq, rqw = oracle.llmint8_quant_weight(W, ridx)
        assert np.array_equal(st["Wq"].cpu().numpy(), rWq)
        rXq, rqx = oracle.llmint8_quant_rows(X, ridx)
        acc = oracle.gemm_i8(rXq, rWq)
        y = oracle.llmint8_combine(acc, rqx, rqw, X, W, ridx)
        Xf, Wf = npf(X).astype(np.float64), npf(W).astype(np.float64)
        terms = np.abs(oracle.dequant(acc, rqx, rqw)) + np.abs(Xf[:, ridx]) @ np.abs(Wf[:, ridx]).T
        assert_close_16(Y, y, torch.float16, terms)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("n_out,thr", [(40, 6.0), (0, 3.0)])
def test_llmint8_beyond_compact_cap(dtype, n_out, thr):
    """|O| above the 32 outlier columns the epilogue keeps as compact fp32
    copies: 40 planted dimensions at the 6.0 threshold, and a threshold of 3.0
    on N(0, 1) data (about half of all columns). The GEMM epilogue then reads
    the 16-bit operands of every outlier column directly."""
    M, K, N = 256, 512, 384
    X, W, dims = _llm_case(M, K, N, n_out, seed=77 + n_out, dtype=dtype)
    ridx = oracle.llmint8_outliers(X, thr, 0.0)
    assert ridx.size > 32
    if n_out:
        assert ridx.tolist() == dims.tolist()
    Xd = X.to(DEV)
    st = sq.llmint8_weight_state(W.to(DEV))
    Y = torch.empty((M, N), dtype=dtype, device=DEV)
    idx = torch.empty(K, dtype=torch.int32, device=DEV)
    n = torch.empty(1, dtype=torch.int32, device=DEV)
    ws = sq.workspace(sq.SQ_OP_LLMINT8, M, N, K)
    sq.sq_llmint8_matmul(Xd, st, thr, 0.0, Y, idx, n, ws)
    torch.cuda.synchronize()
    sq.sq_workspace_status(ws)
    assert int(n.item()) == ridx.size and idx[:ridx.size].cpu().numpy().tolist() == ridx.tolist()
    rXq, rqx = oracle.llmint8_quant_rows(X, ridx)
    rWq, rqw = oracle.llmint8_quant_weight(W, ridx)
    assert np.array_equal(st["Wq"].cpu().numpy(), rWq) and np.array_equal(npf(st["qs_w"]), rqw)
    acc = oracle.gemm_i8(rXq, rWq)
    y = oracle.llmint8_combine(acc, rqx, rqw, X, W, ridx)
    Xf, Wf = npf(X).astype(np.float64), npf(W).astype(np.float64)
    terms = np.abs(oracle.dequant(acc, rqx, rqw)) + np.abs(Xf[:, ridx]) @ np.abs(Wf[:, ridx]).T
    assert_close_16(Y, y, dtype, terms)


def test_llmint8_detect_counters_reset():
    """The detection's arrival counters are back at zero after every call:
    many calls in a row on one workspace, of several sizes, all exact."""
    ws = sq.workspace(sq.SQ_OP_LLMINT8_DETECT, 2048, 0, 4096)
    for i, (M, K, n_out) in enumerate([(2048, 4096, 6), (300, 1024, 3), (1, 256, 0), (700, 4096, 9), (2048, 4096, 6)]):
        X, _, dims = _llm_case(M, K, 16, n_out, seed=500 + i)
        idx = torch.full((K,), -1, dtype=torch.int32, device=DEV)
        n = torch.full((1,), -1, dtype=torch.int32, device=DEV)
        sq.sq_llmint8_detect(X.to(DEV), 6.0, 0.0, idx, n, ws)
        torch.cuda.synchronize()
        assert int(n.item()) == n_out and idx[:n_out].cpu().tolist() == dims.tolist()
    hdr = ws[:256].view(torch.int32).cpu()
    assert int(hdr[2]) == 0  # the count of finished column groups


def test_llmint8_detect_wide_rows():
    """Rows of more than 32 column groups of 256 (more mask words than the
    last group's block takes in one pass) with a ragged last group: outlier
    columns at both ends, on either side of column 8192 and in the last
    group, found in ascending order on one workspace call after call, the
    second call wider than the first: the arrival counters sit at the same
    bytes for every K, so the first call's masks and counts (left behind,
    not cleared) are never read as the second call's counters."""
    ws = sq.workspace(sq.SQ_OP_LLMINT8_DETECT, 300, 0, 16392)
    for i, (M, K, cols) in enumerate([(300, 8200, [0, 17, 8191, 8192, 8199]),
                                      (129, 16392, [5, 4000, 8192, 12000, 16384, 16391]),
                                      (300, 8200, [1, 8198])]):
        X = rnd((M, K), 900 + i, torch.float16).clamp(-5, 5)
        for j, c in enumerate(cols):
            X[(7 * j) % M, c] = 6.5 + j
        idx = torch.full((K,), -1, dtype=torch.int32, device=DEV)
        n = torch.full((1,), -1, dtype=torch.int32, device=DEV)
        sq.sq_llmint8_detect(X.to(DEV), 6.0, 0.0, idx, n, ws)
        torch.cuda.synchronize()
        ref = oracle.llmint8_outliers(X, 6.0, 0.0).tolist()
        assert ref == cols
        assert int(n.item()) == len(cols) and idx[:len(cols)].cpu().tolist() == cols
    assert int(ws[:256].view(torch.int32)[2].item()) == 0  # the count of finished column groups


def test_llmint8_min_ratio():
    M, K = 200, 256
    X = rnd((M, K), 61, torch.float16).clamp(-5, 5)
    X[:13, 10] = 7.0   # 13/200 = 0.065 > 0.06
    X[:12, 20] = -9.0  # 12/200 = 0.06, not > 0.06
    X[:1, 30] = 6.5
    idx = torch.empty(K, dtype=torch.int32, device=DEV)
    n = torch.empty(1, dtype=torch.int32, device=DEV)
    ws = sq.workspace(sq.SQ_OP_LLMINT8_DETECT, M, 0, K)
    for mr in (0.0, 0.06, 0.1):
        sq.sq_llmint8_detect(X.to(DEV), 6.0, mr, idx, n, ws)
        ref = oracle.llmint8_outliers(X, 6.0, mr).tolist()
        assert idx[: int(n.item())].cpu().tolist() == ref


def test_llmint8_full_size_sampled():
    """The 6.7B-shaped case ([2048,4096] x [16384,4096]) in the benchmark's
    launch configuration; outlier set exact, sampled rows against the oracle."""
    d = inputs.c4_llmint8(device=DEV)
    X, W = d["X"], d["W"]
    M, K = X.shape
    N = W.shape[0]
    st = sq.llmint8_weight_state(W)
    Y = torch.empty((M, N), dtype=torch.float16, device=DEV)
    idx = torch.empty(K, dtype=torch.int32, device=DEV)
    n = torch.empty(1, dtype=torch.int32, device=DEV)
    ws = sq.workspace(sq.SQ_OP_LLMINT8, M, N, K)
    sq.sq_llmint8_matmul(X, st, 6.0, 0.0, Y, idx, n, ws)
    torch.cuda.synchronize()
    Xc, Wc = X.cpu(), W.cpu()
    ridx = oracle.llmint8_outliers(Xc, 6.0, 0.0)
    assert ridx.tolist() == d["dims"].tolist()
    assert idx[: int(n.item())].cpu().tolist() == ridx.tolist()
    rWq, rqw = oracle.llmint8_quant_weight(Wc, ridx)
    assert np.array_equal(st["qs_w"].cpu().numpy(), rqw)
    assert np.array_equal(st["Wq"].cpu().numpy(), rWq)
    rows = np.array([0, 5, 511, 1024, 2047])
    rXq, rqx = oracle.llmint8_quant_rows(Xc[rows], ridx)
    acc = oracle.gemm_i8(rXq, rWq)
    y = oracle.llmint8_combine(acc, rqx, rqw, Xc[rows], Wc, ridx)
    Xf, Wf = npf(Xc[rows]).astype(np.float64), npf(Wc).astype(np.float64)
    terms = np.abs(oracle.dequant(acc, rqx, rqw)) + np.abs(Xf[:, ridx]) @ np.abs(Wf[:, ridx]).T
    assert_close_16(Y[rows].contiguous(), y, torch.float16, terms)


# ---------------------------------------------------------------- edges
def test_empty_inputs():
    ws = sq.workspace(0, 1, 16, 16)
    e = torch.empty((0, 16), dtype=torch.int8, device=DEV)
    W = rand_i8((16, 16), 1).to(DEV)
    Y = torch.empty((0, 16), dtype=torch.bfloat16, device=DEV)
    sq.sq_gemm_w8a8(e, W, torch.ones(1, device=DEV), torch.ones(1, device=DEV), None, Y, ws)
    xmax = torch.full((16,), 3.0, device=DEV)
    sq.sq_calib_absmax(torch.empty((0, 16), dtype=torch.bfloat16, device=DEV), xmax)
    assert torch.all(xmax == 3.0)
    n = torch.full((1,), 99, dtype=torch.int32, device=DEV)
    idx = torch.empty(16, dtype=torch.int32, device=DEV)
    sq.sq_llmint8_detect(torch.empty((0, 16), dtype=torch.float16, device=DEV), 6.0, 0.0, idx, n,
                         sq.workspace(3, 0, 0, 16))
    assert int(n.item()) == 0


def test_errors_raise():
    with pytest.raises(sq.SqError) as ei:
        sq.sq_gemm_w8a8(torch.zeros((4, 24), dtype=torch.int8, device=DEV),
                        torch.zeros((4, 24), dtype=torch.int8, device=DEV), None, None, None,
                        torch.empty((4, 4), dtype=torch.int32, device=DEV), sq.workspace(0, 4, 4, 24))
    assert ei.value.status == 2


# ---------------------------------------------------------------- FP8 variant
def _fp8_bits(t):
    return t.cpu().numpy().view(np.uint8)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("per_row,with_s", [(True, True), (True, False), (False, True)])
@pytest.mark.parametrize("K", [1024, 4112, 20480])
def test_quantize_fp8(dtype, per_row, with_s, K):
    """E4M3 codes and scales of weights (x s) and activations (/ s), bit for bit."""
    M = 131 if K > 4112 else 517
    X = rnd((M, K), K + 21, dtype, 0.05)
    X[3, 5] = 0.0
    s = torch.rand(K, generator=torch.Generator().manual_seed(22)) * 30 + 0.05 if with_s else None
    Q = torch.empty((M, K), dtype=torch.uint8, device=DEV)
    qs = torch.empty(M if per_row else 1, device=DEV)
    ws = sq.workspace(sq.SQ_OP_QUANT_WEIGHT, 0, M, K)
    Xd, sd = X.to(DEV), None if s is None else s.to(DEV)
    sq.sq_quantize_weight_fp8(Xd, sd, per_row, Q, qs, ws)
    rQ, rqs = oracle.quantize_fp8(X.float().numpy(), None if s is None else s.numpy(), s_div=False, per_row=per_row)
    assert np.array_equal(npf(qs), rqs)
    assert np.array_equal(_fp8_bits(Q), rQ)
    sq.sq_quantize_act_fp8(Xd, sd, per_row, None, Q, qs, ws)
    rQ, rqs = oracle.quantize_fp8(X.float().numpy(), None if s is None else s.numpy(), s_div=True, per_row=per_row)
    assert np.array_equal(npf(qs), rqs)
    assert np.array_equal(_fp8_bits(Q), rQ)


def _fp8_codes(shape, seed):
    """Random finite E4M3 codes (NaN codes 0x7F / 0xFF redrawn)."""
    g = torch.Generator().manual_seed(seed)
    b = torch.randint(0, 256, shape, generator=g, dtype=torch.int32)
    b = torch.where((b & 0x7F) == 0x7F, b ^ 0x01, b)
    return b.to(torch.uint8)


def _fp8_tol(A, B, rows):
    """|error| bound of an fp32 accumulation of K products: K * 2^-23 * sum |a b|."""
    av = np.vectorize(oracle.e4m3_value)
    a = np.abs(av(A[rows].numpy()))
    b = np.abs(av(B.numpy()))
    return a @ b.T * (A.shape[1] * 2.0 ** -23)


@pytest.mark.parametrize("M,N,K", [(16, 256, 64), (200, 300, 272), (257, 513, 1040), (129, 4096, 1024)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_fp8(M, N, K, out_dtype):
    """FP8 products are exact in fp32; the tensor core sums them in fp32, so the
    result is within K * 2^-23 * sum|a b| of the exact sum (fp32 out), plus
    one rounding to bf16."""
    A, B = _fp8_codes((M, K), M + 5), _fp8_codes((N, K), N + 6)
    g = torch.Generator().manual_seed(M + N)
    qx = torch.rand(M, generator=g) * 10 + 1
    qw = torch.rand(N, generator=g) * 10 + 1
    bias = torch.randn(N, generator=g)
    Y = torch.empty((M, N), dtype=out_dtype, device=DEV)
    sq.sq_gemm_fp8(A.to(DEV), B.to(DEV), qx.to(DEV), qw.to(DEV), bias.to(DEV), Y, sq.workspace(0, M, N, K))
    rows = sorted({0, 1, M // 2, M - 1})
    acc = oracle.gemm_fp8(A.numpy(), B.numpy(), rows=rows)
    y = oracle.dequant_f64(acc, qx.numpy()[rows], qw.numpy(), bias.numpy())
    d = (qx.numpy()[rows].astype(np.float64)[:, None] * qw.numpy().astype(np.float64)[None, :])
    tol = _fp8_tol(A, B, rows) / d + 1e-6 * (np.abs(y) + 1e-30)
    got = Y[rows].float().cpu().numpy().astype(np.float64)
    if out_dtype == torch.bfloat16:
        tol = tol + np.abs(y) * 2.0 ** -8
    assert np.all(np.abs(got - y) <= tol)


def test_fp8_path_end_to_end():
    """Quantise X (/ s) and W (x s) to E4M3 with the library, multiply, and
    compare with the oracle's chain from the same inputs."""
    M, N, K = 256, 512, 1024
    X = rnd((M, K), 70, torch.bfloat16, 1.0)
    X[:, 7] *= 40
    W = rnd((N, K), 71, torch.bfloat16, 0.02)
    s = torch.rand(K, generator=torch.Generator().manual_seed(72)) * 4 + 0.25
    Xq = torch.empty((M, K), dtype=torch.uint8, device=DEV)
    Wq = torch.empty((N, K), dtype=torch.uint8, device=DEV)
    qx, qw = torch.empty(M, device=DEV), torch.empty(N, device=DEV)
    sq.sq_quantize_act_fp8(X.to(DEV), s.to(DEV), True, None, Xq, qx)
    sq.sq_quantize_weight_fp8(W.to(DEV), s.to(DEV), True, Wq, qw)
    Y = torch.empty((M, N), dtype=torch.float32, device=DEV)
    sq.sq_gemm_fp8(Xq, Wq, qx, qw, None, Y, sq.workspace(0, M, N, K))
    rXq, rqx = oracle.quantize_fp8(X.float().numpy(), s.numpy(), s_div=True)
    rWq, rqw = oracle.quantize_fp8(W.float().numpy(), s.numpy(), s_div=False)
    assert np.array_equal(_fp8_bits(Xq), rXq) and np.array_equal(_fp8_bits(Wq), rWq)
    rows = [0, 100, 255]
    y = oracle.dequant_f64(oracle.gemm_fp8(rXq, rWq, rows=rows), rqx[rows], rqw)
    tol = _fp8_tol(torch.from_numpy(rXq), torch.from_numpy(rWq), rows) / (
        rqx[rows].astype(np.float64)[:, None] * rqw.astype(np.float64)[None, :]) + 1e-6 * np.abs(y)
    assert np.all(np.abs(Y[rows].cpu().numpy().astype(np.float64) - y) <= tol)
    # and the FP8 W8A8 product approximates X W^T
    ref = X.float().numpy().astype(np.float64)[rows] @ W.float().numpy().astype(np.float64).T
    assert np.max(np.abs(y - ref)) / np.max(np.abs(ref)) < 0.1


# ---------------------------------------------------------------- batched int8 GEMM (attention)
@pytest.mark.parametrize("batch,M,N,K", [(3, 200, 300, 272), (4, 128, 256, 128), (2, 1, 16, 16), (16, 257, 130, 1040)])
def test_bmm_int32_exact(batch, M, N, K):
    """Every problem exact against torch._int_mm (library cross-check) and
    sampled rows against the oracle; problems never bleed into each other
    (M, N not multiples of the tile)."""
    A = torch.stack([rand_i8((M, K), 90 + b) for b in range(batch)])
    B = torch.stack([rand_i8((N, K), 190 + b) for b in range(batch)])
    Ad, Bd = A.to(DEV), B.to(DEV)
    Y = torch.empty((batch, M, N), dtype=torch.int32, device=DEV)
    sq.sq_bmm_w8a8(Ad, Bd, None, None, Y, sq.workspace(0, M, N, K))
    if M > 16 and N % 8 == 0:
        for b in range(batch):
            assert torch.equal(Y[b], torch._int_mm(Ad[b], Bd[b].t()))
    rows = sorted({0, M // 2, M - 1})
    ref = oracle.bmm_i8(A.numpy(), B.numpy(), rows=rows)
    assert np.array_equal(Y[:, rows].cpu().numpy().astype(np.int64), ref)


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_bmm_attention(out_dtype):
    """QK^T with per-(head, token) scales and PV with P per row and V^T per
    (head, channel), quantised by the library, against the oracle's chain."""
    H, T, d = 4, 256, 128
    Q, Kt, V = (rnd((H, T, d), 95 + i, torch.bfloat16) for i in range(3))
    Qq, Kq = torch.empty((H, T, d), dtype=torch.int8, device=DEV), torch.empty((H, T, d), dtype=torch.int8, device=DEV)
    qq, qk = torch.empty((H, T), device=DEV), torch.empty((H, T), device=DEV)
    sq.sq_quantize_act(Q.to(DEV).view(H * T, d), None, True, None, Qq.view(H * T, d), qq.view(-1))
    sq.sq_quantize_act(Kt.to(DEV).view(H * T, d), None, True, None, Kq.view(H * T, d), qk.view(-1))
    S = torch.empty((H, T, T), dtype=out_dtype, device=DEV)
    sq.sq_bmm_w8a8(Qq, Kq, qq, qk, S, sq.workspace(0, T, T, d))
    rq = [oracle.quantize_act(Q[h].float().numpy(), None, per_token=True) for h in range(H)]
    rk = [oracle.quantize_act(Kt[h].float().numpy(), None, per_token=True) for h in range(H)]
    assert np.array_equal(Qq.cpu().numpy(), np.stack([r[0] for r in rq]))
    rows = [0, 17, 255]
    ys = oracle.bmm_dequant(oracle.bmm_i8(np.stack([r[0] for r in rq]), np.stack([r[0] for r in rk]), rows=rows),
                            [r[1] for r in rq], [r[1] for r in rk], rows=rows)
    for h in range(H):
        if out_dtype == torch.float32:
            assert_close_f32(S[h, rows].contiguous(), ys[h], np.abs(ys[h]))
        else:
            assert_close_16(S[h, rows].contiguous(), ys[h], out_dtype)
    # PV: P per row, V^T per (head, channel)
    P = torch.softmax(S.float() / 16.0, dim=-1).to(torch.bfloat16)
    Vt = V.to(DEV).transpose(1, 2).contiguous()  # [H, d, T]
    Pq, Vq = torch.empty((H, T, T), dtype=torch.int8, device=DEV), torch.empty((H, d, T), dtype=torch.int8, device=DEV)
    qp, qv = torch.empty((H, T), device=DEV), torch.empty((H, d), device=DEV)
    sq.sq_quantize_act(P.view(H * T, T), None, True, None, Pq.view(H * T, T), qp.view(-1))
    sq.sq_quantize_act(Vt.view(H * d, T), None, True, None, Vq.view(H * d, T), qv.view(-1))
    O = torch.empty((H, T, d), dtype=out_dtype, device=DEV)
    sq.sq_bmm_w8a8(Pq, Vq, qp, qv, O, sq.workspace(0, T, d, T))
    acc = oracle.bmm_i8(Pq.cpu().numpy(), Vq.cpu().numpy(), rows=rows)
    yo = oracle.bmm_dequant(acc, qp.cpu().numpy(), qv.cpu().numpy(), rows=rows)
    for h in range(H):
        if out_dtype == torch.float32:
            assert_close_f32(O[h, rows].contiguous(), yo[h], np.abs(yo[h]))
        else:
            assert_close_16(O[h, rows].contiguous(), yo[h], out_dtype)


# ---------------------------------------------------------------- the benchmark's whole step
def test_every_row_step_against_oracle():
    """The Qwen3-0.6B-shaped layer with every row in one step (on its streams,
    captured in a CUDA graph) against the oracle on the same inputs: the
    weight side in full, the token side on sampled rows. Stages after a 16-bit
    GEMM output take the device's output as their input, so each stage is held
    to its own bar."""
    import c2_every_row as bench

    dev = torch.device(DEV, 0)
    L = bench.Layer(dev)
    L.step()
    torch.cuda.synchronize()
    eager = [y.clone() for y in L.outputs()]
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        L.step()  # warm-up on the capture stream
    torch.cuda.synchronize()
    with torch.cuda.graph(graph, stream=stream):
        L.step()
    for _ in range(2):
        for y in L.outputs():
            y.zero_()
        graph.replay()
        torch.cuda.synchronize()
        for a, b in zip(eager, L.outputs()):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))

    d = {k: v for k, v in L.d.items() if torch.is_tensor(v)}
    d = {k: v.cpu() for k, v in d.items()}
    W = {k: v.cpu() for k, v in L.d["W"].items()}
    eps, alpha, I = L.d["eps"], L.d["alpha"], L.I
    rows = [0, 1, 127, 128, 1029, bench.M_TOKENS - 1]
    # calibration input, maxima, smoothing factors, folded gamma
    s, gp = {}, {}
    V16 = {}
    for k, w in (("attn", "qkv"), ("mlp", "gateup")):
        V = oracle.norm_smooth_quant(d["h_" + k], oracle.RMSNORM, d["gamma_" + k].numpy(), None, eps,
                                     quantize=False, want_v=True)["V"]
        V16[k] = torch.from_numpy(V).to(torch.bfloat16)
        assert np.array_equal(npu16(L.V[k]), npu16(V16[k]))
        xmax = oracle.col_absmax(V16[k])
        assert np.array_equal(npf(L.xmax[k]), xmax)
        wmax = oracle.col_absmax(W[w])
        assert np.array_equal(npf(L.wmax[k]), wmax)
        s[k] = oracle.smooth_scales(xmax, wmax, alpha)
        assert np.array_equal(npf(L.s[k]), s[k])
        gp[k], _ = oracle.fold_norm(d["gamma_" + k].numpy(), None, s[k])
        assert np.array_equal(npf(L.gp[k]), gp[k])
    # weight side: down_proj's factors s_down come from the set-up's
    # calibration pass, checked stage by stage on every channel: the norm
    # output and its per-token int8 (bit-exact), the int8 gate/up weight
    # (bit-exact), the calibration GEMM's bf16 output (within one ulp, on
    # sampled rows), then, from the device's own bf16 output, the SwiGLU
    # maxima, down_proj's weight maxima and s_down (bit-exact)
    c = L.calib
    Vc = oracle.norm_smooth_quant(d["h_calib"], oracle.RMSNORM, d["gamma_mlp"].numpy(), None, eps,
                                  quantize=False, want_v=True)["V"]
    Vc16 = torch.from_numpy(Vc).to(torch.bfloat16)
    assert np.array_equal(npu16(c["V"]), npu16(Vc16))
    Xc, qc = oracle.quantize_act(Vc16.float().numpy(), None, per_token=True)
    assert np.array_equal(c["Xq"].cpu().numpy(), Xc) and np.array_equal(npf(c["qx"]), qc)
    Wc, qwc = oracle.quantize_weight(W["gateup"], True)
    assert np.array_equal(c["Wq"].cpu().numpy(), Wc) and np.array_equal(npf(c["qw"]), qwc)
    assert_close_16(c["Y"][rows], oracle.dequant(oracle.gemm_i8(Xc[rows], Wc), qc[rows], qwc), torch.bfloat16)
    hmax = oracle.act_quant(npf(c["Y"]), oracle.SWIGLU, quantize=False, absmax=np.zeros(I, np.float32))["absmax"]
    assert np.array_equal(npf(c["hmax"]), hmax)
    wmax_down = oracle.col_absmax(W["down"])
    assert np.array_equal(npf(c["wmax"]), wmax_down)
    s_down = oracle.smooth_scales(hmax, wmax_down, alpha)
    assert np.array_equal(npf(L.s_down), s_down)
    up_f, _ = oracle.fold_prev_linear(W["gateup"][I:], s_down)
    ref_w = {
        "qkv": oracle.fold_weight(W["qkv"], s["attn"]),
        "gateup": np.concatenate([oracle.fold_weight(W["gateup"][:I], s["mlp"]), oracle.fold_weight(up_f, s["mlp"])]),
        "o": oracle.f32(W["o"]),
        "down": oracle.fold_weight(W["down"], s_down),
    }
    Wq, qw = {}, {}
    for w, Wp in ref_w.items():
        Wq[w], qw[w] = oracle.quantize_weight(Wp, True)
        assert np.array_equal(L.Wq[w].cpu().numpy(), Wq[w]), w
        assert np.array_equal(npf(L.qw[w]), qw[w]), w
    # token side on sampled rows
    for k, w in (("attn", "qkv"), ("mlp", "gateup")):
        r = oracle.norm_smooth_quant(d["h_" + k][rows], oracle.RMSNORM, gp[k], None, eps, True)
        assert np.array_equal(L.Xq[k][rows].cpu().numpy(), r["Xq"])
        assert np.array_equal(npf(L.qx[k][rows]), r["qs"])
        y = oracle.dequant(oracle.gemm_i8(r["Xq"], Wq[w]), r["qs"], qw[w])
        assert_close_16(L.Y[w][rows], y, torch.bfloat16)
    xo, so = L.act_in["o"]
    xs, ss = xo[rows].cpu().numpy(), npf(so[rows])
    assert_close_16(L.Y["o"][rows], oracle.dequant(oracle.gemm_i8(xs, Wq["o"]), ss, qw["o"]), torch.bfloat16)
    a = oracle.act_quant(npf(L.Y["gateup"][rows]), oracle.SWIGLU)
    assert np.array_equal(L.Xq_down[rows].cpu().numpy(), a["Xq"])
    assert np.array_equal(npf(L.qx_down[rows]), a["qs"])
    y = oracle.dequant(oracle.gemm_i8(a["Xq"], Wq["down"]), a["qs"], qw["down"])
    assert_close_16(L.Y["down"][rows], y, torch.bfloat16)
    # LLM.int8 of the q/k/v projection: outlier set over every token
    idx = oracle.llmint8_outliers(V16["attn"], 6.0, 0.0)
    n = int(L.nidx.item())
    assert n == idx.size and L.idx[:n].cpu().numpy().tolist() == idx.tolist()
    Xs = V16["attn"][rows]
    Xq8, qx8 = oracle.llmint8_quant_rows(Xs, idx)
    Wq8, qw8 = oracle.llmint8_quant_weight(W["qkv"], idx)
    acc = oracle.gemm_i8(Xq8, Wq8)
    y = oracle.llmint8_combine(acc, qx8, qw8, Xs, W["qkv"], idx)
    Xf, Wf = npf(Xs).astype(np.float64), npf(W["qkv"]).astype(np.float64)
    terms = np.abs(oracle.dequant(acc, qx8, qw8)) + np.abs(Xf[:, idx]) @ np.abs(Wf[:, idx]).T
    assert_close_16(L.Y["llm"][rows], y, torch.bfloat16, terms)
    del graph
