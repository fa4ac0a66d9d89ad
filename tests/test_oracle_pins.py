"""Pins for the CPU oracle: it is checked against what the pages and the
mathematics fix, never against itself or the GPU path.

Each test names the fact it pins. A plausible slip in the oracle (a dropped
clamp, a transposed fold, a wrong rounding mode, a wrong comparison) fails at
least one of them.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------ smoothing factors: pins
def test_closed_form_scales(orc):
    """"大语言模型量化技术（四）：SmoothQuant", section 缩放因子: closed forms of
    s_j = x^a / w^(1-a) at powers of two, including a = 0 and a = 1."""
    for c in _load("closed_forms_scale.json")["cases"]:
        s = orc.smooth_scales([c["x"]], [c["w"]], c["alpha"])
        assert s[0] == np.float32(c["s"]), c


def test_worked_example(orc):
    """Same page, section 缩放的效果: the two-channel example. s_A = 100,
    s_B ~ 7.07; a value 0.4 in channel B quantises to 1 before smoothing and
    to 7 after; the error drops from 0.387 to about 0.010 (about 2.5%)."""
    g = _load("worked_example_wangyu.json")
    p = g["printed"]
    s = orc.smooth_scales(g["x_max"], g["w_max"], g["alpha"])
    assert s[0] == np.float32(100.0)
    assert abs(s[1] - p["s_B"]) < 5e-3
    # an activation tensor whose channel maxima are 100 and 0.5, holding 0.4
    X = np.array([[100.0, 0.5], [0.0, 0.4]], np.float32)
    Xq, qs = orc.quantize_act(X, None, per_token=False)
    assert abs(1.0 / qs[0] - p["delta_before"]) < 5e-4
    assert Xq[1, 1] == p["q_before"]
    deq = Xq[1, 1] / qs[0]
    assert abs(deq - p["dequant_before"]) < 5e-4
    assert abs(deq - 0.4 - p["abs_error_before"]) < 5e-4
    Xq2, qs2 = orc.quantize_act(X, s, per_token=False)
    assert abs(1.0 / qs2[0] - p["delta_after"]) < 5e-6
    assert Xq2[1, 1] == p["q_after"]
    deq2 = Xq2[1, 1] / qs2[0] * s[1]
    assert abs(deq2 - p["dequant_after"]) < 1e-3
    assert abs(deq2 - 0.4) == pytest.approx(p["abs_error_after"], abs=5e-4)
    assert 100 * abs(deq2 - 0.4) / 0.4 == pytest.approx(p["rel_error_after_percent"], abs=0.1)
    # the smoothed channel B maximum equals the smoothed weight maximum
    assert abs(0.5 / s[1] - p["channel_B_max_after"]) < 5e-4
    assert abs(s[1] * 0.01 - p["channel_B_max_after"]) < 5e-4


def test_clamps(orc):
    """lpnh.cn SmoothQuant article §3.2: clamp(min=1e-5) on both statistics and
    on s. A zero statistic must not produce 0, inf or nan."""
    s = orc.smooth_scales([0.0, 1e-5, 1e-7, 4.0], [1e5, 0.0, 4.0, 0.0], 0.5)
    assert np.all(np.isfinite(s)) and np.all(s >= np.float32(1e-5))
    assert s[0] == np.float32(1e-5)  # sqrt(1e-5 / 1e5) = 1e-5 exactly at the clamp
    assert s[1] == np.float32(1.0)   # both clamped to 1e-5
    # x = 4, w clamped to 1e-5: sqrt(4 / 1e-5)
    assert s[3] == np.float32(np.sqrt(np.float64(np.float32(4.0)) / np.float64(np.float32(1e-5))))


def test_balance_alpha_half(orc):
    """Section 缩放因子: at a = 0.5 the smoothed maxima match,
    x_j / s_j = s_j * w_j (to fp32 rounding of s)."""
    rng = np.random.default_rng(3)
    x = (rng.random(4096) * 300 + 1e-3).astype(np.float32)
    w = (rng.random(4096) * 0.2 + 1e-4).astype(np.float32)
    s = orc.smooth_scales(x, w, 0.5).astype(np.float64)
    a = x.astype(np.float64) / s
    b = s * w.astype(np.float64)
    assert np.max(np.abs(a - b) / b) < 4 * 2.0 ** -24


def test_power_law_general_alpha(orc):
    """s_j against an independent evaluation of the formula through logs
    (exp(a ln x - (1-a) ln w)), relative 1e-6, for a in {0.4, 0.6}."""
    rng = np.random.default_rng(4)
    x = (rng.random(2000) * 100 + 1e-2).astype(np.float32)
    w = (rng.random(2000) * 0.1 + 1e-3).astype(np.float32)
    for a in (0.4, 0.6, 0.75):
        s = orc.smooth_scales(x, w, a).astype(np.float64)
        ref = np.exp(a * np.log(x.astype(np.float64)) - (1 - a) * np.log(w.astype(np.float64)))
        assert np.max(np.abs(s - ref) / ref) < 1e-6


# ------------------------------------------------------------------ fold pins
def test_equivalence_identity_fp64(orc):
    """"SmoothQuant 的原理": Y = XW = (X S^-1)(S W), exact in the reals. In fp64
    with the oracle's own fold (input channel j of W times s_j) the two
    products agree to 1e-12 relative (max-norm)."""
    rng = np.random.default_rng(5)
    M, K, N = 24, 96, 40
    X = rng.normal(size=(M, K))
    X[:, 3] *= 80.0
    W = rng.normal(scale=0.02, size=(N, K))
    x = np.abs(X).max(0).astype(np.float32)
    w = np.abs(W).max(0).astype(np.float32)
    for a in (0.4, 0.5, 0.6):
        s = orc.smooth_scales(x, w, a).astype(np.float64)
        Wp = orc.fold_weight(W, s, round_f32=False)
        Y = X @ W.T
        Y2 = (X / s) @ Wp.T
        assert np.max(np.abs(Y2 - Y)) / np.max(np.abs(Y)) < 1e-12
    # a fold along the wrong axis breaks the identity (the test has power)
    Wbad = W * s[:N, None] if N <= K else None
    assert np.max(np.abs((X / s) @ Wbad.T - Y)) / np.max(np.abs(Y)) > 1e-3


def test_fold_f32_is_one_rounding(orc):
    """The fp32 fold is the fp32 product: fp64 product of two fp32 values is
    exact, so rounding it once equals the IEEE fp32 multiply."""
    rng = np.random.default_rng(6)
    W = rng.normal(scale=0.02, size=(17, 33)).astype(np.float32)
    s = (rng.random(33) * 10).astype(np.float32)
    Wp = orc.fold_weight(W, s, round_f32=True)
    assert np.array_equal(Wp, (W * s[None, :]).astype(np.float32))


def test_norm_fold_f32_is_one_division(orc):
    """The fp32 norm fold gamma' = gamma/s, beta' = beta/s ("融入 LayerNorm")
    is the IEEE fp32 quotient: the fp64 quotient of two fp32 values rounded
    to fp32 is the correctly rounded fp32 quotient (53 >= 2*24 + 2, so the
    double rounding is innocuous). RMSNorm has no beta."""
    rng = np.random.default_rng(8)
    K = 4099
    gamma = (1 + 0.1 * rng.normal(size=K)).astype(np.float32)
    beta = (0.1 * rng.normal(size=K)).astype(np.float32)
    s = (rng.random(K) * 20 + 1e-3).astype(np.float32)
    gp, bp = orc.fold_norm(gamma, beta, s)
    assert np.array_equal(gp, gamma / s) and np.array_equal(bp, beta / s)
    gp2, bp2 = orc.fold_norm(gamma, None, s)
    assert bp2 is None and np.array_equal(gp2, gp)


def test_norm_fold_identity_fp64(orc):
    """"融入 LayerNorm": with gamma' = gamma/s and beta' = beta/s the norm output
    is y/s (fp64, 1e-12), for LayerNorm and RMSNorm."""
    rng = np.random.default_rng(7)
    M, K = 8, 256
    H = rng.normal(size=(M, K))
    H[:, 5] *= 50
    gamma = 1 + 0.1 * rng.normal(size=K)
    beta = 0.1 * rng.normal(size=K)
    s = (rng.random(K) * 20 + 0.05)
    gp, bp = orc.fold_norm(gamma, beta, s, round_f32=False)
    for norm, b, bpp in ((orc.LAYERNORM, beta, bp), (orc.RMSNORM, None, None)):
        V = orc.norm_f64(H, norm, gamma, b, 1e-5)
        V2 = orc.norm_f64(H, norm, gp, bpp, 1e-5)
        assert np.max(np.abs(V2 - V / s)) / np.max(np.abs(V / s)) < 1e-12


# ------------------------------------------------------------------ norm pins
@pytest.mark.parametrize("K", [1024, 7168, 1000, 8])
def test_norm_fp32_matches_fp64(orc, K):
    """The fp32 fused path (fixed reduction order) agrees with the fp64 norm
    to 1e-6 relative per row, LayerNorm and RMSNorm."""
    rng = np.random.default_rng(K)
    M = 6
    H = rng.normal(size=(M, K)).astype(np.float32)
    H[:, min(3, K - 1)] *= 60
    gamma = (1 + 0.1 * rng.normal(size=K)).astype(np.float32)
    beta = (0.1 * rng.normal(size=K)).astype(np.float32)
    for norm, b, eps in ((orc.LAYERNORM, beta, 1e-5), (orc.RMSNORM, None, 1e-6)):
        r = orc.norm_smooth_quant(H, norm, gamma, b, eps, quantize=False, want_v=True)
        V64 = orc.norm_f64(H, norm, gamma, b, eps)
        err = np.max(np.abs(r["V"] - V64), axis=1) / np.max(np.abs(V64), axis=1)
        assert np.all(err < 1e-6), err


def test_norm_special_rows(orc):
    """Closed forms: an alternating row +-c has mean 0 and variance c^2, so
    LayerNorm gives +-1/sqrt(1 + eps/c^2) (times gamma, plus beta); a
    constant row c gives RMSNorm c/sqrt(c^2 + eps)."""
    K = 512
    c = 3.0
    row = np.tile([c, -c], K // 2).astype(np.float32)
    gamma = np.full(K, 2.0, np.float32)
    beta = np.full(K, 0.5, np.float32)
    r = orc.norm_smooth_quant(row[None], orc.LAYERNORM, gamma, beta, 1e-5, quantize=False, want_v=True)
    expect = np.sign(row) * 2.0 / np.sqrt(1 + 1e-5 / c ** 2) + 0.5
    assert np.max(np.abs(r["V"][0] - expect)) < 1e-6
    const = np.full(K, -c, np.float32)
    r = orc.norm_smooth_quant(const[None], orc.RMSNORM, gamma, None, 1e-6, quantize=False, want_v=True)
    assert np.max(np.abs(r["V"][0] - (-c) * 2.0 / np.sqrt(c * c + 1e-6))) < 1e-6


def test_norm_quant_per_token_scale(orc):
    """Per-token quantisation of the norm output: the largest |v| of every
    row maps to +-127 and qs = 127 / max|v| ("8位量化" §2.1)."""
    rng = np.random.default_rng(8)
    H = rng.normal(size=(16, 256)).astype(np.float32)
    gamma = (1 + 0.1 * rng.normal(size=256)).astype(np.float32)
    r = orc.norm_smooth_quant(H, orc.RMSNORM, gamma, None, 1e-6, want_v=True)
    for i in range(16):
        m = np.max(np.abs(r["V"][i]))
        assert r["qs"][i] == np.float32(127.0) / np.float32(m)
        assert np.max(np.abs(r["Xq"][i].astype(np.int32))) == 127


def test_norm_absmax_calibration(orc):
    """Calibration mode keeps a running per-channel max of |v| across batches."""
    rng = np.random.default_rng(9)
    gamma = np.ones(64, np.float32)
    am = np.zeros(64, np.float32)
    Vs = []
    for b in range(3):
        H = rng.normal(size=(5, 64)).astype(np.float32)
        r = orc.norm_smooth_quant(H, orc.RMSNORM, gamma, None, 1e-6, quantize=False, absmax=am,
                                  want_v=True)
        am = r["absmax"]
        Vs.append(r["V"])
    assert np.array_equal(am, np.abs(np.concatenate(Vs)).max(0))


# ------------------------------------------------------------------ quant pins
def test_round_half_even_and_clip(orc):
    """"8位量化" §2.1: q = clip(round(x * scale), -127, 127) with numpy's
    round (half to even)."""
    X = np.array([[2.5, -2.5, 3.5, 0.5, 1.5, -0.5, 127.4, 200.0, -300.0, 126.5]], np.float32)
    Xq, qs = orc.quantize_act(X, None, per_token=False, static_qs=1.0)
    assert Xq.tolist() == [[2, -2, 4, 0, 2, 0, 127, 127, -127, 126]]
    assert qs[0] == 1.0
    # per token: the row max maps to 127; 63.5 ties to 64
    Xq, qs = orc.quantize_act(np.array([[127.0, 63.5, -0.5]], np.float32), None, per_token=True)
    assert qs[0] == 1.0 and Xq.tolist() == [[127, 64, 0]]


def _check_symmetric_int8(v, q, qs, keep=None):
    """Invariants of absmax int8 with scale qs = 127 / max|v| per row ("8位量化"
    §2.1): codes in [-127, 127]; the row's largest |v| maps to +-127; every
    code is the nearest integer to v*qs (within 0.5 plus the fp32 rounding of
    the product); codes keep the sign of v. Columns outside `keep` are 0."""
    v = v.astype(np.float64)
    qs = np.asarray(qs, np.float64).reshape(-1, 1)
    q = q.astype(np.int64)
    if keep is not None:
        out = np.setdiff1d(np.arange(v.shape[1]), keep)
        assert np.all(q[:, out] == 0)
        v, q = v[:, keep], q[:, keep]
    assert np.all(np.abs(q) <= 127)
    am = np.argmax(np.abs(v), axis=1)
    rows = np.arange(v.shape[0])
    nz = np.abs(v[rows, am]) > 0
    assert np.all(np.abs(q[rows, am])[nz] == 127)
    assert np.max(np.abs(v * qs - q)) <= 0.5 + 127 * 2.0 ** -23
    assert np.all((q == 0) | (np.sign(q) == np.sign(v)))


def test_int8_quantisers_invariants(orc):
    """Every absmax int8 quantiser of the oracle on random data with outlier
    channels: activations per token, weights per output channel, the LLM.int8
    rows and weight columns outside O, the fused norm output and the SwiGLU
    output. A truncating or half-away rounding, an inverted scale or a clip at
    128 fails here."""
    rng = np.random.default_rng(60)
    M, K, N = 37, 200, 29
    X = rng.normal(size=(M, K)).astype(np.float32)
    X[:, [3, 77]] *= 40
    Xq, qx = orc.quantize_act(X, None, per_token=True)
    _check_symmetric_int8(X, Xq, qx)
    W = rng.normal(scale=0.02, size=(N, K)).astype(np.float32)
    Wq, qw = orc.quantize_weight(W, per_channel=True)
    _check_symmetric_int8(W, Wq, qw)
    idx = orc.llmint8_outliers(X, 6.0, 0.0)
    assert set(idx.tolist()) >= {3, 77}
    keep = np.setdiff1d(np.arange(K), idx)
    Xq8, qx8 = orc.llmint8_quant_rows(X, idx)
    _check_symmetric_int8(X, Xq8, qx8, keep)
    Wq8, qw8 = orc.llmint8_quant_weight(W, idx)
    _check_symmetric_int8(W, Wq8, qw8, keep)
    gamma = (1 + 0.1 * rng.normal(size=K)).astype(np.float32)
    for norm in (orc.LAYERNORM, orc.RMSNORM):
        r = orc.norm_smooth_quant(X, norm, gamma, None, 1e-5, True, want_v=True)
        _check_symmetric_int8(r["V"], r["Xq"], r["qs"])
    A = (rng.normal(size=(M, 2 * K)) * 3).astype(np.float32)
    r = orc.act_quant(A, orc.SWIGLU, want_h=True)
    _check_symmetric_int8(r["H"], r["Xq"], r["qs"])


def test_zero_row_scale_floor(orc):
    """An all-zero row takes the 1e-8 floor of quantize_vectorwise and gives 0."""
    Xq, qs = orc.quantize_act(np.zeros((2, 16), np.float32), None, per_token=True)
    assert np.all(Xq == 0) and np.all(qs == np.float32(127.0) / np.float32(1e-8))


def test_weight_quant_group_scaling_invariance(orc):
    """"缩放的代价": relative quantisation error is unchanged when a whole
    quantisation group is scaled. With per-output-channel groups and power of
    two factors, codes are identical and scales divide exactly."""
    rng = np.random.default_rng(10)
    W = rng.normal(scale=0.02, size=(32, 128)).astype(np.float32)
    f = (2.0 ** rng.integers(-6, 7, size=32)).astype(np.float32)
    Wq, qs = orc.quantize_weight(W, per_channel=True)
    Wq2, qs2 = orc.quantize_weight(W * f[:, None], per_channel=True)
    assert np.array_equal(Wq, Wq2)
    assert np.array_equal(qs2, (qs / f).astype(np.float32))
    e1 = np.abs(W - Wq / qs[:, None]).max(1) / np.abs(W).max(1)
    e2 = np.abs(W * f[:, None] - Wq2 / qs2[:, None]).max(1) / np.abs(W * f[:, None]).max(1)
    assert np.allclose(e1, e2, rtol=1e-6)


def test_weight_quant_per_tensor(orc):
    W = np.array([[0.5, -1.0], [0.25, 2.0]], np.float32)
    Wq, qs = orc.quantize_weight(W, per_channel=False)
    assert qs[0] == np.float32(63.5)
    assert Wq.tolist() == [[32, -64], [16, 127]]  # 31.75 -> 32, 15.875 -> 16


# ------------------------------------------------------------------ GEMM pins
def test_gemm_bruteforce_random(orc):
    rng = np.random.default_rng(11)
    for (M, N, K) in [(1, 1, 1), (3, 5, 7), (17, 9, 64), (33, 40, 130)]:
        X = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
        W = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
        ref = X.astype(np.int64) @ W.astype(np.int64).T
        assert np.array_equal(orc.gemm_i8(X, W), ref)
        r = orc.gemm_i8(X, W, rows=(M // 2, M))
        assert np.array_equal(r, ref[M // 2:])


@pytest.mark.parametrize("K", [1, 2, 3])
def test_gemm_exhaustive_small_k(orc, K):
    vals = [-127, -1, 0, 1, 127]
    rows = np.array(list(itertools.product(vals, repeat=K)), np.int8)
    acc = orc.gemm_i8(rows, rows)
    ref = np.array([[sum(int(a) * int(b) for a, b in zip(r1, r2)) for r2 in rows] for r1 in rows])
    assert np.array_equal(acc, ref)


def test_gemm_no_overflow_bound(orc):
    """"8位量化" §2.1: int32 accumulation does not overflow. |acc| <= 127^2 K;
    at the largest K here (49152) all-127 operands give exactly 792,772,608."""
    K = 49152
    X = np.full((2, K), 127, np.int8)
    X[1] = -127
    W = np.full((1, K), 127, np.int8)
    acc = orc.gemm_i8(X, W)
    assert acc[0, 0] == 792_772_608 and acc[1, 0] == -792_772_608
    assert abs(int(acc[0, 0])) < 2 ** 31
    assert 127 * 127 * 133_144 < 2 ** 31 < 127 * 127 * 133_145


def test_dequant_closed_form(orc):
    """out = acc / (c_x * c_w) + bias ("8位量化" §2.1 outer-product dequant)."""
    acc = np.array([[127 * 127, -127 * 64]], np.int64)
    y = orc.dequant(acc, np.array([63.5], np.float32), np.array([254.0, 127.0], np.float32),
                    bias=np.array([0.25, -1.0], np.float32))
    assert y[0, 0] == 16129 / (63.5 * 254) + 0.25
    assert y[0, 1] == -127 * 64 / (63.5 * 127) - 1.0


def test_static_scale_from_calibration_absmax(orc):
    """A static per-tensor scale is 127 over the largest calibrated channel
    absmax ("8位量化" §2.1, one scale for the whole tensor): closed forms, the
    1e-8 floor of an all-zero calibration, and agreement with the dynamic
    per-tensor scale of a tensor whose absmax is that value."""
    assert orc.scale_from_absmax(np.array([0.5, 2.0, 1.0], np.float32)) == np.float32(63.5)
    assert orc.scale_from_absmax(np.array([127.0], np.float32)) == np.float32(1.0)
    assert orc.scale_from_absmax(np.zeros(4, np.float32)) == np.float32(127.0) / np.float32(1e-8)
    rng = np.random.default_rng(13)
    X = rng.normal(size=(9, 48)).astype(np.float32)
    Xq, qs = orc.quantize_act(X, None, per_token=False)
    assert qs[0] == orc.scale_from_absmax(np.abs(X).max(0))
    Xq2, _ = orc.quantize_act(X, None, per_token=False, static_qs=qs[0])
    assert np.array_equal(Xq, Xq2)


def test_dequant_f64_accumulators(orc):
    """The fp64-accumulator dequant (for FP8 products, whose sums are not
    integers) is the same outer-product formula: exact on power-of-two
    scales, per-tensor and per-row/per-column indexing, bias added last."""
    acc = np.array([[1.5, -3.0, 0.0], [96.0, 0.25, -7.75]], np.float64)
    qx = np.array([2.0, 0.5], np.float32)
    qw = np.array([4.0, 8.0, 0.25], np.float32)
    b = np.array([1.0, -0.5, 0.125], np.float32)
    y = orc.dequant_f64(acc, qx, qw, bias=b)
    ref = acc / (qx.astype(np.float64)[:, None] * qw.astype(np.float64)[None, :]) + b.astype(np.float64)
    assert np.array_equal(y, ref)
    y1 = orc.dequant_f64(acc, np.array([2.0], np.float32), np.array([4.0], np.float32))
    assert np.array_equal(y1, acc / 8.0)
    assert np.array_equal(orc.dequant_f64(acc.astype(np.int64).astype(np.float64), qx, qw),
                          orc.dequant(acc.astype(np.int64), qx, qw))


def test_dequant_row_and_column_scales(orc):
    """Scales factor out only per row (token) and per column (output channel):
    Y = diag(dX) Xq Wq^T diag(dW) ("为什么激活不能用逐通道量化")."""
    rng = np.random.default_rng(12)
    X = rng.integers(-127, 128, size=(5, 32)).astype(np.int8)
    W = rng.integers(-127, 128, size=(7, 32)).astype(np.int8)
    qx = (rng.random(5) * 10 + 1).astype(np.float32)
    qw = (rng.random(7) * 10 + 1).astype(np.float32)
    y = orc.dequant(orc.gemm_i8(X, W), qx, qw)
    ref = np.diag(1 / qx.astype(np.float64)) @ (X.astype(np.float64) @ W.astype(np.float64).T) \
        @ np.diag(1 / qw.astype(np.float64))
    assert np.max(np.abs(y - ref) / (np.abs(ref) + 1e-30)) < 1e-14


# ------------------------------------------------------------------ rounding pins
def test_round_bf16_matches_torch_on_fp32(orc):
    rng = np.random.default_rng(13)
    v = np.concatenate([rng.normal(size=2000) * 10.0 ** rng.integers(-20, 20, size=2000),
                        [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 3.3e38, -3.4e38]]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.round_bf16_bits(v.astype(np.float64)), ref)


def test_round_fp16_matches_numpy(orc):
    rng = np.random.default_rng(14)
    v = np.concatenate([rng.normal(size=3000) * 10.0 ** rng.integers(-9, 5, size=3000),
                        [0.0, -0.0, 1 + 2 ** -11, 1 + 3 * 2 ** -11, 65504.0, 65519.9, 65520.0,
                         2 ** -25, 3 * 2 ** -26, 1e-9]])
    with np.errstate(over="ignore"):  # values past 65520 overflow to inf on purpose
        ref = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(orc.round_fp16_bits(v), ref)


# ------------------------------------------------------------------ LLM.int8 pins
def test_outliers_bruteforce(orc):
    """"8位量化" §2.2 split_outliers: columns where the share of |x| > alpha
    exceeds min_ratio; §4.1: any value over the threshold marks the column."""
    rng = np.random.default_rng(15)
    X = rng.normal(size=(32, 40)).astype(np.float32)
    X[3, 7] = 6.0         # not > 6.0
    X[5, 9] = 6.00390625  # next fp16 above 6: counts
    X[0:2, 20] = -7.0     # 2/32 = 0.0625
    X[0:3, 30] = 9.0      # 3/32
    X[:, 7] = np.clip(X[:, 7], -5, 5); X[3, 7] = 6.0
    for thr, mr in [(6.0, 0.0), (6.0, 0.06), (6.0, 0.0625), (2.0, 0.1), (100.0, 0.0)]:
        ref = [j for j in range(40) if np.mean(np.abs(X[:, j]) > thr) > mr]
        assert orc.llmint8_outliers(X, thr, mr).tolist() == ref
    assert 9 in orc.llmint8_outliers(X, 6.0, 0.0).tolist()
    assert 7 not in orc.llmint8_outliers(X, 6.0, 0.0).tolist()
    assert 20 in orc.llmint8_outliers(X, 6.0, 0.06).tolist()
    assert 20 not in orc.llmint8_outliers(X, 6.0, 0.0625).tolist()


def test_decomposition_identity_fp64():
    """§2.2: X_O W_O + X_notO W_notO = X W (exact split of the inner product)."""
    rng = np.random.default_rng(16)
    X = rng.normal(size=(9, 50))
    W = rng.normal(size=(50, 11))
    O = [3, 17, 44]
    m = np.ones(50, bool)
    m[O] = False
    assert np.max(np.abs(X[:, O] @ W[O] + X[:, m] @ W[m] - X @ W)) < 1e-12


def test_llmint8_no_outliers_reduces_to_vectorwise(orc):
    """With O empty the decomposition is the vector-wise int8 path."""
    rng = np.random.default_rng(17)
    X = rng.normal(size=(12, 64)).astype(np.float32)
    W = rng.normal(scale=0.02, size=(20, 64)).astype(np.float32)
    y, idx, Xq, qx, Wq, qw = orc.llmint8_matmul(X, W, 6.0)
    assert idx.size == 0
    Xq2, qx2 = orc.quantize_act(X, None, per_token=True)
    Wq2, qw2 = orc.quantize_weight(W, per_channel=True)
    assert np.array_equal(Xq, Xq2) and np.array_equal(Wq, Wq2)
    assert np.array_equal(y, orc.dequant(orc.gemm_i8(Xq2, Wq2), qx2, qw2))


def test_llmint8_planted_and_accuracy(orc):
    """Planted outlier dims are found exactly; outlier columns are zero in both
    int8 operands; the result is close to the exact product, and much closer
    than plain vector-wise int8 on the same data."""
    rng = np.random.default_rng(18)
    M, K, N = 64, 256, 48
    X = np.clip(rng.normal(size=(M, K)), -5.9, 5.9).astype(np.float32)
    dims = [11, 100, 200]
    for d in dims:
        X[rng.permutation(M)[:16], d] = 30.0
    W = rng.normal(scale=0.02, size=(N, K)).astype(np.float32)
    y, idx, Xq, qx, Wq, qw = orc.llmint8_matmul(X, W, 6.0)
    assert idx.tolist() == dims
    assert np.all(Xq[:, dims] == 0) and np.all(Wq[:, dims] == 0)
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    err = np.max(np.abs(y - ref)) / np.max(np.abs(ref))
    Xv, qxv = orc.quantize_act(X, None, per_token=True)
    Wv, qwv = orc.quantize_weight(W, per_channel=True)
    err_v = np.max(np.abs(orc.dequant(orc.gemm_i8(Xv, Wv), qxv, qwv) - ref)) / np.max(np.abs(ref))
    assert err < 2e-2 and err < err_v / 2


def test_llmint8_exact_on_dyadic_grid(orc):
    """When every row of X outside O has absmax 127/32 and every row of W
    outside O has absmax 127/64, with all entries on those grids, the
    vector-wise codes are the grid integers and the dequantised int8 part is
    exact; the outlier term (whole numbers times grid values) is exact too.
    The decomposition then returns X·Wᵀ exactly, so a dropped or doubled
    outlier term, an outlier column left in a row's absmax, a transposed
    operand or a wrong scale fails it (LLM.int8() decomposition, the
    outlier/vector-wise split of "LLM.int8()" §2.2)."""
    rng = np.random.default_rng(20)
    M, K, N = 24, 96, 40
    dims = [5, 47, 90]
    X = rng.integers(-127, 128, size=(M, K)).astype(np.float32) / 32.0
    X[:, 0] = np.where(rng.random(M) < 0.5, -127.0, 127.0) / 32.0  # row absmax outside O
    for d in dims:
        X[rng.permutation(M)[:6], d] = rng.choice([-40.0, -30.0, 9.0, 30.0, 40.0], 6)
    W = rng.integers(-127, 128, size=(N, K)).astype(np.float32) / 64.0
    W[:, 1] = np.where(rng.random(N) < 0.5, -127.0, 127.0) / 64.0
    y, idx, Xq, qx, Wq, qw = orc.llmint8_matmul(X, W, 6.0)
    assert idx.tolist() == dims
    assert np.all(qx == 32.0) and np.all(qw == 64.0)
    keep = np.setdiff1d(np.arange(K), dims)
    assert np.array_equal(Xq[:, keep].astype(np.float64), X[:, keep].astype(np.float64) * 32)
    assert np.array_equal(Wq[:, keep].astype(np.float64), W[:, keep].astype(np.float64) * 64)
    assert np.array_equal(y, X.astype(np.float64) @ W.astype(np.float64).T)


def test_vectorwise_toy_magnitude(orc):
    """"8位量化" §2.1 toy: X(4x8), W(8x16) from default_rng(0), X[0,3] = 40;
    vector-wise int8 gives a relative error of order 1e-3..1e-2. A magnitude
    check only: the page prints no tensors."""
    rng = np.random.default_rng(0)
    X = rng.normal(0, 1, (4, 8)).astype(np.float16)
    W = rng.normal(0, 1, (8, 16)).astype(np.float16)
    X[0, 3] = 40.0
    Xq, qx = orc.quantize_act(X.astype(np.float32), None, per_token=True)
    Wq, qw = orc.quantize_weight(W.T.astype(np.float32), per_channel=True)
    y = orc.dequant(orc.gemm_i8(Xq, Wq), qx, qw)
    ref = X.astype(np.float32).astype(np.float64) @ W.astype(np.float32).astype(np.float64)
    err = np.abs(y - ref).max() / np.abs(ref).max()
    assert 1e-4 < err < 5e-2


def test_col_absmax_bruteforce(orc):
    rng = np.random.default_rng(19)
    X = rng.normal(size=(37, 29)).astype(np.float32)
    prev = np.abs(rng.normal(size=29)).astype(np.float32) * 2
    got = orc.col_absmax(X, prev)
    ref = np.array([max(prev[j], max(abs(float(X[i, j])) for i in range(37))) for j in range(29)],
                   np.float32)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- MLP activation; fold into the previous linear
def _ulps(got, ref64):
    """|got - ref| in units of the fp32 spacing at ref."""
    ref32 = ref64.astype(np.float32)
    return np.abs(got.astype(np.float64) - ref64) / np.spacing(np.abs(ref32)).astype(np.float64)


def test_expf_within_4ulp_of_fp64(orc):
    """The fixed fp32 exponential against the fp64 exp on a dense grid of its
    finite range, and its end values."""
    x = np.linspace(-87.0, 88.0, 400_001).astype(np.float32)
    e = orc.expf(x)
    assert np.max(_ulps(e, np.exp(x.astype(np.float64)))) <= 4.0
    assert orc.expf(0.0)[0] == 1.0
    assert np.isinf(orc.expf(88.5)[0]) and orc.expf(-87.5)[0] == 0.0
    # across the 2^n seams of the reduction (x = (n + 1/2) ln 2) the result
    # stays monotone
    seams = (np.arange(-120, 120) + 0.5) * np.log(2.0)
    xs = np.concatenate([np.nextafter(seams.astype(np.float32), -np.inf), seams.astype(np.float32),
                         np.nextafter(seams.astype(np.float32), np.inf)]).astype(np.float32)
    xs = np.sort(xs[(xs > -87) & (xs < 88)])
    assert np.all(np.diff(orc.expf(xs)) >= 0)


def test_silu_identities(orc):
    """silu(g) = g * sigmoid(g): silu(g) - silu(-g) = g; silu(0) = 0; silu(g)
    = g once exp(-g) vanishes next to 1; within a few ulp of the fp64 value."""
    g = np.linspace(-60, 60, 240_001).astype(np.float32)
    s = orc.silu(g).astype(np.float64)
    sn = orc.silu(-g).astype(np.float64)
    assert np.max(np.abs((s - sn) - g.astype(np.float64)) / np.maximum(np.abs(g), 1e-3)) < 2e-6
    g64 = g.astype(np.float64)
    ref = g64 / (1.0 + np.exp(-g64))
    big = np.abs(ref) > 1e-30
    assert np.max(_ulps(orc.silu(g)[big], ref[big])) <= 6.0
    assert orc.silu(0.0)[0] == 0.0
    assert orc.silu(30.0)[0] == 30.0 and orc.silu(1000.0)[0] == 1000.0
    assert orc.silu(-100.0)[0] == 0.0


def test_swiglu_quant_against_fp64(orc):
    """h = silu(gate) * up per element ([gate | up] halves of a row), per-token
    int8: h within a few ulp of the fp64 value and the codes those of the fp64
    h wherever the fp64 value is not within 1e-3 of a rounding tie. Swapping
    the halves (a plausible mistake) is far off."""
    rng = np.random.default_rng(30)
    M, I = 40, 96
    A = (rng.normal(size=(M, 2 * I)) * 3).astype(np.float32)
    r = orc.act_quant(A, orc.SWIGLU, want_h=True)
    g64, u64 = A[:, :I].astype(np.float64), A[:, I:].astype(np.float64)
    h64 = g64 / (1.0 + np.exp(-g64)) * u64
    big = np.abs(h64) > 1e-20
    assert np.max(_ulps(r["H"][big], h64[big])) <= 8.0
    qs64 = 127.0 / np.max(np.abs(h64), axis=1)
    assert np.max(np.abs(r["qs"] / qs64 - 1)) < 1e-6
    t = h64 * qs64[:, None]
    clear = np.abs(np.abs(t - np.floor(t)) - 0.5) > 1e-3
    assert np.array_equal(r["Xq"][clear], np.rint(t)[clear].astype(np.int8))
    swapped = u64 / (1.0 + np.exp(-u64)) * g64
    assert np.max(np.abs(swapped - h64)) > 1.0


def _gelu64(x, c, k):
    """The tanh-form GELU in fp64, written x / (1 + exp(-2u)): the same
    function as 0.5 x (1 + tanh(u)) without its cancellation for x < 0."""
    x = np.asarray(x, np.float64)
    u = c * (x + k * x ** 3)
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-2.0 * u))


def test_gelu_against_fp64_and_library(orc):
    """The fixed fp32 GELU (reading R15) against an fp64 evaluation with the
    same fp32 constants (few ulp: only the sequence's roundings and exp's
    error remain), against a library GELU (torch, tanh form, fp64, exact
    constants) to 1e-5 relative where |gelu| > 1e-6, and its identities:
    gelu(x) - gelu(-x) = x, gelu(0) = 0, gelu(x) = x and 0 far from 0. A
    plausible mistake (the erf form, or a dropped cubic term) is far off."""
    import math

    c32, k32 = float(np.float32(math.sqrt(2 / math.pi))), float(np.float32(0.044715))
    x = np.concatenate([np.linspace(-12, 12, 200001), np.geomspace(1e-30, 1e3, 5001),
                        -np.geomspace(1e-30, 9.0, 5001)]).astype(np.float32)
    g = orc.gelu(x).astype(np.float64)
    g64 = _gelu64(x, c32, k32)
    big = np.abs(g64) > 1e-30
    # exp(z) carries the relative error of z times |z|: the bound grows with
    # |2u| where exp(-2u) dominates (x < 0)
    z = np.abs(2 * c32 * (x.astype(np.float64) + k32 * x.astype(np.float64) ** 3))
    assert np.all(_ulps(g[big].astype(np.float32), g64[big]) <= 16.0 + 8.0 * z[big])
    lib = torch.nn.functional.gelu(torch.from_numpy(x.astype(np.float64)), approximate="tanh").numpy()
    m = np.abs(lib) > 1e-6
    assert np.max(np.abs(g[m] - lib[m]) / np.abs(lib[m])) < 1e-5
    d = g - orc.gelu(-x).astype(np.float64) - x.astype(np.float64)
    assert np.all(np.abs(d) <= 4 * np.spacing(np.abs(x)).astype(np.float64) + 1e-38)
    assert orc.gelu(np.float32(0.0))[0] == 0.0
    assert orc.gelu(np.float32(40.0))[0] == np.float32(40.0) and orc.gelu(np.float32(-40.0))[0] == 0.0
    erf_form = torch.nn.functional.gelu(torch.from_numpy(x.astype(np.float64))).numpy()
    assert np.max(np.abs(erf_form - g)) > 1e-4
    assert np.max(np.abs(_gelu64(x, c32, 0.0) - g)) > 1e-2


def test_gelu_quant_against_fp64(orc):
    """GELU then per-token int8: the codes those of the fp64 GELU wherever the
    fp64 value is not within 1e-3 of a rounding tie."""
    import math

    rng = np.random.default_rng(31)
    A = (rng.normal(size=(40, 256)) * 3).astype(np.float32)
    r = orc.act_quant(A, orc.GELU, want_h=True)
    h64 = _gelu64(A, float(np.float32(math.sqrt(2 / math.pi))), float(np.float32(0.044715)))
    qs64 = 127.0 / np.max(np.abs(h64), axis=1)
    assert np.max(np.abs(r["qs"] / qs64 - 1)) < 1e-6
    t = h64 * qs64[:, None]
    clear = np.abs(np.abs(t - np.floor(t)) - 0.5) > 1e-3
    assert np.array_equal(r["Xq"][clear], np.rint(t)[clear].astype(np.int8))


def test_relu_quant_bruteforce(orc):
    """ReLU MLP input: h = max(x, 0), then int8 per token or with a static scale."""
    rng = np.random.default_rng(31)
    X = rng.normal(size=(7, 24)).astype(np.float32)
    X[2] = -np.abs(X[2])  # an all-negative row: h = 0, scale from the 1e-8 floor
    r = orc.act_quant(X, orc.RELU, want_h=True)
    for i in range(7):
        h = [max(float(v), 0.0) for v in X[i]]
        m = max(h)
        qs = np.float32(127.0) / np.float32(max(m, 1e-8))
        assert r["qs"][i] == qs
        for j in range(24):
            assert r["H"][i, j] == np.float32(h[j])
            assert r["Xq"][i, j] == int(np.clip(np.rint(np.float32(h[j]) * qs), -127, 127))
    rs = orc.act_quant(X, orc.RELU, per_token=False, static_qs=40.0)
    assert rs["qs"][0] == np.float32(40.0)
    assert np.array_equal(rs["Xq"], np.clip(np.rint(np.maximum(X, 0) * np.float32(40.0)), -127, 127).astype(np.int8))


def _silu64(x):
    return x / (1.0 + np.exp(-x))


def test_fold_prev_linear_identity_mlp(orc):
    """[SQ-p2] 融入前序线性层的权重: up_proj's output channel j divided by s_j and
    down_proj's input channel j multiplied by s_j leave the FFN output
    unchanged (fp64, exact folds); folding up_proj on its input axis instead
    does not."""
    rng = np.random.default_rng(32)
    M, D, I = 6, 16, 24
    x = rng.normal(size=(M, D))
    Wg, Wu = rng.normal(size=(I, D)), rng.normal(size=(I, D))
    Wd = rng.normal(size=(D, I))
    bu = rng.normal(size=I)
    s = np.exp(rng.normal(size=I))
    y = (_silu64(x @ Wg.T) * (x @ Wu.T + bu)) @ Wd.T
    Wu2, bu2 = orc.fold_prev_linear(Wu, s, bu, round_f32=False)
    Wd2 = orc.fold_weight(Wd, s, round_f32=False)
    h2 = _silu64(x @ Wg.T) * (x @ Wu2.T + bu2)
    assert np.allclose(h2, (_silu64(x @ Wg.T) * (x @ Wu.T + bu)) / s, rtol=1e-12, atol=0)
    y2 = h2 @ Wd2.T
    assert np.max(np.abs(y2 - y)) / np.max(np.abs(y)) < 1e-12
    s_in = np.exp(rng.normal(size=D))
    Wu_bad = orc.fold_weight(Wu, s_in, round_f32=False)  # the input axis: wrong
    y_bad = (_silu64(x @ Wg.T) * (x @ Wu_bad.T + bu)) @ Wd.T
    assert np.max(np.abs(y_bad - y)) / np.max(np.abs(y)) > 1e-3


def test_fold_prev_linear_identity_attention(orc):
    """o_proj's input is a convex mix of v_proj's outputs (attention weights P
    with rows summing to 1), so v_proj rows / s and o_proj columns * s leave
    the attention output unchanged (fp64)."""
    rng = np.random.default_rng(33)
    T, D = 9, 12
    x = rng.normal(size=(T, D))
    Wv, Wo = rng.normal(size=(D, D)), rng.normal(size=(D, D))
    P = np.exp(rng.normal(size=(T, T)))
    P /= P.sum(axis=1, keepdims=True)
    s = np.exp(rng.normal(size=D))
    y = (P @ (x @ Wv.T)) @ Wo.T
    Wv2, _ = orc.fold_prev_linear(Wv, s, round_f32=False)
    Wo2 = orc.fold_weight(Wo, s, round_f32=False)
    y2 = (P @ (x @ Wv2.T)) @ Wo2.T
    assert np.max(np.abs(y2 - y)) / np.max(np.abs(y)) < 1e-12


def test_fold_prev_linear_fp32_is_one_division(orc):
    """In fp32 each folded value is the correctly rounded quotient: an fp64
    quotient of fp32 operands rounded once (53 >= 2*24 + 2 bits, so the double
    rounding is innocuous), equal to numpy's float32 division."""
    rng = np.random.default_rng(34)
    W = rng.normal(size=(33, 17)).astype(np.float32)
    b = rng.normal(size=33).astype(np.float32)
    s = np.exp(rng.normal(size=33)).astype(np.float32)
    Wp, bp = orc.fold_prev_linear(W, s, b)
    assert np.array_equal(Wp, W / s[:, None])
    assert np.array_equal(bp, b / s)


# ---------------------------------------------------------------- FP8 variant
def test_e4m3_codes_round_trip(orc):
    """Every finite E4M3 code decodes to a value that rounds and re-encodes to
    the same code; 0x7F / 0xFF (NaN) are the only codes left out; the largest
    finite value is 448 and the smallest subnormal 2^-9."""
    vals = {}
    for b in range(256):
        if (b & 0x7F) == 0x7F:
            continue
        v = orc.e4m3_value(b)
        assert orc.e4m3_bits(orc.e4m3_round(np.float32(v))) == b or v == 0.0
        vals[b] = v
    assert max(vals.values()) == 448.0 and min(v for v in vals.values() if v > 0) == 2.0 ** -9
    assert len(set(vals.values())) == 253  # +0 and -0 compare equal


def test_e4m3_rounding_ties_and_saturation(orc):
    """Midpoints between neighbouring values go to the even code; magnitudes
    past 448 saturate; the conversion agrees with torch's float8_e4m3fn inside
    the finite range."""
    pos = sorted({orc.e4m3_value(b) for b in range(127)})
    for lo, hi in zip(pos[:-1], pos[1:]):
        mid = np.float32((lo + hi) / 2)
        got = orc.e4m3_round(mid)
        lo_even = orc.e4m3_bits(np.float32(lo)) % 2 == 0
        assert got == (lo if lo_even else hi), (lo, hi, got)
        assert orc.e4m3_round(-mid) == -got
    for big in (448.0, 463.9, 464.0, 500.0, 1e30):
        assert orc.e4m3_round(np.float32(big)) == 448.0 and orc.e4m3_round(np.float32(-big)) == -448.0
    rng = np.random.default_rng(40)
    x = (rng.normal(size=20000) * 60).astype(np.float32)
    x = x[np.abs(x) < 440]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float32).numpy()
    got = np.array([orc.e4m3_round(v) for v in x], np.float32)
    assert np.array_equal(got, ref)
    # codes, over the whole finite range on a log scale, down past the
    # smallest subnormal: negative values that round to zero keep the sign
    mag = np.exp(rng.uniform(np.log(1e-5), np.log(440), 50000))
    x = (mag * rng.choice([-1.0, 1.0], mag.size)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_bits(orc.e4m3_round(v)) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_fp8_quant_and_gemm_bruteforce(orc):
    """Row scales 448 / max|v|, codes of v * qs, and the exact GEMM of the
    decoded codes, against plain Python on a tiny case."""
    rng = np.random.default_rng(41)
    X = (rng.normal(size=(3, 16)) * 5).astype(np.float32)
    W = (rng.normal(size=(4, 16)) * 0.1).astype(np.float32)
    Xq, qx = orc.quantize_fp8(X, per_row=True)
    Wq, qw = orc.quantize_fp8(W, per_row=True)
    for i in range(3):
        m = max(abs(float(v)) for v in X[i])
        assert qx[i] == np.float32(448.0) / np.float32(m)
        for j in range(16):
            assert orc.e4m3_value(Xq[i, j]) == orc.e4m3_round(np.float32(X[i, j]) * qx[i])
    acc = orc.gemm_fp8(Xq, Wq)
    for i in range(3):
        for j in range(4):
            t = sum(orc.e4m3_value(Xq[i, k]) * orc.e4m3_value(Wq[j, k]) for k in range(16))
            assert acc[i, j] == t
    # the dequantised product approximates X W^T to the FP8 quantisation error
    y = acc / (qx.astype(np.float64)[:, None] * qw.astype(np.float64)[None, :])
    ref = X.astype(np.float64) @ W.astype(np.float64).T
    assert np.max(np.abs(y - ref)) / np.max(np.abs(ref)) < 0.1


# ---------------------------------------------------------------- batched int8 GEMM (attention)
def test_bmm_bruteforce(orc):
    """Each problem of the batch is its own int64 product (einsum brute force)."""
    rng = np.random.default_rng(50)
    A = rng.integers(-127, 128, size=(3, 5, 7)).astype(np.int8)
    B = rng.integers(-127, 128, size=(3, 4, 7)).astype(np.int8)
    ref = np.einsum("bik,bjk->bij", A.astype(np.int64), B.astype(np.int64))
    assert np.array_equal(orc.bmm_i8(A, B), ref)


def test_bmm_dequant_per_problem_scales(orc):
    """Problem b divides by its own row and column scales, and a row subset
    picks the matching row scales; exact on power-of-two scales."""
    rng = np.random.default_rng(52)
    B, T, S = 3, 6, 5
    acc = rng.integers(-2 ** 20, 2 ** 20, size=(B, T, S)).astype(np.int64)
    qa = [(2.0 ** rng.integers(-4, 5, size=T)).astype(np.float32) for _ in range(B)]
    qb = [(2.0 ** rng.integers(-4, 5, size=S)).astype(np.float32) for _ in range(B)]
    y = orc.bmm_dequant(acc, qa, qb)
    ref = np.stack([acc[b] / (qa[b].astype(np.float64)[:, None] * qb[b].astype(np.float64)[None, :])
                    for b in range(B)])
    assert np.array_equal(y, ref)
    rows = [1, 4]
    ys = orc.bmm_dequant(acc[:, rows], qa, qb, rows=rows)
    assert np.array_equal(ys, ref[:, rows])


def test_bmm_attention_scores_magnitude(orc):
    """lpnh.cn SmoothQuant practice article §2.2: QK^T in int8 with one scale
    per (head, token) on Q and on K approximates the fp64 scores; PV with P
    per row and V^T per (head, channel) approximates P V. Magnitude checks."""
    rng = np.random.default_rng(51)
    H, T, d = 2, 16, 32
    Q, K, V = (rng.normal(size=(H, T, d)).astype(np.float32) for _ in range(3))
    qq = [orc.quantize_act(Q[h], None, per_token=True) for h in range(H)]
    kq = [orc.quantize_act(K[h], None, per_token=True) for h in range(H)]
    S = orc.bmm_dequant(orc.bmm_i8(np.stack([q[0] for q in qq]), np.stack([k[0] for k in kq])),
                        [q[1] for q in qq], [k[1] for k in kq])
    ref = np.einsum("htd,hsd->hts", Q.astype(np.float64), K.astype(np.float64))
    assert np.max(np.abs(S - ref)) / np.max(np.abs(ref)) < 0.03
    P = np.exp(ref - ref.max(axis=2, keepdims=True))
    P = (P / P.sum(axis=2, keepdims=True)).astype(np.float32)
    pq = [orc.quantize_act(P[h], None, per_token=True) for h in range(H)]
    vq = [orc.quantize_act(np.ascontiguousarray(V[h].T), None, per_token=True) for h in range(H)]
    O = orc.bmm_dequant(orc.bmm_i8(np.stack([p[0] for p in pq]), np.stack([v[0] for v in vq])),
                        [p[1] for p in pq], [v[1] for v in vq])
    refo = np.einsum("hts,hsd->htd", P.astype(np.float64), V.astype(np.float64))
    assert np.max(np.abs(O - refo)) / np.max(np.abs(refo)) < 0.05
