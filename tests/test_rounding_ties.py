"""Round-half-even at exact ties ("8位量化：异常值与混合精度分解实战" §2.1:
round, then clip to [-127, 127]; numpy and torch round halves to even).

Inputs are built so that t = v * qs is exactly k + 1/2 for many k of both
signs (2.5 -> 2, -2.5 -> -2, 63.5 -> 64, 126.5 -> 126, 0.5 -> 0, 1.5 -> 2),
and the scale is exactly 1: a per-tensor static scale of 1, or a row whose
largest magnitude is 127. Each quantiser of the path is checked on the oracle
(CPU) and, through the C ABI, on the GPU: the activation quantiser (with and
without the 1/s division), the weight quantiser (per tensor and per channel),
the MLP activation quantiser (ReLU, static scale) and the fused norm (static
and per-token scales, with epsilon 0 and rows of +-1 so that r = 1 exactly).
A fused multiply-add in place of the separate multiply and add of the
rounding step would give the wrong code at +-63.5, so those values are in
every row."""
import numpy as np
import pytest
import torch

import oracle

HALVES = np.array([0.5, 1.5, 2.5, 3.5, 62.5, 63.5, 64.5, 100.5, 125.5, 126.5], np.float64)


def tie_row(K):
    """K values: the halves with both signs, cycled, and 127 at position 0
    (so a per-row absmax scale is exactly 1)."""
    vals = np.concatenate([HALVES, -HALVES])
    row = np.resize(vals, K)
    row[0] = 127.0
    return row


def rne(t):
    return np.clip(np.rint(t), -127, 127).astype(np.int8)


def gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import w8a8_post_quantization_sq_b200 as sq

    return sq


# ---------------------------------------------------------------- oracle
def test_oracle_act_ties(orc):
    X = np.stack([tie_row(64), -tie_row(64)]).astype(np.float16)
    q, qs = oracle.quantize_act(X, None, per_token=True)
    assert np.array_equal(qs, np.ones(2, np.float32)) and np.array_equal(q, rne(X.astype(np.float64)))
    # with the division by s: x = 2 v, s = 2
    q2, _ = oracle.quantize_act((2 * X.astype(np.float32)).astype(np.float16), np.full(64, 2, np.float32), True)
    assert np.array_equal(q2, q)
    q3, qs3 = oracle.quantize_act(X, None, per_token=False, static_qs=1.0)
    assert qs3[0] == 1 and np.array_equal(q3, q)


def test_oracle_weight_and_norm_ties(orc):
    W = np.stack([tie_row(128), -tie_row(128)]).astype(np.float32)
    for per_channel in (True, False):
        q, qs = oracle.quantize_weight(W, per_channel)
        assert np.all(qs == 1) and np.array_equal(q, rne(W))
    # RMSNorm, eps 0, rows of +-1: r = 1, v = x * gamma
    K = 256
    x = np.where(np.arange(K) % 2 == 0, 1.0, -1.0)[None, :].astype(np.float32)
    gamma = tie_row(K).astype(np.float32)
    r = oracle.norm_smooth_quant(x, oracle.RMSNORM, gamma, None, 0.0, True)
    assert r["qs"][0] == 1 and np.array_equal(r["Xq"], rne(x * gamma))
    r = oracle.norm_smooth_quant(x, oracle.LAYERNORM, gamma, np.zeros(K, np.float32), 0.0, False, 1.0)
    assert np.array_equal(r["Xq"], rne(x * gamma))


def test_oracle_relu_ties(orc):
    A = np.stack([tie_row(64), -tie_row(64)]).astype(np.float16)
    r = oracle.act_quant(A, oracle.RELU, per_token=False, static_qs=1.0)
    assert np.array_equal(r["Xq"], rne(np.maximum(A.astype(np.float64), 0)))


# ---------------------------------------------------------------- GPU
@pytest.mark.gpu
def test_gpu_quantize_act_ties():
    sq = gpu()
    X = torch.from_numpy(np.stack([tie_row(1024), -tie_row(1024), tie_row(1024)[::-1].copy()])).to(torch.float16)
    expect = rne(X.double().numpy())
    Xd = X.cuda()
    Xq = torch.empty(X.shape, dtype=torch.int8, device="cuda")
    qs = torch.empty(3, device="cuda")
    sq.sq_quantize_act(Xd, None, True, None, Xq, qs)
    torch.cuda.synchronize()
    assert torch.equal(qs.cpu(), torch.ones(3)) and np.array_equal(Xq.cpu().numpy(), expect)
    # v = x / s with s = 2
    s = torch.full((1024,), 2.0, device="cuda")
    sq.sq_quantize_act((2 * Xd.float()).to(torch.float16), s, True, None, Xq, qs)
    torch.cuda.synchronize()
    assert np.array_equal(Xq.cpu().numpy(), expect)
    # static per-tensor scale 1
    q1 = torch.empty(1, device="cuda")
    sq.sq_quantize_act(Xd, None, False, torch.ones(1, device="cuda"), Xq, q1)
    torch.cuda.synchronize()
    assert np.array_equal(Xq.cpu().numpy(), expect)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("per_channel", [True, False])
def test_gpu_quantize_weight_ties(dtype, per_channel):
    sq = gpu()
    rows = [tie_row(2048), -tie_row(2048), np.roll(tie_row(2048), 7)]
    W = torch.from_numpy(np.stack(rows)).to(dtype)
    expect = rne(W.double().numpy())
    Wq = torch.empty(W.shape, dtype=torch.int8, device="cuda")
    qs = torch.empty(3 if per_channel else 1, device="cuda")
    ws = None if per_channel else sq.workspace(sq.SQ_OP_QUANT_WEIGHT, 0, 3, 2048)
    sq.sq_quantize_weight(W.cuda(), None, per_channel, Wq, qs, ws)
    torch.cuda.synchronize()
    assert bool((qs.cpu() == 1).all()) and np.array_equal(Wq.cpu().numpy(), expect)


@pytest.mark.gpu
@pytest.mark.parametrize("I", [64, 3072, 28672])
def test_gpu_relu_ties(I):
    sq = gpu()
    A = torch.from_numpy(np.stack([tie_row(I), -tie_row(I)])).to(torch.float16)
    expect = rne(np.maximum(A.double().numpy(), 0))
    Xq = torch.empty(A.shape, dtype=torch.int8, device="cuda")
    qs = torch.empty(1, device="cuda")
    sq.sq_act_quant(A.cuda(), sq.SQ_ACT_RELU, False, torch.ones(1, device="cuda"), Xq, qs)
    torch.cuda.synchronize()
    assert np.array_equal(Xq.cpu().numpy(), expect)


@pytest.mark.gpu
@pytest.mark.parametrize("K", [1024, 4096, 12288])
@pytest.mark.parametrize("norm", ["ln", "rms"])
@pytest.mark.parametrize("per_token", [True, False])
def test_gpu_norm_ties(K, norm, per_token):
    """eps = 0 and rows of +-1 (mean 0 and mean square 1 exactly, in any
    summation order): r = 1, so v = x gamma (+ 0) hits the ties exactly."""
    sq = gpu()
    M = 4
    x = np.where((np.arange(K)[None, :] + np.arange(M)[:, None]) % 2 == 0, 1.0, -1.0)
    H = torch.from_numpy(x).to(torch.bfloat16)
    gamma = torch.from_numpy(tie_row(K)).float()
    beta = torch.zeros(K) if norm == "ln" else None
    expect = rne(x * tie_row(K)[None, :])
    Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    qs = torch.empty(M if per_token else 1, device="cuda")
    sq.sq_norm_smooth_quant(H.cuda(), sq.SQ_LAYERNORM if norm == "ln" else sq.SQ_RMSNORM, gamma.cuda(),
                            None if beta is None else beta.cuda(), 0.0, per_token,
                            None if per_token else torch.ones(1, device="cuda"), Xq, qs)
    torch.cuda.synchronize()
    if per_token:
        assert bool((qs.cpu() == 1).all())
    assert np.array_equal(Xq.cpu().numpy(), expect)
    # and the oracle agrees
    r = oracle.norm_smooth_quant(H, 0 if norm == "ln" else 1, gamma.numpy(), None if beta is None else beta.numpy(),
                                 0.0, per_token, None if per_token else 1.0)
    assert np.array_equal(r["Xq"], expect)


# ---------------------------------------------------------------- all-zero rows
@pytest.mark.gpu
@pytest.mark.parametrize("K", [1024, 12288])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_gpu_zero_rows_take_the_floor(K, dtype):
    """A row whose largest |v| is 0 takes the scale 127 / 1e-8 ("8位量化" §2.1:
    the absmax guarded by a small floor) and codes 0, in the activation
    quantiser and in the fused norm (RMSNorm, and LayerNorm without a shift,
    where a zero row stays zero), bit for bit with the oracle; the rows around
    it are unaffected."""
    sq = gpu()
    g = torch.Generator().manual_seed(K)
    X = torch.randn((6, K), generator=g).to(dtype)
    X[1] = 0
    X[4] = 0
    Xd = X.cuda()
    Xq = torch.empty((6, K), dtype=torch.int8, device="cuda")
    qs = torch.empty(6, device="cuda")
    sq.sq_quantize_act(Xd, None, True, None, Xq, qs)
    torch.cuda.synchronize()
    rq, rqs = oracle.quantize_act(X.float().numpy(), None, per_token=True)
    assert np.array_equal(Xq.cpu().numpy(), rq) and np.array_equal(qs.cpu().numpy(), rqs)
    assert qs.cpu()[1] == np.float32(127.0) / np.float32(1e-8) and not Xq[1].any()
    gamma = 1 + 0.1 * torch.randn(K, generator=g)
    for nt, on in ((sq.SQ_RMSNORM, oracle.RMSNORM), (sq.SQ_LAYERNORM, oracle.LAYERNORM)):
        sq.sq_norm_smooth_quant(Xd, nt, gamma.cuda(), None, 1e-5, True, None, Xq, qs)
        torch.cuda.synchronize()
        r = oracle.norm_smooth_quant(X, on, gamma.numpy(), None, 1e-5, True)
        assert np.array_equal(Xq.cpu().numpy(), r["Xq"]) and np.array_equal(qs.cpu().numpy(), r["qs"])
        assert qs.cpu()[4] == np.float32(127.0) / np.float32(1e-8) and not Xq[4].any()
