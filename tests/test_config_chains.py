"""End-to-end parity of every configuration's chain, through the C ABI,
against the CPU oracle on the same inputs.

C1 (the single linear layer of "如何通过 SmoothQuant 解决激活值离群点难题" §3):
calibration on X itself, s, per-tensor int8 of X/s and of W·s, the int32 GEMM
(bit-exact) and the fp16 output (within one ulp).

C2, C3, C5: the benchmark's own deploy-mode stacks (bench.Stack), offline pass
then one online step, checked stage by stage:
  calibration maxima (the running column absmax over every calibration batch,
  or the norm's calibration mode), the weight maxima of each consumer, the
  smoothing factors for every alpha of the configuration and the folded gamma
  and beta, the static per-tensor scales (C3) -- all bit-exact and in full;
  the int8 weights and their scales on sampled output channels (bit-exact,
  every input channel); the norm + smoothing + int8 codes and scales on
  sampled tokens (bit-exact); the four GEMM outputs on sampled tokens (within
  one ulp of the oracle's fp64 value rounded to the output type), each GEMM
  taking the device's int8 operands, which the stages before it checked.
"""
import numpy as np
import pytest
import torch

import bench
import oracle
import w8a8_post_quantization_sq_b200 as sq
from parity_helpers import assert_close_16, npf
from w8a8_post_quantization_sq_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sq.lib()
    oracle.lib()


def test_c1_single_linear_chain():
    """X fp16 [16, 1024] (channel 0 x50), W fp16 [1024, 1024], alpha 0.5,
    per-tensor int8 for both, calibrated on X itself; int32 and fp16 out."""
    d = inputs.c1_single_linear()
    X, W = d["X"], d["W"]
    M, K, N = 16, 1024, 1024
    xmax = torch.zeros(K, device=DEV)
    wmax = torch.zeros(K, device=DEV)
    sq.sq_calib_absmax(X.to(DEV), xmax)
    sq.sq_weight_absmax(W.to(DEV), wmax)
    s = torch.empty(K, device=DEV)
    sq.sq_smooth_scales(xmax, wmax, d["alpha"], s)
    Xq = torch.empty((M, K), dtype=torch.int8, device=DEV)
    qx = torch.empty(1, device=DEV)
    sq.sq_quantize_act(X.to(DEV), s, False, None, Xq, qx, sq.workspace(sq.SQ_OP_QUANT_ACT, M, 0, K))
    Wq = torch.empty((N, K), dtype=torch.int8, device=DEV)
    qw = torch.empty(1, device=DEV)
    sq.sq_quantize_weight(W.to(DEV), s, False, Wq, qw, sq.workspace(sq.SQ_OP_QUANT_WEIGHT, 0, N, K))
    acc = torch.empty((M, N), dtype=torch.int32, device=DEV)
    ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K)
    sq.sq_gemm_w8a8(Xq, Wq, qx, qw, None, acc, ws)
    Y = torch.empty((M, N), dtype=torch.float16, device=DEV)
    sq.sq_gemm_w8a8(Xq, Wq, qx, qw, None, Y, ws)
    torch.cuda.synchronize()
    sq.sq_workspace_status(ws)

    rx, rw = oracle.col_absmax(X), oracle.col_absmax(W)
    assert np.array_equal(npf(xmax), rx) and np.array_equal(npf(wmax), rw)
    rs = oracle.smooth_scales(rx, rw, d["alpha"])
    assert np.array_equal(npf(s), rs)
    rXq, rqx = oracle.quantize_act(X, rs, per_token=False)
    assert np.array_equal(Xq.cpu().numpy(), rXq) and np.array_equal(npf(qx), rqx)
    rWq, rqw = oracle.quantize_weight(oracle.fold_weight(W, rs), per_channel=False)
    assert np.array_equal(Wq.cpu().numpy(), rWq) and np.array_equal(npf(qw), rqw)
    racc = oracle.gemm_i8(rXq, rWq)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), racc)
    assert_close_16(Y, oracle.dequant(racc, rqx, rqw), torch.float16)
    # the smoothing did its job on the outlier channel: X/s has a far smaller
    # per-tensor range than X, so fewer codes of the other channels round to 0
    q0, _ = oracle.quantize_act(X, None, per_token=False)
    assert np.count_nonzero(rXq[:, 1:]) > np.count_nonzero(q0[:, 1:])


def sample_rows(n, k, seed):
    g = np.random.default_rng(seed)
    fixed = {0, 1, 127, 128, n // 2, n - 1}
    return np.array(sorted(fixed | set(g.choice(n, size=min(k, n), replace=False).tolist())))


def col_absmax_chunked(X, running=None, chunk=4096):
    """The oracle's running column absmax over a device tensor, a row block at
    a time (the running max is the same over any split of the rows)."""
    r = running
    for a in range(0, X.shape[0], chunk):
        r = oracle.col_absmax(X[a:a + chunk].cpu(), r)
    return r


@pytest.mark.parametrize("name", ["c2", "c3", "c5"])
def test_stack_chain(name):
    st = bench.Stack(name, torch.device(DEV, 0))
    cfg = st.cfg
    st.offline()
    st.step()
    torch.cuda.synchronize()
    for w in st.ws:
        sq.sq_workspace_status(st.ws[w])
    d = st.d
    eps, M, K = d["eps"], st.M, st.K
    norm = oracle.LAYERNORM if cfg["norm"] == "layer" else oracle.RMSNORM
    g = {k: npf(st.gamma[k]) for k in st.sides}
    b = {k: None if st.beta[k] is None else npf(st.beta[k]) for k in st.sides}

    # calibration maxima over every batch
    x = {}
    for k in st.sides:
        r = np.zeros(K, np.float32)
        for X in d["calib"]:
            if cfg["calib"] == "absmax":
                r = col_absmax_chunked(X, r)
            else:
                r = oracle.norm_smooth_quant(X.cpu(), norm, g[k], b[k], eps, quantize=False, absmax=r)["absmax"]
        x[k] = r
        assert np.array_equal(npf(st.xmax[k]), r), f"calibration maxima ({k})"
    # weight maxima of each side's consumer
    wmax = {}
    for k in st.sides:
        wmax[k] = col_absmax_chunked(st.W[st.consumer[k]])
        assert np.array_equal(npf(st.wmax[k]), wmax[k]), f"weight maxima ({k})"
    # smoothing factors for every alpha, folded norm parameters for the deployed one
    s = {}
    for a in cfg["alphas"]:
        for k in st.sides:
            ra = oracle.smooth_scales(x[k], wmax[k], a)
            assert np.array_equal(npf(st.s[a][k]), ra), f"s (alpha {a}, {k})"
            if a == cfg["alpha"]:
                s[k] = ra
    gp, bp = {}, {}
    for k in st.sides:
        gp[k], bp[k] = oracle.fold_norm(g[k], b[k], s[k])
        assert np.array_equal(npf(st.gp[k]), gp[k])
        if bp[k] is not None:
            assert np.array_equal(npf(st.bp[k]), bp[k])
    # static per-tensor scales: a calibration pass of the smoothed norm
    qs_static = {}
    if not cfg["per_token"]:
        for k in st.sides:
            v = np.zeros(K, np.float32)
            for X in d["calib"]:
                v = oracle.norm_smooth_quant(X.cpu(), norm, gp[k], bp[k], eps, quantize=False, absmax=v)["absmax"]
            assert np.array_equal(npf(st.vmax[k]), v)
            qs_static[k] = oracle.scale_from_absmax(v)
            assert npf(st.qs_static[k])[0] == qs_static[k]
    # int8 weights on sampled output channels
    for i, (w, src) in enumerate(cfg["gemms"]):
        W = st.W[w]
        rows = sample_rows(W.shape[0], 58, i)
        Wr = W[torch.from_numpy(rows).to(W.device)].cpu()
        Wp = oracle.fold_weight(Wr, s[src]) if src != "syn" else oracle.f32(Wr)
        rq, rqs = oracle.quantize_weight(Wp, True)
        assert np.array_equal(st.Wq[w][torch.from_numpy(rows).to(W.device)].cpu().numpy(), rq), w
        assert np.array_equal(npf(st.qw[w])[rows], rqs), w
    # the online step on sampled tokens
    toks = sample_rows(M, 10, 99)
    ti = torch.from_numpy(toks).to(DEV)
    for k in st.sides:
        r = oracle.norm_smooth_quant(st.h[k][ti].cpu(), norm, gp[k], bp[k], eps, cfg["per_token"],
                                     None if cfg["per_token"] else qs_static[k])
        assert np.array_equal(st.Xq[k][ti].cpu().numpy(), r["Xq"]), f"norm codes ({k})"
        got_qs = npf(st.qx[k])[toks] if cfg["per_token"] else npf(st.qx[k])
        assert np.array_equal(got_qs, r["qs"]), f"norm scales ({k})"
    for w, src in cfg["gemms"]:
        if src == "syn":
            xq, qx = st.syn[w]
        else:
            xq, qx = st.Xq[src], st.qx[src]
        qxs = npf(qx)
        qxs = qxs[toks] if qxs.size > 1 else qxs
        y = oracle.dequant(oracle.gemm_i8(xq[ti].cpu().numpy(), st.Wq[w].cpu().numpy()), qxs, npf(st.qw[w]))
        assert_close_16(st.Y[w][ti], y, st.out_dtype)
