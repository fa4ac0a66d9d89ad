"""The int8 GEMM with the MLP activation in its epilogue (sq_gemm_w8a8_act)
against the oracle ("大语言模型量化技术（四）：SmoothQuant", 融入前序线性层的权重:
down_proj's input is act(gate) * up of the gate/up projection's output).

Stage by stage: the plain GEMM's 16-bit output Y (same operands, scales and
bias) within one ulp of the oracle; then, from the device's own Y bits, the
oracle's activation (SwiGLU on the interleaved gate/up channel pairs, ReLU,
GELU) rounded once to the output dtype must equal the fused H bit for bit,
and with a static per-tensor scale the fused int8 codes must equal the
oracle's codes of the fp32 h. Both CTA-pair and single-CTA tilings (with the
stream-K split where the plan makes one)."""
import numpy as np
import pytest
import torch

import oracle
import w8a8_post_quantization_sq_b200 as sq
from parity_helpers import assert_close_16, npf, npu16

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sq.lib()
    oracle.lib()


def rand_i8(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(-127, 128, shape, generator=g, dtype=torch.int32).to(torch.int8)


def case(M, N, K, seed, with_bias):
    g = torch.Generator().manual_seed(seed)
    Xq, Wq = rand_i8((M, K), seed + 1), rand_i8((N, K), seed + 2)
    # scales that put Y in the activation's interesting range (|y| up to ~10)
    qx = torch.rand(M, generator=g) * 30 + 20
    qw = torch.rand(N, generator=g) * 300 + 200 * (K / 1024) ** 0.5
    bias = torch.randn(N, generator=g) if with_bias else None
    return Xq, Wq, qx, qw, bias


def oracle_act(y, act):
    """h (fp32) of the oracle's activation of a 16-bit Y given as fp32."""
    if act == oracle.SWIGLU:
        A = np.concatenate([y[:, 0::2], y[:, 1::2]], axis=1)  # de-interleave to [gate | up]
    else:
        A = y
    return oracle.act_quant(A, act, quantize=False, want_h=True)["H"]


SHAPES = [(300, 520, 272), (129, 6144, 1024), (1029, 2048, 7200), (2048, 6144, 1024)]


@pytest.mark.parametrize("act", [0, 1, 2])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("pairs", ["", "0"])
def test_gemm_act_16bit(act, dtype, M, N, K, pairs, monkeypatch):
    if pairs:
        monkeypatch.setenv("SQ_GEMM_CTA_PAIRS", pairs)
    else:
        monkeypatch.delenv("SQ_GEMM_CTA_PAIRS", raising=False)
    Xq, Wq, qx, qw, bias = case(M, N, K, M + N + act, with_bias=(act == 2))
    Xd, Wd, qxd, qwd = Xq.to(DEV), Wq.to(DEV), qx.to(DEV), qw.to(DEV)
    bd = None if bias is None else bias.to(DEV)
    ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K)
    Y = torch.empty((M, N), dtype=dtype, device=DEV)
    sq.sq_gemm_w8a8(Xd, Wd, qxd, qwd, bd, Y, ws)
    width = N // 2 if act == 0 else N
    H = torch.full((M, width), 7.0, dtype=dtype, device=DEV)
    sq.sq_gemm_w8a8_act(Xd, Wd, qxd, qwd, bd, act, H, ws)
    torch.cuda.synchronize()
    sq.sq_workspace_status(ws)
    # the plain GEMM on sampled rows against the oracle
    rows = sorted({0, 1, 127, 128, M // 2, M - 1})
    acc = oracle.gemm_i8(Xq[rows].numpy(), Wq.numpy())
    y = oracle.dequant(acc, qx.numpy()[rows], qw.numpy(), None if bias is None else bias.numpy())
    terms = None if bias is None else np.abs(oracle.dequant(acc, qx.numpy()[rows], qw.numpy())) + np.abs(
        bias.numpy().astype(np.float64))[None]
    assert_close_16(Y[rows], y, dtype, terms)
    # the fused activation from the device's own Y bits, every element
    h = oracle_act(npf(Y), act)
    ref = torch.from_numpy(h).to(dtype)
    assert np.array_equal(npu16(H), npu16(ref))


@pytest.mark.parametrize("act", [0, 1, 2])
@pytest.mark.parametrize("M,N,K", [(300, 520, 272), (1029, 2048, 7200), (2048, 6144, 1024)])
def test_gemm_act_static_int8(act, M, N, K):
    """With a static per-tensor scale the epilogue writes the int8 codes of
    the fp32 h: those of sq_act_quant (and of the oracle) with that scale on
    the same Y, values past the scale's range clipped."""
    dtype = torch.float16
    Xq, Wq, qx, qw, bias = case(M, N, K, 7 * M + act, with_bias=False)
    Xd, Wd, qxd, qwd = Xq.to(DEV), Wq.to(DEV), qx.to(DEV), qw.to(DEV)
    ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K)
    Y = torch.empty((M, N), dtype=dtype, device=DEV)
    sq.sq_gemm_w8a8(Xd, Wd, qxd, qwd, None, Y, ws)
    width = N // 2 if act == 0 else N
    torch.cuda.synchronize()
    y = npf(Y)
    A = np.concatenate([y[:, 0::2], y[:, 1::2]], axis=1) if act == 0 else y
    # a scale that clips the largest 1 % of |h|
    h = oracle.act_quant(A, act, quantize=False, want_h=True)["H"]
    qsv = float(np.float32(127.0 / np.quantile(np.abs(h), 0.99)))
    qs = torch.tensor([qsv], device=DEV)
    Q = torch.full((M, width), 99, dtype=torch.int8, device=DEV)
    sq.sq_gemm_w8a8_act(Xd, Wd, qxd, qwd, None, act, Q, ws, static_qs=qs, out_dtype=dtype)
    torch.cuda.synchronize()
    sq.sq_workspace_status(ws)
    r = oracle.act_quant(A, act, per_token=False, static_qs=qsv)
    assert np.array_equal(Q.cpu().numpy(), r["Xq"])
    assert np.abs(r["Xq"]).max() == 127  # the clip was exercised
    if width % 8:
        return  # sq_act_quant takes widths that are multiples of 8
    # the unfused path on the device gives the same codes
    Q2 = torch.empty_like(Q)
    q2 = torch.empty(1, device=DEV)
    Ad = torch.cat([Y[:, 0::2], Y[:, 1::2]], dim=1).contiguous() if act == 0 else Y
    sq.sq_act_quant(Ad, act, False, qs, Q2, q2)
    torch.cuda.synchronize()
    assert torch.equal(Q, Q2)


def test_gemm_act_mlp_chain_c2():
    """The Qwen3-0.6B-shaped MLP with the fused SwiGLU: gate and up weights
    interleaved, smoothed and quantised (up's rows divided by down_proj's
    factors), the gate/up GEMM writing h, per-token int8 of h, the down GEMM;
    h bit for bit against the oracle's SwiGLU of the device's Y, the codes
    and scales against the oracle's quantisation of h, and the down
    projection within one ulp."""
    from w8a8_post_quantization_sq_b200 import inputs

    d = inputs.c2_qwen3_06b(device=DEV)
    M, K, I = 2048, 1024, 3072
    Wg, Wu = d["W"]["gateup"][:I], d["W"]["gateup"][I:]
    W_il = torch.stack([Wg, Wu], dim=1).reshape(2 * I, K).contiguous()  # rows g0, u0, g1, u1, ...
    g = torch.Generator(device=DEV).manual_seed(3)
    s = torch.rand(K, generator=g, device=DEV) + 0.5
    s_next = torch.ones(2 * I, device=DEV)
    s_next[1::2] = torch.rand(I, generator=g, device=DEV) + 0.5
    Wq = torch.empty((2 * I, K), dtype=torch.int8, device=DEV)
    qw = torch.empty(2 * I, device=DEV)
    sq.sq_quantize_weight_fold_prev(W_il, s_next, s, Wq, qw)
    Xq, qx = d["down_in"]  # a stand-in int8 input of the gate/up projection
    Xq = Xq[:, :K].contiguous()
    ws = sq.workspace(sq.SQ_OP_GEMM, M, 2 * I, K)
    H = torch.empty((M, I), dtype=torch.bfloat16, device=DEV)
    sq.sq_gemm_w8a8_act(Xq, Wq, qx, qw, None, sq.SQ_ACT_SWIGLU, H, ws)
    Y = torch.empty((M, 2 * I), dtype=torch.bfloat16, device=DEV)
    sq.sq_gemm_w8a8(Xq, Wq, qx, qw, None, Y, ws)
    Xd = torch.empty((M, I), dtype=torch.int8, device=DEV)
    qd = torch.empty(M, device=DEV)
    sq.sq_quantize_act(H, None, True, None, Xd, qd)
    Wdq = torch.empty((K, I), dtype=torch.int8, device=DEV)
    qwd = torch.empty(K, device=DEV)
    sq.sq_quantize_weight(d["W"]["down"], None, True, Wdq, qwd)
    Out = torch.empty((M, K), dtype=torch.bfloat16, device=DEV)
    sq.sq_gemm_w8a8(Xd, Wdq, qd, qwd, None, Out, sq.workspace(sq.SQ_OP_GEMM, M, K, I))
    torch.cuda.synchronize()
    h = oracle_act(npf(Y), oracle.SWIGLU)
    assert np.array_equal(npu16(H), npu16(torch.from_numpy(h).to(torch.bfloat16)))
    rq, rqs = oracle.quantize_act(npf(H), None, per_token=True)
    assert np.array_equal(Xd.cpu().numpy(), rq) and np.array_equal(npf(qd), rqs)
    rows = [0, 1, 1029, M - 1]
    acc = oracle.gemm_i8(rq[rows], Wdq.cpu().numpy())
    assert_close_16(Out[rows], oracle.dequant(acc, rqs[rows], npf(qwd)), torch.bfloat16)
