"""The int8 GEMM on CTA pairs (cta_group::2: 256-row tiles, each CTA of the
pair loading its own rows of Xq and half of the weight tile) against the
oracle, and against the single-CTA kernel bit for bit: both sum the same
exact int32 products and run the same epilogue arithmetic, so every output
type must agree exactly. SQ_GEMM_CTA_PAIRS=1 makes the plan use pairs for
every 256-wide tiling, whatever the size."""
import numpy as np
import pytest
import torch

import oracle
import w8a8_post_quantization_sq_b200 as sq
from parity_helpers import assert_close_16, assert_close_f32, npf

pytestmark = pytest.mark.gpu
DEV = "cuda"

# ragged in every dimension: M past a 256-row pair tile (the second CTA's rows
# all past M), N not a multiple of 256, K with a partial last k-block, and
# shapes with several waves of pairs
SHAPES = [(256, 256, 128), (300, 520, 272), (129, 4096, 1024), (1000, 1000, 1040), (2048, 4096, 1024),
          (512, 768, 16400)]


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sq.lib()
    oracle.lib()


def rand_i8(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(-127, 128, shape, generator=g, dtype=torch.int32).to(torch.int8)


def run(Xd, Wd, qx, qw, bias, Y, mode, monkeypatch, fp8=False):
    monkeypatch.setenv("SQ_GEMM_CTA_PAIRS", mode)
    M, K = Xd.shape
    N = Wd.shape[0]
    ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K)
    if fp8:
        sq.sq_gemm_fp8(Xd, Wd, qx, qw, bias, Y, ws)
    else:
        sq.sq_gemm_w8a8(Xd, Wd, qx, qw, bias, Y, ws)
    torch.cuda.synchronize()
    sq.sq_workspace_status(ws)


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_pairs_int32_exact(M, N, K, monkeypatch):
    Xq, Wq = rand_i8((M, K), M + 11), rand_i8((N, K), N + 12)
    Xd, Wd = Xq.to(DEV), Wq.to(DEV)
    Y2 = torch.full((M, N), 7, dtype=torch.int32, device=DEV)
    run(Xd, Wd, None, None, None, Y2, "1", monkeypatch)
    ref = oracle.gemm_i8(Xq.numpy(), Wq.numpy())
    assert np.array_equal(Y2.cpu().numpy().astype(np.int64), ref)
    Y1 = torch.empty_like(Y2)
    run(Xd, Wd, None, None, None, Y1, "0", monkeypatch)
    assert torch.equal(Y1, Y2)


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("per_token,per_channel,with_bias", [(True, True, False), (False, False, True)])
def test_pairs_dequant(out_dtype, per_token, per_channel, with_bias, monkeypatch):
    M, N, K = 300, 520, 1040
    Xq, Wq = rand_i8((M, K), 41), rand_i8((N, K), 42)
    g = torch.Generator().manual_seed(43)
    qx = torch.rand(M if per_token else 1, generator=g) * 100 + 1
    qw = torch.rand(N if per_channel else 1, generator=g) * 5000 + 100
    bias = torch.randn(N, generator=g) if with_bias else None
    args = (Xq.to(DEV), Wq.to(DEV), qx.to(DEV), qw.to(DEV), None if bias is None else bias.to(DEV))
    Y2 = torch.empty((M, N), dtype=out_dtype, device=DEV)
    run(*args, Y2, "1", monkeypatch)
    acc = oracle.gemm_i8(Xq.numpy(), Wq.numpy())
    y = oracle.dequant(acc, qx.numpy(), qw.numpy(), None if bias is None else bias.numpy())
    terms = np.abs(oracle.dequant(acc, qx.numpy(), qw.numpy()))
    if bias is not None:
        terms = terms + np.abs(bias.numpy().astype(np.float64))[None, :]
    if out_dtype == torch.float32:
        assert_close_f32(Y2, y, terms)
    else:
        assert_close_16(Y2, y, out_dtype, terms if bias is not None else None)
    Y1 = torch.empty_like(Y2)
    run(*args, Y1, "0", monkeypatch)
    assert torch.equal(Y1.view(torch.uint8), Y2.view(torch.uint8))


def test_pairs_strided_output(monkeypatch):
    """Y with a row stride past N: the pair kernel writes no byte outside the
    [M, N] window."""
    M, N, K = 300, 520, 272
    Xq, Wq = rand_i8((M, K), 51), rand_i8((N, K), 52)
    big = torch.full((M, N + 40), -3, dtype=torch.int32, device=DEV)
    run(Xq.to(DEV), Wq.to(DEV), None, None, None, big[:, :N], "1", monkeypatch)
    assert np.array_equal(big[:, :N].cpu().numpy().astype(np.int64), oracle.gemm_i8(Xq.numpy(), Wq.numpy()))
    assert bool((big[:, N:] == -3).all())


def test_pairs_fp8(monkeypatch):
    M, N, K = 300, 520, 1040
    g = torch.Generator().manual_seed(61)
    A = torch.randint(0, 256, (M, K), generator=g, dtype=torch.int32)
    B = torch.randint(0, 256, (N, K), generator=g, dtype=torch.int32)
    A = torch.where((A & 0x7F) == 0x7F, A - 1, A).to(torch.uint8)
    B = torch.where((B & 0x7F) == 0x7F, B - 1, B).to(torch.uint8)
    qx = torch.rand(M, generator=g) + 1
    qw = torch.rand(N, generator=g) + 10
    args = (A.to(DEV), B.to(DEV), qx.to(DEV), qw.to(DEV), None)
    Y2 = torch.empty((M, N), dtype=torch.float32, device=DEV)
    run(*args, Y2, "1", monkeypatch, fp8=True)
    Y1 = torch.empty_like(Y2)
    run(*args, Y1, "0", monkeypatch, fp8=True)
    assert torch.equal(Y1, Y2)
    acc = oracle.gemm_fp8(A.numpy(), B.numpy())
    y = oracle.dequant_f64(acc, qx.numpy(), qw.numpy())
    # the fp32 tensor-core sum of exact products: within K 2^-23 sum|a b| / (qx qw)
    av = np.vectorize(oracle.e4m3_value)(A.numpy()).astype(np.float64)
    bv = np.vectorize(oracle.e4m3_value)(B.numpy()).astype(np.float64)
    bound = K * 2.0 ** -23 * (np.abs(av) @ np.abs(bv).T) / np.outer(qx.numpy(), qw.numpy()) + 1e-6 * np.abs(y)
    assert np.all(np.abs(npf(Y2) - y) <= bound)


def test_pairs_batched(monkeypatch):
    """The batched form (attention's products) on pairs: each problem's rows
    past M read as zero rows of its own problem, never the next problem's."""
    b, M, N, K = 3, 200, 300, 272
    A, B = rand_i8((b, M, K), 71), rand_i8((b, N, K), 72)
    Y = torch.empty((b, M, N), dtype=torch.int32, device=DEV)
    monkeypatch.setenv("SQ_GEMM_CTA_PAIRS", "1")
    ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K)
    sq.sq_bmm_w8a8(A.to(DEV), B.to(DEV), None, None, Y, ws)
    torch.cuda.synchronize()
    sq.sq_workspace_status(ws)
    assert np.array_equal(Y.cpu().numpy().astype(np.int64), oracle.bmm_i8(A.numpy(), B.numpy()))


def test_pairs_llmint8_epilogue(monkeypatch):
    """The LLM.int8 call (int8 GEMM with the fused 16-bit outlier term) on
    pairs agrees bit for bit with the single-CTA kernel."""
    from w8a8_post_quantization_sq_b200 import inputs

    d = inputs.c4_llmint8(device="cpu", M=300, K=1024, N=520, n_out=5, seed=9)
    X = d["X"].to(DEV)
    out = []
    for mode in ("1", "0"):
        monkeypatch.setenv("SQ_GEMM_CTA_PAIRS", mode)
        st = sq.llmint8_weight_state(d["W"].to(DEV))
        Y = torch.empty((300, 520), dtype=torch.float16, device=DEV)
        idx = torch.empty(1024, dtype=torch.int32, device=DEV)
        n = torch.empty(1, dtype=torch.int32, device=DEV)
        ws = sq.workspace(sq.SQ_OP_LLMINT8, 300, 520, 1024)
        sq.sq_llmint8_matmul(X, st, 6.0, 0.0, Y, idx, n, ws)
        torch.cuda.synchronize()
        sq.sq_workspace_status(ws)
        out.append(Y)
    assert torch.equal(out[0].view(torch.int16), out[1].view(torch.int16))


@pytest.mark.parametrize("act", [0, 1, 2])
def test_pairs_fused_activation(act, monkeypatch):
    """The fused activation on CTA pairs equals the single-CTA kernel's bit
    for bit (16-bit h and static-scale codes)."""
    M, N, K = 300, 1040, 1040
    Xq, Wq = rand_i8((M, K), 81 + act), rand_i8((N, K), 82 + act)
    g = torch.Generator().manual_seed(83)
    qx = torch.rand(M, generator=g) * 30 + 20
    qw = torch.rand(N, generator=g) * 300 + 200
    Xd, Wd, qxd, qwd = Xq.to(DEV), Wq.to(DEV), qx.to(DEV), qw.to(DEV)
    width = N // 2 if act == 0 else N
    outs = []
    for mode in ("1", "0"):
        monkeypatch.setenv("SQ_GEMM_CTA_PAIRS", mode)
        ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K)
        H = torch.empty((M, width), dtype=torch.bfloat16, device=DEV)
        sq.sq_gemm_w8a8_act(Xd, Wd, qxd, qwd, None, act, H, ws)
        Q = torch.empty((M, width), dtype=torch.int8, device=DEV)
        sq.sq_gemm_w8a8_act(Xd, Wd, qxd, qwd, None, act, Q, ws, static_qs=torch.tensor([3.0], device=DEV),
                            out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        sq.sq_workspace_status(ws)
        outs.append((H, Q))
    assert torch.equal(outs[0][0].view(torch.int16), outs[1][0].view(torch.int16))
    assert torch.equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("M,N,K,dtype", [(2048, 6144, 8192, torch.bfloat16), (2000, 6100, 8320, torch.float16),
                                         (2048, 6144, 8192, torch.float32)])
def test_pairs_stream_k(M, N, K, dtype, monkeypatch):
    """A ragged last wave of pair tiles cut by k-blocks, one range per CTA pair
    (each CTA of a pair parks and counts its own half of a tile; the piece
    that completes a half adds the parks up): 192 pair tiles over 74 pairs,
    k-loops of 64 and 65 blocks.
    int32 sums exact against the CUDA library's int8 matmul, the dequantised
    output bit for bit against the single-CTA kernel (same int32 sums, same
    epilogue arithmetic), and sampled rows against the oracle; the split's
    counters are left at zero, so a second call on the workspace is exact too."""
    monkeypatch.delenv("SQ_GEMM_CTA_PAIRS", raising=False)
    if M == 2048:
        assert sq.sq_workspace_size(sq.SQ_OP_GEMM, M, N, K) > 30 << 20, "the plan was expected to split on pairs"
    Xq, Wq = rand_i8((M, K), M + 21), rand_i8((N, K), N + 22)
    Xd, Wd = Xq.to(DEV), Wq.to(DEV)
    ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K)
    Y32 = torch.empty((M, N), dtype=torch.int32, device=DEV)
    for _ in range(2):
        sq.sq_gemm_w8a8(Xd, Wd, None, None, None, Y32, ws)
        torch.cuda.synchronize()
        sq.sq_workspace_status(ws)
        if N % 8 == 0:
            assert torch.equal(Y32, torch._int_mm(Xd, Wd.t()))
    rows = [0, 255, 256, M // 2, M - 1]
    ref = oracle.gemm_i8(Xq[rows].numpy(), Wq.numpy())
    assert np.array_equal(Y32[rows].cpu().numpy().astype(np.int64), ref)
    g = torch.Generator().manual_seed(M + N)
    qx = (torch.rand(M, generator=g) * 30 + 20).to(DEV)
    qw = (torch.rand(N, generator=g) * 300 + 200).to(DEV)
    Y2 = torch.empty((M, N), dtype=dtype, device=DEV)
    sq.sq_gemm_w8a8(Xd, Wd, qx, qw, None, Y2, ws)
    torch.cuda.synchronize()
    sq.sq_workspace_status(ws)
    Y1 = torch.empty_like(Y2)
    run(Xd, Wd, qx, qw, None, Y1, "0", monkeypatch)
    assert torch.equal(Y1.view(torch.int16 if dtype != torch.float32 else torch.int32),
                       Y2.view(torch.int16 if dtype != torch.float32 else torch.int32))


def test_stream_k_workspace_shared_between_shapes(monkeypatch):
    """One workspace, sized for the larger of two shapes that both split their
    last wave, used by each in turn: single CTAs cutting 76 tiles
    (1024 x 7168 x 7168), then CTA pairs cutting 44 pair tiles
    (2048 x 6144 x 8192), then the first shape again. The arrival counters sit
    at the same bytes for every shape, so the partial sums one shape parks
    are never read as the other's counters: every call exact against the
    CUDA library's int8 matmul."""
    monkeypatch.delenv("SQ_GEMM_CTA_PAIRS", raising=False)
    shapes = [(1024, 7168, 7168), (2048, 6144, 8192), (1024, 7168, 7168)]
    size = max(sq.sq_workspace_size(sq.SQ_OP_GEMM, M, N, K) for M, N, K in shapes)
    assert all(sq.sq_workspace_size(sq.SQ_OP_GEMM, M, N, K) > 256 for M, N, K in shapes), "both shapes split"
    ws = torch.zeros(size, dtype=torch.uint8, device=DEV)
    for i, (M, N, K) in enumerate(shapes):
        Xd, Wd = rand_i8((M, K), 700 + i).to(DEV), rand_i8((N, K), 800 + i).to(DEV)
        Y32 = torch.empty((M, N), dtype=torch.int32, device=DEV)
        sq.sq_gemm_w8a8(Xd, Wd, None, None, None, Y32, ws)
        torch.cuda.synchronize()
        sq.sq_workspace_status(ws)
        assert torch.equal(Y32, torch._int_mm(Xd, Wd.t())), f"call {i}: {M} x {N} x {K}"
