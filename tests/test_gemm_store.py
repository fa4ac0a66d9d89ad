"""The GEMM's 16-bit outputs leave by TMA store (32 x 32 boxes from a
64-byte-swizzled staging area, rows and columns past the edge clipped by the
copy engine). These tests check every output element and every byte around
the output ("8位量化：异常值与混合精度分解实战" §2.1: Y = acc / (qs_x qs_w)):

  - Y as a strided view into a larger buffer (ldy > N, extra rows below M)
    filled with a sentinel: the padding columns and rows keep the sentinel,
    so no box writes past the edges the call was given;
  - every element against the same dequantisation written in plain PyTorch
    fp32 from the kernel's own exact int32 sums (the int32 output is pinned
    against the oracle elsewhere): y = fl(acc * fl(fl(1/qs_x) fl(1/qs_w)))
    rounded once to 16 bits, bit for bit;
  - batched problems with a ragged last row tile: no problem's rows spill into
    the next one's, and nothing lands past the last problem.
Shapes cover a single row, ragged row and column tiles, CTA pairs and single
CTAs (with the stream-K split where the plan makes one)."""
import numpy as np
import pytest
import torch

import w8a8_post_quantization_sq_b200 as sq

pytestmark = pytest.mark.gpu
DEV = "cuda"
SENTINEL = 0x7E55  # a NaN pattern in both 16-bit types: never a GEMM result


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sq.lib()


def rand_i8(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(-127, 128, shape, generator=g, dtype=torch.int32).to(torch.int8)


def dequant_ref(acc, qx, qw, dtype):
    """The epilogue's arithmetic in torch fp32 (correctly rounded operations
    in the kernel's order), then one rounding to 16 bits."""
    d = (1.0 / qx)[:, None] * (1.0 / qw)[None, :]
    return (acc.float() * d).to(dtype)


SHAPES = [(1, 8, 16), (129, 40, 64), (300, 520, 272), (257, 264, 128), (1029, 2048, 7200), (2048, 6144, 1024)]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("pairs", ["", "0"])
def test_tma_store_edges(dtype, M, N, K, pairs, monkeypatch):
    if pairs:
        monkeypatch.setenv("SQ_GEMM_CTA_PAIRS", pairs)
    else:
        monkeypatch.delenv("SQ_GEMM_CTA_PAIRS", raising=False)
    g = torch.Generator().manual_seed(M + N + K)
    Xq, Wq = rand_i8((M, K), M + 1).to(DEV), rand_i8((N, K), N + 2).to(DEV)
    qx = (torch.rand(M, generator=g) * 30 + 20).to(DEV)
    qw = (torch.rand(N, generator=g) * 300 + 200).to(DEV)
    ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K)
    acc = torch.empty((M, N), dtype=torch.int32, device=DEV)
    sq.sq_gemm_w8a8(Xq, Wq, None, None, None, acc, ws)
    ldy = N + 24  # a multiple of 8: 16-byte aligned rows
    big = torch.full((M + 3, ldy), SENTINEL, dtype=torch.int16, device=DEV)
    Y = big.view(dtype)[:M, :N]
    sq.sq_gemm_w8a8(Xq, Wq, qx, qw, None, Y, ws)
    torch.cuda.synchronize()
    sq.sq_workspace_status(ws)
    ref = dequant_ref(acc, qx, qw, dtype)
    assert torch.equal(Y.contiguous().view(torch.int16), ref.view(torch.int16))
    assert bool((big[:, N:] == SENTINEL).all()), "a store landed in the padding columns"
    assert bool((big[M:] == SENTINEL).all()), "a store landed below the last row"


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("batch,M,N,K", [(3, 100, 72, 64), (5, 257, 136, 128), (2, 2048, 2048, 128)])
def test_tma_store_batched(dtype, batch, M, N, K):
    A = torch.stack([rand_i8((M, K), 300 + b) for b in range(batch)]).to(DEV)
    B = torch.stack([rand_i8((N, K), 400 + b) for b in range(batch)]).to(DEV)
    g = torch.Generator().manual_seed(batch * M)
    qa = (torch.rand(batch * M, generator=g) * 30 + 20).to(DEV)
    qb = (torch.rand(batch * N, generator=g) * 300 + 200).to(DEV)
    ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K)
    acc = torch.empty((batch, M, N), dtype=torch.int32, device=DEV)
    sq.sq_bmm_w8a8(A, B, None, None, acc, ws)
    n = batch * M * N
    flat = torch.full((n + 4096,), SENTINEL, dtype=torch.int16, device=DEV)
    Y = flat[:n].view(dtype).view(batch, M, N)
    sq.sq_bmm_w8a8(A, B, qa.view(batch, M), qb.view(batch, N), Y, ws)
    torch.cuda.synchronize()
    sq.sq_workspace_status(ws)
    for b in range(batch):
        ref = dequant_ref(acc[b], qa[b * M:(b + 1) * M], qb[b * N:(b + 1) * N], dtype)
        assert torch.equal(Y[b].view(torch.int16), ref.view(torch.int16)), f"problem {b}"
    assert bool((flat[n:] == SENTINEL).all()), "a store landed past the last problem"


def test_unaligned_rows_take_plain_stores():
    """Rows that do not start on 16-byte boundaries (ldy = N + 3) cannot be
    described to the copy engine; the plain-store path writes the same values
    and leaves the padding alone."""
    M, N, K = 200, 72, 128
    Xq, Wq = rand_i8((M, K), 1).to(DEV), rand_i8((N, K), 2).to(DEV)
    qx, qw = torch.full((M,), 40.0, device=DEV), torch.linspace(200, 500, N, device=DEV)
    ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K)
    acc = torch.empty((M, N), dtype=torch.int32, device=DEV)
    sq.sq_gemm_w8a8(Xq, Wq, None, None, None, acc, ws)
    big = torch.full((M, N + 3), SENTINEL, dtype=torch.int16, device=DEV)
    Y = big.view(torch.bfloat16)[:, :N]
    sq.sq_gemm_w8a8(Xq, Wq, qx, qw, None, Y, ws)
    torch.cuda.synchronize()
    ref = dequant_ref(acc, qx, qw, torch.bfloat16)
    assert np.array_equal(Y.contiguous().view(torch.int16).cpu().numpy(), ref.view(torch.int16).cpu().numpy())
    assert bool((big[:, N:] == SENTINEL).all())
