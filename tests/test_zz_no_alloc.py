"""sq_llmint8_detect_noalloc: outlier detection for callers that cannot
allocate device memory or pass scratch to the library (a plugin slot that is
given only its inputs and outputs, a memory plan with no room to spare, a
service that must not allocate while serving). Its scratch is a fixed device
array inside the library, so its results must equal those of
sq_llmint8_detect, which takes a caller workspace, call after call.

This file is collected last on purpose; it passes on its own in a fresh
process and after the rest of the suite.
"""
import ctypes

import pytest
import torch

import w8a8_post_quantization_sq_b200 as sq
from w8a8_post_quantization_sq_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sq.lib()


def _detect_both(X, thr, min_ratio):
    M, K = X.shape
    idx_ws = torch.full((K,), -1, dtype=torch.int32, device="cuda")
    n_ws = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    ws = sq.workspace(sq.SQ_OP_LLMINT8_DETECT, M, 0, K)
    sq.sq_llmint8_detect(X, thr, min_ratio, idx_ws, n_ws, ws)
    idx_na = torch.full((K,), -2, dtype=torch.int32, device="cuda")
    n_na = torch.full((1,), -2, dtype=torch.int32, device="cuda")
    sq.sq_llmint8_detect_noalloc(X, thr, min_ratio, idx_na, n_na)
    torch.cuda.synchronize()
    n1, n2 = int(n_ws.item()), int(n_na.item())
    return n1, idx_ws[:n1].cpu().tolist(), n2, idx_na[:n2].cpu().tolist()


def test_noalloc_matches_workspace_entry_point_two_calls_in_a_row():
    # first call: the 6.7B-shaped input (16 bands x 4096 columns of counts)
    d = inputs.c4_llmint8(device="cpu", M=2048, K=4096, N=64, n_out=6, seed=0)
    n1, i1, n2, i2 = _detect_both(d["X"].cuda(), 6.0, 0.0)
    assert n1 == n2 == 6 and i1 == i2 == d["dims"].tolist()
    # second call right after: another size, dtype and ratio; stale counts
    # from the first call must not leak into it
    d = inputs.c4_llmint8(device="cpu", M=300, K=1024, N=64, n_out=3, seed=5)
    X = d["X"].to(torch.bfloat16).cuda()
    for mr in (0.0, 0.06):
        n1, i1, n2, i2 = _detect_both(X, 6.0, mr)
        assert n1 == n2 and i1 == i2
    n1, i1, n2, i2 = _detect_both(X, 6.0, 0.0)
    assert i1 == i2 == d["dims"].tolist()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    L = sq.lib()
    X = torch.zeros((8, 8192), dtype=torch.float16, device="cuda")
    idx = torch.zeros(8192, dtype=torch.int32, device="cuda")
    n = torch.full((1,), 77, dtype=torch.int32, device="cuda")
    # 1000 bands x 8192 columns of counts do not fit in 4 MiB; nothing may run
    st = L.sq_llmint8_detect_noalloc(ctypes.c_void_p(X.data_ptr()), 1, 128 * 1000, 8192, 8192, 6.0, 0.0,
                                     ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(n.data_ptr()), None)
    assert st == 2
    assert "scratch" in L.sq_last_error_string().decode()
    torch.cuda.synchronize()
    assert int(n.item()) == 77
