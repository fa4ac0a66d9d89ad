"""The fused norm + int8 codes against the fp64 norm, independently of the
summation order ("大语言模型量化技术（四）：SmoothQuant", 融入 LayerNorm;
"8位量化：异常值与混合精度分解实战" §2.1 round / clip): every code that the
fp64 value decides (no tie point within the error bound of norm_bound.py) is
the fp64 code exactly; the rest are neighbours and are counted. The oracle is
checked here on the CPU; the GPU path against the same reference in
test_norm_orderfree_gpu."""
import numpy as np
import pytest
import torch

import oracle
from norm_bound import check_codes, reference_codes


def inputs(M, K, seed, norm, outliers=True):
    g = torch.Generator().manual_seed(seed)
    h = torch.randn((M, K), generator=g)
    if outliers:
        ch = torch.randperm(K, generator=g)[:max(1, K // 1000)]
        h[:, ch] *= 60.0
    H = h.to(torch.bfloat16)
    gamma = (1 + 0.1 * torch.randn(K, generator=g)).numpy()
    beta = (0.1 * torch.randn(K, generator=g)).numpy() if norm == 0 else None
    return H, gamma, beta


@pytest.mark.parametrize("norm", [0, 1])
@pytest.mark.parametrize("K", [1024, 7168, 12288])
@pytest.mark.parametrize("per_token", [True, False])
def test_oracle_norm_codes_order_free(norm, K, per_token, orc):
    M = 48
    H, gamma, beta = inputs(M, K, K + norm, norm)
    eps = 1e-5 if norm == 0 else 1e-6
    Hf = H.float().numpy()
    static = None
    if not per_token:
        v = oracle.norm_f64(Hf, norm, gamma, beta, eps)
        static = float(np.float32(127.0 / np.abs(v).max() * 1.3))  # some values clip
    r = oracle.norm_smooth_quant(H, norm, gamma, beta, eps, per_token, static)
    ref = reference_codes(Hf, norm, gamma, beta, eps, per_token, static)
    n_near, n_diff = check_codes(r["Xq"], r["qs"], ref, per_token)
    # the bound leaves few codes undecided (it is a worst case over orders)
    assert n_near <= 1e-3 * M * K, (n_near, n_diff)
    print(f"norm={norm} K={K} per_token={per_token}: {n_near} of {M * K} undecided, {n_diff} differ")


def test_order_free_check_catches_mistakes(orc):
    """Negative controls: a norm with a wrong epsilon, a dropped beta or a
    scale of 128/max fails the order-free check."""
    M, K = 16, 1024
    H, gamma, beta = inputs(M, K, 5, 0)
    Hf = H.float().numpy()
    ref = reference_codes(Hf, 0, gamma, beta, 1e-5)
    wrong = [
        oracle.norm_smooth_quant(H, 0, gamma, None, 1e-5, True),          # beta dropped
        oracle.norm_smooth_quant(H, 0, gamma, beta, 1.0, True),           # epsilon far off
        oracle.norm_smooth_quant(H, 0, gamma * 128 / 127, beta * 128 / 127, 1e-5, True),  # codes of 128/max
    ]
    for r in wrong[:2]:
        with pytest.raises(AssertionError):
            check_codes(r["Xq"], r["qs"], ref)
    r = wrong[2]
    with pytest.raises(AssertionError):
        check_codes(r["Xq"], r["qs"] * 127 / 128, ref)


@pytest.mark.gpu
@pytest.mark.parametrize("norm", [0, 1])
@pytest.mark.parametrize("K", [1024, 7168, 12288])
@pytest.mark.parametrize("per_token", [True, False])
def test_gpu_norm_codes_order_free(norm, K, per_token):
    """The library's fused norm + int8 on the GPU against the fp64 norm, with
    the same order-free bound (warp kernel at K = 1024, bulk-staged kernel at
    7168 and 12288)."""
    import w8a8_post_quantization_sq_b200 as sq

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    M = 300
    H, gamma, beta = inputs(M, K, 2 * K + norm, norm)
    eps = 1e-5 if norm == 0 else 1e-6
    Hf = H.float().numpy()
    static = None
    if not per_token:
        v = oracle.norm_f64(Hf, norm, gamma, beta, eps)
        static = float(np.float32(127.0 / np.abs(v).max() * 1.3))
    Xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    qs = torch.empty(M if per_token else 1, device="cuda")
    sq.sq_norm_smooth_quant(H.cuda(), sq.SQ_LAYERNORM if norm == 0 else sq.SQ_RMSNORM, torch.from_numpy(gamma).cuda(),
                            None if beta is None else torch.from_numpy(beta).cuda(), eps, per_token,
                            None if static is None else torch.tensor([static], device="cuda"), Xq, qs)
    torch.cuda.synchronize()
    ref = reference_codes(Hf, norm, gamma, beta, eps, per_token, static)
    n_near, n_diff = check_codes(Xq.cpu().numpy(), qs.cpu().numpy(), ref, per_token)
    assert n_near <= 1e-3 * M * K, (n_near, n_diff)
