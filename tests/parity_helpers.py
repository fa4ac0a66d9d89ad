"""Comparison helpers shared by the GPU parity tests: host copies of device
tensors and the output tolerances (16-bit outputs within one unit in the last
place of the oracle's fp64 value rounded to the same type, fp32 outputs within
1e-6 of the sum of the magnitudes of the terms)."""
import numpy as np
import torch

import oracle


def npf(t):
    return t.detach().to("cpu", torch.float32).numpy()


def npu16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def ord16(bits):
    b = bits.astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def ulp16(bits, dtype):
    """Spacing of the 16-bit grid at each value (bits of a finite value)."""
    v = torch.from_numpy(bits.view(np.int16)).view(dtype).double().numpy()
    nxt = torch.from_numpy((bits.astype(np.int32) + 1).astype(np.uint16).view(np.int16)).view(dtype).double().numpy()
    return np.abs(nxt - v)


def assert_close_16(got, y, dtype, terms=None):
    """got: torch 16-bit tensor; y: oracle fp64; terms: sum of |terms| (fp64)."""
    gb = npu16(got)
    rb = oracle.round_bf16_bits(y) if dtype == torch.bfloat16 else oracle.round_fp16_bits(y)
    d = np.abs(ord16(gb) - ord16(rb))
    ok = d <= 1
    if terms is not None:
        g = npf(got).astype(np.float64)
        ok |= np.abs(g - y) <= ulp16(rb, dtype) + 2.0 ** -20 * terms
    bad = np.argwhere(~ok)
    assert bad.size == 0, f"{bad.shape[0]} outputs beyond tolerance, first {bad[:5].tolist()} d={d[~ok][:5]}"


def assert_close_f32(got, y, terms):
    g = npf(got).astype(np.float64)
    err = np.abs(g - y)
    bad = err > 1e-6 * terms
    assert not bad.any(), f"max rel {np.max(err / np.maximum(terms, 1e-300))}"
