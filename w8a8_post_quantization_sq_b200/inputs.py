"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random numbers and arranges them into tensors. It holds
none of the method's arithmetic (no absmax, no scales, no quantisation), so
both the GPU path and the CPU oracle can take their inputs from it.

Shapes and value structure follow the workloads the pages describe:

* ``c1_single_linear``: the toy of "如何通过 SmoothQuant 解决激活值离群点难题" §3
  (nn.Linear(1024, 1024), input randn(1, 16, 1024) with channel 0 x50).
* ``c2_qwen3_06b``: Qwen3-0.6B projection shapes from "大语言模型量化技术（四）：
  SmoothQuant" (hidden 1024; q 2048, k/v 1024, o 2048->1024, gate/up 3072,
  down 3072->1024; weight std about 0.03; a few activation channels with
  magnitudes in the hundreds).
* ``c3_opt30b``: OPT-30B decoder linear shapes (hidden 7168) at 4 x 256 tokens,
  LayerNorm input with 0.1% outlier channels.
* ``c4_llmint8``: 6.7B shapes of "8位量化：异常值与混合精度分解实战" §2.2 (6
  outlier dimensions with |x| above 6 on a quarter of the tokens).
* ``c5_175b``: 175B-class shapes (hidden 12288) at 4096 tokens.

Every generator takes a device; the same seed gives the same tensor on the
same device type. Large weights are drawn on the GPU when one is given.
"""
from __future__ import annotations

import math

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn(shape, seed, device="cpu", std=1.0, dtype=torch.float32, gen=None):
    g = gen if gen is not None else _gen(seed, device)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def synthetic_int8(M, K, seed, device="cpu"):
    """Bell-shaped int8 codes in [-127, 127] plus positive per-row scales.

    Stand-in for a quantised activation whose producer (attention, SiLU) is
    outside the linear-layer path."""
    g = _gen(seed, device)
    t = torch.randn((M, K), generator=g, device=device) * 32.0
    q = t.round().clamp_(-127, 127).to(torch.int8)
    sc = torch.rand((M,), generator=g, device=device) * 50.0 + 25.0
    return q, sc


def c1_single_linear(device="cpu"):
    """X fp16 [16,1024] ~N(0,1) with channel 0 x50; W fp16 [1024 out,1024 in]
    ~N(0, 0.02); both from one generator seeded 0 (X drawn first)."""
    g = _gen(0, device)
    X = torch.randn((1, 16, 1024), generator=g, device=device)
    X[:, :, 0] *= 50.0
    W = torch.randn((1024, 1024), generator=g, device=device) * 0.02
    return {"X": X.reshape(16, 1024).to(torch.float16), "W": W.to(torch.float16), "alpha": 0.5}


def outlier_channels(K, n, seed, device="cpu"):
    g = _gen(seed, "cpu")
    return torch.randperm(K, generator=g)[:n].sort().values.to(device)


def c2_qwen3_06b(device="cpu", M=2048):
    K = 1024
    ch = outlier_channels(K, 6, 1234)
    mags = torch.tensor([20.0, 36.0, 52.0, 68.0, 84.0, 100.0], device=device)

    def act(seed):
        h = randn((M, K), seed, device)
        h[:, ch] *= mags
        return h.to(torch.bfloat16)

    g = _gen(7, device)
    gamma_attn = (1.0 + 0.1 * torch.randn((K,), generator=g, device=device))
    gamma_mlp = (1.0 + 0.1 * torch.randn((K,), generator=g, device=device))
    w = {}
    for i, (name, shape) in enumerate([("qkv", (4096, 1024)), ("o", (1024, 2048)),
                                       ("gateup", (6144, 1024)), ("down", (1024, 3072))]):
        w[name] = randn(shape, 100 + i, device, std=0.03, dtype=torch.bfloat16)
    xo, so = synthetic_int8(M, 2048, 200, device)
    xd, sd = synthetic_int8(M, 3072, 201, device)
    return {
        "h_attn": act(0), "h_mlp": act(2), "h_calib": act(1),
        "gamma_attn": gamma_attn, "gamma_mlp": gamma_mlp, "eps": 1e-6,
        "W": w, "o_in": (xo, so), "down_in": (xd, sd), "alpha": 0.5,
        "outlier_channels": ch,
    }


def _weights(spec, device, std, dtype, w_frac):
    """Weights [N, K] ~N(0, std) per name; with w_frac < 1 only the first
    ceil(N * w_frac) output rows are drawn (a sample of the output channels)."""
    w = {}
    for name, (N, K, seed) in spec.items():
        n = N if w_frac >= 1 else max(1, math.ceil(N * w_frac))
        w[name] = randn((n, K), seed, device, std=std, dtype=dtype)
    return w


def c2_block(device="cpu", M=2048, w_frac=1.0):
    """The Qwen3-0.6B-shaped layer of ``c2_qwen3_06b`` in the block layout the
    linear-stack benchmark uses: the attention and MLP sides' pre-norm inputs,
    one calibration batch, per-side gamma (RMSNorm, no beta), the four weights
    and the synthetic int8 inputs of o_proj and down_proj."""
    d = c2_qwen3_06b(device=device, M=M)
    W = d["W"]
    if w_frac < 1:
        W = {k: v[: max(1, math.ceil(v.shape[0] * w_frac))].contiguous() for k, v in W.items()}
    return {
        "h": {"attn": d["h_attn"], "mlp": d["h_mlp"]}, "calib": [d["h_calib"]],
        "gamma": {"attn": d["gamma_attn"], "mlp": d["gamma_mlp"]}, "beta": {"attn": None, "mlp": None},
        "eps": d["eps"], "W": W, "syn": {"o": d["o_in"], "down": d["down_in"]},
        "outlier_channels": d["outlier_channels"],
    }


def _stacked(act, seeds, M, K, dtype, device):
    """Calibration batches drawn one by one into one contiguous [n, M, K]
    buffer: the list of batches (views) and the same tokens as one [n M, K]
    matrix, for a single pass over all of them."""
    buf = torch.empty((len(seeds), M, K), dtype=dtype, device=device)
    for i, s in enumerate(seeds):
        buf[i].copy_(act(s))
    return [buf[i] for i in range(len(seeds))], buf.view(len(seeds) * M, K)


def c3_opt30b(device="cpu", M=1024, n_calib=8, w_frac=1.0):
    """OPT-30B decoder linear stack at 4 x 256 tokens: fp16 pre-norm inputs of
    the attention and MLP sides (7 channels, 0.1% of 7168, x60), 8 calibration
    batches of the same kind, one LayerNorm gamma/beta, fp16 weights
    ~N(0, 0.02) and per-tensor synthetic int8 inputs of out and FC2."""
    K = 7168
    ch = outlier_channels(K, 7, 4321)

    def act(seed):
        h = randn((M, K), seed, device)
        h[:, ch] *= 60.0
        return h.to(torch.float16)

    g = _gen(9, device)
    gamma = 1.0 + 0.1 * torch.randn((K,), generator=g, device=device)
    beta = 0.1 * torch.randn((K,), generator=g, device=device)
    w = _weights({"qkv": (21504, K, 300), "out": (K, K, 301), "fc1": (28672, K, 302), "fc2": (K, 28672, 303)},
                 device, 0.02, torch.float16, w_frac)
    xo, so = synthetic_int8(M, K, 400, device)
    xf, sf = synthetic_int8(M, 28672, 401, device)
    calib, calib_all = _stacked(act, range(1, n_calib + 1), M, K, torch.float16, device)
    return {
        "h": {"attn": act(0), "mlp": act(9)}, "calib": calib, "calib_all": calib_all,
        "gamma": {"attn": gamma, "mlp": gamma}, "beta": {"attn": beta, "mlp": beta}, "eps": 1e-5, "W": w,
        "syn": {"out": (xo, so[:1].contiguous()), "fc2": (xf, sf[:1].contiguous())},
        "outlier_channels": ch,
    }


def c4_llmint8(device="cpu", M=2048, K=4096, N=16384, n_out=6, seed=0):
    """X fp16 [M,K]: N(0,1) with every |x| >= 6 redrawn (so no ordinary entry
    exceeds 6.0 after fp16 rounding); n_out dimensions where M/4 tokens get
    sign * U(6.0625, 40]. W fp16 [N out, K in] ~N(0, 0.02)."""
    g = _gen(seed, "cpu")
    X = torch.randn((M, K), generator=g)
    bad = X.abs() >= 6.0
    while bool(bad.any()):
        X[bad] = torch.randn((int(bad.sum()),), generator=g)
        bad = X.abs() >= 6.0
    dims = torch.randperm(K, generator=g)[:n_out].sort().values
    for d in dims.tolist():
        rows = torch.randperm(M, generator=g)[: M // 4]
        mag = 40.0 - torch.rand((rows.numel(),), generator=g) * (40.0 - 6.0625)
        sign = torch.where(torch.rand((rows.numel(),), generator=g) < 0.5, -1.0, 1.0)
        X[rows, d] = sign * mag
    W = randn((N, K), seed + 1, device, std=0.02, dtype=torch.float16)
    return {"X": X.to(torch.float16).to(device), "W": W, "dims": dims, "threshold": 6.0}


def c5_175b(device="cpu", M=4096, n_calib=16, w_frac=1.0):
    """175B-class block, hidden 12288, at M tokens: n_calib calibration batches
    of linear inputs (bf16 [M, 12288] ~N(0,1), 8 channels x100), the attention
    and MLP sides' pre-norm inputs with the same outlier channels, one
    LayerNorm gamma/beta, fp32 weights ~N(0, 0.01) (QKV, out, FC1, FC2) and
    per-token synthetic int8 inputs of out and FC2."""
    K = 12288
    ch = outlier_channels(K, 8, 5555)

    def act(seed):
        h = randn((M, K), seed, device)
        h[:, ch] *= 100.0
        return h.to(torch.bfloat16)

    g = _gen(11, device)
    gamma = 1.0 + 0.1 * torch.randn((K,), generator=g, device=device)
    beta = 0.1 * torch.randn((K,), generator=g, device=device)
    w = _weights({"qkv": (36864, K, 500), "out": (K, K, 501), "fc1": (49152, K, 502), "fc2": (K, 49152, 503)},
                 device, 0.01, torch.float32, w_frac)
    xo, so = synthetic_int8(M, K, 600, device)
    xf, sf = synthetic_int8(M, 49152, 601, device)
    calib, calib_all = _stacked(act, range(100, 100 + n_calib), M, K, torch.bfloat16, device)
    return {
        "h": {"attn": act(200), "mlp": act(201)}, "calib": calib, "calib_all": calib_all,
        "gamma": {"attn": gamma, "mlp": gamma}, "beta": {"attn": beta, "mlp": beta}, "eps": 1e-5, "W": w,
        "syn": {"out": (xo, so), "fc2": (xf, sf)}, "outlier_channels": ch,
    }
