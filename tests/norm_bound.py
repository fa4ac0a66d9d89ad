"""An order-free check of the fused norm + int8 codes.

The fp32 norm ("大语言模型量化技术（四）：SmoothQuant", 融入 LayerNorm) sums K
values per row; the pages fix no summation order, and the library and the
oracle share one. This module checks int8 codes and scales against the fp64
norm instead, with an error bound that holds for ANY evaluation whose row sums
are summation trees of depth at most n (n = K/256 + 8 covers a fold of K/256
values per lane followed by a 32-lane butterfly and an 8-way tree) and whose
other steps are single correctly rounded fp32 operations:

  sum of K terms, depth n     |err| <= g(n) * sum|terms|,  g(n) = n u / (1 - n u)
  every other step            one rounding, relative error <= u = 2^-24

Propagated through mu, d = x - mu, the variance, r = 1/sqrt(var + eps),
v = (d r) gamma + beta (LayerNorm) or v = (x r) gamma (RMSNorm), the row's
scale qs = 127 / max|v| and t = v qs, this gives per element a bound B on
|t_fp32 - t_fp64| (doubled to cover the second-order terms). A code is
decided by t_fp64 alone when no tie point k + 1/2 lies within B of it; there
the fp32 code must equal round-half-even(t_fp64) exactly. Elsewhere either
neighbour is accepted, and those elements are counted.
"""
import numpy as np

U = 2.0 ** -24


def _g(n):
    return n * U / (1 - n * U)


def depth(K):
    return -(-K // 256) + 8


def reference_codes(H, norm, gamma, beta, eps, per_token=True, static_qs=None):
    """fp64 norm, its scales, t = v qs, the rounded codes and the bound B of
    |t_fp32 - t_fp64| for every element. norm: 0 LayerNorm, 1 RMSNorm."""
    x = np.asarray(H, np.float64)
    M, K = x.shape
    g = np.asarray(gamma, np.float64)[None, :]
    b = np.zeros_like(g) if beta is None else np.asarray(beta, np.float64)[None, :]
    n = depth(K)
    if norm == 0:
        s1 = x.sum(axis=1, keepdims=True)
        mu = s1 / K
        e_mu = _g(n) * np.abs(x).sum(axis=1, keepdims=True) / K + 2 * U * np.abs(mu)
        d = x - mu
        e_d = e_mu * (1 + U) + U * (np.abs(d) + e_mu)
        s2 = (d * d).sum(axis=1, keepdims=True)
        e_s2 = _g(n) * ((np.abs(d) + e_d) ** 2).sum(axis=1, keepdims=True) + (2 * np.abs(d) * e_d + e_d ** 2).sum(
            axis=1, keepdims=True)
        base, e_base = d, e_d
    else:
        s2 = (x * x).sum(axis=1, keepdims=True)
        e_s2 = _g(n) * s2
        base, e_base = x, np.zeros_like(x)
    var = s2 / K
    w = var + eps
    rel_w = (e_s2 / K) / w + 3 * U  # the division by K and the add
    r = 1.0 / np.sqrt(w)
    rel_r = 0.5 * rel_w + 2 * U  # sqrt and reciprocal
    y = base * r
    z = y * g
    v = z + b
    e_v = (e_base * r + np.abs(base) * r * rel_r) * np.abs(g) + 3 * U * (np.abs(z) + np.abs(b)) + U * np.abs(v)
    e_v = 2 * e_v
    if per_token:
        m = np.abs(v).max(axis=1, keepdims=True)
        m_safe = np.maximum(m, 1e-8)
        qs = 127.0 / m_safe
        rel_qs = np.where(m > 1e-8, e_v.max(axis=1, keepdims=True) / m_safe, 0.0) + U
    else:
        qs = np.full((M, 1), float(static_qs))
        rel_qs = np.zeros((M, 1))
    t = v * qs
    B = 2 * (e_v * qs + np.abs(t) * rel_qs) + U * np.abs(t)
    tc = np.clip(t, -127, 127)
    codes = np.rint(tc)  # numpy rounds half to even
    return {"t": t, "B": B, "codes": codes.astype(np.int64), "qs": qs[:, 0], "rel_qs": rel_qs[:, 0]}


def check_codes(Xq, qs, ref, per_token=True):
    """Exact agreement of the codes wherever no tie point lies within the
    bound, a neighbouring code elsewhere, the scales within their bound;
    returns (undecided elements, how many of them differ)."""
    t, B = ref["t"], ref["B"]
    frac = np.abs(t - np.floor(t) - 0.5)  # distance to the nearest tie k + 1/2
    near = (frac <= B) & (np.abs(t) < 127.5)
    got = np.asarray(Xq, np.int64)
    exact = ~near
    bad = np.argwhere(exact & (got != ref["codes"]))
    assert bad.size == 0, f"{bad.shape[0]} decided codes differ, first {bad[:5].tolist()}"
    alt = np.abs(got - ref["codes"])
    assert np.all(alt[near] <= 1), "an undecided code is not a neighbour of the fp64 rounding"
    if per_token:
        q = np.asarray(qs, np.float64)
        assert np.all(np.abs(q - ref["qs"]) <= ref["qs"] * ref["rel_qs"] * 2 + 1e-30), "row scales beyond the bound"
    return int(near.sum()), int((near & (got != ref["codes"])).sum())
