"""Benchmark of the SmoothQuant W8A8 linear-layer path on B200.

The headline workload is the 175B-shaped block (hidden 12288, 4096 tokens) in
deploy mode: the weights are smoothed and quantised once, offline, and one
step is the block's online linear stack

  LayerNorm (gamma', beta' folded) + per-token int8 of the attention side
  QKV GEMM 12288 -> 36864, int8 x int8 -> int32, dequantised to bf16
  out GEMM 12288 -> 12288 on a per-token int8 input (attention is not on the path)
  LayerNorm + per-token int8 of the MLP side
  FC1 GEMM 12288 -> 49152
  FC2 GEMM 49152 -> 12288 on a per-token int8 input (the activation is not on the path)

tokens/s = tokens / step time. The offline work is timed on its own and
reported beside the step, not inside it: the calibration pass (running
per-channel absmax over 16 calibration batches of [4096, 12288] bf16), the
weight maxima, the smoothing factors for alpha in {0.4, 0.5, 0.6} (gamma and
beta folded for alpha = 0.5) and the per-channel int8 weights.

Every timed step is one CUDA graph replay after an L2 flush (a 256 MB write,
then a 256 MB read of another buffer, outside the timed interval), bracketed
by CUDA events on the stream it runs on. Per-kernel durations come from a
second capture of the same step with events around every launch, replayed
after the timed region. The Qwen3-0.6B-, OPT-30B- and LLM.int8-shaped
configurations are timed the same way and reported under "configs".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --kernel gemm --shape M,N,K     (one entry point alone)

Prints one JSON line (rank 0). Under torchrun (N > 1) every rank runs its own
replica of the step on its own GPU (no data-path collective; weak scaling).
"""
from __future__ import annotations

import argparse
import contextlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W8A8 GEMM TOPS & tokens/s at 1 B200; % of INT8 TC peak / HBM GB/s"
NOMINAL_INT8_TOPS = 4500.0  # B200 dense int8 (spec sheet), for context beside the measured-derived peak

# Deploy-mode linear stacks. gemms: (weight, source) in launch order; source is
# the norm side whose int8 output the GEMM reads, or "syn" for a synthetic
# int8 input whose producer (attention, the MLP activation) is off the path.
CONFIGS = {
    "c5": {
        "workload": "175B-shaped W8A8 block, hidden 12288, 4096 tokens, deploy mode: LayerNorm + smoothing + "
                    "per-token int8 of the attention and MLP inputs, QKV/out/FC1/FC2 int8 GEMMs to bf16 "
                    "(weights smoothed and quantised offline)",
        "gen": "c5_175b", "tokens": 4096, "hidden": 12288, "norm": "layer", "per_token": True,
        "calib": "absmax", "alphas": (0.4, 0.5, 0.6), "alpha": 0.5, "out": "bf16",
        "gemms": (("qkv", "attn"), ("out", "syn"), ("fc1", "mlp"), ("fc2", "syn")),
    },
    "c3": {
        "workload": "OPT-30B-shaped decoder linear stack, 4 x 256 tokens, hidden 7168, deploy mode: LayerNorm + "
                    "smoothing + static per-tensor int8 (scales from 8 calibration batches), QKV/out/FC1/FC2 int8 "
                    "GEMMs to fp16",
        "gen": "c3_opt30b", "tokens": 1024, "hidden": 7168, "norm": "layer", "per_token": False,
        "calib": "norm", "alphas": (0.5,), "alpha": 0.5, "out": "fp16",
        "gemms": (("qkv", "attn"), ("out", "syn"), ("fc1", "mlp"), ("fc2", "syn")),
    },
    "c2": {
        "workload": "Qwen3-0.6B-shaped decoder layer linear stack, 2048 tokens, hidden 1024, deploy mode: RMSNorm + "
                    "smoothing + per-token int8, q/k/v, o, gate/up, down int8 GEMMs to bf16",
        "gen": "c2_block", "tokens": 2048, "hidden": 1024, "norm": "rms", "per_token": True,
        "calib": "norm", "alphas": (0.5,), "alpha": 0.5, "out": "bf16",
        "gemms": (("qkv", "attn"), ("o", "syn"), ("gateup", "mlp"), ("down", "syn")),
    },
}
C4 = {"workload": "LLM.int8() decomposition at 6.7B shapes: X fp16 [2048, 4096] with 6 outlier dims, W fp16 "
                  "[16384, 4096], threshold 6.0, fp16 out (weight cache warm: the outlier set is unchanged)",
      "tokens": 2048, "M": 2048, "K": 4096, "N": 16384}
HEADLINE = "c5"
L2_NOTE = ("L2 flushed before every timed step (256 MB write + 256 MB read, outside the timed interval); "
           "the step's operands (1.8 GB of int8 weights) are far larger than L2 as well")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def int8_peaks():
    """Dense int8 peaks in TOPS: the measured bf16 GEMM (burst, sustained) x 2,
    the nominal int8:bf16 ratio (4.5 vs 2.25 PFLOP/s), and the spec-sheet
    nominal 4.5 POPS."""
    pk, src = peaks()
    return {"burst": 2.0 * pk["bf16_tflops"], "sustained": 2.0 * pk.get("bf16_tflops_sustained", pk["bf16_tflops"]),
            "nominal": NOMINAL_INT8_TOPS, "source": src}


# ------------------------------------------------------------------ ranks
def max_over_ranks(x, dev):
    """The maximum of a per-rank number over all ranks (timing: the slowest
    rank's clock decides); x itself with one rank."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ DRAM traffic
GEMM_SOURCES = ["w8a8_post_quantization_sq_b200/csrc/gemm_w8a8.cu", "w8a8_post_quantization_sq_b200/csrc/sq_common.cuh",
                "w8a8_post_quantization_sq_b200/csrc/sq_wait.cuh", "w8a8_post_quantization_sq_b200/csrc/sq_internal.h"]


def gemm_sources_digest():
    import hashlib

    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def gemm_traffic(shapes):
    """DRAM bytes (read + write) of one launch of each GEMM shape (M, N, K),
    from the ncu counters recorded in profiles/gemm_traffic.json; None when a
    shape is missing or the kernel's sources differ from those the counters
    were taken on."""
    p = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("sources_sha256") != gemm_sources_digest():
        return None
    per = d.get("bytes_per_launch")
    if not isinstance(per, dict):
        return None
    keys = ["x".join(str(v) for v in s) for s in shapes]
    if not all(k in per for k in keys):
        return None
    return [float(per[k]) for k in keys]


# ------------------------------------------------------------------ clocks
class ClockSampler:
    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.proc = None
        self.index = index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(index), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        return parse_clocks(out)


def parse_clocks(out):
    rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
    if not rows:
        return None
    num = lambda x: x.strip().replace(".", "", 1).isdigit()  # noqa: E731
    sm = [float(r[1]) for r in rows if num(r[1])]
    mx = [float(r[2]) for r in rows if num(r[2])]
    pw = [float(r[3]) for r in rows if num(r[3])]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i] and "Not" not in r[5 + i]})
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
            "sm_mhz_min": min(sm) if sm else None, "power_w_max": max(pw) if pw else None,
            "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ GPU helpers
class L2Flush:
    """Evicts L2 before a timed interval: a 256 MB write, then a 256 MB read of
    another buffer, so the dirty lines of the write are written back before the
    interval starts rather than inside it."""

    def __init__(self, dev):
        import torch

        self.w = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        self.r = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)
        self.out = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self, i=1):
        import torch

        self.w.fill_(i & 0xFF)
        torch.sum(self.r, dim=0, out=self.out)


class EventBank:
    """CUDA event pairs around launches captured in a graph (external events,
    so every replay records them), each tagged with its kernel and its
    algorithmic work."""

    def __init__(self):
        self.pairs = []

    def pair(self, tag, work):
        import torch

        e = (torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
        self.pairs.append((tag, work, e))
        return e

    def read(self):
        return [a.elapsed_time(b) for _, _, (a, b) in self.pairs]


def esize(t):
    return t.element_size()


# ------------------------------------------------------------------ the deploy-mode stacks
class Stack:
    """Device buffers, offline pass and online step of one deploy-mode linear
    stack (CONFIGS). `offline()` calibrates, smooths and quantises the weights;
    `step()` is the online linear stack. Every launch goes through `launch`,
    which brackets it with events when an EventBank is attached."""

    def __init__(self, name, dev, M=None, n_calib=None):
        import torch

        import w8a8_post_quantization_sq_b200 as sq
        from w8a8_post_quantization_sq_b200 import inputs

        cfg = CONFIGS[name]
        self.name, self.cfg, self.sq, self.torch, self.dev = name, cfg, sq, torch, dev
        self.M = M = M or cfg["tokens"]
        kw = {} if n_calib is None else {"n_calib": n_calib}
        d = getattr(inputs, cfg["gen"])(device=dev, M=M, **kw)
        self.d = d
        K = cfg["hidden"]
        self.K = K
        self.norm = sq.SQ_LAYERNORM if cfg["norm"] == "layer" else sq.SQ_RMSNORM
        self.per_token = cfg["per_token"]
        self.alpha, self.alphas = cfg["alpha"], cfg["alphas"]
        self.out_dtype = torch.bfloat16 if cfg["out"] == "bf16" else torch.float16
        f32 = lambda *s: torch.empty(s, dtype=torch.float32, device=dev)  # noqa: E731
        self.sides = ("attn", "mlp")
        self.consumer = {src: w for w, src in cfg["gemms"] if src != "syn"}
        self.gamma = {k: d["gamma"][k].float().contiguous() for k in self.sides}
        self.beta = {k: None if d["beta"][k] is None else d["beta"][k].float().contiguous() for k in self.sides}
        self.h, self.syn, self.W = dict(d["h"]), dict(d["syn"]), d["W"]
        # running maxima (cleared by one fill per offline pass): the linear
        # inputs' per channel (one vector for both sides when the calibration
        # batches are the linear inputs themselves), the consumers' weights,
        # and the smoothed norm outputs (static per-tensor scales)
        self.cal = torch.zeros((6, K), dtype=torch.float32, device=dev)
        shared = cfg["calib"] == "absmax"
        self.xmax = {"attn": self.cal[0], "mlp": self.cal[0] if shared else self.cal[1]}
        self.wmax = {"attn": self.cal[2], "mlp": self.cal[3]}
        self.vmax = {"attn": self.cal[4], "mlp": self.cal[5]}
        self.s = {a: {k: f32(K) for k in self.sides} for a in self.alphas}
        self.gp = {k: f32(K) for k in self.sides}
        self.bp = {k: None if self.beta[k] is None else f32(K) for k in self.sides}
        self.qs_static = {k: f32(1) for k in self.sides}
        self.Wq = {w: torch.empty(self.W[w].shape, dtype=torch.int8, device=dev) for w, _ in cfg["gemms"]}
        self.qw = {w: f32(self.W[w].shape[0]) for w, _ in cfg["gemms"]}
        self.Xq = {k: torch.empty((M, K), dtype=torch.int8, device=dev) for k in self.sides}
        self.qx = {k: f32(M if self.per_token else 1) for k in self.sides}
        self.Y = {w: torch.empty((M, self.W[w].shape[0]), dtype=self.out_dtype, device=dev) for w, _ in cfg["gemms"]}
        self.ws = {w: sq.workspace(sq.SQ_OP_GEMM, M, self.W[w].shape[0], self.W[w].shape[1], device=dev)
                   for w, _ in cfg["gemms"]}
        self.bank = None
        self.by_phase = False  # with a bank: events around each phase of the offline pass, not each launch

    # one launch, bracketed by events when a bank is attached (per launch)
    def launch(self, tag, work, fn, *a):
        if self.bank is None or self.by_phase:
            fn(*a)
            return
        e0, e1 = self.bank.pair(tag, work)
        e0.record()
        fn(*a)
        e1.record()

    @contextlib.contextmanager
    def phase(self, tag, work):
        """A group of launches timed as one (events before the first and after
        the last) when a bank is attached in phase mode."""
        if self.bank is None or not self.by_phase:
            yield
            return
        e0, e1 = self.bank.pair(tag, work)
        e0.record()
        yield
        e1.record()

    def gemm_shapes(self):
        return [(self.M, self.W[w].shape[0], self.W[w].shape[1]) for w, _ in self.cfg["gemms"]]

    def offline(self):
        """Calibration, weight maxima, smoothing factors for every alpha (gamma
        and beta folded for the deployed one), static per-tensor scales where
        the configuration uses them, and the int8 weights."""
        sq, d = self.sq, self.d
        L = self.launch
        eps = d["eps"]
        self.cal.zero_()
        cb = sum(X.numel() * esize(X) for X in d["calib"])
        # the batches sit back to back in HBM: one pass over all their tokens
        # (the running maxima are the same as batch by batch)
        batches = [d["calib_all"]] if "calib_all" in d else d["calib"]
        if self.cfg["calib"] == "absmax":
            with self.phase("calib_absmax", ("hbm", cb)):
                for X in batches:
                    L("calib_absmax", ("hbm", X.numel() * esize(X)), sq.sq_calib_absmax, X, self.xmax["attn"])
        else:
            with self.phase("calib_norm", ("hbm", cb * 2)):
                for X in batches:
                    for k in self.sides:
                        L("calib_norm", ("hbm", X.numel() * esize(X)), sq.sq_norm_smooth_quant, X, self.norm,
                          self.gamma[k], self.beta[k], eps, True, None, None, None, self.xmax[k])
        with self.phase("weight_absmax", ("hbm", sum(self.W[self.consumer[k]].numel() *
                                                      esize(self.W[self.consumer[k]]) for k in self.sides))):
            for k in self.sides:
                W = self.W[self.consumer[k]]
                L("weight_absmax", ("hbm", W.numel() * esize(W)), sq.sq_weight_absmax, W, self.wmax[k])
        with self.phase("smoothing", ("latency", 0)):
            for a in self.alphas:
                for k in self.sides:
                    if a == self.alpha:
                        L("smooth_fold_norm", ("latency", 0), sq.sq_smooth_fold_norm, self.xmax[k], self.wmax[k], a,
                          self.gamma[k], self.beta[k], self.s[a][k], self.gp[k], self.bp[k])
                    else:
                        L("smooth_scales", ("latency", 0), sq.sq_smooth_scales, self.xmax[k], self.wmax[k], a,
                          self.s[a][k])
        if not self.per_token:
            with self.phase("static_scales", ("hbm", cb * 2)):
                for X in batches:
                    for k in self.sides:
                        L("calib_norm_smoothed", ("hbm", X.numel() * esize(X)), sq.sq_norm_smooth_quant, X,
                          self.norm, self.gp[k], self.bp[k], eps, True, None, None, None, self.vmax[k])
                for k in self.sides:
                    L("scale_from_absmax", ("latency", 0), sq.sq_scale_from_absmax, self.vmax[k], self.qs_static[k])
        wq = sum(self.W[w].numel() * (esize(self.W[w]) + 1) + 4 * self.W[w].shape[0] for w, _ in self.cfg["gemms"])
        with self.phase("quantize_weight", ("hbm", wq)):
            for w, src in self.cfg["gemms"]:
                W = self.W[w]
                s = None if src == "syn" else self.s[self.alpha][src]
                L("quantize_weight", ("hbm", W.numel() * (esize(W) + 1) + 4 * W.shape[0]), sq.sq_quantize_weight,
                  W, s, True, self.Wq[w], self.qw[w])

    def norm_instances(self, n_sets=4):
        """The norm + smoothing + int8 of this stack alone, on n_sets distinct
        inputs (the step's two and fresh draws of the same kind), for a
        back-to-back bandwidth figure; returns (launches, bytes per launch)."""
        torch, sq = self.torch, self.sq
        g = torch.Generator(device=self.dev).manual_seed(1234)
        hs = [self.h["attn"], self.h["mlp"]]
        while len(hs) < n_sets:
            hs.append((torch.randn(hs[0].shape, generator=g, device=self.dev) * 3).to(hs[0].dtype))
        outs = [(torch.empty(h.shape, dtype=torch.int8, device=self.dev),
                 torch.empty(self.M if self.per_token else 1, device=self.dev)) for h in hs]
        st = None if self.per_token else self.qs_static["attn"]
        eps = self.d["eps"]

        def one(h, o):
            return lambda: sq.sq_norm_smooth_quant(h, self.norm, self.gp["attn"], self.bp["attn"], eps,
                                                   self.per_token, st, o[0], o[1])
        nbytes = self.M * self.K * esize(hs[0]) + self.M * self.K + 4 * outs[0][1].numel()
        return [one(h, o) for h, o in zip(hs, outs)], nbytes

    def step(self):
        """The online linear stack: per side, norm + smoothing + int8 then the
        GEMM that reads it; the synthetic-input GEMMs in block order."""
        sq, M, K = self.sq, self.M, self.K
        L = self.launch
        eps = self.d["eps"]
        ob = esize(self.Y[self.cfg["gemms"][0][0]])
        for w, src in self.cfg["gemms"]:
            if src == "syn":
                xq, qx = self.syn[w]
            else:
                h = self.h[src]
                st = None if self.per_token else self.qs_static[src]
                L("norm_quant", ("hbm", M * K * esize(h) + M * K + 4 * self.qx[src].numel()), sq.sq_norm_smooth_quant,
                  h, self.norm, self.gp[src], self.bp[src], eps, self.per_token, st, self.Xq[src], self.qx[src])
                xq, qx = self.Xq[src], self.qx[src]
            N, Kw = self.W[w].shape
            L("gemm_w8a8", ("tensor", 2.0 * M * N * Kw, M * Kw + N * Kw + M * N * ob), sq.sq_gemm_w8a8, xq,
              self.Wq[w], qx, self.qw[w], None, self.Y[w], self.ws[w])

    def launches_per_step(self):
        return sum(2 if src != "syn" else 1 for _, src in self.cfg["gemms"])

    # per-step inputs and outputs (the e2e leg copies them to and from the host)
    def io(self):
        ins = [self.h[k] for k in self.sides] + [t for w in self.syn for t in self.syn[w]]
        outs = [self.Y[w] for w, _ in self.cfg["gemms"]]
        return ins, outs

    def swap_io(self, other=None):
        """Point the step at another set of input/output buffers (fresh ones
        when other is None); returns the previous set."""
        torch = self.torch
        old = (self.h, self.syn, self.Y)
        if other is None:
            other = ({k: torch.empty_like(v).copy_(v) for k, v in self.h.items()},
                     {k: tuple(torch.empty_like(t).copy_(t) for t in v) for k, v in self.syn.items()},
                     {k: torch.empty_like(v) for k, v in self.Y.items()})
        self.h, self.syn, self.Y = other
        return old


class LlmInt8Stack:
    """The LLM.int8() call at 6.7B shapes: offline = the weight's int8 copy for
    the outlier set; step = one sq_llmint8_matmul (detection, row
    quantisation, the int8 GEMM with the fused 16-bit outlier term) with the
    weight cache warm."""

    def __init__(self, dev):
        import torch

        import w8a8_post_quantization_sq_b200 as sq
        from w8a8_post_quantization_sq_b200 import inputs

        self.sq, self.torch, self.dev = sq, torch, dev
        M, K, N = C4["M"], C4["K"], C4["N"]
        self.M, self.K, self.N = M, K, N
        self.d = inputs.c4_llmint8(device=dev, M=M, K=K, N=N)
        self.st = sq.llmint8_weight_state(self.d["W"])
        self.Y = torch.empty((M, N), dtype=torch.float16, device=dev)
        self.idx = torch.empty(K, dtype=torch.int32, device=dev)
        self.n = torch.empty(1, dtype=torch.int32, device=dev)
        self.ws = sq.workspace(sq.SQ_OP_LLMINT8, M, N, K, device=dev)
        self.ws_det = sq.workspace(sq.SQ_OP_LLMINT8_DETECT, M, N, K, device=dev)
        self.bank = None
        self.by_phase = False

    launch = Stack.launch

    def gemm_shapes(self):
        return [(self.M, self.N, self.K)]

    def offline(self):
        sq, X, W = self.sq, self.d["X"], self.d["W"]
        self.launch("llmint8_detect", ("hbm", X.numel() * 2), sq.sq_llmint8_detect, X, 6.0, 0.0, self.idx, self.n,
                    self.ws_det)
        self.launch("llmint8_quant_weight", ("hbm", W.numel() * 3 + 4 * self.N), sq.sq_llmint8_quant_weight, W,
                    self.idx, self.n, self.st["Wq"], self.st["qs_w"])

    def step(self):
        M, N, K = self.M, self.N, self.K
        self.launch("llmint8_matmul", ("tensor", 2.0 * M * N * K, M * K * 2 + N * K + M * N * 2),
                    self.sq.sq_llmint8_matmul, self.d["X"], self.st, 6.0, 0.0, self.Y, self.idx, self.n, self.ws)

    def launches_per_step(self):
        return 5  # counts, compaction, weight-side pass, row quantisation, GEMM


class Fp8Stack:
    """The 175B-shaped block's linear stack on FP8 units (E4M3 codes,
    per-token and per-channel scales, fp32 tensor-core accumulation): the
    smoothed per-token FP8 quantisation of both sides' [4096, 12288] bf16
    linear inputs and the four GEMMs (out and FC2 on synthetic E4M3 inputs).
    Offline: the int8 stack's calibration and smoothing factors, then the FP8
    weights."""

    def __init__(self, dev):
        import torch

        import w8a8_post_quantization_sq_b200 as sq

        self.sq, self.torch, self.dev = sq, torch, dev
        base = Stack("c5", dev)
        with torch.cuda.stream(torch.cuda.Stream(device=dev)):
            base.offline()
        torch.cuda.synchronize()
        self.base = base
        self.M, self.K = base.M, base.K
        self.s = {k: base.s[base.alpha][k] for k in base.sides}
        self.W = base.W
        self.gemms = base.cfg["gemms"]
        u8 = lambda *sh: torch.empty(sh, dtype=torch.uint8, device=dev)  # noqa: E731
        self.Wq = {w: u8(*self.W[w].shape) for w, _ in self.gemms}
        self.qw = {w: torch.empty(self.W[w].shape[0], device=dev) for w, _ in self.gemms}
        self.Xq = {k: u8(self.M, self.K) for k in base.sides}
        self.qx = {k: torch.empty(self.M, device=dev) for k in base.sides}
        g = torch.Generator(device=dev).manual_seed(77)
        self.syn = {}
        for w, src in self.gemms:
            if src == "syn":
                c = torch.randint(0, 256, (self.M, self.W[w].shape[1]), generator=g, device=dev, dtype=torch.int32)
                c = torch.where((c & 0x7F) == 0x7F, c - 1, c).to(torch.uint8)  # no NaN codes
                self.syn[w] = (c, torch.rand(self.M, generator=g, device=dev) + 1.0)
        self.Y = base.Y
        self.ws = base.ws
        self.d = {}
        self.bank = None
        self.by_phase = False

    launch = Stack.launch

    def gemm_shapes(self):
        return self.base.gemm_shapes()

    def offline(self):
        for w, src in self.gemms:
            W = self.W[w]
            s = None if src == "syn" else self.s[src]
            self.launch("quantize_weight_fp8", ("hbm", W.numel() * (esize(W) + 1) + 4 * W.shape[0]),
                        self.sq.sq_quantize_weight_fp8, W, s, True, self.Wq[w], self.qw[w])

    def step(self):
        sq, M, K = self.sq, self.M, self.K
        for w, src in self.gemms:
            if src == "syn":
                xq, qx = self.syn[w]
            else:
                h = self.base.h[src]
                self.launch("quantize_act_fp8", ("hbm", M * K * esize(h) + M * K + 4 * M), sq.sq_quantize_act_fp8, h,
                            self.s[src], True, None, self.Xq[src], self.qx[src])
                xq, qx = self.Xq[src], self.qx[src]
            N, Kw = self.W[w].shape
            ob = esize(self.Y[w])
            self.launch("gemm_fp8", ("tensor", 2.0 * M * N * Kw, M * Kw + N * Kw + M * N * ob), sq.sq_gemm_fp8, xq,
                        self.Wq[w], qx, self.qw[w], None, self.Y[w], self.ws[w])

    def launches_per_step(self):
        return 6


class AttnStack:
    """Attention's two products in int8 at the 175B-shaped block's head
    layout (96 heads of 128 channels, 2048 tokens of one sequence): per-(head,
    token) int8 of Q and K, the batched QK^T to bf16, per-(head, channel) int8
    of V^T, and the batched PV on int8 probabilities (the softmax between
    them is not on the path: P stands as synthetic int8 codes with per-row
    scales)."""

    def __init__(self, dev, heads=96, T=2048, d=128):
        import torch

        import w8a8_post_quantization_sq_b200 as sq

        self.sq, self.torch, self.dev = sq, torch, dev
        self.H, self.T, self.dh = heads, T, d
        g = torch.Generator(device=dev).manual_seed(5)
        bf = lambda *sh: torch.randn(sh, generator=g, device=dev).to(torch.bfloat16)  # noqa: E731
        self.Q, self.Kt, self.Vt = bf(heads * T, d), bf(heads * T, d), bf(heads * d, T)
        i8 = lambda *sh: torch.empty(sh, dtype=torch.int8, device=dev)  # noqa: E731
        self.Qq, self.Kq, self.Vq = i8(heads, T, d), i8(heads, T, d), i8(heads, d, T)
        self.qq, self.qk, self.qv = (torch.empty(n, device=dev) for n in (heads * T, heads * T, heads * d))
        t = torch.randn((heads, T, T), generator=g, device=dev) * 40
        self.Pq = t.round().clamp_(-127, 127).to(torch.int8)
        del t
        self.qp = torch.rand(heads * T, generator=g, device=dev) * 100 + 100
        self.S = torch.empty((heads, T, T), dtype=torch.bfloat16, device=dev)
        self.O = torch.empty((heads, T, d), dtype=torch.bfloat16, device=dev)
        self.ws1 = sq.workspace(sq.SQ_OP_GEMM, T, T, d, device=dev)
        self.ws2 = sq.workspace(sq.SQ_OP_GEMM, T, d, T, device=dev)
        self.d = {}
        self.bank = None
        self.by_phase = False

    launch = Stack.launch

    def gemm_shapes(self):
        return [(self.T, self.T, self.dh), (self.T, self.dh, self.T)]

    has_offline = False

    def offline(self):
        pass

    def step(self):
        sq, H, T, dh = self.sq, self.H, self.T, self.dh
        for X, Xq, qs in ((self.Q, self.Qq, self.qq), (self.Kt, self.Kq, self.qk)):
            self.launch("quantize_act", ("hbm", X.numel() * 3 + 4 * X.shape[0]), sq.sq_quantize_act, X, None, True,
                        None, Xq.view(H * T, dh), qs)
        # both products are bound by HBM at this head dimension (2 T^2 d operations
        # against the 2 T^2 bytes of S or the T^2 of P: 128 and 256 operations per
        # byte, under the int8 ridge of ~500): judged by their bytes
        self.launch("bmm_qk", ("hbm", H * (2 * T * dh + 2 * T * T + 8 * T)), sq.sq_bmm_w8a8,
                    self.Qq, self.Kq, self.qq.view(H, T), self.qk.view(H, T), self.S, self.ws1)
        self.launch("quantize_act", ("hbm", self.Vt.numel() * 3 + 4 * self.Vt.shape[0]), sq.sq_quantize_act, self.Vt,
                    None, True, None, self.Vq.view(H * dh, T), self.qv)
        self.launch("bmm_pv", ("hbm", H * (T * T + dh * T + 2 * T * dh + 4 * (T + dh))), sq.sq_bmm_w8a8,
                    self.Pq, self.Vq, self.qp.view(H, T), self.qv.view(H, dh), self.O, self.ws2)

    def launches_per_step(self):
        return 5


def summarise(bank, per_launch_ms, ipk, hbm):
    """Per-kernel figures from an instrumented replay: launches, mean time per
    launch, achieved throughput from the algorithmic work, and the fraction
    of the peak that bounds the kernel (int8 dense for the GEMMs, measured
    copy bandwidth for the memory-bound kernels)."""
    out = {}
    for (tag, work, _), ms in zip(bank.pairs, per_launch_ms):
        r = out.setdefault(tag, {"kernel": tag, "launches": 0, "ms": 0.0, "work": 0.0, "bytes": 0.0, "bound": work[0]})
        r["launches"] += 1
        r["ms"] += ms
        r["work"] += work[1]
        if work[0] == "tensor":
            r["bytes"] += work[2]
    rows = []
    for r in out.values():
        t = r["ms"] * 1e-3
        e = {"kernel": r["kernel"], "launches": r["launches"], "us_per_launch": r["ms"] * 1e3 / r["launches"],
             "us_total": r["ms"] * 1e3, "bound": r["bound"]}
        if r["bound"] == "tensor":
            a = r["work"] / t / 1e12
            e.update({"ops_per_launch": r["work"] / r["launches"], "achieved": a, "unit": "TOPS",
                      "peak": ipk["burst"], "frac": a / ipk["burst"], "frac_sustained": a / ipk["sustained"],
                      "frac_nominal": a / ipk["nominal"], "algorithmic_bytes_per_launch": r["bytes"] / r["launches"]})
        elif r["bound"] == "hbm":
            a = r["work"] / t / 1e9
            e.update({"bytes_per_launch": r["work"] / r["launches"], "achieved": a, "unit": "GB/s", "peak": hbm,
                      "frac": a / hbm})
        rows.append(e)
    return rows


def capture(fn, stream):
    import torch

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def timed_replays(graph, bank, n, flush, stream):
    """Per-launch durations (ms) of an instrumented graph, averaged over n
    replays, each after an L2 flush."""
    import torch

    acc = None
    with torch.cuda.stream(stream):
        for i in range(n):
            flush(i)
            graph.replay()
            stream.synchronize()
            v = np.array(bank.read())
            acc = v if acc is None else acc + v
    return (acc / n).tolist()


def run_stack(st, args, rank, world, dev, flush, e2e=True):
    """Time one stack: the offline pass (instrumented), the online step (plain
    graph, timed; then instrumented, for per-kernel times) and, with e2e, the
    step through the public API with pinned host buffers."""
    import torch
    import torch.distributed as dist

    ipk = int8_peaks()
    hbm = peaks()[0]["hbm_gbs"]
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        st.offline()
        st.step()
    stream.synchronize()
    g_step = capture(st.step, stream)
    st.bank = EventBank()
    g_step_ev = capture(st.step, stream)
    bank_step = st.bank
    st.bank = EventBank()
    st.by_phase = hasattr(st, "phase")  # the offline pass: one interval per phase
    # (a stack with no offline work captures no graph for it: an empty graph)
    g_off_ev = capture(st.offline, stream) if getattr(st, "has_offline", True) else None
    bank_off = st.bank
    st.bank, st.by_phase = None, False
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            g_step.replay()
        if g_off_ev is not None:
            g_off_ev.replay()
        g_step_ev.replay()
    torch.cuda.synchronize()

    # the timed region: K replays of the step, each after an L2 flush
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(dev.index if dev.index is not None else 0) if rank == 0 else None
    time.sleep(0.05)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush(i)
            ev[i][0].record(stream)
            g_step.replay()
            ev[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    step_ms = [a.elapsed_time(b) for a, b in ev]
    ms_per_step = max_over_ranks(sum(step_ms), dev) / args.steps

    n_ev = max(3, min(args.steps, 50))
    k_step = summarise(bank_step, timed_replays(g_step_ev, bank_step, n_ev, flush, stream), ipk, hbm)
    k_off = []
    if g_off_ev is not None:
        k_off = summarise(bank_off, timed_replays(g_off_ev, bank_off, max(3, min(args.steps, 10)), flush, stream),
                          ipk, hbm)
    r = {"ms_per_step": ms_per_step, "step_ms_median": statistics.median(step_ms), "clocks": clk,
         "kernels": k_step, "offline": k_off, "instrumented_replays": n_ev, "ipk": ipk, "hbm": hbm,
         "launches_per_step": st.launches_per_step(),
         "n_calib": len(st.d["calib"]) if isinstance(st.d, dict) and "calib" in st.d else None}
    if hasattr(st, "norm_instances"):
        r["norm_bandwidth"] = time_back_to_back(st.norm_instances(), args, dev, flush, hbm, stream)
    if e2e:
        r.update(run_e2e(st, g_step, args, world, dev, stream))
    del g_step, g_step_ev, g_off_ev
    return r


def time_back_to_back(inst, args, dev, flush, hbm, stream):
    """Launches of one kernel cycled over distinct input sets (together larger
    than L2), back to back in one graph after one L2 flush: the mean time per
    launch, the achieved bandwidth and its fraction of the measured copy
    bandwidth, with the clocks sampled during the replay."""
    import torch

    fns, nbytes = inst
    reps = max(5, min(args.steps, 20))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(reps):
            for f in fns:
                f()
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    time.sleep(0.05)
    with torch.cuda.stream(stream):
        flush()
        a.record(stream)
        g.replay()
        b.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    n = reps * len(fns)
    us = a.elapsed_time(b) * 1e3 / n
    gbs = nbytes / (us * 1e-6) / 1e9
    del g
    return {"launches": n, "input_sets": len(fns), "us_per_launch": us, "bytes_per_launch": nbytes,
            "achieved": gbs, "unit": "GB/s", "peak": hbm, "frac": gbs / hbm, "clocks": clk,
            "timing": f"{n} launches back to back over {len(fns)} input sets, one L2 flush before"}


def run_e2e(st, graph, args, world, dev, stream):
    """The step through the public API with host buffers: every step copies
    its inputs in from pinned host memory, runs the step and copies every
    output back, all inside the timed region. Two buffer sets (a second capture
    of the step on the other set) let step i's outputs go out and step i+1's
    inputs come in on copy streams while step i+1 computes."""
    import torch
    import torch.distributed as dist

    ins_a, outs_a = st.io()
    host_in = [t.cpu().pin_memory() for t in ins_a]
    main = st.swap_io()
    graph_b = capture(st.step, stream)
    ins_b, outs_b = st.io()
    st.swap_io(main)
    sets = [(ins_a, outs_a, graph), (ins_b, outs_b, graph_b)]
    host_out = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs_a] for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(o.numel() * o.element_size() for o in outs_a)
    n = max(3, min(args.steps, 20))
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for i in range(n):
        b = i % 2
        ins, outs, g = sets[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[b])  # step i-2 has read this input set
            for t, th in zip(ins, host_in):
                t.copy_(th, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # step i-2's outputs are out
            g.replay()
            ev_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            for o, oh in zip(outs, host_out[b]):
                oh.copy_(o, non_blocking=True)
            ev_out[b].record(s_out)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n, dev)
    del graph_b
    return {"e2e_ms": e2e_ms, "h2d": h2d, "d2h": d2h, "e2e_steps": n}


GEMM_TAGS = ("gemm_w8a8", "llmint8_matmul", "gemm_fp8", "bmm_qk")
EXTRA_WORKLOADS = {
    "c4": C4["workload"],
    "c5_fp8": "175B-shaped block on FP8 units: smoothed per-token E4M3 quantisation of both sides' [4096, 12288] "
              "bf16 linear inputs, QKV/out/FC1/FC2 E4M3 GEMMs to bf16 (weights E4M3 per channel, offline)",
    "attn_int8": "attention products in int8 at the 175B-shaped head layout: 96 heads x 128 channels, 2048 tokens; "
                 "per-(head, token) int8 of Q and K, batched QK^T to bf16, per-(head, channel) int8 of V^T, batched PV "
                 "on synthetic int8 probabilities",
}


def gemm_roofline(r, shapes):
    """The dominant kernel's roofline: the int8 GEMM over its launches in one
    step (sum of 2MNK over sum of launch durations)."""
    g = [k for k in r["kernels"] if k["kernel"] in GEMM_TAGS][0]
    ipk = r["ipk"]
    traffic = gemm_traffic(shapes)
    return {"bound": "tensor", "achieved": g["achieved"], "peak": ipk["burst"], "unit": "TOPS",
            "frac": g["achieved"] / ipk["burst"], "traffic": None if traffic is None else sum(traffic),
            "kernel": "gemm_w8a8_kernel", "launches_per_step": g["launches"],
            "ops_per_step": g["ops_per_launch"] * g["launches"],
            "algorithmic_bytes_per_step": g["algorithmic_bytes_per_launch"] * g["launches"],
            "traffic_per": f"one step ({g['launches']} launches)",
            "peak_source": f"{ipk['source']} bf16 burst x 2 (nominal int8:bf16 ratio)",
            "peak_sustained": ipk["sustained"], "frac_sustained": g["achieved"] / ipk["sustained"],
            "peak_nominal": ipk["nominal"], "frac_nominal": g["achieved"] / ipk["nominal"],
            "timing": f"CUDA events around each launch of an instrumented copy of the step's graph, "
                      f"{r['instrumented_replays']} replays after the timed region, L2 flushed before each"}


def config_summary(name, r, tokens, world, shapes):
    """A compact line for a non-headline configuration."""
    g = [k for k in r["kernels"] if k["kernel"] in GEMM_TAGS][0]
    out = {"workload": (CONFIGS[name]["workload"] if name in CONFIGS else EXTRA_WORKLOADS[name]),
           "tokens": tokens, "tokens_per_s": tokens * world / (r["ms_per_step"] * 1e-3),
           "ms_per_step": r["ms_per_step"], "gemm_bound": g["bound"], "gemm_frac": g["frac"],
           "gemm_shapes": shapes, "kernels": r["kernels"], "offline": r["offline"], "clocks": r["clocks"]}
    if g["bound"] == "tensor":
        out.update({"gemm_tops": g["achieved"], "gemm_frac_nominal": g["frac_nominal"]})
    else:
        out["gemm_gbs"] = g["achieved"]
    return out


def json_line(args, world, r, shapes, tokens=None, cfg=None):
    """The benchmark's JSON line (without the CPU baseline) from the measured
    headline stack."""
    cfg = cfg or CONFIGS[HEADLINE]
    tokens = tokens or cfg["tokens"]
    calib = [k for k in r["offline"] if k["kernel"] == "calib_absmax"]
    line = {
        "metric": METRIC, "value": tokens * world / (r["ms_per_step"] * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8",
        "data": "synthetic (seeded draws with the configuration's shapes and outlier channels; no dataset)",
        "config": {"workload": cfg["workload"], "tokens": tokens, "hidden": cfg["hidden"],
                   "parallelism": f"replicas x{world}", "l2": L2_NOTE},
        "roofline": gemm_roofline(r, shapes),
        "kernels": r["kernels"],
        "offline": {"kernels": r["offline"], "ms": sum(k["us_total"] for k in r["offline"]) * 1e-3,
                    "note": "calibration, weight maxima, smoothing factors for every alpha, int8 weights: "
                            "timed separately, not part of the step"},
        "calibration": None if not calib else {
            "batches": r.get("n_calib"), "us_total": calib[0]["us_total"],
            "us_per_batch": calib[0]["us_total"] / max(r.get("n_calib") or 1, 1),
            "bytes": calib[0]["bytes_per_launch"] * calib[0]["launches"], "achieved": calib[0]["achieved"],
            "unit": "GB/s", "peak": r["hbm"], "frac": calib[0]["frac"],
            "timing": "one interval around the whole pass (all batches' tokens in one sq_calib_absmax call over "
                      "the batches stacked in HBM), L2 flushed before"},
        "norm_bandwidth": r.get("norm_bandwidth"),
        "gpu_launches": r["launches_per_step"] * args.steps,
        "clocks": r["clocks"],
    }
    if "e2e_ms" in r:
        line["e2e"] = {"value": tokens * world / (r["e2e_ms"] * 1e-3), "unit": "tokens/s",
                       "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                       "ms_per_step": r["e2e_ms"], "steps": r["e2e_steps"]}
    return line


# MLP chains of the configurations: (name, tokens, hidden, intermediate, act,
# static per-tensor scale for FC2's input?, output dtype)
MLP_CHAINS = (("c2_swiglu", 2048, 1024, 3072, 0, False, "bf16"),
              ("c3_relu_static", 1024, 7168, 28672, 1, True, "fp16"),
              ("c5_gelu", 4096, 12288, 49152, 2, False, "bf16"))


# int8 ops per SM per clock of the dense tensor-core path: 8192 MACs (the
# nominal 4.5 POPS at 148 SMs and 1.855 GHz)
INT8_OPS_PER_SM_CLK = 16384


def int8_ceiling(args, dev, flush, shapes=((8192, 8192, 8192), (4096, 36864, 12288)), reps=10):
    """The measured int8 ceiling beside the library's own GEMM: this library's
    GEMM (int32 and bf16 outputs) against the CUDA library int8 matmul torch
    exposes (torch._int_mm, int32 output) on the same operands, at 8192^3 and
    at the 175B-shaped QKV shape, each launch after an L2 flush, with the
    clocks during the timing and the clock-scaled dense peak (SM count x 16384
    ops/clock x the median SM clock)."""
    import torch

    import w8a8_post_quantization_sq_b200 as sq

    res = {"timing": f"median of {reps} launches, each after an L2 flush", "shapes": []}
    for M, N, K in shapes:
        g = torch.Generator(device=dev).manual_seed(8)
        A = torch.randint(-127, 128, (M, K), generator=g, device=dev, dtype=torch.int8)
        B = torch.randint(-127, 128, (N, K), generator=g, device=dev, dtype=torch.int8)
        qa = torch.rand(M, generator=g, device=dev) + 1
        qb = torch.rand(N, generator=g, device=dev) + 100
        Y32 = torch.empty((M, N), dtype=torch.int32, device=dev)
        Y16 = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K, device=dev)
        Bt = B.t()  # [K, N] column-major view: torch._int_mm computes A @ Bt = A B^T, the same product
        arms = {"ours_int32": lambda: sq.sq_gemm_w8a8(A, B, None, None, None, Y32, ws),
                "ours_bf16": lambda: sq.sq_gemm_w8a8(A, B, qa, qb, None, Y16, ws),
                "torch_int_mm_int32": lambda: torch._int_mm(A, Bt)}
        out = {"shape": [M, N, K]}
        for f in arms.values():
            f()
        torch.cuda.synchronize()
        out["int32_outputs_equal"] = bool(torch.equal(torch._int_mm(A, Bt), Y32))
        clocks = ClockSampler(dev.index if dev.index is not None else 0)
        time.sleep(0.05)
        for name, f in arms.items():
            ms = []
            for _ in range(reps):
                flush(0)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                f()
                b.record()
                torch.cuda.synchronize()
                ms.append(a.elapsed_time(b))
            t = statistics.median(ms) * 1e-3
            out[name] = {"us": t * 1e6, "tops": 2.0 * M * N * K / t / 1e12}
        clk = clocks.stop()
        out["clocks"] = clk
        if clk and clk.get("sm_mhz"):
            sms = torch.cuda.get_device_properties(dev).multi_processor_count
            peak = sms * INT8_OPS_PER_SM_CLK * clk["sm_mhz"] * 1e6 / 1e12
            out["clock_scaled_peak_tops"] = peak
            for name in arms:
                out[name]["frac_clock_scaled"] = out[name]["tops"] / peak
        res["shapes"].append(out)
        del A, B, Y32, Y16, ws
        torch.cuda.empty_cache()
    return res


def time_mlp_chains(args, dev, flush):
    """The MLP of each configuration from an int8 input to the down/FC2
    output, unfused (GEMM to 16-bit Y, the activation + int8 kernel, GEMM)
    and with the activation in the first GEMM's epilogue (its 16-bit h, or
    with a static scale its int8 codes, then GEMM). Synthetic int8 operands;
    each chain one CUDA graph, timed after an L2 flush, mean of the replays."""
    import torch

    import w8a8_post_quantization_sq_b200 as sq

    out = {}
    stream = torch.cuda.Stream(device=dev)
    for name, M, D, I, act, static, odt in MLP_CHAINS:
        dt = torch.bfloat16 if odt == "bf16" else torch.float16
        g = torch.Generator(device=dev).manual_seed(I)
        N1 = 2 * I if act == 0 else I
        ri = lambda *sh: torch.randint(-127, 128, sh, generator=g, device=dev, dtype=torch.int8)  # noqa: E731
        Xq, W1, W2 = ri(M, D), ri(N1, D), ri(D, I)
        qx = torch.rand(M, generator=g, device=dev) * 30 + 20
        q1 = torch.rand(N1, generator=g, device=dev) * 300 + 200 * (D / 1024) ** 0.5
        q2 = torch.rand(D, generator=g, device=dev) * 300 + 200 * (I / 1024) ** 0.5
        Y = torch.empty((M, N1), dtype=dt, device=dev)
        H = torch.empty((M, I), dtype=dt, device=dev)
        X2 = torch.empty((M, I), dtype=torch.int8, device=dev)
        qa = torch.empty(M if not static else 1, device=dev)
        st = torch.tensor([8.0], device=dev) if static else None
        Out = torch.empty((M, D), dtype=dt, device=dev)
        ws1 = sq.workspace(sq.SQ_OP_GEMM, M, N1, D, device=dev)
        ws2 = sq.workspace(sq.SQ_OP_GEMM, M, D, I, device=dev)

        def unfused():
            sq.sq_gemm_w8a8(Xq, W1, qx, q1, None, Y, ws1)
            sq.sq_act_quant(Y, act, not static, st, X2, qa)
            sq.sq_gemm_w8a8(X2, W2, qa, q2, None, Out, ws2)

        def fused():
            if static:
                sq.sq_gemm_w8a8_act(Xq, W1, qx, q1, None, act, X2, ws1, static_qs=st, out_dtype=dt)
                sq.sq_gemm_w8a8(X2, W2, st, q2, None, Out, ws2)
            else:
                sq.sq_gemm_w8a8_act(Xq, W1, qx, q1, None, act, H, ws1)
                sq.sq_quantize_act(H, None, True, None, X2, qa)
                sq.sq_gemm_w8a8(X2, W2, qa, q2, None, Out, ws2)

        r = {"tokens": M, "hidden": D, "intermediate": I, "act": ["swiglu", "relu", "gelu"][act],
             "fc2_input_scale": "static per-tensor" if static else "per token"}
        for key, fn in (("unfused", unfused), ("fused", fused)):
            with torch.cuda.stream(stream):
                fn()
            stream.synchronize()
            reps = max(3, min(args.steps, 20))
            graph = capture(fn, stream)
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
            with torch.cuda.stream(stream):
                graph.replay()
                for i in range(reps):
                    flush(i)
                    ev[i][0].record(stream)
                    graph.replay()
                    ev[i][1].record(stream)
            torch.cuda.synchronize()
            r[key + "_us"] = 1e3 * sum(a.elapsed_time(b) for a, b in ev) / reps
            del graph
        r["speedup"] = r["unfused_us"] / r["fused_us"]
        out[name] = r
        del Xq, W1, W2, Y, H, X2, Out
        torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, dev):
    import torch

    torch.cuda.set_device(dev)
    flush = L2Flush(dev)
    st = Stack(args.workload, dev)
    shapes = st.gemm_shapes()
    r = run_stack(st, args, rank, world, dev, flush, e2e=True)
    cfg = CONFIGS[args.workload]
    line = json_line(args, world, r, shapes, cfg["tokens"], cfg)
    del st
    torch.cuda.empty_cache()
    names = [c for c in args.configs.split(",") if c and c not in ("none", args.workload)]
    for c in names:
        if c not in EXTRA_WORKLOADS and c not in CONFIGS:
            raise SystemExit(f"unknown configuration {c}")
    if names:
        extra = {}
        for name in names:
            if name in EXTRA_WORKLOADS:
                s = {"c4": LlmInt8Stack, "c5_fp8": Fp8Stack, "attn_int8": AttnStack}[name](dev)
                rr = run_stack(s, args, rank, world, dev, flush, e2e=False)
                tokens = {"c4": C4["tokens"], "c5_fp8": 4096, "attn_int8": 2048}[name]
                extra[name] = config_summary(name, rr, tokens, world, s.gemm_shapes())
            else:
                s = Stack(name, dev)
                rr = run_stack(s, args, rank, world, dev, flush, e2e=False)
                extra[name] = config_summary(name, rr, CONFIGS[name]["tokens"], world, s.gemm_shapes())
            del s
            torch.cuda.empty_cache()
        line["configs"] = extra
    if args.mlp_chains:
        line["mlp_chains"] = time_mlp_chains(args, dev, flush)
    if args.ceiling:
        line["int8_ceiling"] = int8_ceiling(args, dev, flush)
    return line


# ------------------------------------------------------------------ CPU arm (the oracle)
class CpuStack:
    """The oracle, as it stands, on the deploy-mode linear stack of a
    configuration, on a sample: `rows` tokens through every online step and the
    first `wfrac` of every weight's output channels. The offline part (the
    calibration maxima, smoothing factors, folded norm parameters, static
    scales and int8 weights of the sampled channels) is made once, untimed.
    A step's time for the whole workload is t_norm * M / rows +
    t_gemm * M / rows / wfrac: both parts are linear in what they process.
    threads > 1 runs the oracle's calls on disjoint row and channel blocks in
    a thread pool (the oracle's C calls release the GIL); the arithmetic is
    the same."""

    def __init__(self, name, rows, wfrac, threads=1):
        import torch

        import oracle
        from w8a8_post_quantization_sq_b200 import inputs

        oracle.lib()
        cfg = CONFIGS[name]
        self.o, self.torch, self.cfg = oracle, torch, cfg
        self.rows, self.wfrac, self.threads = rows, wfrac, threads
        d = getattr(inputs, cfg["gen"])(device="cpu", M=rows, w_frac=wfrac)
        self.d = d
        o = oracle
        self.norm = o.LAYERNORM if cfg["norm"] == "layer" else o.RMSNORM
        eps, alpha = d["eps"], cfg["alpha"]
        sides = ("attn", "mlp")
        consumer = {src: w for w, src in cfg["gemms"] if src != "syn"}
        g = {k: d["gamma"][k].numpy() for k in sides}
        b = {k: None if d["beta"][k] is None else d["beta"][k].numpy() for k in sides}
        xmax = {}
        for k in sides:
            x = np.zeros(cfg["hidden"], np.float32)
            for X in d["calib"]:
                if cfg["calib"] == "absmax":
                    x = o.col_absmax(X, x)
                else:
                    x = o.norm_smooth_quant(X, self.norm, g[k], b[k], eps, quantize=False, absmax=x)["absmax"]
            xmax[k] = x
        self.gp, self.bp, self.qs = {}, {}, {}
        s = {}
        for k in sides:
            s[k] = o.smooth_scales(xmax[k], o.col_absmax(d["W"][consumer[k]]), alpha)
            self.gp[k], self.bp[k] = o.fold_norm(g[k], b[k], s[k])
            if not cfg["per_token"]:
                v = np.zeros(cfg["hidden"], np.float32)
                for X in d["calib"]:
                    v = o.norm_smooth_quant(X, self.norm, self.gp[k], self.bp[k], eps, quantize=False,
                                            absmax=v)["absmax"]
                self.qs[k] = float(o.scale_from_absmax(v))
        self.Wq, self.qw = {}, {}
        for w, src in cfg["gemms"]:
            W = d["W"][w]
            Wp = o.fold_weight(W, s[src]) if src != "syn" else o.f32(W)
            self.Wq[w], self.qw[w] = o.quantize_weight(Wp, True)
        self.h = {k: d["h"][k] for k in sides}
        self.syn = {w: (t[0].numpy(), t[1].numpy()) for w, t in d["syn"].items()}
        self.sides = sides

    def step(self, threads=None):
        """(seconds of norm + int8 work, seconds of GEMM + dequant work) for
        the sample's tokens and weight channels, on `threads` host threads."""
        from concurrent.futures import ThreadPoolExecutor

        o, cfg = self.o, self.cfg
        rows = self.rows
        eps = self.d["eps"]
        T = threads or self.threads
        rnd = o.round_bf16_bits if cfg["out"] == "bf16" else o.round_fp16_bits
        pool = ThreadPoolExecutor(max_workers=T) if T > 1 else None

        def rowblocks(n):
            k = max(1, min(T, n))
            return [(i * n // k, (i + 1) * n // k) for i in range(k)]

        t0 = time.perf_counter()
        Xq, qx = {}, {}
        for k in self.sides:
            h = self.h[k][:rows]
            st = None if cfg["per_token"] else self.qs[k]

            def nq(a, b_, h=h, k=k, st=st):
                return o.norm_smooth_quant(h[a:b_], self.norm, self.gp[k], self.bp[k], eps, cfg["per_token"], st)
            parts = list(pool.map(lambda ab: nq(*ab), rowblocks(rows))) if pool else [nq(0, rows)]
            Xq[k] = np.concatenate([p["Xq"] for p in parts])
            qx[k] = np.concatenate([p["qs"] for p in parts]) if cfg["per_token"] else parts[0]["qs"]
        t_norm = time.perf_counter() - t0
        t0 = time.perf_counter()
        for w, src in cfg["gemms"]:
            if src == "syn":
                xq, q = self.syn[w][0][:rows], self.syn[w][1]
                q = q[:rows] if q.size > 1 else q
            else:
                xq, q = Xq[src], qx[src]
            Wq, qw = self.Wq[w], self.qw[w]
            N = Wq.shape[0]

            def gm(a, b_, xq=xq, q=q, Wq=Wq, qw=qw):
                return rnd(o.dequant(o.gemm_i8(xq, Wq[a:b_]), q, qw[a:b_]))
            if pool:
                list(pool.map(lambda ab: gm(*ab), rowblocks(N)))
            else:
                gm(0, N)
        t_gemm = time.perf_counter() - t0
        if pool:
            pool.shutdown()
        return t_norm, t_gemm

    def full_step_s(self, t_norm, t_gemm):
        M = self.cfg["tokens"]
        return t_norm * M / self.rows + t_gemm * M / self.rows / self.wfrac


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def cpu_baseline(name, rows, wfrac):
    """The oracle on the headline stack, on one core and on every core of
    this host, same sample; returns the line's cpu_baseline entry."""
    M = CONFIGS[name]["tokens"]
    out = {}
    c = CpuStack(name, rows, wfrac)
    c.step(1)  # warm-up: page in the sample
    for T in (1, cpu_threads()):
        tn, tg = c.step(T)
        s = c.full_step_s(tn, tg)
        out[T] = {"value": M / s, "unit": "tokens/s", "cores": T, "step_s": s,
                  "sample_s": tn + tg}
        if T == 1 and cpu_threads() == 1:
            break
    T = max(out)
    smp = (f"{rows} of {M} tokens through the online stack against the first 1/{round(1 / wfrac)} of every "
           f"weight's output channels (weights smoothed and quantised beforehand, untimed), extrapolated "
           f"linearly in tokens and channels")
    return {"value": out[T]["value"], "unit": "tokens/s", "cores": T, "kind": "oracle",
            "sample": smp + f"; measured {out[T]['sample_s']:.2f} s for the sample on {T} threads",
            "single_core": {"value": out[1]["value"], "cores": 1,
                            "sample": f"the same sample, {out[1]['sample_s']:.2f} s on one thread"}}


REF_BUDGET_S = 150.0  # wall time of the reference arm's timed steps, whatever --steps asks for


def ref_sample(t_row_norm, t_row_gemm_full, per_step):
    """Token rows (1..64) and weight fraction (1/16, 1/32, ..., 1/256) of one
    reference step that fit `per_step` seconds, given one token row's norm
    time and one token row's GEMM time against the full weights: the largest
    sample that fits."""
    wfrac = 1 / 16
    while wfrac > 1 / 256 and t_row_norm + t_row_gemm_full * wfrac > per_step:
        wfrac /= 2
    rows = int(max(1, min(64, per_step // max(t_row_norm + t_row_gemm_full * wfrac, 1e-9))))
    return rows, wfrac


def run_reference(args, rank, world):
    """The oracle as the reference arm: the headline stack's online step on a
    bounded sample per step, on one host core, extrapolated to the whole
    workload (the line says so)."""
    if rank != 0:
        return
    name = args.workload
    cfg = CONFIGS[name]
    M = cfg["tokens"]
    probe = CpuStack(name, 2, 1 / 64)
    tn, tg = probe.step()
    t_row_norm, t_row_gemm_full = tn / 2, tg / 2 * 64
    n_warm = min(max(args.warmup, 1), 3)
    rows, wfrac = ref_sample(t_row_norm, t_row_gemm_full, REF_BUDGET_S / max(args.steps + n_warm, 1))
    c = CpuStack(name, rows, wfrac)
    for _ in range(n_warm):
        c.step()
    full, meas = [], []
    for _ in range(args.steps):
        tn, tg = c.step()
        meas.append(tn + tg)
        full.append(c.full_step_s(tn, tg))
    step_s = sum(full) / len(full)
    v = M / step_s
    sample = (f"each step: {rows} of {M} tokens against the first 1/{round(1 / wfrac)} of every weight's output "
              f"channels, timed, then extrapolated linearly in tokens and channels")
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8",
        "data": "synthetic (seeded draws with the configuration's shapes and outlier channels; no dataset)",
        "config": {"workload": cfg["workload"], "tokens": M, "hidden": cfg["hidden"],
                   "parallelism": f"replicas x{args.gpus}", "l2": L2_NOTE},
        "ms_per_step_extrapolated": True,
        "ms_per_step_measured_sample": 1e3 * sum(meas) / len(meas),
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ single kernels
def run_kernel(args):
    """Time one entry point alone on one shape:
    gemm M,N,K | gemm_fp8 M,N,K | bmm B,M,N,K | norm M,K | norm_calib M,K | absmax M,K | act M,I |
    quant_weight N,K |
    llmint8 M,K,N.
    --sets 1: every launch after an L2 flush, each launch timed on its own.
    --sets S > 1: S distinct input/output sets, launches cycling through them
    back to back (one flush before the run); the time per launch is the run's
    time divided by the launches. With S sets larger than L2 in all, no launch
    finds its inputs in L2 (e.g. absmax 4096,12288 --sets 16 is the 16-batch
    calibration pass of the 175B-shaped configuration). The clocks are sampled
    during the timed replay."""
    import torch

    import w8a8_post_quantization_sq_b200 as sq
    from w8a8_post_quantization_sq_b200 import build

    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    shape = [int(x) for x in args.shape.split(",")]
    g = torch.Generator(device=dev).manual_seed(0)
    pk, src = peaks()
    ipk = int8_peaks()
    flush = L2Flush(dev)
    out = {"kernel": args.kernel, "shape": shape, "dtype": args.dtype}

    def make(i):
        """Inputs and outputs of set i; returns the launch."""
        if args.kernel == "gemm":
            M, N, K = shape
            Xq = torch.randint(-127, 128, (M, K), generator=g, device=dev, dtype=torch.int8)
            Wq = torch.randint(-127, 128, (N, K), generator=g, device=dev, dtype=torch.int8)
            qx = torch.rand(M, generator=g, device=dev) + 1
            qw = torch.rand(N, generator=g, device=dev) + 100
            Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            # a 256-byte workspace has no room for a stream-K split: whole tiles only
            ws = (torch.zeros(256, dtype=torch.uint8, device=dev) if args.whole_tiles
                  else sq.workspace(sq.SQ_OP_GEMM, M, N, K, device=dev))
            return lambda: sq.sq_gemm_w8a8(Xq, Wq, qx, qw, None, Y, ws)
        if args.kernel == "gemm_fp8":
            M, N, K = shape
            # random finite E4M3 codes (0x7F / 0xFF, the NaN codes, moved to 0x7E / 0xFE)
            Xq = torch.randint(0, 256, (M, K), generator=g, device=dev, dtype=torch.int32)
            Wq = torch.randint(0, 256, (N, K), generator=g, device=dev, dtype=torch.int32)
            Xq = torch.where((Xq & 0x7F) == 0x7F, Xq - 1, Xq).to(torch.uint8)
            Wq = torch.where((Wq & 0x7F) == 0x7F, Wq - 1, Wq).to(torch.uint8)
            qx = torch.rand(M, generator=g, device=dev) + 1
            qw = torch.rand(N, generator=g, device=dev) + 100
            Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K, device=dev)
            return lambda: sq.sq_gemm_fp8(Xq, Wq, qx, qw, None, Y, ws)
        if args.kernel == "bmm":
            B, M, N, K = shape
            Aq = torch.randint(-127, 128, (B, M, K), generator=g, device=dev, dtype=torch.int8)
            Bq = torch.randint(-127, 128, (B, N, K), generator=g, device=dev, dtype=torch.int8)
            qa = torch.rand(B * M, generator=g, device=dev) + 1
            qb = torch.rand(B * N, generator=g, device=dev) + 100
            Y = torch.empty((B, M, N), dtype=torch.bfloat16, device=dev)
            ws = sq.workspace(sq.SQ_OP_GEMM, M, N, K, device=dev)
            return lambda: sq.sq_bmm_w8a8(Aq, Bq, qa, qb, Y, ws)
        if args.kernel in ("norm", "norm_calib"):
            M, K = shape
            dt16 = torch.float16 if args.dtype == "fp16" else torch.bfloat16
            H = torch.randn((M, K), generator=g, device=dev).to(dt16)
            gamma = torch.rand(K, generator=g, device=dev) + 0.5
            beta = torch.randn(K, generator=g, device=dev) * 0.1 if args.norm == "ln" else None
            nt = sq.SQ_LAYERNORM if args.norm == "ln" else sq.SQ_RMSNORM
            if args.kernel == "norm_calib":  # calibration mode: running max |v| per channel, no codes
                am = torch.zeros(K, device=dev)
                return lambda: sq.sq_norm_smooth_quant(H, nt, gamma, beta, 1e-5, True, None, None, None, am)
            Xq = torch.empty((M, K), dtype=torch.int8, device=dev)
            qs = torch.empty(M, device=dev)
            return lambda: sq.sq_norm_smooth_quant(H, nt, gamma, beta, 1e-5, True, None, Xq, qs)
        if args.kernel == "absmax":
            M, K = shape
            dtx = {"fp16": torch.float16, "bf16": torch.bfloat16, "fp32": torch.float32}[args.dtype]
            X = torch.randn((M, K), generator=g, device=dev).to(dtx)
            return lambda: sq.sq_calib_absmax(X, xmax)
        if args.kernel == "act":
            M, I = shape
            dt16 = torch.float16 if args.dtype == "fp16" else torch.bfloat16
            act = sq.SQ_ACT_RELU if args.act == "relu" else sq.SQ_ACT_SWIGLU
            A = (torch.randn((M, 2 * I if act == sq.SQ_ACT_SWIGLU else I), generator=g, device=dev) * 2).to(dt16)
            Xq = torch.empty((M, I), dtype=torch.int8, device=dev)
            qs = torch.empty(M, device=dev)
            return lambda: sq.sq_act_quant(A, act, True, None, Xq, qs)
        if args.kernel == "quant_weight":
            N, K = shape
            dtx = {"fp16": torch.float16, "bf16": torch.bfloat16, "fp32": torch.float32}[args.dtype]
            W = (torch.randn((N, K), generator=g, device=dev) * 0.02).to(dtx)
            s_ = torch.rand(K, generator=g, device=dev) * 10 + 0.1
            Wq = torch.empty((N, K), dtype=torch.int8, device=dev)
            qw = torch.empty(N, device=dev)
            return lambda: sq.sq_quantize_weight(W, s_, True, Wq, qw)
        if args.kernel == "llmint8":
            from w8a8_post_quantization_sq_b200 import inputs

            M, K, N = shape
            d = inputs.c4_llmint8(device=dev, M=M, K=K, N=N, n_out=args.outliers, seed=i)
            st = sq.llmint8_weight_state(d["W"])
            Y = torch.empty((M, N), dtype=torch.float16, device=dev)
            idx = torch.empty(K, dtype=torch.int32, device=dev)
            n = torch.empty(1, dtype=torch.int32, device=dev)
            ws = sq.workspace(sq.SQ_OP_LLMINT8, M, N, K, device=dev)
            return lambda: sq.sq_llmint8_matmul(d["X"], st, 6.0, 0.0, Y, idx, n, ws)
        raise SystemExit(f"unknown kernel {args.kernel}")

    if args.kernel in ("gemm", "gemm_fp8", "llmint8"):
        if args.kernel == "llmint8":
            M, K, N = shape
        else:
            M, N, K = shape
        # dense int8 and fp8 peaks are both twice the bf16 one (4.5 vs 2.25 PFLOP/s nominal)
        work, unit, peak = 2.0 * M * N * K / 1e12, "TOPS", ipk["burst"]
        out["whole_tiles"] = bool(args.whole_tiles)
    elif args.kernel == "bmm":
        B, M, N, K = shape
        # int8 operands, bf16 output, fp32 row scales: the bytes that must cross HBM once
        nbytes = B * (M * K + N * K + 2 * M * N + 4 * (M + N))
        work, unit, peak = nbytes / 1e9, "GB/s", pk["hbm_gbs"]
        out["ops"] = 2.0 * B * M * N * K
        out["bytes"] = nbytes
    elif args.kernel == "norm":
        M, K = shape
        work, unit, peak = (3.0 * M * K + 4 * M) / 1e9, "GB/s", pk["hbm_gbs"]
        out["norm"] = args.norm
    elif args.kernel == "norm_calib":
        M, K = shape
        work, unit, peak = 2.0 * M * K / 1e9, "GB/s", pk["hbm_gbs"]
        out["norm"] = args.norm
    elif args.kernel == "absmax":
        M, K = shape
        eb = 4 if args.dtype == "fp32" else 2
        work, unit, peak = eb * M * K / 1e9, "GB/s", pk["hbm_gbs"]
        xmax = torch.zeros(K, device=dev)
    elif args.kernel == "act":
        M, I = shape
        work, unit, peak = ((2 if args.act == "relu" else 4) * M * I + M * I + 4 * M) / 1e9, "GB/s", pk["hbm_gbs"]
        out["act"] = args.act
    elif args.kernel == "quant_weight":
        N, K = shape
        eb = 4 if args.dtype == "fp32" else 2
        work, unit, peak = ((eb + 1.0) * N * K + 4 * N) / 1e9, "GB/s", pk["hbm_gbs"]
    else:
        raise SystemExit(f"unknown kernel {args.kernel}")
    fns = [make(i) for i in range(max(args.sets, 1))]
    for _ in range(max(args.warmup, 3)):
        for f in fns:
            f()
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    clocks = None
    if len(fns) == 1:
        # the launches, each preceded by an L2 flush, captured in one CUDA graph
        # so host launch latency stays out of the timed intervals; the events
        # are external, so the replay records them
        ev = [(torch.cuda.Event(enable_timing=True, external=True),
               torch.cuda.Event(enable_timing=True, external=True)) for _ in range(args.steps)]
        with torch.cuda.graph(graph, stream=stream):
            for a, b in ev:
                flush()
                a.record()
                fns[0]()
                b.record()
        clocks = ClockSampler(0)
        time.sleep(0.05)
        graph.replay()
        torch.cuda.synchronize()
        clk = clocks.stop()
        ms = [a.elapsed_time(b) for a, b in ev]
        avg, best = sum(ms) / len(ms), min(ms)
        out["timing"] = "each launch after an L2 flush"
    else:
        n = args.steps * len(fns)
        with torch.cuda.graph(graph, stream=stream):
            for _ in range(args.steps):
                for f in fns:
                    f()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clocks = ClockSampler(0)
        time.sleep(0.05)
        with torch.cuda.stream(stream):
            flush()
            a.record(stream)
            graph.replay()
            b.record(stream)
        torch.cuda.synchronize()
        clk = clocks.stop()
        avg = best = a.elapsed_time(b) / n
        out["timing"] = f"{n} launches back to back over {len(fns)} input sets"
    ach = work / (avg * 1e-3)
    out.update({"avg_us": avg * 1e3, "min_us": best * 1e3, "achieved": ach, "unit": unit,
                "peak": peak, "frac": ach / peak, "peak_source": src, "clocks": clk})
    if unit == "TOPS":
        out.update({"frac_sustained": ach / ipk["sustained"], "frac_nominal": ach / ipk["nominal"]})
    if "ops" in out:
        out["tops"] = out["ops"] / (avg * 1e-3) / 1e12
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", default=None, help="time one entry point alone: gemm|norm|absmax|quant_weight|llmint8")
    ap.add_argument("--shape", default="4096,36864,12288")
    ap.add_argument("--dtype", default="bf16", help="input dtype of --kernel absmax|quant_weight|norm")
    ap.add_argument("--norm", default="rms", help="--kernel norm: rms|ln")
    ap.add_argument("--act", default="swiglu", help="--kernel act: swiglu|relu")
    ap.add_argument("--whole-tiles", action="store_true", help="--kernel gemm: a workspace without stream-K scratch")
    ap.add_argument("--outliers", type=int, default=6, help="--kernel llmint8: outlier dimensions in X")
    ap.add_argument("--sets", type=int, default=1, help="--kernel: input sets cycled back to back (1: flush each)")
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(CONFIGS), help="the headline stack")
    ap.add_argument("--configs", default="c2,c3,c4,c5_fp8,attn_int8",
                    help="other stacks timed and reported under 'configs' (none: only the headline)")
    ap.add_argument("--no-mlp-chains", dest="mlp_chains", action="store_false",
                    help="skip the MLP chains (activation unfused / in the GEMM epilogue)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=64, help="token rows of the CPU baseline sample")
    ap.add_argument("--cpu-wfrac", type=float, default=1 / 16, help="fraction of weight channels in the CPU sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-ceiling", dest="ceiling", action="store_false",
                    help="skip the int8 ceiling (this library's GEMM against torch._int_mm at 8192^3)")
    args = ap.parse_args()
    if args.kernel:
        run_kernel(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    from w8a8_post_quantization_sq_b200 import build

    if rank == 0:
        build.build()
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        torch.cuda.set_device(dev)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
        dist.barrier()
    line = run_ours(args, rank, world, dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_rows, args.cpu_wfrac)
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
