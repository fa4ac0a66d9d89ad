"""Benchmark of the SmoothQuant W8A8 linear-layer path on B200.

One step = one pass of every hot-path row over one batch of synthetic input
shaped like a Qwen3-0.6B decoder layer at 2048 tokens (hidden 1024; q/k/v
fused 1024->4096, o 2048->1024, gate/up fused 1024->6144, down 3072->1024;
6 activation channels x20..x100):
  norm pass producing the linear input (RMSNorm, original gamma)        x2
  calibration absmax of that input                                      x2
  weight absmax over the fused consumers                                x2
  smoothing factors and gamma' = gamma / s (one launch)                 x2
  weight fold + int8 quantisation (per output channel)                  x5
    (up_proj's also takes 1/s of down_proj's input on its output channels)
  fused RMSNorm + smoothing + per-token int8                            x2
  int8 GEMM + dequant epilogue to bf16                                  x4
  SwiGLU of the gate/up output + per-token int8 (down_proj's input)     x1
  LLM.int8 decomposition of the q/k/v projection (bf16)                 x1
The independent chains of the step (the attention-side and MLP-side
calibration/quantisation chains, the weight-side work, the o/down GEMMs and the
LLM.int8 call) run on their own streams inside the step, joined at its end.
The step is captured once in a CUDA graph and replayed. L2 is flushed (a
256 MB write, then a 256 MB read of another buffer so that no dirty line of the
flush is left to be written back) before every timed step, outside the timed
interval; each step is bracketed by CUDA events on the stream it runs on. The
GEMMs' launch durations come from a second capture of the step with events
around each GEMM, replayed after the timed region (event nodes inside the
graph cut the programmatic chaining of a GEMM to its producer, which costs the
step 10-25 us, so they stay out of the timed graph).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). With torchrun (N > 1) every rank runs its own
replica of the step on its own GPU (no data-path collective; weak scaling).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

M_TOKENS, HIDDEN = 2048, 1024
WORKLOAD = ("qwen3-0.6b-shaped decoder layer linear stack, 2048 tokens, hidden 1024, bf16 in/out, int8 GEMMs; "
            "down_proj input from the SwiGLU of the gate/up output")
METRIC = "W8A8 GEMM TOPS & tokens/s at 1 B200; % of INT8 TC peak / HBM GB/s"
# GEMM (M, N, K) of one step: qkv, o, gate/up, down, LLM.int8 q/k/v
GEMMS = [(2048, 4096, 1024), (2048, 1024, 2048), (2048, 6144, 1024), (2048, 1024, 3072), (2048, 4096, 1024)]
# our kernels in one step: weight absmax 2, calibration absmax 2, smoothing +
# gamma fold 2, norm passes 4, weight quantisation 5 (up_proj's with the fold
# of down_proj's s), GEMMs 4, SwiGLU + int8 1, LLM.int8 5 (counts, compaction,
# weight-side pass, row quantisation, GEMM)
# steps of the instrumented copy of the step that time the GEMM launches
GEMM_TIMED_STEPS = 200
LAUNCHES_PER_STEP = (2 * 1 + 2 * 1 + 2 * 1 + 2 * 2 + 5 * 1 + 4 * 1 + 1 + 5)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


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


def gemm_traffic():
    """DRAM bytes per launch of the step's four GEMMs, from the ncu counters
    recorded in profiles/gemm_traffic.json, or None once the kernel's sources
    differ from those the counters were taken on."""
    p = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    return d.get("bytes_per_launch") if d.get("sources_sha256") == gemm_sources_digest() else None


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
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i] and "Not" not in r[5 + i]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ GPU arm
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


class Layer:
    """Device buffers and the step for the Qwen3-0.6B-shaped layer."""

    def __init__(self, dev):
        import torch

        import w8a8_post_quantization_sq_b200 as sq
        from w8a8_post_quantization_sq_b200 import inputs

        self.sq, self.torch = sq, torch
        d = inputs.c2_qwen3_06b(device=dev)
        self.d = d
        M, K = M_TOKENS, HIDDEN
        e = lambda *s, dt=torch.float32: torch.empty(s, dtype=dt, device=dev)  # noqa: E731
        self.h = {"attn": d["h_attn"], "mlp": d["h_mlp"]}
        self.gamma = {"attn": d["gamma_attn"].float().contiguous(), "mlp": d["gamma_mlp"].float().contiguous()}
        self.W = d["W"]
        self.V = {k: e(M, K, dt=torch.bfloat16) for k in ("attn", "mlp")}
        # the four running maxima share one buffer, cleared by one fill per step
        self.maxima = e(4, K)
        self.xmax = {"attn": self.maxima[0], "mlp": self.maxima[1]}
        self.wmax = {"attn": self.maxima[2], "mlp": self.maxima[3]}
        self.s = {k: e(K) for k in ("attn", "mlp")}
        self.gp = {k: e(K) for k in ("attn", "mlp")}
        self.Wq = {k: e(*self.W[k].shape, dt=torch.int8) for k in self.W}
        self.qw = {k: e(self.W[k].shape[0]) for k in self.W}
        self.Xq = {k: e(M, K, dt=torch.int8) for k in ("attn", "mlp")}
        self.qx = {k: e(M) for k in ("attn", "mlp")}
        xo, so = d["o_in"]
        xd, sd = d["down_in"]
        self.act_in = {"o": (xo, so), "down": (xd, sd)}
        self.Y = {k: e(M, self.W[k].shape[0], dt=torch.bfloat16) for k in self.W}
        self.Y["llm"] = e(M, 4096, dt=torch.bfloat16)
        self.ws = sq.workspace(sq.SQ_OP_LLMINT8, M, 4096, K, device=dev)
        self.ws_gemm = {k: sq.workspace(sq.SQ_OP_GEMM, M, 4096, K, device=dev) for k in ("qkv", "o", "gateup", "down")}
        self.llm = sq.llmint8_weight_state(self.W["qkv"])
        self.idx = e(K, dt=torch.int32)
        self.nidx = e(1, dt=torch.int32)
        # down_proj's input: SwiGLU of the gate/up output, smoothed by s_down
        # folded into up_proj's output channels
        I = self.W["down"].shape[1]
        self.I = I
        self.W_gate, self.W_up = self.W["gateup"][:I], self.W["gateup"][I:]
        self.Xq_down = e(M, I, dt=torch.int8)
        self.qx_down = e(M)
        self.s_down = self.calibrate_down()
        self.streams = [torch.cuda.Stream(device=dev) for _ in range(5)]
        self.events = {n: torch.cuda.Event() for n in ("wmax_attn", "wmax_mlp", "V_attn", "V_mlp", "s_attn", "s_mlp",
                                                      "wq_qkv", "wq_gateup", "wq_down")}

    def calibrate_down(self):
        """s for down_proj's input, from one pass of the MLP input through the
        unsmoothed int8 gate/up projection: running max of |silu(gate) * up|
        (calibration mode of sq_act_quant) against down_proj's weight maxima. Done once, at
        set-up; the step then folds it (1/s into up_proj's rows, s into
        down_proj's columns)."""
        sq, d, torch = self.sq, self.d, self.torch
        M, K, I = M_TOKENS, HIDDEN, self.I
        dev = self.h["mlp"].device
        e = lambda *s_, dt=torch.float32: torch.empty(s_, dtype=dt, device=dev)  # noqa: E731
        V = e(M, K, dt=torch.bfloat16)
        sq.sq_norm_smooth_quant(self.d["h_calib"].to(dev), sq.SQ_RMSNORM, self.gamma["mlp"], None, d["eps"], True, None,
                                None, None, None, V)
        Xq, qx = e(M, K, dt=torch.int8), e(M)
        sq.sq_quantize_act(V, None, True, None, Xq, qx)
        Wq, qw = e(2 * I, K, dt=torch.int8), e(2 * I)
        sq.sq_quantize_weight(self.W["gateup"], None, True, Wq, qw)
        Y = e(M, 2 * I, dt=torch.bfloat16)
        sq.sq_gemm_w8a8(Xq, Wq, qx, qw, None, Y, sq.workspace(sq.SQ_OP_GEMM, M, 2 * I, K, device=dev))
        hmax = torch.zeros(I, device=dev)
        sq.sq_act_quant(Y, sq.SQ_ACT_SWIGLU, True, None, None, None, hmax)
        wmax = torch.zeros(I, device=dev)
        sq.sq_weight_absmax(self.W["down"], wmax)
        s = e(I)
        sq.sq_smooth_scales(hmax, wmax, d["alpha"], s)
        torch.cuda.synchronize()
        return s

    def step(self, gemm_ev=None):
        """One pass of every row. Independent chains run on their own streams
        (forked from and joined back into the current stream), so the
        latency-bound small kernels of one chain overlap the others."""
        sq, d, torch = self.sq, self.d, self.torch
        eps = d["eps"]
        I = self.I
        main = torch.cuda.current_stream()
        sA, sB, sC, sD, sE = self.streams
        ev = self.events
        self.maxima.zero_()
        for s_ in self.streams:
            s_.wait_stream(main)

        def gemm(i, w, xq, qx):
            if gemm_ev is not None:
                gemm_ev[i][0].record()
            sq.sq_gemm_w8a8(xq, self.Wq[w], qx, self.qw[w], None, self.Y[w], self.ws_gemm[w])
            if gemm_ev is not None:
                gemm_ev[i][1].record()

        # the MLP chain (norm -> gate/up GEMM -> SwiGLU -> down GEMM) is the
        # longest, so the weight-side work it waits for goes first on each stream
        with torch.cuda.stream(sC):
            sq.sq_weight_absmax(self.W["gateup"], self.wmax["mlp"])
            ev["wmax_mlp"].record()
            sq.sq_weight_absmax(self.W["qkv"], self.wmax["attn"])
            ev["wmax_attn"].record()
            sq.sq_quantize_weight(self.W["down"], self.s_down, True, self.Wq["down"], self.qw["down"])
            ev["wq_down"].record()
            sq.sq_quantize_weight(self.W["o"], None, True, self.Wq["o"], self.qw["o"])
            gemm(1, "o", *self.act_in["o"])
        chains = (("attn", "qkv", sA, 0), ("mlp", "gateup", sB, 2))
        for k, w, s_, i in chains:
            with torch.cuda.stream(s_):
                # norm (calibration pass) -> linear input; its column absmax
                sq.sq_norm_smooth_quant(self.h[k], sq.SQ_RMSNORM, self.gamma[k], None, eps, True, None, None,
                                        None, None, self.V[k])
                ev["V_" + k].record()
                sq.sq_calib_absmax(self.V[k], self.xmax[k])
                s_.wait_event(ev["wmax_" + k])
                # s and gamma' = gamma / s in one launch
                sq.sq_smooth_fold_norm(self.xmax[k], self.wmax[k], d["alpha"], self.gamma[k], None, self.s[k],
                                       self.gp[k])
                ev["s_" + k].record()
                sq.sq_norm_smooth_quant(self.h[k], sq.SQ_RMSNORM, self.gp[k], None, eps, True, None,
                                        self.Xq[k], self.qx[k], None, None)
        with torch.cuda.stream(sD):  # weight quantisation once s is known
            sD.wait_event(ev["s_mlp"])
            sq.sq_quantize_weight(self.W_gate, self.s["mlp"], True, self.Wq["gateup"][:I], self.qw["gateup"][:I])
            # up_proj: 1/s_down folded into its output channels (down_proj takes
            # s_down) and its own s, in the quantising pass
            sq.sq_quantize_weight_fold_prev(self.W_up, self.s_down, self.s["mlp"], self.Wq["gateup"][I:],
                                            self.qw["gateup"][I:])
            ev["wq_gateup"].record()
            sD.wait_event(ev["s_attn"])
            sq.sq_quantize_weight(self.W["qkv"], self.s["attn"], True, self.Wq["qkv"], self.qw["qkv"])
            ev["wq_qkv"].record()
        for k, w, s_, i in chains:
            with torch.cuda.stream(s_):
                s_.wait_event(ev["wq_" + w])
                gemm(i, w, self.Xq[k], self.qx[k])
        with torch.cuda.stream(sB):
            # down_proj's input from the SwiGLU of the gate/up output
            sq.sq_act_quant(self.Y["gateup"], sq.SQ_ACT_SWIGLU, True, None, self.Xq_down, self.qx_down)
            sB.wait_event(ev["wq_down"])
            gemm(3, "down", self.Xq_down, self.qx_down)
        with torch.cuda.stream(sE):  # LLM.int8 decomposition
            sE.wait_event(ev["V_attn"])
            sq.sq_llmint8_matmul(self.V["attn"], self.llm, 6.0, 0.0, self.Y["llm"], self.idx, self.nidx, self.ws)
        for s_ in self.streams:
            main.wait_stream(s_)

    def outputs(self):
        return [self.Y[k] for k in ("qkv", "o", "gateup", "down", "llm")]


def run_ours(args, rank, world, dev):
    import torch
    import torch.distributed as dist

    torch.cuda.set_device(dev)
    L = Layer(dev)
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        L.step()
        L.step()
    stream.synchronize()
    # the step as timed: one CUDA graph with nothing but the step in it
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        L.step()
    # a second capture of the same step with events around its four GEMMs, for
    # their launch durations; event nodes break the programmatic chaining of
    # the GEMMs with their producers, so this copy is replayed after the timed
    # region, not inside it (external events are re-recorded by every replay)
    n_g = 4
    gemm_ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in range(n_g)]
    graph_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_ev, stream=stream):
        L.step(gemm_ev)
    flush = L2Flush(dev)
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            graph.replay()
            graph_ev.replay()
    torch.cuda.synchronize()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    time.sleep(0.05)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(args.steps):
            flush(i)
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(step_ms), dev)
    ms_per_step = total_ms / args.steps

    # GEMM launch durations: the instrumented step, L2 flushed before each
    gemm_ms = []
    n_ev = min(args.steps, GEMM_TIMED_STEPS)
    with torch.cuda.stream(stream):
        for i in range(n_ev):
            flush(i)
            graph_ev.replay()
            stream.synchronize()
            gemm_ms.append([gemm_ev[j][0].elapsed_time(gemm_ev[j][1]) for j in range(n_g)])
    torch.cuda.synchronize()

    # e2e through the public API with host buffers: every step copies its
    # inputs in from pinned host memory, runs the step and copies every output
    # back, all inside the timed region. Two buffer sets (a second capture of
    # the step on the other set) let step i's outputs go out and step i+1's
    # inputs come in on copy streams while step i+1 computes.
    h_host = {k: L.h[k].cpu().pin_memory() for k in L.h}
    h_alt = {k: torch.empty_like(v) for k, v in L.h.items()}
    y_alt = {k: torch.empty_like(v) for k, v in L.Y.items()}
    h_main, y_main = L.h, L.Y
    L.h, L.Y = h_alt, y_alt
    graph_b = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_b, stream=stream):
        L.step()
    outs_b = L.outputs()
    L.h, L.Y = h_main, y_main
    sets = [(L.h, L.outputs(), graph), (h_alt, outs_b, graph_b)]
    o_host = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs_b] for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in h_host.values())
    d2h = sum(o.numel() * o.element_size() for o in outs_b)
    e2e_steps = max(3, min(args.steps, 50))
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
    for i in range(e2e_steps):
        b = i % 2
        h_dev, outs, g = sets[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[b])  # step i-2 has read this input set
            for k in h_dev:
                h_dev[k].copy_(h_host[k], non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # step i-2's outputs are out
            g.replay()
            ev_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            for o, oh in zip(outs, o_host[b]):
                oh.copy_(o, non_blocking=True)
            ev_out[b].record(s_out)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
    del graph_b

    gm = np.array(gemm_ms)  # [steps, 4]
    gemm_ops = [2.0 * m * n * k for (m, n, k) in GEMMS[:4]]
    gemm_avg_ms = gm.mean(axis=0)
    gemm_tops = sum(gemm_ops) / (gemm_avg_ms.sum() * 1e-3) / 1e12
    pk, src = peaks()
    i8_peak = 2.0 * pk["bf16_tflops"]  # dense int8 = 2 x dense bf16 (nominal 4.5 vs 2.25 PFLOP/s)
    del graph, graph_ev
    return {
        "ms_per_step": ms_per_step, "e2e_ms": e2e_ms, "h2d": h2d, "d2h": d2h, "clocks": clk,
        "gemm_avg_ms": gemm_avg_ms.tolist(), "gemm_timed_steps": n_ev, "gemm_tops": gemm_tops, "i8_peak": i8_peak, "peak_src": src,
        "step_ms_median": statistics.median(step_ms),
    }


# ------------------------------------------------------------------ CPU arm
class CpuStep:
    """The oracle, as it stands, on the benchmark's step, timed on a sample.

    The inputs, and the step's set-up (down_proj's smoothing factors from a
    calibration pass, and the full int8 weights the token rows multiply), are
    made once, untimed. Each call of ``step(rows, wfrac)`` then times the
    whole path on a sample: the per-token work for ``rows`` tokens, and the
    weight-side work (maxima, smoothing factors, folds, quantisation, the
    LLM.int8 weight requantisation) on the first ``wfrac`` of every weight's
    output channels. Both are linear in what they process, so the step time
    of the full workload is t_weights / wfrac + t_rows * tokens / rows."""

    def __init__(self, rows=64):
        import torch

        import oracle
        from w8a8_post_quantization_sq_b200 import inputs

        oracle.lib()
        self.o, self.torch = oracle, torch
        d = inputs.c2_qwen3_06b(device="cpu")
        self.d = d
        self.gamma = {"attn": d["gamma_attn"].numpy(), "mlp": d["gamma_mlp"].numpy()}
        self.W = W = {k: oracle.f32(v) for k, v in d["W"].items()}
        self.I = I = W["down"].shape[1]
        sl = slice(0, rows)
        # down_proj's smoothing factors, from a calibration pass over the sample
        Vc = oracle.norm_smooth_quant(d["h_calib"][sl], oracle.RMSNORM, self.gamma["mlp"], None, d["eps"],
                                      quantize=False, want_v=True)["V"]
        Vc16 = torch.from_numpy(Vc).to(torch.bfloat16).float().numpy()
        Xc, qc = oracle.quantize_act(Vc16, None, per_token=True)
        Wc, qwc = oracle.quantize_weight(W["gateup"], True)
        hmax = oracle.act_quant(self.bf16(oracle.dequant(oracle.gemm_i8(Xc, Wc), qc, qwc)), oracle.SWIGLU,
                                quantize=False, absmax=np.zeros(I, np.float32))["absmax"]
        self.s_down = oracle.smooth_scales(hmax, oracle.col_absmax(W["down"]), d["alpha"])
        # the full weight side once, for the token rows of every sampled step
        h = {"attn": d["h_attn"][sl], "mlp": d["h_mlp"][sl]}
        V = {k: oracle.norm_smooth_quant(h[k], oracle.RMSNORM, self.gamma[k], None, d["eps"], quantize=False,
                                         want_v=True)["V"] for k in h}
        V16 = {k: torch.from_numpy(V[k]).to(torch.bfloat16) for k in V}
        self.xmax = {k: oracle.col_absmax(V16[k]) for k in V}
        self.gp, self.Wq, self.qw, self.s = {}, {}, {}, {}
        _, self.llm_idx = self.weight_side(1.0, self.gp, self.Wq, self.qw, self.s,
                                           oracle.llmint8_outliers(V16["attn"], 6.0, 0.0))

    def bf16(self, y):
        torch = self.torch
        return torch.from_numpy(self.o.round_bf16_bits(y).view(np.int16)).view(torch.bfloat16).float().numpy()

    def weight_side(self, wfrac, gp, Wq, qw, s, idx):
        """Maxima, smoothing factors, folds and int8 weights on the first
        wfrac of every weight's output channels; returns (seconds, idx)."""
        o, W, I, d = self.o, self.W, self.I, self.d
        part = lambda w: w[: max(1, int(round(w.shape[0] * wfrac)))]  # noqa: E731
        t0 = time.perf_counter()
        for k, w in (("attn", "qkv"), ("mlp", "gateup")):
            wmax = o.col_absmax(part(W[w]))
            s[k] = o.smooth_scales(self.xmax[k], wmax, d["alpha"])
            gp[k], _ = o.fold_norm(self.gamma[k], None, s[k])
        Wq["qkv"], qw["qkv"] = o.quantize_weight(o.fold_weight(part(W["qkv"]), s["attn"]), True)
        up_f, _ = o.fold_prev_linear(part(W["gateup"][I:]), self.s_down[: part(W["gateup"][I:]).shape[0]])
        gate_q, gate_s = o.quantize_weight(o.fold_weight(part(W["gateup"][:I]), s["mlp"]), True)
        up_q, up_s = o.quantize_weight(o.fold_weight(up_f, s["mlp"]), True)
        Wq["gateup"], qw["gateup"] = np.concatenate([gate_q, up_q]), np.concatenate([gate_s, up_s])
        Wq["o"], qw["o"] = o.quantize_weight(part(W["o"]), True)
        Wq["down"], qw["down"] = o.quantize_weight(o.fold_weight(part(W["down"]), self.s_down), True)
        Wq["llm"], qw["llm"] = o.llmint8_quant_weight(part(W["qkv"]), idx)
        return time.perf_counter() - t0, idx

    def step(self, rows, wfrac=1.0):
        """(seconds of weight-side work scaled to all channels, seconds of
        per-token work for `rows` tokens)."""
        o, d, torch = self.o, self.d, self.torch
        sl = slice(0, rows)
        h = {"attn": d["h_attn"][sl], "mlp": d["h_mlp"][sl]}
        t0 = time.perf_counter()
        V = {k: o.norm_smooth_quant(h[k], o.RMSNORM, self.gamma[k], None, d["eps"], quantize=False,
                                    want_v=True)["V"] for k in h}
        V16 = {k: torch.from_numpy(V[k]).to(torch.bfloat16) for k in V}
        for k in V:
            o.col_absmax(V16[k])
        t_rows = time.perf_counter() - t0
        t_w, _ = self.weight_side(wfrac, {}, {}, {}, {}, self.llm_idx)
        gp, Wq, qw = self.gp, self.Wq, self.qw
        t0 = time.perf_counter()
        Xq, qx = {}, {}
        for k in h:
            r = o.norm_smooth_quant(h[k], o.RMSNORM, gp[k], None, d["eps"], True)
            Xq[k], qx[k] = r["Xq"], r["qs"]
        xo, so = d["o_in"]
        Y = {}
        for w, xq, q in (("qkv", Xq["attn"], qx["attn"]), ("o", xo[sl].numpy(), so[sl].numpy()),
                         ("gateup", Xq["mlp"], qx["mlp"])):
            Y[w] = self.bf16(o.dequant(o.gemm_i8(xq, Wq[w]), q, qw[w]))
        a = o.act_quant(Y["gateup"], o.SWIGLU)
        self.bf16(o.dequant(o.gemm_i8(a["Xq"], Wq["down"]), a["qs"], qw["down"]))
        # LLM.int8 of the q/k/v projection: outlier set over the sample rows,
        # row quantisation, GEMM + outlier term (the weight requantisation for
        # the set is on the weight side)
        idx = o.llmint8_outliers(V16["attn"], 6.0, 0.0)
        Xq8, qx8 = o.llmint8_quant_rows(V16["attn"], idx)
        t_rows += time.perf_counter() - t0
        if not np.array_equal(idx, self.llm_idx):  # untimed here: the weight side times the requantisation
            Wq["llm"], qw["llm"] = o.llmint8_quant_weight(self.W["qkv"], idx)
            self.llm_idx = idx
        t0 = time.perf_counter()
        y = o.llmint8_combine(o.gemm_i8(Xq8, Wq["llm"]), qx8, qw["llm"], V16["attn"], d["W"]["qkv"], idx)
        o.round_bf16_bits(y)
        t_rows += time.perf_counter() - t0
        return t_w / wfrac, t_rows


def cpu_baseline(rows):
    t_w, t_rows = CpuStep(rows).step(rows)
    step_s = t_w + t_rows * (M_TOKENS / rows)
    return {"value": M_TOKENS / step_s, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{rows} of {M_TOKENS} tokens through every step (weights in full: {t_w:.2f} s; "
                      f"token rows: {t_rows:.2f} s), extrapolated linearly in tokens",
            "step_s": step_s}


REF_BUDGET_S = 150.0  # wall time of the reference arm's timed steps, whatever --steps asks for


def ref_sample(t_w_full, t_row, per_step):
    """Token rows (1..64) and weight fraction (1, 1/2, ..., 1/64) of one
    reference step that fit `per_step` seconds, given the full weight side's
    time and one token row's time: the largest sample that fits, weights in
    full and 64 rows when there is room."""
    rows, wfrac = 64, 1.0
    if t_w_full + 64 * t_row <= per_step:
        return rows, wfrac
    while wfrac > 1 / 64 and t_w_full * wfrac > per_step / 2:
        wfrac /= 2
    rows = int(max(1, min(64, (per_step - t_w_full * wfrac) // max(t_row, 1e-9))))
    return rows, wfrac


def run_reference(args, rank, world):
    if rank != 0:
        return
    ctx = CpuStep()
    t_w_full, t16 = ctx.step(16)  # the first warm-up step also sizes the sample
    rows, wfrac = ref_sample(t_w_full, t16 / 16, REF_BUDGET_S / max(args.steps, 1))
    for _ in range(min(max(args.warmup, 1), 3) - 1):
        ctx.step(rows, wfrac)
    times = []
    for _ in range(args.steps):
        t_w, t_rows = ctx.step(rows, wfrac)
        times.append(t_w + t_rows * (M_TOKENS / rows))
    step_s = sum(times) / len(times)
    v = M_TOKENS / step_s
    wpart = "weights in full" if wfrac == 1 else f"1/{round(1 / wfrac)} of every weight's output channels"
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens": M_TOKENS, "hidden": HIDDEN},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: {rows} of {M_TOKENS} tokens and {wpart}, extrapolated linearly"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ single kernels
def run_kernel(args):
    """Time one entry point alone on one shape:
    gemm M,N,K | gemm_fp8 M,N,K | norm M,K | absmax M,K | act M,I | quant_weight N,K | llmint8 M,K,N.
    --sets 1: every launch after an L2 flush, each launch timed on its own.
    --sets S > 1: S distinct input/output sets, launches cycling through them
    back to back (one flush before the run); the time per launch is the run's
    time divided by the launches. With S sets larger than L2 in all, no launch
    finds its inputs in L2 (e.g. absmax 4096,12288 --sets 16 is the 16-batch
    calibration pass of the 175B-shaped configuration)."""
    import torch

    import w8a8_post_quantization_sq_b200 as sq
    from w8a8_post_quantization_sq_b200 import build

    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    shape = [int(x) for x in args.shape.split(",")]
    g = torch.Generator(device=dev).manual_seed(0)
    pk, src = peaks()
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
        if args.kernel == "norm":
            M, K = shape
            dt16 = torch.float16 if args.dtype == "fp16" else torch.bfloat16
            H = torch.randn((M, K), generator=g, device=dev).to(dt16)
            gamma = torch.rand(K, generator=g, device=dev) + 0.5
            beta = torch.randn(K, generator=g, device=dev) * 0.1 if args.norm == "ln" else None
            nt = sq.SQ_LAYERNORM if args.norm == "ln" else sq.SQ_RMSNORM
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
            d = inputs.c4_llmint8(device=dev, M=M, K=K, N=N, seed=i)
            st = sq.llmint8_weight_state(d["W"])
            Y = torch.empty((M, N), dtype=torch.float16, device=dev)
            idx = torch.empty(K, dtype=torch.int32, device=dev)
            n = torch.empty(1, dtype=torch.int32, device=dev)
            ws = sq.workspace(sq.SQ_OP_LLMINT8, M, N, K, device=dev)
            return lambda: sq.sq_llmint8_matmul(d["X"], st, 6.0, 0.0, Y, idx, n, ws)
        raise SystemExit(f"unknown kernel {args.kernel}")

    if args.kernel in ("gemm", "gemm_fp8"):
        M, N, K = shape
        # dense int8 and fp8 peaks are both twice the bf16 one (4.5 vs 2.25 PFLOP/s nominal)
        work, unit, peak = 2.0 * M * N * K / 1e12, "TOPS", 2.0 * pk["bf16_tflops"]
        out["whole_tiles"] = bool(args.whole_tiles)
    elif args.kernel == "norm":
        M, K = shape
        work, unit, peak = (3.0 * M * K + 4 * M) / 1e9, "GB/s", pk["hbm_gbs"]
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
    elif args.kernel == "llmint8":
        M, K, N = shape
        work, unit, peak = 2.0 * M * N * K / 1e12, "TOPS", 2.0 * pk["bf16_tflops"]
    else:
        raise SystemExit(f"unknown kernel {args.kernel}")
    fns = [make(i) for i in range(max(args.sets, 1))]
    for _ in range(max(args.warmup, 3)):
        for f in fns:
            f()
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
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
        graph.replay()
        torch.cuda.synchronize()
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
        with torch.cuda.stream(stream):
            flush()
            a.record(stream)
            graph.replay()
            b.record(stream)
        torch.cuda.synchronize()
        avg = best = a.elapsed_time(b) / n
        out["timing"] = f"{n} launches back to back over {len(fns)} input sets"
    out.update({"avg_us": avg * 1e3, "min_us": best * 1e3, "achieved": work / (avg * 1e-3), "unit": unit,
                "peak": peak, "frac": work / (avg * 1e-3) / peak, "peak_source": src})
    print(json.dumps(out), flush=True)


def json_line(args, world, r):
    """The benchmark's JSON line (without the CPU baseline) from the measured
    step: r holds the step time, the e2e time, the GEMM intervals and peaks,
    the copy sizes and the clock record of run_ours."""
    value = M_TOKENS * world / (r["ms_per_step"] * 1e-3)
    e2e = M_TOKENS * world / (r["e2e_ms"] * 1e-3)
    gemm_avg_s = sum(r["gemm_avg_ms"]) * 1e-3
    gemm_ops = sum(2.0 * m * n * k for (m, n, k) in GEMMS[:4])
    achieved = gemm_ops / gemm_avg_s / 1e12
    traffic = gemm_traffic()
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens": M_TOKENS, "hidden": HIDDEN, "parallelism": f"replicas x{world}",
                   "l2": "flushed before every timed step (256 MB write + 256 MB read, outside the timed interval)",
                   "graph": "one CUDA graph per step"},
        "gemm_tops": r["gemm_tops"], "gemm_avg_us": [x * 1e3 for x in r["gemm_avg_ms"]],
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": r["i8_peak"], "unit": "TOPS",
                     "frac": achieved / r["i8_peak"], "traffic": traffic,
                     "kernel": "gemm_w8a8_kernel", "peak_source": f"{r['peak_src']} bf16 burst x 2 (int8 nominal ratio)",
                     "timing": f"CUDA events around each GEMM of an instrumented copy of the step's graph, "
                               f"{r['gemm_timed_steps']} replays after the timed region, L2 flushed before each"},
        "e2e": {"value": e2e, "unit": "tokens/s", "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "clocks": r["clocks"],
    }
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", default=None, help="time one entry point alone: gemm|norm|absmax|quant_weight|llmint8")
    ap.add_argument("--shape", default="4096,36864,12288")
    ap.add_argument("--dtype", default="bf16", help="input dtype of --kernel absmax|quant_weight|norm")
    ap.add_argument("--norm", default="rms", help="--kernel norm: rms|ln")
    ap.add_argument("--act", default="swiglu", help="--kernel act: swiglu|relu")
    ap.add_argument("--whole-tiles", action="store_true", help="--kernel gemm: a workspace without stream-K scratch")
    ap.add_argument("--sets", type=int, default=1, help="--kernel: input sets cycled back to back (1: flush each)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=256, help="token rows of the CPU baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
    r = run_ours(args, rank, world, dev)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = json_line(args, world, r)
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = {k: v for k, v in cpu_baseline(args.cpu_rows).items() if k != "step_s"}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
