"""The Qwen3-0.6B-shaped decoder layer with every row of the path in one step
(test helper for the whole-step parity test).

One step runs, on five streams forked from and joined back into the current
stream: the calibration norm pass and column absmax of both linear inputs,
the weight maxima, the smoothing factors with gamma folded, the int8 weights
(up_proj's with the fold of down_proj's factors), the fused RMSNorm +
smoothing + per-token int8, the four GEMMs, the SwiGLU + int8 of the gate/up
output feeding down_proj, and the LLM.int8 decomposition of the q/k/v
projection. It exercises every entry point together, on concurrent streams
and inside a CUDA graph.
"""
from __future__ import annotations

M_TOKENS, HIDDEN = 2048, 1024


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
        # kept for the parity test: every stage of the set-up is checked
        self.calib = {"V": V, "Xq": Xq, "qx": qx, "Wq": Wq, "qw": qw, "Y": Y, "hmax": hmax, "wmax": wmax}
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


