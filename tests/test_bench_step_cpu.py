"""The benchmark step's launch claim against its code (CPU, no kernels run).

bench.py reports `gpu_launches` = LAUNCHES_PER_STEP x steps. This test runs the
step's host code against stand-ins that record which entry points it calls,
and adds up the kernels each entry point launches in the step's configuration
(16-bit inputs under 16 MB for the absmax calls, per-channel weights, K = 1024
norms, the LLM.int8 weight state keeping its W_O copy, O unchanged)."""
from unittest import mock

import bench

# kernels per call of each entry point in the step's configuration
KERNELS = {
    "sq_weight_absmax": 1,
    "sq_calib_absmax": 1,
    "sq_smooth_fold_norm": 1,
    "sq_norm_smooth_quant": 1,
    "sq_quantize_weight": 1,
    "sq_quantize_weight_fold_prev": 1,
    "sq_gemm_w8a8": 1,
    "sq_act_quant": 1,
    # counts, compaction, weight-side pass, row quantisation, GEMM
    "sq_llmint8_matmul": 5,
}


class RecordingSQ:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if name.startswith("SQ_"):
            return 0

        def call(*args, **kwargs):
            self.calls.append(name)
        return call


def run_step_host_code():
    sq = RecordingSQ()
    layer = mock.MagicMock()
    layer.sq = sq
    layer.torch = mock.MagicMock()
    layer.d = {"eps": 1e-6, "alpha": 0.5}
    layer.I = 3072
    layer.streams = [mock.MagicMock() for _ in range(5)]
    layer.act_in = {"o": (mock.MagicMock(), mock.MagicMock()), "down": (mock.MagicMock(), mock.MagicMock())}
    bench.Layer.step(layer)
    return sq.calls


def test_step_calls_known_entry_points():
    calls = run_step_host_code()
    assert calls, "the step made no calls"
    assert set(calls) <= set(KERNELS), set(calls) - set(KERNELS)


def test_launch_claim_matches_the_step():
    calls = run_step_host_code()
    assert sum(KERNELS[c] for c in calls) == bench.LAUNCHES_PER_STEP
    # every row of the path is in the step
    for row in ("sq_calib_absmax", "sq_weight_absmax", "sq_smooth_fold_norm", "sq_quantize_weight",
                "sq_norm_smooth_quant", "sq_gemm_w8a8", "sq_llmint8_matmul", "sq_act_quant",
                "sq_quantize_weight_fold_prev"):
        assert row in calls, row


def test_reference_sample_fits_the_budget():
    """The reference arm's per-step sample fits its share of the wall-time
    budget for any --steps, and is the full 64-row, full-weight sample when
    there is room."""
    t_w, t_row = 0.25, 0.0066  # seconds: full weight side, one token row (oracle on one core)
    assert bench.ref_sample(t_w, t_row, bench.REF_BUDGET_S / 20) == (64, 1.0)
    for steps in (200, 500, 2000, 10000):
        per_step = bench.REF_BUDGET_S / steps
        rows, wfrac = bench.ref_sample(t_w, t_row, per_step)
        assert 1 <= rows <= 64 and 1 / 64 <= wfrac <= 1
        assert wfrac == 1 or t_w * wfrac <= per_step / 2 or wfrac == 1 / 64
        if steps <= 2000:
            assert t_w * wfrac + rows * t_row <= per_step


def test_json_line_contract():
    """The benchmark's JSON line from a synthetic measurement: every key the
    line must carry, whole-job tokens/s over the ranks, the roofline fraction
    as achieved / peak, and the launch claim as kernels per step x steps."""
    import json
    import types

    args = types.SimpleNamespace(steps=100, warmup=5)
    r = {"ms_per_step": 0.125, "e2e_ms": 1.25, "gemm_avg_ms": [0.03, 0.02, 0.05, 0.02], "gemm_tops": 500.0,
         "i8_peak": 3300.0, "peak_src": "measured", "gemm_timed_steps": 200, "h2d": 8 << 20, "d2h": 64 << 20,
         "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}}
    line = json.loads(json.dumps(bench.json_line(args, 2, r)))
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in line, k
    assert line["value"] == bench.M_TOKENS * 2 / 0.125e-3
    assert line["e2e"]["value"] == bench.M_TOKENS * 2 / 1.25e-3
    assert line["e2e"]["h2d_bytes_per_step"] == 8 << 20 and line["e2e"]["d2h_bytes_per_step"] == 64 << 20
    ops = sum(2.0 * m * n * k for (m, n, k) in bench.GEMMS[:4])
    assert abs(line["roofline"]["achieved"] - ops / 0.12e-3 / 1e12) < 1e-9 * line["roofline"]["achieved"]
    assert line["roofline"]["frac"] == line["roofline"]["achieved"] / 3300.0
    assert line["roofline"]["bound"] == "tensor" and line["roofline"]["unit"] == "TOPS"
    assert line["gpu_launches"] == bench.LAUNCHES_PER_STEP * 100
    assert line["n_gpus"] == 2 and line["scaling"] == "weak" and line["higher_is_better"] is True
    assert "workload" in line["config"] and "l2" in line["config"]
