"""The benchmark's host logic on CPU (no kernels run): the launch claim of the
headline step against its code, the reference arm's sample sizing, the JSON
line's keys and arithmetic, and the CPU oracle stack on a tiny sample.

bench.py reports `gpu_launches` = launches per step x steps. The step's host
code runs here against stand-ins that record which entry points it calls; each
of those entry points launches exactly one kernel in the step's configuration
(per-token or static norm + int8 at K <= 16384, the int8 GEMM)."""
import json
import types
from unittest import mock

import pytest

import bench

KERNELS = {"sq_norm_smooth_quant": 1, "sq_gemm_w8a8": 1}


class RecordingSQ:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if name.startswith("SQ_"):
            return 0

        def call(*args, **kwargs):
            self.calls.append(name)
        return call


def fake_stack(name):
    st = mock.MagicMock()
    st.cfg = bench.CONFIGS[name]
    st.sq = RecordingSQ()
    st.bank = None
    st.by_phase = False
    st.M, st.K = 8, 16
    st.d = {"eps": 1e-5}
    st.per_token = st.cfg["per_token"]
    st.launch = lambda tag, work, fn, *a: bench.Stack.launch(st, tag, work, fn, *a)
    W = mock.MagicMock()
    W.shape = (32, 16)
    st.W = {w: W for w, _ in st.cfg["gemms"]}
    y = mock.MagicMock()
    y.element_size.return_value = 2
    st.Y = {w: y for w, _ in st.cfg["gemms"]}
    h = mock.MagicMock()
    h.element_size.return_value = 2
    st.h = {"attn": h, "mlp": h}
    q = mock.MagicMock()
    q.numel.return_value = 8
    st.qx = {"attn": q, "mlp": q}
    st.syn = {w: (mock.MagicMock(), mock.MagicMock()) for w, src in st.cfg["gemms"] if src == "syn"}
    return st


@pytest.mark.parametrize("name", sorted(bench.CONFIGS))
def test_launch_claim_matches_the_step(name):
    st = fake_stack(name)
    bench.Stack.step(st)
    calls = st.sq.calls
    assert set(calls) <= set(KERNELS), set(calls) - set(KERNELS)
    assert sum(KERNELS[c] for c in calls) == bench.Stack.launches_per_step(st)
    # two norm + int8 passes and the four GEMMs
    assert calls.count("sq_norm_smooth_quant") == 2 and calls.count("sq_gemm_w8a8") == 4


def test_instrumented_step_brackets_every_launch():
    """With an event bank attached every launch gets its own event pair,
    tagged with its kernel and its algorithmic work."""
    st = fake_stack("c5")

    class Bank:
        def __init__(self):
            self.pairs = []

        def pair(self, tag, work):
            e = (mock.MagicMock(), mock.MagicMock())
            self.pairs.append((tag, work, e))
            return e

    st.bank = Bank()
    bench.Stack.step(st)
    tags = [t for t, _, _ in st.bank.pairs]
    assert tags == ["norm_quant", "gemm_w8a8", "gemm_w8a8", "norm_quant", "gemm_w8a8", "gemm_w8a8"]
    for tag, work, (a, b) in st.bank.pairs:
        assert a.record.called and b.record.called
        if tag == "gemm_w8a8":
            assert work[0] == "tensor" and work[1] == 2.0 * 8 * 32 * 16
        else:
            assert work[0] == "hbm" and work[1] == 8 * 16 * 2 + 8 * 16 + 4 * 8


def test_reference_sample_fits_the_budget():
    """The reference arm's per-step sample fits its share of the wall-time
    budget for any --steps and stays within 1..64 rows and 1/256..1/16 of the
    weight channels."""
    t_norm, t_gemm = 0.0004, 0.72  # seconds per token row: norm, GEMMs against the full weights
    for steps in (20, 100, 1000, 10000):
        per_step = bench.REF_BUDGET_S / steps
        rows, wfrac = bench.ref_sample(t_norm, t_gemm, per_step)
        assert 1 <= rows <= 64 and 1 / 256 <= wfrac <= 1 / 16
        if rows > 1:
            assert rows * (t_norm + t_gemm * wfrac) <= per_step
    assert bench.ref_sample(t_norm, t_gemm, 7.5) == (64, 1 / 16)


def synthetic_measurement():
    k_step = [
        {"kernel": "norm_quant", "launches": 2, "us_per_launch": 40.0, "us_total": 80.0, "bound": "hbm",
         "achieved": 5000.0, "unit": "GB/s", "peak": 6548.2, "frac": 5000.0 / 6548.2},
        {"kernel": "gemm_w8a8", "launches": 4, "us_per_launch": 1300.0, "us_total": 5200.0, "bound": "tensor",
         "ops_per_launch": 3.7e12, "achieved": 2846.0, "unit": "TOPS", "peak": 3306.6, "frac": 2846.0 / 3306.6,
         "frac_sustained": 2846.0 / 2779.0, "frac_nominal": 2846.0 / 4500.0, "algorithmic_bytes_per_launch": 7.6e8},
    ]
    k_off = [{"kernel": "calib_absmax", "launches": 1, "us_per_launch": 288.0, "us_total": 288.0, "bound": "hbm",
              "bytes_per_launch": 1.61e9, "achieved": 5600.0, "unit": "GB/s", "peak": 6548.2, "frac": 5600.0 / 6548.2}]
    return {"ms_per_step": 5.5, "e2e_ms": 20.0, "h2d": 450 << 20, "d2h": 900 << 20, "e2e_steps": 20,
            "kernels": k_step, "offline": k_off, "instrumented_replays": 20,
            "ipk": {"burst": 3306.6, "sustained": 2779.0, "nominal": 4500.0, "source": "measured"}, "hbm": 6548.2,
            "launches_per_step": 6, "n_calib": 16, "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []},
            "norm_bandwidth": {"us_per_launch": 30.0, "achieved": 5033.0, "frac": 5033.0 / 6548.2}}


def test_json_line_contract():
    """The benchmark's JSON line from a synthetic measurement: every key the
    line must carry, whole-job tokens/s over the ranks, the roofline fraction
    as achieved / peak (with the sustained and nominal peaks beside it), and
    the launch claim as kernels per step x steps."""
    args = types.SimpleNamespace(steps=20, warmup=5)
    r = synthetic_measurement()
    shapes = [(4096, 36864, 12288), (4096, 12288, 12288), (4096, 49152, 12288), (4096, 12288, 49152)]
    line = json.loads(json.dumps(bench.json_line(args, 2, r, shapes)))
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in line, k
    assert line["value"] == 4096 * 2 / 5.5e-3
    assert line["e2e"]["value"] == 4096 * 2 / 20.0e-3
    assert line["e2e"]["h2d_bytes_per_step"] == 450 << 20 and line["e2e"]["d2h_bytes_per_step"] == 900 << 20
    rf = line["roofline"]
    assert rf["bound"] == "tensor" and rf["unit"] == "TOPS" and rf["achieved"] == 2846.0
    assert rf["frac"] == 2846.0 / 3306.6 and rf["frac_nominal"] == 2846.0 / 4500.0
    assert rf["frac_sustained"] == 2846.0 / 2779.0
    assert rf["ops_per_step"] == 4 * 3.7e12
    assert line["gpu_launches"] == 6 * 20
    assert line["n_gpus"] == 2 and line["scaling"] == "weak" and line["higher_is_better"] is True
    assert line["config"]["workload"] == bench.CONFIGS["c5"]["workload"] and "l2" in line["config"]
    assert line["config"]["tokens"] == 4096 and line["config"]["hidden"] == 12288
    assert line["calibration"]["batches"] == 16 and line["calibration"]["us_per_batch"] == 18.0
    assert line["calibration"]["bytes"] == 1.61e9 and line["norm_bandwidth"]["us_per_launch"] == 30.0
    assert abs(line["offline"]["ms"] - 0.288) < 1e-12


def test_reference_line_has_the_same_config():
    """The reference arm prints the same `config` as the GPU arm (one workload,
    one comparison) and flags its extrapolated step time."""
    import inspect

    src = inspect.getsource(bench.run_reference)
    assert '"config": {"workload": cfg["workload"], "tokens": M, "hidden": cfg["hidden"]' in src
    assert '"parallelism": f"replicas x{args.gpus}", "l2": L2_NOTE' in src
    assert "ms_per_step_extrapolated" in src and "ms_per_step_measured_sample" in src
    src_j = inspect.getsource(bench.json_line)
    assert '"config": {"workload": cfg["workload"], "tokens": tokens, "hidden": cfg["hidden"]' in src_j
    assert '"parallelism": f"replicas x{world}", "l2": L2_NOTE' in src_j


def test_clock_record_parsing():
    out = ("2026/01/01 00:00:00.000, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active\n"
           "2026/01/01 00:00:00.020, 1500, 1965, 999.0, 0x4, Not Active, Not Active, Not Active, Active\n"
           "2026/01/01 00:00:00.040, 1700, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n")
    c = bench.parse_clocks(out)
    assert c["sm_mhz"] == 1700 and c["sm_max_mhz"] == 1965 and c["sm_mhz_min"] == 1500
    assert c["reasons"] == ["sw_power_cap"] and c["samples"] == 3 and c["power_w_max"] == 999.0


@pytest.mark.parametrize("name", ["c2", "c3"])
def test_cpu_stack_runs_on_a_tiny_sample(name):
    """The oracle's stack (the CPU baseline and the reference arm) on two
    tokens and a sliver of the weights, on one thread and on two: the same
    step, and positive times."""
    c = bench.CpuStack(name, 2, 1 / 64)
    for T in (1, 2):
        tn, tg = c.step(T)
        assert tn > 0 and tg > 0
        assert c.full_step_s(tn, tg) > tn + tg


def _recording_stack(cls):
    st = object.__new__(cls)
    st.sq = RecordingSQ()
    st.bank = None
    st.by_phase = False
    return st


def _t(*shape, es=2):
    t = mock.MagicMock()
    t.shape = shape
    t.element_size.return_value = es
    n = 1
    for s in shape:
        n *= s
    t.numel.return_value = n
    t.view.return_value = t
    return t


def test_fp8_stack_launch_claim():
    """The FP8 stack: one E4M3 quantisation per smoothed side and the four
    E4M3 GEMMs, each one kernel."""
    st = _recording_stack(bench.Fp8Stack)
    st.M, st.K = 8, 16
    st.gemms = bench.CONFIGS["c5"]["gemms"]
    st.W = {w: _t(32, 16, es=4) for w, _ in st.gemms}
    st.base = types.SimpleNamespace(h={"attn": _t(8, 16), "mlp": _t(8, 16)})
    st.s = {"attn": _t(16), "mlp": _t(16)}
    st.Xq = {k: _t(8, 16, es=1) for k in ("attn", "mlp")}
    st.qx = {k: _t(8, es=4) for k in ("attn", "mlp")}
    st.syn = {w: (_t(8, 16, es=1), _t(8, es=4)) for w, src in st.gemms if src == "syn"}
    st.Y = {w: _t(8, 32) for w, _ in st.gemms}
    st.Wq = {w: _t(32, 16, es=1) for w, _ in st.gemms}
    st.qw = {w: _t(32, es=4) for w, _ in st.gemms}
    st.ws = {w: _t(256, es=1) for w, _ in st.gemms}
    bench.Fp8Stack.step(st)
    c = st.sq.calls
    assert c.count("sq_quantize_act_fp8") == 2 and c.count("sq_gemm_fp8") == 4
    assert len(c) == bench.Fp8Stack.launches_per_step(st)


def test_attention_stack_launch_claim():
    """The attention products: int8 of Q, K and V^T and the two batched
    GEMMs, each one kernel."""
    st = _recording_stack(bench.AttnStack)
    H, T, d = 2, 32, 16
    st.H, st.T, st.dh = H, T, d
    for k in ("Q", "Kt"):
        setattr(st, k, _t(H * T, d))
    st.Vt = _t(H * d, T)
    for k in ("Qq", "Kq", "Vq", "Pq", "qq", "qk", "qv", "qp", "S", "O", "ws1", "ws2"):
        setattr(st, k, _t(4))

    class Bank:
        def __init__(self):
            self.pairs = []

        def pair(self, tag, work):
            self.pairs.append((tag, work))
            return mock.MagicMock(), mock.MagicMock()

    st.bank = Bank()
    bench.AttnStack.step(st)
    c = st.sq.calls
    assert c.count("sq_quantize_act") == 3 and c.count("sq_bmm_w8a8") == 2
    assert len(c) == bench.AttnStack.launches_per_step(st)
    tags = dict(st.bank.pairs)
    # both products judged by their bytes: S written in bf16, P read in int8
    assert tags["bmm_qk"] == ("hbm", H * (2 * T * d + 2 * T * T + 8 * T))
    assert tags["bmm_pv"] == ("hbm", H * (T * T + d * T + 2 * T * d + 4 * (T + d)))
