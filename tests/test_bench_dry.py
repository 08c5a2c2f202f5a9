"""bench.py's host flow on the CPU, device objects faked (tests/fake_device.py): every mode
runs to its JSON line, and the line carries every key of the benchmark contract. The
numbers are meaningless here; a B200 run produces the real ones."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RUN = """
import sys
sys.path.insert(0, {root!r})
import tests.fake_device as fd
fd.install()
import bench
from synth import inputs as synth
bench.ClockSampler.start = lambda self: None
bench.ClockSampler.stop = lambda self: {{"sm_mhz": None, "sm_max_mhz": None, "reasons": []}}
if {small_prefill}:  # the 64K-token prefill's queries would need 8.6 GB of host memory
    synth.WORKLOADS[4] = synth.Workload("small_prefill", "prefill", B=1, m=4, H=128, H_I=64,
                                        k=1024, P=512, T=1100, seed=4)
    import torch
    real = synth.prefill_inputs_device
    synth.prefill_inputs_device = lambda *a, device="cuda", **k: {{
        key: v.to("meta") if isinstance(v, torch.Tensor) else v
        for key, v in real(*a, device="cpu", **k).items()}}
sys.argv = ["bench.py"] + {argv!r}
bench.main()
"""


# Every mode's run, by key: (bench.py arguments, whether the prefill workload is shrunk).
RUNS = {
    "default": (["--steps", "20", "--warmup", "3"], False),
    "flash": (["--workload", "flash", "--steps", "16", "--warmup", "3"], False),
    "tiny": (["--workload", "tiny", "--steps", "16", "--warmup", "3"], False),
    "hca": (["--workload", "hca", "--steps", "20", "--warmup", "3"], False),
    "prefill": (["--workload", "prefill", "--steps", "2", "--warmup", "3"], True),
    "reference": (["--impl", "reference", "--steps", "1", "--warmup", "0"], False),
}
TEST_RUNS = {"test_default_decode_line": "default", "test_hca_line": "hca",
             "test_prefill_line": "prefill", "test_reference_line": "reference"}


def _key(item):
    if item.originalname == "test_other_decode_lines":
        return item.callspec.params["mode"]
    return TEST_RUNS.get(item.originalname)


@pytest.fixture(scope="module")
def runs(request):
    """Start the runs of every selected test of this module at once (each is a separate
    process of about 2 GB); a test then waits for its own. Runs still going when the module
    ends (a test failed first under -x) are ended by their process ids."""
    keys = {_key(it) for it in request.session.items if it.module is request.module}
    procs = {}
    for k in sorted(x for x in keys if x):
        argv, small = RUNS[k]
        code = RUN.format(root=ROOT, argv=argv, small_prefill=small)
        procs[k] = subprocess.Popen([sys.executable, "-c", code], cwd=ROOT, text=True,
                                    stdout=subprocess.PIPE, stderr=subprocess.PIPE)
    yield procs
    for pr in procs.values():
        if pr.poll() is None:
            pr.kill()
            pr.communicate()


def _line(runs, key):
    out, err = runs[key].communicate(timeout=600)
    assert runs[key].returncode == 0, err[-3000:]
    lines = [ln for ln in out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out[-2000:]
    return json.loads(lines[0])


def _contract(d, cpu_baseline=True):
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "clocks", "e2e", "gpu_launches"):
        assert key in d, key
    assert "workload" in d["config"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in d["roofline"], key
    for key in ("sm_mhz", "sm_max_mhz", "reasons"):
        assert key in d["clocks"], key
    for key in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert key in d["e2e"], key
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] > 0 and d["n_gpus"] == 1
    if cpu_baseline:
        for key in ("value", "unit", "cores", "kind", "sample"):
            assert key in d["cpu_baseline"], key


def _arith(d, units_per_step, kernel_ms):
    """The line's numbers agree with one another: the rate is the step's units over its
    time, end to end too; the roofline's achieved rate is its work per launch over the
    kernel's time, and its fractions are that rate over the stated peaks."""
    approx = lambda x: pytest.approx(x, rel=1e-9)
    assert d["value"] == approx(units_per_step * d["n_gpus"] / (d["ms_per_step"] * 1e-3))
    assert d["e2e"]["value"] == approx(units_per_step * d["n_gpus"] /
                                       (d["e2e"]["ms_per_step"] * 1e-3))
    r = d["roofline"]
    assert r["frac"] == approx(r["achieved"] / r["peak"])
    assert r["frac_of_nominal"] == approx(r["achieved"] / r["nominal_peak"])
    if r["bound"] == "hbm":
        assert r["achieved"] == approx(r["algorithmic_bytes_per_launch"] / (kernel_ms * 1e-3)
                                       / 1e9)


@pytest.mark.slow
def test_default_decode_line(runs):
    d = _line(runs, "default")
    _contract(d)
    assert d["steps"] == 20
    assert d["config"]["workload"] == "csa_decode_pro_1m" and d["roofline"]["bound"] == "hbm"
    # per query: 262,144 keys of 64 B codes + 4 B scales, 64 indexer heads of 64 B codes +
    # 4 B scales + a 4 B weight, 1,024 indices out, the length
    assert d["roofline"]["algorithmic_bytes_per_launch"] == \
        4 * (262144 * 68 + 64 * (64 + 4 + 4) + 1024 * 4 + 4) == 71338000
    # and the attention: 1,024 rows of 576 B + a 4 B scale, 128 window rows of 1 KB, Q and O
    # (128 heads x 1 KB each), the indices read back, position and length, 128 sink logits
    assert d["config"]["step_algorithmic_bytes"] == 71338000 + \
        4 * (1024 * 580 + 128 * 1024 + 2 * 128 * 1024 + 1024 * 4 + 8 + 128 * 4)
    c = d["config"]
    _arith(d, c["queries_per_step_per_gpu"], c["indexer_topk_ms"])
    assert c["step_achieved_gbs"] == pytest.approx(
        c["step_algorithmic_bytes"] / (d["ms_per_step"] * 1e-3) / 1e9, rel=1e-9)


@pytest.mark.parametrize("mode,workload", [("flash", "csa_decode_flash_128k"),
                                           ("tiny", "csa_decode_8k_tiny")])
def test_other_decode_lines(runs, mode, workload):
    d = _line(runs, mode)
    _contract(d)
    assert d["config"]["workload"] == workload and d["steps"] == 16
    assert d["roofline"]["bound"] == "hbm"
    _arith(d, d["config"]["queries_per_step_per_gpu"], d["config"]["indexer_topk_ms"])


def test_hca_line(runs):
    d = _line(runs, "hca")
    _contract(d)
    assert d["config"]["workload"] == "hca_decode_128k"
    assert d["steps"] == 20  # graphs of 4 steps: exactly the steps asked for
    # the step is the attention call alone, so the kernel time is the step time
    _arith(d, d["config"]["queries_per_step_per_gpu"], d["ms_per_step"])


def test_prefill_line(runs):
    d = _line(runs, "prefill")
    _contract(d)
    assert d["roofline"]["bound"] == "tensor"
    c, r = d["config"], d["roofline"]
    _arith(d, c["new_tokens"], d["ms_per_step"])
    # FLOPs of the shrunk workload by the layer's definition, restated here per query
    P, T, m, H, H_I, k = c["prefix_tokens"], c["new_tokens"], 4, c["heads"], \
        c["indexer_heads"], c["top_k"]
    f4 = f16 = 0
    for t in range(P, P + T):
        n = (t + 1) // m
        f4 += 2 * H_I * 128 * n
        f16 += 4 * H * 512 * (min(k, n) + min(128, t + 1))
    assert c["fp4_tflop"] == pytest.approx(f4 / 1e12, rel=1e-12)
    assert c["bf16_tflop"] == pytest.approx(f16 / 1e12, rel=1e-12)
    ratio = r["mma_peak"]["fp4_over_bf16"]
    assert r["achieved"] == pytest.approx(
        (f4 / ratio + f16) / (d["ms_per_step"] * 1e-3) / 1e12, rel=1e-9)


def test_reference_line(runs):
    d = _line(runs, "reference")
    assert d["impl"] == "reference" and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_full_prefill_flops_match_the_workload_figures():
    # 65,536 new tokens after a 196,608-token prefix, m = 4, 128 heads, 64 indexer heads,
    # top-1024: sum of n(t) = 3.758e9 eligible entries, so 61.57 TFLOP of FP4 indexer work;
    # every query attends to 1,024 + 128 rows, so 128 x 1152 x 512 x 4 x 65,536 = 19.79 TFLOP
    import bench

    f4, f16 = bench.prefill_flops(196608, 65536, 4, 128, 64, 1024)
    assert f4 == pytest.approx(61.57e12, rel=1e-3)
    assert f16 == 128 * 1152 * 512 * 4 * 65536
