"""The multi-rank logic of bench.py on CPU: gloo, world size 2 (no GPU)."""

import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    # rank r took (1 + r) ms per step and (5 - r) ms end to end
    ms, e2e = bench.max_over_ranks([1.0 + rank, 5.0 - rank], world, "cpu")
    q.put((rank, ms, e2e, bench.whole_job_rate(4, world, ms)))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, e2e, rate in res:
        assert ms == 2.0 and e2e == 5.0  # the slowest rank sets both times
        assert rate == pytest.approx(2 * 4 / 2e-3)  # 8 queries in 2 ms


def test_reference_arm_runs_on_rank_zero_only():
    # a non-zero rank of the reference arm exits at once without touching the oracle
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_prefill_cpu_baseline_on_a_small_host_bundle():
    # the prefill line's oracle leg, on inputs drawn by the device generator on the CPU
    from types import SimpleNamespace

    sys.path.insert(0, ROOT)
    import bench
    from synth import inputs as synth

    d = synth.prefill_inputs_device(512, 300, 4, 64, 16, seed=3, device="cpu")
    r = bench.prefill_cpu_baseline(d, SimpleNamespace(k=64, seed=3), nrows=12)
    assert r["kind"] == "oracle" and r["unit"] == "tokens/s" and r["value"] > 0
    assert r["cores"] >= 1 and "12 query rows" in r["sample"]


def test_hca_step_bytes_of_the_128k_workload():
    # 8 sequences x (1,024 rows x 580 B + 128 window rows x 1 KB + Q and O of 64 heads x
    # 1 KB + position and length + 64 sink logits)
    sys.path.insert(0, ROOT)
    import bench
    from synth import inputs as synth

    d = synth.decode_inputs(synth.WORKLOADS[bench.HCA_ID])
    assert bench.hca_step_bytes(d) == 8 * (1024 * 580 + 128 * 1024 + 2 * 64 * 1024 + 8 + 256)
