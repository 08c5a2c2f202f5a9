"""Benchmark of the CSA decode step at 1M context (V4-Pro-shaped layer).

One step = one decode query for each of the B = 4 sequences of the workload
(context 1,048,576 tokens -> 262,144 compressed entries, 128 heads sharing one KV of
head_dim 512, indexer 64 heads x 128 FP4 dims, top-k 1024, 128-token window, sink):
  csa_indexer_topk  (FP4 indexer scores over every entry + top-k selection)
  csa_sparse_attn_decode  (shared-KV MQA over the selected entries + window + sink)
Metric: decode queries/s (whole job). Inputs are synthetic and seeded; device copies of the
streamed inputs are rotated step by step (inside each replayed graph too) so that
consecutive steps never hit in L2. The compressed cache sits in pages of 512 entries
(2,048 tokens) behind a shuffled block table (--page-entries 0: contiguous per sequence).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                       [--workload decode|prefill|hca]
Under torchrun every rank runs its own 4-sequence batch (weak scaling, no collective on
the data path); rank 0 prints one JSON line.

--workload prefill times csa_prefill instead: 65,536 new tokens after a 196,608-token
prefix (one sequence, 128 heads, indexer 64 heads, top-k 1024); one step is the whole
prefill call (compression, indexer top-k and attention for every new token).
--workload hca times hca_attn_decode: 8 sequences at 128K context (1,024 entries each,
64 heads), dense MQA over every entry + window + sink, graphs over 24 device copies.
--workload flash times the same CSA decode step as the default on the V4-Flash-shaped
workload (32 sequences of 64K-128K tokens, 64 heads, indexer 64 heads, top-k 512), and
--workload tiny on one 8K-token sequence (64 heads, indexer 16 heads, top-k 512); each
rotates over enough device copies that one rotation exceeds twice the L2.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

WORKLOAD_ID = 3
METRIC = "CSA decode queries/s at 1M ctx; achieved HBM GB/s as % of B200 peak"
UNIT = "queries/s"
COPIES = 4
# nominal B200 figures, reported beside the measured peaks: HBM3e bandwidth (HGX) and dense
# BF16 tensor throughput
NOMINAL_HBM_GBS = 7700.0
NOMINAL_BF16_TFLOPS = 2250.0


def algorithmic_bytes(d: dict) -> tuple[int, int]:
    """(indexer_topk bytes per call, whole decode step bytes) by the layer's definition:
    per query 68 B per eligible entry (64 B E2M1 key + 4 B E8M0 scales), the FP4 query
    (H_I x 68 B) and weights, the k selected rows of 580 B (576 B + fp32 scale), 128 window
    rows of 1 KB, Q and O (H x 1 KB each), the indices and positions."""
    w = d["workload"]
    n = d["n_entries"].astype(np.int64)
    idx = int((n * 68).sum() + d["B"] * (w.H_I * 72 + w.k * 4 + 4))
    attn = d["B"] * (w.k * 580 + 128 * 1024 + 2 * w.H * 1024 + w.k * 4 + 8 + w.H * 4)
    return idx, idx + attn


def peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "src": "measured"}
    return {"hbm_gbs": 6650.0, "src": "fallback"}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the GPU is busy."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        mhz, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) != 6:
                continue
            try:
                mhz.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for nm, v in zip(names, f[2:]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(mhz) if mhz else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(mhz)}


def ncu_traffic() -> dict | None:
    """DRAM bytes per launch of the indexer call from the committed ncu summary, if it was
    taken on the current sources of that kernel."""
    p = os.path.join(ROOT, "profiles", "indexer_topk_csa_decode_pro_1m.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    from long_context_compressed_layer_b200 import build as b
    if d.get("sources_sha") != b.sources_sha(d.get("sources")):
        return None
    return d


PREFILL_ID = 4
PREFILL_METRIC = "CSA prefill tokens/s (65,536 new tokens after a 196,608-token prefix)"


def prefill_flops(P: int, T: int, m: int, H: int, H_I: int, k: int) -> tuple[int, int]:
    """(FP4 indexer FLOPs, BF16/FP16 attention FLOPs) of one prefill by the layer's
    definition: every query scores its n(t) = floor((t+1)/m) eligible entries with H_I heads
    of 128 dims; attention forms S = Q V^T and O = P V over min(k, n(t)) entries + the
    window rows (at most 128) for H heads of 512 dims."""
    t = P + np.arange(T, dtype=np.int64)
    n = (t + 1) // m
    rows = np.minimum(k, n) + np.minimum(128, t + 1)
    return int(2 * H_I * 128 * n.sum()), int(4 * H * 512 * rows.sum())


def capture_graph(torch, warm, body):
    """A CUDA graph of `body`, captured on a side stream after one uncaptured `warm` call
    (which fills the library's tensor-map and attribute caches)."""
    g = torch.cuda.CUDAGraph()
    s_cap = torch.cuda.Stream()
    s_cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s_cap):
        warm()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s_cap):
            body()
    torch.cuda.current_stream().wait_stream(s_cap)
    torch.cuda.synchronize()
    return g


def rotation_graphs(torch, step, copies, reps):
    """CUDA graphs of `reps` steps each in which the global step s runs on device copy
    copies[s % len(copies)], so that no two consecutive steps read the same copy; replaying
    the returned graphs round robin continues that sequence."""
    n = len(copies)
    graphs = []
    for gi in range(n // math.gcd(n, reps)):
        seq = [copies[(gi * reps + j) % n] for j in range(reps)]
        graphs.append(capture_graph(torch, lambda seq=seq: step(seq[0]),
                                    lambda seq=seq: [step(c) for c in seq]))
    return graphs


def packed(torch, specs: dict, host: bool):
    """One byte buffer (pinned host memory, or device memory) holding a tensor per entry of
    `specs` (name -> (shape, dtype)) at 256-byte aligned offsets: (buffer, {name: view})."""
    offs, off = {}, 0
    for key, (shape, dtype) in specs.items():
        nbytes = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
        offs[key] = (off, nbytes)
        off += -(-nbytes // 256) * 256
    if host:
        buf = torch.empty(off, dtype=torch.uint8, pin_memory=True)
    else:
        buf = torch.empty(off, dtype=torch.uint8, device="cuda")
    return buf, {key: buf[o:o + nb].view(specs[key][1]).view(specs[key][0])
                 for key, (o, nb) in offs.items()}


def e2e_graphs(torch, launch, copies, inputs: dict, out_specs: dict, reps):
    """CUDA graphs of `reps` end-to-end steps each, pipelined across steps. Step j uploads
    its query-side inputs (`inputs`, host tensors, packed into one pinned buffer) in one copy
    into device slot j % 2 on an upload stream, runs its kernels on the capture stream once
    that copy is done (launch(copy, device input views, device output views)), and
    downloads its packed outputs to pinned host memory in one copy on a download stream.
    Slot reuse waits on events: an upload waits for the kernels two steps back, and kernels
    wait for the download two steps back. Device copies rotate as in rotation_graphs.
    Returns (graphs, h2d bytes per step, d2h bytes per step, host output views)."""
    in_specs = {key: (tuple(v.shape), v.dtype) for key, v in inputs.items()}
    h_in, h_in_v = packed(torch, in_specs, True)
    for key, v in inputs.items():
        h_in_v[key].copy_(v)
    d_in = [packed(torch, in_specs, False) for _ in range(2)]
    d_out = [packed(torch, out_specs, False) for _ in range(2)]
    h_out, h_out_v = packed(torch, out_specs, True)
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    n = len(copies)

    def body(seq):
        comp = torch.cuda.current_stream()
        up.wait_stream(comp)
        down.wait_stream(comp)
        done, fetched = [], []
        for j, c in enumerate(seq):
            s = j % 2
            with torch.cuda.stream(up):
                if j >= 2:
                    up.wait_event(done[j - 2])
                d_in[s][0].copy_(h_in, non_blocking=True)
                e_up = torch.cuda.Event()
                e_up.record(up)
            comp.wait_event(e_up)
            if j >= 2:
                comp.wait_event(fetched[j - 2])
            launch(c, d_in[s][1], d_out[s][1])
            e_done = torch.cuda.Event()
            e_done.record(comp)
            done.append(e_done)
            with torch.cuda.stream(down):
                down.wait_event(e_done)
                h_out.copy_(d_out[s][0], non_blocking=True)
                e_f = torch.cuda.Event()
                e_f.record(down)
                fetched.append(e_f)
        comp.wait_stream(up)
        comp.wait_stream(down)

    graphs = []
    for gi in range(n // math.gcd(n, reps)):
        seq = [copies[(gi * reps + j) % n] for j in range(reps)]
        graphs.append(capture_graph(torch, lambda seq=seq: launch(seq[0], d_in[0][1], d_out[0][1]),
                                    lambda seq=seq: body(seq)))
    return graphs, h_in.numel(), h_out.numel(), h_out_v


def fp4_bf16_mma_rates(torch, csa, stream, iters: int = 20000) -> dict:
    """Rates (TFLOP/s) of csa_mma_peak's back-to-back MMA loops, BF16 at N = 64 and 256 and
    MXFP4 at N = 64, each timed with CUDA events after a warm-up launch, and the FP4 / BF16
    ratio at the common shape N = 64."""
    out = {}
    for name, kind, N in (("bf16_n64", 1, 64), ("bf16_n256", 1, 256), ("mxf4_n64", 0, 64)):
        csa.mma_peak(kind, N, iters)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        flops = sum(csa.mma_peak(kind, N, iters) for _ in range(5))
        e1.record(stream)
        torch.cuda.synchronize()
        out[name] = flops / (e0.elapsed_time(e1) * 1e-3) / 1e12
    out["fp4_over_bf16"] = out["mxf4_n64"] / out["bf16_n64"]
    return out


def max_over_ranks(vals: list[float], world: int, device) -> list[float]:
    """Per-rank timings -> their maxima over all ranks (one all-reduce of a few floats,
    outside the data path)."""
    if world <= 1:
        return list(vals)
    import torch
    import torch.distributed as dist
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def whole_job_rate(units_per_rank: int, world: int, ms: float) -> float:
    """Units processed by all ranks per second, from the slowest rank's time."""
    return world * units_per_rank / (ms * 1e-3)


def bench_prefill(args, rank: int, world: int, local: int) -> None:
    import torch

    import long_context_compressed_layer_b200 as csa
    from synth import inputs as synth

    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    w = synth.WORKLOADS[PREFILL_ID]
    d = synth.prefill_inputs_device(w.P, w.T, w.m, w.H, w.H_I, seed=w.seed + 1000 * rank)
    T, k = w.T, w.k
    kv0 = d["kv"].clone()
    ws = csa.prefill_workspace(T, d["Nmax"], w.H, k)
    out = torch.empty((T, w.H, 512), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    bf = lambda x: x.view(torch.bfloat16) if x.dtype == torch.int16 else x

    def step():
        csa.prefill(w.P, w.m, k, a=d["a"], b=d["b"], za=d["za"], zb=d["zb"], bias=d["bias"],
                    kv=d["kv"], kv_scale=d["kv_scale"], q_fp4=d["q_fp4"], q_sf=d["q_sf"],
                    w=d["w"], k_fp4=d["k_fp4"], k_sf=d["k_sf"], q=d["q"], sink=d["sink"],
                    prev_b=d["prev_b"], prev_zb=d["prev_zb"], swa_prefix=d["swa_prefix"],
                    workspace=ws, out=out, dev_status=status)

    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1) / args.steps
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during the benchmark")

    # the indexer keys of the new blocks (csa_compress_index_keys over the 65,536 new
    # tokens -> 16,384 MXFP4 keys): an HBM stream of 6,144 bytes read and 68 written per key
    ik_fp4 = torch.zeros((1, d["Nmax"], 64), dtype=torch.uint8, device="cuda")
    ik_sf = torch.zeros((1, d["Nmax"] // 128 * 512), dtype=torch.uint8, device="cuda")

    def ikeys():
        csa.compress_index_keys(d["ia"][None], d["iza"][None], d["ibias"], w.m, True,
                                b=d["ib"][None], zb=d["izb"][None], pos0=w.P,
                                prev_b=d["iprev_b"][None], prev_zb=d["iprev_zb"][None],
                                k_fp4=ik_fp4, k_sf=ik_sf)

    for _ in range(3):
        ikeys()
    k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    k0.record(stream)
    for _ in range(20):
        ikeys()
    k1.record(stream)
    torch.cuda.synchronize()
    ik_ms = k0.elapsed_time(k1) / 20
    n_keys = T // w.m
    ik_bytes = n_keys * (2 * w.m * 128 * 6 + 68)
    hbm = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["hbm_gbs"] if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else 6650.0

    # the indexer queries of the new tokens (csa_indexer_query: a [65,536 x 1536] x
    # [1536 x 8192] BF16 product quantised to MXFP4 per head), timed alone
    g = torch.Generator(device="cuda")
    g.manual_seed(w.seed + 17)
    rq = 1536
    cq = torch.randn((T, rq), generator=g, device="cuda").to(torch.bfloat16)
    Wq = (torch.randn((w.H_I * 128, rq), generator=g, device="cuda") * rq ** -0.5).to(
        torch.bfloat16)
    qf_out = torch.empty((T, w.H_I, 64), dtype=torch.uint8, device="cuda")
    qs_out = torch.empty((T, w.H_I, 4), dtype=torch.uint8, device="cuda")
    for _ in range(3):
        csa.indexer_query(cq, Wq, w.H_I, q_fp4=qf_out, q_sf=qs_out)
    k0.record(stream)
    for _ in range(10):
        csa.indexer_query(cq, Wq, w.H_I, q_fp4=qf_out, q_sf=qs_out)
    k1.record(stream)
    torch.cuda.synchronize()
    iq_ms = k0.elapsed_time(k1) / 10
    iq_flop = 2 * T * rq * w.H_I * 128
    peaks_file = os.path.join(ROOT, "MEASURED_PEAKS.json")
    pkd = json.load(open(peaks_file)) if os.path.exists(peaks_file) else {}
    bf16_burst = pkd.get("bf16_tflops", 1590.0)  # a kernel timed alone: the burst figure
    del cq, Wq

    # the grouped output projection of the prefill's attention output (16 groups of 8
    # heads reduced to 1024 each, then 16,384 -> 7168), timed alone
    G, d_g, d_model = 16, 1024, 7168
    K1 = w.H // G * 512
    Wg = (torch.randn((G, d_g, K1), generator=g, device="cuda") * K1 ** -0.5).to(torch.bfloat16)
    Wo = (torch.randn((d_model, G * d_g), generator=g, device="cuda") * (G * d_g) ** -0.5).to(
        torch.bfloat16)
    op_out = torch.empty((T, d_model), dtype=torch.bfloat16, device="cuda")
    op_ws = torch.empty(T * G * d_g * 2 + 256, dtype=torch.uint8, device="cuda")
    csa.grouped_out_proj(out, Wg, Wo, workspace=op_ws, out=op_out)
    k0.record(stream)
    for _ in range(3):
        csa.grouped_out_proj(out, Wg, Wo, workspace=op_ws, out=op_out)
    k1.record(stream)
    torch.cuda.synchronize()
    op_ms = k0.elapsed_time(k1) / 3
    op_flop = 2 * T * (G * d_g * K1 + d_model * G * d_g)
    del Wg, Wo, op_out, op_ws

    # the tensor pipes' FP4 / BF16 rate ratio at one MMA shape (csa_mma_peak: back-to-back
    # MMAs on shared-memory operands, M = 128, N = 64), which scales the measured BF16 GEMM
    # peak into the FP4 peak of the roofline below
    mma_rates = fp4_bf16_mma_rates(torch, csa, stream)

    # end to end: the new tokens' inputs go up from pinned host memory and the output
    # comes back, around the same call
    up = ("a", "b", "za", "zb", "q", "q_fp4", "q_sf", "w")
    pinned = {x: d[x].cpu().pin_memory() for x in up}
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = out_h.numel() * out_h.element_size()
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(stream)
    for _ in range(args.steps):
        for x in up:
            d[x].copy_(pinned[x], non_blocking=True)
        step()
        out_h.copy_(out, non_blocking=True)
    x1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = x0.elapsed_time(x1) / args.steps
    d["kv"].copy_(kv0)
    ms, e2e_ms = max_over_ranks([ms, e2e_ms], world, "cuda")
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    f4, f16 = prefill_flops(w.P, T, w.m, w.H, w.H_I, k)
    pk = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    bf16_peak = pk.get("bf16_tflops_sustained", 1400.0)  # a long step: the sustained figure
    # FP4 FLOPs weighted by the measured BF16 / FP4 tensor-rate ratio (1/4 nominally)
    fp4_ratio = mma_rates["fp4_over_bf16"]
    eq_tflops = (f4 / fp4_ratio + f16) / (ms * 1e-3) / 1e12
    line = {
        "metric": PREFILL_METRIC, "value": whole_job_rate(T, world, ms), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp4+fp16", "data": "synthetic",
        "config": {"workload": w.name, "prefix_tokens": w.P, "new_tokens": T, "heads": w.H,
                   "indexer_heads": w.H_I, "top_k": k, "window": 128,
                   "l2": "inputs larger than L2 (8.6 GB of queries)",
                   "fp4_tflop": f4 / 1e12, "bf16_tflop": f16 / 1e12,
                   "index_key_compress": {"ms": ik_ms, "keys": n_keys,
                                          "algorithmic_bytes": ik_bytes,
                                          "gbs": ik_bytes / (ik_ms * 1e-3) / 1e9,
                                          "frac_of_hbm": ik_bytes / (ik_ms * 1e-3) / 1e9 / hbm},
                   "index_query": {"ms": iq_ms, "latent_dim": rq, "tflop": iq_flop / 1e12,
                                   "tflops": iq_flop / (iq_ms * 1e-3) / 1e12,
                                   "frac_of_bf16_burst": iq_flop / (iq_ms * 1e-3) / 1e12
                                   / bf16_burst},
                   "grouped_out_proj": {"ms": op_ms, "groups": G, "group_rank": d_g,
                                        "d_model": d_model, "tflop": op_flop / 1e12,
                                        "tflops": op_flop / (op_ms * 1e-3) / 1e12,
                                        "frac_of_bf16_burst": op_flop / (op_ms * 1e-3) / 1e12
                                        / bf16_burst}},
        "roofline": {"bound": "tensor", "kernel": "csa_prefill (whole call)",
                     "achieved": eq_tflops, "peak": bf16_peak, "unit": "TFLOP/s",
                     "frac": eq_tflops / bf16_peak,
                     "nominal_peak": NOMINAL_BF16_TFLOPS,
                     "frac_of_nominal": eq_tflops / NOMINAL_BF16_TFLOPS,
                     "peak_src": (f"measured sustained bf16; FP4 FLOPs weighted 1/{fp4_ratio:.2f} "
                                  "(FP4 / BF16 tensor-rate ratio measured by csa_mma_peak)"
                                  if "bf16_tflops_sustained" in pk else "fallback"),
                     "fp4_peak_tflops": bf16_peak * fp4_ratio,
                     "mma_peak": mma_rates,
                     "traffic": None},
        "clocks": clocks,
        "e2e": {"value": whole_job_rate(T, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        # per call: compression of the new blocks, the window-row prep, the FP16 entry rows,
        # then per 1024 queries the scoring, selection and attention kernels
        "gpu_launches": args.steps * ((1 if T // w.m else 0) + 1 + (1 if (w.P + T) // w.m else 0)
                                      + 3 * (-(-T // 1024))),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = prefill_cpu_baseline(d, w)
    print(json.dumps(line), flush=True)


def prefill_cpu_baseline(d: dict, w, nrows: int = 128) -> dict:
    """The oracle timed on a bounded sample of one prefill (inputs as drawn on the device,
    copied to the host): its compression of every new block, then `nrows` query rows (the
    first tokens, the edges of the 1024-query chunks, the last token and seeded random
    ones). Tokens/s is extrapolated from the two times: T / (t_compress + T * t_row)."""
    import torch

    import oracle

    T = d["T"]
    fixed = [r for r in (0, 1, 2, 3, 1023, 1024, T - 1) if r < T]
    rng = np.random.default_rng(w.seed)
    extra = rng.choice(T, min(T, max(0, nrows - len(fixed))), replace=False)
    rows = np.unique(np.concatenate([fixed, extra]).astype(np.int32))[:nrows]

    def host(x):
        x = x.cpu().numpy()
        return x.view(np.uint16) if x.dtype == np.int16 else x

    inp = {key: d[key] for key in ("P", "T", "m", "H", "H_I", "Nmax")}
    for key in ("kv", "kv_scale", "k_fp4", "k_sf", "q_fp4", "q_sf", "w", "sink", "swa_prefix",
                "a", "b", "za", "zb", "bias", "prev_b", "prev_zb"):
        if key in d:
            inp[key] = host(d[key])
    q = np.zeros(tuple(d["q"].shape), dtype=np.uint16)  # only the sampled rows are read
    q[rows] = host(d["q"].index_select(0, torch.as_tensor(rows, dtype=torch.long,
                                                          device=d["q"].device)))
    inp["q"] = q
    t0 = time.perf_counter()
    oracle.prefill(inp, w.k, np.zeros(0, np.int32))
    t1 = time.perf_counter()
    oracle.prefill(inp, w.k, rows)
    t2 = time.perf_counter()
    t_comp = t1 - t0
    t_row = max(0.0, (t2 - t1) - t_comp) / len(rows)
    return {"value": T / (t_comp + T * t_row), "unit": "tokens/s", "cores": os.cpu_count() or 1,
            "kind": "oracle",
            "sample": f"compression of all {T // d['m']} new blocks ({t_comp:.1f} s) and "
                      f"{len(rows)} query rows ({t2 - t1 - t_comp:.1f} s), fp64, all host "
                      "threads; tokens/s extrapolated per query row"}


HCA_ID = 1
HCA_METRIC = "HCA decode queries/s (8 sequences at 128K context, 1,024 entries each)"
HCA_COPIES = 24  # 24 x 6.3 MB of streamed inputs: more than L2 across the rotation


def hca_step_bytes(d: dict) -> int:
    """Algorithmic bytes of one HCA decode step: per sequence every eligible row of 580 B
    (576 B + fp32 scale), 128 window rows of 1 KB, Q and O (H x 1 KB each), the position
    and length, and the H sink logits."""
    H = d["workload"].H
    n = d["n_entries"].astype(np.int64)
    return int((n * 580).sum() + d["B"] * (128 * 1024 + 2 * H * 1024 + 8 + H * 4))


def bench_hca(args, rank: int, world: int, local: int) -> None:
    """The HCA decode (hca_attn_decode) of the 128K-context workload, replayed from CUDA
    graphs over device copies of its inputs; roofline against the measured HBM copy rate."""
    import torch

    import long_context_compressed_layer_b200 as csa
    from synth import inputs as synth

    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    w = synth.WORKLOADS[HCA_ID]
    d = synth.decode_inputs(w, seed=w.seed + 1000 * rank)
    B, Nmax = d["B"], d["Nmax"]

    def dev(x):
        x = np.ascontiguousarray(x)
        return torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x).cuda()

    streamed = ("kv", "kv_scale", "q", "swa")
    base = {key: dev(d[key]) for key in streamed + ("n_entries", "pos", "sink")}
    copies = [base] + [{key: (base[key].clone() if key in streamed else base[key])
                        for key in base} for _ in range(HCA_COPIES - 1)]
    ws = csa.attn_workspace(B, w.H, Nmax + 128)
    out = torch.empty((B, w.H, 512), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def step(c):
        csa.hca_attn_decode(c["q"], c["pos"], c["n_entries"], c["kv"], c["kv_scale"], c["swa"],
                            c["sink"], workspace=ws, out=out, dev_status=status)

    graph_steps = next(g for g in (8, 4, 2, 1) if args.steps % g == 0)  # exactly --steps

    def timed(graphs, n, per_graph=graph_steps):
        for i in range(max(3, 2 * len(graphs))):  # warm-up replays
            graphs[i % len(graphs)].replay()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n):
            graphs[i % len(graphs)].replay()
        e1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return e0.elapsed_time(e1) / (n * per_graph)

    # every step of a graph moves to the next device copy of the inputs
    graphs = rotation_graphs(torch, step, copies, graph_steps)
    replays = max(1, (args.steps + graph_steps - 1) // graph_steps)
    sampler = ClockSampler(local)
    sampler.start()
    ms = timed(graphs, replays)
    clocks = sampler.stop()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during the benchmark")

    # end to end: every step uploads its queries, positions and lengths from pinned host
    # memory (one packed copy) and downloads its output (one copy), on copy streams that
    # overlap the neighbouring steps' kernels
    q_inputs = ("q", "pos", "n_entries")

    def e2e_launch(c, din, dout):
        csa.hca_attn_decode(din["q"], din["pos"], din["n_entries"], c["kv"], c["kv_scale"],
                            c["swa"], c["sink"], workspace=ws, out=dout["out"],
                            dev_status=status)

    e2e_steps = 24
    e2e_g, h2d, d2h, h_out = e2e_graphs(torch, e2e_launch, copies,
                                         {key: base[key].cpu() for key in q_inputs},
                                         {"out": (tuple(out.shape), out.dtype)}, e2e_steps)
    e2e_ms = timed(e2e_g, max(len(e2e_g), min(replays, 64)), e2e_steps)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the end-to-end run")
    if not torch.equal(h_out["out"], out.cpu()):
        raise RuntimeError("end-to-end output differs from the device-resident call's")
    ms, e2e_ms = max_over_ranks([ms, e2e_ms], world, "cuda")
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    pk = peaks()
    step_bytes = hca_step_bytes(d)
    streamed_bytes = sum(base[key].numel() * base[key].element_size() for key in streamed)
    achieved = step_bytes / (ms * 1e-3) / 1e9
    line = {
        "metric": HCA_METRIC, "value": whole_job_rate(B, world, ms), "unit": UNIT,
        "n_gpus": world, "steps": replays * graph_steps, "warmup": max(3, 2 * len(graphs)) * graph_steps,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp16", "data": "synthetic",
        "config": {"workload": w.name, "queries_per_step_per_gpu": B, "context": w.L,
                   "entries_per_seq": int(d["n_entries"][0]), "heads": w.H, "window": 128,
                   "l2": f"inputs rotated over {HCA_COPIES} device copies "
                         f"({HCA_COPIES * streamed_bytes / 1e6:.0f} MB of streamed inputs)",
                   "launch": f"CUDA graphs of {graph_steps} steps, programmatic dependent launch",
                   "e2e_launch": f"CUDA graphs of {e2e_steps} steps; one packed upload and one "
                                 "download per step on two copy streams, device inputs and "
                                 "outputs double-buffered"},
        "roofline": {"bound": "hbm", "kernel": "hca_attn_decode (chunk + combine kernels)",
                     "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"], "peak_src": pk["src"],
                     "nominal_peak": NOMINAL_HBM_GBS,
                     "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                     "algorithmic_bytes_per_launch": step_bytes, "traffic": None},
        "clocks": clocks,
        "e2e": {"value": whole_job_rate(B, world, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": 2 * replays * graph_steps,
    }
    if world == 1 and not args.no_cpu_baseline:
        import oracle

        t0 = time.perf_counter()
        oracle.attention(d["q"], d["pos"], d["n_entries"], d["kv"], d["kv_scale"], d["swa"],
                         d["sink"])
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": B / dt, "unit": UNIT, "cores": os.cpu_count() or 1,
                                "kind": "oracle",
                                "sample": f"one whole step ({B} queries), fp64, all host threads"}
    print(json.dumps(line), flush=True)


def run_reference(args, rank: int) -> None:
    """The fp64 CPU oracle, as it stands, on the host cores: each step is one decode query
    (one sequence of the workload: indexer over 262,144 entries, top-k, attention)."""
    if rank != 0:
        return
    import oracle
    from synth import inputs as synth

    w = synth.WORKLOADS[WORKLOAD_ID]
    d = synth.decode_inputs(w, B=1)
    cores = os.cpu_count() or 1

    def step():
        s = oracle.indexer_scores(d["n_entries"], d["q_fp4"], d["q_sf"], d["w"], d["k_fp4"],
                                  d["k_sf"])
        idx = oracle.topk(s[0], int(d["n_entries"][0]), w.k)[None]
        oracle.attention(d["q"], d["pos"], d["n_entries"], d["kv"], d["kv_scale"], d["swa"],
                         d["sink"], idx=idx)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    v = args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "queries_per_step": 1, "context": w.L, "heads": w.H,
                   "indexer_heads": w.H_I, "top_k": w.k, "l2": "host run"},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": "one decode query (one sequence of the workload) per step"},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline_sample(d_host, w) -> dict:
    """The oracle timed on a bounded sample: 2 decode queries of the workload."""
    import oracle
    cores = os.cpu_count() or 1
    q = min(2, d_host["B"])
    t0 = time.perf_counter()
    for b in range(q):
        sl = slice(b, b + 1)
        s = oracle.indexer_scores(d_host["n_entries"][sl], d_host["q_fp4"][sl],
                                  d_host["q_sf"][sl], d_host["w"][sl], d_host["k_fp4"][sl],
                                  d_host["k_sf"][sl])
        idx = oracle.topk(s[0], int(d_host["n_entries"][b]), w.k)[None]
        oracle.attention(d_host["q"][sl], d_host["pos"][sl], d_host["n_entries"][sl],
                         d_host["kv"][sl], d_host["kv_scale"][sl], d_host["swa"][sl],
                         d_host["sink"], idx=idx)
    dt = time.perf_counter() - t0
    return {"value": q / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{q} decode queries (the first sequences of the workload), fp64, all "
                      "host threads"}


# CSA decode workloads timed like the default one: the workload index in synth.WORKLOADS
# and the metric name of its line
DECODE_MODES = {
    "decode": (WORKLOAD_ID, METRIC),
    "flash": (2, "CSA decode queries/s (V4-Flash-shaped: 32 sequences of 64K-128K tokens)"),
    "tiny": (0, "CSA decode queries/s (one sequence of 8K tokens, 64 heads, k = 512)"),
}
L2_BYTES = 126 << 20


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 20000 for decode modes, 5 for prefill)")
    ap.add_argument("--warmup", type=int, default=None,
                    help="untimed steps first (default 500 for decode modes, 3 for prefill)")
    ap.add_argument("--impl", default="csa", choices=["csa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--copies", type=int, default=0,
                    help="device copies of the streamed inputs rotated across steps "
                         "(0: enough that one rotation exceeds twice the L2)")
    ap.add_argument("--workload", default="decode",
                    choices=sorted(DECODE_MODES) + ["prefill", "hca"])
    ap.add_argument("--page-entries", type=int, default=512,
                    help="decode modes: compressed cache in pages of this many entries "
                         "behind a shuffled block table (0: contiguous per sequence)")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = 5 if args.workload == "prefill" else 20000
    if args.warmup is None:
        args.warmup = 3 if args.workload == "prefill" else 500

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.workload == "prefill":
        bench_prefill(args, rank, world, local)
        return
    if args.workload == "hca":
        bench_hca(args, rank, world, local)
        return

    import torch
    import torch.distributed as dist

    import long_context_compressed_layer_b200 as csa
    from synth import inputs as synth

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    wid, metric = DECODE_MODES[args.workload]
    w = synth.WORKLOADS[wid]
    d = synth.decode_inputs(w, seed=w.seed + 1000 * rank)
    B, k, Nmax = d["B"], w.k, d["Nmax"]

    def dev(x):
        x = np.ascontiguousarray(x)
        return torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x).cuda()

    # the compressed cache (entries and indexer keys) in pages of P entries behind a
    # shuffled block table, as a serving cache holds it; the oracle keeps the contiguous d
    P = args.page_entries
    dd, paging, cache_cfg = d, None, {"layout": "contiguous per sequence"}
    if P:
        table, num_pages = synth.page_table(np.random.default_rng(w.seed + 77), B, -(-Nmax // P))
        dd = dict(d)
        dd["k_fp4"] = synth.place_in_pages(d["k_fp4"], table, P, num_pages)
        dd["k_sf"] = synth.place_in_pages(d["k_sf"].reshape(B, Nmax // 128, 512), table, P,
                                          num_pages, group=128)
        dd["kv"] = synth.place_in_pages(d["kv"], table, P, num_pages)
        dd["kv_scale"] = synth.place_in_pages(d["kv_scale"], table, P, num_pages)
        paging = csa.Paging(dev(table), P, Nmax)
        cache_cfg = {"layout": "paged", "page_entries": P, "page_tokens": P * w.m,
                     "block_table": "shuffled", "pool_pages": num_pages}

    streamed = ("k_fp4", "k_sf", "kv", "kv_scale", "q_fp4", "q_sf", "w", "q", "swa")
    base = {key: dev(dd[key]) for key in streamed + ("n_entries", "pos", "sink")}
    copy_bytes = sum(base[key].numel() * base[key].element_size() for key in streamed)
    ncopy = args.copies if args.copies > 0 else min(512, max(COPIES, -(-2 * L2_BYTES // copy_bytes)))
    copies = [base] + [{key: (base[key].clone() if key in streamed else base[key])
                        for key in base} for _ in range(ncopy - 1)]
    ws_idx = csa.indexer_topk_workspace(B, Nmax, k)
    ws_att = csa.attn_workspace(B, w.H, k + 128)
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    out = torch.empty((B, w.H, 512), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def step_idx(c):
        csa.indexer_topk(c["n_entries"], c["q_fp4"], c["q_sf"], c["w"], c["k_fp4"], c["k_sf"],
                         k, workspace=ws_idx, idx=idx, dev_status=status, paging=paging)

    def step_att(c):
        csa.sparse_attn_decode(c["q"], c["pos"], c["n_entries"], c["kv"], c["kv_scale"],
                               c["swa"], c["sink"], idx, workspace=ws_att, out=out,
                               dev_status=status, paging=paging)

    def step(c):
        step_idx(c)
        step_att(c)

    # The decode step is replayed from CUDA graphs (as a serving loop would), each holding
    # GRAPH_STEPS steps that move to the next device copy of the inputs at every step.
    # Kernels launched with programmatic stream serialisation keep their programmatic edges
    # inside the graph. Graphs of 8 steps when --steps allows it, else of the largest power
    # of two dividing it, so that the timed region runs exactly --steps steps.
    GRAPH_STEPS = next(g for g in (8, 4, 2, 1) if args.steps % g == 0)
    step_graphs = rotation_graphs(torch, step, copies, GRAPH_STEPS)
    idx_graphs = rotation_graphs(torch, step_idx, copies, GRAPH_STEPS)
    att_graphs = rotation_graphs(torch, step_att, copies, GRAPH_STEPS)
    replays = max(1, (args.steps + GRAPH_STEPS - 1) // GRAPH_STEPS)
    steps_run = replays * GRAPH_STEPS

    def run_graphs(graphs, n):
        for i in range(n):
            graphs[i % len(graphs)].replay()

    sampler = ClockSampler(local)
    sampler.start()
    run_graphs(step_graphs, max(args.warmup // GRAPH_STEPS, 3))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    run_graphs(step_graphs, replays)
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = t0.elapsed_time(t1)

    # live per-call timing of each ABI call (graphs of that call alone, same rotation)
    def time_graphs(graphs, n, per_graph=GRAPH_STEPS):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        run_graphs(graphs, 2 * len(graphs))
        e0.record(stream)
        run_graphs(graphs, n)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / (n * per_graph)

    nprobe = max(4, min(replays, 256))
    t_idx = time_graphs(idx_graphs, nprobe)
    t_att = time_graphs(att_graphs, nprobe)

    # the selection on BF16-rounded index scores: its call time, and how much of the fp32
    # selection it keeps (recall) on the first device copy
    idx_bf = torch.empty_like(idx)

    def step_idx_bf(c):
        csa.indexer_topk(c["n_entries"], c["q_fp4"], c["q_sf"], c["w"], c["k_fp4"], c["k_sf"],
                         k, workspace=ws_idx, idx=idx_bf, dev_status=status, bf16_scores=True,
                         paging=paging)

    bf_graphs = rotation_graphs(torch, step_idx_bf, copies, GRAPH_STEPS)
    t_idx_bf = time_graphs(bf_graphs, nprobe)
    step_idx(copies[0])
    step_idx_bf(copies[0])
    torch.cuda.synchronize()
    a32, a16 = idx.cpu().numpy(), idx_bf.cpu().numpy()
    recall = float(np.mean([len(np.intersect1d(a32[b][a32[b] >= 0], a16[b][a16[b] >= 0])) /
                            max(1, int((a32[b] >= 0).sum())) for b in range(B)]))
    clocks = sampler.stop()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during the benchmark")

    # end to end through host buffers: every step uploads its query-side inputs from pinned
    # host memory (one packed copy) and downloads its outputs and selected indices (one
    # packed copy), on copy streams that overlap the neighbouring steps' kernels
    q_inputs = ("q", "q_fp4", "q_sf", "w", "pos", "n_entries")
    out_specs = {"out": (tuple(out.shape), out.dtype), "idx": (tuple(idx.shape), idx.dtype)}

    def e2e_launch(c, din, dout):
        csa.indexer_topk(din["n_entries"], din["q_fp4"], din["q_sf"], din["w"], c["k_fp4"],
                         c["k_sf"], k, workspace=ws_idx, idx=dout["idx"], dev_status=status,
                         paging=paging)
        csa.sparse_attn_decode(din["q"], din["pos"], din["n_entries"], c["kv"], c["kv_scale"],
                               c["swa"], c["sink"], dout["idx"], workspace=ws_att,
                               out=dout["out"], dev_status=status, paging=paging)

    E2E_STEPS = 32
    e2e_g, h2d, d2h, h_out = e2e_graphs(torch, e2e_launch, copies,
                                         {key: base[key].cpu() for key in q_inputs},
                                         out_specs, E2E_STEPS)
    e2e_ms = time_graphs(e2e_g, max(len(e2e_g), min(replays, 64)), E2E_STEPS)
    if not torch.equal(h_out["idx"], idx.cpu()):
        raise RuntimeError("end-to-end indices differ from the device-resident call's")

    ms_step, e2e_ms = max_over_ranks([ms_total / steps_run, e2e_ms], world, "cuda")
    value = whole_job_rate(B, world, ms_step)
    e2e_value = whole_job_rate(B, world, e2e_ms)

    if rank == 0:
        idx_bytes, step_bytes = algorithmic_bytes(d)
        pk = peaks()
        achieved = idx_bytes / (t_idx * 1e-3) / 1e9
        # the committed capture is of the 1M workload's indexer call; other workloads have none
        traffic = ncu_traffic() if w.name == "csa_decode_pro_1m" else None
        line = {
            "metric": metric, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": steps_run, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp4+fp16",
            "data": "synthetic",
            "config": {"workload": w.name, "queries_per_step_per_gpu": B, "context": w.L,
                       "entries_per_seq": int(d["n_entries"][0]), "heads": w.H,
                       "indexer_heads": w.H_I, "top_k": w.k, "window": 128,
                       "cache": cache_cfg,
                       "l2": f"inputs rotated over {ncopy} device copies "
                             f"({ncopy * copy_bytes / 1e6:.0f} MB of streamed inputs)",
                       "step_algorithmic_bytes": step_bytes,
                       "step_achieved_gbs": step_bytes / (ms_step * 1e-3) / 1e9,
                       "step_frac_of_peak": step_bytes / (ms_step * 1e-3) / 1e9 / pk["hbm_gbs"],
                       # each call timed in graphs of that call alone: the indexer's keys
                       # stream from HBM there as in the step, but the attention's inputs and
                       # code stay in L2 between its calls; inside the step the indexer's
                       # stream flushes them, so the attention's share of the step is the
                       # step time minus the indexer's
                       "indexer_topk_ms": t_idx, "sparse_attn_ms_alone": t_att,
                       "sparse_attn_ms_in_step": ms_step - t_idx,
                       "bf16_index_scores": {"indexer_topk_ms": t_idx_bf,
                                             "recall_of_fp32_topk": recall},
                       "launch": f"CUDA graphs of {GRAPH_STEPS} steps, programmatic dependent launch",
                       "e2e_launch": f"CUDA graphs of {E2E_STEPS} steps; one packed upload and "
                                     "one packed download per step on two copy streams, "
                                     "device inputs and outputs double-buffered"},
            "roofline": {"bound": "hbm", "kernel": "csa_indexer_topk (score + select)",
                         "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "peak_src": pk["src"],
                         "nominal_peak": NOMINAL_HBM_GBS,
                         "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                         "algorithmic_bytes_per_launch": idx_bytes,
                         "traffic": traffic["dram_bytes_per_launch"] if traffic else None},
            "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            # per step: the cooperative indexer launch (scores + selection) and the two
            # attention kernels
            "gpu_launches": 3 * steps_run,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_sample(d, w)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
