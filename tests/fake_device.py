"""Shape-only stand-ins for the CUDA device, so that bench.py's host flow (argument
handling, graph capture and replay calls, timing arithmetic, the JSON line) can run on a
machine without a GPU. Tensors asked for on "cuda" live on the meta device (shapes, no
data); graphs, streams and events do nothing and every timing reads 1 ms; the library's
compute entry points return success without running, while its workspace-size queries
(host functions) run for real. Numbers produced this way mean nothing; only the flow and
the keys of the output are under test. Used by tests/test_bench_dry.py in child processes.
"""

import contextlib

import torch

import long_context_compressed_layer_b200 as csa


class _Graph:
    def replay(self):
        pass


class _Event:
    def __init__(self, *a, **k):
        pass

    def record(self, *a, **k):
        pass

    def elapsed_time(self, other):
        return 1.0


class _Stream:
    cuda_stream = 0

    def wait_stream(self, *a, **k):
        pass

    def wait_event(self, *a, **k):
        pass


class _FakeLib:
    def __init__(self, real):
        self.real = real

    def __getattr__(self, name):
        if name.endswith("_workspace_size") or name == "csa_status_string":
            return getattr(self.real, name)
        if name.endswith("_flops"):
            return lambda *a: 1.0
        return lambda *a: csa.CSA_OK


def _to_meta_device(fn):
    def g(*a, **k):
        if str(k.get("device", "")).startswith("cuda"):
            k["device"] = "meta"
            k.pop("generator", None)
        k.pop("pin_memory", None)
        return fn(*a, **k)
    return g


def install() -> None:
    for name in ("empty", "zeros", "ones", "full", "randn", "rand", "randint", "arange",
                 "empty_like", "zeros_like"):
        setattr(torch, name, _to_meta_device(getattr(torch, name)))
    real_gen = torch.Generator

    class _CpuGenerator(real_gen):
        def __new__(cls, device=None):
            return real_gen()

    torch.Generator = _CpuGenerator
    T = torch.Tensor
    real_cpu, real_item, real_copy = T.cpu, T.item, T.copy_
    T.cuda = lambda self, *a, **k: self.to("meta")
    T.cpu = lambda self, *a, **k: (torch.zeros(self.shape, dtype=self.dtype) if self.is_meta
                                   else real_cpu(self, *a, **k))
    T.item = lambda self: 0 if self.is_meta else real_item(self)
    # a copy from the device leaves zeros in a host tensor (the fake device reads as zeros)
    T.copy_ = lambda self, src, non_blocking=False: (
        self if self.is_meta else self.zero_() if src.is_meta
        else real_copy(self, src, non_blocking))
    T.pin_memory = lambda self, *a, **k: self
    c = torch.cuda
    c.is_available = lambda: True
    c.init = lambda: None
    c.synchronize = lambda *a, **k: None
    c.set_device = lambda *a, **k: None
    c.current_device = lambda: 0
    c.CUDAGraph = _Graph
    c.graph = lambda *a, **k: contextlib.nullcontext()
    c.Stream = lambda *a, **k: _Stream()
    c.stream = lambda *a, **k: contextlib.nullcontext()
    c.current_stream = lambda *a, **k: _Stream()
    c.Event = _Event
    fake = _FakeLib(csa.lib())
    csa.lib = lambda: fake
    csa._stream = lambda s: 0
    real_ptr = csa._ptr

    def ptr(t, *, elem=None, name=""):
        if t is not None and t.is_meta:
            if elem is not None and t.element_size() != elem:
                raise ValueError(f"{name}: expected {elem}-byte elements, got {t.dtype}")
            return 0
        return real_ptr(t, elem=elem, name=name)

    csa._ptr = ptr
