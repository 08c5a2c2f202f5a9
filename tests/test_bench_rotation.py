"""bench.py's graph layout on the CPU with a recording stand-in for the CUDA graph calls:
inside every captured graph consecutive steps use different device copies of the inputs
(so no step finds the previous step's inputs in L2), and replaying the graphs round robin
continues the sequence copy 0, 1, 2, ... without a repeat at graph boundaries."""

import contextlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _Rec:
    """Just enough of torch for bench.capture_graph: graphs record the steps of their body."""

    def __init__(self):
        self.log = None

    class _Graph:
        def __init__(self):
            self.steps = []

    class _Stream:
        def wait_stream(self, *a):
            pass

    def make(self):
        rec = self

        class Cuda:
            @staticmethod
            def CUDAGraph():
                return rec._Graph()

            @staticmethod
            def Stream():
                return rec._Stream()

            @staticmethod
            def current_stream():
                return rec._Stream()

            @staticmethod
            def stream(s):
                return contextlib.nullcontext()

            @staticmethod
            def synchronize():
                pass

            @staticmethod
            @contextlib.contextmanager
            def graph(g, stream=None):
                rec.log = g.steps
                yield
                rec.log = None

        class Torch:
            cuda = Cuda

        return Torch


@pytest.mark.parametrize("ncopy,reps", [(4, 8), (4, 2), (3, 8), (512, 8), (24, 8), (1, 4)])
def test_rotation_graphs_alternate_copies(ncopy, reps):
    rec = _Rec()
    torch = rec.make()
    copies = list(range(ncopy))

    def step(c):
        if rec.log is not None:
            rec.log.append(c)

    graphs = bench.rotation_graphs(torch, step, copies, reps)
    seq = [c for _ in range(3) for g in graphs for c in g.steps]  # three rounds of replays
    assert all(len(g.steps) == reps for g in graphs)
    assert seq == [i % ncopy for i in range(len(seq))]
    if ncopy > 1:
        assert all(a != b for a, b in zip(seq, seq[1:]))
