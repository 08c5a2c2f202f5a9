"""bench.e2e_graphs' pipelining on the CPU with a recording stand-in for torch's streams,
events, copies and graphs: step j uses device slot j % 2; its upload waits for the kernels
of step j - 2 (which read that slot), its kernels wait for its upload and for the download
of step j - 2 (which reads that output slot), and its download waits for its kernels; every
step moves its inputs up and its outputs down in one copy each."""

import contextlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _fake_torch(log):
    class Tensor:
        def __init__(self, nbytes, where):
            self.nbytes, self.where = nbytes, where

        def numel(self):
            return self.nbytes

        def __getitem__(self, sl):
            return View(self, sl)

        def copy_(self, src, non_blocking=False):
            log.append(("copy", cur[-1].name, src.where, self.where))
            return self

    class View(Tensor):
        def __init__(self, base, sl):
            super().__init__(0, base.where)

        def view(self, *a):
            return self

    class Stream:
        n = 0

        def __init__(self):
            Stream.n += 1
            self.name = f"s{Stream.n}"

        def wait_stream(self, other):
            log.append(("wait_stream", self.name, other.name))

        def wait_event(self, ev):
            log.append(("wait", self.name, ev.tag))

    class _Ev:
        def record(self, stream):
            self.tag = (stream.name, len(log))
            log.append(("record", stream.name, self.tag))

    cap = Stream()
    cur = [cap]

    class Cuda:
        Event = _Ev

        @staticmethod
        def Stream():
            return Stream()

        @staticmethod
        def current_stream():
            return cur[-1]

        @staticmethod
        @contextlib.contextmanager
        def stream(s):
            cur.append(s)
            yield
            cur.pop()

        @staticmethod
        def synchronize():
            pass

        @staticmethod
        def CUDAGraph():
            return object()

        @staticmethod
        @contextlib.contextmanager
        def graph(g, stream=None):
            log.append(("capture_begin",))
            yield
            log.append(("capture_end",))

    class Torch:
        cuda = Cuda
        uint8 = "u8"

        @staticmethod
        def empty(n, dtype=None, device=None, pin_memory=False):
            where = f"host{len(log)}" if pin_memory else f"dev{len(log)}"
            log.append(("alloc", where))
            return Tensor(n, where)

    Torch.cur = cur
    return Torch


def test_e2e_steps_alternate_slots_and_wait_on_reuse(monkeypatch):
    log = []
    torch = _fake_torch(log)
    steps = []

    class Spec:
        shape = (4,)
        dtype = "u8"

    def launch(c, din, dout):
        steps.append((c, torch.cuda.current_stream().name))
        log.append(("launch", torch.cuda.current_stream().name, c))

    monkeypatch.setattr(bench, "packed", lambda torch_, specs, host: (
        torch_.empty(64, pin_memory=host), {k: torch_.empty(8, pin_memory=host) for k in specs}))
    inputs = {"q": type("T", (), {"shape": (4,), "dtype": "u8", "where": "input"})()}
    graphs, h2d, d2h, _ = bench.e2e_graphs(torch, launch, [0, 1, 2], inputs,
                                           {"out": ((4,), "u8")}, 6)
    # the captured body of the single graph (3 copies, 6 steps: 6 / gcd(3, 6) = 1 graph)
    assert len(graphs) == 1
    b0 = log.index(("capture_begin",))
    body = log[b0:log.index(("capture_end",))]
    launches = [e for e in body if e[0] == "launch"]
    assert [e[2] for e in launches] == [0, 1, 2, 0, 1, 2]  # device copies rotate
    uploads = [e for e in body if e[0] == "copy" and e[2].startswith("host")]
    downloads = [e for e in body if e[0] == "copy" and e[3].startswith("host")]
    assert len(uploads) == 6 and len(downloads) == 6
    up_slots = [e[3] for e in uploads]
    assert up_slots[0::2] == [up_slots[0]] * 3 and up_slots[1::2] == [up_slots[1]] * 3
    assert up_slots[0] != up_slots[1]  # two device input slots, alternating
    down_slots = [e[2] for e in downloads]
    assert down_slots[0::2] == [down_slots[0]] * 3 and down_slots[1] != down_slots[0]
    # uploads and downloads run on their own streams, never on the launching stream
    comp = launches[0][1]
    assert all(e[1] != comp for e in uploads + downloads)
    assert len({e[1] for e in uploads}) == 1 and len({e[1] for e in downloads}) == 1
    assert uploads[0][1] != downloads[0][1]
    # ordering: step j's upload waits for step j - 2's kernels, its kernels wait for its
    # upload and for step j - 2's download, its download waits for its kernels
    rec = {}  # event tag -> ("done" | "up" | "down", step)
    step = {"up": 0, "done": 0, "down": 0}
    for e in body:
        if e[0] == "record":
            kind = "done" if e[1] == comp else ("up" if e[1] == uploads[0][1] else "down")
            rec[e[2]] = (kind, step[kind])
            step[kind] += 1
    waits = [(e[1], rec[e[2]]) for e in body if e[0] == "wait"]
    up_s, down_s = uploads[0][1], downloads[0][1]
    assert [w[1] for w in waits if w[0] == up_s] == [("done", j - 2) for j in range(2, 6)]
    assert [w[1] for w in waits if w[0] == down_s] == [("done", j) for j in range(6)]
    comp_waits = [w[1] for w in waits if w[0] == comp]
    assert [w for w in comp_waits if w[0] == "up"] == [("up", j) for j in range(6)]
    assert [w for w in comp_waits if w[0] == "down"] == [("down", j - 2) for j in range(2, 6)]
