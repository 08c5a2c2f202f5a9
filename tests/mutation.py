"""Helpers of the mutation checks (test infrastructure): plant one mistake at a time in a
scratch copy of some source and require a chosen set of test files to fail on every copy
while passing on the unmutated one.

Each copy's tests run in a child forked from a small server that has already imported
torch, numpy and pytest, instead of a fresh interpreter per copy. The child moves into its
copy first, so that `oracle`, `synth` and `tests` resolve there (none of them is imported
before the fork), runs the test files whose names start with the given prefixes with
pytest -x, and exits with pytest's status."""

import json
import os
import subprocess
import sys

_SERVER = r"""
import json, os, sys
import numpy, torch, pytest
dirs, workers, prefixes = json.loads(sys.argv[1]), int(sys.argv[2]), json.loads(sys.argv[3])
status, running, todo = {}, {}, list(dirs)
while todo or running:
    while todo and len(running) < workers:
        d = todo.pop(0)
        pid = os.fork()
        if pid == 0:
            try:
                os.chdir(d)
                fd = os.open(os.path.join(d, "pins.log"), os.O_WRONLY | os.O_CREAT, 0o644)
                os.dup2(fd, 1)
                os.dup2(fd, 2)
                sys.path.insert(0, d)
                tests = sorted(os.path.join("tests", f) for f in os.listdir("tests")
                               if f.endswith(".py") and f.startswith(tuple(prefixes)))
                rc = pytest.main(["-x", "-q", "-m", "not gpu", "-p", "no:cacheprovider",
                                  *tests])
                sys.stdout.flush()
                sys.stderr.flush()
                os._exit(int(rc))
            except BaseException:
                os._exit(99)
        running[pid] = d
    pid, st = os.wait()
    status[running.pop(pid)] = os.waitstatus_to_exitcode(st)
print(json.dumps(status))
"""


def apply(src: str, old: str, new: str, which: int) -> str:
    """src with occurrence `which` of `old` replaced by `new` (the pattern must exist)."""
    parts = src.split(old)
    assert len(parts) >= which + 2, f"pattern not in the source: {old[:60]!r}"
    return old.join(parts[:which + 1]) + new + old.join(parts[which + 1:])


def last_line(d: str) -> str:
    try:
        with open(os.path.join(d, "pins.log")) as f:
            lines = f.read().strip().splitlines()
        return lines[-1] if lines else ""
    except OSError:
        return "no log"


def run(dirs: list[str], prefixes: list[str], cwd: str, workers: int) -> dict:
    """Run the test files named by `prefixes` in every copy; {copy directory: status}."""
    r = subprocess.run([sys.executable, "-c", _SERVER, json.dumps(dirs), str(workers),
                        json.dumps(prefixes)],
                       cwd=cwd, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stderr[-600:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def verdict(names: list[str], dirs: list[str], status: dict, what: str) -> None:
    """The first copy is the unmutated one and must pass; every other copy must fail a test
    (status 1) or crash on a signal (negative). Any other status (interrupted, internal or
    usage error, nothing collected) means the harness is broken."""
    res = [(n, status[d], last_line(d)) for n, d in zip(names, dirs)]
    control = res[0]
    assert control[1] == 0, f"the unmutated {what} fails its tests: {control[2]}"
    broken = [(n, rc, msg) for n, rc, msg in res[1:] if rc > 1]
    assert not broken, f"test runs that ended without a verdict: {broken}"
    survivors = [(n, msg) for n, rc, msg in res[1:] if rc == 0]
    assert not survivors, f"planted mistakes no test catches: {survivors}"
