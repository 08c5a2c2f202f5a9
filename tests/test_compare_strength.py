"""Strength of the parity comparison rules (tests/compare.py): plant one loosening at a
time in a scratch copy of the rules (a wider tolerance, a check skipped, a window scaled
up) and require their own tests (tests/test_compare.py) to fail on every copy while
passing on the unmutated one (no GPU). Each mutant is (name, text in compare.py,
replacement, which occurrence)."""

import os
import shutil
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle
from tests import mutation

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = [
    ("max_abs_loose", "MAX_ABS = 1e-2", "MAX_ABS = 1e-1", 0),
    ("rel_l2_loose", "REL_L2 = 5e-3", "REL_L2 = 5e-2", 0),
    ("close_ignores_l2", "assert ma <= max_abs and rl <= rel_l2",
     "assert ma <= max_abs", 0),
    ("close_ignores_max", "assert ma <= max_abs and rl <= rel_l2",
     "assert rl <= rel_l2", 0),
    ("mid_rel_loose", "MID_REL = 1e-5", "MID_REL = 1e-2", 0),
    ("tie_rel_loose", "TIE_REL = 1e-6", "TIE_REL = 1e-3", 0),
    ("e4m3_codes_unchecked", "d8 = g8 != o8", "d8 = g8 != g8", 0),
    ("bf16_codes_unchecked", "d2 = rg != ro", "d2 = rg != rg", 0),
    ("e4m3_window_wide",
     "delta8 = MID_REL * np.maximum(np.abs(v[d8]), rms[d8])",
     "delta8 = MID_REL * np.maximum(np.abs(v[d8]), 1e3 * rms[d8])", 0),
    ("bf16_window_wide",
     "delta = MID_REL * np.maximum(np.abs(yr[d2]), pair[d2])",
     "delta = MID_REL * np.maximum(np.abs(yr[d2]), 1e3 * pair[d2])", 0),
    ("scale_unchecked",
     'np.testing.assert_allclose(scale_gpu, ora["kv_scale"], rtol=1e-5, err_msg=what)',
     "pass", 0),
    ("topk_padding_unchecked", 'assert (got[keep:] == -1).all(), f"{what}: padding"',
     "pass", 0),
    ("topk_order_unchecked",
     'assert (np.diff(g) > 0).all(), f"{what}: not strictly ascending"', "pass", 0),
    ("topk_far_below_accepted", "s[extra] >= sk * (1 - 10 * TIE_REL)",
     "s[extra] >= -np.inf", 0),
    ("mxfp4_scale_anywhere", "(np.abs(l2 - np.round(l2)) < sf_rel)",
     "(np.abs(l2 - np.round(l2)) < 1.0)", 0),
    ("mxfp4_codes_unchecked", "d = g_codes[keep] != o_codes[keep]",
     "d = g_codes[keep] != g_codes[keep]", 0),
    ("bf16_topk_step_wide", "step = np.abs(rk) * 2.0 ** -7", "step = np.abs(rk) * 2.0 ** -3", 0),
    ("bf16_topk_padding_unchecked", 'assert (got[keep:] == -1).all(), f"{what}: padding"',
     "pass", 1),
]


def _ignore(_, names):
    return [n for n in names if n in ("__pycache__", "c") or
            (n.startswith("test_") and n != "test_compare.py")]


def _prepare(base, name, text):
    d = os.path.join(base, name)
    shutil.copytree(os.path.join(ROOT, "synth"), os.path.join(d, "synth"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    shutil.copytree(os.path.join(ROOT, "tests"), os.path.join(d, "tests"), ignore=_ignore)
    with open(os.path.join(d, "tests", "compare.py"), "w") as f:
        f.write(text)
    os.makedirs(os.path.join(d, "oracle"))
    # the built oracle is copied with its times, so the copy does not rebuild it
    for f in ("__init__.py", "csa_oracle.cpp", "liboracle.so"):
        shutil.copy2(os.path.join(ROOT, "oracle", f), os.path.join(d, "oracle", f))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), d)
    return name, d


@pytest.mark.slow
def test_every_loosened_rule_fails_its_tests(tmp_path):
    oracle.build()
    with open(os.path.join(ROOT, "tests", "compare.py")) as f:
        src = f.read()
    jobs = [("unmutated", src)] + [(n, mutation.apply(src, o, r, w)) for n, o, r, w in MUTANTS]
    workers = max(1, min(8, os.cpu_count() or 2))
    with ThreadPoolExecutor(workers) as ex:
        built = list(ex.map(lambda j: _prepare(str(tmp_path), *j), jobs))
    names, dirs = [b[0] for b in built], [b[1] for b in built]
    status = mutation.run(dirs, ["test_compare"], str(tmp_path), workers)
    mutation.verdict(names, dirs, status, "comparison rules")
