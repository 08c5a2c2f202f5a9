"""The comparison rules the GPU parity tests apply (tests/compare.py) catch planted
deviations and accept only what they are meant to accept (no GPU)."""

import numpy as np
import pytest

import oracle
from synth import inputs as synth
from tests import compare


def test_close_bounds_both_the_largest_error_and_the_relative_l2():
    rng = np.random.default_rng(1)
    want = rng.standard_normal(4096)
    compare.close(want.copy(), want)
    one_off = want.copy()
    one_off[17] += 2e-2  # a single element past the max-abs bound
    with pytest.raises(AssertionError, match="max-abs"):
        compare.close(one_off, want)
    small = want * 1e-3
    with pytest.raises(AssertionError, match="rel-L2"):
        compare.close(small * 1.01, small)  # tiny values, 1 % off everywhere
    compare.close(want + 1e-4, want)


def _entries():
    inp = synth.compress_inputs(2, 64, 4, True, seed=3)
    ora = oracle.compress(inp["a"], inp["za"], inp["bias"], 4, True, b=inp["b"], zb=inp["zb"])
    return ora["kv"].copy(), ora["kv_scale"].copy(), ora["y"].astype(np.float32), ora


def test_entries_accept_the_oracle_and_catch_planted_deviations():
    kv, sc, dbg, ora = _entries()
    assert compare.compare_entries(kv, sc, dbg, ora) == 0
    bad = kv.copy()
    bad[0, 3, 10] ^= 0x08  # an E4M3 code one exponent step away: not a midpoint flip
    with pytest.raises(AssertionError, match="E4M3"):
        compare.compare_entries(bad, sc, dbg, ora)
    rope = kv.copy()
    rope[1, 2, 448 + 2 * 5 + 1] ^= 0x40  # a BF16 RoPE dim's exponent bit
    with pytest.raises(AssertionError, match="BF16"):
        compare.compare_entries(rope, sc, dbg, ora)
    with pytest.raises(AssertionError):
        compare.compare_entries(kv, sc * 1.001, dbg, ora)
    with pytest.raises(AssertionError, match="pre-quantisation"):
        compare.compare_entries(kv, sc, dbg + 0.05, ora)


def test_topk_is_exact_except_inside_a_tie():
    rng = np.random.default_rng(2)
    n, k = 1000, 100
    s = rng.standard_normal(n)
    want = np.sort(np.lexsort((np.arange(n), -s))[:k])
    assert compare.compare_topk(want, s, n, k) == 0
    order = np.lexsort((np.arange(n), -s))
    wrong = np.sort(np.r_[order[:k - 1], order[500]])  # the k-th swapped for a far one
    with pytest.raises(AssertionError):
        compare.compare_topk(wrong, s, n, k)
    with pytest.raises(AssertionError, match="ascending"):
        compare.compare_topk(want[::-1].copy(), s, n, k)
    short = np.r_[np.arange(10), np.full(k - 10, -1)]  # n < k: all 10 then padding
    assert compare.compare_topk(short, s[:10], 10, k) == 0
    with pytest.raises(AssertionError, match="padding"):
        compare.compare_topk(np.r_[np.arange(10), np.full(k - 10, 0)], s[:10], 10, k)
    # a near tie at the boundary: the (k+1)-th within 1e-6 of the k-th may replace it
    t = s.copy()
    t[order[k]] = t[order[k - 1]] * (1 - 1e-7)
    swapped = np.sort(np.r_[order[:k - 1], order[k]])
    assert compare.compare_topk(swapped, t, n, k) == 1


def test_bf16_topk_accepts_only_boundary_neighbours():
    rng = np.random.default_rng(3)
    n, k = 2000, 300
    s = np.abs(rng.standard_normal(n)) + 1.0
    want = oracle.topk_bf16(s, n, k)
    assert compare.compare_topk_bf16(want, s, n, k) == 0
    r = compare._bf16_round(s)
    far = int(np.argmin(r))  # the smallest score, far below the boundary
    wrong = np.sort(np.r_[want[:k - 1], far]) if far not in want else want
    with pytest.raises(AssertionError):
        compare.compare_topk_bf16(wrong, s, n, k)
