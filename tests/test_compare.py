"""The comparison rules the GPU parity tests apply (tests/compare.py) catch planted
deviations and accept only what they are meant to accept (no GPU)."""

import numpy as np
import pytest

import oracle
from synth import inputs as synth
from tests import compare, indep


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


def test_code_flips_must_be_the_rounding_of_a_value_near_the_oracles():
    # an E4M3 value placed exactly on the midpoint of two codes: either neighbour passes,
    # a code two steps away does not (the older rule looked only at where the oracle's
    # value lay and accepted any code there)
    kv, sc, dbg, ora = _entries()
    y = ora["y"].copy()
    lo = int(kv[0, 1, 7]) & 0x7F
    if lo in (0, 0x7E):
        lo = 0x30
    pair = indep.e4m3_to_f64(np.array([lo, lo + 1], dtype=np.uint8))
    y[0, 1, 7] = (pair[0] + pair[1]) / 2 * float(sc[0, 1])
    ref = kv.copy()
    ref[0, 1, 7] = lo
    for code, ok in ((lo, True), (lo + 1, True), (lo + 2, False), (lo - 1, False)):
        got = ref.copy()
        got[0, 1, 7] = code
        if ok:
            compare.check_codes(got, ref, y, sc)
        else:
            with pytest.raises(AssertionError, match="E4M3"):
                compare.check_codes(got, ref, y, sc)


def test_rotated_bf16_codes_follow_the_pair_norm_window():
    # a rotated dim that nearly cancels (|v| = 1e-7 of its pair's norm): fp32 rounding of
    # the pair moves it by several of its own BF16 steps, and the rule admits exactly the
    # codes within 1e-5 of the pair norm, not arbitrary ones
    kv, sc, dbg, ora = _entries()
    y = ora["y"].copy()
    y[0, 0, 448], y[0, 0, 449] = 1e-7, 1.0  # pair (x0, x1) with a tiny x0
    ref = kv.copy()
    ref[0, 0, 448:452] = np.frombuffer(indep.f64_to_bf16(np.array([1e-7, 1.0])).tobytes(),
                                       np.uint8)
    close_by = ref.copy()
    close_by[0, 0, 448:452] = np.frombuffer(indep.f64_to_bf16(np.array([3e-6, 1.0])).tobytes(),
                                            np.uint8)
    assert compare.check_codes(close_by, ref, y, sc) == 1
    far = ref.copy()
    far[0, 0, 448:452] = np.frombuffer(indep.f64_to_bf16(np.array([3e-4, 1.0])).tobytes(),
                                       np.uint8)
    with pytest.raises(AssertionError, match="BF16"):
        compare.check_codes(far, ref, y, sc)
    sign = ref.copy()
    sign[0, 0, 448:452] = np.frombuffer(indep.f64_to_bf16(np.array([-2e-5, 1.0])).tobytes(),
                                        np.uint8)
    with pytest.raises(AssertionError, match="BF16"):
        compare.check_codes(sign, ref, y, sc)


def test_mxfp4_rule_accepts_the_oracle_and_catches_planted_deviations():
    inp = synth.compress_inputs(1, 64, 4, True, seed=5, dim=128)
    kf, ks, y = oracle.compress_index_keys(inp["a"], inp["za"], inp["bias"], 4, True, 128,
                                           b=inp["b"], zb=inp["zb"])
    rows = np.arange(16)
    sf = np.array([[ks[0, oracle.key_sf_offset(r, s)] for s in range(4)] for r in rows])
    codes = compare.unpack_nibbles(kf[0, rows]).reshape(-1, 32)
    yb = y[0].reshape(-1, 32)
    assert compare.check_mxfp4(codes, codes, sf.reshape(-1), sf.reshape(-1), yb) == 0
    # an element moved to the next code although the value is nowhere near a midpoint
    X = np.ldexp(1.0, sf.reshape(-1).astype(np.int64) - 127)[:, None]
    r = np.abs(yb / X)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    far = np.min(np.abs(r[..., None] - mids), axis=-1) > 0.1
    blk, el = np.argwhere(far & (codes & 7 < 7) & (codes & 7 > 0))[0]
    bad = codes.copy()
    bad[blk, el] += 1
    with pytest.raises(AssertionError, match="E2M1"):
        compare.check_mxfp4(bad, codes, sf.reshape(-1), sf.reshape(-1), yb)
    # a scale one step off on a block whose maximum is not a power of two
    sfb = sf.reshape(-1).copy()
    amax = np.abs(yb).max(axis=1)
    i = int(np.argmax(np.abs(np.log2(amax) - np.round(np.log2(amax))) > 0.1))
    sfb[i] += 1
    with pytest.raises(AssertionError, match="scale"):
        compare.check_mxfp4(codes, codes, sfb, sf.reshape(-1), yb)
    # at an exact midpoint both neighbours pass
    mid = yb.copy()
    mid[0, 0] = 1.25 * X[0, 0]
    two = codes.copy()
    two[:1, :1] = 2
    three = codes.copy()
    three[:1, :1] = 3
    assert compare.check_mxfp4(three, two, sf.reshape(-1), sf.reshape(-1), mid) <= 1


def test_a_boundary_gap_above_the_tie_tolerance_is_not_a_tie():
    # the (k+1)-th score 1e-4 (relative) below the k-th: outside the 1e-6 tie window, so a
    # set that takes it instead of the k-th is wrong
    rng = np.random.default_rng(4)
    n, k = 1000, 100
    s = rng.standard_normal(n)
    order = np.lexsort((np.arange(n), -s))
    s[order[k]] = s[order[k - 1]] * (1 - 1e-4)
    swapped = np.sort(np.r_[order[:k - 1], order[k]])
    with pytest.raises(AssertionError, match="gap"):
        compare.compare_topk(swapped, s, n, k)


def test_inside_a_tie_every_chosen_entry_is_still_at_the_boundary():
    # an exact tie between the k-th and (k+1)-th scores lets either be chosen, but not an
    # entry far below them
    rng = np.random.default_rng(5)
    n, k = 1000, 100
    s = rng.standard_normal(n)
    order = np.lexsort((np.arange(n), -s))
    s[order[k]] = s[order[k - 1]]
    wrong = np.sort(np.r_[order[:k - 1], order[500]])
    with pytest.raises(AssertionError, match="far below"):
        compare.compare_topk(wrong, s, n, k)


def test_a_flip_past_the_midpoint_window_is_rejected():
    # the oracle's value 2e-3 of the row's RMS above a midpoint: well outside the 1e-5
    # window, so the code below that midpoint is not a rounding of a nearby value
    kv, sc, dbg, ora = _entries()
    y = ora["y"].copy()
    v = y[0, 1, :448] / float(sc[0, 1])
    rms = float(np.sqrt(np.mean(v * v)))
    lo = int(indep.f64_to_e4m3(np.array([rms]))[0]) & 0x7F
    lo = lo - 1 if lo & 7 == 7 else lo
    pair = indep.e4m3_to_f64(np.array([lo, lo + 1], dtype=np.uint8))
    y[0, 1, 7] = ((pair[0] + pair[1]) / 2 + 2e-3 * rms) * float(sc[0, 1])
    ref = kv.copy()
    ref[0, 1, 7] = lo + 1  # the nearest code of the oracle's value
    got = ref.copy()
    got[0, 1, 7] = lo
    with pytest.raises(AssertionError, match="E4M3"):
        compare.check_codes(got, ref, y, sc)


def test_bf16_topk_rejects_an_entry_several_steps_below_the_boundary():
    # scores on the BF16 grid of [2, 4) (step 2^-6): the top 40 of 120 start at 3.25; an
    # entry 3 grid steps below (0.047, above the rule's one step of 3.25 x 2^-7 = 0.025)
    # may not replace the boundary entry
    n, k = 120, 40
    s = 2.0 + np.arange(n) * 2.0 ** -6
    want = oracle.topk_bf16(s, n, k)
    assert compare.compare_topk_bf16(want, s, n, k) == 0
    wrong = np.sort(np.r_[np.setdiff1d(want, [80]), 77])
    with pytest.raises(AssertionError, match="BF16 step"):
        compare.compare_topk_bf16(wrong, s, n, k)


def test_bf16_topk_checks_the_padding():
    s = 1.0 + np.arange(10) * 0.25
    want = oracle.topk_bf16(s, 10, 16)
    assert compare.compare_topk_bf16(want, s, 10, 16) == 0
    bad = want.copy()
    bad[10:] = 0
    with pytest.raises(AssertionError, match="padding"):
        compare.compare_topk_bf16(bad, s, 10, 16)
