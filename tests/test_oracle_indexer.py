"""Pins of the oracle's lightning-indexer scores and top-k selection."""

import numpy as np
import torch
import pytest

import oracle
from synth import inputs as synth
from tests import indep


def _scores_library(n, q_fp4, q_sf, w, k_fp4, k_sf):
    """Scores from table decoding and einsum (no oracle code)."""
    B, H_I, _ = q_fp4.shape
    Nmax = k_fp4.shape[1]
    q = indep.e2m1_to_f64(indep.unpack_fp4(q_fp4)) * np.repeat(
        indep.e8m0_to_f64(q_sf), 32, axis=-1)
    out = np.full((B, Nmax), np.nan)
    for b in range(B):
        ks = indep.key_scales(k_sf[b], Nmax)
        k = indep.e2m1_to_f64(indep.unpack_fp4(k_fp4[b])) * np.repeat(
            indep.e8m0_to_f64(ks), 32, axis=-1)
        dots = np.einsum("hd,jd->jh", q[b], k[: n[b]])
        out[b, : n[b]] = np.maximum(dots, 0.0) @ w[b].astype(np.float64)
    return out


def _small(seed=0, B=2, H_I=4, Nmax=256, planted=0):
    rng = np.random.default_rng(seed)
    n = np.array([Nmax - 37, Nmax][:B], dtype=np.int32)
    return n, synth.indexer_inputs(rng, B, H_I, Nmax, n, planted)


def test_scores_match_table_decode_and_einsum():
    n, ix = _small(seed=1)
    got = oracle.indexer_scores(n, ix["q_fp4"], ix["q_sf"], ix["w"], ix["k_fp4"], ix["k_sf"])
    want = _scores_library(n, ix["q_fp4"], ix["q_sf"], ix["w"], ix["k_fp4"], ix["k_sf"])
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=0)
    assert np.isnan(got[0, n[0]:]).all()


def test_single_block_scores_are_integer_exact():
    # all scales 2^0 and w = 1: twice each E2M1 value is an integer, so 4 * dot is an
    # integer sum that int64 arithmetic reproduces exactly
    n, ix = _small(seed=2, B=1, H_I=3)
    ix["q_sf"][:] = 127
    ix["k_sf"][:] = 127
    ix["w"][:] = 1.0
    got = oracle.indexer_scores(n, ix["q_fp4"], ix["q_sf"], ix["w"], ix["k_fp4"], ix["k_sf"])
    tab2 = (2 * indep.E2M1_TABLE).astype(np.int64)

    def ints(p):
        c = indep.unpack_fp4(p)
        v = tab2[c & 7]
        return np.where(c & 8, -v, v)

    qi, ki = ints(ix["q_fp4"][0]), ints(ix["k_fp4"][0][: n[0]])
    dots4 = ki @ qi.T
    want = np.maximum(dots4, 0).sum(1) / 4.0
    np.testing.assert_array_equal(got[0, : n[0]], want)


def test_nibble_order_and_scale_layout():
    B, H_I, Nmax = 1, 1, 256
    q = np.zeros((B, H_I, 64), np.uint8)
    k = np.zeros((B, Nmax, 64), np.uint8)
    q_sf = np.full((B, H_I, 4), 127, np.uint8)
    k_sf = np.full((B, Nmax // 128 * 512), 127, np.uint8)
    w = np.ones((B, H_I), np.float32)
    q[0, 0, 0] = 0x02  # element 0 = 1.0 (low nibble), element 1 = 0
    k[0, 5, 0] = 0x02  # entry 5, element 0 = 1.0
    k[0, 6, 0] = 0x20  # entry 6, element 1 = 1.0 (high nibble) -> no overlap with q
    q[0, 0, 40] = 0x30  # element 81 = 1.5 (high nibble of byte 40), block 2
    k[0, 200, 40] = 0x70  # entry 200, element 81 = 6.0
    k_sf[0, oracle.key_sf_offset(200, 2)] = 130  # x8 on block 2 of entry 200
    n = np.array([Nmax], np.int32)
    s = oracle.indexer_scores(n, q, q_sf, w, k, k_sf)[0]
    assert s[5] == 1.0 and s[6] == 0.0
    assert s[200] == 1.5 * 6.0 * 8.0
    assert np.count_nonzero(s) == 2
    # the same scale byte under the plain row-major reading would have hit another entry
    assert oracle.key_sf_offset(200, 2) != 200 * 4 + 2


def test_positive_rescale_and_head_permutation_keep_topk():
    n, ix = _small(seed=3, B=1, H_I=8, Nmax=1024, planted=4)
    args = (ix["q_fp4"], ix["q_sf"])
    s1 = oracle.indexer_scores(n, *args, ix["w"], ix["k_fp4"], ix["k_sf"])
    s2 = oracle.indexer_scores(n, *args, ix["w"] * 2, ix["k_fp4"], ix["k_sf"])
    np.testing.assert_array_equal(s2, 2 * s1)  # exact: power-of-two rescale
    perm = np.random.default_rng(0).permutation(8)
    s3 = oracle.indexer_scores(n, ix["q_fp4"][:, perm], ix["q_sf"][:, perm], ix["w"][:, perm],
                               ix["k_fp4"], ix["k_sf"])
    np.testing.assert_allclose(s3, s1, rtol=1e-14)
    k = 37
    t1 = oracle.topk(s1[0], int(n[0]), k)
    t3 = oracle.topk(s3[0], int(n[0]), k)
    gap = np.sort(s1[0, : n[0]])[::-1]
    if abs(gap[k - 1] - gap[k]) > 1e-9 * gap[k - 1]:
        np.testing.assert_array_equal(t1, t3)


def test_topk_matches_lexsort_with_ties():
    rng = np.random.default_rng(4)
    s = rng.integers(0, 50, size=3000).astype(np.float64)  # many exact ties
    for k in (1, 7, 64, 2999, 3000, 5000):
        got = oracle.topk(s, 3000, k)
        order = np.lexsort((np.arange(3000), -s))  # score desc, index asc
        keep = np.sort(order[: min(k, 3000)])
        want = np.full(k, -1, np.int32)
        want[: len(keep)] = keep
        np.testing.assert_array_equal(got, want)


def test_topk_only_sees_the_first_n():
    s = np.arange(100, dtype=np.float64)
    got = oracle.topk(s, 10, 3)  # entries 10.. are not eligible
    np.testing.assert_array_equal(got, [7, 8, 9])


def test_planted_blocks_dominate_topk():
    rng = np.random.default_rng(5)
    n = np.array([4096], np.int32)
    ix = synth.indexer_inputs(rng, 1, 64, 4096, n, planted_runs=8)
    s = oracle.indexer_scores(n, ix["q_fp4"], ix["q_sf"], ix["w"], ix["k_fp4"], ix["k_sf"])
    top = oracle.topk(s[0], 4096, 64)
    assert ix["planted"][0, top].mean() > 0.9


def test_eligible_counts_of_the_workloads():
    # the entry count of every decode workload is floor(L/m) at the query t = L-1
    for cid, n_expect in ((0, 2048), (1, 1024), (3, 262144)):
        w = synth.WORKLOADS[cid]
        t = w.L - 1
        assert (t + 1) // w.m == n_expect
    w = synth.WORKLOADS[2]
    L = synth.seq_lengths(w)
    assert ((L >= 65536) & (L <= 131072)).all() and len(L) == 32


def test_bf16_topk_orders_rounded_ties_by_index():
    # near 1.0 the BF16 spacing is 2^-7: 1.001 and 1 + 2^-10 both round to 1.0, so the
    # three entries at 1.0 tie and the smallest index wins the last slot
    s = np.array([1.0, 1.001, 3.0, 2.0, 1.0 + 2.0 ** -10, 0.5])
    np.testing.assert_array_equal(oracle.topk_bf16(s, 6, 3), [0, 2, 3])
    np.testing.assert_array_equal(oracle.topk(s, 6, 3), [1, 2, 3])
    np.testing.assert_array_equal(oracle.topk_bf16(s, 4, 8), [0, 1, 2, 3, -1, -1, -1, -1])


def test_bf16_topk_matches_library_rounding_and_lexsort():
    # an independent statement: torch's round-to-nearest-even BF16 cast, then numpy's
    # lexsort on (value descending, index ascending)
    rng = np.random.default_rng(5)
    for n, k in ((1000, 100), (4096, 512), (257, 300)):
        s = rng.standard_normal(n) * rng.choice([1.0, 1e3], size=n)
        r = torch.from_numpy(s).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
        # torch rounds through fp32; keep cases where that equals direct rounding
        order = np.lexsort((np.arange(n), -r))
        keep = min(k, n)
        want = np.concatenate([np.sort(order[:keep]), np.full(k - keep, -1)])
        got = oracle.topk_bf16(s.astype(np.float32).astype(np.float64), n, k)
        np.testing.assert_array_equal(got, want)


def test_bf16_topk_equals_exact_topk_on_distinct_bf16_values():
    rng = np.random.default_rng(6)
    vals = np.unique(rng.integers(0x3C00, 0x4400, size=3000).astype(np.uint16))
    s = torch.from_numpy(vals.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    rng.shuffle(s)
    n = len(s)
    np.testing.assert_array_equal(oracle.topk_bf16(s, n, 700), oracle.topk(s, n, 700))
