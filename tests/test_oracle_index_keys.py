"""Pins of the oracle's indexer-key compression: the E2M1 encoder, the MXFP4 block rule,
the gated merge on the 128-dim stream and the stored layout the indexer reads."""

import numpy as np
import pytest

import oracle
from synth import inputs as synth
from tests import indep

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])


def _nearest_even(x):
    """Brute force: the nearest E2M1 magnitude, ties to the even mantissa bit, saturate."""
    a = min(abs(x), 6.0)
    d = np.abs(E2M1 - a)
    best = np.flatnonzero(d == d.min())
    c = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
    return (8 if np.signbit(x) else 0) | int(c)


def test_e2m1_encode_is_nearest_with_even_ties():
    xs = np.concatenate([np.arange(-8, 8, 1 / 64), [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0],
                         [-0.25, -0.75, -5.0, 1e9, -1e9, 0.0, -0.0]])
    got = oracle.e2m1_encode(xs)
    want = np.array([_nearest_even(x) for x in xs], dtype=np.uint8)
    np.testing.assert_array_equal(got, want)


def test_e2m1_encode_round_trips_every_code():
    codes = np.arange(16, dtype=np.uint8)
    np.testing.assert_array_equal(oracle.e2m1_encode(oracle.e2m1_decode(codes)), codes)


def test_mxfp4_block_hand_examples():
    # amax 7: floor(log2 7) = 2, shared exponent 0 -> 6, 3, 1.5 exact; 0.75 and 5 tie to
    # 1.0 and 4.0; -0.25 ties to -0; 7 saturates to 6
    nib, sf = oracle.mxfp4_block(np.r_[[6, 3, 1.5, 0.75, -0.25, 5, 7], np.zeros(25)])
    assert sf == 127
    np.testing.assert_array_equal(nib[:8], [7, 5, 3, 2, 8, 6, 7, 0])
    # amax 0.3: floor(log2 0.3) = -2, exponent -4, 0.3 * 16 = 4.8 -> 4.0
    nib, sf = oracle.mxfp4_block(np.r_[[0.3, -0.1], np.zeros(30)])
    assert sf == 127 - 4
    np.testing.assert_array_equal(nib[:2], [6, 8 | 3])  # -0.1 * 16 = -1.6 -> -1.5
    nib, sf = oracle.mxfp4_block(np.zeros(32))
    assert sf == 0 and not nib.any()


def test_mxfp4_block_error_bound_and_top_code():
    rng = np.random.default_rng(3)
    for _ in range(200):
        v = rng.standard_normal(32) * 10.0 ** rng.uniform(-3, 3)
        nib, sf = oracle.mxfp4_block(v)
        X = 2.0 ** (sf - 127)
        dq = oracle.e2m1_decode(nib) * X
        r = np.abs(v) / X
        assert r.max() >= 4 and r.max() < 8  # the shared exponent puts the max in [4X, 8X)
        inside = r <= 6
        # half of the widest E2M1 step (2) inside the range; the rule saturates the rest
        assert (np.abs(v - dq)[inside] <= X).all()
        assert (np.abs(dq[~inside]) == 6 * X).all()


def test_key_merge_with_uniform_gates_is_the_block_mean():
    inp = synth.compress_inputs(2, 64, 4, True, seed=5, dim=128)
    inp["za"][:] = 0
    inp["zb"][:] = 0
    inp["bias"][:] = 0
    _, _, y = oracle.compress_index_keys(inp["a"], inp["za"], inp["bias"], 4, True, 128,
                                         b=inp["b"], zb=inp["zb"])
    a = indep.bf16_to_f64(inp["a"])
    b = indep.bf16_to_f64(inp["b"])
    want0 = a[:, 0:4].mean(axis=1)  # the first entry has no previous block
    want5 = (a[:, 20:24].sum(axis=1) + b[:, 16:20].sum(axis=1)) / 8
    np.testing.assert_allclose(y[:, 0], want0, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(y[:, 5], want5, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("m,pos0", [(4, 0), (4, 512), (2, 8)])
def test_key_merge_matches_library_softmax(m, pos0):
    # random gates and bias: every candidate slot keeps its own bias term
    inp = synth.compress_inputs(2, 16 * m, m, True, seed=21 + m + pos0, dim=128, pos0=pos0)
    Nmax = (pos0 // m + 16 + 127) // 128 * 128
    _, _, y = oracle.compress_index_keys(inp["a"], inp["za"], inp["bias"], m, True, Nmax,
                                         b=inp["b"], zb=inp["zb"], pos0=pos0,
                                         prev_b=inp.get("prev_b"), prev_zb=inp.get("prev_zb"))
    np.testing.assert_allclose(y, indep.gated_merge(inp, m, True, pos0), rtol=1e-12,
                               atol=1e-12)


def test_stored_keys_are_the_mxfp4_of_the_merge_in_the_indexer_layout():
    inp = synth.compress_inputs(1, 4 * 200, 4, True, seed=6, dim=128, pos0=512)
    k_fp4, k_sf, y = oracle.compress_index_keys(inp["a"], inp["za"], inp["bias"], 4, True,
                                                384, b=inp["b"], zb=inp["zb"], pos0=512,
                                                prev_b=inp["prev_b"], prev_zb=inp["prev_zb"])
    assert not k_fp4[0, :128].any()  # rows before pos0 / m are left alone
    for i in (0, 1, 77, 199):
        row = 128 + i
        lo, hi = k_fp4[0, row] & 15, k_fp4[0, row] >> 4
        codes = np.stack([lo, hi], axis=1).reshape(128)
        for s in range(4):
            nib, sf = oracle.mxfp4_block(y[0, i, 32 * s:32 * s + 32])
            np.testing.assert_array_equal(codes[32 * s:32 * s + 32], nib)
            assert k_sf[0, oracle.key_sf_offset(row, s)] == sf
    # the indexer reads these keys back as the dequantised merge (one query, one head)
    q = np.zeros((1, 16, 64), np.uint8)
    q[0, 0] = 0x22  # every query element 1.0 (code 2 in both nibbles)
    qsf = np.full((1, 16, 4), 127, np.uint8)
    w = np.zeros((1, 16), np.float32)
    w[0, 0] = 1.0
    s = oracle.indexer_scores(np.array([328], np.int32), q, qsf, w, k_fp4, k_sf)[0]
    for i in (0, 77, 199):
        dq = np.concatenate([oracle.e2m1_decode(oracle.mxfp4_block(y[0, i, 32 * t:32 * t + 32])[0])
                             * 2.0 ** (oracle.mxfp4_block(y[0, i, 32 * t:32 * t + 32])[1] - 127)
                             for t in range(4)])
        assert abs(s[128 + i] - max(0.0, dq.sum())) <= 1e-9 * max(1.0, abs(dq).sum())


def test_indexer_query_is_the_library_matmul_then_mxfp4_per_head():
    rng = np.random.default_rng(8)
    T, r, H_I = 37, 192, 4
    c = synth.bf16_normal(rng, (T, r))
    W = synth.bf16_normal(rng, (H_I * 128, r), std=r ** -0.5)
    q_fp4, q_sf, y = oracle.indexer_query(c, W, H_I)
    want = indep.bf16_to_f64(c) @ indep.bf16_to_f64(W).T  # numpy's matmul in fp64
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)
    for t in (0, 17, 36):
        for h in range(H_I):
            codes = np.stack([q_fp4[t, h] & 15, q_fp4[t, h] >> 4], axis=1).reshape(128)
            for s in range(4):
                nib, sf = oracle.mxfp4_block(y[t, h * 128 + 32 * s:h * 128 + 32 * s + 32])
                np.testing.assert_array_equal(codes[32 * s:32 * s + 32], nib)
                assert q_sf[t, h, s] == sf
