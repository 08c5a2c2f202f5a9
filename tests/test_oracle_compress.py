"""Pins of the oracle's gated compression (gated merge, RMSNorm, RoPE, split store)."""

import numpy as np
import pytest

import oracle
from synth import inputs as synth
from tests import indep


@pytest.mark.parametrize("m,overlap,pos0", [(4, True, 0), (2, True, 8), (4, False, 0),
                                            (1, True, 4), (128, False, 0)])
def test_merge_matches_library_softmax(m, overlap, pos0):
    T = max(4 * m, 16)
    inp = synth.compress_inputs(2, T, m, overlap, seed=11 + m, pos0=pos0)
    r = oracle.compress(inp["a"], inp["za"], inp["bias"], m, overlap, b=inp.get("b"),
                        zb=inp.get("zb"), pos0=pos0, prev_b=inp.get("prev_b"),
                        prev_zb=inp.get("prev_zb"))
    np.testing.assert_allclose(r["e"], indep.gated_merge(inp, m, overlap, pos0), rtol=1e-12,
                               atol=1e-12)


def test_uniform_gates_give_block_mean():
    m, T = 4, 16
    inp = synth.compress_inputs(1, T, m, True, seed=3)
    za = np.full_like(inp["za"], 0.7)
    zb = np.full_like(inp["zb"], 0.7)
    bias = np.zeros(2 * m, np.float32)
    r = oracle.compress(inp["a"], za, bias, m, True, b=inp["b"], zb=zb)
    a = indep.bf16_to_f64(inp["a"])[0]
    bb = indep.bf16_to_f64(inp["b"])[0]
    # first block: own 4 tokens only; later blocks: own 4 of a + previous 4 of b
    np.testing.assert_allclose(r["e"][0, 0], a[0:4].mean(0), rtol=0, atol=1e-14)
    for i in range(1, T // m):
        want = np.concatenate([a[4 * i:4 * i + 4], bb[4 * i - 4:4 * i]]).mean(0)
        np.testing.assert_allclose(r["e"][0, i], want, rtol=0, atol=1e-14)


def test_single_token_gate_reproduces_raw_kv():
    # m = 1, overlap on: bias (0, -1000) keeps only the own token of a; (-1000, 0) keeps
    # only the previous token of b (exp(-1000) underflows to exactly 0 in fp64). Catches
    # a swapped slot order or an off-by-one previous block.
    T = 8
    inp = synth.compress_inputs(1, T, 1, True, seed=4)
    own = oracle.compress(inp["a"], inp["za"], np.array([0, -1000], np.float32), 1, True,
                          b=inp["b"], zb=inp["zb"])
    np.testing.assert_array_equal(own["e"][0], indep.bf16_to_f64(inp["a"][0]))
    prev = oracle.compress(inp["a"], inp["za"], np.array([-1000, 0], np.float32), 1, True,
                           b=inp["b"], zb=inp["zb"])
    np.testing.assert_array_equal(prev["e"][0, 1:], indep.bf16_to_f64(inp["b"][0, :-1]))
    # the first entry of a sequence has no previous block, so only a[0] can be chosen
    np.testing.assert_array_equal(prev["e"][0, 0], indep.bf16_to_f64(inp["a"][0, 0]))
    # and m = 1 at position t equals the sliding-window form of token t
    for t in range(T):
        row = oracle.swa_row(inp["a"][0, t], t)
        assert (oracle.bf16_encode(own["y"][0, t]) == row).all()


def test_rmsnorm_closed_form_at_position_zero():
    # entry 0 sits at position 0 where the rotation is the identity
    inp = synth.compress_inputs(3, 8, 4, True, seed=5)
    r = oracle.compress(inp["a"], inp["za"], inp["bias"], 4, True, b=inp["b"], zb=inp["zb"],
                        eps=1e-6)
    for b in range(3):
        e, y = r["e"][b, 0], r["y"][b, 0]
        ms = np.mean(e * e)
        np.testing.assert_allclose(y, e / np.sqrt(ms + 1e-6), rtol=1e-13)
        np.testing.assert_allclose(np.mean(y * y), ms / (ms + 1e-6), rtol=1e-12)


def test_rmsnorm_weight_scales_each_normalised_dim():
    # the optional RMSNorm weight multiplies dim d of the normalised entry by w[d]; with
    # equal weights on the two dims of each RoPE pair the rotation commutes with it
    rng = np.random.default_rng(12)
    inp = synth.compress_inputs(2, 32, 4, True, seed=12)
    w = rng.uniform(0.5, 2.0, 512).astype(np.float32)
    w[449::2] = w[448::2]
    base = oracle.compress(inp["a"], inp["za"], inp["bias"], 4, True, b=inp["b"], zb=inp["zb"])
    wt = oracle.compress(inp["a"], inp["za"], inp["bias"], 4, True, b=inp["b"], zb=inp["zb"],
                         norm_w=w)
    np.testing.assert_array_equal(wt["e"], base["e"])
    np.testing.assert_allclose(wt["y"], base["y"] * w.astype(np.float64), rtol=1e-13,
                               atol=1e-15)


def test_window_row_norm_weight_by_powers_of_two():
    # powers of two scale binary floating point exactly, so the stored BF16 window row with
    # such weights is the row without them times the weights
    rng = np.random.default_rng(13)
    a = synth.bf16_normal(rng, (512,))
    w = (2.0 ** rng.integers(-2, 3, 512)).astype(np.float32)
    w[449::2] = w[448::2]
    for t in (0, 5, 1000):
        plain = indep.bf16_to_f64(oracle.swa_row(a, t))
        weighted = indep.bf16_to_f64(oracle.swa_row(a, t, norm_w=w))
        np.testing.assert_array_equal(weighted, plain * w.astype(np.float64))


def test_rope_pairs_keep_norm_and_turn_by_position():
    m = 4
    inp = synth.compress_inputs(1, 64, m, True, seed=6)
    rot = oracle.compress(inp["a"], inp["za"], inp["bias"], m, True, b=inp["b"], zb=inp["zb"])
    e = rot["e"][0]
    n = e / np.sqrt(np.mean(e * e, axis=1, keepdims=True) + 1e-6)
    y = rot["y"][0]
    np.testing.assert_allclose(y[:, :448], n[:, :448], rtol=1e-13)
    for i in range(e.shape[0]):
        p = m * i
        x0, x1 = n[i, 448::2], n[i, 449::2]
        y0, y1 = y[i, 448::2], y[i, 449::2]
        np.testing.assert_allclose(np.hypot(y0, y1), np.hypot(x0, x1), rtol=1e-12)
        turn = np.angle((y0 + 1j * y1) / (x0 + 1j * x1))
        # pair 0 turns by p rad (theta_0 = 1); pair 16 by p/100 (10000^(-1/2)); pair 8 by
        # p/10 (10000^(-1/4))
        for j, f in ((0, 1.0), (16, 0.01), (8, 0.1)):
            want = np.angle(np.exp(1j * p * f))
            assert abs(np.angle(np.exp(1j * (turn[j] - want)))) < 1e-9, (i, j)


def test_rope_turn_is_additive_in_position():
    # the rotation at positions p1 then p2 equals the rotation at p1 + p2
    inp = synth.compress_inputs(1, 4 * 9, 4, False, seed=7)
    r = oracle.compress(inp["a"], inp["za"], inp["bias"], 4, False)
    e = r["e"][0]
    n = e / np.sqrt(np.mean(e * e, axis=1, keepdims=True) + 1e-6)
    z = (r["y"][0, :, 448::2] + 1j * r["y"][0, :, 449::2]) / (n[:, 448::2] + 1j * n[:, 449::2])
    # entries 2 (p=8), 3 (p=12) and 5 (p=20): turn(8) * turn(12) == turn(20)
    np.testing.assert_allclose(z[2] * z[3], z[5], rtol=0, atol=1e-12)


def test_split_store_matches_library_casts():
    inp = synth.compress_inputs(2, 64, 4, True, seed=8)
    r = oracle.compress(inp["a"], inp["za"], inp["bias"], 4, True, b=inp["b"], zb=inp["zb"])
    y = r["y"]
    amax = np.abs(y[..., :448]).max(-1)
    np.testing.assert_array_equal(r["kv_scale"], (amax / 448.0).astype(np.float32))
    codes = indep.f64_to_e4m3(y[..., :448] / r["kv_scale"][..., None].astype(np.float64))
    np.testing.assert_array_equal(r["kv"][..., :448], codes)
    rope = np.ascontiguousarray(r["kv"][..., 448:]).view(np.uint16)
    np.testing.assert_array_equal(rope, indep.f64_to_bf16(y[..., 448:]))
    # the largest magnitude maps to the top code 448
    top = np.abs(indep.e4m3_to_f64(r["kv"][..., :448])).max(-1)
    assert (top == 448.0).all()


def test_zero_entry_gets_unit_scale():
    a = np.zeros((1, 4, 512), np.uint16)
    z = np.zeros((1, 4, 512), np.float32)
    r = oracle.compress(a, z, np.zeros(4, np.float32), 4, False)
    assert r["kv_scale"][0, 0] == 1.0 and (r["kv"] == 0).all()


def test_tail_tokens_are_not_emitted_and_prev_block_is_required():
    inp = synth.compress_inputs(1, 10, 4, True, seed=9)
    r = oracle.compress(inp["a"], inp["za"], inp["bias"], 4, True, b=inp["b"], zb=inp["zb"])
    assert r["kv"].shape == (1, 2, 576)
    with pytest.raises(ValueError):
        oracle.compress(inp["a"], inp["za"], inp["bias"], 4, True, b=inp["b"], zb=inp["zb"],
                        pos0=8)  # a later chunk needs the previous block's tail
    with pytest.raises(ValueError):
        oracle.compress(inp["a"], inp["za"], inp["bias"], 4, True, b=inp["b"], zb=inp["zb"],
                        pos0=6)  # chunk start not on a block boundary
