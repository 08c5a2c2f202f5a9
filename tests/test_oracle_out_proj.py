"""Pins of the oracle's grouped output projection."""

import numpy as np

import oracle
from synth import inputs as synth
from tests import indep


def _case(T, H, G, d_g, d_model, seed):
    rng = np.random.default_rng(seed)
    attn = synth.bf16_normal(rng, (T, H, 512))
    Wg = synth.bf16_normal(rng, (G, d_g, H // G * 512), std=(H // G * 512) ** -0.5)
    Wo = synth.bf16_normal(rng, (d_model, G * d_g), std=(G * d_g) ** -0.5)
    return attn, Wg, Wo


def test_groups_equal_one_block_diagonal_projection():
    # an independent statement: the group projections are one projection of the whole
    # head vector by the block-diagonal matrix diag(Wg[0], ..., Wg[G-1]), done by numpy
    T, H, G, d_g, d_model = 9, 16, 4, 32, 48
    attn, Wg, Wo = _case(T, H, G, d_g, d_model, 1)
    out, mid = oracle.grouped_out_proj(attn, Wg, Wo)
    K1 = H // G * 512
    D = np.zeros((G * d_g, H * 512))
    for g in range(G):
        D[g * d_g:(g + 1) * d_g, g * K1:(g + 1) * K1] = indep.bf16_to_f64(Wg[g])
    x = indep.bf16_to_f64(attn).reshape(T, H * 512)
    m = x @ D.T
    # mid is the BF16 rounding of the block-diagonal product
    np.testing.assert_allclose(mid, m, rtol=2.0 ** -8, atol=1e-12)
    np.testing.assert_array_equal(oracle.bf16_decode(oracle.bf16_encode(mid)), mid)
    np.testing.assert_allclose(out, mid @ indep.bf16_to_f64(Wo).T, rtol=1e-12, atol=1e-12)


def test_single_group_is_a_plain_two_layer_projection():
    T, H, d_g, d_model = 5, 8, 64, 96
    attn, Wg, Wo = _case(T, H, 1, d_g, d_model, 2)
    out, mid = oracle.grouped_out_proj(attn, Wg, Wo)
    m = indep.bf16_to_f64(attn).reshape(T, -1) @ indep.bf16_to_f64(Wg[0]).T
    assert (np.abs(mid - m) <= np.abs(m) * 2.0 ** -8 + 1e-300).all()
    np.testing.assert_allclose(out, mid @ indep.bf16_to_f64(Wo).T, rtol=1e-12, atol=1e-12)
