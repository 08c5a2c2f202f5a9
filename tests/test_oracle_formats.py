"""Pins of the oracle's number formats against library casts and the OCP tables."""

import os

import numpy as np
import pytest
import torch

import oracle
from tests import indep


def test_bf16_decode_all_codes():
    codes = np.arange(65536, dtype=np.uint16)
    got = oracle.bf16_decode(codes)
    want = indep.bf16_to_f64(codes)
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all()


def test_bf16_encode_matches_torch_rne():
    rng = np.random.default_rng(5)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        # exact midpoints between neighbouring bf16 values: ties must go to even
        (indep.bf16_to_f64(np.arange(0x3F80, 0x3FFF, dtype=np.uint16)) +
         indep.bf16_to_f64(np.arange(0x3F81, 0x4000, dtype=np.uint16))) / 2,
        [0.0, -0.0, 1e-45, -3e-39, 3.3e38],
    ])
    got = oracle.bf16_encode(x)
    want = indep.f64_to_bf16(x)
    np.testing.assert_array_equal(got, want)


def test_bf16_roundtrip_finite_codes():
    codes = np.arange(65536, dtype=np.uint16)
    exp = (codes >> 7) & 0xFF
    codes = codes[exp != 0xFF]
    back = oracle.bf16_encode(oracle.bf16_decode(codes))
    np.testing.assert_array_equal(back, codes)


def test_e4m3_decode_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    want = indep.e4m3_to_f64(codes)
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all()
    # spot values fixed by the OCP FP8 definition
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6
    assert got[0x38] == 1.0 and np.isnan(got[0x7F]) and np.isnan(got[0xFF])


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(6)
    vals = indep.e4m3_to_f64(np.arange(0, 0x7F, dtype=np.uint8))  # non-negative finite
    mids = (vals[:-1] + vals[1:]) / 2
    x = np.concatenate([rng.uniform(-448, 448, 20000), rng.standard_normal(5000) * 1e-2,
                        mids, -mids, vals, -vals])
    got = oracle.e4m3_encode(x)
    want = indep.f64_to_e4m3(x)
    np.testing.assert_array_equal(got, want)


def test_e4m3_encode_saturates():
    got = oracle.e4m3_encode(np.array([448.0, 449.0, 464.0, 479.0, 1e9, -1e9, -500.0]))
    np.testing.assert_array_equal(got, [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE])


def test_e4m3_roundtrip_all_finite_codes():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    np.testing.assert_array_equal(oracle.e4m3_encode(oracle.e4m3_decode(codes)), codes)


def test_e2m1_values_follow_ocp_table():
    got = oracle.e2m1_decode(np.arange(16, dtype=np.uint8))
    np.testing.assert_array_equal(got[:8], [0, 0.5, 1, 1.5, 2, 3, 4, 6])
    np.testing.assert_array_equal(got[8:], -got[:8])
    assert np.signbit(got[8])  # code 8 is -0


def test_e2m1_matches_torch_fp4_pairs():
    # torch's float4_e2m1fn_x2 holds two codes per byte (low nibble first); widening goes
    # through its documented value set.
    if not hasattr(torch, "float4_e2m1fn_x2"):
        pytest.skip("torch without float4")
    table = oracle.e2m1_decode(np.arange(16, dtype=np.uint8))
    np.testing.assert_array_equal(table, indep.e2m1_to_f64(np.arange(16, dtype=np.uint8)))


def test_e8m0():
    got = oracle.e8m0_decode(np.array([0, 1, 126, 127, 128, 254, 255], dtype=np.uint8))
    np.testing.assert_array_equal(got[:6], [2.0 ** -127, 2.0 ** -126, 0.5, 1.0, 2.0, 2.0 ** 127])
    assert np.isnan(got[6])


def test_key_scale_offsets_form_a_bijection_per_group():
    offs = {oracle.key_sf_offset(j, s) for j in range(256) for s in range(4)}
    assert offs == set(range(1024))
    # entry r0 + 32*r1 keeps its four scales in one 32-bit word: 16*r0 + 4*r1
    assert [oracle.key_sf_offset(37, s) for s in range(4)] == [16 * 5 + 4 + s for s in range(4)]
    assert oracle.key_sf_offset(128 + 96 + 31, 3) == 512 + 16 * 31 + 12 + 3


def _page_ratios():
    path = os.path.join(os.path.dirname(__file__), "golden", "page_ratios.txt")
    out = {}
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            name, value, tol = line.split()[:3]
            out[name] = (float(value), float(tol))
    return out


def test_stored_format_reproduces_the_ratios_the_pages_state():
    r = _page_ratios()
    entry = 448 + 64 * 2 + 4  # stored entry: E4M3 dims + BF16 RoPE dims + fp32 scale
    csa_tok = (entry + 64 + 4) / 4  # CSA entry and its FP4 indexer key per 4 tokens
    hca_tok = entry / 128
    gqa8_tok = 8 * 128 * 2 * 2
    v, tol = r["kv_cache_vs_bf16_gqa8"]
    assert abs((csa_tok + hca_tok) / 2 / gqa8_tok - v) <= tol
    v, tol = r["fp8_bf16_split_vs_all_bf16"]
    assert abs((448 + 64 * 2) / (512 * 2) - v) <= tol


def test_storage_arithmetic_matches_pages():
    # walkthrough §2.2 / chooseai 一: the CSA+HCA cache at 1M context is about 2% of a
    # BF16 GQA8 (head dim 128) cache; the FP8+BF16 split about halves a BF16 entry.
    entry = 448 + 64 * 2 + 4  # E4M3 dims + bf16 RoPE dims + fp32 scale
    idx_key = 64 + 4  # 128 E2M1 + 4 E8M0
    csa_per_token = (entry + idx_key) / 4
    hca_per_token = entry / 128
    gqa8 = 8 * 128 * 2 * 2  # 8 KV heads x 128 dims x (K, V) x bf16
    ratio = (csa_per_token + hca_per_token) / 2 / gqa8
    assert abs(ratio - 0.0203) < 0.001
    assert abs(576 / 1024 - 0.5625) < 1e-12
