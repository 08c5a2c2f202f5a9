"""The seeded input generators draw what they promise (no GPU): E4M3 codes never NaN and
near the top of the range, E2M1 magnitudes from the table with balanced signs, E8M0 codes
in their stated range, the workloads' shapes and lengths, planted runs of 16 with large
keys, and a device generator that matches the host distributions."""

import numpy as np
import torch

from synth import inputs as synth


def test_e4m3_codes_never_nan_and_sit_near_the_top_of_the_range():
    rng = np.random.default_rng(0)
    c = synth.e4m3_codes(rng, (200000,))
    assert not ((c & 0x7F) == 0x7F).any()  # S.1111.111 is the NaN code
    exp = (c >> 3) & 15
    assert np.mean(exp >= 10) > 0.7  # the exponent field is drawn near its top


def test_sliced_generation_equals_one_pass_over_the_draws(monkeypatch):
    """The E4M3 and table-sampled codes do not depend on the slice length: a length that
    leaves a ragged last slice gives the same codes as one slice over the whole draw."""
    shape = (3, 1000, 448)
    monkeypatch.setattr(synth, "_CHUNK", 1 << 30)
    whole = synth.e4m3_codes(np.random.default_rng(7), shape)
    nib_whole = synth.e2m1_nibbles(np.random.default_rng(8), (5, 70001))
    monkeypatch.setattr(synth, "_CHUNK", 100003)
    np.testing.assert_array_equal(synth.e4m3_codes(np.random.default_rng(7), shape), whole)
    np.testing.assert_array_equal(synth.e2m1_nibbles(np.random.default_rng(8), (5, 70001)),
                                  nib_whole)
    # the codes are the sign, exponent and mantissa fields of the draws, S.1111.111 excluded
    assert whole.dtype == np.uint8 and not ((whole & 0x7F) == 0x7F).any()


def test_e2m1_magnitudes_follow_the_table_and_signs_are_balanced():
    rng = np.random.default_rng(1)
    nib = synth.e2m1_nibbles(rng, (400000,))
    freq = np.bincount(nib & 7, minlength=8) / nib.size
    np.testing.assert_allclose(freq, synth._E2M1_MAG_P / synth._E2M1_MAG_P.sum(), atol=0.005)
    assert abs(np.mean(nib >> 3) - 0.5) < 0.005


def test_e8m0_codes_stay_in_the_stated_range():
    c = synth.e8m0_codes(np.random.default_rng(2), (10000,))
    assert c.min() == 124 and c.max() == 130


def test_workload_shapes_and_lengths():
    w2 = synth.WORKLOADS[2]
    L = synth.seq_lengths(w2)
    assert len(L) == 32 and L.min() >= 65536 and L.max() <= 131072
    w3 = synth.WORKLOADS[3]
    assert (synth.seq_lengths(w3) == 1 << 20).all() and w3.k == 1024 and w3.H == 128


def test_planted_runs_are_runs_of_16_with_large_keys():
    rng = np.random.default_rng(3)
    n = np.array([4096], np.int32)
    ix = synth.indexer_inputs(rng, 1, 64, 4096, n, planted_runs=8)
    planted = ix["planted"][0]
    assert planted.sum() == 8 * 16
    starts = np.flatnonzero(np.diff(np.r_[0, planted.astype(int)]) == 1)
    assert len(starts) == 8 and (starts % 16 == 0).all()
    lo = ix["k_fp4"][0][planted] & 15
    assert ((lo & 7) >= 4).all()  # magnitudes from the four largest codes


def test_device_generator_matches_the_host_distributions():
    # same recipe, different random stream: compare summary statistics, not values
    host = synth.prefill_inputs(512, 256, 4, 64, 16, seed=5)
    dev = synth.prefill_inputs_device(512, 256, 4, 64, 16, seed=5, device="cpu")

    def f32(x):
        x = x.numpy() if torch.is_tensor(x) else x
        if x.dtype in (np.int16, np.uint16):
            return (x.astype(np.uint16).astype(np.uint32) << 16).view(np.float32)
        return x.astype(np.float32)

    for k in ("q", "a", "b"):
        h, d = f32(host[k]), f32(dev[k])
        assert abs(h.mean() - d.mean()) < 0.02 and abs(h.std() - d.std()) < 0.02, k
    for k in ("za", "zb", "w"):
        h, d = f32(host[k]), f32(dev[k])
        assert abs(h.mean() - d.mean()) < 0.05 and abs(h.std() - d.std()) < 0.05, k
    hq = np.bincount((host["q_fp4"] & 7).ravel(), minlength=8) / host["q_fp4"].size
    dq = np.bincount((dev["q_fp4"].numpy() & 7).ravel(), minlength=8) / dev["q_fp4"].numel()
    np.testing.assert_allclose(hq, dq, atol=0.01)
    assert dev["q_sf"].min() >= 124 and dev["q_sf"].max() <= 130
    for k in ("kv", "kv_scale", "k_fp4", "k_sf", "swa_prefix", "prev_b", "prev_zb"):
        assert tuple(dev[k].shape) == tuple(np.shape(host[k])), k
