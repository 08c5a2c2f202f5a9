"""How far the drawn inputs sit from the recipe they stand in for (no GPU).

The 1M-token caches cannot be made by the fp64 oracle's compression in a test's time, so
the generators draw stored codes directly. These tests bound the departure on sizes the
oracle finishes in seconds: the drawn KV entries dequantise to the same scale as the
oracle's compression of N(0, 1) token streams, the drawn E2M1 magnitudes follow the
oracle's MXFP4 encoding of N(0, 1) blocks, and the drawn queries have the per-head RMS
that the recipe's RMSNorm would give them."""

import numpy as np

import oracle
from synth import inputs as synth


def _rms(x):
    return float(np.sqrt(np.mean(np.square(x, dtype=np.float64))))


def test_drawn_kv_entries_have_the_scale_of_compressed_ones():
    ci = synth.compress_inputs(B=1, T=4096, m=4, overlap=True, seed=11)
    comp = oracle.compress(ci["a"], ci["za"], ci["bias"], 4, True, b=ci["b"], zb=ci["zb"])
    kv, sc = synth.kv_cache(np.random.default_rng(12), 1, 1024)
    made = oracle.dequant_rows(comp["kv"][0], comp["kv_scale"][0])
    drawn = oracle.dequant_rows(kv[0], sc[0])
    # both parts of the row: the E4M3 dims and the BF16 RoPE dims
    for lo, hi in ((0, 448), (448, 512)):
        assert abs(_rms(drawn[:, lo:hi]) / _rms(made[:, lo:hi]) - 1) < 0.06
    # the per-entry scales overlap: the drawn range covers the bulk of the compressed ones
    s = comp["kv_scale"][0]
    assert np.mean((s >= 0.004) & (s < 0.012)) > 0.8
    # E4M3 exponent fields: same top-heavy shape, the drawn one somewhat wider
    ex_made = np.bincount((comp["kv"][0, :, :448] >> 3).ravel() & 15, minlength=16)
    ex_drawn = np.bincount((kv[0, :, :448] >> 3).ravel() & 15, minlength=16)
    p, q = ex_made / ex_made.sum(), ex_drawn / ex_drawn.sum()
    assert 0.5 * np.abs(p - q).sum() < 0.3
    assert p[10:].sum() > 0.9 and q[10:].sum() > 0.7


def test_drawn_e2m1_magnitudes_follow_mxfp4_of_unit_normal_blocks():
    rng = np.random.default_rng(13)
    mags, scales = [], []
    for _ in range(1500):
        codes, e = oracle.mxfp4_block(rng.standard_normal(32))
        mags.append(codes & 7)
        scales.append(e)
    made = np.bincount(np.concatenate(mags), minlength=8) / (1500 * 32)
    drawn = synth._E2M1_MAG_P / synth._E2M1_MAG_P.sum()
    assert 0.5 * np.abs(made - drawn).sum() < 0.1
    # the recipe's scale codes sit at 125..127; the drawn ones (124..130) contain them
    assert set(scales) <= set(range(124, 131))


def test_drawn_queries_have_unit_rms_per_head():
    w = synth.WORKLOADS[0]
    d = synth.decode_inputs(w)
    q = oracle.bf16_decode(d["q"]).reshape(-1, 512)
    r = np.sqrt(np.mean(q * q, axis=1))
    # RMSNorm would set every head's RMS to 1 exactly; the drawn heads are within a few %
    assert np.all(np.abs(r - 1) < 0.15) and abs(r.mean() - 1) < 0.02
