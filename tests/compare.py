"""Comparison rules between the CUDA path and the oracle (tolerances of the layer spec).

- fp32/bf16 outputs: max-abs <= 1e-2 and relative L2 <= 5e-3 against the fp64 oracle.
- stored E4M3/BF16 codes: bit-exact, except where the oracle's value v lies within
  delta = 1e-5 (relative) of a rounding midpoint. There the GPU's code must be the
  round-to-nearest-even code of some value in [v - delta, v + delta]: normally the other
  code of that midpoint, the neighbour of the oracle's code. Such flips are counted and
  returned. "Relative" is to the scale the fp32 value was computed at, which is not always
  the value itself: an E4M3 dim is a gated average of O(1) inputs that can cancel, then
  normalised by the row's RMS, so its fp32 error scales with the row's RMS (delta = 1e-5 x
  max(|v|, RMS of the row's v)); a rotated BF16 dim x0*cos - x1*sin is formed from a pair,
  so its error scales with the pair's norm (delta = 1e-5 x max(|v|, pair norm)). Where the
  value is tiny next to that scale the interval can span more than two codes, and the
  rule then admits exactly the codes that rounding of a value within that error can give.
- top-k sets: bit-exact, unless the oracle's k-th and (k+1)-th scores are within 1e-6
  (relative) of each other; mismatches are then counted and returned.
"""

import numpy as np

from tests import indep

MAX_ABS = 1e-2
REL_L2 = 5e-3
MID_REL = 1e-5
TIE_REL = 1e-6


def close(got, want, max_abs=MAX_ABS, rel_l2=REL_L2, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = got - want
    ma = float(np.abs(err).max()) if err.size else 0.0
    rl = float(np.linalg.norm(err) / max(np.linalg.norm(want), 1e-30)) if err.size else 0.0
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max-abs {ma:.3e}, rel-L2 {rl:.3e}"
    return ma, rl


def _ordinal(code, sign_bit):
    """Sign-magnitude codes -> integers in value order (+0 and -0 both 0)."""
    c = np.asarray(code, dtype=np.int64)
    mag = c & (sign_bit - 1)
    return np.where(c & sign_bit, -mag, mag)


def _e4m3_ordinal(x):
    return _ordinal(indep.f64_to_e4m3(np.clip(x, -448.0, 448.0)), 0x80)


def _bf16_ordinal(x):
    return _ordinal(indep.f64_to_bf16(x), 0x8000)


def _codes_in_window(got, v, delta, ordinal, sign_bit):
    """Every code of `got` is the rounding of some value within delta of v: its ordinal
    lies between those of RNE(v - delta) and RNE(v + delta)."""
    g = _ordinal(got, sign_bit)
    return (g >= ordinal(v - delta)) & (g <= ordinal(v + delta))


def check_codes(kv_gpu, kv_ora, y, scale, what=""):
    """Stored rows (E4M3 dims times `scale`, then BF16 dims) against the oracle's rows and
    its values y before quantisation -> number of codes that differ from the oracle's."""
    y = np.asarray(y, dtype=np.float64)
    v = y[..., :448] / np.asarray(scale, dtype=np.float64)[..., None]
    rms = np.sqrt(np.mean(v * v, axis=-1, keepdims=True)) * np.ones_like(v)
    g8, o8 = kv_gpu[..., :448], kv_ora[..., :448]
    d8 = g8 != o8
    delta8 = MID_REL * np.maximum(np.abs(v[d8]), rms[d8])
    ok8 = _codes_in_window(g8[d8], v[d8], delta8, _e4m3_ordinal, 0x80)
    if not ok8.all():
        i = int(np.flatnonzero(~ok8)[0])
        raise AssertionError(
            f"{what}: {int((~ok8).sum())} E4M3 codes are not a rounding of a value within the "
            f"midpoint tolerance of the oracle's (first: v = {v[d8][i]!r}, row RMS "
            f"{rms[d8][i]:.4g}, oracle code {int(o8[d8][i]):#04x}, GPU code "
            f"{int(g8[d8][i]):#04x})")
    rg = np.ascontiguousarray(kv_gpu[..., 448:]).view(np.uint16)
    ro = np.ascontiguousarray(kv_ora[..., 448:]).view(np.uint16)
    d2 = rg != ro
    yr = y[..., 448:]
    pair = np.hypot(y[..., 448::2], y[..., 449::2]).repeat(2, axis=-1)
    delta = MID_REL * np.maximum(np.abs(yr[d2]), pair[d2])
    ok2 = _codes_in_window(rg[d2], yr[d2], delta, _bf16_ordinal, 0x8000)
    if not ok2.all():
        i = int(np.flatnonzero(~ok2)[0])
        raise AssertionError(
            f"{what}: {int((~ok2).sum())} BF16 codes are not a rounding of a value within the "
            f"midpoint tolerance of the oracle's (first: v = {yr[d2][i]!r}, pair norm "
            f"{pair[d2][i]:.4g}, oracle code {int(ro[d2][i]):#06x}, GPU code "
            f"{int(rg[d2][i]):#06x})")
    return int(d8.sum()) + int(d2.sum())


def _e2m1_ordinal(x):
    """Nearest E2M1 value of x (brute force over the OCP magnitudes, ties to the code with
    an even mantissa bit, saturating at 6) as a signed ordinal."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), 6.0)
    d = np.abs(indep.E2M1_TABLE[None, :] - a.reshape(-1, 1))
    cand = d == d.min(axis=1, keepdims=True)
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    code = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1)).reshape(x.shape)
    return np.where(np.signbit(x), -code, code)


def unpack_nibbles(packed):
    """[..., 64] bytes -> [..., 128] E2M1 codes (element 2i in the low nibble of byte i)."""
    return indep.unpack_fp4(packed)


def check_mxfp4(g_codes, o_codes, g_sf, o_sf, y, mid_rel=MID_REL, sf_rel=1e-6, what=""):
    """MXFP4 blocks: codes [nblk][32] and E8M0 scales [nblk] of the GPU and of the oracle,
    the oracle's values y [nblk][32] -> number of differing codes and scales. A scale may
    differ only where the block maximum sits at a power of two (floor(log2) then depends
    on the last bit); where the scales agree, every element code must be the E2M1 rounding
    of a value within mid_rel of the oracle's y / 2^e."""
    g_codes, o_codes = np.asarray(g_codes), np.asarray(o_codes)
    y = np.asarray(y, dtype=np.float64)
    flips = 0
    sd = np.asarray(g_sf) != np.asarray(o_sf)
    if sd.any():
        amax = np.abs(y[sd]).max(axis=1)
        l2 = np.log2(np.maximum(amax, 1e-300))
        assert ((amax > 0) & (np.abs(l2 - np.round(l2)) < sf_rel)).all(), \
            f"{what}: a block scale differs away from a power-of-two maximum"
        flips += int(sd.sum())
    keep = ~sd
    X = np.ldexp(1.0, np.asarray(o_sf, dtype=np.int64)[keep] - 127)[:, None]
    r = y[keep] / X
    d = g_codes[keep] != o_codes[keep]
    if d.any():
        gc = g_codes[keep][d].astype(np.int64)
        go = np.where(gc & 8, -(gc & 7), gc & 7)
        rv = r[d]
        delta = mid_rel * np.abs(rv)
        ok = (go >= _e2m1_ordinal(rv - delta)) & (go <= _e2m1_ordinal(rv + delta))
        assert ok.all(), (f"{what}: {int((~ok).sum())} E2M1 codes are not a rounding of a "
                          "value within the midpoint tolerance of the oracle's")
        flips += int(d.sum())
    return flips


def compare_entries(kv_gpu, scale_gpu, dbg_gpu, ora, what=""):
    """GPU compress output vs oracle.compress -> number of tolerated code flips."""
    y = ora["y"]
    close(dbg_gpu, y, what=f"{what} pre-quantisation")
    np.testing.assert_allclose(scale_gpu, ora["kv_scale"], rtol=1e-5, err_msg=what)
    return check_codes(kv_gpu, ora["kv"], y, ora["kv_scale"], what)


def compare_topk(idx_gpu, scores_ora, n, k, what=""):
    """One sequence -> number of tolerated mismatching indices."""
    s = np.asarray(scores_ora[:n], dtype=np.float64)
    order = np.lexsort((np.arange(n), -s))
    keep = min(k, n)
    want = np.sort(order[:keep])
    got = np.asarray(idx_gpu)
    assert (got[keep:] == -1).all(), f"{what}: padding"
    g = got[:keep]
    assert (np.diff(g) > 0).all(), f"{what}: not strictly ascending"
    if np.array_equal(g, want):
        return 0
    assert n > k, what
    sk, sk1 = s[order[k - 1]], s[order[k]]
    assert abs(sk - sk1) <= TIE_REL * abs(sk), \
        f"{what}: sets differ but the k-th/(k+1)-th gap {abs(sk - sk1) / abs(sk):.2e} is wide"
    extra = np.setdiff1d(g, want)
    assert (s[extra] >= sk * (1 - 10 * TIE_REL)).all(), f"{what}: a chosen entry is far below the k-th"
    return int(len(extra))


def _bf16_round(x):
    import torch
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).to(
        torch.float64).numpy()


def compare_topk_bf16(idx_gpu, scores_ora, n, k, what=""):
    """One sequence of the BF16-score selection -> number of tolerated mismatches.
    The GPU rounds its fp32 score to BF16, the oracle its fp64 score, so an entry whose
    score sits next to a BF16 rounding midpoint may land one BF16 step apart; the sets may
    differ only in entries within one BF16 step of the boundary value."""
    import oracle
    want = oracle.topk_bf16(np.asarray(scores_ora[:n], dtype=np.float64), n, k)
    got = np.asarray(idx_gpu)
    keep = min(k, n)
    assert (got[keep:] == -1).all(), f"{what}: padding"
    g = got[:keep]
    assert (np.diff(g) > 0).all(), f"{what}: not strictly ascending"
    if np.array_equal(g, want[:keep]):
        return 0
    assert n > k, what
    r = _bf16_round(scores_ora[:n])
    rk = np.sort(r)[::-1][k - 1]
    step = np.abs(rk) * 2.0 ** -7
    diff = np.setxor1d(g, want[:keep])
    assert (np.abs(r[diff] - rk) <= step).all(), \
        f"{what}: a differing entry is more than one BF16 step from the boundary"
    return int(len(diff))
