"""Comparison rules between the CUDA path and the oracle (tolerances of the layer spec).

- fp32/bf16 outputs: max-abs <= 1e-2 and relative L2 <= 5e-3 against the fp64 oracle.
- stored E4M3/BF16 codes: bit-exact, except a code whose oracle value lies within 1e-5
  (relative) of a rounding midpoint; such flips are counted and returned. For the rotated
  BF16 dims "relative" means relative to the norm of the value's RoPE pair.
- top-k sets: bit-exact, unless the oracle's k-th and (k+1)-th scores are within 1e-6
  (relative) of each other; mismatches are then counted and returned.
"""

import numpy as np

from tests import indep

MAX_ABS = 1e-2
REL_L2 = 5e-3
MID_REL = 1e-5
TIE_REL = 1e-6

_E4M3_POS = np.sort(np.unique(indep.e4m3_to_f64(np.arange(0, 0x7F, dtype=np.uint8))))


def close(got, want, max_abs=MAX_ABS, rel_l2=REL_L2, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = got - want
    ma = float(np.abs(err).max()) if err.size else 0.0
    rl = float(np.linalg.norm(err) / max(np.linalg.norm(want), 1e-30)) if err.size else 0.0
    assert ma <= max_abs and rl <= rel_l2, f"{what}: max-abs {ma:.3e}, rel-L2 {rl:.3e}"
    return ma, rl


def _near_mid_e4m3(v):
    a = np.minimum(np.abs(v), 448.0)
    i = np.clip(np.searchsorted(_E4M3_POS, a) - 1, 0, len(_E4M3_POS) - 2)
    mid = (_E4M3_POS[i] + _E4M3_POS[i + 1]) / 2
    return np.abs(a - mid) <= MID_REL * np.maximum(a, 1e-30)


def _near_mid_bf16(v, ref):
    """`ref` is the magnitude the value was computed from: for a rotated dim, the norm of
    its RoPE pair (x0*cos - x1*sin can cancel, so the value itself is the wrong yardstick)."""
    f = np.abs(v).astype(np.float32)
    lo = (f.view(np.uint32) & 0xFFFF0000).view(np.float32).astype(np.float64)
    hi = ((f.view(np.uint32) & 0xFFFF0000) + 0x10000).view(np.float32).astype(np.float64)
    mid = (lo + hi) / 2
    a = np.abs(v)
    return np.abs(a - mid) <= MID_REL * np.maximum(np.maximum(a, ref), 1e-30)


def compare_entries(kv_gpu, scale_gpu, dbg_gpu, ora, what=""):
    """GPU compress output vs oracle.compress -> number of tolerated code flips."""
    y = ora["y"]
    close(dbg_gpu, y, what=f"{what} pre-quantisation")
    np.testing.assert_allclose(scale_gpu, ora["kv_scale"], rtol=1e-5, err_msg=what)
    v = y[..., :448] / ora["kv_scale"][..., None].astype(np.float64)
    diff = kv_gpu[..., :448] != ora["kv"][..., :448]
    flips = int(diff.sum())
    assert _near_mid_e4m3(v[diff]).all(), f"{what}: E4M3 code differs away from a midpoint"
    rg = np.ascontiguousarray(kv_gpu[..., 448:]).view(np.uint16)
    ro = np.ascontiguousarray(ora["kv"][..., 448:]).view(np.uint16)
    d2 = rg != ro
    flips2 = int(d2.sum())
    pair = np.hypot(y[..., 448::2], y[..., 449::2]).repeat(2, axis=-1)
    assert _near_mid_bf16(y[..., 448:][d2], pair[d2]).all(), \
        f"{what}: BF16 code differs away from a midpoint"
    return flips + flips2


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
