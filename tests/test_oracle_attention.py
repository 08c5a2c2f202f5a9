"""Pins of the oracle's shared-KV MQA (window, sink, de-rotation) and of the prefill."""

import numpy as np
import pytest

import oracle
from synth import inputs as synth
from tests import indep

TAU = 1.0 / np.sqrt(512.0)


def _small_decode(seed=0, B=2, H=4, Nmax=256, L=(700, 1000), m=4):
    rng = np.random.default_rng(seed)
    L = np.array(L[:B])
    n = (L // m).astype(np.int32)
    kv, sc = synth.kv_cache(rng, B, Nmax)
    return {
        "q": synth.bf16_normal(rng, (B, H, 512)), "pos": (L - 1).astype(np.int32),
        "n": n, "kv": kv, "sc": sc, "swa": synth.bf16_normal(rng, (B, 128, 512)),
        "sink": rng.standard_normal(H).astype(np.float32),
    }


def _window_rows(swa_b, t):
    ps = np.arange(max(0, t - 127), t + 1)
    return indep.bf16_to_f64(swa_b[ps % 128])


def _textbook(d, rows_of, sink_zero_value_row=True):
    """softmax over [sink, rows] with the sink as a row of value zero."""
    B, H, _ = d["q"].shape
    out = np.empty((B, H, 512)); lse = np.empty((B, H))
    for b in range(B):
        V = rows_of(b)
        q = indep.bf16_to_f64(d["q"][b])
        logits = TAU * q @ V.T
        full = np.concatenate([d["sink"].astype(np.float64)[:, None], logits], 1)
        p = indep.softmax(full, axis=1)
        out[b] = p[:, 1:] @ V
        lse[b] = np.log(np.exp(full - full.max(1, keepdims=True)).sum(1)) + full.max(1)
    return out, lse


def test_dense_hca_equals_textbook_softmax_with_window_and_sink():
    d = _small_decode(1)

    def rows(b):
        ent = indep.dequant_rows(d["kv"][b, : d["n"][b]], d["sc"][b, : d["n"][b]])
        return np.concatenate([ent, _window_rows(d["swa"][b], d["pos"][b])])

    got, lse = oracle.attention(d["q"], d["pos"], d["n"], d["kv"], d["sc"], d["swa"],
                                d["sink"], derotate=False)
    want, wlse = _textbook(d, rows)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, wlse, rtol=1e-12)


def test_sink_minus_inf_restores_plain_softmax():
    d = _small_decode(2)
    d["sink"][:] = -np.inf
    idx = np.stack([np.sort(np.random.default_rng(b).choice(d["n"][b], 33, replace=False))
                    for b in range(2)]).astype(np.int32)

    def rows(b):
        ent = indep.dequant_rows(d["kv"][b, idx[b]], d["sc"][b, idx[b]])
        return np.concatenate([ent, _window_rows(d["swa"][b], d["pos"][b])])

    got, _ = oracle.attention(d["q"], d["pos"], d["n"], d["kv"], d["sc"], d["swa"], d["sink"],
                              idx=idx, derotate=False)
    for b in range(2):
        V = rows(b)
        p = indep.softmax(TAU * indep.bf16_to_f64(d["q"][b]) @ V.T, axis=1)
        np.testing.assert_allclose(got[b], p @ V, rtol=1e-10, atol=1e-12)


def test_probabilities_and_sink_sum_to_one():
    d = _small_decode(3)
    _, lse = oracle.attention(d["q"], d["pos"], d["n"], d["kv"], d["sc"], d["swa"], d["sink"],
                              derotate=False)
    for b in range(2):
        V = np.concatenate([indep.dequant_rows(d["kv"][b, : d["n"][b]], d["sc"][b, : d["n"][b]]),
                            _window_rows(d["swa"][b], d["pos"][b])])
        logits = TAU * indep.bf16_to_f64(d["q"][b]) @ V.T
        total = np.exp(d["sink"] - lse[b]) + np.exp(logits - lse[b][:, None]).sum(1)
        np.testing.assert_allclose(total, 1.0, rtol=1e-12)


def test_sink_plus_inf_gives_zero_output():
    d = _small_decode(4)
    d["sink"][1] = np.inf
    got, lse = oracle.attention(d["q"], d["pos"], d["n"], d["kv"], d["sc"], d["swa"], d["sink"])
    assert (got[:, 1] == 0).all() and np.isinf(lse[:, 1]).all()
    assert (np.abs(got[:, 0]).sum(-1) > 0).all()


def test_topk_covering_all_entries_reduces_csa_to_hca():
    d = _small_decode(5)
    k = 300
    idx = np.full((2, k), -1, np.int32)
    for b in range(2):
        idx[b, : d["n"][b]] = np.arange(d["n"][b])
    dense = oracle.attention(d["q"], d["pos"], d["n"], d["kv"], d["sc"], d["swa"], d["sink"])
    sparse = oracle.attention(d["q"], d["pos"], d["n"], d["kv"], d["sc"], d["swa"], d["sink"],
                              idx=idx)
    np.testing.assert_array_equal(dense[0], sparse[0])
    np.testing.assert_array_equal(dense[1], sparse[1])


def test_row_order_does_not_matter():
    d = _small_decode(6)
    rng = np.random.default_rng(0)
    idx = np.stack([np.sort(rng.choice(d["n"][b], 50, replace=False)) for b in range(2)])
    perm = np.stack([rng.permutation(r) for r in idx]).astype(np.int32)
    a = oracle.attention(d["q"], d["pos"], d["n"], d["kv"], d["sc"], d["swa"], d["sink"],
                         idx=idx.astype(np.int32))
    b = oracle.attention(d["q"], d["pos"], d["n"], d["kv"], d["sc"], d["swa"], d["sink"],
                         idx=perm)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-12, atol=1e-14)


def test_derotation_undoes_the_query_position_turn():
    d = _small_decode(7)
    plain, _ = oracle.attention(d["q"], d["pos"], d["n"], d["kv"], d["sc"], d["swa"],
                                d["sink"], derotate=False)
    der, _ = oracle.attention(d["q"], d["pos"], d["n"], d["kv"], d["sc"], d["swa"], d["sink"],
                              derotate=True)
    np.testing.assert_array_equal(der[..., :448], plain[..., :448])
    for b in range(2):
        t = d["pos"][b]
        zp = plain[b, :, 448::2] + 1j * plain[b, :, 449::2]
        zd = der[b, :, 448::2] + 1j * der[b, :, 449::2]
        # pair 0 turns by -t rad, pair 16 by -t/100
        for j, f in ((0, 1.0), (16, 0.01)):
            np.testing.assert_allclose(zd[:, j], zp[:, j] * np.exp(-1j * t * f), rtol=1e-9,
                                       atol=1e-14)


def test_early_position_sees_only_t_plus_one_window_rows():
    d = _small_decode(8, L=(3, 60), Nmax=128)
    d["sink"][:] = -np.inf
    # poison the ring slots a query at t must not see
    for b in range(2):
        d["swa"][b, d["pos"][b] + 1:] = 0x7FC0  # bf16 NaN
    out, _ = oracle.attention(d["q"], d["pos"], d["n"], d["kv"], d["sc"], d["swa"], d["sink"])
    assert np.isfinite(out).all()


def test_bad_index_is_rejected():
    d = _small_decode(9)
    idx = np.zeros((2, 4), np.int32)
    idx[1, 2] = d["n"][1]  # not eligible
    with pytest.raises(ValueError):
        oracle.attention(d["q"], d["pos"], d["n"], d["kv"], d["sc"], d["swa"], d["sink"], idx=idx)


# ----------------------------------------------------------------- prefill
@pytest.mark.parametrize("weighted,strict", [(False, False), (True, False), (False, True)])
def test_prefill_row_matches_independent_recomputation(weighted, strict):
    P, T, m, H, H_I, k = 512, 64, 4, 2, 4, 40
    inp = synth.prefill_inputs(P, T, m, H, H_I, seed=10)
    norm_w = None
    if weighted:  # the optional RMSNorm weight reaches the entries and the window rows
        norm_w = np.random.default_rng(10).uniform(0.5, 2.0, 512).astype(np.float32)
        inp["norm_w"] = norm_w
    rows = [0, 1, 3, 4, 31, 63]
    r = oracle.prefill(inp, k, rows, strict=strict)
    # the new entries match a stand-alone compression of the new tokens
    comp = oracle.compress(inp["a"][None], inp["za"][None], inp["bias"], m, True,
                           b=inp["b"][None], zb=inp["zb"][None], pos0=P,
                           prev_b=inp["prev_b"][None], prev_zb=inp["prev_zb"][None],
                           norm_w=norm_w)
    n0 = P // m
    np.testing.assert_array_equal(r["kv"][n0:n0 + T // m], comp["kv"][0])
    np.testing.assert_array_equal(r["kv"][:n0], inp["kv"][:n0])
    Nmax = inp["Nmax"]
    ks = indep.key_scales(inp["k_sf"], Nmax)
    kdec = indep.e2m1_to_f64(indep.unpack_fp4(inp["k_fp4"])) * np.repeat(
        indep.e8m0_to_f64(ks), 32, -1)
    for i, row in enumerate(rows):
        t = P + row
        # inclusive: the block whose last token is t counts; strict: blocks ending before t
        n = t // m if strict else (t + 1) // m
        q = indep.e2m1_to_f64(indep.unpack_fp4(inp["q_fp4"][row])) * np.repeat(
            indep.e8m0_to_f64(inp["q_sf"][row]), 32, -1)
        s = np.maximum(kdec[:n] @ q.T, 0) @ inp["w"][row].astype(np.float64)
        order = np.lexsort((np.arange(n), -s))
        sel = np.sort(order[:k])
        assert (r["idx"][i, : len(sel)] == sel).all() and (r["idx"][i, len(sel):] == -1).all()
        ent = indep.dequant_rows(r["kv"][sel], r["kv_scale"][sel])
        win = []
        for p in range(t - 127, t + 1):
            if p < P:
                win.append(indep.bf16_to_f64(inp["swa_prefix"][p % 128]))
            else:
                win.append(indep.bf16_to_f64(oracle.swa_row(inp["a"][p - P], p,
                                                            norm_w=norm_w)))
        V = np.concatenate([ent, np.array(win)])
        qh = indep.bf16_to_f64(inp["q"][row])
        full = np.concatenate([inp["sink"].astype(np.float64)[:, None], TAU * qh @ V.T], 1)
        o = indep.softmax(full, 1)[:, 1:] @ V
        z = (o[:, 448::2] + 1j * o[:, 449::2]) * np.exp(
            -1j * t * 10000.0 ** (-np.arange(32) / 32.0))
        o[:, 448::2], o[:, 449::2] = z.real, z.imag
        np.testing.assert_allclose(r["out"][i], o, rtol=1e-9, atol=1e-12)


def test_prefill_eligibility_counts_the_block_ending_at_t():
    P, T, m = 0, 16, 4
    inp = synth.prefill_inputs(P, T, m, 1, 2, seed=11)
    r = oracle.prefill(inp, 100, list(range(T)))
    for t in range(T):
        sel = r["idx"][t]
        assert (sel >= 0).sum() == (t + 1) // m
        assert sel[sel >= 0].max(initial=-1) == (t + 1) // m - 1


def test_prefill_strict_eligibility_takes_blocks_completed_before_t():
    # "completed before t": block i (tokens m*i .. m*i+m-1) is visible at t iff
    # m*i + m - 1 < t; the block closing at t itself is not. Counted by hand for m = 4:
    # t = 0..4 see 0 blocks, t = 4 is the first to see block 0 (its last token is 3).
    P, T, m = 0, 16, 4
    inp = synth.prefill_inputs(P, T, m, 1, 2, seed=11)
    r = oracle.prefill(inp, 100, list(range(T)), strict=True)
    want = [0, 0, 0, 0, 1, 1, 1, 1, 2, 2, 2, 2, 3, 3, 3, 3]
    for t in range(T):
        sel = r["idx"][t]
        assert (sel >= 0).sum() == want[t]
        assert sel[sel >= 0].max(initial=-1) == want[t] - 1


def test_prefill_strict_row_at_t_equals_inclusive_row_at_t_minus_1_selection():
    # with k >= n the set is every eligible entry, so under the strict reading the set at
    # t is the inclusive reading's set at t - 1 (floor(t/m) = floor(((t-1)+1)/m))
    P, T, m = 64, 40, 4
    inp = synth.prefill_inputs(P, T, m, 2, 2, seed=13)
    rows = list(range(1, T))
    s = oracle.prefill(inp, 64, rows, strict=True)
    i = oracle.prefill(inp, 64, [r - 1 for r in rows])
    np.testing.assert_array_equal(s["idx"], i["idx"])


def test_swa_row_at_position_zero_is_the_normalised_token():
    rng = np.random.default_rng(12)
    a = synth.bf16_normal(rng, 512)
    x = indep.bf16_to_f64(a)
    want = indep.f64_to_bf16(x / np.sqrt(np.mean(x * x) + 1e-6))
    np.testing.assert_array_equal(oracle.swa_row(a, 0), want)


def test_online_blocking_over_any_split_equals_the_oracle():
    # P-11: merging running (max, sum, output) over arbitrary blocks of the row list, the
    # sink entering only the denominator, reproduces the oracle's result to 1e-12
    d = _small_decode(9)
    rng = np.random.default_rng(9)
    got, lse = oracle.attention(d["q"], d["pos"], d["n"], d["kv"], d["sc"], d["swa"],
                                d["sink"], derotate=False)
    for b in range(2):
        ent = indep.dequant_rows(d["kv"][b, : d["n"][b]], d["sc"][b, : d["n"][b]])
        V = np.concatenate([ent, _window_rows(d["swa"][b], d["pos"][b])])
        q = indep.bf16_to_f64(d["q"][b])
        for _ in range(3):
            perm = rng.permutation(len(V))
            cuts = np.sort(rng.choice(np.arange(1, len(V)), size=7, replace=False))
            M = np.full(q.shape[0], -np.inf)
            S = np.zeros(q.shape[0])
            O = np.zeros((q.shape[0], 512))
            for blk in np.split(perm, cuts):
                lg = TAU * q @ V[blk].T
                mb = lg.max(1)
                Mn = np.maximum(M, mb)
                a = np.exp(M - Mn)
                e = np.exp(lg - Mn[:, None])
                S = S * a + e.sum(1)
                O = O * a[:, None] + e @ V[blk]
                M = Mn
            sink = d["sink"].astype(np.float64)
            Z = S + np.exp(sink - M)
            np.testing.assert_allclose(O / Z[:, None], got[b], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(M + np.log(Z), lse[b], rtol=1e-12)
