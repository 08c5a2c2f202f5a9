"""CUDA prefill (csa_prefill) vs the fp64 oracle's prefill on seeded inputs (needs a B200)."""

import numpy as np
import pytest
import torch

import oracle
from synth import inputs as synth
from tests import compare

pytestmark = pytest.mark.gpu

csa = pytest.importorskip("long_context_compressed_layer_b200")


def dev(x):
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        x = x.view(np.int16)
    return torch.from_numpy(x).cuda()


def host(t):
    return t.cpu().numpy()


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    csa.lib()


def run_prefill(inp, k, derotate=True, strict=False):
    kv, sc = dev(inp["kv"]), dev(inp["kv_scale"])
    opt = {x: dev(inp[x]) for x in ("prev_b", "prev_zb", "norm_w") if x in inp}
    if inp["P"] > 0:
        opt["swa_prefix"] = dev(inp["swa_prefix"])
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, idx = csa.prefill(
        inp["P"], inp["m"], k, a=dev(inp["a"]), b=dev(inp["b"]), za=dev(inp["za"]),
        zb=dev(inp["zb"]), bias=dev(inp["bias"]), kv=kv, kv_scale=sc, q_fp4=dev(inp["q_fp4"]),
        q_sf=dev(inp["q_sf"]), w=dev(inp["w"]), k_fp4=dev(inp["k_fp4"]), k_sf=dev(inp["k_sf"]),
        q=dev(inp["q"]), sink=dev(inp["sink"]), derotate=derotate,
        strict_eligibility=strict, lse=True, idx=True,
        dev_status=st, **opt)
    torch.cuda.synchronize()
    assert int(st.item()) == 0, f"device status {int(st.item())}"
    return dict(out=out.float().cpu().numpy(), lse=host(lse), idx=host(idx), kv=host(kv),
                kv_scale=host(sc))


def check_rows(inp, k, got, rows, ora, strict=False):
    P, m = inp["P"], inp["m"]
    flips = 0
    for i, r in enumerate(rows):
        n = (P + r + (0 if strict else 1)) // m
        s = oracle.indexer_scores(np.array([n], np.int32), inp["q_fp4"][r:r + 1],
                                  inp["q_sf"][r:r + 1], inp["w"][r:r + 1],
                                  inp["k_fp4"][None], inp["k_sf"][None])[0]
        flips += compare.compare_topk(got["idx"][r], s, n, k, what=f"row {r}")
    assert flips <= 2
    compare.close(got["out"][rows], ora["out"], what="prefill out")
    np.testing.assert_allclose(got["lse"][rows], ora["lse"], rtol=1e-4, atol=1e-4)


def check_cache(inp, got, ora):
    P, T, m = inp["P"], inp["T"], inp["m"]
    n0, n1 = P // m, (P + T) // m
    np.testing.assert_array_equal(got["kv"][:n0], inp["kv"][:n0])  # prefix rows untouched
    np.testing.assert_allclose(got["kv_scale"][n0:n1], ora["kv_scale"][n0:n1], rtol=1e-5)
    if n1 == n0:
        return
    # the oracle's values before quantisation: its compression of the new tokens
    comp = oracle.compress(inp["a"][None], inp["za"][None], inp["bias"], m, True,
                           b=inp["b"][None], zb=inp["zb"][None], pos0=P,
                           prev_b=inp["prev_b"][None] if P else None,
                           prev_zb=inp["prev_zb"][None] if P else None,
                           norm_w=inp.get("norm_w"))
    np.testing.assert_array_equal(comp["kv"][0], ora["kv"][n0:n1])
    flips = compare.check_codes(got["kv"][n0:n1], ora["kv"][n0:n1], comp["y"][0],
                                ora["kv_scale"][n0:n1], what="prefill cache rows")
    assert flips <= max(4, (n1 - n0) * 576 // 5000), f"{flips} stored codes differ"


@pytest.mark.parametrize("P,T,H,H_I,k", [
    (512, 301, 64, 16, 64),     # a tail of one token; every row checked
    (4096, 160, 128, 64, 1024), # n(t) around k: the set is everything, then a true top-k
])
def test_prefill_small_all_rows(P, T, H, H_I, k):
    inp = synth.prefill_inputs(P, T, 4, H, H_I, seed=P + T)
    got = run_prefill(inp, k)
    rows = np.arange(T, dtype=np.int32)
    ora = oracle.prefill(inp, k, rows)
    check_cache(inp, got, ora)
    check_rows(inp, k, got, rows, ora)


@pytest.mark.parametrize("P,T,H,H_I,k", [
    (0, 300, 64, 16, 64),       # from an empty prefix: t = 0..3 see nothing, t = 4 block 0
    (4096, 160, 128, 64, 1024), # n(t) = floor(t/m) around k
])
def test_prefill_strict_eligibility_all_rows(P, T, H, H_I, k):
    # the reading "only blocks completed before t": n(t) = floor(t/m)
    inp = synth.prefill_inputs(P, T, 4, H, H_I, seed=P + T + 1)
    got = run_prefill(inp, k, strict=True)
    rows = np.arange(T, dtype=np.int32)
    ora = oracle.prefill(inp, k, rows, strict=True)
    check_cache(inp, got, ora)
    check_rows(inp, k, got, rows, ora, strict=True)
    n = (P + rows) // 4
    assert ((got["idx"] >= 0).sum(axis=1) == np.minimum(n, k)).all()


def test_prefill_with_rmsnorm_weight():
    # the optional RMSNorm weight reaches the new entries and the new window rows
    inp = synth.prefill_inputs(512, 200, 4, 64, 16, seed=23)
    inp["norm_w"] = np.random.default_rng(23).uniform(0.5, 2.0, 512).astype(np.float32)
    got = run_prefill(inp, 64)
    rows = np.array([0, 1, 2, 3, 100, 127, 128, 199], np.int32)
    ora = oracle.prefill(inp, 64, rows)
    check_cache(inp, got, ora)
    check_rows(inp, 64, got, rows, ora)


def test_prefill_from_empty_prefix_over_two_query_chunks():
    # P = 0: the first queries see no entry at all (n = 0) and a short window; 1100 queries
    # span two launches of 1024
    inp = synth.prefill_inputs(0, 1100, 4, 128, 32, seed=11)
    got = run_prefill(inp, 128)
    rows = np.array([0, 1, 2, 3, 4, 5, 127, 128, 511, 512, 1022, 1023, 1024, 1025, 1099],
                    np.int32)
    ora = oracle.prefill(inp, 128, rows)
    check_cache(inp, got, ora)
    check_rows(inp, 128, got, rows, ora)
    assert (got["idx"][0] == -1).all() and (got["idx"][4][1:] == -1).all()


def test_prefill_long_prefix_sampled_rows():
    # the 1M-class shape scaled down: H = 128, H_I = 64, k = 1024, n(t) ~ 4.1-4.5K
    P, T, k = 16384, 1536, 1024
    inp = synth.prefill_inputs(P, T, 4, 128, 64, seed=4)
    got = run_prefill(inp, k)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1, 2, 3, 1023, 1024, T - 1],
                                     rng.choice(T, 17, replace=False)])).astype(np.int32)
    ora = oracle.prefill(inp, k, rows)
    check_cache(inp, got, ora)
    check_rows(inp, k, got, rows, ora)


def test_prefill_without_derotation_and_deterministic():
    inp = synth.prefill_inputs(1024, 200, 4, 64, 16, seed=9)
    a = run_prefill(inp, 128, derotate=False)
    b = run_prefill(inp, 128, derotate=False)
    for key in ("out", "lse", "idx", "kv"):
        np.testing.assert_array_equal(a[key], b[key])
    rows = np.array([0, 57, 199], np.int32)
    ora = oracle.prefill(inp, 128, rows, derotate=False)
    check_rows(inp, 128, a, rows, ora)


def _host_inputs(d, rows):
    """Host copies of a device-drawn prefill bundle for the oracle: every input except the
    queries, which only the sampled rows need (the rest of the array stays untouched
    zero pages)."""
    def h(x):
        x = x.cpu().numpy()
        return x.view(np.uint16) if x.dtype == np.int16 else x

    inp = {k: d[k] for k in ("P", "T", "m", "H", "H_I", "Nmax")}
    for k in ("kv", "kv_scale", "k_fp4", "k_sf", "q_fp4", "q_sf", "w", "sink", "swa_prefix",
              "a", "b", "za", "zb", "bias", "prev_b", "prev_zb"):
        if k in d:
            inp[k] = h(d[k])
    q = np.zeros(tuple(d["q"].shape), dtype=np.uint16)
    idx = torch.as_tensor(rows, dtype=torch.long, device=d["q"].device)
    q[rows] = h(d["q"].index_select(0, idx))
    inp["q"] = q
    return inp


@pytest.mark.slow
def test_prefill_full_size_sampled_rows():
    # the 64K-token prefill after a 192K-token prefix, as bench.py --workload prefill runs
    # it, checked on rows at the start, chunk boundaries and the end
    w = synth.WORKLOADS[4]
    d = synth.prefill_inputs_device(w.P, w.T, w.m, w.H, w.H_I, seed=w.seed)
    kv0 = d["kv"].clone()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, idx = csa.prefill(
        w.P, w.m, w.k, a=d["a"], b=d["b"], za=d["za"], zb=d["zb"], bias=d["bias"], kv=d["kv"],
        kv_scale=d["kv_scale"], q_fp4=d["q_fp4"], q_sf=d["q_sf"], w=d["w"], k_fp4=d["k_fp4"],
        k_sf=d["k_sf"], q=d["q"], sink=d["sink"], prev_b=d["prev_b"], prev_zb=d["prev_zb"],
        swa_prefix=d["swa_prefix"], lse=True, idx=True, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows = np.array([0, 1, 1023, 1024, 32767, 40000, w.T - 2, w.T - 1], np.int32)
    kv_gpu = d["kv"]
    d["kv"] = kv0  # the oracle compresses the new blocks itself from the prefix cache
    inp = _host_inputs(d, rows)
    ora = oracle.prefill(inp, w.k, rows)
    got = dict(out=out.float().cpu().numpy(), lse=host(lse), idx=host(idx), kv=host(kv_gpu),
               kv_scale=host(d["kv_scale"]))
    check_cache(inp, got, ora)
    check_rows(inp, w.k, got, rows, ora)


@pytest.mark.parametrize("P,T,page_entries", [(512, 300, 128), (2048, 700, 256)])
def test_prefill_on_a_paged_cache_equals_contiguous(P, T, page_entries):
    # the cache and keys behind a shuffled block table: the same outputs, selected sets and
    # lse bits as the contiguous call, the prefix rows untouched in their pages and the new
    # rows written to the pages the table names
    inp = synth.prefill_inputs(P, T, 4, 64, 16, seed=P + T)
    flat = run_prefill(inp, 64)
    Nmax = inp["kv"].shape[0]
    rng = np.random.default_rng(page_entries)
    table, num_pages = synth.page_table(rng, 1, Nmax // page_entries)
    kvp = synth.place_in_pages(inp["kv"][None], table, page_entries, num_pages)
    scp = synth.place_in_pages(inp["kv_scale"][None], table, page_entries, num_pages)
    kfp = synth.place_in_pages(inp["k_fp4"][None], table, page_entries, num_pages)
    ksp = synth.place_in_pages(inp["k_sf"].reshape(1, Nmax // 128, 512), table, page_entries,
                               num_pages, group=128)
    kv_d, sc_d = dev(kvp), dev(scp)
    opt = {x: dev(inp[x]) for x in ("prev_b", "prev_zb") if x in inp}
    opt["swa_prefix"] = dev(inp["swa_prefix"])
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse, idx = csa.prefill(
        P, 4, 64, a=dev(inp["a"]), b=dev(inp["b"]), za=dev(inp["za"]), zb=dev(inp["zb"]),
        bias=dev(inp["bias"]), kv=kv_d, kv_scale=sc_d, q_fp4=dev(inp["q_fp4"]),
        q_sf=dev(inp["q_sf"]), w=dev(inp["w"]), k_fp4=dev(kfp), k_sf=dev(ksp), q=dev(inp["q"]),
        sink=dev(inp["sink"]), lse=True, idx=True, dev_status=st,
        paging=csa.Paging(dev(table), page_entries, Nmax), **opt)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(out.float().cpu().numpy(), flat["out"])
    np.testing.assert_array_equal(host(lse), flat["lse"])
    np.testing.assert_array_equal(host(idx), flat["idx"])
    n1 = (P + T) // 4
    view_kv = oracle.paged_view(host(kv_d), table, page_entries)[0]
    view_sc = oracle.paged_view(host(sc_d), table, page_entries)[0]
    np.testing.assert_array_equal(view_kv[:n1], flat["kv"][:n1])
    np.testing.assert_array_equal(view_sc[:n1], flat["kv_scale"][:n1])
