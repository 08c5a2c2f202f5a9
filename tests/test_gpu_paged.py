"""The paged compressed cache on the GPU (csa_pages): indexer top-k, sparse and dense
attention and the decode-step append, each through a shuffled block table, against the
oracle reading the pool through its own paged view, and bit for bit against the same call
on the contiguous layout. (walkthrough §3.5: the classical cache holds the compressed
entries in blocks aligned to 128 tokens.)"""

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
    return torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x).cuda()


def host(t):
    return t.cpu().numpy()


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    csa.lib()


@pytest.mark.parametrize("page_entries", [128, 256, 512, 2048])
@pytest.mark.parametrize("separate", [False, True])
def test_indexer_through_shuffled_pages(page_entries, separate):
    rng = np.random.default_rng(page_entries + separate)
    B, H_I, Nmax, k = 3, 64, 8192, 512
    n = np.array([8192, 5000, 700], np.int32)
    ix = synth.indexer_inputs(rng, B, H_I, Nmax, n, 3)
    table, num_pages = synth.page_table(rng, B, Nmax // page_entries)
    kp = synth.place_in_pages(ix["k_fp4"], table, page_entries, num_pages)
    sp = synth.place_in_pages(ix["k_sf"].reshape(B, Nmax // 128, 512), table, page_entries,
                              num_pages, group=128)
    paging = csa.Paging(dev(table), page_entries)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = (dev(n), dev(ix["q_fp4"]), dev(ix["q_sf"]), dev(ix["w"]))
    got = host(csa.indexer_topk(*q, dev(kp), dev(sp), k, paging=paging, dev_status=st,
                                separate_select=separate))
    flat = host(csa.indexer_topk(*q, dev(ix["k_fp4"]), dev(ix["k_sf"]), k,
                                 separate_select=separate))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(got, flat)  # same scores, same selection
    ora = oracle.indexer_scores(n, ix["q_fp4"], ix["q_sf"], ix["w"],
                                oracle.paged_view(kp, table, page_entries),
                                oracle.paged_view(sp, table, page_entries, group=128).reshape(B, -1))
    flips = sum(compare.compare_topk(got[b], ora[b], int(n[b]), k, what=f"seq {b}")
                for b in range(B))
    assert flips <= 2


def _attn_inputs(rng, B, H, Nmax, n, pos, k):
    kv, sc = synth.kv_cache(rng, B, Nmax)
    q = synth.bf16_normal(rng, (B, H, 512))
    swa = synth.bf16_normal(rng, (B, 128, 512))
    sink = rng.standard_normal(H).astype(np.float32)
    idx = None
    if k is not None:
        idx = np.full((B, k), -1, np.int32)
        for b in range(B):
            c = min(k - 3, int(n[b]))
            idx[b, :c] = np.sort(rng.choice(int(n[b]), c, replace=False))
    return kv, sc, q, swa, sink, idx


@pytest.mark.parametrize("page_entries", [128, 1024])
@pytest.mark.parametrize("sparse", [True, False])
def test_attention_through_shuffled_pages(page_entries, sparse):
    rng = np.random.default_rng(page_entries * 3 + sparse)
    B, H, Nmax = 3, 128, 4096
    n = np.array([4096, 2500, 9], np.int32)
    pos = np.array([16383, 10001, 40], np.int32)
    k = 1024 if sparse else None
    kv, sc, q, swa, sink, idx = _attn_inputs(rng, B, H, Nmax, n, pos, k)
    table, num_pages = synth.page_table(rng, B, Nmax // page_entries)
    kvp = synth.place_in_pages(kv, table, page_entries, num_pages)
    scp = synth.place_in_pages(sc, table, page_entries, num_pages)
    paging = csa.Paging(dev(table), page_entries)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    common = (dev(q), dev(pos), dev(n))
    rest = (dev(swa), dev(sink))
    if sparse:
        got = csa.sparse_attn_decode(*common, dev(kvp), dev(scp), *rest, dev(idx),
                                     paging=paging, dev_status=st)
        flat = csa.sparse_attn_decode(*common, dev(kv), dev(sc), *rest, dev(idx))
    else:
        got = csa.hca_attn_decode(*common, dev(kvp), dev(scp), *rest, paging=paging,
                                  dev_status=st)
        flat = csa.hca_attn_decode(*common, dev(kv), dev(sc), *rest)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(got.view(torch.int16), flat.view(torch.int16))
    want, _ = oracle.attention(q, pos, n, oracle.paged_view(kvp, table, page_entries),
                               oracle.paged_view(scp, table, page_entries), swa, sink, idx=idx)
    compare.close(got.float().cpu().numpy(), want, what="paged attention")


def test_appends_into_shuffled_pages():
    # token-by-token appends into a paged cache land where the table says, with the same
    # bits as appends into the contiguous cache
    B, S, m, Nmax, P = 2, 4 * 300 + 3, 4, 512, 128
    rng = np.random.default_rng(8)
    kvs = synth.compress_inputs(B, S, m, True, seed=81)
    iks = synth.compress_inputs(B, S, m, True, seed=82, dim=128)
    table, num_pages = synth.page_table(rng, B, Nmax // P)
    paging = csa.Paging(dev(table), P)
    flat = csa.new_decode_state(B, Nmax, m)
    paged = csa.new_decode_state(B, Nmax, m)
    paged["kv"] = torch.zeros((num_pages, P, 576), dtype=torch.uint8, device="cuda")
    paged["kv_scale"] = torch.zeros((num_pages, P), dtype=torch.float32, device="cuda")
    paged["k_fp4"] = torch.zeros((num_pages, P, 64), dtype=torch.uint8, device="cuda")
    paged["k_sf"] = torch.zeros((num_pages, P // 128, 512), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    d = {k_: dev(v) for k_, v in kvs.items()}
    di = {k_: dev(v) for k_, v in iks.items()}
    for t in range(S):
        pos = torch.full((B,), t, dtype=torch.int32, device="cuda")
        tok = dict(b=d["b"][:, t].contiguous(), zb=d["zb"][:, t].contiguous(), m=m,
                   ia=di["a"][:, t].contiguous(), ib=di["b"][:, t].contiguous(),
                   iza=di["za"][:, t].contiguous(), izb=di["zb"][:, t].contiguous(),
                   ibias=di["bias"], dev_status=st)
        a_t, za_t = d["a"][:, t].contiguous(), d["za"][:, t].contiguous()
        csa.decode_append(pos, a_t, za_t, d["bias"], flat, **tok)
        csa.decode_append(pos, a_t, za_t, d["bias"], paged, paging=paging, **tok)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    n = S // m
    assert (host(paged["n_entries"]) == n).all()
    view = lambda key, group=1: oracle.paged_view(host(paged[key]), table, P, group)
    np.testing.assert_array_equal(view("kv")[:, :n], host(flat["kv"])[:, :n])
    np.testing.assert_array_equal(view("kv_scale")[:, :n], host(flat["kv_scale"])[:, :n])
    np.testing.assert_array_equal(view("k_fp4")[:, :n], host(flat["k_fp4"])[:, :n])
    np.testing.assert_array_equal(view("k_sf", 128).reshape(B, -1)[:, :(n + 127) // 128 * 512],
                                  host(flat["k_sf"])[:, :(n + 127) // 128 * 512])
    # and the appended entries against the oracle's whole-stream compression
    ora = oracle.compress(kvs["a"], kvs["za"], kvs["bias"], m, True, b=kvs["b"], zb=kvs["zb"])
    flips = compare.check_codes(view("kv")[:, :n], ora["kv"], ora["y"], ora["kv_scale"],
                                what="paged appends")
    assert flips <= max(4, ora["kv"].size // 5000)


def test_page_outside_the_pool_is_reported():
    rng = np.random.default_rng(12)
    B, H, Nmax, P = 1, 64, 1024, 256
    n = np.array([1000], np.int32)
    kv, sc, q, swa, sink, idx = _attn_inputs(rng, B, H, Nmax, n, np.array([4000], np.int32), 256)
    table, num_pages = synth.page_table(rng, B, Nmax // P)
    kvp = synth.place_in_pages(kv, table, P, num_pages)
    scp = synth.place_in_pages(sc, table, P, num_pages)
    table[0, 2] = num_pages + 7  # a page the pool does not have: never dereferenced
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    csa.sparse_attn_decode(dev(q), dev(np.array([4000], np.int32)), dev(n), dev(kvp), dev(scp),
                           dev(swa), dev(sink), dev(idx), paging=csa.Paging(dev(table), P),
                           dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == csa.CSA_ERR_DEVICE
    ix = synth.indexer_inputs(rng, B, 16, Nmax, n)
    kp = synth.place_in_pages(ix["k_fp4"], table.clip(0, num_pages - 1), P, num_pages)
    sp = synth.place_in_pages(ix["k_sf"].reshape(B, -1, 512), table.clip(0, num_pages - 1), P,
                              num_pages, group=128)
    st.zero_()
    csa.indexer_topk(dev(n), dev(ix["q_fp4"]), dev(ix["q_sf"]), dev(ix["w"]), dev(kp), dev(sp),
                     64, paging=csa.Paging(dev(table), P), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == csa.CSA_ERR_DEVICE
