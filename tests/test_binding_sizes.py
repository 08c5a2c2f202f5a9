"""The binding's buffer-size checks, on shape-only ("meta") tensors, without a GPU: calls
shaped as the parity tests and the benchmark make them pass the checks (and stop at the
device-pointer check, since meta tensors live on no device); a buffer one element short of
its layout is refused by name before any pointer reaches the library."""

import pytest
import torch

import long_context_compressed_layer_b200 as csa

U8, I16, I32, F32 = torch.uint8, torch.int16, torch.int32, torch.float32


def t(*shape, dtype=F32):
    return torch.empty(shape, dtype=dtype, device="meta")


def short(x):
    return t(x.numel() - 1, dtype=x.dtype)


def passes_checks(fn, *args, **kw):
    with pytest.raises(ValueError, match="CUDA tensor"):
        fn(*args, **kw)


def refused(name, fn, *args, **kw):
    with pytest.raises(ValueError, match=f"^{name}: expected at least"):
        fn(*args, **kw)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    csa.lib()  # the workspace-size queries are host functions of the library


def _compress_kw(B=2, T=64, m=4, pos0=8, dim=512):
    return dict(a=t(B, T, dim, dtype=I16), za=t(B, T, dim), bias=t(2 * m), m=m, overlap=True,
                b=t(B, T, dim, dtype=I16), zb=t(B, T, dim), pos0=pos0,
                prev_b=t(B, m, dim, dtype=I16), prev_zb=t(B, m, dim))


def test_compress():
    kw = _compress_kw()
    call = lambda **o: csa.compress(**{**kw, **o}, Nmax=128)
    passes_checks(call)
    passes_checks(call, norm_w=t(512), kv=t(2, 128, 576, dtype=U8), kv_scale=t(2, 128))
    for name in ("za", "b", "zb", "bias", "prev_b", "prev_zb"):
        refused(name, call, **{name: short(kw[name])})
    refused("norm_w", call, norm_w=t(511))
    refused("kv", call, kv=t(2 * 128 * 576 - 1, dtype=U8))
    with pytest.raises(ValueError, match="^a: dimension 2"):
        call(a=t(2, 64, 256, dtype=I16))


def test_compress_index_keys():
    kw = _compress_kw(dim=128)
    call = lambda **o: csa.compress_index_keys(**{**kw, **o})
    passes_checks(call)
    for name in ("za", "b", "zb", "bias", "prev_b", "prev_zb"):
        refused(name, call, **{name: short(kw[name])})
    refused("k_sf", call, k_fp4=t(2, 128, 64, dtype=U8), k_sf=t(2 * 512 - 1, dtype=U8))


def test_decode_append():
    B, m = 2, 4
    st = csa.new_decode_state(B, 128, m, device="meta")
    kw = dict(pos=t(B, dtype=I32), a=t(B, 512, dtype=I16), za=t(B, 512), bias=t(2 * m),
              state=st, b=t(B, 512, dtype=I16), zb=t(B, 512), m=m, ia=t(B, 128, dtype=I16),
              ib=t(B, 128, dtype=I16), iza=t(B, 128), izb=t(B, 128), ibias=t(2 * m))
    call = lambda **o: csa.decode_append(**{**kw, **o})
    passes_checks(call)
    for name in ("pos", "za", "b", "zb", "ibias", "ia"):
        refused(name, call, **{name: short(kw[name])})
    small = dict(st, swa=t(B * 128 * 512 - 1, dtype=I16))
    refused("swa", call, state=small)


def test_indexer_query():
    call = lambda **o: csa.indexer_query(**{**dict(c=t(300, 256, dtype=I16),
                                                   W=t(16 * 128, 256, dtype=I16), H_I=16), **o})
    passes_checks(call)
    refused("W", call, W=t(16 * 128 * 256 - 1, dtype=I16))
    refused("q_sf", call, q_fp4=t(300, 16, 64, dtype=U8), q_sf=t(300 * 16 * 4 - 1, dtype=U8))


def test_grouped_out_proj():
    kw = dict(attn=t(200, 64, 512, dtype=I16), Wg=t(16, 128, 4 * 512, dtype=I16),
              Wo=t(256, 16 * 128, dtype=I16))
    call = lambda **o: csa.grouped_out_proj(**{**kw, **o})
    passes_checks(call)
    refused("Wo", call, Wo=short(kw["Wo"]))
    refused("out", call, out=t(200 * 256 - 1, dtype=I16))


def test_indexer_topk():
    B, H_I, Nmax, k = 4, 64, 262144, 1024
    kw = dict(n_entries=t(B, dtype=I32), q_fp4=t(B, H_I, 64, dtype=U8),
              q_sf=t(B, H_I, 4, dtype=U8), w=t(B, H_I), k_fp4=t(B, Nmax, 64, dtype=U8),
              k_sf=t(B, Nmax // 128 * 512, dtype=U8), k=k)
    call = lambda **o: csa.indexer_topk(**{**kw, **o})
    passes_checks(call)
    passes_checks(call, idx=t(B, k, dtype=I32), workspace=t(256, dtype=U8))
    for name in ("n_entries", "q_sf", "w", "k_sf"):
        refused(name, call, **{name: short(kw[name])})
    refused("k_fp4", call, k_fp4=t(B - 1, Nmax, 64, dtype=U8))
    refused("idx", call, idx=t(B, k - 1, dtype=I32))


def test_paged_indexer_and_attention_arguments():
    # pools of 512-entry pages behind a [B][pages_max] table: a well-shaped call reaches the
    # device-pointer check; a table of the wrong type or row count, a pool that is not a
    # whole number of pages, and a pool one element short are refused on the host
    B, H_I, H, P, pages_max, k = 4, 64, 128, 512, 8, 1024
    pool = (B * pages_max + 3) * P
    paging = csa.Paging(t(B, pages_max, dtype=I32), P)
    assert paging.Nmax == pages_max * P
    kw = dict(n_entries=t(B, dtype=I32), q_fp4=t(B, H_I, 64, dtype=U8),
              q_sf=t(B, H_I, 4, dtype=U8), w=t(B, H_I), k_fp4=t(pool, 64, dtype=U8),
              k_sf=t(pool // 128 * 512, dtype=U8), k=k, paging=paging)
    call = lambda **o: csa.indexer_topk(**{**kw, **o})
    passes_checks(call)
    with pytest.raises(ValueError, match="block_table: int32"):
        csa.Paging(t(B, pages_max, dtype=torch.int64), P)
    with pytest.raises(ValueError, match="rows for 4 sequences"):
        call(paging=csa.Paging(t(B - 1, pages_max, dtype=I32), P))
    with pytest.raises(ValueError, match="whole number of pages"):
        call(k_fp4=t(pool + 128, 64, dtype=U8), k_sf=t((pool + 128) // 128 * 512, dtype=U8))
    refused("k_sf", call, k_sf=short(kw["k_sf"]))
    akw = dict(q=t(B, H, 512, dtype=I16), pos=t(B, dtype=I32), n_entries=t(B, dtype=I32),
               kv=t(pool, 576, dtype=U8), kv_scale=t(pool), swa=t(B, 128, 512, dtype=I16),
               sink=t(H), idx=t(B, k, dtype=I32), paging=paging)
    attn = lambda **o: csa.sparse_attn_decode(**{**akw, **o})
    passes_checks(attn)
    refused("kv_scale", attn, kv_scale=short(akw["kv_scale"]))
    with pytest.raises(ValueError, match="whole number of pages"):
        attn(kv=t(pool + 1, 576, dtype=U8), kv_scale=t(pool + 1))


def test_attention():
    B, H, Nmax, k = 4, 128, 262144, 1024
    kw = dict(q=t(B, H, 512, dtype=I16), pos=t(B, dtype=I32), n_entries=t(B, dtype=I32),
              kv=t(B, Nmax, 576, dtype=U8), kv_scale=t(B, Nmax), swa=t(B, 128, 512, dtype=I16),
              sink=t(H))
    sparse = lambda **o: csa.sparse_attn_decode(**{**kw, "idx": t(B, k, dtype=I32), **o})
    dense = lambda **o: csa.hca_attn_decode(**{**kw, **o})
    passes_checks(sparse)
    passes_checks(dense)
    passes_checks(sparse, out=t(B, H, 512, dtype=I16))
    for name in ("pos", "n_entries", "kv_scale", "swa", "sink"):
        refused(name, sparse, **{name: short(kw[name])})
        refused(name, dense, **{name: short(kw[name])})
    refused("idx", sparse, idx=t(B - 1, k, dtype=I32))
    refused("out", dense, out=t(B, H, 511, dtype=I16))


def test_prefill():
    P, T, m, H, H_I, k, Nmax = 512, 301, 4, 64, 16, 64, 256
    kw = dict(a=t(T, 512, dtype=I16), b=t(T, 512, dtype=I16), za=t(T, 512), zb=t(T, 512),
              bias=t(2 * m), kv=t(Nmax, 576, dtype=U8), kv_scale=t(Nmax),
              q_fp4=t(T, H_I, 64, dtype=U8), q_sf=t(T, H_I, 4, dtype=U8), w=t(T, H_I),
              k_fp4=t(Nmax, 64, dtype=U8), k_sf=t(Nmax // 128 * 512, dtype=U8),
              q=t(T, H, 512, dtype=I16), sink=t(H), prev_b=t(m, 512, dtype=I16),
              prev_zb=t(m, 512), swa_prefix=t(128, 512, dtype=I16))
    call = lambda **o: csa.prefill(P, m, k, **{**kw, **o})
    passes_checks(call)
    passes_checks(call, norm_w=t(512), out=t(T, H, 512, dtype=I16))
    for name in ("b", "za", "zb", "bias", "kv_scale", "q_sf", "w", "k_fp4", "k_sf", "sink",
                 "prev_b", "prev_zb", "swa_prefix"):
        refused(name, call, **{name: short(kw[name])})
    refused("q", call, q=t(T - 1, H, 512, dtype=I16))
    refused("norm_w", call, norm_w=t(100))


def test_paged_append_and_prefill_arguments():
    # the append's state and the prefill's cache as page pools: well-shaped calls reach the
    # device-pointer check; a table whose row count is not the batch's, or a pool that is
    # not a whole number of pages, is refused on the host
    B, m, P, pages_max = 2, 4, 256, 4
    pool = (B * pages_max + 3) * P
    st = csa.new_decode_state(B, 128, m, device="meta")
    st.update(kv=t(pool, 576, dtype=U8), kv_scale=t(pool), k_fp4=t(pool, 64, dtype=U8),
              k_sf=t(pool // 128 * 512, dtype=U8))
    paging = csa.Paging(t(B, pages_max, dtype=I32), P)
    kw = dict(pos=t(B, dtype=I32), a=t(B, 512, dtype=I16), za=t(B, 512), bias=t(2 * m),
              state=st, b=t(B, 512, dtype=I16), zb=t(B, 512), m=m, ia=t(B, 128, dtype=I16),
              ib=t(B, 128, dtype=I16), iza=t(B, 128), izb=t(B, 128), ibias=t(2 * m),
              paging=paging)
    call = lambda **o: csa.decode_append(**{**kw, **o})
    passes_checks(call)
    with pytest.raises(ValueError, match="rows for 2 sequences"):
        call(paging=csa.Paging(t(B + 1, pages_max, dtype=I32), P))
    refused("k_sf", call, state=dict(st, k_sf=short(st["k_sf"])))

    Pp, T, H, H_I, k = 512, 301, 64, 16, 64
    pk = dict(a=t(T, 512, dtype=I16), b=t(T, 512, dtype=I16), za=t(T, 512), zb=t(T, 512),
              bias=t(2 * m), kv=t(pool, 576, dtype=U8), kv_scale=t(pool),
              q_fp4=t(T, H_I, 64, dtype=U8), q_sf=t(T, H_I, 4, dtype=U8), w=t(T, H_I),
              k_fp4=t(pool, 64, dtype=U8), k_sf=t(pool // 128 * 512, dtype=U8),
              q=t(T, H, 512, dtype=I16), sink=t(H), prev_b=t(m, 512, dtype=I16),
              prev_zb=t(m, 512), swa_prefix=t(128, 512, dtype=I16),
              paging=csa.Paging(t(1, pages_max, dtype=I32), P))
    pre = lambda **o: csa.prefill(Pp, m, k, **{**pk, **o})
    passes_checks(pre)
    with pytest.raises(ValueError, match="rows for 1 sequences"):
        pre(paging=paging)  # a prefill is one sequence: its table has one row
    with pytest.raises(ValueError, match="whole number of pages"):
        pre(kv=t(pool + 7, 576, dtype=U8), kv_scale=t(pool + 7), k_fp4=t(pool + 7, 64, dtype=U8))
