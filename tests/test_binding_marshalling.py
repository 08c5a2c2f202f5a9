"""The binding hands each call's arguments to the library as the C structs say (no GPU):
with the library replaced by a recorder and device pointers by stand-in addresses, every
paged call passes the table row length, the entries per page and the pool's page count
(the pool's entries over the page size), every contiguous call passes an empty page
struct, and the sizes, flags and scalars arrive as given. Host logic only: nothing here
reaches a kernel."""

import pytest
import torch

import long_context_compressed_layer_b200 as csa

U8, I16, I32, F32 = torch.uint8, torch.int16, torch.int32, torch.float32
B, M, P, PAGES_MAX = 2, 4, 256, 4
POOL = (B * PAGES_MAX + 3) * P  # three spare pages


def t(*shape, dtype=F32):
    return torch.empty(shape, dtype=dtype)


class Recorder:
    """Stands in for the library: records each call's arguments and returns OK."""

    def __init__(self):
        self.pages = {}
        self.args = {}

    def _rec(self, name, args):
        self.args[name] = args._obj
        pg = args._obj.pages
        self.pages[name] = (bool(pg.block_table), pg.pages_max, pg.page_entries, pg.num_pages)
        return 0

    def csa_indexer_topk(self, args, ws, n, stream):
        return self._rec("topk", args)

    def csa_sparse_attn_decode(self, args, ws, n, stream):
        return self._rec("attn", args)

    def csa_decode_append(self, args, stream):
        return self._rec("append", args)

    def csa_prefill(self, args, ws, n, stream):
        return self._rec("prefill", args)

    def csa_status_string(self, s):
        return b"ok"


@pytest.fixture
def rec(monkeypatch):
    r = Recorder()
    monkeypatch.setattr(csa, "lib", lambda: r)
    monkeypatch.setattr(csa, "_ptr", lambda x, **k: None if x is None else 4096)
    monkeypatch.setattr(csa, "_stream", lambda s: None)
    return r


def _calls(paged):
    pool = POOL if paged else B * 512
    kv = t(pool, 576, dtype=U8) if paged else t(B, 512, 576, dtype=U8)
    scale = t(pool) if paged else t(B, 512)
    k_fp4 = t(pool, 64, dtype=U8) if paged else t(B, 512, 64, dtype=U8)
    k_sf = t(pool // 128 * 512, dtype=U8) if paged else t(B, 512 // 128 * 512, dtype=U8)
    table = csa.Paging(t(B, PAGES_MAX, dtype=I32), P) if paged else None
    ws = t(256, dtype=U8)
    csa.indexer_topk(t(B, dtype=I32), t(B, 16, 64, dtype=U8), t(B, 16, 4, dtype=U8), t(B, 16),
                     k_fp4, k_sf, 64, workspace=ws, idx=t(B, 64, dtype=I32), paging=table)
    csa.sparse_attn_decode(t(B, 64, 512, dtype=I16), t(B, dtype=I32), t(B, dtype=I32), kv,
                           scale, t(B, 128, 512, dtype=I16), t(64), t(B, 64, dtype=I32),
                           workspace=ws, out=t(B, 64, 512, dtype=I16), paging=table)
    st = csa.new_decode_state(B, 128, M, device="cpu")
    st.update(kv=kv if paged else t(B, 128, 576, dtype=U8),
              kv_scale=scale if paged else t(B, 128),
              k_fp4=k_fp4 if paged else t(B, 128, 64, dtype=U8),
              k_sf=k_sf if paged else t(B, 512, dtype=U8))
    csa.decode_append(t(B, dtype=I32), t(B, 512, dtype=I16), t(B, 512), t(2 * M), st,
                      b=t(B, 512, dtype=I16), zb=t(B, 512), m=M, ia=t(B, 128, dtype=I16),
                      ib=t(B, 128, dtype=I16), iza=t(B, 128), izb=t(B, 128), ibias=t(2 * M),
                      paging=table)
    T = 301
    one = csa.Paging(t(1, PAGES_MAX, dtype=I32), P) if paged else None
    n1 = POOL if paged else 1024
    csa.prefill(512, M, 64, a=t(T, 512, dtype=I16), b=t(T, 512, dtype=I16), za=t(T, 512),
                zb=t(T, 512), bias=t(2 * M), kv=t(n1, 576, dtype=U8), kv_scale=t(n1),
                q_fp4=t(T, 16, 64, dtype=U8), q_sf=t(T, 16, 4, dtype=U8), w=t(T, 16),
                k_fp4=t(n1, 64, dtype=U8), k_sf=t(n1 // 128 * 512, dtype=U8),
                q=t(T, 64, 512, dtype=I16), sink=t(64), prev_b=t(M, 512, dtype=I16),
                prev_zb=t(M, 512), swa_prefix=t(128, 512, dtype=I16), workspace=ws,
                out=t(T, 64, 512, dtype=I16), paging=one)


def test_paged_calls_pass_the_table_and_the_pool_size(rec):
    _calls(paged=True)
    want = (True, PAGES_MAX, P, POOL // P)
    assert rec.pages == {"topk": want, "attn": want, "append": want, "prefill": want}


def test_contiguous_calls_pass_an_empty_struct(rec):
    _calls(paged=False)
    assert set(rec.pages.values()) == {(False, 0, 0, 0)}


def test_sizes_flags_and_scalars_arrive_as_given(rec):
    ws = t(256, dtype=U8)
    kf, ksf = t(B, 1024, 64, dtype=U8), t(B, 1024 // 128 * 512, dtype=U8)
    common = (t(B, dtype=I32), t(B, 32, 64, dtype=U8), t(B, 32, 4, dtype=U8), t(B, 32), kf, ksf)
    csa.indexer_topk(*common, 128, workspace=ws, idx=t(B, 128, dtype=I32))
    a = rec.args["topk"]
    assert (a.B, a.H_I, a.k, a.Nmax, a.flags, a.select_wait_ns) == (B, 32, 128, 1024, 0, 0)
    csa.indexer_topk(*common, 128, workspace=ws, idx=t(B, 128, dtype=I32),
                     separate_select=True, select_wait_ns=5000)
    a = rec.args["topk"]
    assert (a.flags & csa.TOPK_SEPARATE_SELECT, a.select_wait_ns) == (1, 5000)

    csa.sparse_attn_decode(t(B, 128, 512, dtype=I16), t(B, dtype=I32), t(B, dtype=I32),
                           t(B, 2048, 576, dtype=U8), t(B, 2048), t(B, 128, 512, dtype=I16),
                           t(128), t(B, 512, dtype=I32), workspace=ws,
                           out=t(B, 128, 512, dtype=I16), tau=0.125, rope_base=5e5,
                           derotate=False)
    a = rec.args["attn"]
    assert (a.B, a.H, a.k, a.Nmax, a.derotate) == (B, 128, 512, 2048, 0)
    assert (a.tau, a.rope_base) == (0.125, 5e5)

    T = 301
    csa.prefill(1024, M, 256, a=t(T, 512, dtype=I16), b=t(T, 512, dtype=I16), za=t(T, 512),
                zb=t(T, 512), bias=t(2 * M), kv=t(1024, 576, dtype=U8), kv_scale=t(1024),
                q_fp4=t(T, 16, 64, dtype=U8), q_sf=t(T, 16, 4, dtype=U8), w=t(T, 16),
                k_fp4=t(1024, 64, dtype=U8), k_sf=t(1024 // 128 * 512, dtype=U8),
                q=t(T, 64, 512, dtype=I16), sink=t(64), prev_b=t(M, 512, dtype=I16),
                prev_zb=t(M, 512), swa_prefix=t(128, 512, dtype=I16), workspace=ws,
                out=t(T, 64, 512, dtype=I16), strict_eligibility=True, eps=1e-5)
    a = rec.args["prefill"]
    assert (a.P, a.T, a.m, a.H, a.H_I, a.k, a.Nmax) == (1024, T, M, 64, 16, 256, 1024)
    assert (a.strict_eligibility, a.derotate) == (1, 1)
    assert a.eps == pytest.approx(1e-5, rel=1e-7)
