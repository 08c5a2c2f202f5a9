"""The C-ABI library: it builds, loads without a GPU, exports every symbol the headers
declare, and rejects bad arguments on the host before touching the device."""

import ctypes as C
import glob
import os
import re

import pytest

import long_context_compressed_layer_b200 as csa
from long_context_compressed_layer_b200 import build as csa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    csa_build.build()
    return csa.lib()


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(\w+)\s*\([^;{]*\)\s*;",
                            text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert "csa_indexer_topk" in names and "hca_attn_decode" in names
    for n in names:
        assert hasattr(L, n), n
    assert set(csa.EXPORTS) == set(names)  # the binding covers every entry point


def test_status_strings(L):
    for code in range(7):
        assert L.csa_status_string(code)
    assert b"unknown" in L.csa_status_string(99)


def test_workspace_sizes_are_host_only(L):
    a = L.csa_indexer_topk_workspace_size(4, 262144, 1024)
    assert a >= 4 * 262144 * (4 + 8) + 4 * 2048 * 4  # scores, candidates, 11-bit histograms
    assert L.csa_indexer_topk_workspace_size(-1, 128, 4) == 0
    b = L.csa_attn_workspace_size(4, 128, 1024 + 128)
    assert b >= 4 * 18 * 128 * 512 * 2  # fp16 partial outputs per 64-row chunk
    assert L.csa_attn_workspace_size(1, 0, 10) == 0


def test_workspace_sizes_grow_with_every_argument(L):
    # one workspace serves every smaller problem (the header's promise), so no size may
    # shrink when a dimension grows; sizes come in whole 256-byte blocks
    ix = L.csa_indexer_topk_workspace_size
    at = L.csa_attn_workspace_size
    pf = L.csa_prefill_workspace_size
    op = L.csa_grouped_out_proj_workspace_size
    for B in (1, 2, 4, 32, 1024):
        for N in (128, 4096, 262144):
            for k in (1, 512, 2048):
                v = ix(B, N, k)
                assert v % 256 == 0
                assert v <= ix(2 * B, N, k) and v <= ix(B, 2 * N, k) and v <= ix(B, N, 2 * k)
    for B in (1, 4, 32):
        for H in (64, 128):
            for rows in (129, 1152, 2176, 8320):
                v = at(B, H, rows)
                assert v % 256 == 0 and v <= at(2 * B, H, rows) and v <= at(B, H, rows + 64)
    for T in (1, 1024, 1100, 65536):
        for N in (128, 65536):
            v = pf(T, N, 128, 1024)
            assert v % 256 == 0 and v <= pf(T + 1, N, 128, 1024) and v <= pf(T, N + 128, 128, 1024)
            assert v >= ix(min(T, 1024), N, 1024)  # holds the indexer workspace of one chunk
    assert op(100, 16, 1024) <= op(101, 16, 1024) and op(1, 1, 1) % 256 == 0


FAKE = 1 << 20  # a 256-aligned non-null address: never dereferenced on a rejected call


def _topk_args(**over):
    a = csa.TopkArgs(2, 64, 512, 1024, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None)
    for k, v in over.items():
        setattr(a, k, v)
    return a


def test_indexer_rejects_on_host(L):
    ws_ok = L.csa_indexer_topk_workspace_size(2, 1024, 512)
    call = lambda a, ws=FAKE, n=ws_ok: L.csa_indexer_topk(C.byref(a), ws, n, None)
    assert L.csa_indexer_topk(None, FAKE, ws_ok, None) == csa.CSA_ERR_INVALID_ARG
    assert call(_topk_args(Nmax=1000)) == csa.CSA_ERR_INVALID_ARG  # not a multiple of 128
    assert call(_topk_args(k=0)) == csa.CSA_ERR_INVALID_ARG
    assert call(_topk_args(flags=2)) == csa.CSA_ERR_INVALID_ARG  # an unknown flag bit
    assert call(_topk_args(select_wait_ns=-1)) == csa.CSA_ERR_INVALID_ARG
    assert call(_topk_args(H_I=8)) == csa.CSA_ERR_UNSUPPORTED
    assert call(_topk_args(k=4096)) == csa.CSA_ERR_UNSUPPORTED
    assert call(_topk_args(q_fp4=FAKE + 8)) == csa.CSA_ERR_INVALID_ARG  # misaligned
    assert call(_topk_args(w=None)) == csa.CSA_ERR_INVALID_ARG
    assert call(_topk_args(), ws=None) == csa.CSA_ERR_WORKSPACE
    assert call(_topk_args(), ws=FAKE + 16) == csa.CSA_ERR_WORKSPACE
    assert call(_topk_args(), n=ws_ok - 1) == csa.CSA_ERR_WORKSPACE
    assert call(_topk_args(B=0)) == csa.CSA_OK  # nothing to do


def _attn_args(**over):
    a = csa.AttnArgs(2, 128, 1024, 4096, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.0,
                     10000.0, 1, FAKE, None, None)
    for k, v in over.items():
        setattr(a, k, v)
    return a


def test_attention_rejects_on_host(L):
    ws_ok = L.csa_attn_workspace_size(2, 128, 1024 + 128)
    f = lambda a, ws=FAKE, n=ws_ok: L.csa_sparse_attn_decode(C.byref(a), ws, n, None)
    assert f(_attn_args(H=96)) == csa.CSA_ERR_UNSUPPORTED
    assert f(_attn_args(k=0)) == csa.CSA_ERR_INVALID_ARG
    assert f(_attn_args(derotate=2)) == csa.CSA_ERR_INVALID_ARG
    # paged-cache descriptors: page size a power of two >= 128, pages covering Nmax,
    # an aligned table, a pool of at least one page
    for pages in (csa.Pages(FAKE, 32, 100, 8), csa.Pages(FAKE, 64, 64, 8),
                  csa.Pages(FAKE, 3, 1024, 8), csa.Pages(FAKE + 4, 32, 128, 8),
                  csa.Pages(FAKE, 32, 128, 0), csa.Pages(FAKE, 0, 4096, 8)):
        assert f(_attn_args(pages=pages)) == csa.CSA_ERR_INVALID_ARG
    assert f(_attn_args(pages=csa.Pages(None, 0, 0, 0))) != csa.CSA_ERR_INVALID_ARG
    assert f(_attn_args(idx=None)) == csa.CSA_ERR_INVALID_ARG
    assert f(_attn_args(out=FAKE + 4)) == csa.CSA_ERR_INVALID_ARG
    assert f(_attn_args(), n=ws_ok - 1) == csa.CSA_ERR_WORKSPACE
    # HCA sizes its workspace from Nmax, not k
    hca_ws = L.csa_attn_workspace_size(2, 128, 4096 + 128)
    assert L.hca_attn_decode(C.byref(_attn_args(idx=None)), FAKE, ws_ok, None) == \
        csa.CSA_ERR_WORKSPACE
    assert hca_ws > ws_ok


def test_compress_rejects_on_host(L):
    def args(**over):
        a = csa.CompressArgs(1, 64, 4, 1, 0, 10000.0, 1e-6, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                             None, None, FAKE, FAKE, 16, None)
        for k, v in over.items():
            setattr(a, k, v)
        return a

    f = lambda a: L.csa_compress(C.byref(a), None)
    assert f(args(m=0)) == csa.CSA_ERR_INVALID_ARG
    assert f(args(m=129)) == csa.CSA_ERR_INVALID_ARG
    assert f(args(pos0=6)) == csa.CSA_ERR_INVALID_ARG  # not a block boundary
    assert f(args(pos0=8)) == csa.CSA_ERR_INVALID_ARG  # needs prev_b/prev_zb
    assert f(args(Nmax=15)) == csa.CSA_ERR_INVALID_ARG  # 16 entries do not fit
    assert f(args(b=None)) == csa.CSA_ERR_INVALID_ARG
    assert f(args(overlap=2)) == csa.CSA_ERR_INVALID_ARG
    assert f(args(T=3)) == csa.CSA_OK  # no complete block: nothing to do


def _prefill_args(**over):
    a = csa.PrefillArgs(4096, 300, 4, 128, 64, 1024, 1152, 0.0, 10000.0, 1e-6, 1, 0,
                        *([FAKE] * 5), None, FAKE, FAKE, *([FAKE] * 10), FAKE, None,
                        None, None)
    for k, v in over.items():
        setattr(a, k, v)
    return a


def test_prefill_rejects_on_host(L):
    ws_ok = L.csa_prefill_workspace_size(300, 1152, 128, 1024)
    assert ws_ok > 300 * 4 * 2 + (300 + 127) * 1024  # lengths, positions, window rows
    f = lambda a, ws=FAKE, n=ws_ok: L.csa_prefill(C.byref(a), ws, n, None)
    assert L.csa_prefill(None, FAKE, ws_ok, None) == csa.CSA_ERR_INVALID_ARG
    assert f(_prefill_args(P=4094)) == csa.CSA_ERR_INVALID_ARG   # not a block boundary
    assert f(_prefill_args(Nmax=1100)) == csa.CSA_ERR_INVALID_ARG  # not a multiple of 128
    assert f(_prefill_args(Nmax=1024)) == csa.CSA_ERR_INVALID_ARG  # 1099 entries do not fit
    # no capacity at all, even with no complete block: rejected before any launch
    assert f(_prefill_args(P=0, T=3, Nmax=0)) == csa.CSA_ERR_INVALID_ARG
    assert f(_prefill_args(k=0)) == csa.CSA_ERR_INVALID_ARG
    assert f(_prefill_args(strict_eligibility=2)) == csa.CSA_ERR_INVALID_ARG
    assert f(_prefill_args(H=96)) == csa.CSA_ERR_UNSUPPORTED
    assert f(_prefill_args(H_I=8)) == csa.CSA_ERR_UNSUPPORTED
    assert f(_prefill_args(k=4096)) == csa.CSA_ERR_UNSUPPORTED
    assert f(_prefill_args(swa_prefix=None)) == csa.CSA_ERR_INVALID_ARG  # P > 0 needs it
    assert f(_prefill_args(prev_b=None)) == csa.CSA_ERR_INVALID_ARG
    assert f(_prefill_args(q=FAKE + 2)) == csa.CSA_ERR_INVALID_ARG
    assert f(_prefill_args(), n=ws_ok - 1) == csa.CSA_ERR_WORKSPACE
    assert f(_prefill_args(), ws=FAKE + 64) == csa.CSA_ERR_WORKSPACE
    assert f(_prefill_args(T=0)) == csa.CSA_OK  # nothing to do


def test_cuda_sources_are_sm100a_only():
    src = open(os.path.join(ROOT, "long_context_compressed_layer_b200", "build.py")).read()
    assert "arch=compute_100a,code=sm_100a" in src
    for f in glob.glob(os.path.join(ROOT, "long_context_compressed_layer_b200", "csrc", "*")):
        text = open(f).read()
        assert "multicast" not in text  # no TMA multicast anywhere
        assert "wgmma" not in text and "mma.sync" not in text


def test_index_key_compression_rejects_on_host(L):
    def args(**over):
        a = csa.IkeyArgs(1, 64, 4, 1, 0, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE,
                         128, None)
        for k, v in over.items():
            setattr(a, k, v)
        return a

    f = lambda a: L.csa_compress_index_keys(C.byref(a), None)
    assert L.csa_compress_index_keys(None, None) == csa.CSA_ERR_INVALID_ARG
    assert f(args(Nmax=100)) == csa.CSA_ERR_INVALID_ARG      # not a multiple of 128
    assert f(args(pos0=6)) == csa.CSA_ERR_INVALID_ARG        # not a block boundary
    assert f(args(pos0=512)) == csa.CSA_ERR_INVALID_ARG      # 144 entries > Nmax, no tail
    assert f(args(b=None)) == csa.CSA_ERR_INVALID_ARG
    assert f(args(k_sf=FAKE + 4)) == csa.CSA_ERR_INVALID_ARG
    assert f(args(T=3)) == csa.CSA_OK                        # no complete block


def test_indexer_query_rejects_on_host(L):
    def args(**over):
        a = csa.IqueryArgs(16, 1536, 64, FAKE, FAKE, FAKE, FAKE, None, None)
        for k, v in over.items():
            setattr(a, k, v)
        return a

    f = lambda a: L.csa_indexer_query(C.byref(a), None)
    assert f(args(r=100)) == csa.CSA_ERR_INVALID_ARG   # not a multiple of 64
    assert f(args(r=32768)) == csa.CSA_ERR_UNSUPPORTED
    assert f(args(H_I=8)) == csa.CSA_ERR_UNSUPPORTED
    assert f(args(W=None)) == csa.CSA_ERR_INVALID_ARG
    assert f(args(T=0)) == csa.CSA_OK


def test_grouped_out_proj_rejects_on_host(L):
    ws_ok = L.csa_grouped_out_proj_workspace_size(64, 16, 1024)
    assert ws_ok >= 64 * 16 * 1024 * 2

    def args(**over):
        a = csa.OprojArgs(64, 128, 16, 1024, 7168, FAKE, FAKE, FAKE, FAKE, None)
        for k, v in over.items():
            setattr(a, k, v)
        return a

    f = lambda a, ws=FAKE, n=ws_ok: L.csa_grouped_out_proj(C.byref(a), ws, n, None)
    assert f(args(G=3)) == csa.CSA_ERR_UNSUPPORTED        # does not divide 128 heads
    assert f(args(d_g=1000)) == csa.CSA_ERR_UNSUPPORTED   # not a multiple of 128
    assert f(args(H=96)) == csa.CSA_ERR_UNSUPPORTED
    assert f(args(out=None)) == csa.CSA_ERR_INVALID_ARG
    assert f(args(), n=ws_ok - 1) == csa.CSA_ERR_WORKSPACE
    assert f(args(T=0)) == csa.CSA_OK


def test_decode_append_rejects_on_host(L):
    def args(**over):
        a = csa.AppendArgs(2, 4, 1, 10000.0, 1e-6, *([FAKE] * 6), None, *([FAKE] * 7), 128,
                           FAKE, *([None] * 11), None)
        for k, v in over.items():
            setattr(a, k, v)
        return a

    f = lambda a: L.csa_decode_append(C.byref(a), None)
    assert L.csa_decode_append(None, None) == csa.CSA_ERR_INVALID_ARG
    assert f(args(m=0)) == csa.CSA_ERR_INVALID_ARG
    assert f(args(Nmax=100)) == csa.CSA_ERR_INVALID_ARG
    assert f(args(tail_b=None)) == csa.CSA_ERR_INVALID_ARG     # overlap needs the ring
    assert f(args(ia=FAKE)) == csa.CSA_ERR_INVALID_ARG         # a key stream needs its state
    assert f(args(B=0)) == csa.CSA_OK


def test_bf16_index_scores_share_the_indexer_checks(L):
    ws_ok = L.csa_indexer_topk_workspace_size(2, 1024, 512)
    call = lambda a, ws=FAKE, n=ws_ok: L.csa_indexer_topk_bf16(C.byref(a), ws, n, None)
    assert call(_topk_args(Nmax=1000)) == csa.CSA_ERR_INVALID_ARG
    assert call(_topk_args(H_I=8)) == csa.CSA_ERR_UNSUPPORTED
    assert call(_topk_args(), n=ws_ok - 1) == csa.CSA_ERR_WORKSPACE
    assert call(_topk_args(B=0)) == csa.CSA_OK
