"""ctypes binding of the fp64 CPU oracle (csa_oracle.cpp).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the CUDA library. It takes and returns numpy
arrays; the shared object is built on first use (or by the package build step).
"""

from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (plain -O2, no fast-math: IEEE fp64 throughout)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _p(a, ctype):
    return None if a is None else a.ctypes.data_as(C.POINTER(ctype))


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            d, i, i64 = C.c_double, C.c_int, C.c_int64
            P = C.POINTER
            u8, u16, f32, f64, i32 = (P(C.c_uint8), P(C.c_uint16), P(C.c_float),
                                      P(C.c_double), P(C.c_int32))
            L.or_bf16_decode.restype = d
            L.or_bf16_decode.argtypes = [C.c_uint16]
            L.or_bf16_encode.restype = C.c_uint16
            L.or_bf16_encode.argtypes = [d]
            L.or_e4m3_decode.restype = d
            L.or_e4m3_decode.argtypes = [C.c_uint8]
            L.or_e4m3_encode.restype = C.c_uint8
            L.or_e4m3_encode.argtypes = [d]
            L.or_e2m1_decode.restype = d
            L.or_e2m1_decode.argtypes = [C.c_uint8]
            L.or_e8m0_decode.restype = d
            L.or_e8m0_decode.argtypes = [C.c_uint8]
            L.or_key_sf_offset.restype = C.c_size_t
            L.or_key_sf_offset.argtypes = [i64, i]
            L.or_compress.restype = i
            L.or_compress.argtypes = [i, i, i, i, i64, d, d, u16, u16, f32, f32, f32, f32,
                                      u16, f32, f64, f64, u8, f32]
            L.or_dequant_row.restype = None
            L.or_dequant_row.argtypes = [u8, C.c_float, f64]
            L.or_indexer_scores.restype = i
            L.or_indexer_scores.argtypes = [i, i, i64, i32, u8, u8, f32, u8, u8, f64, i]
            L.or_topk.restype = i
            L.or_topk.argtypes = [i64, i, f64, i32]
            L.or_e2m1_encode.restype = C.c_uint8
            L.or_e2m1_encode.argtypes = [d]
            L.or_mxfp4_block.restype = None
            L.or_mxfp4_block.argtypes = [f64, u8, u8]
            L.or_compress_index_keys.restype = i
            L.or_compress_index_keys.argtypes = [i, i, i, i, i64, u16, u16, f32, f32, f32, u16,
                                                 f32, i64, u8, u8, f64]
            L.or_indexer_query.restype = i
            L.or_indexer_query.argtypes = [i, i, i, u16, u16, u8, u8, f64]
            L.or_grouped_out_proj.restype = i
            L.or_grouped_out_proj.argtypes = [i, i, i, i, i, u16, u16, u16, f64, f64]
            L.or_topk_bf16.restype = i
            L.or_topk_bf16.argtypes = [i64, i, f64, i32]
            L.or_attention.restype = i
            L.or_attention.argtypes = [i, i, i, i64, i, u16, i32, i32, i32, u8, f32, u16,
                                       f32, d, d, i, f64, f64, i]
            L.or_swa_row.restype = None
            L.or_swa_row.argtypes = [u16, i64, d, d, f32, u16]
            L.or_prefill.restype = i
            L.or_prefill.argtypes = [i64, i, i, i, i, i, d, d, d, i, i, u16, u16, f32, f32, f32,
                                     f32, u16, f32, u8, f32, i64, u8, u8, f32, u8, u8, u16,
                                     f32, u16, i, i32, f64, f64, i32, i]
            _lib = L
    return _lib


def _c(a, dtype):
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


# ------------------------------------------------------------------ formats
def bf16_decode(h):
    h = np.asarray(h, dtype=np.uint16)
    return np.vectorize(lambda x: lib().or_bf16_decode(int(x)), otypes=[np.float64])(h)


def bf16_encode(x):
    return np.vectorize(lambda v: lib().or_bf16_encode(float(v)), otypes=[np.uint16])(x)


def e4m3_decode(c):
    return np.vectorize(lambda x: lib().or_e4m3_decode(int(x)), otypes=[np.float64])(c)


def e4m3_encode(x):
    return np.vectorize(lambda v: lib().or_e4m3_encode(float(v)), otypes=[np.uint8])(x)


def e2m1_decode(c):
    return np.vectorize(lambda x: lib().or_e2m1_decode(int(x)), otypes=[np.float64])(c)


def e8m0_decode(c):
    return np.vectorize(lambda x: lib().or_e8m0_decode(int(x)), otypes=[np.float64])(c)


def key_sf_offset(j: int, s: int) -> int:
    return int(lib().or_key_sf_offset(int(j), int(s)))


def dequant_rows(kv_rows: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """[n][576] stored rows + [n] scales -> [n][512] float64."""
    kv_rows = _c(kv_rows, np.uint8).reshape(-1, 576)
    scale = _c(scale, np.float32).reshape(-1)
    out = np.empty((kv_rows.shape[0], 512), dtype=np.float64)
    for r in range(kv_rows.shape[0]):
        lib().or_dequant_row(_p(kv_rows[r], C.c_uint8), float(scale[r]),
                             _p(out[r], C.c_double))
    return out


# ------------------------------------------------------------------ layer
def compress(a, za, bias, m: int, overlap: bool, b=None, zb=None, pos0: int = 0,
             prev_b=None, prev_zb=None, rope_base: float = 10000.0, eps: float = 1e-6,
             norm_w=None) -> dict:
    """a, b bf16 bits [B][T][512]; za, zb float32 [B][T][512] -> dict with e, y
    (float64 [B][N][512]), kv (uint8 [B][N][576]) and kv_scale (float32 [B][N])."""
    a = _c(a, np.uint16)
    B, T, _ = a.shape
    N = T // m
    e = np.empty((B, N, 512)); y = np.empty((B, N, 512))
    kv = np.empty((B, N, 576), dtype=np.uint8); sc = np.empty((B, N), dtype=np.float32)
    args = [_c(b, np.uint16), _c(za, np.float32), _c(zb, np.float32), _c(bias, np.float32),
            _c(norm_w, np.float32), _c(prev_b, np.uint16), _c(prev_zb, np.float32)]
    rc = lib().or_compress(B, T, m, int(overlap), pos0, rope_base, eps, _p(a, C.c_uint16),
                           _p(args[0], C.c_uint16), _p(args[1], C.c_float),
                           _p(args[2], C.c_float), _p(args[3], C.c_float),
                           _p(args[4], C.c_float), _p(args[5], C.c_uint16),
                           _p(args[6], C.c_float), _p(e, C.c_double), _p(y, C.c_double),
                           _p(kv, C.c_uint8), _p(sc, C.c_float))
    if rc:
        raise ValueError("oracle compress rejected its arguments")
    return {"e": e, "y": y, "kv": kv, "kv_scale": sc}


def indexer_scores(n_entries, q_fp4, q_sf, w, k_fp4, k_sf, nthreads: int = 0) -> np.ndarray:
    """-> float64 [B][Nmax] (NaN past n_entries[b])."""
    q_fp4 = _c(q_fp4, np.uint8)
    B, H_I, _ = q_fp4.shape
    k_fp4 = _c(k_fp4, np.uint8)
    Nmax = k_fp4.shape[1]
    n = _c(np.asarray(n_entries, dtype=np.int32), np.int32)
    out = np.empty((B, Nmax))
    qs, ww, ks = _c(q_sf, np.uint8), _c(w, np.float32), _c(k_sf, np.uint8)
    rc = lib().or_indexer_scores(B, H_I, Nmax, _p(n, C.c_int32), _p(q_fp4, C.c_uint8),
                                 _p(qs, C.c_uint8), _p(ww, C.c_float),
                                 _p(k_fp4, C.c_uint8), _p(ks, C.c_uint8),
                                 _p(out, C.c_double), nthreads)
    if rc:
        raise ValueError("oracle indexer rejected its arguments")
    return out


def topk(scores: np.ndarray, n: int, k: int) -> np.ndarray:
    s = _c(np.asarray(scores[:n], dtype=np.float64), np.float64)
    idx = np.empty(k, dtype=np.int32)
    if lib().or_topk(n, k, _p(s, C.c_double), _p(idx, C.c_int32)):
        raise ValueError("oracle topk rejected its arguments")
    return idx


def e2m1_encode(x):
    return np.vectorize(lambda v: lib().or_e2m1_encode(float(v)), otypes=[np.uint8])(x)


def mxfp4_block(v) -> tuple[np.ndarray, int]:
    """32 values -> (32 E2M1 codes, E8M0 scale code)."""
    v = _c(np.asarray(v, dtype=np.float64), np.float64)
    nib = np.empty(32, dtype=np.uint8)
    sf = np.zeros(1, dtype=np.uint8)
    lib().or_mxfp4_block(_p(v, C.c_double), _p(nib, C.c_uint8), _p(sf, C.c_uint8))
    return nib, int(sf[0])


def compress_index_keys(a, za, bias, m: int, overlap: bool, Nmax: int, b=None, zb=None,
                        pos0: int = 0, prev_b=None, prev_zb=None):
    """[B][T][128] indexer-key streams -> (k_fp4 [B][Nmax][64], k_sf [B][Nmax/128*512],
    y [B][N][128]); rows pos0/m .. pos0/m + N - 1 are written, the rest stay zero."""
    B, T, _ = a.shape
    N = T // m
    k_fp4 = np.zeros((B, Nmax, 64), dtype=np.uint8)
    k_sf = np.zeros((B, Nmax // 128 * 512), dtype=np.uint8)
    y = np.empty((B, N, 128))
    g = {x: _c(v, t) for x, v, t in (("a", a, np.uint16), ("b", b, np.uint16),
                                      ("za", za, np.float32), ("zb", zb, np.float32),
                                      ("bias", bias, np.float32), ("pb", prev_b, np.uint16),
                                      ("pz", prev_zb, np.float32))}
    rc = lib().or_compress_index_keys(
        B, T, m, int(overlap), pos0, _p(g["a"], C.c_uint16), _p(g["b"], C.c_uint16),
        _p(g["za"], C.c_float), _p(g["zb"], C.c_float), _p(g["bias"], C.c_float),
        _p(g["pb"], C.c_uint16), _p(g["pz"], C.c_float), Nmax, _p(k_fp4, C.c_uint8),
        _p(k_sf, C.c_uint8), _p(y, C.c_double))
    if rc:
        raise ValueError("oracle key compression rejected its arguments")
    return k_fp4, k_sf, y


def indexer_query(c, W, H_I: int):
    """c bf16 [T][r], W bf16 [H_I * 128][r] -> (q_fp4 [T][H_I][64], q_sf [T][H_I][4],
    y [T][H_I * 128])."""
    T, r = c.shape
    q_fp4 = np.empty((T, H_I, 64), dtype=np.uint8)
    q_sf = np.empty((T, H_I, 4), dtype=np.uint8)
    y = np.empty((T, H_I * 128))
    cc, ww = _c(c, np.uint16), _c(W, np.uint16)
    if lib().or_indexer_query(T, r, H_I, _p(cc, C.c_uint16), _p(ww, C.c_uint16),
                              _p(q_fp4, C.c_uint8), _p(q_sf, C.c_uint8), _p(y, C.c_double)):
        raise ValueError("oracle indexer query rejected its arguments")
    return q_fp4, q_sf, y


def grouped_out_proj(attn, Wg, Wo):
    """attn bf16 [T][H][512], Wg bf16 [G][d_g][H/G*512], Wo bf16 [d_model][G*d_g] ->
    (out [T][d_model], mid [T][G*d_g]) in float64."""
    T, H, _ = attn.shape
    G, d_g, _ = Wg.shape
    d_model = Wo.shape[0]
    out = np.empty((T, d_model))
    mid = np.empty((T, G * d_g))
    a, g, o = _c(attn, np.uint16), _c(Wg, np.uint16), _c(Wo, np.uint16)
    if lib().or_grouped_out_proj(T, H, G, d_g, d_model, _p(a, C.c_uint16), _p(g, C.c_uint16),
                                 _p(o, C.c_uint16), _p(out, C.c_double), _p(mid, C.c_double)):
        raise ValueError("oracle output projection rejected its arguments")
    return out, mid


def topk_bf16(scores: np.ndarray, n: int, k: int) -> np.ndarray:
    """Top-k on the scores rounded to BF16 (ties in the rounded value broken by index)."""
    s = _c(np.asarray(scores[:n], dtype=np.float64), np.float64)
    idx = np.empty(k, dtype=np.int32)
    if lib().or_topk_bf16(n, k, _p(s, C.c_double), _p(idx, C.c_int32)):
        raise ValueError("oracle topk rejected its arguments")
    return idx


def attention(q, pos, n_entries, kv, kv_scale, swa, sink, idx=None, k: int = 0,
              tau: float | None = None, rope_base: float = 10000.0, derotate: bool = True,
              nthreads: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """q bf16 bits [B][H][512]; kv [B][Nmax][576]; kv_scale [B][Nmax]; swa [B][128][512];
    idx [B][k] (CSA) or None (HCA: all n_entries) -> (out float64 [B][H][512], lse [B][H])."""
    q = _c(q, np.uint16)
    B, H, _ = q.shape
    kv = _c(kv, np.uint8)
    Nmax = kv.shape[1]
    sparse = idx is not None
    if sparse:
        idx = _c(np.asarray(idx, dtype=np.int32), np.int32)
        k = idx.shape[1]
    tau = 1.0 / np.sqrt(512.0) if tau is None else tau
    pos = _c(np.asarray(pos, dtype=np.int32), np.int32)
    n = _c(np.asarray(n_entries, dtype=np.int32), np.int32)
    sc, sw, sk = _c(kv_scale, np.float32), _c(swa, np.uint16), _c(sink, np.float32)
    out = np.empty((B, H, 512)); lse = np.empty((B, H))
    rc = lib().or_attention(B, H, k, Nmax, int(sparse), _p(q, C.c_uint16), _p(pos, C.c_int32),
                            _p(idx, C.c_int32), _p(n, C.c_int32), _p(kv, C.c_uint8),
                            _p(sc, C.c_float), _p(sw, C.c_uint16), _p(sk, C.c_float), tau,
                            rope_base, int(derotate), _p(out, C.c_double),
                            _p(lse, C.c_double), nthreads)
    if rc:
        raise ValueError("oracle attention rejected its arguments")
    return out, lse


def swa_row(a_row, t: int, rope_base: float = 10000.0, eps: float = 1e-6,
            norm_w=None) -> np.ndarray:
    a_row = _c(a_row, np.uint16)
    out = np.empty(512, dtype=np.uint16)
    nw = _c(norm_w, np.float32)
    lib().or_swa_row(_p(a_row, C.c_uint16), t, rope_base, eps, _p(nw, C.c_float),
                     _p(out, C.c_uint16))
    return out


def prefill(inp: dict, k: int, q_rows, tau: float | None = None, rope_base: float = 10000.0,
            eps: float = 1e-6, derotate: bool = True, strict: bool = False,
            nthreads: int = 0) -> dict:
    """Evaluate the rows `q_rows` of a prefill described by a synth.prefill_inputs dict
    (with an optional RMSNorm weight under "norm_w"). Returns out [nq][H][512], lse [nq][H],
    idx [nq][k] and the cache after compression. strict=True takes the eligibility
    n(t) = floor(t/m) (blocks completed before t) instead of floor((t+1)/m)."""
    P, T, m, H, H_I, Nmax = (inp[x] for x in ("P", "T", "m", "H", "H_I", "Nmax"))
    tau = 1.0 / np.sqrt(512.0) if tau is None else tau
    kv = np.array(inp["kv"], dtype=np.uint8, copy=True)
    sc = np.array(inp["kv_scale"], dtype=np.float32, copy=True)
    rows = _c(np.asarray(q_rows, dtype=np.int32), np.int32)
    nq = rows.shape[0]
    out = np.empty((nq, H, 512)); lse = np.empty((nq, H)); idx = np.empty((nq, k), np.int32)
    g = {x: _c(inp.get(x), t) for x, t in (
        ("a", np.uint16), ("b", np.uint16), ("za", np.float32), ("zb", np.float32),
        ("bias", np.float32), ("prev_b", np.uint16), ("prev_zb", np.float32),
        ("q_fp4", np.uint8), ("q_sf", np.uint8), ("w", np.float32), ("k_fp4", np.uint8),
        ("k_sf", np.uint8), ("q", np.uint16), ("sink", np.float32),
        ("swa_prefix", np.uint16), ("norm_w", np.float32))}
    U16, F32, U8 = C.c_uint16, C.c_float, C.c_uint8
    rc = lib().or_prefill(P, T, m, H, H_I, k, rope_base, eps, tau, int(derotate), int(strict),
                          _p(g["a"], U16), _p(g["b"], U16), _p(g["za"], F32),
                          _p(g["zb"], F32), _p(g["bias"], F32), _p(g["norm_w"], F32),
                          _p(g["prev_b"], U16), _p(g["prev_zb"], F32), _p(kv, U8),
                          _p(sc, F32), Nmax, _p(g["q_fp4"], U8), _p(g["q_sf"], U8),
                          _p(g["w"], F32), _p(g["k_fp4"], U8), _p(g["k_sf"], U8),
                          _p(g["q"], U16), _p(g["sink"], F32), _p(g["swa_prefix"], U16),
                          nq, _p(rows, C.c_int32), _p(out, C.c_double), _p(lse, C.c_double),
                          _p(idx, C.c_int32), nthreads)
    if rc:
        raise ValueError("oracle prefill rejected its arguments")
    return {"out": out, "lse": lse, "idx": idx, "kv": kv, "kv_scale": sc}


# ------------------------------------------------------------------ paged cache
# The classical cache of compressed entries (walkthrough §3.5) kept in pages: pools of
# pages that hold page_entries entries each, and a block table per sequence naming the
# page of each logical page of the sequence. Entry j of sequence b lives in slot
# j % page_entries of page block_table[b][j // page_entries]. Arrays grouped by 128 entries
# (the indexer key scales, 512 bytes per group) page by whole groups: group g of sequence
# b is group (g * 128 % page_entries) / 128 of page block_table[b][g * 128 // page_entries].
# These two functions are the definition the paged kernels are checked against: the
# oracle's own computations take the contiguous view.

def paged_view(pool, block_table, page_entries: int, group: int = 1) -> np.ndarray:
    """Contiguous per-sequence view [B][pages_max * page_entries / group][...] of a pool
    [num_pages][page_entries / group][...]; units on table entries outside the pool
    (e.g. -1 for pages not yet given) read as zeros."""
    pool = np.asarray(pool)
    table = np.asarray(block_table, dtype=np.int64)
    B, pages_max = table.shape
    per_page = page_entries // group
    out = np.zeros((B, pages_max * per_page) + pool.shape[2:], dtype=pool.dtype)
    for b in range(B):
        for lp in range(pages_max):
            page = int(table[b, lp])
            if 0 <= page < pool.shape[0]:
                out[b, lp * per_page:(lp + 1) * per_page] = pool[page]
    return out


def paged_scatter(view, block_table, page_entries: int, num_pages: int,
                  group: int = 1) -> np.ndarray:
    """The pool [num_pages][page_entries / group][...] that holds each sequence's units of
    a contiguous view [B][units][...] at the places the block table names (pages the
    table does not name are zero)."""
    view = np.asarray(view)
    table = np.asarray(block_table, dtype=np.int64)
    B, pages_max = table.shape
    per_page = page_entries // group
    pool = np.zeros((num_pages, per_page) + view.shape[2:], dtype=view.dtype)
    for b in range(B):
        for lp in range(pages_max):
            page = int(table[b, lp])
            lo = lp * per_page
            if 0 <= page < num_pages and lo < view.shape[1]:
                hi = min(lo + per_page, view.shape[1])
                pool[page, :hi - lo] = view[b, lo:hi]
    return pool
