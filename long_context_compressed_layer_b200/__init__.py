"""Python binding of the B200 CSA/HCA compressed attention library (libcsa_b200.so).

Argument marshalling only: every step of the layer runs in the sm_100a kernels behind the
C ABI declared in include/csa.h. PyTorch supplies device memory and the current stream.
If the shared library is missing the import of a function raises; there is no fallback.

bf16 inputs may be torch.bfloat16 tensors or 16-bit integer tensors holding bf16 bits.
"""

from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa_b200.so")

HEAD_DIM, NOPE_DIM, ROPE_DIM, ROW_BYTES, INDEX_DIM, WINDOW = 512, 448, 64, 576, 128, 128

CSA_OK, CSA_ERR_INVALID_ARG, CSA_ERR_UNSUPPORTED, CSA_ERR_WORKSPACE = 0, 1, 2, 3
CSA_ERR_CUDA, CSA_ERR_DEVICE, CSA_ERR_TIMEOUT = 4, 5, 6
TOPK_SEPARATE_SELECT = 1

_vp = C.c_void_p


class CompressArgs(C.Structure):
    _fields_ = [("B", C.c_int32), ("T", C.c_int32), ("m", C.c_int32), ("overlap", C.c_int32),
                ("pos0", C.c_int64), ("rope_base", C.c_float), ("eps", C.c_float),
                ("a", _vp), ("b", _vp), ("za", _vp), ("zb", _vp), ("bias", _vp),
                ("norm_w", _vp), ("prev_b", _vp), ("prev_zb", _vp), ("kv", _vp),
                ("kv_scale", _vp), ("Nmax", C.c_int64), ("dbg", _vp)]


class IkeyArgs(C.Structure):
    _fields_ = [("B", C.c_int32), ("T", C.c_int32), ("m", C.c_int32), ("overlap", C.c_int32),
                ("pos0", C.c_int64), ("a", _vp), ("b", _vp), ("za", _vp), ("zb", _vp),
                ("bias", _vp), ("prev_b", _vp), ("prev_zb", _vp), ("k_fp4", _vp),
                ("k_sf", _vp), ("Nmax", C.c_int64), ("dbg", _vp)]


class IqueryArgs(C.Structure):
    _fields_ = [("T", C.c_int32), ("r", C.c_int32), ("H_I", C.c_int32), ("c", _vp), ("W", _vp),
                ("q_fp4", _vp), ("q_sf", _vp), ("dbg", _vp), ("dev_status", _vp)]


class OprojArgs(C.Structure):
    _fields_ = [("T", C.c_int32), ("H", C.c_int32), ("G", C.c_int32), ("d_g", C.c_int32),
                ("d_model", C.c_int32), ("attn", _vp), ("Wg", _vp), ("Wo", _vp), ("out", _vp),
                ("dev_status", _vp)]


class Pages(C.Structure):
    """csa_pages: the block table of a paged compressed cache (all zero: contiguous)."""
    _fields_ = [("block_table", _vp), ("pages_max", C.c_int32), ("page_entries", C.c_int32),
                ("num_pages", C.c_int32)]


class Paging:
    """A paged compressed cache: block_table int32 [B][pages_max] (device) names the pool
    page of each logical page of page_entries entries; Nmax is the entry capacity per
    sequence (default pages_max * page_entries). Pools are kv uint8
    [num_pages][page_entries][576], kv_scale float32 [num_pages][page_entries], k_fp4 uint8
    [num_pages][page_entries][64] and k_sf uint8 [num_pages][page_entries // 128][512]."""

    def __init__(self, block_table: torch.Tensor, page_entries: int, Nmax: int | None = None):
        if block_table.dtype != torch.int32 or block_table.dim() != 2:
            raise ValueError("block_table: int32 [B][pages_max]")
        self.block_table = block_table.contiguous()
        self.page_entries = int(page_entries)
        self.pages_max = block_table.shape[1]
        self.Nmax = int(Nmax) if Nmax is not None else self.pages_max * self.page_entries

    def struct(self, pool_entries: int) -> Pages:
        return Pages(_ptr(self.block_table, elem=4, name="block_table"), self.pages_max,
                     self.page_entries, pool_entries // self.page_entries)


def _pages(paging: "Paging | None", pool_entries: int, B: int) -> Pages:
    if paging is None:
        return Pages()
    if paging.block_table.shape[0] != B:
        raise ValueError(f"block_table: {paging.block_table.shape[0]} rows for {B} sequences")
    if pool_entries % paging.page_entries:
        raise ValueError("pool size is not a whole number of pages")
    return paging.struct(pool_entries)


class AppendArgs(C.Structure):
    _fields_ = [("B", C.c_int32), ("m", C.c_int32), ("overlap", C.c_int32),
                ("rope_base", C.c_float), ("eps", C.c_float), ("pos", _vp), ("a", _vp),
                ("b", _vp), ("za", _vp), ("zb", _vp), ("bias", _vp), ("norm_w", _vp),
                ("tail_a", _vp), ("tail_za", _vp), ("tail_b", _vp), ("tail_zb", _vp),
                ("swa", _vp), ("kv", _vp), ("kv_scale", _vp), ("Nmax", C.c_int64),
                ("n_entries", _vp), ("ia", _vp), ("ib", _vp), ("iza", _vp), ("izb", _vp),
                ("ibias", _vp), ("itail_a", _vp), ("itail_za", _vp), ("itail_b", _vp),
                ("itail_zb", _vp), ("k_fp4", _vp), ("k_sf", _vp), ("dev_status", _vp),
                ("pages", Pages)]


class TopkArgs(C.Structure):
    _fields_ = [("B", C.c_int32), ("H_I", C.c_int32), ("k", C.c_int32), ("Nmax", C.c_int64),
                ("n_entries", _vp), ("q_fp4", _vp), ("q_sf", _vp), ("w", _vp),
                ("k_fp4", _vp), ("k_sf", _vp), ("idx", _vp), ("scores", _vp),
                ("dev_status", _vp), ("flags", C.c_uint32), ("select_wait_ns", C.c_int64),
                ("pages", Pages)]


class AttnArgs(C.Structure):
    _fields_ = [("B", C.c_int32), ("H", C.c_int32), ("k", C.c_int32), ("Nmax", C.c_int64),
                ("q", _vp), ("pos", _vp), ("idx", _vp), ("n_entries", _vp), ("kv", _vp),
                ("kv_scale", _vp), ("swa", _vp), ("sink", _vp), ("tau", C.c_float),
                ("rope_base", C.c_float), ("derotate", C.c_int32), ("out", _vp), ("lse", _vp),
                ("dev_status", _vp), ("pages", Pages)]


class PrefillArgs(C.Structure):
    _fields_ = [("P", C.c_int64), ("T", C.c_int32), ("m", C.c_int32), ("H", C.c_int32),
                ("H_I", C.c_int32), ("k", C.c_int32), ("Nmax", C.c_int64), ("tau", C.c_float),
                ("rope_base", C.c_float), ("eps", C.c_float), ("derotate", C.c_int32),
                ("strict_eligibility", C.c_int32),
                ("a", _vp), ("b", _vp), ("za", _vp), ("zb", _vp), ("bias", _vp),
                ("norm_w", _vp), ("prev_b", _vp), ("prev_zb", _vp), ("kv", _vp),
                ("kv_scale", _vp), ("q_fp4", _vp), ("q_sf", _vp), ("w", _vp), ("k_fp4", _vp),
                ("k_sf", _vp), ("q", _vp), ("sink", _vp), ("swa_prefix", _vp), ("out", _vp),
                ("lse", _vp), ("idx", _vp), ("dev_status", _vp), ("pages", Pages)]


EXPORTS = ["csa_status_string", "csa_compress", "csa_compress_index_keys", "csa_decode_append",
           "csa_indexer_query", "csa_grouped_out_proj_workspace_size", "csa_grouped_out_proj",
           "csa_indexer_topk_workspace_size",
           "csa_indexer_topk", "csa_indexer_topk_bf16", "csa_attn_workspace_size", "csa_sparse_attn_decode",
           "hca_attn_decode", "csa_sparse_attn_decode_noalloc", "csa_prefill_workspace_size",
           "csa_prefill", "csa_mma_peak", "csa_mma_peak_flops"]

NOALLOC_SCRATCH_BYTES = 12 << 20

_lib = None


def lib() -> C.CDLL:
    """Load libcsa_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m long_context_compressed_layer_b200.build`")
        L = C.CDLL(LIB_PATH)
        L.csa_status_string.restype = C.c_char_p
        L.csa_status_string.argtypes = [C.c_int]
        L.csa_compress.restype = C.c_int
        L.csa_compress.argtypes = [C.POINTER(CompressArgs), _vp]
        L.csa_decode_append.restype = C.c_int
        L.csa_decode_append.argtypes = [C.POINTER(AppendArgs), _vp]
        L.csa_compress_index_keys.restype = C.c_int
        L.csa_compress_index_keys.argtypes = [C.POINTER(IkeyArgs), _vp]
        L.csa_indexer_query.restype = C.c_int
        L.csa_indexer_query.argtypes = [C.POINTER(IqueryArgs), _vp]
        L.csa_grouped_out_proj_workspace_size.restype = C.c_size_t
        L.csa_grouped_out_proj_workspace_size.argtypes = [C.c_int32, C.c_int32, C.c_int32]
        L.csa_grouped_out_proj.restype = C.c_int
        L.csa_grouped_out_proj.argtypes = [C.POINTER(OprojArgs), _vp, C.c_size_t, _vp]
        L.csa_indexer_topk_workspace_size.restype = C.c_size_t
        L.csa_indexer_topk_workspace_size.argtypes = [C.c_int32, C.c_int64, C.c_int32]
        for f in ("csa_indexer_topk", "csa_indexer_topk_bf16"):
            getattr(L, f).restype = C.c_int
            getattr(L, f).argtypes = [C.POINTER(TopkArgs), _vp, C.c_size_t, _vp]
        L.csa_attn_workspace_size.restype = C.c_size_t
        L.csa_attn_workspace_size.argtypes = [C.c_int32, C.c_int32, C.c_int32]
        for f in ("csa_sparse_attn_decode", "hca_attn_decode"):
            getattr(L, f).restype = C.c_int
            getattr(L, f).argtypes = [C.POINTER(AttnArgs), _vp, C.c_size_t, _vp]
        L.csa_prefill_workspace_size.restype = C.c_size_t
        L.csa_prefill_workspace_size.argtypes = [C.c_int32, C.c_int64, C.c_int32, C.c_int32]
        L.csa_prefill.restype = C.c_int
        L.csa_prefill.argtypes = [C.POINTER(PrefillArgs), _vp, C.c_size_t, _vp]
        L.csa_sparse_attn_decode_noalloc.restype = C.c_int
        L.csa_sparse_attn_decode_noalloc.argtypes = [C.POINTER(AttnArgs), _vp]
        L.csa_mma_peak.restype = C.c_int
        L.csa_mma_peak.argtypes = [C.c_int32, C.c_int32, C.c_int32, _vp, _vp]
        L.csa_mma_peak_flops.restype = C.c_double
        L.csa_mma_peak_flops.argtypes = [C.c_int32, C.c_int32, C.c_int32]
        _lib = L
    return _lib


class CSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {lib().csa_status_string(status).decode()} ({status})")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != CSA_OK:
        raise CSAError(status, where)


def _ptr(t: torch.Tensor | None, *, elem: int | None = None, name: str = "") -> int | None:
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        # the kernels run on the current device and would dereference another GPU's memory
        raise ValueError(f"{name}: on {t.device}, but the current device is "
                         f"cuda:{torch.cuda.current_device()}")
    if elem is not None and t.element_size() != elem:
        raise ValueError(f"{name}: expected {elem}-byte elements, got {t.dtype}")
    return t.data_ptr()


def _sizes(**named) -> None:
    """Each named (tensor, n): a given tensor must hold at least n elements, the count its
    layout needs; a shorter buffer would let a kernel read or write past its end."""
    for name, (t, n) in named.items():
        if t is not None and t.numel() < n:
            raise ValueError(f"{name}: expected at least {n} elements, got {t.numel()} "
                             f"(shape {tuple(t.shape)})")


def _dim(t, axis: int, n: int, name: str) -> None:
    if t.shape[axis] != n:
        raise ValueError(f"{name}: dimension {axis} must be {n}, got shape {tuple(t.shape)}")


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ------------------------------------------------------------------ compress
def compress(a, za, bias, m: int, overlap: bool, *, b=None, zb=None, pos0: int = 0,
             prev_b=None, prev_zb=None, kv=None, kv_scale=None, Nmax: int | None = None,
             rope_base: float = 10000.0, eps: float = 1e-6, norm_w=None, dbg: bool = False,
             stream=None):
    """Compress a [B][T][512] stream into entries pos0/m .. pos0/m + T/m - 1.
    Returns (kv [B][Nmax][576] uint8, kv_scale [B][Nmax] float32, dbg [B][N][512] or None);
    kv/kv_scale are written in place when given."""
    B, T, _ = a.shape
    _dim(a, 2, HEAD_DIM, "a")
    N = T // m
    if Nmax is None:
        Nmax = kv.shape[1] if kv is not None else pos0 // m + N
    tok = B * T * HEAD_DIM
    _sizes(za=(za, tok), b=(b, tok), zb=(zb, tok), bias=(bias, 2 * m if overlap else m),
           norm_w=(norm_w, HEAD_DIM), prev_b=(prev_b, B * m * HEAD_DIM),
           prev_zb=(prev_zb, B * m * HEAD_DIM), kv=(kv, B * Nmax * ROW_BYTES),
           kv_scale=(kv_scale, B * Nmax))
    dev = a.device
    if kv is None:
        kv = torch.zeros((B, Nmax, ROW_BYTES), dtype=torch.uint8, device=dev)
    if kv_scale is None:
        kv_scale = torch.zeros((B, Nmax), dtype=torch.float32, device=dev)
    d = torch.empty((B, N, HEAD_DIM), dtype=torch.float32, device=dev) if dbg else None
    args = CompressArgs(B, T, m, int(overlap), pos0, rope_base, eps,
                        _ptr(a, elem=2, name="a"), _ptr(b, elem=2, name="b"),
                        _ptr(za, elem=4, name="za"), _ptr(zb, elem=4, name="zb"),
                        _ptr(bias, elem=4, name="bias"), _ptr(norm_w, elem=4, name="norm_w"),
                        _ptr(prev_b, elem=2, name="prev_b"), _ptr(prev_zb, elem=4, name="prev_zb"),
                        _ptr(kv, elem=1, name="kv"), _ptr(kv_scale, elem=4, name="kv_scale"),
                        Nmax, _ptr(d, elem=4, name="dbg"))
    _check(lib().csa_compress(C.byref(args), _stream(stream)), "csa_compress")
    return kv, kv_scale, d


def new_decode_state(B: int, Nmax: int, m: int = 4, index_keys: bool = True, device="cuda"):
    """Zeroed per-sequence decode state: block tails, the window ring, the compressed cache
    and (optionally) the indexer-key tails and keys."""
    z = lambda shape, dt: torch.zeros(shape, dtype=dt, device=device)
    st = {"tail_a": z((B, m, HEAD_DIM), torch.int16), "tail_za": z((B, m, HEAD_DIM), torch.float32),
          "tail_b": z((B, 2, m, HEAD_DIM), torch.int16),
          "tail_zb": z((B, 2, m, HEAD_DIM), torch.float32),
          "swa": z((B, WINDOW, HEAD_DIM), torch.int16), "kv": z((B, Nmax, ROW_BYTES), torch.uint8),
          "kv_scale": z((B, Nmax), torch.float32), "n_entries": z((B,), torch.int32)}
    if index_keys:
        st.update({"itail_a": z((B, m, INDEX_DIM), torch.int16),
                   "itail_za": z((B, m, INDEX_DIM), torch.float32),
                   "itail_b": z((B, 2, m, INDEX_DIM), torch.int16),
                   "itail_zb": z((B, 2, m, INDEX_DIM), torch.float32),
                   "k_fp4": z((B, Nmax, 64), torch.uint8),
                   "k_sf": z((B, Nmax // 128 * 512), torch.uint8)})
    return st


def decode_append(pos, a, za, bias, state, *, b=None, zb=None, m: int = 4, overlap: bool = True,
                  norm_w=None, rope_base: float = 10000.0, eps: float = 1e-6, ia=None, ib=None,
                  iza=None, izb=None, ibias=None, dev_status=None,
                  paging: Paging | None = None, stream=None):
    """Append one token per sequence (a, b bf16 [B][512]; za, zb [B][512]; ia.. [B][128]) at
    positions pos [B] to a state from new_decode_state. With paging, the state's kv,
    kv_scale, k_fp4 and k_sf are page pools (Paging) and a closed block's entry goes to
    the slot its block table names."""
    B = a.shape[0]
    _dim(a, -1, HEAD_DIM, "a")
    if paging is None:
        Nmax, pool = state["kv"].shape[1], B * state["kv"].shape[1]
    else:
        Nmax, pool = paging.Nmax, state["kv"].numel() // ROW_BYTES
    row, irow = B * HEAD_DIM, B * INDEX_DIM
    _sizes(pos=(pos, B), za=(za, row), b=(b, row), zb=(zb, row),
           bias=(bias, 2 * m if overlap else m), norm_w=(norm_w, HEAD_DIM), ia=(ia, irow),
           ib=(ib, irow), iza=(iza, irow), izb=(izb, irow), ibias=(ibias, 2 * m),
           tail_a=(state["tail_a"], B * m * HEAD_DIM), tail_za=(state["tail_za"], B * m * HEAD_DIM),
           tail_b=(state.get("tail_b"), 2 * B * m * HEAD_DIM),
           tail_zb=(state.get("tail_zb"), 2 * B * m * HEAD_DIM),
           swa=(state["swa"], B * WINDOW * HEAD_DIM), kv=(state["kv"], pool * ROW_BYTES),
           kv_scale=(state["kv_scale"], pool), n_entries=(state["n_entries"], B))
    if ia is not None:
        _sizes(itail_a=(state["itail_a"], B * m * INDEX_DIM),
               itail_za=(state["itail_za"], B * m * INDEX_DIM),
               itail_b=(state["itail_b"], 2 * B * m * INDEX_DIM),
               itail_zb=(state["itail_zb"], 2 * B * m * INDEX_DIM),
               k_fp4=(state["k_fp4"], pool * 64), k_sf=(state["k_sf"], pool // 128 * 512))
    pg = _pages(paging, pool, B)
    g = lambda k_, el: _ptr(state.get(k_), elem=el, name=k_)
    args = AppendArgs(B, m, int(overlap), rope_base, eps, _ptr(pos, elem=4, name="pos"),
                      _ptr(a, elem=2, name="a"), _ptr(b, elem=2, name="b"),
                      _ptr(za, elem=4, name="za"), _ptr(zb, elem=4, name="zb"),
                      _ptr(bias, elem=4, name="bias"), _ptr(norm_w, elem=4, name="norm_w"),
                      g("tail_a", 2), g("tail_za", 4), g("tail_b", 2), g("tail_zb", 4),
                      g("swa", 2), g("kv", 1), g("kv_scale", 4), Nmax,
                      g("n_entries", 4), _ptr(ia, elem=2, name="ia"), _ptr(ib, elem=2, name="ib"),
                      _ptr(iza, elem=4, name="iza"), _ptr(izb, elem=4, name="izb"),
                      _ptr(ibias, elem=4, name="ibias"),
                      g("itail_a", 2) if ia is not None else None,
                      g("itail_za", 4) if ia is not None else None,
                      g("itail_b", 2) if ia is not None else None,
                      g("itail_zb", 4) if ia is not None else None,
                      g("k_fp4", 1) if ia is not None else None,
                      g("k_sf", 1) if ia is not None else None,
                      _ptr(dev_status, elem=4, name="dev_status"), pg)
    _check(lib().csa_decode_append(C.byref(args), _stream(stream)), "csa_decode_append")


def compress_index_keys(a, za, bias, m: int, overlap: bool, *, b=None, zb=None, pos0: int = 0,
                        prev_b=None, prev_zb=None, k_fp4=None, k_sf=None,
                        Nmax: int | None = None, dbg: bool = False, stream=None):
    """Compress a [B][T][128] indexer-key stream into MXFP4 keys at rows pos0/m ...
    Returns (k_fp4 [B][Nmax][64], k_sf [B][Nmax/128*512], dbg [B][N][128] or None);
    k_fp4 / k_sf are written in place when given."""
    B, T, _ = a.shape
    _dim(a, 2, INDEX_DIM, "a")
    N = T // m
    if Nmax is None:
        Nmax = k_fp4.shape[1] if k_fp4 is not None else -(-(pos0 // m + N) // 128) * 128
    tok = B * T * INDEX_DIM
    _sizes(za=(za, tok), b=(b, tok), zb=(zb, tok), bias=(bias, 2 * m if overlap else m),
           prev_b=(prev_b, B * m * INDEX_DIM), prev_zb=(prev_zb, B * m * INDEX_DIM),
           k_fp4=(k_fp4, B * Nmax * 64), k_sf=(k_sf, B * Nmax // 128 * 512))
    dev = a.device
    if k_fp4 is None:
        k_fp4 = torch.zeros((B, Nmax, 64), dtype=torch.uint8, device=dev)
    if k_sf is None:
        k_sf = torch.zeros((B, Nmax // 128 * 512), dtype=torch.uint8, device=dev)
    d = torch.empty((B, N, INDEX_DIM), dtype=torch.float32, device=dev) if dbg else None
    args = IkeyArgs(B, T, m, int(overlap), pos0, _ptr(a, elem=2, name="a"),
                    _ptr(b, elem=2, name="b"), _ptr(za, elem=4, name="za"),
                    _ptr(zb, elem=4, name="zb"), _ptr(bias, elem=4, name="bias"),
                    _ptr(prev_b, elem=2, name="prev_b"), _ptr(prev_zb, elem=4, name="prev_zb"),
                    _ptr(k_fp4, elem=1, name="k_fp4"), _ptr(k_sf, elem=1, name="k_sf"), Nmax,
                    _ptr(d, elem=4, name="dbg"))
    _check(lib().csa_compress_index_keys(C.byref(args), _stream(stream)),
           "csa_compress_index_keys")
    return k_fp4, k_sf, d


def indexer_query(c, W, H_I: int, *, q_fp4=None, q_sf=None, dbg: bool = False,
                  dev_status=None, stream=None):
    """Indexer queries of T tokens: c bf16 [T][r], W bf16 [H_I * 128][r] -> (q_fp4
    [T][H_I][64], q_sf [T][H_I][4], dbg [T][H_I * 128] or None)."""
    T, r = c.shape
    _sizes(W=(W, H_I * INDEX_DIM * r), q_fp4=(q_fp4, T * H_I * 64), q_sf=(q_sf, T * H_I * 4))
    dev = c.device
    if q_fp4 is None:
        q_fp4 = torch.empty((T, H_I, 64), dtype=torch.uint8, device=dev)
    if q_sf is None:
        q_sf = torch.empty((T, H_I, 4), dtype=torch.uint8, device=dev)
    d = torch.empty((T, H_I * 128), dtype=torch.float32, device=dev) if dbg else None
    args = IqueryArgs(T, r, H_I, _ptr(c, elem=2, name="c"), _ptr(W, elem=2, name="W"),
                      _ptr(q_fp4, elem=1, name="q_fp4"), _ptr(q_sf, elem=1, name="q_sf"),
                      _ptr(d, elem=4, name="dbg"), _ptr(dev_status, elem=4, name="dev_status"))
    _check(lib().csa_indexer_query(C.byref(args), _stream(stream)), "csa_indexer_query")
    return q_fp4, q_sf, d


def grouped_out_proj(attn, Wg, Wo, *, workspace=None, out=None, dev_status=None, stream=None):
    """attn bf16 [T][H][512], Wg bf16 [G][d_g][H/G*512], Wo bf16 [d_model][G*d_g] ->
    out bf16 [T][d_model]."""
    T, H, _ = attn.shape
    _dim(attn, 2, HEAD_DIM, "attn")
    G, d_g, _ = Wg.shape
    d_model = Wo.shape[0]
    _sizes(Wg=(Wg, G * d_g * (H // G) * HEAD_DIM), Wo=(Wo, d_model * G * d_g),
           out=(out, T * d_model))
    dev = attn.device
    if workspace is None:
        n = lib().csa_grouped_out_proj_workspace_size(T, G, d_g)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
    if out is None:
        out = torch.empty((T, d_model), dtype=torch.bfloat16, device=dev)
    args = OprojArgs(T, H, G, d_g, d_model, _ptr(attn, elem=2, name="attn"),
                     _ptr(Wg, elem=2, name="Wg"), _ptr(Wo, elem=2, name="Wo"),
                     _ptr(out, elem=2, name="out"), _ptr(dev_status, elem=4, name="dev_status"))
    _check(lib().csa_grouped_out_proj(C.byref(args), workspace.data_ptr(), workspace.numel(),
                                      _stream(stream)), "csa_grouped_out_proj")
    return out


# ------------------------------------------------------------- indexer top-k
def mma_peak(kind: int, N: int, iters: int, *, dev_status=None, stream=None) -> float:
    """Launch csa_mma_peak (a tensor-pipe throughput measurement: kind 0 = MXFP4 N = 64,
    kind 1 = BF16 N = 64 or 256) on the stream; returns the FLOPs of the launch, which the
    caller divides by the time it measures."""
    _check(lib().csa_mma_peak(kind, N, iters, _ptr(dev_status, elem=4, name="dev_status"),
                              _stream(stream)), "csa_mma_peak")
    return float(lib().csa_mma_peak_flops(kind, N, iters))


def indexer_topk_workspace(B: int, Nmax: int, k: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace (the library keeps it zeroed between calls)."""
    n = lib().csa_indexer_topk_workspace_size(B, Nmax, k)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


def indexer_topk(n_entries, q_fp4, q_sf, w, k_fp4, k_sf, k: int, *, workspace=None, idx=None,
                 scores: bool = False, bf16_scores: bool = False, dev_status=None,
                 separate_select: bool = False, select_wait_ns: int = 0,
                 paging: Paging | None = None, stream=None):
    """Top-k entry indices [B][k] (ascending, -1 padded) and optionally their scores.
    bf16_scores selects on scores rounded to BF16 (csa_indexer_topk_bf16).
    separate_select runs the selection as separate kernels instead of inside the
    cooperative scoring launch; select_wait_ns bounds that launch's grid-barrier waits
    (0 = the library default). After a call whose dev_status reports an error, zero-fill
    the workspace before reusing it. With paging, k_fp4 / k_sf are page pools (Paging)."""
    B, H_I, _ = q_fp4.shape
    _dim(q_fp4, 2, 64, "q_fp4")
    if paging is None:
        Nmax, pool = k_fp4.shape[1], B * k_fp4.shape[1]
    else:
        Nmax, pool = paging.Nmax, k_fp4.numel() // 64
    _sizes(n_entries=(n_entries, B), q_sf=(q_sf, B * H_I * 4), w=(w, B * H_I),
           k_fp4=(k_fp4, pool * 64), k_sf=(k_sf, pool // 128 * 512), idx=(idx, B * k))
    pg = _pages(paging, pool, B)
    dev = q_fp4.device
    if workspace is None:
        workspace = indexer_topk_workspace(B, Nmax, k, dev)
    if idx is None:
        idx = torch.empty((B, k), dtype=torch.int32, device=dev)
    sc = torch.empty((B, k), dtype=torch.float32, device=dev) if scores else None
    args = TopkArgs(B, H_I, k, Nmax, _ptr(n_entries, elem=4, name="n_entries"),
                    _ptr(q_fp4, elem=1, name="q_fp4"), _ptr(q_sf, elem=1, name="q_sf"),
                    _ptr(w, elem=4, name="w"), _ptr(k_fp4, elem=1, name="k_fp4"),
                    _ptr(k_sf, elem=1, name="k_sf"), _ptr(idx, elem=4, name="idx"),
                    _ptr(sc, elem=4, name="scores"), _ptr(dev_status, elem=4, name="dev_status"),
                    TOPK_SEPARATE_SELECT if separate_select else 0, int(select_wait_ns), pg)
    fn = "csa_indexer_topk_bf16" if bf16_scores else "csa_indexer_topk"
    _check(getattr(lib(), fn)(C.byref(args), workspace.data_ptr(), workspace.numel(),
                              _stream(stream)), fn)
    return (idx, sc) if scores else idx


# ------------------------------------------------------------------ attention
def attn_workspace(B: int, H: int, rows_max: int, device="cuda") -> torch.Tensor:
    n = lib().csa_attn_workspace_size(B, H, rows_max)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def _attn(fn: str, sparse: bool, q, pos, n_entries, kv, kv_scale, swa, sink, idx, *,
          tau: float = 0.0, rope_base: float = 10000.0, derotate: bool = True,
          workspace=None, out=None, lse: bool = False, dev_status=None,
          paging: Paging | None = None, stream=None):
    B, H, _ = q.shape
    _dim(q, 2, HEAD_DIM, "q")
    if paging is None:
        Nmax, pool = kv.shape[1], B * kv.shape[1]
    else:
        Nmax, pool = paging.Nmax, kv.numel() // ROW_BYTES
    k = idx.shape[1] if sparse else 0
    _sizes(pos=(pos, B), n_entries=(n_entries, B), kv=(kv, pool * ROW_BYTES),
           kv_scale=(kv_scale, pool), swa=(swa, B * WINDOW * HEAD_DIM), sink=(sink, H),
           idx=(idx if sparse else None, B * k), out=(out, B * H * HEAD_DIM))
    pg = _pages(paging, pool, B)
    dev = q.device
    noalloc = fn.endswith("_noalloc")
    if workspace is None and not noalloc:
        workspace = attn_workspace(B, H, (k if sparse else Nmax) + WINDOW, dev)
    if out is None:
        out = torch.empty((B, H, HEAD_DIM), dtype=torch.bfloat16, device=dev)
    l = torch.empty((B, H), dtype=torch.float32, device=dev) if lse else None
    args = AttnArgs(B, H, k, Nmax, _ptr(q, elem=2, name="q"), _ptr(pos, elem=4, name="pos"),
                    _ptr(idx, elem=4, name="idx") if sparse else None,
                    _ptr(n_entries, elem=4, name="n_entries"), _ptr(kv, elem=1, name="kv"),
                    _ptr(kv_scale, elem=4, name="kv_scale"), _ptr(swa, elem=2, name="swa"),
                    _ptr(sink, elem=4, name="sink"), tau, rope_base, int(derotate),
                    _ptr(out, elem=2, name="out"), _ptr(l, elem=4, name="lse"),
                    _ptr(dev_status, elem=4, name="dev_status"), pg)
    if noalloc:
        _check(getattr(lib(), fn)(C.byref(args), _stream(stream)), fn)
    else:
        _check(getattr(lib(), fn)(C.byref(args), workspace.data_ptr(), workspace.numel(),
                                  _stream(stream)), fn)
    return (out, l) if lse else out


def sparse_attn_decode(q, pos, n_entries, kv, kv_scale, swa, sink, idx, **kw):
    """CSA decode: MQA over idx [B][k] + window + sink -> bf16 [B][H][512] (and lse)."""
    return _attn("csa_sparse_attn_decode", True, q, pos, n_entries, kv, kv_scale, swa, sink,
                 idx, **kw)


def sparse_attn_decode_noalloc(q, pos, n_entries, kv, kv_scale, swa, sink, idx, **kw):
    """sparse_attn_decode with the library's static per-device scratch instead of a workspace
    (no scratch allocation; overlapping calls on one device race on the shared scratch)."""
    if kw.get("workspace") is not None:
        raise ValueError("sparse_attn_decode_noalloc takes no workspace")
    return _attn("csa_sparse_attn_decode_noalloc", True, q, pos, n_entries, kv, kv_scale, swa,
                 sink, idx, **kw)


def hca_attn_decode(q, pos, n_entries, kv, kv_scale, swa, sink, **kw):
    """HCA decode: MQA over all n_entries[b] entries + window + sink."""
    return _attn("hca_attn_decode", False, q, pos, n_entries, kv, kv_scale, swa, sink, None,
                 **kw)


# -------------------------------------------------------------------- prefill
def prefill_workspace(T: int, Nmax: int, H: int, k: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace (the parts that must start at zero are left zeroed)."""
    n = lib().csa_prefill_workspace_size(T, Nmax, H, k)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


def prefill(P: int, m: int, k: int, *, a, b, za, zb, bias, kv, kv_scale, q_fp4, q_sf, w,
            k_fp4, k_sf, q, sink, prev_b=None, prev_zb=None, swa_prefix=None, norm_w=None,
            tau: float = 0.0, rope_base: float = 10000.0, eps: float = 1e-6,
            derotate: bool = True, strict_eligibility: bool = False, workspace=None,
            out=None, lse: bool = False, idx: bool = False, dev_status=None,
            paging: Paging | None = None, stream=None):
    """Causal CSA prefill of the T new tokens after a P-token prefix (one sequence).
    kv / kv_scale [Nmax] are updated in place with the new entries. Returns out
    [T][H][512] bf16 and, when asked, lse [T][H] and the selected sets idx [T][k].
    strict_eligibility: a query at t sees only blocks completed before t (floor(t/m)
    entries) instead of also the block closing at t (floor((t+1)/m)).
    With paging (a one-row block table), kv, kv_scale, k_fp4 and k_sf are page pools."""
    T = a.shape[0]
    H, H_I = q.shape[1], q_fp4.shape[1]
    if paging is None:
        Nmax = pool = kv.shape[0]
    else:
        Nmax, pool = paging.Nmax, kv.numel() // ROW_BYTES
    tok = T * HEAD_DIM
    _sizes(a=(a, tok), b=(b, tok), za=(za, tok), zb=(zb, tok), bias=(bias, 2 * m),
           kv=(kv, pool * ROW_BYTES), kv_scale=(kv_scale, pool), q_fp4=(q_fp4, T * H_I * 64),
           q_sf=(q_sf, T * H_I * 4), w=(w, T * H_I), k_fp4=(k_fp4, pool * 64),
           k_sf=(k_sf, pool // 128 * 512), q=(q, T * H * HEAD_DIM), sink=(sink, H),
           prev_b=(prev_b, m * HEAD_DIM), prev_zb=(prev_zb, m * HEAD_DIM),
           swa_prefix=(swa_prefix, WINDOW * HEAD_DIM), norm_w=(norm_w, HEAD_DIM),
           out=(out, T * H * HEAD_DIM))
    pg = _pages(paging, pool, 1)
    dev = q.device
    if workspace is None:
        workspace = prefill_workspace(T, Nmax, H, k, dev)
    if out is None:
        out = torch.empty((T, H, HEAD_DIM), dtype=torch.bfloat16, device=dev)
    l = torch.empty((T, H), dtype=torch.float32, device=dev) if lse else None
    ix = torch.empty((T, k), dtype=torch.int32, device=dev) if idx else None
    args = PrefillArgs(P, T, m, H, H_I, k, Nmax, tau, rope_base, eps, int(derotate),
                       int(strict_eligibility),
                       _ptr(a, elem=2, name="a"), _ptr(b, elem=2, name="b"),
                       _ptr(za, elem=4, name="za"), _ptr(zb, elem=4, name="zb"),
                       _ptr(bias, elem=4, name="bias"), _ptr(norm_w, elem=4, name="norm_w"),
                       _ptr(prev_b, elem=2, name="prev_b"),
                       _ptr(prev_zb, elem=4, name="prev_zb"), _ptr(kv, elem=1, name="kv"),
                       _ptr(kv_scale, elem=4, name="kv_scale"),
                       _ptr(q_fp4, elem=1, name="q_fp4"), _ptr(q_sf, elem=1, name="q_sf"),
                       _ptr(w, elem=4, name="w"), _ptr(k_fp4, elem=1, name="k_fp4"),
                       _ptr(k_sf, elem=1, name="k_sf"), _ptr(q, elem=2, name="q"),
                       _ptr(sink, elem=4, name="sink"),
                       _ptr(swa_prefix, elem=2, name="swa_prefix"),
                       _ptr(out, elem=2, name="out"), _ptr(l, elem=4, name="lse"),
                       _ptr(ix, elem=4, name="idx"),
                       _ptr(dev_status, elem=4, name="dev_status"), pg)
    _check(lib().csa_prefill(C.byref(args), workspace.data_ptr(), workspace.numel(),
                             _stream(stream)), "csa_prefill")
    res = [out]
    if lse:
        res.append(l)
    if idx:
        res.append(ix)
    return res[0] if len(res) == 1 else tuple(res)
