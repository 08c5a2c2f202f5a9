"""Seeded synthetic inputs for the CSA/HCA layer, shared by the tests, the benchmark
and the smoke check.

This module holds none of the layer's arithmetic. It draws raw bit patterns only:
bf16 values are the upper halves of float32 normal samples, FP8 E4M3 / FP4 E2M1 /
E8M0 values are drawn directly as codes from fixed categorical distributions, and
gate logits, biases, weights and sink logits are plain float32 samples. Everything a
later stage of the layer would compute (compressed entries, indexer scores, window
rows) is left to the oracle or to the CUDA library.

Workload shapes follow the five configurations of the benchmark table (the
DeepSeek-V4 Flash/Pro-shaped layers of the pages: head_dim 512, 64 or 128 query
heads, indexer 16/64 heads x 128 dims, top-k 512/1024, m = 4 or 128).
"""

from __future__ import annotations

import dataclasses

import numpy as np

D = 512
D_NOPE = 448
D_ROPE = 64
D_I = 128
W_SWA = 128
ROW_BYTES = 576


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str  # "csa", "hca" or "prefill"
    B: int
    m: int
    H: int
    H_I: int = 0
    k: int = 0
    L: int = 0  # context length (decode: query at position L-1)
    L_min: int = 0  # seeded per-sequence lengths in [L_min, L] when set
    P: int = 0  # prefill: cached prefix tokens
    T: int = 0  # prefill: new tokens
    planted_runs: int = 0  # runs of 16 high-affinity entries per sequence
    seed: int = 0


WORKLOADS = {
    0: Workload("csa_decode_8k_tiny", "csa", B=1, m=4, H=64, H_I=16, k=512, L=8192, seed=0),
    1: Workload("hca_decode_128k", "hca", B=8, m=128, H=64, L=131072, seed=1),
    2: Workload("csa_decode_flash_128k", "csa", B=32, m=4, H=64, H_I=64, k=512,
                L=131072, L_min=65536, seed=2),
    3: Workload("csa_decode_pro_1m", "csa", B=4, m=4, H=128, H_I=64, k=1024,
                L=1 << 20, planted_runs=164, seed=3),
    4: Workload("csa_prefill_pro_64k_on_192k", "prefill", B=1, m=4, H=128, H_I=64,
                k=1024, P=196608, T=65536, seed=4),
}


def round_up(x: int, q: int) -> int:
    return (x + q - 1) // q * q


# ------------------------------------------------------------------ raw codes
def bf16_normal(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    """bf16 bit patterns: the upper 16 bits of float32 N(0, std^2) samples."""
    x = (rng.standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


# E4M3 codes for a stored compressed entry: random sign, exponent field drawn around
# the top of the range (entries are scaled so the largest magnitude sits near 448),
# uniform mantissa; the NaN code S.1111.111 never occurs.
_E4M3_EXP_P = np.array([1, 1, 1, 1, 1, 2, 2, 3, 4, 6, 9, 13, 17, 19, 14, 6], dtype=np.float64)
_E4M3_EXP_P /= _E4M3_EXP_P.sum()


# Elementwise work on large draws runs over slices of this many elements, so that the
# temporaries stay cache-sized; the random draws themselves are taken whole, in a fixed
# order, so the values do not depend on the slicing.
_CHUNK = 1 << 22


def e4m3_codes(rng: np.random.Generator, shape) -> np.ndarray:
    n = int(np.prod(shape))
    e = _lut_sample(rng, n, _E4M3_EXP_P)
    low = rng.integers(0, 16, size=n, dtype=np.uint8)  # 3 mantissa bits + sign bit
    out = np.empty(n, dtype=np.uint8)
    for c in range(0, n, _CHUNK):
        ec, lc, oc = e[c:c + _CHUNK], low[c:c + _CHUNK], out[c:c + _CHUNK]
        mant = lc & 7
        mant[(ec == 15) & (mant == 7)] = 6
        np.left_shift(lc >> 3, 7, out=oc)
        oc |= ec << 3
        oc |= mant
    return out.reshape(shape)


# E2M1 magnitude codes 0..7 (values 0, .5, 1, 1.5, 2, 3, 4, 6) drawn with the
# frequencies a unit normal block of 32 shows after MXFP4 scaling.
_E2M1_MAG_P = np.array([0.10, 0.19, 0.17, 0.15, 0.17, 0.13, 0.07, 0.02])


def _lut_sample(rng: np.random.Generator, n: int, p: np.ndarray) -> np.ndarray:
    """Categorical samples through a 65536-entry lookup table of uniform u16 draws."""
    edges = np.cumsum(p) / p.sum()
    u = (np.arange(65536, dtype=np.float64) + 0.5) / 65536.0
    lut = np.searchsorted(edges, u, side="right").clip(0, len(p) - 1).astype(np.uint8)
    idx = rng.integers(0, 65536, size=n, dtype=np.uint16)
    out = np.empty(n, dtype=np.uint8)
    for c in range(0, n, _CHUNK):
        np.take(lut, idx[c:c + _CHUNK], out=out[c:c + _CHUNK])
    return out


def e2m1_nibbles(rng: np.random.Generator, shape, sign_bias: np.ndarray | None = None,
                 agree: float = 0.5, big: bool = False) -> np.ndarray:
    """One E2M1 code per element (0..15). With `sign_bias` (+-1 per element of the last
    axis) the sign matches it with probability `agree`; `big` draws magnitudes from the
    four largest codes (2, 3, 4, 6)."""
    n = int(np.prod(shape))
    if big:
        mag = (4 + rng.integers(0, 4, size=n, dtype=np.uint8)).astype(np.uint8)
    else:
        mag = _lut_sample(rng, n, _E2M1_MAG_P)
    if sign_bias is None:
        sign = rng.integers(0, 2, size=n, dtype=np.uint8)
    else:
        want_neg = np.broadcast_to(sign_bias < 0, shape).reshape(-1)
        keep = rng.random(n) < agree
        rand = rng.integers(0, 2, size=n, dtype=np.uint8).astype(bool)
        sign = np.where(keep, want_neg, rand).astype(np.uint8)
    return ((sign << 3) | mag).astype(np.uint8).reshape(shape)


def pack_nibbles(nib: np.ndarray) -> np.ndarray:
    """Element 2i in the low nibble of byte i, element 2i+1 in the high nibble."""
    return (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)


def e8m0_codes(rng: np.random.Generator, shape, lo: int = 124, hi: int = 130) -> np.ndarray:
    return rng.integers(lo, hi + 1, size=shape, dtype=np.uint8)


# ------------------------------------------------------------- input bundles
def compress_inputs(B: int, T: int, m: int, overlap: bool, seed: int,
                    pos0: int = 0, dim: int = D) -> dict:
    """Token streams for one compression call: a, b bf16 [B][T][dim], gate logits za, zb
    float32 [B][T][dim] ~ N(0,1), bias [2m] (CSA) or [m] (HCA) ~ N(0, 0.1), and when
    pos0 > 0 the previous block's tail prev_b / prev_zb [B][m][dim]. dim is 512 for the
    KV stream and 128 for the indexer-key stream."""
    rng = np.random.default_rng(seed)
    out = {
        "a": bf16_normal(rng, (B, T, dim)),
        "za": rng.standard_normal((B, T, dim), dtype=np.float32),
        "bias": (rng.standard_normal(2 * m if overlap else m) * 0.1).astype(np.float32),
    }
    if overlap:
        out["b"] = bf16_normal(rng, (B, T, dim))
        out["zb"] = rng.standard_normal((B, T, dim), dtype=np.float32)
        if pos0 > 0:
            out["prev_b"] = bf16_normal(rng, (B, m, dim))
            out["prev_zb"] = rng.standard_normal((B, m, dim), dtype=np.float32)
    return out


def seq_lengths(w: Workload) -> np.ndarray:
    if w.L_min:
        rng = np.random.default_rng(1000 + w.seed)
        return rng.integers(w.L_min, w.L + 1, size=w.B).astype(np.int64)
    return np.full(w.B, w.L, dtype=np.int64)


def kv_cache(rng: np.random.Generator, B: int, Nmax: int) -> tuple[np.ndarray, np.ndarray]:
    """A stored cache of compressed entries: rows of 448 E4M3 codes + 64 bf16, and a
    float32 per-entry scale in [0.004, 0.012) so dequantised values are O(1)."""
    kv = np.empty((B, Nmax, ROW_BYTES), dtype=np.uint8)
    kv[:, :, :D_NOPE] = e4m3_codes(rng, (B, Nmax, D_NOPE))
    kv[:, :, D_NOPE:] = bf16_normal(rng, (B, Nmax, D_ROPE)).view(np.uint8).reshape(
        B, Nmax, 2 * D_ROPE)
    scale = rng.uniform(0.004, 0.012, size=(B, Nmax)).astype(np.float32)
    return kv, scale


def indexer_inputs(rng: np.random.Generator, B: int, H_I: int, Nmax: int,
                   n_entries: np.ndarray, planted_runs: int = 0) -> dict:
    """FP4 indexer queries and keys. With planted_runs > 0, every sequence gets that many
    runs of 16 consecutive entries whose key signs follow a hidden direction u that the
    queries also lean towards, so the top-k set is drawn from a structured minority."""
    u = np.where(rng.random((B, 1, D_I)) < 0.5, -1.0, 1.0)
    if planted_runs:
        qn = e2m1_nibbles(rng, (B, H_I, D_I), sign_bias=u, agree=0.8)
    else:
        qn = e2m1_nibbles(rng, (B, H_I, D_I))
    kn = e2m1_nibbles(rng, (B, Nmax, D_I))
    planted = np.zeros((B, Nmax), dtype=bool)
    for b in range(B if planted_runs else 0):
        nruns = min(planted_runs, int(n_entries[b]) // 16)
        starts = rng.choice(int(n_entries[b]) // 16, size=nruns, replace=False) * 16
        for s in starts:
            kn[b, s:s + 16] = e2m1_nibbles(rng, (16, D_I), sign_bias=u[b, 0], agree=1.0,
                                           big=True)
            planted[b, s:s + 16] = True
    return {
        "q_fp4": pack_nibbles(qn),
        "q_sf": e8m0_codes(rng, (B, H_I, 4)),
        "w": rng.random((B, H_I), dtype=np.float32),
        "k_fp4": pack_nibbles(kn),
        "k_sf": e8m0_codes(rng, (B, Nmax // 128 * 512)),
        "planted": planted,
    }


def decode_inputs(w: Workload, seed: int | None = None, B: int | None = None) -> dict:
    """Everything one decode step reads: queries at position L_b - 1, the compressed
    cache (Nmax rows per sequence, n_b = floor(L_b / m) valid), the window ring
    swa[b][p % 128] (bf16 ~ N(0,1)), sink logits ~ N(0,1), and for CSA the FP4 indexer
    inputs. `B` overrides the batch (taking the first B sequence lengths)."""
    seed = w.seed if seed is None else seed
    rng = np.random.default_rng(seed)
    L = seq_lengths(w)
    if B is not None:
        L = np.resize(L, B)
    Bn = len(L)
    n = (L // w.m).astype(np.int32)
    Nmax = round_up(int(n.max()), 128)
    kv, scale = kv_cache(rng, Bn, Nmax)
    out = {
        "workload": w,
        "B": Bn,
        "Nmax": Nmax,
        "pos": (L - 1).astype(np.int32),
        "n_entries": n,
        "q": bf16_normal(rng, (Bn, w.H, D)),
        "kv": kv,
        "kv_scale": scale,
        "swa": bf16_normal(rng, (Bn, W_SWA, D)),
        "sink": rng.standard_normal(w.H, dtype=np.float32),
    }
    if w.kind == "csa":
        out.update(indexer_inputs(rng, Bn, w.H_I, Nmax, n, w.planted_runs))
    return out


def prefill_inputs(P: int, T: int, m: int, H: int, H_I: int, seed: int) -> dict:
    """One sequence: a P-token cached prefix (P/m stored entries, indexer keys for every
    entry up to (P+T)/m, the window ring of the prefix and the previous block's tail)
    and T new tokens (a, b, za, zb, Q, FP4 indexer queries and weights)."""
    rng = np.random.default_rng(seed)
    Nmax = round_up(max((P + T) // m, 1), 128)
    kv, scale = kv_cache(rng, 1, Nmax)
    n_all = np.array([(P + T) // m], dtype=np.int32)
    ix = indexer_inputs(rng, 1, H_I, Nmax, n_all)
    tok = compress_inputs(1, T, m, True, seed + 7919, pos0=P)
    q_nib = e2m1_nibbles(rng, (T, H_I, D_I))
    out = {
        "P": P, "T": T, "m": m, "H": H, "H_I": H_I, "Nmax": Nmax,
        "kv": kv[0], "kv_scale": scale[0],
        "k_fp4": ix["k_fp4"][0], "k_sf": ix["k_sf"][0],
        "q_fp4": pack_nibbles(q_nib),
        "q_sf": e8m0_codes(rng, (T, H_I, 4)),
        "w": rng.random((T, H_I), dtype=np.float32),
        "q": bf16_normal(rng, (T, H, D)),
        "sink": rng.standard_normal(H, dtype=np.float32),
        "swa_prefix": bf16_normal(rng, (W_SWA, D)),
        "a": tok["a"][0], "b": tok["b"][0], "za": tok["za"][0], "zb": tok["zb"][0],
        "bias": tok["bias"],
    }
    if P > 0:
        out["prev_b"] = tok["prev_b"][0]
        out["prev_zb"] = tok["prev_zb"][0]
    return out


# ------------------------------------------------------- device-side generation
def prefill_inputs_device(P: int, T: int, m: int, H: int, H_I: int, seed: int,
                          device="cuda") -> dict:
    """The bundle of prefill_inputs drawn on the GPU with torch's seeded generator, for
    sizes where host generation would take minutes (the 64K-token prefill holds 4.3 G query
    values). Same distributions as the host generators (bf16 by truncating float32 N(0,1),
    E2M1 magnitudes and E4M3 exponents through the same 65536-entry lookup tables, E8M0
    in 124..130, w ~ U(0,1)); a different random stream, so values differ from
    prefill_inputs with the same seed. The stored prefix cache and the indexer keys come
    from the host generators (they are small). Returns torch tensors on `device`."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    rng = np.random.default_rng(seed)
    Nmax = round_up(max((P + T) // m, 1), 128)
    CH = 1 << 26  # elements per generation chunk (bounds the temporaries)

    def chunked(n, fn, dtype):
        out = torch.empty(n, dtype=dtype, device=device)
        for s in range(0, n, CH):
            e = min(n, s + CH)
            out[s:e] = fn(e - s)
        return out

    def bf16n(shape):
        n = int(np.prod(shape))
        f = lambda c: (torch.randn(c, generator=g, device=device).view(torch.int32) >> 16) \
            .to(torch.int16)
        return chunked(n, f, torch.int16).view(shape)

    def lut_of(p):
        edges = np.cumsum(p) / p.sum()
        u = (np.arange(65536, dtype=np.float64) + 0.5) / 65536.0
        lut = np.searchsorted(edges, u, side="right").clip(0, len(p) - 1).astype(np.uint8)
        return torch.from_numpy(lut).to(device)

    mag_lut = lut_of(_E2M1_MAG_P)

    def fp4_packed(shape):  # shape ends with the element count; returns packed bytes
        n = int(np.prod(shape)) // 2

        def f(c):
            lo = mag_lut[torch.randint(0, 65536, (c,), generator=g, device=device)] | \
                (torch.randint(0, 2, (c,), generator=g, device=device, dtype=torch.uint8) << 3)
            hi = mag_lut[torch.randint(0, 65536, (c,), generator=g, device=device)] | \
                (torch.randint(0, 2, (c,), generator=g, device=device, dtype=torch.uint8) << 3)
            return lo | (hi << 4)
        return chunked(n, f, torch.uint8).view(*shape[:-1], shape[-1] // 2)

    kv, scale = kv_cache(rng, 1, Nmax)
    n_all = np.array([(P + T) // m], dtype=np.int32)
    ix = indexer_inputs(rng, 1, H_I, Nmax, n_all)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(
        x.view(np.int16) if x.dtype == np.uint16 else x)).to(device)
    out = {
        "P": P, "T": T, "m": m, "H": H, "H_I": H_I, "Nmax": Nmax,
        "kv": t(kv[0]), "kv_scale": t(scale[0]),
        "k_fp4": t(ix["k_fp4"][0]), "k_sf": t(ix["k_sf"][0]),
        "q_fp4": fp4_packed((T, H_I, D_I)),
        "q_sf": torch.randint(124, 131, (T, H_I, 4), generator=g, device=device,
                              dtype=torch.uint8),
        "w": torch.rand((T, H_I), generator=g, device=device),
        "q": bf16n((T, H, D)),
        "sink": torch.randn(H, generator=g, device=device),
        "swa_prefix": bf16n((W_SWA, D)),
        "a": bf16n((T, D)), "b": bf16n((T, D)),
        "za": torch.randn((T, D), generator=g, device=device),
        "zb": torch.randn((T, D), generator=g, device=device),
        "bias": torch.randn(2 * m, generator=g, device=device) * 0.1,
    }
    # the indexer-key stream of the new tokens (128 dims), for the key compressor
    out["ia"], out["ib"] = bf16n((T, D_I)), bf16n((T, D_I))
    out["iza"] = torch.randn((T, D_I), generator=g, device=device)
    out["izb"] = torch.randn((T, D_I), generator=g, device=device)
    out["ibias"] = torch.randn(2 * m, generator=g, device=device) * 0.1
    if P > 0:
        out["prev_b"] = bf16n((m, D))
        out["prev_zb"] = torch.randn((m, D), generator=g, device=device)
        out["iprev_b"] = bf16n((m, D_I))
        out["iprev_zb"] = torch.randn((m, D_I), generator=g, device=device)
    return out


def page_table(rng: np.random.Generator, B: int, pages_max: int, spare: int = 3
               ) -> tuple[np.ndarray, int]:
    """A shuffled block table int32 [B][pages_max] over a pool of B * pages_max + spare
    pages (the spare pages are never named): (table, num_pages)."""
    num_pages = B * pages_max + spare
    table = rng.permutation(num_pages)[:B * pages_max].reshape(B, pages_max)
    return table.astype(np.int32), num_pages


def place_in_pages(per_seq: np.ndarray, table: np.ndarray, page_entries: int,
                   num_pages: int, group: int = 1, fill: int = 0x5A) -> np.ndarray:
    """Lay per-sequence rows [B][units][...] (a unit = `group` entries) out in a page pool
    [num_pages][page_entries // group][...]: logical page lp of sequence b goes to pool
    page table[b][lp]. Pool bytes no sequence owns hold `fill` (never read when the
    table is honoured)."""
    per_page = page_entries // group
    B, units = per_seq.shape[:2]
    flat = np.ascontiguousarray(per_seq)
    pool = np.empty((num_pages, per_page) + flat.shape[2:], dtype=flat.dtype)
    pool.view(np.uint8)[...] = fill
    for b in range(B):
        for lp in range(table.shape[1]):
            lo, hi = lp * per_page, min((lp + 1) * per_page, units)
            if lo < hi:
                pool[table[b, lp], :hi - lo] = flat[b, lo:hi]
    return pool
