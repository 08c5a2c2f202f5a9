"""Independent decoders and reductions used only to pin the oracle.

They go through library routines (torch's float8/bfloat16 casts, numpy/scipy
softmax, einsum, lexsort) or the literal OCP value tables, never through the oracle's
own code paths, so a mistake in the oracle does not cancel out here.
"""

import numpy as np
import torch

# OCP MX specification, E2M1 magnitudes for codes 0..7
E2M1_TABLE = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def bf16_to_f64(h):
    h = np.asarray(h, dtype=np.uint16)
    with np.errstate(invalid="ignore"):  # signalling-NaN codes widen to NaN, quietly
        return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def e4m3_to_f64(c):
    c = torch.from_numpy(np.ascontiguousarray(np.asarray(c, dtype=np.uint8)))
    return c.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def f64_to_e4m3(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def f64_to_bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).view(
        torch.int16).numpy().astype(np.uint16)


def e2m1_to_f64(nib):
    nib = np.asarray(nib, dtype=np.uint8)
    v = E2M1_TABLE[nib & 7]
    return np.where(nib & 8, -v, v)


def unpack_fp4(packed):
    """[..., 64] bytes -> [..., 128] codes, element 2i = low nibble of byte i."""
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


def e8m0_to_f64(e):
    return np.ldexp(1.0, np.asarray(e, dtype=np.int64) - 127)


def key_scales(k_sf_seq, nmax):
    """Grouped key-scale bytes of one sequence -> [nmax][4] E8M0 codes.
    Group g (512 bytes) holds entry 128g + r0 + 32*r1 at bytes 16*r0 + 4*r1 .. +3."""
    g = np.asarray(k_sf_seq, dtype=np.uint8).reshape(nmax // 128, 32, 4, 4)  # g, r0, r1, s
    return g.transpose(0, 2, 1, 3).reshape(nmax, 4)  # g, r1, r0, s -> entry order


def dequant_rows(kv_rows, scale):
    kv_rows = np.asarray(kv_rows, dtype=np.uint8).reshape(-1, 576)
    v = np.empty((kv_rows.shape[0], 512))
    v[:, :448] = e4m3_to_f64(kv_rows[:, :448]) * np.asarray(scale, np.float64).reshape(-1, 1)
    v[:, 448:] = bf16_to_f64(np.ascontiguousarray(kv_rows[:, 448:]).view(np.uint16))
    return v


def softmax(x, axis=-1):
    from scipy.special import softmax as sp_softmax
    return sp_softmax(x, axis=axis)


def gated_merge(inp, m, overlap, pos0=0):
    """The gated merge of a compression input bundle (streams a, b, logits za, zb, bias
    [2m]) by the library softmax over an explicit candidate axis: entry i takes the m own
    tokens of a with logits za + bias[:m] and, with overlap, the m previous-block tokens of
    b (or of prev_b for the first entry of a later chunk) with logits zb + bias[m:]."""
    a = bf16_to_f64(inp["a"])
    B, T, D = a.shape
    N = T // m
    bias = inp["bias"].astype(np.float64)
    e = np.empty((B, N, D))
    for b in range(B):
        for i in range(N):
            xs = [a[b, m * i:m * i + m]]
            zs = [inp["za"][b, m * i:m * i + m].astype(np.float64) + bias[:m, None]]
            if overlap and (i > 0 or pos0 > 0):
                if i > 0:
                    xb = bf16_to_f64(inp["b"][b, m * (i - 1):m * i])
                    zb = inp["zb"][b, m * (i - 1):m * i].astype(np.float64)
                else:
                    xb = bf16_to_f64(inp["prev_b"][b])
                    zb = inp["prev_zb"][b].astype(np.float64)
                xs.append(xb)
                zs.append(zb + bias[m:, None])
            x = np.concatenate(xs, 0)
            z = np.concatenate(zs, 0)
            e[b, i] = (softmax(z, axis=0) * x).sum(0)
    return e
