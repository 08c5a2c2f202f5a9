"""csa_sparse_attn_decode_noalloc (static per-device scratch) against the workspace entry point.

Named to be collected last, so that it runs after every other test has used the library on
the same device, and it also passes on its own.
"""

import ctypes as C

import numpy as np
import pytest
import torch

from synth import inputs as synth
from tests import compare

csa = pytest.importorskip("long_context_compressed_layer_b200")

FAKE = 1 << 20  # a 256-aligned non-null address: never dereferenced on a rejected call


def _args(B, H, k, Nmax=4096):
    return csa.AttnArgs(B, H, k, Nmax, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.0,
                        10000.0, 1, FAKE, None, None)


def test_noalloc_rejects_oversized_problems_on_the_host():
    L = csa.lib()
    assert csa.NOALLOC_SCRATCH_BYTES == 12 << 20
    # 64 sequences x 128 heads x (2048 + 128) rows needs far more than the static scratch
    big = _args(64, 128, 2048)
    assert L.csa_attn_workspace_size(64, 128, 2048 + 128) > csa.NOALLOC_SCRATCH_BYTES
    assert L.csa_sparse_attn_decode_noalloc(C.byref(big), None) == csa.CSA_ERR_UNSUPPORTED
    # the ordinary argument checks still apply
    assert L.csa_sparse_attn_decode_noalloc(None, None) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_sparse_attn_decode_noalloc(C.byref(_args(1, 96, 64)), None) == \
        csa.CSA_ERR_UNSUPPORTED
    assert L.csa_sparse_attn_decode_noalloc(C.byref(_args(1, 64, 0)), None) == \
        csa.CSA_ERR_INVALID_ARG
    assert L.csa_sparse_attn_decode_noalloc(C.byref(_args(0, 64, 64)), None) == csa.CSA_OK
    # the largest decode it is meant for fits: 4 x 128 heads x (1024 + 128) rows
    assert L.csa_attn_workspace_size(4, 128, 1024 + 128) <= csa.NOALLOC_SCRATCH_BYTES


def _case(B, H, Nmax, n, pos, k, seed):
    rng = np.random.default_rng(seed)
    kv, sc = synth.kv_cache(rng, B, Nmax)
    q = synth.bf16_normal(rng, (B, H, 512))
    swa = synth.bf16_normal(rng, (B, 128, 512))
    sink = rng.standard_normal(H).astype(np.float32)
    idx = np.full((B, k), -1, np.int32)
    for b in range(B):
        c = min(k - 3, int(n[b]))
        idx[b, :c] = np.sort(rng.choice(int(n[b]), c, replace=False))

    def dev(x):
        x = np.ascontiguousarray(x)
        return torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x).cuda()

    return [dev(q), dev(np.asarray(pos, np.int32)), dev(np.asarray(n, np.int32)), dev(kv),
            dev(sc), dev(swa), dev(sink), dev(idx)]


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    cases = [_case(4, 128, 4096, [4096, 3000, 1500, 1100], [16383, 12001, 6000, 4411], 1024,
                   seed=41),
             _case(2, 64, 2048, [2048, 700], [8191, 2803], 512, seed=42)]
    got = []
    for args in cases:  # two no-alloc calls back to back on one stream, one sync at the end
        got.append(csa.sparse_attn_decode_noalloc(*args, lse=True))
    torch.cuda.synchronize()
    for args, (out, lse) in zip(cases, got):
        want, wlse = csa.sparse_attn_decode(*args, lse=True)
        torch.cuda.synchronize()
        compare.close(out.float().cpu().numpy(), want.float().cpu().numpy(),
                      what="no-alloc vs workspace")
        np.testing.assert_allclose(lse.cpu().numpy(), wlse.cpu().numpy(), rtol=1e-5, atol=1e-5)
