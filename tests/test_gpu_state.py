"""Decode-step state updates (csa_decode_append) against the oracle's whole-stream
compression (and the library's own whole-stream calls)."""

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


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    csa.lib()


@pytest.mark.parametrize("weighted", [False, True])
def test_token_by_token_appends_equal_whole_stream_compression(weighted):
    B, S, m = 2, 4 * 37 + 2, 4  # 37 closed blocks, two tokens left in the tail
    kvs = synth.compress_inputs(B, S, m, True, seed=61)
    iks = synth.compress_inputs(B, S, m, True, seed=62, dim=128)
    # the optional RMSNorm weight of the entries and window rows
    w = np.random.default_rng(61).uniform(0.5, 2.0, 512).astype(np.float32) if weighted else None
    w_dev = dev(w) if weighted else None
    Nmax = 128
    st = csa.new_decode_state(B, Nmax, m)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    d = {k: dev(v) for k, v in kvs.items()}
    di = {k: dev(v) for k, v in iks.items()}
    for t in range(S):
        pos = torch.full((B,), t, dtype=torch.int32, device="cuda")
        csa.decode_append(pos, d["a"][:, t].contiguous(), d["za"][:, t].contiguous(), d["bias"],
                          st, b=d["b"][:, t].contiguous(), zb=d["zb"][:, t].contiguous(), m=m,
                          ia=di["a"][:, t].contiguous(), ib=di["b"][:, t].contiguous(),
                          iza=di["za"][:, t].contiguous(), izb=di["zb"][:, t].contiguous(),
                          ibias=di["bias"], norm_w=w_dev, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert (st["n_entries"].cpu().numpy() == S // m).all()
    # the entries and keys against the oracle's whole-stream compression of the same tokens
    n = S // m
    ora = oracle.compress(kvs["a"], kvs["za"], kvs["bias"], m, True, b=kvs["b"], zb=kvs["zb"],
                          norm_w=w)
    kv_h, sc_h = st["kv"].cpu().numpy(), st["kv_scale"].cpu().numpy()
    np.testing.assert_allclose(sc_h[:, :n], ora["kv_scale"], rtol=1e-5)
    flips = compare.check_codes(kv_h[:, :n], ora["kv"], ora["y"], ora["kv_scale"],
                                what="appended entries")
    assert flips <= max(4, ora["kv"].size // 5000)
    okf, oks, oy = oracle.compress_index_keys(iks["a"], iks["za"], iks["bias"], m, True, Nmax,
                                              b=iks["b"], zb=iks["zb"])
    kf_h, ks_h = st["k_fp4"].cpu().numpy(), st["k_sf"].cpu().numpy()
    rows = np.arange(n)
    kflips = 0
    for bb in range(B):
        sf_g = np.array([[ks_h[bb, oracle.key_sf_offset(r, s)] for s in range(4)] for r in rows])
        sf_o = np.array([[oks[bb, oracle.key_sf_offset(r, s)] for s in range(4)] for r in rows])
        kflips += compare.check_mxfp4(
            compare.unpack_nibbles(kf_h[bb, rows]).reshape(-1, 32),
            compare.unpack_nibbles(okf[bb, rows]).reshape(-1, 32), sf_g.reshape(-1),
            sf_o.reshape(-1), oy[bb].reshape(-1, 32), what=f"appended keys seq {bb}")
    assert kflips <= max(2, n * B // 500)
    # and bit for bit the same as the library's whole-stream calls (one block arithmetic)
    kv, sc, _ = csa.compress(d["a"], d["za"], d["bias"], m, True, b=d["b"], zb=d["zb"],
                             Nmax=Nmax, norm_w=w_dev)
    kf, ks, _ = csa.compress_index_keys(di["a"], di["za"], di["bias"], m, True, b=di["b"],
                                        zb=di["zb"], Nmax=Nmax)
    torch.cuda.synchronize()
    assert torch.equal(st["kv"][:, :n], kv[:, :n]) and torch.equal(st["kv_scale"][:, :n],
                                                                   sc[:, :n])
    assert torch.equal(st["k_fp4"][:, :n], kf[:, :n]) and torch.equal(st["k_sf"], ks)
    # the window ring holds the last 128 tokens' window rows
    ring = st["swa"].cpu().numpy().view(np.uint16)
    for bb in range(B):
        for p in (S - 128, S - 57, S - 1):
            want = oracle.swa_row(kvs["a"][bb, p], p, norm_w=w)
            got = ring[bb, p % 128]
            wf = want.astype(np.uint32) << 16
            gf = got.astype(np.uint32) << 16
            np.testing.assert_allclose(gf.view(np.float32), wf.view(np.float32), rtol=2.0 ** -7,
                                       atol=1e-6)
