"""CUDA path vs the fp64 oracle, element by element, on seeded inputs (needs a B200)."""

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
    if x.dtype == np.uint16:
        x = x.view(np.int16)
    return torch.from_numpy(x).cuda()


def host(t):
    return t.cpu().numpy()


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    csa.lib()
    torch.cuda.init()


# ------------------------------------------------------------------ compress
def _run_compress(inp, m, overlap, pos0=0, Nmax=None, norm_w=None):
    B, T, _ = inp["a"].shape
    N = T // m
    Nmax = Nmax or pos0 // m + N
    kv, sc, dbg = csa.compress(dev(inp["a"]), dev(inp["za"]), dev(inp["bias"]), m, overlap,
                               b=dev(inp["b"]) if overlap else None,
                               zb=dev(inp["zb"]) if overlap else None, pos0=pos0,
                               prev_b=dev(inp["prev_b"]) if "prev_b" in inp else None,
                               prev_zb=dev(inp["prev_zb"]) if "prev_zb" in inp else None,
                               Nmax=Nmax, dbg=True,
                               norm_w=dev(norm_w) if norm_w is not None else None)
    torch.cuda.synchronize()
    n0 = pos0 // m
    return host(kv)[:, n0:n0 + N], host(sc)[:, n0:n0 + N], host(dbg)


@pytest.mark.parametrize("B,T,m,overlap,pos0", [
    (2, 4 * 37 + 3, 4, True, 0),      # CSA, ragged tail (3 tokens stay in state)
    (1, 4 * 64, 4, True, 4096),       # CSA chunk after a prefix: previous block from state
    (3, 128 * 3, 128, False, 0),      # HCA
    (1, 128 * 2, 128, False, 1 << 20),  # HCA at 1M positions (RoPE angle range)
    (1, 24, 1, True, 0),              # m = 1
])
def test_compress_matches_oracle(B, T, m, overlap, pos0):
    inp = synth.compress_inputs(B, T, m, overlap, seed=100 + m + B, pos0=pos0)
    kv, sc, dbg = _run_compress(inp, m, overlap, pos0, Nmax=pos0 // m + T // m + 5)
    ora = oracle.compress(inp["a"], inp["za"], inp["bias"], m, overlap, b=inp.get("b"),
                          zb=inp.get("zb"), pos0=pos0, prev_b=inp.get("prev_b"),
                          prev_zb=inp.get("prev_zb"))
    flips = compare.compare_entries(kv, sc, dbg, ora, what=f"compress m={m}")
    assert flips <= max(4, kv.size // 5000)


def test_compress_with_rmsnorm_weight():
    # the optional RMSNorm weight (dims scaled after the norm, before RoPE)
    inp = synth.compress_inputs(2, 4 * 40, 4, True, seed=131, pos0=256)
    w = np.random.default_rng(131).uniform(0.5, 2.0, 512).astype(np.float32)
    kv, sc, dbg = _run_compress(inp, 4, True, 256, norm_w=w)
    ora = oracle.compress(inp["a"], inp["za"], inp["bias"], 4, True, b=inp["b"], zb=inp["zb"],
                          pos0=256, prev_b=inp["prev_b"], prev_zb=inp["prev_zb"], norm_w=w)
    flips = compare.compare_entries(kv, sc, dbg, ora, what="compress with norm weight")
    assert flips <= max(4, kv.size // 5000)


def test_compress_workload0_full():
    # the 8192-token CSA stream of the tiny decode workload -> 2048 entries
    inp = synth.compress_inputs(1, 8192, 4, True, seed=0)
    kv, sc, dbg = _run_compress(inp, 4, True)
    ora = oracle.compress(inp["a"], inp["za"], inp["bias"], 4, True, b=inp["b"], zb=inp["zb"])
    flips = compare.compare_entries(kv, sc, dbg, ora, what="workload 0 compress")
    assert flips <= kv.size // 5000


# ------------------------------------------------------- indexer-key compression
@pytest.mark.parametrize("B,T,m,pos0", [
    (2, 4 * 37 + 3, 4, 0),      # ragged tail, first entry without a previous block
    (1, 4 * 64, 4, 4096),       # previous block from the caller's tail
    (1, 8192, 4, 0),            # the 8K stream of the tiny decode workload -> 2048 keys
])
def test_index_key_compression_matches_oracle(B, T, m, pos0):
    inp = synth.compress_inputs(B, T, m, True, seed=300 + T, pos0=pos0, dim=128)
    N = T // m
    Nmax = -(-(pos0 // m + N) // 128) * 128
    kf, ks, dbg = csa.compress_index_keys(
        dev(inp["a"]), dev(inp["za"]), dev(inp["bias"]), m, True, b=dev(inp["b"]),
        zb=dev(inp["zb"]), pos0=pos0, prev_b=dev(inp["prev_b"]) if pos0 else None,
        prev_zb=dev(inp["prev_zb"]) if pos0 else None, Nmax=Nmax, dbg=True)
    torch.cuda.synchronize()
    kf, ks, dbg = host(kf), host(ks), host(dbg)
    okf, oks, oy = oracle.compress_index_keys(
        inp["a"], inp["za"], inp["bias"], m, True, Nmax, b=inp["b"], zb=inp["zb"], pos0=pos0,
        prev_b=inp.get("prev_b"), prev_zb=inp.get("prev_zb"))
    np.testing.assert_allclose(dbg, oy, rtol=1e-5, atol=1e-5)
    n0 = pos0 // m
    rows = np.arange(n0, n0 + N)
    flips = 0
    for bb in range(B):
        sf_g = np.array([[ks[bb, oracle.key_sf_offset(r, s)] for s in range(4)] for r in rows])
        sf_o = np.array([[oks[bb, oracle.key_sf_offset(r, s)] for s in range(4)] for r in rows])
        flips += compare.check_mxfp4(
            compare.unpack_nibbles(kf[bb, rows]).reshape(-1, 32),
            compare.unpack_nibbles(okf[bb, rows]).reshape(-1, 32), sf_g.reshape(-1),
            sf_o.reshape(-1), oy[bb].reshape(-1, 32), what=f"index keys seq {bb}")
    assert flips <= max(2, N * B // 500)


@pytest.mark.parametrize("T,r,H_I", [
    (300, 256, 16),    # three token tiles, the last one ragged
    (4, 1536, 64),     # one decode step of the 1M workload, latent rank 1536
    (129, 64, 32),     # a single K block
])
def test_indexer_query_matches_oracle(T, r, H_I):
    rng = np.random.default_rng(T + r)
    c = synth.bf16_normal(rng, (T, r))
    W = synth.bf16_normal(rng, (H_I * 128, r), std=r ** -0.5)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qf, qs, dbg = csa.indexer_query(dev(c), dev(W), H_I, dbg=True, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    qf, qs, dbg = host(qf), host(qs), host(dbg)
    of, os_, y = oracle.indexer_query(c, W, H_I)
    np.testing.assert_allclose(dbg, y, rtol=1e-4, atol=1e-4)
    flips = compare.check_mxfp4(compare.unpack_nibbles(qf).reshape(-1, 32),
                                compare.unpack_nibbles(of).reshape(-1, 32), qs.reshape(-1),
                                os_.reshape(-1), y.reshape(-1, 32), mid_rel=1e-4,
                                sf_rel=1e-5, what="indexer queries")
    assert flips <= max(4, T * H_I * 128 // 2000)


# -------------------------------------------------------- grouped output projection
@pytest.mark.parametrize("T,H,G,d_g,d_model", [
    (200, 64, 16, 128, 256),     # two token tiles, the second ragged
    (4, 128, 16, 1024, 1024),    # one decode step of the 1M workload's heads
    (130, 128, 8, 256, 384),
])
def test_grouped_out_proj_matches_oracle(T, H, G, d_g, d_model):
    rng = np.random.default_rng(T + H + G)
    attn = synth.bf16_normal(rng, (T, H, 512))
    K1 = H // G * 512
    Wg = synth.bf16_normal(rng, (G, d_g, K1), std=0.5 * K1 ** -0.5)
    Wo = synth.bf16_normal(rng, (d_model, G * d_g), std=0.5 * (G * d_g) ** -0.5)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = csa.grouped_out_proj(dev(attn), dev(Wg), dev(Wo), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    want, _ = oracle.grouped_out_proj(attn, Wg, Wo)
    compare.close(out.float().cpu().numpy(), want, what="grouped output projection")


# ------------------------------------------------------------- indexer top-k
def _topk_case(B, H_I, Nmax, n, k, planted=0, seed=0, separate=False):
    rng = np.random.default_rng(seed)
    n = np.asarray(n, dtype=np.int32)
    ix = synth.indexer_inputs(rng, B, H_I, Nmax, n, planted)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, sc = csa.indexer_topk(dev(n), dev(ix["q_fp4"]), dev(ix["q_sf"]), dev(ix["w"]),
                               dev(ix["k_fp4"]), dev(ix["k_sf"]), k, scores=True,
                               separate_select=separate, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ora = oracle.indexer_scores(n, ix["q_fp4"], ix["q_sf"], ix["w"], ix["k_fp4"], ix["k_sf"])
    return host(idx), host(sc), ora, n


@pytest.mark.parametrize("B,H_I,Nmax,n,k,planted", [
    (1, 16, 2048, [2048], 512, 0),              # workload 0 shape
    (3, 64, 4096, [4096, 2999, 130], 512, 0),   # ragged lengths, n < k in one sequence
    (2, 32, 1024, [1000, 0], 64, 2),            # an empty sequence
    (2, 64, 16384, [16384, 12345], 1024, 8),    # planted runs, several CTAs per sequence
    (1, 64, 256, [1], 1, 0),                    # one entry: most CTAs own no tile
    # many short sequences: CTAs spanning several sequences, some empty, some n <= k
    (200, 32, 3072, list(np.random.default_rng(5).integers(0, 3072, 200)), 1000, 0),
])
@pytest.mark.parametrize("separate", [False, True])
def test_indexer_topk_matches_oracle(B, H_I, Nmax, n, k, planted, separate):
    # separate: the selection as stand-alone kernels, the path the library takes when the
    # runtime refuses the cooperative launch
    idx, sc, ora, n = _topk_case(B, H_I, Nmax, n, k, planted, seed=B * 7 + k,
                                 separate=separate)
    total = 0
    for b in range(B):
        total += compare.compare_topk(idx[b], ora[b], int(n[b]), k, what=f"seq {b}")
        sel = idx[b][idx[b] >= 0]
        np.testing.assert_allclose(sc[b][: len(sel)], ora[b][sel], rtol=2e-5, atol=1e-6)
    assert total <= 2


@pytest.mark.parametrize("B,H_I,Nmax,n,k,planted", [
    (1, 16, 2048, [2048], 512, 0),
    (3, 64, 4096, [4096, 2999, 130], 512, 0),
    (2, 64, 16384, [16384, 12345], 1024, 8),
])
def test_indexer_topk_bf16_scores_match_oracle(B, H_I, Nmax, n, k, planted):
    rng = np.random.default_rng(B * 11 + k)
    n = np.asarray(n, dtype=np.int32)
    ix = synth.indexer_inputs(rng, B, H_I, Nmax, n, planted)
    idx, sc = csa.indexer_topk(dev(n), dev(ix["q_fp4"]), dev(ix["q_sf"]), dev(ix["w"]),
                               dev(ix["k_fp4"]), dev(ix["k_sf"]), k, scores=True,
                               bf16_scores=True)
    torch.cuda.synchronize()
    idx, sc = host(idx), host(sc)
    ora = oracle.indexer_scores(n, ix["q_fp4"], ix["q_sf"], ix["w"], ix["k_fp4"], ix["k_sf"])
    total = 0
    for b in range(B):
        total += compare.compare_topk_bf16(idx[b], ora[b], int(n[b]), k, what=f"seq {b}")
        sel = idx[b][idx[b] >= 0]
        want = compare._bf16_round(ora[b][sel])
        # each returned score is a BF16 value within one BF16 step of the oracle's
        assert (compare._bf16_round(sc[b][: len(sel)]) == sc[b][: len(sel)]).all()
        np.testing.assert_allclose(sc[b][: len(sel)], want, rtol=2.0 ** -7, atol=1e-6)
    assert total <= 2 * B


@pytest.mark.parametrize("B,H_I,Nmax,n,k,planted", [
    (1, 16, 2048, [2048], 512, 0),
    (3, 64, 4096, [4096, 2999, 130], 512, 0),
    (2, 64, 16384, [16384, 12345], 1024, 8),
    (4, 64, 65536, [65536, 60000, 30000, 900], 1024, 16),
])
def test_indexer_bf16_fused_selection_equals_separate_kernels(B, H_I, Nmax, n, k, planted):
    # the cooperative launch's BF16 path (counts by the 5 key bits below the bin, ties
    # split by index across CTAs) and the stand-alone selection kernels select on the same
    # scores: the same indices
    rng = np.random.default_rng(B * 13 + k)
    n = np.asarray(n, dtype=np.int32)
    ix = synth.indexer_inputs(rng, B, H_I, Nmax, n, planted)
    args = (dev(n), dev(ix["q_fp4"]), dev(ix["q_sf"]), dev(ix["w"]), dev(ix["k_fp4"]),
            dev(ix["k_sf"]), k)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fused = host(csa.indexer_topk(*args, bf16_scores=True, dev_status=st))
    sep = host(csa.indexer_topk(*args, bf16_scores=True, separate_select=True, dev_status=st))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(fused, sep)


@pytest.mark.parametrize("separate", [False, True])
def test_indexer_bf16_heavy_ties_exact(separate):
    # unit scales and w = 1: scores are multiples of 1/4, exact in fp32 and, at these sizes,
    # spread over few BF16 values, so thousands of entries tie at the cut; the selection
    # must take the smallest indices among them, exactly as the oracle's BF16 selection
    B, H_I, Nmax, k = 2, 16, 32768, 1024
    rng = np.random.default_rng(17)
    n = np.array([32768, 20000], np.int32)
    ix = synth.indexer_inputs(rng, B, H_I, Nmax, n)
    ix["q_sf"][:] = 127
    ix["k_sf"][:] = 127
    ix["w"][:] = 1.0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx = host(csa.indexer_topk(dev(n), dev(ix["q_fp4"]), dev(ix["q_sf"]), dev(ix["w"]),
                                dev(ix["k_fp4"]), dev(ix["k_sf"]), k, bf16_scores=True,
                                separate_select=separate, dev_status=st))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ora = oracle.indexer_scores(n, ix["q_fp4"], ix["q_sf"], ix["w"], ix["k_fp4"], ix["k_sf"])
    for b in range(B):
        r = compare._bf16_round(ora[b][: n[b]])
        assert (r == np.sort(r)[::-1][k - 1]).sum() > 50  # the case really has heavy ties
        np.testing.assert_array_equal(idx[b], oracle.topk_bf16(ora[b][: n[b]], int(n[b]), k))


def test_indexer_scores_exact_on_integer_case():
    # unit scales, w = 1: every score is a multiple of 1/4 below 2^24, exact in fp32
    B, H_I, Nmax, k = 1, 64, 1024, 1024
    rng = np.random.default_rng(3)
    n = np.array([1000], np.int32)
    ix = synth.indexer_inputs(rng, B, H_I, Nmax, n)
    ix["q_sf"][:] = 127
    ix["k_sf"][:] = 127
    ix["w"][:] = 1.0
    idx, sc = csa.indexer_topk(dev(n), dev(ix["q_fp4"]), dev(ix["q_sf"]), dev(ix["w"]),
                               dev(ix["k_fp4"]), dev(ix["k_sf"]), k, scores=True)
    ora = oracle.indexer_scores(n, ix["q_fp4"], ix["q_sf"], ix["w"], ix["k_fp4"], ix["k_sf"])
    idx, sc = host(idx)[0], host(sc)[0]
    assert (idx[:1000] == np.arange(1000)).all() and (idx[1000:] == -1).all()
    np.testing.assert_array_equal(sc[:1000], ora[0, :1000])


@pytest.mark.parametrize("separate", [False, True])
@pytest.mark.parametrize("k", [1, 100, 777, 2048])
def test_indexer_exact_ties_keep_smaller_indices(k, separate):
    # unit scales, w = 1, every query element 1.0 and key elements 0 or 1: each score is
    # 16 x (an integer dot <= 128), so the cut falls inside a group of exactly equal scores
    # and must keep the smaller indices (no tolerance here)
    B, H_I, Nmax = 1, 16, 5120
    rng = np.random.default_rng(k)
    n = np.array([5000], np.int32)
    ix = synth.indexer_inputs(rng, B, H_I, Nmax, n)
    ix["q_sf"][:] = 127
    ix["k_sf"][:] = 127
    ix["w"][:] = 1.0
    ix["q_fp4"][:] = 0x22
    ix["k_fp4"][:] = rng.choice(np.array([0x00, 0x02, 0x20, 0x22], np.uint8), size=ix["k_fp4"].shape)
    ora = oracle.indexer_scores(n, ix["q_fp4"], ix["q_sf"], ix["w"], ix["k_fp4"], ix["k_sf"])
    s = ora[0, :5000]
    assert len(np.unique(s)) <= 129  # the case really is tie-heavy
    want = oracle.topk(ora[0], 5000, k)
    idx = csa.indexer_topk(dev(n), dev(ix["q_fp4"]), dev(ix["q_sf"]), dev(ix["w"]),
                           dev(ix["k_fp4"]), dev(ix["k_sf"]), k, separate_select=separate)
    np.testing.assert_array_equal(host(idx)[0], want)


def test_indexer_selection_wait_that_runs_out_reports_a_timeout():
    # a 1 ns limit on the grid-barrier waits of the fused selection: every CTA that is not
    # the last to arrive gives up at once. The waits bounded here start after scoring has
    # drained its copies and MMAs. The call must return with CSA_ERR_TIMEOUT; after the
    # workspace is zero-filled again (as the interface asks after any error) the next
    # normal call on it matches the oracle.
    B, H_I, Nmax, k = 4, 64, 32768, 1024
    rng = np.random.default_rng(31)
    n = np.array([32768, 30000, 20000, 1000], np.int32)
    ix = synth.indexer_inputs(rng, B, H_I, Nmax, n, 4)
    args = [dev(n), dev(ix["q_fp4"]), dev(ix["q_sf"]), dev(ix["w"]), dev(ix["k_fp4"]),
            dev(ix["k_sf"]), k]
    ws = csa.indexer_topk_workspace(B, Nmax, k)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    csa.indexer_topk(*args, workspace=ws, dev_status=st, select_wait_ns=1)
    torch.cuda.synchronize()
    assert int(st.item()) == csa.CSA_ERR_TIMEOUT
    ws.zero_()
    st.zero_()
    idx = csa.indexer_topk(*args, workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ora = oracle.indexer_scores(n, ix["q_fp4"], ix["q_sf"], ix["w"], ix["k_fp4"], ix["k_sf"])
    idx = host(idx)
    flips = sum(compare.compare_topk(idx[b], ora[b], int(n[b]), k, what=f"seq {b}")
                for b in range(B))
    assert flips <= 2


def test_indexer_workspace_stays_clean_across_calls():
    B, H_I, Nmax, k = 2, 64, 2048, 256
    rng = np.random.default_rng(4)
    n = np.array([2048, 1500], np.int32)
    ix = synth.indexer_inputs(rng, B, H_I, Nmax, n, 3)
    args = [dev(n), dev(ix["q_fp4"]), dev(ix["q_sf"]), dev(ix["w"]), dev(ix["k_fp4"]),
            dev(ix["k_sf"]), k]
    ws = csa.indexer_topk_workspace(B, Nmax, k)
    first = host(csa.indexer_topk(*args, workspace=ws))
    for _ in range(3):
        again = host(csa.indexer_topk(*args, workspace=ws))
        np.testing.assert_array_equal(again, first)


def test_indexer_workspace_shared_across_batch_sizes():
    # one workspace sized for the largest call serves smaller batches in between
    rng = np.random.default_rng(21)
    big_n = np.array([4096, 3000, 2500], np.int32)
    big = synth.indexer_inputs(rng, 3, 64, 4096, big_n)
    small_n = np.array([1500], np.int32)
    small = synth.indexer_inputs(rng, 1, 64, 4096, small_n)
    ws = csa.indexer_topk_workspace(3, 4096, 512)

    def run(ix, n):
        return host(csa.indexer_topk(dev(n), dev(ix["q_fp4"]), dev(ix["q_sf"]), dev(ix["w"]),
                                     dev(ix["k_fp4"]), dev(ix["k_sf"]), 512, workspace=ws))

    first = run(big, big_n)
    one = run(small, small_n)
    again = run(big, big_n)
    np.testing.assert_array_equal(again, first)
    ora = oracle.indexer_scores(small_n, small["q_fp4"], small["q_sf"], small["w"],
                                small["k_fp4"], small["k_sf"])
    assert compare.compare_topk(one[0], ora[0], 1500, 512, what="small batch") <= 1


# ------------------------------------------------------------------ attention
def _attn_case(B, H, Nmax, n, pos, k=None, seed=0, sink_override=None):
    rng = np.random.default_rng(seed)
    n = np.asarray(n, np.int32)
    pos = np.asarray(pos, np.int32)
    kv, sc = synth.kv_cache(rng, B, Nmax)
    q = synth.bf16_normal(rng, (B, H, 512))
    swa = synth.bf16_normal(rng, (B, 128, 512))
    sink = rng.standard_normal(H).astype(np.float32)
    if sink_override is not None:
        sink[:] = sink_override
    idx = None
    if k is not None:
        idx = np.full((B, k), -1, np.int32)
        for b in range(B):
            c = min(k - 3, int(n[b]))  # leave some padding
            idx[b, :c] = np.sort(rng.choice(int(n[b]), c, replace=False))
    return dict(q=q, pos=pos, n=n, kv=kv, sc=sc, swa=swa, sink=sink, idx=idx)


def _gpu_attn(d, derotate=True, raw=False):
    args = (dev(d["q"]), dev(d["pos"]), dev(d["n"]), dev(d["kv"]), dev(d["sc"]), dev(d["swa"]),
            dev(d["sink"]))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kw = dict(lse=True, derotate=derotate, dev_status=st)
    if d["idx"] is not None:
        out, lse = csa.sparse_attn_decode(*args, dev(d["idx"]), **kw)
    else:
        out, lse = csa.hca_attn_decode(*args, **kw)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    if raw:
        return out.view(torch.int16).cpu().numpy(), host(lse)
    return out.float().cpu().numpy(), host(lse)


def _ora_attn(d, derotate=True):
    return oracle.attention(d["q"], d["pos"], d["n"], d["kv"], d["sc"], d["swa"], d["sink"],
                            idx=d["idx"], derotate=derotate)


@pytest.mark.parametrize("B,H,Nmax,n,pos,k", [
    (2, 64, 2048, [2048, 1000], [8191, 4003], 512),      # CSA, workload 0/2 heads
    (2, 128, 4096, [4096, 3000], [16383, 12001], 1024),  # CSA, workload 3 heads
    (3, 64, 1024, [1024, 7, 0], [131071, 900, 50], None),  # HCA, ragged, early positions
    (1, 128, 256, [200], [803], 100),                     # CSA, k not a multiple of 64
    (1, 128, 4096, [4096], [16383], 2048),                # CSA at the largest k
    (1, 64, 8192, [8192], [1048575], None),               # HCA over a 1M-token context
])
def test_attention_matches_oracle(B, H, Nmax, n, pos, k):
    d = _attn_case(B, H, Nmax, n, pos, k, seed=H + B)
    out, lse = _gpu_attn(d)
    want, wlse = _ora_attn(d)
    compare.close(out, want, what="attention out")
    np.testing.assert_allclose(lse, wlse, rtol=1e-4, atol=1e-4)


def test_attention_workspace_reused_across_calls_and_batches():
    # one workspace for calls whose chunk counts per sequence change (HCA lengths grow
    # between steps)
    ws = csa.attn_workspace(3, 64, 2048 + 128)
    for trial, n in enumerate(([2048, 100, 900], [700, 2048, 5], [64, 1, 2000])):
        d = _attn_case(3, 64, 2048, n, [9000, 8000, 7000], None, seed=trial)
        args = (dev(d["q"]), dev(d["pos"]), dev(d["n"]), dev(d["kv"]), dev(d["sc"]),
                dev(d["swa"]), dev(d["sink"]))
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = csa.hca_attn_decode(*args, workspace=ws, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        want, _ = _ora_attn(d)
        compare.close(out.float().cpu().numpy(), want, what=f"call {trial}")


def test_attention_sink_limits():
    d = _attn_case(2, 64, 512, [512, 300], [2047, 1300], 256, seed=5)
    d["sink"][:5] = -np.inf
    d["sink"][5:8] = np.inf
    out, lse = _gpu_attn(d)
    want, wlse = _ora_attn(d)
    assert (out[:, 5:8] == 0).all() and np.isinf(lse[:, 5:8]).all()
    compare.close(out, want, what="sink limits")
    np.testing.assert_allclose(lse[:, :5], wlse[:, :5], rtol=1e-4)


def test_attention_without_derotation():
    d = _attn_case(1, 128, 1024, [1024], [4095], 512, seed=6)
    out, _ = _gpu_attn(d, derotate=False)
    want, _ = _ora_attn(d, derotate=False)
    compare.close(out, want, what="no derotation")


def test_attention_bad_index_is_reported():
    d = _attn_case(1, 64, 512, [300], [1203], 64, seed=7)
    d["idx"][0, 5] = 400  # beyond n_entries: skipped and reported
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    csa.sparse_attn_decode(dev(d["q"]), dev(d["pos"]), dev(d["n"]), dev(d["kv"]), dev(d["sc"]),
                           dev(d["swa"]), dev(d["sink"]), dev(d["idx"]), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == csa.CSA_ERR_DEVICE


# ------------------------------------------------------- invariance, determinism
def test_batch_invariance_and_determinism():
    w = synth.WORKLOADS[0]
    full = synth.decode_inputs(synth.Workload("inv", "csa", B=3, m=4, H=64, H_I=64, k=512,
                                              L=40000, L_min=9000, seed=11))
    B = full["B"]

    def step(sl):
        n = dev(full["n_entries"][sl])
        idx = csa.indexer_topk(n, dev(full["q_fp4"][sl]), dev(full["q_sf"][sl]),
                               dev(full["w"][sl]), dev(full["k_fp4"][sl]),
                               dev(full["k_sf"][sl]), 512)
        out = csa.sparse_attn_decode(dev(full["q"][sl]), dev(full["pos"][sl]), n,
                                     dev(full["kv"][sl]), dev(full["kv_scale"][sl]),
                                     dev(full["swa"][sl]), dev(full["sink"]), idx)
        torch.cuda.synchronize()
        return host(idx), out.view(torch.int16).cpu().numpy()

    idx_all, out_all = step(slice(0, B))
    idx_again, out_again = step(slice(0, B))
    np.testing.assert_array_equal(idx_all, idx_again)
    np.testing.assert_array_equal(out_all, out_again)
    for b in range(B):
        idx_b, out_b = step(slice(b, b + 1))
        np.testing.assert_array_equal(idx_b[0], idx_all[b])
        np.testing.assert_array_equal(out_b[0], out_all[b])


def test_attention_bits_do_not_depend_on_the_output_split():
    # a chunk's output is computed by one CTA (all 512 dims) when the batch's chunks fill
    # the SMs, and by two (one per half) when twice the chunks still fit one wave; 8
    # sequences of 18 chunks take the first path, each of them alone the second
    d = _attn_case(8, 128, 2048, [2048, 1900, 1700, 1500, 1300, 1100, 900, 700],
                   [9000, 8000, 7000, 6000, 5000, 4500, 3700, 2900], 1024, seed=23)
    full = csa.sparse_attn_decode(dev(d["q"]), dev(d["pos"]), dev(d["n"]), dev(d["kv"]),
                                  dev(d["sc"]), dev(d["swa"]), dev(d["sink"]), dev(d["idx"]))
    full = full.view(torch.int16).cpu().numpy()
    for b in range(8):
        sl = slice(b, b + 1)
        one = csa.sparse_attn_decode(dev(d["q"][sl]), dev(d["pos"][sl]), dev(d["n"][sl]),
                                     dev(d["kv"][sl]), dev(d["sc"][sl]), dev(d["swa"][sl]),
                                     dev(d["sink"]), dev(d["idx"][sl]))
        np.testing.assert_array_equal(one.view(torch.int16).cpu().numpy()[0], full[b])


# --------------------------------------------------- full decode, small workloads
def test_workload0_decode_chain():
    """Compress the 8192-token stream, score/select, attend: each stage vs the oracle fed
    with the oracle's own upstream result."""
    w = synth.WORKLOADS[0]
    inp = synth.compress_inputs(1, w.L, w.m, True, seed=w.seed)
    d = synth.decode_inputs(w)
    ora_c = oracle.compress(inp["a"], inp["za"], inp["bias"], 4, True, b=inp["b"], zb=inp["zb"])
    kv_gpu, sc_gpu, dbg = _run_compress(inp, 4, True)
    compare.compare_entries(kv_gpu, sc_gpu, dbg, ora_c, what="workload 0")
    n = d["n_entries"]
    idx = host(csa.indexer_topk(dev(n), dev(d["q_fp4"]), dev(d["q_sf"]), dev(d["w"]),
                                dev(d["k_fp4"]), dev(d["k_sf"]), w.k))
    ora_s = oracle.indexer_scores(n, d["q_fp4"], d["q_sf"], d["w"], d["k_fp4"], d["k_sf"])
    compare.compare_topk(idx[0], ora_s[0], int(n[0]), w.k, what="workload 0 top-k")
    ora_idx = oracle.topk(ora_s[0], int(n[0]), w.k)[None]
    kv, sc = ora_c["kv"], ora_c["kv_scale"]
    out = csa.sparse_attn_decode(dev(d["q"]), dev(d["pos"]), dev(n), dev(kv), dev(sc),
                                 dev(d["swa"]), dev(d["sink"]), dev(ora_idx))
    want, _ = oracle.attention(d["q"], d["pos"], n, kv, sc, d["swa"], d["sink"], idx=ora_idx)
    compare.close(out.float().cpu().numpy(), want, what="workload 0 attention")


def test_workload1_hca_decode():
    w = synth.WORKLOADS[1]
    d = synth.decode_inputs(w)
    out, lse = csa.hca_attn_decode(dev(d["q"]), dev(d["pos"]), dev(d["n_entries"]),
                                   dev(d["kv"]), dev(d["kv_scale"]), dev(d["swa"]),
                                   dev(d["sink"]), lse=True)
    want, wlse = oracle.attention(d["q"], d["pos"], d["n_entries"], d["kv"], d["kv_scale"],
                                  d["swa"], d["sink"])
    compare.close(out.float().cpu().numpy(), want, what="workload 1")
    np.testing.assert_allclose(host(lse), wlse, rtol=1e-4, atol=1e-4)


def _full_size_decode(wid):
    """A decode step of a whole workload through the calls bench.py times: every
    sequence's top-k set against the oracle's scores, then the attention output of every
    head against the oracle on the same quantised cache and the same sets."""
    w = synth.WORKLOADS[wid]
    d = synth.decode_inputs(w)
    n = d["n_entries"]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, sc = csa.indexer_topk(dev(n), dev(d["q_fp4"]), dev(d["q_sf"]), dev(d["w"]),
                               dev(d["k_fp4"]), dev(d["k_sf"]), w.k, scores=True,
                               dev_status=status)
    out, lse = csa.sparse_attn_decode(dev(d["q"]), dev(d["pos"]), dev(n), dev(d["kv"]),
                                      dev(d["kv_scale"]), dev(d["swa"]), dev(d["sink"]), idx,
                                      lse=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    idx_h, sc_h = host(idx), host(sc)
    ora_s = oracle.indexer_scores(n, d["q_fp4"], d["q_sf"], d["w"], d["k_fp4"], d["k_sf"])
    flips = 0
    for b in range(d["B"]):
        flips += compare.compare_topk(idx_h[b], ora_s[b], int(n[b]), w.k, what=f"{w.name} {b}")
        keep = min(w.k, int(n[b]))
        np.testing.assert_allclose(sc_h[b][:keep], ora_s[b][idx_h[b][:keep]], rtol=2e-5,
                                   atol=1e-6)
    assert flips <= 2 * d["B"]
    want, wlse = oracle.attention(d["q"], d["pos"], n, d["kv"], d["kv_scale"], d["swa"],
                                  d["sink"], idx=idx_h)
    compare.close(out.float().cpu().numpy(), want, what=f"{w.name} attention")
    np.testing.assert_allclose(host(lse), wlse, rtol=1e-4, atol=1e-4)


def test_workload2_full_size_decode():
    # 32 sequences of 64K-128K tokens (16K-32K entries), 64 heads, top-k 512
    _full_size_decode(2)


def test_workload3_full_size_decode():
    # 4 sequences at 1M tokens (262,144 entries), 128 heads, top-k 1024, planted runs
    _full_size_decode(3)
