"""Pins of the oracle's paged-cache view (oracle.paged_view / paged_scatter): a worked
example by hand, the one-page-per-sequence case that is the contiguous layout itself,
round trips through shuffled tables, and the 128-entry grouping of the key scales
agreeing with the per-entry placement. (walkthrough §3.5: the classical cache holds the
compressed entries; pages are whole multiples of 128 tokens.)"""

import numpy as np
import pytest

import oracle


def test_worked_example_by_hand():
    # two entries per page; sequence 0 uses pages 2 then 0, sequence 1 page 1 then none
    pool = np.array([[0, 1], [10, 11], [20, 21]], np.int32)[:, :, None]
    table = np.array([[2, 0], [1, -1]], np.int32)
    view = oracle.paged_view(pool, table, 2)[:, :, 0]
    np.testing.assert_array_equal(view, [[20, 21, 0, 1], [10, 11, 0, 0]])


def test_one_page_per_sequence_is_the_contiguous_layout():
    rng = np.random.default_rng(0)
    B, Nmax = 3, 256
    kv = rng.integers(0, 256, (B, Nmax, 576), dtype=np.uint8)
    ksf = rng.integers(0, 256, (B, Nmax // 128, 512), dtype=np.uint8)
    table = np.arange(B, dtype=np.int32)[:, None]
    np.testing.assert_array_equal(oracle.paged_view(kv, table, Nmax), kv)
    np.testing.assert_array_equal(oracle.paged_view(ksf, table, Nmax, group=128), ksf)


@pytest.mark.parametrize("page_entries", [128, 256, 512, 2048])
def test_shuffled_tables_round_trip(page_entries):
    rng = np.random.default_rng(page_entries)
    B, Nmax = 3, 4096
    pages_max = Nmax // page_entries
    num_pages = B * pages_max + 5  # spare pages stay unused
    table = rng.permutation(num_pages)[:B * pages_max].reshape(B, pages_max).astype(np.int32)
    kv = rng.integers(0, 256, (B, Nmax, 576), dtype=np.uint8)
    ksf = rng.integers(0, 256, (B, Nmax // 128, 512), dtype=np.uint8)
    pool = oracle.paged_scatter(kv, table, page_entries, num_pages)
    sf_pool = oracle.paged_scatter(ksf, table, page_entries, num_pages, group=128)
    assert pool.shape == (num_pages, page_entries, 576)
    assert sf_pool.shape == (num_pages, page_entries // 128, 512)
    np.testing.assert_array_equal(oracle.paged_view(pool, table, page_entries), kv)
    np.testing.assert_array_equal(oracle.paged_view(sf_pool, table, page_entries, group=128), ksf)
    # and entry j really sits in slot j % P of page table[b][j // P]
    for b, j in ((0, 0), (1, page_entries - 1), (2, Nmax - 1), (1, 3 * page_entries // 2)):
        np.testing.assert_array_equal(pool[table[b, j // page_entries], j % page_entries], kv[b, j])


def test_grouped_scales_follow_their_entries():
    # the scale bytes of entry j (at the grouped offset of j) land in the page that holds
    # entry j, at the grouped offset of its slot j % P
    rng = np.random.default_rng(3)
    B, Nmax, P = 2, 1024, 256
    pages_max = Nmax // P
    num_pages = B * pages_max
    table = rng.permutation(num_pages).reshape(B, pages_max).astype(np.int32)
    ksf = rng.integers(0, 256, (B, Nmax // 128, 512), dtype=np.uint8)
    sf_pool = oracle.paged_scatter(ksf, table, P, num_pages, group=128)
    for b in range(B):
        for j in rng.integers(0, Nmax, 40):
            for s in range(4):
                want = ksf[b].reshape(-1)[oracle.key_sf_offset(int(j), s)]
                page = table[b, j // P]
                got = sf_pool[page].reshape(-1)[oracle.key_sf_offset(int(j % P), s)]
                assert got == want


def test_indexer_scores_through_pages_equal_contiguous():
    from synth import inputs as synth
    rng = np.random.default_rng(5)
    B, H_I, Nmax, P = 2, 16, 1024, 256
    n = np.array([1024, 700], np.int32)
    ix = synth.indexer_inputs(rng, B, H_I, Nmax, n)
    pages_max = Nmax // P
    table = rng.permutation(B * pages_max).reshape(B, pages_max).astype(np.int32)
    kp = oracle.paged_scatter(ix["k_fp4"], table, P, B * pages_max)
    sp = oracle.paged_scatter(ix["k_sf"].reshape(B, Nmax // 128, 512), table, P, B * pages_max,
                              group=128)
    got = oracle.indexer_scores(n, ix["q_fp4"], ix["q_sf"], ix["w"],
                                oracle.paged_view(kp, table, P),
                                oracle.paged_view(sp, table, P, group=128).reshape(B, -1))
    want = oracle.indexer_scores(n, ix["q_fp4"], ix["q_sf"], ix["w"], ix["k_fp4"], ix["k_sf"])
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    np.testing.assert_array_equal(got[~np.isnan(got)], want[~np.isnan(want)])
