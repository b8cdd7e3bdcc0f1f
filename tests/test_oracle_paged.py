"""Pins for the paged-cache oracle: it is the contiguous definition on the gathered cache, so
scattering a contiguous cache into a shuffled page pool and gathering it back is the identity,
and paged decode equals contiguous decode on the same data."""

import numpy as np
import pytest

import oracle


def _scatter(cache, lengths, page_size, num_pages, rng):
    """A shuffled page pool plus block table that spell out ``cache`` (B, h_kv, T, d)."""
    B, h_kv, T, d = cache.shape
    max_pages = (T + page_size - 1) // page_size
    pool = rng.standard_normal((num_pages, h_kv, page_size, d))
    table = np.full((B, max_pages), -1, np.int64)
    free = list(rng.permutation(num_pages))
    for b in range(B):
        for i in range((int(lengths[b]) + page_size - 1) // page_size):
            page = free.pop()
            table[b, i] = page
            m = min(page_size, T - i * page_size)
            pool[page, :, :m] = cache[b, :, i * page_size:i * page_size + m]
    return pool, table


@pytest.mark.parametrize("page_size", [1, 4, 16])
def test_gather_inverts_scatter_and_decode_matches(page_size):
    rng = np.random.default_rng(1949)
    B, h_q, h_kv, T, d = 3, 8, 2, 37, 8
    k = rng.standard_normal((B, h_kv, T, d))
    v = rng.standard_normal((B, h_kv, T, d))
    q = rng.standard_normal((B, h_q, d))
    lens = np.array([37, 20, 1])
    n_pages = 3 * ((T + page_size - 1) // page_size) + 5
    kp, table = _scatter(k, lens, page_size, n_pages, rng)
    vp = np.zeros_like(kp)  # V uses the same block table
    for b in range(B):
        for i in range((int(lens[b]) + page_size - 1) // page_size):
            m = min(page_size, T - i * page_size)
            vp[table[b, i], :, :m] = v[b, :, i * page_size:i * page_size + m]
    g = oracle.gather_pages(kp, table, lens, T_max=T)
    for b in range(B):
        assert np.array_equal(g[b, :, :lens[b]], k[b, :, :lens[b]])
        assert np.isnan(g[b, :, lens[b]:]).all()
    O, L = oracle.paged_decode_ref(q, kp, vp, table, lens)
    Oc, Lc = oracle.decode_ref(q, k, v, kv_len=lens)
    assert np.array_equal(O, Oc) and np.array_equal(L, Lc)


def test_paged_append_writes_exactly_the_mapped_rows():
    rng = np.random.default_rng(2)
    num_pages, h_kv, ps, d = 6, 2, 4, 3
    kp = rng.integers(0, 60000, size=(num_pages, h_kv, ps, d), dtype=np.uint16)
    vp = rng.integers(0, 60000, size=(num_pages, h_kv, ps, d), dtype=np.uint16)
    table = np.array([[5, 1, 3], [0, 2, 4]])
    kn = rng.integers(0, 60000, size=(2, h_kv, 3, d), dtype=np.uint16)
    vn = rng.integers(0, 60000, size=(2, h_kv, 3, d), dtype=np.uint16)
    k2, v2 = oracle.paged_append_ref(kp, vp, kn, vn, table, [3, 8])
    # seq 0: positions 3,4,5 -> page 5 row 3, page 1 rows 0,1; seq 1: 8,9,10 -> page 4 rows 0,1,2
    assert np.array_equal(k2[5, :, 3], kn[0, :, 0]) and np.array_equal(k2[1, :, 0], kn[0, :, 1])
    assert np.array_equal(k2[1, :, 1], kn[0, :, 2]) and np.array_equal(v2[4, :, 2], vn[1, :, 2])
    touched = np.zeros(kp.shape, bool)
    touched[5, :, 3] = touched[1, :, 0] = touched[1, :, 1] = True
    touched[4, :, 0] = touched[4, :, 1] = touched[4, :, 2] = True
    assert np.array_equal(k2[~touched], kp[~touched]) and np.array_equal(v2[~touched], vp[~touched])
    with pytest.raises(ValueError):
        oracle.paged_append_ref(kp, vp, kn, vn, table, [10, 0])  # runs past the table
    with pytest.raises(ValueError):
        oracle.paged_append_ref(kp, vp, kn, vn, np.array([[9, 1, 3], [0, 2, 4]]), [0, 0])
