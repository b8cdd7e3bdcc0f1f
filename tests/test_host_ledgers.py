"""Host-side logic without a GPU: the bench's algorithmic-work ledgers against the oracle's
ledgers, and the paged-cache input generator's block tables."""

import numpy as np
import pytest

import bench
import oracle
import workloads
from oracle import ledgers


@pytest.mark.parametrize("window", [0, 1, 100, 1024, 5000])
def test_prefill_flops_ledger_matches_visible_pairs(window):
    S, T, q_start, h_q, d = 300, 700, 400, 8, 64
    pairs = sum(oracle.visible_count(q_start + i, T, window=window or None) for i in range(S))
    assert bench.prefill_flops(1, h_q, d, S, q_start, T, window) == 4 * d * h_q * pairs
    if window == 0:
        assert bench.prefill_flops(1, h_q, d, S, q_start, T) == ledgers.prefill_flops(1, h_q, d, S, q_start, T)


def test_decode_bytes_ledger_matches_oracle_ledger():
    lens = [8192] * 8
    for h_kv in (32, 8, 1):
        assert bench.decode_kv_bytes(8, h_kv, lens, 128) == ledgers.decode_kv_read_bytes(lens, h_kv, 128, 2)


@pytest.mark.parametrize("page_size", [1, 16, 48])
def test_paged_block_table_assigns_distinct_pages(page_size):
    lens = np.array([1, 16, 17, 300, 0 + 5])
    table, num_pages = workloads.paged_block_table(lens, page_size, seed=3, spare_pages=4)
    need = [(int(n) + page_size - 1) // page_size for n in lens]
    assert num_pages == sum(need) + 4
    used = []
    for b, n in enumerate(need):
        assert np.all(table[b, :n] >= 0) and np.all(table[b, :n] < num_pages)
        assert np.all(table[b, n:] == -1)
        used.extend(table[b, :n].tolist())
    assert len(used) == len(set(used))  # no page shared between sequences


def test_paged_decode_inputs_spell_out_a_finite_cache():
    shape = workloads.DecodeShape(B=3, h_q=4, h_kv=2, T_max=100, d_h=16)
    q, k, v, bt, kl = workloads.paged_decode_inputs(shape, 16, seed=2, lengths=[100, 33, 1])
    kc = oracle.gather_pages(workloads.to_f64(k), bt.numpy(), kl.numpy(), 100)
    for b, n in enumerate([100, 33, 1]):
        assert np.isfinite(kc[b, :, :n]).all() and np.isnan(kc[b, :, n:]).all()
    # every row of the pool that no sequence reads is NaN
    assert np.isnan(workloads.to_f64(k)).sum() == (k.shape[0] * 16 - 134) * 2 * 16
