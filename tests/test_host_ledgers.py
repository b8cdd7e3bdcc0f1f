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


def test_bench_ledgers_at_the_five_configs():
    """The bench's algorithmic work at the five workloads equals the closed forms: causal prefill
    4 d_h B h_q sum_i (q_start + i + 1) FLOPs; decode 2 B h_kv T d_h 2 KV bytes; the backward's five
    GEMMs per visible pair are 2.5x the forward's two."""
    # prefill_small: 4 * 4 * 64 * (256 * 257 / 2)
    assert bench.prefill_flops(1, 4, 64, 256, 0, 256) == 33_685_504
    # prefill_4k: 4 * 32 * 128 * (4096 * 4097 / 2)
    assert bench.prefill_flops(1, 32, 128, 4096, 0, 4096) == 137_472_507_904
    # chunked prefill: 512 rows at positions 32256..32767, each sees position + 1 keys
    assert bench.prefill_flops(1, 32, 128, 512, 32256, 32768) == 272_734_617_600
    # decode_8k: 1 GiB / 256 MiB / 32 MiB of K/V for h_kv = 32 / 8 / 1
    for h_kv, nbytes in ((32, 1_073_741_824), (8, 268_435_456), (1, 33_554_432)):
        assert bench.decode_kv_bytes(8, h_kv, [8192] * 8, 128) == nbytes
    # ragged_decode: 2 * 8 * 128 * 2 = 4096 bytes per visible key
    lens = workloads.ragged_lengths(0)
    assert bench.decode_kv_bytes(64, 8, lens.tolist(), 128) == 4096 * int(lens.sum())
    assert lens.min() >= 1024 and lens.max() <= 32768 and lens.shape == (64,)
    # backward of prefill_4k, as the bench line states it
    assert 5 * bench.prefill_flops(1, 32, 128, 4096, 0, 4096) // 2 == 343_681_269_760
