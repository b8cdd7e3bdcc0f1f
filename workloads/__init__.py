"""Seeded synthetic inputs shaped like the pages' workloads.

This module is shared by the tests, the oracle side and the benchmark.  It generates numbers and
shapes only: it contains none of the attention arithmetic.  Every tensor is drawn in fp32 from a
seeded generator, scaled, and rounded once to bf16 (round-to-nearest-even, done by
``Tensor.to(torch.bfloat16)``); both the CUDA path and the oracle read that single copy (the
oracle upcasts it to fp64, which is exact).

Workloads (sizes from the pages: h_q = 32, d_h = 128, T = 8192 and the 32/8/1 KV-head sweep from
the MHA/MQA/GQA walkthrough's parameter table; 64 query / 8 KV heads from 第三章 §3.3):

* ``prefill_small``   causal prefill, B=1, h_q=4, h_kv=2, T=256, d_h=64, N(0,1).
* ``decode_8k``       decode, B=8, h_q=32, d_h=128, T=8192, h_kv in {32, 8, 1}, N(0,1);
                      the query sits at position 8191 and sees every key.
* ``prefill_4k``      causal prefill, B=1, h_q=32, h_kv=8, T=4096, d_h=128, N(0,1)*0.5.
* ``ragged_decode``   decode, B=64, h_q=64, h_kv=8, d_h=128, lengths uniform integers on
                      [1024, 32768] (inclusive), cache allocated at 32768, tail filled with NaN.
* ``chunked_prefill`` B=1, h_q=32, h_kv=8, d_h=128: 32256 cached positions, then 512 new
                      queries at positions 32256..32767 over T=32768 after appending their K/V.
* paged variants of the decode workloads: the same q and lengths over K/V pools of fixed-size
  pages, assigned to sequences in a seeded random order (``paged_decode_inputs``).
"""

from __future__ import annotations

import dataclasses

import numpy as np
import torch

DEFAULT_SEED = 0
PAGES_SEED = 1949  # the seed the 第 09 章 checks were recorded with (§09.6)


@dataclasses.dataclass(frozen=True)
class PrefillShape:
    B: int
    h_q: int
    h_kv: int
    S_q: int
    T_max: int
    d_h: int
    q_start: int
    kv_len: int
    std: float = 1.0


@dataclasses.dataclass(frozen=True)
class DecodeShape:
    B: int
    h_q: int
    h_kv: int
    T_max: int
    d_h: int
    std: float = 1.0
    ragged: bool = False
    len_lo: int = 0
    len_hi: int = 0


PREFILL_SMALL = PrefillShape(B=1, h_q=4, h_kv=2, S_q=256, T_max=256, d_h=64, q_start=0, kv_len=256)
PREFILL_4K = PrefillShape(B=1, h_q=32, h_kv=8, S_q=4096, T_max=4096, d_h=128, q_start=0,
                          kv_len=4096, std=0.5)
CHUNKED_PREFILL = PrefillShape(B=1, h_q=32, h_kv=8, S_q=512, T_max=32768, d_h=128, q_start=32256,
                               kv_len=32768)
DECODE_8K = {h_kv: DecodeShape(B=8, h_q=32, h_kv=h_kv, T_max=8192, d_h=128) for h_kv in (32, 8, 1)}
RAGGED_DECODE = DecodeShape(B=64, h_q=64, h_kv=8, T_max=32768, d_h=128, ragged=True,
                            len_lo=1024, len_hi=32768)


def ragged_lengths(seed: int, B: int = 64, lo: int = 1024, hi: int = 32768) -> np.ndarray:
    """Per-request cached lengths, uniform integers on [lo, hi] inclusive."""
    return np.random.default_rng(seed).integers(lo, hi + 1, size=B).astype(np.int32)


def _generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn_bf16(shape, gen: torch.Generator, std: float = 1.0, device="cpu",
               dtype=torch.bfloat16) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 from ``gen``, rounded once to ``dtype``."""
    x = torch.randn(shape, generator=gen, dtype=torch.float32, device=device)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def prefill_inputs(shape: PrefillShape, seed: int = DEFAULT_SEED, device="cpu",
                   dtype=torch.bfloat16):
    """Q (B,h_q,S_q,d_h) and the K/V cache (B,h_kv,T_max,d_h); draw order Q, K, V."""
    g = _generator(seed, device)
    q = randn_bf16((shape.B, shape.h_q, shape.S_q, shape.d_h), g, shape.std, device, dtype)
    k = randn_bf16((shape.B, shape.h_kv, shape.T_max, shape.d_h), g, shape.std, device, dtype)
    v = randn_bf16((shape.B, shape.h_kv, shape.T_max, shape.d_h), g, shape.std, device, dtype)
    return q, k, v


def chunked_prefill_inputs(shape: PrefillShape = CHUNKED_PREFILL, seed: int = DEFAULT_SEED,
                           device="cpu", dtype=torch.bfloat16):
    """Cache with positions < q_start filled (rest zero), the new K/V chunk and the new queries.

    Draw order: K cache, V cache, K new, V new, Q.
    """
    g = _generator(seed, device)
    B, h_kv, T, d = shape.B, shape.h_kv, shape.T_max, shape.d_h
    k = torch.zeros((B, h_kv, T, d), dtype=dtype, device=device)
    v = torch.zeros((B, h_kv, T, d), dtype=dtype, device=device)
    k[:, :, :shape.q_start] = randn_bf16((B, h_kv, shape.q_start, d), g, shape.std, device, dtype)
    v[:, :, :shape.q_start] = randn_bf16((B, h_kv, shape.q_start, d), g, shape.std, device, dtype)
    k_new = randn_bf16((B, h_kv, shape.S_q, d), g, shape.std, device, dtype)
    v_new = randn_bf16((B, h_kv, shape.S_q, d), g, shape.std, device, dtype)
    q = randn_bf16((B, shape.h_q, shape.S_q, d), g, shape.std, device, dtype)
    return k, v, k_new, v_new, q


def decode_inputs(shape: DecodeShape, seed: int = DEFAULT_SEED, device="cpu",
                  dtype=torch.bfloat16, nan_tail: bool = True):
    """q (B,h_q,d_h), K/V cache (B,h_kv,T_max,d_h), kv_len (B,) int32.

    Draw order: q, K, V.  For ragged shapes the positions at or beyond each request's length
    are overwritten with NaN (a sentinel that must never reach an output).
    """
    g = _generator(seed, device)
    q = randn_bf16((shape.B, shape.h_q, shape.d_h), g, shape.std, device, dtype)
    k = randn_bf16((shape.B, shape.h_kv, shape.T_max, shape.d_h), g, shape.std, device, dtype)
    v = randn_bf16((shape.B, shape.h_kv, shape.T_max, shape.d_h), g, shape.std, device, dtype)
    if shape.ragged:
        lens = ragged_lengths(seed, shape.B, shape.len_lo, shape.len_hi)
        if nan_tail:
            for b in range(shape.B):
                k[b, :, int(lens[b]):] = float("nan")
                v[b, :, int(lens[b]):] = float("nan")
    else:
        lens = np.full(shape.B, shape.T_max, np.int32)
    kv_len = torch.from_numpy(lens).to(device)
    return q, k, v, kv_len


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact upcast of a (bf16 or fp32) tensor to a float64 NumPy array on the host."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def paged_block_table(lengths, page_size: int, seed: int, spare_pages: int = 3,
                      max_pages: int | None = None):
    """A shuffled page assignment for sequences of the given lengths.

    Returns (block_table (B, max_pages) int32, num_pages). Sequence b owns ceil(len_b / page_size)
    distinct pages drawn in a seeded random order from a pool that also holds ``spare_pages``
    unused pages; table entries past a sequence's last page are -1 (never read).
    """
    lengths = np.asarray(lengths, np.int64)
    need = [(int(n) + page_size - 1) // page_size for n in lengths]
    num_pages = int(sum(need)) + spare_pages
    perm = np.random.default_rng(seed).permutation(num_pages).astype(np.int32)
    mp = max(need) if max_pages is None else max_pages
    table = np.full((len(lengths), max(mp, 1)), -1, np.int32)
    at = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[at:at + n]
        at += n
    return table, num_pages


def paged_decode_inputs(shape: DecodeShape, page_size: int, seed: int = DEFAULT_SEED, device="cpu",
                        dtype=torch.bfloat16, lengths=None, spare_pages: int = 3):
    """q (B,h_q,d_h), K/V page pools (num_pages, h_kv, page_size, d_h), block_table (B, max_pages)
    int32, kv_len (B,) int32.

    Draw order: q, K pool, V pool (the pool is drawn whole, then every row that holds no visible
    position -- spare pages and the tail of each sequence's last page -- is set to NaN). Lengths
    are ``lengths`` if given, else ragged_lengths for ragged shapes, else T_max.
    """
    if lengths is None:
        lengths = (ragged_lengths(seed, shape.B, shape.len_lo, shape.len_hi) if shape.ragged
                   else np.full(shape.B, shape.T_max, np.int32))
    lengths = np.asarray(lengths, np.int32)
    table, num_pages = paged_block_table(lengths, page_size, seed + 1, spare_pages,
                                         max_pages=(shape.T_max + page_size - 1) // page_size)
    g = _generator(seed, device)
    q = randn_bf16((shape.B, shape.h_q, shape.d_h), g, shape.std, device, dtype)
    pool = (num_pages, shape.h_kv, page_size, shape.d_h)
    k = randn_bf16(pool, g, shape.std, device, dtype)
    v = randn_bf16(pool, g, shape.std, device, dtype)
    used = np.zeros((num_pages, page_size), bool)
    for b, n in enumerate(lengths):
        for t0 in range(0, int(n), page_size):
            used[table[b, t0 // page_size], :min(page_size, int(n) - t0)] = True
    unused = torch.from_numpy(~used).to(device)
    k.transpose(1, 2)[unused] = float("nan")  # (num_pages, page_size) rows, every KV head
    v.transpose(1, 2)[unused] = float("nan")
    return q, k, v, torch.from_numpy(table).to(device), torch.from_numpy(lengths).to(device)


@dataclasses.dataclass(frozen=True)
class MlaShape:
    B: int
    h_q: int
    T_max: int
    d_qk: int = 576  # latent 512 + decoupled rotary key 64 (DeepSeek-V2/V3 widths)
    d_v: int = 512
    d_nope: int = 128  # per-head widths of the original (non-absorbed) heads, for the scale
    d_rope: int = 64

    @property
    def scale(self) -> float:
        return (self.d_nope + self.d_rope) ** -0.5


# MLA decode at the decode_8k sizes: B=8, T=8192, 16 heads per GPU (128 heads split 8 ways) and
# all 128 heads on one GPU.
MLA_DECODE = {h: MlaShape(B=8, h_q=h, T_max=8192) for h in (16, 128)}


def mla_decode_inputs(shape: MlaShape, seed: int = DEFAULT_SEED, device="cpu", dtype=torch.bfloat16,
                      lengths=None, nan_tail: bool = True):
    """q (B, h_q, d_qk), cache (B, T_max, d_qk), kv_len (B,) int32. Draw order: q, cache.
    Rows at or past each length are NaN when ``nan_tail``."""
    g = _generator(seed, device)
    q = randn_bf16((shape.B, shape.h_q, shape.d_qk), g, 1.0, device, dtype)
    cache = randn_bf16((shape.B, shape.T_max, shape.d_qk), g, 1.0, device, dtype)
    lens = (np.full(shape.B, shape.T_max, np.int32) if lengths is None
            else np.asarray(lengths, np.int32))
    if nan_tail:
        for b in range(shape.B):
            cache[b, int(lens[b]):] = float("nan")
    return q, cache, torch.from_numpy(lens).to(device)
