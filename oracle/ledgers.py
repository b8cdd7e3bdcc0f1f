"""Byte, parameter and FLOP ledgers the pages write out, as plain integer formulas.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``). The benchmark's algorithmic byte and FLOP
counts are defined by these same formulas, restated independently in ``bench.py``'s accounting;
the tests pin both to the pages' printed values.
"""

from __future__ import annotations


def kv_cache_bytes(L: int, B: int, T: int, h_kv: int, d_h: int, s: int) -> int:
    """C_KV = 2 L B T h_kv d_h s: K and V, each B*T*h_kv*d_h scalars of s bytes, per layer.

    [序列计算与存储 §缓存字节; 第三章 §3.2 (KVBytes = 2 B L N H_KV d_h s); 第 09 章 §09.1.]
    """
    return 2 * L * B * T * h_kv * d_h * s


def kv_bytes_per_token_layer(h_kv: int, d_h: int, s: int) -> int:
    """Cache payload one token adds to one layer: 2 h_kv d_h s [MHA/MQA/GQA 逐步算例 §4-§6]."""
    return 2 * h_kv * d_h * s


def kv_ratio_vs_mha(h_q: int, h_kv: int) -> float:
    """Cache size relative to MHA with the same query heads: h_kv / h_q [序列计算与存储 §缓存字节]."""
    return h_kv / h_q


def projection_params(d: int, h_q: int, h_kv: int, d_h: int) -> int:
    """Bias-free projection parameters, counted Q, K, V, output [序列计算与存储 §头与投影].

    W_Q: d x h_q d_h; W_K, W_V: d x h_kv d_h; W_O: h_q d_h x d.
    """
    return d * h_q * d_h + 2 * d * h_kv * d_h + h_q * d_h * d


def decode_flops(h_q: int, T: int, d_h: int) -> int:
    """QK plus PV FLOPs of one decode token in one layer: 4 h_q T d_h [MHA/MQA/GQA 逐步算例 §8].

    Each query head does a (1 x d_h)(d_h x T) and a (1 x T)(T x d_h) product, 2 FLOPs per
    multiply-add.
    """
    return 4 * h_q * T * d_h


def kv_read_intensity(h_q: int, h_kv: int, d_h: int, s: int, T: int) -> float:
    """Ideal FLOPs per KV byte read once from HBM for one decode token [MHA/MQA/GQA 逐步算例 §8]."""
    return decode_flops(h_q, T, d_h) / (T * kv_bytes_per_token_layer(h_kv, d_h, s))


def score_tensor_elements(B: int, h_q: int, T: int) -> int:
    """Elements of the full score tensor over all heads, B h_q T^2 [序列计算与存储 §资源变化]."""
    return B * h_q * T * T


def prefill_visible_pairs(S_q: int, q_start: int, kv_len: int, causal: bool = True) -> int:
    """Number of (query, key) pairs a causal prefill actually scores for one head.

    Query i sits at q_start + i and sees min(kv_len, q_start + i + 1) keys.
    """
    total = 0
    for i in range(S_q):
        n = min(kv_len, q_start + i + 1) if causal else kv_len
        total += max(0, n)
    return total


def prefill_flops(B: int, h_q: int, d_h: int, S_q: int, q_start: int, kv_len: int,
                  causal: bool = True) -> int:
    """Algorithmic FLOPs of a (causal) prefill: 4 d_h per visible pair per head (QK and PV)."""
    return 4 * d_h * B * h_q * prefill_visible_pairs(S_q, q_start, kv_len, causal)


def decode_kv_read_bytes(lengths, h_kv: int, d_h: int, s: int) -> int:
    """KV bytes a decode must read once: sum over sequences of 2 h_kv len d_h s."""
    return sum(2 * h_kv * int(n) * d_h * s for n in lengths)
