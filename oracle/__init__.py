"""Plain, slow, fp64 CPU oracle for causal grouped-query attention over an unexpanded KV cache.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package. The CUDA library never imports it, and it imports
nothing from the CUDA library: the two share no code, headers, tables or helpers. The only module
both sides use is ``workloads`` (seeded input generators, none of the method's arithmetic).

Sources are the five web pages this project is built from, cited by title and section:

* [序列计算与存储] "序列计算与存储" (efficient sequence models notes), sections 分组查询注意力,
  头与投影, 缓存字节, 分块注意力, 在线 softmax, 两块算例, 资源变化.
* [第三章] "第三章：MHA 的局限与 MQA、GQA、Flash Attention", sections 3.1-3.7.
* [MHA/MQA/GQA 逐步算例] the MHA / MQA / GQA walkthrough (zane-jiang.github.io, mha-mqa-gqa),
  sections 1-9 and its parameter table.
* [04 注意力表示与 KV Cache 演进] sections on evidence levels.
* [第 09 章] "第 09 章 GQA、MLA 与跨层 KV 共享", sections 09.1-09.6.

Every function is pinned by ``tests/test_oracle_pins.py`` against values the pages print, closed
forms, invariants and independent library routines; nothing here is "parity unpinned".
"""

from .attention_ref import (
    group_of,
    head_attention,
    attention_ref,
    decode_ref,
    visible_count,
)
from .online_softmax import online_softmax_row, merge_states, blockwise_attention_row
from .kv_append_ref import kv_append_ref
from .paged import gather_pages, paged_append_ref, paged_decode_ref
from .backward import attention_backward_ref, softmax_backward_rowterm
from .mla import mla_decode_ref, mla_explicit_ref
from . import ledgers

__all__ = [
    "group_of",
    "head_attention",
    "attention_ref",
    "decode_ref",
    "visible_count",
    "online_softmax_row",
    "merge_states",
    "blockwise_attention_row",
    "kv_append_ref",
    "gather_pages",
    "paged_decode_ref",
    "paged_append_ref",
    "attention_backward_ref",
    "softmax_backward_rowterm",
    "mla_decode_ref",
    "mla_explicit_ref",
    "ledgers",
]
