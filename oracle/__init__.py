"""Oracle for the paged decode-attention path — TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct CPU code (NumPy, float64) that states what the
GPU library computes, so that the library can be checked against it.  Only
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference
leg of ``bench.py`` may import it.  The product package never imports this
module, and this module never imports the product package: the two share no
code.  The seeded input generators both sides use live in ``workloads/``.

Sources (web pages on PagedAttention):

* "什么是分页注意力（PagedAttention）" (aiboss88.com wiki), section 边界与常见误解:
  paging changes neither the weights nor the mathematical definition of
  attention, only where the KV cache lives and how it is addressed.
* "PagedAttention" concept card (awesome-system-papers), sections 核心思想 and
  实现要点: fixed-size physical blocks (16 tokens typical), a per-sequence block
  table from logical block index to physical block, the kernel reads K/V
  through the table; copy-on-write with reference counts on fork.
* "深入解析 PagedAttention" (cygnushan.xyz), sections 工作原理 (block table with
  ``-1`` padding, shared prefix) and 多序列共享 (free at refcount 0, copy on
  write).
* "什么是 LLM 中的分页注意力" (news.rkmt.cn/news/13929), sections 使用分页注意力
  and 块表: the worked example (block size 4, ten tokens, table 0→5, 1→12,
  2→3, two empty slots in the last block).

Modules:

* ``oracle.decode``    — ``ref_decode``: gather K/V through the table into
  contiguous float64 arrays, then scaled dot-product softmax attention.
* ``oracle.cache_ops`` — ``ref_reshape_and_cache``, ``ref_copy_blocks``.
* ``oracle.allocator`` — ``RefAllocator``: the block allocator with reference
  counts (free list, fork, append with copy-on-write, free).

Parity status: every function here is pinned by ``tests/test_oracle.py``
against facts the pages print (the worked example, the sharing diagram) and
against mathematics (brute-force loops, closed forms, invariants, a library
attention routine).  No function is "parity unpinned".
"""

from .decode import gather_kv, ref_decode
from .cache_ops import ref_reshape_and_cache, ref_copy_blocks
from .allocator import RefAllocator, OutOfBlocks, splitmix64_stream

__all__ = [
    "gather_kv",
    "ref_decode",
    "ref_reshape_and_cache",
    "ref_copy_blocks",
    "RefAllocator",
    "OutOfBlocks",
    "splitmix64_stream",
]
