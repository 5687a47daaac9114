"""Oracle: the two kernels that keep the paged KV pool consistent.

TEST INFRASTRUCTURE ONLY — see ``oracle/__init__.py``.

* ``ref_reshape_and_cache`` — each decode step computes one new key and value
  per token and stores them in the cache for later steps ("什么是 LLM 中的分页注意力",
  section 快速回顾:KV 缓存); the paged form writes token ``t``'s K/V into the slot
  the slot mapping gives, slot ``s`` meaning physical block ``s // block_size``
  at offset ``s % block_size`` (the same addressing as the section 块表 table).
  A negative slot means "skip this token".
* ``ref_copy_blocks`` — copy on write: before a forked sequence writes into a
  block it still shares, the block is copied so that the sibling's prefix is
  not modified ("PagedAttention" concept card, section 实现要点; "深入解析
  PagedAttention", section 多序列共享).  The whole block is copied (every slot,
  K and V).

Both return new arrays; the inputs are not modified.
"""

from __future__ import annotations

import numpy as np


def ref_reshape_and_cache(key, value, k_pool, v_pool, slot_mapping):
    """Scatter ``key[t]``/``value[t]`` (``[T, Hkv, D]``) into copies of the pools.

    ``slot_mapping[t]`` is the flat slot of token ``t``; ``< 0`` skips it.
    """
    block_size = k_pool.shape[1]
    k_new = np.array(k_pool, copy=True)
    v_new = np.array(v_pool, copy=True)
    for t in range(len(slot_mapping)):
        s = int(slot_mapping[t])
        if s < 0:
            continue
        k_new[s // block_size, s % block_size] = key[t]
        v_new[s // block_size, s % block_size] = value[t]
    return k_new, v_new


def ref_copy_blocks(k_pool, v_pool, pairs):
    """Copy whole physical blocks ``src → dst`` for each ``(src, dst)`` in ``pairs``."""
    k_new = np.array(k_pool, copy=True)
    v_new = np.array(v_pool, copy=True)
    for src, dst in pairs:
        k_new[int(dst)] = k_pool[int(src)]
        v_new[int(dst)] = v_pool[int(src)]
    return k_new, v_new
