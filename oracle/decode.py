"""Oracle: batched single-token decode attention over a paged KV pool (float64).

TEST INFRASTRUCTURE ONLY — see ``oracle/__init__.py``.

What it computes
----------------
Paging does not change the attention math ("什么是分页注意力", section
边界与常见误解); only the addressing of K/V changes.  So the oracle first undoes
the paging — it gathers each sequence's keys and values through its block
table into contiguous arrays, the contiguous form that paging replaces
("PagedAttention" concept card, section 核心思想) — and then applies the plain
scaled dot-product attention definition the concept card cites (section
引用本概念的论文, "Attention Is All You Need") to the single new query token.

Readings where the pages are silent (each listed in the design notes):

* GQA: query head ``h`` reads KV head ``h // (Hq // Hkv)``.
* ``seq_lens[b]`` counts every cached token of sequence ``b``, including the
  one written this step; the query attends to all of them (a single decode
  token needs no causal mask).
* ``seq_lens[b] == 0`` gives an all-zero output row (an empty sum).
* Table entries at logical index ``>= ceil(L / block_size)`` are never read
  (they may be ``-1``, as in the sharing diagram of "深入解析 PagedAttention",
  section 工作原理); slots of the last block past ``L`` are never read.

Token ``t`` of sequence ``b`` lives in physical block
``block_tables[b, t // block_size]`` at offset ``t % block_size`` ("什么是 LLM
中的分页注意力", section 块表: the table maps the numbered logical blocks 0, 1,
2 to positions in memory).
"""

from __future__ import annotations

import numpy as np


def _f64(x):
    """Exact float64 values of ``x``; ``uint16`` arrays are bfloat16 bit patterns."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def gather_kv(k_pool, v_pool, block_table, seq_len, kv_head):
    """Return the contiguous ``(K, V)`` of one sequence and one KV head.

    ``k_pool``/``v_pool``: ``[num_blocks, block_size, Hkv, D]``.
    ``block_table``: 1-D logical→physical block ids of this sequence.
    Returns two float64 arrays of shape ``[seq_len, D]``; row ``t`` is token
    ``t`` read from block ``block_table[t // block_size]``, offset
    ``t % block_size``.
    """
    block_size = k_pool.shape[1]
    D = k_pool.shape[3]
    K = np.zeros((seq_len, D), dtype=np.float64)
    V = np.zeros((seq_len, D), dtype=np.float64)
    for t in range(seq_len):
        phys = int(block_table[t // block_size])
        off = t % block_size
        K[t] = _f64(k_pool[phys, off, kv_head])
        V[t] = _f64(v_pool[phys, off, kv_head])
    return K, V


def ref_decode(q, k_pool, v_pool, block_tables, seq_lens, scale):
    """Decode attention for every (sequence, query head), in float64.

    q            ``[B, Hq, D]`` float, or uint16 holding bfloat16 bit patterns
                 (values are taken exactly in either case; same for the pools)
    k_pool       ``[num_blocks, block_size, Hkv, D]``
    v_pool       same shape as ``k_pool``
    block_tables ``[B, max_blocks]`` integer
    seq_lens     ``[B]`` integer
    scale        float multiplying ``q·k``
    returns      ``[B, Hq, D]`` float64

    For each ``b`` and ``h`` with ``g = h // (Hq // Hkv)`` and ``L = seq_lens[b]``:
    ``s_t = scale * q[b,h]·K[t]``, ``p = softmax(s)``, ``out[b,h] = Σ_t p_t V[t]``
    over ``t < L``.
    """
    B, Hq, D = q.shape
    Hkv = k_pool.shape[2]
    assert Hq % Hkv == 0, "query heads must be a multiple of KV heads"
    group = Hq // Hkv
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        L = int(seq_lens[b])
        if L == 0:
            continue
        for g in range(Hkv):
            K, V = gather_kv(k_pool, v_pool, block_tables[b], L, g)
            for h in range(g * group, (g + 1) * group):
                qh = _f64(q[b, h])
                s = float(scale) * (K @ qh)
                s = s - s.max()
                w = np.exp(s)
                p = w / w.sum()
                out[b, h] = p @ V
    return out
