"""Seeded synthetic inputs for the paged decode-attention path.

Shared by the tests, ``bench.py`` and the oracle's callers.  This module holds
NONE of the method's arithmetic: it draws shapes, lengths, random values and
an allocator op script, and nothing else.  Slot mappings, block tables and
copy-on-write pairs are produced by running the script through an allocator
(the C library's on the product side, ``oracle.RefAllocator`` on the oracle
side); attention outputs come from the kernels or the oracle.

Value recipe (every workload):

* q, K, V ~ N(0, 1): drawn as float32 by ``numpy.random.PCG64`` and rounded
  to bfloat16 (round to nearest, ties to even) for bf16 workloads, so the GPU
  and the oracle see identical values.  Pools are drawn whole, so the unused
  slots of a block hold random values too.
* Pools are drawn in fixed chunks of ``2**22`` elements, chunk ``i`` from
  ``SeedSequence(seed, spawn_key=(stream, i))``: the draw does not depend on
  the number of threads.
* Physical blocks come from the allocator's seeded free-list permutation
  (``alloc_seed``); the pool holds the blocks the workload needs plus 10 % free.

Workloads (the serving shapes the PagedAttention pages motivate):

* ``tiny``        fp32, B=2, Hq=Hkv=4, D=64, block_size=4, 16 blocks, decode
                  lengths 10 and 7; the step writes one token per sequence and
                  copies one shared partial block (sequence 1 was forked).
* ``mha``         bf16 Llama-7B-shaped: B=64, Hq=Hkv=32, D=128, bs=16,
                  lengths U[128, 2048].
* ``gqa``         bf16 Llama-3-8B-shaped: B=256, Hq=32, Hkv=8, D=128, bs=16,
                  lengths log-normal (median 1024, sigma 0.6) clipped [64, 4096].
* ``prefix``      bf16 parallel sampling: 32 prompts of 1024 tokens, each
                  forked into 8 samples with U{0..256} private tokens.
* ``prefix_cow``  as ``prefix`` but 1000-token prompts and the step is the
                  first divergence: 7 of every 8 forks copy the shared partial
                  last prompt block (224 copy pairs).
* ``long``        bf16 long context: B=8, Hq=64, Hkv=8, D=128, bs=16,
                  lengths U[32768, 131072].

Each builder takes size overrides so the tests can run scaled-down versions
with the same structure.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

CHUNK = 1 << 22

# Op script entries (executed by each side's allocator):
#   ("add", seq_id, num_tokens)   register a sequence already holding num_tokens
#   ("fork", parent_id, child_id) child shares all of parent's blocks
#   ("append", seq_id, count)     append count tokens (setup only; no K/V written)


@dataclass
class Workload:
    name: str
    dtype: str                 # "f32" or "bf16"
    B: int
    Hq: int
    Hkv: int
    D: int
    block_size: int
    num_blocks: int
    scale: float
    alloc_seed: int            # allocator free-list shuffle seed
    setup_ops: list            # op script run before the step
    step_seqs: list            # the batch: one sequence id per row, in order
    seed: int
    pop_order: list | None = None   # explicit free-list pop order (overrides alloc_seed)
    max_blocks: int = 0        # block-table width (>= blocks of the longest sequence after the step)
    meta: dict = field(default_factory=dict)
    _cache: dict = field(default_factory=dict, repr=False)

    # ---- random tensors (lazily drawn, cached) ------------------------------
    def _draw(self, key, shape, stream):
        if key not in self._cache:
            self._cache[key] = draw_normal(shape, self.seed, stream, self.dtype)
        return self._cache[key]

    @property
    def pool_shape(self):
        return (self.num_blocks, self.block_size, self.Hkv, self.D)

    def k_pool(self):
        """Initial key pool; uint16 bf16 bit patterns or float32."""
        return self._draw("k_pool", self.pool_shape, 1)

    def v_pool(self):
        return self._draw("v_pool", self.pool_shape, 2)

    def q(self):
        return self._draw("q", (self.B, self.Hq, self.D), 3)

    def new_k(self):
        """The step's new key row per batch entry, ``[B, Hkv, D]``."""
        return self._draw("new_k", (self.B, self.Hkv, self.D), 4)

    def new_v(self):
        return self._draw("new_v", (self.B, self.Hkv, self.D), 5)


def _round_bf16_bits(x):
    """float32 → bfloat16 bit patterns, round to nearest, ties to even."""
    u = x.view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits):
    """bfloat16 bit patterns (uint16) → exactly equal float32 values."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def draw_normal(shape, seed, stream, dtype):
    """N(0,1) array of ``shape``; uint16 bf16 bits for ``bf16``, float32 for ``f32``."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16 if dtype == "bf16" else np.float32)
    nchunks = max(1, -(-n // CHUNK))

    def fill(i):
        lo, hi = i * CHUNK, min(n, (i + 1) * CHUNK)
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(stream, i))))
        x = rng.standard_normal(hi - lo, dtype=np.float32)
        out[lo:hi] = _round_bf16_bits(x) if dtype == "bf16" else x

    if nchunks == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(min(nchunks, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(nchunks)))
    return out.reshape(shape)


def _blocks(ntok, bs):
    return -(-ntok // bs)


# ---- builders ----------------------------------------------------------------

def tiny(seed=1000, worked_example=False):
    """fp32, two sequences (decode lengths 10 and 7), 16 blocks of 4 tokens.

    Setup: sequence 0 holds 9 tokens, sequence 1 holds 6 and is forked into
    sequence 2, so sequence 1's last block (2 of 4 slots used) is shared.  The
    step appends one token to sequences 0 and 1: sequence 1's append copies
    the shared partial block first.  With ``worked_example`` the free list pops
    5, 12, 3 first, so sequence 0 gets the worked example's table 0→5, 1→12,
    2→3 and its 10 tokens leave 2 slots empty.
    """
    pop_order = None
    if worked_example:
        rest = [b for b in range(16) if b not in (5, 12, 3)]
        pop_order = [5, 12, 3] + rest
    return Workload(
        name="tiny" + ("_worked_example" if worked_example else ""),
        dtype="f32", B=2, Hq=4, Hkv=4, D=64, block_size=4, num_blocks=16,
        scale=1.0 / math.sqrt(64), alloc_seed=seed,
        setup_ops=[("add", 0, 9), ("add", 1, 6), ("fork", 1, 2)],
        step_seqs=[0, 1], seed=seed, pop_order=pop_order, max_blocks=4,
        meta={"decode_lens": [10, 7]},
    )


def _independent(name, seed, dtype, B, Hq, Hkv, D, bs, lens_after, max_blocks=None):
    """B independent sequences; sequence b holds lens_after[b]-1 tokens before the step."""
    lens_after = [int(x) for x in lens_after]
    need = sum(_blocks(L, bs) for L in lens_after)
    nb = max(1, math.ceil(1.1 * need))
    mb = max_blocks or max(1, max(_blocks(L, bs) for L in lens_after))
    return Workload(
        name=name, dtype=dtype, B=B, Hq=Hq, Hkv=Hkv, D=D, block_size=bs, num_blocks=nb,
        scale=1.0 / math.sqrt(D), alloc_seed=seed,
        setup_ops=[("add", b, L - 1) for b, L in enumerate(lens_after)],
        step_seqs=list(range(B)), seed=seed, max_blocks=mb,
        meta={"decode_lens": lens_after},
    )


def independent(lens_after, seed=2000, Hq=8, Hkv=2, D=128, bs=16, dtype="bf16", max_blocks=None,
                name="explicit"):
    """Independent sequences with the given decode lengths (each >= 1)."""
    return _independent(name, seed, dtype, len(lens_after), Hq, Hkv, D, bs, lens_after, max_blocks)


def mha(seed=1001, B=64, lo=128, hi=2048, Hq=32, D=128, bs=16, dtype="bf16"):
    """Llama-7B-shaped MHA decode: lengths uniform in [lo, hi]."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(lo, hi + 1, size=B)
    return _independent("mha", seed, dtype, B, Hq, Hq, D, bs, lens)


def gqa(seed=1002, B=256, median=1024, sigma=0.6, lo=64, hi=4096, Hq=32, Hkv=8, D=128, bs=16,
        dtype="bf16"):
    """Llama-3-8B-shaped GQA decode: log-normal lengths (median, sigma) clipped to [lo, hi]."""
    rng = np.random.default_rng(seed)
    lens = np.clip(np.rint(rng.lognormal(math.log(median), sigma, size=B)), lo, hi).astype(np.int64)
    return _independent("gqa", seed, dtype, B, Hq, Hkv, D, bs, lens)


def long_context(seed=1004, B=8, lo=32768, hi=131072, Hq=64, Hkv=8, D=128, bs=16, dtype="bf16"):
    """Long-context GQA decode: lengths uniform in [lo, hi]."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(lo, hi + 1, size=B)
    return _independent("long", seed, dtype, B, Hq, Hkv, D, bs, lens)


def prefix(seed=1003, prompts=32, n=8, prompt_len=1024, max_private=256, Hq=32, Hkv=8, D=128,
           bs=16, dtype="bf16", first_divergence=False):
    """Parallel sampling: each prompt forked into ``n`` samples sharing the prompt blocks.

    Default: every sample holds U{0..max_private} private tokens before the
    step.  ``first_divergence``: no private tokens; the step is every sample's
    first own token, so a partial last prompt block gets copied on write.
    """
    rng = np.random.default_rng(seed)
    ops = []
    seqs = []
    need = 0
    max_tok = 0
    for p in range(prompts):
        parent = p * n
        ops.append(("add", parent, prompt_len))
        need += _blocks(prompt_len, bs)
        for k in range(1, n):
            ops.append(("fork", parent, parent + k))
        for k in range(n):
            sid = parent + k
            priv = 0 if first_divergence else int(rng.integers(0, max_private + 1))
            if priv:
                ops.append(("append", sid, priv))
            seqs.append(sid)
            total = prompt_len + priv + 1
            max_tok = max(max_tok, total)
            # private blocks of this sample (upper bound, counting a copied partial block)
            need += _blocks(total, bs) - (prompt_len // bs)
    nb = max(1, math.ceil(1.1 * need))
    name = "prefix_cow" if first_divergence else "prefix"
    return Workload(
        name=name, dtype=dtype, B=prompts * n, Hq=Hq, Hkv=Hkv, D=D, block_size=bs,
        num_blocks=nb, scale=1.0 / math.sqrt(D), alloc_seed=seed, setup_ops=ops,
        step_seqs=seqs, seed=seed, max_blocks=_blocks(max_tok, bs),
        meta={"prompts": prompts, "n": n, "prompt_len": prompt_len},
    )


def families(seed=1021, sizes=(16, 3, 6, 1, 9), solo=3, prompt_len=140, max_private=70,
             Hq=32, Hkv=8, D=128, bs=16, dtype="bf16"):
    """Fork families of mixed sizes (each prompt forked into ``sizes[i]`` samples holding
    U{0..max_private} private tokens) and ``solo`` unforked sequences of U{1..300} tokens,
    in one batch: units of different row counts meet in one launch."""
    rng = np.random.default_rng(seed)
    ops, seqs = [], []
    need, max_tok, sid = 0, 0, 0
    for n in sizes:
        parent = sid
        ops.append(("add", parent, prompt_len))
        need += _blocks(prompt_len, bs)
        for k in range(1, n):
            ops.append(("fork", parent, parent + k))
        for k in range(n):
            priv = int(rng.integers(0, max_private + 1))
            if priv:
                ops.append(("append", parent + k, priv))
            seqs.append(parent + k)
            total = prompt_len + priv + 1
            max_tok = max(max_tok, total)
            need += _blocks(total, bs) - (prompt_len // bs)
        sid += n
    for _ in range(solo):
        L = int(rng.integers(1, 301))
        ops.append(("add", sid, L - 1))
        seqs.append(sid)
        need += _blocks(L, bs)
        max_tok = max(max_tok, L)
        sid += 1
    nb = max(1, math.ceil(1.1 * need))
    return Workload(
        name="families", dtype=dtype, B=len(seqs), Hq=Hq, Hkv=Hkv, D=D, block_size=bs,
        num_blocks=nb, scale=1.0 / math.sqrt(D), alloc_seed=seed, setup_ops=ops,
        step_seqs=seqs, seed=seed, max_blocks=_blocks(max_tok, bs),
        meta={"sizes": list(sizes), "solo": solo, "prompt_len": prompt_len},
    )


def prefix_cow(seed=1013, prompts=32, n=8, prompt_len=1000, **kw):
    return prefix(seed=seed, prompts=prompts, n=n, prompt_len=prompt_len, first_divergence=True, **kw)


BUILDERS = {
    "tiny": tiny,
    "mha": mha,
    "gqa": gqa,
    "prefix": prefix,
    "prefix_cow": prefix_cow,
    "long": long_context,
}


def build(name, **overrides):
    return BUILDERS[name](**overrides)


# ---- running the op script through an allocator --------------------------------
# ``alloc`` is either side's allocator object; both expose add_seq, fork,
# append_slot and block_table with the same meaning.

def run_setup(w, alloc):
    """Execute ``w.setup_ops``; returns the copy pairs the setup produced, in order.

    They are none unless a fork appends into a partial prompt block during setup
    (prompt lengths that are not block multiples); each side then applies them to
    its pools before the step."""
    pairs = []
    for op in w.setup_ops:
        if op[0] == "add":
            alloc.add_seq(op[1], op[2])
        elif op[0] == "fork":
            alloc.fork(op[1], op[2])
        elif op[0] == "append":
            for _ in range(op[2]):
                _, src, dst = alloc.append_slot(op[1])
                if src >= 0:
                    pairs.append((src, dst))
        else:
            raise ValueError(op)
    return pairs


def run_step_allocation(w, alloc):
    """Reserve the step's slot for every batch row, in batch order.

    Returns ``slot_mapping [B] int64``, ``pairs [n, 2] int32`` (copy-on-write
    ``src, dst``), ``block_tables [B, max_blocks] int32`` padded with ``-1`` and
    ``seq_lens [B] int32`` — all read back from the allocator.
    """
    slots = np.empty(w.B, dtype=np.int64)
    pairs = []
    for i, sid in enumerate(w.step_seqs):
        slot, src, dst = alloc.append_slot(sid)
        slots[i] = slot
        if src >= 0:
            pairs.append((src, dst))
    tables = np.full((w.B, w.max_blocks), -1, dtype=np.int32)
    lens = np.empty(w.B, dtype=np.int32)
    for i, sid in enumerate(w.step_seqs):
        table, ntok = alloc.block_table(sid)
        tables[i, : len(table)] = table
        lens[i] = ntok
    return slots, np.asarray(pairs, dtype=np.int32).reshape(-1, 2), tables, lens


# ---- a multi-step serving trace (continuous batching) -----------------------------

@dataclass
class ServingTrace:
    """Per-step events of a serving loop; every live sequence decodes one token per step.

    ``events[t]`` lists ("admit", seq_id, prompt_len), ("fork", parent, child),
    ("retire", seq_id), ("select", beam_ids, parent_indices) and ("truncate", seq_id,
    num_tokens) applied before step t's decode.  The prompt K/V of an admission
    and every step's q / new K / new V are drawn with ``draw_normal`` from ``seed`` and
    the stream numbers ``prompt_stream`` / ``step_stream`` give.
    """
    seed: int
    dtype: str
    Hq: int
    Hkv: int
    D: int
    block_size: int
    num_blocks: int
    scale: float
    alloc_seed: int
    events: list
    max_blocks: int

    def prompt_kv(self, seq_id, n):
        shape = (n, self.Hkv, self.D)
        return (draw_normal(shape, self.seed, 100000 + 2 * seq_id, self.dtype),
                draw_normal(shape, self.seed, 100001 + 2 * seq_id, self.dtype))

    def step_inputs(self, t, B):
        return (draw_normal((B, self.Hq, self.D), self.seed, 200000 + 3 * t, self.dtype),
                draw_normal((B, self.Hkv, self.D), self.seed, 200001 + 3 * t, self.dtype),
                draw_normal((B, self.Hkv, self.D), self.seed, 200002 + 3 * t, self.dtype))

    def pool(self, which):
        shape = (self.num_blocks, self.block_size, self.Hkv, self.D)
        return draw_normal(shape, self.seed, 1 if which == "k" else 2, self.dtype)


def serving_trace(seed=3000, steps=40, start=6, max_live=12, prompt_lo=1, prompt_hi=90,
                  p_admit=0.25, p_retire=0.15, p_fork=0.2, Hq=16, Hkv=2, D=128, bs=16,
                  dtype="bf16", num_blocks=None):
    """Random admissions, forks (parallel sampling) and retirements over ``steps`` steps."""
    rng = np.random.default_rng(seed)
    live = []
    next_id = 0
    events = []
    max_tokens = 0
    tokens = {}
    for t in range(steps):
        ev = []
        n_admit = start if t == 0 else int(rng.random() < p_admit)
        for _ in range(n_admit):
            if len(live) >= max_live:
                break
            n = int(rng.integers(prompt_lo, prompt_hi + 1))
            ev.append(("admit", next_id, n))
            live.append(next_id)
            tokens[next_id] = n
            next_id += 1
        if live and len(live) < max_live and rng.random() < p_fork:
            parent = int(rng.choice(live))
            ev.append(("fork", parent, next_id))
            live.append(next_id)
            tokens[next_id] = tokens[parent]
            next_id += 1
        if len(live) > 1 and rng.random() < p_retire:
            gone = int(rng.choice(live))
            ev.append(("retire", gone))
            live.remove(gone)
        events.append(ev)
        for sid in live:
            tokens[sid] += 1
            max_tokens = max(max_tokens, tokens[sid])
    mb = _blocks(max_tokens, bs) + 1
    nb = num_blocks or (max_live + 2) * mb * 2
    return ServingTrace(seed=seed, dtype=dtype, Hq=Hq, Hkv=Hkv, D=D, block_size=bs,
                        num_blocks=nb, scale=1.0 / math.sqrt(D), alloc_seed=seed + 1,
                        events=events, max_blocks=mb)


def beam_trace(seed=3300, beams=4, steps=30, prompt_len=37, p_select=0.6, p_truncate=0.25,
               Hq=16, Hkv=2, D=128, bs=16, dtype="bf16"):
    """Beam search with speculative rollback: one prompt forked into ``beams`` beams;
    before a step the beams may be re-selected from random parents, and one beam may be
    rolled back by 1-3 tokens (never into the prompt)."""
    rng = np.random.default_rng(seed)
    events = [[("admit", 0, prompt_len)] + [("fork", 0, b) for b in range(1, beams)]]
    ntok = [prompt_len] * beams
    for t in range(1, steps):
        ev = []
        if rng.random() < p_select:
            parents = [int(x) for x in rng.integers(0, beams, size=beams)]
            ev.append(("select", tuple(range(beams)), tuple(parents)))
            ntok = [ntok[p] for p in parents]
        if rng.random() < p_truncate:
            b = int(rng.integers(0, beams))
            n = max(prompt_len, ntok[b] - int(rng.integers(1, 4)))
            ev.append(("truncate", b, n))
            ntok[b] = n
        events.append(ev)
        ntok = [n + 1 for n in ntok]
    ntok = [n + 1 for n in ntok]
    mb = _blocks(prompt_len + steps + 1, bs) + 1
    nb = beams * mb * 3 + 8
    return ServingTrace(seed=seed, dtype=dtype, Hq=Hq, Hkv=Hkv, D=D, block_size=bs,
                        num_blocks=nb, scale=1.0 / math.sqrt(D), alloc_seed=seed + 1,
                        events=events, max_blocks=mb)
