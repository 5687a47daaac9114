"""Pins for the oracle (CPU only).

Each test checks the oracle against something other than itself: values the
pages print (tests/golden/), brute-force loops written independently, closed
forms, invariants and a library attention routine.  The planted-mistake test
at the end shows that plausible mistakes in the oracle fail these pins.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import (RefAllocator, OutOfBlocks, gather_kv, ref_copy_blocks, ref_decode,
                    ref_reshape_and_cache, splitmix64_stream)
from oracle import decode as oracle_decode

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------
# Worked example: block size 4, ten tokens, table 0→5, 1→12, 2→3
# ----------------------------------------------------------------------------

def _worked_example_allocator(ex):
    table = [ex["block_table"][str(i)] for i in range(len(ex["block_table"]))]
    rest = [b for b in range(16) if b not in table]
    return RefAllocator(16, ex["block_size"], pop_order=table + rest), table


def test_worked_example_on_demand_blocks_and_table():
    ex = load("worked_example.json")
    bs = ex["block_size"]
    alloc, table = _worked_example_allocator(ex)
    alloc.add_seq(0, 0)
    nblocks_seen = []
    slots = []
    for _ in ex["tokens"]:
        slot, src, dst = alloc.append_slot(0)
        assert (src, dst) == (-1, -1)
        slots.append(slot)
        nblocks_seen.append(len(alloc.block_table(0)[0]))
    # a new block is taken only when the previous one is full (steps 1, 2, 3)
    assert nblocks_seen == [1, 1, 1, 1, 2, 2, 2, 2, 3, 3]
    got_table, ntok = alloc.block_table(0)
    assert got_table == table == [5, 12, 3]
    assert ntok == len(ex["tokens"]) == ex["contiguous_used_slots"]
    # paged layout wastes only the 2 empty slots of the last block ...
    assert alloc.internal_waste_slots() == ex["paged_wasted_slots"]
    assert len(got_table) * bs - ntok == ex["paged_wasted_slots"]
    # ... against 6 for the 16-slot contiguous reservation
    assert ex["contiguous_reserved_slots"] - ntok == ex["contiguous_wasted_slots"]

    # write token ids through the slots; the physical blocks must read as the page prints them
    vocab = {tok: i + 1 for i, tok in enumerate(ex["tokens"])}
    pool = np.zeros((16, bs, 1, 1), dtype=np.int64)
    ids = np.array([vocab[t] for t in ex["tokens"]], dtype=np.int64).reshape(-1, 1, 1)
    kp, _ = ref_reshape_and_cache(ids, ids, pool, pool, np.array(slots))
    for logical, words in enumerate(ex["blocks"]):
        phys = ex["block_table"][str(logical)]
        want = [vocab[w] if w is not None else 0 for w in words]
        assert kp[phys, :, 0, 0].tolist() == want


def test_worked_example_gather_order():
    ex = load("worked_example.json")
    bs = ex["block_size"]
    table = np.array([ex["block_table"][str(i)] for i in range(3)] + [-1])
    pool = np.full((16, bs, 1, 1), np.nan)
    # fill the three blocks exactly as the page shows them (empty slots stay NaN)
    vocab = {tok: i + 1 for i, tok in enumerate(ex["tokens"])}
    for logical, words in enumerate(ex["blocks"]):
        for off, w in enumerate(words):
            if w is not None:
                pool[table[logical], off, 0, 0] = vocab[w]
    K, V = gather_kv(pool, pool, table, len(ex["tokens"]), 0)
    assert K[:, 0].tolist() == [float(i + 1) for i in range(10)]
    assert np.all(np.isfinite(V))


# ----------------------------------------------------------------------------
# Sharing diagram: tables [0, 1, 2] and [0, 1, -1, -1]; refcounts; free at 0
# ----------------------------------------------------------------------------

def test_sharing_diagram_refcounts_and_free():
    ex = load("sharing_diagram.json")
    bs = ex["tokens_per_block"]
    alloc = RefAllocator(8, bs)
    alloc.add_seq(1, 2 * bs)      # tokens 1..8 in blocks 0, 1
    alloc.fork(1, 2)              # sequence 2 shares the prefix
    alloc.append_slot(1)          # token 9 of sequence 1 starts block 2
    t1, _ = alloc.block_table(1)
    t2, _ = alloc.block_table(2)
    assert t1 == ex["tables"]["1"]
    assert t2 == [b for b in ex["tables"]["2"] if b >= 0]
    assert [alloc.refcount(b) for b in range(3)] == [2, 2, 1]
    nfree = alloc.num_free()
    alloc.free_seq(1)
    assert [alloc.refcount(b) for b in range(3)] == [1, 1, 0]
    assert alloc.num_free() == nfree + 1
    alloc.free_seq(2)
    assert [alloc.refcount(b) for b in range(3)] == [0, 0, 0]
    assert alloc.num_free() == 8


def test_copy_on_write_rule_n_forks():
    bs = 4
    alloc = RefAllocator(32, bs)
    alloc.add_seq(0, 6)                  # blocks [0, 1]; block 1 holds 2 of 4
    for c in range(1, 4):
        alloc.fork(0, c)
    assert alloc.refcount(1) == 4
    copies = []
    for s in range(4):
        slot, src, dst = alloc.append_slot(s)
        copies.append((src, dst))
        table, ntok = alloc.block_table(s)
        assert ntok == 7
        assert slot == table[-1] * bs + 2
    # the first three writers copy the shared partial block, the last writes in place
    assert [c[0] for c in copies] == [1, 1, 1, -1]
    assert len({c[1] for c in copies[:3]}) == 3
    assert alloc.refcount(1) == 1
    assert alloc.block_table(3)[0] == [0, 1]
    assert alloc.refcount(0) == 4


def test_full_shared_block_needs_no_copy():
    alloc = RefAllocator(8, 4)
    alloc.add_seq(0, 8)
    alloc.fork(0, 1)
    slot, src, dst = alloc.append_slot(0)
    assert (src, dst) == (-1, -1)
    assert alloc.block_table(0)[0] == [0, 1, 2] and slot == 8


def test_out_of_blocks_leaves_state_unchanged():
    alloc = RefAllocator(3, 4)
    alloc.add_seq(0, 6)
    alloc.fork(0, 1)
    alloc.add_seq(2, 4)
    before = (list(alloc.free), list(alloc.ref), {k: list(v) for k, v in alloc.tables.items()},
              dict(alloc.ntok))
    with pytest.raises(OutOfBlocks):
        alloc.append_slot(0)            # needs a copy-on-write block; none free
    with pytest.raises(OutOfBlocks):
        alloc.add_seq(3, 1)
    after = (list(alloc.free), list(alloc.ref), {k: list(v) for k, v in alloc.tables.items()},
             dict(alloc.ntok))
    assert before == after


def test_truncate_releases_tail_blocks_and_rewrites_shared_partial_block():
    alloc = RefAllocator(8, 4)
    alloc.add_seq(0, 10)                 # blocks [0, 1, 2], 2 of 4 used in block 2
    alloc.fork(0, 1)
    alloc.truncate(0, 5)                 # keeps blocks [0, 1]; block 2 still held by 1
    assert alloc.block_table(0) == ([0, 1], 5)
    assert [alloc.refcount(b) for b in range(3)] == [2, 2, 1]
    slot, src, dst = alloc.append_slot(0)   # block 1 is shared and partial: copy on write
    assert src == 1 and slot == dst * 4 + 1
    alloc.truncate(1, 0)                 # all of sequence 1's blocks released
    assert alloc.block_table(1) == ([], 0)
    assert alloc.refcount(2) == 0 and alloc.refcount(0) == 1
    alloc.truncate(0, 4)                 # exactly one block: the copied block goes back
    assert alloc.block_table(0) == ([0], 4) and alloc.refcount(dst) == 0


def test_beam_select_shares_parent_blocks_and_frees_dropped_beams():
    alloc = RefAllocator(16, 4)
    alloc.add_seq(0, 4)                  # prompt in block 0
    for c in (1, 2, 3):
        alloc.fork(0, c)
    for s in range(4):                   # each beam writes its own block 1..4
        alloc.append_slot(s)
    private = [alloc.block_table(s)[0][1] for s in range(4)]
    alloc.beam_select([0, 1, 2, 3], [2, 2, 0, 2])
    for s, p in zip(range(4), [2, 2, 0, 2]):
        assert alloc.block_table(s)[0] == [0, private[p]]
    assert alloc.refcount(0) == 4
    assert alloc.refcount(private[2]) == 3 and alloc.refcount(private[0]) == 1
    assert alloc.refcount(private[1]) == 0 and alloc.refcount(private[3]) == 0
    assert alloc.num_free() == 16 - 3


def test_splitmix64_published_vectors():
    # splitmix64 reference implementation (Vigna, prng.di.unimi.it/splitmix64.c), seed 1234567
    g = splitmix64_stream(1234567)
    assert [next(g) for _ in range(5)] == [6457827717110365317, 3203168211198807973,
                                           9817491932198370423, 4593380528125082431,
                                           16408922859458223821]


def test_shuffled_free_list_is_a_permutation():
    a = RefAllocator(97, 16, shuffle_seed=42)
    order = list(reversed(a.free))
    assert sorted(order) == list(range(97)) and order != list(range(97))
    assert list(reversed(RefAllocator(97, 16).free)) == list(range(97))


# ----------------------------------------------------------------------------
# Decode attention: brute force, library cross-check, closed forms, invariants
# ----------------------------------------------------------------------------

def _random_case(rng, B=3, Hq=4, Hkv=2, D=8, bs=4, lens=(5, 9, 1), NB=12):
    q = rng.standard_normal((B, Hq, D))
    kp = rng.standard_normal((NB, bs, Hkv, D))
    vp = rng.standard_normal((NB, bs, Hkv, D))
    perm = rng.permutation(NB)
    MB = max(-(-L // bs) for L in lens) + 1
    tables = np.full((B, MB), -1, dtype=np.int64)
    k = 0
    for b, L in enumerate(lens):
        n = -(-L // bs)
        tables[b, :n] = perm[k:k + n]
        k += n
    return q, kp, vp, tables, np.array(lens), 0.37


def brute_force(q, kp, vp, tables, lens, scale):
    """Literal double loop over tokens with math.exp; K/V addressed through the table."""
    B, Hq, D = q.shape
    bs, Hkv = kp.shape[1], kp.shape[2]
    G = Hq // Hkv
    out = [[[0.0] * D for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        L = int(lens[b])
        for h in range(Hq):
            kvh = h // G
            logits = []
            for t in range(L):
                blk = int(tables[b][t // bs])
                logits.append(scale * sum(q[b][h][d] * kp[blk][t % bs][kvh][d] for d in range(D)))
            if not logits:
                continue
            mx = max(logits)
            w = [math.exp(x - mx) for x in logits]
            z = sum(w)
            for d in range(D):
                out[b][h][d] = sum(w[t] * vp[int(tables[b][t // bs])][t % bs][kvh][d]
                                   for t in range(L)) / z
    return np.array(out)


def test_decode_matches_brute_force():
    rng = np.random.default_rng(0)
    case = _random_case(rng)
    np.testing.assert_allclose(ref_decode(*case), brute_force(*case), rtol=0, atol=1e-12)


def test_decode_matches_library_sdpa():
    rng = np.random.default_rng(1)
    q, kp, vp, tables, lens, scale = _random_case(rng, B=4, Hq=8, Hkv=2, D=16, bs=4,
                                                  lens=(13, 4, 7, 16), NB=20)
    out = ref_decode(q, kp, vp, tables, lens, scale)
    bs, G = kp.shape[1], q.shape[1] // kp.shape[2]
    for b, L in enumerate(lens):
        t = np.arange(L)
        phys = tables[b][t // bs]
        K = torch.from_numpy(kp[phys, t % bs])          # [L, Hkv, D] (numpy fancy gather)
        V = torch.from_numpy(vp[phys, t % bs])
        K = K.repeat_interleave(G, dim=1).permute(1, 0, 2)   # [Hq, L, D]
        V = V.repeat_interleave(G, dim=1).permute(1, 0, 2)
        Q = torch.from_numpy(q[b]).unsqueeze(1)               # [Hq, 1, D]
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=scale)
        np.testing.assert_allclose(out[b], ref[:, 0].numpy(), rtol=0, atol=1e-12)


def test_single_token_returns_its_value():
    rng = np.random.default_rng(2)
    q, kp, vp, tables, lens, scale = _random_case(rng, lens=(1, 1, 1))
    out = ref_decode(q, kp, vp, tables, lens, scale)
    for b in range(3):
        for h in range(4):
            assert np.array_equal(out[b, h], vp[tables[b, 0], 0, h // 2])


def test_zero_query_or_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(3)
    q, kp, vp, tables, lens, scale = _random_case(rng, lens=(5, 9, 3))
    bs = kp.shape[1]
    mean = lambda b, g: np.mean([vp[tables[b][t // bs], t % bs, g] for t in range(lens[b])], axis=0)
    out = ref_decode(np.zeros_like(q), kp, vp, tables, lens, scale)
    for b in range(3):
        for h in range(4):
            np.testing.assert_allclose(out[b, h], mean(b, h // 2), atol=1e-13)
    kp_eq = np.broadcast_to(kp[:1, :1], kp.shape).copy()   # every key identical
    out = ref_decode(q, kp_eq, vp, tables, lens, scale)
    for b in range(3):
        for h in range(4):
            np.testing.assert_allclose(out[b, h], mean(b, h // 2), atol=1e-13)


def test_dominant_logit_and_huge_scale_select_that_value():
    rng = np.random.default_rng(4)
    q, kp, vp, tables, lens, _ = _random_case(rng, B=1, Hq=2, Hkv=1, lens=(9,))
    bs = kp.shape[1]
    j = 6
    target = kp[tables[0][j // bs], j % bs, 0]
    q[0, :] = target            # q·k_j = |k_j|^2 is the largest logit by a margin for this draw
    logits = [q[0, 0] @ kp[tables[0][t // bs], t % bs, 0] for t in range(9)]
    assert int(np.argmax(logits)) == j
    out = ref_decode(q, kp, vp, tables, lens, 1e4)   # exp of raw logits would overflow
    assert np.all(np.isfinite(out))
    np.testing.assert_array_equal(out[0, 0], vp[tables[0][j // bs], j % bs, 0])


def test_empty_sequence_gives_zeros_and_tails_are_never_read():
    rng = np.random.default_rng(5)
    q, kp, vp, tables, lens, scale = _random_case(rng, lens=(6, 0, 3))
    base = ref_decode(q, kp, vp, tables, lens, scale)
    assert np.array_equal(base[1], np.zeros_like(base[1]))
    kp2, vp2 = kp.copy(), vp.copy()
    bs = kp.shape[1]
    for b, L in enumerate(lens):
        used = -(-L // bs)
        if used:
            last = tables[b][used - 1]
            kp2[last, (L - 1) % bs + 1:] = np.nan      # unused slots of the last block
            vp2[last, (L - 1) % bs + 1:] = np.inf
    np.testing.assert_array_equal(ref_decode(q, kp2, vp2, tables, lens, scale), base)


def test_gqa_head_mapping_consecutive_groups():
    rng = np.random.default_rng(6)
    q, kp, vp, tables, lens, scale = _random_case(rng, B=2, Hq=6, Hkv=3, lens=(5, 7))
    vp2 = vp.copy()
    vp2[:, :, 2] = np.nan       # KV head 2 serves only query heads 4 and 5
    out = ref_decode(q, kp, vp2, tables, lens, scale)
    assert np.all(np.isfinite(out[:, :4])) and np.all(np.isnan(out[:, 4:]))


def test_block_placement_permutation_invariant():
    rng = np.random.default_rng(7)
    q, kp, vp, tables, lens, scale = _random_case(rng, lens=(5, 9, 2))
    NB = kp.shape[0]
    perm = rng.permutation(NB)                  # physical block i moves to perm[i]
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp
    tables2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1)
    np.testing.assert_array_equal(ref_decode(q, kp2, vp2, tables2, lens, scale),
                                  ref_decode(q, kp, vp, tables, lens, scale))


def test_shared_prefix_equals_duplicated_private_copies():
    rng = np.random.default_rng(8)
    bs, D = 4, 8
    kp = rng.standard_normal((10, bs, 1, D))
    vp = rng.standard_normal((10, bs, 1, D))
    q = rng.standard_normal((2, 2, D))
    lens = np.array([10, 11])
    shared = np.array([[0, 1, 2], [0, 1, 3]])           # blocks 0, 1 shared
    kd, vd = kp.copy(), vp.copy()
    kd[4], kd[5], vd[4], vd[5] = kp[0], kp[1], vp[0], vp[1]
    dup = np.array([[0, 1, 2], [4, 5, 3]])              # sequence 1 owns private copies
    np.testing.assert_array_equal(ref_decode(q, kp, vp, shared, lens, 0.3),
                                  ref_decode(q, kd, vd, dup, lens, 0.3))


def test_copy_on_write_then_write_leaves_sibling_unchanged():
    rng = np.random.default_rng(9)
    bs, Hkv, D = 4, 2, 8
    NB = 8
    kp = rng.standard_normal((NB, bs, Hkv, D))
    vp = rng.standard_normal((NB, bs, Hkv, D))
    alloc = RefAllocator(NB, bs, shuffle_seed=3)
    alloc.add_seq(0, 6)
    alloc.fork(0, 1)
    q = rng.standard_normal((1, 4, D))

    def decode(seq, k, v):
        t, n = alloc.block_table(seq)
        return ref_decode(q, k, v, np.array([t]), np.array([n]), 0.25)

    before = decode(1, kp, vp)
    slot, src, dst = alloc.append_slot(0)        # sequence 0 diverges
    assert src >= 0
    kp, vp = ref_copy_blocks(kp, vp, [(src, dst)])
    kp, vp = ref_reshape_and_cache(rng.standard_normal((1, Hkv, D)), rng.standard_normal((1, Hkv, D)),
                                   kp, vp, np.array([slot]))
    np.testing.assert_array_equal(decode(1, kp, vp), before)
    # and the writer sees its copy of the prefix plus the new token
    t0, n0 = alloc.block_table(0)
    assert n0 == 7 and t0[-1] == dst and slot == dst * bs + 2


def test_bf16_bit_patterns_are_read_exactly():
    x = np.array([1.0, -2.5, 3.140625, 0.0078125], dtype=np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)      # exactly representable values
    np.testing.assert_array_equal(oracle_decode._f64(bits), x.astype(np.float64))


# ----------------------------------------------------------------------------
# Cache ops
# ----------------------------------------------------------------------------

def test_reshape_and_cache_literal_and_skip():
    rng = np.random.default_rng(10)
    kp = rng.standard_normal((4, 4, 2, 3))
    vp = rng.standard_normal((4, 4, 2, 3))
    key = rng.standard_normal((3, 2, 3))
    val = rng.standard_normal((3, 2, 3))
    k2, v2 = ref_reshape_and_cache(key, val, kp, vp, np.array([13, -1, 2]))
    exp_k, exp_v = kp.copy(), vp.copy()
    exp_k[3, 1], exp_v[3, 1] = key[0], val[0]       # slot 13 = block 3, offset 1
    exp_k[0, 2], exp_v[0, 2] = key[2], val[2]       # slot 2 = block 0, offset 2
    np.testing.assert_array_equal(k2, exp_k)
    np.testing.assert_array_equal(v2, exp_v)


def test_copy_blocks_whole_block_only_dst_changes():
    rng = np.random.default_rng(11)
    kp = rng.standard_normal((6, 4, 2, 3))
    vp = rng.standard_normal((6, 4, 2, 3))
    k2, v2 = ref_copy_blocks(kp, vp, [(1, 4), (2, 5)])
    for b in range(6):
        src = {4: 1, 5: 2}.get(b, b)
        np.testing.assert_array_equal(k2[b], kp[src])
        np.testing.assert_array_equal(v2[b], vp[src])


# ----------------------------------------------------------------------------
# Planted mistakes: each plausible oracle bug must fail at least one pin
# ----------------------------------------------------------------------------

def _mutant_decode(kind):
    def f(q, kp, vp, tables, lens, scale):
        B, Hq, D = q.shape
        bs, Hkv = kp.shape[1], kp.shape[2]
        G = Hq // Hkv
        out = np.zeros((B, Hq, D))
        for b in range(B):
            L = int(lens[b])
            if L == 0:
                continue
            for h in range(Hq):
                g = (h % Hkv) if kind == "head_mod" else h // G
                t = np.arange(L)
                blk = (t // bs + 1) if kind == "off_by_one" else t // bs
                blk = np.minimum(blk, tables.shape[1] - 1)
                phys = tables[b][blk]
                K, V = kp[phys, t % bs, g], vp[phys, t % bs, g]
                s = (K @ q[b, h]) * (1.0 if kind == "no_scale" else scale)
                if kind == "wrong_sign":
                    s = -s
                p = np.exp(s - s.max())
                p = p / (p.sum() if kind != "no_norm" else 1.0)
                out[b, h] = (p @ K) if kind == "k_for_v" else (p @ V)
        return out
    return f


@pytest.mark.parametrize("kind", ["head_mod", "off_by_one", "no_scale", "wrong_sign", "no_norm",
                                  "k_for_v"])
def test_planted_mistakes_fail_brute_force(kind):
    rng = np.random.default_rng(12)
    case = _random_case(rng)
    bad = _mutant_decode(kind)(*case)
    assert not np.allclose(bad, brute_force(*case), atol=1e-6)
    # the same structure without a mutation passes
    np.testing.assert_allclose(_mutant_decode("none")(*case), brute_force(*case), atol=1e-12)
