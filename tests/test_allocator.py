"""CPU: the C allocator (pa_alloc_*) against oracle.RefAllocator, state compared
bit-exactly (free stack order, refcounts, tables, token counts)."""

import numpy as np
import pytest

import workloads
from oracle import OutOfBlocks, RefAllocator


def _alloc(*a, **k):
    from paged_kv_cache_350_b200 import Allocator
    return Allocator(*a, **k)


def state(a, seqs, nb):
    tables = {s: (a.block_table(s), [int(x) for x in a.seq_slots(s)]) for s in sorted(seqs)}
    refs = [a.refcount(b) for b in range(nb)]
    free = a.free_list() if hasattr(a, "free_list") else None
    return tables, refs, free, a.num_free(), a.internal_waste_slots()


def ref_state(r, seqs, nb):
    tables = {s: (r.block_table(s), r.seq_slots(s)) for s in sorted(seqs)}
    return tables, [r.refcount(b) for b in range(nb)], list(r.free), r.num_free(), \
        r.internal_waste_slots()


@pytest.mark.parametrize("seed", range(12))
def test_random_op_sequences_bit_exact(seed):
    from paged_kv_cache_350_b200 import PAError
    rng = np.random.default_rng(seed)
    nb, bs = int(rng.integers(8, 64)), int(rng.choice([4, 8, 16]))
    shuffle = int(rng.integers(0, 2**63)) if seed % 2 else 0
    c = _alloc(nb, bs, shuffle_seed=shuffle)
    r = RefAllocator(nb, bs, shuffle_seed=shuffle)
    live = set()
    next_id = 0
    for _ in range(300):
        op = rng.choice(["add", "fork", "append", "append", "append", "free", "truncate", "select"])
        c_exc = r_exc = None
        if op == "add" or not live:
            sid, n = next_id, int(rng.integers(0, 3 * bs))
            next_id += 1
            try:
                c.add_seq(sid, n)
            except PAError as e:
                c_exc = e.status
            try:
                r.add_seq(sid, n)
                live.add(sid)
            except OutOfBlocks:
                r_exc = 3
        elif op == "fork":
            parent = int(rng.choice(sorted(live)))
            sid = next_id
            next_id += 1
            c.fork(parent, sid)
            r.fork(parent, sid)
            live.add(sid)
        elif op == "append":
            sid = int(rng.choice(sorted(live)))
            try:
                cres = c.append_slot(sid)
            except PAError as e:
                c_exc, cres = e.status, None
            try:
                rres = r.append_slot(sid)
            except OutOfBlocks:
                r_exc, rres = 3, None
            assert cres == rres
        elif op == "truncate":
            sid = int(rng.choice(sorted(live)))
            n = int(rng.integers(0, r.ntok[sid] + 1))
            c.truncate(sid, n)
            r.truncate(sid, n)
        elif op == "select":
            beams = [int(x) for x in rng.choice(sorted(live), size=min(len(live), 4), replace=False)]
            parents = [int(x) for x in rng.integers(0, len(beams), size=len(beams))]
            c.beam_select(beams, parents)
            r.beam_select(beams, parents)
        else:
            sid = int(rng.choice(sorted(live)))
            c.free_seq(sid)
            r.free_seq(sid)
            live.discard(sid)
        assert c_exc == r_exc
        assert state(c, live, nb) == ref_state(r, live, nb)


def test_worked_example_through_the_c_allocator():
    order = [5, 12, 3] + [b for b in range(16) if b not in (5, 12, 3)]
    c = _alloc(16, 4, pop_order=order)
    c.add_seq(0, 0)
    slots = [c.append_slot(0)[0] for _ in range(10)]
    r = RefAllocator(16, 4, pop_order=order)
    r.add_seq(0, 0)
    assert slots == [r.append_slot(0)[0] for _ in range(10)]
    assert c.block_table(0) == ([5, 12, 3], 10) and c.internal_waste_slots() == 2


def test_batched_append_matches_sequential_and_is_all_or_nothing():
    from paged_kv_cache_350_b200 import PAError
    w = workloads.prefix_cow(prompts=3, prompt_len=40)
    c = _alloc(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed)
    r = RefAllocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed)
    workloads.run_setup(w, c)
    workloads.run_setup(w, r)
    slots, pairs = c.append_slots(w.step_seqs)
    ref_slots, ref_pairs, ref_tables, ref_lens = workloads.run_step_allocation(w, r)
    assert slots.tolist() == ref_slots.tolist() and pairs.tolist() == ref_pairs.tolist()
    tables, lens = c.block_tables(w.step_seqs, w.max_blocks)
    assert np.array_equal(tables, ref_tables) and np.array_equal(lens, ref_lens)
    # out of blocks in the middle of a batch: nothing changes
    small = _alloc(4, 4)
    small.add_seq(0, 4)
    small.add_seq(1, 4)
    small.add_seq(2, 4)
    before = state(small, {0, 1, 2}, 4)
    with pytest.raises(PAError) as e:
        small.append_slots([0, 1, 2])        # needs 3 fresh blocks, 1 free
    assert e.value.status == 3 and state(small, {0, 1, 2}, 4) == before
    with pytest.raises(PAError):
        small.append_slots([0, 0])           # duplicate id
    with pytest.raises(PAError):
        small.append_slots([0, 99])          # unknown id
    assert state(small, {0, 1, 2}, 4) == before


def test_errors_leave_state_unchanged():
    from paged_kv_cache_350_b200 import PAError
    c = _alloc(3, 4)
    c.add_seq(0, 6)
    c.fork(0, 1)
    c.add_seq(2, 4)
    before = state(c, {0, 1, 2}, 3)
    for f, args in ((c.append_slot, (0,)), (c.add_seq, (3, 1)), (c.add_seq, (0, 1)),
                    (c.fork, (9, 10)), (c.fork, (0, 2)), (c.free_seq, (42,))):
        with pytest.raises(PAError):
            f(*args)
    assert state(c, {0, 1, 2}, 3) == before
    with pytest.raises(PAError):
        _alloc(4, 4, pop_order=[0, 1, 1, 2])


def test_truncate_and_beam_select_reject_bad_arguments_without_change():
    from paged_kv_cache_350_b200 import PAError
    c = _alloc(16, 4)
    c.add_seq(0, 6)
    c.add_seq(1, 3)
    before = state(c, {0, 1}, 16)
    for f, args in ((c.truncate, (0, 7)), (c.truncate, (0, -1)), (c.truncate, (9, 0)),
                    (c.beam_select, ([0, 1], [0, 2])), (c.beam_select, ([0, 0], [0, 0])),
                    (c.beam_select, ([0, 5], [0, 0]))):
        with pytest.raises(PAError):
            f(*args)
    assert state(c, {0, 1}, 16) == before
