"""Structure of the seeded workloads, run through the oracle's allocator (CPU)."""

import numpy as np

import workloads
from oracle import RefAllocator


def _plan(w):
    alloc = RefAllocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed, pop_order=w.pop_order)
    assert workloads.run_setup(w, alloc) == []
    return alloc, workloads.run_step_allocation(w, alloc)


def test_tiny_step_has_one_copy_and_decode_lengths_10_7():
    w = workloads.tiny()
    alloc, (slots, pairs, tables, lens) = _plan(w)
    assert lens.tolist() == [10, 7] and pairs.shape == (1, 2)
    assert (tables >= -1).all() and slots.dtype == np.int64


def test_tiny_worked_example_table():
    w = workloads.tiny(worked_example=True)
    alloc, (slots, pairs, tables, lens) = _plan(w)
    assert tables[0, :3].tolist() == [5, 12, 3] and lens[0] == 10
    assert slots[0] == 3 * 4 + 1


def test_prefix_refcounts_and_copy_counts():
    w = workloads.prefix(prompts=4)
    alloc = RefAllocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed)
    workloads.run_setup(w, alloc)
    table, _ = alloc.block_table(0)
    assert all(alloc.refcount(b) == 8 for b in table[:64])
    _, pairs, _, lens = workloads.run_step_allocation(w, alloc)
    assert pairs.shape[0] == 0 and lens.min() >= 1025
    w = workloads.prefix_cow()
    _, (_, pairs, _, lens) = _plan(w)
    assert pairs.shape[0] == 32 * 7 and (lens == 1001).all()


def test_families_mixed_sizes():
    """Fork families of the given sizes share their prompt's full blocks (refcount = family
    size); unforked sequences hold blocks of their own; every pool block fits."""
    w = workloads.families()
    sizes, solo, P = w.meta["sizes"], w.meta["solo"], w.meta["prompt_len"]
    assert w.B == sum(sizes) + solo
    alloc = RefAllocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed)
    workloads.run_setup(w, alloc)
    first = 0
    for n in sizes:
        table, _ = alloc.block_table(first)
        assert all(alloc.refcount(b) == n for b in table[:P // w.block_size])
        first += n
    _, pairs, tables, lens = workloads.run_step_allocation(w, alloc)
    assert (lens[:sum(sizes)] >= P + 1).all() and (lens[sum(sizes):] >= 1).all()
    assert tables.shape[1] <= w.max_blocks and alloc.num_free() >= 0


def test_length_distributions():
    w = workloads.gqa()
    L = np.array(w.meta["decode_lens"])
    assert L.min() >= 64 and L.max() <= 4096 and 800 < np.median(L) < 1300
    L = np.array(workloads.mha().meta["decode_lens"])
    assert L.min() >= 128 and L.max() <= 2048
    L = np.array(workloads.long_context().meta["decode_lens"])
    assert L.min() >= 32768 and L.max() <= 131072


def test_draws_are_seeded_and_bf16_exact():
    a = workloads.draw_normal((3, 5_000_000), 7, 1, "bf16")
    b = workloads.draw_normal((3, 5_000_000), 7, 1, "bf16")
    assert a.dtype == np.uint16 and np.array_equal(a, b)
    f = workloads.bf16_bits_to_f32(a[0, :1000])
    assert abs(float(f.std()) - 1.0) < 0.1
