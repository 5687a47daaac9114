"""CPU: the all-cores oracle runner gives exactly the single-call oracle's output.

tests/_oracle_pool.py cuts a batch into (row, KV head) items for spawned workers; the
full-size GPU parity test relies on it computing the same float64 values as one
oracle.ref_decode call over the batch.
"""

import numpy as np

import workloads
from _oracle_pool import decode_all_rows
from oracle import ref_decode


def test_all_cores_runner_equals_one_oracle_call():
    w = workloads.gqa(B=7, median=40, lo=1, hi=90, seed=77)
    from oracle import RefAllocator
    alloc = RefAllocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed)
    workloads.run_setup(w, alloc)
    _, _, tables, lens = workloads.run_step_allocation(w, alloc)
    lens = lens.copy()
    lens[3] = 0  # an empty row stays zero
    args = (w.q(), w.k_pool(), w.v_pool(), tables, lens, w.scale)
    want = ref_decode(*args)
    got = decode_all_rows(*args, workers=2)
    assert np.array_equal(got, want)
