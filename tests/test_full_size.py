"""GPU parity at the full serving sizes, in the launch configuration bench.py times
(automatic path and partitioning, workspace from pa_decode_workspace_size).

Every output row of every serving batch is compared with the float64 oracle.  The oracle
runs on all host cores (tests/_oracle_pool.py), once per batch, and serves both the fused
step (pa_decode_append, the call bench.py times) and the unfused one (pa_reshape_and_cache
+ pa_decode).  The pools after the fused step are compared bit for bit with the oracle's
pools after copy_blocks and reshape_and_cache.
"""

import numpy as np
import pytest
import torch

import workloads
from _oracle_pool import decode_all_rows
from _parity import assert_close, gpu_step, oracle_bits, pool_bits
from oracle import RefAllocator, ref_copy_blocks, ref_reshape_and_cache

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

FULL = {
    "gqa": workloads.gqa,
    "mha": workloads.mha,
    "long": workloads.long_context,
    "prefix": workloads.prefix,
    "prefix_cow": workloads.prefix_cow,
}


def _oracle_every_row(w):
    """The oracle side of one workload step, with the decode over every row on all cores."""
    alloc = RefAllocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed, pop_order=w.pop_order)
    setup_pairs = workloads.run_setup(w, alloc)
    slots, pairs, tables, lens = workloads.run_step_allocation(w, alloc)
    kp, vp = ref_copy_blocks(w.k_pool(), w.v_pool(), setup_pairs)
    kp, vp = ref_copy_blocks(kp, vp, [tuple(p) for p in pairs])
    kp, vp = ref_reshape_and_cache(w.new_k(), w.new_v(), kp, vp, slots)
    out = decode_all_rows(w.q(), kp, vp, tables, lens, w.scale)
    return {"out": out, "slots": slots, "pairs": pairs, "tables": tables, "lens": lens,
            "k_pool": kp, "v_pool": vp}


@pytest.mark.parametrize("name", sorted(FULL))
def test_full_size_every_row(name):
    w = FULL[name]()
    r = _oracle_every_row(w)
    for fused in (True, False):
        g = gpu_step(w, fused=fused, keep=fused)
        assert g["err"] == 0
        np.testing.assert_array_equal(g["slots"], r["slots"])
        np.testing.assert_array_equal(g["pairs"], r["pairs"])
        np.testing.assert_array_equal(g["tables"], r["tables"])
        np.testing.assert_array_equal(g["lens"], r["lens"])
        assert_close(w, g["out"], r["out"])
        if fused:
            # the decode kernel wrote every row's new K/V into its slot, and nothing else
            for pool, ref in ((g["k_pool"], r["k_pool"]), (g["v_pool"], r["v_pool"])):
                assert np.array_equal(pool_bits(pool), oracle_bits(ref, w))
        del g
        torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["prefix", "prefix_cow"])
def test_full_size_shared_prefix_every_row(name):
    """pa_decode_shared_prefix in the grouping bench.py times (whole fork families of
    8 samples x 4 heads as one unit), every row against the oracle."""
    import paged_kv_cache_350_b200 as pa
    w = FULL[name]()
    r = _oracle_every_row(w)
    g = gpu_step(w, keep=True)
    maxm = min(32, 64 // (w.Hq // w.Hkv))
    gof, gpre, gmem = g["alloc"].prefix_groups(w.step_seqs, maxm, pa.binding.PA_SHARED_PREFIX_ALIGN)
    assert len(gpre) == w.meta["prompts"]
    n = pa.pa_decode_shared_prefix_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.block_size, len(gpre))
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    out = torch.full_like(g["q"], float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_decode_shared_prefix(out, g["q"], g["k_pool"], g["v_pool"], g["t_d"], g["l_d"], w.scale,
                               torch.from_numpy(gof).cuda(), torch.from_numpy(gpre).cuda(),
                               torch.from_numpy(np.ascontiguousarray(gmem)).cuda(), ws,
                               err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert_close(w, out, r["out"])
