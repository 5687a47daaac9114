"""GPU parity at the full serving sizes, in the launch configuration bench.py times
(automatic path and partitioning, workspace from pa_decode_workspace_size).

The oracle computes a sample of batch rows one by one; the remaining rows are
checked for the properties that hold at any size (finite, and each output row
inside the convex hull bound max|v| of its values)."""

import numpy as np
import pytest
import torch

import workloads
from _parity import assert_close, gpu_step, oracle_step

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

FULL = {
    "gqa": (workloads.gqa, [0, 1, 77, 128, 255]),
    "mha": (workloads.mha, [0, 31, 63]),
    "long": (workloads.long_context, [0, 5]),
    "prefix": (workloads.prefix, [0, 9, 255]),
    "prefix_cow": (workloads.prefix_cow, [0, 7, 8, 250]),
}


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("name", sorted(FULL))
def test_full_size_sampled_rows(name, fused):
    """fused: pa_decode_append, the call bench.py times; else reshape_and_cache + pa_decode."""
    build, rows = FULL[name]
    w = build()
    g = gpu_step(w, fused=fused, keep=fused)
    assert g["err"] == 0
    if fused:
        # every row's new K/V sits in the slot the allocator reserved for it
        slots = torch.from_numpy(g["slots"]).cuda()
        for pool, new in ((g["k_pool"], g["nk"]), (g["v_pool"], g["nv"])):
            rows_at = pool.view(-1, w.Hkv, w.D)[slots]
            assert torch.equal(rows_at, new)
    out = g["out"].float()
    assert torch.isfinite(out).all()
    # |o| <= max |v| for a convex combination: a property of every row
    assert float(out.abs().max()) <= 6.0
    r = oracle_step(w, rows=rows)
    np.testing.assert_array_equal(g["slots"], r["slots"])
    np.testing.assert_array_equal(g["pairs"], r["pairs"])
    np.testing.assert_array_equal(g["tables"], r["tables"])
    assert_close(w, g["out"][torch.as_tensor(rows)], r["out"])
