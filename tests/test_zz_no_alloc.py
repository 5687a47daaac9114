"""GPU: pa_decode_no_alloc, the decode entry point that allocates nothing.

It serves callers that cannot allocate device memory (a runtime that owns every
device buffer through its own pool, or a caller that cannot afford cudaMalloc),
so it takes no workspace and uses the library's static device scratch instead.
Its output must match the float64 oracle's and pa_decode's (same inputs, workspace
supplied) within the parity tolerance, on two calls in a row with different batches, so
that whatever the first call left in the shared scratch cannot leak into the second.

This file is collected last on purpose: it runs after every other test in a
full session, and must also pass alone in a fresh process.
"""

import numpy as np
import pytest
import torch

import workloads
from _parity import assert_close, to_device
from oracle import ref_decode

pytestmark = pytest.mark.gpu


def _host_tables(w):
    import paged_kv_cache_350_b200 as pa
    alloc = pa.Allocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed, pop_order=w.pop_order)
    workloads.run_setup(w, alloc)
    _, _, tables, lens = workloads.run_step_allocation(w, alloc)
    return tables, lens


def _inputs(w):
    tables, lens = _host_tables(w)
    return (to_device(w.q(), w), to_device(w.k_pool(), w), to_device(w.v_pool(), w),
            torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda())


def _reference(w, q, kp, vp, tables, lens):
    import paged_kv_cache_350_b200 as pa
    n = pa.pa_decode_workspace_size(w.B, w.Hq, w.Hkv, w.D, tables.shape[1] * w.block_size,
                                    w.block_size, 0)
    ws = torch.empty(max(n, 1), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    pa.pa_decode(out, q, kp, vp, tables, lens, w.scale, workspace=ws)
    return out


def test_no_alloc_matches_oracle_and_pa_decode_on_two_calls_in_a_row():
    import paged_kv_cache_350_b200 as pa
    cases = [workloads.gqa(B=40, median=300, lo=1, hi=1200, seed=5100),
             workloads.long_context(B=3, lo=2000, hi=9000, Hq=32, seed=5101)]
    for w in cases:
        q, kp, vp, tables, lens = _inputs(w)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = torch.full_like(q, float("nan"))
        pa.pa_decode_no_alloc(out, q, kp, vp, tables, lens, w.scale, err_flag=err)
        ref = _reference(w, q, kp, vp, tables, lens)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert torch.isfinite(out.float()).all()
        tables, lens = _host_tables(w)
        assert_close(w, out, ref_decode(w.q(), w.k_pool(), w.v_pool(), tables, lens, w.scale))
        assert_close(w, out, ref.float().cpu().numpy(), exact_ref=False)


def test_no_alloc_rejects_what_it_does_not_take():
    import paged_kv_cache_350_b200 as pa
    w = workloads.independent([5, 9], Hq=4, Hkv=4, D=64, bs=4, dtype="f32")
    q, kp, vp, tables, lens = _inputs(w)
    with pytest.raises(pa.PAError) as e:
        pa.pa_decode_no_alloc(torch.empty_like(q), q, kp, vp, tables, lens, w.scale)
    assert e.value.status == pa.binding.PA_ERR_UNSUPPORTED
