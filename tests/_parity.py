"""Helpers for the parity tests: run one workload step on each side.

Product side: the C allocator and the CUDA kernels through the binding.
Oracle side:  ``oracle.RefAllocator`` and the float64 CPU functions.
Both start from the same seeded inputs (``workloads``); neither side's
outputs feed the other.
"""

import numpy as np
import torch

import workloads
from oracle import RefAllocator, ref_copy_blocks, ref_decode, ref_reshape_and_cache

# Tolerances of the bf16 attention outputs: max-abs-error <= 1e-2 and max-rel-error <= 2e-2
# against the float64 oracle; <= 1e-4 abs for fp32 inputs.
BF16_ABS = 1e-2     # elementwise |g - r|, where the bf16 output format can hold it (below)
BF16_REL = 2e-2     # elementwise |g - r| / max(|r|, REL_FLOOR)
REL_FLOOR = 1e-3    # so that outputs near zero do not turn rounding noise into a ratio
F32_ABS = 1e-4      # fp32 inputs: max |g - r|
# What the bf16 path may differ from the exact value by before its one final rounding to
# bf16.  It computes in fp32; the largest term is P entering the P.V product as two bf16
# parts, hi = rn(p) and lo = rn(p - hi), so |p - hi - lo| <= 2^-18 p and the output moves
# by at most 2^-18 * sum_t p_t |v_t| <= 2^-18 * max|v| (< 8 for N(0,1) draws): 3.1e-5.
# exp2, the fp32 sums and the tensor cores' fp32 accumulation add orders of magnitude
# less at these logit sizes.  The slack is about three times that bound.
F32_SLACK = 1e-4


def torch_dtype(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def to_device(arr, w, device="cuda"):
    """Host draw (uint16 bf16 bits or float32) -> device tensor of the workload dtype."""
    if w.dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(arr)).to(device)


def gpu_step(w, partition_tokens=0, path=0, device="cuda", keep=False, max_ctas=0, fused=False):
    """The product path: allocator, copy_blocks, reshape_and_cache, decode. Returns dict.

    With ``fused`` the cache write and the decode are one pa_decode_append call, which
    derives each row's slot from its table and length (the allocator's slots are only
    compared, not passed)."""
    import paged_kv_cache_350_b200 as pa
    alloc = pa.Allocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed, pop_order=w.pop_order)
    setup_pairs = workloads.run_setup(w, alloc)
    slots, pairs, tables, lens = workloads.run_step_allocation(w, alloc)
    kp = to_device(w.k_pool(), w, device)
    vp = to_device(w.v_pool(), w, device)
    if setup_pairs:  # copy-on-write during setup (forks appending into a partial prompt block)
        pa.pa_copy_blocks(kp, vp, torch.tensor(setup_pairs, dtype=torch.int32, device=device))
    q = to_device(w.q(), w, device)
    nk = to_device(w.new_k(), w, device)
    nv = to_device(w.new_v(), w, device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    pa.pa_copy_blocks(kp, vp, torch.from_numpy(pairs).to(device), err_flag=err)
    if not fused:
        pa.pa_reshape_and_cache(nk, nv, kp, vp, torch.from_numpy(slots).to(device), err_flag=err)
    out = torch.empty_like(q)
    nws = pa.pa_decode_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.max_blocks * w.block_size,
                                      w.block_size, partition_tokens)
    ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=device)
    t_d = torch.from_numpy(tables).to(device)
    l_d = torch.from_numpy(lens).to(device)
    if fused:
        pa.pa_decode_append(out, q, nk, nv, kp, vp, t_d, l_d, w.scale, workspace=ws, err_flag=err,
                            partition_tokens=partition_tokens, path=path, max_ctas=max_ctas)
    else:
        pa.pa_decode(out, q, kp, vp, t_d, l_d, w.scale, workspace=ws, err_flag=err,
                     partition_tokens=partition_tokens, path=path, max_ctas=max_ctas)
    torch.cuda.synchronize()
    res = {"out": out, "slots": slots, "pairs": pairs, "tables": tables, "lens": lens,
           "err": int(err.item()), "alloc": alloc}
    if keep:
        res.update(k_pool=kp, v_pool=vp, q=q, ws=ws, t_d=t_d, l_d=l_d, nk=nk, nv=nv)
    return res


def oracle_step(w, rows=None):
    """The oracle path; ``rows`` restricts the decode to a subset of batch rows."""
    alloc = RefAllocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed, pop_order=w.pop_order)
    setup_pairs = workloads.run_setup(w, alloc)
    slots, pairs, tables, lens = workloads.run_step_allocation(w, alloc)
    kp, vp = ref_copy_blocks(w.k_pool(), w.v_pool(), setup_pairs)
    kp, vp = ref_copy_blocks(kp, vp, [tuple(p) for p in pairs])
    kp, vp = ref_reshape_and_cache(w.new_k(), w.new_v(), kp, vp, slots)
    rows = np.arange(w.B) if rows is None else np.asarray(rows)
    out = ref_decode(w.q()[rows], kp, vp, tables[rows], lens[rows], w.scale)
    return {"out": out, "slots": slots, "pairs": pairs, "tables": tables, "lens": lens,
            "k_pool": kp, "v_pool": vp, "alloc": alloc, "rows": rows}


def pool_bits(t):
    """Device pool -> host array of its raw element bits (int16 for bf16, float32 else)."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy()
    return t.cpu().numpy()


def oracle_bits(a, w):
    """Oracle pool (uint16 bf16 bits or float32) -> the same form as pool_bits."""
    return np.asarray(a).view(np.int16) if w.dtype == "bf16" else np.asarray(a, dtype=np.float32)


def bf16_ulp(x):
    """Spacing of bfloat16 numbers at |x| (8 significant bits; normal range)."""
    ax = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(ax)) - 7)


def abs_bar(r, exact_ref=True):
    """Elementwise bound on |g - r| for a bf16 output g.

    The literal 1e-2, except where bf16 cannot resolve it: a kernel that computes in fp32
    and rounds once to nearest lands within half a bf16 ulp of its fp32 value, which is
    within F32_SLACK of the exact value, so the bound is max(1e-2, ulp(r)/2 + F32_SLACK).
    Half an ulp exceeds 1e-2 only for |r| >= 4 (ulp 2^-5 there).  With ``exact_ref`` False
    the reference r is itself a rounded GPU output (two GPU paths compared): both lie
    within that bound of the exact value, so they may differ by twice it."""
    r = np.asarray(r, dtype=np.float64)
    k = 1.0 if exact_ref else 2.0
    return np.maximum(BF16_ABS, k * (0.5 * bf16_ulp(r) + F32_SLACK))


def errors(gpu_out, ref_out, bf16=False, exact_ref=True):
    """Parity figures of gpu vs reference outputs (``[..., D]``), as a dict:

    abs       max |g - r|
    abs_bar   max |g - r| / abs_bar(r)  (bf16; <= 1 passes)
    rel       max elementwise |g - r| / max(|r|, REL_FLOOR)  (the asserted relative error)
    rel_unfloored  max elementwise |g - r| / |r| over r != 0  (reported only)
    rel_row   max over rows of max_d |g - r| / max_d |r|     (reported only)
    """
    g = gpu_out.float().cpu().numpy().astype(np.float64) if hasattr(gpu_out, "cpu") \
        else np.asarray(gpu_out, dtype=np.float64)
    r = np.asarray(ref_out, dtype=np.float64)
    diff = np.abs(g - r)
    res = {"abs": float(diff.max()) if diff.size else 0.0, "abs_bar": 0.0, "rel": 0.0,
           "rel_unfloored": 0.0, "rel_row": 0.0, "n": int(diff.size)}
    if not diff.size:
        return res
    if bf16:
        res["abs_bar"] = float((diff / abs_bar(r, exact_ref)).max())
    ar = np.abs(r)
    res["rel"] = float((diff / np.maximum(ar, REL_FLOOR)).max())
    nz = ar > 0
    res["rel_unfloored"] = float((diff[nz] / ar[nz]).max()) if nz.any() else 0.0
    scale = ar.max(axis=-1)
    row_err = diff.max(axis=-1)
    rows = scale > 0
    res["rel_row"] = float((row_err[rows] / scale[rows]).max()) if rows.any() else 0.0
    # rows whose reference is exactly zero (empty sequences) must be exactly zero
    if (~rows).any():
        assert float(row_err[~rows].max()) == 0.0, "a zero reference row is not zero"
    return res


def _log(w, res, exact_ref):
    """Append the figures to the file named by PA_PARITY_LOG (when set), one JSON line per
    comparison, so that a GPU run leaves a record of the errors it saw."""
    import json
    import os
    path = os.environ.get("PA_PARITY_LOG")
    if not path:
        return
    rec = {"test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], "workload": w.name,
           "dtype": w.dtype, "exact_ref": exact_ref, **res}
    with open(path, "a") as f:
        f.write(json.dumps(rec) + "\n")


def assert_close(w, gpu_out, ref_out, exact_ref=True):
    """Assert the tolerances: bf16, elementwise |g - r| <= abs_bar(r) and
    |g - r| / max(|r|, 1e-3) <= 2e-2; fp32, |g - r| <= 1e-4.  ``exact_ref``: the reference
    is the float64 oracle (False: another GPU path's bf16 output).  Returns the figures."""
    bf16 = w.dtype == "bf16"
    res = errors(gpu_out, ref_out, bf16=bf16, exact_ref=exact_ref)
    _log(w, res, exact_ref)
    if bf16:
        assert res["abs_bar"] <= 1.0 and res["rel"] <= BF16_REL, res
    else:
        assert res["abs"] <= F32_ABS, res
    return res
