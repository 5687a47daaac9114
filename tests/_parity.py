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

BF16_ABS = 1e-2   # bf16: max |gpu - oracle|, or one bf16 ulp of the oracle value if larger
BF16_REL = 2e-2   # bf16: max over (b, h) rows of max|gpu - oracle| / max|oracle|
F32_ABS = 1e-4    # fp32 inputs: max |gpu - oracle|


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


def errors(gpu_out, ref_out, bf16=False):
    """(max abs error, max row-normwise relative error) of gpu vs oracle outputs.

    With ``bf16`` the absolute error is measured in excess of the output
    format's resolution: elementwise ``|g - r|`` where one bf16 ulp of ``r`` is
    at most 1e-2, and ``|g - r| * 1e-2 / ulp(r)`` where it is larger (|r| >= 2),
    so the bar 1e-2 means "within 1e-2, or within one bf16 ulp of the exact
    value when 1e-2 is finer than the format"."""
    g = gpu_out.float().cpu().numpy().astype(np.float64)
    r = np.asarray(ref_out, dtype=np.float64)
    diff = np.abs(g - r)
    scaled = diff
    if bf16:
        ulp = bf16_ulp(r)
        scaled = np.where(ulp > BF16_ABS, diff * BF16_ABS / ulp, diff)
    abs_err = float(scaled.max()) if diff.size else 0.0
    scale = np.abs(r).max(axis=-1)
    row_err = diff.max(axis=-1)
    nz = scale > 0
    rel = float((row_err[nz] / scale[nz]).max()) if nz.any() else 0.0
    # rows whose reference is exactly zero (empty sequences) must be exactly zero
    if (~nz).any():
        assert float(row_err[~nz].max()) == 0.0
    return abs_err, rel


def assert_close(w, gpu_out, ref_out):
    a, r = errors(gpu_out, ref_out, bf16=(w.dtype == "bf16"))
    if w.dtype == "bf16":
        assert a <= BF16_ABS and r <= BF16_REL, (a, r)
    else:
        assert a <= F32_ABS, a
    return a, r
