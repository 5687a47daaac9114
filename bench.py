#!/usr/bin/env python
"""Benchmark: paged decode attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config gqa] [--impl ours|reference]

One step = one decode step of the whole hot path over one synthetic batch:
copy-on-write block copies (when the step has any), then pa_decode_append: the
step's new K/V written to their slots (reshape_and_cache, fused into the decode
kernel) and the decode attention (plus its reduce).  ``--unfused`` runs
pa_reshape_and_cache and pa_decode as two calls instead.  The allocator's
slot mapping, copy pairs, tables and lengths for the step are computed on the
host before timing and are resident in HBM; the timed steps repeat the same
step (the cache writes are idempotent), over pools larger than the 126 MB L2.

Prints ONE JSON line (rank 0).  ``value`` = algorithmic KV bytes of pa_decode
per step x steps x ranks / max-over-ranks device time, in GB/s (the whole step
is in the denominator).  ``e2e`` = the same metric through
``PagedKVCache.pipeline`` with host buffers: per step the allocator, a host->device
copy, the kernels and a device->host copy of the output, steps queued back to back.  ``roofline`` is the decode
call alone (pa_decode_append, or pa_decode with ``--unfused``) against the
measured HBM copy bandwidth.

With ``--impl reference`` the float64 CPU oracle is timed instead, on a
bounded sample of the same workload per step.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "paged decode attention KV GB/s"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0

CONFIG_TEXT = {
    "gqa": "Llama-3-8B-shaped GQA decode, bf16: B=256, Hq=32, Hkv=8, D=128, block_size=16, "
           "seq_lens log-normal(median 1024, sigma 0.6) clipped [64, 4096], shuffled blocks, "
           "one new token per sequence via reshape_and_cache before attention",
    "mha": "Llama-7B-shaped MHA decode, bf16: B=64, Hq=Hkv=32, D=128, block_size=16, "
           "seq_lens U[128, 2048], shuffled blocks",
    "long": "long-context GQA decode, bf16: B=8, Hq=64, Hkv=8, D=128, block_size=16, "
            "seq_lens U[32768, 131072], shuffled blocks",
    "prefix": "parallel sampling, bf16: 32 prompts x 8 samples sharing 1024-token prompt "
              "blocks (refcount 8), U{0..256} private tokens, Hq=32, Hkv=8, D=128, bs=16",
    "prefix_cow": "parallel sampling first divergence, bf16: 32 prompts of 1000 tokens x 8 "
                  "samples; 224 copy-on-write block copies in the step; Hq=32, Hkv=8, D=128",
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="gqa", choices=sorted(CONFIG_TEXT))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-all-cores", type=int, default=1,
                    help="also time the oracle in one spawned process per host core (0: off)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--shared-prefix", action="store_true",
                    help="decode with pa_decode_shared_prefix (fork groups read shared blocks once)")
    ap.add_argument("--block-size", type=int, default=0,
                    help="override the workload's block size (8, 16 or 32) for a sweep")
    ap.add_argument("--long", type=int, default=1,
                    help="with the gqa config, also time the long-context batch in the same run "
                         "(reported under \"long\"; 0: off)")
    ap.add_argument("--unfused", action="store_true",
                    help="pa_reshape_and_cache + pa_decode as two calls (default: pa_decode_append)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# accounting
# ---------------------------------------------------------------------------

def decode_bytes(lens, B, Hq, Hkv, D, bs, esize):
    """Algorithmic bytes of one pa_decode call: K/V once per KV head, q, out, tables, lens."""
    lens = np.asarray(lens, dtype=np.int64)
    kv = int(2 * lens.sum() * Hkv * D * esize)
    qo = 2 * B * Hq * D * esize
    tab = int(np.sum(-(-lens // bs)) * 4) + 4 * B
    return kv + qo + tab, kv


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _code_only(text):
    """C/CUDA source without comments and blank lines (so a comment edit keeps the hash)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln.strip())


def decode_kernel_hash():
    """Hash of the decode kernels' code; a recorded ncu traffic figure holds while it matches."""
    h = hashlib.sha256()
    for f in ("decode_stream.cu", "decode_tc.cu", "tc_tile.cuh", "pa_device.cuh"):
        with open(os.path.join(ROOT, "paged_kv_cache_350_b200", "csrc", f)) as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(config, call):
    """DRAM bytes per call from a committed ncu summary, if it covers this call and the kernel
    sources are unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(config)
    except Exception:
        return None
    if not rec or rec.get("call") != call or rec.get("kernel_hash") != decode_kernel_hash():
        return None
    return rec.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, sampled in a thread)
# ---------------------------------------------------------------------------

_REASONS = [(0x4, "sw_power_cap"), (0x8, "hw_slowdown"), (0x20, "sw_thermal_slowdown"),
            (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown"),
            (0x2, "applications_clocks_setting"), (0x10, "sync_boost")]


class ClockSampler:
    def __init__(self, device_index, period_s=0.02):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _reasons(self):
        nv = self.nv
        for fn in ("nvmlDeviceGetCurrentClocksEventReasons", "nvmlDeviceGetCurrentClocksThrottleReasons"):
            if hasattr(nv, fn):
                return getattr(nv, fn)(self.h)
        return 0

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self._reasons())
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if self.nv is None or not self.samples:
            return None
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": [n for bit, n in _REASONS if self.reasons & bit],
                "samples": len(self.samples), "source": "nvml"}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas: one process per GPU, no data-path collective)
# ---------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init_dist(world, local_rank, backend="nccl"):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    kw = {"timeout": datetime.timedelta(seconds=300)}
    if backend == "nccl":
        import torch
        kw["device_id"] = torch.device("cuda", local_rank)
    dist.init_process_group(backend, **kw)
    return dist


def max_over_ranks(x, dist, device=None):
    """Max of a float over all ranks (identity without a process group)."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device=None):
    if dist is not None:
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_sample_rate(w, tables, lens, seconds, row_order=None, max_tokens=None):
    """Time oracle.ref_decode on whole sequences until ``seconds`` pass; returns (GB/s, desc)."""
    from oracle import ref_decode
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(limits=1)
    except Exception:
        limiter = None
    q, kp, vp = w.q(), w.k_pool(), w.v_pool()
    esize = 2 if w.dtype == "bf16" else 4
    rows = list(row_order) if row_order is not None else list(range(w.B))
    done_bytes = 0
    done_rows = 0
    tokens = 0
    t0 = time.perf_counter()
    for r in rows:
        L = int(lens[r]) if max_tokens is None else min(int(lens[r]), max_tokens)
        ref_decode(q[r:r + 1], kp, vp, tables[r:r + 1], np.array([L]), w.scale)
        done_bytes += decode_bytes([L], 1, w.Hq, w.Hkv, w.D, w.block_size, esize)[0]
        done_rows += 1
        tokens += L
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    if limiter is not None:
        limiter.unregister()
    desc = (f"oracle.ref_decode (float64 NumPy, 1 BLAS thread) on {done_rows} sequence(s) "
            f"({tokens} tokens x {w.Hkv} KV heads) of the {w.name} batch")
    return done_bytes / dt / 1e9, desc, dt


def _oracle_worker(task):
    """One spawned worker of oracle_rate_all_cores: ref_decode on its rows until the time
    budget passes, reading the pools from shared memory.  Returns (bytes, seconds)."""
    from multiprocessing import shared_memory
    from oracle import ref_decode
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except Exception:
        pass
    name, shape, dtype, qshape, tables, lens, rows, scale, seconds, Hq, Hkv, D, bs, esize = task
    shm = shared_memory.SharedMemory(name=name)
    try:
        nb = int(np.prod(shape)) * np.dtype(dtype).itemsize
        kp = np.ndarray(shape, dtype=dtype, buffer=shm.buf)
        vp = np.ndarray(shape, dtype=dtype, buffer=shm.buf, offset=nb)
        q = np.ndarray(qshape, dtype=dtype, buffer=shm.buf, offset=2 * nb)
        done = 0
        t0 = time.perf_counter()
        for r in rows:
            ref_decode(q[r:r + 1], kp, vp, tables[r:r + 1], lens[r:r + 1], scale)
            done += decode_bytes([int(lens[r])], 1, Hq, Hkv, D, bs, esize)[0]
            if time.perf_counter() - t0 >= seconds:
                break
        dt = time.perf_counter() - t0
        del kp, vp, q
    finally:
        shm.close()
    return done, dt


def oracle_rate_all_cores(w, tables, lens, seconds, workers=None):
    """The same oracle on every host core: one spawned process per core, each on its own
    rows of the batch (round robin), the pools shared read-only through shared memory.
    Returns (GB/s = all bytes / the slowest worker's time, processes, description)."""
    import multiprocessing as mp
    from multiprocessing import shared_memory
    workers = workers or len(os.sched_getaffinity(0))
    kp, vp, q = w.k_pool(), w.v_pool(), w.q()
    shm = shared_memory.SharedMemory(create=True, size=kp.nbytes + vp.nbytes + q.nbytes)
    try:
        np.ndarray(kp.shape, dtype=kp.dtype, buffer=shm.buf)[...] = kp
        np.ndarray(vp.shape, dtype=vp.dtype, buffer=shm.buf, offset=kp.nbytes)[...] = vp
        np.ndarray(q.shape, dtype=q.dtype, buffer=shm.buf, offset=2 * kp.nbytes)[...] = q
        esize = 2 if w.dtype == "bf16" else 4
        tasks = [(shm.name, kp.shape, kp.dtype, q.shape, tables, lens,
                  list(range(i, w.B, workers)), w.scale, seconds, w.Hq, w.Hkv, w.D,
                  w.block_size, esize)
                 for i in range(min(workers, w.B))]
        del kp, vp, q
        # a worker that dies raises here instead of being respawned for ever
        from concurrent.futures import ProcessPoolExecutor
        with ProcessPoolExecutor(len(tasks), mp_context=mp.get_context("spawn")) as ex:
            res = list(ex.map(_oracle_worker, tasks, timeout=10 * seconds + 120))
    finally:
        shm.close()
        shm.unlink()
    total = sum(r[0] for r in res)
    slowest = max(r[1] for r in res)
    desc = (f"oracle.ref_decode (float64 NumPy) in {len(tasks)} spawned processes, one per "
            f"core, each on every {len(tasks)}-th sequence of the {w.name} batch for about "
            f"{seconds:.0f} s; the pools shared read-only")
    return total / slowest / 1e9, len(tasks), desc


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    from oracle import RefAllocator
    w = workloads.build(args.config)
    alloc = RefAllocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed, pop_order=w.pop_order)
    workloads.run_setup(w, alloc)
    _, _, tables, lens = workloads.run_step_allocation(w, alloc)
    # per-step sample: one sequence, truncated so the whole run stays within ~3 minutes
    budget = 150.0 / max(1, args.steps + args.warmup)
    _, _, dt1 = oracle_sample_rate(w, tables, lens, 0.0, row_order=[0], max_tokens=256)
    per_token = dt1 / 256
    max_tok = max(16, int(budget / per_token))
    rates, times, nbytes = [], [], []
    esize = 2 if w.dtype == "bf16" else 4
    for i in range(args.warmup + args.steps):
        r = i % w.B
        t0 = time.perf_counter()
        rate, desc, dt = oracle_sample_rate(w, tables, lens, 0.0, row_order=[r], max_tokens=max_tok)
        if i >= args.warmup:
            times.append(dt)
            nbytes.append(decode_bytes([min(int(lens[r]), max_tok)], 1, w.Hq, w.Hkv, w.D,
                                       w.block_size, esize)[0])
    value = sum(nbytes) / sum(times) / 1e9
    sampled = [int(lens[i % w.B]) for i in range(args.warmup, args.warmup + args.steps)]
    cut = (f"truncated to its first {max_tok} tokens" if max(sampled) > max_tok
           else "whole (no sampled sequence is longer than the per-step cap)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": CONFIG_TEXT[args.config],
                   "sample": f"per step one sequence of the batch (round robin), {cut}, "
                             f"all {w.Hkv} KV heads"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"oracle.ref_decode per step on one sequence, {cut} "
                                   f"(float64 NumPy, 1 thread)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def to_device(arr, w, device):
    import torch
    if w.dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(arr)).to(device)


def prepare(args, pa, device, config, block_size=0):
    """Inputs of one config resident on the device, and the step closure that runs the hot
    path over them (the allocator's output for the step computed on the host first)."""
    import torch
    w = workloads.build(config, **({"bs": block_size} if block_size else {}))
    esize = 2 if w.dtype == "bf16" else 4
    dtype_pa = pa.PA_BF16 if w.dtype == "bf16" else pa.PA_F32

    alloc = pa.Allocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed, pop_order=w.pop_order)
    assert workloads.run_setup(w, alloc) == []
    slots, pairs, tables, lens = workloads.run_step_allocation(w, alloc)
    MB = w.max_blocks + (args.e2e_steps + w.block_size - 1) // w.block_size + 1
    tables_wide = np.full((w.B, MB), -1, dtype=np.int32)
    tables_wide[:, : tables.shape[1]] = tables

    kp = to_device(w.k_pool(), w, device)
    vp = to_device(w.v_pool(), w, device)
    q = to_device(w.q(), w, device)
    nk = to_device(w.new_k(), w, device)
    nv = to_device(w.new_v(), w, device)
    slots_d = torch.from_numpy(slots).to(device)
    pairs_d = torch.from_numpy(np.ascontiguousarray(pairs)).to(device)
    tables_d = torch.from_numpy(tables_wide).to(device)
    lens_d = torch.from_numpy(lens).to(device)
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    nws = pa.pa_decode_workspace_size(w.B, w.Hq, w.Hkv, w.D, MB * w.block_size, w.block_size, 0)
    ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=device)
    plan = pa.pa_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.block_size, MB, dtype_pa, nws)
    npairs = int(pairs.shape[0])
    stream = torch.cuda.current_stream(device)
    fused = not (args.unfused or args.shared_prefix)
    # the fused call adds an append kernel only on the paths whose decode kernel does
    # not write the token itself
    append_launch = 1 if (not fused or plan["kernel"] != pa.binding.PA_KERNEL_TC_STREAM) else 0
    launches_per_step = plan["launches"] + append_launch + (1 if npairs else 0)
    unique_kv = None
    sp = None
    if args.shared_prefix:
        maxm = max(1, min(32, 64 // (w.Hq // w.Hkv)))
        gof, gpre, gmem = alloc.prefix_groups(w.step_seqs, maxm, pa.binding.PA_SHARED_PREFIX_ALIGN)
        ng = len(gpre)
        sp = {"gof": torch.from_numpy(np.ascontiguousarray(gof)).to(device),
              "gpre": torch.from_numpy(np.ascontiguousarray(gpre) if ng else np.zeros(1, np.int32)).to(device),
              "gmem": torch.from_numpy(np.ascontiguousarray(gmem).reshape(ng, maxm)).to(device)}
        nws = pa.pa_decode_shared_prefix_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.block_size, ng)
        ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=device)
        pre_of = np.where(gof >= 0, np.asarray(gpre, dtype=np.int64)[np.maximum(gof, 0)] if ng else 0, 0)
        tok_unique = int(np.asarray(gpre, dtype=np.int64).sum()) + int((lens - pre_of).sum())
        unique_kv = 2 * tok_unique * w.Hkv * w.D * esize
        plan = {"kernel": "shared_prefix", "groups": ng, "max_members": maxm, "launches": 1}
        launches_per_step = 1 + 1 + (1 if npairs else 0)

    def step(ev=None):
        if npairs:
            pa.pa_copy_blocks(kp, vp, pairs_d, err_flag=err, stream=stream)
        if fused:
            if ev is not None:
                ev[0].record(stream)
            pa.pa_decode_append(out, q, nk, nv, kp, vp, tables_d, lens_d, w.scale, workspace=ws,
                                err_flag=err, stream=stream)
            if ev is not None:
                ev[1].record(stream)
            return
        pa.pa_reshape_and_cache(nk, nv, kp, vp, slots_d, err_flag=err, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        if args.shared_prefix:
            pa.pa_decode_shared_prefix(out, q, kp, vp, tables_d, lens_d, w.scale, sp["gof"],
                                       sp["gpre"], sp["gmem"], ws, err_flag=err, stream=stream)
        else:
            pa.pa_decode(out, q, kp, vp, tables_d, lens_d, w.scale, workspace=ws, err_flag=err,
                         stream=stream)
        if ev is not None:
            ev[1].record(stream)

    alg_bytes, kv_bytes = decode_bytes(lens, w.B, w.Hq, w.Hkv, w.D, w.block_size, esize)
    # bytes that must cross HBM: with shared prefixes, each group's shared tokens once
    roof_bytes = alg_bytes if unique_kv is None else alg_bytes - kv_bytes + unique_kv
    # the fused call also writes each row's new K/V to its slot (its read replaces the
    # read of that slot, already counted in the decode bytes)
    append_bytes = 2 * w.B * w.Hkv * w.D * esize if fused else 0
    roof_bytes += append_bytes
    return {"w": w, "config": config, "esize": esize, "alloc": alloc, "slots": slots,
            "pairs": pairs, "tables": tables, "lens": lens, "MB": MB, "kp": kp, "vp": vp,
            "q": q, "nk": nk, "nv": nv, "err": err, "plan": plan, "npairs": npairs,
            "stream": stream, "fused": fused, "launches_per_step": launches_per_step,
            "unique_kv": unique_kv, "step": step, "alg_bytes": alg_bytes, "kv_bytes": kv_bytes,
            "roof_bytes": roof_bytes, "append_bytes": append_bytes}


def time_steps(st, K, W, dist, device):
    """W untimed steps, then K steps bracketed by a barrier and a synchronize on both sides,
    timed with CUDA events on the launching stream; then the same K steps again with an
    event pair around each decode call (the kernel's own time: an event between two
    kernels stops the second from launching while the first drains, so the whole-region
    figure is taken without them).  The clocks are sampled during both.  Times are the max
    over ranks."""
    import torch
    step, err, stream = st["step"], st["err"], st["stream"]
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flag {int(err.item())} during warm-up")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(device.index)
    barrier(dist, device)
    torch.cuda.synchronize()
    clocks.start()
    t_start.record(stream)
    for i in range(K):
        step()
    t_end.record(stream)
    torch.cuda.synchronize()
    for i in range(K):
        step(evs[i])
    torch.cuda.synchronize()
    clocks.stop()
    barrier(dist, device)
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), dist, device)
    dec_avg_ms = max_over_ranks(statistics.fmean(a.elapsed_time(b) for a, b in evs), dist, device)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flag {int(err.item())} during timing")
    return elapsed_ms, dec_avg_ms, clocks.summary()


def roofline(st, dec_avg_ms, config):
    """The decode call of one step against the measured HBM copy bandwidth."""
    peak, peak_src = measured_peak()
    achieved = st["roof_bytes"] / (dec_avg_ms / 1e3) / 1e9
    fused = st["fused"]
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak,
            "traffic": recorded_traffic(config, "pa_decode_append" if fused else "pa_decode"),
            "kernel": ("pa_decode_append call (decode kernel with the fused cache write + its "
                       "reduce)" if fused else
                       "pa_decode_shared_prefix call (one kernel; cut units merged inside it)"
                       if st["unique_kv"] is not None else
                       "pa_decode call (main kernel + its reduce)") + ", CUDA events per call",
            "append_bytes_per_call": st["append_bytes"],
            "peak_source": f"{peak_src} HBM copy bandwidth (burst)"}


def run_ours(args):
    import torch
    rank, local_rank, world = dist_env()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    dist = init_dist(world, local_rank)
    if rank == 0:
        from paged_kv_cache_350_b200.build import build
        build()
    barrier(dist, device)
    import paged_kv_cache_350_b200 as pa

    st = prepare(args, pa, device, args.config, args.block_size)
    w, esize, alloc = st["w"], st["esize"], st["alloc"]
    tables, lens, MB = st["tables"], st["lens"], st["MB"]
    kp, vp, q, nk, nv = st["kp"], st["vp"], st["q"], st["nk"], st["nv"]
    plan, npairs, stream, fused = st["plan"], st["npairs"], st["stream"], st["fused"]
    unique_kv, alg_bytes, kv_bytes = st["unique_kv"], st["alg_bytes"], st["kv_bytes"]

    K = args.steps
    elapsed_ms, dec_avg_ms, clock_summary = time_steps(st, K, args.warmup, dist, device)
    value = alg_bytes * K * world / (elapsed_ms / 1e3) / 1e9
    tokens_per_s = w.B * K * world / (elapsed_ms / 1e3)
    roof = roofline(st, dec_avg_ms, args.config)

    # ---- end to end through the public API with host buffers -------------------------
    # PagedKVCache.pipeline: every step is one C call (pa_pipeline_submit) that runs the
    # allocator, one host->device copy of the step input (q, new K/V, tables, lengths, copy
    # pairs), pa_copy_blocks + pa_decode_append and a device->host copy of the output; steps
    # are queued back to back over three staging slots, and each step's output is read two
    # steps later (so the host and the copies of neighbouring steps stay off the GPU's
    # critical path).
    # Shared-prefix runs take the pipeline's shared-prefix steps (fork groups formed in the
    # same C call; copy_blocks, reshape_and_cache and pa_decode_shared_prefix), on a pool of
    # their own with room for every step's appends (zeroed blocks: the work does not depend
    # on the values; the batch's 10 % of free blocks would last a few steps).
    e2e = None
    if not args.no_e2e and args.e2e_steps > 0:
        members = plan["max_members"] if args.shared_prefix else 0
        if members:
            nb_e2e = w.num_blocks + w.B * ((args.e2e_steps + 8 + w.block_size - 1) // w.block_size + 1)
            cache = pa.PagedKVCache(nb_e2e, w.block_size, w.Hkv, w.D, dtype=kp.dtype, device=device,
                                    shuffle_seed=w.alloc_seed, pop_order=w.pop_order)
        else:
            cache = pa.PagedKVCache(w.num_blocks, w.block_size, w.Hkv, w.D, dtype=kp.dtype,
                                    device=device, shuffle_seed=w.alloc_seed, pop_order=w.pop_order,
                                    k_pool=kp, v_pool=vp)
        workloads.run_setup(w, cache.alloc)
        pipe = cache.pipeline(w.B, w.Hq, MB, depth=3, stream=stream, shared_prefix_members=members)
        lag = pipe.depth - 1
        q_c, nk_c, nv_c = q.cpu(), nk.cpu(), nv.cpu()
        ids = np.asarray(w.step_seqs, dtype=np.int64)
        warm = max(2, pipe.depth)
        nbytes = []
        host_s = []
        cur = lens.astype(np.int64).copy()
        t0 = None
        done = 0
        for i in range(warm + args.e2e_steps):
            if i < pipe.depth:  # the same inputs every step: each staging slot written once
                for dst, src in zip(pipe.inputs(), (q_c, nk_c, nv_c)):
                    dst.copy_(src)
            if i == warm:
                pipe.sync()
                barrier(dist, device)
                t0 = time.perf_counter()
            try:
                h0 = time.perf_counter()
                pipe.submit(ids, w.scale)
                if i >= warm:
                    host_s.append(time.perf_counter() - h0)
            except pa.PAError:  # the pool ran out of blocks for more appends
                break
            if i >= lag:
                pipe.result(i - lag)
            if i >= warm:
                nbytes.append(decode_bytes(cur, w.B, w.Hq, w.Hkv, w.D, w.block_size, esize)[0])
                done += 1
            cur += 1
        pipe.result(pipe.next - 1)
        dt = time.perf_counter() - t0 if t0 is not None else 0.0
        cache.check_device_errors()
        if done:
            dt = max_over_ranks(dt, dist, device)
            e2e = {"value": sum(nbytes) * world / dt / 1e9, "unit": UNIT,
                   "h2d_bytes_per_step": int(pipe.bytes_in), "d2h_bytes_per_step": int(pipe.bytes_out),
                   "ms_per_step": 1e3 * dt / done, "steps": done,
                   "host_us_per_submit": 1e6 * statistics.median(host_s) if host_s else None,
                   "timing": "host perf_counter over the steps of PagedKVCache.pipeline: per step "
                             "one C call (pa_pipeline_submit: the allocator%s, one host->device "
                             "copy of the step input, the kernels, a device->host copy of the "
                             "output, read two steps later); steps queued back to back over three "
                             "staging slots%s" % (
                                 " and the fork grouping" if members else "",
                                 "; the batch grows a token per step, so only the first step "
                                 "copies blocks on write" if members else "")}

    # ---- the long-context batch, timed in the same run ---------------------------------
    # The decode must hold its bandwidth on both serving shapes: the GQA batch above and
    # long contexts (B=8, 32K-128K tokens), where every unit is split over many streams.
    long_line = None
    gpu_launches = st["launches_per_step"] * K
    if args.config == "gqa" and args.long and not args.shared_prefix and not args.block_size:
        sl = prepare(args, pa, device, "long")
        l_ms, l_dec_ms, l_clocks = time_steps(sl, K, args.warmup, dist, device)
        wl = sl["w"]
        long_line = {
            "workload": CONFIG_TEXT["long"], "name": "long", "B": wl.B, "Hq": wl.Hq,
            "Hkv": wl.Hkv, "head_dim": wl.D, "block_size": wl.block_size,
            "mean_seq_len": float(np.mean(sl["lens"])), "steps": K, "warmup": args.warmup,
            "value": sl["alg_bytes"] * K * world / (l_ms / 1e3) / 1e9, "unit": UNIT,
            "ms_per_step": l_ms / K,
            "decode_tokens_per_s": wl.B * K * world / (l_ms / 1e3),
            "alg_bytes_per_step": sl["alg_bytes"], "decode_plan": sl["plan"],
            "step_calls": "pa_decode_append" if sl["fused"] else "pa_reshape_and_cache + pa_decode",
            "roofline": roofline(sl, l_dec_ms, "long"),
            "clocks": l_clocks,
            "l2": "inputs larger than L2 (K/V pools of %.2f GB vs 126 MB L2); not flushed"
                  % (2 * sl["kp"].numel() * sl["esize"] / 1e9),
        }
        gpu_launches += sl["launches_per_step"] * K
        del sl

    # ---- CPU oracle baseline (rank 0, one GPU only) --------------------------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, desc, _ = oracle_sample_rate(w, tables, lens, args.cpu_seconds)
        cpu = {"value": rate, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc}
        if args.cpu_all_cores:
            try:
                need = 2 * w.k_pool().nbytes + w.q().nbytes
                fs = os.statvfs("/dev/shm")
                if fs.f_bavail * fs.f_frsize < 1.2 * need:
                    raise RuntimeError(f"/dev/shm has less than {1.2 * need / 1e9:.1f} GB free")
                rate_n, procs, desc_n = oracle_rate_all_cores(w, tables, lens, args.cpu_seconds / 2)
                cpu["all_cores"] = {"value": rate_n, "unit": UNIT, "cores": procs, "sample": desc_n}
            except Exception as exc:  # the single-thread figure stands on its own
                cpu["all_cores"] = {"skipped": f"{type(exc).__name__}: {exc}"}

    if dist is not None:
        barrier(dist, device)
        dist.destroy_process_group()
    if rank != 0:
        return 0

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {
            "workload": CONFIG_TEXT[args.config], "name": args.config, "B": w.B, "Hq": w.Hq,
            "Hkv": w.Hkv, "head_dim": w.D, "block_size": w.block_size,
            "num_blocks": w.num_blocks, "mean_seq_len": float(np.mean(lens)),
            "kv_bytes_per_step": kv_bytes, "alg_bytes_per_step": alg_bytes,
            "copy_pairs_per_step": npairs, "decode_plan": plan,
            "step_calls": ("pa_copy_blocks + " if npairs else "") + (
                "pa_decode_append" if fused else "pa_reshape_and_cache + " + (
                    "pa_decode_shared_prefix" if args.shared_prefix else "pa_decode")),
            "internal_waste_slots": int(alloc.internal_waste_slots()),
            "kv_bytes_unique_per_step": unique_kv,
            "l2": "inputs larger than L2 (K/V pools of %.2f GB vs 126 MB L2); not flushed"
                  % (2 * kp.numel() * esize / 1e9),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        },
        "decode_tokens_per_s": tokens_per_s,
        "kernel_kv_gbs": alg_bytes / (dec_avg_ms / 1e3) / 1e9,
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": gpu_launches,
        "clocks": clock_summary,
    }
    if long_line is not None:
        line["long"] = long_line
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
