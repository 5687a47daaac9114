"""Multi-step decode with continuous batching: admissions (prefill of the prompt K/V),
forks for parallel sampling (copy on write at the first divergent token), retirements
(blocks back to the pool at refcount 0), and one decode step per live sequence per step.

The product side runs PagedKVCache (C allocator + kernels); the oracle side replays the
same trace with RefAllocator and the float64 functions.  Every step's slots, copy pairs,
tables and lengths must be identical, every step's outputs within tolerance, and the
pools bit-identical at the end."""

import numpy as np
import pytest
import torch

import workloads
from _parity import assert_close
from oracle import RefAllocator, ref_copy_blocks, ref_decode, ref_reshape_and_cache


def _oracle_replay(tr):
    alloc = RefAllocator(tr.num_blocks, tr.block_size, shuffle_seed=tr.alloc_seed)
    kp, vp = tr.pool("k"), tr.pool("v")
    live, outs, plans = [], [], []
    for t, ev in enumerate(tr.events):
        for e in ev:
            if e[0] == "admit":
                alloc.add_seq(e[1], e[2])
                pk, pv = tr.prompt_kv(e[1], e[2])
                kp, vp = ref_reshape_and_cache(pk, pv, kp, vp, np.array(alloc.seq_slots(e[1])))
                live.append(e[1])
            elif e[0] == "fork":
                alloc.fork(e[1], e[2])
                live.append(e[2])
            elif e[0] == "select":
                alloc.beam_select(e[1], e[2])
            elif e[0] == "truncate":
                alloc.truncate(e[1], e[2])
            else:
                alloc.free_seq(e[1])
                live.remove(e[1])
        ids = sorted(live)
        q, nk, nv = tr.step_inputs(t, len(ids))
        slots, pairs = [], []
        for sid in ids:
            slot, src, dst = alloc.append_slot(sid)
            slots.append(slot)
            if src >= 0:
                pairs.append((src, dst))
        kp, vp = ref_copy_blocks(kp, vp, pairs)
        kp, vp = ref_reshape_and_cache(nk, nv, kp, vp, np.array(slots))
        tables = np.full((len(ids), tr.max_blocks), -1, dtype=np.int32)
        lens = np.zeros(len(ids), dtype=np.int32)
        for i, sid in enumerate(ids):
            tab, n = alloc.block_table(sid)
            tables[i, :len(tab)] = tab
            lens[i] = n
        outs.append(ref_decode(q, kp, vp, tables, lens, tr.scale))
        plans.append((np.array(slots), np.array(pairs, dtype=np.int32).reshape(-1, 2), tables, lens))
    return outs, plans, kp, vp, alloc


def test_trace_replay_keeps_allocator_invariants():
    tr = workloads.serving_trace(seed=3101, steps=30)
    _, _, _, _, alloc = _oracle_replay(tr)
    used = {}
    for sid, tab in alloc.tables.items():
        for b in tab:
            used[b] = used.get(b, 0) + 1
    for b in range(tr.num_blocks):
        assert alloc.refcount(b) == used.get(b, 0)
    assert alloc.num_free() + len(used) == tr.num_blocks
    assert any(e[0] == "fork" for ev in tr.events for e in ev)
    assert any(e[0] == "retire" for ev in tr.events for e in ev)


TRACES = {
    "serve_bs16_g8": lambda: workloads.serving_trace(seed=3201, steps=36, bs=16, Hq=16, Hkv=2),
    "serve_bs8_g4": lambda: workloads.serving_trace(seed=3202, steps=36, bs=8, Hq=8, Hkv=2),
    "serve_bs32_g2": lambda: workloads.serving_trace(seed=3203, steps=36, bs=32, Hq=4, Hkv=2),
    "beam_bs16": lambda: workloads.beam_trace(seed=3301, bs=16),
    "beam_bs8": lambda: workloads.beam_trace(seed=3302, bs=8, Hq=8, Hkv=2, prompt_len=20),
}


def test_beam_trace_replay_keeps_allocator_invariants():
    tr = workloads.beam_trace(seed=3401)
    _, _, _, _, alloc = _oracle_replay(tr)
    used = {}
    for sid, tab in alloc.tables.items():
        for b in tab:
            used[b] = used.get(b, 0) + 1
    for b in range(tr.num_blocks):
        assert alloc.refcount(b) == used.get(b, 0)
    assert any(e[0] == "select" for ev in tr.events for e in ev)
    assert any(e[0] == "truncate" for ev in tr.events for e in ev)


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(TRACES))
def test_serving_trace_matches_oracle_replay(name):
    import paged_kv_cache_350_b200 as pa
    tr = TRACES[name]()
    outs, plans, ref_kp, ref_vp, ref_alloc = _oracle_replay(tr)

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)

    def host(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    cache = pa.PagedKVCache(tr.num_blocks, tr.block_size, tr.Hkv, tr.D, shuffle_seed=tr.alloc_seed,
                            k_pool=dev(tr.pool("k")), v_pool=dev(tr.pool("v")))
    live = []
    for t, ev in enumerate(tr.events):
        for e in ev:
            if e[0] == "admit":
                pk, pv = tr.prompt_kv(e[1], e[2])
                cache.admit(e[1], host(pk), host(pv))
                live.append(e[1])
            elif e[0] == "fork":
                cache.fork(e[1], e[2])
                live.append(e[2])
            elif e[0] == "select":
                cache.beam_select(e[1], e[2])
            elif e[0] == "truncate":
                cache.truncate(e[1], e[2])
            else:
                cache.retire(e[1])
                live.remove(e[1])
        ids = sorted(live)
        q, nk, nv = tr.step_inputs(t, len(ids))
        qh, kh, vh = cache.host_inputs(len(ids), tr.Hq, tr.max_blocks)
        qh.copy_(host(q))
        kh.copy_(host(nk))
        vh.copy_(host(nv))
        out, _ = cache.step_staged(ids, tr.scale, tr.max_blocks)
        slots, pairs, tables, lens = plans[t]
        lay = cache._lay
        got_slots = cache._view(cache._hbuf, "slots", (len(ids),), torch.int64).numpy()
        got_tables = cache._view(cache._hbuf, "tables", (len(ids), tr.max_blocks), torch.int32).numpy()
        got_lens = cache._view(cache._hbuf, "lens", (len(ids),), torch.int32).numpy()
        assert np.array_equal(got_slots, slots) and np.array_equal(got_tables, tables)
        assert np.array_equal(got_lens, lens)
        w = workloads.independent([1], dtype="bf16")
        assert_close(w, out.clone(), outs[t])
    cache.check_device_errors()
    kd = cache.k_pool.view(torch.int16).cpu().numpy().view(np.uint16)
    vd = cache.v_pool.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(kd, ref_kp) and np.array_equal(vd, ref_vp)
    assert cache.alloc.free_list() == list(ref_alloc.free)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["serve_bs16_g8", "serve_bs8_g4", "serve_bs32_g2"])
def test_serving_trace_shared_prefix_matches_oracle_replay(name):
    """The same traces through PagedKVCache.step_shared_prefix: each step groups the
    sequences that share a prompt's blocks and reads those blocks once per group.  Every
    step's output matches the oracle replay, the pools end bit-identical and the free list
    equal."""
    import paged_kv_cache_350_b200 as pa
    tr = TRACES[name]()
    outs, _, ref_kp, ref_vp, ref_alloc = _oracle_replay(tr)

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)

    def host(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    cache = pa.PagedKVCache(tr.num_blocks, tr.block_size, tr.Hkv, tr.D, shuffle_seed=tr.alloc_seed,
                            k_pool=dev(tr.pool("k")), v_pool=dev(tr.pool("v")))
    maxm = min(32, 64 // (tr.Hq // tr.Hkv))
    live, groups = [], 0
    w = workloads.independent([1], dtype="bf16")
    for t, ev in enumerate(tr.events):
        for e in ev:
            if e[0] == "admit":
                pk, pv = tr.prompt_kv(e[1], e[2])
                cache.admit(e[1], host(pk), host(pv))
                live.append(e[1])
            elif e[0] == "fork":
                cache.fork(e[1], e[2])
                live.append(e[2])
            elif e[0] == "select":
                cache.beam_select(e[1], e[2])
            elif e[0] == "truncate":
                cache.truncate(e[1], e[2])
            else:
                cache.retire(e[1])
                live.remove(e[1])
        ids = sorted(live)
        q, nk, nv = tr.step_inputs(t, len(ids))
        out = torch.empty((len(ids), tr.Hq, tr.D), dtype=torch.bfloat16).pin_memory()
        cache.step_shared_prefix(ids, host(q).pin_memory(), host(nk).pin_memory(),
                                 host(nv).pin_memory(), out, tr.scale, tr.max_blocks, maxm)
        groups += cache.last_prefix_groups
        assert_close(w, out.clone(), outs[t])
    assert groups > 0
    cache.check_device_errors()
    kd = cache.k_pool.view(torch.int16).cpu().numpy().view(np.uint16)
    vd = cache.v_pool.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(kd, ref_kp) and np.array_equal(vd, ref_vp)
    assert cache.alloc.free_list() == list(ref_alloc.free)


@pytest.mark.gpu
@pytest.mark.parametrize("wl, members", [("cow", 0), ("cow", 8), ("solo", 4)])
@pytest.mark.parametrize("depth", [1, 2, 3])
def test_step_pipeline_matches_oracle_step_by_step(depth, wl, members):
    """StepPipeline: steps queued back to back over `depth` staging slots, with different
    inputs every step and copy-on-write in the first; each step's output (read one step
    late, as a serving loop would) must match the oracle, the final pools bit for bit.
    members > 0: the shared-prefix steps (fork groups of up to `members` samples; "solo":
    unforked sequences, so that no group forms in any step)."""
    import paged_kv_cache_350_b200 as pa
    w = (workloads.prefix_cow(prompts=2, prompt_len=100) if wl == "cow"
         else workloads.gqa(B=6, median=100, lo=1, hi=200))
    steps = 7
    MB = w.max_blocks + steps // w.block_size + 2
    B = len(w.step_seqs)

    def draws(t):
        shapes = ((B, w.Hq, w.D), (B, w.Hkv, w.D), (B, w.Hkv, w.D))
        return [workloads.draw_normal(s, w.seed + 17, 5000 + 3 * t + i, w.dtype)
                for i, s in enumerate(shapes)]

    # oracle replay
    ref = RefAllocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed, pop_order=w.pop_order)
    kp, vp = ref_copy_blocks(w.k_pool(), w.v_pool(), workloads.run_setup(w, ref))
    outs = []
    for t in range(steps):
        q, nk, nv = draws(t)
        slots, pairs = [], []
        for sid in w.step_seqs:
            slot, src, dst = ref.append_slot(sid)
            slots.append(slot)
            if src >= 0:
                pairs.append((src, dst))
        if t == 0 and wl == "cow":
            assert pairs, "the first step copies on write"
        kp, vp = ref_copy_blocks(kp, vp, pairs)
        kp, vp = ref_reshape_and_cache(nk, nv, kp, vp, np.array(slots))
        tables = np.full((B, MB), -1, dtype=np.int32)
        lens = np.zeros(B, dtype=np.int32)
        for i, sid in enumerate(w.step_seqs):
            tab, n = ref.block_table(sid)
            tables[i, :len(tab)] = tab
            lens[i] = n
        outs.append(ref_decode(q, kp, vp, tables, lens, w.scale))

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)

    cache = pa.PagedKVCache(w.num_blocks, w.block_size, w.Hkv, w.D, shuffle_seed=w.alloc_seed,
                            pop_order=w.pop_order, k_pool=dev(w.k_pool()), v_pool=dev(w.v_pool()))
    setup_pairs = workloads.run_setup(w, cache.alloc)
    pa.pa_copy_blocks(cache.k_pool, cache.v_pool,
                      torch.tensor(setup_pairs, dtype=torch.int32, device="cuda").reshape(-1, 2))
    pipe = cache.pipeline(B, w.Hq, MB, depth=depth, shared_prefix_members=members)
    got = []
    lag = min(1, depth - 1)  # a slot holds its output until it is reused
    for t in range(steps):
        qh, kh, vh = pipe.inputs()
        for dst, src in zip((qh, kh, vh), draws(t)):
            dst.copy_(torch.from_numpy(np.ascontiguousarray(src).view(np.int16)).view(torch.bfloat16))
        assert pipe.submit(w.step_seqs, w.scale) == t
        if t >= lag:
            got.append(pipe.result(t - lag).clone())
    for t in range(steps - lag, steps):
        got.append(pipe.result(t).clone())
    pipe.sync()
    cache.check_device_errors()
    for t in range(steps):
        assert_close(w, got[t], outs[t])
    assert np.array_equal(cache.k_pool.view(torch.int16).cpu().numpy().view(np.uint16), kp)
    assert np.array_equal(cache.v_pool.view(torch.int16).cpu().numpy().view(np.uint16), vp)
