"""Shared-prefix decode: fork groups read their common prompt blocks once.

The result is plain attention, so the GPU output is checked against the float64
oracle (and against pa_decode) on the same seeded inputs; the grouping helper is
checked for the properties the kernel relies on."""

import numpy as np
import pytest
import torch

import workloads
from _parity import assert_close, gpu_step, oracle_step


def _alloc_after_step(w):
    import paged_kv_cache_350_b200 as pa
    a = pa.Allocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed, pop_order=w.pop_order)
    workloads.run_setup(w, a)  # copy pairs of the setup only matter for pool contents
    workloads.run_step_allocation(w, a)
    return a


@pytest.mark.parametrize("maxm", [2, 4, 8])
def test_prefix_groups_properties(maxm):
    w = workloads.prefix(prompts=3, n=8, prompt_len=100, max_private=40)
    a = _alloc_after_step(w)
    gof, gpre, gmem = a.prefix_groups(w.step_seqs, maxm, 32)
    assert len(gpre) == 3 * (8 // maxm)
    for g in range(len(gpre)):
        members = [int(m) for m in gmem[g] if m >= 0]
        assert 2 <= len(members) <= maxm and gpre[g] % 32 == 0 and gpre[g] > 0
        tabs = [a.block_table(w.step_seqs[m]) for m in members]
        nshared = -(-int(gpre[g]) // w.block_size)
        assert all(t[0][:nshared] == tabs[0][0][:nshared] for t in tabs)
        assert all(int(gpre[g]) <= t[1] for t in tabs)
        assert all(gof[m] == g for m in members)
    assert (gof >= 0).all()
    # an unrelated batch forms no group
    w2 = workloads.gqa(B=6, median=100, lo=1, hi=300)
    a2 = _alloc_after_step(w2)
    gof2, gpre2, _ = a2.prefix_groups(w2.step_seqs, 4, 32)
    assert len(gpre2) == 0 and (gof2 == -1).all()


def _shared_prefix_gpu(w, maxm):
    import paged_kv_cache_350_b200 as pa
    g = gpu_step(w, keep=True)
    gof, gpre, gmem = g["alloc"].prefix_groups(w.step_seqs, maxm, pa.binding.PA_SHARED_PREFIX_ALIGN)
    n = pa.pa_decode_shared_prefix_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.block_size, len(gpre))
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    out = torch.full_like(g["q"], float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_decode_shared_prefix(out, g["q"], g["k_pool"], g["v_pool"], g["t_d"], g["l_d"], w.scale,
                               torch.from_numpy(gof).cuda(),
                               torch.from_numpy(np.ascontiguousarray(gpre) if len(gpre) else np.zeros(1, np.int32)).cuda(),
                               torch.from_numpy(np.ascontiguousarray(gmem).reshape(len(gpre), maxm)).cuda(),
                               ws, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return out, g, len(gpre)


CASES = {
    "prefix_g4_m4": (lambda: workloads.prefix(prompts=3, n=8, prompt_len=150, max_private=60), 4),
    "prefix_g4_m2": (lambda: workloads.prefix(prompts=2, n=8, prompt_len=96, max_private=40), 2),
    "cow_g4_m4": (lambda: workloads.prefix_cow(prompts=2, n=8, prompt_len=100), 4),
    "prefix_g8_m2": (lambda: workloads.prefix(prompts=2, n=4, prompt_len=200, max_private=30,
                                              Hq=16, Hkv=2), 2),
    "prefix_bs8": (lambda: workloads.prefix(prompts=2, n=4, prompt_len=70, max_private=50,
                                            bs=8), 4),
    "prefix_bs32_d64": (lambda: workloads.prefix(prompts=2, n=4, prompt_len=130, max_private=50,
                                                 bs=32, D=64), 4),
    "mixed_no_groups": (lambda: workloads.gqa(B=5, median=100, lo=1, hi=200), 4),
    # whole fork families as one unit: 32 and 64 stacked rows
    "prefix_g4_m8": (lambda: workloads.prefix(prompts=3, n=8, prompt_len=150, max_private=60), 8),
    "prefix_g4_m16": (lambda: workloads.prefix(prompts=2, n=16, prompt_len=130, max_private=70), 16),
    "prefix_g8_m8": (lambda: workloads.prefix(prompts=2, n=8, prompt_len=200, max_private=30,
                                              Hq=16, Hkv=2), 8),
    "cow_g4_m8": (lambda: workloads.prefix_cow(prompts=2, n=8, prompt_len=100), 8),
    "prefix_g1_m32": (lambda: workloads.prefix(prompts=1, n=32, prompt_len=64, max_private=40,
                                               Hq=4, Hkv=4), 32),
    "prefix_bs8_m8": (lambda: workloads.prefix(prompts=2, n=8, prompt_len=70, max_private=50,
                                               bs=8), 8),
    "prefix_bs32_d64_m8": (lambda: workloads.prefix(prompts=2, n=8, prompt_len=130,
                                                    max_private=50, bs=32, D=64), 8),
    # long prompts: units span several CTAs, so cut units are merged across CTAs
    "long_prompt_m8": (lambda: workloads.prefix(prompts=4, n=8, prompt_len=2000,
                                                max_private=300), 8),
    # G = 2 (2 rows a member) and G = 16 (a member fills a sub-partition)
    "prefix_g2_m16": (lambda: workloads.prefix(prompts=2, n=16, prompt_len=140, max_private=60,
                                               Hq=16, Hkv=8), 16),
    "prefix_g16_m4": (lambda: workloads.prefix(prompts=2, n=4, prompt_len=140, max_private=60,
                                               Hq=32, Hkv=2), 4),
    "prefix_g16_m2": (lambda: workloads.prefix(prompts=2, n=4, prompt_len=140, max_private=60,
                                               Hq=32, Hkv=2), 2),
    # units of 64, 36, 24, 12 and 4 rows (and ungrouped sequences) in one launch, so a CTA
    # moves between units whose rows fill different numbers of sub-partitions
    "families_mixed_m16": (lambda: workloads.families(), 16),
    "families_mixed_long_m16": (lambda: workloads.families(seed=1022, sizes=(9, 16, 2, 5),
                                                           solo=4, prompt_len=1500,
                                                           max_private=200), 16),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(CASES))
def test_shared_prefix_matches_oracle_and_pa_decode(name):
    build, maxm = CASES[name]
    w = build()
    out, g, ng = _shared_prefix_gpu(w, maxm)
    if not name.startswith("mixed"):
        assert ng > 0
    r = oracle_step(w)
    assert_close(w, out, r["out"])
    assert_close(w, out, g["out"].float().cpu().numpy(), exact_ref=False)


@pytest.mark.gpu
def test_member_with_no_own_tokens_and_empty_rows():
    """Two rows share every token (prefix == length); one row is empty."""
    import paged_kv_cache_350_b200 as pa
    from oracle import ref_decode
    rng = np.random.default_rng(11)
    B, Hq, Hkv, D, bs, NB = 3, 8, 2, 128, 16, 12
    kp = torch.from_numpy(rng.standard_normal((NB, bs, Hkv, D)).astype(np.float32)).to(torch.bfloat16)
    vp = torch.from_numpy(rng.standard_normal((NB, bs, Hkv, D)).astype(np.float32)).to(torch.bfloat16)
    q = torch.from_numpy(rng.standard_normal((B, Hq, D)).astype(np.float32)).to(torch.bfloat16)
    tables = np.array([[3, 7, 1, 4], [3, 7, 1, 4], [-1, -1, -1, -1]], dtype=np.int32)
    lens = np.array([64, 64, 0], dtype=np.int32)
    h = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    ref = ref_decode(h(q), h(kp), h(vp), tables, lens, 0.1)
    n = pa.pa_decode_shared_prefix_workspace_size(B, Hq, Hkv, D, bs, 1)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    out = torch.full_like(q, float("nan")).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_decode_shared_prefix(out, q.cuda(), kp.cuda(), vp.cuda(), torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens).cuda(), 0.1,
                               torch.tensor([0, 0, -1], dtype=torch.int32, device="cuda"),
                               torch.tensor([64], dtype=torch.int32, device="cuda"),
                               torch.tensor([[0, 1]], dtype=torch.int32, device="cuda"), ws, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert_close(workloads.independent([1]), out, ref)


@pytest.mark.gpu
@pytest.mark.parametrize("all_empty", [False, True])
def test_group_with_no_shared_tokens(all_empty):
    """A group whose prefix is 0 streams only its members' own tokens.  A member of length
    0 gets a zero row; so does every member when all are empty (the group has no tile)."""
    import paged_kv_cache_350_b200 as pa
    from oracle import ref_decode
    rng = np.random.default_rng(12)
    B, Hq, Hkv, D, bs, NB = 4, 8, 2, 128, 16, 16
    kp = torch.from_numpy(rng.standard_normal((NB, bs, Hkv, D)).astype(np.float32)).to(torch.bfloat16)
    vp = torch.from_numpy(rng.standard_normal((NB, bs, Hkv, D)).astype(np.float32)).to(torch.bfloat16)
    q = torch.from_numpy(rng.standard_normal((B, Hq, D)).astype(np.float32)).to(torch.bfloat16)
    tables = np.array([[3, 7, 1, -1], [2, 9, -1, -1], [-1, -1, -1, -1], [5, 11, 0, 4]],
                      dtype=np.int32)
    lens = np.array([0, 0, 0, 50] if all_empty else [40, 21, 0, 50], dtype=np.int32)
    h = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    ref = ref_decode(h(q), h(kp), h(vp), tables, lens, 0.1)
    n = pa.pa_decode_shared_prefix_workspace_size(B, Hq, Hkv, D, bs, 1)
    ws = torch.full((n,), 0xA5, dtype=torch.uint8, device="cuda")
    out = torch.full_like(q, float("nan")).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_decode_shared_prefix(out, q.cuda(), kp.cuda(), vp.cuda(), torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens).cuda(), 0.1,
                               torch.tensor([0, 0, 0, -1], dtype=torch.int32, device="cuda"),
                               torch.tensor([0], dtype=torch.int32, device="cuda"),
                               torch.tensor([[0, 1, 2, -1]], dtype=torch.int32, device="cuda"),
                               ws, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = out.float().cpu().numpy()
    for b in np.flatnonzero(lens == 0):
        assert (got[b] == 0).all()
    assert_close(workloads.independent([1]), out, ref)


@pytest.mark.gpu
def test_shared_prefix_replayed_from_a_cuda_graph():
    """The shared-prefix call captured in a CUDA graph and replayed, on a batch whose units
    span several CTAs (cut units merged across CTAs, through flags tagged per call): a
    replay keeps the call's tag, so the flags must be cleared once consumed.  After a call
    no flag is left set (the flags lead the workspace, one 8-byte word per CTA), and every
    replay, each with new queries, matches an eager call on the same inputs bit for bit."""
    import paged_kv_cache_350_b200 as pa
    w = workloads.prefix(prompts=4, n=8, prompt_len=2000, max_private=300)
    maxm = 8
    _, g, _ = _shared_prefix_gpu(w, maxm)
    gof, gpre, gmem = g["alloc"].prefix_groups(w.step_seqs, maxm, pa.binding.PA_SHARED_PREFIX_ALIGN)
    n = pa.pa_decode_shared_prefix_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.block_size, len(gpre))
    gof_d = torch.from_numpy(gof).cuda()
    gpre_d = torch.from_numpy(np.ascontiguousarray(gpre)).cuda()
    gmem_d = torch.from_numpy(np.ascontiguousarray(gmem).reshape(len(gpre), maxm)).cuda()
    q = g["q"].clone()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def call(out, ws, stream=None):
        pa.pa_decode_shared_prefix(out, q, g["k_pool"], g["v_pool"], g["t_d"], g["l_d"], w.scale,
                                   gof_d, gpre_d, gmem_d, ws, err_flag=err, stream=stream)

    # flags: zero before, zero after (each one set by a later piece is cleared by its owner)
    ws_eager = torch.zeros(n, dtype=torch.uint8, device="cuda")
    ref = torch.empty_like(q)
    call(ref, ws_eager)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ctas = torch.cuda.get_device_properties(0).multi_processor_count
    assert int(ws_eager[: ctas * 8].count_nonzero()) == 0

    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up on the capture stream (first-call setup)
        call(out, ws, stream=s)
    s.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        call(out, ws, stream=s)
    gen = torch.Generator(device="cuda").manual_seed(7700)
    for _ in range(3):
        q.copy_(torch.randn(q.shape, generator=gen, device="cuda", dtype=torch.float32).to(q.dtype))
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        call(ref, ws_eager)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    del graph
