"""GPU parity of pa_decode_append (cache write fused into the decode) against the oracle.

The oracle side is the unfused definition: the allocator reserves each row's slot,
``ref_reshape_and_cache`` writes the new K/V there and ``ref_decode`` attends.  The
GPU side passes no slots: the kernel derives each row's slot from its block table and
length.  Outputs are held to the decode tolerances; the pools must match bit for bit.
"""

import numpy as np
import pytest
import torch

import workloads
from _parity import assert_close, gpu_step, oracle_bits, oracle_step, pool_bits
from oracle import ref_decode, ref_reshape_and_cache

pytestmark = pytest.mark.gpu

AUTO, GENERIC, TENSOR = 0, 1, 2


def check_fused(w, partition_tokens=0, path=AUTO, max_ctas=0):
    g = gpu_step(w, partition_tokens=partition_tokens, path=path, max_ctas=max_ctas, keep=True,
                 fused=True)
    r = oracle_step(w)
    assert g["err"] == 0
    np.testing.assert_array_equal(g["tables"], r["tables"])
    np.testing.assert_array_equal(pool_bits(g["k_pool"]), oracle_bits(r["k_pool"], w))
    np.testing.assert_array_equal(pool_bits(g["v_pool"]), oracle_bits(r["v_pool"], w))
    return assert_close(w, g["out"], r["out"])


SCALED = {
    "mha": lambda: workloads.mha(B=6, lo=1, hi=300),
    "gqa": lambda: workloads.gqa(B=12, median=200, lo=1, hi=700),
    "long": lambda: workloads.long_context(B=2, lo=1500, hi=5000),
    "prefix": lambda: workloads.prefix(prompts=2, prompt_len=96, max_private=40),
    "prefix_cow": lambda: workloads.prefix_cow(prompts=2, prompt_len=100),
}


@pytest.mark.parametrize("worked", [False, True])
def test_tiny_fp32_append_kernel_then_generic(worked):
    check_fused(workloads.tiny(worked_example=worked))


@pytest.mark.parametrize("name", sorted(SCALED))
@pytest.mark.parametrize("partition,path,ctas", [(0, AUTO, 0), (0, TENSOR, 1), (0, TENSOR, 37),
                                                 (64, TENSOR, 0), (0, GENERIC, 0)])
def test_scaled_workloads_fused(name, partition, path, ctas):
    """AUTO/TENSOR with partition 0: the stream kernel writes the token itself; the
    partition and CUDA-core paths run the append kernel first."""
    check_fused(SCALED[name](), partition_tokens=partition, path=path, max_ctas=ctas)


EDGE_LENS = [1, 2, 15, 16, 17, 31, 32, 33, 47, 48, 49, 63, 64, 65, 127, 129]


@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("G", [1, 4, 12, 16])
@pytest.mark.parametrize("D", [64, 128])
def test_edge_lengths_fused_stream_kernel(bs, G, D):
    """The new token at every offset of a stage (first, last, middle row; first and last
    block of a stage), with streams cut inside units (max_ctas 2)."""
    w = workloads.independent(EDGE_LENS, Hq=2 * G, Hkv=2, D=D, bs=bs, seed=5000 + bs + G + D)
    check_fused(w, path=TENSOR)
    check_fused(w, path=TENSOR, max_ctas=2)


@pytest.mark.parametrize("name", ["gqa", "prefix_cow"])
@pytest.mark.parametrize("path,partition", [(TENSOR, 0), (TENSOR, 64), (GENERIC, 0)])
def test_fused_equals_unfused_bitwise(name, path, partition):
    """The fused call computes exactly what reshape_and_cache + pa_decode compute."""
    w = SCALED[name]()
    a = gpu_step(w, path=path, partition_tokens=partition, keep=True)
    b = gpu_step(w, path=path, partition_tokens=partition, keep=True, fused=True)
    assert a["err"] == 0 and b["err"] == 0
    assert torch.equal(a["out"], b["out"])
    assert torch.equal(a["k_pool"], b["k_pool"]) and torch.equal(a["v_pool"], b["v_pool"])


def _bf16_host(t):
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _direct(q, nk, nv, kp, vp, tables, lens, scale, path, partition=0, max_ctas=0):
    import paged_kv_cache_350_b200 as pa
    B, Hq, D = q.shape
    bs, Hkv = kp.shape[1], kp.shape[2]
    n = pa.pa_decode_workspace_size(B, Hq, Hkv, D, tables.shape[1] * bs, bs, partition)
    ws = torch.empty(max(n, 1), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    pa.pa_decode_append(out, q, nk, nv, kp, vp, tables, lens, scale, workspace=ws, err_flag=err,
                        partition_tokens=partition, path=path, max_ctas=max_ctas)
    torch.cuda.synchronize()
    return out, int(err.item())


@pytest.mark.parametrize("path,partition,ctas", [(TENSOR, 0, 0), (TENSOR, 0, 1), (TENSOR, 16, 0),
                                                 (GENERIC, 0, 0)])
def test_zero_length_rows_write_nothing(path, partition, ctas):
    rng = np.random.default_rng(11)
    B, Hq, Hkv, D, bs, NB = 5, 8, 2, 128, 16, 30
    lens = np.array([0, 1, 16, 0, 33], dtype=np.int32)
    perm = rng.permutation(NB)
    MB = 4
    tables = np.full((B, MB), -1, dtype=np.int32)
    k = 0
    for b, L in enumerate(lens):
        n = -(-int(L) // bs)
        tables[b, :n] = perm[k:k + n]
        k += n
    q = torch.randn(B, Hq, D).to(torch.bfloat16)
    nk = torch.randn(B, Hkv, D).to(torch.bfloat16)
    nv = torch.randn(B, Hkv, D).to(torch.bfloat16)
    kp = torch.randn(NB, bs, Hkv, D).to(torch.bfloat16)
    vp = torch.randn(NB, bs, Hkv, D).to(torch.bfloat16)
    slots = np.array([-1 if L == 0 else tables[b, (L - 1) // bs] * bs + (L - 1) % bs
                      for b, L in enumerate(lens)], dtype=np.int64)
    rk, rv = ref_reshape_and_cache(_bf16_host(nk), _bf16_host(nv), _bf16_host(kp),
                                   _bf16_host(vp), slots)
    ref = ref_decode(_bf16_host(q), rk, rv, tables, lens, 0.09)
    kd, vd = kp.cuda(), vp.cuda()
    out, err = _direct(q.cuda(), nk.cuda(), nv.cuda(), kd, vd, torch.from_numpy(tables).cuda(),
                       torch.from_numpy(lens).cuda(), 0.09, path, partition, ctas)
    assert err == 0
    assert_close(workloads.independent([1]), out, ref)
    assert torch.equal(out[0].float().cpu(), torch.zeros(Hq, D))
    np.testing.assert_array_equal(kd.view(torch.int16).cpu().numpy().view(np.uint16), rk)
    np.testing.assert_array_equal(vd.view(torch.int16).cpu().numpy().view(np.uint16), rv)


def test_bad_table_entry_and_bad_length_write_nothing_and_flag():
    import paged_kv_cache_350_b200 as pa
    B, Hq, Hkv, D, bs, NB = 2, 4, 1, 128, 16, 8
    q = torch.randn(B, Hq, D, device="cuda").to(torch.bfloat16)
    nk = torch.randn(B, Hkv, D, device="cuda").to(torch.bfloat16)
    kp = torch.randn(NB, bs, Hkv, D, device="cuda").to(torch.bfloat16)
    vp = torch.randn_like(kp)
    # row 0's token lands in logical block 2, whose entry is out of range; row 1 is fine
    tables = torch.tensor([[0, 1, 99], [2, 3, -1]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([40, 30], dtype=torch.int32, device="cuda")
    for path, part in ((TENSOR, 0), (TENSOR, 16), (GENERIC, 0)):
        k0, v0 = kp.clone(), vp.clone()
        out, err = _direct(q, nk, nk, k0, v0, tables, lens, 0.1, path, part)
        assert err & pa.binding.PA_DEVERR_BAD_BLOCK_ID
        # only row 1's slot (block 3, offset 13) changed
        changed = (k0 != kp).any(dim=-1).any(dim=-1).nonzero().tolist()
        assert changed == [[3, 13]]
        assert torch.equal(k0[3, 13], nk[1]) and torch.equal(v0[3, 13], nk[1])
        # a length beyond max_blocks * block_size: flagged, nothing written
        k1 = kp.clone()
        out, err = _direct(q, nk, nk, k1, vp.clone(), tables[:, :1].contiguous(),
                           torch.tensor([17, 5], dtype=torch.int32, device="cuda"), 0.1, path,
                           part)
        assert err & pa.binding.PA_DEVERR_BAD_SEQ_LEN
        assert (k1 != kp).any(dim=-1).any(dim=-1).nonzero().tolist() == [[2, 4]]



def test_workspace_contents_do_not_matter():
    """The workspace needs no initialisation: NaN- or garbage-filled, the result is the
    same bit for bit as with a zeroed one (every word a call reads it writes first)."""
    import paged_kv_cache_350_b200 as pa
    w = SCALED["gqa"]()
    g = gpu_step(w, keep=True, fused=True, max_ctas=5)  # few CTAs: many cut units
    outs = []
    for fill in (0, 0xFF, 0x7F):
        ws = torch.full_like(g["ws"], fill)
        kp, vp = g["k_pool"].clone(), g["v_pool"].clone()
        out = torch.empty_like(g["q"])
        nk, nv = g["nk"], g["nv"]
        pa.pa_decode_append(out, g["q"], nk, nv, kp, vp, g["t_d"], g["l_d"], w.scale,
                            workspace=ws, max_ctas=5)
        torch.cuda.synchronize()
        outs.append(out)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    assert torch.equal(outs[0], g["out"])


def test_step_replayed_from_a_cuda_graph():
    """One fused decode step captured in a CUDA graph and replayed: every replay gives the
    eager call's output bit for bit (the cache write is idempotent for a repeated step)."""
    import paged_kv_cache_350_b200 as pa
    w = SCALED["gqa"]()
    g = gpu_step(w, keep=True, fused=True)
    kp, vp = g["k_pool"], g["v_pool"]
    out = torch.empty_like(g["q"])
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up on the capture stream (first-call setup)
        pa.pa_decode_append(out, g["q"], g["nk"], g["nv"], kp, vp, g["t_d"], g["l_d"], w.scale,
                            workspace=g["ws"], err_flag=err, stream=s)
    s.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        pa.pa_decode_append(out, g["q"], g["nk"], g["nv"], kp, vp, g["t_d"], g["l_d"], w.scale,
                            workspace=g["ws"], err_flag=err, stream=s)
    for _ in range(3):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert torch.equal(out, g["out"])
    del graph


def test_plan_on_b200_takes_the_stream_kernel_for_every_block_size():
    import paged_kv_cache_350_b200 as pa
    for bs in (8, 16, 32):
        n = pa.pa_decode_workspace_size(256, 32, 8, 128, 4096, bs, 0)
        plan = pa.pa_decode_plan(256, 32, 8, 128, bs, 4096 // bs, pa.PA_BF16, n)
        assert plan["kernel"] == pa.binding.PA_KERNEL_TC_STREAM
        assert plan["launches"] == 2  # the kernel and its cut-unit reduce
        assert plan["grid"] % torch.cuda.get_device_properties(0).multi_processor_count == 0


def test_batch_beyond_the_stream_kernel_limit():
    """B > 8192 (the balanced kernel's prefix sums live in shared memory): the plan falls
    back to the partition kernel, and the fused call to the append kernel + that decode."""
    import paged_kv_cache_350_b200 as pa
    rng = np.random.default_rng(4400)
    lens = rng.integers(1, 41, size=8200)
    w = workloads.independent(lens, Hq=8, Hkv=2, bs=16, seed=4401)
    n = pa.pa_decode_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.max_blocks * w.block_size,
                                    w.block_size, 0)
    plan = pa.pa_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.block_size, w.max_blocks, pa.PA_BF16, n)
    assert plan["kernel"] == pa.binding.PA_KERNEL_TC_PARTITION
    check_fused(w)
