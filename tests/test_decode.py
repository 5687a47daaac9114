"""GPU parity of pa_decode against the float64 oracle (through the C ABI).

Tolerances: bf16 max-abs <= 1e-2 and max row-normwise relative <= 2e-2;
fp32 inputs max-abs <= 1e-4.  The three invariants are checked bit-exactly
on the GPU: the kernels' arithmetic order depends only on the logical token
order and the sequence lengths.
"""

import numpy as np
import pytest
import torch

import workloads
from _parity import assert_close, gpu_step, oracle_step, to_device
from oracle import ref_decode

pytestmark = pytest.mark.gpu

AUTO, GENERIC, TENSOR = 0, 1, 2


def check(w, partition_tokens=0, path=AUTO, max_ctas=0):
    g = gpu_step(w, partition_tokens=partition_tokens, path=path, max_ctas=max_ctas)
    r = oracle_step(w)
    assert g["err"] == 0
    np.testing.assert_array_equal(g["slots"], r["slots"])
    np.testing.assert_array_equal(g["tables"], r["tables"])
    return assert_close(w, g["out"], r["out"])


# ---- the tiny fp32 case (CUDA-core path) -------------------------------------

@pytest.mark.parametrize("worked", [False, True])
@pytest.mark.parametrize("partition", [0, 4, 8])
def test_tiny_fp32(worked, partition):
    check(workloads.tiny(worked_example=worked), partition_tokens=partition)


# ---- scaled-down versions of the serving workloads ------------------------------

SCALED = {
    "mha": lambda: workloads.mha(B=6, lo=1, hi=300),
    "gqa": lambda: workloads.gqa(B=12, median=200, lo=1, hi=700),
    "long": lambda: workloads.long_context(B=2, lo=1500, hi=5000),
    "prefix": lambda: workloads.prefix(prompts=2, prompt_len=96, max_private=40),
    "prefix_cow": lambda: workloads.prefix_cow(prompts=2, prompt_len=100),
}


@pytest.mark.parametrize("name", sorted(SCALED))
@pytest.mark.parametrize("partition,path,ctas", [(0, AUTO, 0), (0, TENSOR, 1), (0, TENSOR, 3),
                                                 (0, TENSOR, 37), (16, TENSOR, 0), (64, TENSOR, 0),
                                                 (0, GENERIC, 0), (32, GENERIC, 0)])
def test_scaled_workloads(name, partition, path, ctas):
    """AUTO/TENSOR with partition 0 run the balanced stream kernel (max_ctas varies where
    the tile ranges cut units); partition > 0 runs the partition kernels."""
    check(SCALED[name](), partition_tokens=partition, path=path, max_ctas=ctas)


# ---- lengths around block and tile boundaries ---------------------------------

EDGE_LENS = [1, 2, 15, 16, 17, 31, 32, 33, 47, 48, 49, 63, 64, 65, 127, 129]


@pytest.mark.parametrize("bs", [8, 16, 32])
@pytest.mark.parametrize("G", [1, 2, 4, 8, 12, 16])
def test_edge_lengths_tensor_path(bs, G):
    w = workloads.independent(EDGE_LENS, Hq=2 * G, Hkv=2, bs=bs, seed=3000 + bs + G)
    check(w, path=TENSOR)
    check(w, path=TENSOR, max_ctas=2)
    check(w, partition_tokens=32, path=TENSOR)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("bs", [4, 16])
def test_edge_lengths_generic_path(D, dtype, bs):
    w = workloads.independent(EDGE_LENS, Hq=6, Hkv=2, D=D, bs=bs, dtype=dtype, seed=4000 + D + bs)
    check(w, path=GENERIC)
    check(w, partition_tokens=2 * bs, path=GENERIC)


def test_head_dim_64_tensor_path():
    w = workloads.independent([5, 70, 300, 33], Hq=16, Hkv=2, D=64, bs=16, seed=4100)
    check(w, path=TENSOR)
    check(w, path=TENSOR, max_ctas=1)
    check(w, partition_tokens=64, path=TENSOR)


def test_gqa_group_wider_than_16_uses_cuda_cores():
    w = workloads.independent([40, 9], Hq=32, Hkv=1, bs=16, seed=4200)
    check(w)  # auto path -> CUDA-core path


# ---- direct decode cases (no allocator): empty rows, poisoned slots, logits ----

def _decode_direct(q, kp, vp, tables, lens, scale, path=AUTO, partition=0, dev="cuda", max_ctas=0):
    import paged_kv_cache_350_b200 as pa
    out = torch.full_like(q, float("nan"))
    B, Hq, D = q.shape
    bs, Hkv = kp.shape[1], kp.shape[2]
    n = pa.pa_decode_workspace_size(B, Hq, Hkv, D, tables.shape[1] * bs, bs, partition)
    ws = torch.empty(max(n, 1), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pa.pa_decode(out, q, kp, vp, tables, lens, scale, workspace=ws, err_flag=err,
                 partition_tokens=partition, path=path, max_ctas=max_ctas)
    torch.cuda.synchronize()
    return out, int(err.item())


def _bf16_host(t):
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("path,partition,ctas", [(TENSOR, 0, 0), (TENSOR, 0, 1), (TENSOR, 16, 0),
                                                 (GENERIC, 0, 0), (GENERIC, 16, 0)])
def test_empty_rows_poisoned_tails_and_minus_one_tables(path, partition, ctas):
    rng = np.random.default_rng(5)
    B, Hq, Hkv, D, bs, NB = 6, 8, 2, 128, 16, 40
    lens = np.array([0, 1, 17, 0, 33, 50], dtype=np.int32)
    perm = rng.permutation(NB)
    MB = 6
    tables = np.full((B, MB), -1, dtype=np.int32)
    k = 0
    for b, L in enumerate(lens):
        n = -(-int(L) // bs)
        tables[b, :n] = perm[k:k + n]
        k += n
    q = torch.randn(B, Hq, D).to(torch.bfloat16)
    kp = torch.randn(NB, bs, Hkv, D).to(torch.bfloat16)
    vp = torch.randn(NB, bs, Hkv, D).to(torch.bfloat16)
    ref = ref_decode(_bf16_host(q), _bf16_host(kp), _bf16_host(vp), tables, lens, 0.088)
    # poison every slot no sequence uses, including the tails of the last blocks
    used = np.zeros((NB, bs), dtype=bool)
    for b, L in enumerate(lens):
        for t in range(int(L)):
            used[tables[b, t // bs], t % bs] = True
    mask = torch.from_numpy(~used)
    kp[mask] = float("nan")
    vp[mask] = float("inf")
    out, err = _decode_direct(q.cuda(), kp.cuda(), vp.cuda(), torch.from_numpy(tables).cuda(),
                              torch.from_numpy(lens).cuda(), 0.088, path=path, partition=partition,
                              max_ctas=ctas)
    assert err == 0
    w = workloads.independent([1], dtype="bf16")
    assert_close(w, out, ref)
    assert torch.equal(out[0].float().cpu(), torch.zeros(Hq, D))


@pytest.mark.parametrize("path,ctas", [(TENSOR, 0), (TENSOR, 1), (GENERIC, 0)])
def test_large_logits_and_rising_logits_force_rescaling(path, ctas):
    rng = np.random.default_rng(6)
    B, Hq, Hkv, D, bs = 2, 8, 1, 128, 16
    L = 300
    NB = 2 * (-(-L // bs))
    u = rng.standard_normal(D)
    u /= np.linalg.norm(u)
    kp = rng.standard_normal((NB, bs, Hkv, D)) * 0.1
    # sequence 0: logits rise along the sequence, so the running max changes at every tile
    for t in range(L):
        kp[t // bs, t % bs, 0] += u * (t / 10.0)
    vp = rng.standard_normal((NB, bs, Hkv, D))
    q = rng.standard_normal((B, Hq, D))
    q[0] = u * 8.0
    q[1] *= 30.0          # huge logits for sequence 1
    tables = np.arange(NB, dtype=np.int32).reshape(B, -1)
    tables[1] = np.arange(NB // 2, NB)
    lens = np.array([L, L], dtype=np.int32)
    tq, tk, tv = (torch.from_numpy(x).to(torch.bfloat16) for x in (q, kp, vp))
    ref = ref_decode(_bf16_host(tq), _bf16_host(tk), _bf16_host(tv), tables, lens, 1.0)
    out, err = _decode_direct(tq.cuda(), tk.cuda(), tv.cuda(), torch.from_numpy(tables).cuda(),
                              torch.from_numpy(lens).cuda(), 1.0, path=path,
                              partition=0 if path == TENSOR else 64, max_ctas=ctas)
    assert err == 0 and torch.isfinite(out.float()).all()
    assert_close(workloads.independent([1]), out, ref)


# ---- invariants, bit-exact on the GPU ---------------------------------------

@pytest.mark.parametrize("path", [TENSOR, GENERIC])
def test_block_permutation_invariant_bitwise(path):
    w = SCALED["gqa"]()
    g = gpu_step(w, path=path, keep=True)
    NB = w.num_blocks
    perm = torch.from_numpy(np.random.default_rng(7).permutation(NB)).cuda()
    kp2 = torch.empty_like(g["k_pool"])
    vp2 = torch.empty_like(g["v_pool"])
    kp2[perm] = g["k_pool"]
    vp2[perm] = g["v_pool"]
    t = g["t_d"].long()
    t2 = torch.where(t >= 0, perm[t.clamp(min=0)], t).int()
    out2, err = _decode_direct(g["q"], kp2, vp2, t2, g["l_d"], w.scale, path=path)
    assert err == 0 and torch.equal(out2, g["out"])


@pytest.mark.parametrize("path", [TENSOR, GENERIC])
def test_shared_prefix_equals_private_copies_bitwise(path):
    w = SCALED["prefix"]()
    g = gpu_step(w, path=path, keep=True)
    tables = g["t_d"].clone()
    kp, vp = g["k_pool"].clone(), g["v_pool"].clone()
    # give every sample its own copy of the shared prompt blocks (appended to the pool)
    nshared = w.meta["prompt_len"] // w.block_size
    extra = []
    for row in range(w.B):
        for j in range(nshared):
            src = int(tables[row, j])
            extra.append(src)
            tables[row, j] = w.num_blocks + len(extra) - 1
    idx = torch.tensor(extra, device="cuda")
    kp = torch.cat([kp, kp[idx]])
    vp = torch.cat([vp, vp[idx]])
    out2, err = _decode_direct(g["q"], kp, vp, tables, g["l_d"], w.scale, path=path)
    assert err == 0 and torch.equal(out2, g["out"])


@pytest.mark.parametrize("path", [TENSOR, GENERIC])
def test_copy_on_write_leaves_sibling_bitwise_unchanged(path):
    import paged_kv_cache_350_b200 as pa
    w = workloads.prefix_cow(prompts=1, prompt_len=100)
    alloc = pa.Allocator(w.num_blocks, w.block_size, shuffle_seed=w.alloc_seed)
    workloads.run_setup(w, alloc)
    kp, vp = to_device(w.k_pool(), w), to_device(w.v_pool(), w)
    q = to_device(w.q(), w)[:1]
    sib = 7  # the sibling that will not write

    def decode_sibling():
        t, n = alloc.block_table(sib)
        tab = torch.tensor([t + [-1] * (w.max_blocks - len(t))], dtype=torch.int32, device="cuda")
        out, err = _decode_direct(q, kp, vp, tab, torch.tensor([n], dtype=torch.int32, device="cuda"),
                                  w.scale, path=path)
        assert err == 0
        return out

    before = decode_sibling()
    slot, src, dst = alloc.append_slot(0)      # sample 0 diverges first: copy on write
    assert src >= 0
    pa.pa_copy_blocks(kp, vp, torch.tensor([[src, dst]], dtype=torch.int32, device="cuda"))
    nk = torch.randn(1, w.Hkv, w.D, device="cuda").to(torch.bfloat16)
    pa.pa_reshape_and_cache(nk, nk, kp, vp, torch.tensor([slot], device="cuda"))
    assert torch.equal(decode_sibling(), before)


# ---- corrupted inputs raise the device flag and never fault -----------------------

def test_bad_block_id_and_bad_length_set_the_flag():
    import paged_kv_cache_350_b200 as pa
    B, Hq, Hkv, D, bs, NB = 2, 4, 1, 128, 16, 8
    q = torch.randn(B, Hq, D, device="cuda").to(torch.bfloat16)
    kp = torch.randn(NB, bs, Hkv, D, device="cuda").to(torch.bfloat16)
    vp = torch.randn_like(kp)
    tables = torch.tensor([[0, 99, 1], [2, 3, -7]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([40, 30], dtype=torch.int32, device="cuda")
    for path, part in ((TENSOR, 0), (TENSOR, 16), (GENERIC, 0)):
        out, err = _decode_direct(q, kp, vp, tables, lens, 0.1, path=path, partition=part)
        assert err & pa.binding.PA_DEVERR_BAD_BLOCK_ID
        assert pa.pa_status_from_device_flag(err) == pa.binding.PA_ERR_BAD_BLOCK_ID
        out, err = _decode_direct(q, kp, vp, tables[:, :1].contiguous(),
                                  torch.tensor([17, -1], dtype=torch.int32, device="cuda"), 0.1,
                                  path=path, partition=part)
        assert err & pa.binding.PA_DEVERR_BAD_SEQ_LEN


def test_bounded_wait_runs_out_sets_the_flag_and_the_context_survives():
    """Failure detection on the GPU without a fault: a wait on a barrier phase nothing
    completes (the decode kernels' bounded wait, limited to 20 ms) ends with
    PA_DEVERR_TIMEOUT; afterwards the same context runs a decode correctly."""
    import time
    import paged_kv_cache_350_b200 as pa
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    pa.binding.pa_selftest_bounded_wait(err, 20000)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert int(err.item()) == pa.binding.PA_DEVERR_TIMEOUT
    assert pa.pa_status_from_device_flag(int(err.item())) == pa.binding.PA_ERR_TIMEOUT
    check(SCALED["gqa"](), path=TENSOR)
