"""GPU: pa_reshape_and_cache and pa_copy_blocks are bit-exact against the oracle
over the whole pools (untouched blocks included)."""

import numpy as np
import pytest
import torch

from oracle import ref_copy_blocks, ref_reshape_and_cache

pytestmark = pytest.mark.gpu


def _pools(rng, NB, bs, Hkv, D, dtype):
    k = torch.from_numpy(rng.standard_normal((NB, bs, Hkv, D)).astype(np.float32)).to(dtype)
    v = torch.from_numpy(rng.standard_normal((NB, bs, Hkv, D)).astype(np.float32)).to(dtype)
    return k, v


def _np(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("bs,Hkv,D,T", [(16, 8, 128, 256), (4, 4, 64, 37), (32, 2, 64, 70000),
                                        (8, 1, 128, 1)])
def test_reshape_and_cache_bit_exact(dtype, bs, Hkv, D, T):
    import paged_kv_cache_350_b200 as pa
    rng = np.random.default_rng(T + bs)
    NB = max(8, -(-T * 2 // bs))
    kp, vp = _pools(rng, NB, bs, Hkv, D, dtype)
    key = torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)).to(dtype)
    val = torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)).to(dtype)
    slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int64)
    slots[rng.random(T) < 0.1] = -1                     # skipped tokens
    ek, ev = ref_reshape_and_cache(_np(key), _np(val), _np(kp), _np(vp), slots)
    kd, vd = kp.cuda(), vp.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_reshape_and_cache(key.cuda(), val.cuda(), kd, vd, torch.from_numpy(slots).cuda(),
                            err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(_np(kd), ek) and np.array_equal(_np(vd), ev)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("bs,Hkv,D,n", [(16, 8, 128, 224), (4, 4, 64, 3), (32, 1, 64, 1)])
def test_copy_blocks_bit_exact(dtype, bs, Hkv, D, n):
    import paged_kv_cache_350_b200 as pa
    rng = np.random.default_rng(n)
    NB = 3 * n + 5
    kp, vp = _pools(rng, NB, bs, Hkv, D, dtype)
    ids = rng.permutation(NB)
    pairs = np.stack([ids[:n], ids[n:2 * n]], axis=1).astype(np.int32)   # disjoint src / dst
    ek, ev = ref_copy_blocks(_np(kp), _np(vp), [tuple(p) for p in pairs])
    kd, vd = kp.cuda(), vp.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_copy_blocks(kd, vd, torch.from_numpy(pairs).cuda(), err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(_np(kd), ek) and np.array_equal(_np(vd), ev)


def test_bad_slot_and_bad_pair_set_the_flag_and_write_nothing():
    import paged_kv_cache_350_b200 as pa
    kp = torch.zeros(4, 16, 2, 64, dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    key = torch.ones(2, 2, 64, dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_reshape_and_cache(key, key, kp, vp, torch.tensor([64, 10**12], device="cuda"), err_flag=err)
    pa.pa_copy_blocks(kp, vp, torch.tensor([[0, 4], [-1, 2]], dtype=torch.int32, device="cuda"),
                      err_flag=err)
    torch.cuda.synchronize()
    f = int(err.item())
    assert f & pa.binding.PA_DEVERR_BAD_SLOT and f & pa.binding.PA_DEVERR_BAD_BLOCK_ID
    assert int(torch.count_nonzero(kp.float())) == 0 and int(torch.count_nonzero(vp.float())) == 0
