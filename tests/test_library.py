"""CPU: the C-ABI library loads, exports every symbol include/pa.h declares, and
rejects bad arguments on the host before touching a GPU."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    from paged_kv_cache_350_b200 import binding
    syms = declared_symbols()
    assert len(syms) >= 20
    for s in syms:
        assert hasattr(binding.lib, s), s
    assert sorted(binding.EXPORTED) == syms


def test_status_strings_and_flag_mapping():
    from paged_kv_cache_350_b200 import binding as b
    for s in range(13):
        assert b.lib.pa_status_string(s) != b"unknown status"
    assert b.lib.pa_status_string(b.PA_ERR_HOST_MEMORY) == b"out of host memory"
    assert b.lib.pa_status_string(99) == b"unknown status"
    assert b.lib.pa_status_from_device_flag(0) == b.PA_OK
    assert b.lib.pa_status_from_device_flag(b.PA_DEVERR_BAD_BLOCK_ID | 8) == b.PA_ERR_BAD_BLOCK_ID
    assert b.lib.pa_status_from_device_flag(b.PA_DEVERR_TIMEOUT) == b.PA_ERR_TIMEOUT


def test_workspace_size_bounds_every_partition():
    from paged_kv_cache_350_b200 import binding as b
    assert b.pa_decode_workspace_size(8, 64, 8, 128, 512, 4, 0) == 0     # CUDA cores, one pass
    n0 = b.pa_decode_workspace_size(256, 32, 8, 128, 4096, 16, 0)
    parts = 4096 // 512
    assert n0 >= 256 * 32 * parts * (128 + 2) * 4
    assert b.pa_decode_workspace_size(2, 4, 4, 64, 64, 4, 4) >= 2 * 4 * 16 * 66 * 4
    # the balanced kernel needs room for two partial pieces per stream, whatever B
    assert b.pa_decode_workspace_size(1, 8, 1, 128, 16, 16, 0) >= 4 * 2 * 8 * 130 * 4
    with pytest.raises(b.PAError):
        b.pa_decode_workspace_size(2, 4, 4, 64, 64, 4, 6)   # not a multiple of block_size
    with pytest.raises(b.PAError):
        b.pa_decode_workspace_size(2, 6, 4, 64, 64, 4, 0)   # Hq % Hkv


def _call_decode(**kw):
    from paged_kv_cache_350_b200 import binding as b
    a = dict(out=16, q=16, k=16, v=16, t=16, l=16, B=2, Hq=8, Hkv=2, D=128, bs=16, MB=4, NB=8,
             scale=0.1, dtype=b.PA_BF16, ws=0, wsb=0, err=0, stream=0, part=0, path=0)
    a.update(kw)
    opts = b.pa_decode_opts(a["part"], a["path"], 0)
    vp = ctypes.c_void_p
    return b.lib.pa_decode_ex(vp(a["out"]), vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["t"]),
                              vp(a["l"]), a["B"], a["Hq"], a["Hkv"], a["D"], a["bs"], a["MB"],
                              a["NB"], a["scale"], a["dtype"], vp(a["ws"]), a["wsb"], vp(a["err"]),
                              vp(a["stream"]), ctypes.byref(opts))


def test_plan_on_a_machine_without_gpu_falls_back_to_partitions():
    from paged_kv_cache_350_b200 import binding as b
    import torch
    if torch.cuda.is_available():
        pytest.skip("plan depends on the device here")
    n = b.pa_decode_workspace_size(256, 32, 8, 128, 4112, 16, 0)
    plan = b.pa_decode_plan(256, 32, 8, 128, 16, 257, b.PA_BF16, n)
    assert plan["kernel"] == b.PA_KERNEL_TC_PARTITION and plan["launches"] == 2
    plan = b.pa_decode_plan(2, 4, 4, 64, 4, 4, b.PA_F32, 0)
    assert plan["kernel"] == b.PA_KERNEL_GENERIC and plan["launches"] == 1
    assert b.pa_decode_plan(0, 4, 4, 64, 4, 4, b.PA_F32, 0)["launches"] == 0


def test_decode_argument_errors_are_reported_before_any_launch():
    from paged_kv_cache_350_b200 import binding as b
    assert _call_decode(B=0) == b.PA_OK                       # empty batch: nothing to do
    assert _call_decode(Hq=6, Hkv=4) == b.PA_ERR_INVALID_ARG  # Hq % Hkv
    assert _call_decode(D=96) == b.PA_ERR_UNSUPPORTED
    assert _call_decode(bs=12) == b.PA_ERR_UNSUPPORTED
    assert _call_decode(q=8) == b.PA_ERR_INVALID_ARG          # misaligned pointer
    assert _call_decode(q=0) == b.PA_ERR_INVALID_ARG          # NULL
    assert _call_decode(scale=float("nan")) == b.PA_ERR_INVALID_ARG
    assert _call_decode(part=24) == b.PA_ERR_INVALID_ARG      # not a multiple of block_size
    assert _call_decode(dtype=b.PA_F32, path=b.PA_PATH_TENSOR) == b.PA_ERR_UNSUPPORTED
    assert _call_decode(bs=4, path=b.PA_PATH_TENSOR) == b.PA_ERR_UNSUPPORTED
    assert _call_decode(part=32, MB=8, wsb=0) == b.PA_ERR_INVALID_ARG   # explicit split, no workspace
    assert _call_decode(path=7) == b.PA_ERR_INVALID_ARG


def _call_append(**kw):
    from paged_kv_cache_350_b200 import binding as b
    a = dict(out=16, q=16, kn=16, vn=16, k=16, v=16, t=16, l=16, B=2, Hq=8, Hkv=2, D=128, bs=16,
             MB=4, NB=8, scale=0.1, dtype=b.PA_BF16)
    a.update(kw)
    vp = ctypes.c_void_p
    return b.lib.pa_decode_append(vp(a["out"]), vp(a["q"]), vp(a["kn"]), vp(a["vn"]), vp(a["k"]),
                                  vp(a["v"]), vp(a["t"]), vp(a["l"]), a["B"], a["Hq"], a["Hkv"],
                                  a["D"], a["bs"], a["MB"], a["NB"], a["scale"], a["dtype"],
                                  vp(0), 0, vp(0), vp(0), None)


def test_decode_append_argument_errors_are_reported_before_any_launch():
    from paged_kv_cache_350_b200 import binding as b
    assert _call_append(B=0, kn=0, vn=0) == b.PA_OK           # empty batch: nothing to do
    assert _call_append(kn=0) == b.PA_ERR_INVALID_ARG         # no new keys
    assert _call_append(vn=0) == b.PA_ERR_INVALID_ARG
    assert _call_append(vn=24) == b.PA_ERR_INVALID_ARG        # misaligned new values
    assert _call_append(D=96) == b.PA_ERR_UNSUPPORTED
    assert _call_append(Hq=6, Hkv=4) == b.PA_ERR_INVALID_ARG


def test_selftest_rejects_bad_arguments_before_any_launch():
    from paged_kv_cache_350_b200 import binding as b
    vp = ctypes.c_void_p
    assert b.lib.pa_selftest_bounded_wait(vp(0), 1000, vp(0)) == b.PA_ERR_INVALID_ARG
    assert b.lib.pa_selftest_bounded_wait(vp(16), 0, vp(0)) == b.PA_ERR_INVALID_ARG
    assert b.lib.pa_selftest_bounded_wait(vp(16), 2000000, vp(0)) == b.PA_ERR_INVALID_ARG


def test_cache_op_argument_errors():
    from paged_kv_cache_350_b200 import binding as b
    vp = ctypes.c_void_p
    L = b.lib
    assert L.pa_reshape_and_cache(vp(16), vp(16), vp(16), vp(16), vp(16), 0, 8, 128, 16, 4,
                                  b.PA_BF16, vp(0), vp(0)) == b.PA_OK
    assert L.pa_reshape_and_cache(vp(16), vp(16), vp(16), vp(16), vp(12), 3, 8, 128, 16, 4,
                                  b.PA_BF16, vp(0), vp(0)) == b.PA_ERR_INVALID_ARG
    assert L.pa_reshape_and_cache(vp(16), vp(16), vp(16), vp(16), vp(16), 3, 8, 80, 16, 4,
                                  b.PA_BF16, vp(0), vp(0)) == b.PA_ERR_UNSUPPORTED
    assert L.pa_copy_blocks(vp(16), vp(16), vp(16), 0, 16, 8, 128, 4, b.PA_BF16, vp(0),
                            vp(0)) == b.PA_OK
    assert L.pa_copy_blocks(vp(16), vp(16), vp(0), 2, 16, 8, 128, 4, b.PA_BF16, vp(0),
                            vp(0)) == b.PA_ERR_INVALID_ARG
    assert L.pa_copy_blocks(vp(16), vp(16), vp(16), -1, 16, 8, 128, 4, b.PA_BF16, vp(0),
                            vp(0)) == b.PA_ERR_INVALID_ARG


def _call_shared_prefix(**kw):
    from paged_kv_cache_350_b200 import binding as b
    a = dict(out=16, q=16, k=16, v=16, t=16, l=16, B=2, Hq=8, Hkv=2, D=128, bs=16, MB=4, NB=8,
             scale=0.1, dtype=b.PA_BF16, gof=16, gpre=16, gmem=16, ng=1, maxm=2, ws=256, wsb=1 << 20,
             err=0)
    a.update(kw)
    vp = ctypes.c_void_p
    return b.lib.pa_decode_shared_prefix(
        vp(a["out"]), vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["t"]), vp(a["l"]), a["B"], a["Hq"],
        a["Hkv"], a["D"], a["bs"], a["MB"], a["NB"], a["scale"], a["dtype"], vp(a["gof"]),
        vp(a["gpre"]), vp(a["gmem"]), a["ng"], a["maxm"], vp(a["ws"]), a["wsb"], vp(a["err"]),
        vp(0))


def test_shared_prefix_argument_errors_are_reported_before_any_launch():
    from paged_kv_cache_350_b200 import binding as b
    assert _call_shared_prefix(B=0) == b.PA_OK                    # empty batch: nothing to do
    assert _call_shared_prefix(Hq=6, Hkv=4) == b.PA_ERR_INVALID_ARG
    assert _call_shared_prefix(maxm=0) == b.PA_ERR_INVALID_ARG
    assert _call_shared_prefix(ng=-1) == b.PA_ERR_INVALID_ARG
    assert _call_shared_prefix(scale=float("inf")) == b.PA_ERR_INVALID_ARG
    assert _call_shared_prefix(maxm=17) == b.PA_ERR_UNSUPPORTED   # 17 members x 4 heads > 64 rows
    assert _call_shared_prefix(maxm=33, Hq=4, Hkv=4) == b.PA_ERR_UNSUPPORTED  # > 32 members
    assert _call_shared_prefix(dtype=b.PA_F32) == b.PA_ERR_UNSUPPORTED
    assert _call_shared_prefix(D=96) == b.PA_ERR_UNSUPPORTED
    assert _call_shared_prefix(B=8000, ng=500) == b.PA_ERR_UNSUPPORTED  # more rows than the kernel takes
    assert _call_shared_prefix(gof=0) == b.PA_ERR_INVALID_ARG
    assert _call_shared_prefix(gmem=0) == b.PA_ERR_INVALID_ARG    # groups without member lists
    assert _call_shared_prefix(gpre=18) == b.PA_ERR_INVALID_ARG   # misaligned int32 arrays
    assert _call_shared_prefix(gmem=18) == b.PA_ERR_INVALID_ARG
    assert _call_shared_prefix(gof=18) == b.PA_ERR_INVALID_ARG
    assert _call_shared_prefix(out=8) == b.PA_ERR_INVALID_ARG
    assert _call_shared_prefix(ws=0) == b.PA_ERR_INVALID_ARG
    assert _call_shared_prefix(ws=128) == b.PA_ERR_INVALID_ARG    # workspace not 256-byte aligned
    assert _call_shared_prefix(err=2) == b.PA_ERR_INVALID_ARG
    # no groups: the group arrays other than group_of may be NULL
    assert _call_shared_prefix(ng=0, gpre=0, gmem=0, out=8) == b.PA_ERR_INVALID_ARG
    assert b.pa_decode_shared_prefix_workspace_size(2, 8, 2, 128, 16, 1) > 0


def test_binding_rejects_host_tensors_before_the_c_call():
    """The library takes raw device pointers: a host tensor must never reach a kernel."""
    import torch
    from paged_kv_cache_350_b200 import binding as b
    q = torch.zeros(2, 8, 128, dtype=torch.bfloat16)
    kp = torch.zeros(4, 16, 2, 128, dtype=torch.bfloat16)
    tab = torch.zeros(2, 4, dtype=torch.int32)
    lens = torch.ones(2, dtype=torch.int32)
    kn = torch.zeros(2, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        b.pa_decode(q.clone(), q, kp, kp.clone(), tab, lens, 0.1)
    with pytest.raises(ValueError, match="CUDA"):
        b.pa_decode_append(q.clone(), q, kn, kn.clone(), kp, kp.clone(), tab, lens, 0.1)
    with pytest.raises(ValueError, match="CUDA"):
        b.pa_decode_no_alloc(q.clone(), q, kp, kp.clone(), tab, lens, 0.1)
    with pytest.raises(ValueError, match="CUDA"):
        b.pa_reshape_and_cache(kn, kn.clone(), kp, kp.clone(), torch.zeros(2, dtype=torch.int64))
    with pytest.raises(ValueError, match="CUDA"):
        b.pa_copy_blocks(kp, kp.clone(), torch.zeros(1, 2, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA"):
        b.pa_decode_shared_prefix(q.clone(), q, kp, kp.clone(), tab, lens, 0.1,
                                  torch.zeros(2, dtype=torch.int32), torch.zeros(1, dtype=torch.int32),
                                  torch.zeros(1, 2, dtype=torch.int32), torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="err_flag is required"):
        b.pa_selftest_bounded_wait(None, 1000)
    # shape and dtype errors come first, with their own messages
    with pytest.raises(ValueError, match="group_prefix int32"):
        b.pa_decode_shared_prefix(q.clone(), q, kp, kp.clone(), tab, lens, 0.1,
                                  torch.zeros(2, dtype=torch.int32), torch.zeros(1, dtype=torch.int64),
                                  torch.zeros(1, 2, dtype=torch.int32), torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ValueError, match="pools must be"):
        b.pa_copy_blocks(kp, kp[:2], torch.zeros(1, 2, dtype=torch.int32))


def test_header_compiles_as_c_and_the_allocator_runs_from_plain_c(tmp_path):
    """include/pa.h is a C header (strict C11) and the library serves a C client: the
    allocator's copy-on-write story, the fork grouping for the shared-prefix decode and the
    pipeline's slot layout, run from tests/c/alloc_abi.c, no Python in the path."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    from paged_kv_cache_350_b200 import binding
    libdir = os.path.dirname(binding._LIB_PATH)
    libname = os.path.basename(binding._LIB_PATH)
    if libname != "libpagedattn.so":
        pytest.skip("a renamed build of the library is loaded")
    exe = str(tmp_path / "alloc_abi")
    subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "alloc_abi.c"),
                    "-L", libdir, "-lpagedattn", f"-Wl,-rpath,{libdir}", "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr


def test_pipeline_layout_and_argument_errors_before_any_cuda_call():
    """pa_pipeline_*: the input-slot layout, descriptors rejected on the host, and the
    allocator check that keeps a step that cannot be described from changing state."""
    from paged_kv_cache_350_b200 import binding as b
    import numpy as np
    offs = (ctypes.c_size_t * 6)()
    total = b.lib.pa_pipeline_input_bytes(3, 8, 2, 128, 5, b.PA_BF16, offs)
    sizes = [3 * 8 * 128 * 2, 3 * 2 * 128 * 2, 3 * 2 * 128 * 2, 3 * 5 * 4, 3 * 4, 3 * 8]
    up = lambda n: (n + 255) // 256 * 256  # noqa: E731
    assert list(offs) == [sum(up(s) for s in sizes[:i]) for i in range(6)]
    assert total == sum(up(s) for s in sizes)
    assert b.lib.pa_pipeline_input_bytes(0, 8, 2, 128, 5, b.PA_BF16, None) == 0
    assert b.lib.pa_pipeline_input_bytes(3, 8, 2, 128, 5, 7, None) == 0
    # the shared-prefix slot: the same six sections, then slot_mapping, group_of,
    # group_prefix and group_members [B][m]
    offs10 = (ctypes.c_size_t * 10)()
    assert b.lib.pa_pipeline_input_bytes_prefix(3, 8, 2, 128, 5, b.PA_BF16, 0, offs10) == total
    sizes10 = sizes + [3 * 8, 3 * 4, 3 * 4, 3 * 6 * 4]
    total10 = b.lib.pa_pipeline_input_bytes_prefix(3, 8, 2, 128, 5, b.PA_BF16, 6, offs10)
    assert list(offs10) == [sum(up(s) for s in sizes10[:i]) for i in range(10)]
    assert total10 == sum(up(s) for s in sizes10)
    for m in (-1, 33):
        assert b.lib.pa_pipeline_input_bytes_prefix(3, 8, 2, 128, 5, b.PA_BF16, m, None) == 0

    a = b.Allocator(8, 4)
    h = ctypes.c_void_p()
    desc = b.pa_pipeline_desc()  # all zero: B = 0, no buffers
    assert b.lib.pa_pipeline_create(a._h, ctypes.byref(desc), ctypes.byref(h)) == b.PA_ERR_INVALID_ARG
    assert not h.value
    desc.shared_prefix_members = 33  # out of range as well
    assert b.lib.pa_pipeline_create(a._h, ctypes.byref(desc), ctypes.byref(h)) == b.PA_ERR_INVALID_ARG
    # a shared-prefix descriptor the decode would refuse (fp32; 16 members x G = 8 > 64
    # rows; no workspace) is refused when the pipeline is made, before any CUDA call
    bufs = (ctypes.c_void_p * 1)(16)
    for dtype, m, ws in ((b.PA_F32, 4, 256), (b.PA_BF16, 16, 256), (b.PA_BF16, 4, None)):
        d2 = b.pa_pipeline_desc(4, 16, 2, 128, 16, 8, 64, dtype, 1, 16, 16, ws, 1 << 30, None,
                                bufs, bufs, bufs, bufs, None, None, None, m)
        assert b.lib.pa_pipeline_create(a._h, ctypes.byref(d2), ctypes.byref(h)) == \
            b.PA_ERR_INVALID_ARG
        assert not h.value
    assert b.lib.pa_pipeline_create(None, ctypes.byref(desc), ctypes.byref(h)) == b.PA_ERR_INVALID_ARG
    slot = ctypes.c_int()
    assert b.lib.pa_pipeline_next_slot(None, ctypes.byref(slot)) == b.PA_ERR_INVALID_ARG
    assert b.lib.pa_pipeline_result(None, 0, ctypes.byref(slot)) == b.PA_ERR_INVALID_ARG
    assert b.lib.pa_pipeline_sync(None) == b.PA_ERR_INVALID_ARG
    b.lib.pa_pipeline_destroy(None)

    # the append check: sequence 1 holds 8 tokens = 2 full blocks of 4
    a.add_seq(0, 3)
    a.add_seq(1, 8)
    ids = np.array([0, 1], dtype=np.int64)
    chk = lambda i, mb: b.lib.pa_alloc_check_append_fits(a._h, b._i64p(i), i.size, mb)  # noqa: E731
    assert chk(ids, 3) == b.PA_OK
    assert chk(ids, 2) == b.PA_ERR_INVALID_ARG           # token 9 needs a third block
    assert chk(np.array([0], dtype=np.int64), 1) == b.PA_OK
    assert chk(np.array([5], dtype=np.int64), 3) == b.PA_ERR_NOT_FOUND
    free = a.num_free()
    assert free == 8 - 1 - 2 and a.block_table(1)[1] == 8   # the checks changed nothing


def test_step_shared_prefix_refuses_bad_group_size_before_any_change():
    """PagedKVCache.step_shared_prefix: a group size the decode cannot take (over 32
    members, or members x Hq/Hkv over 64 rows) is refused before the allocator changes."""
    import torch
    import paged_kv_cache_350_b200 as pa
    cache = pa.PagedKVCache(16, 16, 2, 128, device="cpu")
    cache.alloc.add_seq(0, 20)
    cache.alloc.fork(0, 1)
    free = cache.alloc.num_free()
    q = torch.zeros((2, 16, 128), dtype=torch.bfloat16)
    kv = torch.zeros((2, 2, 128), dtype=torch.bfloat16)
    for m in (0, 33, 9):  # 9 members x G = 8 is 72 rows
        with pytest.raises(pa.PAError):
            cache.step_shared_prefix([0, 1], q, kv, kv, torch.empty_like(q), 0.1, 4, m)
        assert cache.alloc.num_free() == free
