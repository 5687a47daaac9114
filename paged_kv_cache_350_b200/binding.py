"""ctypes binding of libpagedattn (include/pa.h): argument marshalling only.

Every function keeps the C name and takes torch tensors (device memory and
streams come from PyTorch); shapes are read from the tensors, pointers and
sizes are passed to the C ABI, and a non-OK status raises ``PAError``.  No
computation happens here.  If the shared library is missing this module
raises at import: there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

# The in-tree build; PAGEDATTN_LIB may name another build of the same library.
_LIB_PATH = os.environ.get("PAGEDATTN_LIB") or os.path.join(
    os.path.dirname(os.path.abspath(__file__)), "libpagedattn.so")

# pa_status
PA_OK = 0
PA_ERR_INVALID_ARG = 1
PA_ERR_UNSUPPORTED = 2
PA_ERR_OUT_OF_BLOCKS = 3
PA_ERR_BAD_BLOCK_ID = 4
PA_ERR_CUDA = 5
PA_ERR_NOT_FOUND = 6
PA_ERR_EXISTS = 7
PA_ERR_BAD_SEQ_LEN = 8
PA_ERR_BAD_SLOT = 9
PA_ERR_TIMEOUT = 10
PA_ERR_SCRATCH_LIMIT = 11
PA_ERR_HOST_MEMORY = 12

# pa_dtype
PA_F32 = 0
PA_BF16 = 1

# pa_decode_path
PA_PATH_AUTO = 0
PA_PATH_GENERIC = 1
PA_PATH_TENSOR = 2

# device error flag bits
PA_DEVERR_BAD_BLOCK_ID = 0x1
PA_DEVERR_BAD_SEQ_LEN = 0x2
PA_DEVERR_BAD_SLOT = 0x4
PA_DEVERR_TIMEOUT = 0x8


class PAError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = status
        msg = lib.pa_status_string(status).decode() if lib is not None else str(status)
        super().__init__(f"{where}: {msg} (status {status})" if where else msg)


# pa_decode_kernel
PA_KERNEL_NONE = 0
PA_KERNEL_GENERIC = 1
PA_KERNEL_TC_PARTITION = 2
PA_KERNEL_TC_STREAM = 3


class pa_decode_opts(ctypes.Structure):
    _fields_ = [("partition_tokens", ctypes.c_int), ("path", ctypes.c_int),
                ("max_ctas", ctypes.c_int)]


class pa_decode_plan_info(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int), ("partition_tokens", ctypes.c_int),
                ("max_parts", ctypes.c_int), ("grid", ctypes.c_int), ("launches", ctypes.c_int)]


class pa_pipeline_desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("D", ctypes.c_int), ("block_size", ctypes.c_int), ("max_blocks", ctypes.c_int),
                ("num_blocks", ctypes.c_int), ("dtype", ctypes.c_int), ("depth", ctypes.c_int),
                ("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("dev_err_flag", ctypes.c_void_p),
                ("host_in", ctypes.POINTER(ctypes.c_void_p)),
                ("dev_in", ctypes.POINTER(ctypes.c_void_p)),
                ("host_out", ctypes.POINTER(ctypes.c_void_p)),
                ("dev_out", ctypes.POINTER(ctypes.c_void_p)),
                ("compute", ctypes.c_void_p), ("copy_in", ctypes.c_void_p),
                ("copy_out", ctypes.c_void_p), ("shared_prefix_members", ctypes.c_int)]


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"libpagedattn.so not found at {_LIB_PATH}; build it with "
            "`python -m paged_kv_cache_350_b200.build` (there is no non-CUDA fallback)")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    pi32 = ctypes.POINTER(ctypes.c_int32)
    pi64 = ctypes.POINTER(ctypes.c_int64)
    pint = ctypes.POINTER(ctypes.c_int)
    sig = {
        "pa_status_string": (ctypes.c_char_p, [i32]),
        "pa_status_from_device_flag": (i32, [ctypes.c_int32]),
        "pa_version": (ctypes.c_char_p, []),
        "pa_decode_workspace_size": (sz, [i32, i32, i32, i32, i32, i32, i32]),
        "pa_decode": (i32, [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, i32,
                            vp, sz, vp, vp]),
        "pa_decode_ex": (i32, [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32,
                               i32, vp, sz, vp, vp, ctypes.POINTER(pa_decode_opts)]),
        "pa_decode_append": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                   i32, f32, i32, vp, sz, vp, vp,
                                   ctypes.POINTER(pa_decode_opts)]),
        "pa_decode_plan": (i32, [i32, i32, i32, i32, i32, i32, i32, sz,
                                 ctypes.POINTER(pa_decode_opts), ctypes.POINTER(pa_decode_plan_info)]),
        "pa_decode_shared_prefix_workspace_size": (sz, [i32, i32, i32, i32, i32, i32]),
        "pa_decode_shared_prefix": (i32, [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                          i32, f32, i32, vp, vp, vp, i32, i32, vp, sz, vp, vp]),
        "pa_alloc_prefix_groups": (i32, [vp, pi64, i32, i32, i32, pi32, pi32, pi32, pint]),
        "pa_decode_no_alloc": (i32, [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                     f32, i32, vp, vp]),
        "pa_selftest_bounded_wait": (i32, [vp, ctypes.c_uint, vp]),
        "pa_reshape_and_cache": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp]),
        "pa_copy_blocks": (i32, [vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, vp]),
        "pa_alloc_create": (i32, [i32, i32, ctypes.c_uint64, ctypes.POINTER(vp)]),
        "pa_alloc_create_ordered": (i32, [i32, i32, pi32, ctypes.POINTER(vp)]),
        "pa_alloc_destroy": (None, [vp]),
        "pa_alloc_add_seq": (i32, [vp, i64, i32]),
        "pa_alloc_fork": (i32, [vp, i64, i64]),
        "pa_alloc_append_slot": (i32, [vp, i64, pi64, pi32, pi32]),
        "pa_alloc_append_slots": (i32, [vp, pi64, i32, pi64, pi32, pint]),
        "pa_alloc_free_seq": (i32, [vp, i64]),
        "pa_alloc_truncate": (i32, [vp, i64, i32]),
        "pa_alloc_beam_select": (i32, [vp, pi64, pi32, i32]),
        "pa_alloc_block_table": (i32, [vp, i64, pi32, i32, pint, pint]),
        "pa_alloc_block_tables": (i32, [vp, pi64, i32, pi32, i32, pi32]),
        "pa_alloc_seq_slots": (i32, [vp, i64, pi64, i32, pint]),
        "pa_alloc_refcount": (i32, [vp, ctypes.c_int32]),
        "pa_alloc_num_free": (i32, [vp]),
        "pa_alloc_internal_waste_slots": (i64, [vp]),
        "pa_alloc_free_list": (i32, [vp, pi32, i32]),
        "pa_alloc_check_append_fits": (i32, [vp, pi64, i32, i32]),
        "pa_pipeline_input_bytes": (sz, [i32, i32, i32, i32, i32, i32, ctypes.POINTER(sz)]),
        "pa_pipeline_input_bytes_prefix": (sz, [i32, i32, i32, i32, i32, i32, i32,
                                                ctypes.POINTER(sz)]),
        "pa_pipeline_create": (i32, [vp, ctypes.POINTER(pa_pipeline_desc), ctypes.POINTER(vp)]),
        "pa_pipeline_destroy": (None, [vp]),
        "pa_pipeline_next_slot": (i32, [vp, pint]),
        "pa_pipeline_submit": (i32, [vp, pi64, f32, pi64, ctypes.POINTER(sz)]),
        "pa_pipeline_result": (i32, [vp, i64, pint]),
        "pa_pipeline_sync": (i32, [vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = None
lib = _load()

#: every symbol include/pa.h declares
EXPORTED = (
    "pa_status_string", "pa_status_from_device_flag", "pa_version", "pa_decode_workspace_size",
    "pa_decode", "pa_decode_ex", "pa_decode_append", "pa_decode_plan", "pa_decode_no_alloc",
    "pa_decode_shared_prefix_workspace_size", "pa_decode_shared_prefix", "pa_alloc_prefix_groups",
    "pa_reshape_and_cache", "pa_copy_blocks", "pa_selftest_bounded_wait", "pa_alloc_create",
    "pa_alloc_create_ordered", "pa_alloc_destroy", "pa_alloc_add_seq", "pa_alloc_fork",
    "pa_alloc_append_slot", "pa_alloc_append_slots", "pa_alloc_free_seq", "pa_alloc_truncate",
    "pa_alloc_beam_select", "pa_alloc_block_table",
    "pa_alloc_block_tables", "pa_alloc_seq_slots", "pa_alloc_refcount", "pa_alloc_num_free",
    "pa_alloc_internal_waste_slots", "pa_alloc_free_list", "pa_alloc_check_append_fits",
    "pa_pipeline_input_bytes", "pa_pipeline_input_bytes_prefix", "pa_pipeline_create",
    "pa_pipeline_destroy",
    "pa_pipeline_next_slot", "pa_pipeline_submit", "pa_pipeline_result", "pa_pipeline_sync",
)


def _check(status, where):
    if status != PA_OK:
        raise PAError(status, where)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_of(t):
    import torch
    if t.dtype == torch.bfloat16:
        return PA_BF16
    if t.dtype == torch.float32:
        return PA_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _need(cond, msg):
    if not cond:
        raise ValueError(msg)


def _on_device(*ts, err_flag=None):
    """Every tensor (None skipped) must live on the current CUDA device: the library takes
    raw device pointers and launches there, so a host tensor would be read by a kernel.
    err_flag, when given, is an int32 device tensor of at least one element."""
    import torch
    dev = torch.cuda.current_device() if torch.cuda.is_available() else None
    for t in (*ts, err_flag):
        if t is None:
            continue
        _need(t.is_cuda, "tensors must be CUDA tensors (the library takes device pointers)")
        _need(t.device.index == dev, f"tensors must be on the current device (cuda:{dev})")
    _need(err_flag is None or (err_flag.dtype == torch.int32 and err_flag.numel() >= 1),
          "err_flag must be an int32 tensor of at least one element")


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------

def pa_decode_workspace_size(B, Hq, Hkv, D, max_seq_len, block_size, partition_tokens=0):
    n = lib.pa_decode_workspace_size(B, Hq, Hkv, D, max_seq_len, block_size, partition_tokens)
    if n == ctypes.c_size_t(-1).value:
        raise PAError(PA_ERR_INVALID_ARG, "pa_decode_workspace_size")
    return n


def pa_decode_plan(B, Hq, Hkv, D, block_size, max_blocks, dtype, workspace_bytes=0,
                   partition_tokens=0, path=PA_PATH_AUTO, max_ctas=0):
    """dict(kernel, partition_tokens, max_parts, grid, launches) pa_decode would use."""
    info = pa_decode_plan_info()
    opts = pa_decode_opts(partition_tokens, path, max_ctas)
    _check(lib.pa_decode_plan(B, Hq, Hkv, D, block_size, max_blocks, dtype, workspace_bytes,
                              ctypes.byref(opts), ctypes.byref(info)), "pa_decode_plan")
    return {"kernel": info.kernel, "partition_tokens": info.partition_tokens,
            "max_parts": info.max_parts, "grid": info.grid, "launches": info.launches}


def pa_decode(out, q, k_pool, v_pool, block_tables, seq_lens, scale, workspace=None,
              err_flag=None, stream=None, partition_tokens=0, path=PA_PATH_AUTO, max_ctas=0):
    """out[B,Hq,D] = paged decode attention of q[B,Hq,D] over the pools (see include/pa.h)."""
    import torch
    _need(q.dim() == 3 and out.shape == q.shape, "q/out must be [B, Hq, D]")
    _need(k_pool.dim() == 4 and v_pool.shape == k_pool.shape, "pools must be [NB, bs, Hkv, D]")
    _need(block_tables.dim() == 2 and block_tables.dtype == torch.int32, "block_tables int32 [B, MB]")
    _need(seq_lens.dtype == torch.int32 and seq_lens.numel() == q.shape[0], "seq_lens int32 [B]")
    for t in (out, q, k_pool, v_pool, block_tables, seq_lens):
        _need(t.is_contiguous(), "tensors must be contiguous")
    _on_device(out, q, k_pool, v_pool, block_tables, seq_lens, workspace, err_flag=err_flag)
    _need(q.dtype == out.dtype == k_pool.dtype == v_pool.dtype, "q, out and pools share a dtype")
    B, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_pool.shape
    _need(D2 == D, "head dim mismatch")
    _need(block_tables.shape[0] == B, "block_tables rows != B")
    wbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    opts = pa_decode_opts(partition_tokens, path, max_ctas)
    st = lib.pa_decode_ex(_ptr(out), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables),
                          _ptr(seq_lens), B, Hq, Hkv, D, bs, block_tables.shape[1], NB,
                          float(scale), _dtype_of(q), _ptr(workspace), wbytes, _ptr(err_flag),
                          _stream(stream), ctypes.byref(opts))
    _check(st, "pa_decode")
    return out


def pa_decode_append(out, q, k_new, v_new, k_pool, v_pool, block_tables, seq_lens, scale,
                     workspace=None, err_flag=None, stream=None, partition_tokens=0,
                     path=PA_PATH_AUTO, max_ctas=0):
    """One decode step with the cache write fused: k_new/v_new[B,Hkv,D] go to position
    seq_lens[b]-1 of each row's table, then out = pa_decode (see include/pa.h)."""
    import torch
    _need(q.dim() == 3 and out.shape == q.shape, "q/out must be [B, Hq, D]")
    _need(k_pool.dim() == 4 and v_pool.shape == k_pool.shape, "pools must be [NB, bs, Hkv, D]")
    _need(block_tables.dim() == 2 and block_tables.dtype == torch.int32, "block_tables int32 [B, MB]")
    _need(seq_lens.dtype == torch.int32 and seq_lens.numel() == q.shape[0], "seq_lens int32 [B]")
    B, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_pool.shape
    _need(D2 == D and block_tables.shape[0] == B, "shape mismatch")
    _need(k_new.shape == (B, Hkv, D) and v_new.shape == k_new.shape, "k_new/v_new must be [B, Hkv, D]")
    for t in (out, q, k_new, v_new, k_pool, v_pool, block_tables, seq_lens):
        _need(t.is_contiguous(), "tensors must be contiguous")
    _on_device(out, q, k_new, v_new, k_pool, v_pool, block_tables, seq_lens, workspace,
               err_flag=err_flag)
    _need(q.dtype == out.dtype == k_new.dtype == v_new.dtype == k_pool.dtype == v_pool.dtype,
          "q, out, new K/V and pools share a dtype")
    wbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    opts = pa_decode_opts(partition_tokens, path, max_ctas)
    st = lib.pa_decode_append(_ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool),
                              _ptr(v_pool), _ptr(block_tables), _ptr(seq_lens), B, Hq, Hkv, D, bs,
                              block_tables.shape[1], NB, float(scale), _dtype_of(q),
                              _ptr(workspace), wbytes, _ptr(err_flag), _stream(stream),
                              ctypes.byref(opts))
    _check(st, "pa_decode_append")
    return out


def decode_append_args(out, q, k_new, v_new, k_pool, v_pool, block_tables, seq_lens,
                       workspace=None, err_flag=None, stream=None, partition_tokens=0,
                       path=PA_PATH_AUTO, max_ctas=0):
    """The checked argument list of a pa_decode_append call whose tensors stay fixed (a
    caller that repeats the call, such as StepPipeline); run it with decode_append_call."""
    import torch
    _need(q.dim() == 3 and out.shape == q.shape, "q/out must be [B, Hq, D]")
    _need(k_pool.dim() == 4 and v_pool.shape == k_pool.shape, "pools must be [NB, bs, Hkv, D]")
    _need(block_tables.dim() == 2 and block_tables.dtype == torch.int32, "block_tables int32 [B, MB]")
    _need(seq_lens.dtype == torch.int32 and seq_lens.numel() == q.shape[0], "seq_lens int32 [B]")
    B, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_pool.shape
    _need(D2 == D and block_tables.shape[0] == B, "shape mismatch")
    _need(k_new.shape == (B, Hkv, D) and v_new.shape == k_new.shape, "k_new/v_new must be [B, Hkv, D]")
    for t in (out, q, k_new, v_new, k_pool, v_pool, block_tables, seq_lens):
        _need(t.is_contiguous(), "tensors must be contiguous")
    _on_device(out, q, k_new, v_new, k_pool, v_pool, block_tables, seq_lens, workspace,
               err_flag=err_flag)
    _need(q.dtype == out.dtype == k_new.dtype == v_new.dtype == k_pool.dtype == v_pool.dtype,
          "q, out, new K/V and pools share a dtype")
    wbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    opts = pa_decode_opts(partition_tokens, path, max_ctas)
    return [_ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool), _ptr(v_pool),
            _ptr(block_tables), _ptr(seq_lens), B, Hq, Hkv, D, bs, block_tables.shape[1], NB,
            0.0, _dtype_of(q), _ptr(workspace), wbytes, _ptr(err_flag), _stream(stream),
            ctypes.byref(opts), opts]


def decode_append_call(args, scale):
    """Run a pa_decode_append argument list from decode_append_args with this scale."""
    a = list(args[:-1])
    a[15] = float(scale)
    _check(lib.pa_decode_append(*a), "pa_decode_append")


def pa_decode_no_alloc(out, q, k_pool, v_pool, block_tables, seq_lens, scale, err_flag=None,
                       stream=None):
    """pa_decode without a workspace, for callers that cannot allocate device memory.

    The library's static device scratch (PA_NO_ALLOC_SCRATCH_BYTES per device) stands in
    for the workspace; calls that overlap on the GPU race on it (see include/pa.h)."""
    import torch
    _need(q.dim() == 3 and out.shape == q.shape, "q/out must be [B, Hq, D]")
    _need(k_pool.dim() == 4 and v_pool.shape == k_pool.shape, "pools must be [NB, bs, Hkv, D]")
    _need(block_tables.dim() == 2 and block_tables.dtype == torch.int32, "block_tables int32 [B, MB]")
    _need(seq_lens.dtype == torch.int32 and seq_lens.numel() == q.shape[0], "seq_lens int32 [B]")
    for t in (out, q, k_pool, v_pool, block_tables, seq_lens):
        _need(t.is_contiguous(), "tensors must be contiguous")
    _on_device(out, q, k_pool, v_pool, block_tables, seq_lens, err_flag=err_flag)
    _need(q.dtype == out.dtype == k_pool.dtype == v_pool.dtype, "q, out and pools share a dtype")
    B, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_pool.shape
    _need(D2 == D and block_tables.shape[0] == B, "shape mismatch")
    st = lib.pa_decode_no_alloc(_ptr(out), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                _ptr(block_tables), _ptr(seq_lens), B, Hq, Hkv, D, bs,
                                block_tables.shape[1], NB, float(scale), _dtype_of(q),
                                _ptr(err_flag), _stream(stream))
    _check(st, "pa_decode_no_alloc")
    return out


PA_SHARED_PREFIX_ALIGN = 32


def pa_decode_shared_prefix_workspace_size(B, Hq, Hkv, D, block_size, ngroups):
    n = lib.pa_decode_shared_prefix_workspace_size(B, Hq, Hkv, D, block_size, ngroups)
    if n == ctypes.c_size_t(-1).value:
        raise PAError(PA_ERR_INVALID_ARG, "pa_decode_shared_prefix_workspace_size")
    return n


def pa_decode_shared_prefix(out, q, k_pool, v_pool, block_tables, seq_lens, scale, group_of,
                            group_prefix, group_members, workspace, err_flag=None, stream=None):
    """pa_decode reading each group's shared prefix once (device int32 group arrays; see
    include/pa.h and Allocator.prefix_groups)."""
    import torch
    _need(q.dim() == 3 and out.shape == q.shape, "q/out must be [B, Hq, D]")
    _need(k_pool.dim() == 4 and v_pool.shape == k_pool.shape, "pools must be [NB, bs, Hkv, D]")
    _need(block_tables.dim() == 2 and block_tables.dtype == torch.int32, "block_tables int32 [B, MB]")
    _need(seq_lens.dtype == torch.int32 and seq_lens.numel() == q.shape[0], "seq_lens int32 [B]")
    _need(group_of.dtype == torch.int32 and group_of.numel() == q.shape[0], "group_of int32 [B]")
    _need(group_prefix.dtype == torch.int32, "group_prefix int32 [ngroups]")
    _need(group_members.dim() == 2 and group_members.dtype == torch.int32, "members int32 [ng, m]")
    for t in (out, q, k_pool, v_pool, block_tables, seq_lens, group_of, group_prefix, group_members):
        _need(t.is_contiguous(), "tensors must be contiguous")
    _on_device(out, q, k_pool, v_pool, block_tables, seq_lens, group_of, group_prefix,
               group_members, workspace, err_flag=err_flag)
    _need(q.dtype == out.dtype == k_pool.dtype == v_pool.dtype, "q, out and pools share a dtype")
    B, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_pool.shape
    _need(D2 == D and block_tables.shape[0] == B, "shape mismatch")
    ng, maxm = group_members.shape
    _need(group_prefix.numel() >= ng, "group_prefix [ngroups]")
    wbytes = workspace.numel() * workspace.element_size()
    st = lib.pa_decode_shared_prefix(
        _ptr(out), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), _ptr(seq_lens), B, Hq,
        Hkv, D, bs, block_tables.shape[1], NB, float(scale), _dtype_of(q), _ptr(group_of),
        _ptr(group_prefix), _ptr(group_members), ng, max(maxm, 1), _ptr(workspace), wbytes,
        _ptr(err_flag), _stream(stream))
    _check(st, "pa_decode_shared_prefix")
    return out


def pa_reshape_and_cache(key, value, k_pool, v_pool, slot_mapping, err_flag=None, stream=None):
    """Scatter key/value [T,Hkv,D] into the pools at slot_mapping[T] (int64; < 0 skips)."""
    import torch
    _need(key.dim() == 3 and value.shape == key.shape, "key/value must be [T, Hkv, D]")
    _need(slot_mapping.dtype == torch.int64 and slot_mapping.numel() == key.shape[0],
          "slot_mapping int64 [T]")
    _need(key.dtype == value.dtype == k_pool.dtype == v_pool.dtype, "dtype mismatch")
    _need(k_pool.dim() == 4 and v_pool.shape == k_pool.shape, "pools must be [NB, bs, Hkv, D]")
    for t in (key, value, k_pool, v_pool, slot_mapping):
        _need(t.is_contiguous(), "tensors must be contiguous")
    _on_device(key, value, k_pool, v_pool, slot_mapping, err_flag=err_flag)
    NB, bs, Hkv, D = k_pool.shape
    _need(key.shape[1:] == (Hkv, D), "key rows must be [Hkv, D] of the pool")
    st = lib.pa_reshape_and_cache(_ptr(key), _ptr(value), _ptr(k_pool), _ptr(v_pool),
                                  _ptr(slot_mapping), key.shape[0], Hkv, D, bs, NB,
                                  _dtype_of(key), _ptr(err_flag), _stream(stream))
    _check(st, "pa_reshape_and_cache")


def pa_copy_blocks(k_pool, v_pool, pairs, err_flag=None, stream=None):
    """Copy whole blocks pairs[i][0] -> pairs[i][1] (device int32 [n, 2]) in both pools."""
    import torch
    _need(pairs.dtype == torch.int32 and (pairs.numel() == 0 or pairs.shape[-1] == 2),
          "pairs int32 [n, 2]")
    _need(k_pool.dim() == 4 and v_pool.shape == k_pool.shape and v_pool.dtype == k_pool.dtype,
          "pools must be [NB, bs, Hkv, D] of one dtype")
    _need(pairs.is_contiguous() and k_pool.is_contiguous() and v_pool.is_contiguous(),
          "tensors must be contiguous")
    _on_device(k_pool, v_pool, pairs, err_flag=err_flag)
    NB, bs, Hkv, D = k_pool.shape
    n = pairs.numel() // 2
    st = lib.pa_copy_blocks(_ptr(k_pool), _ptr(v_pool), _ptr(pairs), n, bs, Hkv, D, NB,
                            _dtype_of(k_pool), _ptr(err_flag), _stream(stream))
    _check(st, "pa_copy_blocks")


def pa_selftest_bounded_wait(err_flag, limit_us, stream=None):
    """Run the bounded-wait self-test (see include/pa.h): err_flag gets PA_DEVERR_TIMEOUT."""
    _need(err_flag is not None, "err_flag is required")
    _on_device(err_flag=err_flag)
    _check(lib.pa_selftest_bounded_wait(_ptr(err_flag), int(limit_us), _stream(stream)),
           "pa_selftest_bounded_wait")


def pa_status_from_device_flag(flag):
    return lib.pa_status_from_device_flag(int(flag))


# ---------------------------------------------------------------------------
# host allocator
# ---------------------------------------------------------------------------

def _i32p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _i64p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


class Allocator:
    """The pa_alloc_* block allocator (C++), one handle per pool."""

    def __init__(self, num_blocks, block_size, shuffle_seed=0, pop_order=None):
        h = ctypes.c_void_p()
        if pop_order is not None:
            order = np.ascontiguousarray(pop_order, dtype=np.int32)
            _need(order.size == num_blocks, "pop_order must list every block")
            st = lib.pa_alloc_create_ordered(num_blocks, block_size, _i32p(order), ctypes.byref(h))
        else:
            st = lib.pa_alloc_create(num_blocks, block_size, ctypes.c_uint64(shuffle_seed),
                                     ctypes.byref(h))
        _check(st, "pa_alloc_create")
        self._h = h
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self):
        if getattr(self, "_h", None):
            lib.pa_alloc_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_seq(self, seq_id, num_tokens):
        _check(lib.pa_alloc_add_seq(self._h, seq_id, num_tokens), "pa_alloc_add_seq")

    def fork(self, parent_id, child_id):
        _check(lib.pa_alloc_fork(self._h, parent_id, child_id), "pa_alloc_fork")

    def append_slot(self, seq_id):
        slot, src, dst = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib.pa_alloc_append_slot(self._h, seq_id, ctypes.byref(slot), ctypes.byref(src),
                                        ctypes.byref(dst)), "pa_alloc_append_slot")
        return slot.value, src.value, dst.value

    def append_slots(self, seq_ids, slot_out=None, pairs_out=None):
        """append_slot for every id, all or nothing; returns (slots int64[n], pairs int32[k,2])."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.size
        slots = slot_out if slot_out is not None else np.empty(n, dtype=np.int64)
        pairs = pairs_out if pairs_out is not None else np.empty((max(n, 1), 2), dtype=np.int32)
        k = ctypes.c_int()
        _check(lib.pa_alloc_append_slots(self._h, _i64p(ids), n, _i64p(slots), _i32p(pairs),
                                         ctypes.byref(k)), "pa_alloc_append_slots")
        return slots[:n], pairs[: k.value]

    def free_seq(self, seq_id):
        _check(lib.pa_alloc_free_seq(self._h, seq_id), "pa_alloc_free_seq")

    def prefix_groups(self, seq_ids, max_members, align_tokens=PA_SHARED_PREFIX_ALIGN):
        """(group_of [n], group_prefix [ng], group_members [ng, max_members]) int32 arrays."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.size
        gof = np.empty(max(n, 1), np.int32)
        gpre = np.empty(max(n, 1), np.int32)
        gmem = np.empty((max(n, 1), max_members), np.int32)
        ng = ctypes.c_int()
        _check(lib.pa_alloc_prefix_groups(self._h, _i64p(ids), n, max_members, align_tokens,
                                          _i32p(gof), _i32p(gpre), _i32p(gmem), ctypes.byref(ng)),
               "pa_alloc_prefix_groups")
        return gof[:n], gpre[: ng.value], gmem[: ng.value]

    def truncate(self, seq_id, num_tokens):
        _check(lib.pa_alloc_truncate(self._h, seq_id, num_tokens), "pa_alloc_truncate")

    def beam_select(self, seq_ids, parent_idx):
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        par = np.ascontiguousarray(parent_idx, dtype=np.int32)
        _need(ids.size == par.size, "one parent index per beam")
        _check(lib.pa_alloc_beam_select(self._h, _i64p(ids), _i32p(par), ids.size),
               "pa_alloc_beam_select")

    def block_table(self, seq_id):
        n, ntok = ctypes.c_int(), ctypes.c_int()
        _check(lib.pa_alloc_block_table(self._h, seq_id, None, 0, ctypes.byref(n),
                                        ctypes.byref(ntok)), "pa_alloc_block_table")
        out = np.empty(max(n.value, 1), dtype=np.int32)
        _check(lib.pa_alloc_block_table(self._h, seq_id, _i32p(out), n.value, ctypes.byref(n),
                                        ctypes.byref(ntok)), "pa_alloc_block_table")
        return out[: n.value].tolist(), ntok.value

    def block_tables(self, seq_ids, max_blocks, tables_out=None, lens_out=None):
        """Padded tables int32[n, max_blocks] (-1 tail) and seq_lens int32[n]."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.size
        tables = tables_out if tables_out is not None else np.empty((n, max_blocks), np.int32)
        lens = lens_out if lens_out is not None else np.empty(n, np.int32)
        _check(lib.pa_alloc_block_tables(self._h, _i64p(ids), n, _i32p(tables), max_blocks,
                                         _i32p(lens)), "pa_alloc_block_tables")
        return tables, lens

    def seq_slots(self, seq_id):
        """Slots of all tokens of the sequence (int64 array)."""
        n = ctypes.c_int()
        _check(lib.pa_alloc_seq_slots(self._h, seq_id, None, 0, ctypes.byref(n)), "pa_alloc_seq_slots")
        out = np.empty(max(n.value, 1), dtype=np.int64)
        _check(lib.pa_alloc_seq_slots(self._h, seq_id, _i64p(out), n.value, ctypes.byref(n)),
               "pa_alloc_seq_slots")
        return out[: n.value]

    def refcount(self, block):
        return lib.pa_alloc_refcount(self._h, block)

    def num_free(self):
        return lib.pa_alloc_num_free(self._h)

    def internal_waste_slots(self):
        return lib.pa_alloc_internal_waste_slots(self._h)

    def free_list(self):
        n = lib.pa_alloc_free_list(self._h, None, 0)
        out = np.empty(max(n, 1), dtype=np.int32)
        lib.pa_alloc_free_list(self._h, _i32p(out), n)
        return out[:n].tolist()
