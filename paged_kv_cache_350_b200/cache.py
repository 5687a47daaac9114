"""PagedKVCache: one decode step through the library, host buffers in and out.

The public call for a serving loop.  It owns the device K/V pools (PyTorch
memory), the C allocator and the split-context workspace; ``step`` takes the
step's query and new K/V rows in host memory, and returns the attention output
in host memory:

1. ``pa_alloc_append_slots`` (C, host): a slot per sequence, copy-on-write
   pairs for partial blocks that are still shared;
2. ``pa_alloc_block_tables`` (C, host): padded tables and lengths;
3. host→device copies of those and of q / new K / new V (pinned staging);
4. ``pa_copy_blocks`` (when a shared partial block is appended to), then
   ``pa_decode_append``: the decode kernel itself writes each sequence's new K/V at
   its last position (the slot the allocator reserved) and attends;
5. device→host copy of the output, then a stream synchronise.

Everything between the copies runs in the library's kernels.

``host_inputs`` + ``step_staged`` do the same with one host→device copy: the
caller writes the step's q / new K / new V straight into the cache's pinned
input buffer, the allocator writes slots, tables and lengths behind them, and a
single copy moves the whole step input.

``step_shared_prefix`` is ``step`` for parallel sampling: the sequences that share a
prompt's blocks are grouped (``pa_alloc_prefix_groups``), the new tokens' K/V go to their
slots with ``pa_reshape_and_cache``, and ``pa_decode_shared_prefix`` reads each group's
shared blocks once.

``pipeline`` (``StepPipeline``, the C ``pa_pipeline_*`` calls) queues such steps back to
back, one C call per step: staging in several slots, the copies on their own streams, so
the host and the copy engines work on neighbouring steps while the GPU decodes the
current one.
"""

from __future__ import annotations

import numpy as np
import torch

from . import binding as _b


class PagedKVCache:
    def __init__(self, num_blocks, block_size, Hkv, D, dtype=torch.bfloat16, device="cuda",
                 shuffle_seed=0, pop_order=None, k_pool=None, v_pool=None):
        self.device = torch.device(device)
        self.block_size, self.Hkv, self.D, self.dtype = block_size, Hkv, D, dtype
        shape = (num_blocks, block_size, Hkv, D)
        self.k_pool = k_pool if k_pool is not None else torch.zeros(shape, dtype=dtype, device=self.device)
        self.v_pool = v_pool if v_pool is not None else torch.zeros(shape, dtype=dtype, device=self.device)
        assert tuple(self.k_pool.shape) == shape and tuple(self.v_pool.shape) == shape
        self.alloc = _b.Allocator(num_blocks, block_size, shuffle_seed=shuffle_seed,
                                  pop_order=pop_order)
        self.err = torch.zeros(1, dtype=torch.int32, device=self.device)
        self._ws = None
        self._staging = {}

    # -- host buffers ------------------------------------------------------------
    def _pinned(self, key, shape, dtype):
        t = self._staging.get(key)
        if t is None or tuple(t.shape) != tuple(shape):
            t = torch.empty(shape, dtype=dtype, pin_memory=True)
            self._staging[key] = t
        return t

    def _dev(self, key, shape, dtype):
        k = ("dev",) + key
        t = self._staging.get(k)
        if t is None or tuple(t.shape) != tuple(shape):
            t = torch.empty(shape, dtype=dtype, device=self.device)
            self._staging[k] = t
        return t

    def workspace(self, B, Hq, max_blocks):
        n = _b.pa_decode_workspace_size(B, Hq, self.Hkv, self.D, max_blocks * self.block_size,
                                        self.block_size, 0)
        if n and (self._ws is None or self._ws.numel() < n):
            self._ws = torch.empty(n, dtype=torch.uint8, device=self.device)
        return self._ws if n else None

    # -- one decode step ---------------------------------------------------------
    def step(self, seq_ids, q_host, k_host, v_host, out_host, scale, max_blocks, stream=None):
        """Append one token to each sequence, cache its K/V, attend; output into out_host.

        q_host [B,Hq,D], k_host/v_host [B,Hkv,D] and out_host [B,Hq,D] are pinned
        host tensors of the pool dtype.  Returns (h2d_bytes, d2h_bytes).
        """
        stream = stream or torch.cuda.current_stream(self.device)
        B, Hq, D = q_host.shape
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        slots_h = self._pinned(("slots",), (B,), torch.int64)
        pairs_h = self._pinned(("pairs",), (B, 2), torch.int32)
        tables_h = self._pinned(("tables",), (B, max_blocks), torch.int32)
        lens_h = self._pinned(("lens",), (B,), torch.int32)
        _, pairs = self.alloc.append_slots(ids, slot_out=slots_h.numpy(), pairs_out=pairs_h.numpy())
        self.alloc.block_tables(ids, max_blocks, tables_out=tables_h.numpy(), lens_out=lens_h.numpy())
        npairs = pairs.shape[0]

        with torch.cuda.stream(stream):
            q = self._dev(("q",), q_host.shape, self.dtype)
            kn = self._dev(("k",), k_host.shape, self.dtype)
            vn = self._dev(("v",), v_host.shape, self.dtype)
            tables = self._dev(("tables",), (B, max_blocks), torch.int32)
            lens = self._dev(("lens",), (B,), torch.int32)
            out = self._dev(("out",), q_host.shape, self.dtype)
            h2d = 0
            # the slots stay on the host: the kernel derives them from tables and lengths
            for dst, src in ((q, q_host), (kn, k_host), (vn, v_host), (tables, tables_h),
                             (lens, lens_h)):
                dst.copy_(src, non_blocking=True)
                h2d += src.numel() * src.element_size()
            if npairs:
                pairs_d = self._dev(("pairs",), (B, 2), torch.int32)
                pairs_d[:npairs].copy_(pairs_h[:npairs], non_blocking=True)
                h2d += npairs * 8
                _b.pa_copy_blocks(self.k_pool, self.v_pool, pairs_d[:npairs], err_flag=self.err,
                                  stream=stream)
            ws = self.workspace(B, Hq, max_blocks)
            _b.pa_decode_append(out, q, kn, vn, self.k_pool, self.v_pool, tables, lens, scale,
                                workspace=ws, err_flag=self.err, stream=stream)
            out_host.copy_(out, non_blocking=True)
        stream.synchronize()
        return h2d, out_host.numel() * out_host.element_size()

    # -- one decode step reading each fork group's shared prompt once ------------------
    def step_shared_prefix(self, seq_ids, q_host, k_host, v_host, out_host, scale, max_blocks,
                           max_members, stream=None):
        """``step`` with the shared-prefix attention.

        Sequences forked from one prompt point at the same physical blocks ("深入解析
        PagedAttention", 多序列共享); after this step's appends (so that a block copied on
        write is a member's own), ``pa_alloc_prefix_groups`` groups them, up to
        ``max_members`` per group, and ``pa_decode_shared_prefix`` reads each group's shared
        blocks once (``max_members`` <= 32 and ``max_members`` * Hq / Hkv <= 64).  The new
        tokens' K/V are written to their slots by ``pa_reshape_and_cache`` first.  Same
        tensors as ``step``; returns (h2d_bytes, d2h_bytes), and ``last_prefix_groups`` is the
        number of groups formed.
        """
        B, Hq, D = q_host.shape
        # refused before the allocator or the pools change
        if not (1 <= max_members <= 32 and max_members * (Hq // self.Hkv) <= 64):
            raise _b.PAError(_b.PA_ERR_UNSUPPORTED, "step_shared_prefix: max_members")
        stream = stream or torch.cuda.current_stream(self.device)
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        slots_h = self._pinned(("slots",), (B,), torch.int64)
        pairs_h = self._pinned(("pairs",), (B, 2), torch.int32)
        tables_h = self._pinned(("tables",), (B, max_blocks), torch.int32)
        lens_h = self._pinned(("lens",), (B,), torch.int32)
        _, pairs = self.alloc.append_slots(ids, slot_out=slots_h.numpy(), pairs_out=pairs_h.numpy())
        self.alloc.block_tables(ids, max_blocks, tables_out=tables_h.numpy(), lens_out=lens_h.numpy())
        npairs = pairs.shape[0]
        gof, gpre, gmem = self.alloc.prefix_groups(ids, max_members)
        ng = len(gpre)
        self.last_prefix_groups = ng
        gof_h = self._pinned(("gof",), (B,), torch.int32)
        gpre_h = self._pinned(("gpre",), (B,), torch.int32)
        gmem_h = self._pinned(("gmem",), (B, max_members), torch.int32)
        gof_h.numpy()[:] = gof
        gpre_h.numpy()[:ng] = gpre
        gmem_h.numpy()[:ng] = gmem

        with torch.cuda.stream(stream):
            q = self._dev(("q",), q_host.shape, self.dtype)
            kn = self._dev(("k",), k_host.shape, self.dtype)
            vn = self._dev(("v",), v_host.shape, self.dtype)
            tables = self._dev(("tables",), (B, max_blocks), torch.int32)
            lens = self._dev(("lens",), (B,), torch.int32)
            slots = self._dev(("slots",), (B,), torch.int64)
            gof_d = self._dev(("gof",), (B,), torch.int32)
            gpre_d = self._dev(("gpre",), (B,), torch.int32)
            gmem_d = self._dev(("gmem",), (B, max_members), torch.int32)
            out = self._dev(("out",), q_host.shape, self.dtype)
            h2d = 0
            for dst, src in ((q, q_host), (kn, k_host), (vn, v_host), (tables, tables_h),
                             (lens, lens_h), (slots, slots_h), (gof_d, gof_h)):
                dst.copy_(src, non_blocking=True)
                h2d += src.numel() * src.element_size()
            if ng:
                gpre_d[:ng].copy_(gpre_h[:ng], non_blocking=True)
                gmem_d[:ng].copy_(gmem_h[:ng], non_blocking=True)
                h2d += ng * 4 * (1 + max_members)
            if npairs:
                pairs_d = self._dev(("pairs",), (B, 2), torch.int32)
                pairs_d[:npairs].copy_(pairs_h[:npairs], non_blocking=True)
                h2d += npairs * 8
                _b.pa_copy_blocks(self.k_pool, self.v_pool, pairs_d[:npairs], err_flag=self.err,
                                  stream=stream)
            _b.pa_reshape_and_cache(kn, vn, self.k_pool, self.v_pool, slots, err_flag=self.err,
                                    stream=stream)
            n = _b.pa_decode_shared_prefix_workspace_size(B, Hq, self.Hkv, self.D,
                                                          self.block_size, ng)
            ws = getattr(self, "_ws_prefix", None)
            if ws is None or ws.numel() < max(n, 1):
                ws = self._ws_prefix = torch.empty(max(n, 1), dtype=torch.uint8,
                                                   device=self.device)
            _b.pa_decode_shared_prefix(out, q, self.k_pool, self.v_pool, tables, lens, scale,
                                       gof_d, gpre_d, gmem_d[:ng], ws, err_flag=self.err,
                                       stream=stream)
            out_host.copy_(out, non_blocking=True)
        stream.synchronize()
        return h2d, out_host.numel() * out_host.element_size()

    # -- one decode step, single staged copy -----------------------------------------
    def _layout(self, B, Hq, max_blocks):
        """Byte offsets of the sections of the step input buffer (256-byte aligned)."""
        esz = torch.tensor([], dtype=self.dtype).element_size()
        # slots last: the allocator writes them but the device never reads them
        sizes = [("q", B * Hq * self.D * esz), ("k", B * self.Hkv * self.D * esz),
                 ("v", B * self.Hkv * self.D * esz), ("tables", B * max_blocks * 4),
                 ("lens", B * 4), ("pairs", B * 8), ("slots", B * 8)]
        off, lay = 0, {}
        for name, n in sizes:
            lay[name] = (off, n)
            off += (n + 255) // 256 * 256
        return lay, off

    def host_inputs(self, B, Hq, max_blocks):
        """Pinned host views (q [B,Hq,D], k [B,Hkv,D], v [B,Hkv,D]) for step_staged to read.

        The buffers only grow, so a batch that changes size from step to step (sequences
        admitted and retired) reuses them."""
        lay, total = self._layout(B, Hq, max_blocks)
        out_elems = B * Hq * self.D
        if getattr(self, "_hbuf", None) is None or self._hbuf.numel() < total:
            self._hbuf = torch.empty(total, dtype=torch.uint8, pin_memory=True)
            self._dbuf = torch.empty(total, dtype=torch.uint8, device=self.device)
        if getattr(self, "_out_hbuf", None) is None or self._out_hbuf.numel() < out_elems:
            self._out_hbuf = torch.empty(out_elems, dtype=self.dtype, pin_memory=True)
            self._out_dbuf = torch.empty(out_elems, dtype=self.dtype, device=self.device)
        self._stage_key, self._lay = (B, Hq, max_blocks), lay
        self._out_h = self._out_hbuf[:out_elems].view(B, Hq, self.D)
        self._out_d = self._out_dbuf[:out_elems].view(B, Hq, self.D)
        return (self._view(self._hbuf, "q", (B, Hq, self.D), self.dtype),
                self._view(self._hbuf, "k", (B, self.Hkv, self.D), self.dtype),
                self._view(self._hbuf, "v", (B, self.Hkv, self.D), self.dtype))

    def _view(self, buf, name, shape, dtype):
        off, n = self._lay[name]
        return buf[off:off + n].view(dtype).view(shape)

    def step_staged(self, seq_ids, scale, max_blocks, stream=None):
        """One decode step whose q / new K / new V the caller wrote into host_inputs().

        Returns the pinned host output [B, Hq, D] (valid until the next call) and the
        (h2d_bytes, d2h_bytes) moved.
        """
        stream = stream or torch.cuda.current_stream(self.device)
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        B = ids.size
        Hq = self._stage_key[1]
        assert self._stage_key == (B, Hq, max_blocks), "call host_inputs() with this shape first"
        h = self._hbuf
        slots_h = self._view(h, "slots", (B,), torch.int64).numpy()
        pairs_h = self._view(h, "pairs", (B, 2), torch.int32).numpy()
        tables_h = self._view(h, "tables", (B, max_blocks), torch.int32).numpy()
        lens_h = self._view(h, "lens", (B,), torch.int32).numpy()
        _, pairs = self.alloc.append_slots(ids, slot_out=slots_h, pairs_out=pairs_h)
        self.alloc.block_tables(ids, max_blocks, tables_out=tables_h, lens_out=lens_h)
        npairs = pairs.shape[0]
        used = self._lay["pairs"][0] + npairs * 8 if npairs else self._lay["lens"][0] + B * 4
        d = self._dbuf
        with torch.cuda.stream(stream):
            d[:used].copy_(h[:used], non_blocking=True)
            kp, vp = self.k_pool, self.v_pool
            if npairs:
                _b.pa_copy_blocks(kp, vp, self._view(d, "pairs", (B, 2), torch.int32)[:npairs],
                                  err_flag=self.err, stream=stream)
            _b.pa_decode_append(self._out_d, self._view(d, "q", (B, Hq, self.D), self.dtype),
                                self._view(d, "k", (B, self.Hkv, self.D), self.dtype),
                                self._view(d, "v", (B, self.Hkv, self.D), self.dtype), kp, vp,
                                self._view(d, "tables", (B, max_blocks), torch.int32),
                                self._view(d, "lens", (B,), torch.int32), scale,
                                workspace=self.workspace(B, Hq, max_blocks), err_flag=self.err,
                                stream=stream)
            self._out_h.copy_(self._out_d, non_blocking=True)
        stream.synchronize()
        return self._out_h, (used, self._out_h.numel() * self._out_h.element_size())

    def pipeline(self, B, Hq, max_blocks, depth=2, stream=None, shared_prefix_members=0):
        """A StepPipeline over this cache: decode steps queued back to back (with
        ``shared_prefix_members`` > 0, the steps of ``step_shared_prefix``)."""
        return StepPipeline(self, B, Hq, max_blocks, depth=depth, stream=stream,
                            shared_prefix_members=shared_prefix_members)

    # -- sequence management ------------------------------------------------------------
    def admit(self, seq_id, k_host, v_host, stream=None):
        """Register a sequence and write its prompt's K/V ([n, Hkv, D] host) into its blocks."""
        stream = stream or torch.cuda.current_stream(self.device)
        n = k_host.shape[0]
        self.alloc.add_seq(seq_id, n)
        if n == 0:
            return
        slots = torch.from_numpy(self.alloc.seq_slots(seq_id))
        with torch.cuda.stream(stream):
            k = k_host.to(self.device, non_blocking=True)
            v = v_host.to(self.device, non_blocking=True)
            sl = slots.to(self.device, non_blocking=True)
            _b.pa_reshape_and_cache(k, v, self.k_pool, self.v_pool, sl, err_flag=self.err,
                                    stream=stream)
        stream.synchronize()  # the host tensors above must outlive the copies

    def fork(self, parent_id, child_id):
        """The child shares every block of the parent (copy on write at its first append)."""
        self.alloc.fork(parent_id, child_id)

    def beam_select(self, seq_ids, parent_idx):
        """Beam search: beam i continues from beam parent_idx[i] (blocks shared, no copy)."""
        self.alloc.beam_select(seq_ids, parent_idx)

    def truncate(self, seq_id, num_tokens):
        """Roll a sequence back to its first num_tokens tokens (rejected speculation)."""
        self.alloc.truncate(seq_id, num_tokens)

    def retire(self, seq_id):
        """Free the sequence; blocks no other sequence holds return to the pool."""
        self.alloc.free_seq(seq_id)

    def check_device_errors(self):
        flag = int(self.err.item())
        if flag:
            raise _b.PAError(_b.pa_status_from_device_flag(flag), "device")


class StepPipeline:
    """Decode steps of a fixed batch shape queued back to back: ``pa_pipeline_*`` (C).

    Each step is the same work as ``PagedKVCache.step_staged``: the allocator reserves a
    slot per sequence, one host->device copy moves the step's q / new K / new V, tables,
    lengths and copy pairs, ``pa_copy_blocks`` + ``pa_decode_append`` run, and the output
    is copied back to pinned host memory.  The whole step is one C call
    (``pa_pipeline_submit``), which returns once the step is queued.  The step input and
    output buffers come in ``depth`` slots and the copies run on their own streams, so
    the host prepares step t+1 and the copy engines move its input and step t-1's output
    while the GPU decodes step t; events order every reuse of a slot.  This class owns
    the buffers and streams (PyTorch memory) and marshals the calls.

        pipe = cache.pipeline(B, Hq, max_blocks)
        q, k, v = pipe.inputs()        # pinned views of the next step's input slot
        ...                            # write the step's q [B,Hq,D], k/v [B,Hkv,D]
        t = pipe.submit(seq_ids, scale)
        out = pipe.result(t)           # waits for step t's output copy (pinned [B,Hq,D])

    ``result(t)`` stays valid until step t + depth is submitted.

    With ``shared_prefix_members`` > 0 each step is that of ``PagedKVCache.step_shared_prefix``
    (fork groups formed by the C allocator in the same call; ``pa_copy_blocks``,
    ``pa_reshape_and_cache`` and ``pa_decode_shared_prefix`` queued).
    """

    def __init__(self, cache, B, Hq, max_blocks, depth=2, stream=None, shared_prefix_members=0):
        import ctypes
        assert depth >= 1
        self.cache, self.B, self.Hq, self.max_blocks, self.depth = cache, B, Hq, max_blocks, depth
        self.dev = cache.device
        self.stream = stream or torch.cuda.current_stream(self.dev)
        self.copy_in = torch.cuda.Stream(self.dev)
        self.copy_out = torch.cuda.Stream(self.dev)
        D, Hkv, dt = cache.D, cache.Hkv, cache.dtype
        pdt = _b.PA_BF16 if dt == torch.bfloat16 else _b.PA_F32
        m = int(shared_prefix_members)
        offs = (ctypes.c_size_t * 10)()
        total = _b.lib.pa_pipeline_input_bytes_prefix(B, Hq, Hkv, D, max_blocks, pdt, m, offs)
        if total == 0:
            raise _b.PAError(_b.PA_ERR_INVALID_ARG, "pa_pipeline_input_bytes_prefix")
        self.offsets = list(offs)
        n_out = B * Hq * D
        self.h_in = [torch.empty(total, dtype=torch.uint8, pin_memory=True) for _ in range(depth)]
        self.d_in = [torch.empty(total, dtype=torch.uint8, device=self.dev) for _ in range(depth)]
        self.h_out = [torch.empty(n_out, dtype=dt, pin_memory=True).view(B, Hq, D)
                      for _ in range(depth)]
        self.d_out = [torch.empty(n_out, dtype=dt, device=self.dev).view(B, Hq, D)
                      for _ in range(depth)]
        if m:
            # the shared-prefix workspace: its size does not grow with the groups of a step
            # (at most B / 2: a group has two members or more)
            n = _b.pa_decode_shared_prefix_workspace_size(B, Hq, Hkv, D, cache.block_size, B // 2)
            self.ws = torch.empty(max(n, 1), dtype=torch.uint8, device=self.dev)
        else:
            self.ws = cache.workspace(B, Hq, max_blocks)
        esz = self.h_out[0].element_size()
        sec = [B * Hq * D * esz, B * Hkv * D * esz, B * Hkv * D * esz]
        self._in_views = [tuple(h[o:o + n].view(dt).view(shape) for o, n, shape in
                                zip(self.offsets[:3], sec, ((B, Hq, D), (B, Hkv, D), (B, Hkv, D))))
                          for h in self.h_in]
        arr = lambda ts: (ctypes.c_void_p * depth)(*[t.data_ptr() for t in ts])  # noqa: E731
        self._arrays = (arr(self.h_in), arr(self.d_in), arr(self.h_out), arr(self.d_out))
        desc = _b.pa_pipeline_desc(
            B, Hq, Hkv, D, cache.block_size, max_blocks, cache.k_pool.shape[0], pdt, depth,
            cache.k_pool.data_ptr(), cache.v_pool.data_ptr(),
            self.ws.data_ptr() if self.ws is not None else None,
            self.ws.numel() if self.ws is not None else 0, cache.err.data_ptr(), *self._arrays,
            self.stream.cuda_stream, self.copy_in.cuda_stream, self.copy_out.cuda_stream, m)
        h = ctypes.c_void_p()
        _b._check(_b.lib.pa_pipeline_create(cache.alloc._h, ctypes.byref(desc), ctypes.byref(h)),
                  "pa_pipeline_create")
        self._h = h
        self._slot = ctypes.c_int()
        self._step = ctypes.c_int64()
        self._h2d = ctypes.c_size_t()
        self.next = 0
        self.bytes_in = 0
        self.bytes_out = n_out * esz

    def close(self):
        if getattr(self, "_h", None):
            _b.lib.pa_pipeline_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def inputs(self):
        """Pinned host (q, k, v) of the next step's slot, once its previous copy is done."""
        import ctypes
        _b._check(_b.lib.pa_pipeline_next_slot(self._h, ctypes.byref(self._slot)),
                  "pa_pipeline_next_slot")
        return self._in_views[self._slot.value]

    def submit(self, seq_ids, scale):
        """Queue one decode step for seq_ids (the inputs() of this step must be written)."""
        import ctypes
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        assert ids.size == self.B, "the batch shape is fixed per pipeline"
        _b._check(_b.lib.pa_pipeline_submit(self._h, _b._i64p(ids), float(scale),
                                            ctypes.byref(self._step), ctypes.byref(self._h2d)),
                  "pa_pipeline_submit")
        self.bytes_in = self._h2d.value
        self.next = self._step.value + 1
        return self._step.value

    def result(self, t):
        """Pinned host output [B, Hq, D] of step t (waits for its copy)."""
        import ctypes
        _b._check(_b.lib.pa_pipeline_result(self._h, int(t), ctypes.byref(self._slot)),
                  "pa_pipeline_result")
        return self.h_out[self._slot.value]

    def sync(self):
        """Wait for every queued step."""
        _b._check(_b.lib.pa_pipeline_sync(self._h), "pa_pipeline_sync")
