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

``pipeline`` (``StepPipeline``) queues such steps back to back: double-buffered
staging, the copies on their own streams, so the host and the copy engines work on
neighbouring steps while the GPU decodes the current one.
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

    def pipeline(self, B, Hq, max_blocks, depth=2, stream=None):
        """A StepPipeline over this cache: decode steps queued back to back."""
        return StepPipeline(self, B, Hq, max_blocks, depth=depth, stream=stream)

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
    """Decode steps of a fixed batch shape queued back to back, host and device overlapped.

    Each step is the same work as ``PagedKVCache.step_staged``: the allocator reserves a
    slot per sequence, one host->device copy moves the step's q / new K / new V, tables,
    lengths and copy pairs, ``pa_copy_blocks`` + ``pa_decode_append`` run, and the output
    is copied back to pinned host memory.  Here the step input and output buffers come in
    ``depth`` slots, the copies run on their own streams, and ``submit`` returns once the
    step is queued.  So the host prepares step t+1 and the copy engines move its input
    and step t-1's output while the GPU decodes step t.  Events order every reuse of a
    slot: a host input buffer is rewritten only after its copy has finished, a device
    input buffer only after the kernels that read it, a device output buffer only after
    its copy to the host.

        pipe = cache.pipeline(B, Hq, max_blocks)
        q, k, v = pipe.inputs()        # pinned views of the next step's input slot
        ...                            # write the step's q [B,Hq,D], k/v [B,Hkv,D]
        t = pipe.submit(seq_ids, scale)
        out = pipe.result(t)           # waits for step t's output copy (pinned [B,Hq,D])

    ``result(t)`` stays valid until step t + depth is submitted.
    """

    def __init__(self, cache, B, Hq, max_blocks, depth=2, stream=None):
        assert depth >= 1
        self.cache, self.B, self.Hq, self.max_blocks, self.depth = cache, B, Hq, max_blocks, depth
        self.dev = cache.device
        self.stream = stream or torch.cuda.current_stream(self.dev)
        self.copy_in = torch.cuda.Stream(self.dev)
        self.copy_out = torch.cuda.Stream(self.dev)
        self.lay, total = cache._layout(B, Hq, max_blocks)
        n_out = B * Hq * cache.D
        self.h_in = [torch.empty(total, dtype=torch.uint8, pin_memory=True) for _ in range(depth)]
        self.d_in = [torch.empty(total, dtype=torch.uint8, device=self.dev) for _ in range(depth)]
        self.h_out = [torch.empty(n_out, dtype=cache.dtype, pin_memory=True).view(B, Hq, cache.D)
                      for _ in range(depth)]
        self.d_out = [torch.empty(n_out, dtype=cache.dtype, device=self.dev).view(B, Hq, cache.D)
                      for _ in range(depth)]
        ev = lambda: [torch.cuda.Event() for _ in range(depth)]  # noqa: E731
        self.h2d_done, self.kern_done, self.d2h_done = ev(), ev(), ev()
        self.used = [False] * depth   # slot has a step in flight (its events are recorded)
        self.next = 0                 # index of the next step to submit
        self.bytes_in = self.bytes_out = 0
        self.ws = cache.workspace(B, Hq, max_blocks)
        # Per slot, built once (the per-step host work is the allocator and the queueing):
        # the allocator's output views in the pinned input, the device views the kernels
        # read, and the argument list of the pa_decode_append call.
        D, Hkv, dt = cache.D, cache.Hkv, cache.dtype
        self.h_views, self.d_pairs, self.decode_args = [], [], []
        for k in range(depth):
            h, d = self.h_in[k], self.d_in[k]
            self.h_views.append((self._view(h, "slots", (B,), torch.int64).numpy(),
                                 self._view(h, "pairs", (B, 2), torch.int32).numpy(),
                                 self._view(h, "tables", (B, max_blocks), torch.int32).numpy(),
                                 self._view(h, "lens", (B,), torch.int32).numpy()))
            self.d_pairs.append(self._view(d, "pairs", (B, 2), torch.int32))
            self.decode_args.append(_b.decode_append_args(
                self.d_out[k], self._view(d, "q", (B, Hq, D), dt), self._view(d, "k", (B, Hkv, D), dt),
                self._view(d, "v", (B, Hkv, D), dt), cache.k_pool, cache.v_pool,
                self._view(d, "tables", (B, max_blocks), torch.int32),
                self._view(d, "lens", (B,), torch.int32), workspace=self.ws, err_flag=cache.err,
                stream=self.stream))

    def _view(self, buf, name, shape, dtype):
        off, n = self.lay[name]
        return buf[off:off + n].view(dtype).view(shape)

    def inputs(self):
        """Pinned host (q, k, v) of the next step's slot, once its previous copy is done."""
        k = self.next % self.depth
        if self.used[k]:
            self.h2d_done[k].synchronize()
        c, h = self.cache, self.h_in[k]
        return (self._view(h, "q", (self.B, self.Hq, c.D), c.dtype),
                self._view(h, "k", (self.B, c.Hkv, c.D), c.dtype),
                self._view(h, "v", (self.B, c.Hkv, c.D), c.dtype))

    def submit(self, seq_ids, scale):
        """Queue one decode step for seq_ids (the inputs() of this step must be written)."""
        c, B = self.cache, self.B
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        assert ids.size == B, "the batch shape is fixed per pipeline"
        t, k = self.next, self.next % self.depth
        h, d = self.h_in[k], self.d_in[k]
        slots_h, pairs_h, tables_h, lens_h = self.h_views[k]
        if self.used[k]:
            self.h2d_done[k].synchronize()   # normally long done: the copy of step t - depth
        _, pairs = c.alloc.append_slots(ids, slot_out=slots_h, pairs_out=pairs_h)
        c.alloc.block_tables(ids, self.max_blocks, tables_out=tables_h, lens_out=lens_h)
        npairs = pairs.shape[0]
        used = self.lay["pairs"][0] + npairs * 8 if npairs else self.lay["lens"][0] + B * 4
        if self.used[k]:
            self.copy_in.wait_event(self.kern_done[k])     # step t - depth has read d_in[k]
        with torch.cuda.stream(self.copy_in):
            d[:used].copy_(h[:used], non_blocking=True)
        self.h2d_done[k].record(self.copy_in)
        s = self.stream
        s.wait_event(self.h2d_done[k])
        if self.used[k]:
            s.wait_event(self.d2h_done[k])                 # d_out[k] was copied out
        if npairs:
            _b.pa_copy_blocks(c.k_pool, c.v_pool, self.d_pairs[k][:npairs], err_flag=c.err,
                              stream=s)
        _b.decode_append_call(self.decode_args[k], scale)
        self.kern_done[k].record(s)
        self.copy_out.wait_event(self.kern_done[k])
        with torch.cuda.stream(self.copy_out):
            self.h_out[k].copy_(self.d_out[k], non_blocking=True)
        self.d2h_done[k].record(self.copy_out)
        self.used[k] = True
        self.bytes_in = used
        self.bytes_out = self.h_out[k].numel() * self.h_out[k].element_size()
        self.next = t + 1
        return t

    def result(self, t):
        """Pinned host output [B, Hq, D] of step t (waits for its copy)."""
        assert self.next - self.depth <= t < self.next, "step no longer (or not yet) held"
        k = t % self.depth
        self.d2h_done[k].synchronize()
        return self.h_out[k]

    def sync(self):
        """Wait for every queued step."""
        for k in range(self.depth):
            if self.used[k]:
                self.d2h_done[k].synchronize()
