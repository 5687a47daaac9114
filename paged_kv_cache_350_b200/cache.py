"""PagedKVCache: one decode step through the library, host buffers in and out.

The public call for a serving loop.  It owns the device K/V pools (PyTorch
memory), the C allocator and the split-context workspace; ``step`` takes the
step's query and new K/V rows in host memory, and returns the attention output
in host memory:

1. ``pa_alloc_append_slots`` (C, host): a slot per sequence, copy-on-write
   pairs for partial blocks that are still shared;
2. ``pa_alloc_block_tables`` (C, host): padded tables and lengths;
3. host→device copies of those and of q / new K / new V (pinned staging);
4. ``pa_copy_blocks`` → ``pa_reshape_and_cache`` → ``pa_decode`` on the stream;
5. device→host copy of the output, then a stream synchronise.

Everything between the copies runs in the library's kernels.
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
            slots = self._dev(("slots",), (B,), torch.int64)
            tables = self._dev(("tables",), (B, max_blocks), torch.int32)
            lens = self._dev(("lens",), (B,), torch.int32)
            out = self._dev(("out",), q_host.shape, self.dtype)
            h2d = 0
            for dst, src in ((q, q_host), (kn, k_host), (vn, v_host), (slots, slots_h),
                             (tables, tables_h), (lens, lens_h)):
                dst.copy_(src, non_blocking=True)
                h2d += src.numel() * src.element_size()
            if npairs:
                pairs_d = self._dev(("pairs",), (B, 2), torch.int32)
                pairs_d[:npairs].copy_(pairs_h[:npairs], non_blocking=True)
                h2d += npairs * 8
                _b.pa_copy_blocks(self.k_pool, self.v_pool, pairs_d[:npairs], err_flag=self.err,
                                  stream=stream)
            _b.pa_reshape_and_cache(kn, vn, self.k_pool, self.v_pool, slots, err_flag=self.err,
                                    stream=stream)
            ws = self.workspace(B, Hq, max_blocks)
            _b.pa_decode(out, q, self.k_pool, self.v_pool, tables, lens, scale, workspace=ws,
                         err_flag=self.err, stream=stream)
            out_host.copy_(out, non_blocking=True)
        stream.synchronize()
        return h2d, out_host.numel() * out_host.element_size()

    def check_device_errors(self):
        flag = int(self.err.item())
        if flag:
            raise _b.PAError(_b.pa_status_from_device_flag(flag), "device")
