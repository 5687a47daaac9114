"""The float64 oracle over every row of a full-size batch, on all host cores.

Test infrastructure.  The batch's decode is cut into (batch row, KV head) items, each
one call of ``oracle.ref_decode`` on that row's query heads of that KV head, with the
pools viewed at that KV head: the same arithmetic as one call over the whole batch
(query head h reads KV head h // G; here G heads over a single KV head).  Items run
longest first in one spawned process per host core; the pools and q sit once in a
shared-memory segment that the workers map read-only.

Spawned, not forked: CUDA is live in the test process, and a process forked after it
was initialised can hang.
"""

from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor
from multiprocessing import shared_memory

import numpy as np

_W = {}  # worker state: the shared segment and the arrays viewed on it


def _attach(name, layout, tables, lens, scale, G):
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except Exception:
        pass
    shm = shared_memory.SharedMemory(name=name)
    try:  # the creating process unlinks the segment; this one only maps it
        from multiprocessing import resource_tracker
        resource_tracker.unregister(shm._name, "shared_memory")
    except Exception:
        pass
    arrs = {k: np.ndarray(shape, dtype=np.dtype(dt), buffer=shm.buf, offset=off)
            for k, (off, shape, dt) in layout.items()}
    _W.update(shm=shm, tables=tables, lens=lens, scale=scale, G=G, **arrs)


def _item(task):
    from oracle import ref_decode
    b, g = task
    G = _W["G"]
    q = _W["q"][b:b + 1, g * G:(g + 1) * G]
    kp = _W["k_pool"][:, :, g:g + 1]
    vp = _W["v_pool"][:, :, g:g + 1]
    o = ref_decode(q, kp, vp, _W["tables"][b:b + 1], _W["lens"][b:b + 1], _W["scale"])
    return b, g, o[0]


def decode_all_rows(q, k_pool, v_pool, tables, lens, scale, workers=None):
    """ref_decode(q, k_pool, v_pool, tables, lens, scale) for the whole batch, computed on
    ``workers`` processes (default: every core this process may run on)."""
    B, Hq, D = q.shape
    Hkv = k_pool.shape[2]
    G = Hq // Hkv
    workers = workers or len(os.sched_getaffinity(0))
    arrays = {"q": q, "k_pool": k_pool, "v_pool": v_pool}
    layout, off = {}, 0
    for k, a in arrays.items():
        layout[k] = (off, a.shape, a.dtype.str)
        off += (a.nbytes + 4095) // 4096 * 4096
    st = os.statvfs("/dev/shm")
    if st.f_bavail * st.f_frsize < off * 1.05:
        raise RuntimeError(f"/dev/shm holds less than the {off / 1e9:.1f} GB the oracle needs")
    shm = shared_memory.SharedMemory(create=True, size=off)
    out = np.zeros((B, Hq, D), dtype=np.float64)
    try:
        for k, a in arrays.items():
            o, shape, dt = layout[k]
            np.ndarray(shape, dtype=np.dtype(dt), buffer=shm.buf, offset=o)[...] = a
        lens = np.ascontiguousarray(lens)
        tasks = sorted(((b, g) for b in range(B) for g in range(Hkv) if lens[b] > 0),
                       key=lambda t: -int(lens[t[0]]))
        n = max(1, min(workers, len(tasks)))
        with ProcessPoolExecutor(n, mp_context=mp.get_context("spawn"), initializer=_attach,
                                 initargs=(shm.name, layout, np.ascontiguousarray(tables), lens,
                                           float(scale), G)) as ex:
            for b, g, o in ex.map(_item, tasks, chunksize=1):
                out[b, g * G:(g + 1) * G] = o
    finally:
        shm.close()
        shm.unlink()
    return out
