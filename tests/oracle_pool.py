"""The oracle's attention on many row ranges at once, in a pool of worker processes
(test infrastructure: lets full-size tests compare whole tiles with the fp64 oracle in
minutes rather than tens of minutes).

The bf16 inputs are placed once in shared memory; each worker views them as float64
where it indexes them and runs ``oracle.spava_oracle.approx_attention`` on its row
ranges, storing only those rows.  The pool is started with ``spawn`` (a process forked
after CUDA has been initialised can hang) and every worker limits its BLAS to one
thread, so the workers together use the host's cores once.
"""

import os
from concurrent.futures import ProcessPoolExecutor
from multiprocessing import get_context, shared_memory

import numpy as np

_ARRAYS = {}
_SHM = []


class _LazyF64:
    """bf16 bit patterns viewed as float64, converted only where indexed."""

    def __init__(self, bits):
        self.bits = bits
        self.shape = bits.shape

    def __getitem__(self, key):
        b = np.ascontiguousarray(self.bits[key], dtype=np.uint16)
        return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def _init(specs):
    from threadpoolctl import threadpool_limits
    threadpool_limits(1)
    for name, (shm_name, shape) in specs.items():
        shm = shared_memory.SharedMemory(name=shm_name)
        _SHM.append(shm)
        _ARRAYS[name] = np.ndarray(shape, dtype=np.uint16, buffer=shm.buf)


def _work(args):
    from oracle import spava_oracle as orc
    r0, r1, off, anchor, sel, scale = args
    q, k, v = (_LazyF64(_ARRAYS[x]) for x in ("q", "k", "v"))
    return orc.approx_attention(q, k, v, off, anchor, sel, scale, row_range=(r0, r1), compact=True)


def attention_rows_ranges(bits, off, anchor, sel, scale, ranges, workers=None):
    """O [r1-r0, hq, d] and lse [hq, r1-r0] (fp64) of every range (r0, r1) of rows, in
    the order given.  ``bits``: dict of the bf16 bit arrays q, k, v (uint16)."""
    workers = workers or max(1, min(len(ranges), os.cpu_count() or 1))
    shms, specs = [], {}
    try:
        for name in ("q", "k", "v"):
            a = np.ascontiguousarray(bits[name]).view(np.uint16)
            shm = shared_memory.SharedMemory(create=True, size=max(1, a.nbytes))
            shms.append(shm)
            np.ndarray(a.shape, dtype=np.uint16, buffer=shm.buf)[...] = a
            specs[name] = (shm.name, a.shape)
        jobs = [(int(r0), int(r1), off, anchor, sel, scale) for r0, r1 in ranges]
        with ProcessPoolExecutor(max_workers=workers, mp_context=get_context("spawn"), initializer=_init,
                                 initargs=(specs,)) as ex:
            return list(ex.map(_work, jobs))
    finally:
        for shm in shms:
            shm.close()
            shm.unlink()
