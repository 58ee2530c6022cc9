"""The oracle over many sequences at once: one spawned process per host core,
one sequence per job (test infrastructure).

A job carries one sequence's tokens (bf16 bit patterns, copied from wherever
the GPU side drew them, so both sides see the same values) and, optionally,
its query row.  The worker appends the tokens to an oracle cache in the order
the GPU side appended them -- the first L - 1 tokens (in chunks: the bytes do
not depend on how an append is split) and then the decode step's token -- and
returns the oracle's tiles of that sequence (every INT4 page it owns and its
INT8 store) and the oracle's attention row.  The processes are spawned, never
forked, so the parent may hold a CUDA context.
"""

import os

import numpy as np

_STATE = {}


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def _init(cfg, table):
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"
    _STATE["cfg"] = dict(cfg)
    _STATE["table"] = np.asarray(table, np.int32)


def _f32(bits):
    """bf16 bit patterns (uint16) -> fp32 values (exact)."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _run(job):
    from threadpoolctl import threadpool_limits
    from oracle import OracleKV4Cache, decode_attention
    layer, seq, k_bits, v_bits, q, chunk = job
    cfg, table = _STATE["cfg"], _STATE["table"]
    with threadpool_limits(1):
        orc = OracleKV4Cache(cfg, table)
        L = k_bits.shape[0]
        done = 0
        while done < L - 1:                           # the population, then the decode step's token
            n = min(chunk, L - 1 - done)
            orc.append(layer, [seq], [0, n], _f32(k_bits[done:done + n]), _f32(v_bits[done:done + n]))
            done += n
        orc.append(layer, [seq], [0, 1], _f32(k_bits[L - 1:L]), _f32(v_bits[L - 1:L]))
        pages = {pg: t for (lay, pg), t in orc.pages.items() if lay == layer}
        prot = orc.prot.get((layer, seq))
        ref = None
        if q is not None:
            r = decode_attention(orc, layer, [seq], q[None].astype(np.float32))
            ref = {"out_bf16": r["out_bf16"], "out_f64": r["out_f64"]}
    return seq, pages, prot, ref


class OraclePool:
    """A pool of oracle processes for one cache configuration and block table."""

    def __init__(self, cfg, table, procs=None):
        import multiprocessing as mp
        self.procs = procs or host_cores()
        self.pool = mp.get_context("spawn").Pool(self.procs, initializer=_init, initargs=(cfg, table))

    def run(self, jobs, batch=None):
        """jobs: an iterable of (layer, seq, k_bits [L, Hkv, D] uint16, v_bits, q [Hq, D] fp32 or None);
        yields the results as they finish, keeping at most `batch` jobs in flight (the iterable is consumed
        lazily, so the tokens of a large batch are never all on the host at once)."""
        batch = batch or 2 * self.procs
        it = iter(jobs)
        pending = []
        while True:
            while len(pending) < batch:
                try:
                    layer, seq, kb, vb, q = next(it)
                except StopIteration:
                    break
                pending.append(self.pool.apply_async(_run, ((layer, seq, kb, vb, q, 16384),)))
            if not pending:
                return
            done = [p for p in pending if p.ready()]
            if not done:
                pending[0].wait()
                continue
            for p in done:
                pending.remove(p)
                yield p.get()

    def close(self):
        self.pool.close()
        self.pool.join()

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.pool.terminate()
        self.pool.join()
