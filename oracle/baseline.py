"""CPU timing of the float64 oracle (the reported CPU baseline).

TEST INFRASTRUCTURE: used only by bench.py's CPU-baseline / reference leg.
Independent (sequence, head) units run in a pool of worker processes started
with the ``spawn`` method, one BLAS thread each.
"""
from __future__ import annotations

import os
import time


def _unit(args):
    os.environ.setdefault('OPENBLAS_NUM_THREADS', '1')
    from oracle import kda_oracle as ko
    (x, f, bl, g, cw, al, dtb, nw, cu) = args
    t0 = time.perf_counter()
    ko.layer(x=x, f=f, beta_logit=bl, g=g, conv_w=cw, A_log=al, dt_bias=dtb, norm_w=nw,
             cu_seqlens=cu)
    return time.perf_counter() - t0


def _warm(_):
    from oracle import kda_oracle  # noqa: F401  (import cost outside the timed region)
    return 0


def time_units(units, workers=None):
    """Run ``oracle.layer`` on each unit in a spawn pool; return (wall seconds, workers)."""
    import multiprocessing as mp
    workers = max(1, min(workers or os.cpu_count() or 1, len(units)))
    for var in ('OPENBLAS_NUM_THREADS', 'OMP_NUM_THREADS', 'MKL_NUM_THREADS'):
        os.environ[var] = '1'
    ctx = mp.get_context('spawn')
    with ctx.Pool(workers) as pool:
        pool.map(_warm, range(workers))
        t0 = time.perf_counter()
        pool.map(_unit, units)
        wall = time.perf_counter() - t0
    return wall, workers
