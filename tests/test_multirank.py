"""The N>1 host path of bench.py with world_size-2 gloo ranks on CPU.

The layer needs no collective (every (sequence, head) unit is independent), so
the multi-GPU bench runs replicas: each rank its own batch, a barrier around
the timed region and a max-over-ranks reduction of the elapsed time only.
"""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(('127.0.0.1', 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR='127.0.0.1', MASTER_PORT=str(port))
    import bench
    d = bench.Dist()
    try:
        d.barrier()
        t = d.max(10.0 + rank)              # each rank's elapsed time; all get the max
        seed = 1 + 1000 * d.rank            # per-rank batch seed used by run_prefill
        out.put((rank, d.world, t, seed))
    finally:
        d.close()


def test_two_gloo_ranks_share_max_time_and_use_distinct_batches():
    ctx = mp.get_context('spawn')
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [2, 2]
    assert [r[2] for r in res] == [11.0, 11.0]
    assert res[0][3] != res[1][3]
