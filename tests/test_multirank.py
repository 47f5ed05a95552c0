"""The N>1 host path of bench.py on CPU: two gloo ranks agree on the max-over-ranks
time and draw distinct batches (the path shards by sequence with no data exchange)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    from paged_kv_cache_363_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world, init_method="tcp://127.0.0.1:%d" % port,
                            timeout=datetime.timedelta(seconds=60))
    t = bench.reduce_max(10.0 + rank)
    wl = W.make_workload(2, seed=bench.rank_seed(0, rank))
    out.put((rank, t, int(wl.context_lens.sum()), wl.free_order[:8].tolist()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_shard():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [11.0, 11.0]
    assert res[0][2:] != res[1][2:]      # different batches per rank
