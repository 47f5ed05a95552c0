"""The N>1 host path on CPU with gloo ranks: the ranks agree on the max-over-ranks
time and draw distinct batches (the path shards by sequence with no data exchange);
sequence shards of one global batch are disjoint and cover it; kv-head shards are
disjoint and cover the heads, and every rank's allocator builds the same tables."""
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


def _split_worker(rank, world, port, out):
    """One rank of each split: its shard of a global 64-sequence batch, and, for the
    kv-head split, its head ranges and the block tables its own allocator builds."""
    import datetime
    import hashlib
    import sys
    import numpy as np
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    from paged_kv_cache_363_b200 import pa, runner
    from paged_kv_cache_363_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world, init_method="tcp://127.0.0.1:%d" % port,
                            timeout=datetime.timedelta(seconds=60))
    # data-parallel by sequence: this rank's part of one global batch
    wl = W.make_workload(2, seed=0)
    seqs = list(runner.sequence_shard(wl.num_seqs, world, rank))
    # tensor-parallel by kv head: the same allocator script on every rank
    wg = W.make_workload(3, seed=0)
    if wg.num_kv_heads % world == 0:
        qh, kh = runner.kv_head_shard(wg.num_heads, wg.num_kv_heads, world, rank)
    else:                                       # 8 kv heads do not split 3 ways: refused
        try:
            runner.kv_head_shard(wg.num_heads, wg.num_kv_heads, world, rank)
            raise AssertionError("an uneven kv-head split was accepted")
        except ValueError:
            qh, kh = range(0), range(0)
    alloc = pa.Allocator(wg.num_blocks, wg.block_size, wg.free_order)
    for s in range(wg.num_seqs):
        alloc.add_seq(s, int(wg.context_lens[s]))
    tables, lens = alloc.block_tables(np.arange(wg.num_seqs, dtype=np.int64),
                                      int(-(-wg.context_lens.max() // wg.block_size)), fill=-1)
    digest = hashlib.sha256(tables.tobytes() + lens.tobytes()).hexdigest()
    got = [None] * world
    dist.all_gather_object(got, (seqs, list(qh), list(kh), digest))
    if rank == 0:
        out.put(got)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_shard_by_sequence_and_by_kv_head(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    seqs = [g[0] for g in got]
    # sequence shards: disjoint, and together the whole batch in order
    assert sum(seqs, []) == list(range(64))
    assert max(map(len, seqs)) - min(map(len, seqs)) <= 1
    if 8 % world == 0:
        qheads = [g[1] for g in got]
        kvheads = [g[2] for g in got]
        assert sum(kvheads, []) == list(range(8))               # kv heads: disjoint, covering
        assert sum(qheads, []) == list(range(32))               # query heads follow their kv heads
        for qh, kh in zip(qheads, kvheads):
            assert [h // 4 for h in qh] == [k for k in kh for _ in range(4)]
    assert len({g[3] for g in got}) == 1                        # replicated tables: identical on every rank
