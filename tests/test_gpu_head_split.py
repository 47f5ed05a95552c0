"""The tensor-parallel split by kv head, emulated on one GPU.

A rank of that split holds kv heads [k0, k1) of every block and the query heads
that read them, with the same block tables as every other rank (a table names
whole blocks: "PagedAttention Paper Breakdown", section 2, the per-request block
table).  Decoding each head slice with its own pools and concatenating the outputs
must give the full decode: bit for bit with a fixed partition size (the same units,
the same reduction order), within tolerance under automatic partitions (the plan
may choose another size for fewer heads), and within tolerance of the oracle.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_363_b200 import workloads as W
from pa_testlib import TOL, max_abs, oracle_logical_all

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_363_b200 import pa as _pa
    return _pa


def _bits(t):
    return t.view(torch.int32) if t.dtype == torch.float32 else t.view(torch.int16)


def _split_decode(pa, runner, batch, world, part):
    wl = batch.wl
    outs = []
    for rank in range(world):
        qh, kh = runner.kv_head_shard(wl.num_heads, wl.num_kv_heads, world, rank)
        q = batch.q[:, qh.start:qh.stop].contiguous()
        k = batch.k_cache[:, kh.start:kh.stop].contiguous()
        v = batch.v_cache[:, kh.start:kh.stop].contiguous()
        out = torch.empty_like(q)
        pa.pa_decode(out, q, k, v, batch.block_tables, batch.context_lens, batch.max_context_len, wl.scale, part)
        outs.append(out)
        del k, v
    return torch.cat(outs, dim=1)


@pytest.mark.parametrize("wid,world,over", [
    (1, 2, {}), (1, 4, {}),
    (2, 2, {"num_seqs": 24, "num_blocks": 4000}), (2, 4, {"num_seqs": 24, "num_blocks": 4000}),
    (3, 2, {}), (3, 8, {}),
    (5, 4, {"num_seqs": 3, "num_blocks": 3200}),
])
def test_kv_head_split_equals_full_decode(pa, wid, world, over):
    from paged_kv_cache_363_b200 import runner
    wl = W.make_workload(wid, seed=4, **over)
    vals = W.decode_values(wl, "cuda")
    batch = runner.DecodeBatch(wl, "cuda", values=vals)
    batch.append()
    tol = TOL[wl.dtype]
    # fixed partitions: the same units in the same order, so the same bits
    part = 4 * wl.block_size
    full = torch.empty_like(batch.q)
    pa.pa_decode(full, batch.q, batch.k_cache, batch.v_cache, batch.block_tables, batch.context_lens,
                 batch.max_context_len, wl.scale, part)
    split = _split_decode(pa, runner, batch, world, part)
    torch.cuda.synchronize()
    assert torch.equal(_bits(split), _bits(full))
    # automatic partitions: each rank's plan sees fewer heads
    auto_full = batch.decode(partition_size=0).clone()
    auto_split = _split_decode(pa, runner, batch, world, 0)
    torch.cuda.synchronize()
    assert max_abs(auto_split.float().cpu().numpy(), auto_full.float().cpu().numpy()) <= tol
    assert pa.pa_device_status() == 0
    # and the split result against the oracle
    q, keys, values, off = vals
    kc, vc = keys.float().cpu().numpy(), values.float().cpu().numpy()
    ref = oracle_logical_all(q.float().cpu().numpy(), lambda s: (kc[off[s]:off[s + 1]], vc[off[s]:off[s + 1]]),
                             wl.block_size, wl.scale)
    assert max_abs(split.float().cpu().numpy(), ref) <= tol
