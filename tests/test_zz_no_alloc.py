"""pa_decode_static_workspace: decode attention for callers that cannot allocate
device memory (a host that only lends pointers to tensors it owns, or a process
whose memory pool must not be bypassed).  It uses the library's fixed 16 MiB
device workspace instead of one passed in.

Checked through the C ABI against pa_decode with a caller workspace, on calls in
a row with different inputs: the shared array keeps the previous call's contents
(another batch's plan and partition states), which must not leak into the next
result.  Both paths run the same kernels, so they must agree bit for bit; the
result is also checked against the fp64 oracle directly.  This file is collected
last and also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from oracle import oracle
from paged_kv_cache_363_b200 import workloads as W
from pa_testlib import TOL, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_363_b200 import pa as _pa
    return _pa


def _case(dtype, Hq, Hkv, lens, seed):
    g = torch.Generator().manual_seed(seed)
    dt = W.torch_dtype(dtype)
    S, D, B = len(lens), 128, 16
    nblk = [(L + B - 1) // B for L in lens]
    NB = sum(nblk) + 5
    perm = np.random.default_rng(seed).permutation(NB)
    tables = np.full((S, max(nblk)), -1, np.int32)
    pos = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = perm[pos:pos + n]
        pos += n
    q = torch.randn(S, Hq, D, generator=g).to(dt).cuda()
    k = torch.randn(NB, Hkv, B, D, generator=g).to(dt).cuda()
    v = torch.randn(NB, Hkv, B, D, generator=g).to(dt).cuda()
    return q, k, v, torch.from_numpy(tables).cuda(), torch.tensor(lens, dtype=torch.int32).cuda()


def _bits(t):
    return t.view(torch.int32) if t.dtype == torch.float32 else t.view(torch.int16)


@pytest.mark.parametrize("dtype,Hq,Hkv", [("bf16", 32, 8), ("bf16", 8, 8), ("f32", 4, 2)])
def test_static_workspace_matches_caller_workspace_twice(pa, dtype, Hq, Hkv):
    scale = 128 ** -0.5
    # the inputs under test, and another batch (more sequences, longer contexts, so
    # more partitions) whose call runs first and leaves its state in the shared array
    lens_a = [1, 17, 300, 1500, 64, 999]
    lens_b = [3000, 5, 2047, 640, 1, 2500, 33, 1200]
    a = _case(dtype, Hq, Hkv, lens_a, seed=Hq + Hkv)
    b = _case(dtype, Hq, Hkv, lens_b, seed=Hq + Hkv + 1)
    calls = [(b, lens_b), (a, lens_a), (a, lens_a)]
    for (q, k, v, tables, ctx), lens in calls:
        ref = torch.empty_like(q)
        pa.pa_decode(ref, q, k, v, tables, ctx, max(lens), scale, partition_size=64)   # split: uses the merge
        out = torch.full_like(q, 5.0)
        pa.pa_decode_static_workspace(out, q, k, v, tables, ctx, max(lens), scale, partition_size=64)
        torch.cuda.synchronize()
        assert max_abs(out.float().cpu().numpy(), ref.float().cpu().numpy()) <= TOL[dtype]
        assert torch.equal(_bits(out), _bits(ref))        # same kernels: the same bits
    q, k, v, tables, ctx = a
    want = oracle.decode(q.float().cpu().numpy(), k.float().cpu().numpy(), v.float().cpu().numpy(),
                         tables.cpu().numpy(), ctx.cpu().numpy(), scale, nthreads=4)
    assert max_abs(out.float().cpu().numpy(), want) <= TOL[dtype]
    assert pa.pa_device_status() == 0


def test_static_workspace_rejects_what_does_not_fit(pa):
    # 4096 sequences x 64 heads x 64 partitions of 16 tokens need far more than 16 MiB
    need = pa.pa_decode_workspace_size(4096, 64, 8, 128, 16, 1024, 16)
    assert need > pa.PA_STATIC_WORKSPACE_BYTES
    q = torch.zeros(4096, 64, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(8, 8, 16, 128, dtype=torch.bfloat16, device="cuda")
    tables = torch.zeros(4096, 64, dtype=torch.int32, device="cuda")
    ctx = torch.zeros(4096, dtype=torch.int32, device="cuda")
    with pytest.raises(pa.PAError) as e:
        pa.pa_decode_static_workspace(torch.empty_like(q), q, k, k, tables, ctx, 1024, 1.0, partition_size=16)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED
    assert "workspace" in str(e.value)
