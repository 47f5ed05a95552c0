"""The library at its documented limits (needs a B200): the most partitions a
sequence may have (2048) and the largest partition (4096 tokens), one past each
refused; the most copy pairs a call takes (65535); the most sequences a decode call
takes (65535, with contexts of one and zero tokens); a large append."""
import numpy as np
import pytest
import torch

from oracle import oracle
from pa_testlib import TOL, bits, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_363_b200 import pa as _pa
    return _pa


def _pool_for(lens, B, Hkv, D, dt, seed):
    g = torch.Generator().manual_seed(seed)
    nblk = [max(1, -(-L // B)) for L in lens]
    NB = sum(nblk)
    tables = np.full((len(lens), max(nblk)), -1, np.int32)
    perm = np.random.default_rng(seed).permutation(NB)
    pos = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = perm[pos:pos + n]
        pos += n
    k = torch.randn(NB, Hkv, B, D, generator=g).to(dt)
    v = torch.randn(NB, Hkv, B, D, generator=g).to(dt)
    return k, v, tables


@pytest.mark.parametrize("part,ok", [(16, True), (4096, True)])
def test_most_partitions_and_largest_partition(pa, part, ok):
    B, Hkv, G, D = 16, 2, 4, 128
    lens = [2048 * 16, 5000, 1]            # 2048 partitions of 16 tokens for the first sequence
    k, v, tables = _pool_for(lens, B, Hkv, D, torch.bfloat16, seed=part)
    g = torch.Generator().manual_seed(part + 1)
    q = torch.randn(len(lens), Hkv * G, D, generator=g).to(torch.bfloat16)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    pa.pa_decode(out, q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(tables).cuda(),
                 torch.tensor(lens, dtype=torch.int32).cuda(), max(lens), 128 ** -0.5, part)
    torch.cuda.synchronize()
    assert pa.pa_device_status() == 0
    ref = oracle.decode(q.float().numpy(), k.float().numpy(), v.float().numpy(), tables, np.array(lens, np.int32),
                        128 ** -0.5, nthreads=16)
    assert max_abs(out.float().cpu().numpy(), ref) <= TOL["bf16"]


def test_one_partition_too_many_or_too_large_is_refused(pa):
    B = 16
    for part, mcl in ((16, 2048 * 16 + 1), (4096 + 16, 5000)):
        with pytest.raises(pa.PAError):
            pa.pa_decode_partition_size(1, 8, 2, 128, B, mcl, part)
        k = torch.zeros(4, 2, B, 128, dtype=torch.bfloat16, device="cuda")
        q = torch.zeros(1, 8, 128, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(pa.PAError):
            pa.pa_decode(torch.empty_like(q), q, k, k, torch.zeros(1, 4, dtype=torch.int32, device="cuda"),
                         torch.zeros(1, dtype=torch.int32, device="cuda"), mcl, 1.0, part,
                         workspace=torch.empty(1 << 20, dtype=torch.uint8, device="cuda"))


def test_most_copy_pairs_in_one_call(pa):
    B, Hkv, D, n = 16, 1, 64, 65535
    NB = 2 * n
    kc = torch.arange(NB * Hkv * B * D, dtype=torch.int32).view(NB, Hkv, B, D).to(torch.float32).cuda()
    vc = (-kc).contiguous()
    perm = np.random.default_rng(5).permutation(NB)
    pairs = np.stack([perm[:n], perm[n:]], 1).astype(np.int64)
    want_k, want_v = kc.cpu().numpy().copy(), vc.cpu().numpy().copy()
    want_k[pairs[:, 1]], want_v[pairs[:, 1]] = want_k[pairs[:, 0]], want_v[pairs[:, 0]]
    pa.pa_copy_blocks(kc, vc, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    assert pa.pa_device_status() == 0
    assert np.array_equal(kc.cpu().numpy(), want_k) and np.array_equal(vc.cpu().numpy(), want_v)
    with pytest.raises(pa.PAError):
        pa.pa_copy_blocks(kc, vc, torch.zeros(n + 1, 2, dtype=torch.int64, device="cuda"))


def test_most_sequences_in_one_decode(pa):
    S, B, Hkv, G, D = 65535, 16, 1, 2, 64
    rng = np.random.default_rng(6)
    lens = rng.integers(0, 3, size=S).astype(np.int32)            # contexts of 0, 1 and 2 tokens
    k, v, tables = _pool_for(lens.tolist(), B, Hkv, D, torch.float32, seed=6)
    q = torch.randn(S, Hkv * G, D, generator=torch.Generator().manual_seed(7))
    out = torch.full(q.shape, 9.0, device="cuda")
    pa.pa_decode(out, q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(),
                 2, 0.125, 0)
    torch.cuda.synchronize()
    assert pa.pa_device_status() == 0
    ref = oracle.decode(q.numpy(), k.numpy(), v.numpy(), tables, lens, 0.125, nthreads=16)
    assert max_abs(out.cpu().numpy(), ref) <= TOL["f32"]
    assert np.all(out.cpu().numpy()[lens == 0] == 0.0)
    with pytest.raises(pa.PAError):
        pa.pa_decode(torch.empty(S + 1, Hkv * G, D, device="cuda"), torch.empty(S + 1, Hkv * G, D, device="cuda"),
                     k.cuda(), v.cuda(), torch.zeros(S + 1, tables.shape[1], dtype=torch.int32, device="cuda"),
                     torch.zeros(S + 1, dtype=torch.int32, device="cuda"), 2, 0.125, 0)


def test_large_append(pa):
    N, Hkv, B, D, NB = 1 << 18, 8, 16, 128, (1 << 18) // 16 + 8
    g = torch.Generator(device="cuda").manual_seed(8)
    key = torch.randn(N, Hkv, D, generator=g, device="cuda").to(torch.bfloat16)
    val = torch.randn(N, Hkv, D, generator=g, device="cuda").to(torch.bfloat16)
    kc = torch.zeros(NB, Hkv, B, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    slots = torch.from_numpy(np.random.default_rng(9).permutation(NB * B)[:N].astype(np.int64)).cuda()
    pa.pa_reshape_and_cache(key, val, kc, vc, slots)
    torch.cuda.synchronize()
    assert pa.pa_device_status() == 0
    s = slots.cpu().numpy()
    blk, off = s // B, s % B
    got = kc.cpu()[torch.from_numpy(blk), :, torch.from_numpy(off)]
    assert np.array_equal(bits(got), bits(key.cpu()))
    gotv = vc.cpu()[torch.from_numpy(blk), :, torch.from_numpy(off)]
    assert np.array_equal(bits(gotv), bits(val.cpu()))
