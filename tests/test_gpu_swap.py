"""CPU-GPU block swapping ([fullstackaihub] "Engineering Limitations") on the GPU path.

pa_swap_blocks copies whole blocks between a device pool and a pinned host pool in
either direction; checked bit for bit against plain copies.  End to end: sequences
swapped out through the allocator's host tier, their device blocks reused and
overwritten by another sequence, then swapped back in, decode to the same bits as
before (decode does not depend on where the blocks sit).
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_363_b200 import workloads as W
from pa_testlib import bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_363_b200 import pa as _pa
    return _pa


@pytest.mark.parametrize("dtype,D,B,Hkv", [("bf16", 128, 16, 8), ("f32", 64, 32, 2), ("bf16", 64, 16, 32)])
@pytest.mark.parametrize("mapping_on_host", [False, True])
def test_swap_blocks_bit_exact_both_directions(pa, dtype, D, B, Hkv, mapping_on_host):
    dt = W.torch_dtype(dtype)
    g = torch.Generator().manual_seed(D + B + Hkv)
    NB, NH, n = 97, 41, 29
    kd = torch.randn(NB, Hkv, B, D, generator=g).to(dt).cuda()
    vd = torch.randn(NB, Hkv, B, D, generator=g).to(dt).cuda()
    kh = torch.full((NH, Hkv, B, D), 3.0, dtype=dt).pin_memory()
    vh = torch.full((NH, Hkv, B, D), -3.0, dtype=dt).pin_memory()
    rng = np.random.default_rng(D)
    src = rng.choice(NB, n, replace=False)
    dst = rng.choice(NH, n, replace=False)
    out_pairs = torch.from_numpy(np.stack([src, dst], 1).astype(np.int64))
    out_pairs = out_pairs.pin_memory() if mapping_on_host else out_pairs.cuda()
    want_kh, want_vh = bits(kh).copy(), bits(vh).copy()
    want_kh[dst], want_vh[dst] = bits(kd)[src], bits(vd)[src]
    pa.pa_swap_blocks(kh, vh, kd, vd, out_pairs)
    torch.cuda.synchronize()
    assert np.array_equal(bits(kh), want_kh) and np.array_equal(bits(vh), want_vh)
    # back in, to other device blocks
    dst2 = rng.choice(NB, n, replace=False)
    in_pairs = torch.from_numpy(np.stack([dst, dst2], 1).astype(np.int64))
    in_pairs = in_pairs.pin_memory() if mapping_on_host else in_pairs.cuda()
    want_kd, want_vd = bits(kd).copy(), bits(vd).copy()
    want_kd[dst2], want_vd[dst2] = want_kh[dst], want_vh[dst]
    pa.pa_swap_blocks(kd, vd, kh, vh, in_pairs)
    torch.cuda.synchronize()
    assert np.array_equal(bits(kd), want_kd) and np.array_equal(bits(vd), want_vd)
    assert pa.pa_device_status() == 0


def test_swap_refuses_pageable_memory_and_flags_bad_pairs(pa):
    kd = torch.zeros(8, 2, 16, 64, dtype=torch.bfloat16, device="cuda")
    pageable = torch.zeros(8, 2, 16, 64, dtype=torch.bfloat16)
    pairs = torch.tensor([[0, 1]], dtype=torch.int64, device="cuda")
    with pytest.raises(ValueError):
        pa.pa_swap_blocks(pageable, pageable, kd, kd, pairs)
    # the C entry point itself refuses pageable host memory
    st = pa.lib.pa_swap_blocks(pageable.data_ptr(), pageable.data_ptr(), kd.data_ptr(), kd.data_ptr(),
                               pairs.data_ptr(), 1, 2, 64, 16, 8, 8, pa.PA_DTYPE_BF16, None)
    assert st == pa.PA_ERR_INVALID and "pinned" in pa.lib.pa_last_error_string().decode()
    kh = torch.full((4, 2, 16, 64), 5.0, dtype=torch.bfloat16).pin_memory()
    bad = torch.tensor([[0, 4], [9, 0], [1, 2]], dtype=torch.int64, device="cuda")
    before = bits(kh).copy()
    pa.pa_swap_blocks(kh, kh, kd, kd, bad)
    torch.cuda.synchronize()
    assert pa.pa_device_status() == pa.PA_DEV_BAD_PAIR
    after = bits(kh)
    assert np.array_equal(after[[0, 1, 3]], before[[0, 1, 3]])    # only the valid pair (1 -> 2) landed
    assert np.array_equal(after[2], bits(kd)[1])


def test_swap_round_trip_decodes_to_the_same_bits(pa):
    from paged_kv_cache_363_b200 import runner
    wl = W.make_workload(3, seed=4, num_seqs=24, num_blocks=3000)
    batch = runner.DecodeBatch(wl, "cuda")
    batch.append()
    ref = batch.decode(out=torch.empty_like(batch.q)).clone()
    S, Hkv, B, D = wl.num_seqs, wl.num_kv_heads, wl.block_size, wl.head_dim
    NH = 2000
    kh = torch.zeros(NH, Hkv, B, D, dtype=torch.bfloat16).pin_memory()
    vh = torch.zeros(NH, Hkv, B, D, dtype=torch.bfloat16).pin_memory()
    a = batch.alloc
    a.add_host_pool(NH)
    out_ids = list(range(1, S, 2))
    for s in out_ids:
        pairs = a.swap_out(s)
        pa.pa_swap_blocks(kh, vh, batch.k_cache, batch.v_cache, torch.from_numpy(pairs).cuda())
    assert a.stats()["swapped_seqs"] == len(out_ids)
    # another sequence takes every free device block (the released ones included) and overwrites it
    filler = a.add_seq(10_000, B * a.num_free())
    junk = torch.full((len(filler), Hkv, D), 9.0, dtype=torch.bfloat16, device="cuda")
    pa.pa_reshape_and_cache(junk, junk, batch.k_cache, batch.v_cache, torch.from_numpy(filler).cuda())
    a.free_seq(10_000)
    for s in reversed(out_ids):
        pairs = a.swap_in(s)
        pa.pa_swap_blocks(batch.k_cache, batch.v_cache, kh, vh, torch.from_numpy(pairs).cuda())
    tables, lens = batch.tables_now()
    out = torch.empty_like(batch.q)
    pa.pa_decode(out, batch.q, batch.k_cache, batch.v_cache, torch.from_numpy(tables).cuda(),
                 torch.from_numpy(lens).cuda(), batch.max_context_len, wl.scale, 0)
    torch.cuda.synchronize()
    assert np.array_equal(bits(out), bits(ref))
    assert pa.pa_device_status() == 0
