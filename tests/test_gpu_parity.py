"""Parity of the CUDA path with the fp64 oracle (needs a B200).

Every comparison runs the library through its C ABI (binding in
paged_kv_cache_363_b200.pa) and the oracle on the same seeded generator values.
Block tables, slots, appended rows and copied blocks must match bit for bit; the
attention output within max-abs 1e-5 (fp32) or 2e-2 (bf16 output, fp32
accumulation).  Unused pool slots hold NaN, so any stray read shows up.
"""
import numpy as np
import pytest
import torch

from oracle import oracle
from oracle.allocator import OracleAllocator
from paged_kv_cache_363_b200 import workloads as W
from pa_testlib import (TOL, bits, bits_to_f32, max_abs, nan_bits, oracle_decode_side, oracle_logical,
                        oracle_logical_all, report_error)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_363_b200 import pa as _pa
    return _pa


@pytest.fixture(scope="module")
def runner(pa):
    from paged_kv_cache_363_b200 import runner as _r
    return _r


def _status_clean(pa):
    assert pa.pa_device_status() == 0


# ------------------------------------------------------------------ decode-tiny-f32, end to end

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_f32_end_to_end(pa, runner, seed):
    wl = W.make_workload(1, seed=seed)
    vals = W.decode_values(wl, "cpu")
    ref = oracle_decode_side(wl, vals)
    batch = runner.DecodeBatch(wl, "cuda", values=vals)
    # decode over the prefill (before the step's append): contexts L-1, some of them 0
    t_pre, l_pre = batch.prefill_tables
    assert np.array_equal(t_pre[:, :ref["tables_pre"].shape[1]], ref["tables_pre"])
    assert np.array_equal(l_pre, ref["lens_pre"])
    out_pre = torch.empty_like(batch.q)
    pa.pa_decode(out_pre, batch.q, batch.k_cache, batch.v_cache, torch.from_numpy(t_pre).cuda(),
                 torch.from_numpy(l_pre).cuda(), int(l_pre.max()), wl.scale, 0, batch.workspace)
    assert max_abs(out_pre.cpu().numpy(), ref["out_pre"]) <= TOL["f32"]
    # the step: append one token per sequence, then decode over L
    out = batch.step()
    torch.cuda.synchronize()
    assert np.array_equal(batch.block_tables.cpu().numpy(), ref["tables"])
    assert np.array_equal(batch.context_lens.cpu().numpy(), ref["lens"])
    assert np.array_equal(bits(batch.k_cache), ref["kpool"])      # whole pool, bit for bit
    assert np.array_equal(bits(batch.v_cache), ref["vpool"])
    assert max_abs(out.cpu().numpy(), ref["out"]) <= TOL["f32"]
    _status_clean(pa)


# ------------------------------------------------------------------ shape/dtype matrix, small sizes

def _small_workload(dtype, D, B, G, lens, seed=0, Hkv=2, partition=0):
    nblk = sum(-(-L // B) for L in lens)
    return W.make_workload(1, seed=seed, num_heads=Hkv * G, num_kv_heads=Hkv, head_dim=D, block_size=B,
                           dtype=dtype, num_blocks=nblk + 37, context_lens=lens, partition_size=partition)


MATRIX = [(dt, D, B, G) for dt in ("f32", "bf16") for D in (64, 128) for B in (16, 32) for G in (1, 2, 4, 8)]


@pytest.mark.parametrize("dtype,D,B,G", MATRIX)
def test_decode_matrix_against_oracle(pa, runner, dtype, D, B, G):
    # ragged lengths: single token, partial and exact blocks, several partitions of 64 tokens
    lens = [1, B - 1, B, B + 1, 3 * B + 5, 200, 517]
    wl = _small_workload(dtype, D, B, G, lens, seed=D + B + G)
    vals = W.decode_values(wl, "cpu")
    ref = oracle_decode_side(wl, vals)
    batch = runner.DecodeBatch(wl, "cuda", values=vals)
    batch.append()
    assert np.array_equal(bits(batch.k_cache), ref["kpool"])
    assert np.array_equal(bits(batch.v_cache), ref["vpool"])
    for part in (0, 64, 2 * B, 4096):
        out = batch.decode(partition_size=part)
        got = out.float().cpu().numpy()
        assert np.isfinite(got).all()
        assert max_abs(got, ref["out"]) <= TOL[dtype], (part, max_abs(got, ref["out"]))
    _status_clean(pa)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_partitions_agree_with_each_other(pa, runner, dtype):
    wl = _small_workload(dtype, 128, 16, 4, [1000, 31, 4096, 513, 17], Hkv=3)
    vals = W.decode_values(wl, "cpu")
    batch = runner.DecodeBatch(wl, "cuda", values=vals)
    batch.append()
    outs = [batch.decode(out=torch.empty_like(batch.q), partition_size=p).float().cpu().numpy()
            for p in (16, 48, 512, 4096)]
    for o in outs[1:]:
        assert max_abs(o, outs[0]) <= TOL[dtype]
    _status_clean(pa)


def test_placement_does_not_change_a_single_bit(pa, runner):
    """Paged attention equals attention over the logical sequence, whatever the
    physical placement: two different placements give identical outputs."""
    lens = [700, 33, 1, 256, 95]
    wl1 = _small_workload("bf16", 128, 16, 4, lens, seed=3)
    wl2 = _small_workload("bf16", 128, 16, 4, lens, seed=3)
    wl2.free_order = np.random.default_rng(99).permutation(wl2.num_blocks).astype(np.int32)
    vals = W.decode_values(wl1, "cpu")
    o1 = runner.DecodeBatch(wl1, "cuda", values=vals).step().cpu()
    o2 = runner.DecodeBatch(wl2, "cuda", values=vals).step().cpu()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


@pytest.mark.parametrize("wid,overrides", [(3, {}), (2, {}), (5, {}), (3, {"dtype": "f32", "num_seqs": 48})])
def test_decode_is_reproducible_under_a_changing_schedule(pa, runner, wid, overrides):
    """Units go to CTAs through a dynamic work counter, so which CTA runs a unit, and
    after which others, changes from call to call.  The result must not: repeat the
    decode while a matmul on another stream takes SMs away at different moments."""
    wl = W.make_workload(wid, seed=1, **overrides)
    batch = runner.DecodeBatch(wl, "cuda", values=W.decode_values(wl, "cuda"))
    batch.append()
    ref = batch.decode(out=torch.empty_like(batch.q)).clone()
    side = torch.cuda.Stream()
    a = torch.randn(4096, 4096, device="cuda", dtype=torch.bfloat16)
    for k in range(6):
        with torch.cuda.stream(side):
            for _ in range(k):
                a = (a @ a).clamp_(-1, 1)
        out = batch.decode(out=torch.empty_like(batch.q))
        torch.cuda.synchronize()
        assert np.array_equal(bits(out), bits(ref)), "call %d differs" % k
    _status_clean(pa)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_zero_length_context_gives_zero_row(pa, dtype):
    dt = W.torch_dtype(dtype)
    S, Hq, Hkv, D, B, NB = 3, 4, 2, 128, 16, 8
    g = torch.Generator().manual_seed(5)
    q = torch.randn(S, Hq, D, generator=g).to(dt)
    k = torch.randn(NB, Hkv, B, D, generator=g).to(dt)
    v = torch.randn(NB, Hkv, B, D, generator=g).to(dt)
    tables = torch.tensor([[-1, -1], [3, 5], [-1, -1]], dtype=torch.int32)
    lens = torch.tensor([0, 20, 0], dtype=torch.int32)
    out = torch.full((S, Hq, D), 7.0, dtype=dt, device="cuda")
    pa.pa_decode(out, q.cuda(), k.cuda(), v.cuda(), tables.cuda(), lens.cuda(), 20, 0.3)
    ref = oracle.decode(q.float().numpy(), k.float().numpy(), v.float().numpy(), tables.numpy(), lens.numpy(), 0.3)
    o = out.float().cpu().numpy()
    assert np.all(o[0] == 0) and np.all(o[2] == 0)
    assert max_abs(o, ref) <= TOL[dtype]
    _status_clean(pa)


@pytest.mark.parametrize("dtype,G", [("bf16", 1), ("bf16", 4), ("f32", 2)])
def test_many_short_and_empty_sequences(pa, dtype, G):
    """Hundreds of tiny or empty contexts: many work units per persistent CTA, units
    without blocks, partial blocks everywhere, a few sequences split in partitions."""
    rng = np.random.default_rng(G)
    S, Hkv, D, B = 600, 2, 128, 16
    lens = rng.choice([0, 0, 1, 2, 15, 16, 17, 33, 100], size=S).astype(np.int32)
    lens[::97] = 700
    dt = W.torch_dtype(dtype)
    nblk = [(int(L) + B - 1) // B for L in lens]
    NB = sum(nblk) + 11
    perm = rng.permutation(NB)
    tables = np.full((S, max(nblk)), -1, np.int32)
    pos = 0
    for s_, n in enumerate(nblk):
        tables[s_, :n] = perm[pos:pos + n]
        pos += n
    g = torch.Generator().manual_seed(G)
    q = torch.randn(S, Hkv * G, D, generator=g).to(dt)
    k = torch.randn(NB, Hkv, B, D, generator=g).to(dt)
    v = torch.randn(NB, Hkv, B, D, generator=g).to(dt)
    out = torch.full((S, Hkv * G, D), 3.0, dtype=dt, device="cuda")
    pa.pa_decode(out, q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(),
                 int(lens.max()), 0.2, partition_size=256)
    ref = oracle.decode(q.float().numpy(), k.float().numpy(), v.float().numpy(), tables, lens, 0.2, nthreads=8)
    o = out.float().cpu().numpy()
    assert np.all(o[lens == 0] == 0)
    assert max_abs(o, ref) <= TOL[dtype]
    _status_clean(pa)


# ------------------------------------------------------------------ companions, bit-exact

@pytest.mark.parametrize("dtype,D,B", [("f32", 64, 16), ("bf16", 128, 16), ("bf16", 128, 32), ("f32", 128, 32)])
def test_reshape_and_cache_bit_exact(pa, dtype, D, B):
    rng = np.random.default_rng(D + B)
    NB, Hkv, N = 40, 3, 300
    dt = W.torch_dtype(dtype)
    g = torch.Generator().manual_seed(D)
    key = torch.randn(N, Hkv, D, generator=g).to(dt)
    val = torch.randn(N, Hkv, D, generator=g).to(dt)
    pool0 = torch.randn(NB, Hkv, B, D, generator=g).to(dt)
    slots = rng.choice(NB * B, size=N, replace=False).astype(np.int64)
    slots[rng.random(N) < 0.1] = -1                       # padding tokens
    kc, vc = pool0.clone().cuda(), pool0.clone().cuda()
    pa.pa_reshape_and_cache(key.cuda(), val.cuda(), kc, vc, torch.from_numpy(slots).cuda())
    rk, rv = oracle.reshape_and_cache(bits(key), bits(val), bits(pool0), bits(pool0), slots)
    assert np.array_equal(bits(kc), rk) and np.array_equal(bits(vc), rv)
    _status_clean(pa)


@pytest.mark.parametrize("dtype,D,B,Hkv", [("bf16", 128, 16, 32), ("f32", 64, 16, 4), ("bf16", 64, 32, 8)])
def test_copy_blocks_bit_exact(pa, dtype, D, B, Hkv):
    rng = np.random.default_rng(Hkv)
    NB = 64
    dt = W.torch_dtype(dtype)
    pool_k = torch.randn(NB, Hkv, B, D, generator=torch.Generator().manual_seed(1)).to(dt)
    pool_v = torch.randn(NB, Hkv, B, D, generator=torch.Generator().manual_seed(2)).to(dt)
    perm = rng.permutation(NB)
    src, dst = perm[:20], perm[20:40]                     # distinct destinations, none a source
    src[5] = src[6]                                       # one source copied twice
    pairs = np.stack([src, dst], 1).astype(np.int64)
    kc, vc = pool_k.clone().cuda(), pool_v.clone().cuda()
    pa.pa_copy_blocks(kc, vc, torch.from_numpy(pairs).cuda())
    rk, rv = oracle.copy_blocks(bits(pool_k), bits(pool_v), pairs)
    assert np.array_equal(bits(kc), rk) and np.array_equal(bits(vc), rv)
    _status_clean(pa)


def test_checked_copy_and_append_refuse_racing_mappings_before_any_write(pa):
    """check=True runs the host-side checks first: a racing mapping is refused and the
    pools stay as they were; a sound one goes through bit-exact."""
    NB, Hkv, B, D = 16, 2, 16, 64
    pool_k = torch.randn(NB, Hkv, B, D, generator=torch.Generator().manual_seed(3))
    pool_v = torch.randn(NB, Hkv, B, D, generator=torch.Generator().manual_seed(4))
    kc, vc = pool_k.clone().cuda(), pool_v.clone().cuda()
    for bad in ([[0, 3], [1, 3]], [[0, 3], [3, 5]]):
        with pytest.raises(pa.PAError):
            pa.pa_copy_blocks(kc, vc, torch.tensor(bad, dtype=torch.int64, device="cuda"), check=True)
    key = torch.ones(3, Hkv, D, device="cuda")
    with pytest.raises(pa.PAError):
        pa.pa_reshape_and_cache(key, key, kc, vc, torch.tensor([5, 40, 5], dtype=torch.int64, device="cuda"),
                                check=True)
    torch.cuda.synchronize()
    assert torch.equal(kc.cpu(), pool_k) and torch.equal(vc.cpu(), pool_v)
    good = np.array([[0, 3], [0, 4], [1, 5]], np.int64)
    pa.pa_copy_blocks(kc, vc, torch.from_numpy(good).cuda(), check=True)
    rk, rv = oracle.copy_blocks(bits(pool_k), bits(pool_v), good)
    assert np.array_equal(bits(kc), rk) and np.array_equal(bits(vc), rv)
    _status_clean(pa)


# ------------------------------------------------------------------ device-side checks

def test_device_checks_flag_bad_inputs_without_touching_memory(pa):
    dt = torch.bfloat16
    S, Hq, Hkv, D, B, NB = 2, 4, 4, 128, 16, 8
    q = torch.randn(S, Hq, D, device="cuda").to(dt)
    k = torch.randn(NB, Hkv, B, D, device="cuda").to(dt)
    v = torch.randn(NB, Hkv, B, D, device="cuda").to(dt)
    out = torch.empty_like(q)
    _status_clean(pa)
    # block-table entry past the pool: flagged, never dereferenced
    tables = torch.tensor([[1, 99], [2, 3]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([20, 20], dtype=torch.int32, device="cuda")
    pa.pa_decode(out, q, k, v, tables, lens, 32, 0.1)
    assert pa.pa_device_status() & pa.PA_DEV_BAD_BLOCK
    # context length beyond max_context_len: flagged and clamped
    tables = torch.tensor([[1, 2], [2, 3]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([20, 40], dtype=torch.int32, device="cuda")
    pa.pa_decode(out, q, k, v, tables, lens, 32, 0.1)
    assert pa.pa_device_status() & pa.PA_DEV_BAD_CONTEXT
    # slot past the pool: flagged and skipped (pool unchanged)
    k0 = k.clone()
    pa.pa_reshape_and_cache(torch.ones(1, Hkv, D, dtype=dt, device="cuda"), torch.ones(1, Hkv, D, dtype=dt, device="cuda"),
                            k, v, torch.tensor([NB * B], dtype=torch.int64, device="cuda"))
    assert pa.pa_device_status() & pa.PA_DEV_BAD_SLOT
    assert torch.equal(k, k0)
    # copy pair outside the pool: flagged and skipped
    pa.pa_copy_blocks(k, v, torch.tensor([[0, NB]], dtype=torch.int64, device="cuda"))
    assert pa.pa_device_status() & pa.PA_DEV_BAD_PAIR
    assert torch.equal(k, k0)
    _status_clean(pa)


# ------------------------------------------------------------------ full sizes, bench launch configuration

@pytest.mark.parametrize("wid,seed", [(2, 0), (3, 0), (3, 1), (5, 0)])
def test_full_size_workloads_every_row(pa, runner, wid, seed):
    """The bench's workloads at full size, in the bench's launch configuration
    (automatic partitions): every output row against the oracle, every appended
    row bit for bit at its slot."""
    wl = W.make_workload(wid, seed=seed)
    vals = W.decode_values(wl, "cuda")
    q, keys, values, off = vals
    batch = runner.DecodeBatch(wl, "cuda", values=vals)
    out = batch.step()
    torch.cuda.synchronize()
    _status_clean(pa)
    got = out.float().cpu().numpy()
    # the appended rows landed at their slots, bit for bit, for every sequence
    slots = batch.slot_mapping.cpu()
    last = torch.from_numpy(np.asarray(off[1:], np.int64) - 1)
    blk, o = slots // wl.block_size, slots % wl.block_size
    assert torch.equal(bits_t(batch.k_cache.cpu()[blk, :, o]), bits_t(keys.cpu()[last]))
    assert torch.equal(bits_t(batch.v_cache.cpu()[blk, :, o]), bits_t(values.cpu()[last]))
    kc, vc = keys.float().cpu().numpy(), values.float().cpu().numpy()
    ref = oracle_logical_all(q.float().cpu().numpy(),
                             lambda s: (kc[off[s]:off[s + 1]], vc[off[s]:off[s + 1]]), wl.block_size, wl.scale)
    err = max_abs(got, ref)
    report_error("%s seed %d" % (wl.name, seed), err, wl.num_seqs * wl.num_heads)
    assert err <= TOL["bf16"], err


def test_cow_sampling_full_size(pa, runner):
    wl = W.make_workload(4, seed=0)
    vals = W.cow_values(wl, "cuda")
    q, pk, pv, poff, xk, xv, xoff = vals
    batch = runner.CowBatch(wl, "cuda", values=vals)
    # the oracle allocator replays the same script: identical slots, copy pairs, tables
    P, n = wl.num_prompts, wl.streams_per_prompt
    ora = OracleAllocator(wl.num_blocks, wl.block_size, wl.free_order)
    for p in range(P):
        ora.add_seq(p * n, int(wl.prompt_lens[p]))
    for p in range(P):
        for j in range(1, n):
            ora.fork(p * n, p * n + j)
    for active, slots, pairs in batch.log:
        res = [ora.append_slot(int(s)) for s in active]
        assert slots.tolist() == [r[0] for r in res]
        assert [tuple(x) for x in pairs.tolist()] == [r[1] for r in res if r[1] is not None]
    for s in range(wl.num_seqs):
        row = batch.block_tables[s].cpu().numpy()
        assert row[:len(ora.tables[s])].tolist() == ora.tables[s]
    assert ora.cow_count == sum(len(p) for _, _, p in batch.log) > 0
    out = batch.step()
    torch.cuda.synchronize()
    _status_clean(pa)
    got = out.float().cpu().numpy()
    # each stream attends over its prompt followed by its own private tokens: every stream
    pkc, pvc = pk.float().cpu().numpy(), pv.float().cpu().numpy()
    xkc, xvc = xk.float().cpu().numpy(), xv.float().cpu().numpy()

    def rows(s):
        p = s // n
        return (np.concatenate([pkc[poff[p]:poff[p + 1]], xkc[xoff[s]:xoff[s + 1]]]),
                np.concatenate([pvc[poff[p]:poff[p + 1]], xvc[xoff[s]:xoff[s + 1]]]))

    ref = oracle_logical_all(q.float().cpu().numpy(), rows, wl.block_size, wl.scale)
    err = max_abs(got, ref)
    report_error("%s seed 0" % wl.name, err, wl.num_seqs * wl.num_heads)
    assert err <= TOL["bf16"], err


def test_cow_small_pool_bit_exact(pa, runner):
    """Small parallel-sampling run: the whole pool after all copy-on-write copies and
    appends equals the oracle's (oracle allocator + oracle copy + oracle scatter)."""
    wl = W.make_workload(4, seed=1, num_prompts=5, num_heads=4, num_kv_heads=2, head_dim=64,
                         prompt_lens=(17, 60), private_tokens=(1, 20), num_blocks=120)
    vals = W.cow_values(wl, "cpu")
    q, pk, pv, poff, xk, xv, xoff = vals
    batch = runner.CowBatch(wl, "cuda", values=vals)
    P, n, B = wl.num_prompts, wl.streams_per_prompt, wl.block_size
    ora = OracleAllocator(wl.num_blocks, B, wl.free_order)
    nb = nan_bits(wl.dtype)
    kp = np.full((wl.num_blocks, wl.num_kv_heads, B, wl.head_dim), nb)
    vp = np.full_like(kp, nb)
    slots = []
    for p in range(P):
        slots += ora.add_seq(p * n, int(wl.prompt_lens[p]))
    kp, vp = oracle.reshape_and_cache(bits(pk), bits(pv), kp, vp, np.array(slots))
    for p in range(P):
        for j in range(1, n):
            ora.fork(p * n, p * n + j)
    priv = np.asarray(wl.private_tokens)
    for t in range(int(priv.max())):
        active = [s for s in range(wl.num_seqs) if priv[s] > t]
        res = [ora.append_slot(s) for s in active]
        pairs = [r[1] for r in res if r[1] is not None]
        if pairs:
            kp, vp = oracle.copy_blocks(kp, vp, np.array(pairs))
        rows = [xoff[s] + t for s in active]
        kp, vp = oracle.reshape_and_cache(bits(xk)[rows], bits(xv)[rows], kp, vp, np.array([r[0] for r in res]))
    assert np.array_equal(bits(batch.k_cache), kp) and np.array_equal(bits(batch.v_cache), vp)
    mb = max(len(t) for t in ora.tables.values())
    tables = np.full((wl.num_seqs, mb), -1, np.int32)
    for s in range(wl.num_seqs):
        tables[s, :len(ora.tables[s])] = ora.tables[s]
    lens = np.array([ora.ntokens[s] for s in range(wl.num_seqs)], np.int32)
    ref = oracle.decode(bits_to_f32(bits(q)), bits_to_f32(kp), bits_to_f32(vp), tables, lens, wl.scale)
    out = batch.step()
    assert max_abs(out.float().cpu().numpy(), ref) <= TOL["bf16"]
    _status_clean(pa)


@pytest.mark.parametrize("wid,part,full", [(3, 0, False), (3, 0, True), (2, 256, False), (5, 512, False),
                                           (1, 0, False)])
def test_plan_once_then_run_per_layer(pa, runner, wid, part, full):
    """One plan per step, one run per layer: each run equals a whole pa_decode of the
    same layer bit for bit (the runs reuse the plan; the last CTA of each resets its
    work counter, or the next run would skip units).  The full-size GQA batch takes the
    1024-token starting partition, which plan and run must both choose."""
    over = {"num_seqs": 40, "num_blocks": 6000} if wid in (2, 3) and not full else {}
    wl = W.make_workload(wid, seed=2, **over)
    wl.partition_size = part
    batch = runner.DecodeBatch(wl, "cuda")
    batch.append()
    ws = torch.empty(pa.pa_decode_workspace_size(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim,
                                                 wl.block_size, batch.max_context_len, part) + 16,
                     dtype=torch.uint8, device="cuda")
    pa.pa_decode_plan(batch.block_tables, batch.context_lens, batch.max_context_len, wl.num_heads, batch.k_cache, ws,
                      part)
    if full:
        # 1024 (sequence, kv head) pairs and contexts up to 4096: the plan starts at 1024 tokens
        torch.cuda.synchronize()
        pb = int(ws[8:12].cpu().view(torch.int32)[0])
        assert pb * wl.block_size == 1024, pb
    g = torch.Generator(device="cuda").manual_seed(wid)
    for layer in range(4):
        q = torch.randn(batch.q.shape, generator=g, device="cuda").to(batch.q.dtype)
        kL = (batch.k_cache * (1.0 + 0.25 * layer)).contiguous()
        vL = (batch.v_cache * (1.0 - 0.125 * layer)).contiguous()
        got = torch.empty_like(q)
        pa.pa_decode_run(got, q, kL, vL, batch.block_tables, batch.context_lens, batch.max_context_len, wl.scale, ws,
                         part)
        ref = torch.empty_like(q)
        pa.pa_decode(ref, q, kL, vL, batch.block_tables, batch.context_lens, batch.max_context_len, wl.scale, part)
        torch.cuda.synchronize()
        assert torch.equal(bits_t(got), bits_t(ref)), "layer %d" % layer
    _status_clean(pa)


def bits_t(t):
    return t.view(torch.int32) if t.dtype == torch.float32 else t.view(torch.int16)


@pytest.mark.parametrize("G", [1, 4])
def test_adaptive_partition_grows_without_first_wave(pa, G):
    """A batch of 96 sequences of 12-16k tokens (1.36M tokens, more than four 1024-token
    partitions per CTA): the automatic partition grows in the plan kernel.  No CTA may
    then start before the plan (the first wave needs a partition length the host can
    fix), so this runs the path in which every CTA waits for the plan.  Every row matches
    the oracle, and a second run from the same plan gives the same bits."""
    S, Hkv, D, B = 96, 2, 128, 16
    Hq = Hkv * G
    rng = np.random.default_rng(40 + G)
    lens = rng.integers(12000, 16385, size=S).astype(np.int32)
    nblk = (lens + B - 1) // B
    NB = int(nblk.sum()) + 7
    perm = rng.permutation(NB).astype(np.int32)
    tables = np.full((S, int(nblk.max())), -1, np.int32)
    pos = 0
    for s in range(S):
        tables[s, :nblk[s]] = perm[pos:pos + nblk[s]]
        pos += nblk[s]
    g = torch.Generator(device="cuda").manual_seed(G)
    k = torch.randn((NB, Hkv, B, D), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((NB, Hkv, B, D), generator=g, device="cuda").to(torch.bfloat16)
    q = torch.randn((S, Hq, D), generator=g, device="cuda").to(torch.bfloat16)
    t_d = torch.from_numpy(tables).cuda()
    l_d = torch.from_numpy(lens).cuda()
    maxL = int(lens.max())
    ws = torch.zeros(pa.pa_decode_workspace_size(S, Hq, Hkv, D, B, maxL, 0) + 16, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    pa.pa_decode(out, q, k, v, t_d, l_d, maxL, D ** -0.5, 0, ws)
    torch.cuda.synchronize()
    _status_clean(pa)
    # the plan's partition (blocks per partition, third word of the work plan) grew past the smallest
    pb = int(ws[8:12].cpu().view(torch.int32).item())
    assert pb * B > pa.pa_decode_partition_size(S, Hq, Hkv, D, B, maxL, 0)
    again = torch.empty_like(q)
    pa.pa_decode_run(again, q, k, v, t_d, l_d, maxL, D ** -0.5, ws, 0)
    torch.cuda.synchronize()
    assert torch.equal(bits_t(again), bits_t(out))
    kc, vc = k.float().cpu().numpy(), v.float().cpu().numpy()

    def rows(s):
        blk = tables[s, :nblk[s]]
        kk = kc[blk].transpose(0, 2, 1, 3).reshape(-1, Hkv, D)[:lens[s]]
        vv = vc[blk].transpose(0, 2, 1, 3).reshape(-1, Hkv, D)[:lens[s]]
        return kk, vv

    ref = oracle_logical_all(q.float().cpu().numpy(), rows, B, D ** -0.5)
    err = max_abs(out.float().cpu().numpy(), ref)
    report_error("adaptive partition, G=%d (96 x 12-16k tokens)" % G, err, S * Hq)
    assert err <= TOL["bf16"], err
