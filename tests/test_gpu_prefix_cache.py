"""Prefix caching on the GPU path ("PagedAttention Paper Breakdown", "Paper Methods":
shared prefix caching in a radix tree), against the oracle.

Requests share system prompts; the library allocator's prefix cache places them and
only the tokens past the cached prefix are written.  The library's tables must equal
the oracle allocator's on the same script, the pools must equal the oracle's scatter
of the same rows bit for bit, and decode through the shared tables must match the
oracle's attention over each request's own logical tokens.
"""
import numpy as np
import pytest
import torch

from oracle import oracle
from oracle.allocator import OracleAllocator
from paged_kv_cache_363_b200 import workloads as W
from pa_testlib import TOL, bits, bits_to_f32, max_abs, nan_bits, oracle_logical, oracle_logical_all, report_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def runner():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_363_b200 import runner as _r
    return _r


def _logical(wl, vals, r):
    """Request r's logical K/V rows (its stem's, then its own suffix's), fp32."""
    q, sk, sv, soff, xk, xv, xoff = vals
    rows = W.prefix_logical_rows(wl, r, soff, xoff)
    which = np.array([s for s, _ in rows])
    idx = torch.tensor([i for _, i in rows], dtype=torch.int64)
    out = []
    for stem, own in ((sk, xk), (sv, xv)):
        x = torch.empty((len(rows),) + tuple(stem.shape[1:]), dtype=torch.float32)
        m0, m1 = torch.from_numpy(which == 0), torch.from_numpy(which == 1)
        x[m0] = stem[idx[m0]].float()
        x[m1] = own[idx[m1]].float()
        out.append(x.numpy())
    return out[0], out[1]


@pytest.mark.parametrize("seed", [0, 1])
def test_small_prefix_batch_bit_exact_against_oracle(runner, seed):
    wl = W.make_workload(6, seed=seed, num_prompts=3, requests_per_prompt=4, stem_lens=(20, 70),
                         suffix_lens=(1, 40), num_blocks=300)
    vals = W.prefix_values(wl, "cpu")
    batch = runner.PrefixBatch(wl, "cuda", values=vals)
    torch.cuda.synchronize()
    q, sk, sv, soff, xk, xv, xoff = vals
    S, Hkv, D, B, NB = wl.num_seqs, wl.num_kv_heads, wl.head_dim, wl.block_size, wl.num_blocks
    # the oracle replays the same script: prompts by token ids, then one append each
    ora = OracleAllocator(NB, B, wl.free_order)
    nb = nan_bits(wl.dtype)
    kpool = np.full((NB, Hkv, B, D), nb)
    vpool = np.full((NB, Hkv, B, D), nb)
    srcbits = {0: (bits(sk), bits(sv)), 1: (bits(xk), bits(xv))}
    for r in range(S):
        slots, nc = ora.add_seq_cached(r, wl.tokens(r)[:-1])
        assert nc == batch.cached_tokens[r]
        rows = W.prefix_logical_rows(wl, r, soff, xoff)[:-1]
        for src in (0, 1):
            pick = [(i, sl) for (s_, i), sl in zip(rows[nc:], slots[nc:]) if s_ == src]
            if pick:
                kb, vb = srcbits[src]
                idx = [i for i, _ in pick]
                kpool, vpool = oracle.reshape_and_cache(kb[idx], vb[idx], kpool, vpool,
                                                        np.array([sl for _, sl in pick]))
    assert sum(batch.cached_tokens) > 0                       # later requests hit their stems
    new = ora.append_slots(list(range(S)))
    assert batch.slot_mapping.cpu().tolist() == [x for x, _ in new]
    kb, vb = srcbits[1]
    last = [int(xoff[r + 1]) - 1 for r in range(S)]
    kpool, vpool = oracle.reshape_and_cache(kb[last], vb[last], kpool, vpool, np.array([x for x, _ in new]))
    mb = batch.block_tables.shape[1]
    tables = np.full((S, mb), -1, np.int32)
    for r in range(S):
        tables[r, :len(ora.tables[r])] = ora.tables[r]
    assert np.array_equal(batch.block_tables.cpu().numpy(), tables)
    out = batch.step()
    torch.cuda.synchronize()
    assert np.array_equal(bits(batch.k_cache), kpool) and np.array_equal(bits(batch.v_cache), vpool)
    lens = np.array([ora.ntokens[r] for r in range(S)], np.int32)
    ref = oracle.decode(bits_to_f32(bits(q)), bits_to_f32(kpool), bits_to_f32(vpool), tables, lens, wl.scale,
                        nthreads=4)
    assert max_abs(out.float().cpu().numpy(), ref) <= TOL[wl.dtype]
    # and the shared tables give each request its own logical attention
    ks, vs = zip(*[_logical(wl, vals, r) for r in range(S)])
    logical = oracle_logical(q.float().numpy(), list(ks), list(vs), B, wl.scale)
    assert max_abs(out.float().cpu().numpy(), logical) <= TOL[wl.dtype]


def test_full_size_prefix_batch_every_row(runner):
    wl = W.make_workload(6, seed=0)
    vals = W.prefix_values(wl, "cpu")
    batch = runner.PrefixBatch(wl, "cuda", values=vals)
    out = batch.step()
    torch.cuda.synchronize()
    from paged_kv_cache_363_b200 import pa
    assert pa.pa_device_status() == 0
    S, B = wl.num_seqs, wl.block_size
    # blocks in use = distinct full-block prefixes + one private partial per request
    prompts = [wl.tokens(r)[:-1] for r in range(S)]
    prefixes = {tuple(p[:(j + 1) * B]) for p in prompts for j in range(len(p) // B)}
    st = batch.alloc.stats()
    assert st["cached_blocks"] == len(prefixes)
    assert batch.written_tokens < sum(len(p) for p in prompts) // 2
    got = out.float().cpu().numpy()
    # every request against the oracle's attention over its own logical tokens
    q = vals[0]
    ref = oracle_logical_all(q.float().numpy(), lambda r: _logical(wl, vals, r), B, wl.scale)
    err = max_abs(got, ref)
    report_error("%s seed 0" % wl.name, err, S * wl.num_heads)
    assert err <= TOL["bf16"], err
