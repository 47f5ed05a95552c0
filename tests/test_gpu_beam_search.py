"""Beam search on the GPU path ([fullstackaihub] section 3 and [initnode] section 3:
beams share blocks by copy-on-write until one writes), against the oracle.

Every beam step goes through pa_alloc_beam_step, one pa_copy_blocks for the step's
copies and one pa_reshape_and_cache for the new tokens.  The oracle allocator replays
the same steps with the oracle's copy and scatter: tables, slots, copy pairs and both
pools must match bit for bit, and decode must match the oracle's attention over each
beam's own history (prompt, then the tokens of its ancestors and itself).
"""
import numpy as np
import pytest
import torch

from oracle import oracle
from oracle.allocator import OracleAllocator
from paged_kv_cache_363_b200 import workloads as W
from pa_testlib import TOL, bits, bits_to_f32, max_abs, nan_bits, oracle_logical, report_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def runner():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_363_b200 import runner as _r
    return _r


def _logical(wl, vals, beams):
    """Each beam's logical K/V rows (prompt rows, then its ancestors' and its own new
    tokens), fp32."""
    q, pk, pv, poff, nk, nv = vals
    hist = W.beam_histories(wl, poff)
    ks, vs = [], []
    for b in beams:
        which = torch.tensor([s for s, _ in hist[b]]) == 0
        idx = torch.tensor([i for _, i in hist[b]], dtype=torch.int64)
        for prompt, new, acc in ((pk, nk, ks), (pv, nv, vs)):
            x = torch.empty((len(idx),) + tuple(prompt.shape[1:]), dtype=torch.float32)
            x[which] = prompt[idx[which]].float()
            x[~which] = new[idx[~which]].float()
            acc.append(x.numpy())
    return ks, vs


@pytest.mark.parametrize("seed,B", [(0, 16), (1, 16), (2, 32)])
def test_small_beam_search_bit_exact_against_oracle(runner, seed, B):
    wl = W.make_workload(7, seed=seed, num_requests=3, beam_width=3, prompt_lens=(20, 70), beam_steps=12,
                         block_size=B, num_blocks=300)
    vals = W.beam_values(wl, "cpu")
    batch = runner.BeamBatch(wl, "cuda", values=vals)
    out = batch.step()
    torch.cuda.synchronize()
    q, pk, pv, poff, nk, nv = vals
    S, Wd, Hkv, D, NB = wl.num_seqs, wl.beam_width, wl.num_kv_heads, wl.head_dim, wl.num_blocks
    ora = OracleAllocator(NB, B, wl.free_order)
    nb = nan_bits(wl.dtype)
    kpool = np.full((NB, Hkv, B, D), nb)
    vpool = np.full((NB, Hkv, B, D), nb)
    slots = []
    for r in range(wl.num_requests):
        slots += ora.add_seq(r * Wd, int(wl.prompt_lens[r]))
        for j in range(1, Wd):
            ora.fork(r * Wd, r * Wd + j)
    kpool, vpool = oracle.reshape_and_cache(bits(pk), bits(pv), kpool, vpool, np.array(slots))
    ids = list(range(S))
    ncopies = 0
    for t in range(wl.beam_steps):
        res = ora.beam_step(ids, wl.parents[t].tolist(), ids)
        pairs = [c for _, c in res if c is not None]
        ncopies += len(pairs)
        if pairs:
            kpool, vpool = oracle.copy_blocks(kpool, vpool, np.array(pairs))
        kpool, vpool = oracle.reshape_and_cache(bits(nk[t * S:(t + 1) * S]), bits(nv[t * S:(t + 1) * S]), kpool,
                                                vpool, np.array([x for x, _ in res]))
    assert ncopies == sum(batch.copies_per_step) and ncopies > 0
    assert batch.slot_mapping.cpu().tolist() == [x for x, _ in res]
    assert [tuple(p) for p in batch.cow_pairs.cpu().tolist()] == pairs
    mb = batch.block_tables.shape[1]
    tables = np.full((S, mb), -1, np.int32)
    for b in ids:
        tables[b, :len(ora.tables[b])] = ora.tables[b]
    assert np.array_equal(batch.block_tables.cpu().numpy(), tables)
    assert np.array_equal(bits(batch.k_cache), kpool) and np.array_equal(bits(batch.v_cache), vpool)
    lens = np.array([ora.ntokens[b] for b in ids], np.int32)
    ref = oracle.decode(bits_to_f32(bits(q)), bits_to_f32(kpool), bits_to_f32(vpool), tables, lens, wl.scale,
                        nthreads=4)
    got = out.float().cpu().numpy()
    assert max_abs(got, ref) <= TOL[wl.dtype]
    ks, vs = _logical(wl, vals, ids)
    assert max_abs(got, oracle_logical(q.float().numpy(), ks, vs, B, wl.scale)) <= TOL[wl.dtype]
    # the step repeats: copies and append rewrite the same bytes
    batch.step()
    torch.cuda.synchronize()
    assert np.array_equal(bits(batch.k_cache), kpool)


def test_full_size_beam_search_every_row(runner):
    wl = W.make_workload(7, seed=0)
    vals = W.beam_values(wl, "cpu")
    batch = runner.BeamBatch(wl, "cuda", values=vals)
    out = batch.step()
    torch.cuda.synchronize()
    from paged_kv_cache_363_b200 import pa
    assert pa.pa_device_status() == 0
    got = out.float().cpu().numpy()
    ks, vs = _logical(wl, vals, range(wl.num_seqs))
    ref = oracle_logical(vals[0].float().numpy(), ks, vs, wl.block_size, wl.scale)
    err = max_abs(got, ref)
    report_error("%s seed 0" % wl.name, err, wl.num_seqs * wl.num_heads)
    assert err <= TOL["bf16"], err
