"""Chunked prefill on the tensor cores (pa_prefill) against the oracle.

Each query row attends causally to its prefix through the block table; the oracle
computes the same in fp64 (oracle.prefill, pinned in tests/test_oracle_prefill.py).
bf16 output, fp32 accumulation: max-abs 2e-2.  Unused pool slots hold NaN, so a
stray read or an unmasked key shows up.
"""
import numpy as np
import pytest
import torch

from oracle import oracle
from pa_testlib import NTHREADS, TOL, max_abs, oracle_logical_prefill, report_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_363_b200 import pa as _pa
    return _pa


def _case(seed, lens, nq, Hq, Hkv, B, D=128):
    rng = np.random.default_rng(seed)
    g = torch.Generator().manual_seed(seed)
    S = len(lens)
    nblk = [-(-L // B) for L in lens]
    NB = sum(nblk) + 11
    order = rng.permutation(NB)
    tables = np.full((S, max(nblk)), -1, np.int32)
    pos = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = order[pos:pos + n]
        pos += n
    k = torch.full((NB, Hkv, B, D), float("nan"), dtype=torch.bfloat16)
    v = torch.full((NB, Hkv, B, D), float("nan"), dtype=torch.bfloat16)
    for s, L in enumerate(lens):          # fill exactly the slots of the context tokens
        for t in range(L):
            k[tables[s][t // B], :, t % B] = torch.randn(Hkv, D, generator=g).to(torch.bfloat16)
            v[tables[s][t // B], :, t % B] = torch.randn(Hkv, D, generator=g).to(torch.bfloat16)
    q_start = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    q = torch.randn(int(q_start[-1]), Hq, D, generator=g).to(torch.bfloat16)
    return q, k, v, tables, np.array(lens, np.int32), q_start


def _run(pa, q, k, v, tables, lens, q_start, scale, ws=True, calls=1):
    """pa_prefill_ws (one CTA per SM taking items from a counter) or, with ws=False, pa_prefill (one item per
    CTA); `calls` > 1 repeats the call on the same workspace and checks that every call gives the same bits."""
    out = torch.full(q.shape, 7.0, dtype=torch.bfloat16, device="cuda")
    workspace = torch.empty(pa.pa_prefill_workspace_size(), dtype=torch.uint8, device="cuda") if ws else None
    first = None
    for _ in range(calls):
        pa.pa_prefill(out, q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(tables).cuda(),
                      torch.from_numpy(lens).cuda(), torch.from_numpy(q_start).cuda(), int(np.max(np.diff(q_start))),
                      scale, workspace=workspace)
        torch.cuda.synchronize()
        if first is None:
            first = out.clone()
        else:
            assert torch.equal(out, first), "a repeated call on the same workspace changed the output"
    return out.float().cpu().numpy()


def _oracle(q, k, v, tables, lens, q_start, scale):
    return oracle.prefill(q.float().numpy(), np.nan_to_num(k.float().numpy()), np.nan_to_num(v.float().numpy()),
                          tables, lens, q_start, scale, nthreads=NTHREADS)


CASES = [
    # (lens, query counts): full prefills, chunks, single tokens, ragged tiles of q and of keys
    ([1, 17, 128, 129, 300], [1, 17, 128, 129, 300]),
    ([200, 531, 64, 1000], [13, 200, 1, 77]),
    ([700, 33], [1, 1]),
    ([257], [257]),
]


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("B", [16, 32])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_prefill_matches_oracle(pa, G, B, case):
    lens, nq = CASES[case]
    Hkv = 2
    q, k, v, tables, L, qs = _case(100 * G + B + case, lens, nq, Hkv * G, Hkv, B)
    scale = 128 ** -0.5
    got = _run(pa, q, k, v, tables, L, qs, scale, calls=2)
    assert np.isfinite(got).all()
    assert max_abs(got, _oracle(q, k, v, tables, L, qs, scale)) <= TOL["bf16"]
    # the grid of one item per CTA computes each item the same way: the same bits
    assert np.array_equal(_run(pa, q, k, v, tables, L, qs, scale, ws=False), got)
    assert pa.pa_device_status() == 0


def test_single_token_chunks_agree_with_decode(pa):
    lens = [5, 300, 129, 1000, 16]
    q, k, v, tables, L, qs = _case(7, lens, [1] * 5, 32, 8, 16)
    scale = 0.09
    got = _run(pa, q, k, v, tables, L, qs, scale)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    pa.pa_decode(out, q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(tables).cuda(), torch.from_numpy(L).cuda(),
                 int(L.max()), scale, 0)
    torch.cuda.synchronize()
    assert max_abs(got, out.float().cpu().numpy()) <= TOL["bf16"]


def test_long_chunk_every_row(pa):
    lens, nq = [2100, 1500, 4096], [640, 1500, 300]
    q, k, v, tables, L, qs = _case(9, lens, nq, 32, 8, 16)
    scale = 128 ** -0.5
    got = _run(pa, q, k, v, tables, L, qs, scale)
    err = max_abs(got, _oracle(q, k, v, tables, L, qs, scale))
    report_error("prefill long chunks (contexts 2100/1500/4096)", err, got.shape[0] * got.shape[1])
    assert err <= TOL["bf16"], err


def test_bad_chunk_is_flagged_and_skipped(pa):
    q, k, v, tables, L, qs = _case(3, [40, 20], [10, 20], 4, 2, 16)
    L_bad = L.copy()
    L_bad[1] = 19                               # 20 queries but only 19 tokens
    got = _run(pa, q, k, v, tables, L_bad, qs, 0.1)
    assert pa.pa_device_status() == pa.PA_DEV_BAD_CONTEXT
    assert np.all(got[10:] == 7.0)              # the bad sequence's rows are untouched
    assert max_abs(got[:10], _oracle(q[:10], k, v, tables[:1], L[:1], qs[:2], 0.1)) <= TOL["bf16"]


@pytest.mark.parametrize("ws", [True, False])
@pytest.mark.parametrize("bad", ["past_end", "backwards", "negative_start", "over_max_query_len"])
def test_bad_query_rows_are_flagged_and_skipped(pa, bad, ws):
    """q_start is device data: a sequence whose query rows leave [0, num_query_tokens),
    run backwards, or outnumber max_query_len is flagged and skipped whole before any
    store, and the other sequence still matches the oracle."""
    lens, nq = [60, 70], [10, 20]
    q, k, v, tables, L, qs = _case(31, lens, nq, 8, 2, 16)
    max_q = 20
    good = 0                                   # the sequence left intact
    qs_bad = qs.copy()
    if bad == "past_end":
        qs_bad[2] = qs[2] + 5                   # rows 10..34 of a 30-row q
    elif bad == "backwards":
        qs_bad[2] = 5                           # sequence 1 would run from row 10 back to row 5
    elif bad == "negative_start":
        qs_bad[0] = -5                          # sequence 0 starts before row 0
        good = 1
    elif bad == "over_max_query_len":
        max_q = 15                              # sequence 1 has 20 rows
    out = torch.full(q.shape, 7.0, dtype=torch.bfloat16, device="cuda")
    workspace = torch.empty(pa.pa_prefill_workspace_size(), dtype=torch.uint8, device="cuda") if ws else None
    pa.pa_prefill(out, q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(tables).cuda(), torch.from_numpy(L).cuda(),
                  torch.from_numpy(qs_bad).cuda(), max_q, 0.1, workspace=workspace)
    torch.cuda.synchronize()
    assert pa.pa_device_status() == pa.PA_DEV_BAD_CONTEXT
    got = out.float().cpu().numpy()
    ref = _oracle(q, k, v, tables, L, qs, 0.1)
    if good == 0:
        assert np.all(got[10:] == 7.0)         # the bad sequence's rows are untouched
        assert max_abs(got[:10], ref[:10]) <= TOL["bf16"]
    else:
        assert np.all(got[:10] == 7.0)
        assert max_abs(got[10:], ref[10:]) <= TOL["bf16"]
    assert pa.pa_device_status() == 0


def test_unsupported_shapes_are_refused(pa):
    q = torch.zeros(4, 4, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(4, 2, 16, 64, dtype=torch.bfloat16, device="cuda")
    t = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    with pytest.raises(pa.PAError) as e:
        pa.pa_prefill(torch.empty_like(q), q, k, k, t, torch.tensor([4], dtype=torch.int32, device="cuda"),
                      torch.tensor([0, 4], dtype=torch.int32, device="cuda"), 4, 1.0)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED


def test_prefill_workload_full_size_every_row(pa):
    """The bench's prefill workload at full size: all 16,384 query rows of the 16
    sequences against the oracle, sequence by sequence."""
    from paged_kv_cache_363_b200 import runner
    from paged_kv_cache_363_b200 import workloads as W
    wl = W.make_workload(8, seed=0)
    vals = W.prefill_values(wl, "cpu")
    batch = runner.PrefillBatch(wl, "cuda", values=vals)
    out = batch.step()
    torch.cuda.synchronize()
    assert pa.pa_device_status() == 0
    got = out.float().cpu().numpy()
    q, keys, values = vals
    koff = np.concatenate([[0], np.cumsum(wl.context_lens)])
    qs = batch.q_start_np
    err = 0.0
    for s in range(wl.num_seqs):
        L = int(wl.context_lens[s])
        ref = oracle_logical_prefill(q[qs[s]:qs[s + 1]].float().numpy(), keys[koff[s]:koff[s] + L].float().numpy(),
                                     values[koff[s]:koff[s] + L].float().numpy(), wl.block_size, wl.scale)
        err = max(err, max_abs(got[qs[s]:qs[s + 1]], ref))
    report_error("%s seed 0" % wl.name, err, got.shape[0] * got.shape[1])
    assert err <= TOL["bf16"], err


@pytest.mark.parametrize("scale", [0.0, -0.06, 0.3])
def test_any_finite_scale(pa, scale):
    lens, nq = [130, 70], [130, 20]
    q, k, v, tables, L, qs = _case(21, lens, nq, 8, 2, 16)
    got = _run(pa, q, k, v, tables, L, qs, scale)
    assert np.isfinite(got).all()
    assert max_abs(got, _oracle(q, k, v, tables, L, qs, scale)) <= TOL["bf16"]


def test_workspace_call_replays_from_a_cuda_graph(pa):
    """pa_prefill_ws zeroes its counter on the stream before the launch, so a captured call replays: every
    replay of the graph gives the direct call's bits."""
    q, k, v, tables, L, qs = _case(77, [300, 129, 1000], [300, 17, 64], 8, 2, 16)
    want = _run(pa, q, k, v, tables, L, qs, 0.09)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    td, ld, sd = torch.from_numpy(tables).cuda(), torch.from_numpy(L).cuda(), torch.from_numpy(qs).cuda()
    ws = torch.empty(pa.pa_prefill_workspace_size(), dtype=torch.uint8, device="cuda")
    out = torch.full(q.shape, 7.0, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        pa.pa_prefill(out, qd, kd, vd, td, ld, sd, int(np.max(np.diff(qs))), 0.09, stream=s, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        pa.pa_prefill(out, qd, kd, vd, td, ld, sd, int(np.max(np.diff(qs))), 0.09,
                      stream=torch.cuda.current_stream(), workspace=ws)
    for _ in range(3):
        out.fill_(7.0)
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(out.float().cpu().numpy(), want)
    assert pa.pa_device_status() == 0
    del g


@pytest.mark.parametrize("ws", [True, False])
def test_sequences_without_queries(pa, ws):
    """Sequences with no query rows (n_s = 0, with or without context) have no work items; the others match the
    oracle and no status bit is raised."""
    lens, nq = [50, 0, 300, 40, 1], [10, 0, 0, 40, 1]
    q, k, v, tables, L, qs = _case(91, [max(x, 1) for x in lens], nq, 4, 2, 16)
    L = np.array(lens, np.int32)
    got = _run(pa, q, k, v, tables, L, qs, 0.1, ws=ws)
    assert pa.pa_device_status() == 0
    assert max_abs(got, _oracle(q, k, v, tables, L, qs, 0.1)) <= TOL["bf16"]


def test_many_small_items_through_the_ring(pa):
    """4,800 items of one to four key tiles each (600 short sequences x 8 kv heads): every CTA of the
    persistent grid takes ~32 of them, so the two-slot item ring is refilled as fast as it can be.  A reader
    that used a slot after releasing it would put rows in the wrong place; every row is compared."""
    rng = np.random.default_rng(31)
    g = torch.Generator().manual_seed(31)
    S, Hkv, G, B, D = 600, 8, 4, 16, 128
    lens = rng.integers(1, 201, size=S).astype(np.int32)
    nq = np.minimum(lens, rng.integers(1, 41, size=S)).astype(np.int32)
    nblk = -(-lens // B)
    NB = int(nblk.sum()) + 7
    order = rng.permutation(NB).astype(np.int32)
    tables = np.full((S, int(nblk.max())), -1, np.int32)
    starts = np.concatenate([[0], np.cumsum(nblk)])
    for s in range(S):
        tables[s, :nblk[s]] = order[starts[s]:starts[s + 1]]
    # the context's slots get random rows; every other slot of the pools stays NaN
    tok_s = np.repeat(np.arange(S), lens)
    tok_t = np.concatenate([np.arange(L) for L in lens])
    blk = torch.from_numpy(tables[tok_s, tok_t // B].astype(np.int64))
    off = torch.from_numpy((tok_t % B).astype(np.int64))
    k = torch.full((NB, Hkv, B, D), float("nan"), dtype=torch.bfloat16)
    v = torch.full((NB, Hkv, B, D), float("nan"), dtype=torch.bfloat16)
    k[blk, :, off] = torch.randn(len(tok_s), Hkv, D, generator=g).to(torch.bfloat16)
    v[blk, :, off] = torch.randn(len(tok_s), Hkv, D, generator=g).to(torch.bfloat16)
    q_start = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    q = torch.randn(int(q_start[-1]), Hkv * G, D, generator=g).to(torch.bfloat16)
    scale = 128 ** -0.5
    got = _run(pa, q, k, v, tables, lens, q_start, scale, calls=3)
    assert np.isfinite(got).all()
    err = max_abs(got, _oracle(q, k, v, tables, lens, q_start, scale))
    report_error("prefill, 600 short sequences (4,800 small items)", err, got.shape[0] * got.shape[1])
    assert err <= TOL["bf16"], err
    assert np.array_equal(_run(pa, q, k, v, tables, lens, q_start, scale, ws=False), got)
    assert pa.pa_device_status() == 0
