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
from pa_testlib import TOL, max_abs

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


def _run(pa, q, k, v, tables, lens, q_start, scale):
    out = torch.full(q.shape, 7.0, dtype=torch.bfloat16, device="cuda")
    pa.pa_prefill(out, q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(),
                  torch.from_numpy(q_start).cuda(), int(np.max(np.diff(q_start))), scale)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


def _oracle(q, k, v, tables, lens, q_start, scale):
    return oracle.prefill(q.float().numpy(), np.nan_to_num(k.float().numpy()), np.nan_to_num(v.float().numpy()),
                          tables, lens, q_start, scale, nthreads=8)


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
    got = _run(pa, q, k, v, tables, L, qs, scale)
    assert np.isfinite(got).all()
    assert max_abs(got, _oracle(q, k, v, tables, L, qs, scale)) <= TOL["bf16"]
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


def test_long_chunk_sampled_rows(pa):
    lens, nq = [2100, 1500, 4096], [640, 1500, 300]
    q, k, v, tables, L, qs = _case(9, lens, nq, 32, 8, 16)
    scale = 128 ** -0.5
    got = _run(pa, q, k, v, tables, L, qs, scale)
    rows = np.array([0, 1, 127, 128, 639, 640, 641, 1500, 2139, 2140, 2439])
    # the oracle on the sampled rows only: each row is its own one-row chunk at its position
    ref = np.zeros((len(rows),) + q.shape[1:])
    for i, r in enumerate(rows):
        s = int(np.searchsorted(qs, r, side="right") - 1)
        pos = int(L[s] - (qs[s + 1] - qs[s]) + (r - qs[s]))
        ref[i] = oracle.prefill(q[r:r + 1].float().numpy(), np.nan_to_num(k.float().numpy()),
                                np.nan_to_num(v.float().numpy()), tables[s:s + 1], np.array([pos + 1], np.int32),
                                np.array([0, 1], np.int32), scale)[0]
    assert max_abs(got[rows], ref) <= TOL["bf16"]


def test_bad_chunk_is_flagged_and_skipped(pa):
    q, k, v, tables, L, qs = _case(3, [40, 20], [10, 20], 4, 2, 16)
    L_bad = L.copy()
    L_bad[1] = 19                               # 20 queries but only 19 tokens
    got = _run(pa, q, k, v, tables, L_bad, qs, 0.1)
    assert pa.pa_device_status() == pa.PA_DEV_BAD_CONTEXT
    assert np.all(got[10:] == 7.0)              # the bad sequence's rows are untouched
    assert max_abs(got[:10], _oracle(q[:10], k, v, tables[:1], L[:1], qs[:2], 0.1)) <= TOL["bf16"]


def test_unsupported_shapes_are_refused(pa):
    q = torch.zeros(4, 4, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(4, 2, 16, 64, dtype=torch.bfloat16, device="cuda")
    t = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    with pytest.raises(pa.PAError) as e:
        pa.pa_prefill(torch.empty_like(q), q, k, k, t, torch.tensor([4], dtype=torch.int32, device="cuda"),
                      torch.tensor([0, 4], dtype=torch.int32, device="cuda"), 4, 1.0)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED


def test_prefill_workload_full_size_sampled(pa):
    from paged_kv_cache_363_b200 import runner
    from paged_kv_cache_363_b200 import workloads as W
    from pa_testlib import oracle_logical
    wl = W.make_workload(8, seed=0)
    vals = W.prefill_values(wl, "cpu")
    batch = runner.PrefillBatch(wl, "cuda", values=vals)
    out = batch.step()
    torch.cuda.synchronize()
    assert pa.pa_device_status() == 0
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    q, keys, values = vals
    koff = np.concatenate([[0], np.cumsum(wl.context_lens)])
    qs = batch.q_start_np
    rows, ks, vs = [], [], []
    for s in (0, 5, wl.num_seqs - 1):
        for i in (0, 1, 511, int(wl.query_lens[s]) - 1):
            pos = int(wl.prefix_lens[s]) + i
            rows.append(int(qs[s]) + i)
            ks.append(keys[koff[s]:koff[s] + pos + 1].float().numpy())
            vs.append(values[koff[s]:koff[s] + pos + 1].float().numpy())
    ref = oracle_logical(q[rows].float().numpy(), ks, vs, wl.block_size, wl.scale)
    assert max_abs(got[rows], ref) <= TOL["bf16"]


@pytest.mark.parametrize("scale", [0.0, -0.06, 0.3])
def test_any_finite_scale(pa, scale):
    lens, nq = [130, 70], [130, 20]
    q, k, v, tables, L, qs = _case(21, lens, nq, 8, 2, 16)
    got = _run(pa, q, k, v, tables, L, qs, scale)
    assert np.isfinite(got).all()
    assert max_abs(got, _oracle(q, k, v, tables, L, qs, scale)) <= TOL["bf16"]
