"""Pins of the oracle's chunked prefill (CPU only).

Query i of a sequence with L tokens and n queries sits at position L - n + i and
attends causally to tokens 0..L-n+i through the block table.  Pinned against: torch
SDPA with its own causal flag when the whole sequence is the query (n = L), SDPA
with the bottom-right causal mask for chunks, the independently pinned decode oracle
when every chunk is one token, exact invariance under block placement, the first
token's closed form (its output is V_0), and a pure-Python brute force.
"""
import numpy as np
import pytest
import torch

from oracle import oracle


def _case(rng, lens, nq, Hq, Hkv, D, B, perm=True):
    S = len(lens)
    nblk = [-(-L // B) for L in lens]
    NB = sum(nblk) + 3
    order = rng.permutation(NB) if perm else np.arange(NB)
    tables = np.full((S, max(nblk)), -1, np.int32)
    pos = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = order[pos:pos + n]
        pos += n
    k = rng.standard_normal((NB, Hkv, B, D)).astype(np.float32)
    v = rng.standard_normal((NB, Hkv, B, D)).astype(np.float32)
    q_start = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    q = rng.standard_normal((int(q_start[-1]), Hq, D)).astype(np.float32)
    return q, k, v, tables, np.array(lens, np.int32), q_start


def _logical(k, tables, s, L, B):
    """[L, Hkv, D] rows of sequence s in logical order."""
    return np.stack([k[tables[s][i // B], :, i % B] for i in range(L)])


def _sdpa(q, kl, vl, scale, G, mask=None, causal=False):
    qt = torch.from_numpy(q.astype(np.float64)).permute(1, 0, 2)[None]              # [1, Hq, n, D]
    kt = torch.from_numpy(kl.astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)[None]
    vt = torch.from_numpy(vl.astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, is_causal=causal, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("G", [1, 4])
def test_whole_sequence_as_query_is_causal_sdpa(G):
    rng = np.random.default_rng(G)
    Hkv, D, B = 2, 16, 4
    lens = [1, 7, 13]
    q, k, v, tables, L, qs = _case(rng, lens, lens, Hkv * G, Hkv, D, B)
    out = oracle.prefill(q, k, v, tables, L, qs, 0.37)
    for s, Ls in enumerate(lens):
        ref = _sdpa(q[qs[s]:qs[s + 1]], _logical(k, tables, s, Ls, B), _logical(v, tables, s, Ls, B), 0.37, G,
                    causal=True)
        assert np.allclose(out[qs[s]:qs[s + 1]], ref, rtol=0, atol=1e-12)


def test_chunk_is_bottom_right_causal_sdpa():
    rng = np.random.default_rng(3)
    Hkv, G, D, B = 2, 2, 8, 4
    lens, nq = [9, 20, 5], [3, 7, 5]
    q, k, v, tables, L, qs = _case(rng, lens, nq, Hkv * G, Hkv, D, B)
    out = oracle.prefill(q, k, v, tables, L, qs, 0.3)
    for s, (Ls, n) in enumerate(zip(lens, nq)):
        mask = torch.tensor([[t <= Ls - n + i for t in range(Ls)] for i in range(n)])
        ref = _sdpa(q[qs[s]:qs[s + 1]], _logical(k, tables, s, Ls, B), _logical(v, tables, s, Ls, B), 0.3, G,
                    mask=mask)
        assert np.allclose(out[qs[s]:qs[s + 1]], ref, rtol=0, atol=1e-12)


def test_one_token_chunks_are_the_decode_oracle():
    rng = np.random.default_rng(4)
    lens = [5, 1, 33, 16]
    q, k, v, tables, L, qs = _case(rng, lens, [1] * 4, 8, 2, 16, 8)
    out = oracle.prefill(q, k, v, tables, L, qs, 0.25)
    ref = oracle.decode(q, k, v, tables, L, 0.25)
    assert np.array_equal(out, ref)


def test_placement_does_not_change_the_result_and_first_token_is_v0():
    rng = np.random.default_rng(5)
    lens, nq = [11, 6], [11, 2]
    q, k, v, tables, L, qs = _case(rng, lens, nq, 4, 2, 8, 4, perm=False)
    out = oracle.prefill(q, k, v, tables, L, qs, 0.5)
    # move every block to a new place and rewrite the tables
    NB = k.shape[0]
    perm = rng.permutation(NB)
    k2, v2 = np.empty_like(k), np.empty_like(v)
    k2[perm], v2[perm] = k, v
    t2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1).astype(np.int32)
    assert np.array_equal(oracle.prefill(q, k2, v2, t2, L, qs, 0.5), out)
    # the first query of a sequence starting at position 0 sees one token: out = V_0
    for h in range(4):
        assert np.array_equal(out[0, h], v[tables[0][0], h // 2, 0].astype(np.float64))


def test_pure_python_brute_force_tiny():
    rng = np.random.default_rng(6)
    lens, nq = [6, 4], [4, 2]
    q, k, v, tables, L, qs = _case(rng, lens, nq, 2, 1, 4, 2)
    out = oracle.prefill(q, k, v, tables, L, qs, 0.7)
    for s in range(2):
        for i in range(nq[s]):
            p = lens[s] - nq[s] + i
            row = q[qs[s] + i][None]
            ref = oracle.decode_bruteforce(row, k, v, tables[s:s + 1], np.array([p + 1]), 0.7)
            assert np.allclose(out[qs[s] + i], ref[0], rtol=0, atol=1e-12)


def test_bad_arguments_are_rejected():
    rng = np.random.default_rng(7)
    q, k, v, tables, L, qs = _case(rng, [4], [4], 2, 1, 4, 2)
    with pytest.raises(ValueError):
        oracle.prefill(q, k, v, tables, np.array([3], np.int32), qs, 1.0)     # more queries than tokens


# ---- the pins catch plausible mistakes: a CPU restatement with one planted at a time

PREFILL_MUTATIONS = ["none", "top_left_causal", "position_off_by_one", "sees_next_token", "kv_head_modulo"]


def _prefill_copy(q, k, v, tables, L, qs, scale, mut):
    Hq, D = q.shape[1], q.shape[2]
    NB, Hkv, B, _ = k.shape
    G = Hq // Hkv
    out = np.zeros(q.shape)
    for s in range(len(L)):
        n = int(qs[s + 1] - qs[s])
        for i in range(n):
            p = {"top_left_causal": i, "position_off_by_one": L[s] - n + i - 1,
                 "sees_next_token": min(L[s] - 1, L[s] - n + i + 1)}.get(mut, L[s] - n + i)
            for h in range(Hq):
                kvh = h % Hkv if mut == "kv_head_modulo" else h // G
                rows = [(tables[s][t // B], t % B) for t in range(p + 1)]
                z = np.array([scale * float(q[qs[s] + i, h].astype(np.float64) @ k[b, kvh, o].astype(np.float64))
                              for b, o in rows])
                w = np.exp(z - z.max())
                w /= w.sum()
                out[qs[s] + i, h] = sum(wt * v[b, kvh, o].astype(np.float64) for wt, (b, o) in zip(w, rows))
    return out


def _passes_pins(mut):
    rng = np.random.default_rng(11)
    Hkv, G, D, B = 2, 2, 8, 4
    for lens, nq in (([7, 12], [7, 12]), ([9, 14], [3, 6])):
        q, k, v, tables, L, qs = _case(rng, lens, nq, Hkv * G, Hkv, D, B)
        try:
            got = _prefill_copy(q, k, v, tables, L, qs, 0.4, mut)
        except ValueError:                          # e.g. a row left with no token at all
            return False
        for s, (Ls, n) in enumerate(zip(lens, nq)):
            mask = torch.tensor([[t <= Ls - n + i for t in range(Ls)] for i in range(n)])
            ref = _sdpa(q[qs[s]:qs[s + 1]], _logical(k, tables, s, Ls, B), _logical(v, tables, s, Ls, B), 0.4, G,
                        mask=mask)
            if not np.allclose(got[qs[s]:qs[s + 1]], ref, rtol=0, atol=1e-10):
                return False
    return True


@pytest.mark.parametrize("mut", PREFILL_MUTATIONS)
def test_planted_prefill_mistakes_fail_a_pin(mut):
    assert _passes_pins(mut) == (mut == "none")
