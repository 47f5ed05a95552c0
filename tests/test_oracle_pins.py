"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test pins the oracle to something it does not compute itself: the worked
examples the pages print, a library routine on a special case (torch's
scaled_dot_product_attention when the block table is the identity), invariants
(permutation of physical blocks, weights summing to one), closed forms and an
independent pure-Python brute force.
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from oracle import oracle
from paged_kv_cache_363_b200 import workloads as W


def _pool(NB, Hkv, B, D, rng, dtype=np.float32):
    return rng.standard_normal((NB, Hkv, B, D)).astype(dtype)


def _random_case(rng, S=3, Hq=4, Hkv=2, D=16, B=4, NB=40, maxL=23, lens=None):
    if lens is None:
        lens = rng.integers(0, maxL + 1, size=S).astype(np.int32)
    lens = np.asarray(lens, np.int32)
    MB = max(1, -(-int(lens.max()) // B))
    perm = rng.permutation(NB)
    tables = np.full((S, MB), -1, np.int32)
    pos = 0
    for s in range(S):
        n = -(-int(lens[s]) // B)
        tables[s, :n] = perm[pos:pos + n]
        pos += n
    q = rng.standard_normal((S, Hq, D)).astype(np.float32)
    k = _pool(NB, Hkv, B, D, rng)
    v = _pool(NB, Hkv, B, D, rng)
    return q, k, v, tables, lens


# ---------------------------------------------------------------- translation

def test_translation_matches_fullstackaihub_worked_example():
    hdr, rows = read_golden("translation_fullstackaihub.txt")
    B, table = hdr["block_size"], hdr["table"]
    for tok, blk, off, slot in rows:
        got = oracle.physical_slot(table, B, tok)
        assert got == slot
        assert (got // B, got % B) == (blk, off)


def test_translation_matches_initnode_walk():
    hdr, rows = read_golden("walk_initnode.txt")
    B, table = hdr["block_size"], hdr["table"]
    for tok, blk, off, slot in rows:
        assert oracle.physical_slot(table, B, tok) == slot
    # tokens in logical order visit the physical blocks in table order
    visited = []
    for i in range(len(table) * B):
        p = oracle.physical_slot(table, B, i) // B
        if not visited or visited[-1] != p:
            visited.append(p)
    assert visited == list(table)


def test_translation_brute_force_all_tokens():
    rng = np.random.default_rng(5)
    for B in (16, 32):
        table = rng.permutation(1000)[:37].astype(np.int32)
        for i in range(37 * B):
            assert oracle.physical_slot(table, B, i) == int(table[i // B]) * B + (i % B)


# ---------------------------------------------------------------- decode

def _sdpa_reference(q, k_seq, v_seq, scale):
    """Contiguous attention of one sequence with torch's SDPA in fp64.
    q [Hq, D]; k_seq, v_seq [L, Hkv, D]; GQA by repeating kv heads consecutively."""
    Hq = q.shape[0]
    Hkv = k_seq.shape[1]
    qt = torch.from_numpy(q.astype(np.float64))[:, None, :]            # [Hq, 1, D]
    kt = torch.from_numpy(k_seq.astype(np.float64)).permute(1, 0, 2)    # [Hkv, L, D]
    vt = torch.from_numpy(v_seq.astype(np.float64)).permute(1, 0, 2)
    kt = kt.repeat_interleave(Hq // Hkv, dim=0)
    vt = vt.repeat_interleave(Hq // Hkv, dim=0)
    o = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None], scale=scale)
    return o[0, :, 0, :].numpy()


@pytest.mark.parametrize("Hq,Hkv,D,B", [(4, 4, 16, 4), (8, 2, 32, 16), (4, 1, 8, 32), (6, 3, 12, 16)])
def test_identity_table_equals_contiguous_sdpa(Hq, Hkv, D, B):
    """With blocks laid out in logical order, paged attention is plain attention."""
    rng = np.random.default_rng(Hq * 100 + D)
    S = 3
    lens = np.array([1, B * 2 + 3, B * 3], np.int32)
    MB = 3
    NB = S * MB
    tables = np.arange(S * MB, dtype=np.int32).reshape(S, MB)
    q = rng.standard_normal((S, Hq, D)).astype(np.float32)
    k = _pool(NB, Hkv, B, D, rng)
    v = _pool(NB, Hkv, B, D, rng)
    scale = 0.37
    out = oracle.decode(q, k, v, tables, lens, scale)
    for s in range(S):
        L = lens[s]
        # contiguous view: blocks s*MB .. s*MB+MB-1 concatenated in token order
        kseq = k[s * MB:(s + 1) * MB].transpose(0, 2, 1, 3).reshape(MB * B, Hkv, D)[:L]
        vseq = v[s * MB:(s + 1) * MB].transpose(0, 2, 1, 3).reshape(MB * B, Hkv, D)[:L]
        ref = _sdpa_reference(q[s], kseq, vseq, scale)
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12)


def test_permutation_of_physical_blocks_changes_nothing():
    rng = np.random.default_rng(11)
    q, k, v, tables, lens = _random_case(rng)
    out = oracle.decode(q, k, v, tables, lens, 0.25)
    NB = k.shape[0]
    perm = rng.permutation(NB)          # new position of old block b is perm[b]
    k2 = np.empty_like(k)
    v2 = np.empty_like(v)
    k2[perm] = k
    v2[perm] = v
    t2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1).astype(np.int32)
    out2 = oracle.decode(q, k2, v2, t2, lens, 0.25)
    assert np.array_equal(out, out2)


def test_single_token_returns_its_value_row():
    rng = np.random.default_rng(3)
    q, k, v, tables, lens = _random_case(rng, S=2, lens=[1, 1])
    out = oracle.decode(q, k, v, tables, lens, 0.5)
    for s in range(2):
        for h in range(q.shape[1]):
            kvh = h // (q.shape[1] // k.shape[1])
            assert np.array_equal(out[s, h], v[tables[s, 0], kvh, 0].astype(np.float64))


def test_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(4)
    q, k, v, tables, lens = _random_case(rng, S=2, lens=[17, 29])
    k[:] = k[0, 0, 0]                      # every key row identical
    out = oracle.decode(q, k, v, tables, lens, 0.9)
    B = k.shape[2]
    for s in range(2):
        for h in range(q.shape[1]):
            kvh = h // (q.shape[1] // k.shape[1])
            rows = [v[tables[s, i // B], kvh, i % B].astype(np.float64) for i in range(lens[s])]
            np.testing.assert_allclose(out[s, h], np.mean(rows, axis=0), rtol=0, atol=1e-14)


def test_dominant_logit_selects_its_value_row():
    rng = np.random.default_rng(6)
    q, k, v, tables, lens = _random_case(rng, S=1, Hq=2, Hkv=2, lens=[37])
    B = k.shape[2]
    j = 21
    kj = k[tables[0, j // B], :, j % B]        # [Hkv, D]
    q[0] = 60.0 * kj / np.linalg.norm(kj, axis=1, keepdims=True)
    out = oracle.decode(q, k, v, tables, lens, 1.0)
    for h in range(2):
        np.testing.assert_allclose(out[0, h], v[tables[0, j // B], h, j % B], rtol=0, atol=1e-6)


def test_weights_are_a_distribution():
    rng = np.random.default_rng(7)
    q, k, v, tables, lens = _random_case(rng, S=4, lens=[0, 50, 3, 17])
    out, w = oracle.decode(q, k, v, tables, lens, 0.3, return_weights=True)
    for s in range(4):
        for h in range(q.shape[1]):
            L = lens[s]
            if L == 0:
                assert np.all(out[s, h] == 0)
                continue
            assert np.all(w[s, h, :L] > 0)
            assert abs(w[s, h, :L].sum() - 1.0) < 1e-14
            assert np.all(w[s, h, L:] == 0)


def test_c_oracle_matches_pure_python_brute_force_on_tiny_workload():
    wl = W.make_workload(1, seed=0)
    q, keys, values, off = W.decode_values(wl, "cpu")
    tables = W.direct_block_tables(wl)
    B, Hkv, D = wl.block_size, wl.num_kv_heads, wl.head_dim
    k = np.full((wl.num_blocks, Hkv, B, D), np.nan, np.float32)
    v = np.full_like(k, np.nan)
    for s in range(wl.num_seqs):
        for i in range(int(wl.context_lens[s])):
            k[tables[s, i // B], :, i % B] = keys[off[s] + i].numpy()
            v[tables[s, i // B], :, i % B] = values[off[s] + i].numpy()
    out = oracle.decode(q.numpy(), k, v, tables, wl.context_lens, wl.scale)
    ref = oracle.decode_bruteforce(q.numpy(), k, v, tables, wl.context_lens, wl.scale)
    assert np.isfinite(out).all()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


def test_threads_do_not_change_results():
    rng = np.random.default_rng(8)
    q, k, v, tables, lens = _random_case(rng, S=5, maxL=60)
    a = oracle.decode(q, k, v, tables, lens, 0.2, nthreads=1)
    b = oracle.decode(q, k, v, tables, lens, 0.2, nthreads=3)
    assert np.array_equal(a, b)


def test_partition_merge_equals_one_pass():
    """Splitting the context into partitions and merging their (m, l, acc) states by
    log-sum-exp reaches the one-pass value (exact up to rounding)."""
    rng = np.random.default_rng(9)
    q, k, v, tables, lens = _random_case(rng, S=1, Hq=2, Hkv=1, lens=[77])
    out = oracle.decode(q, k, v, tables, lens, 0.4)
    for cuts in ([0, 77], [0, 32, 64, 77], [0, 4, 8, 77], [0, 0, 40, 40, 77, 77]):
        ms, ls, accs = [], [], []
        for a, b in zip(cuts[:-1], cuts[1:]):
            m, l, acc = oracle.partial(q[0, 1], k, v, tables[0], 2, 1, a, b, 0.4)
            ms.append(m)
            ls.append(l)
            accs.append(acc)
        merged = oracle.merge_partials(ms, ls, np.array(accs))
        np.testing.assert_allclose(merged, out[0, 1], rtol=0, atol=1e-13)


# ---------------------------------------------------------------- reshape / copy

def test_reshape_lands_tokens_at_the_printed_slots():
    """Writing tokens 0..31 through the fullstackaihub table puts token 17 in
    physical block 4 at offset 1 (slot 65) and token 0 in block 17 at offset 0."""
    hdr, rows = read_golden("translation_fullstackaihub.txt")
    B, table = hdr["block_size"], hdr["table"]
    rng = np.random.default_rng(1)
    Hkv, D = 2, 8
    key = rng.standard_normal((32, Hkv, D)).astype(np.float32)
    val = rng.standard_normal((32, Hkv, D)).astype(np.float32)
    kc = np.zeros((20, Hkv, B, D), np.float32)
    vc = np.zeros_like(kc)
    slots = np.array([oracle.physical_slot(table, B, i) for i in range(32)], np.int64)
    kc2, vc2 = oracle.reshape_and_cache(key, val, kc, vc, slots)
    for tok, blk, off, slot in rows:
        assert np.array_equal(kc2[blk, :, off], key[tok])
        assert np.array_equal(vc2[blk, :, off], val[tok])
    untouched = [b for b in range(20) if b not in table]
    assert np.all(kc2[untouched] == 0) and np.all(vc2[untouched] == 0)


def test_reshape_skips_negative_slots_and_is_bit_exact_on_bf16_bits():
    rng = np.random.default_rng(2)
    bits = rng.integers(0, 2 ** 16, size=(3, 1, 4), dtype=np.uint16)
    kc = np.zeros((2, 1, 4, 4), np.uint16)
    kc2, vc2 = oracle.reshape_and_cache(bits, bits, kc, kc, np.array([5, -1, 2]))
    assert np.array_equal(kc2[1, 0, 1], bits[0, 0]) and np.array_equal(kc2[0, 0, 2], bits[2, 0])
    assert np.count_nonzero(kc2) == np.count_nonzero(bits[0]) + np.count_nonzero(bits[2])
    with pytest.raises(ValueError):
        oracle.reshape_and_cache(bits, bits, kc, kc, np.array([8, 0, 0]))


def test_copy_blocks_copies_whole_blocks_in_pair_order():
    rng = np.random.default_rng(3)
    kc = rng.standard_normal((6, 2, 16, 4)).astype(np.float32)
    vc = rng.standard_normal((6, 2, 16, 4)).astype(np.float32)
    k2, v2 = oracle.copy_blocks(kc, vc, np.array([[0, 3], [3, 5]]))
    assert np.array_equal(k2[3], kc[0]) and np.array_equal(v2[3], vc[0])
    assert np.array_equal(k2[5], kc[0]) and np.array_equal(v2[5], vc[0])   # chained in order
    for b in (0, 1, 2, 4):
        assert np.array_equal(k2[b], kc[b]) and np.array_equal(v2[b], vc[b])
    hdr, _ = read_golden("cow_initnode.txt")
    assert kc.shape[2] == hdr["copied_slots"]            # all 16 slots of the block move
    with pytest.raises(ValueError):
        oracle.copy_blocks(kc, vc, np.array([[0, 6]]))
