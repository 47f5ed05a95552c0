"""The pins are strong enough: plausible mistakes planted in a CPU copy of the
decode definition each fail at least one pin (CPU only).

The copy below is a plain restatement of the oracle's definition with a switch
for one planted mistake.  The unmutated copy passes every pin; each mutated one
fails at least one.  Nothing here touches the real oracle or the library.
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden

MUTATIONS = ["none", "kv_head_modulo", "block_offset_swapped", "scale_dropped", "no_normalise",
             "value_from_key", "table_index_off_by_one", "last_token_dropped"]


def _decode(q, k, v, tables, lens, scale, mut):
    S, Hq, D = q.shape
    NB, Hkv, B, _ = k.shape
    g = Hq // Hkv
    out = np.zeros((S, Hq, D))
    for s in range(S):
        L = int(lens[s]) - (1 if mut == "last_token_dropped" and lens[s] > 1 else 0)
        for h in range(Hq):
            kvh = h % Hkv if mut == "kv_head_modulo" else h // g
            rows = []
            for i in range(L):
                b, o = (i % B, i // B) if mut == "block_offset_swapped" else (i // B, i % B)
                if mut == "table_index_off_by_one":
                    b = min(b + 1, tables.shape[1] - 1)
                if not 0 <= b < tables.shape[1]:
                    return None
                p = int(tables[s][b])
                if not (0 <= p < NB and 0 <= o < B):
                    return None
                rows.append((p, o))
            if not rows:
                continue
            sc = 1.0 if mut == "scale_dropped" else scale
            z = [sc * float(np.dot(q[s, h].astype(np.float64), k[p, kvh, o].astype(np.float64))) for p, o in rows]
            m = max(z)
            e = [math.exp(x - m) for x in z]
            den = 1.0 if mut == "no_normalise" else sum(e)
            src = k if mut == "value_from_key" else v
            for (p, o), w in zip(rows, e):
                out[s, h] += (w / den) * src[p, kvh, o].astype(np.float64)
    return out


def _pin_sdpa(fn):
    rng = np.random.default_rng(0)
    S, Hq, Hkv, D, B, MB = 2, 4, 2, 8, 4, 3
    lens = np.array([9, 12], np.int32)
    tables = np.arange(S * MB, dtype=np.int32).reshape(S, MB)
    q = rng.standard_normal((S, Hq, D)).astype(np.float32)
    k = rng.standard_normal((S * MB, Hkv, B, D)).astype(np.float32)
    v = rng.standard_normal((S * MB, Hkv, B, D)).astype(np.float32)
    out = fn(q, k, v, tables, lens, 0.6)
    if out is None:
        return False
    for s in range(S):
        L = lens[s]
        kk = torch.from_numpy(k[s * MB:(s + 1) * MB].transpose(1, 0, 2, 3).reshape(Hkv, MB * B, D)[:, :L]).double()
        vv = torch.from_numpy(v[s * MB:(s + 1) * MB].transpose(1, 0, 2, 3).reshape(Hkv, MB * B, D)[:, :L]).double()
        qq = torch.from_numpy(q[s]).double()[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(
            qq[None], kk.repeat_interleave(Hq // Hkv, 0)[None], vv.repeat_interleave(Hq // Hkv, 0)[None],
            scale=0.6)[0, :, 0].numpy()
        if not np.allclose(out[s], ref, rtol=0, atol=1e-10):
            return False
    return True


def _pin_golden_walk(fn):
    """Single-token one-hot values reveal which physical row each logical token reads:
    with one-hot values per slot, the output of an all-equal-keys query is the
    histogram of slots read; compare with the slots the pages print."""
    hdr, rows = read_golden("translation_fullstackaihub.txt")
    B, table = hdr["block_size"], hdr["table"]
    NB = max(table) + 1
    D = NB * B
    k = np.zeros((NB, 1, B, D), np.float32)
    v = np.zeros((NB, 1, B, D), np.float32)
    for p in range(NB):
        for o in range(B):
            v[p, 0, o, p * B + o] = 1.0
    q = np.zeros((1, 1, D), np.float32)
    lens = np.array([32], np.int32)
    out = fn(q, k, v, np.array([table], np.int32), lens, 1.0)
    if out is None:
        return False
    read = set(np.nonzero(out[0, 0] > 0)[0].tolist())
    printed = {r[3] for r in rows}                  # slots the golden file lists
    # the diagram: physical block 17 holds tokens 0..15, physical block 4 tokens 16..31
    whole_blocks = {table[0] * B + o for o in range(B)} | {table[1] * B + o for o in range(B)}
    return printed <= read and read == whole_blocks


@pytest.mark.parametrize("mut", MUTATIONS)
def test_planted_mistakes_fail_a_pin(mut):
    f = lambda *a: _decode(*a, mut)
    passed = _pin_sdpa(f) and _pin_golden_walk(f)
    if mut == "none":
        assert passed
    else:
        assert not passed


# ---------------------------------------------------------------- split-K merge

MERGE_MUTATIONS = ["none", "den_without_l", "num_unweighted", "last_partition_dropped",
                   "partition_end_off_by_one"]


def _split_merge(q_row, k, v, table, kvh, cuts, scale, mut):
    """Partition states (m, l, acc) over [t0, t1) and their log-sum-exp merge, restated
    with a switch for one planted mistake."""
    B = k.shape[2]
    states = []
    for t0, t1 in zip(cuts[:-1], cuts[1:]):
        t1 = max(t0, t1 - 1) if mut == "partition_end_off_by_one" else t1
        z = [scale * float(np.dot(q_row.astype(np.float64), k[table[i // B], kvh, i % B].astype(np.float64)))
             for i in range(t0, t1)]
        if not z:
            states.append((-math.inf, 0.0, np.zeros(k.shape[3])))
            continue
        m = max(z)
        e = [math.exp(x - m) for x in z]
        acc = sum(w * v[table[i // B], kvh, i % B].astype(np.float64) for w, i in zip(e, range(t0, t1)))
        states.append((m, sum(e), acc))
    if mut == "last_partition_dropped":
        states = states[:-1]
    M = max(m for m, _, _ in states)
    num, den = 0.0, 0.0
    for m, l, acc in states:
        w = 0.0 if m == -math.inf else math.exp(m - M)
        num = num + (acc if mut == "num_unweighted" else w * acc)
        den += w if mut == "den_without_l" else w * l
    return num / den


def _merge_passes_pin(mut):
    """The split-K pin: for several partitionings (empty ranges included) the merge of the
    partition states equals the one-pass oracle row."""
    from oracle import oracle
    rng = np.random.default_rng(11)
    B, D, L = 4, 8, 23
    tables = np.array([[2, 0, 5, 1, 3, 4]], np.int32)
    q = rng.standard_normal((1, 2, D)).astype(np.float32)
    k = rng.standard_normal((6, 1, B, D)).astype(np.float32)
    v = rng.standard_normal((6, 1, B, D)).astype(np.float32)
    ref = oracle.decode(q, k, v, tables, np.array([L], np.int32), 0.7)[0, 1]
    for cuts in ([0, L], [0, 8, 16, L], [0, 4, 4, 12, L], [0, 1, L, L]):
        try:
            got = _split_merge(q[0, 1], k, v, tables[0], 0, cuts, 0.7, mut)
        except (ValueError, ZeroDivisionError):
            return False          # a mistake that cannot even produce a row fails too
        if not np.allclose(got, ref, rtol=0, atol=1e-12):
            return False
    return True


@pytest.mark.parametrize("mut", MERGE_MUTATIONS)
def test_planted_merge_mistakes_fail_the_split_pin(mut):
    assert _merge_passes_pin(mut) == (mut == "none")


# ---------------------------------------------------------------- append and copy-on-write copy

RESHAPE_MUTATIONS = ["none", "block_offset_swapped", "value_not_written", "negative_slot_written"]
COPY_MUTATIONS = ["none", "key_pool_only", "first_slot_only", "first_head_only", "pair_reversed"]


def _reshape(key, value, kc, vc, slots, mut):
    kc, vc = kc.copy(), vc.copy()
    B = kc.shape[2]
    for t, s in enumerate(slots):
        if s < 0 and mut != "negative_slot_written":
            continue
        s = int(s) % (kc.shape[0] * B)
        b, o = (s % B, s // B) if mut == "block_offset_swapped" else (s // B, s % B)
        kc[b, :, o] = key[t]
        if mut != "value_not_written":
            vc[b, :, o] = value[t]
    return kc, vc


def _copy(kc, vc, pairs, mut):
    kc, vc = kc.copy(), vc.copy()
    for src, dst in pairs:
        if mut == "pair_reversed":
            src, dst = dst, src
        sl = (slice(None), slice(0, 1)) if mut == "first_slot_only" else (slice(0, 1),) if mut == "first_head_only" \
            else (slice(None),)
        kc[(dst,) + sl] = kc[(src,) + sl]
        if mut != "key_pool_only":
            vc[(dst,) + sl] = vc[(src,) + sl]
    return kc, vc


def _reshape_passes_pins(mut):
    from conftest import read_golden
    from oracle import oracle
    hdr, rows = read_golden("translation_fullstackaihub.txt")
    B, table = hdr["block_size"], hdr["table"]
    rng = np.random.default_rng(1)
    key = rng.standard_normal((32, 2, 8)).astype(np.float32)
    val = rng.standard_normal((32, 2, 8)).astype(np.float32)
    kc = np.zeros((20, 2, B, 8), np.float32)
    slots = np.array([oracle.physical_slot(table, B, i) for i in range(32)], np.int64)
    slots[5] = -1                                     # a padding token
    try:
        k2, v2 = _reshape(key, val, kc, kc, slots, mut)
    except IndexError:
        return False                                  # a mistake that writes outside the pool fails too
    for tok, blk, off, _ in rows:
        if tok != 5 and not (np.array_equal(k2[blk, :, off], key[tok]) and np.array_equal(v2[blk, :, off], val[tok])):
            return False
    untouched = [b for b in range(20) if b not in table]
    written = {(table[i // B], i % B) for i in range(32) if i != 5}
    stray = [(b, o) for b in table for o in range(B) if (b, o) not in written and np.any(k2[b, :, o] != 0)]
    return bool(np.all(k2[untouched] == 0) and np.all(v2[untouched] == 0)) and not stray


def _copy_passes_pins(mut):
    rng = np.random.default_rng(3)
    kc = rng.standard_normal((6, 2, 16, 4)).astype(np.float32)
    vc = rng.standard_normal((6, 2, 16, 4)).astype(np.float32)
    k2, v2 = _copy(kc, vc, [(0, 3), (1, 5)], mut)
    if not all(np.array_equal(k2[d], kc[s]) and np.array_equal(v2[d], vc[s]) for s, d in ((0, 3), (1, 5))):
        return False
    return all(np.array_equal(k2[b], kc[b]) and np.array_equal(v2[b], vc[b]) for b in (0, 1, 2, 4))


@pytest.mark.parametrize("mut", RESHAPE_MUTATIONS)
def test_planted_append_mistakes_fail_a_pin(mut):
    assert _reshape_passes_pins(mut) == (mut == "none")


@pytest.mark.parametrize("mut", COPY_MUTATIONS)
def test_planted_copy_mistakes_fail_a_pin(mut):
    assert _copy_passes_pins(mut) == (mut == "none")
