"""Pins of the oracle block allocator to the pages' copy-on-write and waste facts (CPU only)."""
import numpy as np
import pytest

from conftest import read_golden
from oracle import oracle
from oracle.allocator import OracleAllocator, OutOfBlocks


def test_cow_worked_example_initnode():
    hdr, _ = read_golden("cow_initnode.txt")
    B, n, L = hdr["block_size"], hdr["streams"], hdr["prompt_tokens"]
    a = OracleAllocator(64, B, free_order=np.random.default_rng(0).permutation(64))
    a.add_seq(0, L)
    for j in range(1, n):
        a.fork(0, j)
    prompt = a.block_table(0)
    assert [a.ref[b] for b in prompt] == [hdr["ref_before"]] * len(prompt)
    before = {j: a.block_table(j) for j in range(n)}
    # stream 1 of the page writes first
    slot, cow = a.append_slot(1)
    assert cow is not None and cow[0] == prompt[-1]
    assert a.ref[prompt[-1]] == hdr["ref_after_first_write"]
    assert a.ref[cow[1]] == 1
    assert a.block_table(1) == prompt[:-1] + [cow[1]]
    for j in (0, 2, 3):
        assert a.block_table(j) == before[j]                       # others untouched
    assert slot == cow[1] * B + L % B
    # subsequent writes of stream 1 are private: no new copy, same block
    slot2, cow2 = a.append_slot(1)
    assert cow2 is None and slot2 == slot + 1
    # full shared blocks are never copied
    assert a.ref[prompt[0]] == n


def test_cow_order_three_copies_then_in_place():
    a = OracleAllocator(32, 16)
    a.add_seq(0, 20)
    for j in (1, 2, 3):
        a.fork(0, j)
    last = a.block_table(0)[-1]
    cows = [a.append_slot(j)[1] for j in range(4)]
    assert [c is not None for c in cows] == [True, True, True, False]
    assert a.ref[last] == 1 and a.block_table(3)[-1] == last
    # a prompt ending on a block boundary needs no copy at all
    b = OracleAllocator(32, 16)
    b.add_seq(0, 32)
    b.fork(0, 1)
    assert b.append_slot(0)[1] is None and b.append_slot(1)[1] is None


def test_copy_moves_all_slots_of_the_block():
    """The copy-on-write copy duplicates the block's 16 slots, for K and for V."""
    hdr, _ = read_golden("cow_initnode.txt")
    B = hdr["block_size"]
    rng = np.random.default_rng(1)
    kc = rng.standard_normal((8, 2, B, 4)).astype(np.float32)
    vc = rng.standard_normal((8, 2, B, 4)).astype(np.float32)
    a = OracleAllocator(8, B)
    a.add_seq(0, 20)
    a.fork(0, 1)
    _, (src, dst) = a.append_slot(1)
    k2, v2 = oracle.copy_blocks(kc, vc, np.array([[src, dst]]))
    assert np.array_equal(k2[dst], kc[src]) and np.array_equal(v2[dst], vc[src])
    assert k2[dst].shape[1] == hdr["copied_slots"]


def test_waste_bound_initnode():
    hdr, _ = read_golden("waste_initnode.txt")
    B = hdr["block_size"]
    a = OracleAllocator(4096, B)
    worst = 0
    for L in range(0, 700):
        a.add_seq(L, L)
        w = a.waste_tokens(L)
        assert 0 <= w <= B - 1
        worst = max(worst, w)
        a.free_seq(L)
    assert worst == hdr["max_waste_tokens"]
    assert abs(hdr["max_waste_tokens"] / hdr["average_context"] - hdr["waste_fraction"]) < 1e-12


def test_incremental_allocation_takes_a_block_only_on_overflow():
    a = OracleAllocator(16, 4, free_order=list(range(15, -1, -1)))
    a.add_seq(7, 0)
    for i in range(13):
        before = a.num_free()
        slot, cow = a.append_slot(7)
        assert cow is None
        assert a.num_free() == before - (1 if i % 4 == 0 else 0)
        assert slot == a.block_table(7)[i // 4] * 4 + i % 4
    assert a.block_table(7) == [15, 14, 13, 12]


def test_accounting_and_release():
    rng = np.random.default_rng(2)
    NB, B = 300, 16
    a = OracleAllocator(NB, B, free_order=rng.permutation(NB))
    lens = rng.integers(0, 400, size=9)
    for s, L in enumerate(lens):
        slots = a.add_seq(s, int(L))
        assert len(set(slots)) == L
    assert a.num_free() == NB - sum(-(-int(L) // B) for L in lens)
    a.fork(0, 100)
    a.fork(0, 101)
    used = {b for t in a.tables.values() for b in t}
    assert len(used) + a.num_free() == NB
    for s in list(a.tables):
        a.free_seq(s)
    assert a.num_free() == NB and all(r == 0 for r in a.ref)


def test_out_of_blocks_changes_nothing():
    a = OracleAllocator(4, 16)
    a.add_seq(0, 40)
    a.fork(0, 1)
    snap = (list(a.free), list(a.ref), {k: list(v) for k, v in a.tables.items()}, dict(a.ntokens))
    with pytest.raises(OutOfBlocks):
        a.add_seq(2, 33)
    assert snap == (list(a.free), list(a.ref), {k: list(v) for k, v in a.tables.items()}, dict(a.ntokens))
    a.append_slot(0)          # copy-on-write takes the last free block
    assert a.num_free() == 0
    for _ in range(8):        # seq 1 now owns its last block: tokens 40..47 go in place
        assert a.append_slot(1)[1] is None
    snap = (list(a.free), list(a.ref), {k: list(v) for k, v in a.tables.items()}, dict(a.ntokens))
    with pytest.raises(OutOfBlocks):
        a.append_slot(1)      # token 48 needs a fresh block
    assert snap == (list(a.free), list(a.ref), {k: list(v) for k, v in a.tables.items()}, dict(a.ntokens))


# ---------------------------------------------------------------- prefix cache
# "PagedAttention Paper Breakdown" (fullstackaihub.com), "Paper Methods": shared prefix
# caching in a radix tree.  Read at block granularity: a node is one full block, its
# label the block's token ids, its parent the block before it.

def _state(a):
    return (list(a.free), list(a.ref), {k: list(v) for k, v in a.tables.items()}, dict(a.ntokens),
            dict(a.tree), list(a.unreferenced))


def test_prefix_cache_shares_the_common_full_blocks():
    a = OracleAllocator(32, 4)
    s0, c0 = a.add_seq_cached(0, list(range(10)))                        # 2 full blocks + 2 tokens
    assert c0 == 0 and len(a.tree) == 2
    s1, c1 = a.add_seq_cached(1, list(range(8)) + [50, 51, 52, 53, 54])  # same 2 blocks, 1 new full, 1 partial
    t0, t1 = a.block_table(0), a.block_table(1)
    assert c1 == 8 and t1[:2] == t0[:2] and t1[2] not in t0 and t1[3] not in t0
    assert [a.ref[b] for b in t0] == [2, 2, 1] and a.ref[t1[2]] == 1 and a.ref[t1[3]] == 1
    assert len(a.tree) == 3                        # the partial blocks are private, never cached
    assert s1[:8] == s0[:8]                        # shared tokens sit at the same slots


def test_prefix_match_follows_the_path_not_the_block_content():
    """A block is reused only under the same prefix: equal content after a divergence is not shared."""
    a = OracleAllocator(32, 4)
    X, Y, W, Z = [1, 1, 1, 1], [2, 2, 2, 2], [3, 3, 3, 3], [4, 4, 4, 4]
    a.add_seq_cached(0, X + Y + Z)
    _, c = a.add_seq_cached(1, X + W + Z)
    t0, t1 = a.block_table(0), a.block_table(1)
    assert c == 4 and t1[0] == t0[0] and t1[2] != t0[2]
    _, c = a.add_seq_cached(2, Y + Z)              # Y at the root is a different node from Y under X
    assert c == 0


def test_cached_blocks_outlive_their_sequences_and_are_reused():
    a = OracleAllocator(16, 4)
    a.add_seq_cached(0, list(range(9)))            # 2 cached full blocks + 1 private partial
    full = a.block_table(0)[:2]
    partial = a.block_table(0)[2]
    free_before = a.num_free()
    a.free_seq(0)
    assert a.num_free() == free_before + 1 and a.free[-1] == partial      # only the private block returns
    assert a.num_cached_free() == 2 and all(a.ref[b] == 0 for b in full)
    _, c = a.add_seq_cached(1, list(range(8)) + [99])
    assert c == 8 and a.block_table(1)[:2] == full and a.num_cached_free() == 0
    assert all(a.ref[b] == 1 for b in full)


def test_eviction_takes_the_oldest_unreferenced_leaf():
    a = OracleAllocator(5, 2)
    a.add_seq_cached(0, [1, 1, 2, 2])              # chain p1 -> p2
    p1, p2 = a.block_table(0)
    a.add_seq_cached(1, [7, 7])                    # single node c1
    (c1,) = a.block_table(1)
    a.free_seq(0)                                  # released first: p1, then p2
    a.free_seq(1)                                  # released later: c1
    a.add_seq(2, 4)                                # the two free blocks
    assert a.num_free() == 0 and a.num_cached_free() == 3
    a.add_seq(3, 2)                                # p1 is older but has a child: the leaf p2 goes
    assert a.block_table(3) == [p2] and p2 not in a.key_of and a.nchildren[p1] == 0
    a.add_seq(4, 2)                                # now p1 is a leaf, and older than c1
    assert a.block_table(4) == [p1]
    _, c = a.add_seq_cached(5, [7, 7])             # c1 is still cached
    assert c == 2 and a.block_table(5) == [c1]
    with pytest.raises(OutOfBlocks):
        a.add_seq(6, 1)


def test_blocks_in_use_equal_distinct_prefixes_plus_partials():
    rng = np.random.default_rng(5)
    B = 4
    stems = [rng.integers(0, 2, size=int(rng.integers(4, 30))).tolist() for _ in range(4)]
    a = OracleAllocator(400, B, free_order=rng.permutation(400))
    prompts = []
    for sid in range(40):
        stem = stems[sid % 4]
        p = stem[:int(rng.integers(0, len(stem) + 1))] + rng.integers(0, 2, size=int(rng.integers(0, 9))).tolist()
        slots, cached = a.add_seq_cached(sid, p)
        assert cached % B == 0 and cached <= len(p) - len(p) % B
        prompts.append(p)
    prefixes = {tuple(p[:(j + 1) * B]) for p in prompts for j in range(len(p) // B)}
    partials = sum(1 for p in prompts if len(p) % B)
    assert sum(1 for r in a.ref if r > 0) == len(prefixes) + partials
    assert len(a.tree) == len(prefixes)
    for sid in range(40):
        a.free_seq(sid)
    assert a.num_free() + a.num_cached_free() == 400 and not any(a.ref)


def test_cached_add_out_of_blocks_changes_nothing():
    a = OracleAllocator(6, 4)
    a.add_seq_cached(0, list(range(12)))
    a.free_seq(0)
    a.add_seq(1, 12)                               # 3 free blocks taken, 3 cached unreferenced remain
    before = _state(a)
    with pytest.raises(OutOfBlocks):
        a.add_seq_cached(2, list(range(8)) + [9, 9, 9, 9, 9, 9, 9, 9, 9])  # 2 hits, needs 3 more, 1 evictable
    assert _state(a) == before


def test_prefix_shared_tables_give_the_contiguous_attention():
    """Only the uncached tokens of each prompt are written; decode through the shared
    tables must equal plain softmax attention over each prompt's own tokens."""
    rng = np.random.default_rng(11)
    B, Hkv, G, D = 4, 2, 2, 8
    stem = rng.integers(0, 3, size=13).tolist()
    prompts = [stem[:c] + rng.integers(0, 3, size=n).tolist() for c, n in ((13, 3), (9, 6), (13, 0), (4, 7))]

    def kv_of(prefix):                              # a token's K/V depend on the whole prefix up to it
        g = np.random.default_rng(abs(hash(tuple(prefix))) % (2 ** 32))
        return g.standard_normal((2, Hkv, D)).astype(np.float32)

    NB = 64
    a = OracleAllocator(NB, B, free_order=rng.permutation(NB))
    kc = np.full((NB, Hkv, B, D), np.nan, np.float32)
    vc = np.full((NB, Hkv, B, D), np.nan, np.float32)
    written = 0
    for sid, p in enumerate(prompts):
        slots, cached = a.add_seq_cached(sid, p)
        rows = np.stack([kv_of(p[:i + 1]) for i in range(cached, len(p))]) if len(p) > cached else None
        if rows is not None:
            kc, vc = oracle.reshape_and_cache(rows[:, 0], rows[:, 1], kc, vc, np.asarray(slots[cached:]))
            written += len(p) - cached
    assert written < sum(len(p) for p in prompts)   # some K/V really are shared
    S = len(prompts)
    q = rng.standard_normal((S, Hkv * G, D)).astype(np.float32)
    mb = max(len(a.block_table(s)) for s in range(S))
    tables = np.array([a.block_table(s) + [-1] * (mb - len(a.block_table(s))) for s in range(S)], np.int32)
    lens = np.array([len(p) for p in prompts], np.int32)
    scale = D ** -0.5
    out = oracle.decode(q, kc, vc, tables, lens, scale)
    for s, p in enumerate(prompts):
        kv = np.stack([kv_of(p[:i + 1]) for i in range(len(p))]).astype(np.float64)   # [L, 2, Hkv, D]
        for h in range(Hkv * G):
            z = scale * kv[:, 0, h // G] @ q[s, h].astype(np.float64)
            w = np.exp(z - z.max())
            w /= w.sum()
            assert np.allclose(out[s, h], w @ kv[:, 1, h // G], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- beam search
# [fullstackaihub] section 3 and "Summary & Key Takeaways" 3; [initnode] section 3:
# beams share blocks by copy-on-write until one of them writes.

def _beams(a, B, prompt, width):
    a.add_seq(0, prompt)
    for j in range(1, width):
        a.fork(0, j)
    return list(range(width))


def test_beam_step_with_each_parent_once_copies_nothing():
    a = OracleAllocator(64, 4)
    beams = _beams(a, 4, 10, 3)                    # 3 beams sharing 3 blocks (last one partial)
    for j in beams:                                # diverge: first appends copy the shared partial block
        a.append_slot(j)
    before = {j: a.block_table(j) for j in beams}
    res = a.beam_step(beams, [2, 0, 1], [10, 11, 12])   # a permutation: every parent once
    assert all(c is None for _, c in res)          # fork-then-free leaves every last block private
    assert [a.block_table(n) for n in (10, 11, 12)] == [before[2], before[0], before[1]]
    assert all(a.ntokens[n] == 12 for n in (10, 11, 12))
    assert all(b not in a.tables for b in beams)


def test_beam_step_parent_twice_copies_once_and_frees_the_dropped_beam():
    a = OracleAllocator(64, 4)
    beams = _beams(a, 4, 9, 2)
    a.append_slot(0)                               # beam 0 copies the shared partial block
    a.append_slot(1)                               # beam 1 now writes in place
    t0, t1 = a.block_table(0), a.block_table(1)
    private1 = [b for b in t1 if b not in t0]
    free_before = a.num_free()
    res = a.beam_step([0, 1], [0, 0], [0, 1])      # both new beams continue beam 0; beam 1 dropped
    copies = [c for _, c in res if c is not None]
    assert len(copies) == 1 and copies[0][0] == t0[-1]        # k children of one parent: k-1 copies
    # the first child to write copies; the last one writes in place in the parent's block
    assert a.block_table(0)[:-1] == t0[:-1] and a.block_table(0)[-1] == copies[0][1] and a.block_table(1) == t0
    assert all(a.ref[b] == 0 for b in private1) and a.num_free() == free_before + len(private1) - 1
    assert all(a.ref[b] == 2 for b in t0[:-1])                # full shared blocks are never copied


def test_beam_steps_keep_every_beam_its_parent_plus_one_token():
    """After random beam steps, decode through each beam's table equals plain attention
    over the tokens that beam accumulated (its ancestors' tokens, then its own)."""
    rng = np.random.default_rng(3)
    B, Hkv, G, D, W, prompt = 4, 1, 2, 8, 4, 7
    NB = 128
    a = OracleAllocator(NB, B, free_order=rng.permutation(NB))
    kc = np.full((NB, Hkv, B, D), np.nan, np.float32)
    vc = np.full((NB, Hkv, B, D), np.nan, np.float32)
    rows = [rng.standard_normal((2, Hkv, D)).astype(np.float32) for _ in range(prompt)]
    slots = a.add_seq(0, prompt)
    kc, vc = oracle.reshape_and_cache(np.stack([r[0] for r in rows]), np.stack([r[1] for r in rows]), kc, vc,
                                      np.array(slots))
    hist = {0: list(range(prompt))}                # beam -> indices into `rows`
    beams = [0]
    for step in range(9):
        parents = rng.integers(0, len(beams), size=W).tolist()
        new_ids = [100 * (step + 1) + j for j in range(W)]
        res = a.beam_step(beams, parents, new_ids)
        pairs = [c for _, c in res if c is not None]
        if pairs:
            kc, vc = oracle.copy_blocks(kc, vc, np.array(pairs))
        new_rows = []
        for j, (slot, _) in enumerate(res):
            rows.append(rng.standard_normal((2, Hkv, D)).astype(np.float32))
            new_rows.append(len(rows) - 1)
        kc, vc = oracle.reshape_and_cache(np.stack([rows[i][0] for i in new_rows]),
                                          np.stack([rows[i][1] for i in new_rows]), kc, vc,
                                          np.array([s for s, _ in res]))
        hist = {new_ids[j]: hist[beams[p]] + [new_rows[j]] for j, p in enumerate(parents)}
        beams = new_ids
    assert sum(1 for r in a.ref if r > 0) == len({b for n in beams for b in a.block_table(n)})
    q = rng.standard_normal((W, Hkv * G, D)).astype(np.float32)
    mb = max(len(a.block_table(n)) for n in beams)
    tables = np.array([a.block_table(n) + [-1] * (mb - len(a.block_table(n))) for n in beams], np.int32)
    lens = np.array([a.ntokens[n] for n in beams], np.int32)
    scale = D ** -0.5
    out = oracle.decode(q, kc, vc, tables, lens, scale)
    for s, n in enumerate(beams):
        kv = np.stack([rows[i] for i in hist[n]]).astype(np.float64)
        assert len(hist[n]) == lens[s]
        for h in range(Hkv * G):
            z = scale * kv[:, 0, h // G] @ q[s, h].astype(np.float64)
            w = np.exp(z - z.max())
            w /= w.sum()
            assert np.allclose(out[s, h], w @ kv[:, 1, h // G], rtol=0, atol=1e-12)


def test_beam_step_out_of_blocks_changes_nothing():
    a = OracleAllocator(5, 4)
    beams = _beams(a, 4, 6, 2)                     # 2 blocks shared by 2 beams
    a.add_seq(9, 12)                               # the other 3 blocks
    before = _state(a)
    with pytest.raises(OutOfBlocks):
        a.beam_step(beams, [0, 0, 1], [5, 6, 7])   # 3 beams on one shared partial block: 2 copies, 0 free
    assert _state(a) == before
    with pytest.raises(ValueError):
        a.beam_step(beams, [0, 2], [5, 6])
    with pytest.raises(ValueError):
        a.beam_step(beams, [0, 1], [9, 6])         # 9 is held by a sequence outside the beams


# ---------------------------------------------------------------- swapping
# [fullstackaihub] "Engineering Limitations": CPU-GPU block swapping under memory pressure.

def test_swap_out_releases_device_blocks_and_swap_in_restores_the_sequence():
    a = OracleAllocator(16, 4)
    a.add_host_pool(8)
    a.add_seq(0, 10)                               # 3 blocks
    t = a.block_table(0)
    free0 = a.num_free()
    pairs = a.swap_out(0)
    assert [d for d, _ in pairs] == t and [h for _, h in pairs] == [0, 1, 2]     # host FIFO, table order
    assert a.num_free() == free0 + 3 and all(a.ref[b] == 0 for b in t)
    assert a.block_table(0) == [0, 1, 2] and 0 in a.on_host and len(a.host_free) == 5
    with pytest.raises(ValueError):
        a.append_slot(0)
    with pytest.raises(ValueError):
        a.fork(0, 1)
    back = a.swap_in(0)
    assert [h for h, _ in back] == [0, 1, 2] and len(a.host_free) == 8
    assert a.block_table(0) == [d for _, d in back] and all(a.ref[b] == 1 for b in a.block_table(0))
    assert a.ntokens[0] == 10 and a.append_slot(0)[1] is None


def test_swapping_out_one_sharer_leaves_the_shared_blocks_to_the_other():
    a = OracleAllocator(16, 4)
    a.add_host_pool(8)
    a.add_seq(0, 6)
    a.fork(0, 1)
    shared = a.block_table(0)
    a.swap_out(1)
    assert a.block_table(0) == shared and all(a.ref[b] == 1 for b in shared)
    assert a.append_slot(0)[1] is None             # the remaining stream owns the block now: no copy


def test_swap_round_trip_keeps_the_attention_output():
    """Swap half the sequences out, let other sequences reuse the freed device blocks,
    swap back in: decode over the returned tables equals decode before the swap."""
    rng = np.random.default_rng(8)
    B, Hkv, D, NB, NH = 4, 2, 8, 40, 32
    a = OracleAllocator(NB, B, free_order=rng.permutation(NB))
    a.add_host_pool(NH)
    kc = rng.standard_normal((NB, Hkv, B, D)).astype(np.float32)
    vc = rng.standard_normal((NB, Hkv, B, D)).astype(np.float32)
    kh = np.zeros((NH, Hkv, B, D), np.float32)
    vh = np.zeros((NH, Hkv, B, D), np.float32)
    lens = [9, 14, 3, 11]
    for s, L in enumerate(lens):
        a.add_seq(s, L)
    q = rng.standard_normal((4, Hkv, D)).astype(np.float32)

    def run():
        mb = max(len(a.block_table(s)) for s in range(4))
        tab = np.array([a.block_table(s) + [-1] * (mb - len(a.block_table(s))) for s in range(4)], np.int32)
        return oracle.decode(q, kc, vc, tab, np.array(lens, np.int32), 0.3)

    before = run()
    for s in (1, 3):
        for d, h in a.swap_out(s):
            kh[h], vh[h] = kc[d], vc[d]
    a.add_seq(9, 4 * (a.num_free() - 3))           # another sequence takes (and overwrites) freed blocks
    for b in a.block_table(9):
        kc[b] = 7.0
        vc[b] = -7.0
    a.free_seq(9)
    for s in (3, 1):
        for h, d in a.swap_in(s):
            kc[d], vc[d] = kh[h], vh[h]
    assert np.array_equal(run(), before)


def test_swap_out_of_blocks_changes_nothing():
    a = OracleAllocator(8, 4)
    a.add_host_pool(2)
    a.add_seq(0, 12)                               # 3 blocks, host has 2
    before = (_state(a), list(a.host_free), set(a.on_host))
    with pytest.raises(OutOfBlocks):
        a.swap_out(0)
    assert (_state(a), list(a.host_free), set(a.on_host)) == before
    b = OracleAllocator(4, 4)
    b.add_host_pool(4)
    b.add_seq(0, 12)
    b.swap_out(0)
    b.add_seq(1, 13)                               # all 4 device blocks
    before = (_state(b), list(b.host_free), set(b.on_host))
    with pytest.raises(OutOfBlocks):
        b.swap_in(0)
    assert (_state(b), list(b.host_free), set(b.on_host)) == before
