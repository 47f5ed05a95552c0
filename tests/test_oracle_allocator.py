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
