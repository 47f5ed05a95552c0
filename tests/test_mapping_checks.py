"""Host-side checks of the copy pairs and append slots (pa_check_block_mapping,
pa_check_slot_mapping): what they refuse, what they let through, and that the
allocator's own copy-on-write pairs and append slots always pass (CPU only)."""
import numpy as np
import pytest

from paged_kv_cache_363_b200 import pa


def _refused(fn, *args):
    with pytest.raises(pa.PAError) as e:
        fn(*args)
    assert e.value.status == pa.PA_ERR_INVALID
    return str(e.value)


def test_block_mapping_accepts_disjoint_pairs():
    pa.pa_check_block_mapping(np.zeros((0, 2), np.int64), 8)
    pa.pa_check_block_mapping([[0, 1], [0, 2], [3, 4]], 8)   # one source read by two pairs is fine


def test_block_mapping_refuses_out_of_range_repeated_and_chained():
    assert "pair 1" in _refused(pa.pa_check_block_mapping, [[0, 1], [2, 8]], 8)
    assert "pair 0" in _refused(pa.pa_check_block_mapping, [[-1, 1]], 8)
    msg = _refused(pa.pa_check_block_mapping, [[0, 5], [1, 2], [3, 5]], 8)
    assert "same block 5" in msg and "0" in msg and "2" in msg
    # block 2 is written by pair 0 and read by pair 1: the copy order would decide the result
    assert "block 2" in _refused(pa.pa_check_block_mapping, [[1, 2], [2, 3]], 8)
    assert "block 4" in _refused(pa.pa_check_block_mapping, [[4, 4]], 8)


def test_slot_mapping_ignores_padding_and_refuses_repeats_and_overflow():
    pa.pa_check_slot_mapping(np.zeros(0, np.int64), 4, 16)
    pa.pa_check_slot_mapping([-1, 0, -1, 63, 17], 4, 16)
    msg = _refused(pa.pa_check_slot_mapping, [5, 9, 5], 4, 16)
    assert "tokens 0 and 2" in msg and "slot 5" in msg
    assert "token 1" in _refused(pa.pa_check_slot_mapping, [0, 64], 4, 16)


def test_bad_counts_are_refused():
    with pytest.raises(pa.PAError):
        pa.pa_check_block_mapping([[0, 1]], 0)
    with pytest.raises(pa.PAError):
        pa.pa_check_slot_mapping([0], 4, 0)
    assert pa.lib.pa_check_block_mapping(None, 1, 8) == pa.PA_ERR_INVALID
    assert pa.lib.pa_check_slot_mapping(None, 1, 8, 16) == pa.PA_ERR_INVALID
    assert pa.lib.pa_check_block_mapping(None, 0, 8) == pa.PA_OK


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_the_allocators_own_pairs_and_slots_always_pass(seed):
    """Parallel sampling as the pages describe it (prompts forked into streams that then
    append in batches): every batch's copy-on-write pairs and slots pass both checks."""
    rng = np.random.default_rng(seed)
    NB, B = 4096, 16
    alloc = pa.Allocator(NB, B, rng.permutation(NB))
    seqs = []
    for p in range(12):
        sid = 1000 * p
        alloc.add_seq(sid, int(rng.integers(1, 4 * B)))
        seqs.append(sid)
        for c in range(1, int(rng.integers(2, 5))):
            alloc.fork(sid, sid + c)
            seqs.append(sid + c)
    copies = 0
    for _ in range(3 * B):
        batch = [s for s in seqs if rng.random() < 0.8]
        slots, pairs = alloc.append_slots(batch)
        pa.pa_check_slot_mapping(slots, NB, B)
        pa.pa_check_block_mapping(np.asarray(pairs, np.int64).reshape(-1, 2), NB)
        copies += len(pairs)
    assert copies > 0
