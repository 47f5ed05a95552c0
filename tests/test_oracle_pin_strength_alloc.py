"""The prefix-cache, beam-search and swap pins are strong enough: plausible mistakes
planted in a subclass of the oracle allocator each fail at least one pin (CPU only).  The unmutated class
passes them all.  Nothing here changes the real oracle or touches the library."""
import pytest

import test_oracle_allocator as pins
from oracle.allocator import OracleAllocator

BEAM_PINS = [pins.test_beam_step_with_each_parent_once_copies_nothing,
             pins.test_beam_step_parent_twice_copies_once_and_frees_the_dropped_beam,
             pins.test_beam_steps_keep_every_beam_its_parent_plus_one_token,
             pins.test_beam_step_out_of_blocks_changes_nothing]

PREFIX_PINS = [pins.test_prefix_cache_shares_the_common_full_blocks,
               pins.test_prefix_match_follows_the_path_not_the_block_content,
               pins.test_cached_blocks_outlive_their_sequences_and_are_reused,
               pins.test_eviction_takes_the_oldest_unreferenced_leaf,
               pins.test_blocks_in_use_equal_distinct_prefixes_plus_partials,
               pins.test_cached_add_out_of_blocks_changes_nothing,
               pins.test_prefix_shared_tables_give_the_contiguous_attention]


class _EvictAnyOldest(OracleAllocator):
    """Evicts the earliest-released cached block even when it still has children."""
    def _take(self):
        if not self.free and self.unreferenced:
            blk = next(iter(self.unreferenced))
            self.nchildren[blk] = 0
        return super()._take()


class _ContentTree(dict):
    def get(self, key, default=None):
        for (_, toks), blk in self.items():
            if toks == key[1]:
                return blk
        return default


class _MatchContentOnly(OracleAllocator):
    """Looks blocks up by their token ids alone, ignoring the prefix before them."""
    def __init__(self, *args, **kw):
        super().__init__(*args, **kw)
        self.tree = _ContentTree()


class _ReleaseToFree(OracleAllocator):
    """Returns cached blocks to the free queue at count zero (and forgets them)."""
    def _release(self, blk):
        self.ref[blk] -= 1
        if self.ref[blk] == 0:
            if blk in self.key_of:
                key = self.key_of.pop(blk)
                del self.tree[key]
                del self.nchildren[blk]
                if key[0] >= 0 and key[0] in self.nchildren:
                    self.nchildren[key[0]] -= 1
            self.free.append(blk)


class _NoHoldOnHit(OracleAllocator):
    """Reuses cached blocks without counting the new reference."""
    def _hold(self, blk):
        if self.ref[blk] == 0:
            del self.unreferenced[blk]
            self.ref[blk] = 1


class _CachedCountsPartial(OracleAllocator):
    """Reports the partial last block as cached too."""
    def add_seq_cached(self, seq_id, token_ids):
        slots, c = super().add_seq_cached(seq_id, token_ids)
        n = len(token_ids)
        return slots, (n if c == n - n % self.B and c > 0 else c)


class _AppendBeforeFree(OracleAllocator):
    """Beam step that appends the new tokens while the old beams still hold their blocks."""
    def beam_step(self, beam_ids, parents, new_ids):
        trial = __import__("copy").deepcopy(self)
        temp = [("beam", j) for j in range(len(new_ids))]
        for j, p in enumerate(parents):
            trial.fork(beam_ids[p], temp[j])
        res = trial.append_slots(temp)
        for b in beam_ids:
            trial.free_seq(b)
        for j, b in enumerate(new_ids):
            trial.tables[b] = trial.tables.pop(temp[j])
            trial.ntokens[b] = trial.ntokens.pop(temp[j])
        self.__dict__.update(trial.__dict__)
        return res


class _ForkWithoutReference(OracleAllocator):
    """Fork that shares the parent's blocks without counting the child's reference."""
    def fork(self, parent, child):
        self.tables[child] = list(self.tables[parent])
        self.ntokens[child] = self.ntokens[parent]


class _SwapOutKeepsReference(OracleAllocator):
    """Swap-out that gives the sequence host blocks but keeps its device blocks referenced."""
    def swap_out(self, seq_id):
        table = list(self.tables[seq_id])
        self.ref_backup = {b: self.ref[b] for b in table}
        pairs = super().swap_out(seq_id)
        for b, r in self.ref_backup.items():
            if self.ref[b] < r:
                if b in self.free:
                    self.free.remove(b)
                self.ref[b] = r
        return pairs


class _SwapInReversed(OracleAllocator):
    """Swap-in that hands back the host blocks in reverse table order."""
    def swap_in(self, seq_id):
        if seq_id in self.on_host:
            self.tables[seq_id] = self.tables[seq_id][::-1]
        pairs = super().swap_in(seq_id)
        return pairs


class _PartialSwapOut(OracleAllocator):
    """Swap-out that moves what fits on the host instead of refusing when the host is short."""
    def swap_out(self, seq_id):
        if seq_id not in self.tables or seq_id in self.on_host:
            raise ValueError("unknown or swapped-out sequence")
        table = self.tables[seq_id]
        pairs = []
        for i, blk in enumerate(table):
            if not self.host_free:
                break
            h = self.host_free.popleft()
            pairs.append((blk, h))
            self._release(blk)
            table[i] = h
        self.on_host.add(seq_id)
        return pairs


BEAM_MUTANTS = {"none": OracleAllocator, "append_before_free": _AppendBeforeFree,
                "fork_without_reference": _ForkWithoutReference}

SWAP_PINS = [pins.test_swap_out_releases_device_blocks_and_swap_in_restores_the_sequence,
             pins.test_swapping_out_one_sharer_leaves_the_shared_blocks_to_the_other,
             pins.test_swap_round_trip_keeps_the_attention_output,
             pins.test_swap_out_of_blocks_changes_nothing]

SWAP_MUTANTS = {"none": OracleAllocator, "swap_out_keeps_reference": _SwapOutKeepsReference,
                "swap_in_reversed": _SwapInReversed, "partial_swap_out": _PartialSwapOut}

MUTANTS = {"none": OracleAllocator, "evict_any_oldest": _EvictAnyOldest, "match_content_only": _MatchContentOnly,
           "release_to_free": _ReleaseToFree, "no_hold_on_hit": _NoHoldOnHit,
           "cached_counts_partial": _CachedCountsPartial}


def _failures(cls, monkeypatch, which=None):
    monkeypatch.setattr(pins, "OracleAllocator", cls)
    failed = []
    for pin in (PREFIX_PINS if which is None else which):
        try:
            pin()
        except (Exception, pytest.fail.Exception):   # pytest.raises reports through a BaseException
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_allocator_mistakes_fail_a_pin(name, monkeypatch):
    failed = _failures(MUTANTS[name], monkeypatch)
    if name == "none":
        assert failed == []
    else:
        assert failed, "mutation %s passed every prefix-cache pin" % name


@pytest.mark.parametrize("name", sorted(BEAM_MUTANTS))
def test_planted_beam_mistakes_fail_a_pin(name, monkeypatch):
    failed = _failures(BEAM_MUTANTS[name], monkeypatch, BEAM_PINS)
    if name == "none":
        assert failed == []
    else:
        assert failed, "mutation %s passed every beam pin" % name


@pytest.mark.parametrize("name", sorted(SWAP_MUTANTS))
def test_planted_swap_mistakes_fail_a_pin(name, monkeypatch):
    failed = _failures(SWAP_MUTANTS[name], monkeypatch, SWAP_PINS)
    if name == "none":
        assert failed == []
    else:
        assert failed, "mutation %s passed every swap pin" % name
