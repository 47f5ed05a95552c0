"""The parallel-sampling workload's paging, simulated on the host (CPU only).

"PagedAttention Paper Breakdown" (fullstackaihub.com) calls the block manager a
deterministic simulation of multi-tenant paging.  Here the full-size workload (32 prompts
of U[256, 1024] tokens, each forked into 4 streams that append U[1, 40] private tokens
in batches) runs through the library's allocator twice and through the oracle
allocator: tables, slots and copy-on-write pairs agree bit for bit, and the pages'
accounting holds ("PagedAttention and vLLM Architecture", section 3 and "Why Internal
Fragmentation is Bounded")."""
import numpy as np
import pytest

from oracle.allocator import OracleAllocator
from paged_kv_cache_363_b200 import pa
from paged_kv_cache_363_b200 import workloads as W


def _simulate(wl, make):
    P, n, B = wl.num_prompts, wl.streams_per_prompt, wl.block_size
    a = make(wl.num_blocks, B, wl.free_order)
    log = []
    for p in range(P):
        log.append(("prompt", list(a.add_seq(p * n, int(wl.prompt_lens[p])))))
    for p in range(P):
        for j in range(1, n):
            a.fork(p * n, p * n + j)
    priv = np.asarray(wl.private_tokens)
    for t in range(int(priv.max())):
        active = [int(s) for s in np.nonzero(priv > t)[0]]
        res = a.append_slots(active)
        if isinstance(res, tuple):                     # the library: (slots, pairs)
            slots, pairs = list(res[0]), [tuple(p) for p in res[1].tolist()]
        else:                                          # the oracle: [(slot, pair or None)]
            slots, pairs = [r[0] for r in res], [r[1] for r in res if r[1] is not None]
        log.append(("step", slots, pairs))
    tables = [list(a.block_table(s)) for s in range(P * n)]
    return log, tables, a


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_parallel_sampling_paging_is_replayable_and_matches_the_oracle(seed):
    wl = W.make_workload(W.NAME_TO_ID["cow-sampling-bf16"], seed=seed)
    log1, tables1, lib_a = _simulate(wl, pa.Allocator)
    log2, tables2, _ = _simulate(wl, pa.Allocator)
    assert (log1, tables1) == (log2, tables2)                  # deterministic
    log_o, tables_o, ora = _simulate(wl, lambda nb, b, order: OracleAllocator(nb, b, [int(x) for x in order]))
    assert [(e[0], [int(x) for x in e[1]]) + tuple(e[2:]) for e in log1] == \
        [(e[0], [int(x) for x in e[1]]) + tuple(e[2:]) for e in log_o]
    assert tables1 == tables_o

    P, n, B = wl.num_prompts, wl.streams_per_prompt, wl.block_size
    copies = sum(len(e[2]) for e in log1 if e[0] == "step")
    partial = sum(1 for p in range(P) if wl.prompt_lens[p] % B)
    # each prompt with a partial last block is copied by all but the last stream to write
    assert copies == (n - 1) * partial
    for s in range(P * n):
        L = int(wl.prompt_lens[s // n]) + int(wl.private_tokens[s])
        assert len(tables1[s]) * B - L < B                     # waste below one block per stream
    # full prompt blocks stay shared by all n streams; blocks in use = distinct blocks
    used = {b for t in tables1 for b in t}
    assert lib_a.num_free() == wl.num_blocks - len(used)
    for p in range(P):
        for b in tables1[p * n][: int(wl.prompt_lens[p]) // B]:
            assert lib_a.ref_count(b) == n
