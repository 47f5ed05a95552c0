"""The seeded generator: deterministic, shaped like the stated workloads (CPU only)."""
import math

import numpy as np

from paged_kv_cache_363_b200 import workloads as W


def test_deterministic_and_seed_dependent():
    a, b, c = W.make_workload(2, 0), W.make_workload(2, 0), W.make_workload(2, 1)
    assert np.array_equal(a.context_lens, b.context_lens) and np.array_equal(a.free_order, b.free_order)
    assert not np.array_equal(a.context_lens, c.context_lens)


def test_shapes_and_ranges():
    for wid in (1, 2, 3, 5):
        for seed in range(3):
            wl = W.make_workload(wid, seed)
            spec = W.WORKLOADS[wid]
            assert len(wl.context_lens) == spec["num_seqs"]
            if spec["lens"][0] == "uniform":
                assert wl.context_lens.min() >= spec["lens"][1] and wl.context_lens.max() <= spec["lens"][2]
            else:
                assert wl.context_lens.min() >= 16 and wl.context_lens.max() <= 4096
            blocks = sum(-(-int(L) // wl.block_size) for L in wl.context_lens)
            assert blocks <= wl.num_blocks
            assert sorted(wl.free_order.tolist()) == list(range(wl.num_blocks))
            assert math.isclose(wl.scale, 1 / math.sqrt(wl.head_dim))


def test_gqa_lengths_are_lognormal_around_500():
    lens = np.concatenate([W.make_workload(3, s).context_lens for s in range(3)])
    assert 400 <= np.median(lens) <= 620


def test_cow_workload_fits_and_values_line_up():
    wl = W.make_workload(4, 0)
    assert wl.num_seqs == 128 and wl.prompt_lens.min() >= 256 and wl.prompt_lens.max() <= 1024
    assert wl.private_tokens.min() >= 1 and wl.private_tokens.max() <= 40
    q, pk, pv, poff, xk, xv, xoff = W.cow_values(W.make_workload(4, 0, num_prompts=2, head_dim=64), "cpu")
    assert pk.shape[0] == poff[-1] and xk.shape[0] == xoff[-1]


def test_values_depend_only_on_seed():
    wl = W.make_workload(1, 3)
    q1, k1, v1, o1 = W.decode_values(wl, "cpu")
    q2, k2, v2, o2 = W.decode_values(wl, "cpu")
    assert (q1 == q2).all() and (k1 == k2).all() and (v1 == v2).all() and np.array_equal(o1, o2)
    assert k1.shape[0] == int(wl.context_lens.sum())
