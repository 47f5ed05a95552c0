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
