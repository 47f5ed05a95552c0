"""Test helpers: the oracle's side of each comparison, built only from the seeded
generator's values and the oracle (never from anything the CUDA path produced)."""
import json
import os

import numpy as np
import torch

from oracle import oracle
from oracle.allocator import OracleAllocator

TOL = {"f32": 1e-5, "bf16": 2e-2}     # max-abs tolerance on the attention output


def bits(t):
    """Raw element bits of a CPU or CUDA tensor as a numpy array (exact)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32)
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype in (torch.int32, torch.int64):
        return t.numpy()
    raise TypeError(t.dtype)


def bits_to_f32(b):
    """fp32 values of raw fp32 / bf16 bits (bf16 widens exactly)."""
    if b.dtype == np.uint32:
        return b.view(np.float32)
    return (b.astype(np.uint32) << 16).view(np.float32)


def nan_bits(dtype):
    return np.uint32(0x7FC00000) if dtype == "f32" else np.uint16(0x7FC0)


def oracle_decode_side(wl, values):
    """The oracle's own run of a decode workload: oracle allocator places the prefill
    and the appended token, oracle scatter fills NaN-initialised pools, oracle decode
    runs before and after the append.  values = workloads.decode_values(wl, 'cpu')."""
    q, keys, vals, off = values
    S, Hkv, D, B, NB = wl.num_seqs, wl.num_kv_heads, wl.head_dim, wl.block_size, wl.num_blocks
    kb, vb = bits(keys), bits(vals)
    ora = OracleAllocator(NB, B, wl.free_order)
    pre_slots, pre_rows = [], []
    for s in range(S):
        n = int(wl.context_lens[s]) - 1
        pre_slots += ora.add_seq(s, n)
        pre_rows += list(range(off[s], off[s] + n))
    nb = nan_bits(wl.dtype)
    kpool = np.full((NB, Hkv, B, D), nb)
    vpool = np.full((NB, Hkv, B, D), nb)
    if pre_rows:
        kpool, vpool = oracle.reshape_and_cache(kb[pre_rows], vb[pre_rows], kpool, vpool, np.array(pre_slots))
    mb = max(1, max(len(ora.tables[s]) for s in range(S)))
    tables_pre = np.full((S, mb), -1, np.int32)
    for s in range(S):
        tables_pre[s, :len(ora.tables[s])] = ora.tables[s]
    lens_pre = np.array([ora.ntokens[s] for s in range(S)], np.int32)
    qf = bits_to_f32(bits(q))
    out_pre = oracle.decode(qf, bits_to_f32(kpool), bits_to_f32(vpool), tables_pre, lens_pre, wl.scale,
                            nthreads=4)
    new = [ora.append_slot(s) for s in range(S)]
    assert all(c is None for _, c in new)
    last = [off[s + 1] - 1 for s in range(S)]
    kpool, vpool = oracle.reshape_and_cache(kb[last], vb[last], kpool, vpool, np.array([x for x, _ in new]))
    mb = max(len(ora.tables[s]) for s in range(S))
    tables = np.full((S, mb), -1, np.int32)
    for s in range(S):
        tables[s, :len(ora.tables[s])] = ora.tables[s]
    lens = np.array([ora.ntokens[s] for s in range(S)], np.int32)
    out = oracle.decode(qf, bits_to_f32(kpool), bits_to_f32(vpool), tables, lens, wl.scale, nthreads=4)
    return dict(allocator=ora, kpool=kpool, vpool=vpool, tables=tables, lens=lens, out=out,
                tables_pre=tables_pre, lens_pre=lens_pre, out_pre=out_pre)


NTHREADS = max(1, os.cpu_count() or 1)


def _compact_pool(k_seqs, v_seqs, block_size):
    """Sequences given by their logical K/V rows (each [L, Hkv, D] fp32) placed in a
    compact pool, sequence after sequence, with identity block tables."""
    S = len(k_seqs)
    B = block_size
    Hkv, D = k_seqs[0].shape[1], k_seqs[0].shape[2]
    nblk = [max(1, -(-len(k) // B)) for k in k_seqs]
    NB = sum(nblk)
    kp = np.zeros((NB, Hkv, B, D), np.float32)
    vp = np.zeros((NB, Hkv, B, D), np.float32)
    tables = np.full((S, max(nblk)), -1, np.int32)
    base = 0
    for s in range(S):
        L = len(k_seqs[s])
        pad = nblk[s] * B - L
        kk = np.concatenate([k_seqs[s], np.zeros((pad, Hkv, D), np.float32)])
        vv = np.concatenate([v_seqs[s], np.zeros((pad, Hkv, D), np.float32)])
        kp[base:base + nblk[s]] = kk.reshape(nblk[s], B, Hkv, D).transpose(0, 2, 1, 3)
        vp[base:base + nblk[s]] = vv.reshape(nblk[s], B, Hkv, D).transpose(0, 2, 1, 3)
        tables[s, :nblk[s]] = np.arange(base, base + nblk[s])
        base += nblk[s]
    lens = np.array([len(k) for k in k_seqs], np.int32)
    return kp, vp, tables, lens


def oracle_logical(q_rows, k_seqs, v_seqs, block_size, scale):
    """Oracle attention of sequences given directly by their logical K/V rows
    (each [L, Hkv, D] fp32), placed in a compact pool with an identity block table
    (the result does not depend on placement: a pinned property of the oracle)."""
    kp, vp, tables, lens = _compact_pool(k_seqs, v_seqs, block_size)
    return oracle.decode(np.asarray(q_rows, np.float32), kp, vp, tables, lens, scale, nthreads=NTHREADS)


def oracle_logical_all(q, seq_rows, block_size, scale, token_budget=200_000):
    """oracle_logical over a whole batch, a few sequences at a time so the fp32 pools
    stay small.  q: [S, Hq, D]; seq_rows(s) -> (K rows, V rows) of sequence s, each
    [L_s, Hkv, D] fp32.  Returns out [S, Hq, D] float64: every row of the batch."""
    q = np.asarray(q, np.float32)
    S = q.shape[0]
    out = np.zeros(q.shape, np.float64)
    s0 = 0
    while s0 < S:
        ks, vs, s1, tok = [], [], s0, 0
        while s1 < S and (s1 == s0 or tok < token_budget):
            k, v = seq_rows(s1)
            ks.append(np.asarray(k, np.float32))
            vs.append(np.asarray(v, np.float32))
            tok += len(k)
            s1 += 1
        out[s0:s1] = oracle_logical(q[s0:s1], ks, vs, block_size, scale)
        s0 = s1
    return out


def oracle_logical_prefill(q_rows, k_seq, v_seq, block_size, scale):
    """Oracle chunked prefill of one sequence given by its logical K/V rows
    ([L, Hkv, D] fp32): the n = len(q_rows) queries are its last n tokens."""
    kp, vp, tables, lens = _compact_pool([k_seq], [v_seq], block_size)
    n = len(q_rows)
    return oracle.prefill(np.asarray(q_rows, np.float32), kp, vp, tables, lens, np.array([0, n], np.int32), scale,
                          nthreads=NTHREADS)


def report_error(name, err, rows=None):
    """Print a comparison's max-abs error and, when PA_PARITY_REPORT names a file,
    append it there as a JSON line."""
    print("parity %s: max-abs %.4g%s" % (name, err, "" if rows is None else " over %d rows" % rows))
    path = os.environ.get("PA_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": name, "max_abs": err, "rows": rows}) + "\n")


def max_abs(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b))) if a.size else 0.0
