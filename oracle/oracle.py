"""Python face of the fp64 C oracle, plus a pure-Python brute force for tiny cases.

TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU-baseline leg).

Citations are by page title and section:
  "PagedAttention Paper Breakdown" (fullstackaihub.com), section 2, Address
  Translation Formula: b = floor(i/B), o = i mod B, PhysicalAddr(K_i) = T[b]*B + o.
  "PagedAttention and vLLM Architecture" (initnode.dev), section 2 (the decode
  kernel walks the block table, softmaxes across all blocks and weights V) and
  section 3 (copy-on-write copies a whole block).
"""
import ctypes
import math

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        c_i64, c_i32, c_int, c_dbl, c_vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        L.oracle_physical_slot.restype = c_i64
        L.oracle_physical_slot.argtypes = [c_vp, c_int, c_i64]
        L.oracle_decode.restype = c_int
        L.oracle_decode.argtypes = [c_vp, c_vp, c_i64, c_vp, c_vp, c_vp, c_vp, c_vp,
                                    c_int, c_int, c_int, c_int, c_int, c_int, c_dbl, c_int]
        L.oracle_partial.restype = c_int
        L.oracle_partial.argtypes = [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                     c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_dbl]
        L.oracle_merge_partials.restype = None
        L.oracle_merge_partials.argtypes = [c_vp, c_vp, c_vp, c_vp, c_int, c_int]
        L.oracle_reshape_and_cache.restype = c_int
        L.oracle_reshape_and_cache.argtypes = [c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_int, c_int]
        L.oracle_copy_blocks.restype = c_int
        L.oracle_copy_blocks.argtypes = [c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_int, c_int]
        L.oracle_prefill.restype = c_int
        L.oracle_prefill.argtypes = [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_int,
                                     c_int, ctypes.c_double, c_int]
        del c_i32
        _lib = L
    return _lib


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def physical_slot(table, block_size, i):
    """Token-slot address of logical token i through one sequence's block table."""
    t = _c(table, np.int32)
    return int(lib().oracle_physical_slot(_ptr(t), int(block_size), int(i)))


def decode(q, k_cache, v_cache, block_tables, context_lens, scale, nthreads=1, return_weights=False):
    """fp64 paged decode attention.

    q: [S, Hq, D]; k_cache, v_cache: [NB, Hkv, B, D] (any float dtype, widened to
    fp32 exactly: fp32 or bf16 values); block_tables: [S, MB] int; context_lens: [S].
    Returns out [S, Hq, D] float64 (and the softmax weights [S, Hq, max L] if asked).
    """
    q = _c(q, np.float32)
    k = _c(k_cache, np.float32)
    v = _c(v_cache, np.float32)
    T = _c(block_tables, np.int32)
    Ls = _c(context_lens, np.int32)
    S, Hq, D = q.shape
    NB, Hkv, B, D2 = k.shape
    assert D2 == D and v.shape == k.shape and T.shape[0] == S and Ls.shape == (S,)
    MB = T.shape[1] if T.ndim == 2 else 0
    out = np.zeros((S, Hq, D), np.float64)
    wstride = max(1, int(Ls.max()) if S else 1)
    w = np.zeros((S, Hq, wstride), np.float64) if return_weights else None
    rc = lib().oracle_decode(_ptr(out), _ptr(w), wstride, _ptr(q), _ptr(k), _ptr(v), _ptr(T), _ptr(Ls),
                             S, Hq, Hkv, D, B, MB, float(scale), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_decode rejected its arguments")
    return (out, w) if return_weights else out


def partial(q_row, k_cache, v_cache, table, num_heads, h, t0, t1, scale):
    """(m, l, acc) of one (sequence, head) over logical tokens [t0, t1)."""
    q = _c(q_row, np.float32)
    k = _c(k_cache, np.float32)
    v = _c(v_cache, np.float32)
    T = _c(table, np.int32)
    NB, Hkv, B, D = k.shape
    m = np.zeros(1, np.float64)
    l = np.zeros(1, np.float64)
    acc = np.zeros(D, np.float64)
    rc = lib().oracle_partial(_ptr(m), _ptr(l), _ptr(acc), _ptr(q), _ptr(k), _ptr(v), _ptr(T),
                              num_heads, Hkv, D, B, h, t0, t1, float(scale))
    if rc != 0:
        raise ValueError("oracle_partial rejected its arguments")
    return float(m[0]), float(l[0]), acc


def merge_partials(ms, ls, accs):
    ms = _c(ms, np.float64)
    ls = _c(ls, np.float64)
    accs = _c(accs, np.float64)
    n, D = accs.shape
    out = np.zeros(D, np.float64)
    lib().oracle_merge_partials(_ptr(out), _ptr(ms), _ptr(ls), _ptr(accs), n, D)
    return out


def reshape_and_cache(key, value, k_cache, v_cache, slot_mapping):
    """Returns updated copies of (k_cache, v_cache); exact for any element type."""
    key = np.ascontiguousarray(key)
    value = np.ascontiguousarray(value)
    kc = np.array(k_cache, copy=True, order="C")
    vc = np.array(v_cache, copy=True, order="C")
    sm = _c(slot_mapping, np.int64)
    N, Hkv, D = key.shape
    NB, Hkv2, B, D2 = kc.shape
    assert Hkv2 == Hkv and D2 == D and key.dtype == kc.dtype and value.dtype == vc.dtype
    rc = lib().oracle_reshape_and_cache(_ptr(key), _ptr(value), _ptr(kc), _ptr(vc), _ptr(sm),
                                        N, Hkv, D, B, NB, kc.dtype.itemsize)
    if rc != 0:
        raise ValueError("oracle_reshape_and_cache: slot out of range")
    return kc, vc


def copy_blocks(k_cache, v_cache, block_mapping):
    """Returns updated copies of (k_cache, v_cache) after the (src, dst) block copies."""
    kc = np.array(k_cache, copy=True, order="C")
    vc = np.array(v_cache, copy=True, order="C")
    bm = _c(block_mapping, np.int64).reshape(-1, 2)
    NB, Hkv, B, D = kc.shape
    rc = lib().oracle_copy_blocks(_ptr(kc), _ptr(vc), _ptr(bm), bm.shape[0], Hkv, D, B, NB, kc.dtype.itemsize)
    if rc != 0:
        raise ValueError("oracle_copy_blocks: block index out of range")
    return kc, vc


def prefill(q, k_cache, v_cache, block_tables, context_lens, q_start, scale, nthreads=1):
    """fp64 chunked-prefill attention: query i of sequence s (row q_start[s] + i of
    q [Nq, Hq, D]) sits at position context_lens[s] - n_s + i and attends to tokens
    0..that position through the block table.  Returns out [Nq, Hq, D] float64."""
    q = _c(q, np.float32)
    k = _c(k_cache, np.float32)
    v = _c(v_cache, np.float32)
    T = _c(block_tables, np.int32)
    Ls = _c(context_lens, np.int32)
    qs = _c(q_start, np.int32)
    Nq, Hq, D = q.shape
    NB, Hkv, B, D2 = k.shape
    S = Ls.shape[0]
    assert D2 == D and v.shape == k.shape and qs.shape == (S + 1,) and int(qs[-1]) == Nq
    MB = T.shape[1] if T.ndim == 2 else 0
    out = np.zeros((Nq, Hq, D), np.float64)
    rc = lib().oracle_prefill(_ptr(out), _ptr(q), _ptr(k), _ptr(v), _ptr(T), _ptr(Ls), _ptr(qs), S, Hq, Hkv, D,
                              B, MB, float(scale), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_prefill rejected its arguments")
    return out


def decode_bruteforce(q, k_cache, v_cache, block_tables, context_lens, scale):
    """Pure-Python loops (math.exp, Python floats) for tiny inputs: an independent
    restatement of the same definition, used to pin the C oracle."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k_cache, np.float64)
    v = np.asarray(v_cache, np.float64)
    S, Hq, D = q.shape
    NB, Hkv, B, _ = k.shape
    group = Hq // Hkv
    out = [[[0.0] * D for _ in range(Hq)] for _ in range(S)]
    for s in range(S):
        L = int(context_lens[s])
        for h in range(Hq):
            kvh = h // group
            keys, vals = [], []
            for i in range(L):
                blk = int(block_tables[s][i // B])
                off = i % B
                keys.append([float(x) for x in k[blk, kvh, off]])
                vals.append([float(x) for x in v[blk, kvh, off]])
            logits = [scale * sum(float(q[s, h, d]) * kk[d] for d in range(D)) for kk in keys]
            if not logits:
                continue
            top = max(logits)
            e = [math.exp(z - top) for z in logits]
            tot = sum(e)
            for d in range(D):
                out[s][h][d] = sum(e[i] / tot * vals[i][d] for i in range(L))
    return np.array(out, np.float64)
