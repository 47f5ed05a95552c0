"""Thin ctypes binding of libpa.so (include/pa.h), with the C function names.

Argument marshalling only: shapes, dtypes and pointers are read off torch tensors
and handed to the C ABI; every step of the path runs in the library's kernels.
Importing this module loads libpa.so and fails loudly if it is missing: there is
no fallback.  Build it with `python -m paged_kv_cache_363_b200.build`.
"""
import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libpa.so is not built (%s); run `python -m paged_kv_cache_363_b200.build`" % LIB_PATH)

lib = ctypes.CDLL(LIB_PATH)

PA_OK, PA_ERR_INVALID, PA_ERR_UNSUPPORTED, PA_ERR_OOM, PA_ERR_CUDA, PA_ERR_DEVICE_CHECK = 0, -1, -2, -3, -4, -5
PA_DTYPE_F32, PA_DTYPE_BF16 = 0, 1
PA_DEV_BAD_BLOCK, PA_DEV_BAD_CONTEXT, PA_DEV_BAD_SLOT, PA_DEV_BAD_PAIR, PA_DEV_WAIT_TIMEOUT = 1, 2, 4, 8, 16

_i32, _i64, _int, _f32, _vp, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
_u32 = ctypes.c_uint32


class pa_alloc_stats_t(ctypes.Structure):
    _fields_ = [(n, _i64) for n in ("num_blocks", "num_free", "num_seqs", "shared_blocks", "cow_copies",
                                   "tokens", "waste_tokens", "cached_blocks", "cached_free", "host_blocks",
                                   "host_free", "swapped_seqs")]


# (name, restype, argtypes) of every symbol declared in include/pa.h
SIGNATURES = [
    ("pa_decode_partition_size", _int, [_int] * 7),
    ("pa_decode_workspace_size", _sz, [_int] * 7),
    ("pa_decode", _int, [_vp, _vp, _vp, _vp, _vp, _vp] + [_int] * 8 + [_f32, _int, _vp, _sz, _int, _vp]),
    ("pa_decode_plan", _int, [_vp, _vp] + [_int] * 9 + [_vp, _sz, _int, _vp]),
    ("pa_decode_run", _int, [_vp, _vp, _vp, _vp, _vp, _vp] + [_int] * 8 + [_f32, _int, _vp, _sz, _int, _vp]),
    ("pa_decode_static_workspace", _int, [_vp, _vp, _vp, _vp, _vp, _vp] + [_int] * 8 + [_f32, _int, _int, _vp]),
    ("pa_reshape_and_cache", _int, [_vp, _vp, _vp, _vp, _vp] + [_int] * 6 + [_vp]),
    ("pa_prefill", _int, [_vp] * 7 + [_int] * 9 + [_f32, _int, _vp]),
    ("pa_prefill_workspace_size", _sz, []),
    ("pa_prefill_ws", _int, [_vp] * 7 + [_int] * 9 + [_f32, _vp, _sz, _int, _vp]),
    ("pa_copy_blocks", _int, [_vp, _vp, _vp] + [_int] * 6 + [_vp]),
    ("pa_check_block_mapping", _int, [_vp, _int, _int]),
    ("pa_check_slot_mapping", _int, [_vp, _int, _int, _int]),
    ("pa_swap_blocks", _int, [_vp, _vp, _vp, _vp, _vp] + [_int] * 7 + [_vp]),
    ("pa_device_status", _int, [ctypes.POINTER(_u32), _vp]),
    ("pa_selftest_bounded_wait", _int, [ctypes.POINTER(ctypes.c_uint64), _vp]),
    ("pa_alloc_create", _vp, [_int, _int, _vp]),
    ("pa_alloc_destroy", None, [_vp]),
    ("pa_alloc_add_seq", _int, [_vp, _i64, _int, _vp]),
    ("pa_alloc_add_seq_cached", _int, [_vp, _i64, _vp, _int, _vp, ctypes.POINTER(_int)]),
    ("pa_alloc_fork", _int, [_vp, _i64, _i64]),
    ("pa_alloc_append_slot", _int, [_vp, _i64, ctypes.POINTER(_i64), ctypes.POINTER(_i32), ctypes.POINTER(_i32)]),
    ("pa_alloc_append_slots", _int, [_vp, _vp, _int, _vp, _vp, ctypes.POINTER(_int)]),
    ("pa_alloc_beam_step", _int, [_vp, _vp, _int, _vp, _vp, _int, _vp, _vp, ctypes.POINTER(_int)]),
    ("pa_alloc_free_seq", _int, [_vp, _i64]),
    ("pa_alloc_add_host_pool", _int, [_vp, _int]),
    ("pa_alloc_swap_out", _int, [_vp, _i64, _vp, ctypes.POINTER(_int)]),
    ("pa_alloc_swap_in", _int, [_vp, _i64, _vp, ctypes.POINTER(_int)]),
    ("pa_alloc_num_host_free", _int, [_vp]),
    ("pa_alloc_is_swapped", _int, [_vp, _i64]),
    ("pa_alloc_block_table", _int, [_vp, _i64, _vp, _int, ctypes.POINTER(_int)]),
    ("pa_alloc_block_tables", _int, [_vp, _vp, _int, _vp, _int, _i32, _vp]),
    ("pa_alloc_ref_count", _int, [_vp, _i32]),
    ("pa_alloc_num_free", _int, [_vp]),
    ("pa_alloc_num_cached_free", _int, [_vp]),
    ("pa_alloc_num_tokens", _int, [_vp, _i64]),
    ("pa_alloc_stats", _int, [_vp, ctypes.POINTER(pa_alloc_stats_t)]),
    ("pa_last_error_string", ctypes.c_char_p, []),
]

for _name, _res, _args in SIGNATURES:
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class PAError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = lib.pa_last_error_string().decode(errors="replace")
        super().__init__("%s failed with status %d: %s" % (where, status, msg))


class OutOfBlocks(PAError):
    pass


def _check(status, where):
    if status == PA_ERR_OOM:
        raise OutOfBlocks(status, where)
    if status != PA_OK:
        raise PAError(status, where)


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return PA_DTYPE_F32
    if t.dtype == torch.bfloat16:
        return PA_DTYPE_BF16
    raise TypeError("unsupported dtype %s (fp32 or bf16)" % t.dtype)


def _dev_ptr(t, name):
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t.data_ptr()


def _pool_ptr(t, name):
    """A CUDA tensor, or a pinned CPU tensor (the library maps it), contiguous."""
    if not (t.is_cuda or t.is_pinned()):
        raise ValueError("%s must be a CUDA tensor or pinned host memory" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t.data_ptr()


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


# ---------------------------------------------------------------- device calls

def pa_decode_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                             partition_size=0):
    p = lib.pa_decode_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                                     partition_size)
    if p < 0:
        raise PAError(p, "pa_decode_partition_size")
    return p


def pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                             partition_size=0):
    return int(lib.pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                            max_context_len, partition_size))


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale, partition_size=0,
              workspace=None, stream=None):
    """out[S,Hq,D] <- paged decode attention of q[S,Hq,D] over k/v_cache[NB,Hkv,B,D].
    Without `workspace` a buffer of pa_decode_workspace_size() bytes is allocated for the call."""
    S, Hq, D = q.shape
    NB, Hkv, B, D2 = k_cache.shape
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or tuple(context_lens.shape) != (S,):
        raise ValueError("block_tables must be [S, max_blocks] and context_lens [S]")
    dt = _dtype_code(q)
    if any(_dtype_code(t) != dt for t in (out, k_cache, v_cache)):
        raise TypeError("q, out and the caches must share a dtype")
    import torch
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    if workspace is None:
        need = pa_decode_workspace_size(S, Hq, Hkv, D, B, int(max_context_len), int(partition_size))
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    ws_ptr, ws_bytes = _dev_ptr(workspace, "workspace"), workspace.numel() * workspace.element_size()
    st = lib.pa_decode(_dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"),
                       _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables"),
                       _dev_ptr(context_lens, "context_lens"), S, Hq, Hkv, D, B, block_tables.shape[1], NB,
                       int(max_context_len), float(scale), int(partition_size), ws_ptr, ws_bytes, dt,
                       _stream(stream))
    _check(st, "pa_decode")
    return out


PA_STATIC_WORKSPACE_BYTES = 16 * 1024 * 1024


def pa_decode_plan(block_tables, context_lens, max_context_len, num_heads, k_cache, workspace, partition_size=0,
                   dtype=None, stream=None):
    """The work plan of a decode step into `workspace` (run it with pa_decode_run, once per layer).
    k_cache gives the pool's shape and dtype (its data is not read); `dtype`, when given, must be
    that dtype (the plan's choice of kernel depends on it)."""
    NB, Hkv, B, D = k_cache.shape
    S = context_lens.shape[0]
    if dtype is not None and dtype != k_cache.dtype:
        raise ValueError("pa_decode_plan: dtype %s differs from k_cache's %s" % (dtype, k_cache.dtype))
    st = lib.pa_decode_plan(_dev_ptr(block_tables, "block_tables"), _dev_ptr(context_lens, "context_lens"), S,
                            int(num_heads), Hkv, D, B, block_tables.shape[1], NB, int(max_context_len),
                            int(partition_size), _dev_ptr(workspace, "workspace"),
                            workspace.numel() * workspace.element_size(), _dtype_code(k_cache), _stream(stream))
    _check(st, "pa_decode_plan")


def pa_decode_run(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale, workspace,
                  partition_size=0, stream=None):
    """Decode attention from the plan pa_decode_plan left in `workspace`."""
    S, Hq, D = q.shape
    NB, Hkv, B, D2 = k_cache.shape
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("shape mismatch")
    st = lib.pa_decode_run(_dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"),
                           _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables"),
                           _dev_ptr(context_lens, "context_lens"), S, Hq, Hkv, D, B, block_tables.shape[1], NB,
                           int(max_context_len), float(scale), int(partition_size), _dev_ptr(workspace, "workspace"),
                           workspace.numel() * workspace.element_size(), _dtype_code(q), _stream(stream))
    _check(st, "pa_decode_run")


def pa_decode_static_workspace(out, q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale,
                               partition_size=0, stream=None):
    """pa_decode for callers that cannot allocate device memory: the workspace is the
    library's own fixed 16 MiB device array (see include/pa.h).  Calls on one device
    share that array, so calls that could overlap must be ordered on one stream."""
    S, Hq, D = q.shape
    NB, Hkv, B, D2 = k_cache.shape
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or tuple(context_lens.shape) != (S,):
        raise ValueError("block_tables must be [S, max_blocks] and context_lens [S]")
    dt = _dtype_code(q)
    st = lib.pa_decode_static_workspace(_dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"),
                                        _dev_ptr(v_cache, "v_cache"), _dev_ptr(block_tables, "block_tables"),
                                        _dev_ptr(context_lens, "context_lens"), S, Hq, Hkv, D, B,
                                        block_tables.shape[1], NB, int(max_context_len), float(scale),
                                        int(partition_size), dt, _stream(stream))
    _check(st, "pa_decode_static_workspace")
    return out


def _host_int64(a):
    """A C-contiguous int64 numpy copy of a host or device array (for the host-side checks)."""
    import numpy as np
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a), dtype=np.int64)


def pa_check_block_mapping(block_mapping, num_blocks):
    """Host-side check of copy pairs [n, 2] (any array; copied to host): raises PAError if an
    entry is out of range, a destination repeats, or a destination is also a source."""
    m = _host_int64(block_mapping).reshape(-1)
    if m.size % 2:
        raise ValueError("block_mapping must be [n, 2]")
    n = m.size // 2
    _check(lib.pa_check_block_mapping(m.ctypes.data if n else None, n, int(num_blocks)), "pa_check_block_mapping")


def pa_check_slot_mapping(slot_mapping, num_blocks, block_size):
    """Host-side check of append slots (any array; copied to host): raises PAError if a slot
    >= 0 repeats or lies past the pool."""
    m = _host_int64(slot_mapping).reshape(-1)
    _check(lib.pa_check_slot_mapping(m.ctypes.data if m.size else None, m.size, int(num_blocks), int(block_size)),
           "pa_check_slot_mapping")


def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, stream=None, check=False):
    """k/v_cache[slot // B, :, slot % B, :] <- key/value[t] for every slot >= 0.  With check=True
    the slots are first copied to the host and checked (pa_check_slot_mapping; synchronising)."""
    N, Hkv, D = key.shape
    NB, Hkv2, B, D2 = k_cache.shape
    if (Hkv2, D2) != (Hkv, D) or tuple(value.shape) != tuple(key.shape) or tuple(slot_mapping.shape) != (N,):
        raise ValueError("shape mismatch")
    import torch
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    if check:
        pa_check_slot_mapping(slot_mapping, NB, B)
    dt = _dtype_code(key)
    st = lib.pa_reshape_and_cache(_dev_ptr(key, "key"), _dev_ptr(value, "value"), _dev_ptr(k_cache, "k_cache"),
                                  _dev_ptr(v_cache, "v_cache"), _dev_ptr(slot_mapping, "slot_mapping"), N, Hkv, D,
                                  B, NB, dt, _stream(stream))
    _check(st, "pa_reshape_and_cache")


def pa_prefill_workspace_size():
    return int(lib.pa_prefill_workspace_size())


def pa_prefill(out, q, k_cache, v_cache, block_tables, context_lens, q_start, max_query_len, scale, stream=None,
               workspace=None):
    """out[Nq,Hq,D] <- causal attention of the packed query rows q[Nq,Hq,D] (rows q_start[s]..q_start[s+1]-1
    are the last tokens of sequence s) over k/v_cache[NB,Hkv,B,D] through block_tables.  With a device
    `workspace` (at least pa_prefill_workspace_size() bytes) this calls pa_prefill_ws."""
    import torch
    Nq, Hq, D = q.shape
    NB, Hkv, B, D2 = k_cache.shape
    S = context_lens.shape[0]
    if D2 != D or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or tuple(q_start.shape) != (S + 1,):
        raise ValueError("block_tables must be [S, max_blocks] and q_start [S + 1]")
    if any(t.dtype != torch.int32 for t in (block_tables, context_lens, q_start)):
        raise TypeError("block_tables, context_lens and q_start must be int32")
    dt = _dtype_code(q)
    if any(_dtype_code(t) != dt for t in (out, k_cache, v_cache)):
        raise TypeError("q, out and the caches must share a dtype")
    args = (_dev_ptr(out, "out"), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
            _dev_ptr(block_tables, "block_tables"), _dev_ptr(context_lens, "context_lens"),
            _dev_ptr(q_start, "q_start"), S, Hq, Hkv, D, B, block_tables.shape[1], NB, Nq, int(max_query_len),
            float(scale))
    if workspace is None:
        _check(lib.pa_prefill(*args, dt, _stream(stream)), "pa_prefill")
    else:
        nbytes = workspace.numel() * workspace.element_size()
        _check(lib.pa_prefill_ws(*args, _dev_ptr(workspace, "workspace"), nbytes, dt, _stream(stream)),
               "pa_prefill_ws")


def pa_swap_blocks(dst_k_cache, dst_v_cache, src_k_cache, src_v_cache, block_mapping, stream=None):
    """For every (src, dst) row of block_mapping[n, 2] (int64): dst pools[dst] <- src pools[src].
    Pools and block_mapping may be CUDA tensors or pinned CPU tensors."""
    import torch
    NBs, Hkv, B, D = src_k_cache.shape
    NBd = dst_k_cache.shape[0]
    if tuple(dst_k_cache.shape[1:]) != (Hkv, B, D) or dst_k_cache.dtype != src_k_cache.dtype:
        raise ValueError("pools differ in block shape or dtype")
    if block_mapping.dtype != torch.int64 or (block_mapping.numel() and block_mapping.shape[-1] != 2):
        raise TypeError("block_mapping must be int64 [n, 2]")
    n = block_mapping.numel() // 2
    ptr = _pool_ptr(block_mapping, "block_mapping") if n else None
    st = lib.pa_swap_blocks(_pool_ptr(dst_k_cache, "dst_k_cache"), _pool_ptr(dst_v_cache, "dst_v_cache"),
                            _pool_ptr(src_k_cache, "src_k_cache"), _pool_ptr(src_v_cache, "src_v_cache"), ptr, n,
                            Hkv, D, B, NBs, NBd, _dtype_code(src_k_cache), _stream(stream))
    _check(st, "pa_swap_blocks")


def pa_copy_blocks(k_cache, v_cache, block_mapping, stream=None, check=False):
    """For every (src, dst) row of block_mapping[n, 2] (int64): block dst <- block src, both pools.
    With check=True the pairs are first copied to the host and checked (pa_check_block_mapping;
    synchronising)."""
    NB, Hkv, B, D = k_cache.shape
    import torch
    if block_mapping.dtype != torch.int64 or (block_mapping.numel() and block_mapping.shape[-1] != 2):
        raise TypeError("block_mapping must be int64 [n, 2]")
    n = block_mapping.numel() // 2
    if check:
        pa_check_block_mapping(block_mapping, NB)
    ptr = _dev_ptr(block_mapping, "block_mapping") if n else None
    st = lib.pa_copy_blocks(_dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"), ptr, n, Hkv, D, B, NB,
                            _dtype_code(k_cache), _stream(stream))
    _check(st, "pa_copy_blocks")


def pa_selftest_bounded_wait(stream=None):
    """Makes one bounded device wait run out (nothing arrives); returns the nanoseconds it
    waited.  PA_DEV_WAIT_TIMEOUT is then set in the status word."""
    ns = ctypes.c_uint64(0)
    _check(lib.pa_selftest_bounded_wait(ctypes.byref(ns), _stream(stream)), "pa_selftest_bounded_wait")
    return int(ns.value)


def pa_device_status(stream=None):
    """PA_DEV_* bits raised since the last call (waits for the stream; clears them)."""
    v = _u32(0)
    _check(lib.pa_device_status(ctypes.byref(v), _stream(stream)), "pa_device_status")
    return int(v.value)


# ---------------------------------------------------------------- allocator

def _np_ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


class Allocator:
    """Host block allocator with reference-counted copy-on-write (pa_alloc_*)."""

    def __init__(self, num_blocks, block_size, free_order=None):
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        fo = None
        if free_order is not None:
            fo = np.ascontiguousarray(free_order, dtype=np.int32)
            if fo.shape != (self.num_blocks,):
                raise ValueError("free_order must have num_blocks entries")
        h = lib.pa_alloc_create(self.num_blocks, self.block_size, _np_ptr(fo) if fo is not None else None)
        if not h:
            raise PAError(PA_ERR_INVALID, "pa_alloc_create")
        self._h = ctypes.c_void_p(h)
        # held here: at interpreter exit the module's globals may already be gone when __del__ runs
        self._destroy = lib.pa_alloc_destroy

    def close(self):
        if getattr(self, "_h", None):
            self._destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def add_seq(self, seq_id, num_tokens):
        slots = np.empty(max(1, int(num_tokens)), np.int64)
        _check(lib.pa_alloc_add_seq(self._h, int(seq_id), int(num_tokens), _np_ptr(slots)), "pa_alloc_add_seq")
        return slots[:int(num_tokens)]

    def add_seq_cached(self, seq_id, token_ids):
        """New sequence with these token ids, reusing cached prompt blocks.
        Returns (slots of all tokens, number of leading tokens already cached)."""
        ids = np.ascontiguousarray(token_ids, dtype=np.int32)
        n = ids.shape[0]
        slots = np.empty(max(1, n), np.int64)
        ncached = _int(0)
        _check(lib.pa_alloc_add_seq_cached(self._h, int(seq_id), _np_ptr(ids) if n else None, n, _np_ptr(slots),
                                           ctypes.byref(ncached)), "pa_alloc_add_seq_cached")
        return slots[:n], int(ncached.value)

    def fork(self, parent_id, child_id):
        _check(lib.pa_alloc_fork(self._h, int(parent_id), int(child_id)), "pa_alloc_fork")

    def append_slot(self, seq_id):
        slot, src, dst = _i64(0), _i32(-1), _i32(-1)
        _check(lib.pa_alloc_append_slot(self._h, int(seq_id), ctypes.byref(slot), ctypes.byref(src),
                                        ctypes.byref(dst)), "pa_alloc_append_slot")
        return int(slot.value), (None if src.value < 0 else (int(src.value), int(dst.value)))

    def append_slots(self, seq_ids):
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = ids.shape[0]
        slots = np.empty(max(1, n), np.int64)
        pairs = np.empty((max(1, n), 2), np.int64)
        ncow = _int(0)
        _check(lib.pa_alloc_append_slots(self._h, _np_ptr(ids), n, _np_ptr(slots), _np_ptr(pairs),
                                         ctypes.byref(ncow)), "pa_alloc_append_slots")
        return slots[:n], pairs[:ncow.value]

    def beam_step(self, beam_ids, parents, new_ids):
        """Beam j of the new set continues old beam parents[j] under new_ids[j] and gets
        one token.  Returns (slots of the new tokens, copy-on-write pairs [k, 2])."""
        old = np.ascontiguousarray(beam_ids, dtype=np.int64)
        par = np.ascontiguousarray(parents, dtype=np.int32)
        new = np.ascontiguousarray(new_ids, dtype=np.int64)
        if par.shape != new.shape:
            raise ValueError("parents and new_ids differ in length")
        n = new.shape[0]
        slots = np.empty(max(1, n), np.int64)
        pairs = np.empty((max(1, n), 2), np.int64)
        ncow = _int(0)
        _check(lib.pa_alloc_beam_step(self._h, _np_ptr(old), old.shape[0], _np_ptr(par), _np_ptr(new), n,
                                      _np_ptr(slots), _np_ptr(pairs), ctypes.byref(ncow)), "pa_alloc_beam_step")
        return slots[:n], pairs[:ncow.value]

    def free_seq(self, seq_id):
        _check(lib.pa_alloc_free_seq(self._h, int(seq_id)), "pa_alloc_free_seq")

    def add_host_pool(self, num_host_blocks):
        _check(lib.pa_alloc_add_host_pool(self._h, int(num_host_blocks)), "pa_alloc_add_host_pool")

    def _swap(self, fn, name, seq_id):
        cap = max(1, len(self.block_table(seq_id)))
        pairs = np.empty((cap, 2), np.int64)
        n = _int(0)
        _check(fn(self._h, int(seq_id), _np_ptr(pairs), ctypes.byref(n)), name)
        return pairs[:n.value]

    def swap_out(self, seq_id):
        """Moves the sequence to the host tier; returns its (device, host) block pairs."""
        return self._swap(lib.pa_alloc_swap_out, "pa_alloc_swap_out", seq_id)

    def swap_in(self, seq_id):
        """Brings the sequence back; returns its (host, device) block pairs."""
        return self._swap(lib.pa_alloc_swap_in, "pa_alloc_swap_in", seq_id)

    def num_host_free(self):
        return int(lib.pa_alloc_num_host_free(self._h))

    def is_swapped(self, seq_id):
        return int(lib.pa_alloc_is_swapped(self._h, int(seq_id)))

    def block_table(self, seq_id):
        n = _int(0)
        tokens = int(lib.pa_alloc_num_tokens(self._h, int(seq_id)))
        # a table holds ceil(tokens / B) blocks; an unknown id gets the call's own error
        cap = max(1, -(-tokens // self.block_size)) if tokens >= 0 else 1
        out = np.empty(cap, np.int32)
        _check(lib.pa_alloc_block_table(self._h, int(seq_id), _np_ptr(out), cap, ctypes.byref(n)),
               "pa_alloc_block_table")
        return out[:n.value].tolist()

    def block_tables(self, seq_ids, max_blocks, fill=-1):
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        out = np.empty((max(1, len(ids)), max(1, int(max_blocks))), np.int32)
        lens = np.empty(max(1, len(ids)), np.int32)
        _check(lib.pa_alloc_block_tables(self._h, _np_ptr(ids), len(ids), _np_ptr(out), int(max_blocks),
                                         int(fill), _np_ptr(lens)), "pa_alloc_block_tables")
        return out[:len(ids), :int(max_blocks)], lens[:len(ids)]

    def ref_count(self, block):
        return int(lib.pa_alloc_ref_count(self._h, int(block)))

    def num_free(self):
        return int(lib.pa_alloc_num_free(self._h))

    def num_cached_free(self):
        return int(lib.pa_alloc_num_cached_free(self._h))

    def num_tokens(self, seq_id):
        return int(lib.pa_alloc_num_tokens(self._h, int(seq_id)))

    def stats(self):
        s = pa_alloc_stats_t()
        _check(lib.pa_alloc_stats(self._h, ctypes.byref(s)), "pa_alloc_stats")
        return {n: int(getattr(s, n)) for n, _ in pa_alloc_stats_t._fields_}
