"""Decode-step drivers built only from the C-ABI calls in `pa`.

A DecodeBatch holds one serving batch on the device: the two KV pools, the host
block allocator that places the sequences, and the inputs of one decode step.
Its prefill writes every prompt token through pa_reshape_and_cache at the slot the
allocator gives it; a step then appends each sequence's new token (copy-on-write
copies first, then the slot-mapped append) and runs paged decode attention.

A CowBatch does the same for parallel sampling: prompts are forked into streams
that share their blocks, and every stream appends private tokens, which triggers
copy-on-write of the shared partial last blocks.

The torch calls here only allocate memory, move bytes and index tensors.
"""
import math
import time

import numpy as np
import torch

from . import pa
from . import workloads as W


def _round_up(x, m):
    return (x + m - 1) // m * m


class DecodeBatch:
    def __init__(self, wl, device="cuda", values=None, fill=float("nan"), partition_size=None):
        self.wl = wl
        self.device = torch.device(device)
        S, Hq, Hkv, D, B, NB = (wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
                                wl.num_blocks)
        dt = W.torch_dtype(wl.dtype)
        if values is None:
            values = W.decode_values(wl, self.device)
        q, keys, vals, offsets = values
        self.k_cache = torch.full((NB, Hkv, B, D), fill, dtype=dt, device=self.device)
        self.v_cache = torch.full((NB, Hkv, B, D), fill, dtype=dt, device=self.device)
        self.alloc = pa.Allocator(NB, B, wl.free_order)
        lens = np.asarray(wl.context_lens, np.int64)

        # prefill: every token but the last of each sequence
        pre_slots, pre_rows = [], []
        for s in range(S):
            n = int(lens[s]) - 1
            pre_slots.append(self.alloc.add_seq(s, n))
            pre_rows.append(np.arange(offsets[s], offsets[s] + n, dtype=np.int64))
        pre_slots = np.concatenate(pre_slots) if S else np.zeros(0, np.int64)
        pre_rows = np.concatenate(pre_rows) if S else np.zeros(0, np.int64)
        if len(pre_rows):
            idx = torch.from_numpy(pre_rows).to(keys.device)
            pk = keys.index_select(0, idx).to(self.device).contiguous()
            pv = vals.index_select(0, idx).to(self.device).contiguous()
            sm = torch.from_numpy(pre_slots).to(self.device)
            pa.pa_reshape_and_cache(pk, pv, self.k_cache, self.v_cache, sm)
            del pk, pv, sm
        self.prefill_tables = self.tables_now()

        # the step: one new token per sequence
        slots, pairs = self.alloc.append_slots(np.arange(S, dtype=np.int64))
        last = torch.from_numpy(offsets[1:] - 1).to(keys.device)
        self.new_k = keys.index_select(0, last).to(self.device).contiguous()
        self.new_v = vals.index_select(0, last).to(self.device).contiguous()
        self.slot_mapping = torch.from_numpy(slots.copy()).to(self.device)
        self.cow_pairs = torch.from_numpy(pairs.copy()).to(self.device)
        self.q = q.to(self.device).contiguous()
        tables, ctx = self.tables_now()
        self.block_tables = torch.from_numpy(tables).to(self.device)
        self.context_lens = torch.from_numpy(ctx).to(self.device)
        self.max_context_len = int(ctx.max()) if S else 0
        self.partition_size = wl.partition_size if partition_size is None else partition_size
        self.out = torch.empty_like(self.q)
        ws = pa.pa_decode_workspace_size(S, Hq, Hkv, D, B, self.max_context_len, self.partition_size)
        self.workspace = torch.empty(max(ws, 16) // 4 + 4, dtype=torch.float32, device=self.device)

    def tables_now(self):
        S, B = self.wl.num_seqs, self.wl.block_size
        ids = np.arange(S, dtype=np.int64)
        mb = max(1, max((self.alloc.num_tokens(s) + B - 1) // B for s in range(S)) if S else 1)
        return self.alloc.block_tables(ids, mb, fill=-1)

    def append(self, stream=None):
        """Copy-on-write copies (if any), then the slot-mapped append of the new tokens."""
        if self.cow_pairs.numel():
            pa.pa_copy_blocks(self.k_cache, self.v_cache, self.cow_pairs, stream=stream)
        pa.pa_reshape_and_cache(self.new_k, self.new_v, self.k_cache, self.v_cache, self.slot_mapping,
                                stream=stream)

    def decode(self, out=None, stream=None, partition_size=None):
        out = self.out if out is None else out
        part = self.partition_size if partition_size is None else partition_size
        pa.pa_decode(out, self.q, self.k_cache, self.v_cache, self.block_tables, self.context_lens,
                     self.max_context_len, self.wl.scale, part, self.workspace_for(part), stream=stream)
        return out

    def workspace_for(self, part):
        """Workspace large enough for `part` (grown once if needed)."""
        wl = self.wl
        need = pa.pa_decode_workspace_size(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim,
                                           wl.block_size, self.max_context_len, part)
        if need > self.workspace.numel() * 4:
            self.workspace = torch.empty(need // 4 + 4, dtype=torch.float32, device=self.device)
        return self.workspace

    def step(self, stream=None):
        self.append(stream)
        return self.decode(stream=stream)

    # ---- accounting (bytes the step must move, by definition of the computation)
    def decode_bytes(self):
        """K and V rows of every context token, plus q, out, tables and lengths."""
        wl = self.wl
        elt = 4 if wl.dtype == "f32" else 2
        tok = int(np.sum(wl.context_lens))
        blocks = int(sum((int(L) + wl.block_size - 1) // wl.block_size for L in wl.context_lens))
        return (tok * 2 * wl.num_kv_heads * wl.head_dim * elt
                + 2 * wl.num_seqs * wl.num_heads * wl.head_dim * elt
                + 4 * (blocks + wl.num_seqs))

    def append_bytes(self):
        wl = self.wl
        elt = 4 if wl.dtype == "f32" else 2
        row = wl.num_kv_heads * wl.head_dim * elt
        return wl.num_seqs * (2 * row * 2 + 8)


class CowBatch:
    """Parallel sampling: prompts forked into streams, then private appends with copy-on-write."""

    def __init__(self, wl, device="cuda", values=None, fill=float("nan"), partition_size=None):
        self.wl = wl
        self.device = torch.device(device)
        P, n = wl.num_prompts, wl.streams_per_prompt
        Hq, Hkv, D, B, NB = wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size, wl.num_blocks
        dt = W.torch_dtype(wl.dtype)
        if values is None:
            values = W.cow_values(wl, self.device)
        q, pk, pv, poff, xk, xv, xoff = values
        self.k_cache = torch.full((NB, Hkv, B, D), fill, dtype=dt, device=self.device)
        self.v_cache = torch.full((NB, Hkv, B, D), fill, dtype=dt, device=self.device)
        self.alloc = pa.Allocator(NB, B, wl.free_order)
        self.log = []          # per append step: (stream ids, slots, cow pairs)
        slots = [self.alloc.add_seq(p * n, int(wl.prompt_lens[p])) for p in range(P)]
        sm = torch.from_numpy(np.concatenate(slots)).to(self.device)
        pa.pa_reshape_and_cache(pk.to(self.device).contiguous(), pv.to(self.device).contiguous(),
                                self.k_cache, self.v_cache, sm)
        for p in range(P):
            for j in range(1, n):
                self.alloc.fork(p * n, p * n + j)
        priv = np.asarray(wl.private_tokens)
        for t in range(int(priv.max())):
            active = np.nonzero(priv > t)[0].astype(np.int64)
            sl, pairs = self.alloc.append_slots(active)
            self.log.append((active, sl.copy(), pairs.copy()))
            if len(pairs):
                pa.pa_copy_blocks(self.k_cache, self.v_cache, torch.from_numpy(pairs).to(self.device))
            rows = torch.from_numpy(xoff[active] + t).to(xk.device)
            pa.pa_reshape_and_cache(xk.index_select(0, rows).to(self.device).contiguous(),
                                    xv.index_select(0, rows).to(self.device).contiguous(),
                                    self.k_cache, self.v_cache, torch.from_numpy(sl).to(self.device))
        S = wl.num_seqs
        ids = np.arange(S, dtype=np.int64)
        mb = max((self.alloc.num_tokens(s) + B - 1) // B for s in range(S))
        tables, ctx = self.alloc.block_tables(ids, mb, fill=-1)
        self.context_lens_np = ctx
        self.block_tables = torch.from_numpy(tables).to(self.device)
        self.context_lens = torch.from_numpy(ctx).to(self.device)
        self.max_context_len = int(ctx.max())
        self.q = q.to(self.device).contiguous()
        # the decode step re-appends every stream's last private token at its slot
        last_rows = torch.from_numpy(xoff[1:] - 1).to(xk.device)
        self.new_k = xk.index_select(0, last_rows).to(self.device).contiguous()
        self.new_v = xv.index_select(0, last_rows).to(self.device).contiguous()
        last_slot = np.empty(S, np.int64)
        for active, sl, _ in self.log:
            last_slot[active] = sl
        self.slot_mapping = torch.from_numpy(last_slot).to(self.device)
        self.partition_size = wl.partition_size if partition_size is None else partition_size
        self.out = torch.empty_like(self.q)
        ws = pa.pa_decode_workspace_size(S, Hq, Hkv, D, B, self.max_context_len, self.partition_size)
        self.workspace = torch.empty(max(ws, 16) // 4 + 4, dtype=torch.float32, device=self.device)

    def append(self, stream=None):
        pa.pa_reshape_and_cache(self.new_k, self.new_v, self.k_cache, self.v_cache, self.slot_mapping,
                                stream=stream)

    def decode(self, out=None, stream=None, partition_size=None):
        out = self.out if out is None else out
        part = self.partition_size if partition_size is None else partition_size
        pa.pa_decode(out, self.q, self.k_cache, self.v_cache, self.block_tables, self.context_lens,
                     self.max_context_len, self.wl.scale, part, self.workspace_for(part), stream=stream)
        return out

    def workspace_for(self, part):
        """Workspace large enough for `part` (grown once if needed)."""
        wl = self.wl
        need = pa.pa_decode_workspace_size(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim,
                                           wl.block_size, self.max_context_len, part)
        if need > self.workspace.numel() * 4:
            self.workspace = torch.empty(need // 4 + 4, dtype=torch.float32, device=self.device)
        return self.workspace

    def step(self, stream=None):
        self.append(stream)
        return self.decode(stream=stream)

    def decode_bytes(self):
        wl = self.wl
        tok = int(np.sum(self.context_lens_np))
        blocks = int(sum((int(L) + wl.block_size - 1) // wl.block_size for L in self.context_lens_np))
        return tok * 2 * wl.num_kv_heads * wl.head_dim * 2 + 2 * wl.num_seqs * wl.num_heads * wl.head_dim * 2 + \
            4 * (blocks + wl.num_seqs)

    def append_bytes(self):
        wl = self.wl
        return wl.num_seqs * (2 * wl.num_kv_heads * wl.head_dim * 2 * 2 + 8)


class PrefixBatch:
    """Requests sharing system prompts through the allocator's prefix cache.

    Each request's prompt (all its tokens but the last) is added by token ids; only
    the tokens past the cached full-block prefix are written into the pools, so a
    stem's full blocks are written once and read by every request that shares it.
    The decode step appends each request's last token and runs decode attention.
    """

    def __init__(self, wl, device="cuda", values=None, fill=float("nan"), partition_size=None):
        self.wl = wl
        self.device = torch.device(device)
        S, Hq, Hkv, D, B, NB = (wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
                                wl.num_blocks)
        dt = W.torch_dtype(wl.dtype)
        if values is None:
            values = W.prefix_values(wl, self.device)
        q, sk, sv, soff, xk, xv, xoff = values
        self.k_cache = torch.full((NB, Hkv, B, D), fill, dtype=dt, device=self.device)
        self.v_cache = torch.full((NB, Hkv, B, D), fill, dtype=dt, device=self.device)
        self.alloc = pa.Allocator(NB, B, wl.free_order)
        self.cached_tokens = np.zeros(S, np.int64)
        write = {0: ([], []), 1: ([], [])}          # source -> (rows, slots)
        prompts = [wl.tokens(r)[:-1] for r in range(S)]
        t0 = time.perf_counter()
        placed = [self.alloc.add_seq_cached(r, prompts[r]) for r in range(S)]
        self.alloc_us_per_request = 1e6 * (time.perf_counter() - t0) / max(1, S)
        for r in range(S):
            slots, nc = placed[r]
            self.cached_tokens[r] = nc
            rows = W.prefix_logical_rows(wl, r, soff, xoff)[:-1]
            for (src, row), slot in zip(rows[nc:], slots[nc:]):
                write[src][0].append(row)
                write[src][1].append(int(slot))
        for src, (kk, vv) in ((0, (sk, sv)), (1, (xk, xv))):
            rows, slots = write[src]
            if rows:
                idx = torch.tensor(rows, dtype=torch.int64, device=kk.device)
                pa.pa_reshape_and_cache(kk.index_select(0, idx).to(self.device).contiguous(),
                                        vv.index_select(0, idx).to(self.device).contiguous(),
                                        self.k_cache, self.v_cache,
                                        torch.tensor(slots, dtype=torch.int64, device=self.device))
        self.written_tokens = sum(len(write[s][0]) for s in write)
        self.prefill_tables = self.tables_now()
        # the step: each request's last token
        slots, pairs = self.alloc.append_slots(np.arange(S, dtype=np.int64))
        last = torch.from_numpy(xoff[1:] - 1).to(xk.device)
        self.new_k = xk.index_select(0, last).to(self.device).contiguous()
        self.new_v = xv.index_select(0, last).to(self.device).contiguous()
        self.slot_mapping = torch.from_numpy(slots.copy()).to(self.device)
        self.cow_pairs = torch.from_numpy(pairs.copy()).to(self.device)
        self.q = q.to(self.device).contiguous()
        tables, ctx = self.tables_now()
        self.context_lens_np = ctx
        self.block_tables = torch.from_numpy(tables).to(self.device)
        self.context_lens = torch.from_numpy(ctx).to(self.device)
        self.max_context_len = int(ctx.max()) if S else 0
        self.partition_size = wl.partition_size if partition_size is None else partition_size
        self.out = torch.empty_like(self.q)
        ws = pa.pa_decode_workspace_size(S, Hq, Hkv, D, B, self.max_context_len, self.partition_size)
        self.workspace = torch.empty(max(ws, 16) // 4 + 4, dtype=torch.float32, device=self.device)

    tables_now = DecodeBatch.tables_now
    append = DecodeBatch.append
    decode = DecodeBatch.decode
    workspace_for = DecodeBatch.workspace_for
    step = DecodeBatch.step

    def decode_bytes(self):
        """Logical bytes: every request's context read in full, as the decode does."""
        wl = self.wl
        tok = int(np.sum(self.context_lens_np))
        blocks = int(sum((int(L) + wl.block_size - 1) // wl.block_size for L in self.context_lens_np))
        return tok * 2 * wl.num_kv_heads * wl.head_dim * 2 + 2 * wl.num_seqs * wl.num_heads * wl.head_dim * 2 + \
            4 * (blocks + wl.num_seqs)

    def unique_kv_bytes(self):
        """K/V bytes of the distinct blocks the decode reads (each read at least once)."""
        wl = self.wl
        used = np.unique(self.block_tables.cpu().numpy())
        return int((used >= 0).sum()) * wl.block_size * 2 * wl.num_kv_heads * wl.head_dim * 2

    append_bytes = DecodeBatch.append_bytes


class BeamBatch:
    """Beam search through the allocator's beam step.

    Each request's prompt is written once and forked into its beams.  Every beam step
    reshuffles the beams (pa_alloc_beam_step: fork the chosen parents, free the old
    beams, append one slot per new beam), runs the step's copy-on-write copies as one
    pa_copy_blocks, and writes the new tokens with pa_reshape_and_cache.  All steps but
    the last run at construction; the last one is the batch's step (copies, append,
    decode), which can be repeated: the copies and the append rewrite the same bytes.
    """

    def __init__(self, wl, device="cuda", values=None, fill=float("nan"), partition_size=None):
        self.wl = wl
        self.device = torch.device(device)
        S, Hq, Hkv, D, B, NB = (wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
                                wl.num_blocks)
        Wd, T = wl.beam_width, wl.beam_steps
        dt = W.torch_dtype(wl.dtype)
        if values is None:
            values = W.beam_values(wl, self.device)
        q, pk, pv, poff, nk, nv = values
        self.k_cache = torch.full((NB, Hkv, B, D), fill, dtype=dt, device=self.device)
        self.v_cache = torch.full((NB, Hkv, B, D), fill, dtype=dt, device=self.device)
        self.alloc = pa.Allocator(NB, B, wl.free_order)
        ids = np.arange(S, dtype=np.int64)
        slots = []
        for r in range(wl.num_requests):
            slots.append(self.alloc.add_seq(r * Wd, int(wl.prompt_lens[r])))
            for j in range(1, Wd):
                self.alloc.fork(r * Wd, r * Wd + j)
        sl = torch.from_numpy(np.concatenate(slots)).to(self.device)
        pa.pa_reshape_and_cache(pk.to(self.device).contiguous(), pv.to(self.device).contiguous(), self.k_cache,
                                self.v_cache, sl)
        self.copies_per_step = []
        self.host_us_per_step = []
        for t in range(T):
            t0 = time.perf_counter()
            st_slots, pairs = self.alloc.beam_step(ids, wl.parents[t], ids)
            self.host_us_per_step.append(1e6 * (time.perf_counter() - t0))
            self.copies_per_step.append(len(pairs))
            new_k = nk[t * S:(t + 1) * S].to(self.device).contiguous()
            new_v = nv[t * S:(t + 1) * S].to(self.device).contiguous()
            slot_mapping = torch.from_numpy(st_slots.copy()).to(self.device)
            cow_pairs = torch.from_numpy(pairs.copy()).to(self.device)
            if t < T - 1:
                if len(pairs):
                    pa.pa_copy_blocks(self.k_cache, self.v_cache, cow_pairs)
                pa.pa_reshape_and_cache(new_k, new_v, self.k_cache, self.v_cache, slot_mapping)
        self.new_k, self.new_v, self.slot_mapping, self.cow_pairs = new_k, new_v, slot_mapping, cow_pairs
        self.q = q.to(self.device).contiguous()
        tables, ctx = self.tables_now()
        self.context_lens_np = ctx
        self.block_tables = torch.from_numpy(tables).to(self.device)
        self.context_lens = torch.from_numpy(ctx).to(self.device)
        self.max_context_len = int(ctx.max()) if S else 0
        self.partition_size = wl.partition_size if partition_size is None else partition_size
        self.out = torch.empty_like(self.q)
        ws = pa.pa_decode_workspace_size(S, Hq, Hkv, D, B, self.max_context_len, self.partition_size)
        self.workspace = torch.empty(max(ws, 16) // 4 + 4, dtype=torch.float32, device=self.device)

    tables_now = DecodeBatch.tables_now
    append = DecodeBatch.append
    decode = DecodeBatch.decode
    workspace_for = DecodeBatch.workspace_for
    step = DecodeBatch.step
    decode_bytes = PrefixBatch.decode_bytes
    unique_kv_bytes = PrefixBatch.unique_kv_bytes

    def append_bytes(self):
        """The step's new rows (read and written) plus its whole-block copies."""
        wl = self.wl
        row = wl.num_kv_heads * wl.head_dim * 2
        return wl.num_seqs * (2 * row * 2 + 8) + int(self.cow_pairs.shape[0]) * 2 * (row * wl.block_size) * 2


class PrefillBatch:
    """Chunked prefill: every sequence's prefix and chunk placed by the allocator and
    written with pa_reshape_and_cache; the step is one pa_prefill_ws over all chunks."""

    def __init__(self, wl, device="cuda", values=None, fill=float("nan"), partition_size=None):
        self.wl = wl
        self.device = torch.device(device)
        S, Hq, Hkv, D, B, NB = (wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.block_size,
                                wl.num_blocks)
        dt = W.torch_dtype(wl.dtype)
        if values is None:
            values = W.prefill_values(wl, self.device)
        q, keys, vals = values
        self.k_cache = torch.full((NB, Hkv, B, D), fill, dtype=dt, device=self.device)
        self.v_cache = torch.full((NB, Hkv, B, D), fill, dtype=dt, device=self.device)
        self.alloc = pa.Allocator(NB, B, wl.free_order)
        L = wl.context_lens
        slots = np.concatenate([self.alloc.add_seq(s, int(L[s])) for s in range(S)])
        pa.pa_reshape_and_cache(keys.to(self.device).contiguous(), vals.to(self.device).contiguous(), self.k_cache,
                                self.v_cache, torch.from_numpy(slots).to(self.device))
        tables, ctx = DecodeBatch.tables_now(self)
        self.block_tables = torch.from_numpy(tables).to(self.device)
        self.context_lens = torch.from_numpy(ctx).to(self.device)
        qs = np.concatenate([[0], np.cumsum(wl.query_lens)]).astype(np.int32)
        self.q_start_np = qs
        self.q_start = torch.from_numpy(qs).to(self.device)
        self.max_query_len = int(wl.query_lens.max()) if S else 0
        self.q = q.to(self.device).contiguous()
        self.out = torch.empty_like(self.q)
        self.workspace = torch.empty(pa.pa_prefill_workspace_size(), dtype=torch.uint8, device=self.device)

    def step(self, stream=None):
        pa.pa_prefill(self.out, self.q, self.k_cache, self.v_cache, self.block_tables, self.context_lens,
                      self.q_start, self.max_query_len, self.wl.scale, stream=stream, workspace=self.workspace)
        return self.out


def make_batch(wl, device="cuda", values=None, fill=float("nan"), partition_size=None):
    if isinstance(wl, W.CowWorkload):
        cls = CowBatch
    elif isinstance(wl, W.PrefixWorkload):
        cls = PrefixBatch
    elif isinstance(wl, W.BeamWorkload):
        cls = BeamBatch
    elif isinstance(wl, W.PrefillWorkload):
        cls = PrefillBatch
    else:
        cls = DecodeBatch
    return cls(wl, device=device, values=values, fill=fill, partition_size=partition_size)


# ---- stepping a batch whose inputs live in host memory

STEP_INPUTS = ("q", "new_k", "new_v", "slot_mapping", "cow_pairs", "block_tables", "context_lens")


# ---------------------------------------------------------------- multi-GPU splits

def sequence_shard(num_seqs, world, rank):
    """Data-parallel split by sequence: this rank's contiguous range of a global
    batch's sequences (shard sizes differ by at most one).  Each rank keeps its own
    pools and allocator for its sequences; decode needs no exchange between ranks."""
    if world < 1 or not 0 <= rank < world or num_seqs < 0:
        raise ValueError("bad world, rank or num_seqs")
    base, extra = divmod(num_seqs, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def kv_head_shard(num_heads, num_kv_heads, world, rank):
    """Tensor-parallel split by kv head: this rank holds kv heads [k0, k1) of every
    block (pools [num_blocks, k1 - k0, B, D]) and computes the query heads that read
    them, [k0 * G, k1 * G) with G = num_heads / num_kv_heads.  A block table names
    whole blocks, whatever heads they hold, so every rank runs the same allocator
    script and holds the same tables (replicated host state, no device exchange); the
    output stays sharded by head.  Returns (query-head range, kv-head range)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world or rank")
    if num_kv_heads % world or num_heads % num_kv_heads:
        raise ValueError("num_kv_heads must divide by the world size, num_heads by num_kv_heads")
    per = num_kv_heads // world
    g = num_heads // num_kv_heads
    return range(rank * per * g, (rank + 1) * per * g), range(rank * per, (rank + 1) * per)


def pack_layout(tensors, align=256):
    """Byte layout of one step's inputs packed into a single buffer.

    `tensors` maps a name to a tensor (or None / empty, which is left out).  Each
    field starts on an `align`-byte boundary so that the typed views into the packed
    buffer are aligned for every kernel that reads them.  Returns (fields, nbytes):
    fields = [(name, offset, nbytes, dtype, shape)], nbytes = the end of the last
    field, i.e. the size of the one copy that moves them all.
    """
    fields, off, end = [], 0, 0
    for name, t in tensors.items():
        if t is None or t.numel() == 0:
            continue
        n = t.numel() * t.element_size()
        fields.append((name, off, n, t.dtype, tuple(t.shape)))
        end = off + n
        off = _round_up(end, align)
    return fields, end


class HostStepper:
    """Decode steps fed from pinned host memory and read back into it.

    Every step's inputs (q, the new K/V rows and their slots, copy-on-write pairs,
    block tables, context lengths) sit packed in one pinned host buffer and cross to
    the device in ONE copy; the step's output comes back in one copy.  `depth`
    input/output buffer pairs rotate on three streams, so that the upload of step
    k+1 and the read-back of step k-1 run on the copy engines while step k's
    kernels run: each step's own upload still precedes its kernels and its
    read-back follows them (events order them), and the host may refill a buffer
    only after its upload has finished (`host_inputs` waits for that).

    The kernels are the batch's: the copy-on-write copies, the slot-mapped append
    and paged decode attention, all on the compute stream, so steps run in order.
    With `graph=True` each buffer's kernel sequence is captured once as a CUDA graph
    and replayed, which takes the per-launch host work off every step; the captured
    launches have the batch's max_context_len and partition size fixed in them.
    """

    def __init__(self, batch, depth=2, stream=None, graph=False):
        if depth < 1:
            raise ValueError("depth must be >= 1")
        self.batch = batch
        self.depth = depth
        dev = batch.device
        self.stream = stream if stream is not None else torch.cuda.current_stream(dev)
        self.h2d_stream = torch.cuda.Stream(dev)
        self.d2h_stream = torch.cuda.Stream(dev)
        self.fields, self.h2d_bytes = pack_layout({n: getattr(batch, n, None) for n in STEP_INPUTS})
        self.d2h_bytes = batch.out.numel() * batch.out.element_size()
        self.host_in, self.dev_in, self.host_out, self.dev_out = [], [], [], []
        self.host_views, self.dev_views = [], []
        for _ in range(depth):
            h = torch.empty(max(self.h2d_bytes, 1), dtype=torch.uint8).pin_memory()
            d = torch.empty(max(self.h2d_bytes, 1), dtype=torch.uint8, device=dev)
            self.host_in.append(h)
            self.dev_in.append(d)
            self.host_views.append(self._views(h))
            self.dev_views.append(self._views(d))
            self.host_out.append(torch.empty(batch.out.shape, dtype=batch.out.dtype).pin_memory())
            self.dev_out.append(torch.empty_like(batch.out))
            for name, t in self.host_views[-1].items():
                t.copy_(getattr(batch, name))
        ev = lambda: [torch.cuda.Event() for _ in range(depth)]
        self.uploaded, self.computed, self.downloaded = ev(), ev(), ev()
        self.used = [False] * depth
        self.k = 0
        self.graphs = [None] * depth if graph else None

    def _views(self, buf):
        return {name: buf[off:off + n].view(dt).view(shape) for name, off, n, dt, shape in self.fields}

    def host_inputs(self, slot):
        """The pinned input views of buffer `slot`, once its last upload has finished."""
        if self.used[slot]:
            self.uploaded[slot].synchronize()
        return self.host_views[slot]

    def output(self, slot):
        """The pinned output of buffer `slot`, once its last read-back has finished."""
        self.downloaded[slot].synchronize()
        return self.host_out[slot]

    def submit(self, max_context_len=None):
        """Queue one step on buffer k % depth; returns that buffer's index."""
        b, i = self.batch, self.k % self.depth
        mcl = b.max_context_len if max_context_len is None else int(max_context_len)
        with torch.cuda.stream(self.h2d_stream):
            if self.used[i]:
                self.h2d_stream.wait_event(self.computed[i])
            self.dev_in[i].copy_(self.host_in[i], non_blocking=True)
            self.uploaded[i].record(self.h2d_stream)
        s = self.stream
        s.wait_event(self.uploaded[i])
        if self.used[i]:
            s.wait_event(self.downloaded[i])
        if self.graphs is None:
            self._kernels(i, mcl, s)
        else:
            if mcl != b.max_context_len:
                raise ValueError("a captured step has max_context_len %d fixed in it" % b.max_context_len)
            if self.graphs[i] is None:
                self.graphs[i] = self._capture(i, mcl)
            with torch.cuda.stream(s):
                self.graphs[i].replay()
        self.computed[i].record(s)
        with torch.cuda.stream(self.d2h_stream):
            self.d2h_stream.wait_event(self.computed[i])
            self.host_out[i].copy_(self.dev_out[i], non_blocking=True)
            self.downloaded[i].record(self.d2h_stream)
        self.used[i] = True
        self.k += 1
        return i

    def _kernels(self, i, mcl, s):
        b, v = self.batch, self.dev_views[i]
        if "cow_pairs" in v:
            pa.pa_copy_blocks(b.k_cache, b.v_cache, v["cow_pairs"], stream=s)
        pa.pa_reshape_and_cache(v["new_k"], v["new_v"], b.k_cache, b.v_cache, v["slot_mapping"], stream=s)
        pa.pa_decode(self.dev_out[i], v["q"], b.k_cache, b.v_cache, v["block_tables"], v["context_lens"], mcl,
                     b.wl.scale, b.partition_size, b.workspace_for(b.partition_size), stream=s)

    def _capture(self, i, mcl):
        b = self.batch
        b.workspace_for(b.partition_size)             # sized before capture: nothing allocates inside
        self.stream.synchronize()
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(b.device)
        with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
            self._kernels(i, mcl, cap)
        return g

    def drain(self):
        """Make the compute stream wait for every queued read-back."""
        for i in range(self.depth):
            if self.used[i]:
                self.stream.wait_event(self.downloaded[i])
