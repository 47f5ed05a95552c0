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


def make_batch(wl, device="cuda", values=None, fill=float("nan"), partition_size=None):
    cls = CowBatch if isinstance(wl, W.CowWorkload) else DecodeBatch
    return cls(wl, device=device, values=values, fill=fill, partition_size=partition_size)
