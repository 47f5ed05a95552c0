"""Seeded synthetic inputs for the paged decode path.

This module only draws numbers: context lengths, a block-placement order and
N(0,1) tensor values.  It holds none of the method's arithmetic (no address
translation, no softmax), so both the CUDA path and the CPU oracle can consume
its output.  Nothing here needs a GPU.

The workloads mirror the serving scenario the PagedAttention pages describe
(many concurrent requests of different lengths sharing one block pool, and
parallel sampling with copy-on-write); no public dataset is involved.

  decode-tiny-f32     4 seqs, 4/4 heads, D=64,  B=16, fp32, L ~ U[1,100],  pool 64
  decode-mha-bf16     64 seqs, 32/32 heads (Llama-7B shaped), D=128, B=16, bf16,
                      L ~ U[128,2048], pool 20,000
  decode-gqa-bf16     128 seqs, 32 query / 8 kv heads, D=128, B=16, bf16,
                      L ~ round(lognormal(ln 500, 1.0)) clipped to [16,4096], pool 40,000
  cow-sampling-bf16   32 prompts U[256,1024] x 4 streams, + U[1,40] private tokens
                      per stream, 32/32 heads, D=128, B=16, bf16, pool 20,000
  long-splitk-bf16    8 seqs, 32/8 heads, D=128, B=32, bf16, L ~ U[16384,32768],
                      pool 12,000, context partitions of 512 tokens

For the decode workloads the drawn length L_s is the context of the decode step:
L_s - 1 tokens are the prefill and one token is appended by the step itself.
"""
from dataclasses import dataclass, field
import math

import numpy as np

WORKLOADS = {
    1: dict(name="decode-tiny-f32", num_seqs=4, num_heads=4, num_kv_heads=4, head_dim=64, block_size=16,
            dtype="f32", lens=("uniform", 1, 100), num_blocks=64, partition_size=0),
    2: dict(name="decode-mha-bf16", num_seqs=64, num_heads=32, num_kv_heads=32, head_dim=128, block_size=16,
            dtype="bf16", lens=("uniform", 128, 2048), num_blocks=20000, partition_size=0),
    3: dict(name="decode-gqa-bf16", num_seqs=128, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
            dtype="bf16", lens=("lognormal", 500.0, 1.0, 16, 4096), num_blocks=40000, partition_size=0),
    4: dict(name="cow-sampling-bf16", num_prompts=32, streams_per_prompt=4, num_heads=32, num_kv_heads=32,
            head_dim=128, block_size=16, dtype="bf16", prompt_lens=(256, 1024), private_tokens=(1, 40),
            num_blocks=20000, partition_size=0),
    5: dict(name="long-splitk-bf16", num_seqs=8, num_heads=32, num_kv_heads=8, head_dim=128, block_size=32,
            dtype="bf16", lens=("uniform", 16384, 32768), num_blocks=12000, partition_size=512),
    6: dict(name="prefix-cache-bf16", num_prompts=8, requests_per_prompt=16, num_heads=32, num_kv_heads=8,
            head_dim=128, block_size=16, dtype="bf16", stem_lens=(512, 1536), suffix_lens=(16, 256),
            vocab=32000, num_blocks=20000, partition_size=0),
    8: dict(name="prefill-chunk-bf16", num_seqs=16, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
            dtype="bf16", prefix_lens=(0, 2048), chunk=1024, num_blocks=20000, partition_size=0),
    7: dict(name="beam-search-bf16", num_requests=16, beam_width=4, num_heads=32, num_kv_heads=8, head_dim=128,
            block_size=16, dtype="bf16", prompt_lens=(256, 1024), beam_steps=24, num_blocks=20000,
            partition_size=0),
}

NAME_TO_ID = {v["name"]: k for k, v in WORKLOADS.items()}


@dataclass
class DecodeWorkload:
    """Shapes and seeded integer draws of one decode workload."""
    wid: int
    name: str
    seed: int
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str
    num_blocks: int
    partition_size: int
    context_lens: np.ndarray            # int32 [S], decode context after the step's append
    free_order: np.ndarray              # int32 [num_blocks], seeded permutation (block placement)
    scale: float = field(default=0.0)

    @property
    def max_context_len(self):
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def total_tokens(self):
        return int(self.context_lens.sum())


@dataclass
class CowWorkload:
    """Parallel sampling: prompts forked into streams that then append private tokens."""
    wid: int
    name: str
    seed: int
    num_prompts: int
    streams_per_prompt: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str
    num_blocks: int
    partition_size: int
    prompt_lens: np.ndarray             # int32 [P]
    private_tokens: np.ndarray          # int32 [P * n], stream p*n + j
    free_order: np.ndarray              # int32 [num_blocks]
    scale: float = field(default=0.0)

    @property
    def num_seqs(self):
        return self.num_prompts * self.streams_per_prompt


@dataclass
class PrefixWorkload:
    """Requests that share system prompts: request r = stem[r % P] + its own suffix.
    Token ids are seeded; the allocator's prefix cache shares the stems' full blocks."""
    wid: int
    name: str
    seed: int
    num_prompts: int
    requests_per_prompt: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str
    num_blocks: int
    partition_size: int
    stem_lens: np.ndarray               # int32 [P]
    suffix_lens: np.ndarray             # int32 [S]
    stem_tokens: list                   # P lists of token ids
    suffix_tokens: list                 # S lists of token ids
    free_order: np.ndarray              # int32 [num_blocks]
    scale: float = field(default=0.0)

    @property
    def num_seqs(self):
        return self.num_prompts * self.requests_per_prompt

    def prompt_of(self, r):
        return r % self.num_prompts

    def tokens(self, r):
        """Token ids of request r (its decode step appends the last one)."""
        return self.stem_tokens[self.prompt_of(r)] + self.suffix_tokens[r]

    @property
    def context_lens(self):
        return np.array([int(self.stem_lens[self.prompt_of(r)]) + int(self.suffix_lens[r])
                         for r in range(self.num_seqs)], np.int32)


@dataclass
class BeamWorkload:
    """Beam search: each request's prompt is forked into beam_width beams; every step,
    new beam j of a request continues a seeded choice of that request's beams (with
    repeats, so beams die and others split) and appends one token."""
    wid: int
    name: str
    seed: int
    num_requests: int
    beam_width: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str
    num_blocks: int
    partition_size: int
    prompt_lens: np.ndarray             # int32 [R]
    parents: np.ndarray                 # int32 [steps, R * W]: index into the old beams (same request)
    free_order: np.ndarray              # int32 [num_blocks]
    scale: float = field(default=0.0)

    @property
    def num_seqs(self):
        return self.num_requests * self.beam_width

    @property
    def beam_steps(self):
        return int(self.parents.shape[0])

    @property
    def context_lens(self):
        return np.repeat(self.prompt_lens, self.beam_width) + self.beam_steps


@dataclass
class PrefillWorkload:
    """Chunked prefill: sequence s already holds prefix_lens[s] tokens and appends a
    chunk of `chunk` tokens, which are its queries (causal over prefix + chunk)."""
    wid: int
    name: str
    seed: int
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str
    num_blocks: int
    partition_size: int
    prefix_lens: np.ndarray             # int32 [S]
    query_lens: np.ndarray              # int32 [S]
    free_order: np.ndarray
    scale: float = field(default=0.0)

    @property
    def context_lens(self):
        return (self.prefix_lens + self.query_lens).astype(np.int32)

    def flops(self):
        """Causal attention FLOPs: 4 * D per (query, visible key, query head)."""
        tot = 0
        for P, n in zip(self.prefix_lens, self.query_lens):
            keys = int(n) * int(P) + int(n) * (int(n) + 1) // 2
            tot += 4 * self.head_dim * self.num_heads * keys
        return tot


def _rng(seed, salt):
    return np.random.default_rng([int(seed), int(salt)])


def _draw_lengths(spec, n, rng):
    kind = spec[0]
    if kind == "uniform":
        lo, hi = spec[1], spec[2]
        return rng.integers(lo, hi + 1, size=n).astype(np.int32)
    if kind == "lognormal":
        median, sigma, lo, hi = spec[1], spec[2], spec[3], spec[4]
        x = rng.lognormal(mean=math.log(median), sigma=sigma, size=n)
        return np.clip(np.rint(x), lo, hi).astype(np.int32)
    raise ValueError(kind)


def make_workload(wid, seed=0, **overrides):
    """Seeded workload `wid` (1..5); keyword overrides change shapes for small cases."""
    spec = dict(WORKLOADS[wid])
    spec.update(overrides)
    rng = _rng(seed, wid)
    if wid == 4:
        P, n = spec["num_prompts"], spec["streams_per_prompt"]
        plo, phi = spec["prompt_lens"]
        qlo, qhi = spec["private_tokens"]
        prompt_lens = rng.integers(plo, phi + 1, size=P).astype(np.int32)
        private = rng.integers(qlo, qhi + 1, size=P * n).astype(np.int32)
        free_order = rng.permutation(spec["num_blocks"]).astype(np.int32)
        wl = CowWorkload(wid=wid, name=spec["name"], seed=seed, num_prompts=P, streams_per_prompt=n,
                         num_heads=spec["num_heads"], num_kv_heads=spec["num_kv_heads"],
                         head_dim=spec["head_dim"], block_size=spec["block_size"], dtype=spec["dtype"],
                         num_blocks=spec["num_blocks"], partition_size=spec["partition_size"],
                         prompt_lens=prompt_lens, private_tokens=private, free_order=free_order)
    elif wid == 8:
        S = spec["num_seqs"]
        plo, phi = spec["prefix_lens"]
        prefix = rng.integers(plo, phi + 1, size=S).astype(np.int32)
        qlen = np.full(S, spec["chunk"], np.int32) if "query_lens" not in spec else np.asarray(spec["query_lens"],
                                                                                             np.int32)
        free_order = rng.permutation(spec["num_blocks"]).astype(np.int32)
        wl = PrefillWorkload(wid=wid, name=spec["name"], seed=seed, num_seqs=S, num_heads=spec["num_heads"],
                             num_kv_heads=spec["num_kv_heads"], head_dim=spec["head_dim"],
                             block_size=spec["block_size"], dtype=spec["dtype"], num_blocks=spec["num_blocks"],
                             partition_size=spec["partition_size"], prefix_lens=prefix, query_lens=qlen,
                             free_order=free_order)
    elif wid == 7:
        R, Wd, T = spec["num_requests"], spec["beam_width"], spec["beam_steps"]
        plo, phi = spec["prompt_lens"]
        prompt_lens = rng.integers(plo, phi + 1, size=R).astype(np.int32)
        choice = rng.integers(0, Wd, size=(T, R, Wd))
        parents = (np.arange(R)[None, :, None] * Wd + choice).reshape(T, R * Wd).astype(np.int32)
        free_order = rng.permutation(spec["num_blocks"]).astype(np.int32)
        wl = BeamWorkload(wid=wid, name=spec["name"], seed=seed, num_requests=R, beam_width=Wd,
                          num_heads=spec["num_heads"], num_kv_heads=spec["num_kv_heads"], head_dim=spec["head_dim"],
                          block_size=spec["block_size"], dtype=spec["dtype"], num_blocks=spec["num_blocks"],
                          partition_size=spec["partition_size"], prompt_lens=prompt_lens, parents=parents,
                          free_order=free_order)
    elif wid == 6:
        P, n = spec["num_prompts"], spec["requests_per_prompt"]
        slo, shi = spec["stem_lens"]
        xlo, xhi = spec["suffix_lens"]
        stem_lens = rng.integers(slo, shi + 1, size=P).astype(np.int32)
        suffix_lens = rng.integers(xlo, xhi + 1, size=P * n).astype(np.int32)
        stems = [rng.integers(0, spec["vocab"], size=int(L)).tolist() for L in stem_lens]
        suffixes = [rng.integers(0, spec["vocab"], size=int(L)).tolist() for L in suffix_lens]
        free_order = rng.permutation(spec["num_blocks"]).astype(np.int32)
        wl = PrefixWorkload(wid=wid, name=spec["name"], seed=seed, num_prompts=P, requests_per_prompt=n,
                            num_heads=spec["num_heads"], num_kv_heads=spec["num_kv_heads"],
                            head_dim=spec["head_dim"], block_size=spec["block_size"], dtype=spec["dtype"],
                            num_blocks=spec["num_blocks"], partition_size=spec["partition_size"],
                            stem_lens=stem_lens, suffix_lens=suffix_lens, stem_tokens=stems, suffix_tokens=suffixes,
                            free_order=free_order)
    else:
        lens = spec.pop("context_lens", None)
        if lens is None:
            lens = _draw_lengths(spec["lens"], spec["num_seqs"], rng)
        else:
            lens = np.asarray(lens, np.int32)
            spec["num_seqs"] = len(lens)
        free_order = rng.permutation(spec["num_blocks"]).astype(np.int32)
        wl = DecodeWorkload(wid=wid, name=spec["name"], seed=seed, num_seqs=spec["num_seqs"],
                            num_heads=spec["num_heads"], num_kv_heads=spec["num_kv_heads"],
                            head_dim=spec["head_dim"], block_size=spec["block_size"], dtype=spec["dtype"],
                            num_blocks=spec["num_blocks"], partition_size=spec["partition_size"],
                            context_lens=lens, free_order=free_order)
    wl.scale = 1.0 / math.sqrt(wl.head_dim)
    return wl


def torch_dtype(name):
    import torch
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def normal(shape, dtype, device, seed, salt):
    """N(0,1) fp32 values from a seeded torch generator on `device`, cast once to `dtype`.
    CPU and CUDA generators give different streams: tests that need the same values
    on both sides draw on the CPU and copy."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + int(salt) * 7919) % (2 ** 63))
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return x.to(torch_dtype(dtype)) if isinstance(dtype, str) else x.to(dtype)


def decode_values(wl, device="cpu"):
    """q [S, Hq, D] and the K/V rows of every context token, packed per sequence:
    keys/values [sum L_s, Hkv, D]; token i of sequence s is row offsets[s] + i.
    The last row of each sequence is the token its decode step appends."""
    S, Hq, Hkv, D = wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim
    total = wl.total_tokens
    q = normal((S, Hq, D), wl.dtype, device, wl.seed, 1)
    keys = normal((total, Hkv, D), wl.dtype, device, wl.seed, 2)
    values = normal((total, Hkv, D), wl.dtype, device, wl.seed, 3)
    offsets = np.zeros(S + 1, np.int64)
    offsets[1:] = np.cumsum(wl.context_lens)
    return q, keys, values, offsets


def cow_values(wl, device="cpu"):
    """q per stream [P*n, Hq, D]; prompt K/V rows [sum L_p, Hkv, D] with offsets;
    private K/V rows [sum private, Hkv, D] with offsets (stream order)."""
    Hq, Hkv, D = wl.num_heads, wl.num_kv_heads, wl.head_dim
    q = normal((wl.num_seqs, Hq, D), wl.dtype, device, wl.seed, 1)
    pk = normal((int(wl.prompt_lens.sum()), Hkv, D), wl.dtype, device, wl.seed, 2)
    pv = normal((int(wl.prompt_lens.sum()), Hkv, D), wl.dtype, device, wl.seed, 3)
    xk = normal((int(wl.private_tokens.sum()), Hkv, D), wl.dtype, device, wl.seed, 4)
    xv = normal((int(wl.private_tokens.sum()), Hkv, D), wl.dtype, device, wl.seed, 5)
    poff = np.zeros(wl.num_prompts + 1, np.int64)
    poff[1:] = np.cumsum(wl.prompt_lens)
    xoff = np.zeros(wl.num_seqs + 1, np.int64)
    xoff[1:] = np.cumsum(wl.private_tokens)
    return q, pk, pv, poff, xk, xv, xoff


def prefix_values(wl, device="cpu"):
    """q [S, Hq, D]; stem K/V rows [sum stem_lens, Hkv, D] with offsets (a stem token's
    K/V are the same for every request that shares the stem: they depend only on the
    prefix up to that token); suffix K/V rows [sum suffix_lens, Hkv, D] with offsets."""
    Hq, Hkv, D = wl.num_heads, wl.num_kv_heads, wl.head_dim
    q = normal((wl.num_seqs, Hq, D), wl.dtype, device, wl.seed, 1)
    sk = normal((int(wl.stem_lens.sum()), Hkv, D), wl.dtype, device, wl.seed, 2)
    sv = normal((int(wl.stem_lens.sum()), Hkv, D), wl.dtype, device, wl.seed, 3)
    xk = normal((int(wl.suffix_lens.sum()), Hkv, D), wl.dtype, device, wl.seed, 4)
    xv = normal((int(wl.suffix_lens.sum()), Hkv, D), wl.dtype, device, wl.seed, 5)
    soff = np.zeros(wl.num_prompts + 1, np.int64)
    soff[1:] = np.cumsum(wl.stem_lens)
    xoff = np.zeros(wl.num_seqs + 1, np.int64)
    xoff[1:] = np.cumsum(wl.suffix_lens)
    return q, sk, sv, soff, xk, xv, xoff


def prefill_values(wl, device="cpu"):
    """q rows of every chunk [sum query_lens, Hq, D] (packed by sequence) and the K/V
    rows of every context token [sum context_lens, Hkv, D] (packed by sequence)."""
    Hq, Hkv, D = wl.num_heads, wl.num_kv_heads, wl.head_dim
    total = int(wl.context_lens.sum())
    q = normal((int(wl.query_lens.sum()), Hq, D), wl.dtype, device, wl.seed, 1)
    keys = normal((total, Hkv, D), wl.dtype, device, wl.seed, 2)
    vals = normal((total, Hkv, D), wl.dtype, device, wl.seed, 3)
    return q, keys, vals


def beam_values(wl, device="cpu"):
    """q [S, Hq, D]; prompt K/V rows [sum prompt_lens, Hkv, D] with offsets; the K/V of
    the token beam j appends at step t: rows [t * S + j] of new K/V [steps * S, Hkv, D]."""
    Hq, Hkv, D, S = wl.num_heads, wl.num_kv_heads, wl.head_dim, wl.num_seqs
    q = normal((S, Hq, D), wl.dtype, device, wl.seed, 1)
    pk = normal((int(wl.prompt_lens.sum()), Hkv, D), wl.dtype, device, wl.seed, 2)
    pv = normal((int(wl.prompt_lens.sum()), Hkv, D), wl.dtype, device, wl.seed, 3)
    nk = normal((wl.beam_steps * S, Hkv, D), wl.dtype, device, wl.seed, 4)
    nv = normal((wl.beam_steps * S, Hkv, D), wl.dtype, device, wl.seed, 5)
    poff = np.zeros(wl.num_requests + 1, np.int64)
    poff[1:] = np.cumsum(wl.prompt_lens)
    return q, pk, pv, poff, nk, nv


def beam_histories(wl, poff):
    """Per final beam, the (source, row) of every token it holds: source 0 = prompt rows,
    1 = new-token rows.  Follows the parent choices step by step."""
    W, S = wl.beam_width, wl.num_seqs
    hist = [[(0, int(poff[b // W]) + i) for i in range(int(wl.prompt_lens[b // W]))] for b in range(S)]
    for t in range(wl.beam_steps):
        hist = [hist[int(wl.parents[t, j])] + [(1, t * S + j)] for j in range(S)]
    return hist


def prefix_logical_rows(wl, r, soff, xoff):
    """(source, row) of every token of request r: source 0 = stem rows, 1 = suffix rows."""
    p = wl.prompt_of(r)
    stem = [(0, int(soff[p]) + i) for i in range(int(wl.stem_lens[p]))]
    return stem + [(1, int(xoff[r]) + i) for i in range(int(wl.suffix_lens[r]))]


def direct_block_tables(wl):
    """Block tables drawn straight from the placement order, without the allocator:
    sequence s takes the next ceil(L_s/B) entries of free_order.  Entries past a
    sequence's blocks are filled with -1 (never read by a correct kernel)."""
    B = wl.block_size
    nblk = [(int(L) + B - 1) // B for L in wl.context_lens]
    mb = max(1, max(nblk) if nblk else 1)
    if sum(nblk) > wl.num_blocks:
        raise ValueError("pool too small")
    tables = np.full((wl.num_seqs, mb), -1, np.int32)
    pos = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = wl.free_order[pos:pos + n]
        pos += n
    return tables
