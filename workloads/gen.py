"""Seeded synthetic decode workloads for the SPLA decode path.

This module only draws random inputs (queries, keys, values, block tables,
sequence lengths). It holds none of the method's arithmetic: no scores, no
statistics, no attention. Both the CPU oracle (through the tests and the
benchmark's CPU leg) and the CUDA path consume exactly the values produced
here, so the two sides see bit-identical inputs.

The workloads stand in for the long-context decode setting of
"SPLA: Block Sparse Plus Linear Attention for Long Context Modeling"
(gist.science technical summary, section 1 "Problem Statement" and section 4,
RULER up to 256k tokens). No benchmark items are used.

Recipe (every draw comes from NumPy's PCG64, keyed by the workload seed and a
spawn key naming what is drawn, so any part can be regenerated on its own):

* query of decode step s:      N(0, 1), shape [batch][Hq][d]            key ("q", s)
* per-block offsets of seq b:  one vector per (block, K|V, KV head)     key ("off", b)
    - "normal":    N(0, 0.5^2) per element
    - "student_t": 0.5 * t(3 dof) per element (heavy tails)
    - "none":      zero
* token noise, prefix chunk c of seq b: N(0, 1) for K and V             key ("kv", b, c)
* token noise of decode step s (one token per sequence):                 key ("step", s)
* K = noise + key offset of the token's block (+ 2*u if the block is planted)
  V = noise + value offset of the token's block
  u = normalise(sum of the step's query heads in the KV head's group)
* planted blocks of the prefix: a fixed count per (seq, KV head), drawn
  without replacement                                                    key ("plant", b)
  a block first opened by decode step s is planted with probability 1 %  key ("plant_new", b, block)
  and uses u of step s.
* ragged lengths: floor(exp(U[ln lo, ln hi])) per sequence               key ("lens",)
* paged block table: a random permutation of the physical pool           key ("table",)

For bf16 workloads every value is rounded to bf16 (round to nearest even)
before anyone sees it; it is returned as float32 holding bf16-exact values.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np
import torch

# Token chunk used for prefix generation: a multiple of every block size.
CHUNK_TOKENS = 8192

_TAGS = {"q": 1, "off": 2, "kv": 3, "step": 4, "plant": 5, "plant_new": 6,
         "lens": 7, "table": 8, "gamma": 9}


@dataclass(frozen=True)
class Workload:
    """One synthetic decode workload (shapes, distributions, selection knobs)."""
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    context_lens: tuple          # prefix length per sequence
    top_k: int
    n_sink: int = 0
    n_local: int = 0
    dtype: str = "bf16"          # "f32" or "bf16": dtype of q, K, V, out
    offset_kind: str = "none"    # "none" | "normal" | "student_t"
    offset_scale: float = 0.5
    plant_count: int = -1        # planted blocks per (seq, KV head); -1 => round(1 % of blocks)
    plant_new_prob: float = 0.0  # planting probability for blocks opened by decode steps
    paged: bool = False          # random physical block order
    decode_steps: int = 1        # decode steps the workload names (each preceded by one append)
    extra_tokens: int = 1024     # capacity reserved past the prefix for appended tokens
    seed: int = 1
    ragged: tuple = ()           # (lo, hi) for log-uniform lengths; empty when fixed

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def n_blocks(self, length: int) -> int:
        return -(-length // self.block_size)

    def seq_capacity(self, b: int) -> int:
        """Blocks reserved for sequence b (its prefix plus room for appended tokens)."""
        return self.n_blocks(self.context_lens[b] + self.extra_tokens)

    @property
    def capacity_blocks(self) -> int:
        """Width of the block table: the largest per-sequence reservation."""
        return max(self.seq_capacity(b) for b in range(self.batch))

    @property
    def num_phys_blocks(self) -> int:
        return sum(self.seq_capacity(b) for b in range(self.batch))

    def planted_count(self, n_blocks: int) -> int:
        if self.plant_count >= 0:
            return min(self.plant_count, n_blocks)
        return int(round(0.01 * n_blocks))


def _ragged_lens(seed: int, n: int, lo: int, hi: int) -> tuple:
    r = _rng(seed, "lens")
    x = r.uniform(math.log(lo), math.log(hi), size=n)
    return tuple(int(math.floor(math.exp(v))) for v in x)


def _base_configs() -> dict:
    c = {}
    c["cfg1"] = Workload(name="cfg1", batch=1, num_q_heads=4, num_kv_heads=1, head_dim=64,
                         block_size=64, context_lens=(4096,), top_k=8, dtype="f32",
                         offset_kind="none", plant_count=3, seed=1)
    c["cfg2"] = Workload(name="cfg2", batch=8, num_q_heads=32, num_kv_heads=8, head_dim=128,
                         block_size=64, context_lens=(32768,) * 8, top_k=16, n_sink=1, n_local=1,
                         offset_kind="normal", seed=2)
    c["cfg3"] = Workload(name="cfg3", batch=4, num_q_heads=32, num_kv_heads=8, head_dim=128,
                         block_size=64, context_lens=(131072,) * 4, top_k=32,
                         offset_kind="normal", plant_new_prob=0.01, decode_steps=64, seed=3)
    c["cfg4"] = Workload(name="cfg4", batch=1, num_q_heads=32, num_kv_heads=8, head_dim=128,
                         block_size=128, context_lens=(1048576,), top_k=64,
                         offset_kind="student_t", plant_count=0, seed=4)
    c["cfg5"] = Workload(name="cfg5", batch=16, num_q_heads=32, num_kv_heads=8, head_dim=128,
                         block_size=64, context_lens=_ragged_lens(5, 16, 4096, 262144), top_k=32,
                         offset_kind="normal", paged=True, seed=5, ragged=(4096, 262144))
    return c


DESCRIPTIONS = {
    "cfg1": "decode fp32, batch 1, 4 q / 1 kv heads, d 64, 4096 tokens, block 64, top-k 8, 3 planted blocks",
    "cfg2": "decode bf16, batch 8, 32 q / 8 kv heads, d 128, 32768 tokens, block 64, top-k 16 + 1 sink + 1 local",
    "cfg3": "decode bf16, batch 4, 32 q / 8 kv heads, d 128, 131072 tokens, block 64, top-k 32, append+decode per step",
    "cfg4": "decode bf16, batch 1, 32 q / 8 kv heads, d 128, 1048576 tokens, block 128, top-k 64, Student-t offsets",
    "cfg5": "ragged paged decode bf16, 16 seqs log-uniform 4096..262144 tokens, 32 q / 8 kv heads, d 128, block 64, top-k 32",
}


CONFIGS: dict = {}


def get(name: str, **overrides) -> Workload:
    """A named workload, optionally with fields replaced (e.g. shorter contexts)."""
    w = CONFIGS[name]
    if overrides:
        w = replace(w, **overrides)
    return w


def scaled(base: str, context_lens, **overrides) -> Workload:
    """The named workload's structure (heads, d, block, top-k, distributions) at other lengths."""
    lens = tuple(int(x) for x in context_lens)
    overrides.setdefault("name", f"{base}-small")
    return replace(CONFIGS[base], context_lens=lens, batch=len(lens), **overrides)


# --------------------------------------------------------------------------- rng helpers
def _rng(seed: int, tag: str, *ids) -> np.random.Generator:
    ss = np.random.SeedSequence(entropy=seed, spawn_key=(_TAGS[tag],) + tuple(int(i) for i in ids))
    return np.random.Generator(np.random.PCG64(ss))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def _finish(w: Workload, x: np.ndarray) -> np.ndarray:
    x = x.astype(np.float32, copy=False)
    return round_bf16(x) if w.dtype == "bf16" else x


_POOL = None


def _pool() -> ThreadPoolExecutor:
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1))
    return _POOL


# --------------------------------------------------------------------------- queries
def query(w: Workload, step: int = 0) -> np.ndarray:
    """Decode-step query, [batch][Hq][d] float32 (bf16-exact for bf16 workloads)."""
    q = _rng(w.seed, "q", step).standard_normal((w.batch, w.num_q_heads, w.head_dim),
                                                 dtype=np.float32)
    return _finish(w, q)


def gamma(w: Workload, kind: str = "ones") -> np.ndarray:
    """RMSNorm scale [Hq][d]: ones (no trained weights exist) or a seeded random one for tests."""
    if kind == "ones":
        return np.ones((w.num_q_heads, w.head_dim), np.float32)
    return (1.0 + 0.5 * _rng(w.seed, "gamma").standard_normal(
        (w.num_q_heads, w.head_dim))).astype(np.float32)


def _plant_dir(w: Workload, step: int) -> np.ndarray:
    """u = normalise(sum of the group's query heads), [batch][Hkv][d] float64."""
    q = query(w, step).astype(np.float64).reshape(w.batch, w.num_kv_heads, w.group, w.head_dim)
    s = q.sum(axis=2)
    n = np.linalg.norm(s, axis=-1, keepdims=True)
    return s / np.where(n > 0, n, 1.0)


# --------------------------------------------------------------------------- per-sequence structure
class SeqPlan:
    """Offsets and planted blocks of one sequence (cached per workload and sequence)."""

    def __init__(self, w: Workload, b: int):
        self.w = w
        self.b = b
        cap = w.capacity_blocks
        r = _rng(w.seed, "off", b)
        shape = (cap, 2, w.num_kv_heads, w.head_dim)
        if w.offset_kind == "normal":
            off = w.offset_scale * r.standard_normal(shape)
        elif w.offset_kind == "student_t":
            off = w.offset_scale * r.standard_t(3, size=shape)
        else:
            off = np.zeros(shape)
        self.offsets = off.astype(np.float32)           # [cap][K|V][Hkv][d]
        L = w.context_lens[b]
        nb = w.n_blocks(L)
        npl = w.planted_count(nb)
        rp = _rng(w.seed, "plant", b)
        self.planted = np.zeros((cap, w.num_kv_heads), bool)
        for h in range(w.num_kv_heads):
            if npl > 0:
                self.planted[rp.choice(nb, size=npl, replace=False), h] = True
        # blocks opened by decode steps: planted with probability plant_new_prob
        for j in range(nb, cap):
            if w.plant_new_prob > 0:
                rr = _rng(w.seed, "plant_new", b, j)
                self.planted[j, :] = rr.uniform(size=w.num_kv_heads) < w.plant_new_prob
        self.prefix_u = _plant_dir(w, 0)[b].astype(np.float32)       # [Hkv][d]

    def block_u(self, j: int) -> np.ndarray:
        """Planting direction for block j: step 0 for prefix blocks, else the opening step."""
        L = self.w.context_lens[self.b]
        if j * self.w.block_size < L:
            return self.prefix_u
        step = j * self.w.block_size - L
        return _plant_dir(self.w, step)[self.b].astype(np.float32)


_PLANS: dict = {}


def plan(w: Workload, b: int) -> SeqPlan:
    key = (w, b)
    if key not in _PLANS:
        if len(_PLANS) > 64:
            _PLANS.clear()
        _PLANS[key] = SeqPlan(w, b)
    return _PLANS[key]


def _tokens(w: Workload, b: int, pos0: int, noise: np.ndarray) -> tuple:
    """Add block offsets and planting to noise [2][n][Hkv][d] for positions pos0.."""
    p = plan(w, b)
    n = noise.shape[1]
    pos = pos0 + np.arange(n)
    blk = pos // w.block_size
    K = noise[0] + p.offsets[blk, 0]
    V = noise[1] + p.offsets[blk, 1]
    for j in np.unique(blk):
        pl = p.planted[j]
        if pl.any():
            sel = blk == j
            u = p.block_u(int(j))                      # [Hkv][d]
            K[sel] += (2.0 * u * pl[:, None]).astype(np.float32)[None]
    return _finish(w, K), _finish(w, V)


def prefix_chunk(w: Workload, b: int, c: int) -> tuple:
    """Prefix tokens [c*CHUNK, min(L_b, (c+1)*CHUNK)) of sequence b: (K, V) [n][Hkv][d]."""
    L = w.context_lens[b]
    t0 = c * CHUNK_TOKENS
    n = max(0, min(L, t0 + CHUNK_TOKENS) - t0)
    noise = _rng(w.seed, "kv", b, c).standard_normal((2, n, w.num_kv_heads, w.head_dim),
                                                      dtype=np.float32)
    return _tokens(w, b, t0, noise)


def n_prefix_chunks(w: Workload) -> int:
    return max(-(-L // CHUNK_TOKENS) for L in w.context_lens)


def prefix_chunks(w: Workload, c: int) -> list:
    """Chunk c of every sequence, generated in parallel: list of (K, V) per sequence."""
    return list(_pool().map(lambda b: prefix_chunk(w, b, c), range(w.batch)))


def iter_prefix(w: Workload, lookahead: int = 4):
    """Yield (c, [(K, V) per sequence]) for every prefix chunk in order, generating ahead."""
    pool = _pool()
    nc = n_prefix_chunks(w)
    futs = {}

    def submit(c):
        futs[c] = [pool.submit(prefix_chunk, w, b, c) for b in range(w.batch)]

    for c in range(min(lookahead, nc)):
        submit(c)
    for c in range(nc):
        out = [f.result() for f in futs.pop(c)]
        if c + lookahead < nc:
            submit(c + lookahead)
        yield c, out


def prefix_seq(w: Workload, b: int, kv_heads=None) -> tuple:
    """Whole prefix of sequence b as (K, V) [L][Hkv'][d], optionally only some KV heads."""
    nc = -(-w.context_lens[b] // CHUNK_TOKENS)
    parts = list(_pool().map(lambda c: prefix_chunk(w, b, c), range(nc)))
    if kv_heads is not None:
        parts = [(K[:, kv_heads], V[:, kv_heads]) for K, V in parts]
    if not parts:
        shape = (0, w.num_kv_heads if kv_heads is None else len(kv_heads), w.head_dim)
        return np.zeros(shape, np.float32), np.zeros(shape, np.float32)
    return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts])


def step_tokens(w: Workload, step: int) -> tuple:
    """The token each sequence appends before decode step `step`: (k, v) [batch][Hkv][d]."""
    noise = _rng(w.seed, "step", step).standard_normal(
        (2, w.batch, w.num_kv_heads, w.head_dim), dtype=np.float32)
    ks, vs = [], []
    for b in range(w.batch):
        K, V = _tokens(w, b, w.context_lens[b] + step, noise[:, b:b + 1])
        ks.append(K[0])
        vs.append(V[0])
    return np.stack(ks), np.stack(vs)


# --------------------------------------------------------------------------- paging
def block_table(w: Workload) -> np.ndarray:
    """Logical -> physical block map, int32 [batch][capacity_blocks].

    Sequence b owns seq_capacity(b) physical blocks; entries past that are -1.
    """
    cap = w.capacity_blocks
    total = w.num_phys_blocks
    phys = np.arange(total, dtype=np.int32)
    if w.paged:
        phys = _rng(w.seed, "table").permutation(total).astype(np.int32)
    table = np.full((w.batch, cap), -1, np.int32)
    base = 0
    for b in range(w.batch):
        n = w.seq_capacity(b)
        table[b, :n] = phys[base:base + n]
        base += n
    return table


CONFIGS.update(_base_configs())
