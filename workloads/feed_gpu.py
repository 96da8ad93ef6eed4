"""Load a synthetic workload into the CUDA path: allocate the cache, prefill it
through spla_append_kv chunk by chunk, and drive decode steps.

Plumbing only (uploads and calls); all arithmetic happens in libspla.so.
"""
import numpy as np
import torch

from block_sparse_linear_b200 import SplaConfig, SplaDecodeCache

from . import gen


def config_of(w: gen.Workload, **kw) -> SplaConfig:
    return SplaConfig(num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads,
                      head_dim=w.head_dim, block_size=w.block_size, top_k=w.top_k,
                      n_sink=w.n_sink, n_local=w.n_local, dtype=w.dtype, **kw)


def _dt(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def build_cache(w: gen.Workload, device="cuda", cfg: SplaConfig = None) -> SplaDecodeCache:
    """Allocate the cache for w and append every sequence's prefix through the library."""
    cfg = cfg or config_of(w)
    table = torch.from_numpy(gen.block_table(w))
    cache = SplaDecodeCache(cfg, w.batch, table, w.num_phys_blocks, device=device)
    dt = _dt(w)
    ct = gen.CHUNK_TOKENS
    kbuf = torch.zeros((w.batch, ct, w.num_kv_heads, w.head_dim), dtype=dt, device=device)
    vbuf = torch.zeros_like(kbuf)
    n_new = torch.zeros((w.batch,), dtype=torch.int32, device=device)
    for c, chunk in gen.iter_prefix(w):
        hk = torch.zeros((w.batch, ct, w.num_kv_heads, w.head_dim), dtype=dt)
        hv = torch.zeros_like(hk)
        counts = np.zeros(w.batch, np.int32)
        for b, (K, V) in enumerate(chunk):
            n = K.shape[0]
            counts[b] = n
            if n:
                hk[b, :n] = torch.from_numpy(K).to(dt)
                hv[b, :n] = torch.from_numpy(V).to(dt)
        kbuf.copy_(hk, non_blocking=False)
        vbuf.copy_(hv, non_blocking=False)
        n_new.copy_(torch.from_numpy(counts))
        cache.append(kbuf, vbuf, n_new)
    torch.cuda.synchronize(device)
    return cache


def step_inputs(w: gen.Workload, step: int, device="cuda"):
    """Device tensors for decode step `step`: (k_new [batch][1][Hkv][d], v_new, q [batch][Hq][d])."""
    dt = _dt(w)
    k, v = gen.step_tokens(w, step)
    q = gen.query(w, step)
    to = lambda a: torch.from_numpy(a).to(dt).to(device)
    return to(k[:, None]), to(v[:, None]), to(q)
