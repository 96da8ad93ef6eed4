"""Load a synthetic workload into the CPU oracle (test infrastructure only).

Builds an OracleCache for all or some (sequence, KV head) groups by appending
the generator's prefix, and appends the tokens of decode steps.
"""
import numpy as np

from workloads import gen

from . import spla_oracle as so


def params_of(w: gen.Workload, **kw) -> so.OracleParams:
    return so.OracleParams(num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads,
                           head_dim=w.head_dim, block_size=w.block_size, top_k=w.top_k,
                           n_sink=w.n_sink, n_local=w.n_local, **kw)


def build(w: gen.Workload, groups=None, **kw) -> so.OracleCache:
    """Oracle state after every sequence's prefix (one append per sequence)."""
    oc = so.OracleCache(params_of(w, **kw), w.batch, groups)
    seqs = sorted({b for (b, _) in oc.state})
    for b in seqs:
        heads = sorted(h for (bb, h) in oc.state if bb == b)
        K, V = gen.prefix_seq(w, b, kv_heads=heads)
        for i, h in enumerate(heads):
            oc.append_group(b, h, K[:, i], V[:, i])
    return oc


def append_step(oc: so.OracleCache, w: gen.Workload, step: int) -> None:
    k, v = gen.step_tokens(w, step)
    for (b, h) in oc.state:
        oc.append_group(b, h, k[b, h][None], v[b, h][None])
