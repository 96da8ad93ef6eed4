"""Context-sharded decode (spla_shard_candidates / _partials / _merge), the shards of
each sequence's blocks emulated as separate caches on one GPU.

Each shard holds a contiguous range of global blocks (its own pools, statistics and
linear-attention state over its own tokens); some sequences leave the last shards
empty. The sharded result is compared with the oracle, taking the unsharded GPU
decode's selection as the kept set (the sharded kept set must be the same set,
else o_sparse would not match), and with the unsharded GPU outputs themselves.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_linear_b200 import SplaDecodeCache
from block_sparse_linear_b200.sharded import decode_sharded
from oracle import feed as ofeed
from oracle import spla_oracle as so
from workloads import feed_gpu, gen

from . import parity
from .test_gpu_parity import compare_all

pytestmark = pytest.mark.gpu


def _shard_caches(w, oc, bps, nshards, cfg):
    """nshards caches; shard s holds global blocks [s*bps, (s+1)*bps) of every sequence."""
    bs, hkv, d = w.block_size, w.num_kv_heads, w.head_dim
    shards = []
    for s in range(nshards):
        table = torch.arange(w.batch * bps, dtype=torch.int32).reshape(w.batch, bps)
        cache = SplaDecodeCache(cfg, w.batch, table, w.batch * bps, device="cuda")
        lo = s * bps * bs
        counts = [max(0, min(int(L), lo + bps * bs) - lo) for L in w.context_lens]
        nmax = max(max(counts), 1)
        k = np.zeros((w.batch, nmax, hkv, d))
        v = np.zeros_like(k)
        for b in range(w.batch):
            for h in range(hkv):
                g = oc.state[(b, h)]
                n = counts[b]
                k[b, :n, h] = g.K[lo:lo + n]
                v[b, :n, h] = g.V[lo:lo + n]
        to = lambda a: torch.from_numpy(a).to(cfg.torch_dtype).cuda()
        cache.append(to(k), to(v), torch.tensor(counts, dtype=torch.int32, device="cuda"))
        shards.append((cache, s * bps))
    return shards


CASES = [
    # workload, lengths, shards, blocks per shard
    ("cfg2", (5000, 3100), 3, 27),            # sink + local blocks; sequence 1 leaves shard 2 empty
    ("cfg3", (9000, 4097), 4, 40),            # ragged tails
    ("cfg1", (4096,), 4, 20),                 # fp32, d = 64 (the FMA decode kernel)
    ("cfg5", (3000, 300, 6000, 64), 2, 60),   # paged workload's shape, tiny sequences
]


@pytest.mark.parametrize("name,lens,nshards,bps", CASES)
def test_sharded_decode_matches_oracle_and_unsharded(name, lens, nshards, bps):
    w = gen.scaled(name, context_lens=lens, extra_tokens=0)
    cfg = feed_gpu.config_of(w)
    assert nshards * bps >= max(-(-L // w.block_size) for L in lens)
    cache = feed_gpu.build_cache(w)
    oc = ofeed.build(w)
    shards = _shard_caches(w, oc, bps, nshards, cfg)
    q_np, gamma_np = gen.query(w, 0), gen.gamma(w)
    q = torch.from_numpy(q_np).to(cfg.torch_dtype).cuda()
    gamma = torch.from_numpy(gamma_np).float().cuda()
    out, sel, osp, orl = cache.new_outputs(debug=True)
    cache.decode(q, gamma, out, sel, osp, orl)
    gnb = torch.tensor([math.ceil(L / w.block_size) for L in lens], dtype=torch.int32,
                       device="cuda")
    out2, osp2, orl2 = torch.empty_like(out), torch.empty_like(osp), torch.empty_like(orl)
    decode_sharded(shards, q, gnb, gamma, out2, osp2, orl2)
    torch.cuda.synchronize()
    status = cache.status()
    for c, _ in shards:
        status |= c.status()
    res = {"out": out2.float().cpu().numpy(), "sel": sel.cpu().numpy(),
           "o_sparse": osp2.cpu().numpy(), "o_rla": orl2.cpu().numpy()}
    stats = compare_all(res, oc, q_np, gamma_np, w)
    s = parity.check_ill(name, stats, status)
    print(name, "sharded", s)
    # the same numbers as the unsharded decode, up to fp32 summation order
    np.testing.assert_allclose(osp2.cpu().numpy(), osp.cpu().numpy(), rtol=1e-4, atol=1e-5)
    ok = [(x["b"], x["hq"]) for x in stats if x["conditioned"]]
    r1, r2 = orl.cpu().numpy(), orl2.cpu().numpy()
    for b, hq in ok:
        np.testing.assert_allclose(r2[b, hq], r1[b, hq], rtol=1e-3, atol=1e-4)


def test_sharded_decode_keeps_every_block_when_few_remain():
    """top_k above every sequence's block count: every block kept, o_rla exactly zero."""
    w = gen.scaled("cfg3", context_lens=(900, 64 * 5), top_k=64, extra_tokens=0)
    cfg = feed_gpu.config_of(w)
    oc = ofeed.build(w)
    shards = _shard_caches(w, oc, 6, 3, cfg)
    q_np, gamma_np = gen.query(w, 0), gen.gamma(w)
    q = torch.from_numpy(q_np).to(cfg.torch_dtype).cuda()
    gnb = torch.tensor([math.ceil(L / w.block_size) for L in w.context_lens], dtype=torch.int32,
                       device="cuda")
    out = torch.empty_like(q)
    osp = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    orl = torch.empty_like(osp)
    decode_sharded(shards, q, gnb, torch.from_numpy(gamma_np).float().cuda(), out, osp, orl)
    torch.cuda.synchronize()
    assert np.all(orl.cpu().numpy() == 0)
    for b in range(w.batch):
        for hq in range(w.num_q_heads):
            g = oc.state[(b, hq // oc.p.group)]
            ref = so.decode_head(np.asarray(q_np[b, hq], np.float64), g, oc.p, gamma_np[hq])
            np.testing.assert_allclose(osp.cpu().numpy()[b, hq], ref["o_sparse"], atol=2e-2)
