"""Bulk append on the tensor cores (spla_append_kv_bulk) against the oracle's append.

The oracle's append (fp64) is the definition of the state update; the
one-token-at-a-time kernel path (spla_append_kv) is a second, independent GPU
route to the same numbers. Chunks are ragged per sequence (0, 1, 63, 64, 65 and
several thousand tokens, so splits end mid-tile and sequences have no tokens at
all), later chunks raise the running maximum (the old state is rescaled), and the
input rows past each sequence's count hold NaN, which must never reach the state.
"""
import numpy as np
import pytest
import torch

from block_sparse_linear_b200 import SplaConfig, SplaDecodeCache
from oracle import spla_oracle as so

pytestmark = pytest.mark.gpu

D = 128
B = 64


def _cache(batch, hkv, mbp, dtype="bf16", d=D):
    cfg = SplaConfig(num_q_heads=4 * hkv, num_kv_heads=hkv, head_dim=d, block_size=B, top_k=4,
                     dtype=dtype)
    table = torch.arange(batch * mbp, dtype=torch.int32).reshape(batch, mbp)
    return SplaDecodeCache(cfg, batch, table, batch * mbp, device="cuda")


def _chunk(rng, counts, hkv, shift, scale):
    """bf16 K, V [batch][max_new][Hkv][d] with NaN past each count, and their fp64 values."""
    batch, max_new = len(counts), max(max(counts), 1)
    k = rng.standard_normal((batch, max_new, hkv, D)) * scale + shift
    v = rng.standard_normal((batch, max_new, hkv, D))
    kt = torch.from_numpy(k).to(torch.bfloat16)
    vt = torch.from_numpy(v).to(torch.bfloat16)
    for b, n in enumerate(counts):
        kt[b, n:] = float("nan")
        vt[b, n:] = float("nan")
    return kt, vt, kt.double().numpy(), vt.double().numpy()


# (counts per sequence) for successive calls; one key shift per call raises the max
PLAN = [((0, 1, 700, 4100), 0.0, 1.0),
        ((130, 64, 0, 63), 1.5, 1.2),
        ((1, 1, 1, 1), 0.0, 1.0),
        ((2000, 65, 1, 3000), 2.5, 1.5)]


def _run(bulk, hkv=2, seed=7):
    rng = np.random.default_rng(seed)
    batch = 4
    cache = _cache(batch, hkv, mbp=160)
    groups = {(b, h): so.GroupState(D) for b in range(batch) for h in range(hkv)}
    for counts, shift, scale in PLAN:
        kt, vt, k64, v64 = _chunk(rng, counts, hkv, shift, scale)
        n_new = torch.tensor(counts, dtype=torch.int32, device="cuda")
        use_bulk = bulk and max(counts) > 1
        cache.append(kt.cuda(), vt.cuda(), n_new, bulk=use_bulk)
        for (b, h), g in groups.items():
            so.append(g, k64[b, :counts[b], h], v64[b, :counts[b], h])
    torch.cuda.synchronize()
    return cache, groups


def _check_state(cache, groups):
    assert int(cache.dev_status.item()) == 0
    S, z, m = (t.cpu().numpy().astype(np.float64) for t in (cache.S, cache.z, cache.m))
    stats = cache.blk_stats.cpu().numpy()
    lens = cache.context_lens.cpu().numpy()
    for (b, h), g in groups.items():
        assert lens[b] == g.length
        if g.length == 0:
            assert np.all(m[b, h] == -np.inf) and np.all(S[b, h] == 0) and np.all(z[b, h] == 0)
            continue
        np.testing.assert_array_equal(m[b, h], g.m)          # max of bf16 values: exact
        np.testing.assert_allclose(z[b, h], g.z, rtol=2e-5)
        np.testing.assert_allclose(S[b, h], g.S, rtol=2e-5, atol=2e-5 * np.abs(g.S).max())
        n, mean, var = so.block_stats(g.K, B)
        for j in range(len(n)):
            np.testing.assert_allclose(stats[b, h, j, 0], mean[j], rtol=1e-6, atol=1e-7)
            np.testing.assert_allclose(stats[b, h, j, 1], var[j], rtol=1e-6, atol=1e-7)


def test_bulk_append_matches_oracle():
    cache, groups = _run(bulk=True)
    _check_state(cache, groups)


def test_one_token_path_matches_oracle_on_the_same_chunks():
    cache, groups = _run(bulk=False)
    _check_state(cache, groups)


def test_bulk_append_is_deterministic():
    a, _ = _run(bulk=True, seed=3)
    b, _ = _run(bulk=True, seed=3)
    for x, y in ((a.S, b.S), (a.z, b.z), (a.m, b.m), (a.blk_stats, b.blk_stats)):
        assert torch.equal(x, y)


def test_bulk_append_many_groups_one_split_each():
    """batch * Hkv above the SM count: one split per (sequence, KV head)."""
    rng = np.random.default_rng(11)
    batch, hkv = 20, 8
    cache = _cache(batch, hkv, mbp=8)
    counts = [int(c) for c in rng.integers(0, 300, batch)]
    counts[0], counts[1] = 0, 300
    kt, vt, k64, v64 = _chunk(rng, counts, hkv, 0.5, 1.0)
    cache.append(kt.cuda(), vt.cuda(), torch.tensor(counts, dtype=torch.int32, device="cuda"),
                 bulk=True)
    torch.cuda.synchronize()
    groups = {}
    for b in range(batch):
        for h in range(hkv):
            g = so.GroupState(D)
            so.append(g, k64[b, :counts[b], h], v64[b, :counts[b], h])
            groups[(b, h)] = g
    _check_state(cache, groups)


def test_bulk_append_rejects_unsupported_shapes():
    from block_sparse_linear_b200 import SplaError
    cache = _cache(1, 1, mbp=4, dtype="f32")
    k = torch.zeros((1, 64, 1, D), dtype=torch.float32, device="cuda")
    with pytest.raises(SplaError, match="unsupported"):
        cache.append(k, k.clone(), bulk=True)
    cache = _cache(1, 1, mbp=4, d=64)
    k = torch.zeros((1, 64, 1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(SplaError, match="unsupported"):
        cache.append(k, k.clone(), bulk=True)
