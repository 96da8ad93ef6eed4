"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Small workloads keep each configuration's structure (heads, head_dim, block
size, top-k, sink/local, value distribution, paging) at lengths the oracle
handles in seconds, with ragged last blocks, and compare every head. Full-size
workloads run the launch configuration the benchmark times and compare a
sample of (sequence, KV head) groups.
"""
import numpy as np
import pytest
import torch

from oracle import feed as ofeed
from oracle import spla_oracle as so
from workloads import feed_gpu, gen

from . import parity

pytestmark = pytest.mark.gpu


def _np(t):
    return None if t is None else t.float().cpu().numpy()


def gpu_decode(cache, q_np, gamma_np, w):
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q = torch.from_numpy(q_np).to(dt).cuda()
    gamma = torch.from_numpy(gamma_np).float().cuda()
    out, sel, osp, orl = cache.new_outputs(debug=True)
    cache.decode(q, gamma, out, sel, osp, orl)
    torch.cuda.synchronize()
    return dict(out=_np(out), sel=sel.cpu().numpy(), o_sparse=_np(osp), o_rla=_np(orl))


def compare_all(res, oc, q, gamma, w, heads=None):
    stats = []
    p = oc.p
    if heads is None:
        heads = [(b, hq) for (b, h) in oc.state for hq in range(h * p.group, (h + 1) * p.group)]
    for (b, hq) in heads:
        g = {k: v[b, hq] for k, v in res.items()}
        stats.append(parity.compare_head(g, oc, q, gamma, b, hq, w.dtype))
    return stats




SMALL = {
    "cfg1": dict(context_lens=(4096,)),
    "cfg2": dict(context_lens=(4096 + 37, 3001)),
    "cfg3": dict(context_lens=(8192 + 5, 6000)),
    "cfg4": dict(context_lens=(65536 + 77,)),
    "cfg5": dict(context_lens=(5000, 300, 12000, 64)),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_workload_matches_oracle(name):
    w = gen.scaled(name, **SMALL[name])
    cache = feed_gpu.build_cache(w)
    oc = ofeed.build(w)
    q = gen.query(w, 0)
    gamma = gen.gamma(w, "random")
    res = gpu_decode(cache, q, gamma, w)
    st = compare_all(res, oc, q, gamma, w)
    s = parity.check_ill(w.name, st, cache.status())
    print(name, s)


@pytest.mark.parametrize("name,flags", [("cfg1", {}), ("cfg2", {}), ("cfg3", {}), ("cfg4", {}),
                                        ("cfg5", {}), ("cfg3", {"first_order": True})])
def test_block_scores_match_oracle(name, flags):
    """Every block's score, element by element, against the oracle's block_scores: the
    fp64 dot products stored in fp32 (half an ulp) plus the fp32 log1p (one ulp of the
    second-order term), tail blocks and the first-order flag included."""
    w = gen.scaled(name, **SMALL[name])
    cache = feed_gpu.build_cache(w, cfg=feed_gpu.config_of(w, **flags))
    oc = ofeed.build(w, **flags)
    q = gen.query(w, 0)
    gpu_decode(cache, q, gen.gamma(w), w)
    got = cache.scores().cpu().numpy().astype(np.float64)
    p = oc.p
    for (b, h), g in oc.state.items():
        n, mean, var = so.block_stats(g.K, w.block_size)
        for hq in range(h * p.group, (h + 1) * p.group):
            ref = so.block_scores(q[b, hq], n, mean, var, p.scale, p.first_order)
            d = got[b, hq, :len(ref)]
            tol = 2.0 * np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64) + 2e-7
            bad = np.abs(d - ref) > tol
            assert not bad.any(), (b, hq, np.flatnonzero(bad)[:5], (d - ref)[bad][:5])


def _planted_new_groups(w, steps):
    """(sequence, KV head) groups that get a planted block opened by one of the steps."""
    out = set()
    for b in range(w.batch):
        p = gen.plan(w, b)
        L0 = w.context_lens[b]
        for j in range(w.n_blocks(L0), w.n_blocks(L0 + steps)):
            out |= {(b, h) for h in range(w.num_kv_heads) if p.planted[j, h]}
    return out


def test_interleaved_append_and_decode_match_oracle():
    """Several steps of (append one token per sequence, decode), as the 128K workload runs.
    Half of the blocks opened by the steps are planted (the 128K workload plants 1 %), so
    that a planted block is opened during the steps (sequence 0 crosses a block boundary
    at step 2). No head is ill-conditioned here (the oracle's kappa stays below 2e3)."""
    w = gen.scaled("cfg3", context_lens=(4096 - 2, 5100), plant_new_prob=0.5)
    assert _planted_new_groups(w, 5)
    cache = feed_gpu.build_cache(w)
    oc = ofeed.build(w)
    gamma = gen.gamma(w)
    for step in range(5):
        k, v, qt = feed_gpu.step_inputs(w, step)
        cache.append(k, v)
        ofeed.append_step(oc, w, step)
        q = gen.query(w, step)
        res = gpu_decode(cache, q, gamma, w)
        parity.check_ill(w.name, compare_all(res, oc, q, gamma, w), cache.status())
    lens = cache.context_lens.cpu().numpy()
    assert lens.tolist() == [4094 + 5, 5100 + 5]


def test_append_state_matches_oracle():
    """Block statistics and the scaled state after chunked prefill plus single-token appends."""
    w = gen.scaled("cfg5", context_lens=(3000, 130, 9000))
    cache = feed_gpu.build_cache(w)
    oc = ofeed.build(w)
    for step in range(3):
        k, v, _ = feed_gpu.step_inputs(w, step)
        cache.append(k, v)
        ofeed.append_step(oc, w, step)
    torch.cuda.synchronize()
    table = gen.block_table(w)
    stats = cache.blk_stats.cpu().numpy()
    S, z, m = (t.cpu().numpy().astype(np.float64) for t in (cache.S, cache.z, cache.m))
    for (b, h), g in oc.state.items():
        np.testing.assert_array_equal(m[b, h], g.m)          # max of bf16 values: exact
        np.testing.assert_allclose(z[b, h], g.z, rtol=2e-5)
        np.testing.assert_allclose(S[b, h], g.S, rtol=2e-5, atol=2e-5 * np.abs(g.S).max())
        n, mean, var = so.block_stats(g.K, w.block_size)
        for j in range(len(n)):
            st = stats[b, h, j]
            np.testing.assert_allclose(st[0], mean[j], rtol=1e-6, atol=1e-7)
            np.testing.assert_allclose(st[1], var[j], rtol=1e-6, atol=1e-7)


# ----------------------------------------------------------------------------- edge cases
def _tiny(**kw):
    base = dict(context_lens=(700, 64, 1, 129))
    base.update(kw)
    return gen.scaled("cfg2", **base)


def test_edge_lengths_tail_blocks_sink_local():
    """Lengths 1, exactly one block, partial tails; sink and local blocks forced."""
    w = _tiny()
    cache = feed_gpu.build_cache(w)
    oc = ofeed.build(w)
    q, gamma = gen.query(w, 0), gen.gamma(w, "random")
    res = gpu_decode(cache, q, gamma, w)
    compare_all(res, oc, q, gamma, w)
    assert cache.status() == 0


def test_all_blocks_selected_gives_zero_rla():
    """top_k >= blocks: o_rla is exactly zero and out equals o_sparse up to bf16 rounding."""
    w = gen.scaled("cfg3", context_lens=(900, 64 * 5), top_k=64)
    cache = feed_gpu.build_cache(w)
    oc = ofeed.build(w)
    q, gamma = gen.query(w, 0), gen.gamma(w)
    res = gpu_decode(cache, q, gamma, w)
    assert np.all(res["o_rla"] == 0)
    compare_all(res, oc, q, gamma, w)


def test_empty_sequence_in_batch_gives_zero():
    w = gen.scaled("cfg3", context_lens=(1000, 0, 200))
    cache = feed_gpu.build_cache(w)
    q, gamma = gen.query(w, 0), gen.gamma(w)
    res = gpu_decode(cache, q, gamma, w)
    assert np.all(res["out"][1] == 0) and np.all(res["sel"][1] == -1)
    oc = ofeed.build(w, groups=[(0, 0), (2, 3)])
    compare_all(res, oc, q, gamma, w)


@pytest.mark.parametrize("flag", ["no_rla", "first_order"])
def test_ablation_flags_match_oracle(flag):
    w = gen.scaled("cfg2", context_lens=(3000, 2000))
    cache = feed_gpu.build_cache(w, cfg=feed_gpu.config_of(w, **{flag: True}))
    oc = ofeed.build(w, **{flag: True})
    q, gamma = gen.query(w, 0), gen.gamma(w)
    res = gpu_decode(cache, q, gamma, w)
    compare_all(res, oc, q, gamma, w)
    if flag == "no_rla":
        assert np.all(res["o_rla"] == 0)


def test_fp32_path_head_dim_128_block_128():
    """The fp32 kernel at the larger tile shape."""
    w = gen.scaled("cfg4", context_lens=(5000, 2100), dtype="f32", top_k=8)
    cache = feed_gpu.build_cache(w)
    oc = ofeed.build(w)
    q, gamma = gen.query(w, 0), gen.gamma(w, "random")
    res = gpu_decode(cache, q, gamma, w)
    compare_all(res, oc, q, gamma, w)


def test_bad_block_table_entry_is_flagged_not_faulted():
    """An out-of-range physical block id: kernels skip it and set the status bit."""
    w = gen.scaled("cfg3", context_lens=(2000, 2000))
    cache = feed_gpu.build_cache(w)
    cache.block_table[1, 3] = w.num_phys_blocks + 5
    q = torch.from_numpy(gen.query(w, 0)).to(torch.bfloat16).cuda()
    cache.decode(q)
    torch.cuda.synchronize()
    assert cache.status() & 0x1


def test_append_past_capacity_is_flagged():
    w = gen.scaled("cfg3", context_lens=(300, 100), extra_tokens=0)
    cache = feed_gpu.build_cache(w)
    before = cache.context_lens.cpu().numpy().copy()
    n = w.capacity_blocks * w.block_size - 300 + 1          # one token too many for seq 0
    k = torch.zeros((2, n, w.num_kv_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    cache.append(k, k.clone(), torch.tensor([n, 1], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert cache.status() & 0x2
    after = cache.context_lens.cpu().numpy()
    assert after[0] == before[0] and after[1] == before[1] + 1


# ----------------------------------------------------------------------------- full size
# (sequence, KV head) groups compared at full size: at least 8 per workload (all 8 of
# the 1M-token workload, one per sequence of the ragged one); the 128K workload runs
# 8 interleaved append + decode steps.
FULL_SAMPLE = {
    "cfg1": None,                      # small enough: every head
    "cfg2": [(b, (3 * b + 1) % 8) for b in range(8)] + [(0, 0), (5, 7)],
    "cfg3": [(b, h) for b in range(4) for h in (2 * b % 8, (2 * b + 5) % 8)],
    "cfg4": [(0, h) for h in range(8)],
    "cfg5": [(b, (5 * b) % 8) for b in range(16)],
}
FULL_STEPS = {"cfg3": 8}


@pytest.mark.slow
@pytest.mark.parametrize("name", list(FULL_SAMPLE))
def test_full_size_sampled_heads_match_oracle(name):
    w = gen.get(name)
    cache = feed_gpu.build_cache(w)
    groups = FULL_SAMPLE[name]
    oc = ofeed.build(w, groups=groups)
    gamma = gen.gamma(w)
    steps = FULL_STEPS.get(name, 1)
    for step in range(steps):
        if steps > 1:
            k, v, _ = feed_gpu.step_inputs(w, step)
            cache.append(k, v)
            ofeed.append_step(oc, w, step)
        q = gen.query(w, step)
        res = gpu_decode(cache, q, gamma, w)
        st = compare_all(res, oc, q, gamma, w)
        s = parity.check_ill(name, st, cache.status())
        print(name, step, s)


def test_rla_cancellation_sets_unresolved_bit():
    """The residual's denominator D - D~ sums the weights of the unselected tokens. Here the
    one unselected block has keys at -200 (and every query is positive, so that block scores
    lowest); its exp(k - m) is 0 in fp32, so on the GPU
    D - D~ is the difference of two fp32 evaluations of the same sum: its sign is rounding
    noise. Wherever it is not positive the combine step returns o_rla = 0 and must raise
    SPLA_DEV_RLA_UNRESOLVED; a head whose o_rla is exactly zero while a block went
    unselected is such a head, and the bit is set exactly when one exists."""
    from block_sparse_linear_b200 import SplaConfig, SplaDecodeCache, _lib
    rng = np.random.default_rng(21)
    batch, hq, hkv, d, bs, nb = 4, 16, 4, 128, 64, 8
    cfg = SplaConfig(num_q_heads=hq, num_kv_heads=hkv, head_dim=d, block_size=bs, top_k=nb - 1)
    table = torch.arange(batch * nb, dtype=torch.int32).reshape(batch, nb)
    cache = SplaDecodeCache(cfg, batch, table, batch * nb, device="cuda")
    k = rng.standard_normal((batch, nb * bs, hkv, d))
    k[:, 3 * bs:4 * bs] = -200.0                    # block 3: weight exp(-200 - m) = 0 in fp32
    v = rng.standard_normal((batch, nb * bs, hkv, d))
    to = lambda a: torch.from_numpy(a).to(torch.bfloat16).cuda()
    cache.append(to(k), to(v), bulk=False)
    # q > 0 in every dimension: block 3's mean of -200 gives it the lowest score of all
    q = to(np.abs(rng.standard_normal((batch, hq, d))) + 0.1)
    out, sel, osp, orl = cache.new_outputs(debug=True)
    cache.decode(q, None, out, sel, osp, orl)
    torch.cuda.synchronize()
    sel, orl = sel.cpu().numpy(), orl.cpu().numpy()
    assert np.all((sel[..., :nb - 1] >= 0)) and not np.any(sel == 3)   # block 3 never selected
    zero_heads = int(np.sum(np.all(orl == 0, axis=-1)))
    status = cache.status()
    assert status & ~_lib.SPLA_DEV_RLA_UNRESOLVED == 0, status
    assert bool(status & _lib.SPLA_DEV_RLA_UNRESOLVED) == (zero_heads > 0), (status, zero_heads)
    print(f"heads with D - D~ <= 0: {zero_heads} of {batch * hq}")


@pytest.mark.parametrize("n_sink", [0, 1])
def test_block_causal_forward_by_decode_steps(n_sink):
    """The block-causal form over a 330-token sequence: per token, a one-token append and a
    decode with the current block kept as a local block (n_local = 1), against the
    oracle's decode step at every position (which equals its block-causal form row by
    row: tests/test_oracle_pins.py) and against that form directly."""
    from block_sparse_linear_b200 import SplaConfig, SplaDecodeCache
    rng = np.random.default_rng(31 + n_sink)
    L, hq, d, bs = 330, 4, 128, 64
    nb = -(-L // bs)
    cfg = SplaConfig(num_q_heads=hq, num_kv_heads=1, head_dim=d, block_size=bs, top_k=2,
                     n_sink=n_sink, n_local=1)
    off = np.repeat(rng.normal(0.0, 0.5, (nb, d)), bs, axis=0)[:L]
    to16 = lambda a: torch.from_numpy(a).to(torch.bfloat16)
    K = to16(rng.standard_normal((L, d)) + off).double().numpy()
    V = to16(rng.standard_normal((L, d)) + off).double().numpy()
    Q = to16(rng.standard_normal((L, hq, d))).double().numpy()
    gamma = rng.uniform(0.5, 1.5, (hq, d))
    table = torch.arange(nb, dtype=torch.int32).reshape(1, nb)
    cache = SplaDecodeCache(cfg, 1, table, nb, device="cuda")
    p = so.OracleParams(num_q_heads=hq, num_kv_heads=1, head_dim=d, block_size=bs, top_k=2,
                        n_sink=n_sink, n_local=1)
    oc = so.OracleCache(p, 1)
    form = so.block_causal_forward(K, V, Q, so.OracleParams(**{**p.__dict__, "n_local": 0}),
                                   gamma)
    g_t = torch.from_numpy(gamma).float().cuda()
    out, sel, osp, orl = cache.new_outputs(debug=True)
    stats = []
    for t in range(L):
        kt = to16(K[t][None, None, None]).cuda()
        cache.append(kt, to16(V[t][None, None, None]).cuda())
        cache.decode(to16(Q[t][None]).cuda(), g_t, out, sel, osp, orl)
        oc.append_group(0, 0, K[t:t + 1], V[t:t + 1])
        res = {"out": out.float().cpu().numpy()[0], "sel": sel.cpu().numpy()[0],
               "o_sparse": osp.cpu().numpy()[0], "o_rla": orl.cpu().numpy()[0]}
        for h in range(hq):
            stats.append(parity.compare_head({k: v[h] for k, v in res.items()}, oc, Q[t][None],
                                             gamma, 0, h, "bf16"))
            np.testing.assert_allclose(res["o_sparse"][h], form["o_sparse"][t, h], atol=2e-2)
    s = parity.check_ill("cfg2", stats, cache.status())
    print("block-causal", n_sink, s)
