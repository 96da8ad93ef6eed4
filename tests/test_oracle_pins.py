"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks the oracle against a closed form, an invariant, a library
routine or brute force, chosen so that a plausible slip (a dropped term, a
wrong coefficient or sign, a transposed operand, a wrong divisor) fails one
of them. All run on the CPU.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import spla_oracle as so
from workloads import gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _logsumexp(x):
    m = np.max(x)
    return m + math.log(np.sum(np.exp(x - m)))


# ----------------------------------------------------------------------------- a1 score
def test_score_equals_block_mass_when_variance_is_zero():
    """sigma^2 = 0: the second-order term vanishes and the score is the exact log mass.

    Blocks of identical tokens, including a partial last block, so log n_j is
    checked too (a dropped log n_j or a wrong logit scale fails here).
    """
    rng = np.random.default_rng(11)
    d, B, L = 16, 8, 8 * 5 + 3
    rows = rng.standard_normal((-(-L // B), d))
    K = np.repeat(rows, B, axis=0)[:L]
    q = rng.standard_normal(d)
    scale = 1 / math.sqrt(d)
    n, mean, var = so.block_stats(K, B)
    assert np.max(var) < 1e-30          # zero up to the rounding of the mean
    s = so.block_scores(q, n, mean, var, scale)
    for j in range(len(n)):
        toks = K[j * B:min((j + 1) * B, L)]
        assert s[j] == pytest.approx(_logsumexp(scale * toks @ q), abs=1e-12)


def test_score_second_order_term_and_population_variance():
    """Tokens that differ along one axis only: the covariance is exactly diagonal.

    With symmetric offsets +-y the mean of exp(y_t) is 1 + mean(y^2)/2 + O(y^4),
    so the Taylor score matches the true log mass to the fourth-order remainder.
    A missing 1/2, a missing variance term or an n-1 divisor misses by orders
    of magnitude more than that remainder.
    """
    rng = np.random.default_rng(12)
    d, B = 8, 4
    base = rng.standard_normal(d)
    off = np.array([0.3, -0.3, 0.1, -0.1])
    K = np.tile(base, (B, 1))
    K[:, 2] += off
    q = rng.standard_normal(d) * 3
    scale = 1 / math.sqrt(d)
    n, mean, var = so.block_stats(K, B)
    s = so.block_scores(q, n, mean, var, scale)[0]
    true = _logsumexp(scale * K @ q)
    y = scale * q[2] * off
    remainder = np.mean(np.abs(y) ** 4 / 24 * np.exp(np.abs(y)))
    assert abs(s - true) <= 1.01 * remainder
    # the terms the pin separates
    x_pop = np.mean(y ** 2)
    x_sample = np.sum(y ** 2) / (B - 1)
    assert abs(math.log1p(0.5 * x_sample) - math.log1p(0.5 * x_pop)) > 20 * remainder
    assert abs(math.log1p(x_pop) - math.log1p(0.5 * x_pop)) > 20 * remainder
    assert abs(math.log1p(0.5 * x_pop)) > 20 * remainder
    s1 = so.block_scores(q, n, mean, var, scale, first_order=True)[0]
    assert s1 == pytest.approx(math.log(B) + scale * base @ q, abs=1e-12)


def test_score_tracks_gaussian_block_mass_in_rank():
    """Blocks of Gaussian tokens: the score ranks blocks like the brute-force mass."""
    rng = np.random.default_rng(13)
    d, B, nb = 32, 64, 200
    mu = 0.5 * rng.standard_normal((nb, d))
    K = (mu[:, None, :] + 0.5 * rng.standard_normal((nb, B, d))).reshape(nb * B, d)
    q = rng.standard_normal(d)
    scale = 1 / math.sqrt(d)
    n, mean, var = so.block_stats(K, B)
    s = so.block_scores(q, n, mean, var, scale)
    mass = np.array([_logsumexp(scale * K[j * B:(j + 1) * B] @ q) for j in range(nb)])
    rs = np.argsort(np.argsort(s))
    rm = np.argsort(np.argsort(mass))
    rho = np.corrcoef(rs, rm)[0, 1]
    assert rho > 0.97
    assert np.max(np.abs(s - mass)) < 0.15     # sample skew and off-diagonal covariance


# ----------------------------------------------------------------------------- a2 select
def _brute_select(scores, k, n_sink, n_local):
    nb = len(scores)
    forced = set(range(min(n_sink, nb))) | set(range(max(0, nb - n_local), nb))
    pool = [j for j in range(nb) if j not in forced]
    if len(pool) <= k:
        return list(range(nb))
    best = None
    for comb in itertools.combinations(pool, k):
        key = (sum(scores[j] for j in comb), tuple(-j for j in comb))
        if best is None or key > best[0]:
            best = (key, comb)
    return sorted(forced | set(best[1]))


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("k,n_sink,n_local", [(3, 0, 0), (2, 1, 1), (4, 1, 0), (8, 0, 0), (9, 1, 1)])
def test_select_matches_brute_force(seed, k, n_sink, n_local):
    rng = np.random.default_rng(seed)
    nb = 9
    scores = np.round(rng.standard_normal(nb), 1)   # coarse: ties happen
    got = so.select_blocks(scores, k, n_sink, n_local).tolist()
    assert got == _brute_select(scores.tolist(), k, n_sink, n_local)


def test_select_ties_prefer_lower_index():
    scores = np.array([1.0, 2.0, 2.0, 2.0, 0.5])
    assert so.select_blocks(scores, 2).tolist() == [1, 2]


# ----------------------------------------------------------------------------- a3 exact
def _group_with(K, V):
    g = so.GroupState(K.shape[1])
    so.append(g, K, V)
    return g


def test_all_blocks_selected_is_dense_softmax_attention_and_no_rla():
    """k >= number of blocks: sparse attention is dense attention (torch SDPA, fp64)
    and the residual is exactly zero."""
    rng = np.random.default_rng(21)
    d, B, L = 32, 16, 16 * 6 + 5
    K, V = rng.standard_normal((L, d)), rng.standard_normal((L, d))
    q = rng.standard_normal(d)
    p = so.OracleParams(num_q_heads=1, num_kv_heads=1, head_dim=d, block_size=B, top_k=10)
    r = so.decode_head(q, _group_with(K, V), p, np.ones(d))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None, None], torch.from_numpy(K)[None, None],
        torch.from_numpy(V)[None, None])[0, 0, 0].numpy()
    np.testing.assert_allclose(r["o_sparse"], ref, rtol=1e-12, atol=1e-13)
    assert np.all(r["o_rla"] == 0)
    np.testing.assert_array_equal(r["out"], r["o_sparse"])


def test_sparse_attention_is_softmax_over_selected_tokens():
    """A forced selection: equal to SDPA restricted to those tokens (the tail block partial)."""
    rng = np.random.default_rng(22)
    d, B, L = 16, 8, 8 * 7 + 3
    K, V = rng.standard_normal((L, d)), rng.standard_normal((L, d))
    q = rng.standard_normal(d)
    p = so.OracleParams(1, 1, d, B, top_k=3)
    sel = [1, 4, 7]
    r = so.decode_head(q, _group_with(K, V), p, np.ones(d), forced_sel=sel)
    toks = np.r_[8:16, 32:40, 56:59]
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None, None], torch.from_numpy(K[toks])[None, None],
        torch.from_numpy(V[toks])[None, None])[0, 0, 0].numpy()
    np.testing.assert_allclose(r["o_sparse"], ref, rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------- a0/a4 RLA
def _chunked_group(K, V, rng):
    g = so.GroupState(K.shape[1])
    cuts = np.sort(rng.choice(np.arange(1, len(K)), size=5, replace=False))
    for a, b in zip(np.r_[0, cuts], np.r_[cuts, len(K)]):
        so.append(g, K[a:b], V[a:b])
    return g


def test_state_after_chunked_appends_is_the_unscaled_sum():
    """exp(m) * S = sum_t exp(k_t) v_t^T and exp(m) * z = sum_t exp(k_t), for any chunking,
    with keys whose running maximum rises over time."""
    rng = np.random.default_rng(31)
    d, L = 12, 300
    K = rng.standard_normal((L, d)) + np.linspace(0, 3, L)[:, None]
    V = rng.standard_normal((L, d))
    g = _chunked_group(K, V, rng)
    ref = np.exp(K).T @ V
    np.testing.assert_allclose(np.exp(g.m)[:, None] * g.S, ref, rtol=1e-12,
                               atol=1e-13 * np.abs(ref).max())
    np.testing.assert_allclose(np.exp(g.m) * g.z, np.exp(K).sum(0), rtol=1e-12)
    np.testing.assert_array_equal(g.m, K.max(0))


@pytest.mark.parametrize("seed", range(4))
def test_subtraction_rla_equals_direct_linear_attention_over_unselected(seed):
    """(N - N~)/(D - D~) from the state equals linear attention computed directly over the
    unselected tokens with unscaled phi(q).phi(k) = sum_i exp(q_i) exp(k_i)."""
    rng = np.random.default_rng(40 + seed)
    d, B, L = 16, 8, 8 * 9 + 5
    K = rng.standard_normal((L, d)) + np.linspace(-1, 2, L)[:, None]
    V = rng.standard_normal((L, d)) + 0.3
    q = rng.standard_normal(d)
    p = so.OracleParams(1, 1, d, B, top_k=3)
    g = _chunked_group(K, V, rng)
    r = so.decode_head(q, g, p, np.ones(d))
    sel_tok = np.concatenate([np.arange(j * B, min((j + 1) * B, L)) for j in r["sel"]])
    unsel = np.setdiff1d(np.arange(L), sel_tok)
    w = np.exp(K[unsel]) @ np.exp(q)
    direct = (w @ V[unsel]) / w.sum()
    np.testing.assert_allclose(r["o_rla"], direct, rtol=1e-11, atol=1e-13)
    # and the combine
    rms = math.sqrt(np.mean(direct ** 2) + 1e-6)
    np.testing.assert_allclose(r["out"], r["o_sparse"] + direct / rms, rtol=1e-11)


def test_no_rla_ablation_outputs_sparse_only():
    rng = np.random.default_rng(5)
    d, B, L = 8, 4, 40
    K, V = rng.standard_normal((L, d)), rng.standard_normal((L, d))
    p = so.OracleParams(1, 1, d, B, top_k=2, no_rla=True)
    r = so.decode_head(rng.standard_normal(d), _group_with(K, V), p, np.ones(d))
    np.testing.assert_array_equal(r["out"], r["o_sparse"])


# ----------------------------------------------------------------------------- a5 combine
def test_rms_norm_matches_torch():
    rng = np.random.default_rng(7)
    x, gm = rng.standard_normal(64), rng.standard_normal(64)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), [64], torch.from_numpy(gm), eps=1e-6)
    np.testing.assert_allclose(so.rms_norm(x, gm, 1e-6), ref.numpy(), rtol=1e-12)
    assert np.all(so.rms_norm(np.zeros(8), np.ones(8), 1e-6) == 0)


def test_gamma_scales_rla_linearly():
    rng = np.random.default_rng(8)
    d, B, L = 8, 4, 40
    K, V = rng.standard_normal((L, d)), rng.standard_normal((L, d))
    q = rng.standard_normal(d)
    p = so.OracleParams(1, 1, d, B, top_k=2)
    g = _group_with(K, V)
    r1 = so.decode_head(q, g, p, np.ones(d))
    r2 = so.decode_head(q, g, p, 3 * np.ones(d))
    np.testing.assert_allclose(r2["out"] - r1["o_sparse"], 3 * (r1["out"] - r1["o_sparse"]),
                               rtol=1e-12)


def test_empty_cache_gives_zero():
    p = so.OracleParams(1, 1, 8, 4, top_k=2)
    r = so.decode_head(np.ones(8), so.GroupState(8), p, np.ones(8))
    assert np.all(r["out"] == 0) and len(r["sel"]) == 0


# ----------------------------------------------------------------------------- golden
def test_golden_hand_computed_decode():
    """A four-token case worked out by hand (derivation in the fixture)."""
    with open(os.path.join(GOLDEN, "tiny_decode.json")) as f:
        fx = json.load(f)
    p = so.OracleParams(num_q_heads=1, num_kv_heads=1, head_dim=fx["head_dim"],
                        block_size=fx["block_size"], top_k=fx["top_k"])
    g = _group_with(np.array(fx["K"], float), np.array(fx["V"], float))
    r = so.decode_head(np.array(fx["q"], float), g, p, np.ones(fx["head_dim"]))
    assert r["sel"].tolist() == fx["expected_sel"]
    np.testing.assert_allclose(r["scores"], fx["expected_scores"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["o_sparse"], fx["expected_o_sparse"], atol=1e-12)
    np.testing.assert_allclose(r["o_rla"], fx["expected_o_rla"], atol=1e-12)
    np.testing.assert_allclose(r["out"], fx["expected_out"], atol=1e-12)


# ----------------------------------------------------------------------------- workloads
def test_planted_blocks_are_selected_in_the_small_fp32_workload():
    """The fp32 4096-token workload plants 3 blocks along the group's query direction;
    every head must select all three."""
    w = gen.get("cfg1")
    K, V = gen.prefix_seq(w, 0)
    q = gen.query(w, 0)
    p = so.OracleParams(w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.top_k)
    oc = so.OracleCache(p, w.batch)
    oc.append_seq(0, K, V)
    res = oc.decode(q, gen.gamma(w))
    planted = np.nonzero(gen.plan(w, 0).planted[:, 0])[0]
    assert len(planted) == 3
    for (b, h), r in res.items():
        assert set(planted.tolist()) <= set(r["sel"].tolist()), (h, planted, r["sel"])
        assert len(r["sel"]) == w.top_k


# ----------------------------------------------------------------------------- block-causal form
def _bc_case(L=37, d=8, B=4, G=2, top_k=2, n_sink=0, seed=5):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((L, d))
    V = rng.standard_normal((L, d))
    Q = rng.standard_normal((L, G, d))
    p = so.OracleParams(num_q_heads=G, num_kv_heads=1, head_dim=d, block_size=B, top_k=top_k,
                        n_sink=n_sink)
    return K, V, Q, p


def test_block_causal_with_every_block_kept_is_causal_softmax_attention():
    """top_k above every block count: no residual, and each query's exact part is causal
    softmax attention over tokens 0..t (torch SDPA with a causal mask, fp64)."""
    K, V, Q, p = _bc_case(top_k=100)
    r = so.block_causal_forward(K, V, Q, p, np.ones((2, 8)))
    assert np.all(r["o_rla"] == 0)
    for g in range(2):
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q[:, g])[None, None], torch.from_numpy(K)[None, None],
            torch.from_numpy(V)[None, None], is_causal=True, scale=p.scale)[0, 0].numpy()
        np.testing.assert_allclose(r["o_sparse"][:, g], ref, rtol=1e-12, atol=1e-12)


def test_linear_attention_equals_the_unscaled_formula():
    rng = np.random.default_rng(2)
    q, K, V = rng.standard_normal(6), rng.standard_normal((9, 6)), rng.standard_normal((9, 6))
    w = np.exp(K) @ np.exp(q)                      # phi(q).phi(k_t), small values
    np.testing.assert_allclose(so.linear_attention(q, K, V), (w @ V) / w.sum(), rtol=1e-12)


@pytest.mark.parametrize("n_sink", [0, 1])
def test_block_causal_row_is_the_decode_step_with_a_local_block(n_sink):
    """Row t of the block-causal form equals a decode step over tokens 0..t with the last
    (current) block kept as a local block: the state-subtraction residual equals the
    direct one over the candidates left out, and the kept sets agree."""
    K, V, Q, p = _bc_case(n_sink=n_sink)
    gamma = np.linspace(0.5, 1.5, 16).reshape(2, 8)
    r = so.block_causal_forward(K, V, Q, p, gamma)
    pl = so.OracleParams(**{**p.__dict__, "n_local": 1})
    g = so.GroupState(8)
    for t in range(K.shape[0]):
        so.append(g, K[t:t + 1], V[t:t + 1])
        J = t // p.block_size
        for h in range(2):
            ref = so.decode_head(Q[t, h], g, pl, gamma[h])
            assert list(ref["sel"]) == sorted(set(r["sel"][t][h].tolist()) | {J})
            for key in ("out", "o_sparse", "o_rla"):
                np.testing.assert_allclose(r[key][t, h], ref[key], rtol=1e-9, atol=1e-12)
