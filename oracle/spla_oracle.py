"""Plain fp64 CPU oracle of one SPLA decode step.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module:
only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may use it. It shares no code with the CUDA path.

What it follows ("SPLA: Block Sparse Plus Linear Attention for Long Context
Modeling", gist.science technical summary; the German translation on the same
site repeats it):

* section 2.1 "Principled Block Selection via Second-Order Taylor Expansion":
  the block relevance is the integrated attention mass of the block's tokens,
  approximated around the block mean by exp(q.kbar)(1 + 1/2 q^T Cov(k) q) with
  a diagonal covariance;                                    -> block_scores, select_blocks
* section 2 opening paragraph: exact attention over the selected blocks;
  softmax(q k^T / sqrt(d)) V as in the Baidu article, section 1; -> sparse_attention
* section 2.2 "Residual Linear Attention": the long tail is covered by linear
  attention over the unselected blocks, computed as global linear attention
  over all blocks minus linear attention over the selected blocks;
  normalised linear attention phi(q)(phi(K)^T V) / phi(q)(phi(K)^T 1) as in
  the Baidu article, section 7;                  -> append, global_readout, selected_readout, rla
* section 2.3 "Architecture and Integration": parameter-free exponential
  feature map; output = gated sum of the sparse and RLA outputs with an RMS
  norm (whose scale is the only new parameter) on the RLA output. -> combine
* the same sections in block-causal form (each query attends to the tokens up
  to its own, its own block exactly, earlier blocks selected or covered by the
  residual): -> block_causal_forward, linear_attention

Readings where the pages leave a step open (the CUDA path makes the same ones):
 1. logits are q.k/sqrt(d); the Taylor score approximates the mass of those
    logits, so it uses q' = q/sqrt(d) in both of its terms;
 2. the score is the block's integrated mass, n_j times the per-token
    expectation, so the log-domain score carries log n_j (n_j < B only for a
    sequence's last block);
 3. Cov(k) is the population (divide by n_j) diagonal variance of the block's
    stored keys;
 4. phi(x) = exp(x) element-wise on the unscaled q and k;
 5. the global state is kept as S = sum_t exp(k_t - m) v_t^T, z = sum_t exp(k_t - m)
    with m the per-dimension running maximum of the keys: exactly the
    unscaled state times exp(-m), which cancels in the ratio;
 6. o_rla = (N - N~)/(D - D~): the numerator/denominator pairs are subtracted,
    which is exactly linear attention over the unselected blocks; when every
    block is selected o_rla is 0;
 7. out = o_sparse + gamma * o_rla / sqrt(mean(o_rla^2) + eps), eps = 1e-6;
 8. selection is per query head; ties go to the lower block index; sink
    (first) and local (last) blocks are kept on top of the top-k only when a
    workload names them; when k or fewer candidates remain every block is kept;
 9. decode attends over the whole cache, the token just appended included;
    an empty cache gives out = 0;
10. block-causal form: query t sees tokens 0..t, its own block exactly and
    causally, the complete earlier blocks as candidates (top_k after any sink
    blocks kept), the candidates left out by linear attention.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


@dataclass
class OracleParams:
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    top_k: int
    n_sink: int = 0
    n_local: int = 0
    softmax_scale: float = 0.0      # <= 0 means 1/sqrt(head_dim)
    rms_eps: float = 1e-6
    no_rla: bool = False            # the pages' "SPA" ablation (section 4): o_rla = 0
    first_order: bool = False       # mean-only score (section 4 ablation): drop the variance term

    @property
    def scale(self) -> float:
        return self.softmax_scale if self.softmax_scale > 0 else 1.0 / math.sqrt(self.head_dim)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


class GroupState:
    """KV history and linear-attention state of one (sequence, KV head)."""

    def __init__(self, d: int):
        self.K = np.zeros((0, d))
        self.V = np.zeros((0, d))
        self.S = np.zeros((d, d))           # sum_t exp(k_t - m) v_t^T
        self.z = np.zeros(d)                # sum_t exp(k_t - m)
        self.m = np.full(d, -np.inf)        # running max of k per dimension

    @property
    def length(self) -> int:
        return self.K.shape[0]


# ----------------------------------------------------------------------------- a0: state
def append(g: GroupState, k_new: np.ndarray, v_new: np.ndarray) -> None:
    """Append tokens and update the global linear-attention state (section 2.2).

    S and z accumulate phi(k) v^T and phi(k) over every token. Stored scaled by
    exp(-m): when the running max m rises the old rows are rescaled by
    exp(m_old - m_new) before the new tokens are added.
    """
    k_new = np.asarray(k_new, np.float64)
    v_new = np.asarray(v_new, np.float64)
    if k_new.shape[0] == 0:
        return
    m_new = np.maximum(g.m, k_new.max(axis=0))
    rescale = np.exp(g.m - m_new)                    # exp(-inf) = 0 for an empty state
    e = np.exp(k_new - m_new)                        # [n][d]
    g.S = g.S * rescale[:, None] + e.T @ v_new
    g.z = g.z * rescale + e.sum(axis=0)
    g.m = m_new
    g.K = np.concatenate([g.K, k_new])
    g.V = np.concatenate([g.V, v_new])


def block_stats(K: np.ndarray, B: int) -> tuple:
    """Per-block token count, mean and population variance of the keys (section 2.1)."""
    L, d = K.shape
    nb = -(-L // B)
    n = np.array([min(B, L - j * B) for j in range(nb)], np.float64)
    mean = np.zeros((nb, d))
    var = np.zeros((nb, d))
    nfull = L // B
    if nfull:
        blk = K[:nfull * B].reshape(nfull, B, d)
        mean[:nfull] = blk.mean(axis=1)
        var[:nfull] = ((blk - mean[:nfull, None, :]) ** 2).mean(axis=1)
    if nfull < nb:
        blk = K[nfull * B:]
        mean[nfull] = blk.mean(axis=0)
        var[nfull] = ((blk - mean[nfull]) ** 2).mean(axis=0)
    return n, mean, var


# ----------------------------------------------------------------------------- a1: score
def block_scores(q: np.ndarray, n: np.ndarray, mean: np.ndarray, var: np.ndarray,
                 scale: float, first_order: bool = False) -> np.ndarray:
    """Log of the second-order Taylor estimate of each block's attention mass.

    log[ n_j exp(q'.mu_j) (1 + 1/2 q'^T diag(sigma_j^2) q') ] with q' = scale * q.
    """
    qs = scale * np.asarray(q, np.float64)
    first = mean @ qs
    if first_order:
        return np.log(n) + first
    second = 0.5 * (var @ (qs * qs))
    return np.log(n) + first + np.log1p(second)


# ----------------------------------------------------------------------------- a2: select
def select_blocks(scores: np.ndarray, k: int, n_sink: int = 0, n_local: int = 0) -> np.ndarray:
    """Forced sink/local blocks plus the k best of the rest; ascending block ids."""
    nb = len(scores)
    forced = set(range(min(n_sink, nb))) | set(range(max(0, nb - n_local), nb))
    pool = [j for j in range(nb) if j not in forced]
    if len(pool) <= k:
        return np.arange(nb)
    ranked = sorted(pool, key=lambda j: (-scores[j], j))
    return np.array(sorted(forced | set(ranked[:k])), np.int64)


def _tokens_of(blocks: np.ndarray, B: int, L: int) -> np.ndarray:
    if len(blocks) == 0:
        return np.zeros(0, np.int64)
    t = np.concatenate([np.arange(j * B, min((j + 1) * B, L)) for j in blocks])
    return t.astype(np.int64)


# ----------------------------------------------------------------------------- a3: exact
def sparse_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, tokens: np.ndarray,
                     scale: float) -> np.ndarray:
    """softmax(scale * q.k_t) weighted sum of v_t over the selected tokens."""
    if len(tokens) == 0:
        return np.zeros(V.shape[1])
    logits = (K[tokens] @ np.asarray(q, np.float64)) * scale
    p = np.exp(logits - logits.max())
    return (p / p.sum()) @ V[tokens]


# ----------------------------------------------------------------------------- a4: RLA
def query_weights(q: np.ndarray, m: np.ndarray) -> tuple:
    """a_i = exp(q_i + m_i - c), c = max_i (q_i + m_i): phi(q) in the state's scaling."""
    x = np.asarray(q, np.float64) + m
    c = x.max()
    return np.exp(x - c), c


def global_readout(a: np.ndarray, g: GroupState) -> tuple:
    """Linear attention over all blocks: (N, D) = (a^T S, a^T z), both scaled by exp(-c)."""
    return a @ g.S, a @ g.z


def selected_readout(a: np.ndarray, g: GroupState, tokens: np.ndarray) -> tuple:
    """Linear attention over the selected tokens only, in the same scaling."""
    if len(tokens) == 0:
        return np.zeros(g.V.shape[1]), 0.0
    w = np.exp(g.K[tokens] - g.m) @ a                  # phi(q).phi(k_t) * exp(-c)
    return w @ g.V[tokens], w.sum()


def rla(N, D, N_sel, D_sel, all_selected: bool) -> np.ndarray:
    """Residual linear attention by subtraction: (N - N~)/(D - D~), or 0 if nothing is left."""
    if all_selected:
        return np.zeros_like(N)
    return (N - N_sel) / (D - D_sel)


# ----------------------------------------------------------------------------- a5: combine
def rms_norm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    return gamma * x / np.sqrt(np.mean(x * x) + eps)


def combine(o_sparse, o_rla, gamma, eps) -> np.ndarray:
    return o_sparse + rms_norm(o_rla, gamma, eps)


# ----------------------------------------------------------------------------- one head
def decode_head(q: np.ndarray, g: GroupState, p: OracleParams, gamma: np.ndarray,
                forced_sel=None, stats=None) -> dict:
    """Score -> select -> exact attention -> RLA -> combine for one query head."""
    d = p.head_dim
    L = g.length
    if L == 0:
        z = np.zeros(d)
        return dict(out=z, o_sparse=z, o_rla=z, sel=np.zeros(0, np.int64),
                    scores=np.zeros(0), n_blocks=0)
    n, mean, var = stats if stats is not None else block_stats(g.K, p.block_size)
    nb = len(n)
    scores = block_scores(q, n, mean, var, p.scale, p.first_order)
    if forced_sel is None:
        sel = select_blocks(scores, p.top_k, p.n_sink, p.n_local)
    else:
        sel = np.array(sorted(int(j) for j in forced_sel), np.int64)
    tokens = _tokens_of(sel, p.block_size, L)
    o_sparse = sparse_attention(q, g.K, g.V, tokens, p.scale)
    all_sel = len(sel) == nb
    if p.no_rla:
        o_rla = np.zeros(d)
    else:
        a, _ = query_weights(q, g.m)
        N, D = global_readout(a, g)
        Ns, Ds = selected_readout(a, g, tokens)
        o_rla = rla(N, D, Ns, Ds, all_sel)
    out = combine(o_sparse, o_rla, np.asarray(gamma, np.float64), p.rms_eps)
    return dict(out=out, o_sparse=o_sparse, o_rla=o_rla, sel=sel, scores=scores, n_blocks=nb)


# ----------------------------------------------------------------------------- block-causal
def linear_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """Normalised linear attention with phi = exp over the given tokens, evaluated directly:
    sum_t w_t v_t / sum_t w_t, w_t = phi(q).phi(k_t) = sum_i exp(q_i + k_t,i), formed in
    log space (each w_t by a log-sum-exp over i, then all w_t scaled by their maximum)."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1])
    x = np.asarray(q, np.float64)[None, :] + K          # [n][d]: q_i + k_t,i
    xm = x.max(axis=1, keepdims=True)
    lw = xm[:, 0] + np.log(np.exp(x - xm).sum(axis=1))  # log w_t
    w = np.exp(lw - lw.max())
    return (w @ V) / w.sum()


def block_causal_forward(K: np.ndarray, V: np.ndarray, Q: np.ndarray, p: OracleParams,
                         gamma: np.ndarray) -> dict:
    """The block-causal form of the method over one KV head's sequence: query t (row t of
    Q [L][G][d], G heads of the group) sees tokens 0..t. Its own block J = t // B is
    attended exactly (causally: tokens J*B..t); the complete earlier blocks 0..J-1 are
    the candidates, scored by the Taylor estimate and the top_k of them (after any sink
    blocks) attended exactly; the candidates left out are covered by linear attention
    over their tokens (section 2.2: the residual is linear attention over the unselected
    blocks), evaluated here directly from those tokens; out as in section 2.3.
    Returns out, o_sparse, o_rla [L][G][d] and sel (list of kept candidate arrays)."""
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    L, d = K.shape
    G = Q.shape[1]
    B = p.block_size
    n_all, mean_all, var_all = block_stats(K[:(L // B) * B], B) if L >= B else (
        np.zeros(0), np.zeros((0, d)), np.zeros((0, d)))
    res = {k: np.zeros((L, G, d)) for k in ("out", "o_sparse", "o_rla")}
    sels = []
    for t in range(L):
        J = t // B
        row = []
        for g in range(G):
            q = np.asarray(Q[t, g], np.float64)
            sel = np.zeros(0, np.int64)
            if J > 0:
                scores = block_scores(q, n_all[:J], mean_all[:J], var_all[:J], p.scale,
                                      p.first_order)
                sel = select_blocks(scores, p.top_k, p.n_sink, 0)
            tokens = np.concatenate([_tokens_of(sel, B, J * B),
                                     np.arange(J * B, t + 1)]).astype(np.int64)
            o_sparse = sparse_attention(q, K[:t + 1], V[:t + 1], tokens, p.scale)
            left = np.setdiff1d(np.arange(J * B), _tokens_of(sel, B, J * B))
            o_rla = np.zeros(d) if (p.no_rla or len(left) == 0) else \
                linear_attention(q, K[left], V[left])
            res["out"][t, g] = combine(o_sparse, o_rla, np.asarray(gamma[g], np.float64),
                                       p.rms_eps)
            res["o_sparse"][t, g] = o_sparse
            res["o_rla"][t, g] = o_rla
            row.append(sel)
        sels.append(row)
    res["sel"] = sels
    return res


class OracleCache:
    """Oracle view of a batch of sequences: one GroupState per (sequence, KV head).

    ``groups`` restricts the state to some (sequence, KV head) pairs so that
    full-size workloads can be checked on a sample.
    """

    def __init__(self, p: OracleParams, batch: int, groups=None):
        self.p = p
        self.batch = batch
        if groups is None:
            groups = [(b, h) for b in range(batch) for h in range(p.num_kv_heads)]
        self.state = {tuple(gk): GroupState(p.head_dim) for gk in groups}

    def append_seq(self, b: int, K: np.ndarray, V: np.ndarray) -> None:
        """Append tokens K, V [n][Hkv][d] to sequence b."""
        for h in range(self.p.num_kv_heads):
            if (b, h) in self.state:
                append(self.state[(b, h)], K[:, h], V[:, h])

    def append_group(self, b: int, h: int, k: np.ndarray, v: np.ndarray) -> None:
        append(self.state[(b, h)], k, v)

    def decode(self, q: np.ndarray, gamma: np.ndarray, heads=None, forced_sel=None) -> dict:
        """Decode every query head whose group is held (or the listed (b, hq) heads).

        q: [batch][Hq][d]; gamma: [Hq][d]; forced_sel: {(b, hq): blocks} to
        evaluate a given selection instead of the oracle's own.
        Returns {(b, hq): result dict}.
        """
        p = self.p
        res = {}
        want = heads
        if want is None:
            want = [(b, hq) for (b, h) in self.state for hq in range(h * p.group, (h + 1) * p.group)]
        by_group = {}
        for (b, hq) in want:
            by_group.setdefault((b, hq // p.group), []).append(hq)
        for (b, h), hqs in by_group.items():
            g = self.state[(b, h)]
            stats = block_stats(g.K, p.block_size) if g.length else None
            for hq in hqs:
                fs = None if forced_sel is None else forced_sel.get((b, hq))
                res[(b, hq)] = decode_head(np.asarray(q[b, hq], np.float64), g, p,
                                           gamma[hq], forced_sel=fs, stats=stats)
        return res
