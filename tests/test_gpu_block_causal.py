"""The block-causal form over whole sequences (spla_block_causal_forward) against the
oracle's block_causal_forward, every query position of every head.

Sequences of ragged lengths (partial last blocks), two KV groups, with and without a
sink block, the first-order score flag and the residual switched off. o_sparse is compared everywhere; o_rla
and out where the residual's subtraction is well conditioned (kappa as in
tests/parity.py, computed here from the tokens directly), and the count of
ill-conditioned positions is asserted to be zero for these value distributions.
"""
import numpy as np
import pytest
import torch

from block_sparse_linear_b200 import SplaConfig, SplaDecodeCache
from oracle import spla_oracle as so

from . import parity

pytestmark = pytest.mark.gpu

D = 128
BS = 64


def _kappa(q, K, V, kept_tokens, J):
    """max(D / (D - D~), |N|inf / |N - N~|inf) over the candidate tokens 0 .. J*B - 1."""
    cand = np.arange(J * BS)
    left = np.setdiff1d(cand, kept_tokens)
    if len(left) == 0:
        return 1.0
    x = q[None, :] + K[cand]
    xm = x.max(axis=1, keepdims=True)
    lw = xm[:, 0] + np.log(np.exp(x - xm).sum(axis=1))
    w = np.exp(lw - lw.max())
    idx = {int(t): i for i, t in enumerate(cand)}
    keep = np.array([idx[int(t)] for t in kept_tokens], np.int64)
    Dt, Ds = w.sum(), w[keep].sum() if len(keep) else 0.0
    Nt = w @ V[cand]
    Ns = w[keep] @ V[kept_tokens] if len(keep) else np.zeros(V.shape[1])
    dr, nr = Dt - Ds, np.abs(Nt - Ns).max()
    if dr <= 0 or nr == 0:
        return np.inf
    return float(max(Dt / dr, np.abs(Nt).max() / nr))


@pytest.mark.parametrize("n_sink,first_order,no_rla",
                         [(0, False, False), (1, False, False), (0, True, False), (1, False, True)])
def test_block_causal_forward_matches_oracle(n_sink, first_order, no_rla):
    rng = np.random.default_rng(17 + n_sink + 2 * first_order + 4 * no_rla)
    lens, hkv, G, top_k = (330, 200), 2, 4, 2
    batch, hq, max_len = len(lens), hkv * G, max(lens)
    nb = -(-max_len // BS)
    cfg = SplaConfig(num_q_heads=hq, num_kv_heads=hkv, head_dim=D, block_size=BS, top_k=top_k,
                     n_sink=n_sink, first_order=first_order, no_rla=no_rla)
    to16 = lambda a: torch.from_numpy(a).to(torch.bfloat16)
    off = np.repeat(rng.normal(0.0, 0.5, (batch, nb, hkv, D)), BS, axis=1)[:, :max_len]
    K = to16(rng.standard_normal((batch, max_len, hkv, D)) + off)
    V = to16(rng.standard_normal((batch, max_len, hkv, D)) + off)
    Q = to16(rng.standard_normal((batch, max_len, hq, D)))
    gamma = rng.uniform(0.5, 1.5, (hq, D))
    table = torch.arange(batch * nb, dtype=torch.int32).reshape(batch, nb)
    cache = SplaDecodeCache(cfg, batch, table, batch * nb, device="cuda")
    kd, vd, qd = K.cuda(), V.cuda(), Q.cuda()
    cache.append(kd, vd, torch.tensor(lens, dtype=torch.int32, device="cuda"))
    out = torch.zeros_like(qd)
    osp = torch.zeros(qd.shape, dtype=torch.float32, device="cuda")
    orl = torch.zeros_like(osp)
    cache.block_causal_forward(kd, vd, qd, torch.from_numpy(gamma).float().cuda(), out, osp, orl)
    torch.cuda.synchronize()
    status = cache.status()
    assert status & ~parity.RLA_UNRESOLVED == 0, status
    out, osp, orl = out.float().cpu().numpy(), osp.cpu().numpy(), orl.cpu().numpy()
    K64, V64, Q64 = K.double().numpy(), V.double().numpy(), Q.double().numpy()
    p = so.OracleParams(num_q_heads=hq, num_kv_heads=hkv, head_dim=D, block_size=BS,
                        top_k=top_k, n_sink=n_sink, first_order=first_order, no_rla=no_rla)
    tol = parity.TOL["bf16"]
    ill = 0
    for b, L in enumerate(lens):
        for h in range(hkv):
            hs = slice(h * G, (h + 1) * G)
            ref = so.block_causal_forward(K64[b, :L, h], V64[b, :L, h], Q64[b, :L, hs], p,
                                          gamma[hs])
            np.testing.assert_allclose(osp[b, :L, hs], ref["o_sparse"], atol=tol)
            for t in range(L):
                J = t // BS
                for g in range(G):
                    kept = so._tokens_of(ref["sel"][t][g], BS, J * BS)
                    k = _kappa(Q64[b, t, h * G + g], K64[b, :L, h], V64[b, :L, h], kept, J)
                    if k > parity.KAPPA_MAX["bf16"]:
                        ill += 1
                        continue
                    np.testing.assert_allclose(orl[b, t, h * G + g], ref["o_rla"][t, g], atol=tol,
                                               err_msg=f"o_rla b={b} t={t} head={h * G + g}")
                    d = np.abs(out[b, t, h * G + g] - ref["out"][t, g])
                    d = np.maximum(d - 0.5 * parity.bf16_ulp(ref["out"][t, g]), 0.0)
                    assert d.max() <= tol, (b, t, h * G + g, d.max())
        # rows past the sequence's length are not written
        assert np.all(out[b, L:] == 0)
    assert ill == 0, ill
    if no_rla:
        assert np.all(orl == 0)
