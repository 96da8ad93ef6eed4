"""Comparison of CUDA decode results with the CPU oracle (shared by the GPU tests).

Acceptance, per (sequence, query head):
* selection: the GPU's kept set equals the oracle's, except blocks whose
  oracle score lies within SEL_TIE of the oracle's k-th best candidate score
  (relative 1e-6 on the linear score is 1e-6 absolute on its log);
* outputs: the oracle is re-run on the GPU's own selection; o_sparse, o_rla
  and out must match within 1e-4 * max(1, max|ref|) for fp32 workloads and
  2e-2 absolute for bf16 workloads. o_sparse and o_rla come back in fp32; out
  comes back in bf16 for bf16 workloads, so its bound also allows the output
  format's own rounding, half a bf16 ulp of the reference value (|out| >= 8
  has an ulp of 0.0625, beyond 2e-2 for any bf16 number).
o_rla and out are compared only where the RLA subtraction is well
conditioned: kappa = max(D/(D - D~), |N|_inf/|N - N~|_inf), computed by the
oracle in fp64, bounds how much the fp32 state's rounding is amplified. Heads
past KAPPA_MAX are counted, returned with their kappa, and capped by the tests
(ILL_CAP: none outside the 1M-token Student-t workload); o_sparse and the
selection are still checked on them. A head whose residual denominator the GPU
could not resolve (its o_rla set to 0 and SPLA_DEV_RLA_UNRESOLVED raised) must be
one of them.
"""
import numpy as np

from oracle import spla_oracle as so

SEL_TIE = 1e-6
TOL = {"f32": 1e-4, "bf16": 2e-2}
KAPPA_MAX = {"f32": 10.0, "bf16": 2e3}
# Ill-conditioned heads allowed per workload (by the workload's base name). The
# oracle's own kappa over every head (full size and test size) is at most 2 for
# the 4K, 32K, 128K and ragged workloads; only the 1M-token workload, whose
# heavy-tailed (Student-t) key offsets let a few blocks hold nearly all of a
# head's linear-attention mass, has heads past KAPPA_MAX.
ILL_CAP = {"cfg1": 0, "cfg2": 0, "cfg3": 0, "cfg4": None, "cfg5": 0}
ILL_FRACTION_CFG4 = 0.25       # at most a quarter of the compared heads


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (8 significand bits)."""
    ax = np.maximum(np.abs(np.asarray(x, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def kappa(q, g: so.GroupState, p: so.OracleParams, sel) -> float:
    if g.length == 0:
        return 1.0
    tokens = so._tokens_of(np.asarray(sel, np.int64), p.block_size, g.length)
    a, _ = so.query_weights(np.asarray(q, np.float64), g.m)
    N, D = so.global_readout(a, g)
    Ns, Ds = so.selected_readout(a, g, tokens)
    dr = D - Ds
    nr = np.abs(N - Ns).max()
    if dr <= 0 or nr == 0:
        return np.inf
    return float(max(D / dr, np.abs(N).max() / nr))


def check_selection(gpu_sel, ref: dict, p: so.OracleParams):
    """gpu_sel: 1-D int array (-1 padded). Returns the set difference size (allowed ties)."""
    gs = set(int(x) for x in gpu_sel if x >= 0)
    os_ = set(int(x) for x in ref["sel"])
    if gs == os_:
        return 0
    scores = ref["scores"]
    nb = len(scores)
    forced = set(range(min(p.n_sink, nb))) | set(range(max(0, nb - p.n_local), nb))
    pool = sorted((j for j in range(nb) if j not in forced), key=lambda j: (-scores[j], j))
    assert len(pool) > p.top_k, (gs, os_)
    kth = scores[pool[p.top_k - 1]]
    diff = gs ^ os_
    for j in diff:
        assert j not in forced, ("forced block differs", j)
        assert abs(scores[j] - kth) <= SEL_TIE, (
            f"block {j} differs with score gap {scores[j] - kth:.3g} > {SEL_TIE}")
    assert len(gs) == len(os_)
    return len(diff)


def compare_head(gpu: dict, oc: so.OracleCache, q, gamma, b, hq, dtype: str) -> dict:
    """Check one head; gpu holds numpy arrays out, o_sparse, o_rla [d] and sel [kcap]."""
    p = oc.p
    g = oc.state[(b, hq // p.group)]
    ref = so.decode_head(np.asarray(q[b, hq], np.float64), g, p, gamma[hq])
    ties = check_selection(gpu["sel"], ref, p)
    gsel = [int(x) for x in gpu["sel"] if x >= 0]
    fref = so.decode_head(np.asarray(q[b, hq], np.float64), g, p, gamma[hq], forced_sel=gsel)
    tol = TOL[dtype]
    all_kept = len(gsel) == fref["n_blocks"]
    if all_kept or p.no_rla:
        # nothing left for the residual: exactly zero on both sides
        assert np.all(np.asarray(gpu["o_rla"]) == 0) and np.all(fref["o_rla"] == 0)
        k = 1.0
    else:
        k = kappa(q[b, hq], g, p, gsel)

    def err(name):
        r = fref[name]
        scale = max(1.0, float(np.abs(r).max())) if dtype == "f32" else 1.0
        d = np.abs(np.asarray(gpu[name], np.float64) - r)
        if name == "out" and dtype == "bf16":
            # the output format's own rounding (half a bf16 ulp of the value) comes on top
            d = np.maximum(d - 0.5 * bf16_ulp(r), 0.0)
        return float(d.max()) / scale

    e_sp = err("o_sparse")
    assert e_sp <= tol, f"o_sparse ({b},{hq}) err {e_sp:.3g} > {tol}"
    conditioned = k <= KAPPA_MAX[dtype]
    # errors of every head are measured; only conditioned heads must meet the bound
    e_rl = err("o_rla")
    e_out = err("out")
    if conditioned:
        assert e_rl <= tol, f"o_rla ({b},{hq}) err {e_rl:.3g} > {tol} (kappa {k:.3g})"
        assert e_out <= tol, f"out ({b},{hq}) err {e_out:.3g} > {tol} (kappa {k:.3g})"
    unresolved = (not all_kept and not p.no_rla and np.all(np.asarray(gpu["o_rla"]) == 0))
    return dict(b=b, hq=hq, ties=ties, kappa=k, e_sparse=e_sp, e_rla=e_rl, e_out=e_out,
                conditioned=conditioned, unresolved=unresolved)


def summary(stats) -> dict:
    """Counts over compared heads: ill-conditioned heads with their kappa, worst errors."""
    ill = [(s["b"], s["hq"], float(f"{s['kappa']:.3g}")) for s in stats if not s["conditioned"]]
    cond = [s for s in stats if s["conditioned"]]
    return dict(heads=len(stats), ties=sum(s["ties"] for s in stats), ill=len(ill),
                ill_heads=ill,
                max_sparse=max(s["e_sparse"] for s in stats),
                max_rla=max((s["e_rla"] for s in cond), default=0.0),
                max_out=max((s["e_out"] for s in cond), default=0.0),
                unresolved=[(s["b"], s["hq"]) for s in stats if s["unresolved"]])


def check_ill(name: str, stats, status: int, cap: int = None) -> dict:
    """The ill-conditioned heads stay within the workload's cap (or the given one), and
    the status word carries nothing but the unresolved-residual bit, and that only if
    some head is ill."""
    s = summary(stats)
    base = name.split("-")[0]
    if cap is None:
        cap = ILL_CAP[base]
        if cap is None:
            cap = int(ILL_FRACTION_CFG4 * s["heads"])
    assert s["ill"] <= cap, (f"{name}: {s['ill']} of {s['heads']} heads ill-conditioned "
                             f"(cap {cap}); (b, hq, kappa): {s['ill_heads']}")
    assert status & ~RLA_UNRESOLVED == 0, f"{name}: status {status:#x}"
    if status & RLA_UNRESOLVED:
        assert s["ill"] > 0, f"{name}: residual unresolved on the GPU but every head conditioned"
    # a head the GPU left unresolved is one the oracle finds ill-conditioned
    ill_keys = {(b, hq) for (b, hq, _) in s["ill_heads"]}
    for bh in s["unresolved"]:
        assert bh in ill_keys, f"{name}: head {bh} unresolved on the GPU but conditioned"
    return s


RLA_UNRESOLVED = 0x10
