#!/usr/bin/env python
"""SPLA decode benchmark on B200: queries*heads/s and achieved HBM bandwidth.

One step = the whole hot path for one batch: spla_append_kv (one new token
per sequence, updating block statistics and the linear-attention state; two
launches) then spla_decode (four launches: score every block -> select top-k ->
exact attention over the kept blocks with the fused residual-linear-attention
term -> combine of the splits with the residual and the RMS norm).

Default workload: batch 4, 32 query / 8 KV heads, d 128, 131072-token
contexts in 64-token blocks, top-k 32, 64 steps of append + decode (the
128K-context decode workload). Inputs are synthetic and seeded
(workloads/gen.py) and resident in HBM before timing; L2 is flushed (a
512 MiB read) before every timed step and the flush is outside the events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload cfg3]
    python bench.py --impl reference      # the CPU oracle on the host cores

Multi-GPU (torchrun, one rank per GPU): every rank decodes its own
independent batch (weak scaling, no collective on the data path); the step
time is the max over ranks.
"""
import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SPLA decode queries*heads/s (1 x B200), achieved HBM GB/s"
UNIT = "queries*heads/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="cfg3")
    ap.add_argument("--context", type=int, default=0,
                    help="profiling only: same workload at another context length")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--shards", type=int, default=0,
                    help="also time the context-sharded decode with the workload's sequences "
                         "split into this many shard caches on this GPU")
    ap.add_argument("--no-block-causal", action="store_true",
                    help="skip the block-causal forward measurement")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the bulk-append (prefill chunk) measurement")
    ap.add_argument("--also", default="cfg4",
                    help="a second workload measured in the same run ('' for none)")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """NVML samples of SM clock and clock-event reasons every 2 ms during the timed region."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.index]) if vis else self.index
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception:
            self.nv = None
        return self

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((sm, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def __exit__(self, *a):
        self._stop.set()
        if self.nv is not None:
            self.t.join(timeout=2)

    def summary(self):
        sm = [x for x, _ in self.samples]
        reasons = sorted(n for n, bit in self.REASONS.items()
                         if any(r & bit for _, r in self.samples))
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sm), "source": "NVML, 2 ms period"}


class L2Flush:
    """Evict L2 by reading 512 MiB (a read leaves no dirty lines for the next kernel)."""

    def __init__(self, dev):
        import torch
        self.buf = torch.ones(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        self.acc = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        import torch
        torch.sum(self.buf, 0, out=self.acc)


# ----------------------------------------------------------------------------- bytes
def step_bytes(w, sel: np.ndarray, lens: np.ndarray) -> dict:
    """Algorithmic bytes of one decode: union of kept KV per (seq, KV head), all block
    statistics, the S/z/m state (the count the target names), split by kernel."""
    G = w.group
    esz = 2 if w.dtype == "bf16" else 4
    kv = stats = state = 0
    for b in range(w.batch):
        nb = -(-int(lens[b]) // w.block_size)
        for h in range(w.num_kv_heads):
            u = np.unique(sel[b, h * G:(h + 1) * G])
            u = u[u >= 0]
            for j in u:
                n = min(w.block_size, int(lens[b]) - int(j) * w.block_size)
                kv += 2 * n * w.head_dim * esz
            stats += nb * 2 * w.head_dim * 4
            state += (w.head_dim * w.head_dim + 2 * w.head_dim) * 4
    return {"kv": kv, "stats": stats, "state": state, "total": kv + stats + state}


# Kernel of each profiled phase, and the source file that defines it.
KERNELS = {"score": ("score_kernel", "score_select.cu"),
           "select": ("select_kernel", "score_select.cu"),
           "decode": ("decode_mma_kernel", "decode.cu"),
           "combine": ("combine_kernel", "decode.cu")}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.txt")


def source_digest(fname: str) -> str:
    """sha256/16 of a kernel source with its comments and blank lines removed: a capture
    stays valid across comment edits, and only across those."""
    import hashlib
    import re
    path = os.path.join(ROOT, "block_sparse_linear_b200", "csrc", fname)
    with open(path) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    code = "\n".join(ln.rstrip() for ln in src.splitlines() if ln.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def measured_traffic(workload: str, context: int, phase: str):
    """DRAM bytes (read + write) per launch of a phase's kernel, from an ncu capture
    recorded in profiles/dram_traffic.txt; None unless that capture was taken on this
    workload and on the kernel's current source."""
    kname, fname = KERNELS[phase]
    try:
        digest = source_digest(fname)
        with open(TRAFFIC_FILE) as f:
            for line in f:
                parts = line.split()
                if len(parts) != 6 or line.startswith("#"):
                    continue
                wl, ctx, kn, fn, dg, nbytes = parts
                if (wl, int(ctx), kn, fn, dg) == (workload, context, kname, fname, digest):
                    return int(float(nbytes))
    except (OSError, ValueError):
        return None
    return None


def workload_of(args):
    from workloads import gen
    if args.context > 0:
        w = gen.get(args.workload)
        return gen.scaled(args.workload, (args.context,) * w.batch, name=w.name)
    return gen.get(args.workload)


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(vals, dev):
    """Element-wise max over all ranks of a list of floats (one all-reduce; the
    identity without an initialised process group). Every rank must call it."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_value(world: int, units_per_step: int, steps: int, t_ms: float) -> float:
    """Whole-job throughput: every rank processes its own batch of units each step."""
    return world * units_per_step * steps / (t_ms / 1e3)


# ----------------------------------------------------------------------------- our arm
def measure(w, K, W, dev, stream, flush, rank_sync, with_e2e=True):
    """Time K append + decode steps of workload w (after W warm-up steps): pass A gives the
    whole-step CUDA-event time (the value); pass B zeroes the workspace's device timestamps
    before every step and reads them after it (first CTA past its wait to last CTA exit, per
    kernel of the decode chain), which leaves the chain's programmatic overlap untouched."""
    import torch

    from workloads import feed_gpu

    cache = feed_gpu.build_cache(w, device=dev)
    steps = [feed_gpu.step_inputs(w, s, device=dev) for s in range(W + 2 * K)]
    gamma = torch.ones((w.num_q_heads, w.head_dim), dtype=torch.float32, device=dev)
    out = torch.empty((w.batch, w.num_q_heads, w.head_dim), dtype=steps[0][2].dtype, device=dev)
    sels = torch.empty((2 * K, w.batch, w.num_q_heads, w.top_k + w.n_sink + w.n_local),
                       dtype=torch.int32, device=dev)
    ones = torch.ones((w.batch,), dtype=torch.int32, device=dev)    # one new token per sequence

    def step(s, sel=None):
        k, v, q = steps[s]
        cache.append(k, v, ones)
        cache.decode(q, gamma, out, sel)

    for s in range(W):
        step(s)
    torch.cuda.synchronize(dev)
    rank_sync()

    # ---- pass A: whole-step time (the value)
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    lens0 = cache.context_lens.cpu().numpy().copy()
    with ClockSampler(dev.index or 0) as clk:
        torch.cuda.synchronize(dev)
        rank_sync()
        for i in range(K):
            flush()
            ev0[i].record(stream)
            step(W + i, sels[i])
            ev1[i].record(stream)
        torch.cuda.synchronize(dev)
        rank_sync()
    t_steps = [ev0[i].elapsed_time(ev1[i]) for i in range(K)]

    # ---- pass B: per-kernel device timestamps of the pipelined chain
    from block_sparse_linear_b200 import _lib
    stamps = torch.empty((K, 4, 256, 2), dtype=torch.int64, device=dev)
    st_view = cache.stamps()
    _lib.spla_profile_stamps(True)
    for i in range(K):
        flush()
        st_view.zero_()
        step(W + K + i, sels[K + i])
        stamps[i].copy_(st_view)
    _lib.spla_profile_stamps(False)
    torch.cuda.synchronize(dev)
    st = stamps.cpu().numpy().view(np.uint64)
    # per kernel: the earliest first-CTA time and the latest exit over the SM slots
    first = (~st[:, :, :, 0].max(axis=2)).astype(np.float64)   # ns of the first CTA past its wait
    last = st[:, :, :, 1].max(axis=2).astype(np.float64)
    kt = (last - first) / 1e6                            # ms per kernel: score, select, decode, combine
    chain = (last[:, 3] - first[:, 0]) / 1e6             # scoring's first CTA to the combine's last

    sel_np = sels.cpu().numpy()
    lens_a = lens0 + 1 + np.arange(K)[:, None]           # each step appends one token first
    by_a = [step_bytes(w, sel_np[i], lens_a[i]) for i in range(K)]
    lens_b = lens0 + K + 1 + np.arange(K)[:, None]
    by_b = [step_bytes(w, sel_np[K + i], lens_b[i]) for i in range(K)]
    res = {"t_steps": t_steps, "kt": kt, "chain_ms": chain, "by_a": by_a, "by_b": by_b,
           "status": cache.status(), "clocks": clk.summary()}
    if with_e2e:
        res["e2e"] = e2e_pass(w, cache, steps, W + 2 * K, K, gamma, flush, dev, stream, ones)
    del cache
    torch.cuda.empty_cache()
    return res


KERNEL_NAMES = ["score", "select", "decode", "combine"]


def summarise(w, m, K, t_ms_total, hbm, peak_kind, world):
    """Throughput and roofline figures of one measured workload."""
    kt = m["kt"]
    share = kt.sum(axis=0) / kt.sum()
    dom = int(np.argmax(share))
    dec_bytes = float(np.mean([b["kv"] for b in m["by_b"]]))
    sco_bytes = float(np.mean([b["stats"] + b["state"] for b in m["by_b"]]))
    dom_bytes = dec_bytes if dom == 2 else (sco_bytes if dom == 0 else 0.0)
    dom_ms = float(np.mean(kt[:, dom]))
    achieved = dom_bytes / (dom_ms / 1e3) / 1e9
    step_bytes_mean = float(np.mean([b["total"] for b in m["by_a"]]))
    step_gbs = step_bytes_mean / (t_ms_total / K / 1e3) / 1e9
    chain_ms = float(np.mean(m["chain_ms"]))
    chain_gbs = float(np.mean([b["total"] for b in m["by_b"]])) / (chain_ms / 1e3) / 1e9
    return {
        "dom": dom, "dom_bytes": dom_bytes, "dom_ms": dom_ms, "achieved": achieved,
        "value": job_value(world, w.batch * w.num_q_heads, K, t_ms_total),
        "roofline": {"bound": "hbm", "kernel": KERNEL_NAMES[dom], "achieved": round(achieved, 1),
                     "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                     "traffic": measured_traffic(w.name, int(w.context_lens[0]), KERNEL_NAMES[dom]),
                     "peak_kind": f"{peak_kind} hbm_gbs",
                     "bytes_per_launch": int(dom_bytes), "ms_per_launch": round(dom_ms, 5),
                     "timing": "device timestamps: first CTA past its dependency wait to last "
                               "CTA exit, in the pipelined step"},
        "step_roofline": {"bytes_per_step": int(step_bytes_mean),
                          "kv_bytes": int(np.mean([b["kv"] for b in m["by_a"]])),
                          "stats_bytes": int(np.mean([b["stats"] for b in m["by_a"]])),
                          "state_bytes": int(np.mean([b["state"] for b in m["by_a"]])),
                          "achieved_gbs": round(step_gbs, 1),
                          "frac_of_measured_peak": round(step_gbs / hbm, 4),
                          "frac_of_nominal_8tbs": round(step_gbs / 8000.0, 4),
                          "decode_chain_ms": round(chain_ms, 5),
                          "decode_chain_gbs": round(chain_gbs, 1),
                          "decode_chain_frac_of_measured_peak": round(chain_gbs / hbm, 4)},
        "kernels_ms": {n: round(float(np.mean(kt[:, j])), 5) for j, n in enumerate(KERNEL_NAMES)},
        "kernel_share": {n: round(float(share[j]), 4) for j, n in enumerate(KERNEL_NAMES)},
    }


def run_ours(args):
    import torch
    import torch.distributed as dist

    from workloads import gen

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def rank_sync():
        if world > 1:
            dist.barrier()

    w = workload_of(args)
    K, W = args.steps, args.warmup
    stream = torch.cuda.current_stream(dev)
    flush = L2Flush(dev)
    m = measure(w, K, W, dev, stream, flush, rank_sync, with_e2e=not args.no_e2e)
    t_total = sum(m["t_steps"])
    # the other target workload (1M tokens), measured on the same box; every rank takes part
    extra = None
    if args.also and args.also != w.name:
        wx = gen.get(args.also)
        Kx = min(K, 16)
        mx = measure(wx, Kx, W, dev, stream, flush, rank_sync, with_e2e=False)
        extra = (wx, mx, Kx)

    prefill = measure_prefill("cfg4", dev, stream, flush) if not args.no_prefill else None
    sharded = measure_sharded(w, args.shards, K, W, dev, stream, flush) if args.shards > 0 else None
    bcausal = measure_block_causal(dev, stream, flush) if not args.no_block_causal else None

    # ---- max over ranks (the same single collective on every rank)
    t_max, e2e_ms, tx_max = max_over_ranks(
        [t_total, m["e2e"]["ms"] if "e2e" in m else 0.0,
         sum(extra[1]["t_steps"]) if extra else 0.0], dev)

    if rank == 0:
        hbm, peak_kind = peaks()
        sm = summarise(w, m, K, t_max, hbm, peak_kind, world)
        res = {
            "metric": METRIC, "value": round(sm["value"], 1), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": round(t_max / K, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic (seeded, workloads/gen.py)",
            "config": {"workload": gen.DESCRIPTIONS[w.name], "name": w.name, "batch": w.batch,
                       "context": int(w.context_lens[0]), "q_heads": w.num_q_heads,
                       "kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
                       "block": w.block_size, "top_k": w.top_k,
                       "step": "spla_append_kv (1 token/seq) + spla_decode",
                       "l2": "flushed (512 MiB read) before every timed step, outside the events",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "roofline": sm["roofline"],
            "step_hbm": sm["step_roofline"],
            "kernels_ms": sm["kernels_ms"],
            "kernel_share": sm["kernel_share"],
            "clocks": m["clocks"],
            # per step: append, length advance, scoring, selection, decode, combine
            "gpu_launches": 6 * K,
            "dev_status": m["status"],
        }
        if "e2e" in m:
            e = m["e2e"]
            res["e2e"] = {"value": round(job_value(world, w.batch * w.num_q_heads, K, e2e_ms), 1),
                          "unit": UNIT, "h2d_bytes_per_step": e["h2d"],
                          "d2h_bytes_per_step": e["d2h"]}
        if extra:
            wx, mx, Kx = extra
            sx = summarise(wx, mx, Kx, tx_max, hbm, peak_kind, world)
            res[f"also_{wx.name}"] = {
                "workload": gen.DESCRIPTIONS[wx.name], "steps": Kx,
                "ms_per_step": round(tx_max / Kx, 5), "value": round(sx["value"], 1),
                "unit": UNIT, "roofline": sx["roofline"], "step_hbm": sx["step_roofline"],
                "kernels_ms": sx["kernels_ms"], "dev_status": mx["status"],
                "clocks": mx["clocks"]}
        if sharded:
            res["sharded_emulation"] = sharded
        if bcausal:
            res["block_causal"] = bcausal
        if prefill:
            hbm_p = hbm
            prefill["bulk"]["frac_of_measured_peak" if peak_kind == "measured"
                            else "frac_of_fallback_peak"] = round(
                prefill["bulk"]["achieved_gbs"] / hbm_p, 4)
            res["bulk_append"] = prefill
        if not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(res), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def measure_prefill(name, dev, stream, flush, n_tok=65536, K=4, W=3):
    """Bulk append of one n_tok-token chunk per sequence of workload `name`'s shape, through
    spla_append_kv_bulk and through the one-token kernel path (spla_append_kv), each chunk
    timed alone with CUDA events after an L2 flush. Algorithmic bytes per chunk: the new
    K and V read once and written once into the pool, the touched blocks' statistics, and
    S, z, m read and written once."""
    import torch
    from block_sparse_linear_b200 import SplaDecodeCache
    from workloads import feed_gpu, gen
    w = gen.get(name)
    cfg = feed_gpu.config_of(w)
    hkv, d, bs, batch = w.num_kv_heads, w.head_dim, w.block_size, w.batch
    mbp = (W + K) * n_tok // bs + 2
    table = torch.arange(batch * mbp, dtype=torch.int32).reshape(batch, mbp)
    g = torch.Generator(device=dev).manual_seed(5)
    k = torch.randn((batch, n_tok, hkv, d), device=dev, generator=g).to(cfg.torch_dtype)
    v = torch.randn((batch, n_tok, hkv, d), device=dev, generator=g).to(cfg.torch_dtype)
    esz = k.element_size()
    kv = 2 * batch * n_tok * hkv * d * esz
    blocks = batch * hkv * (n_tok // bs + 1)
    by = 2 * kv + blocks * 2 * d * 4 + 2 * batch * hkv * (d * d + 2 * d) * 4
    out = {"workload": f"append of {n_tok} tokens per sequence, batch {batch}, {hkv} KV heads, "
                       f"d {d}, block {bs}, {w.dtype}", "chunks": K, "warmup": W,
           "l2": "flushed before every chunk", "bytes_per_chunk": by}
    for bulk in (True, False):
        cache = SplaDecodeCache(cfg, batch, table, batch * mbp, device=dev)
        ts = []
        for i in range(W + K):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            cache.append(k, v, bulk=bulk)
            e1.record(stream)
            e1.synchronize()
            if i >= W:
                ts.append(e0.elapsed_time(e1))
        ms = float(np.median(ts))
        key = "bulk" if bulk else "one_token_path"
        out[key] = {"ms_per_chunk": round(ms, 5),
                    "tokens_per_s": round(batch * n_tok / (ms * 1e-3), 1),
                    "dev_status": cache.status()}
        if bulk:
            out[key]["achieved_gbs"] = round(by / (ms * 1e-3) / 1e9, 1)
        del cache
    out["speedup"] = round(out["one_token_path"]["ms_per_chunk"] / out["bulk"]["ms_per_chunk"], 1)
    torch.cuda.empty_cache()
    return out


def measure_sharded(w, nshards, K, W, dev, stream, flush):
    """The context-sharded decode with each sequence's blocks split over nshards caches on
    this GPU (shard s holds global blocks [s*bps, (s+1)*bps)). Per step, after an L2 flush,
    CUDA events around every shard's candidates call, every shard's partials call and the
    merge: a rank of an nshards-GPU run would spend one shard's two phases, the merge and
    two all-gathers (not timed here: one GPU)."""
    import math

    import torch
    from block_sparse_linear_b200 import SplaDecodeCache, _lib
    from block_sparse_linear_b200.sharded import rec_doubles
    from workloads import feed_gpu, gen
    cfg = feed_gpu.config_of(w)
    bs, hkv, d, hq, k = w.block_size, w.num_kv_heads, w.head_dim, w.num_q_heads, w.top_k
    nbg = [math.ceil(L / bs) for L in w.context_lens]
    bps = math.ceil(max(nbg) / nshards)
    span = bps * bs
    shards = []
    for s in range(nshards):
        table = torch.arange(w.batch * bps, dtype=torch.int32).reshape(w.batch, bps)
        shards.append((SplaDecodeCache(cfg, w.batch, table, w.batch * bps, device=dev), s * bps))
    ct, dt = gen.CHUNK_TOKENS, cfg.torch_dtype
    for c, chunk in gen.iter_prefix(w):
        t0 = c * ct
        for s, (cache, _) in enumerate(shards):
            lo, hi = max(s * span, t0), min((s + 1) * span, t0 + ct)
            if lo >= hi:
                continue
            parts = [(K[lo - t0:hi - t0], V[lo - t0:hi - t0]) for K, V in chunk]
            counts = [int(p[0].shape[0]) for p in parts]
            if max(counts) == 0:
                continue
            hk = torch.zeros((w.batch, max(counts), hkv, d), dtype=dt)
            hv = torch.zeros_like(hk)
            for b, (Kp, Vp) in enumerate(parts):
                hk[b, :len(Kp)] = torch.from_numpy(Kp).to(dt)
                hv[b, :len(Vp)] = torch.from_numpy(Vp).to(dt)
            cache.append(hk.to(dev), hv.to(dev), torch.tensor(counts, dtype=torch.int32,
                                                              device=dev))
    torch.cuda.synchronize(dev)
    q = torch.from_numpy(gen.query(w, 0)).to(dt).to(dev)
    gamma = torch.ones((hq, d), dtype=torch.float32, device=dev)
    gnb = torch.tensor(nbg, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    cand = torch.empty((nshards, w.batch, hq, k, 2), dtype=torch.int32, device=dev)
    part = torch.empty((nshards, w.batch, hq, rec_doubles(d)), dtype=torch.float64, device=dev)
    st = stream.cuda_stream

    def step(evs=None):
        rec = (lambda i: evs[i].record(stream)) if evs else (lambda i: None)
        for i, (cache, first) in enumerate(shards):
            rec(i)
            _lib.spla_shard_candidates(cache.params, cache.c, first, gnb.data_ptr(), q.data_ptr(),
                                       cand[i].data_ptr(), cache.workspace.data_ptr(),
                                       cache.ws_bytes, cache.dev_status.data_ptr(), st)
        for i, (cache, first) in enumerate(shards):
            rec(nshards + i)
            _lib.spla_shard_partials(cache.params, cache.c, first, gnb.data_ptr(), q.data_ptr(),
                                     cand.data_ptr(), nshards, part[i].data_ptr(),
                                     cache.workspace.data_ptr(), cache.ws_bytes,
                                     cache.dev_status.data_ptr(), st)
        rec(2 * nshards)
        _lib.spla_shard_merge(shards[0][0].params, w.batch, part.data_ptr(), nshards,
                              gamma.data_ptr(), out.data_ptr(), 0, 0,
                              shards[0][0].dev_status.data_ptr(), st)
        rec(2 * nshards + 1)

    for _ in range(W):
        step()
    torch.cuda.synchronize(dev)
    cand_ms, part_ms, merge_ms = [], [], []
    for _ in range(K):
        flush()
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * nshards + 2)]
        step(evs)
        torch.cuda.synchronize(dev)
        t = [evs[i].elapsed_time(evs[i + 1]) for i in range(2 * nshards + 1)]
        cand_ms += t[:nshards]
        part_ms += t[nshards:2 * nshards]
        merge_ms.append(t[2 * nshards])
    status = 0
    for cache, _ in shards:
        status |= cache.status()
    res = {"shards": nshards, "blocks_per_shard": bps, "steps": K, "warmup": W,
           "l2": "flushed before every step",
           "candidates_ms_per_shard": round(float(np.median(cand_ms)), 5),
           "partials_ms_per_shard": round(float(np.median(part_ms)), 5),
           "merge_ms": round(float(np.median(merge_ms)), 5),
           "one_rank_ms": round(float(np.median(cand_ms) + np.median(part_ms) +
                                      np.median(merge_ms)), 5),
           "dev_status": status,
           "not_timed": "the two all-gathers (NCCL) between the phases: one GPU"}
    del shards
    torch.cuda.empty_cache()
    return res


def measure_block_causal(dev, stream, flush, n_tok=8192, K=5, W=3, loop_positions=256):
    """The block-causal forward of one n_tok-token sequence with the 128K workload's heads
    (32 q / 8 kv, d 128, block 64, top-k 32, bf16): spla_block_causal_forward on a cache
    that holds the sequence (CUDA events, L2 flushed before each run), and, for
    comparison, the same outputs as one-token appends and decodes with a local block,
    timed over the sequence's last loop_positions positions and scaled to tokens/s."""
    import torch
    from block_sparse_linear_b200 import SplaConfig, SplaDecodeCache
    hq, hkv, d, bs, k = 32, 8, 128, 64, 32
    nb = -(-n_tok // bs)
    g = torch.Generator(device=dev).manual_seed(9)
    rnd = lambda *shape: torch.randn(shape, device=dev, generator=g).to(torch.bfloat16)
    kk, vv, qq = rnd(1, n_tok, hkv, d), rnd(1, n_tok, hkv, d), rnd(1, n_tok, hq, d)
    cfg = SplaConfig(num_q_heads=hq, num_kv_heads=hkv, head_dim=d, block_size=bs, top_k=k)
    table = torch.arange(nb, dtype=torch.int32).reshape(1, nb)
    cache = SplaDecodeCache(cfg, 1, table, nb, device=dev)
    cache.append(kk, vv)
    out = torch.empty_like(qq)
    ts = []
    for i in range(W + K):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cache.block_causal_forward(kk, vv, qq, None, out)
        e1.record(stream)
        e1.synchronize()
        if i >= W:
            ts.append(e0.elapsed_time(e1))
    ms = float(np.median(ts))
    status = cache.status()
    del cache
    # the per-position path: one-token append + decode with the current block as local block
    cfgl = SplaConfig(num_q_heads=hq, num_kv_heads=hkv, head_dim=d, block_size=bs, top_k=k,
                      n_local=1)
    cl = SplaDecodeCache(cfgl, 1, table, nb, device=dev)
    o1 = torch.empty((1, hq, d), dtype=torch.bfloat16, device=dev)
    n0 = n_tok - loop_positions - W                  # the last positions: the longest contexts
    cl.append(kk[:, :n0].contiguous(), vv[:, :n0].contiguous())
    for t in range(n0, n0 + W):
        cl.append(kk[:, t:t + 1].contiguous(), vv[:, t:t + 1].contiguous())
        cl.decode(qq[:, t].contiguous(), None, o1)
    steps = [(kk[:, t:t + 1].contiguous(), vv[:, t:t + 1].contiguous(), qq[:, t].contiguous())
             for t in range(n0 + W, n_tok)]
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for kt, vt, qt in steps:
        cl.append(kt, vt)
        cl.decode(qt, None, o1)
    e1.record(stream)
    e1.synchronize()
    loop_ms = e0.elapsed_time(e1) / loop_positions
    del cl
    torch.cuda.empty_cache()
    return {"workload": f"block-causal forward of one {n_tok}-token sequence, {hq} q / {hkv} kv "
                        f"heads, d {d}, block {bs}, top-k {k}, bf16",
            "runs": K, "warmup": W, "l2": "flushed before every run",
            "ms_per_sequence": round(ms, 4), "tokens_per_s": round(n_tok / (ms * 1e-3), 1),
            "dev_status": status,
            "per_position_loop": {"positions_timed": loop_positions,
                                  "ms_per_position": round(loop_ms, 5),
                                  "tokens_per_s": round(1.0 / (loop_ms * 1e-3), 1)},
            "speedup": round(loop_ms * n_tok / ms, 1)}


def e2e_pass(w, cache, steps, s0, K, gamma, flush, dev, stream, ones):
    """Per step: one pinned host -> device copy of the step's (k, v, q), packed back to back,
    append + decode on views of the device copy, device -> host of out."""
    import torch
    from workloads import gen
    dt = steps[0][2].dtype
    shapes = [tuple(t.shape) for t in steps[0]]
    sizes = [int(np.prod(sh)) for sh in shapes]
    host = []
    for i in range(K):
        k, v = gen.step_tokens(w, s0 + i)
        q = gen.query(w, s0 + i)
        flat = [torch.from_numpy(np.ascontiguousarray(a)).to(dt).reshape(-1)
                for a in (k[:, None], v[:, None], q)]
        host.append(torch.cat(flat).pin_memory())
    dbuf = torch.empty(sum(sizes), dtype=dt, device=dev)
    offs = np.cumsum([0] + sizes)
    dk, dv, dq = (dbuf[offs[j]:offs[j + 1]].view(shapes[j]) for j in range(3))
    out = torch.empty_like(dq)
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    torch.cuda.synchronize(dev)
    for i in range(K):
        flush()
        e0[i].record(stream)
        dbuf.copy_(host[i], non_blocking=True)
        cache.append(dk, dv, ones)
        cache.decode(dq, gamma, out)
        hout.copy_(out, non_blocking=True)
        e1[i].record(stream)
    torch.cuda.synchronize(dev)
    ms = sum(e0[i].elapsed_time(e1[i]) for i in range(K))
    h2d = host[0].numel() * host[0].element_size()
    return {"ms": ms, "h2d": h2d, "d2h": hout.numel() * hout.element_size()}


# ----------------------------------------------------------------------------- oracle (CPU)
def _threads():
    """Threads of the BLAS pool numpy uses (the oracle's only multi-threaded part)."""
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return 1


def oracle_sample(w, budget_s: float, steps: int = None):
    """Time the oracle's decode (score, select, exact attention, RLA, combine) plus its
    one-token append, on one (sequence, KV head) group of the workload: the G query
    heads of that group are the units. Returns (units/s, units, seconds, description)."""
    from oracle import feed as ofeed
    from workloads import gen
    oc = ofeed.build(w, groups=[(0, 0)])
    gamma = gen.gamma(w)
    units, t_spent, n = 0, 0.0, 0
    # every step appends one token: stay inside the capacity reserved past the prefix
    cap = w.extra_tokens
    while n < cap and ((steps is None and t_spent < budget_s) or (steps is not None and n < steps)):
        k, v = gen.step_tokens(w, n)
        q = gen.query(w, n)
        t0 = time.perf_counter()
        oc.append_group(0, 0, k[0, 0][None], v[0, 0][None])
        oc.decode(q, gamma)
        t_spent += time.perf_counter() - t0
        units += w.group
        n += 1
    desc = (f"oracle append(1 token) + decode of sequence 0, KV head 0 ({w.group} query heads) "
            f"of the workload, {n} steps, {t_spent:.1f} s")
    return units / t_spent, units, t_spent, desc, n


def cpu_baseline(w):
    """The oracle on the host cores, twice: BLAS limited to one thread, and at the default
    pool. numpy runs the oracle's element-wise work on one thread in both; only its matrix
    products use the pool, so the headline figure states the pool's size, not nproc."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        v1, u1, s1, d1, n1 = oracle_sample(w, budget_s=6.0)
    vm, um, sm_, dm, nm = oracle_sample(w, budget_s=6.0)
    return {"value": round(vm, 2), "unit": UNIT, "cores": _threads(), "kind": "oracle",
            "sample": dm, "threads_max": {"value": round(vm, 2), "blas_threads": _threads()},
            "threads_1": {"value": round(v1, 2), "blas_threads": 1, "sample": d1},
            "nproc": os.cpu_count(),
            "parallelism": "numpy: matrix products on the BLAS pool, everything else one thread; "
                           "the oracle decodes one (sequence, KV head) group at a time"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from workloads import gen
    w = workload_of(args)
    if args.warmup > 0:
        oracle_sample(w, 0.0, steps=args.warmup)              # warm-up (untimed)
    v, units, secs, desc, n = oracle_sample(w, 0.0, steps=max(1, args.steps))
    res = {"impl": "reference", "metric": METRIC, "value": round(v, 2), "unit": UNIT,
           "n_gpus": 0, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(secs / n * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded, workloads/gen.py)",
           "config": {"workload": gen.DESCRIPTIONS[w.name], "name": w.name},
           "cpu_baseline": {"value": round(v, 2), "unit": UNIT, "cores": _threads(),
                            "kind": "oracle", "sample": desc, "nproc": os.cpu_count(),
                            "parallelism": "numpy: matrix products on the BLAS pool "
                                           f"({_threads()} threads), everything else one thread"},
           "e2e": {"value": round(v, 2), "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
