"""Context-sharded decode: the shards of one sequence's blocks, each a SplaDecodeCache
holding global blocks [first_block, first_block + max_blocks_per_seq), run the three
phases of include/spla.h's spla_shard_* calls with two all-gathers between them.

`gather(t)` turns this process's stacked per-shard tensor [n_local, ...] into the
stack over every shard [n_total, ...] in global shard order. The default keeps it
as it is (every shard in this process, on one device); `dist_gather` does it with
torch.distributed (NCCL between GPUs, one shard per rank). The binding only
marshals arguments: every step runs in the library's kernels.
"""
import torch

from . import _lib

REC_EXTRA = 8


def rec_doubles(d: int) -> int:
    """fp64 words of one (sequence, query head) record of spla_shard_partials."""
    return REC_EXTRA + 2 * d


def dist_gather(t: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of [n_local, ...] over the process group, ranks in order (every rank
    holds the same number of shards)."""
    import torch.distributed as dist
    ws = dist.get_world_size(group)
    out = torch.empty((ws * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    dist.all_gather_into_tensor(out, t.contiguous(), group=group)
    return out


def _stream(dev, stream):
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    return s.cuda_stream


def decode_sharded(shards, q: torch.Tensor, global_nb: torch.Tensor, gamma: torch.Tensor = None,
                   out: torch.Tensor = None, o_sparse: torch.Tensor = None,
                   o_rla: torch.Tensor = None, gather=None, stream=None) -> torch.Tensor:
    """shards: [(SplaDecodeCache, first_block)] held by this process, all on q's device.
    global_nb: [batch] int32, each sequence's total block count. Returns out."""
    gather = gather or (lambda t: t)
    c0 = shards[0][0]
    cfg, batch, dev = c0.cfg, c0.batch, q.device
    assert q.is_contiguous() and q.dtype == cfg.torch_dtype
    assert global_nb.dtype == torch.int32 and global_nb.device == dev
    hq, d, k = cfg.num_q_heads, cfg.head_dim, cfg.top_k
    st = _stream(dev, stream)
    cand = torch.empty((len(shards), batch, hq, k, 2), dtype=torch.int32, device=dev)
    for i, (cache, first) in enumerate(shards):
        _lib.spla_shard_candidates(cache.params, cache.c, first, global_nb.data_ptr(),
                                   q.data_ptr(), cand[i].data_ptr(), cache.workspace.data_ptr(),
                                   cache.ws_bytes, cache.dev_status.data_ptr(), st)
    cand_all = gather(cand).contiguous()
    nshards = int(cand_all.shape[0])
    part = torch.empty((len(shards), batch, hq, rec_doubles(d)), dtype=torch.float64, device=dev)
    for i, (cache, first) in enumerate(shards):
        _lib.spla_shard_partials(cache.params, cache.c, first, global_nb.data_ptr(), q.data_ptr(),
                                 cand_all.data_ptr(), nshards, part[i].data_ptr(),
                                 cache.workspace.data_ptr(), cache.ws_bytes,
                                 cache.dev_status.data_ptr(), st)
    part_all = gather(part).contiguous()
    if out is None:
        out = torch.empty_like(q)
    ptr = lambda t: 0 if t is None else t.data_ptr()
    _lib.spla_shard_merge(c0.params, batch, part_all.data_ptr(), nshards, ptr(gamma),
                          out.data_ptr(), ptr(o_sparse), ptr(o_rla), c0.dev_status.data_ptr(), st)
    return out
