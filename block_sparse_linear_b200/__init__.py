"""SPLA decode on B200: a C-ABI CUDA library (libspla.so) and its Python binding.

``SplaDecodeCache`` holds the device buffers of include/spla.h's ``spla_cache``
(allocated with PyTorch, which is used for device memory and streams only) and
forwards ``append`` / ``decode`` to ``spla_append_kv`` (or ``spla_append_kv_bulk``
for long chunks) / ``spla_decode``. Every
step of the decode path runs in the library's kernels; there is no fallback.
"""
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import (SPLA_BF16, SPLA_F32, SPLA_FLAG_FIRST_ORDER, SPLA_FLAG_NO_RLA,
                   SPLA_WS_STAMP_BYTES, SplaError, spla_append_bulk_workspace_size, spla_append_kv,
                   spla_append_kv_bulk, spla_cache_init, spla_decode, spla_decode_static_workspace,
                   spla_decode_workspace_size)

__all__ = ["SplaConfig", "SplaDecodeCache", "SplaError", "spla_append_bulk_workspace_size",
           "spla_append_kv", "spla_append_kv_bulk", "spla_cache_init", "spla_decode",
           "spla_decode_static_workspace", "spla_decode_workspace_size"]

# Chunks at least this long go through spla_append_kv_bulk where it applies.
BULK_MIN_TOKENS = 64


@dataclass
class SplaConfig:
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    top_k: int
    n_sink: int = 0
    n_local: int = 0
    dtype: str = "bf16"            # "bf16" or "f32"
    softmax_scale: float = 0.0     # <= 0: 1/sqrt(head_dim)
    rms_eps: float = 1e-6
    no_rla: bool = False
    first_order: bool = False

    def params(self) -> _lib.spla_params:
        flags = (SPLA_FLAG_NO_RLA if self.no_rla else 0) | (
            SPLA_FLAG_FIRST_ORDER if self.first_order else 0)
        return _lib.spla_params(self.num_q_heads, self.num_kv_heads, self.head_dim,
                                self.block_size, self.top_k, self.n_sink, self.n_local,
                                SPLA_BF16 if self.dtype == "bf16" else SPLA_F32,
                                self.softmax_scale, self.rms_eps, flags)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def kcap(self) -> int:
        return self.top_k + self.n_sink + self.n_local


class SplaDecodeCache:
    """Device buffers of one paged SPLA cache plus the decode workspace."""

    def __init__(self, cfg: SplaConfig, batch: int, block_table: torch.Tensor,
                 num_phys_blocks: int, device="cuda", stream=None):
        _lib.load()
        self.cfg = cfg
        self.batch = batch
        self.device = torch.device(device)
        dev = self.device
        Hkv, d, B = cfg.num_kv_heads, cfg.head_dim, cfg.block_size
        self.block_table = block_table.to(device=dev, dtype=torch.int32).contiguous()
        assert self.block_table.shape[0] == batch
        self.max_blocks_per_seq = int(self.block_table.shape[1])
        self.num_phys_blocks = int(num_phys_blocks)
        self.k_pool = torch.empty((num_phys_blocks, Hkv, B, d), dtype=cfg.torch_dtype, device=dev)
        self.v_pool = torch.empty_like(self.k_pool)
        self.blk_stats = torch.zeros((batch, Hkv, self.max_blocks_per_seq, 2, d),
                                     dtype=torch.float32, device=dev)
        self.S = torch.empty((batch, Hkv, d, d), dtype=torch.float32, device=dev)
        self.z = torch.empty((batch, Hkv, d), dtype=torch.float32, device=dev)
        self.m = torch.empty((batch, Hkv, d), dtype=torch.float32, device=dev)
        self.context_lens = torch.empty((batch,), dtype=torch.int32, device=dev)
        self.dev_status = torch.zeros((1,), dtype=torch.int32, device=dev)
        self.params = cfg.params()
        self.c = _lib.spla_cache(self.k_pool.data_ptr(), self.v_pool.data_ptr(),
                                 self.blk_stats.data_ptr(), self.S.data_ptr(), self.z.data_ptr(),
                                 self.m.data_ptr(), self.block_table.data_ptr(),
                                 self.context_lens.data_ptr(), batch, self.max_blocks_per_seq,
                                 self.num_phys_blocks)
        self.ws_bytes = spla_decode_workspace_size(self.params, batch, self.max_blocks_per_seq)
        self.workspace = torch.zeros((self.ws_bytes + 255) // 256 * 256, dtype=torch.uint8,
                                     device=dev)
        self._n_new = torch.zeros((batch,), dtype=torch.int32, device=dev)
        self._bulk_ws = None
        self._bc_ws = None
        spla_cache_init(self.params, self.c, self._stream(stream))

    def _stream(self, stream=None) -> int:
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        return s.cuda_stream

    def block_causal_forward(self, k_all: torch.Tensor, v_all: torch.Tensor, q_all: torch.Tensor,
                             gamma: torch.Tensor = None, out: torch.Tensor = None,
                             o_sparse: torch.Tensor = None, o_rla: torch.Tensor = None,
                             stream=None) -> torch.Tensor:
        """The block-causal form over the sequences this cache holds (appended from k_all,
        v_all [batch][max_len][Hkv][d]); q_all [batch][max_len][Hq][d]. Returns out (same
        layout as q_all; rows past a sequence's length are left as they are)."""
        for t in (k_all, v_all, q_all):
            assert t.is_contiguous() and t.dtype == self.cfg.torch_dtype
        max_len = int(q_all.shape[1])
        need = _lib.spla_block_causal_workspace_size(self.params, self.batch, max_len)
        if self._bc_ws is None or self._bc_ws.numel() < need:
            self._bc_ws = torch.empty((need + 255) // 256 * 256, dtype=torch.uint8,
                                      device=self.device)
        if out is None:
            out = torch.zeros_like(q_all)
        ptr = lambda t: 0 if t is None else t.data_ptr()
        _lib.spla_block_causal_forward(self.params, self.c, k_all.data_ptr(), v_all.data_ptr(),
                                       q_all.data_ptr(), max_len, ptr(gamma), out.data_ptr(),
                                       ptr(o_sparse), ptr(o_rla), self._bc_ws.data_ptr(),
                                       self._bc_ws.numel(), self.dev_status.data_ptr(),
                                       self._stream(stream))
        return out

    def bulk_supported(self) -> bool:
        """Whether spla_append_kv_bulk takes this cache's shape (bf16, head_dim 128)."""
        return self.cfg.dtype == "bf16" and self.cfg.head_dim == 128

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, n_new: torch.Tensor = None,
               stream=None, bulk: bool = None) -> None:
        """k_new, v_new: [batch][max_new][Hkv][d] on the device; n_new: [batch] int32 (device).
        bulk: None picks spla_append_kv_bulk for chunks of BULK_MIN_TOKENS or more where the
        shape allows it; True asks for it (SplaError if unsupported); False never uses it."""
        assert k_new.is_contiguous() and v_new.is_contiguous()
        assert k_new.dtype == self.cfg.torch_dtype and v_new.dtype == self.cfg.torch_dtype
        max_new = int(k_new.shape[1])
        if n_new is None:
            self._n_new.fill_(max_new)
            n_new = self._n_new
        if bulk is None:
            bulk = self.bulk_supported() and max_new >= BULK_MIN_TOKENS
        if bulk:
            need = spla_append_bulk_workspace_size(self.params, self.batch, max_new)
            if self._bulk_ws is None or self._bulk_ws.numel() < need:
                self._bulk_ws = torch.empty((max(need, 16) + 255) // 256 * 256,
                                            dtype=torch.uint8, device=self.device)
            spla_append_kv_bulk(self.params, self.c, k_new.data_ptr(), v_new.data_ptr(),
                                n_new.data_ptr(), max_new, self._bulk_ws.data_ptr(),
                                self._bulk_ws.numel(), self.dev_status.data_ptr(),
                                self._stream(stream))
            return
        spla_append_kv(self.params, self.c, k_new.data_ptr(), v_new.data_ptr(), n_new.data_ptr(),
                       max_new, self.dev_status.data_ptr(), self._stream(stream))

    def decode(self, q: torch.Tensor, gamma: torch.Tensor = None, out: torch.Tensor = None,
               sel_idx: torch.Tensor = None, o_sparse: torch.Tensor = None,
               o_rla: torch.Tensor = None, stream=None) -> torch.Tensor:
        """q: [batch][Hq][d] on the device. Returns out (same dtype)."""
        assert q.is_contiguous() and q.dtype == self.cfg.torch_dtype
        if out is None:
            out = torch.empty_like(q)
        ptr = lambda t: 0 if t is None else t.data_ptr()
        spla_decode(self.params, self.c, q.data_ptr(), ptr(gamma), out.data_ptr(), ptr(sel_idx),
                    ptr(o_sparse), ptr(o_rla), self.workspace.data_ptr(), self.ws_bytes,
                    self.dev_status.data_ptr(), self._stream(stream))
        return out

    def decode_static_workspace(self, q: torch.Tensor, gamma: torch.Tensor = None,
                                out: torch.Tensor = None, sel_idx: torch.Tensor = None,
                                o_sparse: torch.Tensor = None, o_rla: torch.Tensor = None,
                                stream=None) -> torch.Tensor:
        """decode() through spla_decode_static_workspace: the library's built-in scratch
        instead of this object's workspace, for callers that cannot allocate per call."""
        assert q.is_contiguous() and q.dtype == self.cfg.torch_dtype
        if out is None:
            out = torch.empty_like(q)
        ptr = lambda t: 0 if t is None else t.data_ptr()
        spla_decode_static_workspace(self.params, self.c, q.data_ptr(), ptr(gamma), out.data_ptr(),
                                     ptr(sel_idx), ptr(o_sparse), ptr(o_rla),
                                     self.dev_status.data_ptr(), self._stream(stream))
        return out

    def new_outputs(self, debug: bool = True):
        """Preallocated output tensors for decode(): out, sel_idx, o_sparse, o_rla."""
        c, dev = self.cfg, self.device
        out = torch.empty((self.batch, c.num_q_heads, c.head_dim), dtype=c.torch_dtype, device=dev)
        sel = torch.empty((self.batch, c.num_q_heads, c.kcap), dtype=torch.int32, device=dev)
        osp = orl = None
        if debug:
            osp = torch.empty((self.batch, c.num_q_heads, c.head_dim), dtype=torch.float32,
                              device=dev)
            orl = torch.empty_like(osp)
        return out, sel, osp, orl

    def scores(self) -> torch.Tensor:
        """The last decode's block scores, fp32 [batch][Hq][max_blocks_per_seq] (a view of the
        workspace, whose rows are max_blocks_per_seq rounded up to 4 floats apart; valid after
        the stream has reached the end of that decode)."""
        ld = (self.max_blocks_per_seq + 3) // 4 * 4           # rows padded to 16 bytes
        n = self.batch * self.cfg.num_q_heads * ld
        off = SPLA_WS_STAMP_BYTES
        return self.workspace[off:off + 4 * n].view(torch.float32).view(
            self.batch, self.cfg.num_q_heads, ld)[:, :, :self.max_blocks_per_seq]

    def stamps(self) -> torch.Tensor:
        """Device timestamps of the last decode's kernels (scoring, selection, decode, combine), a
        view of the workspace: uint64 [4][256 SM slots][2] = (~ns of the first CTA past its wait, ns
        of the last CTA's exit), per SM. Zero it (stamps().zero_()) before a call whose times
        you want; the kernel's span is max(~first) to max(last) over the slots."""
        return self.workspace[:SPLA_WS_STAMP_BYTES].view(torch.int64).view(4, 256, 2)

    def status(self) -> int:
        """Device-detected fault bits (synchronises)."""
        return int(self.dev_status.item())
