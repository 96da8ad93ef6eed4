"""The C-ABI library loads, exports what include/spla.h declares, and rejects bad
arguments on the host before any CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest

from block_sparse_linear_b200 import _lib
from workloads import gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000          # never dereferenced: every call below fails its host checks first


def declared_functions():
    with open(os.path.join(ROOT, "include", "spla.h")) as f:
        src = f.read()
    return re.findall(r"SPLA_API\s+[\w\s\*]+?\b(spla_\w+)\s*\(", src)


def test_library_exports_every_declared_function(lib):
    names = declared_functions()
    assert set(names) == set(_lib.EXPORTS), names
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert lib.spla_version() >= 100
    for s in range(6):
        assert lib.spla_status_string(s).decode()
    assert lib.spla_last_cuda_error() == 0


def _params(**kw):
    base = dict(num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=64, top_k=32, n_sink=0,
                n_local=0, dtype=_lib.SPLA_BF16, softmax_scale=0.0, rms_eps=1e-6, flags=0)
    base.update(kw)
    return _lib.spla_params(**base)


def _cache(**kw):
    base = dict(k_pool=FAKE, v_pool=FAKE, blk_stats=FAKE, S=FAKE, z=FAKE, m=FAKE,
                block_table=FAKE, context_lens=FAKE, batch=4, max_blocks_per_seq=2064,
                num_phys_blocks=8256)
    base.update(kw)
    return _lib.spla_cache(**base)


@pytest.mark.parametrize("name", ["cfg1", "cfg2", "cfg3", "cfg4", "cfg5"])
def test_workspace_size_is_deterministic(name):
    w = gen.get(name)
    p = _params(num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                block_size=w.block_size, top_k=w.top_k, n_sink=w.n_sink, n_local=w.n_local,
                dtype=_lib.SPLA_BF16 if w.dtype == "bf16" else _lib.SPLA_F32)
    a = _lib.spla_decode_workspace_size(p, w.batch, w.capacity_blocks)
    b = _lib.spla_decode_workspace_size(p, w.batch, w.capacity_blocks)
    assert a == b and a > 0 and a % 256 == 0
    # scores alone need batch*Hq*mbp floats
    assert a >= w.batch * w.num_q_heads * w.capacity_blocks * 4


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), _lib.SPLA_ERR_UNSUPPORTED),
    (dict(block_size=32), _lib.SPLA_ERR_UNSUPPORTED),
    (dict(num_q_heads=24), _lib.SPLA_ERR_UNSUPPORTED),       # group 3
    (dict(num_q_heads=30), _lib.SPLA_ERR_INVALID_ARG),       # not a multiple
    (dict(top_k=0), _lib.SPLA_ERR_INVALID_ARG),
    (dict(n_sink=-1), _lib.SPLA_ERR_INVALID_ARG),
    (dict(dtype=7), _lib.SPLA_ERR_UNSUPPORTED),
    (dict(flags=0x80), _lib.SPLA_ERR_INVALID_ARG),
])
def test_bad_params_rejected(lib, kw, code):
    p, c = _params(**kw), _cache()
    n = ctypes.c_size_t()
    assert lib.spla_decode_workspace_size(ctypes.byref(p), 4, 100, ctypes.byref(n)) == code
    assert lib.spla_decode(ctypes.byref(p), ctypes.byref(c), FAKE, None, FAKE, None, None, None,
                           FAKE, 1 << 40, None, None) == code
    assert lib.spla_append_kv(ctypes.byref(p), ctypes.byref(c), FAKE, FAKE, FAKE, 1, None,
                              None) == code


def test_bad_cache_and_buffers_rejected(lib):
    p = _params()
    B = ctypes.byref
    for field in ("k_pool", "S", "block_table", "context_lens"):
        c = _cache(**{field: None})
        assert lib.spla_decode(B(p), B(c), FAKE, None, FAKE, None, None, None, FAKE, 1 << 40,
                               None, None) == _lib.SPLA_ERR_INVALID_ARG
        assert lib.spla_cache_init(B(p), B(c), None) == _lib.SPLA_ERR_INVALID_ARG
    c = _cache()
    assert lib.spla_decode(B(p), B(c), None, None, FAKE, None, None, None, FAKE, 1 << 40, None,
                           None) == _lib.SPLA_ERR_INVALID_ARG
    assert lib.spla_decode(B(p), B(c), FAKE, None, None, None, None, None, FAKE, 1 << 40, None,
                           None) == _lib.SPLA_ERR_INVALID_ARG
    # workspace: missing, too small, misaligned
    need = _lib.spla_decode_workspace_size(p, 4, 2064)
    assert lib.spla_decode(B(p), B(c), FAKE, None, FAKE, None, None, None, None, need, None,
                           None) == _lib.SPLA_ERR_WORKSPACE
    assert lib.spla_decode(B(p), B(c), FAKE, None, FAKE, None, None, None, FAKE, need - 1, None,
                           None) == _lib.SPLA_ERR_WORKSPACE
    assert lib.spla_decode(B(p), B(c), FAKE, None, FAKE, None, None, None, FAKE + 16, need,
                           None, None) == _lib.SPLA_ERR_WORKSPACE
    # table wider than the selection kernel supports
    c = _cache(max_blocks_per_seq=_lib.SPLA_MAX_BLOCKS_PER_SEQ + 1)
    assert lib.spla_decode(B(p), B(c), FAKE, None, FAKE, None, None, None, FAKE, 1 << 40, None,
                           None) == _lib.SPLA_ERR_CAPACITY
    # append: negative count bound, missing inputs, more tokens than the table holds
    c = _cache()
    assert lib.spla_append_kv(B(p), B(c), FAKE, FAKE, FAKE, -1, None, None) == \
        _lib.SPLA_ERR_INVALID_ARG
    assert lib.spla_append_kv(B(p), B(c), None, FAKE, FAKE, 4, None, None) == \
        _lib.SPLA_ERR_INVALID_ARG
    assert lib.spla_append_kv(B(p), B(c), FAKE, FAKE, None, 4, None, None) == \
        _lib.SPLA_ERR_INVALID_ARG


def test_python_binding_raises_on_error_codes():
    with pytest.raises(_lib.SplaError) as e:
        _lib.spla_decode_workspace_size(_params(head_dim=100), 1, 1)
    assert e.value.status == _lib.SPLA_ERR_UNSUPPORTED


def test_static_workspace_entry_rejects_oversize_shapes_on_the_host(lib):
    """spla_decode_static_workspace checks its fixed scratch size before any CUDA call."""
    B = ctypes.byref
    p = _params()
    c = _cache(batch=64)
    assert _lib.spla_decode_workspace_size(p, 64, 2064) > _lib.SPLA_STATIC_WORKSPACE_BYTES
    assert lib.spla_decode_static_workspace(B(p), B(c), FAKE, None, FAKE, None, None, None, None,
                                            None) == _lib.SPLA_ERR_CAPACITY
    assert lib.spla_decode_static_workspace(B(p), None, FAKE, None, FAKE, None, None, None, None,
                                            None) == _lib.SPLA_ERR_INVALID_ARG
    bad = _params(head_dim=96)
    assert lib.spla_decode_static_workspace(B(bad), B(_cache()), FAKE, None, FAKE, None, None,
                                            None, None, None) == _lib.SPLA_ERR_UNSUPPORTED
    with pytest.raises(_lib.SplaError) as e:
        _lib.spla_decode_static_workspace(p, c, FAKE, 0, FAKE, 0, 0, 0, 0)
    assert e.value.status == _lib.SPLA_ERR_CAPACITY


def test_decode_rejects_misaligned_buffers(lib):
    """q and the cache buffers the kernels move with bulk copies must be 16-byte aligned."""
    B = ctypes.byref
    p = _params()
    need = _lib.spla_decode_workspace_size(p, 4, 2064)
    assert lib.spla_decode(B(p), B(_cache()), FAKE + 2, None, FAKE, None, None, None, FAKE, need,
                           None, None) == _lib.SPLA_ERR_INVALID_ARG
    for field in ("S", "z", "m", "blk_stats", "k_pool", "v_pool"):
        c = _cache(**{field: FAKE + 4})
        assert lib.spla_decode(B(p), B(c), FAKE, None, FAKE, None, None, None, FAKE, need, None,
                               None) == _lib.SPLA_ERR_INVALID_ARG, field


def test_append_rejects_misaligned_cache_buffers(lib):
    """The append kernels read the pools back with 16-byte loads and the bulk merge moves S
    rows as 16-byte vectors: misaligned pools or S are refused on the host."""
    B = ctypes.byref
    p = _params()
    for field in ("k_pool", "v_pool", "S"):
        c = _cache(**{field: FAKE + 8})
        assert lib.spla_append_kv(B(p), B(c), FAKE, FAKE, FAKE, 4, None, None) == \
            _lib.SPLA_ERR_INVALID_ARG, field
        assert lib.spla_append_kv_bulk(B(p), B(c), FAKE, FAKE, FAKE, 4, FAKE, 1 << 40, None,
                                       None) == _lib.SPLA_ERR_INVALID_ARG, field


def test_bulk_append_host_checks(lib):
    """spla_append_kv_bulk: bf16 and head_dim 128 only, aligned inputs, a large enough
    workspace; its size query is a pure function of its arguments."""
    B = ctypes.byref
    p = _params()
    c = _cache()
    need = _lib.spla_append_bulk_workspace_size(p, 4, 8192)
    assert need == _lib.spla_append_bulk_workspace_size(p, 4, 8192) > 0
    assert _lib.spla_append_bulk_workspace_size(p, 4, 64) <= need
    assert _lib.spla_append_bulk_workspace_size(p, 4, 0) == 0
    for bad, code in ((_params(dtype=_lib.SPLA_F32), _lib.SPLA_ERR_UNSUPPORTED),
                      (_params(head_dim=64, num_q_heads=8, num_kv_heads=2),
                       _lib.SPLA_ERR_UNSUPPORTED)):
        assert lib.spla_append_kv_bulk(B(bad), B(c), FAKE, FAKE, FAKE, 8192, FAKE, need, None,
                                       None) == code
        with pytest.raises(_lib.SplaError) as e:
            _lib.spla_append_bulk_workspace_size(bad, 4, 8192)
        assert e.value.status == code
    # inputs: missing or misaligned
    assert lib.spla_append_kv_bulk(B(p), B(c), None, FAKE, FAKE, 8192, FAKE, need, None,
                                   None) == _lib.SPLA_ERR_INVALID_ARG
    assert lib.spla_append_kv_bulk(B(p), B(c), FAKE, FAKE + 2, FAKE, 8192, FAKE, need, None,
                                   None) == _lib.SPLA_ERR_INVALID_ARG
    assert lib.spla_append_kv_bulk(B(p), B(c), FAKE, FAKE, None, 8192, FAKE, need, None,
                                   None) == _lib.SPLA_ERR_INVALID_ARG
    assert lib.spla_append_kv_bulk(B(p), B(c), FAKE, FAKE, FAKE, -1, FAKE, need, None,
                                   None) == _lib.SPLA_ERR_INVALID_ARG
    # workspace: missing, too small, misaligned
    for ws, nbytes in ((None, need), (FAKE, need - 1), (FAKE + 8, need)):
        assert lib.spla_append_kv_bulk(B(p), B(c), FAKE, FAKE, FAKE, 8192, ws, nbytes, None,
                                       None) == _lib.SPLA_ERR_WORKSPACE


def test_sharded_decode_host_checks(lib):
    """spla_shard_*: missing buffers, a negative first block, a short workspace and too many
    gathered candidates are refused on the host, before any CUDA call."""
    B = ctypes.byref
    p = _params()
    c = _cache()
    need = _lib.spla_decode_workspace_size(p, 4, 2064)
    ok = dict(first=0, gnb=FAKE, q=FAKE, ws=FAKE, n=need)
    args = lambda **kw: {**ok, **kw}

    def cand(**kw):
        a = args(**kw)
        return lib.spla_shard_candidates(B(p), B(c), a["first"], a["gnb"], a["q"], FAKE, a["ws"],
                                         a["n"], None, None)

    def part(nshards=2, **kw):
        a = args(**kw)
        return lib.spla_shard_partials(B(p), B(c), a["first"], a["gnb"], a["q"], FAKE, nshards,
                                       FAKE, a["ws"], a["n"], None, None)

    for f in (cand, part):
        assert f(first=-1) == _lib.SPLA_ERR_INVALID_ARG
        assert f(gnb=None) == _lib.SPLA_ERR_INVALID_ARG
        assert f(q=None) == _lib.SPLA_ERR_INVALID_ARG
        assert f(q=FAKE + 4) == _lib.SPLA_ERR_INVALID_ARG
        assert f(ws=None) == _lib.SPLA_ERR_WORKSPACE
        assert f(n=need - 1) == _lib.SPLA_ERR_WORKSPACE
    assert lib.spla_shard_candidates(B(p), B(c), 0, FAKE, FAKE, None, FAKE, need, None,
                                     None) == _lib.SPLA_ERR_INVALID_ARG
    assert part(nshards=0) == _lib.SPLA_ERR_INVALID_ARG
    assert part(nshards=4096 // p.top_k + 1) == _lib.SPLA_ERR_CAPACITY
    assert lib.spla_shard_merge(B(p), 4, None, 2, None, FAKE, None, None, None,
                                None) == _lib.SPLA_ERR_INVALID_ARG
    assert lib.spla_shard_merge(B(p), 0, FAKE, 2, None, FAKE, None, None, None,
                                None) == _lib.SPLA_ERR_INVALID_ARG


def test_block_causal_forward_host_checks(lib):
    """spla_block_causal_forward: bf16 / head_dim 128 / groups of at most 4 heads only, a
    bounded block count and top_k, aligned inputs and a large enough workspace."""
    B = ctypes.byref
    p = _params()
    c = _cache()
    need = _lib.spla_block_causal_workspace_size(p, 4, 8192)
    assert need == _lib.spla_block_causal_workspace_size(p, 4, 8192) > 0

    def fwd(pp=p, k=FAKE, q=FAKE, max_len=8192, ws=FAKE, n=None):
        return lib.spla_block_causal_forward(B(pp), B(c), k, FAKE, q, max_len, None, FAKE, None,
                                             None, ws, need if n is None else n, None, None)

    for bad in (_params(dtype=_lib.SPLA_F32), _params(head_dim=64, num_q_heads=8, num_kv_heads=2),
                _params(num_q_heads=32, num_kv_heads=4)):
        assert fwd(pp=bad) == _lib.SPLA_ERR_UNSUPPORTED
    assert fwd(pp=_params(top_k=257)) == _lib.SPLA_ERR_CAPACITY
    assert fwd(max_len=64 * 4096 + 1) == _lib.SPLA_ERR_CAPACITY
    assert fwd(max_len=0) == _lib.SPLA_ERR_INVALID_ARG
    assert fwd(k=None) == _lib.SPLA_ERR_INVALID_ARG
    assert fwd(q=FAKE + 2) == _lib.SPLA_ERR_INVALID_ARG
    assert fwd(ws=None) == _lib.SPLA_ERR_WORKSPACE
    assert fwd(n=need - 1) == _lib.SPLA_ERR_WORKSPACE
    assert fwd(ws=FAKE + 16) == _lib.SPLA_ERR_WORKSPACE
