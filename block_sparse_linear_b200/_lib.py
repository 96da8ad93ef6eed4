"""ctypes binding of libspla.so: the C ABI of include/spla.h, argument marshalling only.

Functions keep the C names. Pointers are passed as integers (device
addresses, e.g. ``tensor.data_ptr()``); streams as the raw cudaStream_t
(``torch.cuda.current_stream().cuda_stream``). No computation happens here:
if the shared library is missing the import of these functions fails loudly.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libspla.so")

# status codes (spla_status)
SPLA_OK = 0
SPLA_ERR_INVALID_ARG = 1
SPLA_ERR_UNSUPPORTED = 2
SPLA_ERR_WORKSPACE = 3
SPLA_ERR_CAPACITY = 4
SPLA_ERR_CUDA = 5
# device status bits
SPLA_DEV_BAD_BLOCK_TABLE = 0x1
SPLA_DEV_CAPACITY = 0x2
SPLA_DEV_TIMEOUT = 0x4
SPLA_DEV_BAD_COUNT = 0x8
SPLA_DEV_RLA_UNRESOLVED = 0x10
# dtypes and flags
SPLA_F32 = 0
SPLA_BF16 = 1
SPLA_FLAG_NO_RLA = 0x1
SPLA_FLAG_FIRST_ORDER = 0x2
SPLA_MAX_BLOCKS_PER_SEQ = 32768
SPLA_STATIC_WORKSPACE_BYTES = 16 << 20
SPLA_WS_STAMP_BYTES = 16384

EXPORTS = ("spla_cache_init", "spla_append_kv", "spla_append_kv_bulk",
           "spla_append_bulk_workspace_size", "spla_decode_workspace_size", "spla_decode",
           "spla_shard_candidates", "spla_shard_partials", "spla_shard_merge",
           "spla_block_causal_workspace_size", "spla_block_causal_forward",
           "spla_decode_static_workspace", "spla_profile_events", "spla_profile_stamps",
           "spla_status_string", "spla_last_cuda_error", "spla_version")


class spla_params(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("n_sink", ctypes.c_int32),
                ("n_local", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("rms_eps", ctypes.c_float),
                ("flags", ctypes.c_uint32)]


class spla_cache(ctypes.Structure):
    _fields_ = [("k_pool", ctypes.c_void_p), ("v_pool", ctypes.c_void_p),
                ("blk_stats", ctypes.c_void_p), ("S", ctypes.c_void_p), ("z", ctypes.c_void_p),
                ("m", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("context_lens", ctypes.c_void_p), ("batch", ctypes.c_int32),
                ("max_blocks_per_seq", ctypes.c_int32), ("num_phys_blocks", ctypes.c_int32)]


class SplaError(RuntimeError):
    def __init__(self, name, status, lib):
        msg = lib.spla_status_string(status).decode()
        if status == SPLA_ERR_CUDA:
            msg += f" (cudaError {lib.spla_last_cuda_error()})"
        super().__init__(f"{name}: {msg}")
        self.status = status


_LIB = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the shared library once and declare the C signatures."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise RuntimeError(f"libspla.so not built at {path}: run "
                           "`python -m block_sparse_linear_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    P, C, vp, i32, sz = (ctypes.POINTER(spla_params), ctypes.POINTER(spla_cache), ctypes.c_void_p,
                         ctypes.c_int32, ctypes.c_size_t)
    lib.spla_cache_init.argtypes = [P, C, vp]
    lib.spla_append_kv.argtypes = [P, C, vp, vp, vp, i32, vp, vp]
    lib.spla_append_kv_bulk.argtypes = [P, C, vp, vp, vp, i32, vp, sz, vp, vp]
    lib.spla_append_bulk_workspace_size.argtypes = [P, i32, i32, ctypes.POINTER(sz)]
    lib.spla_decode_workspace_size.argtypes = [P, i32, i32, ctypes.POINTER(sz)]
    lib.spla_decode.argtypes = [P, C, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
    lib.spla_decode_static_workspace.argtypes = [P, C, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.spla_shard_candidates.argtypes = [P, C, i32, vp, vp, vp, vp, sz, vp, vp]
    lib.spla_shard_partials.argtypes = [P, C, i32, vp, vp, vp, i32, vp, vp, sz, vp, vp]
    lib.spla_shard_merge.argtypes = [P, i32, vp, i32, vp, vp, vp, vp, vp, vp]
    lib.spla_block_causal_workspace_size.argtypes = [P, i32, i32, ctypes.POINTER(sz)]
    lib.spla_block_causal_forward.argtypes = [P, C, vp, vp, vp, i32, vp, vp, vp, vp, vp, sz, vp,
                                              vp]
    lib.spla_profile_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), i32]
    lib.spla_profile_stamps.argtypes = [i32]
    for f in ("spla_cache_init", "spla_append_kv", "spla_append_kv_bulk",
              "spla_append_bulk_workspace_size", "spla_decode_workspace_size", "spla_decode",
           "spla_shard_candidates", "spla_shard_partials", "spla_shard_merge",
           "spla_block_causal_workspace_size", "spla_block_causal_forward",
              "spla_decode_static_workspace", "spla_profile_events", "spla_profile_stamps",
              "spla_shard_candidates", "spla_shard_partials", "spla_shard_merge",
              "spla_block_causal_workspace_size", "spla_block_causal_forward"):
        getattr(lib, f).restype = ctypes.c_int
    lib.spla_status_string.argtypes = [ctypes.c_int]
    lib.spla_status_string.restype = ctypes.c_char_p
    lib.spla_last_cuda_error.restype = ctypes.c_int32
    lib.spla_version.restype = ctypes.c_int32
    _LIB = lib
    return lib


def _check(name, st):
    if st != SPLA_OK:
        raise SplaError(name, st, load())


# ----------------------------------------------------------------------------- C entry points
def spla_cache_init(params, cache, stream=0):
    _check("spla_cache_init", load().spla_cache_init(ctypes.byref(params), ctypes.byref(cache),
                                                     stream))


def spla_append_kv(params, cache, k_new, v_new, n_new, max_new, dev_status, stream=0):
    _check("spla_append_kv", load().spla_append_kv(ctypes.byref(params), ctypes.byref(cache),
                                                   k_new, v_new, n_new, max_new, dev_status,
                                                   stream))


def spla_append_kv_bulk(params, cache, k_new, v_new, n_new, max_new, workspace, workspace_bytes,
                        dev_status, stream=0):
    _check("spla_append_kv_bulk",
           load().spla_append_kv_bulk(ctypes.byref(params), ctypes.byref(cache), k_new, v_new,
                                      n_new, max_new, workspace, workspace_bytes, dev_status,
                                      stream))


def spla_append_bulk_workspace_size(params, batch, max_new) -> int:
    n = ctypes.c_size_t(0)
    _check("spla_append_bulk_workspace_size",
           load().spla_append_bulk_workspace_size(ctypes.byref(params), batch, max_new,
                                                  ctypes.byref(n)))
    return n.value


def spla_shard_candidates(params, cache, first_block, global_nb, q, cand, workspace,
                          workspace_bytes, dev_status, stream=0):
    _check("spla_shard_candidates",
           load().spla_shard_candidates(ctypes.byref(params), ctypes.byref(cache), first_block,
                                        global_nb, q, cand, workspace, workspace_bytes,
                                        dev_status, stream))


def spla_shard_partials(params, cache, first_block, global_nb, q, cand_all, nshards, part,
                        workspace, workspace_bytes, dev_status, stream=0):
    _check("spla_shard_partials",
           load().spla_shard_partials(ctypes.byref(params), ctypes.byref(cache), first_block,
                                      global_nb, q, cand_all, nshards, part, workspace,
                                      workspace_bytes, dev_status, stream))


def spla_shard_merge(params, batch, part_all, nshards, gamma, out, o_sparse, o_rla, dev_status,
                     stream=0):
    _check("spla_shard_merge",
           load().spla_shard_merge(ctypes.byref(params), batch, part_all, nshards, gamma, out,
                                   o_sparse, o_rla, dev_status, stream))


def spla_block_causal_workspace_size(params, batch, max_len) -> int:
    n = ctypes.c_size_t(0)
    _check("spla_block_causal_workspace_size",
           load().spla_block_causal_workspace_size(ctypes.byref(params), batch, max_len,
                                                   ctypes.byref(n)))
    return n.value


def spla_block_causal_forward(params, cache, k_all, v_all, q_all, max_len, gamma, out, o_sparse,
                              o_rla, workspace, workspace_bytes, dev_status, stream=0):
    _check("spla_block_causal_forward",
           load().spla_block_causal_forward(ctypes.byref(params), ctypes.byref(cache), k_all,
                                            v_all, q_all, max_len, gamma, out, o_sparse, o_rla,
                                            workspace, workspace_bytes, dev_status, stream))


def spla_decode_workspace_size(params, batch, max_blocks_per_seq) -> int:
    n = ctypes.c_size_t(0)
    _check("spla_decode_workspace_size",
           load().spla_decode_workspace_size(ctypes.byref(params), batch, max_blocks_per_seq,
                                             ctypes.byref(n)))
    return n.value


def spla_decode(params, cache, q, rms_gamma, out, sel_idx, o_sparse_dbg, o_rla_dbg, workspace,
                workspace_bytes, dev_status, stream=0):
    _check("spla_decode", load().spla_decode(ctypes.byref(params), ctypes.byref(cache), q,
                                             rms_gamma, out, sel_idx, o_sparse_dbg, o_rla_dbg,
                                             workspace, workspace_bytes, dev_status, stream))


def spla_decode_static_workspace(params, cache, q, rms_gamma, out, sel_idx, o_sparse_dbg,
                                 o_rla_dbg, dev_status, stream=0):
    """spla_decode with the library's own scratch, for callers that cannot allocate."""
    _check("spla_decode_static_workspace",
           load().spla_decode_static_workspace(ctypes.byref(params), ctypes.byref(cache), q,
                                               rms_gamma, out, sel_idx, o_sparse_dbg, o_rla_dbg,
                                               dev_status, stream))


def spla_profile_stamps(on: bool):
    """Turn the kernels' device timestamps (this host thread's decode calls) on or off."""
    _check("spla_profile_stamps", load().spla_profile_stamps(1 if on else 0))


def spla_profile_events(events):
    """events: 2 to 8 cudaEvent_t handles (ints), or an empty sequence to stop recording."""
    arr = (ctypes.c_void_p * max(1, len(events)))(*events)
    _check("spla_profile_events", load().spla_profile_events(arr, len(events)))
