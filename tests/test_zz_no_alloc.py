"""spla_decode_static_workspace (decode with the library's built-in scratch, no
allocation) against spla_decode with a caller workspace, through the C ABI.

Both entry points run the same kernels on the same inputs, so their results
must be bit-identical. Two calls in a row, with an append between them, so that
the second call reuses scratch the first one left behind. The file name makes
pytest collect it last; it also runs alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from block_sparse_linear_b200 import _lib
from workloads import feed_gpu, gen

pytestmark = pytest.mark.gpu


def _run(cache, q, gamma, static: bool):
    out, sel, osp, orl = cache.new_outputs(debug=True)
    if static:
        _lib.spla_decode_static_workspace(cache.params, cache.c, q.data_ptr(), gamma.data_ptr(),
                                          out.data_ptr(), sel.data_ptr(), osp.data_ptr(),
                                          orl.data_ptr(), cache.dev_status.data_ptr(),
                                          torch.cuda.current_stream().cuda_stream)
    else:
        cache.decode(q, gamma, out, sel, osp, orl)
    torch.cuda.synchronize()
    return {k: t.float().cpu().numpy() if t.dtype != torch.int32 else t.cpu().numpy()
            for k, t in dict(out=out, sel=sel, o_sparse=osp, o_rla=orl).items()}


@pytest.mark.parametrize("name,lens", [("cfg3", (8192 + 5, 6000)), ("cfg5", (5000, 300, 12000, 64))])
def test_static_workspace_matches_caller_workspace_on_two_calls(name, lens):
    w = gen.scaled(name, context_lens=lens)
    cache = feed_gpu.build_cache(w)
    need = _lib.spla_decode_workspace_size(cache.params, cache.batch, cache.max_blocks_per_seq)
    assert need <= _lib.SPLA_STATIC_WORKSPACE_BYTES
    dt = cache.cfg.torch_dtype
    gamma = torch.from_numpy(gen.gamma(w, "random")).float().cuda()
    for step in range(2):
        if step:
            k, v, _ = feed_gpu.step_inputs(w, step)
            cache.append(k, v)
        q = torch.from_numpy(gen.query(w, step)).to(dt).cuda()
        ref = _run(cache, q, gamma, static=False)
        got = _run(cache, q, gamma, static=True)
        for key in ("sel", "o_sparse", "o_rla", "out"):
            np.testing.assert_array_equal(got[key], ref[key], err_msg=key)
    assert cache.status() == 0
