"""GPU test of kvq_decode_attention_noalloc, the decode entry point that needs no workspace.

It is meant for callers that cannot allocate device memory when they decode: a plugin
whose host engine plans all device memory and hands it only input and output buffers, a
server whose KV-cache pool already holds nearly all of HBM, or a loop that keeps
cudaMalloc/cudaFree (which can synchronize the device) off its hot path.  The test calls
the entry point through the C ABI twice in a row and checks each result against the
regular entry point (which uses a caller workspace), within the attention tolerance of
the other decode tests.  Its file name sorts last so a run that stops at the first
failure has run every other test first; it also passes alone in a fresh process.
"""

import ctypes

import pytest
import torch

from quantized_paged_kv_02_b200 import inputs
from tests import helpers

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _call_noalloc(kvq, cache, w, out):
    lib = kvq.lib
    fn = lib.kvq_decode_attention_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(kvq.CacheDesc), ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                   ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                   ctypes.c_float, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p]
    q = w.q.cuda()
    tables = w.block_tables.cuda()
    lens = w.context_lens.cuda()
    st = fn(ctypes.byref(cache.desc), q.data_ptr(), q.shape[0], q.shape[1], tables.data_ptr(),
            tables.shape[1], lens.data_ptr(), None, int(w.max_context), 0.0, out.data_ptr(),
            kvq.DTYPE["fp32"], torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return st


@pytest.mark.parametrize("name", ["c5", "c3", "c4"])
def test_noalloc_matches_workspace_entry_point(name):
    helpers.ensure_built()
    from quantized_paged_kv_02_b200 import kvq
    w = inputs.make(name, small=True)
    static = helpers.oracle_static_scales(w)
    cache = helpers.gpu_cache(w, static=static)
    need = cache.workspace_size(w.spec.batch, w.spec.num_q_heads, w.max_context)
    assert 0 < need <= 16 << 20          # the scratch array is really used
    ref = cache.decode(w.q.cuda(), w.block_tables.cuda(), w.context_lens.cuda(), w.max_context)
    torch.cuda.synchronize()
    for _ in range(2):                   # two calls in a row share the same scratch
        out = torch.full_like(ref, float("nan"))
        assert _call_noalloc(kvq, cache, w, out) == 0
        assert torch.isfinite(out).all()
        assert (out - ref).abs().max().item() <= TOL
