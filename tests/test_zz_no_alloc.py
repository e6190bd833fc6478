"""GPU test of kvq_decode_attention_noalloc, the decode entry point that needs no workspace.

It is meant for callers that cannot allocate device memory when they decode: a plugin
whose host engine plans all device memory and hands it only input and output buffers, a
server whose KV-cache pool already holds nearly all of HBM, or a loop that keeps
cudaMalloc/cudaFree (which can synchronize the device) off its hot path.  The test calls
the entry point through the C ABI on workloads of different shapes in turn (so a call
that read what an earlier call left in the shared scratch would show), and requires each
output to equal, bit for bit, the regular entry point's output on the same inputs (same
kernels, same plan, a caller workspace instead of the fixed array), which is itself within
the attention tolerance of the oracle in the other decode tests.  A shape too large for
the array is refused with nothing written.  Its file name sorts last so a run that stops
at the first failure has run every other test first; it also passes alone in a fresh
process.
"""

import ctypes

import pytest
import torch

from quantized_paged_kv_02_b200 import inputs
from tests import helpers

pytestmark = pytest.mark.gpu


def _call_noalloc(kvq, cache, q, tables, lens, max_context, out):
    fn = kvq.lib.kvq_decode_attention_noalloc
    st = fn(ctypes.byref(cache.desc), q.data_ptr(), q.shape[0], q.shape[1], tables.data_ptr(),
            tables.shape[1], lens.data_ptr(), None, int(max_context), 0.0, out.data_ptr(),
            kvq.DTYPE["fp32"], torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return st


def _setup(name):
    w = inputs.make(name, small=True)
    static = helpers.oracle_static_scales(w)
    cache = helpers.gpu_cache(w, static=static)
    need = cache.workspace_size(w.spec.batch, w.spec.num_q_heads, w.max_context)
    assert 0 < need <= 16 << 20          # the scratch array is really used
    q, tables, lens = w.q.cuda(), w.block_tables.cuda(), w.context_lens.cuda()
    ref = cache.decode(q, tables, lens, w.max_context)
    torch.cuda.synchronize()
    return cache, q, tables, lens, w.max_context, ref


def test_noalloc_matches_workspace_entry_point():
    helpers.ensure_built()
    from quantized_paged_kv_02_b200 import kvq
    cases = {name: _setup(name) for name in ("c3", "c5", "c4")}
    # c3, then c5 and c4 (other shapes, other partial layouts in the scratch), then c3 again
    for name in ("c3", "c5", "c4", "c3", "c3"):
        cache, q, tables, lens, mc, ref = cases[name]
        out = torch.full_like(ref, float("nan"))
        assert _call_noalloc(kvq, cache, q, tables, lens, mc, out) == 0, name
        assert torch.equal(out, ref), name


def test_noalloc_refuses_oversize_shape_and_writes_nothing():
    helpers.ensure_built()
    from quantized_paged_kv_02_b200 import kvq
    w = inputs.make("c5", small=True)
    cache = helpers.gpu_cache(w)
    B = 4096                               # partials of 4096 x 2 units need far more than 16 MiB
    assert cache.workspace_size(B, w.spec.num_q_heads, 16384) > 16 << 20
    q = w.q.cuda()[:1].expand(B, -1, -1).contiguous()
    tables = torch.zeros((B, 1024), dtype=torch.int32, device="cuda")
    lens = torch.ones(B, dtype=torch.int32, device="cuda")
    out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    assert _call_noalloc(kvq, cache, q, tables, lens, 16384, out) == 1
    assert torch.isnan(out).all()
