"""GPU parity at the benchmark's full sizes, on sampled sequences.

Each workload is built at full size on the GPU (as the benchmark builds it), written by
kvq_write and decoded by kvq_decode_attention in the benchmark's configuration.  The
oracle cannot hold a full cache, but quantization is per (token, kv head) row (INT4: per
64-row group of one sequence), so a one-sequence oracle cache holds exactly the codes
of that sequence's blocks: those are compared byte for byte, and its attention output
with output row b (max |gpu - oracle| <= 2e-3, float32 output; the bfloat16 output is
that float32 result rounded to nearest even).  This covers what the small cases
cannot: thousands of pages per CTA ring, full batches and full page pools.
"""

import numpy as np
import pytest
import torch

from oracle import attention, fp
from quantized_paged_kv_02_b200 import inputs
from tests import helpers

pytestmark = pytest.mark.gpu

TOL = 2e-3
FULL = ["c2", "c3", "c4", "c4-tok", "c4-fzp", "c4-int2", "c4-int2-tok", "c4-int2-fzp", "c5",
        "c5-fp8", "c5-bf16", "c5-int8-pc", "c5-int8-ph", "c5-int8-pt", "c5-fp8-pt"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    helpers.ensure_built()


def _samples(w):
    lens = w.context_lens.cpu().numpy()
    B = len(lens)
    picks = {0, B // 2, B - 1, int(np.argmin(lens)), int(np.argmax(lens))}
    return sorted(picks)


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_sequences(name):
    dev = torch.device("cuda")
    w = inputs.make(name, small=False, device="cuda")
    static = helpers.oracle_static_scales(w)
    gc = helpers.gpu_cache(w, device=dev, static=static)
    mc = w.max_context
    out = gc.decode(w.q, w.block_tables, w.context_lens, mc)
    outb = gc.decode(w.q, w.block_tables, w.context_lens, mc, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert gc.read_fault() == (0, 0)
    got = out.cpu().numpy().astype(np.float64)
    gotb = outb.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    records = gc.records()
    tables = w.block_tables.cpu()
    for b in _samples(w):
        sub = helpers.single_sequence(w, b)
        oc = helpers.oracle_cache(sub, static)
        nblk = sub.num_blocks
        if sub.context_lens[0] > 0 and (name != "c4" or int(sub.slot_mapping.max()) >= 0):
            mine = records[tables[b, :nblk].to(dev).long()].cpu().numpy()
            np.testing.assert_array_equal(mine, oc.pages[:nblk], err_msg="codes of sequence %d" % b)
        want = attention.decode_attention(oc, helpers.np64(sub.q), sub.block_tables.numpy(),
                                          sub.context_lens.numpy())[0]
        err = np.abs(got[b] - want).max()
        assert err <= TOL, (b, err)
        # bfloat16 output: the float32 result rounded once (same arithmetic, one store),
        # so within the tolerance plus half a bfloat16 ulp of the oracle
        np.testing.assert_array_equal(gotb[b], fp.bf16_round(got[b]))
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), 2.0 ** -126))) - 7)
        assert np.all(np.abs(gotb[b] - want) <= TOL + ulp / 2), b
    del gc, w, out, outb
    torch.cuda.empty_cache()
