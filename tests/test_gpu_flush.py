"""kvq_flush_ring: quantizing the oldest 64 ring rows of a sequence into a page, from the
ring itself, must store what kvq_write stores for those rows, and decode over the longer
quantized prefix must match the oracle taking the same steps."""

import numpy as np
import pytest
import torch

from oracle import attention
from quantized_paged_kv_02_b200 import inputs, kvq
from tests import helpers

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    helpers.ensure_built()


@pytest.mark.parametrize("cd,mode", [("int4", "kivi"), ("int4", "int4_per_token"),
                                     ("int4", "kivi_float_zero"), ("int2", "kivi"),
                                     ("int2", "int4_per_token")])
def test_flush_then_append_then_decode(cd, mode):
    spec = inputs.Spec("flush", cd, "bf16", mode, 2, 16, 2, 128, 64, lens=[485, 300],
                       outliers="k", slack_blocks=3, seed=11)
    w = inputs.from_spec(spec)
    oc = helpers.oracle_cache(w)
    gc = helpers.gpu_cache(w)
    n0 = int(w.context_lens[0])
    qb = 64 * ((n0 - inputs.RESIDUAL_LEN) // 64)          # 320: ring holds [320, 485)
    used = set(w.block_tables.numpy().reshape(-1).tolist())
    free = [b for b in range(w.num_blocks) if b not in used][0]
    sid = torch.tensor([0], dtype=torch.int32)
    pos = torch.tensor([qb], dtype=torch.int32)
    blk = torch.tensor([free], dtype=torch.int32)
    gc.flush_ring(sid.cuda(), pos.cuda(), blk.cuda())
    oc.flush_ring(sid.numpy(), pos.numpy(), blk.numpy())
    torch.cuda.synchronize()
    helpers.assert_same_cache(gc, oc)
    # the flushed page equals kvq_write of the same 64 rows into that block
    ref = helpers.gpu_cache(w)
    r0 = int(w.seq_start[0]) + qb
    slots = (free * 64 + torch.arange(64, dtype=torch.int32)).cuda()
    ref.write(w.k[r0:r0 + 64].cuda(), w.v[r0:r0 + 64].cuda(), slots)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(gc.records()[free].cpu().numpy(), ref.records()[free].cpu().numpy())
    # 64 more tokens of sequence 0 go to the ring; the prefix grows by the flushed block
    g = torch.Generator().manual_seed(12)
    kn = torch.randn((64, 2, 128), generator=g).to(torch.bfloat16)
    vn = torch.randn((64, 2, 128), generator=g).to(torch.bfloat16)
    newpos = torch.arange(n0, n0 + 64, dtype=torch.int32)
    ring = torch.full((64,), -1, dtype=torch.int32)
    seq = torch.zeros(64, dtype=torch.int32)
    gc.write(kn.cuda(), vn.cuda(), ring.cuda(), seq.cuda(), newpos.cuda())
    oc.write(helpers.np64(kn), helpers.np64(vn), ring.numpy(), seq.numpy(), newpos.numpy())
    lens = w.context_lens.clone()
    lens[0] = n0 + 64                                      # prefix 384 = 6 blocks
    tab = torch.zeros((2, max(w.block_tables.shape[1], 6)), dtype=torch.int32)
    tab[:, :w.block_tables.shape[1]] = w.block_tables
    tab[0, qb // 64] = free
    torch.cuda.synchronize()
    helpers.assert_same_cache(gc, oc)
    out = gc.decode(w.q.cuda(), tab.cuda(), lens.cuda(), int(lens.max()))
    want = attention.decode_attention(oc, helpers.np64(w.q), tab.numpy(), lens.numpy())
    err = np.abs(out.cpu().numpy().astype(np.float64) - want).max()
    assert err <= 2e-3, err
    assert gc.read_fault() == (0, 0)


def test_flush_ring_rejects_bad_entries_and_dense_caches():
    w = inputs.make("c4", small=True)
    gc = helpers.gpu_cache(w)
    before = gc.records().clone()
    bad = torch.tensor([5, 0, 0], dtype=torch.int32, device="cuda")       # sequence 5 of 2
    pos = torch.tensor([0, 63, 0], dtype=torch.int32, device="cuda")       # 63: not a group start
    blk = torch.tensor([0, 0, w.num_blocks + 4], dtype=torch.int32, device="cuda")
    gc.flush_ring(bad, pos, blk)
    torch.cuda.synchronize()
    cnt, bits = gc.read_fault()
    assert cnt == 3 and bits == (8 | 16 | 2)
    assert torch.equal(gc.records(), before)
    d = helpers.gpu_cache(inputs.make("c5", small=True))
    with pytest.raises(kvq.KVQError):
        d.flush_ring(bad, pos, blk)
