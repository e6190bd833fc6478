"""GPU parity of quantize-on-write, calibration and dequant against the oracle.

Codes, scales, zero points and residual rows must be byte-identical to the oracle's,
and every byte the write should not touch must keep the sentinel."""

import numpy as np
import pytest
import torch

from quantized_paged_kv_02_b200 import inputs
from tests import helpers

pytestmark = pytest.mark.gpu

SMALL = ["c1", "c2", "c3", "c4", "c4-tok", "c4-fzp", "c4-int2", "c4-int2-tok", "c4-int2-fzp", "c5",
         "c5-fp8", "c5-bf16", "c5-int8-pc", "c5-int8-ph", "c5-int8-pt", "c5-fp8-pt"]


@pytest.fixture(scope="module", autouse=True)
def _built():
    helpers.ensure_built()


def _workload(name):
    return inputs.make(name, small=(name != "c1"))


def _compare_pools(gc, oc):
    helpers.assert_same_cache(gc, oc)


@pytest.mark.parametrize("name", SMALL)
def test_write_bit_exact(name):
    w = _workload(name)
    static = helpers.oracle_static_scales(w)
    oc = helpers.oracle_cache(w, static)
    gc = helpers.gpu_cache(w, static=static)
    torch.cuda.synchronize()
    _compare_pools(gc, oc)
    assert gc.read_fault() == (0, 0)


def test_fp8_calibration_bit_exact():
    from oracle import quant
    from quantized_paged_kv_02_b200 import kvq
    w = inputs.make("c3", small=True)
    for x in (w.warmup_k, w.warmup_v):
        out = torch.empty(x.shape[1], dtype=torch.float32, device="cuda")
        kvq.kvq_calibrate_fp8_scales(x.cuda(), out)
        want = quant.fp8_calibrate(helpers.np64(x).astype(np.float32))
        np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32), want.view(np.uint32))


def test_head_calibration_bit_exact():
    from oracle import quant
    from quantized_paged_kv_02_b200 import kvq
    w = inputs.make("c5-int8-ph", small=True)
    for x in (w.warmup_k, w.warmup_v):
        for qmax in (127.0, 448.0):
            out = torch.empty(x.shape[1], dtype=torch.float32, device="cuda")
            kvq.kvq_calibrate_head_scales(x.cuda(), qmax, out)
            want = quant.head_calibrate(helpers.np64(x).astype(np.float32), qmax)
            np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32), want.view(np.uint32))


def test_channel_calibration_bit_exact():
    from oracle import quant
    from quantized_paged_kv_02_b200 import kvq
    w = inputs.make("c5-int8-pc", small=True)
    for x in (w.warmup_k, w.warmup_v):
        for qmax in (127.0, 448.0):
            out = torch.empty(x.shape[1:], dtype=torch.float32, device="cuda")
            kvq.kvq_calibrate_channel_scales(x.cuda(), qmax, out)
            want = quant.channel_calibrate(helpers.np64(x).astype(np.float32), qmax)
            np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("name", SMALL)
def test_dequant_matches_oracle(name):
    w = _workload(name)
    static = helpers.oracle_static_scales(w)
    oc = helpers.oracle_cache(w, static)
    gc = helpers.gpu_cache(w, static=static)
    used = sorted(set(w.block_tables.cpu().numpy().reshape(-1).tolist()) & set(
        (w.slot_mapping[w.slot_mapping >= 0].cpu().numpy() // w.spec.block_size).tolist()))
    ids = torch.tensor(used, dtype=torch.int32, device="cuda")
    got = gc.dequant(ids).cpu().numpy().astype(np.float64)
    for i, blk in enumerate(used):
        want = oc.dequant_block(blk)
        # code * scale is rounded once to binary32 on the GPU
        np.testing.assert_allclose(got[i], want, rtol=2.0 ** -24, atol=0)


def test_write_edge_cases():
    """Zero rows (scale 0), a row that saturates, skipped (-1) and out-of-range slots."""
    from oracle import cache as ocache
    from quantized_paged_kv_02_b200 import kvq
    H, D, bs, NB = 2, 128, 16, 4
    g = torch.Generator().manual_seed(3)
    k = torch.randn(7, H, D, generator=g).to(torch.bfloat16)
    v = torch.randn(7, H, D, generator=g).to(torch.bfloat16)
    k[1] = 0
    v[2, 0] = 0
    k[3, 1, 5] = 3.0e38                      # huge outlier: everything else rounds to 0
    k[4, 0, 0] = -1e-30                      # tiny negative
    slots = torch.tensor([5, 17, 63, 33, 0, 64, -1], dtype=torch.int32)   # 64 is out of range
    for cd in ("int8", "fp8"):
        mode = "per_token_head"
        oc = ocache.PagedCache(cd, "bf16", mode, NB, bs, H, D)
        oc.write(helpers.np64(k), helpers.np64(v), slots.numpy())
        gc = kvq.PagedKVCache(cd, "bf16", mode, NB, bs, H, D)
        gc.write(k.cuda(), v.cuda(), slots.cuda())
        torch.cuda.synchronize()
        helpers.assert_same_cache(gc, oc)
        assert gc.read_fault() == (1, 1)       # one bad slot, KVQ_FAULT_SLOT
    # static FP8 scale with values far beyond 448 * s: saturation, signed zero
    sk = torch.tensor([0.01, 1e-3]), torch.tensor([0.5, 2.0])
    oc = ocache.PagedCache("fp8", "bf16", "per_head", NB, bs, H, D,
                           static_scales=(sk[0].numpy(), sk[1].numpy()))
    oc.write(helpers.np64(k), helpers.np64(v), slots.numpy())
    gc = kvq.PagedKVCache("fp8", "bf16", "per_head", NB, bs, H, D,
                          static_k_scale=sk[0].cuda(), static_v_scale=sk[1].cuda())
    gc.write(k.cuda(), v.cuda(), slots.cuda())
    torch.cuda.synchronize()
    helpers.assert_same_cache(gc, oc)


def test_write_rounding_midpoints():
    """Quotients x / s exactly on a rounding midpoint (ties to even) and right beside one: an
    INT8 per-token row whose maximum is 127 * 2^-3 (scale 2^-3, quotients n + 1/2), a static
    INT8 scale of 1/2 with the same kind of row plus saturating values, and E4M3 midpoints
    (1 + (2k + 1) / 16) * 2^e against a static FP8 scale of 1."""
    from oracle import cache as ocache
    from quantized_paged_kv_02_b200 import kvq
    H, D, bs, NB = 2, 128, 16, 2
    n = torch.arange(D, dtype=torch.float64)
    half = ((n - 64) + 0.5) * 0.125                   # quotients -63.5 .. 63.5 at scale 2^-3
    half[0] = 127 * 0.125                             # the row maximum: scale exactly 2^-3
    mids = torch.tensor([(1 + (2 * (i % 8) + 1) / 16.0) * 2.0 ** ((i // 8) % 12 - 6) for i in range(D)],
                        dtype=torch.float64)
    mids = torch.where(n % 2 == 0, mids, -mids)
    g = torch.Generator().manual_seed(11)
    rows = torch.randn(6, H, D, generator=g, dtype=torch.float64)
    rows[0, 0] = half
    rows[1, 1] = half * 8                             # scale 1, quotients n + 1/2 up to 127
    rows[2, 0] = mids
    rows[3, 1] = mids * 4
    rows[4, 0, :8] = torch.tensor([300.0, -300.0, 63.75, -63.75, 63.25, 0.25, -0.25, 0.75])
    k = rows.to(torch.bfloat16)
    v = (rows * 0.5).to(torch.bfloat16)
    assert torch.equal(k[0, 0].double(), half) and torch.equal(k[2, 0].double(), mids)
    slots = torch.tensor([0, 3, 16, 17, 30, 31], dtype=torch.int32)
    cases = (("int8", "per_token_head", None), ("int8", "per_head", (0.5, 0.5)),
             ("fp8", "per_head", (1.0, 0.25)))
    for cd, mode, st in cases:
        sk = None if st is None else torch.tensor([st[0], st[1]], dtype=torch.float32)
        kw = {} if st is None else {"static_scales": (sk.numpy(), sk.numpy())}
        oc = ocache.PagedCache(cd, "bf16", mode, NB, bs, H, D, **kw)
        oc.write(helpers.np64(k), helpers.np64(v), slots.numpy())
        gkw = {} if st is None else {"static_k_scale": sk.cuda(), "static_v_scale": sk.cuda()}
        gc = kvq.PagedKVCache(cd, "bf16", mode, NB, bs, H, D, **gkw)
        gc.write(k.cuda(), v.cuda(), slots.cuda())
        torch.cuda.synchronize()
        helpers.assert_same_cache(gc, oc)
        assert gc.read_fault() == (0, 0)


@pytest.mark.parametrize("cd,mode", [("int8", "per_token_head"), ("int8", "per_head"),
                                     ("fp8", "per_head"), ("fp8", "per_token_head")])
def test_write_many_rows_bit_exact(cd, mode):
    """8192 tokens x 4 heads of values spread over 40 binades (row magnitudes 2^-20 .. 2^20,
    some rows with a single large outlier), written with per-token or static scales: every
    code and scale byte-identical to the oracle's binary32 division and rounding."""
    from oracle import cache as ocache
    from quantized_paged_kv_02_b200 import kvq
    T, H, D, bs = 8192, 4, 128, 16
    NB = T // bs
    g = torch.Generator().manual_seed(21)
    mag = torch.pow(2.0, torch.randint(-20, 21, (T, H, 1), generator=g).double())
    k = (torch.randn(T, H, D, generator=g, dtype=torch.float64) * mag)
    v = (torch.rand(T, H, D, generator=g, dtype=torch.float64) - 0.5) * mag
    k[::7, :, 3] *= 50.0
    k, v = k.to(torch.bfloat16), v.to(torch.bfloat16)
    slots = torch.randperm(NB * bs, generator=g)[:T].to(torch.int32)
    kw, gkw = {}, {}
    if mode == "per_head":
        sk = torch.tensor([0.003, 0.5, 7.0, 1e-5], dtype=torch.float32)
        kw = {"static_scales": (sk.numpy(), (sk * 3).numpy())}
        gkw = {"static_k_scale": sk.cuda(), "static_v_scale": (sk * 3).cuda()}
    oc = ocache.PagedCache(cd, "bf16", mode, NB, bs, H, D, **kw)
    oc.write(helpers.np64(k), helpers.np64(v), slots.numpy())
    gc = kvq.PagedKVCache(cd, "bf16", mode, NB, bs, H, D, **gkw)
    gc.write(k.cuda(), v.cuda(), slots.cuda())
    torch.cuda.synchronize()
    helpers.assert_same_cache(gc, oc)
    assert gc.read_fault() == (0, 0)


def test_int4_bad_run_is_skipped_and_counted():
    from quantized_paged_kv_02_b200 import kvq
    H, D = 1, 128
    k = torch.randn(64, H, D).to(torch.bfloat16).cuda()
    slots = torch.arange(64, 128, dtype=torch.int32)
    slots[10] = 200                                   # not one ordered block
    gc = kvq.PagedKVCache("int4", "bf16", "kivi", 4, 64, H, D, max_seqs=1)
    gc.write(k, k, slots.cuda())
    torch.cuda.synchronize()
    assert np.all(helpers.pool_bytes(gc.pages, gc.sizes[1]) == 0x5A)
    cnt, bits = gc.read_fault()
    assert cnt == 1 and bits == 16
