"""kvq_append_decode_attention: one launch that stores each sequence's new K/V row and then
attends must leave the same pool bytes and give the same output, bit for bit, as
kvq_write of that row followed by kvq_decode_attention (and so match the oracle)."""

import numpy as np
import pytest
import torch

from oracle import attention
from quantized_paged_kv_02_b200 import inputs, kvq
from tests import helpers

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    helpers.ensure_built()


def _split_last(w):
    """Slots with each sequence's last row removed, and those last rows as [B][H][D]."""
    s = w.spec
    starts = w.seq_start.tolist()
    slots = w.slot_mapping.clone().cpu()
    k_new = torch.zeros((s.batch, s.num_kv_heads, s.head_dim), dtype=w.k.dtype)
    v_new = torch.zeros_like(k_new)
    for b in range(s.batch):
        if starts[b + 1] > starts[b]:
            last = starts[b + 1] - 1
            slots[last] = -1
            k_new[b] = w.k[last].cpu()
            v_new[b] = w.v[last].cpu()
    return slots, k_new, v_new


def _caches(w, static):
    a = helpers.gpu_cache(w, static=static)          # every row, by kvq_write
    s = w.spec
    sk = sv = None
    if static is not None:
        sk, sv = (torch.as_tensor(np.asarray(x, np.float32), device="cuda") for x in static)
    b = kvq.PagedKVCache(s.cache_dtype, s.act_dtype, s.scale_mode, w.num_blocks, s.block_size,
                         s.num_kv_heads, s.head_dim, device="cuda", max_seqs=max(s.batch, 1),
                         static_k_scale=sk, static_v_scale=sv, fill=0x5A)
    return a, b


def _check(w):
    static = helpers.oracle_static_scales(w)
    ref, fused = _caches(w, static)
    slots, k_new, v_new = _split_last(w)
    fused.write(w.k.cuda(), w.v.cuda(), slots.cuda())
    q, tab, lens = w.q.cuda(), w.block_tables.cuda(), w.context_lens.cuda()
    mc = max(w.max_context, 1)
    want = ref.decode(q, tab, lens, mc)
    got = fused.append_decode(k_new.cuda(), v_new.cuda(), q, tab, lens, mc)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(helpers.pool_bytes(fused.pages, fused.sizes[1]),
                                  helpers.pool_bytes(ref.pages, ref.sizes[1]))
    assert torch.equal(got, want)
    assert fused.read_fault() == (0, 0)
    return got, static


@pytest.mark.parametrize("name", ["c5", "c5-fp8", "c5-bf16", "c5-int8-pc", "c3", "c2"])
def test_append_decode_equals_write_then_decode(name):
    w = inputs.make(name, small=True)
    got, static = _check(w)
    oc = helpers.oracle_cache(w, static)
    want = attention.decode_attention(oc, helpers.np64(w.q), w.block_tables.numpy(),
                                      w.context_lens.numpy())
    assert np.abs(got.cpu().numpy().astype(np.float64) - want).max() <= TOL


@pytest.mark.parametrize("kind", ["int8", "fp8"])
def test_append_decode_with_empty_and_one_token_sequences(kind):
    cd, mode = {"int8": ("int8", "per_token_head"), "fp8": ("fp8", "per_head")}[kind]
    lens = [0, 1, 16, 17, 0, 33, 2, 0, 5, 48, 0, 31]
    spec = inputs.Spec("append-" + kind, cd, "bf16", mode, len(lens), 8, 2, 128, 16, lens=lens,
                       slack_blocks=3, seed=5)
    _check(inputs.from_spec(spec))


def test_append_decode_full_size_c5():
    w = inputs.make("c5", small=False, device="cuda")
    _check(w)


@pytest.mark.parametrize("name", ["c4", "c4-tok", "c4-fzp", "c4-int2", "c4-int2-tok"])
def test_append_decode_low_bit_equals_write_then_decode(name):
    """INT4 / 2-bit: each sequence's newest row goes to the residual ring in the same call as
    decode; pages, ring and output equal kvq_write of every row followed by decode, bit for
    bit (and so the oracle)."""
    w = inputs.make(name, small=True)
    s = w.spec
    ref = helpers.gpu_cache(w)
    fused = kvq.PagedKVCache(s.cache_dtype, s.act_dtype, s.scale_mode, w.num_blocks, s.block_size,
                             s.num_kv_heads, s.head_dim, device="cuda",
                             residual_len=inputs.RESIDUAL_LEN, residual_cap=inputs.RESIDUAL_CAP,
                             max_seqs=max(s.batch, 1), fill=0x5A)
    idx, slots, sid, pos = inputs.int4_group_rows(w)
    starts = w.seq_start.tolist()
    last = {starts[b + 1] - 1 for b in range(s.batch) if starts[b + 1] > starts[b]}
    keep = torch.tensor([int(i) not in last for i in idx.tolist()])
    k, v = w.k.cuda(), w.v.cuda()
    ki = idx[keep].cuda()
    fused.write(k[ki].contiguous(), v[ki].contiguous(), slots[keep].cuda(), sid[keep].cuda(),
                pos[keep].cuda())
    k_new = torch.zeros((s.batch, s.num_kv_heads, s.head_dim), dtype=w.k.dtype)
    v_new = torch.zeros_like(k_new)
    for b in range(s.batch):
        if starts[b + 1] > starts[b]:
            k_new[b] = w.k[starts[b + 1] - 1].cpu()
            v_new[b] = w.v[starts[b + 1] - 1].cpu()
    q, tab, lens = w.q.cuda(), w.block_tables.cuda(), w.context_lens.cuda()
    mc = max(w.max_context, 1)
    want = ref.decode(q, tab, lens, mc)
    got = fused.append_decode(k_new.cuda(), v_new.cuda(), q, tab, lens, mc)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(helpers.pool_bytes(fused.pages, fused.sizes[1]),
                                  helpers.pool_bytes(ref.pages, ref.sizes[1]))
    np.testing.assert_array_equal(helpers.pool_bytes(fused.residual, fused.sizes[3]),
                                  helpers.pool_bytes(ref.residual, ref.sizes[3]))
    assert torch.equal(got, want)
    assert fused.read_fault() == (0, 0)
    oc = helpers.oracle_cache(w)
    exact = attention.decode_attention(oc, helpers.np64(w.q), w.block_tables.numpy(),
                                       w.context_lens.numpy())
    assert np.abs(got.cpu().numpy().astype(np.float64) - exact).max() <= TOL


def test_append_decode_rejects_unsupported_caches():
    w = inputs.make("c4", small=True)                  # INT4 KIVI with no ring: refused
    s = w.spec
    c = kvq.PagedKVCache(s.cache_dtype, s.act_dtype, s.scale_mode, w.num_blocks, s.block_size,
                         s.num_kv_heads, s.head_dim, device="cuda", residual_len=0,
                         residual_cap=inputs.RESIDUAL_CAP, max_seqs=max(s.batch, 1))
    k_new = torch.zeros((s.batch, s.num_kv_heads, s.head_dim), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(kvq.KVQError):
        c.append_decode(k_new, k_new, w.q.cuda(), w.block_tables.cuda(), w.context_lens.cuda(),
                        w.max_context)
    w1 = inputs.make("c1")                             # head_dim 64: CUDA-core decode
    c1 = helpers.gpu_cache(w1)
    k1 = torch.zeros((w1.spec.batch, w1.spec.num_kv_heads, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(kvq.KVQError):
        c1.append_decode(k1, k1, w1.q.cuda(), w1.block_tables.cuda(), w1.context_lens.cuda(),
                         w1.max_context)
