"""kvq_prefill_attention (chunked prefill) against the float64 oracle.

Each sequence's chunk of new queries is its newest tokens (their K/V rows already in the
cache); query i at position p attends to positions <= p.  Tolerance as decode: max
|gpu - oracle| <= 2e-3 with float32 output.
"""

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


def _queries(w, L, seed):
    g = torch.Generator().manual_seed(seed)
    qs = torch.tensor(np.concatenate([[0], np.cumsum(L)]), dtype=torch.int32)
    q = torch.randn((int(qs[-1]), w.spec.num_q_heads, w.spec.head_dim), generator=g)
    return q.to(inputs.act_torch_dtype(w.spec.act_dtype)), qs


def _prefill(gc, w, q, qs, lens=None):
    lens = w.context_lens if lens is None else lens
    L = (qs[1:] - qs[:-1])
    return gc.prefill(q.cuda(), qs.cuda(), int(L.max()), w.block_tables.cuda(), lens.cuda(),
                      int(lens.max()))


@pytest.mark.parametrize("name,L", [("c5", [37, 1, 33]), ("c5-fp8", [64, 5, 17]),
                                    ("c5-bf16", [3, 200, 33]), ("c5-int8-pc", [9, 16, 1]),
                                    ("c3", [7, 30, 1, 12]), ("c2", [40, 19]),
                                    ("c5", [300, 517, 16]), ("c5-int8-ph", [40, 100, 17]),
                                    ("c5-int8-pt", [128, 3, 33]), ("c5-fp8-pt", [1, 64, 20])])
def test_prefill_matches_oracle(name, L):
    w = inputs.make(name, small=True)
    L = [min(x, int(n)) for x, n in zip(L, w.context_lens.tolist())]
    static = helpers.oracle_static_scales(w)
    oc = helpers.oracle_cache(w, static)
    gc = helpers.gpu_cache(w, static=static)
    q, qs = _queries(w, L, 3)
    got = _prefill(gc, w, q, qs).cpu().numpy().astype(np.float64)
    want = attention.prefill_attention(oc, helpers.np64(q), qs.numpy(), w.block_tables.numpy(),
                                       w.context_lens.numpy())
    err = np.abs(got - want).max()
    assert err <= TOL, err
    assert gc.read_fault() == (0, 0)


def test_one_query_chunk_is_decode():
    w = inputs.make("c5", small=True)
    gc = helpers.gpu_cache(w)
    qs = torch.arange(w.spec.batch + 1, dtype=torch.int32)
    pre = _prefill(gc, w, w.q, qs)
    dec = gc.decode(w.q.cuda(), w.block_tables.cuda(), w.context_lens.cuda(), w.max_context)
    torch.cuda.synchronize()
    assert (pre - dec).abs().max().item() <= 1e-5


def test_rejected_sequences_are_counted_and_left_untouched():
    w = inputs.make("c5", small=True)
    gc = helpers.gpu_cache(w)
    L = [5, 4, 2]
    q, qs = _queries(w, L, 4)
    lens = w.context_lens.clone()
    lens[1] = 3                                   # 4 queries but 3 positions: rejected
    out = torch.full((int(qs[-1]), w.spec.num_q_heads, w.spec.head_dim), 7.0, device="cuda")
    kvq.kvq_prefill_attention(gc.desc, q.cuda(), qs.cuda(), 4, w.block_tables.cuda(), lens.cuda(),
                              int(lens.max()), out)  # max_q_len 4 < 5: sequence 0 rejected too
    torch.cuda.synchronize()
    cnt, bits = gc.read_fault()
    assert cnt >= 2 and (bits & 4)
    assert torch.all(out[qs[0]:qs[2]] == 7.0)
    assert torch.all(out[qs[2]:qs[3]] != 7.0)


def test_prefill_rejects_unsupported_caches():
    """head_dim 64 has no tensor-core prefill: refused before any launch."""
    spec = inputs.Spec("pf-d64", "int8", "fp16", "per_token_head", 2, 8, 4, 64, 16, lens=[40, 7],
                       slack_blocks=1, seed=5)
    w = inputs.from_spec(spec)
    c = helpers.gpu_cache(w)
    q, qs = _queries(w, [2, 2], 5)
    with pytest.raises(kvq.KVQError):
        _prefill(c, w, q, qs)


@pytest.mark.parametrize("name,L", [("c4", [100, 60]), ("c4-tok", [200, 1]), ("c4-fzp", [64, 130]),
                                    ("c4-int2", [100, 60]), ("c4-int2-tok", [37, 200]),
                                    ("c4-int2-fzp", [129, 5])])
def test_prefill_low_bit_matches_oracle(name, L):
    """INT4 / 2-bit caches: positions below the quantized prefix come from the 64-token
    blocks (dequantized exactly into bf16 hi + lo tiles), the newest from the residual ring."""
    w = inputs.make(name, small=True)
    oc = helpers.oracle_cache(w)
    gc = helpers.gpu_cache(w)
    q, qs = _queries(w, L, 10)
    got = _prefill(gc, w, q, qs).cpu().numpy().astype(np.float64)
    want = attention.prefill_attention(oc, helpers.np64(q), qs.numpy(), w.block_tables.numpy(),
                                       w.context_lens.numpy())
    err = np.abs(got - want).max()
    assert err <= TOL, err
    assert gc.read_fault() == (0, 0)


@pytest.mark.parametrize("cd,mode", [("int4", "kivi"), ("int2", "int4_per_token")])
def test_prefill_low_bit_long_context(cd, mode):
    """1200 cached tokens (16 blocks of 64 in the quantized prefix, so the four-stage page
    ring of the low-bit prefill turns over four times) and 300 queries."""
    spec = inputs.Spec("pf-%s-long" % cd, cd, "bf16", mode, 1, 16, 2, 128, 64, lens=[1200],
                       outliers="k", slack_blocks=3, seed=35)
    w = inputs.from_spec(spec)
    oc = helpers.oracle_cache(w)
    gc = helpers.gpu_cache(w)
    q, qs = _queries(w, [300], 12)
    got = _prefill(gc, w, q, qs).cpu().numpy().astype(np.float64)
    want = attention.prefill_attention(oc, helpers.np64(q), qs.numpy(), w.block_tables.numpy(),
                                       w.context_lens.numpy())
    assert np.abs(got - want).max() <= TOL
    assert gc.read_fault() == (0, 0)


def test_prefill_low_bit_fp16_activations():
    """fp16 activations with an INT4 cache: q goes to the tensor cores as an exact bf16
    hi + lo pair."""
    spec = inputs.Spec("pf-int4-fp16", "int4", "fp16", "kivi", 2, 8, 1, 128, 64, lens=[300, 150],
                       outliers="k", slack_blocks=2, seed=34)
    w = inputs.from_spec(spec)
    oc = helpers.oracle_cache(w)
    gc = helpers.gpu_cache(w)
    q, qs = _queries(w, [150, 150], 11)
    got = _prefill(gc, w, q, qs).cpu().numpy().astype(np.float64)
    want = attention.prefill_attention(oc, helpers.np64(q), qs.numpy(), w.block_tables.numpy(),
                                       w.context_lens.numpy())
    assert np.abs(got - want).max() <= TOL
    assert gc.read_fault() == (0, 0)


def test_prefill_full_size_sampled_queries():
    """A c5-shaped layer (batch 4, context 4096, 512-query chunks) at full size; sampled
    queries are checked against the oracle's decode at their positions (equal to prefill
    rows by definition, pinned on the CPU)."""
    import dataclasses
    spec = dataclasses.replace(inputs._spec("c5", False), batch=4, lens=[4096] * 4)
    w = inputs.from_spec(spec, "cuda")
    gc = helpers.gpu_cache(w)
    L = [512, 512, 300, 1]
    q, qs = _queries(w, L, 6)
    got = _prefill(gc, w, q, qs).cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    for b in (0, 2, 3):
        sub = helpers.single_sequence(w, b)
        oc = helpers.oracle_cache(sub)
        for i in sorted({0, L[b] // 2, L[b] - 1}):
            p = int(w.context_lens[b]) - L[b] + i
            want = attention.decode_attention(oc, helpers.np64(q[qs[b] + i])[None],
                                              sub.block_tables.numpy(), np.array([p + 1]))[0]
            err = np.abs(got[qs[b] + i] - want).max()
            assert err <= TOL, (b, i, err)
    assert gc.read_fault() == (0, 0)


def test_more_queries_than_max_q_len_are_rejected():
    """max_q_len is the contract's bound even where the grid covers more queries (a CTA
    takes four): a sequence of 4 queries with max_q_len 3 is skipped and counted."""
    w = inputs.make("c5", small=True)
    gc = helpers.gpu_cache(w)
    L = [4, 2, 3]
    q, qs = _queries(w, L, 7)
    out = torch.full((int(qs[-1]), w.spec.num_q_heads, w.spec.head_dim), 7.0, device="cuda")
    kvq.kvq_prefill_attention(gc.desc, q.cuda(), qs.cuda(), 3, w.block_tables.cuda(),
                              w.context_lens.cuda(), w.max_context, out)
    torch.cuda.synchronize()
    cnt, bits = gc.read_fault()
    assert cnt >= 1 and (bits & 4)
    assert torch.all(out[qs[0]:qs[1]] == 7.0)
    assert torch.all(out[qs[1]:qs[3]] != 7.0)


# Other GQA groups, activation types and cache types: g = 2 (64 query tokens per tile) with
# fp16 activations, an fp16 cache, and MHA with fp16 activations; lengths that put query
# tiles across 128-token block boundaries and leave ragged last tiles.
SPECS = {
    "g2-fp16act": (inputs.Spec("pf-g2", "int8", "fp16", "per_token_head", 3, 4, 2, 128, 16,
                               lens=[700, 300, 129], slack_blocks=5, seed=31), [257, 64, 129]),
    "fp16-cache": (inputs.Spec("pf-fp16", "fp16", "fp16", "none", 2, 8, 1, 128, 16,
                               lens=[400, 130], slack_blocks=2, seed=32), [200, 130]),
    "fp8-mha-fp16act": (inputs.Spec("pf-mha", "fp8", "fp16", "per_token_head", 2, 2, 2, 128, 16,
                                    lens=[333, 47], slack_blocks=2, seed=33), [160, 47]),
    # MHA over a bf16 cache: the rows copied straight into the tiles, 128-token query tiles
    "bf16-mha": (inputs.Spec("pf-bf16-mha", "bf16", "bf16", "none", 3, 4, 4, 128, 16,
                             lens=[333, 129, 260], slack_blocks=3, seed=34), [300, 129, 5]),
}


@pytest.mark.parametrize("key", sorted(SPECS))
def test_prefill_groups_and_types(key):
    spec, L = SPECS[key]
    w = inputs.from_spec(spec)
    static = helpers.oracle_static_scales(w)
    oc = helpers.oracle_cache(w, static)
    gc = helpers.gpu_cache(w, static=static)
    q, qs = _queries(w, L, 8)
    got = _prefill(gc, w, q, qs).cpu().numpy().astype(np.float64)
    want = attention.prefill_attention(oc, helpers.np64(q), qs.numpy(), w.block_tables.numpy(),
                                       w.context_lens.numpy())
    err = np.abs(got - want).max()
    assert err <= TOL, err
    assert gc.read_fault() == (0, 0)


@pytest.mark.parametrize("name", ["c5", "c5-bf16"])
def test_prefill_bad_block_is_masked_and_counted(name):
    """A block-table entry outside the pool: its tokens are left out of every query's window
    (as if masked), the fault record counts it, and nothing else changes.  (bf16 caches take
    the path whose pages are copied straight into the tiles: the bad page's rows are never
    written there, so its V rows are zeroed and its scores masked.)"""
    w = inputs.make(name, small=True)
    oc = helpers.oracle_cache(w)
    gc = helpers.gpu_cache(w)
    L = [50, 20, 5]
    q, qs = _queries(w, L, 9)
    tables = w.block_tables.clone()
    tables[0, 2] = w.num_blocks + 3                   # positions 32..47 of sequence 0
    out = gc.prefill(q.cuda(), qs.cuda(), max(L), tables.cuda(), w.context_lens.cuda(),
                     int(w.context_lens.max())).cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    cnt, bits = gc.read_fault()
    assert cnt > 0 and bits == 2                      # the bad entry alone: no wait ran out
    assert np.isfinite(out).all()
    # sequence 0 without positions 32..47: the oracle over the remaining positions
    K, V = oc.gather(w.block_tables.numpy()[0], int(w.context_lens[0]))
    n = int(w.context_lens[0])
    keep = np.array([p for p in range(n) if not 32 <= p < 48])
    g = w.spec.num_q_heads // w.spec.num_kv_heads
    qq = helpers.np64(q)
    for i in (0, 25, 49):
        p = n - L[0] + i
        vis = keep[keep <= p]
        for hq in range(w.spec.num_q_heads):
            want = attention.softmax_attention(qq[i, hq], K[hq // g][vis], V[hq // g][vis],
                                               1.0 / np.sqrt(w.spec.head_dim))
            assert np.abs(out[i, hq] - want).max() <= TOL, (i, hq)
    want = attention.prefill_attention(oc, qq, qs.numpy(), w.block_tables.numpy(),
                                       w.context_lens.numpy())
    assert np.abs(out[qs[1]:] - want[qs[1]:]).max() <= TOL
