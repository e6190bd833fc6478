"""Pins of the paged cache model and of the attention oracle.

Anchors: torch's scaled_dot_product_attention in float64 on the dense, unquantized rows
(a library routine) when quantization is exact; closed-form invariants (one token gives
v_0; q = 0 gives the mean of v; permuting physical blocks changes nothing); the sentinel
bytes of blocks no write touched.
"""

import numpy as np
import pytest
import torch

from oracle import attention, cache, fp, quant
from quantized_paged_kv_02_b200 import inputs


def _np(t):
    return t.detach().to(torch.float64).cpu().numpy()


def _build(w, static_scales=None, max_seqs=None):
    s = w.spec
    c = cache.PagedCache(s.cache_dtype, s.act_dtype, s.scale_mode, w.num_blocks, s.block_size,
                         s.num_kv_heads, s.head_dim, residual_len=inputs.RESIDUAL_LEN,
                         residual_cap=inputs.RESIDUAL_CAP,
                         max_seqs=max_seqs or s.batch, static_scales=static_scales)
    if inputs.low_bit(s.cache_dtype):
        idx, slots, sid, pos = inputs.int4_group_rows(w)
        c.write(_np(w.k)[idx.numpy()], _np(w.v)[idx.numpy()], slots.numpy(), sid.numpy(), pos.numpy())
    else:
        c.write(_np(w.k), _np(w.v), w.slot_mapping.numpy())
    return c


def _sdpa(q, K, V, scale):
    """torch SDPA in float64 for one query row against dense K, V [n, D]."""
    qq = torch.from_numpy(q)[None, None, None, :]
    kk = torch.from_numpy(K)[None, None]
    vv = torch.from_numpy(V)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=scale)[0, 0, 0].numpy()


# ---------------------------------------------------------------- grid-exact special cases
def _grid_int8_rows(rng, T, H, D):
    """Rows k * 2^-e with one element +-127 * 2^-e per row: INT8 is exact on them."""
    e = rng.integers(2, 6, size=(T, H, 1))
    k = rng.integers(-127, 128, size=(T, H, D))
    k[..., 0] = rng.choice([-127, 127], size=(T, H))
    return (k * np.exp2(-e.astype(np.float64)))


def test_int8_grid_exact_attention_equals_sdpa():
    rng = np.random.default_rng(0)
    T, H, D, g, bs = 70, 2, 64, 3, 16
    K = _grid_int8_rows(rng, T, H, D)
    V = _grid_int8_rows(rng, T, H, D)
    nblk = -(-T // bs)
    perm = rng.permutation(nblk + 2)[:nblk]
    slots = np.array([perm[p // bs] * bs + p % bs for p in range(T)])
    c = cache.PagedCache("int8", "bf16", "per_token_head", nblk + 2, bs, H, D)
    c.write(K, V, slots)
    q = rng.standard_normal((1, H * g, D)).astype(np.float32).astype(np.float64)
    q = fp.bf16_round(q)
    out = attention.decode_attention(c, q, perm[None, :], np.array([T]))
    scale = 1.0 / np.sqrt(D)
    for hq in range(H * g):
        ref = _sdpa(q[0, hq], K[:, hq // g], V[:, hq // g], scale)
        np.testing.assert_allclose(out[0, hq], ref, rtol=1e-12, atol=1e-12)


def test_fp8_grid_exact_attention_equals_sdpa():
    rng = np.random.default_rng(1)
    T, H, D, bs = 40, 2, 64, 16
    t = fp.e4m3_decode_table()
    vals = t[np.isfinite(t) & (np.abs(t) <= 16)]
    ks, vs = np.array([0.25, 0.5], np.float32), np.array([2.0, 0.125], np.float32)
    K = rng.choice(vals, size=(T, H, D)) * ks[None, :, None]
    V = rng.choice(vals, size=(T, H, D)) * vs[None, :, None]
    nblk = -(-T // bs)
    slots = np.arange(T)
    c = cache.PagedCache("fp8", "bf16", "per_head", nblk, bs, H, D, static_scales=(ks, vs))
    c.write(K, V, slots)
    q = fp.bf16_round(rng.standard_normal((1, H, D)))
    out = attention.decode_attention(c, q, np.arange(nblk)[None, :], np.array([T]), softmax_scale=0.3)
    for h in range(H):
        np.testing.assert_allclose(out[0, h], _sdpa(q[0, h], K[:, h], V[:, h], 0.3), rtol=1e-12, atol=1e-12)


def test_int8_per_channel_grid_exact_attention_equals_sdpa():
    """Static per-(head, channel) INT8 scales that are powers of two, values k * s_d with
    integer |k| <= 127: quantization is exact, so attention equals dense SDPA."""
    rng = np.random.default_rng(3)
    T, H, D, g, bs = 50, 2, 64, 4, 16
    ks = np.exp2(-rng.integers(0, 6, size=(H, D))).astype(np.float32)
    vs = np.exp2(-rng.integers(0, 6, size=(H, D))).astype(np.float32)
    K = rng.integers(-127, 128, size=(T, H, D)) * ks[None].astype(np.float64)
    V = rng.integers(-127, 128, size=(T, H, D)) * vs[None].astype(np.float64)
    nblk = -(-T // bs)
    perm = rng.permutation(nblk + 1)[:nblk]
    slots = np.array([perm[p // bs] * bs + p % bs for p in range(T)])
    c = cache.PagedCache("int8", "bf16", "per_channel", nblk + 1, bs, H, D, static_scales=(ks, vs))
    c.write(K, V, slots)
    K2, V2 = c.gather(perm, T)
    np.testing.assert_array_equal(K2, np.transpose(K, (1, 0, 2)))
    np.testing.assert_array_equal(V2, np.transpose(V, (1, 0, 2)))
    q = fp.bf16_round(rng.standard_normal((1, H * g, D)))
    out = attention.decode_attention(c, q, perm[None, :], np.array([T]))
    for hq in range(H * g):
        ref = _sdpa(q[0, hq], K[:, hq // g], V[:, hq // g], 1.0 / np.sqrt(D))
        np.testing.assert_allclose(out[0, hq], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("cd", ["int8", "fp8"])
def test_per_channel_with_equal_channels_is_per_head(cd):
    """A per-channel cache whose channels of a head all carry that head's scale stores
    exactly the bytes of the per-head cache (and dequantizes to the same values)."""
    rng = np.random.default_rng(4)
    T, H, D, bs = 37, 3, 64, 16
    x = fp.bf16_round(rng.standard_normal((T, H, D)) * 3)
    y = fp.bf16_round(rng.standard_normal((T, H, D)))
    sh = np.array([0.03, 0.011, 0.2], np.float32)
    nblk = -(-T // bs)
    a = cache.PagedCache(cd, "bf16", "per_head", nblk, bs, H, D, static_scales=(sh, sh * 2))
    b = cache.PagedCache(cd, "bf16", "per_channel", nblk, bs, H, D,
                         static_scales=(np.repeat(sh[:, None], D, 1), np.repeat((sh * 2)[:, None], D, 1)))
    a.write(x, y, np.arange(T))
    b.write(x, y, np.arange(T))
    np.testing.assert_array_equal(a.pages, b.pages)
    for blk in range(nblk):
        np.testing.assert_array_equal(a.dequant_block(blk), b.dequant_block(blk))


def test_channel_calibration():
    """scale[h, d] = binary32(max_t |x[t, h, d]| / qmax); each channel on its own."""
    rng = np.random.default_rng(5)
    w = fp.bf16_round(rng.standard_normal((256, 2, 64))).astype(np.float32)
    s = quant.channel_calibrate(w, 127.0)
    assert s.shape == (2, 64) and s.dtype == np.float32
    for h in range(2):
        for d in (0, 17, 63):
            assert s[h, d] == fp.div32(np.float32(np.abs(w[:, h, d]).max()), np.float32(127.0))
    w2 = w.copy()
    w2[:, 1, 5] *= 4
    s2 = quant.channel_calibrate(w2, 448.0)
    s1 = quant.channel_calibrate(w, 448.0)
    assert s2[1, 5] == fp.div32(np.float32(4 * np.abs(w[:, 1, 5]).max()), np.float32(448.0))
    mask = np.ones_like(s1, bool)
    mask[1, 5] = False
    np.testing.assert_array_equal(s2[mask], s1[mask])


def test_int4_grid_exact_attention_equals_sdpa():
    """Keys on a per-channel grid over each 64-token block, values on a per-token grid
    over each 64-channel group, plus unquantized residual rows: exact."""
    rng = np.random.default_rng(2)
    H, D, n = 1, 128, 64 * 3 + 128 + 21          # 3 blocks + 149 ring rows
    qb = 64 * ((n - 128) // 64)
    assert qb == 192
    K = np.empty((n, H, D))
    V = np.empty((n, H, D))
    for blk in range(qb // 64):
        for d in range(D):
            k = rng.integers(0, 16, 64)
            k[0], k[1] = 0, 15
            z0, e = rng.integers(0, 16), rng.integers(1, 5)
            K[blk * 64:(blk + 1) * 64, 0, d] = (k - z0) * 2.0 ** -e
    for p in range(qb):
        for gi in range(2):
            k = rng.integers(0, 16, 64)
            k[0], k[1] = 0, 15
            z0, e = rng.integers(0, 16), rng.integers(1, 5)
            V[p, 0, gi * 64:(gi + 1) * 64] = (k - z0) * 2.0 ** -e
    K[qb:] = fp.bf16_round(rng.standard_normal((n - qb, H, D)))
    V[qb:] = fp.bf16_round(rng.standard_normal((n - qb, H, D)))
    c = cache.PagedCache("int4", "bf16", "kivi", 5, 64, H, D, max_seqs=2)
    table = np.array([3, 0, 4])
    rows = list(range(qb)) + list(range(qb, n))
    slots = np.array([table[p // 64] * 64 + p % 64 for p in range(qb)] + [-1] * (n - qb))
    pos = np.array([-1] * qb + list(range(qb, n)))
    sid = np.ones(n, np.int64)
    c.write(K[rows], V[rows], slots, sid, pos)
    q = fp.bf16_round(rng.standard_normal((1, 4, D)))
    out = attention.decode_attention(c, q, table[None, :], np.array([n]), seq_ids=np.array([1]))
    for hq in range(4):
        np.testing.assert_allclose(out[0, hq], _sdpa(q[0, hq], K[:, 0], V[:, 0], 1 / np.sqrt(D)),
                                   rtol=1e-12, atol=1e-12)
    # untouched blocks keep the sentinel
    for blk in (1, 2):
        assert np.all(c.k_codes[blk] == cache.SENTINEL) and np.all(c.v_codes[blk] == cache.SENTINEL)


@pytest.mark.parametrize("cd,mode", [("int4", "int4_per_token"), ("int4", "kivi_float_zero"),
                                     ("int2", "kivi"), ("int2", "int4_per_token"),
                                     ("int2", "kivi_float_zero")])
def test_int4_variants_grid_exact_attention_equals_sdpa(cd, mode):
    """The per-token variant (keys grouped per token over 64 channels, like values), the
    float-zero-point variant (offset = group minimum, the range need not include 0) and the
    2-bit caches: on their grids quantization is exact, so attention equals SDPA on the
    dense rows."""
    rng = np.random.default_rng(3)
    H, D, n = 1, 128, 64 * 3 + 128 + 21
    qb = 192
    Q = int(quant.levels(cache.LOW_BIT[cd]))

    def grid():
        k = rng.integers(0, Q + 1, 64)
        k[0], k[1] = 0, Q
        e = rng.integers(1, 5)
        if mode == "kivi_float_zero":
            return rng.integers(-40, 41) * 2.0 ** -3 + k * 2.0 ** -e
        return (k - rng.integers(0, Q + 1)) * 2.0 ** -e

    K = np.empty((n, H, D))
    V = np.empty((n, H, D))
    for p in range(qb):
        for gi in range(2):
            V[p, 0, gi * 64:(gi + 1) * 64] = grid()
            if mode == "int4_per_token":
                K[p, 0, gi * 64:(gi + 1) * 64] = grid()
    if mode != "int4_per_token":
        for blk in range(qb // 64):
            for d in range(D):
                K[blk * 64:(blk + 1) * 64, 0, d] = grid()
    K[qb:] = fp.bf16_round(rng.standard_normal((n - qb, H, D)))
    V[qb:] = fp.bf16_round(rng.standard_normal((n - qb, H, D)))
    assert np.array_equal(fp.bf16_round(K), K) and np.array_equal(fp.bf16_round(V), V)
    c = cache.PagedCache(cd, "bf16", mode, 5, 64, H, D, max_seqs=2)
    table = np.array([3, 0, 4])
    slots = np.array([table[p // 64] * 64 + p % 64 for p in range(qb)] + [-1] * (n - qb))
    pos = np.array([-1] * qb + list(range(qb, n)))
    c.write(K, V, slots, np.ones(n, np.int64), pos)
    assert c.record == {"int4": 9216, "int2": 5120}[cd]
    q = fp.bf16_round(rng.standard_normal((1, 4, D)))
    out = attention.decode_attention(c, q, table[None, :], np.array([n]), seq_ids=np.array([1]))
    for hq in range(4):
        np.testing.assert_allclose(out[0, hq], _sdpa(q[0, hq], K[:, 0], V[:, 0], 1 / np.sqrt(D)),
                                   rtol=1e-12, atol=1e-12)
    if mode == "kivi_float_zero":
        assert np.any(c.k_scales[table, 0, 1, :] > 0)      # minima above 0 occur
    elif mode == "int4_per_token":
        assert c.k_scales.shape[2:] == (64, 2, 2)          # [bs][D/64][(scale, zero)]


# ---------------------------------------------------------------- invariants
@pytest.mark.parametrize("name", ["c1", "c2", "c3", "c4", "c4-tok", "c4-fzp", "c4-int2",
                                  "c4-int2-tok", "c4-int2-fzp", "c5"])
def test_invariants_on_small_workloads(name):
    w = inputs.make(name, small=True)
    s = w.spec
    static = None
    if s.scale_mode == "per_head":
        static = (quant.fp8_calibrate(_np(w.warmup_k).astype(np.float32)),
                  quant.fp8_calibrate(_np(w.warmup_v).astype(np.float32)))
    c = _build(w, static)
    q = _np(w.q)
    lens = w.context_lens.numpy()
    tables = w.block_tables.numpy()
    out = attention.decode_attention(c, q, tables, lens)
    assert np.all(np.isfinite(out))
    # gathered rows reconstruct the inputs within the quantizer's error
    for b in range(s.batch):
        n = int(lens[b])
        K, V = c.gather(tables[b], n, b)
        r0 = int(w.seq_start[b])
        kk = _np(w.k)[r0:r0 + n].transpose(1, 0, 2)
        err = np.abs(K - kk)
        if s.cache_dtype == "int8":          # |x - q s| <= s (1/2 + 2^-17), s = max|row| / 127
            bound = np.abs(kk).max(axis=-1, keepdims=True) / 127 * (0.5 + 2.0 ** -17) * (1 + 2.0 ** -23)
        elif s.cache_dtype == "fp8":         # 3 mantissa bits, plus saturation at 448 s
            sk = static[0].astype(np.float64)[:, None, None]
            bound = np.abs(kk) / 16 + np.maximum(np.abs(kk) - 448 * sk, 0) + sk * 2.0 ** -10
        elif inputs.low_bit(s.cache_dtype):  # half a step of the widest group
            qb = c.quantized_prefix(n)
            rng_ = np.abs(kk).max() * 2
            Q = quant.levels(cache.LOW_BIT[s.cache_dtype])
            bound = np.full(kk.shape, rng_ / Q * (0.5 + Q * 2.0 ** -11))
            bound[:, qb:] = 0                # residual ring rows are exact
        else:
            bound = np.zeros(kk.shape)
        assert np.all(err <= bound + 1e-12)
    # block permutation: move every used block to another physical id, same output
    NB = w.num_blocks
    perm = np.random.default_rng(5).permutation(NB)
    c2 = _build_permuted(w, static, perm)
    out2 = attention.decode_attention(c2, q, perm[tables], lens)
    np.testing.assert_array_equal(out, out2)


def _build_permuted(w, static, perm):
    s = w.spec
    slots = w.slot_mapping.numpy().astype(np.int64)
    new = np.where(slots >= 0, perm[slots // s.block_size] * s.block_size + slots % s.block_size, -1)
    c = cache.PagedCache(s.cache_dtype, s.act_dtype, s.scale_mode, w.num_blocks, s.block_size,
                         s.num_kv_heads, s.head_dim, max_seqs=s.batch, static_scales=static)
    if inputs.low_bit(s.cache_dtype):
        idx, _, sid, pos = inputs.int4_group_rows(w)
        c.write(_np(w.k)[idx.numpy()], _np(w.v)[idx.numpy()], new[idx.numpy()], sid.numpy(), pos.numpy())
    else:
        c.write(_np(w.k), _np(w.v), new)
    return c


def test_one_token_and_zero_query():
    w = inputs.make("c1")
    c = _build(w)
    lens = np.array([1, 77])
    q = _np(w.q)
    out = attention.decode_attention(c, q, w.block_tables.numpy(), lens)
    K, V = c.gather(w.block_tables.numpy()[0], 1)
    for hq in range(8):
        np.testing.assert_array_equal(out[0, hq], V[hq // 2, 0])
    out0 = attention.decode_attention(c, np.zeros_like(q), w.block_tables.numpy(), lens)
    K, V = c.gather(w.block_tables.numpy()[1], 77)
    for hq in range(8):
        np.testing.assert_allclose(out0[1, hq], V[hq // 2].mean(axis=0), rtol=1e-13, atol=1e-13)


def test_empty_context_gives_zeros():
    w = inputs.make("c1")
    c = _build(w)
    out = attention.decode_attention(c, _np(w.q), w.block_tables.numpy(), np.array([0, 5]))
    assert np.all(out[0] == 0)


def test_write_touches_only_its_slots():
    w = inputs.make("c1")
    c = _build(w)
    used = set(w.block_tables.numpy()[0, :8]) | set(w.block_tables.numpy()[1, :5])
    for blk in range(w.num_blocks):
        untouched = np.all(c.k_codes[blk].view(np.uint8) == cache.SENTINEL)
        assert untouched == (blk not in used)
    # block of sequence 1 holding positions 64..76: offsets 13..15 keep the sentinel
    last = w.block_tables.numpy()[1, 4]
    assert np.all(c.k_codes[last][:, 13:].view(np.uint8) == cache.SENTINEL)
    written = c.k_codes[last][:, :13].view(np.uint8)          # [H, 13, D]
    assert not np.any(np.all(written == cache.SENTINEL, axis=-1))
    sc = c.k_scales[last].view(np.uint32)                     # [H, bs]
    assert np.all(sc[:, 13:] == 0x5A5A5A5A) and not np.any(sc[:, :13] == 0x5A5A5A5A)


def test_int4_prefix_split():
    c = cache.PagedCache("int4", "bf16", "kivi", 4, 64, 1, 128, max_seqs=1)
    assert [c.quantized_prefix(n) for n in (0, 100, 128, 191, 192, 255, 256, 32768)] == \
        [0, 0, 0, 0, 64, 64, 128, 32640]


@pytest.mark.parametrize("name", ["c4", "c4-tok", "c4-fzp", "c4-int2", "c4-int2-fzp"])
def test_flush_ring_equals_writing_the_rows(name):
    """Flushing ring rows [p0, p0+64) into a block stores what writing those rows with the
    block's slots stores (the definition in include/kvq.h)."""
    w = inputs.make(name, small=True)
    c = _build(w)
    s = w.spec
    n0 = int(w.context_lens[0])
    qb = 64 * (max(n0 - inputs.RESIDUAL_LEN, 0) // 64)
    used = set(w.block_tables.numpy().reshape(-1).tolist())
    free = [b for b in range(w.num_blocks) if b not in used][0]
    c.flush_ring([0], [qb], [free])
    ref = _build(w)
    rows = np.arange(int(w.seq_start[0]) + qb, int(w.seq_start[0]) + qb + 64)
    ref.write(_np(w.k)[rows], _np(w.v)[rows], free * 64 + np.arange(64))
    np.testing.assert_array_equal(c.pages[free], ref.pages[free])
    assert not np.array_equal(c.pages[free], _build(w).pages[free])       # it did write


def test_prefill_rows_are_decode_at_their_positions():
    """Query i of a chunk at position p sees exactly what decode with context p + 1 sees;
    a one-token chunk is decode."""
    w = inputs.make("c5", small=True)
    c = _build(w)
    lens = w.context_lens.numpy()
    L = np.array([5, 1, 33])                     # chunk lengths (the last L_b tokens)
    qs = np.concatenate([[0], np.cumsum(L)])
    rng = np.random.default_rng(7)
    q = fp.bf16_round(rng.standard_normal((qs[-1], w.spec.num_q_heads, w.spec.head_dim)))
    out = attention.prefill_attention(c, q, qs, w.block_tables.numpy(), lens)
    for b in range(len(lens)):
        for i in range(L[b]):
            p = lens[b] - L[b] + i
            want = attention.decode_attention(c, q[qs[b] + i][None], w.block_tables.numpy()[b:b + 1],
                                              np.array([p + 1]))
            np.testing.assert_array_equal(out[qs[b] + i], want[0])


@pytest.mark.parametrize("name", ["c4", "c4-int2-tok"])
def test_prefill_rows_are_decode_on_low_bit_caches(name):
    """INT4 / 2-bit caches: query i at position p sees blocks for positions below the
    quantized prefix of p + 1 and the residual ring above it, exactly what decode with
    context p + 1 of the same ring sequence sees (the ring holds every position the
    chunk needs, since the chunk's rows were written before it)."""
    w = inputs.make(name, small=True)
    c = _build(w)
    lens = w.context_lens.numpy()
    L = np.array([100, 60])
    qs = np.concatenate([[0], np.cumsum(L)])
    rng = np.random.default_rng(9)
    q = fp.bf16_round(rng.standard_normal((qs[-1], w.spec.num_q_heads, w.spec.head_dim)))
    out = attention.prefill_attention(c, q, qs, w.block_tables.numpy(), lens)
    for b in range(len(lens)):
        for i in (0, L[b] // 2, L[b] - 1):
            p = lens[b] - L[b] + i
            want = attention.decode_attention(c, q[qs[b] + i][None], w.block_tables.numpy()[b:b + 1],
                                              np.array([p + 1]), seq_ids=np.array([b]))
            if c.quantized_prefix(p + 1) == c.quantized_prefix(lens[b]):
                np.testing.assert_array_equal(out[qs[b] + i], want[0])


def test_prefill_grid_exact_equals_causal_sdpa():
    """On a grid-exact INT8 cache the chunk's output equals torch's causal SDPA over the
    dense rows (the prefix positions are all visible, the chunk is causal)."""
    rng = np.random.default_rng(8)
    T, H, D, g, bs, L = 45, 2, 64, 2, 16, 13
    K = _grid_int8_rows(rng, T, H, D)
    V = _grid_int8_rows(rng, T, H, D)
    nblk = -(-T // bs)
    c = cache.PagedCache("int8", "bf16", "per_token_head", nblk, bs, H, D)
    c.write(K, V, np.arange(T))
    q = fp.bf16_round(rng.standard_normal((L, H * g, D)))
    out = attention.prefill_attention(c, q, np.array([0, L]), np.arange(nblk)[None], np.array([T]))
    for hq in range(H * g):
        qq = torch.from_numpy(q[:, hq])[None, None]                     # [1, 1, L, D]
        kk = torch.from_numpy(K[:, hq // g])[None, None]                # [1, 1, T, D]
        vv = torch.from_numpy(V[:, hq // g])[None, None]
        mask = torch.ones(L, T, dtype=torch.bool).tril(diagonal=T - L)  # query i sees t <= T-L+i
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask,
                                                               scale=1.0 / np.sqrt(D))[0, 0]
        np.testing.assert_allclose(out[:, hq], ref.numpy(), rtol=1e-12, atol=1e-12)
