"""Pins of the size formula against the worked examples the pages print."""

import os
from fractions import Fraction

from oracle import bytes_model


def _rows(path):
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [c.strip() for c in line.split("|")]


def test_printed_size_examples(golden_dir):
    rows = list(_rows(os.path.join(golden_dir, "bytes_examples.txt")))
    assert len(rows) == 5
    for name, shape, printed, exact, relation in rows:
        L, H, d, S, B, dt = shape.split()
        got = bytes_model.kv_cache_bytes(int(L), int(H), int(d), int(S), dt, batch=int(B))
        if relation == "exact":
            assert got == int(exact), name
            # and the printed GB figure (binary GB, as in [P-mem] §2.2)
            gb = Fraction(printed.rstrip("GB"))
            assert got == gb * 2 ** 30, name
        else:
            assert got == int(exact), name
            assert abs(got - Fraction(5 * 10 ** 9)) <= Fraction(5 * 10 ** 8), name


def test_bytes_per_value_table(golden_dir):
    rows = list(_rows(os.path.join(golden_dir, "bytes_per_value.txt")))
    for fmt, bpv, ratio in rows:
        assert bytes_model.BYTES_PER_VALUE[fmt] == Fraction(bpv)
        assert Fraction(2) / bytes_model.BYTES_PER_VALUE[fmt] == Fraction(ratio)


def test_int8_halves_fp16():
    # [P-mem] §5: every row has INT8 = FP16 / 2 ("节省比例 50%")
    for L, H, S in ((32, 32, 1024), (40, 40, 2048), (80, 8, 4096)):
        assert 2 * bytes_model.kv_cache_bytes(L, H, 128, S, "int8") == \
            bytes_model.kv_cache_bytes(L, H, 128, S, "fp16")


def test_decode_step_bytes_components():
    """Per-config byte counts, decomposed by hand from the layout in include/kvq.h."""
    # Llama-2-7B layer, INT8 per-token-head, batch 4 x 2048 tokens, MHA 32 heads
    b = bytes_model.decode_step_bytes("int8", "per_token_head", 4, 32, 32, 128, [2048] * 4, 16)
    codes = 2 * 32 * 128 * 2048 * 4           # K and V, 1 byte per value
    scales = 2 * 32 * 2048 * 4 * 4            # fp32 per token per head, K and V
    meta = 4 * (2048 // 16) * 4 + 4 * 4       # block table entries + context lengths
    qo = 2 * 4 * 32 * 128 * 2
    assert codes == 67108864 and scales == 2097152
    assert b == codes + scales + meta + qo
    # the per-layer c2 slice is 1/32 of the [P-mem] §2.2 INT8 total (32 layers)
    assert codes * 32 == bytes_model.kv_cache_bytes(32, 32, 128, 2048, "int8", batch=4)

    # KIVI INT4, 16 x 32768 tokens, 8 kv heads: 32640 quantized + 128 residual
    b4 = bytes_model.decode_step_bytes("int4", "kivi", 16, 64, 8, 128, [32768] * 16, 64)
    per_unit = 2088960 + 261120 + 2088960 + 261120 + 65536     # one (sequence, kv head)
    assert per_unit == 4765696
    meta4 = 16 * (4 * 510 + 4)
    assert b4 == per_unit * 128 + meta4 + 2 * 16 * 64 * 128 * 2

    # 70B-shaped step, 24 x 16384 tokens, 8 kv heads
    b8 = bytes_model.decode_step_bytes("int8", "per_token_head", 24, 64, 8, 128, [16384] * 24, 16)
    assert b8 - (24 * (4 * 1024 + 4) + 2 * 24 * 64 * 128 * 2) == 830472192
    bf = bytes_model.decode_step_bytes("bf16", "none", 24, 64, 8, 128, [16384] * 24, 16)
    assert bf - (24 * (4 * 1024 + 4) + 2 * 24 * 64 * 128 * 2) == 1610612736


def test_decode_step_bytes_low_bit_forms():
    """2-bit codes and keys grouped per token, decomposed by hand per (sequence, kv head)
    from the record layout: 16 x 32768 tokens, 8 kv heads, 32640 tokens in 510 blocks of
    64 and 128 in the bf16 residual ring ([P-prod] "KV Cache 的基本内存模型": 0.25 byte
    per value for 2-bit; the scale and zero-point bytes are the metadata that section says
    makes the gain smaller)."""
    meta = 16 * (4 * 510 + 4)                          # block-table entries + lengths
    qo = 2 * 16 * 64 * 128 * 2                         # q read + out written, bf16
    ring = 2 * 128 * 128 * 2                           # K and V ring rows
    v_sz = 32640 * 2 * 2 * 2                           # V (scale, zero) per token, 2 groups
    k_sz_chan = 510 * 2 * 128 * 2                      # KIVI K (scale, zero) per channel
    k_sz_tok = 32640 * 2 * 2 * 2                       # K (scale, zero) per token, 2 groups
    codes4, codes2 = 32640 * 128 // 2, 32640 * 128 // 4
    assert (codes4, codes2, v_sz, k_sz_chan, k_sz_tok) == (2088960, 1044480, 261120, 261120, 261120)
    cases = {
        ("int4", "kivi"): 2 * codes4 + k_sz_chan + v_sz + ring,
        ("int4", "kivi_float_zero"): 2 * codes4 + k_sz_chan + v_sz + ring,
        ("int4", "int4_per_token"): 2 * codes4 + k_sz_tok + v_sz + ring,
        ("int2", "kivi"): 2 * codes2 + k_sz_chan + v_sz + ring,
        ("int2", "kivi_float_zero"): 2 * codes2 + k_sz_chan + v_sz + ring,
        ("int2", "int4_per_token"): 2 * codes2 + k_sz_tok + v_sz + ring,
    }
    for (cd, mode), per_unit in cases.items():
        got = bytes_model.decode_step_bytes(cd, mode, 16, 64, 8, 128, [32768] * 16, 64)
        assert got == per_unit * 128 + meta + qo, (cd, mode)
    assert cases[("int2", "kivi")] == 2676736
    # short sequences: everything in the ring (n <= 128 + 63 keeps no whole group)
    got = bytes_model.decode_step_bytes("int2", "int4_per_token", 2, 16, 2, 128, [100, 191], 64)
    assert got == 2 * 2 * (100 + 191) * 128 * 2 + 2 * 4 + 2 * 16 * 128 * 4
    # one group: 192 tokens -> 64 in a block, 128 in the ring
    got = bytes_model.decode_step_bytes("int2", "kivi", 1, 8, 1, 128, [192], 64)
    assert got == (2 * 64 * 32 + 2 * 128 * 2 + 64 * 2 * 4 + 2 * 128 * 128 * 2) + 4 + 4 + 8 * 128 * 4


def test_bench_byte_counts_equal_the_oracle_model():
    """The byte counts the benchmark divides by (the package's roofline module) equal the
    oracle's model for every workload the benchmark runs, at full size and on a ragged
    length mix."""
    import random
    import bench
    from quantized_paged_kv_02_b200 import inputs, roofline
    rng = random.Random(7)
    for name in sorted(bench.WORKLOADS):
        s = inputs._spec(name, False)
        mixes = []
        if s.lens:
            mixes.append(s.lens)
        else:
            mixes.append([rng.randint(*s.len_range) for _ in range(s.batch)])
        mixes.append([0, 1, 63, 64, 127, 128, 191, 192, 193, 1000, 4097])
        for lens in mixes:
            want = bytes_model.decode_step_bytes(s.cache_dtype, s.scale_mode, len(lens),
                                                 s.num_q_heads, s.num_kv_heads, s.head_dim,
                                                 lens, s.block_size)
            got = roofline.decode_bytes(s.cache_dtype, s.scale_mode, s.num_q_heads,
                                        s.num_kv_heads, s.head_dim, s.block_size, lens)
            assert want.denominator == 1 and got == int(want), (name, lens)


def test_write_step_bytes_components():
    """The prefill write of the c5 layer (4 x 8192 new tokens, 8 kv heads, D 128, bf16 rows),
    decomposed by hand: rows read 2 x 32768 x 8 x 128 x 2 = 134,217,728 B plus 4 B of slot id
    per token; INT8 per token writes 1 byte per value plus a float32 scale per (token, kv head)
    for K and V (67,108,864 + 2,097,152 = 69,206,016 B); FP8 with a static per-head scale
    writes the codes only."""
    rows_read, slots = 2 * 32768 * 8 * 128 * 2, 4 * 32768
    assert rows_read == 134217728
    i8 = bytes_model.write_step_bytes("int8", "per_token_head", 32768, 8, 128)
    assert i8 == rows_read + slots + 67108864 + 2097152
    f8 = bytes_model.write_step_bytes("fp8", "per_head", 32768, 8, 128)
    assert f8 == rows_read + slots + 67108864
    # the decode step's append: one row per sequence (24), INT8 per token
    a8 = bytes_model.write_step_bytes("int8", "per_token_head", 24, 8, 128)
    assert a8 == 2 * 24 * 8 * 128 * 2 + 4 * 24 + 2 * 24 * 8 * 128 + 2 * 24 * 8 * 4
    # bf16 caches and rows that go to the INT4 residual ring store the rows as they are
    assert bytes_model.write_step_bytes("bf16", "none", 24, 8, 128) == 2 * (2 * 24 * 8 * 128 * 2) + 4 * 24
    assert bytes_model.write_step_bytes("int4", "kivi", 16, 8, 128, to_ring=True) == \
        2 * (2 * 16 * 8 * 128 * 2) + 4 * 16


def test_bench_write_bytes_equal_the_oracle():
    """The write bytes bench.py adds to every step (and reports for the prefill write) are
    the oracle's count, for every bench workload's append and both prefill-write caches."""
    import bench
    from quantized_paged_kv_02_b200 import inputs, roofline
    for name in sorted(bench.WORKLOADS):
        s = inputs._spec(name, False)
        ring = inputs.low_bit(s.cache_dtype)
        got = roofline.write_bytes(s.cache_dtype, s.scale_mode, s.batch, s.num_kv_heads, s.head_dim,
                                   to_ring=ring)
        want = bytes_model.write_step_bytes(s.cache_dtype, s.scale_mode, s.batch, s.num_kv_heads,
                                            s.head_dim, to_ring=ring)
        assert got == want, name
    for cd, mode in (("int8", "per_token_head"), ("fp8", "per_head")):
        assert roofline.write_bytes(cd, mode, 32768, 8, 128) == \
            bytes_model.write_step_bytes(cd, mode, 32768, 8, 128)


def test_prefill_flops_count_visible_pairs():
    """The prefill roofline's numerator: 4 D flops per (query head, visible position), the
    visible positions those the causal window of each query reaches.  Counted here by
    enumerating the mask (query i of an L-query chunk at the end of n cached tokens sees
    position p iff p <= n - L + i), and the c5 prefill figure (4 x 4096 tokens, 512-query
    chunks, 64 query heads, D 128) written out."""
    import bench
    for batch, n, L, hq, d in ((1, 5, 5, 1, 1), (2, 37, 9, 3, 16), (3, 200, 64, 2, 8)):
        pairs = batch * sum(1 for i in range(L) for p in range(n) if p <= n - L + i)
        assert bench.prefill_flops(batch, n, L, hq, d) == 4 * d * hq * pairs
    per_seq = 512 * (4096 - 512) + 512 * 513 // 2            # sum over the chunk of n - L + i + 1
    assert per_seq == 1966336
    assert bench.prefill_flops(4, 4096, 512, 64, 128) == 4 * 128 * 64 * 4 * per_seq == 257731592192
