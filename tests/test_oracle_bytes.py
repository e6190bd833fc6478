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
