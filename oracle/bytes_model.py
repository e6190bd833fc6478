"""KV-cache size formula and the bytes one decode step must read.

TEST INFRASTRUCTURE (oracle): see the package docstring.

The size formula is the one all three pages print:
  bytes = 2 x layers x kv_heads x head_dim x seq_len x bytes_per_value (x batch)
([P-vLLM] "KV Cache显存瓶颈分析与大模型推理优化"; [P-prod] "KV Cache 的基本内存模型";
[P-mem] §2.1 基础计算公式), with the bytes-per-value table of [P-prod]
(FP16/BF16 2, FP8 1, INT8 1, INT4 0.5, 2-bit 0.25).  The real size adds scales, zero
points and residual rows ([P-prod], the sentence after the table).
"""

from fractions import Fraction

BYTES_PER_VALUE = {
    "fp16": Fraction(2), "bf16": Fraction(2), "fp8": Fraction(1), "int8": Fraction(1),
    "int4": Fraction(1, 2), "int2": Fraction(1, 4),
}


def kv_cache_bytes(layers, kv_heads, head_dim, seq_len, dtype, batch=1):
    """2 x L x H_kv x d x S x bytes_per_value x batch, as an exact Fraction."""
    return 2 * layers * kv_heads * head_dim * seq_len * batch * BYTES_PER_VALUE[dtype]


def decode_step_bytes(cache_dtype, scale_mode, batch, num_q_heads, num_kv_heads, head_dim,
                      context_lens, block_size, act_bytes=2, out_bytes=2, group_size=64,
                      residual_len=128):
    """Bytes one decode step must move: cache rows read, metadata read, q read, out written.

    Per token and kv head: K and V codes (head_dim x bytes per value) plus their
    per-token scale bytes; per block and kv head: the KIVI key scales/zeros (per token
    and channel group when keys are grouped per token); per sequence: block-table entries
    and its context length; q and out once.  INT4 and 2-bit caches read the newest tokens
    from the residual ring at act_bytes per value.
    """
    D, H = head_dim, num_kv_heads
    total = Fraction(0)
    for n in context_lens:
        n = int(n)
        if cache_dtype in ("int4", "int2"):
            # 4-bit or 2-bit codes ([P-prod] "KV Cache 的基本内存模型": 0.5 / 0.25 byte per
            # value) in whole groups; the newest tokens stay in the residual ring
            qb = group_size * (max(n - residual_len, 0) // group_size)
            nblk = qb // block_size
            total += 2 * H * qb * D * BYTES_PER_VALUE[cache_dtype]     # K and V codes
            if scale_mode == "int4_per_token":
                # keys grouped like values: (scale, zero) fp16 per token and channel group
                total += H * qb * (D // group_size) * 2 * 2
            else:
                # KIVI keys: (scale, zero or minimum) fp16 per channel and block
                total += H * nblk * 2 * D * 2
            total += H * qb * (D // group_size) * 2 * 2                 # V scale+zero fp16
            total += 2 * H * (n - qb) * D * act_bytes                   # residual rows
            total += 4 * nblk
        else:
            nblk = -(-n // block_size)
            total += 2 * H * n * D * BYTES_PER_VALUE[cache_dtype]
            if scale_mode == "per_token_head":
                total += 2 * H * n * 4
            total += 4 * nblk
        total += 4                                                      # context length
    if scale_mode == "per_head":
        total += 2 * H * 4
    elif scale_mode == "per_tensor":
        total += 2 * 4
    total += batch * num_q_heads * D * act_bytes                        # q
    total += batch * num_q_heads * D * out_bytes                        # out
    return total


def write_step_bytes(cache_dtype, scale_mode, rows, num_kv_heads, head_dim, act_bytes=2,
                     to_ring=False):
    """Bytes one write of `rows` new tokens must move: the K and V rows read (activation
    values) and one int32 slot id per token, then what the cache stores for them -- codes at
    the bytes per value of the size formula, plus one float32 scale per (token, kv head) for
    K and V when scales are per token ([P-mem] §3.2 动态量化策略: a scale per token).  A
    16-bit cache, and a low-bit cache whose new rows go to the residual ring, store the rows
    as they are (act_bytes per value).  Static scales are read from the call's arguments,
    not from the pool, and are not counted.
    """
    H, D = num_kv_heads, head_dim
    total = Fraction(2 * rows * H * D * act_bytes)                      # K and V rows read
    total += 4 * rows                                                   # slot ids
    if to_ring or cache_dtype in ("bf16", "fp16"):
        total += 2 * rows * H * D * act_bytes
        return total
    total += 2 * rows * H * D * BYTES_PER_VALUE[cache_dtype]            # K and V codes
    if scale_mode == "per_token_head":
        total += 2 * rows * H * 4                                       # K and V scales
    return total
