"""Algorithmic byte counts of one decode step, used for KV-GB/s and the HBM roofline.

Per (sequence, kv head) and cached position, decode must read the K and V codes
(head_dim x bytes per value each) and their per-token scales; per block it reads one
block-table entry (and, for INT4, the block's per-channel key scale/zero pairs); INT4
reads the newest positions from the residual ring at the activation width.  q is read
and out written once.  The size model is the one of [P-prod] "KV Cache 的基本内存模型"
(2 x layers x kv_heads x head_dim x tokens x bytes per value) for one layer, plus the
metadata bytes the same section says make the real gain smaller.  Split partials and
the reduce's round trip are not algorithmic and are not counted.
"""

CODE_BYTES = {"bf16": 2.0, "fp16": 2.0, "int8": 1.0, "fp8": 1.0, "int4": 0.5, "int2": 0.25}


def decode_bytes(cache_dtype, scale_mode, num_q_heads, num_kv_heads, head_dim, block_size,
                 context_lens, act_bytes=2, out_bytes=2, residual_len=128, group=64):
    H, D = num_kv_heads, head_dim
    total = 0
    for n in context_lens:
        n = int(n)
        if cache_dtype in ("int4", "int2"):
            qb = group * (max(n - residual_len, 0) // group)
            nblk = qb // block_size
            total += int(2 * H * qb * D * CODE_BYTES[cache_dtype])
            if scale_mode == "int4_per_token":             # key scale + zero, fp16
                total += H * qb * (D // group) * 2 * 2     # per token and channel group
            else:
                total += H * nblk * 2 * D * 2              # per channel and block
            total += H * qb * (D // group) * 2 * 2         # value scale + zero, fp16
            total += 2 * H * (n - qb) * D * act_bytes      # ring rows
            total += 4 * nblk
        else:
            nblk = -(-n // block_size)
            total += int(2 * H * n * D * CODE_BYTES[cache_dtype])
            if scale_mode == "per_token_head":
                total += 2 * H * n * 4
            total += 4 * nblk
        total += 4
    if scale_mode == "per_head":
        total += 2 * H * 4
    elif scale_mode == "per_tensor":
        total += 8
    B = len(context_lens)
    total += B * num_q_heads * D * (act_bytes + out_bytes)
    return total


def write_bytes(cache_dtype, scale_mode, num_rows, num_kv_heads, head_dim, act_bytes=2,
                to_ring=False):
    """Bytes kvq_write moves for `num_rows` new tokens (K and V)."""
    H, D = num_kv_heads, head_dim
    read = 2 * num_rows * H * D * act_bytes + 4 * num_rows
    if to_ring or cache_dtype in ("bf16", "fp16"):
        return read + 2 * num_rows * H * D * act_bytes
    wrote = int(2 * num_rows * H * D * CODE_BYTES[cache_dtype])
    if scale_mode == "per_token_head":
        wrote += 2 * num_rows * H * 4
    return read + wrote
