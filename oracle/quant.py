"""Quantizers and dequantizers, one group at a time, in the pages' steps.

TEST INFRASTRUCTURE (oracle): see the package docstring.

Inputs are activation values (bfloat16 or float16 values, exactly representable in
binary32) given as NumPy arrays; outputs are codes and scales with the bit patterns the
cache stores.

Readings of the pages taken here:
  * "round" is round-half-to-even: the INT8 snippet of [P-mem] §3.1 对称量化算法 uses
    torch.round, which rounds half to even.
  * x / scale and the scale itself are IEEE binary32: the snippet returns the scale as
    ``.float()``; a fp32 scale per token per head is the dynamic variant of [P-mem]
    §3.2 动态量化策略.
  * An all-zero group (max |x| = 0) has scale 0 and codes 0, with no division.
  * INT4 uses the affine form of [P-prod] "量化不是简单截断精度"
    (X_q = round(X/scale) + zero_point; X_deq = (X_q - zero_point) * scale) with the
    range widened to include 0, so the zero point is an integer in [0, 15].
  * 2-bit caches use the same quantizers with 3 as the largest code ([P-prod] "KV Cache 的基本
    内存模型" lists 2-bit at 0.25 byte per value; "误区二：INT4 或 2-bit 一定比 FP8 更划算").
  * The float-zero-point INT4 variant takes the group minimum itself as the offset
    (X_deq = X_q * scale + min, the range not widened); the pages name only the integer
    form, so this variant is a reading of "zero point" as a real offset.
"""

import numpy as np

from . import fp

INT8_QMAX = 127.0
FP8_QMAX = fp.E4M3_MAX
INT4_LEVELS = 15.0


def levels(bits):
    """Largest code of a `bits`-bit unsigned code: 15 for INT4, 3 for 2-bit."""
    return float((1 << bits) - 1)


# ----------------------------------------------------------------------------- INT8
def int8_scale_dynamic(rows):
    """Per-row symmetric MinMax scale s = max|x| / 127 (binary32), rows [..., D].

    [P-mem] §3.1 对称量化算法 (scale = max(abs(x)) / 127) applied per token per kv head
    ([P-mem] §3.2 动态量化策略: a scale for each token's K/V vector).
    """
    rows = np.asarray(rows, dtype=np.float32)
    m = np.max(np.abs(rows), axis=-1)
    return fp.div32(m, np.float32(INT8_QMAX))


def int8_quantize(rows, scale):
    """q = clamp(round_half_even(x / s), -128, 127) with x / s in binary32.

    [P-mem] §3.1 对称量化算法 (torch.clamp(torch.round(x / scale), -128, 127));
    [P-vLLM] "KV Cache量化策略" gives the same q = round(x / scale).  ``scale`` broadcasts
    against rows[..., D] over the last axis; a zero scale gives code 0.
    """
    rows = np.asarray(rows, dtype=np.float32)
    s = np.asarray(scale, dtype=np.float32)[..., None] if np.ndim(scale) == rows.ndim - 1 \
        else np.asarray(scale, dtype=np.float32)
    r = fp.div32(rows, s)
    q = np.clip(fp.round_half_even(r), -128, 127)
    q = np.where(s == 0, 0, q)
    return q.astype(np.int8)


def int8_dequantize(codes, scale):
    """x_hat = q * s ([P-mem] §3.1: q_x.float() * scale), evaluated in float64."""
    s = np.asarray(scale, dtype=np.float64)
    codes = np.asarray(codes)
    if s.ndim == codes.ndim - 1:
        s = s[..., None]
    return codes.astype(np.float64) * s


# ----------------------------------------------------------------------------- FP8
def fp8_scale_dynamic(rows):
    """Per-row scale s = max|x| / 448 (binary32)."""
    rows = np.asarray(rows, dtype=np.float32)
    return fp.div32(np.max(np.abs(rows), axis=-1), np.float32(FP8_QMAX))


def fp8_calibrate(warmup):
    """Per-kv-head scale from warm-up rows [T, H, D]: max over tokens and channels / 448.

    [P-prod] "vLLM：从 FP8 KV Cache 开始试点": per-attention-head FP8 scales may come from a
    random-token warm-up.  448 is the largest finite E4M3 magnitude.
    """
    w = np.asarray(warmup, dtype=np.float32)
    m = np.max(np.abs(w), axis=(0, 2))
    return fp.div32(m, np.float32(FP8_QMAX))


def head_calibrate(warmup, qmax):
    """Per-kv-head static scale from warm-up rows [T, H, D]: max over tokens and channels of
    |x|, divided by qmax in binary32, [H].  qmax is 127 for INT8, 448 for FP8
    (fp8_calibrate is this with 448).

    [P-mem] §3.2 动态量化策略: static quantization keeps one fixed scale; [P-vLLM]
    "KV Cache量化策略：INT8与FP8精度对比与选择": INT8 per tensor; [P-prod] "量化不是简单截断精度":
    scales per tensor or per head.
    """
    w = np.asarray(warmup, dtype=np.float32)
    return fp.div32(np.max(np.abs(w), axis=(0, 2)), np.float32(qmax))


def channel_calibrate(warmup, qmax):
    """Per-(kv head, channel) static scale from warm-up rows [T, H, D]: max over the tokens
    of |x| / qmax (binary32), [H, D].  qmax is 127 for INT8, 448 for FP8.

    [P-vLLM] "KV Cache量化策略：INT8与FP8精度对比与选择" (INT8 with per-tensor or per-channel
    granularity) and "vLLM引擎KV Cache量化配置与启动参数详解" (INT8 scales generated offline from
    calibration data); [P-prod] "量化不是简单截断精度" (scale per tensor, head, channel, token or
    group); [P-mem] §3.2 动态量化策略 (static quantization: fixed scales).
    """
    w = np.asarray(warmup, dtype=np.float32)
    return fp.div32(np.max(np.abs(w), axis=0), np.float32(qmax))


def fp8_quantize(rows, scale):
    """code = E4M3(x / s): binary32 quotient, nearest E4M3 (ties even), saturate at 448.

    [P-vLLM] "KV Cache量化策略" (FP8 E4M3 storage with a scale); a zero scale gives 0x00.
    """
    rows = np.asarray(rows, dtype=np.float32)
    s = np.asarray(scale, dtype=np.float32)
    if s.ndim == rows.ndim - 1:
        s = s[..., None]
    r = fp.div32(rows, s)
    r = np.where(s == 0, np.float32(0.0), r)
    codes = fp.e4m3_encode(r)
    return np.where(np.broadcast_to(s == 0, codes.shape), np.uint8(0), codes).astype(np.uint8)


def fp8_dequantize(codes, scale):
    s = np.asarray(scale, dtype=np.float64)
    codes = np.asarray(codes)
    if s.ndim == codes.ndim - 1:
        s = s[..., None]
    return fp.e4m3_decode(codes) * s


# ----------------------------------------------------------------------------- INT4
def int4_quantize_groups(values, bits=4):
    """Asymmetric 4-bit (or 2-bit) quantization of groups along the last axis (binary32
    values), with Q = 2^bits - 1 the largest code (15, or 3).

    Every group (1-D slice values[..., :]) is quantized on its own.  Returns (codes
    uint8 in 0..Q with the shape of values, scale float16 and zero point float16 with
    the leading shape).
      lo = min(min x, 0); hi = max(max x, 0)
      s  = float16(binary32((hi - lo) / Q))        -- stored, and used from here on
      z  = clamp(round_half_even(-lo / s), 0, Q)
      q  = clamp(round_half_even(x / s) + z, 0, Q)
    A group whose s is 0 (all values 0) gets codes 0, scale 0, zero point 0.
    [P-prod] "量化不是简单截断精度": X_q = round(X/scale) + zero_point.
    """
    Q = levels(bits)
    x = np.asarray(values, dtype=np.float32)
    lo = np.minimum(x.min(axis=-1), np.float32(0.0))
    hi = np.maximum(x.max(axis=-1), np.float32(0.0))
    s32 = fp.div32(fp.sub32(hi, lo), np.float32(Q))
    s16 = fp.f16(s32)
    zero_group = s16 == 0
    sw = np.where(zero_group, np.float32(1.0), np.asarray(s16, np.float32))
    z = np.clip(fp.round_half_even(fp.div32(-lo, sw)), 0, Q)
    q = np.clip(fp.round_half_even(fp.div32(x, sw[..., None])) + z[..., None], 0, Q)
    q = np.where(zero_group[..., None], 0, q)
    z = np.where(zero_group, 0, z)
    return q.astype(np.uint8), np.asarray(s16, np.float16), np.asarray(z, np.float16)


def int4_quantize_groups_float_zero(values, bits=4):
    """Asymmetric 4-bit (or 2-bit) quantization with a float zero point (the group
    minimum), Q = 2^bits - 1 the largest code.

    Every group (1-D slice values[..., :]) on its own.  Returns (codes uint8 in 0..Q,
    scale float16, minimum float16), the last two with the leading shape.
      lo = min x; hi = max x
      s  = float16(binary32((hi - lo) / Q));  m = float16(lo)    -- stored, used from here on
      q  = clamp(round_half_even(binary32(binary32(x - m) / s)), 0, Q)
    A group whose s is 0 (constant, or a range below float16's reach) gets codes 0.
    Dequantized value: q * s + m.
    """
    Q = levels(bits)
    x = np.asarray(values, dtype=np.float32)
    lo = x.min(axis=-1)
    hi = x.max(axis=-1)
    s16 = fp.f16(fp.div32(fp.sub32(hi, lo), np.float32(Q)))
    m16 = fp.f16(lo)
    zero_group = s16 == 0
    sw = np.where(zero_group, np.float32(1.0), np.asarray(s16, np.float32))
    mw = np.asarray(m16, np.float32)
    q = np.clip(fp.round_half_even(fp.div32(fp.sub32(x, mw[..., None]), sw[..., None])), 0, Q)
    q = np.where(zero_group[..., None], 0, q)
    return q.astype(np.uint8), np.asarray(s16, np.float16), np.asarray(m16, np.float16)


def int4_dequantize_float_zero(codes, scale, minimum):
    """X_deq = X_q * scale + min, float64."""
    return np.asarray(codes, np.float64) * np.float64(scale) + np.float64(minimum)


def _groups(float_zero, bits):
    f = int4_quantize_groups_float_zero if float_zero else int4_quantize_groups
    return lambda v: f(v, bits)


def int4_quantize_group(values):
    """int4_quantize_groups for one group (1-D array): (codes, scale, zero point)."""
    q, s, z = int4_quantize_groups(np.asarray(values, dtype=np.float32).reshape(1, -1))
    return q[0], s[0], z[0]


def int4_dequantize(codes, scale, zero):
    """X_deq = (X_q - zero_point) * scale ([P-prod] "量化不是简单截断精度"), float64."""
    return (np.asarray(codes, np.float64) - np.float64(zero)) * np.float64(scale)


def int4_keys_block(k_rows, float_zero=False, bits=4):
    """KIVI keys: one group per channel over the block's tokens.

    k_rows [64, D] (one kv head), or [..., 64, D] for several heads at once.  Returns
    codes [..., 64, D], scale [..., D], zero point (or minimum, float_zero) [..., D].
    [P-prod] "Key 和 Value 的分布不一定相同": key cache per channel (KIVI).
    """
    k_rows = np.asarray(k_rows, dtype=np.float32)
    q, s, z = _groups(float_zero, bits)(np.swapaxes(k_rows, -1, -2))     # groups = channels
    return np.swapaxes(q, -1, -2), s, z


def int4_values_row(v_row, group=64, float_zero=False, bits=4):
    """One group per token over each run of `group` channels: KIVI values, and keys as well
    as values in the per-token variant.

    v_row [D] (one token, one kv head), or [..., D] for several at once.  Returns codes
    [..., D], scale [..., D/group], zero point (or minimum, float_zero) [..., D/group].
    [P-prod] "Key 和 Value 的分布不一定相同": value cache per token (KIVI); the Transformers
    integration quantizes keys and values per token.
    """
    v_row = np.asarray(v_row, dtype=np.float32)
    D = v_row.shape[-1]
    q, s, z = _groups(float_zero, bits)(v_row.reshape(v_row.shape[:-1] + (D // group, group)))
    return q.reshape(v_row.shape), s, z


def pack_codes(codes, bits):
    """Pack `bits`-bit codes (4 or 2) along the last axis, 8 / bits per byte: element
    k*i + e of a run of k = 8 / bits goes to bits [bits*e, bits*e + bits) of byte i."""
    if bits == 4:
        return pack_nibbles(codes)
    c = np.asarray(codes, dtype=np.uint8) & 3
    return c[..., 0::4] | (c[..., 1::4] << 2) | (c[..., 2::4] << 4) | (c[..., 3::4] << 6)


def unpack_codes(packed, bits):
    if bits == 4:
        return unpack_nibbles(packed)
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 4,), np.uint8)
    for e in range(4):
        out[..., e::4] = (p >> (2 * e)) & 3
    return out


def pack_nibbles(codes):
    """Two 4-bit codes per byte along the last axis: element 2i low, 2i+1 high."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_nibbles(packed):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out
