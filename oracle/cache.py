"""Byte-exact model of the paged, quantized KV cache: scatter on write, gather on read.

TEST INFRASTRUCTURE (oracle): see the package docstring.

The pools are NumPy arrays with exactly the layout written in include/kvq.h, filled
with a sentinel byte (0x5A) so that a test can check that a write touched only its own
slots.  A slot is block_id * block_size + offset; each block is managed on its own
([P-vLLM] "PagedAttention与KV Cache量化协同工作原理": fixed-size blocks, usually of 16
tokens, stored as INT8/FP8 and dequantized when attention reads them).
"""

import numpy as np

from . import fp, quant

SENTINEL = 0x5A

DENSE_DTYPES = ("bf16", "fp16", "int8", "fp8")
INT4_MODES = ("kivi", "kivi_float_zero", "int4_per_token")
LOW_BIT = {"int4": 4, "int2": 2}              # group-quantized caches: bits per code


def _bits_of_act(x, act):
    """Bit patterns (uint16) of activation values given as float64 (exact)."""
    if act == "bf16":
        return fp.bf16_bits(np.asarray(x, np.float64).astype(np.float32))
    if act == "fp16":
        v = np.asarray(x, np.float64)
        h = v.astype(np.float16)
        if not np.array_equal(h.astype(np.float64), v):
            raise ValueError("value not representable in float16")
        return h.view(np.uint16)
    raise ValueError(act)


def _value_of_act_bits(bits, act):
    if act == "bf16":
        return fp.bf16_value(bits)
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


class PagedCache:
    """One layer's paged cache.

    cache_dtype: "bf16" | "fp16" | "int8" | "fp8" | "int4" | "int2"
    act_dtype:   "bf16" | "fp16"
    scale_mode:  "none" | "per_token_head" | "per_head" | "per_tensor" | "per_channel" for
                 dense caches; "kivi" | "kivi_float_zero" | "int4_per_token" for INT4 and
                 2-bit caches (the same groups and records, codes of 4 or 2 bits)
    static_scales: (k_scale, v_scale) float32 arrays for static modes: [H] per head, [1]
                   per tensor, [H, D] per (kv head, channel).

    ``pages`` is the byte pool [NB][H][record] of include/kvq.h: per (block, kv head),
    K codes [bs][row_bytes], V codes [bs][row_bytes], then the per-token scales (float32
    K [bs], V [bs]) or the INT4 parameters, padded to a multiple of 128 bytes.  INT4:
    "kivi" float16 K scale [D], K zero point [D], V (scale, zero point) [bs][D/64][2];
    "kivi_float_zero" the same with each zero point field holding the group minimum;
    "int4_per_token" K (scale, zero point) [bs][D/64][2] then V the same.  The attributes k_codes,
    v_codes, k_scales, v_scales are typed views into it (static scales are arrays of
    their own).
    """

    def __init__(self, cache_dtype, act_dtype, scale_mode, num_blocks, block_size,
                 num_kv_heads, head_dim, group_size=64, residual_len=128,
                 residual_cap=192, max_seqs=0, static_scales=None):
        self.cd, self.act, self.mode = cache_dtype, act_dtype, scale_mode
        self.NB, self.bs, self.H, self.D = num_blocks, block_size, num_kv_heads, head_dim
        self.G, self.R, self.cap, self.max_seqs = group_size, residual_len, residual_cap, max_seqs
        NB, bs, H, D = self.NB, self.bs, self.H, self.D
        if cache_dtype in ("bf16", "fp16"):
            assert scale_mode == "none" and cache_dtype == act_dtype
            code_dt, row_bytes = np.uint16, 2 * D
        elif cache_dtype == "int8":
            code_dt, row_bytes = np.int8, D
        elif cache_dtype == "fp8":
            code_dt, row_bytes = np.uint8, D
        elif cache_dtype in LOW_BIT:
            assert scale_mode in INT4_MODES and block_size == group_size == 64
            code_dt, row_bytes = np.uint8, D * LOW_BIT[cache_dtype] // 8
        else:
            raise ValueError(cache_dtype)
        off_s = 2 * bs * row_bytes
        if scale_mode == "per_token_head":
            scale_bytes = 8 * bs
        elif scale_mode in ("kivi", "kivi_float_zero"):
            scale_bytes = 2 * D * 2 + bs * (D // group_size) * 2 * 2
        elif scale_mode == "int4_per_token":
            scale_bytes = 2 * bs * (D // group_size) * 2 * 2
        else:
            scale_bytes = 0
        self.row_bytes = row_bytes
        self.record = -(-(off_s + scale_bytes) // 128) * 128
        self.pages = np.full((NB, H, self.record), SENTINEL, np.uint8)
        pg = self.pages
        n_el = row_bytes // np.dtype(code_dt).itemsize
        self.k_codes = pg[:, :, 0:bs * row_bytes].view(code_dt).reshape(NB, H, bs, n_el)
        self.v_codes = pg[:, :, bs * row_bytes:off_s].view(code_dt).reshape(NB, H, bs, n_el)
        self.k_scales = self.v_scales = None
        self.residual = None
        if scale_mode == "per_token_head":
            self.k_scales = pg[:, :, off_s:off_s + 4 * bs].view(np.float32).reshape(NB, H, bs)
            self.v_scales = pg[:, :, off_s + 4 * bs:off_s + 8 * bs].view(np.float32).reshape(NB, H, bs)
        elif scale_mode in ("per_head", "per_tensor", "per_channel"):
            shape = {"per_head": (H,), "per_tensor": (1,), "per_channel": (H, D)}[scale_mode]
            ks, vs = static_scales
            self.k_scales = np.asarray(ks, np.float32).reshape(shape).copy()
            self.v_scales = np.asarray(vs, np.float32).reshape(shape).copy()
        elif cache_dtype in LOW_BIT:
            if scale_mode == "int4_per_token":
                # K (scale, zero) [bs][D/G][2], then V the same
                half = scale_bytes // 2
                self.k_scales = pg[:, :, off_s:off_s + half].view(np.float16).reshape(
                    NB, H, bs, D // group_size, 2)
            else:
                # K scale [D] then K zero (or minimum) [D] as [NB][H][2][D]
                half = 4 * D
                self.k_scales = pg[:, :, off_s:off_s + half].view(np.float16).reshape(NB, H, 2, D)
            # V (scale, zero or minimum) [bs][D/G][2]
            self.v_scales = pg[:, :, off_s + half:off_s + scale_bytes].view(np.float16).reshape(
                NB, H, bs, D // group_size, 2)
            self.residual = np.full(max_seqs * 2 * H * residual_cap * D * 2, SENTINEL,
                                    np.uint8).view(np.uint16).reshape(max_seqs, 2, H, residual_cap, D)
        # the views must alias the pool
        assert np.shares_memory(self.k_codes, self.pages)

    # ------------------------------------------------------------------ scales
    def _static_scale(self, which):
        """[H] per head or per tensor, [H, D] per channel."""
        s = self.k_scales if which == 0 else self.v_scales
        if self.mode in ("per_head", "per_channel"):
            return s
        return np.broadcast_to(s, (self.H,))          # per tensor

    # ------------------------------------------------------------------ write
    def write(self, k_new, v_new, slot_mapping, seq_ids=None, positions=None):
        """Quantize rows k_new/v_new [T, H, D] (float64 values of act_dtype) into slots.

        Same contract as kvq_write in include/kvq.h.  Out-of-range slots are skipped.
        """
        k_new = np.asarray(k_new, np.float64)
        v_new = np.asarray(v_new, np.float64)
        slots = np.asarray(slot_mapping, np.int64)
        if self.cd in LOW_BIT:
            return self._write_int4(k_new, v_new, slots, seq_ids, positions)
        NB, bs = self.NB, self.bs
        keep = (slots >= 0) & (slots < NB * bs)
        t_idx = np.nonzero(keep)[0]
        if np.unique(slots[t_idx]).size != t_idx.size:
            # a slot named twice: rows are applied in order, so the later one stays
            for t in t_idx:
                self._write_rows(k_new[t:t + 1], v_new[t:t + 1], slots[t:t + 1])
            return
        self._write_rows(k_new[t_idx], v_new[t_idx], slots[t_idx])

    def _write_rows(self, k_rows, v_rows, slots):
        """Quantize rows [n, H, D] into distinct, in-range slots [n].  Every (token, kv
        head) row is quantized on its own, so the rows are processed together."""
        blk, off = np.divmod(slots, self.bs)
        for which, rows in ((0, k_rows), (1, v_rows)):
            codes = self.k_codes if which == 0 else self.v_codes
            x = rows.astype(np.float32)                # [n, H, D], exact
            if self.cd in ("bf16", "fp16"):
                codes[blk, :, off, :] = _bits_of_act(rows, self.act)
                continue
            if self.mode == "per_token_head":
                s = (quant.int8_scale_dynamic(x) if self.cd == "int8"
                     else quant.fp8_scale_dynamic(x))              # [n, H]
                sc = self.k_scales if which == 0 else self.v_scales
                sc[blk, :, off] = s
            elif self.mode == "per_channel":
                s = np.broadcast_to(self._static_scale(which), x.shape)       # [n, H, D]
            else:
                s = np.broadcast_to(self._static_scale(which), x.shape[:2])
            s2 = np.asarray(s, np.float32)
            if self.mode != "per_channel":
                s2 = s2[..., None]
            if self.cd == "int8":
                codes[blk, :, off, :] = quant.int8_quantize(x, s2)
            else:
                codes[blk, :, off, :] = quant.fp8_quantize(x, s2)

    def _write_int4(self, k_new, v_new, slots, seq_ids, positions):
        T = slots.shape[0]
        G, bs = self.G, self.bs
        for u in range(0, T, G):
            rows = range(u, min(u + G, T))
            first = int(slots[u])
            if first >= 0:
                # one whole block, in order
                if len(rows) != G or first % bs != 0 or first >= self.NB * bs:
                    continue
                if not all(int(slots[u + i]) == first + i for i in range(G)):
                    continue
                blk = first // bs
                # keys per (head, channel) over the block's rows; values per (row, head,
                # channel group); every group on its own, all heads at once
                fz = self.mode == "kivi_float_zero"
                bits = LOW_BIT[self.cd]
                kb = np.swapaxes(k_new[u:u + G].astype(np.float32), 0, 1)     # [H, G, D]
                if self.mode == "int4_per_token":
                    kc, ks, kz = quant.int4_values_row(kb, self.G, bits=bits)  # like values
                    self.k_scales[blk, :, :, :, 0] = ks
                    self.k_scales[blk, :, :, :, 1] = kz
                else:
                    kc, ks, kz = quant.int4_keys_block(kb, float_zero=fz, bits=bits)
                    self.k_scales[blk, :, 0, :] = ks
                    self.k_scales[blk, :, 1, :] = kz
                self.k_codes[blk] = quant.pack_codes(kc, bits)
                vb = np.swapaxes(v_new[u:u + G].astype(np.float32), 0, 1)     # [H, G, D]
                vc, vs, vz = quant.int4_values_row(vb, self.G, float_zero=fz, bits=bits)
                self.v_codes[blk] = quant.pack_codes(vc, bits)
                self.v_scales[blk, :, :, :, 0] = vs
                self.v_scales[blk, :, :, :, 1] = vz
            else:
                for t in rows:
                    if int(slots[t]) != -1 or positions is None or int(positions[t]) < 0:
                        continue
                    sid = int(seq_ids[t])
                    if sid < 0 or sid >= self.max_seqs:
                        continue
                    row = int(positions[t]) % self.cap
                    self.residual[sid, 0, :, row, :] = _bits_of_act(k_new[t], self.act)
                    self.residual[sid, 1, :, row, :] = _bits_of_act(v_new[t], self.act)

    def flush_ring(self, seq_ids, positions, block_ids):
        """INT4: quantize ring rows [p0, p0 + 64) of sequence sid into block blk, every kv
        head, exactly as writing those rows to slots blk*64 .. blk*64+63 would (the contract
        of kvq_flush_ring in include/kvq.h).  Entries out of range are skipped."""
        G = self.G
        for sid, p0, blk in zip(np.asarray(seq_ids).tolist(), np.asarray(positions).tolist(),
                                np.asarray(block_ids).tolist()):
            if not (0 <= sid < self.max_seqs) or not (0 <= blk < self.NB) or p0 < 0 or p0 % G:
                continue
            rows = [(p0 + t) % self.cap for t in range(G)]
            k = _value_of_act_bits(self.residual[sid, 0][:, rows, :], self.act)   # [H, G, D]
            v = _value_of_act_bits(self.residual[sid, 1][:, rows, :], self.act)
            slots = blk * G + np.arange(G)
            self._write_int4(np.swapaxes(k, 0, 1), np.swapaxes(v, 0, 1), slots, None, None)

    # ------------------------------------------------------------------ read
    def dequant_block(self, blk):
        """float64 [2, H, bs, D] of one block (index 0 = K, 1 = V)."""
        out = np.empty((2, self.H, self.bs, self.D), np.float64)
        for which in (0, 1):
            codes = self.k_codes if which == 0 else self.v_codes
            c = codes[blk]
            if self.cd in ("bf16", "fp16"):
                out[which] = _value_of_act_bits(c, self.act)
            elif self.cd in ("int8", "fp8"):
                if self.mode == "per_token_head":
                    s = (self.k_scales if which == 0 else self.v_scales)[blk]          # [H, bs]
                elif self.mode == "per_channel":
                    s = np.broadcast_to(self._static_scale(which)[:, None, :],
                                        (self.H, self.bs, self.D))                   # [H, bs, D]
                else:
                    s = np.broadcast_to(self._static_scale(which)[:, None], (self.H, self.bs))
                deq = quant.int8_dequantize if self.cd == "int8" else quant.fp8_dequantize
                out[which] = deq(c, s)
            else:
                q = quant.unpack_codes(c, LOW_BIT[self.cd]).astype(np.float64)  # [H, bs, D]
                if which == 0 and self.mode != "int4_per_token":
                    s = self.k_scales[blk, :, 0, :].astype(np.float64)[:, None, :]   # [H, 1, D]
                    z = self.k_scales[blk, :, 1, :].astype(np.float64)[:, None, :]
                else:
                    sz = (self.k_scales if which == 0 else self.v_scales)[blk].astype(np.float64)
                    s = np.repeat(sz[..., 0], self.G, axis=-1)   # [H, bs, D]
                    z = np.repeat(sz[..., 1], self.G, axis=-1)
                if self.mode == "kivi_float_zero":
                    out[which] = quant.int4_dequantize_float_zero(q, s, z)
                else:
                    out[which] = quant.int4_dequantize(q, s, z)
        return out

    def quantized_prefix(self, n):
        """INT4: number of leading positions read from blocks; the rest is in the ring."""
        if self.cd not in LOW_BIT:
            return n
        return self.G * (max(n - self.R, 0) // self.G)

    def gather(self, block_table_row, n, seq_id=None):
        """Dequantized K and V of one sequence: two float64 arrays [H, n, D]."""
        K = np.empty((self.H, n, self.D), np.float64)
        V = np.empty((self.H, n, self.D), np.float64)
        qb = self.quantized_prefix(n)
        nblk = (qb + self.bs - 1) // self.bs
        for i in range(nblk):
            blk = int(block_table_row[i])
            d = self.dequant_block(blk)
            lo, hi = i * self.bs, min((i + 1) * self.bs, qb)
            K[:, lo:hi] = d[0, :, :hi - lo]
            V[:, lo:hi] = d[1, :, :hi - lo]
        for p in range(qb, n):
            row = p % self.cap
            K[:, p] = _value_of_act_bits(self.residual[seq_id, 0, :, row, :], self.act)
            V[:, p] = _value_of_act_bits(self.residual[seq_id, 1, :, row, :], self.act)
        return K, V
