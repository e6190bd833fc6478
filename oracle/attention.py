"""Single-token decode attention over the dequantized cache, in float64.

TEST INFRASTRUCTURE (oracle): see the package docstring.

For every sequence b and query head hq (kv head kvh = hq // g, g = H_q / H_kv):
    z_p = scale * (q . k_p)         p < context_lens[b], k_p the dequantized key
    w   = exp(z - max z) / sum exp(z - max z)
    o   = sum_p w_p v_p
Decode reads every cached position at each step ([P-prod] "为什么长上下文更需要 KV Cache
Quantization"); the dequantized rows come from the cache model ([P-vLLM]
"PagedAttention与KV Cache量化协同工作原理").  The default scale is 1/sqrt(D) as in
[P-mem] §6 Q1 (its "+0.01" inside the softmax is a constant shift and is not used).
No split, no rescaling trick: one (b, hq) at a time, all in float64.
"""

import numpy as np


def softmax_attention(q, K, V, scale):
    """o = softmax(scale * K q) V for one query vector q [D], K, V [n, D] (float64)."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], np.float64)
    z = (K @ np.asarray(q, np.float64)) * scale
    w = np.exp(z - z.max())
    w /= w.sum()
    return w @ V


def decode_attention(cache, q, block_tables, context_lens, seq_ids=None,
                     softmax_scale=0.0, units=None):
    """Reference output [B, H_q, D] (float64) for the whole batch, or for `units`.

    q: float64 [B, H_q, D].  units: optional iterable of (b, kvh) pairs to compute; the
    other rows are left as NaN (used to sample large workloads).
    """
    q = np.asarray(q, np.float64)
    B, Hq, D = q.shape
    g = Hq // cache.H
    scale = softmax_scale if softmax_scale else 1.0 / np.sqrt(D)
    out = np.full((B, Hq, D), np.nan, np.float64)
    want = None if units is None else set((int(b), int(h)) for b, h in units)
    for b in range(B):
        if want is not None and not any(bb == b for bb, _ in want):
            continue
        n = int(context_lens[b])
        sid = b if seq_ids is None else int(seq_ids[b])
        K, V = cache.gather(block_tables[b], n, sid)
        for kvh in range(cache.H):
            if want is not None and (b, kvh) not in want:
                continue
            for j in range(g):
                hq = kvh * g + j
                out[b, hq] = softmax_attention(q[b, hq], K[kvh], V[kvh], scale)
    return out
