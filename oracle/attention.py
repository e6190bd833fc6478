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


def prefill_attention(cache, q, q_start, block_tables, context_lens, softmax_scale=0.0,
                      seq_ids=None):
    """Causal attention of a chunk of new queries over the dequantized cache, float64.

    q [Tq, H_q, D]; the queries of sequence b are rows q_start[b] .. q_start[b+1]-1, the
    newest tokens of that sequence: query i sits at position p = n_b - L_b + i (n_b =
    context_lens[b], L_b its query count) and attends to every cached position <= p:
        z_t = scale * (q . k_t), t <= p;   o = softmax(z) V
    (chunked prefill, one of the techniques [P-prod] "为什么长上下文更需要 KV Cache
    Quantization" lists beside KV cache quantization; the chunk's own K/V rows are in the
    cache before attention runs).  For INT4 / 2-bit caches the newest positions come from
    ring sequence seq_ids[b] (b when seq_ids is None), as in decode.  Returns [Tq, H_q, D];
    one query row at a time.
    """
    q = np.asarray(q, np.float64)
    Tq, Hq, D = q.shape
    g = Hq // cache.H
    scale = softmax_scale if softmax_scale else 1.0 / np.sqrt(D)
    out = np.zeros((Tq, Hq, D), np.float64)
    qs = np.asarray(q_start)
    for b in range(len(context_lens)):
        n = int(context_lens[b])
        L = int(qs[b + 1] - qs[b])
        if L == 0:
            continue
        K, V = cache.gather(block_tables[b], n, b if seq_ids is None else int(seq_ids[b]))
        for i in range(L):
            p = n - L + i
            for hq in range(Hq):
                kvh = hq // g
                out[qs[b] + i, hq] = softmax_attention(q[qs[b] + i, hq], K[kvh][:p + 1],
                                                       V[kvh][:p + 1], scale)
    return out
