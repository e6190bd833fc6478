"""Shared test helpers: build the CUDA library, fill a GPU cache and an oracle cache from
the same seeded workload, compare them."""

import os

import numpy as np
import torch

from quantized_paged_kv_02_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "quantized_paged_kv_02_b200", "libkvq.so")


def ensure_built():
    from quantized_paged_kv_02_b200 import build
    build.build()
    return LIB


def np64(t):
    return t.detach().to(torch.float64).cpu().numpy()


def oracle_static_scales(w):
    from oracle import quant
    if w.spec.scale_mode == "per_channel":
        qmax = 127.0 if w.spec.cache_dtype == "int8" else 448.0
        return (quant.channel_calibrate(np64(w.warmup_k).astype(np.float32), qmax),
                quant.channel_calibrate(np64(w.warmup_v).astype(np.float32), qmax))
    if w.spec.scale_mode in ("per_head", "per_tensor"):
        qmax = 127.0 if w.spec.cache_dtype == "int8" else 448.0
        ks = quant.head_calibrate(np64(w.warmup_k).astype(np.float32), qmax)
        vs = quant.head_calibrate(np64(w.warmup_v).astype(np.float32), qmax)
        if w.spec.scale_mode == "per_tensor":
            ks, vs = ks.max(keepdims=True), vs.max(keepdims=True)
        return ks, vs
    return None


def oracle_cache(w, static=None):
    """Oracle cache holding every row of workload w."""
    from oracle import cache
    s = w.spec
    c = cache.PagedCache(s.cache_dtype, s.act_dtype, s.scale_mode, w.num_blocks, s.block_size,
                         s.num_kv_heads, s.head_dim, residual_len=inputs.RESIDUAL_LEN,
                         residual_cap=inputs.RESIDUAL_CAP, max_seqs=max(s.batch, 1),
                         static_scales=static)
    k, v = np64(w.k), np64(w.v)
    if inputs.low_bit(s.cache_dtype):
        idx, slots, sid, pos = inputs.int4_group_rows(w)
        c.write(k[idx.numpy()], v[idx.numpy()], slots.numpy(), sid.numpy(), pos.numpy())
    else:
        c.write(k, v, w.slot_mapping.cpu().numpy())
    return c


def gpu_cache(w, device="cuda", static=None, fill=0x5A):
    """GPU cache holding every row of workload w, written by kvq_write."""
    from quantized_paged_kv_02_b200 import kvq
    s = w.spec
    sk = sv = None
    if static is not None:
        sk, sv = (torch.as_tensor(np.asarray(x, np.float32), device=device) for x in static)
    c = kvq.PagedKVCache(s.cache_dtype, s.act_dtype, s.scale_mode, w.num_blocks, s.block_size,
                         s.num_kv_heads, s.head_dim, device=device,
                         residual_len=inputs.RESIDUAL_LEN, residual_cap=inputs.RESIDUAL_CAP,
                         max_seqs=max(s.batch, 1), static_k_scale=sk, static_v_scale=sv, fill=fill)
    k, v = w.k.to(device), w.v.to(device)
    if inputs.low_bit(s.cache_dtype):
        idx, slots, sid, pos = inputs.int4_group_rows(w)
        idx = idx.to(device)
        c.write(k[idx].contiguous(), v[idx].contiguous(), slots.to(device), sid.to(device),
                pos.to(device))
    else:
        c.write(k, v, w.slot_mapping.to(device))
    return c


def pool_bytes(t, n):
    return t[:n].cpu().numpy().view(np.uint8)


def assert_same_cache(gc, oc):
    """Byte-for-byte equality of the GPU cache and the oracle cache (pages pool, ring)."""
    np.testing.assert_array_equal(pool_bytes(gc.pages, gc.sizes[1]), oc.pages.reshape(-1))
    if oc.residual is not None:
        np.testing.assert_array_equal(pool_bytes(gc.residual, gc.sizes[3]),
                                      oc.residual.reshape(-1).view(np.uint8))


def single_sequence(w, b):
    """Workload holding only sequence b of w (batch 1, blocks 0..n-1 of a pool of its own).

    Quantization works row by row (per token and head; INT4 keys per 64-row group of one
    sequence), so the oracle's codes for this workload equal those of sequence b in the
    full cache, and its attention output is output row b of the full batch.  Used to
    check full-size runs on sampled sequences."""
    import dataclasses
    s = w.spec
    r0, r1 = int(w.seq_start[b]), int(w.seq_start[b + 1])
    n = r1 - r0
    int4 = inputs.low_bit(s.cache_dtype)
    paged = inputs.INT4_GROUP * (max(n - inputs.RESIDUAL_LEN, 0) // inputs.INT4_GROUP) if int4 else n
    nblk = max(-(-paged // s.block_size), 1)
    pos = torch.arange(n, dtype=torch.int32)
    slots = torch.full((n,), -1, dtype=torch.int32)
    slots[:paged] = pos[:paged]                    # block j holds positions [j*bs, (j+1)*bs)
    positions = seq_ids = None
    if int4:
        positions = torch.full((n,), -1, dtype=torch.int32)
        positions[paged:] = pos[paged:]
        seq_ids = torch.full((n,), -1, dtype=torch.int32)
        seq_ids[paged:] = 0
    cpu = lambda t: None if t is None else t.cpu()
    return inputs.Workload(
        spec=dataclasses.replace(s, batch=1, lens=[n], len_range=None),
        context_lens=torch.tensor([n], dtype=torch.int32),
        k=w.k[r0:r1].cpu(), v=w.v[r0:r1].cpu(), q=w.q[b:b + 1].cpu(),
        seq_start=torch.tensor([0, n], dtype=torch.int64),
        block_tables=torch.arange(nblk, dtype=torch.int32)[None],
        num_blocks=nblk, slot_mapping=slots, seq_ids=seq_ids, positions=positions,
        warmup_k=cpu(w.warmup_k), warmup_v=cpu(w.warmup_v))
