"""Seeded synthetic workloads shared by the tests, the benchmark and the oracle checks.

This module only draws random numbers and lays out indices (block tables, slot
mappings, ring positions).  It holds none of the quantization or attention arithmetic,
so the CUDA path and the CPU oracle can both take their inputs from it without sharing
any of the method.

Recipe (all on one ``torch.Generator`` seeded with ``seed``, in this order):
  1. context lengths (fixed, or uniform integers in [lo, hi] for variable workloads);
  2. K rows, V rows: ``randn`` float32 [total_tokens, H_kv, D];
  3. q: ``randn`` float32 [B, H_q, D];
  4. outlier channels: for each kv head, ``randperm(D)[:4]``; the listed tensors (K, or
     K and V) are multiplied by 10 on those channels;
  5. block table: ``randperm(num_blocks)``; sequence b takes the next ceil(n_b/bs)
     entries, so tables are non-contiguous and the unused blocks are spread out;
  6. warm-up rows for static scales (per head, per tensor, per channel): ``randn`` float32
     [256, H_kv, D] for K, then V.
Values are cast to the activation dtype (round to nearest even) after step 4.

The five named workloads follow the shapes of the method's benchmark configurations
(Llama-style layers); ``small=True`` shrinks batch, heads and lengths so the float64
oracle finishes in seconds while several blocks and a ragged tail remain.
"""

from dataclasses import dataclass, field
from typing import List, Optional

import torch

RESIDUAL_LEN = 128
RESIDUAL_CAP = 192
INT4_GROUP = 64


def low_bit(cache_dtype):
    """INT4 and 2-bit caches: 64-token groups, a residual ring of recent tokens."""
    return cache_dtype in ("int4", "int2")


@dataclass
class Spec:
    name: str
    cache_dtype: str            # bf16 | fp16 | int8 | fp8 | int4 | int2
    act_dtype: str              # bf16 | fp16
    scale_mode: str             # none | per_token_head | per_head | per_tensor | per_channel |
                                # kivi | kivi_float_zero | int4_per_token
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    lens: Optional[List[int]] = None       # fixed context lengths
    len_range: Optional[tuple] = None      # (lo, hi) inclusive, drawn per sequence
    outliers: str = ""                     # "", "k", "kv"
    slack_blocks: int = 0
    seed: int = 0


def _spec(name, small):
    if name == "c1":
        return Spec("c1", "int8", "fp16", "per_token_head", 2, 8, 4, 64, 16,
                    lens=[128, 77], slack_blocks=3)
    if name == "c2":
        if small:
            return Spec("c2-small", "int8", "bf16", "per_token_head", 2, 4, 4, 128, 16,
                        lens=[300, 211], outliers="kv", slack_blocks=5)
        return Spec("c2", "int8", "bf16", "per_token_head", 4, 32, 32, 128, 16,
                    lens=[2048] * 4, outliers="kv")
    if name == "c3":
        if small:
            return Spec("c3-small", "fp8", "bf16", "per_head", 4, 8, 2, 128, 16,
                        len_range=(100, 700), slack_blocks=9)
        return Spec("c3", "fp8", "bf16", "per_head", 64, 32, 8, 128, 16,
                    len_range=(1024, 8192), slack_blocks=64)
    if name in ("c4", "c4-tok", "c4-fzp", "c4-int2", "c4-int2-tok", "c4-int2-fzp"):
        # -tok: keys and values per token (64-channel groups); -fzp: KIVI groups with the
        # group minimum as a float zero point; -int2: 2-bit codes; shapes and inputs as c4
        mode = "int4_per_token" if name.endswith("-tok") else \
            "kivi_float_zero" if name.endswith("-fzp") else "kivi"
        cd = "int2" if "int2" in name else "int4"
        if small:
            return Spec(name + "-small", cd, "bf16", mode, 2, 16, 2, 128, 64,
                        lens=[485, 200], outliers="k", slack_blocks=3)
        return Spec(name, cd, "bf16", mode, 16, 64, 8, 128, 64,
                    lens=[32768] * 16, outliers="k", slack_blocks=16)
    if name.startswith("c5"):
        # -pc / -ph / -pt: static scales per (kv head, channel), per kv head, per tensor
        cd = {"c5": "int8", "c5-int8": "int8", "c5-fp8": "fp8", "c5-bf16": "bf16",
              "c5-int8-pc": "int8", "c5-int8-ph": "int8", "c5-int8-pt": "int8",
              "c5-fp8-pt": "fp8"}[name]
        mode = {"int8": "per_token_head", "fp8": "per_head", "bf16": "none"}[cd]
        mode = {"pc": "per_channel", "ph": "per_head", "pt": "per_tensor"}.get(name[-2:], mode)
        if small:
            return Spec(name + "-small", cd, "bf16", mode, 3, 16, 2, 128, 16,
                        lens=[1000, 517, 33], slack_blocks=4)
        return Spec(name, cd, "bf16", mode, 24, 64, 8, 128, 16, lens=[16384] * 24)
    raise KeyError(name)


@dataclass
class Workload:
    spec: Spec
    context_lens: torch.Tensor      # int32 [B]
    k: torch.Tensor                 # act dtype [T, H_kv, D]: rows of all sequences
    v: torch.Tensor
    q: torch.Tensor                 # act dtype [B, H_q, D]
    seq_start: torch.Tensor         # int64 [B+1]: row offsets of each sequence in k/v
    block_tables: torch.Tensor      # int32 [B, max_blocks]
    num_blocks: int
    slot_mapping: torch.Tensor      # int32 [T]: slot of each row, -1 for ring rows
    seq_ids: Optional[torch.Tensor] = None     # int32 [T] (INT4 ring rows)
    positions: Optional[torch.Tensor] = None   # int32 [T] (INT4 ring rows, else -1)
    warmup_k: Optional[torch.Tensor] = None    # act dtype [256, H_kv, D]
    warmup_v: Optional[torch.Tensor] = None
    outlier_channels: Optional[torch.Tensor] = None
    extra: dict = field(default_factory=dict)

    @property
    def max_context(self):
        return int(self.context_lens.max().item()) if self.context_lens.numel() else 0


def act_torch_dtype(act):
    return {"bf16": torch.bfloat16, "fp16": torch.float16}[act]


def make(name, small=False, device="cpu", seed=None):
    """Build the named workload ("c1".."c5", "c4-tok", "c4-fzp", "c4-int2", "c4-int2-tok",
    "c4-int2-fzp", "c5-fp8", "c5-bf16", "c5-int8-pc", "c5-int8-ph", "c5-int8-pt",
    "c5-fp8-pt") on `device`."""
    spec = _spec(name, small)
    if seed is not None:
        spec.seed = seed
    return from_spec(spec, device)


def from_spec(spec, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(spec.seed)
    B, Hq, H, D, bs = spec.batch, spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.block_size
    if spec.lens is not None:
        lens = torch.tensor(spec.lens, dtype=torch.int64)
    else:
        lo, hi = spec.len_range
        lens = torch.randint(lo, hi + 1, (B,), generator=g, device=device).to("cpu")
    T = int(lens.sum())
    k = torch.randn((T, H, D), generator=g, device=device, dtype=torch.float32)
    v = torch.randn((T, H, D), generator=g, device=device, dtype=torch.float32)
    q = torch.randn((B, Hq, D), generator=g, device=device, dtype=torch.float32)
    outl = None
    if spec.outliers:
        outl = torch.stack([torch.randperm(D, generator=g, device=device)[:4] for _ in range(H)])
        mult = torch.ones((H, D), device=device, dtype=torch.float32)
        mult.scatter_(1, outl, 10.0)
        k *= mult
        if spec.outliers == "kv":
            v *= mult
    adt = act_torch_dtype(spec.act_dtype)
    k, v, q = k.to(adt), v.to(adt), q.to(adt)

    # paged placement: rows of sequence b at positions 0..n_b-1
    int4 = low_bit(spec.cache_dtype)
    paged = []
    for n in lens.tolist():
        if int4:
            paged.append(INT4_GROUP * (max(n - RESIDUAL_LEN, 0) // INT4_GROUP))
        else:
            paged.append(n)
    blocks_per_seq = [-(-p // bs) for p in paged]
    need = sum(blocks_per_seq)
    num_blocks = need + spec.slack_blocks
    perm = torch.randperm(num_blocks, generator=g, device=device).to("cpu")
    max_blocks = max(max(blocks_per_seq), 1)
    tables = torch.zeros((B, max_blocks), dtype=torch.int32)
    slots = torch.full((T,), -1, dtype=torch.int32)
    positions = torch.full((T,), -1, dtype=torch.int32) if int4 else None
    seq_ids = torch.full((T,), -1, dtype=torch.int32) if int4 else None
    start = [0]
    cursor = 0
    for b, n in enumerate(lens.tolist()):
        nb = blocks_per_seq[b]
        blk = perm[cursor:cursor + nb]
        cursor += nb
        tables[b, :nb] = blk.to(torch.int32)
        r0 = start[-1]
        pos = torch.arange(paged[b], dtype=torch.int64)
        slots[r0:r0 + paged[b]] = (blk[pos // bs].to(torch.int64) * bs + pos % bs).to(torch.int32)
        if int4:
            positions[r0 + paged[b]:r0 + n] = torch.arange(paged[b], n, dtype=torch.int32)
            seq_ids[r0 + paged[b]:r0 + n] = b
        start.append(r0 + n)
    wk = wv = None
    if spec.scale_mode in ("per_head", "per_tensor", "per_channel"):
        wk = torch.randn((256, H, D), generator=g, device=device, dtype=torch.float32).to(adt)
        wv = torch.randn((256, H, D), generator=g, device=device, dtype=torch.float32).to(adt)
    dev = torch.device(device)
    return Workload(
        spec=spec,
        context_lens=lens.to(torch.int32).to(dev),
        k=k, v=v, q=q,
        seq_start=torch.tensor(start, dtype=torch.int64),
        block_tables=tables.to(dev),
        num_blocks=num_blocks,
        slot_mapping=slots.to(dev),
        seq_ids=None if seq_ids is None else seq_ids.to(dev),
        positions=None if positions is None else positions.to(dev),
        warmup_k=wk, warmup_v=wv, outlier_channels=outl,
    )


def int4_group_rows(w):
    """Reorder an INT4 workload's rows for kvq_write: the block rows of every sequence
    first (each sequence has a whole number of 64-row blocks, so every block run starts
    at a multiple of 64), then the ring rows.  Returns (row_index int64 [T], slot,
    seq_ids, positions) in the new order."""
    slots = w.slot_mapping.cpu()
    pos = w.positions.cpu()
    sid = w.seq_ids.cpu()
    paged_rows = torch.nonzero(slots >= 0).flatten()
    ring_rows = torch.nonzero(slots < 0).flatten()
    assert paged_rows.numel() % INT4_GROUP == 0
    idx = torch.cat([paged_rows, ring_rows])
    return (idx, slots[idx].contiguous(), sid[idx].contiguous(), pos[idx].contiguous())
