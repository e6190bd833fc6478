#!/usr/bin/env python
"""Benchmark of the quantized paged KV-cache decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c5] [--impl ours|reference]

A step is one serving step of one layer: kvq_write of the batch's new K/V rows into the
quantized paged cache, then kvq_decode_attention over every cached position (split-K
kernel + reduce).  The cache of the previous positions is resident in HBM; the timed
step is bracketed by CUDA events on the launching stream, with a 512 MiB memset before
every step so no cache byte is served from L2.  Metric: KV GB/s = algorithmic bytes of
the step / step time; tokens/s = batch / step time.  One JSON line on stdout.

--impl reference times the float64 CPU oracle (the only other implementation of the
method) on a bounded sample of the same workload; under torchrun only rank 0 runs it.
"""

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized paged decode attention: KV GB/s and % of HBM roofline; tokens/s"
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0

WORKLOADS = {
    "c5": "Llama-3-70B-shaped layer: batch 24, 64 q heads / 8 kv heads, head_dim 128, "
          "context 16384, block 16, INT8 per-token-head scales",
    "c5-fp8": "Llama-3-70B-shaped layer: batch 24, 64/8 heads, head_dim 128, context 16384, "
              "block 16, FP8 E4M3 per-kv-head scales (256-token warm-up)",
    "c5-bf16": "Llama-3-70B-shaped layer: batch 24, 64/8 heads, head_dim 128, context 16384, "
               "block 16, unquantized bf16 cache",
    "c5-int8-pc": "Llama-3-70B-shaped layer: batch 24, 64/8 heads, head_dim 128, context 16384, "
                  "block 16, INT8 static per-(kv head, channel) scales (256-token warm-up)",
    "c2": "Llama-2-7B-shaped layer: batch 4, 32 heads MHA, head_dim 128, context 2048, block 16, "
          "INT8 per-token-head, 4 outlier channels x10 in K and V",
    "c3": "Llama-3-8B-shaped layer: batch 64, 32/8 heads, head_dim 128, context U[1024, 8192], "
          "block 16, FP8 E4M3 per-kv-head scales",
    "c4": "70B-shaped KIVI INT4 layer: batch 16, 64/8 heads, head_dim 128, context 32768, "
          "block 64, keys per channel / values per token, 128-token bf16 residual",
    "c4-tok": "70B-shaped INT4 layer as c4, keys and values both per token (64-channel groups), "
              "128-token bf16 residual",
    "c4-fzp": "70B-shaped KIVI INT4 layer as c4, float zero points (group minimum), "
              "128-token bf16 residual",
    "c4-int2": "70B-shaped 2-bit KIVI layer as c4 (codes 0..3, four per byte), "
               "128-token bf16 residual",
    "c4-int2-tok": "70B-shaped 2-bit layer as c4, keys and values both per token, "
                   "128-token bf16 residual",
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="c5", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (smaller cases for profiling)")
    ap.add_argument("--min-warmup-s", type=float, default=1.0,
                    help="keep warming up for at least this many seconds")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(values, world, device):
    """Each timing is the slowest rank's: one all-reduce (MAX) of the list over the process
    group (every rank calls this with the same length, in the same order)."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def throughput(nbytes_per_rank, world, ms):
    """Whole-job GB/s: every rank processes its own nbytes per step (weak scaling), the step
    time is the slowest rank's."""
    return world * nbytes_per_rank / (ms * 1e-3) / 1e9


# ----------------------------------------------------------------------------- peaks
def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Measured dense bf16 tensor throughput (burst), TFLOP/s."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def measure_prefill(device, l2, steps=20):
    """Chunked prefill on a c5-shaped layer (INT8 per-token-head cache, 64/8 heads, D 128,
    block 16): 4 sequences of 4096 cached tokens whose newest 512 are this chunk's queries,
    each attending causally.  Algorithmic work: 4 D flops (q.k and p.v) per query head and
    visible position."""
    import dataclasses
    import torch
    from quantized_paged_kv_02_b200 import inputs, kvq
    spec = dataclasses.replace(inputs._spec("c5", False), batch=4, lens=[4096] * 4)
    w = inputs.from_spec(spec, device)
    s = w.spec
    c = kvq.PagedKVCache(s.cache_dtype, s.act_dtype, s.scale_mode, w.num_blocks, s.block_size,
                         s.num_kv_heads, s.head_dim, device=device)
    c.write(w.k, w.v, w.slot_mapping)
    L, n = 512, 4096
    g = torch.Generator(device=device).manual_seed(1)
    q = torch.randn((s.batch * L, s.num_q_heads, s.head_dim), generator=g, device=device).to(torch.bfloat16)
    qs = torch.arange(0, s.batch * L + 1, L, dtype=torch.int32, device=device)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=device)

    def call():
        kvq.kvq_prefill_attention(c.desc, q, qs, L, w.block_tables, w.context_lens, n, out)
    for _ in range(3):
        call()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for a, b in ev:
        l2.flush()
        a.record()
        call()
        b.record()
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    visible = s.batch * sum(n - L + i + 1 for i in range(L))
    flops = 4.0 * s.head_dim * s.num_q_heads * visible
    peak, kind = tensor_peak()
    tf = flops / (ms * 1e-3) / 1e12
    return {"value": round(tf, 2), "unit": "TFLOP/s", "ms_per_call": round(ms, 4),
            "frac_of_peak": round(tf / peak, 4), "peak": peak, "peak_kind": kind + " bf16 dense",
            "config": "c5-shaped layer, INT8 per-token-head cache, 4 sequences x 4096 tokens, "
                      "512-query causal chunks (kvq_prefill_attention)"}


def profile_traffic(workload):
    """dram bytes per launch of the decode kernel from the committed ncu summary, or None
    when the summary is missing or was taken on a different kernel source (the summary
    names the source files its kernel is built from and their hash)."""
    path = os.path.join(ROOT, "profiles", "decode_%s.md" % workload.replace("-", "_"))
    try:
        text = open(path).read()
    except OSError:
        return None
    m = re.search(r"dram_bytes_per_launch:\s*(\d+)", text)
    h = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", text)
    f = re.search(r"kernel_sources:\s*(.+)", text)
    if not m or not h or not f or h.group(1) != kernel_source_hash(f.group(1).split()):
        return None
    return int(m.group(1))


def kernel_source_hash(names):
    """First 16 hex digits of the sha256 of the named files of the library's csrc/, in
    the order given."""
    d = os.path.join(ROOT, "quantized_paged_kv_02_b200", "csrc")
    hsh = hashlib.sha256()
    for name in names:
        with open(os.path.join(d, name), "rb") as fh:
            hsh.update(fh.read())
    return hsh.hexdigest()[:16]


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9 or (self.uuid and self.uuid not in f[0]):
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- oracle
def oracle_unit_step(w, unit_rows, b, kvh, static):
    """Set up an oracle cache for one (sequence, kv head) and return a callable that
    performs the step's work for it: quantize the new row, then attention of its query
    heads over every cached position.  float64 CPU oracle, single process."""
    import numpy as np
    import torch
    from oracle import attention, cache
    from quantized_paged_kv_02_b200 import inputs
    s = w.spec
    n = int(w.context_lens[b])
    r0 = int(w.seq_start[b])
    k = unit_rows["k"][b].astype(np.float64)[:, None, :]      # [n, 1, D]
    v = unit_rows["v"][b].astype(np.float64)[:, None, :]
    st = None
    if static is not None:
        st = (static[0][kvh:kvh + 1], static[1][kvh:kvh + 1])
    bs = s.block_size
    if inputs.low_bit(s.cache_dtype):
        qb = 64 * (max(n - 128, 0) // 64)
        nblk = qb // 64
    else:
        qb, nblk = n, -(-n // bs)
    mode = "per_head" if s.scale_mode in ("per_head", "per_tensor") else s.scale_mode
    oc = cache.PagedCache(s.cache_dtype, s.act_dtype, mode, max(nblk, 1), bs, 1, s.head_dim,
                          residual_len=inputs.RESIDUAL_LEN, residual_cap=inputs.RESIDUAL_CAP,
                          max_seqs=1, static_scales=st)
    table = np.arange(max(nblk, 1))
    slots = np.array([p if p < qb else -1 for p in range(n)])
    pos = np.array([-1 if p < qb else p for p in range(n)])
    oc.write(k[:n - 1], v[:n - 1], slots[:n - 1], np.zeros(n - 1, np.int64), pos[:n - 1])
    g = s.num_q_heads // s.num_kv_heads
    q = unit_rows["q"][b][kvh * g:(kvh + 1) * g].astype(np.float64)[None]
    del r0, torch

    def step():
        oc.write(k[n - 1:n], v[n - 1:n], slots[n - 1:n], np.zeros(1, np.int64), pos[n - 1:n])
        return attention.decode_attention(oc, q, table[None, :], np.array([n]), seq_ids=np.array([0]))
    return step


def oracle_inputs(w, units):
    """Host copies of the rows the sampled units need (read from the seeded workload)."""
    import numpy as np
    import torch
    rows = {"k": {}, "v": {}, "q": {}}
    for b, kvh in units:
        r0, r1 = int(w.seq_start[b]), int(w.seq_start[b + 1])
        rows["k"][b] = w.k[r0:r1, kvh].to(torch.float32).cpu().numpy()
        rows["v"][b] = w.v[r0:r1, kvh].to(torch.float32).cpu().numpy()
        rows["q"][b] = w.q[b].to(torch.float32).cpu().numpy()
    del np
    return rows


def unit_bytes(w, b):
    from quantized_paged_kv_02_b200 import inputs, roofline
    s = w.spec
    g = s.num_q_heads // s.num_kv_heads
    return (roofline.decode_bytes(s.cache_dtype, s.scale_mode, g, 1, s.head_dim, s.block_size,
                                  [int(w.context_lens[b])])
            + roofline.write_bytes(s.cache_dtype, s.scale_mode, 1, 1, s.head_dim,
                                   to_ring=inputs.low_bit(s.cache_dtype)))


def unit_workload(name):
    """One (sequence, kv head) unit of the named workload, on the CPU: batch 1, one kv
    head with its whole GQA group, the workload's context length (mean of the range for
    variable lengths).  Same distributions and layout as the full workload."""
    import dataclasses
    from quantized_paged_kv_02_b200 import inputs
    full = inputs._spec(name, False)
    g = full.num_q_heads // full.num_kv_heads
    n = full.lens[0] if full.lens else (full.len_range[0] + full.len_range[1]) // 2
    spec = dataclasses.replace(full, name=full.name + "-unit", batch=1, num_kv_heads=1,
                               num_q_heads=g, lens=[n], len_range=None, slack_blocks=0)
    return inputs.from_spec(spec, "cpu")


def run_oracle_sample(w, static, budget_s=12.0, wall_cap_s=45.0):
    """Time the oracle on (b, kvh) units, cycling through the batch in order, until about
    budget_s seconds of timed oracle work (or wall_cap_s of wall time, set-up of each
    unit's cache included) have passed.  Only the steps count toward the reported rate."""
    from threadpoolctl import threadpool_limits
    units = [(b, h) for b in range(w.spec.batch) for h in range(w.spec.num_kv_heads)]
    done, nbytes, t_total = 0, 0, 0.0
    t_start = time.perf_counter()
    with threadpool_limits(limits=1):
        while True:
            b, kvh = units[done % len(units)]
            if done and (t_total >= budget_s or time.perf_counter() - t_start >= wall_cap_s):
                break
            rows = oracle_inputs(w, [(b, kvh)])
            step = oracle_unit_step(w, rows, b, kvh, static)
            t0 = time.perf_counter()
            step()
            t_total += time.perf_counter() - t0
            nbytes += unit_bytes(w, b)
            done += 1
    return {"units": done, "bytes": nbytes, "seconds": t_total}


# ----------------------------------------------------------------------------- ours
def build_state(workload, device, seed, batch=0):
    import dataclasses
    import torch
    from quantized_paged_kv_02_b200 import inputs, kvq
    spec = inputs._spec(workload, False)
    spec.seed = seed
    if batch:
        lens = spec.lens[:1] * batch if spec.lens else None
        spec = dataclasses.replace(spec, batch=batch, lens=lens)
    w = inputs.from_spec(spec, device)
    s = w.spec
    static = None
    sk = sv = None
    if s.scale_mode in ("per_head", "per_tensor"):
        sk = torch.empty(s.num_kv_heads, dtype=torch.float32, device=device)
        sv = torch.empty(s.num_kv_heads, dtype=torch.float32, device=device)
        kvq.kvq_calibrate_fp8_scales(w.warmup_k, sk)
        kvq.kvq_calibrate_fp8_scales(w.warmup_v, sv)
        static = (sk.cpu().numpy(), sv.cpu().numpy())
    elif s.scale_mode == "per_channel":
        qmax = 127.0 if s.cache_dtype == "int8" else 448.0
        sk = torch.empty((s.num_kv_heads, s.head_dim), dtype=torch.float32, device=device)
        sv = torch.empty_like(sk)
        kvq.kvq_calibrate_channel_scales(w.warmup_k, qmax, sk)
        kvq.kvq_calibrate_channel_scales(w.warmup_v, qmax, sv)
        static = (sk.cpu().numpy(), sv.cpu().numpy())
    c = kvq.PagedKVCache(s.cache_dtype, s.act_dtype, s.scale_mode, w.num_blocks, s.block_size,
                         s.num_kv_heads, s.head_dim, device=device,
                         residual_len=inputs.RESIDUAL_LEN, residual_cap=inputs.RESIDUAL_CAP,
                         max_seqs=s.batch, static_k_scale=sk, static_v_scale=sv)
    if inputs.low_bit(s.cache_dtype):
        idx, slots, sid, pos = inputs.int4_group_rows(w)
        idx = idx.to(device)
        c.write(w.k[idx].contiguous(), w.v[idx].contiguous(), slots.to(device), sid.to(device),
                pos.to(device))
    else:
        c.write(w.k, w.v, w.slot_mapping)
    # the step's new token: the last position of every sequence
    last = (w.seq_start[1:] - 1).to(device)
    new = {"k": w.k[last].contiguous(), "v": w.v[last].contiguous()}
    if inputs.low_bit(s.cache_dtype):
        new["slots"] = torch.full((s.batch,), -1, dtype=torch.int32, device=device)
        new["seq_ids"] = torch.arange(s.batch, dtype=torch.int32, device=device)
        new["positions"] = (w.context_lens - 1).to(torch.int32)
    else:
        new["slots"] = w.slot_mapping[last].contiguous()
        new["seq_ids"] = new["positions"] = None
    return w, c, new, static


class L2Flush:
    """Empties L2 between timed steps: write 512 MiB (more than the 126 MB L2), then read
    256 MiB so the lines the write left dirty are written back here, outside the timed
    region, instead of being charged to the first kernel of the step."""
    DESCRIPTION = ("flushed before every timed step, outside the events: 512 MiB written, "
                   "then 256 MiB read (L2 left clean and cold)")

    def __init__(self, device):
        import torch
        self.w = torch.empty(512 << 20, dtype=torch.uint8, device=device)
        self.r = torch.zeros(64 << 20, dtype=torch.float32, device=device)
        self.acc = torch.empty((), dtype=torch.float32, device=device)

    def flush(self):
        import torch
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.acc)


def main_ours(args):
    import torch
    import torch.distributed as dist
    from quantized_paged_kv_02_b200 import build
    build.build()
    from quantized_paged_kv_02_b200 import inputs, kvq, roofline

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    w, cache, new, static = build_state(args.workload, device, seed=rank, batch=args.batch)
    s = w.spec
    B = s.batch
    out = torch.empty(w.q.shape, dtype=torch.bfloat16, device=device)
    max_ctx = w.max_context
    ws_n = cache.workspace_size(B, s.num_q_heads, max_ctx)
    ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=device) if ws_n else None
    stream = torch.cuda.current_stream()

    def write():
        cache.write(new["k"], new["v"], new["slots"], new["seq_ids"], new["positions"])

    def decode():
        kvq.kvq_decode_attention(cache.desc, w.q, w.block_tables, w.context_lens, max_ctx, out, ws)

    lens = w.context_lens.cpu().tolist()
    dec_bytes = roofline.decode_bytes(s.cache_dtype, s.scale_mode, s.num_q_heads, s.num_kv_heads,
                                      s.head_dim, s.block_size, lens)
    wr_bytes = roofline.write_bytes(s.cache_dtype, s.scale_mode, B, s.num_kv_heads, s.head_dim,
                                    to_ring=inputs.low_bit(s.cache_dtype))
    step_bytes = dec_bytes + wr_bytes
    l2 = L2Flush(device)

    # warm-up (at least ~1 s under load so the clock sampler sees the steady state)
    sampler = ClockSampler(str(torch.cuda.get_device_properties(device).uuid))
    sampler.start()
    t_w = time.perf_counter()
    i = 0
    while i < max(3, args.warmup) or time.perf_counter() - t_w < args.min_warmup_s:
        l2.flush()
        write()
        decode()
        i += 1
        if i % 50 == 0:
            torch.cuda.synchronize()
    warm = i
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for k in range(K):
        l2.flush()
        e = ev[k]
        e[0].record(stream)
        write()
        e[1].record(stream)
        decode()
        e[2].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    step_ms = [ev[k][0].elapsed_time(ev[k][2]) for k in range(K)]
    dec_ms = [ev[k][1].elapsed_time(ev[k][2]) for k in range(K)]
    ms = statistics.mean(step_ms)
    dms = statistics.mean(dec_ms)
    ms, dms = max_over_ranks([ms, dms], world, device)

    # the same step as one call (kvq_append_decode_attention), dense caches only
    fused = None
    if not inputs.low_bit(s.cache_dtype) and K > 0:
        def fused_step():
            kvq.kvq_append_decode_attention(cache.desc, new["k"], new["v"], w.q, w.block_tables,
                                            w.context_lens, max_ctx, out, ws)
        for _ in range(3):
            l2.flush()
            fused_step()
        fev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
        torch.cuda.synchronize()
        for a, b2 in fev:
            l2.flush()
            a.record(stream)
            fused_step()
            b2.record(stream)
        torch.cuda.synchronize()
        fms = statistics.mean(a.elapsed_time(b2) for a, b2 in fev)
        fms, = max_over_ranks([fms], world, device)
        fused = {"value": round(world * step_bytes / (fms * 1e-3) / 1e9, 2), "unit": "GB/s",
                 "ms_per_step": round(fms, 5), "tokens_per_s": round(world * B / (fms * 1e-3), 1),
                 "frac_of_peak": round(step_bytes / (fms * 1e-3) / 1e9 / hbm_peak()[0], 4),
                 "call": "kvq_append_decode_attention (append step fused into the decode kernel)"}

    # chunked prefill on its own c5-shaped case (default workload only)
    prefill = measure_prefill(device, l2) if args.workload == "c5" and K > 0 else None

    # end to end through the C ABI: the step's inputs (new K/V rows, slots, q, lengths) packed
    # in one pinned host buffer and copied to the device in one transfer inside the timed
    # region, the output copied back; the step is one kvq_append_decode_attention call for
    # dense caches, kvq_write + kvq_decode_attention for INT4 / INT2
    E = args.e2e_steps
    parts = [new["k"], new["v"], new["slots"], w.q, w.context_lens]
    offs, total = [], 0
    for t in parts:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    hbuf = torch.empty(total, dtype=torch.uint8).pin_memory()
    dbuf = torch.empty(total, dtype=torch.uint8, device=device)
    dviews = []
    for t, o in zip(parts, offs):
        n = t.numel() * t.element_size()
        hbuf[o:o + n].copy_(t.detach().contiguous().view(-1).view(torch.uint8).cpu())
        dviews.append(dbuf[o:o + n].view(t.dtype).view(t.shape))
    dk, dv, dslots, dq, dl = dviews
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = hbuf.numel()
    d2h = hout.numel() * hout.element_size()
    fused_e2e = not inputs.low_bit(s.cache_dtype)
    e2e_ms = []
    for k in range(E + 3 if E > 0 else 0):
        l2.flush()
        a, b2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        dbuf.copy_(hbuf, non_blocking=True)
        if fused_e2e:
            kvq.kvq_append_decode_attention(cache.desc, dk, dv, dq, w.block_tables, dl, max_ctx, out, ws)
        else:
            kvq.kvq_write(cache.desc, dk, dv, dslots, new["seq_ids"], new["positions"])
            kvq.kvq_decode_attention(cache.desc, dq, w.block_tables, dl, max_ctx, out, ws)
        hout.copy_(out, non_blocking=True)
        b2.record(stream)
        b2.synchronize()
        if k >= 3:
            e2e_ms.append(a.elapsed_time(b2))
    e2e = statistics.mean(e2e_ms) if e2e_ms else float("nan")
    e2e, = max_over_ranks([e2e], world, device)

    peak, peak_kind = hbm_peak()
    achieved = dec_bytes / (dms * 1e-3) / 1e9
    launches_per_step = 1 + cache.decode_plan(B, s.num_q_heads, max_ctx)[1]
    result = {
        "metric": METRIC,
        "value": round(throughput(step_bytes, world, ms), 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": warm,
        "ms_per_step": round(ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp32",
        "cache_dtype": s.cache_dtype,
        "data": "synthetic",
        "config": {"workload": "%s: %s; step = kvq_write of %d new tokens + decode attention%s"
                               % (args.workload, WORKLOADS[args.workload], B,
                                  "" if not args.batch else
                                  " (batch reduced to %d for profiling: not a benchmark line)" % B),
                   "global_batch": B * world, "seq_len": max_ctx, "parallelism": "dp%d" % world,
                   "l2": L2Flush.DESCRIPTION},
        "tokens_per_s": round(world * B / (ms * 1e-3), 1),
        "hbm_frac_of_%s" % peak_kind: round(step_bytes / (ms * 1e-3) / 1e9 / peak, 4),
        "bytes_per_step": step_bytes,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "peak_kind": peak_kind, "kernel": "kvq_decode_attention (split kernel + reduce)",
                     "bytes_per_launch": dec_bytes, "ms_per_launch": round(dms, 5),
                     "traffic": profile_traffic(args.workload)},
        "e2e": {"value": round(world * step_bytes / (e2e * 1e-3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(e2e, 5), "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "call": ("kvq_append_decode_attention" if fused_e2e
                         else "kvq_write + kvq_decode_attention") +
                        ", one packed host-to-device copy of the step's inputs, output copied back"},
        "append_decode": fused,
        "prefill": prefill,
        "gpu_launches": launches_per_step * K,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = run_oracle_sample(w, static)
        result["cpu_baseline"] = {
            "value": round(r["bytes"] / r["seconds"] / 1e9, 6), "unit": "GB/s", "cores": 1,
            "kind": "oracle",
            "sample": "%d (sequence, kv head) units of the %d in the step, taken in order and "
                      "cycling; each: quantize the new row + float64 attention of its %d query "
                      "heads over all cached positions; %.1f s of timed oracle work"
                      % (r["units"], B * s.num_kv_heads, s.num_q_heads // s.num_kv_heads,
                         r["seconds"])}
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def main_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import torch
    from quantized_paged_kv_02_b200 import inputs
    from threadpoolctl import threadpool_limits
    w = unit_workload(args.workload)
    static = None
    if w.spec.scale_mode in ("per_head", "per_tensor"):
        from oracle import quant
        static = (quant.fp8_calibrate(w.warmup_k.float().numpy()),
                  quant.fp8_calibrate(w.warmup_v.float().numpy()))
    elif w.spec.scale_mode == "per_channel":
        from oracle import quant
        qmax = 127.0 if w.spec.cache_dtype == "int8" else 448.0
        static = (quant.channel_calibrate(w.warmup_k.float().numpy(), qmax),
                  quant.channel_calibrate(w.warmup_v.float().numpy(), qmax))
    rows = oracle_inputs(w, [(0, 0)])
    step = oracle_unit_step(w, rows, 0, 0, static)
    nbytes = unit_bytes(w, 0)
    with threadpool_limits(limits=1):
        for _ in range(max(1, args.warmup)):
            step()
        times = []
        for _ in range(args.steps):
            t0 = time.perf_counter()
            step()
            times.append(time.perf_counter() - t0)
    sec = statistics.mean(times)
    value = nbytes / sec / 1e9
    del torch
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "%s: %s; step = one (sequence, kv head) unit of the serving step"
                               % (args.workload, WORKLOADS[args.workload])},
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": "unit (sequence 0, kv head 0): quantize the new row + float64 "
                                   "attention of its query heads over every cached position"},
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        main_reference(a)
    else:
        main_ours(a)
