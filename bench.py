#!/usr/bin/env python
"""Benchmark of the quantized paged KV-cache decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c5] [--impl ours|reference]

A step is one serving step of one layer: kvq_write of the batch's new K/V rows into the
quantized paged cache, then kvq_decode_attention over every cached position (split
decode kernel with its log-sum-exp merge).  The cache of the previous positions is resident in HBM; the timed
step is bracketed by CUDA events on the launching stream, with a 512 MiB memset before
every step so no cache byte is served from L2.  Metric: KV GB/s = algorithmic bytes of
the step / step time; tokens/s = batch / step time.  One JSON line on stdout.

The default run (workload c5, one GPU) also times, at full size and with the same protocol,
the decode call of the other target configurations ("configs": c2, c3, c4, c4-int2, c5-fp8,
c5-bf16), the kvq_write of a 4 x 8192-token prefill chunk ("write_prefill") and chunked
prefill attention ("prefill"), and the float64 CPU oracle on every host core
("cpu_baseline").

--impl reference times the float64 CPU oracle (the only other implementation of the
method) on every host core, one (sequence, kv head) unit per core per step; under torchrun
only rank 0 runs it.
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
    "c5-int8-ph": "Llama-3-70B-shaped layer: batch 24, 64/8 heads, head_dim 128, context 16384, "
                  "block 16, INT8 static per-kv-head scales (256-token warm-up)",
    "c5-int8-pt": "Llama-3-70B-shaped layer: batch 24, 64/8 heads, head_dim 128, context 16384, "
                  "block 16, INT8 static per-tensor scale (256-token warm-up)",
    "c5-fp8-pt": "Llama-3-70B-shaped layer: batch 24, 64/8 heads, head_dim 128, context 16384, "
                 "block 16, FP8 E4M3 static per-tensor scale (256-token warm-up)",
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
    ap.add_argument("--prefill-only", action="store_true",
                    help="time only chunked prefill on the workload's cache type (--batch "
                         "sequences of 4096 tokens, 512-query chunks; for profiling)")
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


def prefill_flops(batch, n, L, num_q_heads, head_dim):
    """Algorithmic flops of a causal prefill chunk: the newest L of a sequence's n cached
    tokens are its queries, query i (position n - L + i) sees positions 0 .. n - L + i; per
    query head and visible position q.k and p.v take 2 D flops each."""
    visible = batch * sum(n - L + i + 1 for i in range(L))
    return 4.0 * head_dim * num_q_heads * visible


def measure_prefill(device, l2, workload="c5", steps=20, batch=4, n=4096, chunk=512):
    """Chunked prefill on a layer of the named workload's cache type and heads (c5: INT8
    per-token-head, 64/8 heads, D 128, block 16): `batch` sequences of n cached tokens whose
    newest `chunk` are this chunk's queries, each attending causally
    (kvq_prefill_attention).  Algorithmic work: 4 D flops (q.k and p.v) per query head and
    visible position; throughput against the measured dense bf16 tensor peak."""
    import torch
    from quantized_paged_kv_02_b200 import kvq
    w, c, _, _ = build_state(workload, device, 0, batch=batch, lens=[n] * batch)
    s = w.spec
    L = chunk
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
    flops = prefill_flops(s.batch, n, L, s.num_q_heads, s.head_dim)
    peak, kind = tensor_peak()
    tf = flops / (ms * 1e-3) / 1e12
    res = {"value": round(tf, 2), "unit": "TFLOP/s", "ms_per_call": round(ms, 4),
           "frac_of_peak": round(tf / peak, 4), "peak": peak, "peak_kind": kind + " bf16 dense",
           "flops_per_call": flops,
           "config": "%s layer (%s %s cache, %d/%d heads, head_dim %d, block %d), %d sequences x "
                     "%d tokens, %d-query causal chunks (kvq_prefill_attention)"
                     % (workload, s.cache_dtype, s.scale_mode, s.num_q_heads, s.num_kv_heads,
                        s.head_dim, s.block_size, s.batch, n, L)}
    del w, c, q, out
    torch.cuda.empty_cache()
    return res


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


def unit_case(name, tmpdir):
    """The oracle's inputs for one unit of the named workload (seed 0): its rows, query group
    and static scales saved as NumPy arrays under tmpdir, plus the plain numbers the oracle
    needs, so a worker process loads them without torch or a GPU.  Static scales come from
    the oracle's own calibration of the workload's warm-up rows."""
    import numpy as np
    from oracle import quant
    from quantized_paged_kv_02_b200 import inputs
    w = unit_workload(name)
    s = w.spec
    arrays = {"k": w.k[:, 0].float().numpy(), "v": w.v[:, 0].float().numpy(),
              "q": w.q[0].float().numpy()}
    if s.scale_mode in ("per_head", "per_tensor", "per_channel"):
        qmax = 127.0 if s.cache_dtype == "int8" else 448.0
        cal = quant.channel_calibrate if s.scale_mode == "per_channel" else quant.head_calibrate
        arrays["sk"] = cal(w.warmup_k.float().numpy(), qmax)
        arrays["sv"] = cal(w.warmup_v.float().numpy(), qmax)
    path = os.path.join(tmpdir, "unit_%s.npz" % name)
    np.savez(path, **arrays)
    return {"path": path, "cache_dtype": s.cache_dtype, "act_dtype": s.act_dtype,
            "scale_mode": s.scale_mode, "block_size": s.block_size, "head_dim": s.head_dim,
            "n": int(w.context_lens[0]), "low_bit": inputs.low_bit(s.cache_dtype),
            "residual_len": inputs.RESIDUAL_LEN, "residual_cap": inputs.RESIDUAL_CAP,
            "bytes": unit_bytes(w, 0), "g": s.num_q_heads // s.num_kv_heads}


def oracle_unit_step(case):
    """Set up an oracle cache for one (sequence, kv head) holding all but its newest row and
    return a callable that performs the step's work for it: quantize the new row, then
    float64 attention of its query heads over every cached position."""
    import numpy as np
    from oracle import attention, cache
    arr = np.load(case["path"])
    n, bs = case["n"], case["block_size"]
    k = arr["k"].astype(np.float64)[:, None, :]      # [n, 1, D]
    v = arr["v"].astype(np.float64)[:, None, :]
    st = (arr["sk"], arr["sv"]) if "sk" in arr else None
    if case["low_bit"]:
        qb = 64 * (max(n - case["residual_len"], 0) // 64)
        nblk = qb // 64
    else:
        qb, nblk = n, -(-n // bs)
    mode = case["scale_mode"]
    if mode == "per_tensor":           # one kv head: its one scale
        mode, st = "per_head", (st[0][:1], st[1][:1])
    oc = cache.PagedCache(case["cache_dtype"], case["act_dtype"], mode, max(nblk, 1), bs, 1,
                          case["head_dim"], residual_len=case["residual_len"],
                          residual_cap=case["residual_cap"], max_seqs=1, static_scales=st)
    table = np.arange(max(nblk, 1))
    slots = np.array([p if p < qb else -1 for p in range(n)])
    pos = np.array([-1 if p < qb else p for p in range(n)])
    oc.write(k[:n - 1], v[:n - 1], slots[:n - 1], np.zeros(n - 1, np.int64), pos[:n - 1])
    q = arr["q"].astype(np.float64)[None]

    def step():
        oc.write(k[n - 1:n], v[n - 1:n], slots[n - 1:n], np.zeros(1, np.int64), pos[n - 1:n])
        return attention.decode_attention(oc, q, table[None, :], np.array([n]), seq_ids=np.array([0]))
    return step


def _oracle_worker(case, cmd_q, res_q):
    """Worker process of the oracle pool: one BLAS/OpenMP thread, one unit cache; runs one
    unit step per command and reports its start and end (CLOCK_MONOTONIC, shared by all
    processes of the host)."""
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        step = oracle_unit_step(case)
        res_q.put(None)
        while cmd_q.get() is not None:
            t0 = time.perf_counter()
            step()
            res_q.put((t0, time.perf_counter()))


class OraclePool:
    """The float64 oracle on every host core: one spawned process per core of
    os.sched_getaffinity(0) (spawn, so no process is forked from a CUDA context), each holding
    its own copy of one (sequence, kv head) unit of the workload.  A round is one unit step on
    every worker at once; its time is from the first start to the last end."""
    MAX_WORKERS = 256

    def __init__(self, workload, workers=0):
        import multiprocessing as mp
        import tempfile
        self.tmp = tempfile.TemporaryDirectory(prefix="kvq_oracle_")
        self.case = unit_case(workload, self.tmp.name)
        self.cores = len(os.sched_getaffinity(0))
        self.workers = workers or max(1, min(self.cores, self.MAX_WORKERS))
        ctx = mp.get_context("spawn")
        self.res = ctx.Queue()
        self.cmds = [ctx.Queue() for _ in range(self.workers)]
        self.procs = [ctx.Process(target=_oracle_worker, args=(self.case, c, self.res), daemon=True)
                      for c in self.cmds]
        for pr in self.procs:
            pr.start()
        for _ in self.procs:
            self.res.get(timeout=600)

    def round(self):
        for c in self.cmds:
            c.put(1)
        spans = [self.res.get(timeout=600) for _ in self.cmds]
        return max(t1 for _, t1 in spans) - min(t0 for t0, _ in spans)

    def bytes_per_round(self):
        return self.workers * self.case["bytes"]

    def close(self):
        for c in self.cmds:
            c.put(None)
        for pr in self.procs:
            pr.join(timeout=30)
        self.tmp.cleanup()


def run_oracle_sample(workload, budget_s=10.0):
    """cpu_baseline: rounds of the oracle pool until about budget_s seconds of rounds."""
    pool = OraclePool(workload)
    try:
        pool.round()                               # untimed: first touch of every cache
        t, rounds = 0.0, 0
        while t < budget_s:
            t += pool.round()
            rounds += 1
        value = rounds * pool.bytes_per_round() / t / 1e9
        return {"value": round(value, 6), "unit": "GB/s", "cores": pool.workers, "kind": "oracle",
                "host_cores": pool.cores,
                "sample": "%d rounds of one step of a (sequence, kv head) unit (%d cached tokens, "
                          "%d query heads; quantize the new row + float64 attention) on each of "
                          "%d worker processes, one per host core, one thread each; %.1f s"
                          % (rounds, pool.case["n"], pool.case["g"], pool.workers, t)}
    finally:
        pool.close()


# ----------------------------------------------------------------------------- ours
def build_state(workload, device, seed, batch=0, lens=None):
    import dataclasses
    import torch
    from quantized_paged_kv_02_b200 import inputs, kvq
    spec = inputs._spec(workload, False)
    spec.seed = seed
    if batch:
        if lens is None:
            lens = spec.lens[:1] * batch if spec.lens else None
        spec = dataclasses.replace(spec, batch=batch, lens=lens, len_range=None if lens else spec.len_range)
    w = inputs.from_spec(spec, device)
    s = w.spec
    static = None
    sk = sv = None
    if s.scale_mode in ("per_head", "per_tensor"):
        qmax = 127.0 if s.cache_dtype == "int8" else 448.0
        sk = torch.empty(s.num_kv_heads, dtype=torch.float32, device=device)
        sv = torch.empty(s.num_kv_heads, dtype=torch.float32, device=device)
        kvq.kvq_calibrate_head_scales(w.warmup_k, qmax, sk)
        kvq.kvq_calibrate_head_scales(w.warmup_v, qmax, sv)
        if s.scale_mode == "per_tensor":          # one scale: the largest per-head one
            sk, sv = sk.max().reshape(1), sv.max().reshape(1)
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


# full-size configurations measured beside the main workload in the default run: the
# decode call alone, with the main workload's timing protocol
SUB_WORKLOADS = (("c2", "c2"), ("c3", "c3"), ("c4", "c4"), ("c4_int2", "c4-int2"),
                 ("c5_fp8", "c5-fp8"), ("c5_bf16", "c5-bf16"))


def measure_decode_call(workload, device, l2, steps, warmup):
    """kvq_decode_attention alone (every kernel it launches) on the full-size workload: CUDA
    events on the launching stream around each call, L2 emptied before each (outside the
    events), at least `warmup` untimed calls and 0.3 s under load first, clocks sampled."""
    import torch
    from quantized_paged_kv_02_b200 import kvq, roofline
    w, cache, _, _ = build_state(workload, device, seed=0)
    s = w.spec
    out = torch.empty(w.q.shape, dtype=torch.bfloat16, device=device)
    mc = w.max_context
    ws_n = cache.workspace_size(s.batch, s.num_q_heads, mc)
    ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=device) if ws_n else None

    def decode():
        kvq.kvq_decode_attention(cache.desc, w.q, w.block_tables, w.context_lens, mc, out, ws)
    nbytes = roofline.decode_bytes(s.cache_dtype, s.scale_mode, s.num_q_heads, s.num_kv_heads,
                                   s.head_dim, s.block_size, w.context_lens.cpu().tolist())
    sampler = ClockSampler(str(torch.cuda.get_device_properties(device).uuid))
    sampler.start()
    t0, i = time.perf_counter(), 0
    while i < max(3, warmup) or time.perf_counter() - t0 < 0.3:
        l2.flush()
        decode()
        i += 1
        if i % 50 == 0:
            torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    torch.cuda.synchronize()
    for a, b in ev:
        l2.flush()
        a.record()
        decode()
        b.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    peak, kind = hbm_peak()
    gbs = nbytes / (ms * 1e-3) / 1e9
    res = {"workload": "%s: %s" % (workload, WORKLOADS[workload]), "value": round(gbs, 2),
           "unit": "GB/s", "ms_per_call": round(ms, 5), "frac": round(gbs / peak, 4),
           "peak": peak, "peak_kind": kind, "tokens_per_s": round(s.batch / (ms * 1e-3), 1),
           "bytes_per_call": nbytes,
           "launches_per_call": cache.decode_plan(s.batch, s.num_q_heads, mc)[1],
           "calls": steps, "warmup_calls": i, "clocks": clocks}
    del w, cache, out, ws
    torch.cuda.empty_cache()
    return res


def measure_write_prefill(device, l2, steps, warmup):
    """kvq_write of a prefill chunk: 4 sequences x 8192 new tokens of a 70B-shaped layer (8 kv
    heads, head_dim 128), K and V, into an INT8 per-token-head and an FP8 per-kv-head cache.
    Algorithmic bytes: the bf16 rows and slot ids read, the codes (and INT8 scales) written."""
    import dataclasses
    import torch
    from quantized_paged_kv_02_b200 import inputs, kvq, roofline
    peak, kind = hbm_peak()
    res = {}
    for cd, mode in (("int8", "per_token_head"), ("fp8", "per_head")):
        spec = dataclasses.replace(inputs._spec("c5", False), cache_dtype=cd, scale_mode=mode,
                                   batch=4, lens=[8192] * 4)
        w = inputs.from_spec(spec, device)
        s = w.spec
        sk = sv = None
        if mode == "per_head":
            sk = torch.empty(s.num_kv_heads, dtype=torch.float32, device=device)
            sv = torch.empty_like(sk)
            kvq.kvq_calibrate_head_scales(w.warmup_k, 448.0, sk)
            kvq.kvq_calibrate_head_scales(w.warmup_v, 448.0, sv)
        c = kvq.PagedKVCache(cd, s.act_dtype, mode, w.num_blocks, s.block_size, s.num_kv_heads,
                             s.head_dim, device=device, static_k_scale=sk, static_v_scale=sv)
        T = w.k.shape[0]

        def write():
            kvq.kvq_write(c.desc, w.k, w.v, w.slot_mapping)
        for _ in range(max(3, warmup)):
            l2.flush()
            write()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        torch.cuda.synchronize()
        for a, b in ev:
            l2.flush()
            a.record()
            write()
            b.record()
        torch.cuda.synchronize()
        ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
        nbytes = roofline.write_bytes(cd, mode, T, s.num_kv_heads, s.head_dim)
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[cd] = {"value": round(gbs, 2), "unit": "GB/s", "ms_per_call": round(ms, 5),
                   "frac": round(gbs / peak, 4), "peak_kind": kind, "rows": T,
                   "bytes_per_call": nbytes,
                   "cache": "%s %s" % (cd, mode)}
        del w, c
        torch.cuda.empty_cache()
    res["config"] = ("kvq_write of 4 x 8192 new tokens (K and V rows [32768, 8, 128] bf16) "
                     "into a paged cache, block 16; L2 emptied before each call")
    return res


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
    if args.prefill_only:
        r = measure_prefill(device, L2Flush(device), workload=args.workload,
                            steps=max(1, args.steps), batch=args.batch or 4)
        if rank == 0:
            print(json.dumps({"prefill": r, "note": "profiling run, not a benchmark line"}), flush=True)
        return
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
    step_ms = [ev[k][0].elapsed_time(ev[k][2]) for k in range(K)]
    dec_ms = [ev[k][1].elapsed_time(ev[k][2]) for k in range(K)]
    ms_sep = statistics.mean(step_ms) if K else 0.0
    dms = statistics.mean(dec_ms) if K else 0.0
    ms_sep, dms = max_over_ranks([ms_sep, dms], world, device)

    # the headline step: the same step as one call (kvq_append_decode_attention: the new
    # rows quantized and stored inside the decode call; for INT4 / INT2 they go to the ring,
    # as kvq_write puts a row that completes no block there), timed like the loop above
    def fused_step():
        kvq.kvq_append_decode_attention(cache.desc, new["k"], new["v"], w.q, w.block_tables,
                                        w.context_lens, max_ctx, out, ws)
    for _ in range(max(3, args.warmup)):
        l2.flush()
        fused_step()
    fev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for a, b2 in fev:
        l2.flush()
        a.record(stream)
        fused_step()
        b2.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms = statistics.mean(a.elapsed_time(b2) for a, b2 in fev) if K else 0.0
    ms, = max_over_ranks([ms], world, device)
    separate = None
    if K > 0:
        separate = {"value": round(throughput(step_bytes, world, ms_sep), 2), "unit": "GB/s",
                    "ms_per_step": round(ms_sep, 5), "tokens_per_s": round(world * B / (ms_sep * 1e-3), 1),
                    "call": "kvq_write, then kvq_decode_attention (two calls)"}

    # chunked prefill on its own cases (default workload only): the c5-shaped INT8 layer is
    # the headline; FP8, bf16 and INT4 caches of the same shapes beside it
    prefill = prefill_more = None
    if args.workload == "c5" and K > 0 and not args.batch:
        prefill = measure_prefill(device, l2)
        if world == 1:
            prefill_more = {key: measure_prefill(device, l2, workload=name)
                            for key, name in (("c5_fp8", "c5-fp8"), ("c5_bf16", "c5-bf16"), ("c4", "c4"))}

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
    fused_e2e = True                          # every cache form takes the one-call step
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
    e2e_serial = statistics.mean(e2e_ms) if e2e_ms else float("nan")

    # the same steps as a serving loop runs them: step k + 1's inputs go up on a copy stream
    # (into the second of two device buffers) while step k computes, and step k's output
    # comes back on another copy stream while step k + 1 computes.  Every copy is inside the
    # timed region (first input copy to last output copy, events on the copy streams); the
    # cache (hundreds of MB) is larger than L2, so the loop needs no flush between steps.
    e2e_pipe = float("nan")
    if E > 0:
        up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
        dbufs = [dbuf, torch.empty_like(dbuf)]
        views = []
        for bb in dbufs:
            vv = []
            for t, o in zip(parts, offs):
                n = t.numel() * t.element_size()
                vv.append(bb[o:o + n].view(t.dtype).view(t.shape))
            views.append(vv)
        outs = [out, torch.empty_like(out)]
        houts = [hout, torch.empty(out.shape, dtype=out.dtype).pin_memory()]
        copied = [torch.cuda.Event(), torch.cuda.Event()]
        computed = [torch.cuda.Event(), torch.cuda.Event()]
        drained = [torch.cuda.Event(), torch.cuda.Event()]

        def pipelined(nsteps, t0, t1):
            torch.cuda.synchronize()
            t0.record(up)
            for k in range(nsteps):
                i = k % 2
                if k >= 2:
                    up.wait_event(computed[i])          # step k - 2 has read this buffer
                with torch.cuda.stream(up):
                    dbufs[i].copy_(hbuf, non_blocking=True)
                copied[i].record(up)
                stream.wait_event(copied[i])
                if k >= 2:
                    stream.wait_event(drained[i])       # step k - 2's output is on the host
                qk, qv, qs, qq, ql = views[i]
                if fused_e2e:
                    kvq.kvq_append_decode_attention(cache.desc, qk, qv, qq, w.block_tables, ql, max_ctx,
                                                    outs[i], ws)
                else:
                    kvq.kvq_write(cache.desc, qk, qv, qs, new["seq_ids"], new["positions"])
                    kvq.kvq_decode_attention(cache.desc, qq, w.block_tables, ql, max_ctx, outs[i], ws)
                computed[i].record(stream)
                down.wait_event(computed[i])
                with torch.cuda.stream(down):
                    houts[i].copy_(outs[i], non_blocking=True)
                drained[i].record(down)
            up.wait_stream(down)
            t1.record(up)
            t1.synchronize()
            return t0.elapsed_time(t1) / nsteps
        pipelined(3, torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        e2e_pipe = pipelined(E, torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    e2e, e2e_serial = max_over_ranks([e2e_pipe, e2e_serial], world, device)

    # the other target configurations at full size, one GPU only (at N > 1 every rank would
    # have to take the same collective steps for them; the scaling run times the main step)
    configs = None
    write_prefill = None
    if world == 1 and K > 0 and args.workload == "c5" and not args.batch:
        configs = {key: measure_decode_call(name, device, l2, max(K, 20), args.warmup)
                   for key, name in SUB_WORKLOADS}
        write_prefill = measure_write_prefill(device, l2, max(K, 20), args.warmup)

    peak, peak_kind = hbm_peak()
    achieved = dec_bytes / (dms * 1e-3) / 1e9
    launches_per_step = cache.decode_plan(B, s.num_q_heads, max_ctx)[1]   # the append is inside
    result = {
        "metric": METRIC,
        "value": round(throughput(step_bytes, world, ms), 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "warmup_steps_run": warm,
        "ms_per_step": round(ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp32",
        "cache_dtype": s.cache_dtype,
        "data": "synthetic",
        "config": {"workload": "%s: %s; step = one kvq_append_decode_attention call: kvq_write of "
                               "%d new tokens + decode attention%s"
                               % (args.workload, WORKLOADS[args.workload], B,
                                  "" if not args.batch else
                                  " (batch reduced to %d for profiling: not a benchmark line)" % B),
                   "global_batch": B * world, "seq_len": max_ctx, "parallelism": "dp%d" % world,
                   "l2": L2Flush.DESCRIPTION,
                   "warmup": "at least the requested warm-up steps, and at least %.1f s under load "
                             "so the clocks reach their steady state (warmup_steps_run)"
                             % args.min_warmup_s},
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
                        ", one packed host-to-device copy of the step's inputs, output copied back",
                "schedule": "steps pipelined: step k+1's input copy and step k-1's output copy "
                            "overlap step k (two device buffers, two copy streams); no L2 flush "
                            "(the cache is larger than L2)",
                "serial": {"value": round(world * step_bytes / (e2e_serial * 1e-3) / 1e9, 2),
                           "ms_per_step": round(e2e_serial, 5),
                           "schedule": "one step at a time: L2 flush, input copy, call, output "
                                       "copy, host synchronize"}},
        "step_separate": separate,
        "prefill": prefill,
        "prefill_configs": prefill_more,
        "configs": configs,
        "write_prefill": write_prefill,
        "gpu_launches": launches_per_step * K,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = run_oracle_sample(args.workload)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def main_reference(args):
    """The oracle as the reference arm: every host core runs one (sequence, kv head) unit
    step per round (see OraclePool); a step of this arm is one round."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    pool = OraclePool(args.workload)
    try:
        for _ in range(max(1, args.warmup)):
            pool.round()
        times = [pool.round() for _ in range(args.steps)]
    finally:
        pool.close()
    sec = statistics.mean(times)
    value = pool.bytes_per_round() / sec / 1e9
    sample = ("one step of a (sequence, kv head) unit (%d cached tokens, %d query heads; quantize "
              "the new row + float64 attention over every cached position) on each of %d worker "
              "processes, one per host core, one thread each" % (pool.case["n"], pool.case["g"],
                                                                  pool.workers))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sec * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "%s: %s; step = %d (sequence, kv head) units of the serving step, "
                               "one per host core" % (args.workload, WORKLOADS[args.workload],
                                                      pool.workers)},
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": pool.workers,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        main_reference(a)
    else:
        main_ours(a)
