"""Python binding of the kvq C ABI (include/kvq.h): argument marshalling only.

Every call goes through ctypes into libkvq.so; no step of the cache or of attention runs
in Python.  Device memory comes from torch and work is enqueued on torch's current
stream (or the stream given).  If the library is missing, importing this module fails.

The functions keep the C names (kvq_write, kvq_decode_attention, kvq_dequant, ...).
``PagedKVCache`` is a convenience holder: it asks the library for the pool sizes,
allocates them with torch and fills a ``CacheDesc``.
"""

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvq.so")

DTYPE = {"bf16": 0, "fp16": 1, "fp32": 2, "int8": 3, "fp8": 4, "int4": 5, "int2": 6}
SCALE = {"none": 0, "per_token_head": 1, "per_head": 2, "per_tensor": 3, "kivi": 4,
         "per_channel": 5, "int4_per_token": 6, "kivi_float_zero": 7}
STATUS = {0: "KVQ_OK", 1: "KVQ_ERR_INVALID_ARG", 2: "KVQ_ERR_UNSUPPORTED", 3: "KVQ_ERR_CUDA",
          4: "KVQ_ERR_DEVICE_FAULT"}
FAULT_BITS = {"slot": 1, "block": 2, "context": 4, "seq": 8, "int4_run": 16, "timeout": 32}
EXPORTS = ("kvq_status_string", "kvq_version", "kvq_cache_layout", "kvq_write",
           "kvq_decode_workspace_size", "kvq_decode_attention", "kvq_dequant",
           "kvq_calibrate_fp8_scales", "kvq_read_device_fault", "kvq_decode_attention_noalloc",
           "kvq_append_decode_attention", "kvq_calibrate_channel_scales", "kvq_flush_ring",
           "kvq_prefill_attention", "kvq_decode_plan", "kvq_calibrate_head_scales")


class CacheDesc(ctypes.Structure):
    _fields_ = [("cache_dtype", ctypes.c_int32), ("act_dtype", ctypes.c_int32),
                ("scale_mode", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("group_size", ctypes.c_int32),
                ("residual_len", ctypes.c_int32), ("residual_cap", ctypes.c_int32),
                ("max_seqs", ctypes.c_int32), ("reserved0", ctypes.c_int32),
                ("pages", ctypes.c_void_p), ("k_scales", ctypes.c_void_p),
                ("v_scales", ctypes.c_void_p), ("residual", ctypes.c_void_p),
                ("fault", ctypes.c_void_p)]


class KVQError(RuntimeError):
    def __init__(self, status, what):
        super().__init__("%s failed: %s" % (what, STATUS.get(status, status)))
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("kvq CUDA library not built (%s missing); run "
                          "`python -m quantized_paged_kv_02_b200.build`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    D = ctypes.POINTER(CacheDesc)
    sig = {
        "kvq_status_string": (ctypes.c_char_p, [I]),
        "kvq_version": (I, []),
        "kvq_cache_layout": (I, [D, ctypes.POINTER(Z), ctypes.POINTER(Z), ctypes.POINTER(Z),
                                 ctypes.POINTER(Z)]),
        "kvq_write": (I, [D, P, P, I, P, P, P, P]),
        "kvq_decode_workspace_size": (I, [D, I, I, I, ctypes.POINTER(Z)]),
        "kvq_decode_plan": (I, [D, I, I, I, ctypes.POINTER(I), ctypes.POINTER(I), ctypes.POINTER(I)]),
        "kvq_decode_attention": (I, [D, P, I, I, P, I, P, P, I, F, P, ctypes.c_int32, P, Z, P]),
        "kvq_dequant": (I, [D, P, I, P, P]),
        "kvq_calibrate_fp8_scales": (I, [P, I, I, I, ctypes.c_int32, P, P]),
        "kvq_read_device_fault": (I, [D, ctypes.POINTER(ctypes.c_int32), I, P]),
        "kvq_decode_attention_noalloc": (I, [D, P, I, I, P, I, P, P, I, F, P, ctypes.c_int32, P]),
        "kvq_append_decode_attention": (I, [D, P, P, P, I, I, P, I, P, I, F, P, ctypes.c_int32, P,
                                            Z, P]),
        "kvq_calibrate_channel_scales": (I, [P, I, I, I, ctypes.c_int32, F, P, P]),
        "kvq_calibrate_head_scales": (I, [P, I, I, I, ctypes.c_int32, F, P, P]),
        "kvq_flush_ring": (I, [D, P, P, P, I, P]),
        "kvq_prefill_attention": (I, [D, P, I, I, I, P, I, P, I, P, I, F, P, ctypes.c_int32, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(st, what):
    if st != 0:
        raise KVQError(st, what)


def _act(t):
    if t.dtype == torch.bfloat16:
        return "bf16"
    if t.dtype == torch.float16:
        return "fp16"
    raise TypeError("activations must be bfloat16 or float16, got %s" % t.dtype)


def _i32(t):
    if t is None:
        return None
    if t.dtype != torch.int32 or not t.is_contiguous():
        raise TypeError("index tensors must be contiguous int32")
    return t


# ----------------------------------------------------------------------------- C names
def kvq_status_string(status):
    return lib.kvq_status_string(status).decode()


def kvq_version():
    return lib.kvq_version()


def kvq_cache_layout(desc):
    """(record bytes, pages pool bytes, static scale bytes, residual bytes)."""
    sizes = [ctypes.c_size_t(0) for _ in range(4)]
    _check(lib.kvq_cache_layout(ctypes.byref(desc), *[ctypes.byref(s) for s in sizes]),
           "kvq_cache_layout")
    return tuple(s.value for s in sizes)


def kvq_write(desc, k_new, v_new, slot_mapping, seq_ids=None, positions=None, stream=None):
    _check(lib.kvq_write(ctypes.byref(desc), _ptr(k_new), _ptr(v_new), int(k_new.shape[0]),
                         _ptr(_i32(slot_mapping)), _ptr(_i32(seq_ids)), _ptr(_i32(positions)),
                         _stream(stream)), "kvq_write")


def kvq_decode_workspace_size(desc, batch, num_q_heads, max_context):
    n = ctypes.c_size_t(0)
    _check(lib.kvq_decode_workspace_size(ctypes.byref(desc), batch, num_q_heads, max_context,
                                         ctypes.byref(n)), "kvq_decode_workspace_size")
    return n.value


def kvq_decode_plan(desc, batch, num_q_heads, max_context):
    """(kernel, launches per call, splits or CTAs) of kvq_decode_attention for this shape."""
    k, n, s = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(lib.kvq_decode_plan(ctypes.byref(desc), batch, num_q_heads, max_context,
                               ctypes.byref(k), ctypes.byref(n), ctypes.byref(s)), "kvq_decode_plan")
    return k.value, n.value, s.value


def kvq_decode_attention(desc, q, block_tables, context_lens, max_context, out, workspace=None,
                         seq_ids=None, softmax_scale=0.0, stream=None):
    B, Hq, _ = q.shape
    out_dt = {torch.bfloat16: "bf16", torch.float16: "fp16", torch.float32: "fp32"}[out.dtype]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.kvq_decode_attention(
        ctypes.byref(desc), _ptr(q), B, Hq, _ptr(_i32(block_tables)), int(block_tables.shape[1]),
        _ptr(_i32(context_lens)), _ptr(_i32(seq_ids)), int(max_context), float(softmax_scale),
        _ptr(out), DTYPE[out_dt], _ptr(workspace), ws_bytes, _stream(stream)),
        "kvq_decode_attention")
    return out


def kvq_append_decode_attention(desc, k_new, v_new, q, block_tables, context_lens, max_context,
                                out, workspace=None, softmax_scale=0.0, stream=None):
    """Store each sequence's new K/V row at position context_lens[b] - 1, then decode:
    kvq_write followed by kvq_decode_attention in one launch (dense caches)."""
    B, Hq, _ = q.shape
    out_dt = {torch.bfloat16: "bf16", torch.float16: "fp16", torch.float32: "fp32"}[out.dtype]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.kvq_append_decode_attention(
        ctypes.byref(desc), _ptr(k_new), _ptr(v_new), _ptr(q), B, Hq, _ptr(_i32(block_tables)),
        int(block_tables.shape[1]), _ptr(_i32(context_lens)), int(max_context),
        float(softmax_scale), _ptr(out), DTYPE[out_dt], _ptr(workspace), ws_bytes,
        _stream(stream)), "kvq_append_decode_attention")
    return out


def kvq_decode_attention_noalloc(desc, q, block_tables, context_lens, max_context, out,
                                 seq_ids=None, softmax_scale=0.0, stream=None):
    """kvq_decode_attention with the library's own fixed device scratch instead of a
    caller workspace (for callers that cannot allocate device memory when they decode)."""
    B, Hq, _ = q.shape
    out_dt = {torch.bfloat16: "bf16", torch.float16: "fp16", torch.float32: "fp32"}[out.dtype]
    _check(lib.kvq_decode_attention_noalloc(
        ctypes.byref(desc), _ptr(q), B, Hq, _ptr(_i32(block_tables)), int(block_tables.shape[1]),
        _ptr(_i32(context_lens)), _ptr(_i32(seq_ids)), int(max_context), float(softmax_scale),
        _ptr(out), DTYPE[out_dt], _stream(stream)), "kvq_decode_attention_noalloc")
    return out


def kvq_dequant(desc, block_ids, out, stream=None):
    _check(lib.kvq_dequant(ctypes.byref(desc), _ptr(_i32(block_ids)), int(block_ids.numel()),
                           _ptr(out), _stream(stream)), "kvq_dequant")
    return out


def kvq_calibrate_fp8_scales(x, scale_out, stream=None):
    T, H, D = x.shape
    _check(lib.kvq_calibrate_fp8_scales(_ptr(x), T, H, D, DTYPE[_act(x)], _ptr(scale_out),
                                        _stream(stream)), "kvq_calibrate_fp8_scales")
    return scale_out


def kvq_prefill_attention(desc, q, q_start, max_q_len, block_tables, context_lens, max_context,
                          out, softmax_scale=0.0, stream=None):
    """Causal attention of each sequence's chunk of new queries (rows q_start[b] ..
    q_start[b+1]-1 of q) over the cache."""
    Tq, Hq, _ = q.shape
    B = int(q_start.numel()) - 1
    out_dt = {torch.bfloat16: "bf16", torch.float16: "fp16", torch.float32: "fp32"}[out.dtype]
    _check(lib.kvq_prefill_attention(
        ctypes.byref(desc), _ptr(q), Tq, B, Hq, _ptr(_i32(q_start)), int(max_q_len),
        _ptr(_i32(block_tables)), int(block_tables.shape[1]), _ptr(_i32(context_lens)),
        int(max_context), float(softmax_scale), _ptr(out), DTYPE[out_dt], _stream(stream)),
        "kvq_prefill_attention")
    return out


def kvq_flush_ring(desc, seq_ids, positions, block_ids, stream=None):
    """INT4: quantize ring rows [positions[i], positions[i] + 64) of sequence seq_ids[i]
    into block block_ids[i] (all kv heads)."""
    n = int(seq_ids.numel())
    _check(lib.kvq_flush_ring(ctypes.byref(desc), _ptr(_i32(seq_ids)), _ptr(_i32(positions)),
                              _ptr(_i32(block_ids)), n, _stream(stream)), "kvq_flush_ring")


def kvq_calibrate_head_scales(x, qmax, scale_out, stream=None):
    """scale_out[h] = max over tokens and channels |x[t][h][:]| / qmax (127 INT8, 448 FP8)."""
    T, H, D = x.shape
    _check(lib.kvq_calibrate_head_scales(_ptr(x), T, H, D, DTYPE[_act(x)], float(qmax),
                                         _ptr(scale_out), _stream(stream)),
           "kvq_calibrate_head_scales")
    return scale_out


def kvq_calibrate_channel_scales(x, qmax, scale_out, stream=None):
    """scale_out[h][d] = max over tokens |x[t][h][d]| / qmax (127 INT8, 448 FP8)."""
    T, H, D = x.shape
    _check(lib.kvq_calibrate_channel_scales(_ptr(x), T, H, D, DTYPE[_act(x)], float(qmax),
                                            _ptr(scale_out), _stream(stream)),
           "kvq_calibrate_channel_scales")
    return scale_out


def kvq_read_device_fault(desc, reset=True, stream=None):
    out = (ctypes.c_int32 * 2)()
    st = lib.kvq_read_device_fault(ctypes.byref(desc), out, 1 if reset else 0, _stream(stream))
    if st not in (0, 4):
        _check(st, "kvq_read_device_fault")
    return int(out[0]), int(out[1])


# ----------------------------------------------------------------------------- holder
class PagedKVCache:
    """One layer's cache, allocated with torch in the layout of include/kvq.h: the page
    records pool, the static scale arrays (PER_HEAD / PER_TENSOR) and the INT4 ring."""

    def __init__(self, cache_dtype, act_dtype, scale_mode, num_blocks, block_size, num_kv_heads,
                 head_dim, device="cuda", group_size=64, residual_len=128, residual_cap=192,
                 max_seqs=0, static_k_scale=None, static_v_scale=None, fill=0x5A, fault=True):
        self.desc = CacheDesc()
        d = self.desc
        d.cache_dtype, d.act_dtype, d.scale_mode = DTYPE[cache_dtype], DTYPE[act_dtype], SCALE[scale_mode]
        d.num_blocks, d.block_size, d.num_kv_heads, d.head_dim = num_blocks, block_size, num_kv_heads, head_dim
        d.group_size, d.residual_len, d.residual_cap = group_size, residual_len, residual_cap
        d.max_seqs = max_seqs
        self.cache_dtype, self.act_dtype, self.scale_mode = cache_dtype, act_dtype, scale_mode
        self.num_blocks, self.block_size = num_blocks, block_size
        self.num_kv_heads, self.head_dim = num_kv_heads, head_dim
        self.device = torch.device(device)
        self.record, pages_b, ss_b, res_b = kvq_cache_layout(d)
        self.pages = torch.full((pages_b,), fill, dtype=torch.uint8, device=self.device)
        self.k_scales = self.v_scales = self.residual = None
        if ss_b:
            n = ss_b // 4
            self.k_scales = torch.zeros(max(n, 4), dtype=torch.float32, device=self.device)
            self.v_scales = torch.zeros(max(n, 4), dtype=torch.float32, device=self.device)
            if static_k_scale is not None:
                self.k_scales[:n].copy_(static_k_scale.reshape(n).to(torch.float32))
            if static_v_scale is not None:
                self.v_scales[:n].copy_(static_v_scale.reshape(n).to(torch.float32))
        if res_b:
            self.residual = torch.full((res_b,), fill, dtype=torch.uint8, device=self.device)
        self.fault = torch.zeros(4, dtype=torch.int32, device=self.device) if fault else None
        d.pages = self.pages.data_ptr()
        d.k_scales = self.k_scales.data_ptr() if self.k_scales is not None else None
        d.v_scales = self.v_scales.data_ptr() if self.v_scales is not None else None
        d.residual = self.residual.data_ptr() if self.residual is not None else None
        d.fault = self.fault.data_ptr() if self.fault is not None else None
        self.sizes = (self.record, pages_b, ss_b, res_b)

    def records(self):
        """The pages pool as [NB][H][record] bytes."""
        return self.pages.view(self.num_blocks, self.num_kv_heads, self.record)

    def write(self, k_new, v_new, slot_mapping, seq_ids=None, positions=None, stream=None):
        kvq_write(self.desc, k_new, v_new, slot_mapping, seq_ids, positions, stream)

    def workspace_size(self, batch, num_q_heads, max_context):
        return kvq_decode_workspace_size(self.desc, batch, num_q_heads, max_context)

    def decode_plan(self, batch, num_q_heads, max_context):
        return kvq_decode_plan(self.desc, batch, num_q_heads, max_context)

    def decode(self, q, block_tables, context_lens, max_context, out=None, out_dtype=torch.float32,
               workspace=None, seq_ids=None, softmax_scale=0.0, stream=None):
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        if workspace is None:
            n = self.workspace_size(q.shape[0], q.shape[1], max_context)
            workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device) if n else None
        return kvq_decode_attention(self.desc, q, block_tables, context_lens, max_context, out,
                                    workspace, seq_ids, softmax_scale, stream)

    def append_decode(self, k_new, v_new, q, block_tables, context_lens, max_context, out=None,
                      out_dtype=torch.float32, workspace=None, softmax_scale=0.0, stream=None):
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        if workspace is None:
            n = self.workspace_size(q.shape[0], q.shape[1], max_context)
            workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device) if n else None
        return kvq_append_decode_attention(self.desc, k_new, v_new, q, block_tables, context_lens,
                                           max_context, out, workspace, softmax_scale, stream)

    def prefill(self, q, q_start, max_q_len, block_tables, context_lens, max_context, out=None,
                out_dtype=torch.float32, softmax_scale=0.0, stream=None):
        if out is None:
            out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
        return kvq_prefill_attention(self.desc, q, q_start, max_q_len, block_tables, context_lens,
                                     max_context, out, softmax_scale, stream)

    def flush_ring(self, seq_ids, positions, block_ids, stream=None):
        kvq_flush_ring(self.desc, seq_ids, positions, block_ids, stream)

    def dequant(self, block_ids, stream=None):
        out = torch.empty((block_ids.numel(), 2, self.num_kv_heads, self.block_size, self.head_dim),
                          dtype=torch.float32, device=self.device)
        return kvq_dequant(self.desc, block_ids, out, stream)

    def read_fault(self, reset=True):
        return kvq_read_device_fault(self.desc, reset)
