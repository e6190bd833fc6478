"""CPU checks of the C-ABI library: it loads, exports every declared symbol, computes
layouts and workspace sizes on the host, and rejects bad arguments before launching."""

import ctypes
import os
import re

import pytest

from tests.helpers import ROOT, ensure_built

HEADER = os.path.join(ROOT, "include", "kvq.h")


@pytest.fixture(scope="module")
def lib():
    path = ensure_built()
    return ctypes.CDLL(path)


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert len(syms) >= 9
    for s in syms:
        assert hasattr(lib, s), s


def test_binding_names_match_header():
    from quantized_paged_kv_02_b200 import kvq
    assert sorted(kvq.EXPORTS) == declared_symbols()


def test_missing_library_fails_loudly(monkeypatch):
    from quantized_paged_kv_02_b200 import kvq
    monkeypatch.setattr(kvq, "LIB_PATH", "/nonexistent/libkvq.so")
    with pytest.raises(ImportError):
        kvq._load()


def _desc(kvq, **kw):
    d = kvq.CacheDesc()
    base = dict(cache_dtype=3, act_dtype=0, scale_mode=1, num_blocks=16, block_size=16,
                num_kv_heads=4, head_dim=128, group_size=64, residual_len=128, residual_cap=192,
                max_seqs=2)
    base.update(kw)
    for k, v in base.items():
        setattr(d, k, v)
    return d


def test_layout_sizes(lib):
    """Record = K codes + V codes + per-token scales (or KIVI parameters), padded to 128."""
    from quantized_paged_kv_02_b200 import kvq
    # INT8 per token, bs 16, D 128: 2048 + 2048 + 128
    assert kvq.kvq_cache_layout(_desc(kvq)) == (4224, 16 * 4 * 4224, 0, 0)
    assert kvq.kvq_cache_layout(_desc(kvq, cache_dtype=4, scale_mode=2)) == (4096, 16 * 4 * 4096, 16, 0)
    assert kvq.kvq_cache_layout(_desc(kvq, cache_dtype=4, scale_mode=3)) == (4096, 16 * 4 * 4096, 4, 0)
    assert kvq.kvq_cache_layout(_desc(kvq, cache_dtype=0, scale_mode=0)) == (8192, 16 * 4 * 8192, 0, 0)
    # INT4 KIVI, bs 64: 4096 + 4096 + (512 K scale/zero + 512 V scale/zero)
    rec, pg, ss, r = kvq.kvq_cache_layout(_desc(kvq, cache_dtype=5, scale_mode=4, block_size=64))
    assert rec == 9216 and pg == 16 * 4 * 9216 and ss == 0
    assert r == 2 * 2 * 4 * 192 * 128 * 2
    # D 64, bs 16: 1024 + 1024 + 128, already a multiple of 128
    assert kvq.kvq_cache_layout(_desc(kvq, head_dim=64))[0] == 2176
    # bs 5: 640 + 640 + 40 -> 1408 after padding
    assert kvq.kvq_cache_layout(_desc(kvq, block_size=5))[0] == 1408
    with pytest.raises(kvq.KVQError):
        kvq.kvq_cache_layout(_desc(kvq, cache_dtype=5, scale_mode=4, block_size=16))
    # the per-token and float-zero-point INT4 forms keep the record size
    for mode in (6, 7):
        assert kvq.kvq_cache_layout(_desc(kvq, cache_dtype=5, scale_mode=mode, block_size=64))[0] == 9216
    # INT2, bs 64: 2048 + 2048 + 1024, every INT4 form; the ring as INT4
    for mode in (4, 6, 7):
        rec, pg, ss, r = kvq.kvq_cache_layout(_desc(kvq, cache_dtype=6, scale_mode=mode, block_size=64))
        assert (rec, pg, ss, r) == (5120, 16 * 4 * 5120, 0, 2 * 2 * 4 * 192 * 128 * 2)
    # low-bit caches take only the group forms; dense caches not those
    for cd, mode in ((6, 1), (5, 2), (3, 4), (4, 6), (3, 7)):
        with pytest.raises(kvq.KVQError):
            kvq.kvq_cache_layout(_desc(kvq, cache_dtype=cd, scale_mode=mode, block_size=64))


def test_workspace_plan_is_deterministic(lib):
    from quantized_paged_kv_02_b200 import kvq
    d = _desc(kvq, num_kv_heads=8)
    a = kvq.kvq_decode_workspace_size(d, 24, 64, 16384)
    assert a == kvq.kvq_decode_workspace_size(d, 24, 64, 16384) and a > 0
    # the CUDA-core kernel (head_dim 64) with a single split writes the output directly
    assert kvq.kvq_decode_workspace_size(_desc(kvq, num_kv_heads=8, head_dim=64), 1, 8, 16) == 0
    # the tensor-core kernel always merges per-warp partials through the workspace:
    # (units + CTAs - 1) * 4 partials of g heads, each D floats plus (max, sum); 3 CTAs per
    # SM (148 SMs when no device can be queried)
    ctas, D, g, units = 3 * 148, 128, 1, 8
    heads = (units + ctas - 1) * 4 * g
    assert kvq.kvq_decode_workspace_size(d, 1, 8, 16) == (heads * D * 4 + 255) // 256 * 256 + heads * 8
    with pytest.raises(kvq.KVQError):
        kvq.kvq_decode_workspace_size(d, 2, 12, 100)              # 12 not a multiple of 8


def test_decode_plan_names_the_dispatch(lib):
    """kvq_decode_plan (host only) reports the kernel and launch count of a decode call."""
    from quantized_paged_kv_02_b200 import kvq
    d = _desc(kvq, num_kv_heads=8)
    assert kvq.kvq_decode_plan(d, 24, 64, 16384) == (1, 2, 3 * 148)       # tensor cores + merge
    assert kvq.kvq_decode_plan(d, 4, 8, 2048)[:2] == (1, 2)               # MHA too (g = 1)
    assert kvq.kvq_decode_plan(d, 0, 64, 16384)[1] == 0                  # empty batch
    lo = dict(cache_dtype=5, scale_mode=4, block_size=64, num_kv_heads=8)
    k, n, s = kvq.kvq_decode_plan(_desc(kvq, **lo), 16, 64, 32768)
    assert (k, n) == (2, 3) and s >= 2                                  # blocks, ring, reduce
    assert kvq.kvq_decode_plan(_desc(kvq, **dict(lo, cache_dtype=6)), 16, 64, 32768)[:2] == (2, 3)
    assert kvq.kvq_decode_plan(_desc(kvq, **lo), 16, 16, 32768)[0] == 0   # g = 2: CUDA cores
    # CUDA-core kernel: one split writes the output (one launch), more add the reduce
    d64 = _desc(kvq, num_kv_heads=8, head_dim=64)
    assert kvq.kvq_decode_plan(d64, 1, 8, 16)[:2] == (0, 1)
    assert kvq.kvq_decode_plan(d64, 1, 8, 16384)[:2] == (0, 2)
    with pytest.raises(kvq.KVQError):
        kvq.kvq_decode_plan(d, 2, 12, 100)


def test_invalid_arguments_rejected_before_launch(lib):
    from quantized_paged_kv_02_b200 import kvq
    L = kvq.lib
    d = _desc(kvq)                 # null pools
    null = ctypes.c_void_p(0)
    assert L.kvq_write(ctypes.byref(d), null, null, 4, null, null, null, null) == 1
    assert L.kvq_write(None, null, null, 4, null, null, null, null) == 1
    fake = ctypes.c_void_p(0x1000)
    d2 = _desc(kvq)
    d2.pages = 0x1000
    assert L.kvq_write(ctypes.byref(d2), null, null, 4, null, null, null, null) == 1
    assert L.kvq_write(ctypes.byref(d2), fake, fake, -1, fake, null, null, null) == 1
    assert L.kvq_write(ctypes.byref(d2), fake, fake, 0, fake, null, null, null) == 0   # no work
    d3 = _desc(kvq, head_dim=96)
    d3.pages = 0x1000
    assert L.kvq_write(ctypes.byref(d3), fake, fake, 1, fake, null, null, null) == 2   # unsupported
    # decode: bad head count, bad out dtype, missing workspace
    assert L.kvq_decode_attention(ctypes.byref(d2), fake, 2, 6, fake, 4, fake, null, 64, 0.0,
                                  fake, 2, null, 0, null) == 1
    assert L.kvq_decode_attention(ctypes.byref(d2), fake, 2, 8, fake, 4, fake, null, 64, 0.0,
                                  fake, 7, null, 0, null) == 1
    assert L.kvq_decode_attention(ctypes.byref(d2), fake, 24, 32, fake, 1024, fake, null, 16384,
                                  0.0, fake, 2, null, 0, null) == 1
    assert L.kvq_decode_attention(ctypes.byref(d2), fake, 2, 8, fake, 4, fake, null, 64,
                                  ctypes.c_float(float("nan")), fake, 2, null, 0, null) == 1
    # misaligned pool
    d4 = _desc(kvq)
    d4.pages = 0x1001
    assert L.kvq_write(ctypes.byref(d4), fake, fake, 1, fake, null, null, null) == 1
    # mixed passthrough (bf16 cache, fp16 activations) is unsupported
    d5 = _desc(kvq, cache_dtype=0, act_dtype=1, scale_mode=0)
    d5.pages = 0x1000
    # static scales are required for per-head modes
    d6 = _desc(kvq, cache_dtype=4, scale_mode=2)
    d6.pages = 0x1000
    assert L.kvq_write(ctypes.byref(d6), fake, fake, 1, fake, null, null, null) == 1
    assert L.kvq_write(ctypes.byref(d5), fake, fake, 1, fake, null, null, null) == 2
    assert kvq.kvq_status_string(2) == "KVQ_ERR_UNSUPPORTED"


def test_noalloc_rejects_shapes_beyond_its_scratch(lib):
    """The scratch-free decode refuses, on the host and before any device call, a shape whose
    split partials would not fit its fixed 16 MiB array; an empty batch does nothing."""
    from quantized_paged_kv_02_b200 import kvq
    L = kvq.lib
    d = _desc(kvq)
    d.pages = 0x1000
    fake = ctypes.c_void_p(0x1000)
    null = ctypes.c_void_p(0)
    need = kvq.kvq_decode_workspace_size(d, 10000, 32, 16384)
    assert need > 16 << 20
    assert L.kvq_decode_attention_noalloc(ctypes.byref(d), fake, 10000, 32, fake, 1024, fake, null,
                                          16384, 0.0, fake, 2, null) == 1
    assert L.kvq_decode_attention_noalloc(ctypes.byref(d), fake, 0, 32, fake, 1024, fake, null,
                                          16384, 0.0, fake, 2, null) == 0


def test_head_calibration_rejects_bad_arguments(lib):
    from quantized_paged_kv_02_b200 import kvq
    L = kvq.lib
    fake = ctypes.c_void_p(0x1000)
    null = ctypes.c_void_p(0)
    assert L.kvq_calibrate_head_scales(fake, 4, 2, 128, 0, ctypes.c_float(0.0), fake, null) == 1
    assert L.kvq_calibrate_head_scales(fake, 4, 2, 128, 3, ctypes.c_float(127.0), fake, null) == 1
    assert L.kvq_calibrate_head_scales(fake, 4, 2, 128, 0, ctypes.c_float(127.0), null, null) == 1
