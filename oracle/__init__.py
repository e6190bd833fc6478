"""Plain CPU oracle of the quantized paged KV cache and its decode attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this package: only
the tests, the smoke check in ``__graft_entry__`` and the CPU-baseline leg of
``bench.py`` use it.  It shares no code with the CUDA library (no kernels, headers,
tables or helpers); both sides implement the layout and quantizer definitions written
in ``include/kvq.h`` on their own.

Sources (titles of the web pages that describe the method):
  [P-vLLM] "KV Cache量化压缩技术与vLLM推理引擎显存优化实战" (yunthe.com)
  [P-prod] "KV Cache Quantization 生产实战：用低精度缓存降低长上下文推理显存" (oh-bug.com)
  [P-mem]  "大模型KV Cache显存优化与量化技术实践" (intelliparadigm.com)

Modules
  fp         - binary32 / binary16 / E4M3 rounding steps written from their definitions.
  quant      - INT8, FP8 E4M3 and INT4 (KIVI) quantizers and dequantizers.
  cache      - the paged cache: byte-exact pools, scatter on write, gather on read.
  attention  - single-token decode attention over the dequantized cache, float64.
  bytes_model- the KV-cache size formula and the per-step byte count.

Every function is pinned by a ``-m "not gpu"`` test against something other than
itself (worked examples printed on the pages, exact rational arithmetic, brute force,
closed forms, library routines in special cases); see tests/test_oracle_*.py.
"""

from . import fp, quant, cache, attention, bytes_model  # noqa: F401
