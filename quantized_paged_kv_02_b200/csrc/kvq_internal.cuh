// Internal declarations shared by the kvq CUDA sources (not part of the public ABI).
//
// Sources cited in these files (titles of the web pages that describe the method):
//   [P-vLLM] "KV Cache量化压缩技术与vLLM推理引擎显存优化实战" (yunthe.com)
//   [P-prod] "KV Cache Quantization 生产实战：用低精度缓存降低长上下文推理显存" (oh-bug.com)
//   [P-mem]  "大模型KV Cache显存优化与量化技术实践" (intelliparadigm.com)
#pragma once

#include <type_traits>

#include <utility>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------ fault record
// fault[0] counts skipped entries, fault[1] accumulates KVQ_FAULT_* bits.
__device__ __forceinline__ void record_fault(int32_t* fault, int bits) {
  if (fault != nullptr) {
    atomicAdd(&fault[0], 1);
    atomicOr(&fault[1], bits);
  }
}

// ------------------------------------------------------------------ activations
template <typename T> struct Act;
template <> struct Act<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
};
template <> struct Act<__half> {
  static __device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
};

// Eight 16-bit activation values packed in a uint4 -> float (bf16: the bits placed in the
// upper half of a binary32, exact; fp16: the paired conversion).
template <typename T>
__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    } else {
      const float2 p = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      f[2 * i] = p.x;
      f[2 * i + 1] = p.y;
    }
  }
}

__device__ __forceinline__ float e4m3_to_float(uint8_t c) {
  __nv_fp8_e4m3 v;
  v.__x = c;
  return static_cast<float>(v);
}

// Binary32 quotient with round-to-nearest-even, independent of -prec-div.
__device__ __forceinline__ float div_rn(float a, float b) { return __fdiv_rn(a, b); }

// ------------------------------------------------------------------ dense quantizers
// (kvq_write, and the append step of kvq_append_decode_attention: one definition, so the
// two store identical bytes)
template <int CD> struct QMax;
template <> struct QMax<KVQ_DTYPE_INT8> { static constexpr float v = 127.f; };
template <> struct QMax<KVQ_DTYPE_FP8_E4M3> { static constexpr float v = 448.f; };

__device__ __forceinline__ uint8_t quant_int8(float x, float s) {
  if (s == 0.f) return 0;
  int q = __float2int_rn(div_rn(x, s));
  q = max(-128, min(127, q));
  return static_cast<uint8_t>(static_cast<int8_t>(q));
}

__device__ __forceinline__ uint8_t quant_fp8(float x, float s) {
  if (s == 0.f) return 0;
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(div_rn(x, s), __NV_SATFINITE, __NV_E4M3));
}

// Codes of 8 values against one scale s > 0, equal to those of quant_int8 / quant_fp8 (the
// quotient x / s rounded to float32 first).  The quotient is formed without a division by
// Markstein's correction step (P. Markstein, IBM J. Res. Dev. 34(1), 1990): if r = RN(1/s)
// and q is within one ulp of x / s, the remainder x - q s is exact as one FMA and
// RN(q + (x - q s) r) is the correctly rounded quotient, as long as nothing overflows or
// underflows.  q0 = RN(x r) can be up to 1.5 ulp away, so one first step
// q1 = RN(q0 + RN(x - q0 s) r) (error far below one ulp) precedes the exact one.  Quotients
// below 2^-126 in magnitude round to a zero code of the right sign either way.  INT8 then rounds to an integer by adding
// 1.5 * 2^23 (round to nearest even); E4M3 converts with satfinite.  A lane with a quotient
// or reciprocal that is not finite, or a scale below 2^-100, divides instead.  `bounded`:
// |x| is at most 127 s, as for per-token scales taken from the row's own maximum; otherwise
// the quotient is clamped to [-129, 129] before rounding and the code to [-128, 127] after.
__device__ __forceinline__ uint32_t pack4_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040u), __byte_perm(c, d, 0x0040u), 0x5410u);
}

template <int CD>
__device__ __forceinline__ uint2 quant8_same_scale(const float* x, float s, float r, bool bounded) {
  bool hard = !(r <= 3.0e38f) || !(s >= 7.9e-31f);
  uint32_t w0, w1;
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 xv = make_float2(x[i], x[i + 1]);
    const float2 q0 = __fmul2_rn(xv, make_float2(r, r));
    const float2 q1 = __ffma2_rn(__ffma2_rn(q0, make_float2(-s, -s), xv), make_float2(r, r), q0);
    const float2 e = __ffma2_rn(q1, make_float2(-s, -s), xv);          // exact remainder
    float2 q = __ffma2_rn(e, make_float2(r, r), q1);                    // fl(x / s)
    hard = hard || !(fabsf(q.x) <= 3.0e38f) || !(fabsf(q.y) <= 3.0e38f);
    if constexpr (CD == KVQ_DTYPE_INT8) {
      constexpr float kShift = 12582912.f;                               // 1.5 * 2^23
      if (!bounded) q = make_float2(fminf(fmaxf(q.x, -129.f), 129.f), fminf(fmaxf(q.y, -129.f), 129.f));
      const float2 t = __fadd2_rn(q, make_float2(kShift, kShift));
      b[i] = __float_as_uint(t.x) - 0x4B400000u;
      b[i + 1] = __float_as_uint(t.y) - 0x4B400000u;
    } else {
      uint32_t c;
      asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tcvt.u32.u16 %0, t;\n\t}"
          : "=r"(c) : "f"(q.y), "f"(q.x));
      b[i] = c & 0xFFu;
      b[i + 1] = c >> 8;
    }
  }
  if constexpr (CD == KVQ_DTYPE_INT8) {
    if (!bounded) {
#pragma unroll
      for (int i = 0; i < 8; ++i) b[i] = static_cast<uint32_t>(max(-128, min(127, static_cast<int>(b[i]))));
    }
  }
  w0 = pack4_low_bytes(b[0], b[1], b[2], b[3]);
  w1 = pack4_low_bytes(b[4], b[5], b[6], b[7]);
  if (hard) {
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = (CD == KVQ_DTYPE_INT8) ? quant_int8(x[i], s) : quant_fp8(x[i], s);
    w0 = pack4_low_bytes(c[0], c[1], c[2], c[3]);
    w1 = pack4_low_bytes(c[4], c[5], c[6], c[7]);
  }
  return make_uint2(w0, w1);
}

// One lane's share of quantizing one row (one token, one kv head, K or V) into its page
// record.  A row is handled by D / (8 NV) consecutive lanes (a power of two dividing 32);
// lane l holds activation elements [8 NV l, 8 NV l + 8 NV) in u[0..NV).  `write` false: the
// lane joins the shuffles but stores nothing.  Per-token modes reduce max|x| over the
// row's lanes and store the float32 scale; static modes use `static_s`, or per channel the
// row's [D] scales `chan_s`.  INT8: [P-mem] §3.1 对称量化算法 (scale = max|x|/127,
// q = clamp(round(x/scale), -128, 127)); FP8: [P-vLLM] "KV Cache量化策略" (E4M3 storage
// with a scale).
template <typename TA, int CD, int D, int NV = 1>
__device__ __forceinline__ void quantize_row_part(const uint4* u, int l, bool write, int kv, int off,
                                                  int bs, uint8_t* rec, int off_v, int off_s,
                                                  bool per_token, float static_s,
                                                  const float* chan_s = nullptr) {
  constexpr int E = 8 * NV;                 // elements per lane
  constexpr int LPR = D / E;
  constexpr int ROWB = (CD == KVQ_DTYPE_BF16 || CD == KVQ_DTYPE_FP16) ? 2 * D : D;
  uint8_t* dst_row = rec + (kv ? off_v : 0) + off * ROWB;
  if constexpr (CD == KVQ_DTYPE_BF16 || CD == KVQ_DTYPE_FP16) {
    if (write) {
#pragma unroll
      for (int v = 0; v < NV; ++v) reinterpret_cast<uint4*>(dst_row + l * 16 * NV)[v] = u[v];
    }
  } else {
    float x[E];
#pragma unroll
    for (int v = 0; v < NV; ++v) unpack8<TA>(u[v], x + 8 * v);
    float s = static_s;
    if (per_token) {
      float m = 0.f;
#pragma unroll
      for (int i = 0; i < E; ++i) m = fmaxf(m, fabsf(x[i]));
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      s = div_rn(m, QMax<CD>::v);
      if (write && l == 0) reinterpret_cast<float*>(rec + off_s)[(kv ? bs : 0) + off] = s;
    }
    uint32_t w[2 * NV];
    if (chan_s == nullptr && s != 0.f) {
      const float r = __frcp_rn(s);
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const uint2 c = quant8_same_scale<CD>(x + 8 * v, s, r, per_token);
        w[2 * v] = c.x;
        w[2 * v + 1] = c.y;
      }
    } else {
      // PER_CHANNEL: chan_s is the row's [D] scales; this lane's are [E l, E l + E)
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        float cs[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) cs[i] = s;
        if (chan_s != nullptr) {
          const float4 a = reinterpret_cast<const float4*>(chan_s)[(E * l + 8 * v) / 4];
          const float4 b = reinterpret_cast<const float4*>(chan_s)[(E * l + 8 * v) / 4 + 1];
          cs[0] = a.x; cs[1] = a.y; cs[2] = a.z; cs[3] = a.w;
          cs[4] = b.x; cs[5] = b.y; cs[6] = b.z; cs[7] = b.w;
        }
        uint32_t c[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          c[i] = (CD == KVQ_DTYPE_INT8) ? quant_int8(x[8 * v + i], cs[i]) : quant_fp8(x[8 * v + i], cs[i]);
        w[2 * v] = pack4_low_bytes(c[0], c[1], c[2], c[3]);
        w[2 * v + 1] = pack4_low_bytes(c[4], c[5], c[6], c[7]);
      }
    }
    if (write) {
      if constexpr (NV == 1) {
        *reinterpret_cast<uint2*>(dst_row + l * 8) = make_uint2(w[0], w[1]);
      } else {
        static_assert(NV % 2 == 0, "whole 16-byte code stores");
#pragma unroll
        for (int v = 0; v < NV / 2; ++v)
          reinterpret_cast<uint4*>(dst_row + l * 8 * NV)[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
      }
    }
  }
}

// ------------------------------------------------------------------ host helpers
struct Geometry {
  int cache_dtype, act_dtype, scale_mode;
  int NB, bs, H, D;
  int group, residual_len, residual_cap, max_seqs;
  // page record of one (block, kv head): K codes at 0, V codes at off_v, scales at off_s
  int row_bytes, off_v, off_s, scale_bytes, record;
};

kvq_status validate_desc(const kvq_cache_desc* c, Geometry* g);
int code_bits(int cache_dtype);
// Streaming multiprocessors of the current device (148 on B200; 148 too when no device can
// be queried, so host-only size queries work without a GPU).  Grids and split plans are
// sized from it.
int device_sm_count();

// INT4 and INT2 caches: 64-token groups, zero points, a residual ring of recent tokens
__host__ __device__ inline bool low_bit(int cache_dtype) {
  return cache_dtype == KVQ_DTYPE_INT4 || cache_dtype == KVQ_DTYPE_INT2;
}

// Launchers implemented in the .cu files; return a cudaError_t from the launch.
cudaError_t launch_write_dense(const kvq_cache_desc& c, const Geometry& g, const void* k,
                               const void* v, int T, const int32_t* slots, cudaStream_t s);
cudaError_t launch_write_int4(const kvq_cache_desc& c, const Geometry& g, const void* k,
                              const void* v, int T, const int32_t* slots, const int32_t* seq_ids,
                              const int32_t* positions, cudaStream_t s);
cudaError_t launch_flush_ring(const kvq_cache_desc& c, const Geometry& g, const int32_t* seq_ids,
                              const int32_t* positions, const int32_t* blocks, int n, cudaStream_t s);
cudaError_t launch_dequant(const kvq_cache_desc& c, const Geometry& g, const int32_t* ids, int n,
                           float* out, cudaStream_t s);
cudaError_t launch_calibrate(const void* x, int n, int H, int D, int act, float qmax, float* out,
                             cudaStream_t s);
cudaError_t launch_calibrate_channels(const void* x, int n, int H, int D, int act, float qmax,
                                      float* out, cudaStream_t s);

// Plan of the decode kernels.  SIMT and INT4: grid (splits, heads-tiles, batch), chunk
// tokens each.  Dense tensor-core kernel: ctas CTAs over page-balanced ranges.
struct DecodePlan {
  int kernel;        // 0 = SIMT, 1 = tensor-core (mma.sync), 2 = INT4 tensor-core + ring
  int g;             // query heads per kv head
  int g_tile;        // query heads one CTA covers
  int splits;        // S (kernels 0 and 2)
  int chunk;         // tokens per split (multiple of the block size)
  int ctas;          // kernel 1: grid size
  size_t ws_bytes;   // workspace bytes (0 when a single split writes the output)
  size_t ws_ml_off;  // byte offset of the (max, sum) array inside the workspace
  int sms;           // streaming multiprocessors the plan was made for
};

kvq_status plan_decode(const Geometry& g, int batch, int num_q_heads, int max_context,
                       DecodePlan* p);

struct DecodeArgs {
  const kvq_cache_desc* c;
  Geometry geo;
  DecodePlan plan;
  const void* q;
  const void* k_new;         // append step: [B][H][D] act dtype, else null
  const void* v_new;
  const int32_t* q_start;    // prefill: [B+1] query rows of each sequence, else null
  int max_q_len;             // prefill: host bound on q_start[b+1] - q_start[b]
  int batch, Hq;
  const int32_t* block_tables;
  int max_blocks;
  const int32_t* context_lens;
  const int32_t* seq_ids;
  int max_context;
  float scale_log2;          // softmax scale * log2(e)
  void* out;
  int out_dtype;
  float* ws_o;               // partial outputs (layout per kernel)
  float* ws_ml;              // partial (max, sum) pairs
};

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_prefill(const DecodeArgs& a, cudaStream_t s);

// Launch `kernel` so that it may start while the previous kernel in the stream is still
// running (programmatic dependent launch); the kernel must call griddep_wait() before it
// reads anything that kernel could have written.
template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace kvq
