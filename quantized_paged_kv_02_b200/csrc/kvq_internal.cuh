// Internal declarations shared by the kvq CUDA sources (not part of the public ABI).
//
// Sources cited in these files (titles of the web pages that describe the method):
//   [P-vLLM] "KV Cache量化压缩技术与vLLM推理引擎显存优化实战" (yunthe.com)
//   [P-prod] "KV Cache Quantization 生产实战：用低精度缓存降低长上下文推理显存" (oh-bug.com)
//   [P-mem]  "大模型KV Cache显存优化与量化技术实践" (intelliparadigm.com)
#pragma once

#include <utility>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kNumSMs = 148;            // B200
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

// Eight 16-bit activation values packed in a uint4 -> float.
template <typename T>
__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const T* h = reinterpret_cast<const T*>(&u);
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = Act<T>::to_f(h[i]);
}

__device__ __forceinline__ float e4m3_to_float(uint8_t c) {
  __nv_fp8_e4m3 v;
  v.__x = c;
  return static_cast<float>(v);
}

// Binary32 quotient with round-to-nearest-even, independent of -prec-div.
__device__ __forceinline__ float div_rn(float a, float b) { return __fdiv_rn(a, b); }

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

// Launchers implemented in the .cu files; return a cudaError_t from the launch.
cudaError_t launch_write_dense(const kvq_cache_desc& c, const Geometry& g, const void* k,
                               const void* v, int T, const int32_t* slots, cudaStream_t s);
cudaError_t launch_write_int4(const kvq_cache_desc& c, const Geometry& g, const void* k,
                              const void* v, int T, const int32_t* slots, const int32_t* seq_ids,
                              const int32_t* positions, cudaStream_t s);
cudaError_t launch_dequant(const kvq_cache_desc& c, const Geometry& g, const int32_t* ids, int n,
                           float* out, cudaStream_t s);
cudaError_t launch_calibrate(const void* x, int n, int H, int D, int act, float* out,
                             cudaStream_t s);

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
};

kvq_status plan_decode(const Geometry& g, int batch, int num_q_heads, int max_context,
                       DecodePlan* p);

struct DecodeArgs {
  const kvq_cache_desc* c;
  Geometry geo;
  DecodePlan plan;
  const void* q;
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
