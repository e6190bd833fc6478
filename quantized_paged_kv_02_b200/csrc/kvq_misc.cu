// kvq_dequant (debug), kvq_calibrate_fp8_scales, kvq_calibrate_head_scales and
// kvq_calibrate_channel_scales (set-up)
// kernels.
//
// Dequantized values follow the definitions in include/kvq.h: INT8 / FP8 code * scale
// ([P-mem] §3.1 对称量化算法: q.float() * scale), INT4 (code - zero) * scale ([P-prod]
// "量化不是简单截断精度": X_dequant = (X_q - zero_point) * scale), or code * scale + minimum
// for the float-zero-point variant.
// The calibration scale is max|x| / 448 per kv head over warm-up rows ([P-prod]
// "vLLM：从 FP8 KV Cache 开始试点": scales from a random-token warm-up).
#include "kvq_internal.cuh"

namespace kvq {
namespace {

struct DequantParams {
  const int32_t* ids;
  int n;
  const uint8_t* pages;        // [NB][H][record]
  const float* k_static;
  const float* v_static;
  int NB, bs, H, D, cd, act, mode;
  int record, off_v, off_s, row_bytes;
  float* out;
  int32_t* fault;
};

// grid (n_blocks, 2, H): one CTA writes one [bs][D] tile of K or V.
__global__ void __launch_bounds__(256) dequant_kernel(DequantParams p) {
  const int i = blockIdx.x, kv = blockIdx.y, h = blockIdx.z;
  const int blk = p.ids[i];
  if (blk < 0 || blk >= p.NB) {
    if (threadIdx.x == 0 && kv == 0 && h == 0) record_fault(p.fault, KVQ_FAULT_BLOCK);
    return;
  }
  const uint8_t* rec = p.pages + (static_cast<long>(blk) * p.H + h) * p.record;
  const uint8_t* codes = rec + (kv ? p.off_v : 0);
  float* out = p.out + (((static_cast<long>(i) * 2 + kv) * p.H + h) * p.bs) * p.D;
  for (int e = threadIdx.x; e < p.bs * p.D; e += blockDim.x) {
    const int t = e / p.D, d = e % p.D;
    float x;
    switch (p.cd) {
      case KVQ_DTYPE_BF16:
        x = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(codes + t * p.row_bytes)[d]);
        break;
      case KVQ_DTYPE_FP16:
        x = __half2float(reinterpret_cast<const __half*>(codes + t * p.row_bytes)[d]);
        break;
      case KVQ_DTYPE_INT8:
      case KVQ_DTYPE_FP8_E4M3: {
        const uint8_t c = codes[t * p.row_bytes + d];
        const float* s = reinterpret_cast<const float*>(rec + p.off_s) + (kv ? p.bs : 0);
        const float* st = kv ? p.v_static : p.k_static;
        const float sv = p.mode == KVQ_SCALE_PER_TOKEN_HEAD ? s[t]
                         : p.mode == KVQ_SCALE_PER_HEAD   ? st[h]
                         : p.mode == KVQ_SCALE_PER_CHANNEL ? st[h * p.D + d] : st[0];
        const float cv = p.cd == KVQ_DTYPE_INT8 ? static_cast<float>(static_cast<int8_t>(c))
                                                : e4m3_to_float(c);
        x = cv * sv;
        break;
      }
      default: {  // INT4 (two codes per byte) or INT2 (four)
        int c;
        if (p.cd == KVQ_DTYPE_INT4) {
          const uint8_t byte = codes[t * p.row_bytes + d / 2];
          c = (d & 1) ? (byte >> 4) : (byte & 0xF);
        } else {
          c = (codes[t * p.row_bytes + d / 4] >> (2 * (d & 3))) & 3;
        }
        // K per channel [2][D] (KIVI forms) or per token [bs][D/64][2]; V per token
        const __half* sz = reinterpret_cast<const __half*>(rec + p.off_s);
        float s, z;
        if (kv == 0 && p.mode != KVQ_SCALE_INT4_PER_TOKEN) {
          s = __half2float(sz[d]);
          z = __half2float(sz[p.D + d]);
        } else {
          const __half* v = sz + (kv ? 2 * p.D : 0) + (t * (p.D / 64) + d / 64) * 2;
          s = __half2float(v[0]);
          z = __half2float(v[1]);
        }
        // float zero point: code * s + minimum; integer zero point: (code - z) * s
        x = p.mode == KVQ_SCALE_KIVI_FLOAT_ZERO ? fmaf(static_cast<float>(c), s, z)
                                                : (static_cast<float>(c) - z) * s;
      }
    }
    out[e] = x;
  }
}

template <typename TA>
__global__ void __launch_bounds__(256) calibrate_kernel(const TA* x, int n, int H, int D, float qmax,
                                                        float* out) {
  const int h = blockIdx.x;
  float m = 0.f;
  for (long e = threadIdx.x; e < static_cast<long>(n) * D; e += blockDim.x) {
    const long t = e / D, d = e % D;
    m = fmaxf(m, fabsf(Act<TA>::to_f(x[(t * H + h) * D + d])));
  }
  __shared__ float red[32];
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) out[h] = div_rn(m, qmax);
  }
}

// grid H: thread d of CTA h scans the tokens of channel (h, d).
template <typename TA>
__global__ void __launch_bounds__(128) calibrate_channels_kernel(const TA* x, int n, int H, int D,
                                                                 float qmax, float* out) {
  const int h = blockIdx.x;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float m = 0.f;
    for (long t = 0; t < n; ++t) m = fmaxf(m, fabsf(Act<TA>::to_f(x[(t * H + h) * D + d])));
    out[h * D + d] = div_rn(m, qmax);
  }
}

}  // namespace

cudaError_t launch_calibrate_channels(const void* x, int n, int H, int D, int act, float qmax,
                                      float* out, cudaStream_t s) {
  if (act == KVQ_DTYPE_BF16)
    calibrate_channels_kernel<__nv_bfloat16><<<H, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(x), n, H, D,
                                                                qmax, out);
  else
    calibrate_channels_kernel<__half><<<H, 128, 0, s>>>(static_cast<const __half*>(x), n, H, D, qmax, out);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const kvq_cache_desc& c, const Geometry& g, const int32_t* ids, int n,
                           float* out, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  DequantParams p{ids, n, static_cast<const uint8_t*>(c.pages), c.k_scales, c.v_scales,
                  g.NB, g.bs, g.H, g.D, g.cache_dtype, g.act_dtype, g.scale_mode,
                  g.record, g.off_v, g.off_s, g.row_bytes, out, c.fault};
  dequant_kernel<<<dim3(n, 2, g.H), 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_calibrate(const void* x, int n, int H, int D, int act, float qmax, float* out,
                             cudaStream_t s) {
  if (act == KVQ_DTYPE_BF16)
    calibrate_kernel<__nv_bfloat16><<<H, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), n, H, D, qmax,
                                                       out);
  else
    calibrate_kernel<__half><<<H, 256, 0, s>>>(static_cast<const __half*>(x), n, H, D, qmax, out);
  return cudaGetLastError();
}

}  // namespace kvq
