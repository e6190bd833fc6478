// Split-K paged decode attention on CUDA cores (fp32 FMA), and the split reduce.
//
// One CTA covers (split, kv head, up to two query heads of its GQA group, sequence).
// Each warp walks the split's token range in batches; a lane owns a 16-element chunk
// of the head dimension for one row at a time (16 bytes of INT8/FP8 codes, 8 bytes of
// packed INT4, 4 of INT2, 16 bytes of BF16/FP16), so a warp instruction reads whole rows.
// Scores are reduced over the lanes of a row with shuffles; each lane group runs its
// own online softmax (running max, running sum, fp32 accumulator) in the log2 domain,
// and groups, warps and finally splits are merged with log-sum-exp weights.
//
// Dequantization is fused into the inner products ([P-vLLM]
// "PagedAttention与KV Cache量化协同工作原理": INT8/FP8 blocks are dequantized inside the
// attention kernel): per-token / per-head scales multiply the dot product and the
// softmax weight rather than every element; INT4 keys use (code - zero) * scale per
// channel (or per token group in the per-token variant) and INT4 values (code - zero) *
// scale per token group ([P-prod] "量化不是简单截断精度"); the float-zero-point variant
// dequantizes to code * scale + minimum.  Decode reads every cached position of the sequence each step
// ([P-prod] "为什么长上下文更需要 KV Cache Quantization"), so this kernel is bound by
// HBM bandwidth when the ALUs keep up (small GQA groups).
#include "kvq_internal.cuh"
#include "kvq_decode_common.cuh"
#include "kvq_ptx.cuh"

namespace kvq {
namespace {

template <int CD> struct Chunk;
// 1-byte codes: 16 elements in a uint4
template <> struct Chunk<KVQ_DTYPE_INT8> { static constexpr int EPL = 16, BYTES = 16; };
template <> struct Chunk<KVQ_DTYPE_FP8_E4M3> { static constexpr int EPL = 16, BYTES = 16; };
template <> struct Chunk<KVQ_DTYPE_BF16> { static constexpr int EPL = 8, BYTES = 16; };
template <> struct Chunk<KVQ_DTYPE_FP16> { static constexpr int EPL = 8, BYTES = 16; };
template <> struct Chunk<KVQ_DTYPE_INT4> { static constexpr int EPL = 16, BYTES = 8; };
template <> struct Chunk<KVQ_DTYPE_INT2> { static constexpr int EPL = 16, BYTES = 4; };

// Load EPL cache elements of one row chunk as floats (codes only; scales applied outside).
template <int CD>
__device__ __forceinline__ void load_codes(const uint8_t* p, float* f) {
  if constexpr (CD == KVQ_DTYPE_INT8) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const int8_t* c = reinterpret_cast<const int8_t*>(&u);
#pragma unroll
    for (int i = 0; i < 16; ++i) f[i] = static_cast<float>(c[i]);
  } else if constexpr (CD == KVQ_DTYPE_FP8_E4M3) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_fp8x2_storage_t* c = reinterpret_cast<const __nv_fp8x2_storage_t*>(&u);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(c[i], __NV_E4M3);
      const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&hr));
      f[2 * i] = v.x;
      f[2 * i + 1] = v.y;
    }
  } else if constexpr (CD == KVQ_DTYPE_BF16) {
    unpack8<__nv_bfloat16>(*reinterpret_cast<const uint4*>(p), f);
  } else if constexpr (CD == KVQ_DTYPE_FP16) {
    unpack8<__half>(*reinterpret_cast<const uint4*>(p), f);
  } else if constexpr (CD == KVQ_DTYPE_INT2) {  // 4 bytes, element 4i+e in bits [2e, 2e+2)
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
#pragma unroll
    for (int i = 0; i < 16; ++i) f[i] = static_cast<float>((u >> (2 * i)) & 3u);
  } else {  // INT4: 8 bytes, element 2i in the low nibble of byte i
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const uint8_t* c = reinterpret_cast<const uint8_t*>(&u);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      f[2 * i] = static_cast<float>(c[i] & 0xF);
      f[2 * i + 1] = static_cast<float>(c[i] >> 4);
    }
  }
}

template <typename TA, int CD, int D, int GT>
__global__ void __launch_bounds__(128) decode_simt_kernel(DecodeParams p) {
  constexpr int NW = 4;
  constexpr int EPL = Chunk<CD>::EPL;
  constexpr int CB = Chunk<CD>::BYTES;
  constexpr int LPR = D / EPL;          // lanes per row
  constexpr int RPI = 32 / LPR;         // rows per warp instruction
  constexpr int U = 4;                  // rows per lane per batch
  constexpr bool kInt4 = CD == KVQ_DTYPE_INT4 || CD == KVQ_DTYPE_INT2;   // group codes + ring
  constexpr int ROWB = D * CB / EPL;    // bytes per cache row

  // a kernel launched after this one as its dependent may start at once (the INT4 / INT2
  // block kernel, which reads nothing this one writes, or the split reduce, which waits)
  griddep_launch_dependents();
  // ring-only launch (INT4 blocks on tensor cores): this grid covers [qb, n) from the ring
  const bool ring_only = p.ring_split >= 0;
  const int split = ring_only ? p.ring_split : blockIdx.x;
  const int tiles = p.g / GT;
  const int kvh = blockIdx.y / tiles;
  const int hq0 = kvh * p.g + (blockIdx.y % tiles) * GT;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = lane % LPR, grp = lane / LPR;

  const SeqInfo si = seq_info(p, b, kInt4, blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0);
  const int t0 = ring_only ? si.qb : split * p.chunk;
  const int t1 = ring_only ? si.n : min(si.n, t0 + p.chunk);
  // append step (INT4 / INT2 with the ring split): this step's row of sequence b is position
  // n - 1, always in the ring (the ring keeps at least one token); the first head tile of
  // the (sequence, kv head) stores it there as kvq_write would, and every tile reads it from
  // k_new / v_new, so no tile depends on another's store
  const bool app = kInt4 && ring_only && p.k_new != nullptr && si.n > 0;
  if (app && blockIdx.y % tiles == 0 && warp == 0) {
    const long slot = (si.n - 1) % p.cap;
#pragma unroll
    for (int kv = 0; kv < 2; ++kv) {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const TA*>(kv ? p.v_new : p.k_new) +
                                                        (static_cast<long>(b) * p.H + kvh) * D);
      uint4* dst = reinterpret_cast<uint4*>(static_cast<TA*>(p.residual_w) +
                                            ((static_cast<long>(si.sid) * 2 + kv) * p.H * p.cap +
                                             static_cast<long>(kvh) * p.cap + slot) * D);
      for (int i = lane; i < D / 8; i += 32) dst[i] = src[i];
    }
  }

  // query chunk (pre-multiplied by softmax_scale * log2 e)
  float qf[GT][EPL];
#pragma unroll
  for (int h = 0; h < GT; ++h) {
    const TA* qp = static_cast<const TA*>(p.q) + (static_cast<long>(b) * p.Hq + hq0 + h) * D + c * EPL;
#pragma unroll
    for (int i = 0; i < EPL; i += 8) {
      float f[8];
      unpack8<TA>(*reinterpret_cast<const uint4*>(qp + i), f);
#pragma unroll
      for (int j = 0; j < 8; ++j) qf[h][i + j] = f[j] * p.scale_log2;
    }
  }
  float m[GT], l[GT], acc[GT][EPL];
#pragma unroll
  for (int h = 0; h < GT; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) acc[h][i] = 0.f;
  }
  float khead = 1.f, vhead = 1.f;
  if constexpr (!kInt4) {
    if (p.mode == KVQ_SCALE_PER_HEAD) { khead = p.k_static[kvh]; vhead = p.v_static[kvh]; }
    if (p.mode == KVQ_SCALE_PER_TENSOR) { khead = p.k_static[0]; vhead = p.v_static[0]; }
  }

  constexpr int BATCH = RPI * U;
  for (int base = t0 + warp * BATCH; base < t1; base += NW * BATCH) {
    float kf[U][EPL], vf[U][EPL];
    float kscale[U], vscale[U];
    bool valid[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int pos = base + grp + RPI * j;
      valid[j] = pos < t1;
      kscale[j] = khead;
      vscale[j] = vhead;
#pragma unroll
      for (int i = 0; i < EPL; ++i) { kf[j][i] = 0.f; vf[j][i] = 0.f; }
      if (!valid[j]) continue;
      if (kInt4 && pos >= si.qb) {
        // residual ring row (unquantized activations)
        const long rrow = ((static_cast<long>(si.sid) * 2) * p.H + kvh) * p.cap + pos % p.cap;
        const long vrow = ((static_cast<long>(si.sid) * 2 + 1) * p.H + kvh) * p.cap + pos % p.cap;
        const TA* kr = static_cast<const TA*>(p.residual) + rrow * D + c * EPL;
        const TA* vr = static_cast<const TA*>(p.residual) + vrow * D + c * EPL;
        if (app && pos == si.n - 1) {                  // this step's row, from the call
          kr = static_cast<const TA*>(p.k_new) + (static_cast<long>(b) * p.H + kvh) * D + c * EPL;
          vr = static_cast<const TA*>(p.v_new) + (static_cast<long>(b) * p.H + kvh) * D + c * EPL;
        }
#pragma unroll
        for (int i = 0; i < EPL; i += 8) {
          unpack8<TA>(*reinterpret_cast<const uint4*>(kr + i), &kf[j][i]);
          unpack8<TA>(*reinterpret_cast<const uint4*>(vr + i), &vf[j][i]);
        }
        continue;
      }
      const int blk = block_of(p, b, pos / p.bs);
      if (blk < 0) { valid[j] = false; continue; }
      const int off = pos % p.bs;
      const uint8_t* rec = p.pages + (static_cast<long>(blk) * p.H + kvh) * p.record;
      load_codes<CD>(rec + off * ROWB + c * CB, kf[j]);
      load_codes<CD>(rec + p.off_v + off * ROWB + c * CB, vf[j]);
      if constexpr (kInt4) {
        // this lane's EPL channels lie in one 64-channel group
        const __half* sz = reinterpret_cast<const __half*>(rec + p.off_s);
        const int grp64 = (c * EPL) / 64;
        const bool fzp = p.mode == KVQ_SCALE_KIVI_FLOAT_ZERO;
        if (p.mode == KVQ_SCALE_INT4_PER_TOKEN) {          // K (scale, zero) [bs][D/64][2]
          const __half* ksz = sz + (off * (D / 64) + grp64) * 2;
          const float ks = __half2float(ksz[0]), kz = __half2float(ksz[1]);
#pragma unroll
          for (int i = 0; i < EPL; ++i) kf[j][i] = (kf[j][i] - kz) * ks;
        } else {                                           // K scale [D], zero or minimum [D]
#pragma unroll
          for (int i = 0; i < EPL; ++i) {
            const int d = c * EPL + i;
            const float ks = __half2float(sz[d]), kz = __half2float(sz[D + d]);
            kf[j][i] = fzp ? fmaf(kf[j][i], ks, kz) : (kf[j][i] - kz) * ks;
          }
        }
        const __half* vsz = sz + 2 * D + (off * (D / 64) + grp64) * 2;
        const float vs = __half2float(vsz[0]), vz = __half2float(vsz[1]);
        if (fzp) {                                         // code * s + minimum
#pragma unroll
          for (int i = 0; i < EPL; ++i) vf[j][i] = fmaf(vf[j][i], vs, vz);
        } else {                                           // (code - z), s folded into p
          vscale[j] = vs;
#pragma unroll
          for (int i = 0; i < EPL; ++i) vf[j][i] -= vz;
        }
      } else if (p.mode == KVQ_SCALE_PER_TOKEN_HEAD) {
        const float* sc = reinterpret_cast<const float*>(rec + p.off_s);
        kscale[j] = sc[off];
        vscale[j] = sc[p.bs + off];
      }
    }
    // scores of the U rows for each head
    float s[GT][U];
#pragma unroll
    for (int h = 0; h < GT; ++h) {
#pragma unroll
      for (int j = 0; j < U; ++j) {
        float d = 0.f;
#pragma unroll
        for (int i = 0; i < EPL; ++i) d = fmaf(qf[h][i], kf[j][i], d);
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        s[h][j] = valid[j] ? d * kscale[j] : -INFINITY;
      }
    }
#pragma unroll
    for (int h = 0; h < GT; ++h) {
      float mx = m[h];
#pragma unroll
      for (int j = 0; j < U; ++j) mx = fmaxf(mx, s[h][j]);
      if (mx == -INFINITY) continue;
      const float corr = exp2f(m[h] - mx);
      m[h] = mx;
      l[h] *= corr;
#pragma unroll
      for (int i = 0; i < EPL; ++i) acc[h][i] *= corr;
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const float pj = valid[j] ? exp2f(s[h][j] - mx) : 0.f;
        l[h] += pj;
        const float pv = pj * vscale[j];
#pragma unroll
        for (int i = 0; i < EPL; ++i) acc[h][i] = fmaf(pv, vf[j][i], acc[h][i]);
      }
    }
  }

  // merge the lane groups of this warp (lanes with the same chunk c)
#pragma unroll
  for (int h = 0; h < GT; ++h) {
    float M = m[h];
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float f = (M == -INFINITY) ? 0.f : exp2f(m[h] - M);
    float L = l[h] * f;
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      float a = acc[h][i] * f;
#pragma unroll
      for (int o = LPR; o < 32; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      acc[h][i] = a;
    }
    m[h] = M;
    l[h] = L;
  }
  __shared__ float sm_acc[NW][GT][D];
  __shared__ float sm_ml[NW][GT][2];
  if (grp == 0) {
#pragma unroll
    for (int h = 0; h < GT; ++h) {
#pragma unroll
      for (int i = 0; i < EPL; ++i) sm_acc[warp][h][c * EPL + i] = acc[h][i];
      if (c == 0) { sm_ml[warp][h][0] = m[h]; sm_ml[warp][h][1] = l[h]; }
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < GT * D; e += blockDim.x) {
    const int h = e / D, d = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, sm_ml[w][h][0]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float f = (M == -INFINITY) ? 0.f : exp2f(sm_ml[w][h][0] - M);
      L += sm_ml[w][h][1] * f;
      O += sm_acc[w][h][d] * f;
    }
    store_partial_or_output(p, b, hq0 + h, split, d, M, L, O);
  }
}

template <typename TA, int CD, int D>
cudaError_t launch_cd(const DecodeParams& p, dim3 grid, cudaStream_t s) {
  if (p.g % 2 == 0) decode_simt_kernel<TA, CD, D, 2><<<grid, 128, 0, s>>>(p);
  else decode_simt_kernel<TA, CD, D, 1><<<grid, 128, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename TA, int D>
cudaError_t launch_d(int cd, const DecodeParams& p, dim3 grid, cudaStream_t s) {
  switch (cd) {
    case KVQ_DTYPE_INT8: return launch_cd<TA, KVQ_DTYPE_INT8, D>(p, grid, s);
    case KVQ_DTYPE_FP8_E4M3: return launch_cd<TA, KVQ_DTYPE_FP8_E4M3, D>(p, grid, s);
    case KVQ_DTYPE_BF16: return launch_cd<TA, KVQ_DTYPE_BF16, D>(p, grid, s);
    case KVQ_DTYPE_FP16: return launch_cd<TA, KVQ_DTYPE_FP16, D>(p, grid, s);
    case KVQ_DTYPE_INT4: return launch_cd<TA, KVQ_DTYPE_INT4, D>(p, grid, s);
    case KVQ_DTYPE_INT2: return launch_cd<TA, KVQ_DTYPE_INT2, D>(p, grid, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_simt(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s) {
  const int gt = (a.plan.g % 2 == 0) ? 2 : 1;
  const dim3 grid(p.ring_split >= 0 ? 1 : a.plan.splits, a.geo.H * (a.plan.g / gt), a.batch);
  if (a.geo.act_dtype == KVQ_DTYPE_BF16)
    return a.geo.D == 128 ? launch_d<__nv_bfloat16, 128>(a.geo.cache_dtype, p, grid, s)
                          : launch_d<__nv_bfloat16, 64>(a.geo.cache_dtype, p, grid, s);
  return a.geo.D == 128 ? launch_d<__half, 128>(a.geo.cache_dtype, p, grid, s)
                        : launch_d<__half, 64>(a.geo.cache_dtype, p, grid, s);
}

}  // namespace kvq
