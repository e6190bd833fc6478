// kvq_write kernels: quantize new K/V rows into the paged cache.
//
// Dense caches (INT8 / FP8 E4M3 / BF16 / FP16): one group of D*2/16 lanes per
// (kv tensor, token, kv head) row; each lane loads 16 bytes of activations, the group
// reduces max|x| with shuffles, and each lane stores its codes.  Rows are ordered
// (K or V, token, head) so a warp's loads cover contiguous memory.
//   INT8: [P-mem] §3.1 对称量化算法 (scale = max|x|/127, q = clamp(round(x/scale),-128,127))
//         with one fp32 scale per token per head ([P-mem] §3.2 动态量化策略).
//   FP8 : [P-vLLM] "KV Cache量化策略：INT8与FP8精度对比与选择" (E4M3 storage with a scale);
//         per-head static scales as in [P-prod] "vLLM：从 FP8 KV Cache 开始试点".
// INT4: one CTA per (64-row group, kv head).  KIVI quantizes keys per channel over the
// block's 64 tokens and values per token over 64-channel groups ([P-prod] "Key 和 Value
// 的分布不一定相同"), with the affine form of [P-prod] "量化不是简单截断精度"; the per-token
// variant groups keys like values, and the float-zero-point variant offsets each group by
// its minimum.  Rows that belong to no block are copied unquantized into the residual ring.
#include "kvq_internal.cuh"
#include "kvq_ptx.cuh"

namespace kvq {
namespace {

struct WriteParams {
  const void* k;
  const void* v;
  const int32_t* slots;
  int T;
  uint8_t* pages;            // [NB][H][record]
  const float* k_static;     // PER_HEAD / PER_TENSOR scales
  const float* v_static;
  int NB, bs, H;
  int record, off_v, off_s;
  int scale_mode;
  int32_t* fault;
};

// grid (T, ceil(2 H LPR / blockDim)): token t = blockIdx.x; its 2H rows (K rows of heads
// 0..H-1, then V rows) are spread over blockIdx.y and the CTA's threads (2 H LPR rounded up
// to whole warps, at most 256), LPR = D / 32 lanes
// per row with 32 activations (four 16-byte loads) each, so no index needs a division and
// each lane's index and scale work covers 32 values.  bs_shift >= 0: the block size is
// 2^bs_shift.
template <typename TA, int CD, int D>
__global__ void __launch_bounds__(256) write_dense_kernel(WriteParams p, int bs_shift) {
  griddep_launch_dependents();   // a decode launched after this one may start its set-up
  constexpr int NV = 4;             // 16-byte chunks per lane
  constexpr int LPR = D / (8 * NV); // lanes per row
  const int RPB = blockDim.x / LPR;  // rows per CTA
  const int l = threadIdx.x % LPR;
  const int t = blockIdx.x;
  const int r = blockIdx.y * RPB + threadIdx.x / LPR;   // row of the token: (kv, head)
  const bool valid = r < 2 * p.H;
  // rows past the token's 2H (the tail of the last CTA along y) stand in for head 0: they
  // take part in the shuffles of their lane group but read and write nothing
  const int kv = (valid && r >= p.H) ? 1 : 0;
  const int h = valid ? r - kv * p.H : 0;
  const int slot = p.slots[t];
  const long nslots = static_cast<long>(p.NB) * p.bs;
  const bool write = valid && slot >= 0 && slot < nslots;
  if (blockIdx.y == 0 && threadIdx.x == 0 && (slot < -1 || slot >= nslots)) record_fault(p.fault, KVQ_FAULT_SLOT);

  uint4 u[NV];
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const TA*>(kv ? p.v : p.k) +
                                                    (static_cast<long>(t) * p.H + h) * D + l * 8 * NV);
#pragma unroll
  for (int v = 0; v < NV; ++v) u[v] = write ? src[v] : make_uint4(0, 0, 0, 0);
  int blk = 0, off = 0;
  if (write) {
    if (bs_shift >= 0) {
      blk = slot >> bs_shift;
      off = slot & ((1 << bs_shift) - 1);
    } else {
      blk = slot / p.bs;
      off = slot - blk * p.bs;
    }
  }
  // record of (block, head); this row's codes and (per-token) scale inside it
  uint8_t* rec = p.pages + (static_cast<long>(blk) * p.H + h) * p.record;
  const float* sp = kv ? p.v_static : p.k_static;
  const bool is_static = p.scale_mode == KVQ_SCALE_PER_HEAD || p.scale_mode == KVQ_SCALE_PER_TENSOR;
  const float static_s = (valid && is_static) ? sp[p.scale_mode == KVQ_SCALE_PER_HEAD ? h : 0] : 0.f;
  const float* chan_s = p.scale_mode == KVQ_SCALE_PER_CHANNEL ? sp + static_cast<long>(h) * D : nullptr;
  quantize_row_part<TA, CD, D, NV>(u, l, write, kv, off, p.bs, rec, p.off_v, p.off_s,
                                   p.scale_mode == KVQ_SCALE_PER_TOKEN_HEAD, static_s, chan_s);
}

// ------------------------------------------------------------------ INT4 (KIVI)
struct Int4WriteParams {
  const void* k;
  const void* v;
  const int32_t* slots;
  const int32_t* seq_ids;
  const int32_t* positions;
  int T;
  uint8_t* pages;   // [NB][H][record]: K codes, V codes, K scale [D], K zero [D], V (s,z) [64][D/64][2]
  void* residual;   // [max_seqs][2][H][cap][D]
  int NB, H, cap, max_seqs;
  int record, off_v, off_s, mode;
  int32_t* fault;
};

struct Int4Group {
  float sw;       // stored fp16 scale, widened
  __half s16;
  float off;      // integer zero point z, or the stored fp16 minimum m widened
  __half off16;   // what the record stores beside the scale: z or m
};

// lo/hi are the group's min and max; Q = 15 (INT4) or 3 (INT2) is the largest code.
// Integer zero point: the range is widened to include 0 and z = clamp(round(-lo / s), 0, Q).
// Float zero point: the offset is the group minimum m = fp16(lo) itself.
template <int Q>
__device__ __forceinline__ Int4Group int4_group(float lo, float hi, bool float_zero) {
  if (!float_zero) {
    lo = fminf(lo, 0.f);
    hi = fmaxf(hi, 0.f);
  }
  Int4Group g;
  g.s16 = __float2half_rn(div_rn(__fsub_rn(hi, lo), static_cast<float>(Q)));
  g.sw = __half2float(g.s16);
  if (float_zero) {
    g.off16 = __float2half_rn(lo);
    g.off = __half2float(g.off16);
  } else {
    const int z = (g.sw == 0.f) ? 0 : max(0, min(Q, __float2int_rn(div_rn(-lo, g.sw))));
    g.off = static_cast<float>(z);
    g.off16 = __int2half_rn(z);
  }
  return g;
}

// integer zero point: clamp(round(x / s) + z, 0, Q); float: clamp(round((x - m) / s), 0, Q)
template <int Q>
__device__ __forceinline__ int int4_code(float x, const Int4Group& g, bool float_zero) {
  if (g.sw == 0.f) return 0;
  const int r = float_zero ? __float2int_rn(div_rn(__fsub_rn(x, g.off), g.sw))
                           : __float2int_rn(div_rn(x, g.sw)) + static_cast<int>(g.off);
  return max(0, min(Q, r));
}

// Quantize the 64 rows of one (block, kv head) into its page record, BITS-bit codes (4 or
// 2) packed 8 / BITS per byte.  Values: one group per token per 64 channels.  Keys: one group per channel over the
// 64 tokens (KIVI, [P-prod] "Key 和 Value 的分布不一定相同"), or per token like the values
// (INT4_PER_TOKEN, the Transformers integration's choice in the same section).
// row(kv, t) points at row t (act dtype, D values) of K (kv 0) or V (kv 1).  All 128
// threads of the CTA take part.
template <typename TA, int D, int BITS, typename RowFn>
__device__ void quantize_int4_block(RowFn row, uint8_t* rec, int off_v, int off_s, int mode,
                                    float (*xs)[D + 1], uint8_t (*cs)[D]) {
  constexpr int G = 64;
  constexpr int Q = (1 << BITS) - 1;           // largest code
  const int tid = threadIdx.x;
  const bool fz = mode == KVQ_SCALE_KIVI_FLOAT_ZERO;
  const bool k_per_token = mode == KVQ_SCALE_INT4_PER_TOKEN;
  __half* k_sz = reinterpret_cast<__half*>(rec + off_s);   // [2][D] or [64][D/64][2]
  __half* v_sz = k_sz + 2 * D;                             // [64][D/64][2]
  for (int kv = 0; kv < 2; ++kv) {
    // stage the 64 rows of this head as float
    for (int i = tid; i < G * D / 8; i += blockDim.x) {
      const int t = i / (D / 8), c = i % (D / 8);
      const uint4 w = *reinterpret_cast<const uint4*>(row(kv, t) + c * 8);
      float f[8];
      unpack8<TA>(w, f);
#pragma unroll
      for (int j = 0; j < 8; ++j) xs[t][c * 8 + j] = f[j];
    }
    __syncthreads();
    if (kv == 0 && !k_per_token) {
      // keys: one group per channel over the 64 tokens
      for (int d = tid; d < D; d += blockDim.x) {
        float lo = xs[0][d], hi = xs[0][d];
        for (int t = 1; t < G; ++t) { lo = fminf(lo, xs[t][d]); hi = fmaxf(hi, xs[t][d]); }
        const Int4Group g = int4_group<Q>(lo, hi, fz);
        for (int t = 0; t < G; ++t) cs[t][d] = static_cast<uint8_t>(int4_code<Q>(xs[t][d], g, fz));
        k_sz[d] = g.s16;
        k_sz[D + d] = g.off16;
      }
    } else {
      // one group per token per 64 channels
      __half* sz_base = kv ? v_sz : k_sz;
      for (int i = tid; i < G * (D / 64); i += blockDim.x) {
        const int t = i / (D / 64), gi = i % (D / 64);
        float lo = xs[t][gi * 64], hi = lo;
        for (int j = 1; j < 64; ++j) { lo = fminf(lo, xs[t][gi * 64 + j]); hi = fmaxf(hi, xs[t][gi * 64 + j]); }
        const Int4Group g = int4_group<Q>(lo, hi, fz);
        for (int j = 0; j < 64; ++j)
          cs[t][gi * 64 + j] = static_cast<uint8_t>(int4_code<Q>(xs[t][gi * 64 + j], g, fz));
        __half* sz = sz_base + (t * (D / 64) + gi) * 2;
        sz[0] = g.s16;
        sz[1] = g.off16;
      }
    }
    __syncthreads();
    // pack (element k of a run of 32 / BITS in bits [BITS k, BITS k + BITS) of a 32-bit
    // word, i.e. element 2i in the low nibble of byte i, or 4i+e in bits [2e, 2e+2)) and
    // store 16 bytes at a time
    constexpr int PER_WORD = 32 / BITS;          // codes per 32-bit word
    constexpr int PER_16B = 4 * PER_WORD;        // codes per 16-byte store
    uint8_t* dst = rec + (kv ? off_v : 0);
    for (int i = tid; i < G * D / PER_16B; i += blockDim.x) {
      const int t = i / (D / PER_16B), c = i % (D / PER_16B);
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t x = 0;
#pragma unroll
        for (int k = 0; k < PER_WORD; ++k)
          x |= static_cast<uint32_t>(cs[t][c * PER_16B + j * PER_WORD + k]) << (BITS * k);
        w[j] = x;
      }
      *reinterpret_cast<uint4*>(dst + t * (D * BITS / 8) + c * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    __syncthreads();
  }
}

template <typename TA, int D, int BITS>
__global__ void __launch_bounds__(128) write_int4_kernel(Int4WriteParams p) {
  griddep_launch_dependents();   // a decode launched after this one may start its set-up
  constexpr int G = 64;
  __shared__ float xs[G][D + 1];
  __shared__ __align__(16) uint8_t cs[G][D];
  __shared__ int ok_s;
  const int u = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int r0 = u * G;
  const int nr = min(G, p.T - r0);
  const int first = p.slots[r0];

  if (first >= 0) {
    // one whole block, in order
    if (tid == 0) ok_s = (nr == G && first % G == 0 && first / G < p.NB) ? 1 : 0;
    __syncthreads();
    int mine = (tid < nr) ? (p.slots[r0 + tid] == first + tid) : 1;
    int ok = __syncthreads_and(mine && ok_s);
    if (!ok) {
      if (tid == 0) record_fault(p.fault, KVQ_FAULT_INT4_RUN);
      return;
    }
    const long blk = first / G;
    uint8_t* rec = p.pages + (blk * p.H + h) * p.record;
    auto row = [&](int kv, int t) {
      return static_cast<const TA*>(kv ? p.v : p.k) + (static_cast<long>(r0 + t) * p.H + h) * D;
    };
    quantize_int4_block<TA, D, BITS>(row, rec, p.off_v, p.off_s, p.mode, xs, cs);
  } else {
    // residual rows: copied unquantized into ring row positions[t] % cap
    for (int i = tid; i < nr * 2 * (D / 8); i += blockDim.x) {
      const int r = i / (2 * (D / 8));
      const int kv = (i / (D / 8)) % 2;
      const int c = i % (D / 8);
      const int t = r0 + r;
      const int slot = p.slots[t];
      const bool lead = (kv == 0 && c == 0);
      if (slot != -1) {
        if (lead) record_fault(p.fault, KVQ_FAULT_INT4_RUN);
        continue;
      }
      const int pos = p.positions ? p.positions[t] : -1;
      if (pos < 0) continue;
      const int sid = p.seq_ids ? p.seq_ids[t] : -1;
      if (sid < 0 || sid >= p.max_seqs) {
        if (lead) record_fault(p.fault, KVQ_FAULT_SEQ);
        continue;
      }
      const TA* src = static_cast<const TA*>(kv ? p.v : p.k) + (static_cast<long>(t) * p.H + h) * D + c * 8;
      TA* dst = static_cast<TA*>(p.residual) +
                ((static_cast<long>(sid * 2 + kv) * p.H + h) * p.cap + pos % p.cap) * D + c * 8;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    }
  }
}

template <typename TA, int CD, int D>
cudaError_t dense_launch(const WriteParams& p, cudaStream_t s) {
  constexpr int LPR = D / 32;
  if (p.T <= 0) return cudaSuccess;
  const int need = 2 * p.H * LPR;                       // threads of one token
  const int threads = need >= 256 ? 256 : (need + 31) / 32 * 32;
  const int ys = (need + threads - 1) / threads;
  if (ys > 65535) return cudaErrorInvalidValue;
  int bs_shift = -1;
  for (int k = 0; k < 31; ++k)
    if ((1 << k) == p.bs) bs_shift = k;
  write_dense_kernel<TA, CD, D><<<dim3(static_cast<unsigned>(p.T), static_cast<unsigned>(ys)), threads, 0, s>>>(p, bs_shift);
  return cudaGetLastError();
}

template <typename TA, int D>
cudaError_t dense_by_cd(int cd, const WriteParams& p, cudaStream_t s) {
  switch (cd) {
    case KVQ_DTYPE_INT8: return dense_launch<TA, KVQ_DTYPE_INT8, D>(p, s);
    case KVQ_DTYPE_FP8_E4M3: return dense_launch<TA, KVQ_DTYPE_FP8_E4M3, D>(p, s);
    case KVQ_DTYPE_BF16: return dense_launch<TA, KVQ_DTYPE_BF16, D>(p, s);
    case KVQ_DTYPE_FP16: return dense_launch<TA, KVQ_DTYPE_FP16, D>(p, s);
  }
  return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------ INT4 ring flush
struct Int4FlushParams {
  const int32_t* seq_ids;
  const int32_t* positions;
  const int32_t* blocks;
  uint8_t* pages;
  const void* residual;     // [max_seqs][2][H][cap][D]
  int NB, H, cap, max_seqs;
  int record, off_v, off_s, mode;
  int32_t* fault;
};

// grid (entries, H): quantize ring rows [p0, p0 + 64) of one sequence and kv head into the
// block's record, exactly as kvq_write stores those rows with slots blk*64 .. blk*64+63.
template <typename TA, int D, int BITS>
__global__ void __launch_bounds__(128) flush_ring_kernel(Int4FlushParams p) {
  __shared__ float xs[64][D + 1];
  __shared__ __align__(16) uint8_t cs[64][D];
  const int e = blockIdx.x, h = blockIdx.y;
  const int sid = p.seq_ids[e], p0 = p.positions[e], blk = p.blocks[e];
  int bad = 0;
  if (sid < 0 || sid >= p.max_seqs) bad = KVQ_FAULT_SEQ;
  else if (blk < 0 || blk >= p.NB) bad = KVQ_FAULT_BLOCK;
  else if (p0 < 0 || p0 % 64 != 0) bad = KVQ_FAULT_INT4_RUN;
  if (bad) {                                // uniform over the CTA
    if (h == 0 && threadIdx.x == 0) record_fault(p.fault, bad);
    return;
  }
  uint8_t* rec = p.pages + (static_cast<long>(blk) * p.H + h) * p.record;
  auto row = [&](int kv, int t) {
    return static_cast<const TA*>(p.residual) +
           ((static_cast<long>(sid * 2 + kv) * p.H + h) * p.cap + (p0 + t) % p.cap) * D;
  };
  quantize_int4_block<TA, D, BITS>(row, rec, p.off_v, p.off_s, p.mode, xs, cs);
}

}  // namespace

cudaError_t launch_flush_ring(const kvq_cache_desc& c, const Geometry& g, const int32_t* seq_ids,
                              const int32_t* positions, const int32_t* blocks, int n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  Int4FlushParams p{seq_ids, positions, blocks, static_cast<uint8_t*>(c.pages), c.residual,
                    g.NB, g.H, g.residual_cap, g.max_seqs, g.record, g.off_v, g.off_s,
                    g.scale_mode, c.fault};
  const dim3 grid(n, g.H);
  const int sel = (g.cache_dtype == KVQ_DTYPE_INT4 ? 4 : 0) + (g.act_dtype == KVQ_DTYPE_BF16 ? 2 : 0) +
                  (g.D == 128 ? 1 : 0);
  switch (sel) {
    case 7: flush_ring_kernel<__nv_bfloat16, 128, 4><<<grid, 128, 0, s>>>(p); break;
    case 6: flush_ring_kernel<__nv_bfloat16, 64, 4><<<grid, 128, 0, s>>>(p); break;
    case 5: flush_ring_kernel<__half, 128, 4><<<grid, 128, 0, s>>>(p); break;
    case 4: flush_ring_kernel<__half, 64, 4><<<grid, 128, 0, s>>>(p); break;
    case 3: flush_ring_kernel<__nv_bfloat16, 128, 2><<<grid, 128, 0, s>>>(p); break;
    case 2: flush_ring_kernel<__nv_bfloat16, 64, 2><<<grid, 128, 0, s>>>(p); break;
    case 1: flush_ring_kernel<__half, 128, 2><<<grid, 128, 0, s>>>(p); break;
    default: flush_ring_kernel<__half, 64, 2><<<grid, 128, 0, s>>>(p); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_write_dense(const kvq_cache_desc& c, const Geometry& g, const void* k,
                               const void* v, int T, const int32_t* slots, cudaStream_t s) {
  WriteParams p{k, v, slots, T, static_cast<uint8_t*>(c.pages), c.k_scales, c.v_scales,
                g.NB, g.bs, g.H, g.record, g.off_v, g.off_s, g.scale_mode, c.fault};
  if (g.act_dtype == KVQ_DTYPE_BF16)
    return g.D == 128 ? dense_by_cd<__nv_bfloat16, 128>(g.cache_dtype, p, s)
                      : dense_by_cd<__nv_bfloat16, 64>(g.cache_dtype, p, s);
  return g.D == 128 ? dense_by_cd<__half, 128>(g.cache_dtype, p, s)
                    : dense_by_cd<__half, 64>(g.cache_dtype, p, s);
}

cudaError_t launch_write_int4(const kvq_cache_desc& c, const Geometry& g, const void* k,
                              const void* v, int T, const int32_t* slots, const int32_t* seq_ids,
                              const int32_t* positions, cudaStream_t s) {
  Int4WriteParams p{k, v, slots, seq_ids, positions, T, static_cast<uint8_t*>(c.pages),
                    c.residual, g.NB, g.H, g.residual_cap, g.max_seqs, g.record, g.off_v, g.off_s,
                    g.scale_mode, c.fault};
  const dim3 grid((T + 63) / 64, g.H);
  if (grid.x == 0) return cudaSuccess;
  const int sel = (g.cache_dtype == KVQ_DTYPE_INT4 ? 4 : 0) + (g.act_dtype == KVQ_DTYPE_BF16 ? 2 : 0) +
                  (g.D == 128 ? 1 : 0);
  switch (sel) {
    case 7: write_int4_kernel<__nv_bfloat16, 128, 4><<<grid, 128, 0, s>>>(p); break;
    case 6: write_int4_kernel<__nv_bfloat16, 64, 4><<<grid, 128, 0, s>>>(p); break;
    case 5: write_int4_kernel<__half, 128, 4><<<grid, 128, 0, s>>>(p); break;
    case 4: write_int4_kernel<__half, 64, 4><<<grid, 128, 0, s>>>(p); break;
    case 3: write_int4_kernel<__nv_bfloat16, 128, 2><<<grid, 128, 0, s>>>(p); break;
    case 2: write_int4_kernel<__nv_bfloat16, 64, 2><<<grid, 128, 0, s>>>(p); break;
    case 1: write_int4_kernel<__half, 128, 2><<<grid, 128, 0, s>>>(p); break;
    default: write_int4_kernel<__half, 64, 2><<<grid, 128, 0, s>>>(p); break;
  }
  return cudaGetLastError();
}

}  // namespace kvq
