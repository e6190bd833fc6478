// Paged split-K decode attention on tensor cores, for GQA groups of 3..8 query heads
// (head_dim 128, dense caches: INT8, FP8 E4M3, BF16, FP16).
//
// One CTA covers (split, kv head, sequence) and the whole GQA group, so every KV byte of
// its token range is read from HBM exactly once.  Warp 4 is the producer: it walks the
// block table and moves each block's page record (K codes, V codes and per-token scales,
// contiguous in the cache) into a ring of shared-memory stages with one TMA tensor copy
// per page (128-byte swizzle, so the fragment loads below are free of bank conflicts;
// one 4 KiB copy per page instead of several small ones is what lets the copy engine
// keep HBM busy); an mbarrier per stage
// signals "full" to the consumers and another signals "empty" back.  Warps 0-3 consume
// stages round-robin.  For each 16-token tile a warp computes S^T = K Q^T with mma.sync
// m16n8k16 (M = 16 tokens, N = 8 query heads, K = head_dim, fp32 accumulate): the codes
// are turned into fp16/bf16 fragments in registers (int8 through a byte permute onto
// 1024.0, e4m3 through the hardware conversion, both exact), the per-token or per-head
// scales multiply the fp32 scores, an online softmax (running max, running sum) runs in
// the log2 domain, and O^T += V^T P^T is a second mma.sync with P split into hi + lo
// halves (P changes fragment layout in registers with movmatrix).
// Per-token V scales are folded into P with a per-warp power-of-two normaliser.  The four
// warps and then the splits are merged with log-sum-exp weights.
//
// Dequantization is fused into both contractions ([P-vLLM]
// "PagedAttention与KV Cache量化协同工作原理"); the split covers long contexts, whose decode
// reads every cached position each step ([P-prod] "为什么长上下文更需要 KV Cache
// Quantization").  Tensor cores are used because a GQA group makes QK^T a dense tile:
// with 8 query heads per KV byte the CUDA-core FMAs alone would not keep up with HBM.
#include <cudaTypedefs.h>

#include <climits>
#include <mutex>

#include "kvq_decode_common.cuh"
#include "kvq_ptx.cuh"

namespace kvq {
namespace {

constexpr int kConsumers = 4;
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kD = 128;
constexpr float kRescale = 8.f;   // log2 headroom before the running max is re-reduced

template <int CD> struct Code;
template <> struct Code<KVQ_DTYPE_INT8> { static constexpr int B = 1; static constexpr bool kBf16 = false; };
template <> struct Code<KVQ_DTYPE_FP8_E4M3> { static constexpr int B = 1; static constexpr bool kBf16 = false; };
template <> struct Code<KVQ_DTYPE_FP16> { static constexpr int B = 2; static constexpr bool kBf16 = false; };
template <> struct Code<KVQ_DTYPE_BF16> { static constexpr int B = 2; static constexpr bool kBf16 = true; };

// One stage holds one page record of include/kvq.h (K codes, V codes, per-token scales),
// copied by a single TMA with 128-byte swizzle; stages start on 1024-byte boundaries.
template <int CD, int BS, bool PT>
struct Layout {
  static constexpr int ROWB = kD * Code<CD>::B;          // bytes per token row
  static constexpr int OFF_V = BS * ROWB;                 // V codes inside the record
  static constexpr int OFF_S = 2 * BS * ROWB;             // per-token scales
  static constexpr int REC = (OFF_S + (PT ? 8 * BS : 0) + 127) / 128 * 128;
  static constexpr int REC_ROWS = REC / 128;              // TMA box height
  static constexpr int STAGE = (REC + 1023) / 1024 * 1024;
  // ring depth: about 64 KiB of records per CTA (3 CTAs per SM)
  static constexpr int kStages = (65536 / STAGE) < 4 ? 4 : ((65536 / STAGE) > 16 ? 16 : 65536 / STAGE);
  static constexpr int TILES = kStages * STAGE;
  static constexpr int BARS = kStages * 2 * 8;
  static constexpr int FLAGS = kStages * 4;
  static constexpr int MERGE = kConsumers * 8 * (kD + 2) * 4;
  static constexpr int BYTES = 1024 + TILES + BARS + FLAGS;
  static_assert(MERGE <= TILES, "merge buffer reuses the stages");
  static_assert(REC_ROWS <= 256, "TMA box height");
};

// Shared-memory byte offset of record byte `off` after the 128-byte swizzle: the 16-byte
// chunk index is XORed with the 128-byte row index (mod 8).
__device__ __forceinline__ int swzb(int off) {
  return (off & ~127) + ((((off >> 4) & 7) ^ ((off >> 7) & 7)) << 4) + (off & 15);
}

__device__ __forceinline__ float exp2_or_zero(float x) { return x == -INFINITY ? 0.f : exp2f(x); }

template <int CD, int BS, bool PT>
__global__ void __launch_bounds__(kThreads, 3)
decode_mma_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmap) {
  using L = Layout<CD, BS, PT>;
  constexpr int ROWB = L::ROWB;
  constexpr int STAGE = L::STAGE;
  constexpr bool kBf16 = Code<CD>::kBf16;
  constexpr int kStages = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle, by offsetting the shared array itself so
  // the compiler still knows every derived pointer is shared memory (plain loads -> LDS)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* tiles = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::TILES);
  uint64_t* empty = full + kStages;
  int* valid = reinterpret_cast<int*>(empty + kStages);

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SeqInfo si = seq_info(p, b, false, split == 0 && kvh == 0 && threadIdx.x == 0);
  const int t0 = split * p.chunk;                       // a multiple of BS
  const int t1 = min(si.n, t0 + p.chunk);
  const int npages = t1 > t0 ? (t1 - t0 + BS - 1) / BS : 0;
  const int page0 = t0 / BS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();

  // per-warp results for the merge
  float o[8][4];
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  int ev = INT_MIN;                                      // V normaliser exponent (PT only)
  const int r = lane >> 2, j = lane & 3;
#pragma unroll
  for (int md = 0; md < 8; ++md)
#pragma unroll
    for (int c = 0; c < 4; ++c) o[md][c] = 0.f;

  if (warp == kConsumers) {
    // ---------------------------------------------------------------- producer
    const uint32_t stage_bytes = L::REC;
    bool ok_run = true;
    int issued = 0;
    for (int base = 0; base < npages && ok_run; base += 32) {
      int blk = -1;
      if (base + lane < npages) {
        blk = p.tables[static_cast<long>(b) * p.max_blocks + page0 + base + lane];
        if (blk < 0 || blk >= p.NB) {
          record_fault(p.fault, KVQ_FAULT_BLOCK);
          blk = -1;
        }
      }
      const int cnt = min(32, npages - base);
      for (int k = 0; k < cnt; ++k) {
        const int bk = __shfl_sync(0xffffffffu, blk, k);
        const int i = base + k;
        const int s = i % kStages;
        const int round = i / kStages;
        if (lane == 0) {
          if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1)) {
            record_fault(p.fault, KVQ_FAULT_TIMEOUT);
            ok_run = false;
          }
          if (ok_run) {
            valid[s] = bk >= 0;
            if (bk >= 0) {
              // the whole record of (block, kv head) in one copy
              mbar_arrive_expect_tx(&full[s], stage_bytes);
              tma_load_2d(tiles + s * STAGE, &tmap, &full[s], 0, (bk * p.H + kvh) * L::REC_ROWS);
            } else {
              mbar_arrive(&full[s]);
            }
          }
        }
        ok_run = __shfl_sync(0xffffffffu, ok_run, 0);
        if (!ok_run) break;
        issued = i + 1;
      }
    }
    // wait until every copy this CTA issued has landed before anyone reuses the tiles
    if (lane == 0) {
      for (int i = max(0, issued - kStages); i < issued; ++i)
        if (!mbar_wait(&full[i % kStages], (i / kStages) & 1)) record_fault(p.fault, KVQ_FAULT_TIMEOUT);
    }
  } else {
    // ---------------------------------------------------------------- consumers
    const int g = p.g;
    // Q^T fragments for head n = r: thread j covers d in [32j, 32j+32); k-step kc uses
    // d = 32j + 4kc + {0,1} (b0) and {2,3} (b1), the same d <-> k map the K codes use.
    uint32_t qb[8][2];              // fp16/bf16 Q fragments (FP8, BF16, FP16 caches)
    uint32_t qt[3][4][2];           // int8 Q terms (INT8 caches), see below
    float qscale = p.scale_log2;
    {
      float qv[32];
      if (r < g) {
        const uint16_t* qp = static_cast<const uint16_t*>(p.q) +
                             (static_cast<long>(b) * p.Hq + kvh * g + r) * kD + 32 * j;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 u = *reinterpret_cast<const uint4*>(qp + 8 * c);
          const uint16_t* h = reinterpret_cast<const uint16_t*>(&u);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float f = p.act_fp16 ? __half2float(__ushort_as_half(h[e]))
                                       : __bfloat162float(__ushort_as_bfloat16(h[e]));
            qv[8 * c + e] = f;
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) qv[e] = 0.f;
      }
      if constexpr (CD == KVQ_DTYPE_INT8) {
        // q = sq * (Q0 + Q1/128 + Q2/16384) with int8 terms, sq = max|q| / 127 over the
        // group: |Q1|, |Q2| <= 64 and the error is about max|q| * 2^-22, so K . Q runs on
        // the integer tensor cores (K codes used as they are, int32 sums exact).
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(qv[e]));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        const float sq = amax / 127.f;
        const float inv = amax > 0.f ? 127.f / amax : 0.f;
        uint32_t w[3][8];
#pragma unroll
        for (int t = 0; t < 3; ++t)
#pragma unroll
          for (int e = 0; e < 8; ++e) w[t][e] = 0;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float x = qv[e];
          const int q0 = max(-127, min(127, __float2int_rn(x * inv)));
          const float r1 = fmaf(-static_cast<float>(q0), sq, x);
          const int q1 = max(-127, min(127, __float2int_rn(r1 * inv * 128.f)));
          const float r2 = fmaf(-static_cast<float>(q1), sq * (1.f / 128.f), r1);
          const int q2 = max(-127, min(127, __float2int_rn(r2 * inv * 16384.f)));
          const int sh = 8 * (e & 3);
          w[0][e >> 2] |= static_cast<uint32_t>(q0 & 0xFF) << sh;
          w[1][e >> 2] |= static_cast<uint32_t>(q1 & 0xFF) << sh;
          w[2][e >> 2] |= static_cast<uint32_t>(q2 & 0xFF) << sh;
        }
        // k-step kc: b0 <- elements 8kc..8kc+3, b1 <- 8kc+4..8kc+7 of [32j, 32j+32)
#pragma unroll
        for (int t = 0; t < 3; ++t)
#pragma unroll
          for (int kc = 0; kc < 4; ++kc) {
            qt[t][kc][0] = w[t][2 * kc];
            qt[t][kc][1] = w[t][2 * kc + 1];
          }
        qscale *= sq;
      } else if constexpr (kBf16) {
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
          qb[kc][0] = pack_bf16x2(qv[4 * kc], qv[4 * kc + 1]);
          qb[kc][1] = pack_bf16x2(qv[4 * kc + 2], qv[4 * kc + 3]);
        }
      } else {
        // power-of-two scaling keeps the group inside fp16's range; exact for the normal
        // range, and undone on the fp32 scores
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(qv[e]));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        int eq = 0;
        if (!p.act_fp16 && amax > 0.f) eq = ilogbf(amax) - 13;
        const float down = ldexpf(1.f, -eq);
        qscale = ldexpf(qscale, eq);
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
          qb[kc][0] = pack_f16x2(qv[4 * kc] * down, qv[4 * kc + 1] * down);
          qb[kc][1] = pack_f16x2(qv[4 * kc + 2] * down, qv[4 * kc + 3] * down);
        }
      }
    }
    if constexpr (!PT) {
      if (p.mode == KVQ_SCALE_PER_HEAD || p.mode == KVQ_SCALE_PER_TENSOR) {
        const int si_ = p.mode == KVQ_SCALE_PER_HEAD ? kvh : 0;
        qscale *= p.k_static[si_];
      }
    }
    // Per-thread byte offsets inside a stage tile (the swizzle depends only on the row).
    // K: token rows r and r+8, this thread's 32 codes [32j, 32j+32) of each row.
    // V: token rows 2j, 2j+1, 2j+8, 2j+9, this thread's 16 channels [16r, 16r+16).
    constexpr int KCH = 2 * Code<CD>::B;          // 16-byte chunks per K row segment
    constexpr int VCH = Code<CD>::B;              // 16-byte chunks per V row segment
    int koff[2][KCH], voff[4][VCH];
#pragma unroll
    for (int c = 0; c < KCH; ++c) {
      koff[0][c] = swzb(r * ROWB + 32 * Code<CD>::B * j + 16 * c);
      koff[1][c] = swzb((r + 8) * ROWB + 32 * Code<CD>::B * j + 16 * c);
    }
#pragma unroll
    for (int c = 0; c < VCH; ++c) {
      const int b = 16 * Code<CD>::B * r + 16 * c;
      voff[0][c] = swzb(L::OFF_V + (2 * j) * ROWB + b);
      voff[1][c] = swzb(L::OFF_V + (2 * j + 1) * ROWB + b);
      voff[2][c] = swzb(L::OFF_V + (2 * j + 8) * ROWB + b);
      voff[3][c] = swzb(L::OFF_V + (2 * j + 9) * ROWB + b);
    }
    // per-token scales of tokens r and r+8 (K, then V) inside the staged record
    const int sk0 = swzb(L::OFF_S + 4 * r), sk1 = swzb(L::OFF_S + 4 * (r + 8));
    const int sv0 = swzb(L::OFF_S + 4 * BS + 4 * r), sv1 = swzb(L::OFF_S + 4 * BS + 4 * (r + 8));

    float vlim = 0.f, vinv = 0.f;   // 2^(ev+1) and 2^-ev of the V normaliser (PT only)
    for (int i = warp; i < npages; i += kConsumers) {
      const int s = i % kStages;
      // all lanes wait; the decision is made warp-uniform before any shuffle below
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (i / kStages) & 1))) {
        if (lane == 0) record_fault(p.fault, KVQ_FAULT_TIMEOUT);
        break;
      }
      const uint8_t* st = tiles + s * STAGE;
      const bool pvalid = valid[s] != 0;
      const int pos0 = t0 + i * BS;
      const bool full_page = pvalid && pos0 + BS <= t1;          // warp-uniform
      // ------------------------------------------------ stage -> registers, then hand the
      // stage back to the producer before any math, so the ring refills during compute
      uint4 kw[2][KCH], vw[4][VCH];
#pragma unroll
      for (int c = 0; c < KCH; ++c) {
        kw[0][c] = lds128(st + koff[0][c]);
        kw[1][c] = lds128(st + koff[1][c]);
      }
#pragma unroll
      for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int c = 0; c < VCH; ++c) vw[t][c] = lds128(st + voff[t][c]);
      float ks0 = 1.f, ks1 = 1.f, vs0 = 0.f, vs1 = 0.f;
      if constexpr (PT) {
        ks0 = *reinterpret_cast<const float*>(st + sk0);
        ks1 = *reinterpret_cast<const float*>(st + sk1);
        vs0 = *reinterpret_cast<const float*>(st + sv0);
        vs1 = *reinterpret_cast<const float*>(st + sv1);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);

      // ------------------------------------------------ S^T = K Q^T
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (CD == KVQ_DTYPE_INT8) {
        // integer tensor cores: m16n8k32, k-step kc takes words 2kc (a0/a1) and 2kc+1
        // (a2/a3) of rows r and r+8, i.e. d = 32j + 8kc + 0..7, matching the Q terms
        const uint32_t w0[8] = {kw[0][0].x, kw[0][0].y, kw[0][0].z, kw[0][0].w,
                                kw[0][1].x, kw[0][1].y, kw[0][1].z, kw[0][1].w};
        const uint32_t w1[8] = {kw[1][0].x, kw[1][0].y, kw[1][0].z, kw[1][0].w,
                                kw[1][1].x, kw[1][1].y, kw[1][1].z, kw[1][1].w};
        int i0[4] = {0, 0, 0, 0}, i1[4] = {0, 0, 0, 0}, i2[4] = {0, 0, 0, 0};
#pragma unroll
        for (int kc = 0; kc < 4; ++kc) {
          const uint32_t a[4] = {w0[2 * kc], w1[2 * kc], w0[2 * kc + 1], w1[2 * kc + 1]};
          mma_s8(i0, a, qt[0][kc]);
          mma_s8(i1, a, qt[1][kc]);
          mma_s8(i2, a, qt[2][kc]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)
          sa[e] = fmaf(fmaf(static_cast<float>(i2[e]), 1.f / 128.f, static_cast<float>(i1[e])), 1.f / 128.f,
                       static_cast<float>(i0[e]));
      } else if constexpr (Code<CD>::B == 1) {
        const uint32_t w0[8] = {kw[0][0].x, kw[0][0].y, kw[0][0].z, kw[0][0].w,
                                kw[0][1].x, kw[0][1].y, kw[0][1].z, kw[0][1].w};
        const uint32_t w1[8] = {kw[1][0].x, kw[1][0].y, kw[1][0].z, kw[1][0].w,
                                kw[1][1].x, kw[1][1].y, kw[1][1].z, kw[1][1].w};
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
          uint32_t a[4];
          a[0] = e4m3x2_to_f16x2(w0[kc] & 0xFFFFu);
          a[1] = e4m3x2_to_f16x2(w1[kc] & 0xFFFFu);
          a[2] = e4m3x2_to_f16x2(w0[kc] >> 16);
          a[3] = e4m3x2_to_f16x2(w1[kc] >> 16);
          mma_f16((kc & 1) ? sb : sa, a, qb[kc]);
        }
      } else {
        // 16-bit codes: elements 32j + 4kc + {0,1} / {2,3} are whole words
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const uint32_t w0[4] = {kw[0][h].x, kw[0][h].y, kw[0][h].z, kw[0][h].w};
          const uint32_t w1[4] = {kw[1][h].x, kw[1][h].y, kw[1][h].z, kw[1][h].w};
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const uint32_t a[4] = {w0[2 * e], w1[2 * e], w0[2 * e + 1], w1[2 * e + 1]};
            if constexpr (kBf16) mma_bf16(e ? sb : sa, a, qb[2 * h + e]);
            else mma_f16(e ? sb : sa, a, qb[2 * h + e]);
          }
        }
      }
      // ------------------------------------------------ scale, mask, online softmax
      // (token r, head 2j), (r, 2j+1), (r+8, 2j), (r+8, 2j+1)
      const float f0 = qscale * ks0, f1 = qscale * ks1;
      float s00 = (sa[0] + sb[0]) * f0, s01 = (sa[1] + sb[1]) * f0;
      float s10 = (sa[2] + sb[2]) * f1, s11 = (sa[3] + sb[3]) * f1;
      if (!full_page) {
        const bool v0 = pvalid && pos0 + r < t1;
        const bool v1 = pvalid && pos0 + r + 8 < t1;
        if (!v0) { s00 = s01 = -INFINITY; vs0 = 0.f; }
        if (!v1) { s10 = s11 = -INFINITY; vs1 = 0.f; }
      }
      // The running max only needs to move when a score exceeds it by more than 2^8 in
      // weight (one vote); otherwise P <= 2^8 stays well inside fp16 and the softmax is
      // unchanged (the same reference max is used for numerator and denominator).
      const bool grow = s00 > m[0] + kRescale || s10 > m[0] + kRescale ||
                        s01 > m[1] + kRescale || s11 > m[1] + kRescale;
      if (__any_sync(0xffffffffu, grow)) {
        float tm0 = fmaxf(s00, s10), tm1 = fmaxf(s01, s11);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, off));
          tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, off));
        }
        const float mn0 = fmaxf(m[0], tm0), mn1 = fmaxf(m[1], tm1);
        const float c0 = m[0] == -INFINITY ? 0.f : ex2(m[0] - mn0);
        const float c1 = m[1] == -INFINITY ? 0.f : ex2(m[1] - mn1);
        m[0] = mn0;
        m[1] = mn1;
        l[0] *= c0;
        l[1] *= c1;
#pragma unroll
        for (int md = 0; md < 8; ++md) {
          o[md][0] *= c0;
          o[md][1] *= c1;
          o[md][2] *= c0;
          o[md][3] *= c1;
        }
      }
      const float base0 = m[0] == -INFINITY ? 0.f : m[0], base1 = m[1] == -INFINITY ? 0.f : m[1];
      const float p00 = ex2(s00 - base0), p10 = ex2(s10 - base0);
      const float p01 = ex2(s01 - base1), p11 = ex2(s11 - base1);
      l[0] += p00 + p10;
      l[1] += p01 + p11;
      // fold the per-token V scale into P, normalised by 2^ev (a power of two that only
      // grows, re-reduced when some token's scale reaches 2^(ev+1))
      float w0 = 1.f, w1 = 1.f;
      if constexpr (PT) {
        if (__any_sync(0xffffffffu, vs0 >= vlim || vs1 >= vlim)) {
          float vm = fmaxf(vs0, vs1);
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, off));
          if (vm > 0.f) {
            const int e = exponent_of(vm);
            if (e > ev) {
              if (ev != INT_MIN) {
                const float down = pow2i(ev - e);
#pragma unroll
                for (int md = 0; md < 8; ++md)
#pragma unroll
                  for (int c = 0; c < 4; ++c) o[md][c] *= down;
              }
              ev = e;
              vlim = pow2i(ev + 1);
              vinv = pow2i(-ev);
            }
          }
        }
        w0 = vs0 * vinv;
        w1 = vs1 * vinv;
      }
      const float q00 = p00 * w0, q01 = p01 * w0, q10 = p10 * w1, q11 = p11 * w1;
      // ------------------------------------------------ P^T fragments: hi + lo halves,
      // moved from the S^T accumulator layout to the B layout with movmatrix
      uint32_t pbh[2], pbl[2];
      {
        uint32_t h0, h1, e0, e1;
        if constexpr (kBf16) {
          h0 = pack_bf16x2(q00, q01);
          h1 = pack_bf16x2(q10, q11);
          const float2 f0h = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h0));
          const float2 f1h = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h1));
          e0 = pack_bf16x2(q00 - f0h.x, q01 - f0h.y);
          e1 = pack_bf16x2(q10 - f1h.x, q11 - f1h.y);
        } else {
          h0 = pack_f16x2(q00, q01);
          h1 = pack_f16x2(q10, q11);
          const float2 f0h = __half22float2(*reinterpret_cast<const __half2*>(&h0));
          const float2 f1h = __half22float2(*reinterpret_cast<const __half2*>(&h1));
          e0 = pack_f16x2(q00 - f0h.x, q01 - f0h.y);
          e1 = pack_f16x2(q10 - f1h.x, q11 - f1h.y);
        }
        pbh[0] = movmatrix_trans(h0);
        pbh[1] = movmatrix_trans(h1);
        pbl[0] = movmatrix_trans(e0);
        pbl[1] = movmatrix_trans(e1);
      }
      // ------------------------------------------------ O^T += V^T P^T
      // m-tile md, rows r / r+8 <-> d = 16r + 2md / +1; k = tokens 2j, 2j+1, 2j+8, 2j+9.
      // Rows of invalid tokens carry P = 0, but their codes may be anything: zero them.
      if (!full_page) {
        const bool va = pvalid && pos0 + 2 * j < t1, vb = pvalid && pos0 + 2 * j + 1 < t1;
        const bool vc = pvalid && pos0 + 2 * j + 8 < t1, vd = pvalid && pos0 + 2 * j + 9 < t1;
#pragma unroll
        for (int c = 0; c < VCH; ++c) {
          if (!va) vw[0][c] = make_uint4(0, 0, 0, 0);
          if (!vb) vw[1][c] = make_uint4(0, 0, 0, 0);
          if (!vc) vw[2][c] = make_uint4(0, 0, 0, 0);
          if (!vd) vw[3][c] = make_uint4(0, 0, 0, 0);
        }
      }
      if constexpr (Code<CD>::B == 1) {
        const uint32_t x0[4] = {vw[0][0].x, vw[0][0].y, vw[0][0].z, vw[0][0].w};
        const uint32_t x1[4] = {vw[1][0].x, vw[1][0].y, vw[1][0].z, vw[1][0].w};
        const uint32_t x2[4] = {vw[2][0].x, vw[2][0].y, vw[2][0].z, vw[2][0].w};
        const uint32_t x3[4] = {vw[3][0].x, vw[3][0].y, vw[3][0].z, vw[3][0].w};
#pragma unroll
        for (int md = 0; md < 8; ++md) {
          const int w = md >> 1;
          const uint32_t sel = (md & 1) ? 0x7362u : 0x5140u;
          const uint32_t X = prmt(x0[w], x1[w], sel);   // (t0 d0, t1 d0, t0 d1, t1 d1)
          const uint32_t Y = prmt(x2[w], x3[w], sel);
          uint32_t a[4];
          if constexpr (CD == KVQ_DTYPE_INT8) {
            const uint32_t xf = X ^ 0x80808080u, yf = Y ^ 0x80808080u;
            a[0] = i8x2_to_f16x2(xf, kLoPair);
            a[1] = i8x2_to_f16x2(xf, kHiPair);
            a[2] = i8x2_to_f16x2(yf, kLoPair);
            a[3] = i8x2_to_f16x2(yf, kHiPair);
          } else {
            a[0] = e4m3x2_to_f16x2(X & 0xFFFFu);
            a[1] = e4m3x2_to_f16x2(X >> 16);
            a[2] = e4m3x2_to_f16x2(Y & 0xFFFFu);
            a[3] = e4m3x2_to_f16x2(Y >> 16);
          }
          mma_f16(o[md], a, pbh);
          mma_f16(o[md], a, pbl);
        }
      } else {
        uint32_t x0[8], x1[8], x2[8], x3[8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          x0[4 * h] = vw[0][h].x; x0[4 * h + 1] = vw[0][h].y; x0[4 * h + 2] = vw[0][h].z; x0[4 * h + 3] = vw[0][h].w;
          x1[4 * h] = vw[1][h].x; x1[4 * h + 1] = vw[1][h].y; x1[4 * h + 2] = vw[1][h].z; x1[4 * h + 3] = vw[1][h].w;
          x2[4 * h] = vw[2][h].x; x2[4 * h + 1] = vw[2][h].y; x2[4 * h + 2] = vw[2][h].z; x2[4 * h + 3] = vw[2][h].w;
          x3[4 * h] = vw[3][h].x; x3[4 * h + 1] = vw[3][h].y; x3[4 * h + 2] = vw[3][h].z; x3[4 * h + 3] = vw[3][h].w;
        }
#pragma unroll
        for (int md = 0; md < 8; ++md) {
          // word md of a token holds elements (16r + 2md, +1) = (d0, d1)
          const uint32_t a[4] = {prmt(x0[md], x1[md], 0x5410u), prmt(x0[md], x1[md], 0x7632u),
                                 prmt(x2[md], x3[md], 0x5410u), prmt(x2[md], x3[md], 0x7632u)};
          if constexpr (kBf16) {
            mma_bf16(o[md], a, pbh);
            mma_bf16(o[md], a, pbl);
          } else {
            mma_f16(o[md], a, pbh);
            mma_f16(o[md], a, pbl);
          }
        }
      }
    }
    // complete the row sums: lanes with the same j hold the same heads
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l[0] += __shfl_xor_sync(0xffffffffu, l[0], off);
      l[1] += __shfl_xor_sync(0xffffffffu, l[1], off);
    }
  }
  __syncthreads();   // every stage consumed and every copy landed: the tiles become the merge buffer

  float* red_o = reinterpret_cast<float*>(tiles);                  // [warp][head][D]
  float* red_ml = red_o + kConsumers * 8 * kD;                     // [warp][head][2]
  if (warp < kConsumers) {
    float vmul = 1.f;
    if constexpr (PT) vmul = ev == INT_MIN ? 0.f : ldexpf(1.f, ev);
    if constexpr (!PT) {
      if (p.mode == KVQ_SCALE_PER_HEAD) vmul = p.v_static[kvh];
      if (p.mode == KVQ_SCALE_PER_TENSOR) vmul = p.v_static[0];
    }
#pragma unroll
    for (int md = 0; md < 8; ++md) {
      const int d0 = 16 * r + 2 * md;
      red_o[(warp * 8 + 2 * j) * kD + d0] = o[md][0] * vmul;
      red_o[(warp * 8 + 2 * j + 1) * kD + d0] = o[md][1] * vmul;
      red_o[(warp * 8 + 2 * j) * kD + d0 + 1] = o[md][2] * vmul;
      red_o[(warp * 8 + 2 * j + 1) * kD + d0 + 1] = o[md][3] * vmul;
    }
    if (r == 0) {
      red_ml[(warp * 8 + 2 * j) * 2] = m[0];
      red_ml[(warp * 8 + 2 * j) * 2 + 1] = l[0];
      red_ml[(warp * 8 + 2 * j + 1) * 2] = m[1];
      red_ml[(warp * 8 + 2 * j + 1) * 2 + 1] = l[1];
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < p.g * kD; e += kThreads) {
    const int h = e / kD, d = e % kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, red_ml[(w * 8 + h) * 2]);
    float Lsum = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) {
      const float f = M == -INFINITY ? 0.f : exp2_or_zero(red_ml[(w * 8 + h) * 2] - M);
      Lsum += red_ml[(w * 8 + h) * 2 + 1] * f;
      O += red_o[(w * 8 + h) * kD + d] * f;
    }
    store_partial_or_output(p, b, kvh * p.g + h, split, d, M, Lsum, O);
  }
}

template <int CD, int BS, bool PT>
cudaError_t launch_t(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s) {
  using L = Layout<CD, BS, PT>;
  if (a.geo.record != L::REC) return cudaErrorInvalidValue;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(decode_mma_kernel<CD, BS, PT>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
  });
  if (attr_err != cudaSuccess) return attr_err;
  CUtensorMap tm;
  const long rows = static_cast<long>(a.geo.NB) * a.geo.H * L::REC_ROWS;
  if (!make_pages_map(&tm, a.c->pages, rows, L::REC_ROWS)) return cudaErrorInvalidValue;
  const dim3 grid(a.plan.splits, a.geo.H, a.batch);
  decode_mma_kernel<CD, BS, PT><<<grid, kThreads, L::BYTES, s>>>(p, tm);
  return cudaGetLastError();
}

template <int CD, bool PT>
cudaError_t launch_bs(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s) {
  if (a.geo.bs == 16) return launch_t<CD, 16, PT>(a, p, s);
  return cudaErrorInvalidValue;
}

}  // namespace

// ------------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// Tensor map over the pages pool viewed as rows of 128 bytes; one box is one record
// (rec_rows rows), copied with 128-byte swizzle.
bool make_pages_map(CUtensorMap* map, const void* base, long rows, int rec_rows) {
  auto enc = encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {128, static_cast<cuuint32_t>(rec_rows)};
  cuuint32_t es[2] = {1, 1};
  const CUresult res = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                           box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

bool mma_supported(const Geometry& g, int groups) {
  if (g.D != kD || groups < 3 || groups > 8) return false;
  if (g.bs != 16) return false;   // 8 stages of 16-token tiles fit shared memory 3 CTAs/SM
  switch (g.cache_dtype) {
    case KVQ_DTYPE_INT8:
    case KVQ_DTYPE_FP8_E4M3:
    case KVQ_DTYPE_BF16:
    case KVQ_DTYPE_FP16: return true;
  }
  return false;
}

cudaError_t launch_decode_mma(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s) {
  const bool pt = a.geo.scale_mode == KVQ_SCALE_PER_TOKEN_HEAD;
  switch (a.geo.cache_dtype) {
    case KVQ_DTYPE_INT8: return pt ? launch_bs<KVQ_DTYPE_INT8, true>(a, p, s) : launch_bs<KVQ_DTYPE_INT8, false>(a, p, s);
    case KVQ_DTYPE_FP8_E4M3:
      return pt ? launch_bs<KVQ_DTYPE_FP8_E4M3, true>(a, p, s) : launch_bs<KVQ_DTYPE_FP8_E4M3, false>(a, p, s);
    case KVQ_DTYPE_BF16: return launch_bs<KVQ_DTYPE_BF16, false>(a, p, s);
    case KVQ_DTYPE_FP16: return launch_bs<KVQ_DTYPE_FP16, false>(a, p, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kvq
