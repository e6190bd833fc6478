// Paged split-K decode attention over INT4 and INT2 pages on tensor cores (head_dim 128,
// block 64, GQA groups of 3..8 query heads), for the three group forms of include/kvq.h.
//
// KIVI keeps keys per channel and values per token ([P-prod] "Key 和 Value 的分布不一定
// 相同"), each as X_q = round(X/scale) + zero_point ([P-prod] "量化不是简单截断精度"):
//   k_hat[t][d] = (c[t][d] - zk[d]) * sk[d]   (one (scale, zero) per channel per block)
//   v_hat[t][d] = (c[t][d] - zv[t][G]) * sv[t][G]   (G = the 64-channel group of d)
// A per-channel key scale cannot leave the sum over channels, so for each block the
// consumer forms q'[d] = q[d] * sk[d] (fp32; split into fp16 hi + lo halves, 22 bits).  The
// 4-bit codes go to the tensor cores as they are: a code in the mantissa bits of an fp16
// with a zero exponent is the exact subnormal c * 2^-24, so one mask per register pair
// replaces a conversion.  The zero points come out as sums computed beside the MMAs:
//   S^T[t] = 2^24 * (C Q'^T)[t] - sum_d q'[d] zk[d]           (one term per block and head)
//   O[d]   = 2^24 * (C^T P'^T)[d] - sum_t p'[t] zv[t][G(d)]    (one term per head and group)
// where p' is P with each token's value scale folded in (per channel group, with the same
// power-of-two normaliser as the INT8 kernel); the value-side sums follow every rescale
// of O.  Both subtracted terms and the products they cancel are of similar size (codes
// and zero points are both in [0, 15]), so the cancellation costs a few bits of fp32.
// S^T = C Q'^T with two mma.sync m16n8k16 per k-step (hi and lo halves of q').  For P V,
// A holds the codes of two tokens per register, assembled with a byte permute.  The
// residual ring (the newest tokens, unquantized) is a separate split handled by the
// CUDA-core kernel; the reduce merges both.
//
// Float zero point (k_hat = c * sk + mk, v_hat = c * sv + mv, m the group minimum): the
// same products, with the offsets added instead of subtracted:
//   S^T[t] = 2^24 * (C Q'^T)[t] + sum_d q[d] mk[d],   O[d] = 2^24 * (C^T P'^T)[d] + sum_t p[t] mv[t][G(d)].
// Keys per token (k_hat[t][d] = (c[t][d] - zk[t][G]) * sk[t][G], grouped like values): the
// scale cannot be folded into q, but it is constant over each 64-channel group, so each
// lane reads its codes as two 8-byte halves (one per group) and every k-step stays inside
// one group; two accumulators hold the per-group sums and
//   S^T[t] = sum_G sk[t][G] * (2^24 * (C_G q^T)[t] - zk[t][G] * sum_{d in G} q[d]).
// q is then the same for every block: its fp16 fragments (one MMA per k-step, q being an
// activation value scaled by a power of two) and per-group sums are formed once.
//
// 2-bit codes ([P-prod] "KV Cache 的基本内存模型": 0.25 byte per value) take the same path:
// a 2-bit code under a zero exponent is the subnormal c * 2^-24 too; a k-step pairs codes
// s and s + 8 of one 32-bit word instead of s and s + 4, and for P V each token's 16-bit
// slice of a channel group is spread over a register's halves by the same byte permute.
//
// Structure as the dense tensor-core kernel: warp 4 stages one record per block (64
// tokens of K and V codes plus all scales and zero points: 9 KiB for INT4, 5 KiB for INT2)
// with one 128-byte-swizzled TMA copy into an mbarrier ring; warps 0-3 consume blocks
// round-robin (16 tokens per MMA tile, four tiles per block).
#include <cudaTypedefs.h>

#include <climits>
#include <mutex>

#include "kvq_decode_common.cuh"
#include "kvq_ptx.cuh"

namespace kvq {
namespace {

constexpr int kC = 4;                     // consumer warps
constexpr int kT = 32 * (kC + 1);
constexpr int kD = 128;
constexpr int kBS = 64;
// Consumers take blocks round-robin, so every round of a stage must go to the same warp
// (a warp waiting for round r of a stage whose round r-1 belonged to another warp, not yet
// landed, would see the parity of round r-2 as complete): a multiple of kC stages.
constexpr int kStages = 8;
static_assert(kStages % kC == 0, "ring depth is a multiple of the consumers");
constexpr float kRescale4 = 8.f;

// Record of one (block, kv head) for BITS-bit codes (4, or 2), head_dim 128, 64 tokens:
// K codes, V codes, then the float16 parameters (K scale [128] and zero [128], or K (scale,
// zero) [64][2][2] per token; V (scale, zero) [64][2][2]).
template <int BITS>
struct Rec {
  static constexpr int kRowB = kD * BITS / 8;          // bytes of codes per token: 64 or 32
  static constexpr int kOffV = kBS * kRowB;            // V codes: 4096 or 2048
  static constexpr int kOffKs = 2 * kBS * kRowB;       // K parameters: 8192 or 4096
  static constexpr int kOffKz = kOffKs + 2 * kD;       // K zero points (per channel)
  static constexpr int kOffVsz = kOffKs + 4 * kD;      // V (scale, zero) per token
  static constexpr int kRec = kOffVsz + kBS * 2 * 4;   // 9216 or 5120
  static constexpr int kRecRows = kRec / 128;          // TMA box height: 72 or 40
  static constexpr int kStage = kRec;                  // a multiple of 1024
  static constexpr int kTile = 16 * kRowB;             // 16 tokens of codes: 1024 or 512 bytes
  static constexpr int kTiles = kStages * kStage;
  // each consumer lane's 32 q values (KIVI forms: read once per block for the key-scale
  // fold, so they need not stay in registers)
  static constexpr int kQv = kC * 32 * 32 * 4;
  static constexpr int kBytes = 1024 + kTiles + kQv + kStages * 16 + kStages * 4;
  static constexpr int PW = 16 / BITS;                 // codes in each 16-bit half of a word
  static constexpr uint32_t kMask = BITS == 4 ? 0x000F000Fu : 0x00030003u;
  static_assert(kStage % 1024 == 0, "stages start on the swizzle period");
  static_assert(kC * 8 * (kD + 2) * 4 <= kTiles, "merge buffer");
};

__device__ __forceinline__ int swzb4(int off) {
  return (off & ~127) + ((((off >> 4) & 7) ^ ((off >> 7) & 7)) << 4) + (off & 15);
}

// Offsets of the 8-byte (scale, zero) pairs of channel groups 0 and 1 of tokens 16mt + r
// and 16mt + r + 8 in a per-token parameter array that starts at `base` (a multiple of 128)
// of a stage: 16 tokens fill one 128-byte swizzle row, so the two are swzb4 of base + 128mt
// + 8r and of that + 64, in closed form.
__device__ __forceinline__ int2 sz_offsets(int base, int mt, int r) {
  const int x = ((base >> 7) + mt) & 7;
  const int v = ((r >> 1) ^ x) << 4;
  const int b0 = base + 128 * mt + 8 * (r & 1);
  return make_int2(b0 + v, b0 + (v ^ 64));
}

// (code s, code s + 16/BITS) of w -- the codes at the same place in its two 16-bit halves
// -- as fp16 bit patterns: a 4- or 2-bit code anywhere in the low ten bits of a half with a
// zero exponent is an exact fp16 subnormal, c * 2^(BITS pos - 24), so the tensor cores take
// it with one mask and no conversion.  Codes are masked in place at pos = s % PER and only
// every PER-th position needs a shifted copy of the word (ws[k] = w >> k SH): 4-bit codes
// sit at nibble 0 or 1 of a source word (w, w >> 8), 2-bit codes at crumb 0, 1 or 2 (w,
// w >> 6, w >> 12).  The factor 2^(BITS pos) (1 or 16; 1, 4 or 16) is taken out of the
// other operand (keys: q'; values: the output rows).
template <int BITS>
struct CodeSel {
  static constexpr int PER = BITS == 4 ? 2 : 3;       // positions per source word
  static constexpr int SH = BITS * PER;               // shift between source words
  static constexpr int NSRC = 16 / BITS / PER + (16 / BITS % PER ? 1 : 0);   // 2 or 3
  static constexpr int pos(int s) { return s % PER; }
  // log2 of the factor a code at position s carries
  static constexpr int lg(int s) { return BITS * (s % PER); }
};

template <int BITS>
__device__ __forceinline__ void code_sources(uint32_t w, uint32_t (&ws)[CodeSel<BITS>::NSRC]) {
#pragma unroll
  for (int k = 0; k < CodeSel<BITS>::NSRC; ++k) ws[k] = w >> (k * CodeSel<BITS>::SH);
}

template <int BITS>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&ws)[CodeSel<BITS>::NSRC], int s) {
  using C = CodeSel<BITS>;
  return ws[s / C::PER] & (Rec<BITS>::kMask << C::lg(s));
}

// 2^-e for a small compile-time e
__host__ __device__ constexpr float inv_pow2(int e) { return e == 0 ? 1.f : 0.5f * inv_pow2(e - 1); }

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Forms of the kernel (each for 4- and 2-bit codes)
constexpr int kKivi = 0;        // keys per channel, integer zero points
constexpr int kKiviMin = 1;     // keys per channel, the group minimum as a float zero point
constexpr int kPerToken = 2;    // keys per token like values, integer zero points

template <int MODE, int BITS>
__global__ void __launch_bounds__(kT, 2)
decode_int4_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmap) {
  constexpr bool kFz = MODE == kKiviMin;
  constexpr bool kTok = MODE == kPerToken;
  using R = Rec<BITS>;
  constexpr int kRowB = R::kRowB, kOffV = R::kOffV, kOffKs = R::kOffKs, kOffKz = R::kOffKz;
  constexpr int kOffVsz = R::kOffVsz, kRec = R::kRec, kRecRows = R::kRecRows;
  constexpr int kStage = R::kStage, kTiles = R::kTiles, PW = R::PW;
  using CS = CodeSel<BITS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* tiles = smem;
  float4* qvs = reinterpret_cast<float4*>(smem + kTiles);   // [warp][8][lane]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kTiles + R::kQv);
  uint64_t* empty = full + kStages;
  int* valid = reinterpret_cast<int*>(empty + kStages);

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SeqInfo si = seq_info(p, b, true, split == 0 && kvh == 0 && threadIdx.x == 0);
  const int t0 = split * p.chunk;                         // a multiple of 64
  const int t1 = min(si.qb, t0 + p.chunk);                // blocks only; the ring is elsewhere
  const int npages = t1 > t0 ? (t1 - t0) / kBS : 0;
  const int page0 = t0 / kBS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();

  float o[8][4];
  float cz[2][2] = {{0.f, 0.f}, {0.f, 0.f}};      // [group][head 2j, 2j+1]: sum p' z
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  int ev = INT_MIN;
  const int r = lane >> 2, j = lane & 3;
#pragma unroll
  for (int md = 0; md < 8; ++md)
#pragma unroll
    for (int c = 0; c < 4; ++c) o[md][c] = 0.f;

  if (warp == kC) {
    // ---------------------------------------------------------------- producer
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
              mbar_arrive_expect_tx(&full[s], kRec);
              tma_load_2d(tiles + s * kStage, &tmap, &full[s], 0, (bk * p.H + kvh) * kRecRows);
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
    if (lane == 0) {
      for (int i = max(0, issued - kStages); i < issued; ++i)
        if (!mbar_drain(&full[i % kStages], (i / kStages) & 1)) record_fault(p.fault, KVQ_FAULT_TIMEOUT);
    }
  } else {
    // ---------------------------------------------------------------- consumers
    const int g = p.g;
    // q of head r as bf16/fp16 pairs scaled by 2^-eq (exact): channels [32j, 32j+32), or,
    // keys per token, [16j, 16j+16) and [64+16j, 64+16j+16) (the codes this lane reads)
    float qv[32];
    if (r < g) {
      const uint16_t* qp = static_cast<const uint16_t*>(p.q) +
                           (static_cast<long>(b) * p.Hq + kvh * g + r) * kD;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int ch = kTok ? 64 * (c >> 1) + 16 * j + 8 * (c & 1) : 32 * j + 8 * c;
        const uint4 u = *reinterpret_cast<const uint4*>(qp + ch);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (p.act_fp16) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
            qv[8 * c + 2 * e] = f.x;
            qv[8 * c + 2 * e + 1] = f.y;
          } else {
            qv[8 * c + 2 * e] = bf16lo(w[e]);
            qv[8 * c + 2 * e + 1] = bf16hi(w[e]);
          }
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) qv[e] = 0.f;
    }
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(qv[e]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    // keep |q * scale| well inside fp16 for channel scales up to ~1000
    const int eq = amax > 0.f ? exponent_of(amax) - 5 : 0;
    const float qdown = pow2i(-eq);
    // channel e of this lane is code position e % PW of its word, whose in-place code
    // carries 2^lg: q (and with it q') of that channel is taken down by the same factor
#pragma unroll
    for (int e = 0; e < 32; ++e) qv[e] *= qdown * inv_pow2(CS::lg(e % PW));
    if constexpr (!kTok) {
      // kept in shared memory for the per-block fold (conflict-free: lane-consecutive)
#pragma unroll
      for (int c = 0; c < 8; ++c)
        qvs[(warp * 8 + c) * 32 + lane] = make_float4(qv[4 * c], qv[4 * c + 1], qv[4 * c + 2], qv[4 * c + 3]);
    }
    const float qscale = p.scale_log2 * pow2i(eq);
    // keys per token: q's fp16 fragments and per-group sums, the same for every block;
    // k-step kc < 4 covers group 0, kc >= 4 group 1
    uint32_t qt[kTok ? 8 : 1][2];
    float qg[2][2] = {{0.f, 0.f}, {0.f, 0.f}};        // [group][head 2j, 2j+1]
    if constexpr (kTok) {
      float part[2] = {0.f, 0.f};
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) {
        const int e0 = 2 * PW * (kc / (PW / 2)) + 2 * (kc % (PW / 2));
        qt[kc][0] = pack_f16x2(qv[e0], qv[e0 + PW]);
        qt[kc][1] = pack_f16x2(qv[e0 + 1], qv[e0 + PW + 1]);
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&qt[kc][0]));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&qt[kc][1]));
        // what the MMAs multiply, the in-place factors restored (exact powers of two)
        part[kc >> 2] += (f0.x + f0.y) * static_cast<float>(1 << CS::lg(e0 % PW)) +
                         (f1.x + f1.y) * static_cast<float>(1 << CS::lg((e0 + 1) % PW));
      }
#pragma unroll
      for (int G = 0; G < 2; ++G) {
        part[G] += __shfl_xor_sync(0xffffffffu, part[G], 1);
        part[G] += __shfl_xor_sync(0xffffffffu, part[G], 2);
        qg[G][0] = __shfl_sync(0xffffffffu, part[G], 8 * j);
        qg[G][1] = __shfl_sync(0xffffffffu, part[G], 8 * j + 4);
      }
    }

    float vlim = 0.f, vinv = 0.f;
    // Swizzled offsets of this lane's key and value code words in tile 0 of a stage.  A
    // 4-bit tile (16 tokens of 64 bytes) is one 1024-byte swizzle period, so tile mt reads
    // at the same offsets plus 1024 * mt; a 2-bit tile is half a period, so odd tiles also
    // flip the chunk index's top bit (offset bit 6).  The address arithmetic is done once.
    // Keys: 32 channels per lane, [32j, 32j+32); per token, [16j, 16j+16) of each group.
    int ko[4];
    if constexpr (kTok) {
      ko[0] = swzb4(kRowB * r + 2 * BITS * j);
      ko[1] = swzb4(kRowB * r + kRowB / 2 + 2 * BITS * j);
      ko[2] = swzb4(kRowB * (r + 8) + 2 * BITS * j);
      ko[3] = swzb4(kRowB * (r + 8) + kRowB / 2 + 2 * BITS * j);
    } else {
      ko[0] = swzb4(kRowB * r + 4 * BITS * j);
      ko[1] = swzb4(kRowB * (r + 8) + 4 * BITS * j);
      ko[2] = ko[3] = 0;
    }
    // values: tokens 2j, 2j+1, 2j+8, 2j+9; channels 64G + 8r .. 64G + 8r + 7
    int vo[4][2];
    {
      const int dts[4] = {0, 1, 8, 9};
#pragma unroll
      for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int G = 0; G < 2; ++G)
          vo[t][G] = kOffV + swzb4(kRowB * (2 * j + dts[t]) + (kRowB / 2) * G + BITS * r);
    }
    for (int i = warp; i < npages; i += kC) {
      const int s = i % kStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (i / kStages) & 1))) {
        if (lane == 0) record_fault(p.fault, KVQ_FAULT_TIMEOUT);
        break;
      }
      const uint8_t* st = tiles + s * kStage;
      if (valid[s] == 0) {              // bad block id (counted by the producer): skip it
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        continue;
      }
      // ------------------------------------------------ per-block key scales -> Q' and Zk
      // q'[e] = q[32j+e] * sk[32j+e]; k-step kc uses channel pairs (8w+sp, 8w+sp+4) and
      // (8w+sp+1, 8w+sp+5) with w = kc/2, sp = 2*(kc%2): the pairs the nibble extraction
      // of word w yields.  (Keys per token: nothing per block.)
      uint32_t qh[kTok ? 1 : 8][2], ql[kTok ? 1 : 8][2];
      float ck0 = 0.f, ck1 = 0.f;
      if constexpr (!kTok) {
        uint32_t sw[16], zw[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 a = lds128(st + swzb4(kOffKs + 64 * j + 16 * c));
          const uint4 z = lds128(st + swzb4(kOffKz + 64 * j + 16 * c));
          sw[4 * c] = a.x; sw[4 * c + 1] = a.y; sw[4 * c + 2] = a.z; sw[4 * c + 3] = a.w;
          zw[4 * c] = z.x; zw[4 * c + 1] = z.y; zw[4 * c + 2] = z.z; zw[4 * c + 3] = z.w;
        }
        float qq[32];                   // this lane's q, as stored above
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float4 v4 = qvs[(warp * 8 + c) * 32 + lane];
          qq[4 * c] = v4.x;
          qq[4 * c + 1] = v4.y;
          qq[4 * c + 2] = v4.z;
          qq[4 * c + 3] = v4.w;
        }
        float qs[32];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&sw[e]));
          const float2 q2 = __fmul2_rn(make_float2(qq[2 * e], qq[2 * e + 1]), f);
          qs[2 * e] = q2.x;
          qs[2 * e + 1] = q2.y;
        }
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
          const int e0 = 2 * PW * (kc / (PW / 2)) + 2 * (kc % (PW / 2));
          const float a0 = qs[e0], a1 = qs[e0 + PW], c0 = qs[e0 + 1], c1 = qs[e0 + PW + 1];
          const uint32_t h0 = pack_f16x2(a0, a1), h1 = pack_f16x2(c0, c1);
          const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&h0));
          const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&h1));
          qh[kc][0] = h0;
          qh[kc][1] = h1;
          const float2 r0 = __fadd2_rn(make_float2(a0, a1), make_float2(-f0.x, -f0.y));
          const float2 r1 = __fadd2_rn(make_float2(c0, c1), make_float2(-f1.x, -f1.y));
          ql[kc][0] = pack_f16x2(r0.x, r0.y);
          ql[kc][1] = pack_f16x2(r1.x, r1.y);
        }
        // integer zero points: ck = sum q' zk (subtracted); float: ck = -sum q mk; q and q'
        // carry the in-place factors, so the sums are kept per factor and combined after
        float cp[CS::PER];
#pragma unroll
        for (int k = 0; k < CS::PER; ++k) cp[k] = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 z = __half22float2(*reinterpret_cast<const __half2*>(&zw[e]));
          const int k0 = CS::pos((2 * e) % PW), k1 = CS::pos((2 * e + 1) % PW);
          if constexpr (kFz) {
            cp[k0] = fmaf(-qq[2 * e], z.x, cp[k0]);
            cp[k1] = fmaf(-qq[2 * e + 1], z.y, cp[k1]);
          } else {
            cp[k0] = fmaf(qs[2 * e], z.x, cp[k0]);
            cp[k1] = fmaf(qs[2 * e + 1], z.y, cp[k1]);
          }
        }
        float corr = cp[0];
#pragma unroll
        for (int k = 1; k < CS::PER; ++k) corr = fmaf(cp[k], static_cast<float>(1 << (BITS * k)), corr);
        corr += __shfl_xor_sync(0xffffffffu, corr, 1);
        corr += __shfl_xor_sync(0xffffffffu, corr, 2);
        ck0 = __shfl_sync(0xffffffffu, corr, 8 * j);
        ck1 = __shfl_sync(0xffffffffu, corr, 8 * j + 4);
      }
      // The block's four 16-token tiles in three phases, so that the warp has independent
      // work in flight: the scores of every tile, one softmax update and one V-scale check
      // for the block, then P and P V tile by tile.
      // ------------------------------------------------ S^T = (C - Zk) Q'^T, all tiles
      // sv[mt][0..3]: tokens 16mt + r (heads 2j, 2j+1) and 16mt + r + 8 (heads 2j, 2j+1)
      float sv[kBS / 16][4];
#pragma unroll
      for (int mt = 0; mt < kBS / 16; ++mt) {
        // rows r / r + 8 of the tile: tokens tr0 = 16mt + r and tr1 = tr0 + 8
        const uint8_t* sm = st + R::kTile * mt;
        const int flip = BITS == 2 ? 64 * (mt & 1) : 0;      // 2-bit: odd half-periods
        float s00, s01, s10, s11;
        if constexpr (kTok) {
          // codes of channels [16j, 16j+16) and [64+16j, 64+16j+16): the first BITS/2 words
          // hold group 0, so k-steps 0-3 stay in group 0 and 4-7 in group 1
          uint32_t w0[BITS], w1[BITS];
          if constexpr (BITS == 4) {
            const uint2 k0a = *reinterpret_cast<const uint2*>(sm + ko[0]);
            const uint2 k0b = *reinterpret_cast<const uint2*>(sm + ko[1]);
            const uint2 k1a = *reinterpret_cast<const uint2*>(sm + ko[2]);
            const uint2 k1b = *reinterpret_cast<const uint2*>(sm + ko[3]);
            w0[0] = k0a.x; w0[1] = k0a.y; w0[2] = k0b.x; w0[3] = k0b.y;
            w1[0] = k1a.x; w1[1] = k1a.y; w1[2] = k1b.x; w1[3] = k1b.y;
          } else {
            w0[0] = *reinterpret_cast<const uint32_t*>(sm + (ko[0] ^ flip));
            w0[1] = *reinterpret_cast<const uint32_t*>(sm + (ko[1] ^ flip));
            w1[0] = *reinterpret_cast<const uint32_t*>(sm + (ko[2] ^ flip));
            w1[1] = *reinterpret_cast<const uint32_t*>(sm + (ko[3] ^ flip));
          }
          float sg[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
          uint32_t x0[BITS][CS::NSRC], x1[BITS][CS::NSRC];
#pragma unroll
          for (int w = 0; w < BITS; ++w) {
            code_sources<BITS>(w0[w], x0[w]);
            code_sources<BITS>(w1[w], x1[w]);
          }
#pragma unroll
          for (int kc = 0; kc < 8; ++kc) {
            const int w = kc / (PW / 2), sp = 2 * (kc % (PW / 2));
            const uint32_t a[4] = {code_at<BITS>(x0[w], sp), code_at<BITS>(x1[w], sp),
                                   code_at<BITS>(x0[w], sp + 1), code_at<BITS>(x1[w], sp + 1)};
            mma_f16(sg[kc >> 2], a, qt[kc]);
          }
          // (scale, zero) of tokens tr0 / tr1, groups 0 and 1: fp16 at kOffKs + 8t + 4G
          const int2 ko2 = sz_offsets(kOffKs, mt, r);
          const uint2 z0 = *reinterpret_cast<const uint2*>(st + ko2.x);
          const uint2 z1 = *reinterpret_cast<const uint2*>(st + ko2.y);
          const float2 a00 = __half22float2(*reinterpret_cast<const __half2*>(&z0.x));   // t0 G0
          const float2 a01 = __half22float2(*reinterpret_cast<const __half2*>(&z0.y));   // t0 G1
          const float2 a10 = __half22float2(*reinterpret_cast<const __half2*>(&z1.x));
          const float2 a11 = __half22float2(*reinterpret_cast<const __half2*>(&z1.y));
          s00 = (a00.x * fmaf(sg[0][0], 16777216.f, -a00.y * qg[0][0]) +
                 a01.x * fmaf(sg[1][0], 16777216.f, -a01.y * qg[1][0])) * qscale;
          s01 = (a00.x * fmaf(sg[0][1], 16777216.f, -a00.y * qg[0][1]) +
                 a01.x * fmaf(sg[1][1], 16777216.f, -a01.y * qg[1][1])) * qscale;
          s10 = (a10.x * fmaf(sg[0][2], 16777216.f, -a10.y * qg[0][0]) +
                 a11.x * fmaf(sg[1][2], 16777216.f, -a11.y * qg[1][0])) * qscale;
          s11 = (a10.x * fmaf(sg[0][3], 16777216.f, -a10.y * qg[0][1]) +
                 a11.x * fmaf(sg[1][3], 16777216.f, -a11.y * qg[1][1])) * qscale;
        } else {
          // codes of channels [32j, 32j+32): BITS words per row
          uint32_t w0[BITS], w1[BITS];
          if constexpr (BITS == 4) {
            const uint4 k0 = lds128(sm + ko[0]);
            const uint4 k1 = lds128(sm + ko[1]);
            w0[0] = k0.x; w0[1] = k0.y; w0[2] = k0.z; w0[3] = k0.w;
            w1[0] = k1.x; w1[1] = k1.y; w1[2] = k1.z; w1[3] = k1.w;
          } else {
            const uint2 k0 = *reinterpret_cast<const uint2*>(sm + (ko[0] ^ flip));
            const uint2 k1 = *reinterpret_cast<const uint2*>(sm + (ko[1] ^ flip));
            w0[0] = k0.x; w0[1] = k0.y;
            w1[0] = k1.x; w1[1] = k1.y;
          }
          float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
          uint32_t x0[BITS][CS::NSRC], x1[BITS][CS::NSRC];
#pragma unroll
          for (int w = 0; w < BITS; ++w) {
            code_sources<BITS>(w0[w], x0[w]);
            code_sources<BITS>(w1[w], x1[w]);
          }
#pragma unroll
          for (int kc = 0; kc < 8; ++kc) {
            const int w = kc / (PW / 2), sp = 2 * (kc % (PW / 2));
            const uint32_t a[4] = {code_at<BITS>(x0[w], sp), code_at<BITS>(x1[w], sp),
                                   code_at<BITS>(x0[w], sp + 1), code_at<BITS>(x1[w], sp + 1)};
            mma_f16(sa, a, qh[kc]);
            mma_f16(sb, a, ql[kc]);
          }
          const float2 two24 = make_float2(16777216.f, 16777216.f), nck = make_float2(-ck0, -ck1);
          const float2 qsc2 = make_float2(qscale, qscale);
          const float2 t0 = __fmul2_rn(__ffma2_rn(__fadd2_rn(make_float2(sa[0], sa[1]), make_float2(sb[0], sb[1])),
                                                  two24, nck), qsc2);
          const float2 t1 = __fmul2_rn(__ffma2_rn(__fadd2_rn(make_float2(sa[2], sa[3]), make_float2(sb[2], sb[3])),
                                                  two24, nck), qsc2);
          s00 = t0.x;
          s01 = t0.y;
          s10 = t1.x;
          s11 = t1.y;
        }
        sv[mt][0] = s00;
        sv[mt][1] = s01;
        sv[mt][2] = s10;
        sv[mt][3] = s11;
      }
      // ------------------------------------------------ softmax (log2 domain), per block
      {
        float mx0 = fmaxf(sv[0][0], sv[0][2]), mx1 = fmaxf(sv[0][1], sv[0][3]);
#pragma unroll
        for (int mt = 1; mt < kBS / 16; ++mt) {
          mx0 = fmaxf(mx0, fmaxf(sv[mt][0], sv[mt][2]));
          mx1 = fmaxf(mx1, fmaxf(sv[mt][1], sv[mt][3]));
        }
        if (__any_sync(0xffffffffu, mx0 > m[0] + kRescale4 || mx1 > m[1] + kRescale4)) {
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
          }
          const float mn0 = fmaxf(m[0], mx0), mn1 = fmaxf(m[1], mx1);
          const float c0 = m[0] == -INFINITY ? 0.f : ex2(m[0] - mn0);
          const float c1 = m[1] == -INFINITY ? 0.f : ex2(m[1] - mn1);
          m[0] = mn0;
          m[1] = mn1;
          l[0] *= c0;
          l[1] *= c1;
          cz[0][0] *= c0; cz[1][0] *= c0; cz[0][1] *= c1; cz[1][1] *= c1;
#pragma unroll
          for (int md = 0; md < 8; ++md) {
            o[md][0] *= c0;
            o[md][1] *= c1;
            o[md][2] *= c0;
            o[md][3] *= c1;
          }
        }
      }
      // ------------------------------------------------ value scales of the block
      // vsz for token t, group G: (scale, zero) fp16 at kOffVsz + 8t + 4G (read again for
      // each tile below)
      {
        // the largest scale by packed half maxima (the high halves, zero points, unused)
        __half2 vm2 = __halves2half2(__ushort_as_half(0), __ushort_as_half(0));
#pragma unroll
        for (int mt = 0; mt < kBS / 16; ++mt) {
          const int2 vo2 = sz_offsets(kOffVsz, mt, r);
          const uint2 vz0 = *reinterpret_cast<const uint2*>(st + vo2.x);
          const uint2 vz1 = *reinterpret_cast<const uint2*>(st + vo2.y);
          const uint32_t w4[4] = {vz0.x, vz0.y, vz1.x, vz1.y};
#pragma unroll
          for (int k = 0; k < 4; ++k) vm2 = __hmax2(vm2, *reinterpret_cast<const __half2*>(&w4[k]));
        }
        float vm = __low2float(vm2);
        if (__any_sync(0xffffffffu, vm >= vlim)) {
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, off));
          if (vm > 0.f) {
            const int e = exponent_of(vm);
            if (e > ev) {
              if (ev != INT_MIN) {
                const float down = pow2i(ev - e);
                cz[0][0] *= down; cz[0][1] *= down; cz[1][0] *= down; cz[1][1] *= down;
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
      }
      const float base0 = m[0] == -INFINITY ? 0.f : m[0], base1 = m[1] == -INFINITY ? 0.f : m[1];
#pragma unroll
      for (int mt = 0; mt < kBS / 16; ++mt) {
        const uint8_t* sm = st + R::kTile * mt;
        const int flip = BITS == 2 ? 64 * (mt & 1) : 0;
        const float2 nb = make_float2(-base0, -base1);
        const float2 x0 = __fadd2_rn(make_float2(sv[mt][0], sv[mt][1]), nb);
        const float2 x1 = __fadd2_rn(make_float2(sv[mt][2], sv[mt][3]), nb);
        const float p00 = ex2(x0.x), p01 = ex2(x0.y), p10 = ex2(x1.x), p11 = ex2(x1.y);
        {
          const float2 l2 = __fadd2_rn(make_float2(l[0], l[1]),
                                       __fadd2_rn(make_float2(p00, p01), make_float2(p10, p11)));
          l[0] = l2.x;
          l[1] = l2.y;
        }
        const int2 vo2 = sz_offsets(kOffVsz, mt, r);
        const uint2 vz0 = *reinterpret_cast<const uint2*>(st + vo2.x);
        const uint2 vz1 = *reinterpret_cast<const uint2*>(st + vo2.y);
        const uint32_t sz00 = vz0.x, sz01 = vz0.y, sz10 = vz1.x, sz11 = vz1.y;
        float vs[2][2] = {{__half2float(__ushort_as_half(sz00 & 0xFFFF)), __half2float(__ushort_as_half(sz01 & 0xFFFF))},
                          {__half2float(__ushort_as_half(sz10 & 0xFFFF)), __half2float(__ushort_as_half(sz11 & 0xFFFF))}};
        uint32_t pbh[2][2], pbl[2][2];
#pragma unroll
        for (int G = 0; G < 2; ++G) {
          const float w0g = vs[0][G] * vinv, w1g = vs[1][G] * vinv;
          // (q00, q01): token tr0, heads 2j / 2j+1; (q10, q11): token tr1
          const float2 qa = __fmul2_rn(make_float2(p00, p01), make_float2(w0g, w0g));
          const float2 qb = __fmul2_rn(make_float2(p10, p11), make_float2(w1g, w1g));
          const float z0 = __half2float(__ushort_as_half((G ? sz01 : sz00) >> 16));
          const float z1 = __half2float(__ushort_as_half((G ? sz11 : sz10) >> 16));
          float2 c2 = make_float2(cz[G][0], cz[G][1]);
          if constexpr (kFz) {
            // the minima enter unscaled: cz = -vinv * sum_t p mv
            const float nz0 = -vinv * z0, nz1 = -vinv * z1;
            c2 = __ffma2_rn(make_float2(p00, p01), make_float2(nz0, nz0),
                            __ffma2_rn(make_float2(p10, p11), make_float2(nz1, nz1), c2));
          } else {
            c2 = __ffma2_rn(qa, make_float2(z0, z0), __ffma2_rn(qb, make_float2(z1, z1), c2));
          }
          cz[G][0] = c2.x;
          cz[G][1] = c2.y;
          const uint32_t h0 = pack_f16x2(qa.x, qa.y), h1 = pack_f16x2(qb.x, qb.y);
          const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&h0));
          const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&h1));
          const float2 d0 = __fadd2_rn(qa, make_float2(-f0.x, -f0.y));
          const float2 d1 = __fadd2_rn(qb, make_float2(-f1.x, -f1.y));
          const uint32_t e0 = pack_f16x2(d0.x, d0.y), e1 = pack_f16x2(d1.x, d1.y);
          pbh[G][0] = movmatrix_trans(h0);
          pbh[G][1] = movmatrix_trans(h1);
          pbl[G][0] = movmatrix_trans(e0);
          pbl[G][1] = movmatrix_trans(e1);
        }
        // ------------------------------------------------ O^T += (C - Zv)^T P'^T
        // tile md: channel group G = md/4; rows r / r+8 <-> d = 64G + 8r + 2(md%4) / +1.
        // 4-bit: byte md%4 of the word holding channels 64G + 8r .. +7 of a token, its low /
        // high nibble.  2-bit: those channels are 2 bytes; byte (md%4)/2, crumbs 2(md%2), +1.
        // A byte permute puts the byte of tokens (2j, 2j+1) -- and of (2j+8, 2j+9) -- into the
        // two 16-bit halves of a register, where a shift and a mask leave the codes.
        uint32_t vwd[4][2];
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
          for (int G = 0; G < 2; ++G) {
            if constexpr (BITS == 4)
              vwd[t][G] = *reinterpret_cast<const uint32_t*>(sm + vo[t][G]);
            else
              vwd[t][G] = *reinterpret_cast<const uint16_t*>(sm + (vo[t][G] ^ flip));
          }
#pragma unroll
        for (int md = 0; md < 8; ++md) {
          const int G = md >> 2;
          uint32_t Y, Z;
          int sh;
          if constexpr (BITS == 4) {
            const int k = md & 3;
            const uint32_t sel = static_cast<uint32_t>(k | (k << 4) | ((4 + k) << 8) | ((4 + k) << 12));
            Y = prmt(vwd[0][G], vwd[1][G], sel);   // bytes (ta_k, ta_k, tb_k, tb_k)
            Z = prmt(vwd[2][G], vwd[3][G], sel);
            sh = 0;
          } else {
            const int k = (md >> 1) & 1;
            const uint32_t sel = static_cast<uint32_t>(k | (k << 4) | ((2 + k) << 8) | ((2 + k) << 12));
            Y = prmt(vwd[0][G] | (vwd[1][G] << 16), 0u, sel);
            Z = prmt(vwd[2][G] | (vwd[3][G] << 16), 0u, sel);
            sh = 4 * (md & 1);
          }
          // codes masked in place: rows r carry 2^sh, rows r + 8 2^(sh + BITS) (undone at
          // the end; the products and sums are exact power-of-two multiples of the shifted ones)
          constexpr uint32_t m4 = R::kMask;
          const uint32_t a[4] = {Y & (m4 << sh), Y & (m4 << (sh + BITS)), Z & (m4 << sh),
                                 Z & (m4 << (sh + BITS))};
          mma_f16(o[md], a, pbh[G]);
          mma_f16(o[md], a, pbl[G]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l[0] += __shfl_xor_sync(0xffffffffu, l[0], off);
      l[1] += __shfl_xor_sync(0xffffffffu, l[1], off);
#pragma unroll
      for (int G = 0; G < 2; ++G) {
        cz[G][0] += __shfl_xor_sync(0xffffffffu, cz[G][0], off);
        cz[G][1] += __shfl_xor_sync(0xffffffffu, cz[G][1], off);
      }
    }
#pragma unroll
    for (int md = 0; md < 8; ++md) {
      const int G = md >> 2;
      // 2^24 (the subnormal codes) over the in-place factor of the tile's rows
      const int sh = BITS == 4 ? 0 : 4 * (md & 1);
      const float fr = 16777216.f * inv_pow2(sh), fr8 = 16777216.f * inv_pow2(sh + BITS);
      o[md][0] = fmaf(o[md][0], fr, -cz[G][0]);
      o[md][1] = fmaf(o[md][1], fr, -cz[G][1]);
      o[md][2] = fmaf(o[md][2], fr8, -cz[G][0]);
      o[md][3] = fmaf(o[md][3], fr8, -cz[G][1]);
    }
  }
  __syncthreads();
  griddep_launch_dependents();   // the split reduce may be scheduled (it waits for this grid)

  float* red_o = reinterpret_cast<float*>(tiles);           // [warp][head][D]
  float* red_ml = red_o + kC * 8 * kD;                      // [warp][head][2]
  if (warp < kC) {
    const float vmul = ev == INT_MIN ? 0.f : pow2i(ev);
#pragma unroll
    for (int md = 0; md < 8; ++md) {
      const int d0 = 64 * (md >> 2) + 8 * r + 2 * (md & 3);
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
  for (int e = threadIdx.x; e < p.g * kD; e += kT) {
    const int h = e / kD, d = e % kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kC; ++w) M = fmaxf(M, red_ml[(w * 8 + h) * 2]);
    float Lsum = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kC; ++w) {
      const float mw = red_ml[(w * 8 + h) * 2];
      const float f = (M == -INFINITY || mw == -INFINITY) ? 0.f : exp2f(mw - M);
      Lsum += red_ml[(w * 8 + h) * 2 + 1] * f;
      O += red_o[(w * 8 + h) * kD + d] * f;
    }
    store_partial_or_output(p, b, kvh * p.g + h, split, d, M, Lsum, O);
  }
  // launched as the ring kernel's dependent: this grid completes only after that one, so the
  // split reduce (this grid's dependent, waiting for it) sees both kernels' partials
  griddep_wait();
}

}  // namespace

bool int4_mma_supported(const Geometry& g, int group) {
  const bool rec = (g.cache_dtype == KVQ_DTYPE_INT4 && g.record == Rec<4>::kRec) ||
                   (g.cache_dtype == KVQ_DTYPE_INT2 && g.record == Rec<2>::kRec);
  return rec && g.D == kD && g.bs == kBS && group >= 3 && group <= 8;
}

namespace {

template <int BITS>
cudaError_t launch_bits(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s) {
  using R = Rec<BITS>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    // two CTAs per SM (registers): both rings need the maximum shared-memory carveout
    const void* fns[3] = {reinterpret_cast<const void*>(decode_int4_kernel<kKivi, BITS>),
                          reinterpret_cast<const void*>(decode_int4_kernel<kKiviMin, BITS>),
                          reinterpret_cast<const void*>(decode_int4_kernel<kPerToken, BITS>)};
    for (const void* f : fns) {
      if (attr_err == cudaSuccess)
        attr_err = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, R::kBytes);
      if (attr_err == cudaSuccess)
        attr_err = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                                        cudaSharedmemCarveoutMaxShared);
    }
  });
  if (attr_err != cudaSuccess) return attr_err;
  CUtensorMap tm;
  const long rows = static_cast<long>(a.geo.NB) * a.geo.H * R::kRecRows;
  if (!make_pages_map(&tm, a.c->pages, rows, R::kRecRows)) return cudaErrorInvalidValue;
  // page splits only; the ring split is launched separately
  const dim3 grid(p.ring_split, a.geo.H, a.batch);
  switch (a.geo.scale_mode) {
    // launched as the ring kernel's dependent (see the kernel's last lines)
    case KVQ_SCALE_KIVI: return launch_dependent(decode_int4_kernel<kKivi, BITS>, grid, dim3(kT), R::kBytes, s, p, tm);
    case KVQ_SCALE_KIVI_FLOAT_ZERO:
      return launch_dependent(decode_int4_kernel<kKiviMin, BITS>, grid, dim3(kT), R::kBytes, s, p, tm);
    case KVQ_SCALE_INT4_PER_TOKEN:
      return launch_dependent(decode_int4_kernel<kPerToken, BITS>, grid, dim3(kT), R::kBytes, s, p, tm);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_decode_int4(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s) {
  return a.geo.cache_dtype == KVQ_DTYPE_INT2 ? launch_bits<2>(a, p, s) : launch_bits<4>(a, p, s);
}

}  // namespace kvq
