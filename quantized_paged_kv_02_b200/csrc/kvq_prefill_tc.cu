// Chunked-prefill attention over the quantized paged cache on the 5th-generation tensor
// cores (tcgen05.mma, accumulators in tensor memory), for head_dim 128: INT8, FP8 E4M3,
// BF16 and FP16 caches with block size 16, and the INT4 / 2-bit group caches (block 64, the
// newest tokens in the residual ring).
//
// A CTA owns one tile of 128 query rows of one (sequence, kv head): 128 / g query tokens x
// the g query heads that share the kv head (row r = token r / g, head r % g), and walks the
// causal window of its last query in blocks of 128 cached tokens (8 pages).  Each page is
// dequantized ONCE into shared memory for all 128 rows, instead of once per query token.
// Eighteen warps, each role waiting only on what it consumes (mbarriers, every wait
// bounded):
//
//   warp 8      producer: the table entries of a block's pages, then one bulk copy per page
//               record (K codes, V codes, per-token scales) into a ring of raw stages that
//               turns over a block at a time (one full and one empty barrier per block);
//               for 16-bit caches, whose rows are the tiles' values, four TMA tensor copies
//               per page straight into a K / V tile buffer (128-byte swizzle), no raw ring;
//   warps 10-13 K converters and warps 14-17 V converters: codes -> 16-bit tiles in the
//               tensor cores' 128-byte-swizzled layout (INT8 through the exact 1024-magic,
//               E4M3 by the hardware conversion), K as the K-major B operand of S = Q K^T
//               and V as the MN-major B operand of O = P V, plus the per-token multipliers
//               (in four slots of their own) and V scales (for 16-bit caches only these,
//               and zeros over the V rows outside the window); K and V tiles have their own
//               buffer counts (a K tile is free once S has read it, a V tile after P V);
//   warp 9      MMA issuer: S_j = Q K_j^T (M 128, N 128 tokens, K 128) into one of two TMEM
//               score buffers, then O += P_{j-1} V_{j-1} (N 128 channels, K 128 tokens);
//   warps 0-7   softmax: the two warps of a TMEM lane quarter share its 32 query rows,
//               64 score columns each; they read the scores from TMEM (the next 16 columns'
//               load in flight while the current ones are used), scale them (per-token K
//               scale, softmax scale, log2 e), mask the causal boundary, agree on the row
//               maximum through a per-quarter barrier (re-based only when a score exceeds the
//               running maximum by 2^8), keep the row sum, fold the per-token V scale into P
//               and write P back over its scores as fp16 (bf16 for bf16 caches) hi + lo
//               halves, the A operand of the P V MMA.
//
// Q lives in TMEM too (written once by the softmax warps), so shared memory holds only the
// K / V tiles and the raw ring.  The contraction is exact in the codes: for INT8 / FP8 the
// K and V tiles hold the codes themselves (exact in fp16), q is an exact fp16 copy of the
// bf16 activations scaled by a power of two (per-channel K scales fold into q as a hi + lo
// pair), and P's hi + lo halves keep 22 bits.  For INT4 / 2-bit caches the dequantized
// value (code - zero) * scale (at most 15 significant bits) is split exactly into bf16 hi +
// lo tiles; S takes both (and both halves of q when activations are fp16), P V takes
// P hi V hi + P hi V lo + P lo V hi.  Scores, softmax and O accumulate in fp32.
// Chunked prefill is one of the techniques [P-prod] "为什么长上下文更需要 KV Cache
// Quantization" lists beside cache quantization; dequantization inside attention is the
// design of [P-vLLM] "PagedAttention与KV Cache量化协同工作原理".
#include <cudaTypedefs.h>

#include <climits>
#include <mutex>
#include <type_traits>

#include "kvq_decode_common.cuh"
#include "kvq_ptx.cuh"
#include "kvq_tc.cuh"

namespace kvq {
namespace {

constexpr int kRows = 128;          // query rows per tile (MMA M)
constexpr int kBlk = 128;           // cached tokens per block (MMA N of S, K of P V)
constexpr int kD = 128;
constexpr int kPfThreads = 576;     // warps 0-7 softmax, 8 producer, 9 MMA, 10-13 K converters,
                                    // 14-17 V converters
constexpr int kSoftWarps = 8, kProdWarp = 8, kMmaWarp = 9, kConvWarp0 = 10;
constexpr int kNBMax = 3;           // K / V tile buffers at most
constexpr int kNQ = 4;              // slots of the per-token K multipliers (block j: slot j % 4)
constexpr int kTile = 32768;        // 128 x 128 16-bit elements
constexpr float kRescalePf = 8.f;   // log2 headroom before the running max is re-based
// TMEM columns: scores / P of block j in [128 (j % 2), +128), O in [256, 384), Q from 384
constexpr uint32_t kTmemCols = 512, kTmO = 256, kTmQ = 384;

// Code width and tile type per cache dtype: 8-bit codes and fp16 caches use fp16 tiles,
// bf16 caches and the low-bit caches (whose exact values need a bf16 hi + lo pair) bf16.
template <int CD> struct PfCode;
template <> struct PfCode<KVQ_DTYPE_INT8> { static constexpr int BITS = 8; static constexpr bool kBf16 = false; };
template <> struct PfCode<KVQ_DTYPE_FP8_E4M3> { static constexpr int BITS = 8; static constexpr bool kBf16 = false; };
template <> struct PfCode<KVQ_DTYPE_FP16> { static constexpr int BITS = 16; static constexpr bool kBf16 = false; };
template <> struct PfCode<KVQ_DTYPE_BF16> { static constexpr int BITS = 16; static constexpr bool kBf16 = true; };
template <> struct PfCode<KVQ_DTYPE_INT4> { static constexpr int BITS = 4; static constexpr bool kBf16 = true; };
template <> struct PfCode<KVQ_DTYPE_INT2> { static constexpr int BITS = 2; static constexpr bool kBf16 = true; };

template <int CD, bool PT>
struct PfLayout {
  static constexpr int BITS = PfCode<CD>::BITS;
  static constexpr bool LB = BITS < 8;                     // group codes + residual ring
  static constexpr int BS = LB ? 64 : 16;
  static constexpr int PPB = kBlk / BS;                    // pages per block
  static constexpr int ROWB = kD * BITS / 8;
  static constexpr int OFF_V = BS * ROWB;
  static constexpr int OFF_S = 2 * BS * ROWB;
  // scales: per-token float32 K and V (PT), or the group parameters (K 4 D bytes, V
  // (scale, zero) per token and 64-channel group)
  static constexpr int SCALES = LB ? 4 * kD + BS * (kD / 64) * 4 : (PT ? 8 * BS : 0);
  static constexpr int REC = (OFF_S + SCALES + 127) / 128 * 128;
  static constexpr int KP = LB ? 2 : 1;                    // K tiles whose sum is K (hi, lo)
  static constexpr int VP = LB ? 2 : 1;
  // K / V tile buffers: a K tile is free once S has read it, a V tile only after P V.  16-bit
  // caches (no raw ring) keep three of each; INT8 one K and three V tiles beside the
  // two-block raw ring (measured 1% faster than two and two), E4M3 two and two (0.4%
  // faster than one and three)
  static constexpr bool I8 = CD == KVQ_DTYPE_INT8;
  static constexpr int NBK = LB ? 1 : (BITS == 16 ? 3 : (I8 ? 1 : 2));
  static constexpr int NBV = LB ? 1 : (BITS == 16 || I8 ? 3 : 2);
  static constexpr int NB = NBV;                           // 16-bit caches: NBK == NBV
  static constexpr int RS = LB ? 4 : (BITS == 8 ? 16 : 8); // raw ring stages (pages)
  // the ring turns over in groups of one block's pages, each group with one full and one
  // empty barrier: the producer issues a block's pages together and the converters wait
  // once per block
  static constexpr int RG = RS / PPB;
  // 16-bit caches: the rows are the tiles' values, so the producer copies them with TMA
  // straight into the tile buffers (128-byte swizzle) and no raw ring is needed
  static constexpr bool DIRECT = BITS == 16;
  static constexpr int RAWB = DIRECT ? 0 : RS * REC;       // bytes of the raw ring
  static constexpr int NPOK = DIRECT ? NB * PPB : RS;      // page-valid flags: by ring slot,
                                                           // or by (tile buffer, page)
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = NBK * KP * kTile;
  static constexpr int RAW_OFF = V_OFF + NBV * VP * kTile;
  static constexpr int KQ_OFF = RAW_OFF + RAWB;            // float [kNQ][128]: K multiplier
  static constexpr int VS_OFF = KQ_OFF + kNQ * kBlk * 4;   // float [NBV][128]: V scale
  static constexpr int XM_OFF = VS_OFF + NBV * kBlk * 4;    // float [3][2][128]: row maxima of
                                                           // the two halves (by block parity),
                                                           // then the row sums
  static constexpr int MISC_OFF = XM_OFF + 3 * 2 * kRows * 4;  // per (buffer, converter warp)
                                                               // vmax and bad-token counts; flags
  static constexpr int BAR_OFF = MISC_OFF + 192;
  // raw_full, raw_empty [RG]; k_full [NBK]; v_full, vfree [NBV]; s_full, p_full, pv_done [2];
  // q_ready; fin; xch [4]; kq_full, kqfree [kNQ]; tile_full [NB] (16-bit caches)
  static constexpr int NBARS = 2 * RG + NBK + 2 * NBV + 6 + 2 + 4 + 2 * kNQ + NB;
  static constexpr int BYTES = 1024 + BAR_OFF + NBARS * 8 + NPOK * 4 + 64;
  static_assert(BYTES <= 227 * 1024, "fits the shared memory of one CTA");
  static_assert(BYTES > 114 * 1024, "one CTA per SM, so TMEM allocation never waits on a peer");
  static_assert(RS % PPB == 0 && RG >= 1, "the raw ring holds whole blocks");
  static_assert(PPB <= 32, "one producer lane per page of a block");
  static_assert(REC % 16 == 0, "bulk copies move multiples of 16 bytes");
  static_assert(NBV <= kNBMax && NBK <= kNQ, "scale arrays, multiplier slots");
  static_assert(!DIRECT || NBK == NBV, "16-bit caches fill K and V of a buffer together");
};

struct PfShared {
  uint64_t* raw_full;
  uint64_t* raw_empty;
  uint64_t* k_full;
  uint64_t* v_full;
  uint64_t* s_full;
  uint64_t* p_full;
  uint64_t* vfree;
  uint64_t* pv_done;                // [2]: P V of block j commits to pv_done[j % 2]
  uint64_t* q_ready;
  uint64_t* fin;                    // the MMA issuer's final commit
  uint64_t* xch;                    // [4]: the two softmax warps of a TMEM lane quarter
  uint64_t* kq_full;                // [kNQ]: a slot of K multipliers (and bad-token counts) written
  uint64_t* kqfree;                 // [kNQ]: the softmax is done with a slot of K multipliers
  uint64_t* tile_full;              // [NB]: 16-bit caches: a block's K and V rows have landed
  float* xmax;
  int* page_ok;
  float* kq;                        // [NB][128] K multiplier of each token (NaN: bad page)
  float* vs;                        // [NB][128] V scale of each token
  float* vmax;                      // [NB][4] largest V scale seen by each converter warp
  int* nbad;                        // [NB][4] bad-page tokens seen by each converter warp
  float* qscale;
  uint32_t* tmem;
  volatile int* abort;
};

// Bounded wait that also gives up when another role has aborted.  After a first test the
// thread sleeps in the barrier (up to 20 us per try, woken by the phase completing), so the
// roles that wait (producer, MMA issuer, converters) leave the issue slots to the softmax
// warps that share their SM sub-partitions.
__device__ __forceinline__ bool pf_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_sleep(bar, parity, 20000u)) {
    if (*abort) return false;
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}

__device__ __forceinline__ void pf_fail(const DecodeParams& p, volatile int* abort) {
  record_fault(p.fault, KVQ_FAULT_TIMEOUT);
  *abort = 1;
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Eight INT8 codes -> eight fp16 values (exact), packed low element first.
__device__ __forceinline__ uint4 i8x8_to_f16(uint2 w) {
  const uint32_t a = w.x ^ 0x80808080u, b = w.y ^ 0x80808080u;
  return make_uint4(i8x2_to_f16x2(a, kLoPair), i8x2_to_f16x2(a, kHiPair), i8x2_to_f16x2(b, kLoPair),
                    i8x2_to_f16x2(b, kHiPair));
}

__device__ __forceinline__ uint4 e4m3x8_to_f16(uint2 w) {
  return make_uint4(e4m3x2_to_f16x2(w.x & 0xFFFFu), e4m3x2_to_f16x2(w.x >> 16),
                    e4m3x2_to_f16x2(w.y & 0xFFFFu), e4m3x2_to_f16x2(w.y >> 16));
}

// Swizzled byte offset of 16-byte chunk c (8 elements, c < 16) of row t in a 128 x 128 tile.
__device__ __forceinline__ uint32_t tile_off(int t, int c) {
  return static_cast<uint32_t>((c >> 3) * 16384 + t * 128 + (((c & 7) ^ (t & 7)) << 4));
}

// hi + lo split of two fp32 values into 16-bit pairs (fp16, or bf16 for bf16 caches).
template <bool BF>
__device__ __forceinline__ void split2(float2 w, uint32_t& hi, uint32_t& lo) {
  float2 h;
  if constexpr (BF) {
    hi = pack_bf16x2(w.x, w.y);
    h = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hi));
  } else {
    hi = pack_f16x2(w.x, w.y);
    h = __half22float2(*reinterpret_cast<const __half2*>(&hi));
  }
  const float2 r = __fadd2_rn(w, make_float2(-h.x, -h.y));
  lo = BF ? pack_bf16x2(r.x, r.y) : pack_f16x2(r.x, r.y);
}
template <bool BF>
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  split2<BF>(make_float2(a, b), hi, lo);
}

// Largest of three values (one three-input max on sm_100).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ void st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7])
               : "memory");
}

// Dequantized value of one low-bit code: (code - zero) * scale, or code * scale + minimum
// (float zero point); exact in float32 for the integer zero point (<= 15 significant bits).
__device__ __forceinline__ float lb_value(int code, float s, float z, bool fz) {
  return fz ? fmaf(static_cast<float>(code), s, z) : static_cast<float>(code - static_cast<int>(z)) * s;
}

// Eight values -> bf16 hi and lo chunks (value = hi + lo, exactly for <= 16 significant bits).
__device__ __forceinline__ void split8(const float* v, uint4& hi, uint4& lo) {
  split2<true>(v[0], v[1], hi.x, lo.x);
  split2<true>(v[2], v[3], hi.y, lo.y);
  split2<true>(v[4], v[5], hi.z, lo.z);
  split2<true>(v[6], v[7], hi.w, lo.w);
}

// Dense caches, converter thread (c, rr) = (ct % 16, ct / 16): the K (or V) rows of every
// page of block j -> tile buffer kb, chunk c of rows rr and rr + 8 of each page; all loads
// first, then conversions and stores.  Thread ct also writes token ct's multiplier (K:
// softmax scale x K scale, NaN for a bad page; V: the V scale).  Returns 1 for a bad token
// of K (a visible position on a page that failed its table check), token ct's V scale for V.
template <int CD, bool PT>
__device__ __forceinline__ float dense_part(uint8_t* smem, const PfShared& sh, int j, int kb, bool isv,
                                            int ct, int npg, int pmax, float& qsc, bool& have_q) {
  using L = PfLayout<CD, PT>;
  constexpr int PPB = L::PPB, BS = L::BS;
  using RawT = typename std::conditional<L::BITS == 8, uint2, uint4>::type;
  const int c = ct & 15, rr = ct >> 4;
  RawT w[PPB][2];
  uint32_t pok = 0;
#pragma unroll
  for (int pp = 0; pp < PPB; ++pp) {
    const int k = j * PPB + pp, s = k % L::RS;
    if (k < npg && sh.page_ok[s]) pok |= 1u << pp;
    const uint8_t* src = smem + L::RAW_OFF + s * L::REC + (isv ? L::OFF_V : 0);
#pragma unroll
    for (int h = 0; h < 2; ++h)
      w[pp][h] = *reinterpret_cast<const RawT*>(src + (rr + 8 * h) * L::ROWB + static_cast<int>(sizeof(RawT)) * c);
  }
  // every page present and every position visible to some query: no per-row tests
  const bool whole = pok == (1u << PPB) - 1u && j * kBlk + kBlk - 1 <= pmax;
  // row t of the tile: t & 7 == rr & 7 for all of this thread's rows, so the swizzled chunk is
  // the same for all; only the row offset changes
  uint8_t* tile = smem + (isv ? L::V_OFF : L::K_OFF) + kb * kTile + tile_off(rr, c) - rr * 128;
  auto cvt = [&](const RawT& r) -> uint4 {
    if constexpr (L::BITS == 8) return CD == KVQ_DTYPE_INT8 ? i8x8_to_f16(r) : e4m3x8_to_f16(r);
    else return r;
  };
  if (whole) {
#pragma unroll
    for (int pp = 0; pp < PPB; ++pp)
#pragma unroll
      for (int h = 0; h < 2; ++h) *reinterpret_cast<uint4*>(tile + (pp * BS + rr + 8 * h) * 128) = cvt(w[pp][h]);
  } else {
#pragma unroll
    for (int pp = 0; pp < PPB; ++pp)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = pp * BS + rr + 8 * h;
        const bool keep = ((pok >> pp) & 1u) && j * kBlk + t <= pmax;
        *reinterpret_cast<uint4*>(tile + t * 128) = keep ? cvt(w[pp][h]) : make_uint4(0, 0, 0, 0);
      }
  }
  const int t = ct, pp = t >> 4, row = t & 15, k = j * PPB + pp, pos = j * kBlk + t;
  const bool have = k < npg, pk = (pok >> pp) & 1u;
  const bool valid = pk && pos <= pmax;
  const float* sc = reinterpret_cast<const float*>(smem + L::RAW_OFF + (k % L::RS) * L::REC + L::OFF_S);
  if (!isv) {
    if (!have_q) {
      // the first block: q's scale (the tile above is converted meanwhile); a wait that
      // runs out leaves the multipliers at 0 and the abort flag stops every role
      if (pf_wait(sh.q_ready, 0, sh.abort)) qsc = *sh.qscale;
      else *sh.abort = 1;
      have_q = true;
    }
    float ks = 1.f;
    if constexpr (PT) ks = sc[row];
    // positions past the tile's last query are never visible: their multiplier is unused
    const bool badtok = have && !pk && pos <= pmax;
    sh.kq[(j % kNQ) * kBlk + t] = valid ? qsc * ks : (badtok ? __uint_as_float(0x7fffffffu) : 0.f);
    return badtok ? 1.f : 0.f;
  }
  float vv = 1.f;
  if constexpr (PT) vv = sc[BS + row];
  vv = valid ? vv : 0.f;
  sh.vs[kb * kBlk + t] = vv;
  return vv;
}

// 16-bit caches, thread ct = token ct of block j, whose rows the producer copied into tile
// buffer kb: K: the token's multiplier (softmax scale, NaN for a bad page, 0 past the
// window); V: its scale (1 or 0) and, for a token outside the window or on a page that was
// not copied, zeros over its row of the V tile (whatever the buffer held must not reach
// P V; a masked score never does).  Returns as dense_part.
template <int CD, bool PT>
__device__ __forceinline__ float direct_part(uint8_t* smem, const PfShared& sh, int j, int kb, bool isv,
                                             int ct, int npg, int pmax, float& qsc, bool& have_q) {
  using L = PfLayout<CD, PT>;
  constexpr int BS = L::BS;
  const int t = ct, pp = t / BS, k = j * L::PPB + pp, pos = j * kBlk + t;
  const bool have = k < npg, pk = have && sh.page_ok[kb * L::PPB + pp];
  const bool valid = pk && pos <= pmax;
  if (!isv) {
    if (!have_q) {
      if (pf_wait(sh.q_ready, 0, sh.abort)) qsc = *sh.qscale;
      else *sh.abort = 1;
      have_q = true;
    }
    const bool badtok = have && !pk && pos <= pmax;
    sh.kq[(j % kNQ) * kBlk + t] = valid ? qsc : (badtok ? __uint_as_float(0x7fffffffu) : 0.f);
    return badtok ? 1.f : 0.f;
  }
  if (!valid) {
    uint8_t* tile = smem + L::V_OFF + kb * kTile;
#pragma unroll
    for (int c = 0; c < 16; ++c) *reinterpret_cast<uint4*>(tile + tile_off(t, c)) = make_uint4(0, 0, 0, 0);
  }
  const float vv = valid ? 1.f : 0.f;
  sh.vs[kb * kBlk + t] = vv;
  return vv;
}

template <int CD, bool PT, int QP>
__global__ void __launch_bounds__(kPfThreads, 1)
prefill_tc_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap rows) {
  using L = PfLayout<CD, PT>;
  constexpr bool kBf = PfCode<CD>::kBf16;
  constexpr int BS = L::BS, NB = L::NB, NBK = L::NBK, NBV = L::NBV;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, kvh = blockIdx.y;
  const int g = p.g, TQ = kRows / g;
  const int q0 = blockIdx.x * TQ;
  // the sequence's query count L and context n; a sequence with more queries than
  // positions, or than the host bound max_q_len, is rejected (counted once)
  int Lq = p.q_start[b + 1] - p.q_start[b];
  const SeqInfo si = seq_info(p, b, L::LB, blockIdx.x == 0 && kvh == 0 && threadIdx.x == 0);
  const int n = si.n;
  if (Lq > n || Lq > p.max_q_len || Lq < 0) {
    if (blockIdx.x == 0 && kvh == 0 && threadIdx.x == 0) record_fault(p.fault, KVQ_FAULT_CONTEXT);
    Lq = 0;
  }
  if (q0 >= Lq) return;                                   // uniform: no query of this tile
  const int pmin = n - Lq + q0;                           // position of the tile's first query
  const int pmax = n - Lq + min(q0 + TQ, Lq) - 1;         // ... and of its last
  const int J = pmax / kBlk + 1;                          // blocks of the causal window
  // pages to copy: those of the causal window (low-bit caches: of the quantized prefix only;
  // positions from si.qb on come from the residual ring)
  const int npg = L::LB ? min(pmax / BS + 1, si.qb / BS) : pmax / BS + 1;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  PfShared sh;
  sh.raw_full = bars;
  sh.raw_empty = bars + L::RG;
  sh.k_full = bars + 2 * L::RG;
  sh.v_full = sh.k_full + NBK;
  sh.vfree = sh.v_full + NBV;
  sh.s_full = sh.vfree + NBV;
  sh.p_full = sh.s_full + 2;
  sh.pv_done = sh.p_full + 2;
  sh.q_ready = sh.pv_done + 2;
  sh.fin = sh.q_ready + 1;
  sh.xch = sh.fin + 1;
  sh.kq_full = sh.xch + 4;
  sh.kqfree = sh.kq_full + kNQ;
  sh.tile_full = sh.kqfree + kNQ;
  sh.xmax = reinterpret_cast<float*>(smem + L::XM_OFF);
  sh.page_ok = reinterpret_cast<int*>(bars + L::NBARS);
  sh.kq = reinterpret_cast<float*>(smem + L::KQ_OFF);
  sh.vs = reinterpret_cast<float*>(smem + L::VS_OFF);
  sh.vmax = reinterpret_cast<float*>(smem + L::MISC_OFF);            // [kNBMax][4]
  sh.nbad = reinterpret_cast<int*>(smem + L::MISC_OFF + 48);         // [kNQ][4]
  sh.qscale = reinterpret_cast<float*>(smem + L::MISC_OFF + 112);
  sh.tmem = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF + 116);
  sh.abort = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 120);
  float* red = reinterpret_cast<float*>(smem + L::MISC_OFF + 128);  // [8] softmax amax

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::RG; ++s) {
      mbar_init(&sh.raw_full[s], 1);
      mbar_init(&sh.raw_empty[s], 8);                    // the eight converter warps
    }
    for (int k = 0; k < NBK; ++k) mbar_init(&sh.k_full[k], 4);
    for (int k = 0; k < NBV; ++k) {
      mbar_init(&sh.v_full[k], 4);
      mbar_init(&sh.vfree[k], 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&sh.s_full[k], 1);
      mbar_init(&sh.p_full[k], kSoftWarps);
      mbar_init(&sh.pv_done[k], 1);
    }
    mbar_init(sh.q_ready, kSoftWarps);
    mbar_init(sh.fin, 1);
    for (int k = 0; k < 4; ++k) mbar_init(&sh.xch[k], 2);
    for (int k = 0; k < kNQ; ++k) {
      mbar_init(&sh.kq_full[k], 4);
      mbar_init(&sh.kqfree[k], kSoftWarps);
    }
    for (int k = 0; k < NB; ++k) mbar_init(&sh.tile_full[k], 1);
    *sh.abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tc::tmem_alloc(sh.tmem, kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *sh.tmem;

  if (warp == kProdWarp) {
    // ------------------------------------------------------------ producer
    // block j's pages (lane pp: page j PPB + pp) land in ring group j % RG; lane 0 announces
    // the group's bytes on its full barrier before any copy is issued
    const uint8_t* pages = p.pages;
    const int nblk = (npg + L::PPB - 1) / L::PPB;          // blocks with pages to copy
    bool ok_run = true;
    int jb = 0;
    if constexpr (L::DIRECT) {
      // 16-bit rows go straight into tile buffer kb = jb % NB: K rows (16 of a page) as the
      // two 128-byte halves of the K tile's rows, V rows likewise; a buffer is refilled once
      // S of block jb - NB (K) and P V of block jb - NB (V) have read it
      for (; jb < nblk && ok_run; ++jb) {
        const int kb = jb % NB;
        const int k = jb * L::PPB + lane;
        const bool mine = lane < L::PPB && k < npg;
        const int blk = mine ? p.tables[static_cast<long>(b) * p.max_blocks + k] : -1;
        bool ok_lane = true;
        if (lane == 0 && jb >= NB) {
          if (!pf_wait(&sh.s_full[(jb - NB) & 1], ((jb - NB) >> 1) & 1, sh.abort) ||
              !pf_wait(&sh.vfree[kb], ((jb / NB) - 1) & 1, sh.abort))
            ok_lane = false;
        }
        ok_run = __all_sync(0xffffffffu, ok_lane);
        if (!ok_run) {
          if (lane == 0) pf_fail(p, sh.abort);
          break;
        }
        bool valid = false;
        if (mine) {
          valid = blk >= 0 && blk < p.NB;
          sh.page_ok[kb * L::PPB + lane] = valid;
          if (!valid) record_fault(p.fault, KVQ_FAULT_BLOCK);
        }
        const unsigned nvalid = __popc(__ballot_sync(0xffffffffu, valid));
        if (lane == 0) mbar_arrive_expect_tx(&sh.tile_full[kb], nvalid * L::REC);
        __syncwarp();
        if (valid) {
          // the record's 32 rows of 256 bytes: K rows 0..15, V rows from OFF_V (16..31)
          const int y = (blk * p.H + kvh) * (2 * BS);
          const int r0 = lane * BS * 128;                  // page lane's rows in a tile half
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            tma_load_2d(smem + L::K_OFF + kb * kTile + hh * 16384 + r0, &rows, &sh.tile_full[kb], 128 * hh, y);
            tma_load_2d(smem + L::V_OFF + kb * kTile + hh * 16384 + r0, &rows, &sh.tile_full[kb], 128 * hh,
                        y + L::OFF_V / L::ROWB);
          }
        }
      }
      // every copy issued must land before the CTA may exit
      if (lane == 0) {
        for (int j2 = max(0, jb - NB); j2 < jb; ++j2)
          if (!mbar_drain(&sh.tile_full[j2 % NB], (j2 / NB) & 1)) record_fault(p.fault, KVQ_FAULT_TIMEOUT);
      }
    }
    for (; !L::DIRECT && jb < nblk && ok_run; ++jb) {
      const int grp = jb % L::RG, round = jb / L::RG;
      const int k = jb * L::PPB + lane, s = k % L::RS;
      // the table entries are read before the wait for the ring group, so that their
      // latency overlaps it
      const bool mine = lane < L::PPB && k < npg;
      const int blk = mine ? p.tables[static_cast<long>(b) * p.max_blocks + k] : -1;
      bool ok_lane = true;
      if (lane == 0 && round > 0 && !pf_wait(&sh.raw_empty[grp], (round - 1) & 1, sh.abort)) ok_lane = false;
      ok_run = __all_sync(0xffffffffu, ok_lane);
      if (!ok_run) {
        if (lane == 0) pf_fail(p, sh.abort);
        break;
      }
      bool valid = false;
      if (mine) {
        valid = blk >= 0 && blk < p.NB;
        sh.page_ok[s] = valid;
        if (!valid) record_fault(p.fault, KVQ_FAULT_BLOCK);
      }
      const unsigned nvalid = __popc(__ballot_sync(0xffffffffu, valid));
      if (lane == 0) mbar_arrive_expect_tx(&sh.raw_full[grp], nvalid * L::REC);
      __syncwarp();
      if (valid) {
        bulk_load(smem + L::RAW_OFF + s * L::REC, pages + (static_cast<long>(blk) * p.H + kvh) * L::REC, L::REC,
                  &sh.raw_full[grp]);
      }
    }
    // every copy issued must land before the CTA may exit
    if (!L::DIRECT && lane == 0) {
      for (int j2 = max(0, jb - L::RG); j2 < jb; ++j2)
        if (!mbar_drain(&sh.raw_full[j2 % L::RG], (j2 / L::RG) & 1)) record_fault(p.fault, KVQ_FAULT_TIMEOUT);
    }
  } else if (warp >= kConvWarp0) {
    // ------------------------------------------------------------ converters
    // warps 10-13 convert K, warps 14-17 V; thread (c, rr): 16-byte output chunk c (elements
    // 8c..8c+7 of a row) of rows rr + 8i.  K of block j waits for the block's pages, for S of
    // block j - NB (done with this K tile buffer) and for the softmax of block j - kNQ (done
    // with this slot of K multipliers); V of block j for the pages and for P V of block j - NB
    // (done with its V).  The block's ring group is released once all eight warps have read it.
    const int part = warp >= kConvWarp0 + 4 ? 1 : 0;
    const int cw = (warp - kConvWarp0) & 3;
    const int ct = cw * 32 + lane;                        // 0..127
    const int c = ct & 15, rr = ct >> 4;
    // q's power-of-two scale enters only the K multipliers: the K warps wait for it after
    // converting their first block's tile, the V warps never
    float qsc = 0.f;
    bool have_q = part == 1;
    const bool fz = p.mode == KVQ_SCALE_KIVI_FLOAT_ZERO, ktok = p.mode == KVQ_SCALE_INT4_PER_TOKEN;
    const int G = c >> 3;                                 // 64-channel group of the chunk
    for (int j = 0; j < J && !*sh.abort; ++j) {
      // tile buffer of this part: K tiles by j % NBK, V tiles (and V scales) by j % NBV
      const int kb = part == 0 ? j % NBK : j % NBV;
      const bool paged = j * L::PPB < npg;               // the block has pages in the ring
      {
        bool ok = true;
        if (part == 0) {
          // the K tile buffer: S of block j - NB has read it (16-bit caches: the producer
          // waited for that before refilling it); the multiplier slot: the softmax of block
          // j - kNQ is done with it
          if (!L::DIRECT && j >= NBK && !pf_wait(&sh.s_full[(j - NBK) & 1], ((j - NBK) >> 1) & 1, sh.abort))
            ok = false;
          if (ok && j >= kNQ && !pf_wait(&sh.kqfree[j % kNQ], ((j / kNQ) - 1) & 1, sh.abort)) ok = false;
        } else if (!L::DIRECT && j >= NBV && !pf_wait(&sh.vfree[kb], ((j / NBV) - 1) & 1, sh.abort)) {
          ok = false;
        }
        if constexpr (L::DIRECT) {
          // the block's rows in tile buffer kb (its refill waited for P V of block j - NB,
          // so the V scales of buffer kb are free too)
          if (ok && paged && !pf_wait(&sh.tile_full[kb], (j / NB) & 1, sh.abort)) ok = false;
        } else {
          if (ok && paged && !pf_wait(&sh.raw_full[j % L::RG], (j / L::RG) & 1, sh.abort)) ok = false;
        }
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) pf_fail(p, sh.abort);
          break;
        }
        // K: bad-token count; V: largest V scale
        float val = 0.f;
        if constexpr (L::DIRECT) {
          val = direct_part<CD, PT>(smem, sh, j, kb, part == 1, ct, npg, pmax, qsc, have_q);
        } else if constexpr (!L::LB) {
          val = dense_part<CD, PT>(smem, sh, j, kb, part == 1, ct, npg, pmax, qsc, have_q);
        } else if (part == 0) {
          if (!have_q) {
            if (!pf_wait(sh.q_ready, 0, sh.abort)) pf_fail(p, sh.abort);
            qsc = *sh.qscale;
            have_q = true;
          }
          int bad = 0;
          // K: rows rr + 8i of every page of the block, chunk c (low-bit caches)
          for (int pp = 0; pp < L::PPB; ++pp) {
            const int k = j * L::PPB + pp;
            const bool have = k < npg;
            const int s = k % L::RS;
            const bool pok = have && sh.page_ok[s];
            const uint8_t* raw = smem + L::RAW_OFF + s * L::REC;
            {
              // per-channel K parameters of this chunk (KIVI forms): s[8c..8c+7], z or minimum
              float ksc[8], kzp[8];
              if (!ktok && pok) {
                const uint4 su = *reinterpret_cast<const uint4*>(raw + L::OFF_S + 16 * c);
                const uint4 zu = *reinterpret_cast<const uint4*>(raw + L::OFF_S + 2 * kD + 16 * c);
                const __half* sh8 = reinterpret_cast<const __half*>(&su);
                const __half* zh8 = reinterpret_cast<const __half*>(&zu);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  ksc[e] = __half2float(sh8[e]);
                  kzp[e] = __half2float(zh8[e]);
                }
              }
              for (int i = 0; i < BS / 8; ++i) {
                const int row = rr + 8 * i, t = pp * BS + row, pos = j * kBlk + t;
                const bool ring = pos >= si.qb;
                const bool valid = pos <= pmax && (ring || pok);
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = 0.f;
                if (valid && ring) {
                  const long rrow = ((static_cast<long>(si.sid) * 2) * p.H + kvh) * p.cap + pos % p.cap;
                  const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.residual) + rrow * kD + 8 * c);
                  if (p.act_fp16) unpack8<__half>(u, v);
                  else unpack8<__nv_bfloat16>(u, v);
                } else if (valid) {
                  uint32_t w;
                  if constexpr (L::BITS == 4) w = *reinterpret_cast<const uint32_t*>(raw + row * L::ROWB + 4 * c);
                  else w = *reinterpret_cast<const uint16_t*>(raw + row * L::ROWB + 2 * c);
                  float s1 = 0.f, z1 = 0.f;
                  if (ktok) {
                    const __half2 sz = *reinterpret_cast<const __half2*>(raw + L::OFF_S + (row * 2 + G) * 4);
                    s1 = __low2float(sz);
                    z1 = __high2float(sz);
                  }
#pragma unroll
                  for (int e = 0; e < 8; ++e) {
                    const int code = (w >> (L::BITS * e)) & ((1 << L::BITS) - 1);
                    v[e] = ktok ? lb_value(code, s1, z1, false) : lb_value(code, ksc[e], kzp[e], fz);
                  }
                }
                uint4 hi, lo;
                split8(v, hi, lo);
                *reinterpret_cast<uint4*>(smem + L::K_OFF + (kb * 2) * kTile + tile_off(t, c)) = hi;
                *reinterpret_cast<uint4*>(smem + L::K_OFF + (kb * 2 + 1) * kTile + tile_off(t, c)) = lo;
                if (c == 0) {
                  const bool badtok = !ring && have && !pok && pos <= pmax;
                  sh.kq[(j % kNQ) * kBlk + t] = valid ? qsc : (badtok ? __uint_as_float(0x7fffffffu) : 0.f);
                  bad += badtok;
                }
              }
            }
          }
          val = static_cast<float>(bad);
        } else {
          float vm = 0.f;
          for (int pp = 0; pp < L::PPB; ++pp) {
            const int k = j * L::PPB + pp;
            const bool have = k < npg;
            const int s = k % L::RS;
            const bool pok = have && sh.page_ok[s];
            const uint8_t* raw = smem + L::RAW_OFF + s * L::REC;
            {
              for (int i = 0; i < BS / 8; ++i) {
                const int row = rr + 8 * i, t = pp * BS + row, pos = j * kBlk + t;
                const bool ring = pos >= si.qb;
                const bool valid = pos <= pmax && (ring || pok);
                float v[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = 0.f;
                if (valid && ring) {
                  const long vrow = ((static_cast<long>(si.sid) * 2 + 1) * p.H + kvh) * p.cap + pos % p.cap;
                  const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.residual) + vrow * kD + 8 * c);
                  if (p.act_fp16) unpack8<__half>(u, v);
                  else unpack8<__nv_bfloat16>(u, v);
                } else if (valid) {
                  uint32_t w;
                  if constexpr (L::BITS == 4) w = *reinterpret_cast<const uint32_t*>(raw + L::OFF_V + row * L::ROWB + 4 * c);
                  else w = *reinterpret_cast<const uint16_t*>(raw + L::OFF_V + row * L::ROWB + 2 * c);
                  const __half2 sz = *reinterpret_cast<const __half2*>(raw + L::OFF_S + 4 * kD + (row * 2 + G) * 4);
                  const float s1 = __low2float(sz), z1 = __high2float(sz);
#pragma unroll
                  for (int e = 0; e < 8; ++e) v[e] = lb_value((w >> (L::BITS * e)) & ((1 << L::BITS) - 1), s1, z1, fz);
                }
                uint4 hi, lo;
                split8(v, hi, lo);
                *reinterpret_cast<uint4*>(smem + L::V_OFF + (kb * 2) * kTile + tile_off(t, c)) = hi;
                *reinterpret_cast<uint4*>(smem + L::V_OFF + (kb * 2 + 1) * kTile + tile_off(t, c)) = lo;
                if (c == 0) {
                  const float vv = valid ? 1.f : 0.f;
                  sh.vs[kb * kBlk + t] = vv;
                  vm = fmaxf(vm, vv);
                }
              }
            }
          }
          val = vm;
        }
        if (part == 0) {
          const unsigned nbad = __reduce_add_sync(0xffffffffu, static_cast<unsigned>(val));
          if (lane == 0) sh.nbad[(j % kNQ) * 4 + cw] = static_cast<int>(nbad);
        } else {
          // V scales are >= 0: their bit patterns order as the values do
          const unsigned vmb = __reduce_max_sync(0xffffffffu, __float_as_uint(val));
          if (lane == 0) sh.vmax[kb * 4 + cw] = __uint_as_float(vmb);
        }
        tc::fence_async_shared();
        __syncwarp();
        if (lane == 0) {
          if (part == 0) {
            mbar_arrive(&sh.k_full[kb]);
            mbar_arrive(&sh.kq_full[j % kNQ]);
          } else {
            mbar_arrive(&sh.v_full[kb]);
          }
          if (!L::DIRECT && paged) mbar_arrive(&sh.raw_empty[j % L::RG]);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t tiles = smem_u32(smem);
    constexpr uint32_t idS = tc::idesc_f16(kBf, false, kRows, kBlk);
    constexpr uint32_t idPV = tc::idesc_f16(kBf, true, kRows, kD);
    if (lane == 0) {
      bool ok = pf_wait(sh.q_ready, 0, sh.abort);
      tc::fence_after_sync();
      auto pv = [&](int jj) -> bool {
        const int sb = jj & 1, kb = jj % NBV;
        if (!pf_wait(&sh.v_full[kb], (jj / NBV) & 1, sh.abort)) return false;
        if (!pf_wait(&sh.p_full[sb], (jj >> 1) & 1, sh.abort)) return false;
        tc::fence_after_sync();
        // P hi V hi (+ P hi V lo + P lo V hi for split V) + P lo V hi ... : pairs (pa, vp),
        // pa + vp <= 1
        bool first = jj == 0;
#pragma unroll
        for (int pa = 0; pa < 2; ++pa)
#pragma unroll
          for (int vp = 0; vp < L::VP; ++vp) {
            if (pa + vp > 1) continue;
            const uint32_t vt = tiles + L::V_OFF + (kb * L::VP + vp) * kTile;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              // tokens 16 kk .. 16 kk + 15: chunk kk / 2 of P, its hi (pa 0) or lo (pa 1) half
              tc::mma_ts(tbase + kTmO, tbase + 128 * sb + 16 * kk + 8 * pa,
                         tc::desc_mnmajor(vt, kk), idPV, first ? 0u : 1u);
              first = false;
            }
          }
        tc::commit(&sh.vfree[kb]);
        tc::commit(&sh.pv_done[jj & 1]);
        return true;
      };
      for (int j = 0; j < J && ok; ++j) {
        const int sb = j & 1, kb = j % NBK;
        if (!pf_wait(&sh.k_full[kb], (j / NBK) & 1, sh.abort)) { ok = false; break; }
        tc::fence_after_sync();
        bool first = true;
#pragma unroll
        for (int qa = 0; qa < QP; ++qa)
#pragma unroll
          for (int kp = 0; kp < L::KP; ++kp) {
            if (qa + kp > 1) continue;
            const uint32_t kt = tiles + L::K_OFF + (kb * L::KP + kp) * kTile;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              tc::mma_ts(tbase + 128 * sb, tbase + kTmQ + 64 * qa + 8 * kk, tc::desc_kmajor(kt, kk), idS,
                         first ? 0u : 1u);
              first = false;
            }
          }
        tc::commit(&sh.s_full[sb]);
        if (j > 0 && !pv(j - 1)) { ok = false; break; }
      }
      if (ok && !pv(J - 1)) ok = false;
      if (!ok) pf_fail(p, sh.abort);
      // one more commit covers every MMA issued above: TMEM is freed only after it arrives
      tc::commit(sh.fin);
      if (!mbar_drain(sh.fin, 0)) record_fault(p.fault, KVQ_FAULT_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    // warp w: query rows 32 (w % 4) .. + 31 (its TMEM lane quarter), score columns
    // [64 hf, 64 hf + 64) with hf = w / 4; the two warps of a quarter share each row's
    // running max through a per-quarter mbarrier
    const int quarter = warp & 3, hf = warp >> 2;
    const int r = 32 * quarter + lane;                     // query row (TMEM lane)
    const int t_loc = r / g, h = r - t_loc * g;
    const int qi = q0 + t_loc;
    const bool row_ok = qi < Lq;
    const int pos_r = n - Lq + qi;
    const uint32_t lanebase = tbase + (static_cast<uint32_t>(quarter * 32) << 16);
    const int col0 = 64 * hf;                              // this warp's first score column
    // --- q row, columns [64 hf, 64 hf + 64) -> TMEM (exact fp16 scaled by 2^-eq for
    // quantized caches; 16-bit caches as is)
    {
      const long qrow = static_cast<long>(p.q_start[b]) + qi;
      const uint4* qp = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.q) +
                                                       (qrow * p.Hq + static_cast<long>(kvh) * g + h) * kD + col0);
      // per-channel K scales fold into q (then q goes to TMEM as a hi + lo pair); with
      // bf16 tiles and fp16 activations q is split exactly into bf16 hi + lo
      const float* kch = p.mode == KVQ_SCALE_PER_CHANNEL ? p.k_static + kvh * kD + col0 : nullptr;
      auto elem = [&](const uint4& u, int e) {     // element e (0..7) of 8 packed activations
        const uint32_t w2 = (&u.x)[e >> 1];
        const uint16_t hv = static_cast<uint16_t>((e & 1) ? (w2 >> 16) : (w2 & 0xFFFFu));
        return p.act_fp16 ? __half2float(__ushort_as_half(hv)) : __bfloat162float(__ushort_as_bfloat16(hv));
      };
      float qscale = p.scale_log2;
      if (p.mode == KVQ_SCALE_PER_HEAD) qscale *= p.k_static[kvh];
      if (p.mode == KVQ_SCALE_PER_TENSOR) qscale *= p.k_static[0];
      // the row's 64 values in one round of loads, kept in registers for both passes
      uint4 qr[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) qr[i] = row_ok ? qp[i] : make_uint4(0, 0, 0, 0);
      float down = 1.f;
      if constexpr (!kBf) {
        // the tile's largest |q| (times the channel scale) sets a power-of-two scale that
        // keeps q inside fp16
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            amax = fmaxf(amax, fabsf(kch != nullptr ? elem(qr[i], e) * kch[8 * i + e] : elem(qr[i], e)));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (lane == 0) red[warp] = amax;
        named_sync(2, 32 * kSoftWarps);
        amax = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < kSoftWarps; ++w2) amax = fmaxf(amax, red[w2]);
        int eq = 0;
        if (amax > 0.f && !(p.act_fp16 && kch == nullptr)) eq = ilogbf(amax) - 13;
        down = ldexpf(1.f, -eq);
        qscale = ldexpf(qscale, eq);
      }
      // 32 columns (16 TMEM columns of 16-bit pairs) at a time
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 u = qr[4 * hq + i];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const int d = 32 * hq + 8 * i + e;
            float a = elem(u, e), c2 = elem(u, e + 1);
            if (kch != nullptr) {
              a *= kch[d];
              c2 *= kch[d + 1];
            }
            a *= down;
            c2 *= down;
            if constexpr (QP == 2) split2<kBf>(a, c2, hi[4 * i + e / 2], lo[4 * i + e / 2]);
            else hi[4 * i + e / 2] = kBf ? pack_bf16x2(a, c2) : pack_f16x2(a, c2);
          }
        }
        st16(lanebase + kTmQ + 32 * hf + 16 * hq, hi);
        if constexpr (QP == 2) st16(lanebase + kTmQ + 64 + 32 * hf + 16 * hq, lo);
      }
      if (threadIdx.x == 0) *sh.qscale = qscale;
      tc::st_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(sh.q_ready);
    }
    // --- blocks.  Running max m (re-based lazily) and V normaliser 2^ev (the exponent of the
    // largest V scale so far) together set the exponent offset of P: e = 2^(x - m - ev), so
    // that e times a token's V scale stays below 2^10 in fp16; l and O accumulate in that
    // scaled domain, and the offset cancels in O / l.
    float m = -INFINITY, l = 0.f;
    int ev = INT_MIN;
    bool ok = true;
    float* xm = sh.xmax;                                   // [2][2][128]: block parity, half, row
    for (int j = 0; j < J; ++j) {
      const int sb = j & 1, kb = j % NBV, qs = j % kNQ;     // kb: the V buffer
      // the block's K multipliers through their own slot barrier: K of block j + NB may
      // complete k_full once more before this wait (the next phase of kq_full[qs] needs
      // this softmax's release of the slot)
      if (!pf_wait(&sh.kq_full[qs], (j / kNQ) & 1, sh.abort) ||
          !pf_wait(&sh.s_full[sb], (j >> 1) & 1, sh.abort)) {
        ok = false;
      }
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc::fence_after_sync();
      const float* kq = sh.kq + qs * kBlk + col0;
      const bool fast = sh.nbad[qs * 4] + sh.nbad[qs * 4 + 1] + sh.nbad[qs * 4 + 2] + sh.nbad[qs * 4 + 3] == 0 &&
                        j * kBlk + kBlk - 1 <= pmin;   // uniform
      // causal boundary (position <= this row's) and tokens of bad pages (multiplier NaN)
      const int lim = row_ok ? pos_r - j * kBlk - col0 : -1;
      // pass 1: the largest scaled score of this row's 64 columns, 16 at a time (read from
      // TMEM again in pass 2).  Blocks wholly visible to every row of the tile take a path
      // with no per-score tests, in which the load of the next 16 columns is in flight while
      // the current ones are reduced.
      const uint32_t sbase = lanebase + 128 * sb + col0;
      float m0 = -INFINITY, m1 = -INFINITY;
      uint32_t ra[16], rb[16];
      auto max16 = [&](const uint32_t* r, int c0) {
#pragma unroll
        for (int i = 0; i < 16; i += 4) {
          const float4 f = *reinterpret_cast<const float4*>(kq + c0 + i);
          const float2 a = __fmul2_rn(make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])),
                                      make_float2(f.x, f.y));
          const float2 c = __fmul2_rn(make_float2(__uint_as_float(r[i + 2]), __uint_as_float(r[i + 3])),
                                      make_float2(f.z, f.w));
          m0 = max3(m0, a.x, a.y);
          m1 = max3(m1, c.x, c.y);
        }
      };
      if (fast) {
        tc::ld16_issue(sbase, ra);
        tc::ld_wait16(ra);
        tc::ld16_issue(sbase + 16, rb);
        max16(ra, 0);
        tc::ld_wait16(rb);
        tc::ld16_issue(sbase + 32, ra);
        max16(rb, 16);
        tc::ld_wait16(ra);
        tc::ld16_issue(sbase + 48, rb);
        max16(ra, 32);
        tc::ld_wait16(rb);
        max16(rb, 48);
      } else {
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          tc::ld16(sbase + 16 * cc, ra);
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            const int t = 16 * cc + i;
            const float2 f = *reinterpret_cast<const float2*>(kq + t);
            const float2 a = __fmul2_rn(make_float2(__uint_as_float(ra[i]), __uint_as_float(ra[i + 1])), f);
            m0 = fmaxf(m0, (t <= lim && f.x == f.x) ? a.x : -INFINITY);
            m1 = fmaxf(m1, (t + 1 <= lim && f.y == f.y) ? a.y : -INFINITY);
          }
        }
      }
      // the first 16 columns of pass 2 are read while the row maxima are exchanged
      tc::ld16_issue(sbase, ra);
      float mx = fmaxf(m0, m1);
      // the row's max over both halves: exchange with the partner warp of this quarter
      xm[(sb * 2 + hf) * kRows + r] = mx;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.xch[quarter]);
      if (!pf_wait(&sh.xch[quarter], j & 1, sh.abort)) ok = false;
      if (!pf_wait(&sh.v_full[kb], (j / NBV) & 1, sh.abort)) ok = false;
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      mx = fmaxf(mx, xm[(sb * 2 + (hf ^ 1)) * kRows + r]);
      // rescale factor of l and O: the max re-based (beyond 2^8) and / or the V normaliser
      // grown (both the same in the two warps of a row)
      float fo = 1.f;
      const float vmx = fmaxf(fmaxf(sh.vmax[kb * 4], sh.vmax[kb * 4 + 1]),
                              fmaxf(sh.vmax[kb * 4 + 2], sh.vmax[kb * 4 + 3]));
      if (vmx > 0.f) {
        // (floored at 2^-100, so that 2^(x - m - ev) stays finite for any V scale)
        const int e = max(exponent_of(vmx), -100);
        if (e > ev) {
          if (ev != INT_MIN) fo = pow2i(ev - e);
          ev = e;
        }
      }
      if (mx > m + kRescalePf) {
        const float mn = fmaxf(m, mx);
        fo *= m == -INFINITY ? 0.f : ex2(m - mn);
        m = mn;
      }
      l *= fo;
      if (j > 0 && __any_sync(0xffffffffu, fo != 1.f)) {
        // rescale this warp's half of its O rows: P V of block j - 1 must be complete
        if (!pf_wait(&sh.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, sh.abort)) ok = false;
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc::fence_after_sync();
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[16];
          tc::ld16(lanebase + kTmO + col0 + 16 * cc, o);
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * fo);
          st16(lanebase + kTmO + col0 + 16 * cc, o);
        }
      }
      const float off = (m == -INFINITY ? 0.f : m) + (ev == INT_MIN ? 0.f : static_cast<float>(ev));
      const float* vsp = sh.vs + kb * kBlk + col0;
      // pass 2: e = 2^(x - off), the row sum, and e times the token's V scale as hi + lo
      // 16-bit halves, 16 score columns at a time: P of those 16 keys overwrites their scores
      // (hi halves in the first 8 TMEM columns, lo halves in the next 8)
      float2 lsum = make_float2(0.f, 0.f);
      const float2 noff = make_float2(-off, -off);
      auto p16 = [&](const uint32_t* r, int c0, auto masked) {
        uint32_t ph[8], pl[8];
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          const int t = c0 + 2 * i;
          const float4 f = *reinterpret_cast<const float4*>(kq + t);
          const float4 vv = *reinterpret_cast<const float4*>(vsp + t);
          float2 xa = __ffma2_rn(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])),
                                 make_float2(f.x, f.y), noff);
          float2 xb = __ffma2_rn(make_float2(__uint_as_float(r[2 * i + 2]), __uint_as_float(r[2 * i + 3])),
                                 make_float2(f.z, f.w), noff);
          if constexpr (decltype(masked)::value) {
            if (!(t <= lim && f.x == f.x)) xa.x = -INFINITY;
            if (!(t + 1 <= lim && f.y == f.y)) xa.y = -INFINITY;
            if (!(t + 2 <= lim && f.z == f.z)) xb.x = -INFINITY;
            if (!(t + 3 <= lim && f.w == f.w)) xb.y = -INFINITY;
          }
          const float2 ea = make_float2(ex2(xa.x), ex2(xa.y)), eb = make_float2(ex2(xb.x), ex2(xb.y));
          lsum = __fadd2_rn(lsum, __fadd2_rn(ea, eb));
          split2<kBf>(__fmul2_rn(ea, make_float2(vv.x, vv.y)), ph[i], pl[i]);
          split2<kBf>(__fmul2_rn(eb, make_float2(vv.z, vv.w)), ph[i + 1], pl[i + 1]);
        }
        st8(sbase + c0, ph);
        st8(sbase + c0 + 8, pl);
      };
      tc::ld_wait16(ra);
      if (fast) {
        tc::ld16_issue(sbase + 16, rb);
        p16(ra, 0, std::false_type{});
        tc::ld_wait16(rb);
        tc::ld16_issue(sbase + 32, ra);
        p16(rb, 16, std::false_type{});
        tc::ld_wait16(ra);
        tc::ld16_issue(sbase + 48, rb);
        p16(ra, 32, std::false_type{});
        tc::ld_wait16(rb);
        p16(rb, 48, std::false_type{});
      } else {
        p16(ra, 0, std::true_type{});
#pragma unroll 1
        for (int cc = 1; cc < 4; ++cc) {
          tc::ld16(sbase + 16 * cc, rb);
          p16(rb, 16 * cc, std::true_type{});
        }
      }
      l += lsum.x + lsum.y;
      tc::st_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sh.p_full[sb]);
        mbar_arrive(&sh.kqfree[qs]);
      }
    }
    if (!ok) {
      if (lane == 0) pf_fail(p, sh.abort);
    } else {
      // --- epilogue: the row sum over both halves, then O / l (times the static V scales)
      // for this warp's 64 output columns
      xm[(2 * 2 + hf) * kRows + r] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.xch[quarter]);
      if (!pf_wait(&sh.xch[quarter], J & 1, sh.abort)) ok = false;
      if (!pf_wait(&sh.pv_done[(J - 1) & 1], ((J - 1) >> 1) & 1, sh.abort)) ok = false;
      if (__all_sync(0xffffffffu, ok)) {
        tc::fence_after_sync();
        const float lt = l + xm[(2 * 2 + (hf ^ 1)) * kRows + r];
        float vmul = 1.f;
        if (p.mode == KVQ_SCALE_PER_HEAD) vmul = p.v_static[kvh];
        if (p.mode == KVQ_SCALE_PER_TENSOR) vmul = p.v_static[0];
        const float inv = lt > 0.f ? vmul / lt : 0.f;
        const float* vch = (p.mode == KVQ_SCALE_PER_CHANNEL) ? p.v_static + kvh * kD + col0 : nullptr;
        const long orow = (static_cast<long>(p.q_start[b]) + qi) * p.Hq + static_cast<long>(kvh) * g + h;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[16];
          tc::ld16(lanebase + kTmO + col0 + 16 * cc, o);
          if (row_ok) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              v[i] = __uint_as_float(o[i]) * inv * (vch != nullptr ? vch[16 * cc + i] : 1.f);
            const long e0 = orow * kD + col0 + 16 * cc;          // a multiple of 16 elements
            if (p.out_dtype == KVQ_DTYPE_FP32) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + e0);
#pragma unroll
              for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            } else {
              const bool bf = p.out_dtype == KVQ_DTYPE_BF16;
              uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + e0);
#pragma unroll
              for (int i = 0; i < 2; ++i) {
                uint32_t q4[4];
#pragma unroll
                for (int k2 = 0; k2 < 4; ++k2) {
                  const float a0 = v[8 * i + 2 * k2], a1 = v[8 * i + 2 * k2 + 1];
                  q4[k2] = bf ? pack_bf16x2(a0, a1) : pack_f16x2(a0, a1);
                }
                dst[i] = make_uint4(q4[0], q4[1], q4[2], q4[3]);
              }
            }
          }
        }
      } else if (lane == 0) {
        pf_fail(p, sh.abort);
      }
    }
  }
  // ---------------------------------------------------------------- teardown
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    // the issuer waited for its final commit (every MMA complete) before the barrier
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, kTmemCols);
  }
}

template <int CD, bool PT, int QP>
cudaError_t launch_pf(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s) {
  using L = PfLayout<CD, PT>;
  if (a.geo.record != L::REC) return cudaErrorInvalidValue;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(prefill_tc_kernel<CD, PT, QP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    L::BYTES);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int TQ = kRows / a.plan.g;
  const dim3 grid((a.max_q_len + TQ - 1) / TQ, a.geo.H, a.batch);
  CUtensorMap rows = {};                  // 16-bit caches: the pool as rows of 256 bytes
  if constexpr (L::DIRECT) {
    const long nrows = static_cast<long>(a.geo.NB) * a.geo.H * 2 * L::BS;
    if (!make_rows_map(&rows, a.c->pages, nrows, L::ROWB, L::BS)) return cudaErrorInvalidValue;
  }
  prefill_tc_kernel<CD, PT, QP><<<grid, kPfThreads, L::BYTES, s>>>(p, rows);
  return cudaGetLastError();
}

}  // namespace

bool prefill_tc_supported(const Geometry& g, int group) {
  if (g.D != kD || group < 1 || kRows % group != 0) return false;
  switch (g.cache_dtype) {
    case KVQ_DTYPE_INT8:
    case KVQ_DTYPE_FP8_E4M3:
    case KVQ_DTYPE_BF16:
    case KVQ_DTYPE_FP16: return g.bs == 16;
    case KVQ_DTYPE_INT4:
    case KVQ_DTYPE_INT2: return g.bs == 64;
  }
  return false;
}

cudaError_t launch_prefill_tc(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s) {
  const bool pt = a.geo.scale_mode == KVQ_SCALE_PER_TOKEN_HEAD;
  const bool pc = a.geo.scale_mode == KVQ_SCALE_PER_CHANNEL;
  switch (a.geo.cache_dtype) {
    case KVQ_DTYPE_INT8:
      if (pt) return launch_pf<KVQ_DTYPE_INT8, true, 1>(a, p, s);
      return pc ? launch_pf<KVQ_DTYPE_INT8, false, 2>(a, p, s) : launch_pf<KVQ_DTYPE_INT8, false, 1>(a, p, s);
    case KVQ_DTYPE_FP8_E4M3:
      if (pt) return launch_pf<KVQ_DTYPE_FP8_E4M3, true, 1>(a, p, s);
      return pc ? launch_pf<KVQ_DTYPE_FP8_E4M3, false, 2>(a, p, s)
                : launch_pf<KVQ_DTYPE_FP8_E4M3, false, 1>(a, p, s);
    case KVQ_DTYPE_BF16: return launch_pf<KVQ_DTYPE_BF16, false, 1>(a, p, s);
    case KVQ_DTYPE_FP16: return launch_pf<KVQ_DTYPE_FP16, false, 1>(a, p, s);
    // low-bit: bf16 tiles; fp16 activations go to TMEM as an exact bf16 hi + lo pair
    case KVQ_DTYPE_INT4:
      return p.act_fp16 ? launch_pf<KVQ_DTYPE_INT4, false, 2>(a, p, s) : launch_pf<KVQ_DTYPE_INT4, false, 1>(a, p, s);
    case KVQ_DTYPE_INT2:
      return p.act_fp16 ? launch_pf<KVQ_DTYPE_INT2, false, 2>(a, p, s) : launch_pf<KVQ_DTYPE_INT2, false, 1>(a, p, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kvq
