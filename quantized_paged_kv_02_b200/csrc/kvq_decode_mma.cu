// Paged split-K decode attention on tensor cores, for GQA groups of 1..8 query heads
// (head_dim 128, dense caches: INT8, FP8 E4M3, BF16, FP16).
//
// Schedule: one CTA per resident slot (3 per SM).  The pages of all (sequence, kv head)
// units, concatenated, are cut into equal contiguous ranges, one per CTA, so every CTA
// streams the same number of bytes whatever the mix of context lengths, and a CTA's copy
// pipeline never drains between units.  A unit that straddles CTA ranges is finished by
// the segment reduce (log-sum-exp merge of the per-warp partials).
//
// Within a CTA, warp 4 is the producer: it walks the block tables of its range and moves
// each block's page record (K codes, V codes and per-token scales, contiguous in the
// cache) into a ring of shared-memory stages with one TMA tensor copy per page (128-byte
// swizzle, so the fragment loads below are free of bank conflicts; one 4 KiB copy per page
// instead of several small ones is what lets the copy engine keep HBM busy), and notes
// (unit, page, tokens, valid) beside the stage; an mbarrier per stage signals "full" to
// the consumers and another signals "empty" back.  Warps 0-3 consume stages round-robin.
// For each 16-token tile a warp computes S^T = K Q^T with mma.sync (M = 16 tokens, N = 8
// query heads, K = head_dim, fp32 or exact int32 accumulate): INT8 codes go straight into
// the integer tensor cores against a 3-term int8 split of q, e4m3 / 16-bit codes become
// fp16/bf16 fragments in registers (exact).  The per-token or per-head scales multiply the
// fp32 scores, an online softmax (running max, running sum) runs in the log2 domain, and
// O^T += V^T P^T is a second mma.sync with P split into hi + lo halves (P changes
// fragment layout in registers with movmatrix).  Per-token V scales are folded into P
// with a per-warp power-of-two normaliser.  When the unit changes, the warp writes its
// partial (O, max, sum) to the workspace and loads the next query group.
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
constexpr int kIssueLanes = 8;    // producer lanes that issue copies side by side
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
  // ring depth: as many stages as fit the shared memory of 3 CTAs per SM (228 KiB per SM,
  // 1 KiB of it reserved per CTA); bytes in flight are what keeps HBM busy
  static constexpr int kSmemPerCta = 228 * 1024 / 3 - 1024;
  static constexpr int kFixed = 1024 + 16 + 4 * 4 + 32 * 4;  // alignment, range, batch ids
  static constexpr int kStages = (kSmemPerCta - kFixed) / (STAGE + 32) / kConsumers * kConsumers;
  static constexpr int TILES = kStages * STAGE;
  static constexpr int BARS = kStages * 2 * 8;
  static constexpr int META = kStages * 16 + 16 + 32 * 4;  // page records, range, batch ids
  static constexpr int BYTES = 1024 + TILES + BARS + META;
  static_assert(kStages >= 4 && BYTES <= kSmemPerCta, "ring fits 3 CTAs per SM");
  // Consumers take pages round-robin, and every round of a stage must go to the same
  // warp: a warp waiting for round r of a stage whose round r-1 belonged to another warp
  // (and has not landed yet) would see the parity of round r-2 as complete.
  static_assert(kStages % kConsumers == 0, "ring depth is a multiple of the consumers");
  static_assert(kStages >= kIssueLanes, "one issue chunk never waits on its own stages");
  static_assert(REC_ROWS <= 256, "TMA box height");
};

// Shared-memory byte offset of record byte `off` after the 128-byte swizzle: the 16-byte
// chunk index is XORed with the 128-byte row index (mod 8).
__device__ __forceinline__ int swzb(int off) {
  return (off & ~127) + ((((off >> 4) & 7) ^ ((off >> 7) & 7)) << 4) + (off & 15);
}

// PF false: decode, grid p.ctas over page-balanced ranges.  PF true: chunked prefill,
// grid (query groups of kConsumers tokens, kv heads, sequences); each consumer warp owns one
// query token (with its g heads), reads every page its causal window covers and writes
// its output rows itself.
template <int CD, int BS, bool PT, bool PF>
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
  int4* meta = reinterpret_cast<int4*>(empty + kStages);   // per stage: unit, page, tokens, valid
  int* range_pages = reinterpret_cast<int*>(meta + kStages);
  int* ids = range_pages + 4;                               // producer: block ids of a batch
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = p.ctas;                                    // the grid (page partition)
  const int cta = blockIdx.x;

  // inputs (pages, q, tables, lengths) may come from the kernel just before this one
  griddep_wait();
  griddep_launch_dependents();
  // prefill: this CTA's sequence, kv head, first query of its group, and the group's
  // query count L and context n of the sequence
  int pf_b = 0, pf_kvh = 0, pf_q0 = 0, pf_L = 0, pf_n = 0;
  if constexpr (PF) {
    pf_b = blockIdx.z;
    pf_kvh = blockIdx.y;
    pf_q0 = blockIdx.x * kConsumers;
    pf_L = p.q_start[pf_b + 1] - p.q_start[pf_b];
    pf_n = seq_info(p, pf_b, false, blockIdx.x == 0 && pf_kvh == 0 && threadIdx.x == 0).n;
    // more queries than positions, or than the host bound max_q_len (which sizes the
    // grid): rejected
    if (pf_L > pf_n || pf_L > p.max_q_len || pf_L > static_cast<int>(gridDim.x) * kConsumers ||
        pf_L < 0) {
      if (blockIdx.x == 0 && pf_kvh == 0 && threadIdx.x == 0) record_fault(p.fault, KVQ_FAULT_CONTEXT);
      pf_L = 0;
    }
    if (pf_q0 >= pf_L) return;                  // no query of this group (uniform)
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], PF ? kConsumers : 1);   // prefill: every consumer reads every page
    }
    fence_mbar_init();
  }
  // The producer finds this CTA's page range [start, end) and the sequence it starts in.
  long long start = 0, end = 0, seq_first_page = 0;
  int b_first = 0;
  if constexpr (PF) {
    // pages [0, npages) of unit (b, kvh): the causal window of the group's last query
    const int last = pf_n - pf_L + min(pf_q0 + kConsumers, pf_L) - 1;
    const int npb = (pf_n + BS - 1) / BS;
    b_first = pf_b;
    seq_first_page = 0;                         // unit (b, kvh) starts at kvh * npb
    start = static_cast<long long>(pf_kvh) * npb;
    end = start + (last + BS) / BS;
    if (warp == kConsumers && lane == 0) *range_pages = static_cast<int>(end - start);
  } else if (warp == kConsumers) {
    long long tot = 0;
    for (int b0 = 0; b0 < p.batch; b0 += 32) {
      int np = b0 + lane < p.batch ? seq_pages(p, b0 + lane, cta == 0) : 0;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) np += __shfl_xor_sync(0xffffffffu, np, off);
      tot += np;
    }
    const long long P = tot * p.H;
    start = range_start(P, cta, C);
    end = range_start(P, cta + 1, C);
    long long pre = 0;
    for (int b0 = 0; b0 < p.batch && start < end; b0 += 32) {
      const int b = b0 + lane;
      const long long own = b < p.batch ? static_cast<long long>(seq_pages(p, b)) * p.H : 0;
      long long incl = own;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const long long t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, b < p.batch && pre + incl > start);
      if (hit) {
        const int k = __ffs(hit) - 1;
        b_first = b0 + k;
        seq_first_page = __shfl_sync(0xffffffffu, pre + incl - own, k);
        break;
      }
      pre += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) *range_pages = static_cast<int>(end - start);
  }
  __syncthreads();

  if (warp == kConsumers) {
    // ---------------------------------------------------------------- producer
    // The range is walked in batches of up to 32 pages of one unit.  The block ids of the
    // next batch (and the length of the next sequence) are loaded while lane 0 issues the
    // copies of the current batch, so table reads never leave the copy stream idle.
    const uint32_t stage_bytes = L::REC;
    bool ok_run = true;
    int issued = 0;
    // walk cursor: next global page gp; sequence b starts at global page ub and has nb
    // tokens in npb pages; n_ahead is the raw length of sequence b + 1
    long long gp = start, ub = seq_first_page;
    int b = b_first, nb = 0, npb = 0, n_ahead = 0;
    if (gp < end) {
      nb = seq_info(p, b, false).n;
      npb = (nb + BS - 1) / BS;
      n_ahead = b + 1 < p.batch ? p.lens[b + 1] : 0;
    }
    // Append step: quantize this step's K and V rows of (sequence b, kv head) into the
    // unit's last page, exactly as kvq_write stores them (lanes 0-15 the K row, 16-31 the
    // V row), before that page is copied.  Only this CTA reads that page.
    auto append_row = [&](int bq, int kvh, int n) {
      const int pos = n - 1;
      const int blk = p.tables[static_cast<long>(bq) * p.max_blocks + pos / BS];
      if (blk < 0 || blk >= p.NB) return;     // the page is skipped (and counted) when read
      const int kv = lane >> 4, l = lane & 15;
      const uint4 u = reinterpret_cast<const uint4*>(kv ? p.v_new : p.k_new)
          [((static_cast<long>(bq) * p.H + kvh) * kD) / 8 + l];
      uint8_t* rec = p.pages_w + (static_cast<long>(blk) * p.H + kvh) * L::REC;
      float static_s = 0.f;
      const float* chan_s = nullptr;
      if constexpr (!PT && Code<CD>::B == 1) {
        const float* sp = kv ? p.v_static : p.k_static;
        if (p.mode == KVQ_SCALE_PER_CHANNEL) chan_s = sp + kvh * kD;
        else static_s = sp[p.mode == KVQ_SCALE_PER_HEAD ? kvh : 0];
      }
      if (p.act_fp16)
        quantize_row_part<__half, CD, kD>(&u, l, true, kv, pos % BS, BS, rec, L::OFF_V, L::OFF_S, PT,
                                          static_s, chan_s);
      else
        quantize_row_part<__nv_bfloat16, CD, kD>(&u, l, true, kv, pos % BS, BS, rec, L::OFF_V, L::OFF_S, PT,
                                                 static_s, chan_s);
      fence_proxy_async_global();
      __syncwarp();
    };
    struct Batch { int u, kvh, pg0, cnt, nb, raw; };
    auto next_batch = [&]() {
      Batch t{0, 0, 0, 0, 0, -1};
      if (gp >= end) return t;
      // move past finished (or empty) sequences
      while (gp >= ub + static_cast<long long>(p.H) * npb && b + 1 < p.batch) {
        ub += static_cast<long long>(p.H) * npb;
        ++b;
        nb = dense_len(p, n_ahead);
        npb = (nb + BS - 1) / BS;
        n_ahead = b + 1 < p.batch ? p.lens[b + 1] : 0;
      }
      if (gp >= ub + static_cast<long long>(p.H) * npb) {   // not reached: ranges lie inside P
        gp = end;
        return t;
      }
      const long long off = gp - ub;
      t.kvh = static_cast<int>(off / npb);
      t.pg0 = static_cast<int>(off - static_cast<long long>(t.kvh) * npb);
      t.cnt = static_cast<int>(min(min(static_cast<long long>(npb - t.pg0), end - gp), 32LL));
      t.u = b * p.H + t.kvh;
      t.nb = nb;
      if (p.k_new != nullptr && t.pg0 + t.cnt == npb) append_row(b, t.kvh, nb);
      // issued now, checked when the batch is copied (one batch later)
      if (lane < t.cnt) t.raw = p.tables[static_cast<long>(b) * p.max_blocks + t.pg0 + lane];
      gp += t.cnt;
      return t;
    };
    Batch cur = next_batch();
    while (cur.cnt > 0 && ok_run) {
      const Batch nxt = next_batch();
      int blk = cur.raw;
      if (lane < cur.cnt && (blk < 0 || blk >= p.NB)) {
        record_fault(p.fault, KVQ_FAULT_BLOCK);
        blk = -1;
      }
      // lanes 0..7 issue eight pages at once, each: wait for its stage, write the page
      // record, one copy.  The barrier operations of one page form a dependent chain
      // of a few hundred cycles; issuing pages side by side overlaps those chains, which
      // is what lets 4 KiB copies keep pace with HBM.
      ids[lane] = blk;
      __syncwarp();
      for (int k0 = 0; k0 < cur.cnt && ok_run; k0 += kIssueLanes) {
        const int n = min(kIssueLanes, cur.cnt - k0);
        bool ok_lane = true;
        if (lane < n) {
          const int i = issued + lane;
          const int s = i % kStages, round = i / kStages;
          const int bk = ids[k0 + lane];
          if (round > 0 && !mbar_wait(&empty[s], (round - 1) & 1)) {
            record_fault(p.fault, KVQ_FAULT_TIMEOUT);
            ok_lane = false;
          } else {
            meta[s] = make_int4(cur.u, cur.pg0 + k0 + lane, cur.nb, bk >= 0);
            if (bk >= 0) {
              // the whole record of (block, kv head) in one copy
              mbar_arrive_expect_tx(&full[s], stage_bytes);
              tma_load_2d(tiles + s * STAGE, &tmap, &full[s], 0, (bk * p.H + cur.kvh) * L::REC_ROWS);
            } else {
              mbar_arrive(&full[s]);
            }
          }
        }
        ok_run = __all_sync(0xffffffffu, ok_lane);
        issued += n;
      }
      cur = nxt;
    }
    // wait until every copy this CTA issued has landed before the CTA can exit
    if (lane == 0) {
      for (int i = max(0, issued - kStages); i < issued; ++i)
        if (!mbar_drain(&full[i % kStages], (i / kStages) & 1)) record_fault(p.fault, KVQ_FAULT_TIMEOUT);
    }
    return;
  }

  // ---------------------------------------------------------------- consumers
  const int npages = *range_pages;
  const int g = p.g;
  const int r = lane >> 2, j = lane & 3;
  float o[8][4];
  float m[2], l[2];
  int ev;                         // V normaliser exponent (PT only)
  float vlim = 0.f, vinv = 0.f;   // 2^(ev+1) and 2^-ev of the V normaliser (PT only)
  // Q^T fragments for head n = r: thread j covers d in [32j, 32j+32); k-step kc uses
  // d = 32j + 4kc + {0,1} (b0) and {2,3} (b1), the same d <-> k map the K codes use.
  uint32_t qb[8][2];              // fp16/bf16 Q fragments (FP8, BF16, FP16 caches)
  uint32_t qt[3][4][2];           // int8 Q terms (INT8 caches), see below
  float qscale = 0.f;
  int cur_u = -1, kvh = 0;

  // Load the query group of unit u = (sequence, kv head) into fragments and clear the
  // running softmax state.
  auto begin_unit = [&](int u, long qrow) {     // qrow: row of q ([B] decode, [Tq] prefill)
    const int b = u / p.H;
    kvh = u - b * p.H;
    qscale = p.scale_log2;
    // this thread's 32 query elements, kept packed (16-bit) until they are converted
    uint4 qraw[4];
    if (r < g) {
      const uint4* qp = reinterpret_cast<const uint4*>(
          static_cast<const uint16_t*>(p.q) + (qrow * p.Hq + kvh * g + r) * kD + 32 * j);
#pragma unroll
      for (int c = 0; c < 4; ++c) qraw[c] = qp[c];
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) qraw[c] = make_uint4(0, 0, 0, 0);
    }
    // PER_CHANNEL: K's scale of channel d multiplies every code of that channel, so it
    // folds into q_d once per unit (q . (c * s) = (q * s) . c)
    const float* kch = nullptr;
    if constexpr (!PT && Code<CD>::B == 1) {
      if (p.mode == KVQ_SCALE_PER_CHANNEL) kch = p.k_static + kvh * kD + 32 * j;
    }
    auto qv = [&](int e) {
      const uint32_t w2 = (&qraw[e >> 3].x)[(e & 7) >> 1];
      const uint16_t h = static_cast<uint16_t>((e & 1) ? (w2 >> 16) : (w2 & 0xFFFFu));
      const float f = p.act_fp16 ? __half2float(__ushort_as_half(h)) : __bfloat162float(__ushort_as_bfloat16(h));
      return kch != nullptr ? f * kch[e] : f;
    };
    if constexpr (CD == KVQ_DTYPE_INT8) {
      // q = sq * (Q0 + Q1/128 + Q2/16384) with int8 terms, sq = max|q| / 127 over the
      // group: |Q1|, |Q2| <= 64 and the error is about max|q| * 2^-22, so K . Q runs on
      // the integer tensor cores (K codes used as they are, int32 sums exact).
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(qv(e)));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const float sq = amax / 127.f;
      const float inv = amax > 0.f ? 127.f / amax : 0.f;
      // k-step kc: b0 <- elements 8kc..8kc+3, b1 <- 8kc+4..8kc+7 of [32j, 32j+32)
#pragma unroll
      for (int t = 0; t < 3; ++t)
#pragma unroll
        for (int kc = 0; kc < 4; ++kc) qt[t][kc][0] = qt[t][kc][1] = 0;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float x = qv(e);
        const int q0 = max(-127, min(127, __float2int_rn(x * inv)));
        const float r1 = fmaf(-static_cast<float>(q0), sq, x);
        const int q1 = max(-127, min(127, __float2int_rn(r1 * inv * 128.f)));
        const float r2 = fmaf(-static_cast<float>(q1), sq * (1.f / 128.f), r1);
        const int q2 = max(-127, min(127, __float2int_rn(r2 * inv * 16384.f)));
        const int sh = 8 * (e & 3), kc = e >> 3, hb = (e >> 2) & 1;
        qt[0][kc][hb] |= static_cast<uint32_t>(q0 & 0xFF) << sh;
        qt[1][kc][hb] |= static_cast<uint32_t>(q1 & 0xFF) << sh;
        qt[2][kc][hb] |= static_cast<uint32_t>(q2 & 0xFF) << sh;
      }
      qscale *= sq;
    } else if constexpr (kBf16) {
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) {
        qb[kc][0] = pack_bf16x2(qv(4 * kc), qv(4 * kc + 1));
        qb[kc][1] = pack_bf16x2(qv(4 * kc + 2), qv(4 * kc + 3));
      }
    } else {
      // power-of-two scaling keeps the group inside fp16's range; exact for the normal
      // range, and undone on the fp32 scores
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(qv(e)));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      int eq = 0;
      if (!p.act_fp16 && amax > 0.f) eq = ilogbf(amax) - 13;
      const float down = ldexpf(1.f, -eq);
      qscale = ldexpf(qscale, eq);
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) {
        qb[kc][0] = pack_f16x2(qv(4 * kc) * down, qv(4 * kc + 1) * down);
        qb[kc][1] = pack_f16x2(qv(4 * kc + 2) * down, qv(4 * kc + 3) * down);
      }
    }
    if constexpr (!PT) {
      if (p.mode == KVQ_SCALE_PER_HEAD || p.mode == KVQ_SCALE_PER_TENSOR)
        qscale *= p.k_static[p.mode == KVQ_SCALE_PER_HEAD ? kvh : 0];
    }
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
    ev = INT_MIN;
    vlim = 0.f;
    vinv = 0.f;
#pragma unroll
    for (int md = 0; md < 8; ++md)
#pragma unroll
      for (int c = 0; c < 4; ++c) o[md][c] = 0.f;
  };

  // Write this warp's partial of unit cur_u: unnormalised O, running max and sum per head.
  auto end_unit = [&]() {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l[0] += __shfl_xor_sync(0xffffffffu, l[0], off);
      l[1] += __shfl_xor_sync(0xffffffffu, l[1], off);
    }
    float vmul = 1.f;
    if constexpr (PT) vmul = ev == INT_MIN ? 0.f : ldexpf(1.f, ev);
    if constexpr (!PT) {
      if (p.mode == KVQ_SCALE_PER_HEAD) vmul = p.v_static[kvh];
      if (p.mode == KVQ_SCALE_PER_TENSOR) vmul = p.v_static[0];
    }
    // PER_CHANNEL: V's scale of channel d multiplies output channel d
    const float* vch = nullptr;
    if constexpr (!PT && Code<CD>::B == 1) {
      if (p.mode == KVQ_SCALE_PER_CHANNEL) vch = p.v_static + kvh * kD;
    }
    const long slot = (static_cast<long>(cur_u) + cta) * kSegWarps + warp;
    float* wo = p.ws_o + slot * g * kD;
    float* wml = p.ws_ml + slot * g * 2;
    const int h0 = 2 * j, h1 = 2 * j + 1;
#pragma unroll
    for (int md = 0; md < 8; ++md) {
      const int d0 = 16 * r + 2 * md;
      float m0 = vmul, m1 = vmul;
      if (vch != nullptr) {
        const float2 cv = *reinterpret_cast<const float2*>(vch + d0);
        m0 = cv.x;
        m1 = cv.y;
      }
      if (h0 < g) *reinterpret_cast<float2*>(wo + h0 * kD + d0) = make_float2(o[md][0] * m0, o[md][2] * m1);
      if (h1 < g) *reinterpret_cast<float2*>(wo + h1 * kD + d0) = make_float2(o[md][1] * m0, o[md][3] * m1);
    }
    if (r == 0) {
      if (h0 < g) *reinterpret_cast<float2*>(wml + 2 * h0) = make_float2(m[0], l[0]);
      if (h1 < g) *reinterpret_cast<float2*>(wml + 2 * h1) = make_float2(m[1], l[1]);
    }
  };

  // Prefill: normalise and store this warp's output rows (query row qrow, its g heads).
  auto write_rows = [&](long qrow) {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l[0] += __shfl_xor_sync(0xffffffffu, l[0], off);
      l[1] += __shfl_xor_sync(0xffffffffu, l[1], off);
    }
    float vmul = 1.f;
    if constexpr (PT) vmul = ev == INT_MIN ? 0.f : ldexpf(1.f, ev);
    if constexpr (!PT) {
      if (p.mode == KVQ_SCALE_PER_HEAD) vmul = p.v_static[kvh];
      if (p.mode == KVQ_SCALE_PER_TENSOR) vmul = p.v_static[0];
    }
    const float* vch = nullptr;
    if constexpr (!PT && Code<CD>::B == 1) {
      if (p.mode == KVQ_SCALE_PER_CHANNEL) vch = p.v_static + kvh * kD;
    }
    const float inv0 = l[0] > 0.f ? 1.f / l[0] : 0.f, inv1 = l[1] > 0.f ? 1.f / l[1] : 0.f;
    const int h0 = 2 * j, h1 = 2 * j + 1;
    const long base = (qrow * p.Hq + static_cast<long>(kvh) * g) * kD;
#pragma unroll
    for (int md = 0; md < 8; ++md) {
      const int d0 = 16 * r + 2 * md;
      float m0 = vmul, m1 = vmul;
      if (vch != nullptr) {
        const float2 cv = *reinterpret_cast<const float2*>(vch + d0);
        m0 = cv.x;
        m1 = cv.y;
      }
      if (h0 < g) {
        store_out(p, base + h0 * kD + d0, o[md][0] * m0 * inv0);
        store_out(p, base + h0 * kD + d0 + 1, o[md][2] * m1 * inv0);
      }
      if (h1 < g) {
        store_out(p, base + h1 * kD + d0, o[md][1] * m0 * inv1);
        store_out(p, base + h1 * kD + d0 + 1, o[md][3] * m1 * inv1);
      }
    }
  };

  // Per-thread byte offsets inside a stage tile.  The 128-byte swizzle repeats every 8
  // rows of 128 bytes, so token row t + 8 sits exactly 8 * ROWB bytes after row t.
  // K: token rows r and r+8, this thread's 32 codes [32j, 32j+32) of each row.
  // V: token rows 2j, 2j+1, 2j+8, 2j+9, this thread's 16 channels [16r, 16r+16).
  constexpr int KCH = 2 * Code<CD>::B;          // 16-byte chunks per K row segment
  constexpr int VCH = Code<CD>::B;              // 16-byte chunks per V row segment
  constexpr int R8 = 8 * ROWB;
  static_assert(ROWB % 128 == 0, "token rows are whole swizzle rows");
  int koff[KCH], voff[2][VCH];
#pragma unroll
  for (int c = 0; c < KCH; ++c) koff[c] = swzb(r * ROWB + 32 * Code<CD>::B * j + 16 * c);
#pragma unroll
  for (int c = 0; c < VCH; ++c) {
    const int b = 16 * Code<CD>::B * r + 16 * c;
    voff[0][c] = swzb(L::OFF_V + (2 * j) * ROWB + b);
    voff[1][c] = swzb(L::OFF_V + (2 * j + 1) * ROWB + b);
  }
  // per-token scales (K of tokens 0..15, then V) fill one 128-byte row whose index is a
  // multiple of 8, which the swizzle leaves in place
  static_assert(!PT || (L::OFF_S % 1024 == 0 && 8 * BS == 128), "scale row layout");
  const int soff = L::OFF_S + 4 * r;

  // prefill: this warp's query token (row of q and out) and its causal window [0, t1)
  long pf_row = 0;
  int pf_t1 = 0;
  bool pf_active = false;
  if constexpr (PF) {
    const int idx = pf_q0 + warp;
    pf_active = idx < pf_L;
    pf_row = p.q_start[pf_b] + idx;
    pf_t1 = pf_n - pf_L + idx + 1;
    cur_u = pf_b * p.H + pf_kvh;
    if (pf_active) begin_unit(cur_u, pf_row);
  }

  for (int i = PF ? 0 : warp; i < npages; i += PF ? 1 : kConsumers) {
    const int s = i % kStages;
    // all lanes wait; the decision is made warp-uniform before any shuffle below
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (i / kStages) & 1))) {
      if (lane == 0) record_fault(p.fault, KVQ_FAULT_TIMEOUT);
      break;
    }
    const int4 mt = meta[s];
    if constexpr (!PF) {
      if (mt.x != cur_u) {              // warp-uniform: a new (sequence, kv head) unit
        if (cur_u >= 0) end_unit();
        cur_u = mt.x;
        begin_unit(cur_u, cur_u / p.H);
      }
    }
    const uint8_t* st = tiles + s * STAGE;
    const bool pvalid = mt.w != 0;
    const int pos0 = mt.y * BS, t1 = PF ? pf_t1 : mt.z;
    if constexpr (PF) {
      if (!pf_active || pos0 >= t1) {   // nothing of this page is in the warp's window
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        continue;
      }
    }
    const bool full_page = pvalid && pos0 + BS <= t1;          // warp-uniform
    // ------------------------------------------------ stage -> registers, then hand the
    // stage back to the producer before any math, so the ring refills during compute
    // (16-bit codes: V is read after the K contraction, when the K fragments are dead,
    // which keeps 32 fewer registers live; those pages are HBM-bound either way)
    constexpr bool kEarlyV = Code<CD>::B == 1;
    uint4 kw[2][KCH], vw[4][VCH];
#pragma unroll
    for (int c = 0; c < KCH; ++c) {
      kw[0][c] = lds128(st + koff[c]);
      kw[1][c] = lds128(st + koff[c] + R8);
    }
    auto load_v_and_release = [&]() {
#pragma unroll
      for (int c = 0; c < VCH; ++c) {
        vw[0][c] = lds128(st + voff[0][c]);
        vw[1][c] = lds128(st + voff[1][c]);
        vw[2][c] = lds128(st + voff[0][c] + R8);
        vw[3][c] = lds128(st + voff[1][c] + R8);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    };
    float ks0 = 1.f, ks1 = 1.f, vs0 = 0.f, vs1 = 0.f;
    if constexpr (PT) {
      const float* sc = reinterpret_cast<const float*>(st + soff);
      ks0 = sc[0];
      ks1 = sc[8];
      vs0 = sc[BS];
      vs1 = sc[BS + 8];
    }
    if constexpr (kEarlyV) load_v_and_release();
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
    if constexpr (!kEarlyV) load_v_and_release();
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
  if constexpr (PF) {
    if (pf_active) write_rows(pf_row);
  } else {
    if (cur_u >= 0) end_unit();
  }
}

template <int CD, int BS, bool PT, bool PF>
cudaError_t launch_t(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s) {
  using L = Layout<CD, BS, PT>;
  if (a.geo.record != L::REC) return cudaErrorInvalidValue;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(decode_mma_kernel<CD, BS, PT, PF>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES);
    // three rings per SM need the whole unified L1 / shared memory as shared memory
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(decode_mma_kernel<CD, BS, PT, PF>,
                                      cudaFuncAttributePreferredSharedMemoryCarveout,
                                      cudaSharedmemCarveoutMaxShared);
  });
  if (attr_err != cudaSuccess) return attr_err;
  CUtensorMap tm;
  const long rows = static_cast<long>(a.geo.NB) * a.geo.H * L::REC_ROWS;
  if (!make_pages_map(&tm, a.c->pages, rows, L::REC_ROWS)) return cudaErrorInvalidValue;
  const dim3 grid = PF ? dim3((a.max_q_len + kConsumers - 1) / kConsumers, a.geo.H, a.batch)
                       : dim3(a.plan.ctas);
  if (!PF && a.plan.ctas < 1) return cudaErrorInvalidValue;
  return launch_dependent(decode_mma_kernel<CD, BS, PT, PF>, grid, dim3(kThreads), L::BYTES, s, p, tm);
}

template <int CD, bool PT, bool PF>
cudaError_t launch_bs(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s) {
  if (a.geo.bs == 16) return launch_t<CD, 16, PT, PF>(a, p, s);
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
// (rec_rows rows), copied with 128-byte swizzle.  L2 fills are promoted to 256 bytes only
// when records are whole 256-byte units: a 4224-byte record (33 rows) would otherwise pull
// 128 bytes of its neighbour into L2 at every other record.
bool make_pages_map(CUtensorMap* map, const void* base, long rows, int rec_rows) {
  auto enc = encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {128, static_cast<cuuint32_t>(rec_rows)};
  cuuint32_t es[2] = {1, 1};
  const CUresult res = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                           box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           rec_rows % 2 == 0 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B
                                             : CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

bool make_rows_map(CUtensorMap* map, const void* base, long rows, int row_bytes, int box_rows) {
  auto enc = encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  cuuint32_t box[2] = {128, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1, 1};
  const CUresult res = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                           box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS;
}

bool mma_supported(const Geometry& g, int groups) {
  // any group of 1..8 query heads fills (part of) the N = 8 side of the tiles; the kernel
  // is bound by moving pages, so a partly empty tile costs little
  if (g.D != kD || groups < 1 || groups > 8) return false;
  if (g.bs != 16) return false;   // 8 stages of 16-token tiles fit shared memory 3 CTAs/SM
  switch (g.cache_dtype) {
    case KVQ_DTYPE_INT8:
    case KVQ_DTYPE_FP8_E4M3:
    case KVQ_DTYPE_BF16:
    case KVQ_DTYPE_FP16: return true;
  }
  return false;
}

template <bool PF>
static cudaError_t launch_mma_mode(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s) {
  const bool pt = a.geo.scale_mode == KVQ_SCALE_PER_TOKEN_HEAD;
  switch (a.geo.cache_dtype) {
    case KVQ_DTYPE_INT8:
      return pt ? launch_bs<KVQ_DTYPE_INT8, true, PF>(a, p, s) : launch_bs<KVQ_DTYPE_INT8, false, PF>(a, p, s);
    case KVQ_DTYPE_FP8_E4M3:
      return pt ? launch_bs<KVQ_DTYPE_FP8_E4M3, true, PF>(a, p, s)
                : launch_bs<KVQ_DTYPE_FP8_E4M3, false, PF>(a, p, s);
    case KVQ_DTYPE_BF16: return launch_bs<KVQ_DTYPE_BF16, false, PF>(a, p, s);
    case KVQ_DTYPE_FP16: return launch_bs<KVQ_DTYPE_FP16, false, PF>(a, p, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_mma(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s) {
  return launch_mma_mode<false>(a, p, s);
}

cudaError_t launch_prefill_mma(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s) {
  return launch_mma_mode<true>(a, p, s);
}

}  // namespace kvq
