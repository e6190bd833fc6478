// Decode dispatch: split plan, kernel choice, and the split-K log-sum-exp reduce.
//
// The reduce merges the S partials (m_s, l_s, o_s) of each (sequence, query head):
//   M = max_s m_s,  L = sum_s l_s 2^(m_s - M),  out = sum_s o_s 2^(m_s - M) / L,
// the usual merge of softmax partial sums over disjoint token ranges (the pages leave
// the split of long contexts open; it follows from decode reading every cached
// position at each step, [P-prod] "为什么长上下文更需要 KV Cache Quantization").
#include <algorithm>

#include "kvq_decode_common.cuh"
#include "kvq_ptx.cuh"

namespace kvq {
namespace {

// One warp per (sequence, query head): lane k computes the weight of split slot k
// (k < 32; longer lists loop), lanes own 4 consecutive channels of the output.
__global__ void __launch_bounds__(256) split_reduce_kernel(DecodeParams p, bool int4) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);   // b * Hq + hq
  const int lane = threadIdx.x & 31;
  if (row >= p.rows) return;
  const int b = row / p.Hq;
  const SeqInfo si = seq_info(p, b, int4);
  // splits that hold work: the token splits covering [0, n), or, when the INT4 ring has
  // a split of its own, the block splits covering [0, qb) plus the ring split
  const int S = (p.ring_split >= 0 ? si.qb + p.chunk - 1 : si.n + p.chunk - 1) / p.chunk;
  const bool ring = p.ring_split >= 0 && si.n > si.qb;
  const int K = S + (ring ? 1 : 0);
  // the split count depends only on the call's inputs; the partials are read after the
  // decode kernels are done (the last of them waits for the one before it)
  griddep_wait();
  const float* ml = p.ws_ml + static_cast<long>(row) * p.splits * 2;
  const float* o = p.ws_o + static_cast<long>(row) * p.splits * p.D;
  auto slot = [&](int k) { return k < S ? k : p.ring_split; };
  const bool has_d = 4 * lane < p.D;
  auto row_of = [&](int k) {          // this lane's 4 channels of partial k (0 past the list)
    return (has_d && k < K) ? *reinterpret_cast<const float4*>(o + static_cast<long>(slot(k)) * p.D + 4 * lane)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  // every listed split holds work and every partial row is read, so the first sixteen rows
  // are loaded together with the (max, sum) pairs rather than after the weights
  constexpr int kB = 16;
  float4 v[kB];
#pragma unroll
  for (int t = 0; t < kB; ++t) v[t] = row_of(t);
  // max over the splits
  float M = -INFINITY;
  for (int k = lane; k < K; k += 32) M = fmaxf(M, ml[2 * slot(k)]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k0 = 0; k0 < K; k0 += 32) {
    const int k = k0 + lane;
    float w = 0.f;
    if (k < K) {
      const float mk = ml[2 * slot(k)];
      w = (M == -INFINITY || mk == -INFINITY) ? 0.f : exp2f(mk - M);
      L = fmaf(ml[2 * slot(k) + 1], w, L);
    }
    const int n = min(32, K - k0);
    for (int i0 = 0; i0 < n; i0 += kB) {
      if (k0 + i0 > 0) {
#pragma unroll
        for (int t = 0; t < kB; ++t) v[t] = row_of(k0 + i0 + t);
      }
#pragma unroll
      for (int t = 0; t < kB; ++t) {
        const float wi = __shfl_sync(0xffffffffu, w, i0 + t);   // 0 past the list
        acc.x = fmaf(v[t].x, wi, acc.x);
        acc.y = fmaf(v[t].y, wi, acc.y);
        acc.z = fmaf(v[t].z, wi, acc.z);
        acc.w = fmaf(v[t].w, wi, acc.w);
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
  const float inv = L > 0.f ? 1.f / L : 0.f;
  if (has_d) {
    const long base = static_cast<long>(row) * p.D + 4 * lane;
    store_out(p, base, acc.x * inv);
    store_out(p, base + 1, acc.y * inv);
    store_out(p, base + 2, acc.z * inv);
    store_out(p, base + 3, acc.w * inv);
  }
}

// Merge of the dense tensor-core kernel's per-warp partials.  One warp per (sequence,
// query head): it recomputes the page partition (total pages, the pages before its
// sequence), finds the CTAs whose ranges meet its unit's pages, and takes the partial of
// every consumer warp that saw at least one of those pages.  Lane k describes candidate
// k (CTA c_first + k / kSegWarps, warp k % kSegWarps); the partial rows are then read
// sixteen at a time so their loads overlap.
__global__ void __launch_bounds__(256) segment_reduce_kernel(DecodeParams p) {
  const int C = p.ctas;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);   // b * Hq + hq
  const int lane = threadIdx.x & 31;
  // the partition and the candidate range depend only on the call's inputs (context lengths,
  // block tables), which the decode kernel does not write: they are worked out before the
  // wait for its partials, overlapping its tail
  const bool active = row < p.rows;
  const int b = active ? row / p.Hq : 0, hq = active ? row - b * p.Hq : 0;
  const int kvh = hq / p.g, h = hq - kvh * p.g;
  long long tot = 0, before = 0;
  int npb = 0;
  for (int b0 = 0; b0 < p.batch; b0 += 32) {
    const int bb = b0 + lane;
    const int np = bb < p.batch ? seq_pages(p, bb) : 0;
    int t = np, q = bb < b ? np : 0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      t += __shfl_xor_sync(0xffffffffu, t, off);
      q += __shfl_xor_sync(0xffffffffu, q, off);
    }
    tot += t;
    before += q;
    if (b >= b0 && b < b0 + 32) npb = __shfl_sync(0xffffffffu, np, b - b0);
  }
  const long long P = tot * p.H;
  const long long U0 = before * p.H + static_cast<long long>(kvh) * npb, U1 = U0 + npb;
  int c_first = 0, c_last = -1;
  if (npb > 0) {
    // CTA c covers [P c / C, P (c+1) / C): the last one starting at or before U0, and
    // the last one starting before U1
    c_first = static_cast<int>(((U0 + 1) * C + P - 1) / P) - 1;
    c_last = static_cast<int>((U1 * C + P - 1) / P) - 1;
  }
  const int K = (c_last - c_first + 1) * kSegWarps;
  griddep_wait();                      // the partials of the decode kernel
  if (!active) return;
  const long long u = static_cast<long long>(b) * p.H + kvh;
  const float* ml = p.ws_ml;
  const float* o = p.ws_o + 4 * lane;
  const bool has_d = 4 * lane < p.D;
  float M = -INFINITY, L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k0 = 0; k0 < K; k0 += 32) {
    // lane k: does candidate k0 + k hold a partial, and where
    const int k = k0 + lane;
    int slot = -1;
    float mk = -INFINITY, lk = 0.f;
    if (k < K) {
      const int c = c_first + k / kSegWarps, w = k % kSegWarps;
      const long long sc = range_start(P, c, C), ec = range_start(P, c + 1, C);
      const long long lo = sc > U0 ? sc : U0, hi = ec < U1 ? ec : U1;
      const long long len = hi - lo;
      const int first = static_cast<int>((lo - sc) % kSegWarps);   // warp of the first page
      if (len > 0 && (len >= kSegWarps || ((w - first + kSegWarps) % kSegWarps) < len)) {
        slot = static_cast<int>(((u + c) * kSegWarps + w) * p.g + h);
        const float2 v = *reinterpret_cast<const float2*>(ml + 2L * slot);
        mk = v.x;
        lk = v.y;
      }
    }
    // rescale what was merged so far to the new maximum
    float Mc = mk;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) Mc = fmaxf(Mc, __shfl_xor_sync(0xffffffffu, Mc, off));
    const float Mn = fmaxf(M, Mc);
    if (Mn != -INFINITY && Mn > M) {
      const float c0 = M == -INFINITY ? 0.f : exp2f(M - Mn);
      L *= c0;
      acc.x *= c0; acc.y *= c0; acc.z *= c0; acc.w *= c0;
      M = Mn;
    }
    const float w = (slot >= 0 && mk != -INFINITY) ? exp2f(mk - M) : 0.f;
    L = fmaf(lk, w, L);
    const int n = min(32, K - k0);
    constexpr int kRows = 16;          // partial rows in flight per lane
    for (int i0 = 0; i0 < n; i0 += kRows) {
      float wi[kRows];
      int si[kRows];
      float4 v[kRows];
#pragma unroll
      for (int t = 0; t < kRows; ++t) {
        const int i = min(i0 + t, 31);
        wi[t] = __shfl_sync(0xffffffffu, w, i);
        si[t] = __shfl_sync(0xffffffffu, slot, i);
        if (i0 + t >= n) wi[t] = 0.f;
      }
#pragma unroll
      for (int t = 0; t < kRows; ++t)
        v[t] = (has_d && wi[t] != 0.f) ? *reinterpret_cast<const float4*>(o + static_cast<long>(si[t]) * p.D)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int t = 0; t < kRows; ++t) {
        acc.x = fmaf(v[t].x, wi[t], acc.x);
        acc.y = fmaf(v[t].y, wi[t], acc.y);
        acc.z = fmaf(v[t].z, wi[t], acc.z);
        acc.w = fmaf(v[t].w, wi[t], acc.w);
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
  const float inv = L > 0.f ? 1.f / L : 0.f;
  if (has_d) {
    const long base = static_cast<long>(row) * p.D + 4 * lane;
    store_out(p, base, acc.x * inv);
    store_out(p, base + 1, acc.y * inv);
    store_out(p, base + 2, acc.z * inv);
    store_out(p, base + 3, acc.w * inv);
  }
}

}  // namespace

// Splits for the INT4 tensor-core kernel: one CTA per (sequence, kv head, split); pick the
// split count whose CTA count fills whole waves of the resident slots (per_sm CTAs per SM:
// 2 for that kernel, bound by its registers), preferring fewer splits, with at least 256
// tokens per split.
static void plan_mma(const Geometry& g, int batch, int max_context, DecodePlan* p, long per_sm) {
  const long units = static_cast<long>(batch) * g.H;
  const long slots = per_sm * p->sms;
  const long max_s = std::max(1L, std::min(64L, (static_cast<long>(max_context) + 255) / 256));
  long best_s = 1;
  double best = -1.0;
  for (long S = 1; S <= max_s; ++S) {
    const long ctas = units * S;
    const long waves = (ctas + slots - 1) / slots;
    const double eff = static_cast<double>(ctas) / static_cast<double>(waves * slots);
    const double score = eff - 0.004 * static_cast<double>(S);
    if (score > best + 1e-9) { best = score; best_s = S; }
  }
  long chunk = (static_cast<long>(max_context) + best_s - 1) / best_s;
  chunk = std::max(1L, (chunk + g.bs - 1) / g.bs) * g.bs;
  p->splits = static_cast<int>(std::max(1L, (static_cast<long>(max_context) + chunk - 1) / chunk));
  p->chunk = static_cast<int>(chunk);
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
    cudaGetLastError();              // clear the error a failed query leaves behind
    return 148;
  }
  return n;
}

kvq_status plan_decode(const Geometry& g, int batch, int num_q_heads, int max_context,
                       DecodePlan* p) {
  p->sms = device_sm_count();
  p->g = num_q_heads / g.H;
  p->kernel = mma_supported(g, p->g) ? 1 : 0;
  // per-channel scales are folded into q and the output by the tensor-core kernel only
  if (g.scale_mode == KVQ_SCALE_PER_CHANNEL && p->kernel != 1) return KVQ_ERR_UNSUPPORTED;
  if (int4_mma_supported(g, p->g)) {
    // INT4 blocks on tensor cores: splits over the quantized prefix (64-token blocks)
    // plus one split for the residual ring, computed by the CUDA-core kernel
    p->kernel = 2;
    p->g_tile = p->g;
    const int max_qb = 64 * (std::max(max_context - g.residual_len, 0) / 64);
    Geometry gg = g;
    gg.bs = 64;
    plan_mma(gg, batch, std::max(max_qb, 64), p, 2);
    p->splits += 1;                              // the ring
    p->ctas = 0;
    const size_t rows = static_cast<size_t>(batch) * num_q_heads * p->splits;
    p->ws_ml_off = (rows * g.D * sizeof(float) + 255) / 256 * 256;
    p->ws_bytes = p->ws_ml_off + rows * 2 * sizeof(float);
    return KVQ_OK;
  }
  if (p->kernel == 1) {
    // page-balanced CTAs; partial slots (unit + cta) * kSegWarps + warp, g heads each
    p->g_tile = p->g;
    p->splits = 0;
    p->chunk = 0;
    p->ctas = kMmaCtasPerSM * p->sms;
    const size_t slots = (static_cast<size_t>(batch) * g.H + p->ctas - 1) * kSegWarps;
    const size_t heads = slots * p->g;
    p->ws_ml_off = (heads * g.D * sizeof(float) + 255) / 256 * 256;
    p->ws_bytes = p->ws_ml_off + heads * 2 * sizeof(float);
    return KVQ_OK;
  }
  p->g_tile = (p->g % 2 == 0) ? 2 : 1;
  const long units = static_cast<long>(batch) * g.H * (p->g / p->g_tile);
  const int gran = low_bit(g.cache_dtype) ? 64 : g.bs;
  // aim for about 8 resident CTAs per SM, without splits shorter than 256 tokens
  const long target = 8L * p->sms;
  long S = units > 0 ? (target + units - 1) / units : 1;
  const long max_split_by_len = std::max(1L, (static_cast<long>(max_context) + 255) / 256);
  S = std::max(1L, std::min(S, max_split_by_len));
  long chunk = (static_cast<long>(max_context) + S - 1) / S;
  chunk = std::max(1L, (chunk + gran - 1) / gran) * gran;
  S = std::max(1L, (static_cast<long>(max_context) + chunk - 1) / chunk);
  p->splits = static_cast<int>(S);
  p->chunk = static_cast<int>(chunk);
  p->ctas = 0;
  p->ws_bytes = 0;
  p->ws_ml_off = 0;
  if (S > 1) {
    const size_t rows = static_cast<size_t>(batch) * num_q_heads * S;
    p->ws_ml_off = (rows * g.D * sizeof(float) + 255) / 256 * 256;
    p->ws_bytes = p->ws_ml_off + rows * 2 * sizeof(float);
  }
  return KVQ_OK;
}

static DecodeParams make_params(const DecodeArgs& a) {
  const Geometry& g = a.geo;
  DecodeParams p{};
  p.q = a.q;
  p.tables = a.block_tables;
  p.lens = a.context_lens;
  p.seq_ids = a.seq_ids;
  p.max_blocks = a.max_blocks;
  p.max_context = a.max_context;
  p.pages = static_cast<const uint8_t*>(a.c->pages);
  p.k_static = a.c->k_scales;
  p.v_static = a.c->v_scales;
  p.residual = a.c->residual;
  p.record = g.record;
  p.off_v = g.off_v;
  p.off_s = g.off_s;
  p.row_bytes = g.row_bytes;
  p.NB = g.NB;
  p.bs = g.bs;
  p.H = g.H;
  p.Hq = a.Hq;
  p.D = g.D;
  p.g = a.plan.g;
  p.cap = g.residual_cap;
  p.rlen = g.residual_len;
  p.max_seqs = g.max_seqs;
  p.mode = g.scale_mode;
  p.splits = a.plan.splits;
  p.chunk = a.plan.chunk;
  p.ring_split = a.plan.kernel == 2 ? a.plan.splits - 1 : -1;
  p.rows = a.batch * a.Hq;
  p.batch = a.batch;
  p.ctas = a.plan.ctas;
  p.act_fp16 = g.act_dtype == KVQ_DTYPE_FP16;
  p.scale_log2 = a.scale_log2;
  p.out = a.out;
  p.out_dtype = a.out_dtype;
  p.ws_o = a.ws_o;
  p.ws_ml = a.ws_ml;
  p.fault = a.c->fault;
  p.k_new = a.k_new;
  p.v_new = a.v_new;
  p.pages_w = a.k_new != nullptr ? static_cast<uint8_t*>(a.c->pages) : nullptr;
  p.residual_w = a.k_new != nullptr ? a.c->residual : nullptr;
  p.q_start = a.q_start;
  p.max_q_len = a.max_q_len;
  return p;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  const Geometry& g = a.geo;
  DecodeParams p = make_params(a);
  if (a.batch == 0) return cudaSuccess;
  cudaError_t e;
  if (a.plan.kernel == 2) {
    // the ring split first: its kernel is small and releases its dependents as it starts,
    // so the block splits (launched as its dependent, reading nothing it writes) overlap it
    e = launch_decode_simt(a, p, s);                 // ring split
    if (e == cudaSuccess) e = launch_decode_int4(a, p, s);   // block splits
  } else {
    e = a.plan.kernel == 1 ? launch_decode_mma(a, p, s) : launch_decode_simt(a, p, s);
  }
  if (e != cudaSuccess) return e;
  if (a.plan.kernel == 1) {
    e = launch_dependent(segment_reduce_kernel, dim3((a.batch * a.Hq + 7) / 8), dim3(256), 0, s, p);
  } else if (p.splits > 1) {
    e = launch_dependent(split_reduce_kernel, dim3((a.batch * a.Hq + 7) / 8), dim3(256), 0, s, p,
                         low_bit(g.cache_dtype));
  }
  return e;
}

cudaError_t launch_prefill(const DecodeArgs& a, cudaStream_t s) {
  if (a.batch == 0) return cudaSuccess;
  if (prefill_tc_supported(a.geo, a.plan.g)) return launch_prefill_tc(a, make_params(a), s);
  return launch_prefill_mma(a, make_params(a), s);
}

}  // namespace kvq
