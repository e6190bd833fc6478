// Pieces shared by the decode kernels: parameters, per-sequence bounds, block lookup,
// and the epilogue that writes either a split partial or the final output row.
#pragma once

#include <cuda.h>

#include "kvq_internal.cuh"

namespace kvq {

struct DecodeParams {
  const void* q;             // [B][Hq][D] act
  const int32_t* tables;     // [B][max_blocks]
  const int32_t* lens;       // [B]
  const int32_t* seq_ids;    // [B] or null (INT4 ring)
  int max_blocks, max_context;
  const uint8_t* pages;      // [NB][H][record]
  const float* k_static;     // PER_HEAD / PER_TENSOR scales
  const float* v_static;
  const void* residual;
  int record, off_v, off_s, row_bytes;
  int NB, bs, H, Hq, D, g, cap, rlen, max_seqs, mode;
  int splits, chunk;
  int ring_split;            // INT4 with tensor-core pages: slot of the ring partial, else -1
  int rows;                  // batch * Hq
  int batch;
  int ctas;                  // page-balanced tensor-core kernel: its grid size, else 0
  int act_fp16;              // activations (q, ring) are fp16 rather than bf16
  float scale_log2;
  void* out;
  int out_dtype;
  float* ws_o;               // [B][Hq][S][D]
  float* ws_ml;              // [B][Hq][S][2]  (max, sum) in the log2 domain
  int32_t* fault;
  // append step (kvq_append_decode_attention), else null: this step's K / V row of every
  // sequence, [B][H][D] act dtype, stored at position context_lens[b] - 1 before decode
  const void* k_new;
  const void* v_new;
  uint8_t* pages_w;          // the pool, writable (append step only)
  void* residual_w;          // the INT4 / INT2 ring, writable (append step only)
  // prefill (kvq_prefill_attention): q is [Tq][Hq][D]; the queries of sequence b are rows
  // q_start[b] .. q_start[b+1]-1, the newest tokens of the sequence
  const int32_t* q_start;
  int max_q_len;             // prefill: host bound on a sequence's query count
};

struct SeqInfo {
  int n;     // positions to attend to (0 when the entry was rejected)
  int qb;    // INT4: positions read from blocks; the rest come from the ring
  int sid;   // INT4: ring sequence
};

// Bounds of sequence b.  A context length outside [0, max_context] or beyond what the
// block table can address, or an INT4 ring id outside [0, max_seqs), rejects the whole
// sequence (its output row is zero).  `report` selects the one thread that counts it.
__device__ __forceinline__ SeqInfo seq_info(const DecodeParams& p, int b, bool int4,
                                            bool report = false) {
  SeqInfo s;
  int n = p.lens[b];
  int bits = 0;
  if (n < 0 || n > p.max_context) bits |= KVQ_FAULT_CONTEXT;
  s.sid = b;
  s.qb = n;
  if (int4) {
    s.sid = p.seq_ids ? p.seq_ids[b] : b;
    if (s.sid < 0 || s.sid >= p.max_seqs) bits |= KVQ_FAULT_SEQ;
    const int over = n - p.rlen;
    s.qb = over > 0 ? 64 * (over / 64) : 0;
    if (s.qb / 64 > p.max_blocks) bits |= KVQ_FAULT_CONTEXT;
  } else if (static_cast<long>(n) > static_cast<long>(p.max_blocks) * p.bs) {
    bits |= KVQ_FAULT_CONTEXT;
  }
  if (bits) {
    if (report) record_fault(p.fault, bits);
    n = 0;
    s.qb = 0;
  }
  s.n = n;
  return s;
}

// ---------------------------------------------------------------- page-balanced schedule
// The dense tensor-core kernel runs one CTA per resident slot (kMmaCtasPerSM per SM).  The
// pages of all (sequence, kv head) units, concatenated in the order (sequence, kv head,
// page), are cut into ctas contiguous ranges of equal size: CTA c takes
// [P c / C, P (c + 1) / C).  A CTA range crossing unit boundaries covers several segments
// (unit, CTA); each consumer warp of the CTA writes one partial per segment it saw, into
// slot (unit + c) * kSegWarps + warp.  (Going from one segment to the next raises the unit
// index, the CTA index or both, so unit + c never repeats and there are at most
// units + C - 1 segments.)  The segment reduce merges them.
constexpr int kSegWarps = 4;
constexpr int kMmaCtasPerSM = 3;

__device__ __forceinline__ long long range_start(long long P, int c, int C) {
  return P * c / C;
}

// Pages of sequence b (0 when its entry is rejected).
__device__ __forceinline__ int seq_pages(const DecodeParams& p, int b, bool report = false) {
  return (seq_info(p, b, false, report).n + p.bs - 1) / p.bs;
}

// Tokens of a dense-cache sequence whose raw context length is n: n itself, or 0 when
// seq_info would reject it (outside [0, max_context] or beyond the block table).
__device__ __forceinline__ int dense_len(const DecodeParams& p, int n) {
  const bool bad = n < 0 || n > p.max_context ||
                   static_cast<long>(n) > static_cast<long>(p.max_blocks) * p.bs;
  return bad ? 0 : n;
}

// Physical block of page `page` of sequence b, or -1 (counted) when out of range.
__device__ __forceinline__ int block_of(const DecodeParams& p, int b, int page) {
  const int blk = p.tables[static_cast<long>(b) * p.max_blocks + page];
  if (blk < 0 || blk >= p.NB) {
    record_fault(p.fault, KVQ_FAULT_BLOCK);
    return -1;
  }
  return blk;
}

__device__ __forceinline__ void store_out(const DecodeParams& p, long idx, float v) {
  if (p.out_dtype == KVQ_DTYPE_FP32) static_cast<float*>(p.out)[idx] = v;
  else if (p.out_dtype == KVQ_DTYPE_BF16) static_cast<__nv_bfloat16*>(p.out)[idx] = __float2bfloat16_rn(v);
  else static_cast<__half*>(p.out)[idx] = __float2half_rn(v);
}

// M, L: running max and sum (log2 domain) of this CTA's share; O: unnormalised output.
__device__ __forceinline__ void store_partial_or_output(const DecodeParams& p, int b, int hq,
                                                        int split, int d, float M, float L,
                                                        float O) {
  const long row = static_cast<long>(b) * p.Hq + hq;
  if (p.splits == 1) {
    store_out(p, row * p.D + d, L > 0.f ? O / L : 0.f);
    return;
  }
  const long part = row * p.splits + split;
  p.ws_o[part * p.D + d] = O;
  if (d == 0) {
    p.ws_ml[part * 2] = M;
    p.ws_ml[part * 2 + 1] = L;
  }
}

cudaError_t launch_decode_simt(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s);
cudaError_t launch_decode_mma(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s);
cudaError_t launch_prefill_mma(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s);
// chunked prefill on tcgen05 (128-row query tiles): head_dim 128, block 16, dense caches,
// GQA groups dividing 128
bool prefill_tc_supported(const Geometry& g, int group);
cudaError_t launch_prefill_tc(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s);
// true when the tensor-core kernel covers this geometry and GQA group size
bool mma_supported(const Geometry& g, int group);
bool int4_mma_supported(const Geometry& g, int group);
cudaError_t launch_decode_int4(const DecodeArgs& a, const DecodeParams& p, cudaStream_t s);
// Tensor map over the pages pool viewed as rows of 128 bytes; one box = one record.
bool make_pages_map(CUtensorMap* map, const void* base, long rows, int rec_rows);
// Tensor map over `rows` rows of `row_bytes` bytes; one box is 128 bytes of `box_rows`
// consecutive rows, copied with 128-byte swizzle (the tensor cores' tile layout).
bool make_rows_map(CUtensorMap* map, const void* base, long rows, int row_bytes, int box_rows);

}  // namespace kvq
