// C ABI entry points: host-side validation, layout arithmetic and dispatch.
// Declarations and the contract of every call are in include/kvq.h.
#include <cmath>
#include <cstdint>

#include "kvq_decode_common.cuh"

namespace kvq {

int code_bits(int cd) {
  switch (cd) {
    case KVQ_DTYPE_BF16:
    case KVQ_DTYPE_FP16: return 16;
    case KVQ_DTYPE_INT8:
    case KVQ_DTYPE_FP8_E4M3: return 8;
    case KVQ_DTYPE_INT4: return 4;
    case KVQ_DTYPE_INT2: return 2;
  }
  return 0;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Geometry and record layout of a descriptor (no pointer checks).
static kvq_status validate_geometry(const kvq_cache_desc* c, Geometry* g) {
  if (c == nullptr) return KVQ_ERR_INVALID_ARG;
  g->cache_dtype = c->cache_dtype;
  g->act_dtype = c->act_dtype;
  g->scale_mode = c->scale_mode;
  g->NB = c->num_blocks;
  g->bs = c->block_size;
  g->H = c->num_kv_heads;
  g->D = c->head_dim;
  g->group = c->group_size;
  g->residual_len = c->residual_len;
  g->residual_cap = c->residual_cap;
  g->max_seqs = c->max_seqs;
  if (code_bits(c->cache_dtype) == 0) return KVQ_ERR_INVALID_ARG;
  if (c->act_dtype != KVQ_DTYPE_BF16 && c->act_dtype != KVQ_DTYPE_FP16) return KVQ_ERR_INVALID_ARG;
  if (c->num_blocks < 1 || c->num_kv_heads < 1 || c->block_size < 1 || c->block_size > 1024)
    return KVQ_ERR_INVALID_ARG;
  if (c->head_dim != 64 && c->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
  switch (c->cache_dtype) {
    case KVQ_DTYPE_BF16:
    case KVQ_DTYPE_FP16:
      if (c->scale_mode != KVQ_SCALE_NONE) return KVQ_ERR_INVALID_ARG;
      if (c->cache_dtype != c->act_dtype) return KVQ_ERR_UNSUPPORTED;
      break;
    case KVQ_DTYPE_INT8:
    case KVQ_DTYPE_FP8_E4M3:
      if (c->scale_mode != KVQ_SCALE_PER_TOKEN_HEAD && c->scale_mode != KVQ_SCALE_PER_HEAD &&
          c->scale_mode != KVQ_SCALE_PER_TENSOR && c->scale_mode != KVQ_SCALE_PER_CHANNEL)
        return KVQ_ERR_INVALID_ARG;
      break;
    case KVQ_DTYPE_INT4:
    case KVQ_DTYPE_INT2:
      if (c->scale_mode != KVQ_SCALE_KIVI && c->scale_mode != KVQ_SCALE_KIVI_FLOAT_ZERO &&
          c->scale_mode != KVQ_SCALE_INT4_PER_TOKEN)
        return KVQ_ERR_INVALID_ARG;
      if (c->group_size != 64 || c->block_size != 64) return KVQ_ERR_UNSUPPORTED;
      if (c->residual_len < 0 || c->residual_cap < c->residual_len + c->group_size) return KVQ_ERR_INVALID_ARG;
      if (c->max_seqs < 1) return KVQ_ERR_INVALID_ARG;
      break;
  }
  g->row_bytes = c->head_dim * code_bits(c->cache_dtype) / 8;
  g->off_v = g->bs * g->row_bytes;
  g->off_s = 2 * g->bs * g->row_bytes;
  g->scale_bytes = 0;
  if (g->scale_mode == KVQ_SCALE_PER_TOKEN_HEAD) g->scale_bytes = 8 * g->bs;
  // INT4 / INT2: K (scale, zero) per channel [2][D] or per token [bs][D/64][2], then V per
  // token [bs][D/64][2], all float16; with bs = 64 both K forms take 4 * D bytes
  if (low_bit(g->cache_dtype)) g->scale_bytes = 4 * g->D + g->bs * (g->D / 64) * 4;
  g->record = (g->off_s + g->scale_bytes + 127) / 128 * 128;
  return KVQ_OK;
}

kvq_status validate_desc(const kvq_cache_desc* c, Geometry* g) {
  const kvq_status st = validate_geometry(c, g);
  if (st != KVQ_OK) return st;
  if (c->pages == nullptr || !aligned16(c->pages)) return KVQ_ERR_INVALID_ARG;
  if (c->scale_mode == KVQ_SCALE_PER_HEAD || c->scale_mode == KVQ_SCALE_PER_TENSOR ||
      c->scale_mode == KVQ_SCALE_PER_CHANNEL) {
    if (c->k_scales == nullptr || c->v_scales == nullptr) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(c->k_scales) || !aligned16(c->v_scales)) return KVQ_ERR_INVALID_ARG;
  }
  if (low_bit(c->cache_dtype) && (c->residual == nullptr || !aligned16(c->residual)))
    return KVQ_ERR_INVALID_ARG;
  return KVQ_OK;
}

static kvq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

}  // namespace kvq

using namespace kvq;

namespace {

// Shared by kvq_decode_attention and kvq_append_decode_attention (k_new / v_new null for
// the former).
kvq_status decode_entry(const kvq_cache_desc* c, const void* k_new, const void* v_new,
                        const void* q, int batch, int num_q_heads, const int32_t* block_tables,
                        int max_blocks_per_seq, const int32_t* context_lens,
                        const int32_t* seq_ids, int max_context, float softmax_scale, void* out,
                        int32_t out_dtype, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream) {
  Geometry g;
  kvq_status st = validate_desc(c, &g);
  if (st != KVQ_OK) return st;
  if (batch < 0 || num_q_heads < 1 || num_q_heads % g.H != 0 || max_context < 0 ||
      max_blocks_per_seq < 1)
    return KVQ_ERR_INVALID_ARG;
  if (out_dtype != KVQ_DTYPE_BF16 && out_dtype != KVQ_DTYPE_FP16 && out_dtype != KVQ_DTYPE_FP32)
    return KVQ_ERR_INVALID_ARG;
  if (!(softmax_scale >= 0.f) || !std::isfinite(softmax_scale)) return KVQ_ERR_INVALID_ARG;
  const bool append = k_new != nullptr || v_new != nullptr;
  if (append && (k_new == nullptr || v_new == nullptr || !aligned16(k_new) || !aligned16(v_new)))
    return KVQ_ERR_INVALID_ARG;
  if (batch == 0) return KVQ_OK;
  if (q == nullptr || block_tables == nullptr || context_lens == nullptr || out == nullptr)
    return KVQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out)) return KVQ_ERR_INVALID_ARG;
  DecodeArgs a{};
  a.c = c;
  a.geo = g;
  st = plan_decode(g, batch, num_q_heads, max_context, &a.plan);
  if (st != KVQ_OK) return st;
  // the append step lives in the dense tensor-core kernel's producer, or for INT4 / INT2
  // pages in the ring split (the new position is in the ring when the ring keeps >= 1 token)
  if (append && a.plan.kernel != 1 && !(a.plan.kernel == 2 && g.residual_len >= 1)) return KVQ_ERR_UNSUPPORTED;
  if (a.plan.ws_bytes > 0) {
    if (workspace == nullptr || workspace_bytes < a.plan.ws_bytes || !aligned16(workspace))
      return KVQ_ERR_INVALID_ARG;
    a.ws_o = static_cast<float*>(workspace);
    a.ws_ml = reinterpret_cast<float*>(static_cast<char*>(workspace) + a.plan.ws_ml_off);
  }
  a.q = q;
  a.k_new = k_new;
  a.v_new = v_new;
  a.batch = batch;
  a.Hq = num_q_heads;
  a.block_tables = block_tables;
  a.max_blocks = max_blocks_per_seq;
  a.context_lens = context_lens;
  a.seq_ids = seq_ids;
  a.max_context = max_context;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(g.D));
  a.scale_log2 = scale * kLog2e;
  a.out = out;
  a.out_dtype = out_dtype;
  return from_cuda(launch_decode(a, stream));
}

}  // namespace

extern "C" {

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "KVQ_OK";
    case KVQ_ERR_INVALID_ARG: return "KVQ_ERR_INVALID_ARG";
    case KVQ_ERR_UNSUPPORTED: return "KVQ_ERR_UNSUPPORTED";
    case KVQ_ERR_CUDA: return "KVQ_ERR_CUDA";
    case KVQ_ERR_DEVICE_FAULT: return "KVQ_ERR_DEVICE_FAULT";
  }
  return "KVQ_UNKNOWN_STATUS";
}

int kvq_version(void) { return 100; }

kvq_status kvq_cache_layout(const kvq_cache_desc* c, size_t* record_bytes, size_t* pages_bytes,
                            size_t* static_scale_bytes, size_t* residual_bytes) {
  Geometry g;
  const kvq_status st = validate_geometry(c, &g);
  if (st != KVQ_OK) return st;
  size_t ss = 0, rb = 0;
  if (g.scale_mode == KVQ_SCALE_PER_HEAD) ss = static_cast<size_t>(g.H) * 4;
  if (g.scale_mode == KVQ_SCALE_PER_TENSOR) ss = 4;
  if (g.scale_mode == KVQ_SCALE_PER_CHANNEL) ss = static_cast<size_t>(g.H) * g.D * 4;
  if (low_bit(g.cache_dtype))
    rb = static_cast<size_t>(g.max_seqs) * 2 * g.H * g.residual_cap * g.D * 2;
  if (record_bytes) *record_bytes = static_cast<size_t>(g.record);
  if (pages_bytes) *pages_bytes = static_cast<size_t>(g.NB) * g.H * g.record;
  if (static_scale_bytes) *static_scale_bytes = ss;
  if (residual_bytes) *residual_bytes = rb;
  return KVQ_OK;
}

kvq_status kvq_write(const kvq_cache_desc* c, const void* k_new, const void* v_new,
                     int num_tokens, const int32_t* slot_mapping, const int32_t* seq_ids,
                     const int32_t* positions, cudaStream_t stream) {
  Geometry g;
  kvq_status st = validate_desc(c, &g);
  if (st != KVQ_OK) return st;
  if (num_tokens < 0) return KVQ_ERR_INVALID_ARG;
  if (num_tokens == 0) return KVQ_OK;
  if (k_new == nullptr || v_new == nullptr || slot_mapping == nullptr) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new)) return KVQ_ERR_INVALID_ARG;
  if (low_bit(g.cache_dtype))
    return from_cuda(launch_write_int4(*c, g, k_new, v_new, num_tokens, slot_mapping, seq_ids,
                                       positions, stream));
  return from_cuda(launch_write_dense(*c, g, k_new, v_new, num_tokens, slot_mapping, stream));
}

kvq_status kvq_decode_plan(const kvq_cache_desc* c, int batch, int num_q_heads, int max_context,
                           int* kernel_out, int* launches_out, int* splits_out) {
  if (c == nullptr) return KVQ_ERR_INVALID_ARG;
  Geometry g;
  kvq_status st = validate_geometry(c, &g);
  if (st != KVQ_OK) return st;
  if (batch < 0 || num_q_heads < 1 || num_q_heads % g.H != 0 || max_context < 0)
    return KVQ_ERR_INVALID_ARG;
  DecodePlan p;
  st = plan_decode(g, batch, num_q_heads, max_context, &p);
  if (st != KVQ_OK) return st;
  // the launches of launch_decode: kernel 1 + segment merge; INT4/INT2 blocks + ring kernel +
  // split reduce; CUDA-core kernel (+ split reduce when it splits)
  int launches = p.kernel == 1 ? 2 : p.kernel == 2 ? 3 : (p.splits > 1 ? 2 : 1);
  if (batch == 0) launches = 0;                       // nothing to do: nothing launched
  if (kernel_out) *kernel_out = p.kernel;
  if (launches_out) *launches_out = launches;
  if (splits_out) *splits_out = p.kernel == 1 ? p.ctas : p.splits;
  return KVQ_OK;
}

kvq_status kvq_decode_workspace_size(const kvq_cache_desc* c, int batch, int num_q_heads,
                                     int max_context, size_t* bytes) {
  if (c == nullptr || bytes == nullptr) return KVQ_ERR_INVALID_ARG;
  Geometry g;
  kvq_status st = validate_geometry(c, &g);
  if (st != KVQ_OK) return st;
  if (batch < 0 || num_q_heads < 1 || num_q_heads % g.H != 0 || max_context < 0)
    return KVQ_ERR_INVALID_ARG;
  DecodePlan p;
  st = plan_decode(g, batch, num_q_heads, max_context, &p);
  if (st != KVQ_OK) return st;
  *bytes = p.ws_bytes;
  return KVQ_OK;
}


kvq_status kvq_decode_attention(const kvq_cache_desc* c, const void* q, int batch,
                                int num_q_heads, const int32_t* block_tables,
                                int max_blocks_per_seq, const int32_t* context_lens,
                                const int32_t* seq_ids, int max_context, float softmax_scale,
                                void* out, int32_t out_dtype, void* workspace,
                                size_t workspace_bytes, cudaStream_t stream) {
  return decode_entry(c, nullptr, nullptr, q, batch, num_q_heads, block_tables, max_blocks_per_seq,
                      context_lens, seq_ids, max_context, softmax_scale, out, out_dtype, workspace,
                      workspace_bytes, stream);
}

kvq_status kvq_append_decode_attention(const kvq_cache_desc* c, const void* k_new,
                                       const void* v_new, const void* q, int batch,
                                       int num_q_heads, const int32_t* block_tables,
                                       int max_blocks_per_seq, const int32_t* context_lens,
                                       int max_context, float softmax_scale, void* out,
                                       int32_t out_dtype, void* workspace, size_t workspace_bytes,
                                       cudaStream_t stream) {
  if (k_new == nullptr || v_new == nullptr) return KVQ_ERR_INVALID_ARG;
  return decode_entry(c, k_new, v_new, q, batch, num_q_heads, block_tables, max_blocks_per_seq,
                      context_lens, nullptr, max_context, softmax_scale, out, out_dtype, workspace,
                      workspace_bytes, stream);
}

kvq_status kvq_dequant(const kvq_cache_desc* c, const int32_t* block_ids, int n_blocks,
                       float* out, cudaStream_t stream) {
  Geometry g;
  kvq_status st = validate_desc(c, &g);
  if (st != KVQ_OK) return st;
  if (n_blocks < 0) return KVQ_ERR_INVALID_ARG;
  if (n_blocks == 0) return KVQ_OK;
  if (block_ids == nullptr || out == nullptr) return KVQ_ERR_INVALID_ARG;
  return from_cuda(launch_dequant(*c, g, block_ids, n_blocks, out, stream));
}

kvq_status kvq_calibrate_fp8_scales(const void* x, int n_tokens, int num_kv_heads, int head_dim,
                                    int32_t act_dtype, float* scale_out, cudaStream_t stream) {
  if (n_tokens < 0 || num_kv_heads < 1 || head_dim < 1) return KVQ_ERR_INVALID_ARG;
  if (act_dtype != KVQ_DTYPE_BF16 && act_dtype != KVQ_DTYPE_FP16) return KVQ_ERR_INVALID_ARG;
  if (scale_out == nullptr || (n_tokens > 0 && x == nullptr)) return KVQ_ERR_INVALID_ARG;
  return from_cuda(launch_calibrate(x, n_tokens, num_kv_heads, head_dim, act_dtype, 448.f, scale_out,
                                    stream));
}

kvq_status kvq_calibrate_head_scales(const void* x, int n_tokens, int num_kv_heads, int head_dim,
                                     int32_t act_dtype, float qmax, float* scale_out,
                                     cudaStream_t stream) {
  if (n_tokens < 0 || num_kv_heads < 1 || head_dim < 1) return KVQ_ERR_INVALID_ARG;
  if (act_dtype != KVQ_DTYPE_BF16 && act_dtype != KVQ_DTYPE_FP16) return KVQ_ERR_INVALID_ARG;
  if (!(qmax > 0.f) || !std::isfinite(qmax)) return KVQ_ERR_INVALID_ARG;
  if (scale_out == nullptr || (n_tokens > 0 && x == nullptr)) return KVQ_ERR_INVALID_ARG;
  return from_cuda(launch_calibrate(x, n_tokens, num_kv_heads, head_dim, act_dtype, qmax, scale_out,
                                    stream));
}

kvq_status kvq_prefill_attention(const kvq_cache_desc* c, const void* q, int num_q_tokens, int batch,
                                 int num_q_heads, const int32_t* q_start, int max_q_len,
                                 const int32_t* block_tables, int max_blocks_per_seq,
                                 const int32_t* context_lens, int max_context, float softmax_scale,
                                 void* out, int32_t out_dtype, cudaStream_t stream) {
  Geometry g;
  kvq_status st = validate_desc(c, &g);
  if (st != KVQ_OK) return st;
  if (batch < 0 || num_q_tokens < 0 || max_q_len < 0 || num_q_heads < 1 || num_q_heads % g.H != 0 ||
      max_context < 0 || max_blocks_per_seq < 1)
    return KVQ_ERR_INVALID_ARG;
  if (out_dtype != KVQ_DTYPE_BF16 && out_dtype != KVQ_DTYPE_FP16 && out_dtype != KVQ_DTYPE_FP32)
    return KVQ_ERR_INVALID_ARG;
  if (!(softmax_scale >= 0.f) || !std::isfinite(softmax_scale)) return KVQ_ERR_INVALID_ARG;
  DecodeArgs a{};
  a.c = c;
  a.geo = g;
  st = plan_decode(g, std::max(batch, 1), num_q_heads, max_context, &a.plan);
  if (st != KVQ_ERR_UNSUPPORTED && st != KVQ_OK) return st;
  // the tcgen05 kernel (head_dim 128, block 16 dense / 64 low-bit, GQA groups dividing 128),
  // else the warp-per-query mode of the dense tensor-core decode kernel
  a.plan.g = num_q_heads / g.H;
  if (!prefill_tc_supported(g, a.plan.g) && (st != KVQ_OK || a.plan.kernel != 1)) return KVQ_ERR_UNSUPPORTED;
  if (batch == 0 || num_q_tokens == 0 || max_q_len == 0) return KVQ_OK;
  if (q == nullptr || q_start == nullptr || block_tables == nullptr || context_lens == nullptr ||
      out == nullptr)
    return KVQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out)) return KVQ_ERR_INVALID_ARG;
  a.q = q;
  a.q_start = q_start;
  a.max_q_len = max_q_len;
  a.batch = batch;
  a.Hq = num_q_heads;
  a.block_tables = block_tables;
  a.max_blocks = max_blocks_per_seq;
  a.context_lens = context_lens;
  a.max_context = max_context;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(g.D));
  a.scale_log2 = scale * kLog2e;
  a.out = out;
  a.out_dtype = out_dtype;
  return from_cuda(launch_prefill(a, stream));
}

kvq_status kvq_flush_ring(const kvq_cache_desc* c, const int32_t* seq_ids, const int32_t* positions,
                          const int32_t* block_ids, int n, cudaStream_t stream) {
  Geometry g;
  kvq_status st = validate_desc(c, &g);
  if (st != KVQ_OK) return st;
  if (!low_bit(g.cache_dtype)) return KVQ_ERR_UNSUPPORTED;
  if (n < 0) return KVQ_ERR_INVALID_ARG;
  if (n == 0) return KVQ_OK;
  if (seq_ids == nullptr || positions == nullptr || block_ids == nullptr) return KVQ_ERR_INVALID_ARG;
  return from_cuda(launch_flush_ring(*c, g, seq_ids, positions, block_ids, n, stream));
}

kvq_status kvq_calibrate_channel_scales(const void* x, int n_tokens, int num_kv_heads,
                                        int head_dim, int32_t act_dtype, float qmax,
                                        float* scale_out, cudaStream_t stream) {
  if (n_tokens < 0 || num_kv_heads < 1 || head_dim < 1 || head_dim > 1024) return KVQ_ERR_INVALID_ARG;
  if (act_dtype != KVQ_DTYPE_BF16 && act_dtype != KVQ_DTYPE_FP16) return KVQ_ERR_INVALID_ARG;
  if (!(qmax > 0.f) || !std::isfinite(qmax)) return KVQ_ERR_INVALID_ARG;
  if (scale_out == nullptr || (n_tokens > 0 && x == nullptr)) return KVQ_ERR_INVALID_ARG;
  return from_cuda(launch_calibrate_channels(x, n_tokens, num_kv_heads, head_dim, act_dtype, qmax,
                                             scale_out, stream));
}

kvq_status kvq_read_device_fault(const kvq_cache_desc* c, int32_t* out, int reset,
                                 cudaStream_t stream) {
  if (c == nullptr || out == nullptr || c->fault == nullptr) return KVQ_ERR_INVALID_ARG;
  cudaError_t e = cudaMemcpyAsync(out, c->fault, 2 * sizeof(int32_t), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess && reset) e = cudaMemsetAsync(c->fault, 0, 2 * sizeof(int32_t), stream);
  if (e != cudaSuccess) return KVQ_ERR_CUDA;
  return out[0] != 0 ? KVQ_ERR_DEVICE_FAULT : KVQ_OK;
}

}  // extern "C"
