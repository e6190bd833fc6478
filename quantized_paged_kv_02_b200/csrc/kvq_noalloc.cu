// kvq_decode_attention_noalloc: decode attention for callers that cannot allocate.
//
// A plugin inside a host inference engine that owns all device memory, a server that has
// handed nearly all of HBM to the KV-cache pool, or a decode loop that must keep the
// allocator (and the device synchronization cudaMalloc/cudaFree can cause) off its hot
// path cannot pass kvq_decode_attention a workspace.  This entry point runs the same
// decode with the split partials in a fixed device array that lives in this file, so the
// caller supplies only inputs and outputs.  The pages have no counterpart: this is an
// interface convenience, not part of the method.
#include "kvq_internal.cuh"

namespace {

// The scratch itself: one copy per device that loads the library, kept until exit.  Host
// code must not pass `g_decode_scratch` to a kernel (on the host it names a host-side
// stand-in); it passes the device address looked up below.
static __device__ __align__(256) unsigned char g_decode_scratch[KVQ_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch in the current context of the current device.  Looked up
// on every call rather than cached: a cached address would outlive a cudaDeviceReset or
// belong to another context made current on the same device.  Once the module is loaded
// the look-up allocates nothing; under lazy module loading the first look-up on a device
// is what loads it (and reserves the array), and it fails if memory is short.
cudaError_t scratch_of_current_device(void** addr) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess) return e;
  *addr = p;
  return cudaSuccess;
}

}  // namespace

extern "C" kvq_status kvq_decode_attention_noalloc(
    const kvq_cache_desc* cache, const void* q, int batch, int num_q_heads,
    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
    const int32_t* seq_ids, int max_context, float softmax_scale, void* out, int32_t out_dtype,
    cudaStream_t stream) {
  size_t need = 0;
  kvq_status st = kvq_decode_workspace_size(cache, batch, num_q_heads, max_context, &need);
  if (st != KVQ_OK) return st;
  if (need > KVQ_NOALLOC_SCRATCH_BYTES) return KVQ_ERR_INVALID_ARG;   // shape too large
  void* scratch = nullptr;
  // the look-up runs for every non-empty call, whatever this shape needs, so the first
  // call on a device always does the set-up
  if (batch > 0) {
    if (scratch_of_current_device(&scratch) != cudaSuccess) return KVQ_ERR_CUDA;
  }
  return kvq_decode_attention(cache, q, batch, num_q_heads, block_tables, max_blocks_per_seq,
                              context_lens, seq_ids, max_context, softmax_scale, out, out_dtype,
                              scratch, scratch ? KVQ_NOALLOC_SCRATCH_BYTES : 0, stream);
}
