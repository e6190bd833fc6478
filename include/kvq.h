/*
 * kvq.h - C ABI of a quantized paged KV cache with fused-dequant decode attention
 * for NVIDIA B200 (sm_100a).
 *
 * Sources cited below (titles of the web pages that describe the method):
 *   [P-vLLM] "KV Cache量化压缩技术与vLLM推理引擎显存优化实战" (yunthe.com)
 *   [P-prod] "KV Cache Quantization 生产实战：用低精度缓存降低长上下文推理显存" (oh-bug.com)
 *   [P-mem]  "大模型KV Cache显存优化与量化技术实践" (intelliparadigm.com)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument or descriptor field that names tensor data is a DEVICE
 *    pointer, unless the comment says "host".  The caller owns all memory; the library
 *    never allocates or frees device memory and never synchronises a stream, except
 *    kvq_read_device_fault, which copies a few bytes back and waits for them.
 *  - All work is enqueued on the given stream, in order; a NULL stream is the legacy
 *    default stream.
 *  - Device tensor pointers must be 16-byte aligned.  Tensors are dense, row-major,
 *    with the shapes given below (outermost dimension first).
 *  - Arguments are validated on the host before anything is launched: a bad argument
 *    returns KVQ_ERR_INVALID_ARG, a well-formed request this build does not implement
 *    returns KVQ_ERR_UNSUPPORTED, and in both cases nothing is enqueued.  A failed
 *    launch returns KVQ_ERR_CUDA.
 *  - Values the host cannot see (slot ids, block ids, context lengths, sequence ids
 *    inside device arrays) are range-checked by the kernels.  An out-of-range entry is
 *    skipped (its rows are not written / not read) and, when the descriptor carries a
 *    fault record, counted there.  No kernel traps, asserts or spins without a bound.
 *
 * Cache layout ("L0", plain data owned by the caller)
 * ---------------------------------------------------
 *  NB = num_blocks, H = num_kv_heads, bs = block_size, D = head_dim.
 *  A token slot is  slot = block_id * bs + offset,  0 <= offset < bs  ([P-vLLM]
 *  "PagedAttention与KV Cache量化协同工作原理": fixed-size blocks of usually 16 tokens,
 *  each managed on its own, holding INT8/FP8 data that attention dequantizes).
 *
 *  pages : [NB][H][record] bytes.  One record holds everything decode reads for one
 *          (block, kv head), contiguous, so a single copy moves it:
 *            row_bytes   = D * bits / 8            (bits: 16 BF16/FP16, 8 INT8/FP8, 4 INT4,
 *                                                    2 INT2)
 *            K codes     at offset 0              : [bs][row_bytes]
 *            V codes     at offset bs*row_bytes   : [bs][row_bytes]
 *            scales      at offset 2*bs*row_bytes (off_s):
 *              PER_TOKEN_HEAD : float32 K scale [bs], then float32 V scale [bs]
 *                               (one scale per written token and kv head, [P-mem] §3.2
 *                               动态量化策略)
 *              KIVI (INT4)    : float16 K scale [D], float16 K zero point [D] (each channel
 *                               over the block's 64 tokens), then float16 V (scale, zero
 *                               point) [bs][D/64][2] (each token's 64-channel group)
 *                               ([P-prod] "Key 和 Value 的分布不一定相同": keys per channel,
 *                               values per token)
 *              KIVI_FLOAT_ZERO: as KIVI, with each zero point field holding the group's
 *                               float16 minimum m instead of an integer zero point
 *              INT4_PER_TOKEN : float16 K (scale, zero point) [bs][D/64][2], then float16
 *                               V (scale, zero point) [bs][D/64][2] (keys grouped like
 *                               values: [P-prod] "Key 和 Value 的分布不一定相同", the
 *                               Transformers integration quantizes both per token)
 *                               The three INT4 modes have records of the same size; INT2
 *                               caches take the same three modes and parameter layouts.
 *              other modes    : nothing
 *            record      = off_s + scale bytes, rounded up to a multiple of 128 bytes
 *                          (e.g. INT8, bs 16, D 128: 2048 + 2048 + 128 = 4224 bytes)
 *          INT4 codes pack two per byte: element 2i in the low nibble of byte i, element
 *          2i+1 in the high nibble.  INT2 codes pack four per byte: element 4i+e in bits
 *          [2e, 2e+2) of byte i.  Padding bytes at the end of a record are never written.
 *          (INT4, D 128: 4096 + 4096 + 1024 = 9216 bytes; INT2: 2048 + 2048 + 1024 = 5120.)
 *  k_scales, v_scales : static scales only - PER_HEAD: float32 [H] ([P-prod] "vLLM：从 FP8 KV
 *          Cache 开始试点": per-attention-head); PER_TENSOR: float32 [1]; PER_CHANNEL: float32
 *          [H][D], one scale per kv head and channel ([P-vLLM] "KV Cache量化策略：INT8与FP8
 *          精度对比与选择": INT8 per-tensor or per-channel; [P-prod] "量化不是简单截断精度":
 *          scales per tensor, head, channel, token or group).  Unused otherwise.
 *  residual : INT4 and INT2 only.  act_dtype [max_seqs][2][H][residual_cap][D]: the newest tokens of
 *          each sequence kept unquantized ([P-prod] "Key 和 Value 的分布不一定相同": a
 *          fixed-size higher-precision residual of recent K/V).  Index 0 of the second
 *          dimension is K, 1 is V.  Position p of a sequence lives in ring row
 *          p % residual_cap.
 *
 * Quantizers (what kvq_write stores; x is one activation value widened to float32, and
 * every "/" is an IEEE float32 division rounded to nearest-even)
 *  INT8  ([P-mem] §3.1 对称量化算法; [P-vLLM] "KV Cache量化策略"):
 *        dynamic: s = max_d |x_d| / 127  per (token, kv head), stored as float32;
 *        static : s = the caller's per-head, per-tensor or per-(head, channel) scale;
 *        code   = clamp(round_half_even(x / s), -128, 127);  s == 0 gives code 0.
 *        dequantized value = code * s.
 *  FP8 E4M3 (OCP "E4M3FN": bias 7, no infinities, largest finite 448):
 *        dynamic: s = max_d |x_d| / 448;  static: caller's scale.
 *        code = x / s rounded to the nearest E4M3 value (ties to even), magnitudes
 *        beyond 448 saturate to +-448;  s == 0 gives code 0x00.  value = decode(code)*s.
 *  INT4 KIVI ([P-prod] "量化不是简单截断精度": X_q = round(X/scale) + zero_point,
 *        X_deq = (X_q - zero_point) * scale), over a group G of 64 values (one channel
 *        over the 64 tokens of a block for K, one token over 64 channels for V):
 *        lo = min(min_G x, 0), hi = max(max_G x, 0);
 *        s  = float16_rne( (hi - lo) / 15 )      (hi - lo is a float32 subtraction);
 *        z  = clamp(round_half_even(-lo / s), 0, 15)        (float32 ops, s widened);
 *        code = clamp(round_half_even(x / s) + z, 0, 15);   s == 0 gives z = code = 0.
 *        Stored s and z are float16; dequantized value = (code - z) * s.
 *  INT4 KIVI_FLOAT_ZERO (the same groups; the zero point is the group minimum, a float):
 *        lo = min_G x, hi = max_G x;  s = float16_rne( (hi - lo) / 15 );  m = float16_rne(lo);
 *        code = clamp(round_half_even( (x - m) / s ), 0, 15)   (float32 ops, s and m widened);
 *        s == 0 gives code 0.  Stored s and m are float16; dequantized value = code * s + m.
 *  INT4 PER_TOKEN ([P-prod] "Transformers：适合实验和小规模验证": 4 bits, groups of 64,
 *        residual of 128): the KIVI quantizer, every group one token over 64 channels, for
 *        keys as for values.
 *  INT2 ([P-prod] "KV Cache 的基本内存模型": 2-bit, 0.25 byte per value; "误区二：INT4 或
 *        2-bit 一定比 FP8 更划算"): the three INT4 modes with 3 in place of 15 (codes 0..3).
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1,   /* malformed argument; nothing was enqueued */
  KVQ_ERR_UNSUPPORTED = 2,   /* well-formed but not implemented; nothing enqueued */
  KVQ_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
  KVQ_ERR_DEVICE_FAULT = 4   /* kvq_read_device_fault found skipped entries */
} kvq_status;

typedef enum {
  KVQ_DTYPE_BF16 = 0,
  KVQ_DTYPE_FP16 = 1,
  KVQ_DTYPE_FP32 = 2,        /* output only */
  KVQ_DTYPE_INT8 = 3,
  KVQ_DTYPE_FP8_E4M3 = 4,
  KVQ_DTYPE_INT4 = 5,
  KVQ_DTYPE_INT2 = 6
} kvq_dtype;

typedef enum {
  KVQ_SCALE_NONE = 0,
  KVQ_SCALE_PER_TOKEN_HEAD = 1,
  KVQ_SCALE_PER_HEAD = 2,
  KVQ_SCALE_PER_TENSOR = 3,
  KVQ_SCALE_KIVI = 4,
  KVQ_SCALE_PER_CHANNEL = 5,
  KVQ_SCALE_INT4_PER_TOKEN = 6,
  KVQ_SCALE_KIVI_FLOAT_ZERO = 7
} kvq_scale_mode;

/* Bits of fault[1] (fault[0] counts skipped entries). */
enum {
  KVQ_FAULT_SLOT = 1,        /* kvq_write: slot id outside [-1, NB*bs) */
  KVQ_FAULT_BLOCK = 2,       /* block table entry outside [0, NB) */
  KVQ_FAULT_CONTEXT = 4,     /* context length outside [0, max_context] or the table */
  KVQ_FAULT_SEQ = 8,         /* sequence id outside [0, max_seqs) */
  KVQ_FAULT_INT4_RUN = 16,   /* INT4 page rows not one whole, ordered block */
  KVQ_FAULT_TIMEOUT = 32     /* a bounded wait inside a kernel ran out */
};

/*
 * Cache descriptor.  Plain data: it owns nothing and may be copied freely.
 *   cache_dtype   BF16 / FP16 (unquantized, element type must equal act_dtype),
 *                 INT8, FP8_E4M3, INT4 or INT2.
 *   act_dtype     BF16 or FP16: element type of new K/V rows, of q and of the INT4
 *                 residual ring.
 *   scale_mode    NONE for BF16/FP16; PER_TOKEN_HEAD, PER_HEAD, PER_TENSOR or
 *                 PER_CHANNEL for INT8 and FP8; KIVI, KIVI_FLOAT_ZERO or INT4_PER_TOKEN
 *                 for INT4 and INT2.  PER_CHANNEL decodes on
 *                 the tensor-core path only (block_size 16, head_dim 128).
 *   block_size    tokens per block: 1..1024 for dense caches; INT4 / INT2 require
 *                 block_size == group_size == 64.
 *   head_dim      64 or 128.
 *   group_size, residual_len, residual_cap, max_seqs: INT4 / INT2 only (64, r, cap, seqs);
 *                 residual_cap >= residual_len + group_size.  Ignored otherwise.
 *   fault         optional device int32[2] fault record (NULL: faults are skipped
 *                 silently).  fault[0] += entries skipped; fault[1] |= KVQ_FAULT_* bits.
 */
typedef struct {
  int32_t cache_dtype;
  int32_t act_dtype;
  int32_t scale_mode;
  int32_t num_blocks;
  int32_t block_size;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t group_size;
  int32_t residual_len;
  int32_t residual_cap;
  int32_t max_seqs;
  int32_t reserved0;
  void* pages;         /* [NB][H][record] */
  float* k_scales;     /* static scales (PER_HEAD / PER_TENSOR / PER_CHANNEL) */
  float* v_scales;
  void* residual;      /* INT4 ring */
  int32_t* fault;
} kvq_cache_desc;

/* Human-readable name of a status code (static storage, never NULL). */
const char* kvq_status_string(kvq_status status);

/* Library version as an integer (major*10000 + minor*100 + patch). */
int kvq_version(void);

/*
 * Sizes for a cache described by `cache` (pointer fields are ignored): bytes of one
 * record, of the whole `pages` pool (NB*H records), of each static scale array, and of
 * the residual ring.  Any out pointer may be NULL.  Host-only; never touches the device.
 * The sizes follow the layout above ([P-prod] "KV Cache 的基本内存模型": 2 x layers x
 * kv_heads x head_dim x tokens x bytes per value, per layer here, plus the scale,
 * zero-point and residual bytes that make the real gain smaller).
 */
kvq_status kvq_cache_layout(const kvq_cache_desc* cache, size_t* record_bytes,
                            size_t* pages_bytes, size_t* static_scale_bytes,
                            size_t* residual_bytes);

/*
 * kvq_write - quantize new K/V rows into the cache ("quantize on write").
 *   k_new, v_new  act_dtype [num_tokens][H][D], device.
 *   slot_mapping  int32 [num_tokens], device: destination slot of each row, or -1.
 *   seq_ids, positions  int32 [num_tokens], device, INT4 / INT2 only (NULL otherwise): a row
 *                 with slot -1 and positions[t] >= 0 is copied unquantized into ring row
 *                 positions[t] % residual_cap of sequence seq_ids[t].
 *   Dense caches: row t goes to slot slot_mapping[t]; slot -1 skips the row.  K and V
 *   are quantized separately, each per (token, kv head) for dynamic modes.
 *   INT4 / INT2 caches: rows are taken in groups of 64 (rows 64u .. 64u+63).  A group whose
 *   first slot is >= 0 must map, in order, onto one whole block (slots b*64 .. b*64+63);
 *   it is quantized as one key group per channel and 64 value groups per channel group.
 *   A group whose first slot is -1 holds ring rows or skipped rows only.  A trailing
 *   partial group may hold ring rows only.
 *   Duplicate destination slots inside one call give an undefined winner.
 *   Quantizer definitions: see the header comment ([P-mem] §3.1 / §3.2, [P-vLLM]
 *   "KV Cache量化策略", [P-prod] "量化不是简单截断精度").
 */
kvq_status kvq_write(const kvq_cache_desc* cache, const void* k_new, const void* v_new,
                     int num_tokens, const int32_t* slot_mapping, const int32_t* seq_ids,
                     const int32_t* positions, cudaStream_t stream);

/*
 * kvq_flush_ring - INT4 / INT2: move whole groups of the residual ring into pages.
 *   For each entry i < n: ring rows of sequence seq_ids[i] at positions
 *   [positions[i], positions[i] + 64) (ring row p % residual_cap) are quantized into block
 *   block_ids[i] of every kv head, with exactly the codes, scales and zero points kvq_write
 *   stores when given those rows with slots block_ids[i]*64 + 0..63.  The ring rows are left
 *   in place.
 *   seq_ids, positions, block_ids  int32 [n], device.  positions[i] must be a multiple of 64
 *   and the 64 positions must still be in the ring (at most residual_cap positions behind
 *   the newest one written); an entry with a sequence id, block id or position out of range
 *   is skipped and counted (KVQ_FAULT_SEQ / _BLOCK / _INT4_RUN).
 *   The residual window of [P-prod] "Key 和 Value 的分布不一定相同" keeps the newest tokens
 *   unquantized; once more than residual_len + 64 are there, the oldest 64 become one key
 *   group (one block) and are quantized, which this call does from the ring itself, so the
 *   caller need not keep its own copy of those rows.
 *   INT4 and INT2 caches only (others: KVQ_ERR_UNSUPPORTED).
 */
kvq_status kvq_flush_ring(const kvq_cache_desc* cache, const int32_t* seq_ids,
                          const int32_t* positions, const int32_t* block_ids, int n,
                          cudaStream_t stream);

/*
 * Workspace bytes kvq_decode_attention needs for this shape (host-only: it reads the
 * current device's SM count, and launches nothing).  The split plan depends only on (cache
 * geometry, batch, num_q_heads, max_context) and that SM count (148 on B200, and 148 when
 * no device can be queried), so the same arguments on the same device always give the same
 * size.  *bytes may be 0 (no split needed).
 */
kvq_status kvq_decode_workspace_size(const kvq_cache_desc* cache, int batch,
                                     int num_q_heads, int max_context, size_t* bytes);

/*
 * kvq_decode_plan - which kernels kvq_decode_attention launches for these arguments (host
 * only: no device access, no launch; the pages give no counterpart, it reports this
 * library's dispatch).  Any output pointer may be NULL.
 *   kernel_out    0: the CUDA-core split kernel; 1: the page-balanced tensor-core kernel
 *                 (dense caches); 2: the low-bit (INT4 / INT2) tensor-core block kernel
 *                 plus the CUDA-core kernel for the residual ring.
 *   launches_out  kernels one call launches, the merge included (1: 2; 2: 3; 0: 1, or 2
 *                 with more than one split; 0 when batch is 0).
 *   splits_out    token splits of kernels 0 and 2 (the ring counted as one); for kernel 1,
 *                 its CTA count (the page ranges).
 *   Errors as kvq_decode_workspace_size.
 */
kvq_status kvq_decode_plan(const kvq_cache_desc* cache, int batch, int num_q_heads,
                           int max_context, int* kernel_out, int* launches_out,
                           int* splits_out);

/*
 * kvq_decode_attention - one query token per sequence attends to its cached context.
 *   q             act_dtype [batch][num_q_heads][D], device.  num_q_heads must be a
 *                 multiple of H; query head hq reads kv head hq / (num_q_heads / H).
 *   block_tables  int32 [batch][max_blocks_per_seq], device: block ids of each sequence
 *                 in token order; entries past ceil(len/bs) are not read.
 *   context_lens  int32 [batch], device: tokens to attend to (the current token
 *                 included); 0 gives an all-zero output row.
 *   seq_ids       INT4 / INT2 only, int32 [batch] device or NULL: ring sequence of each batch
 *                 entry (NULL: entry b uses ring sequence b).
 *   max_context   host upper bound of context_lens, used to plan the split.
 *   softmax_scale 0 selects 1/sqrt(D) ([P-mem] §6 Q1 writes softmax(q k^T / sqrt(d))).
 *   out           out_dtype [batch][num_q_heads][D], device; out_dtype BF16, FP16 or FP32.
 *   workspace     device scratch of at least kvq_decode_workspace_size() bytes (may be
 *                 NULL when that size is 0).  Its contents need no initialisation; two
 *                 calls that overlap on the GPU must not share a workspace.
 *   For each (b, hq): o = sum_p softmax_p(scale * q . k_p) v_p over p < context_lens[b],
 *   where k_p, v_p are the dequantized cache rows; for INT4 / INT2, positions p < Qb come
 *   from blocks and the rest from the residual ring, Qb = 64*floor(max(len-residual_len,0)/64).
 *   Dequantization happens inside the kernel ([P-vLLM] "PagedAttention与KV Cache量化协同
 *   工作原理"); long contexts are split across CTAs and merged by a log-sum-exp reduce.
 *   Kernels: head_dim 128 with block_size 16 and 1..8 query heads per kv head runs on the
 *   tensor-core kernel (dense caches); INT4 / INT2 with head_dim 128 and 3..8 query heads per
 *   kv head on the low-bit tensor-core kernel; everything else on the CUDA-core kernel.
 *   PER_CHANNEL caches need the tensor-core kernel (KVQ_ERR_UNSUPPORTED otherwise).
 */
kvq_status kvq_decode_attention(const kvq_cache_desc* cache, const void* q, int batch,
                                int num_q_heads, const int32_t* block_tables,
                                int max_blocks_per_seq, const int32_t* context_lens,
                                const int32_t* seq_ids, int max_context, float softmax_scale,
                                void* out, int32_t out_dtype, void* workspace,
                                size_t workspace_bytes, cudaStream_t stream);

/*
 * kvq_append_decode_attention - one serving step in one call: store this step's K/V row
 * of every sequence, then attend (kvq_write followed by kvq_decode_attention).
 *   k_new, v_new  act_dtype [batch][H][D], device: the new token's key and value rows of
 *                 each sequence.  Row b is stored at position context_lens[b] - 1 of
 *                 sequence b, i.e. slot block_tables[b][(len-1)/bs]*bs + (len-1)%bs, with
 *                 exactly the codes and scales kvq_write would store there; a sequence with
 *                 context_lens[b] == 0 stores nothing.  Then decode attends to positions
 *                 p < context_lens[b], the new one included.
 *   Other arguments as kvq_decode_attention (the workspace size is the same; there is no
 *   seq_ids argument).
 *   Dense caches (INT8, FP8 E4M3, BF16, FP16) with block_size 16 and head_dim 128; and
 *   INT4 / INT2 caches on the tensor-core path (head_dim 128, 3..8 query heads per kv head)
 *   whose ring keeps at least one token (residual_len >= 1): there the new row of sequence b
 *   goes to the residual ring of ring sequence b at position context_lens[b] - 1, as
 *   kvq_write stores a row that completes no block (a 64-token group that has left the ring
 *   window still needs kvq_flush_ring before the step).  Other caches return
 *   KVQ_ERR_UNSUPPORTED (use kvq_write + kvq_decode_attention).
 *   The pages quantize on write and dequantize inside attention ([P-vLLM]
 *   "PagedAttention与KV Cache量化协同工作原理"); doing both in one launch saves a kernel and
 *   its launch per step.  Results equal kvq_write followed by kvq_decode_attention, bit
 *   for bit.
 */
kvq_status kvq_append_decode_attention(const kvq_cache_desc* cache, const void* k_new,
                                       const void* v_new, const void* q, int batch,
                                       int num_q_heads, const int32_t* block_tables,
                                       int max_blocks_per_seq, const int32_t* context_lens,
                                       int max_context, float softmax_scale, void* out,
                                       int32_t out_dtype, void* workspace, size_t workspace_bytes,
                                       cudaStream_t stream);

/*
 * kvq_prefill_attention - causal attention of a chunk of new queries per sequence over the
 *   cache (chunked prefill).  The chunk's own K/V rows must already be in the cache
 *   (kvq_write); the queries are the newest tokens of each sequence.
 *   q             act_dtype [num_q_tokens][num_q_heads][D], device: the queries of sequence b
 *                 are rows q_start[b] .. q_start[b+1]-1, in token order.
 *   q_start       int32 [batch+1], device, non-decreasing, q_start[batch] <= num_q_tokens.
 *   max_q_len     host upper bound of q_start[b+1] - q_start[b] (sizes the grid); a sequence
 *                 with more queries, or with more queries than context_lens[b], is skipped
 *                 and counted (KVQ_FAULT_CONTEXT).
 *   context_lens  int32 [batch], device: tokens in the cache for sequence b, the chunk's own
 *                 included.
 *   out           out_dtype [num_q_tokens][num_q_heads][D], device.
 *   Other arguments as kvq_decode_attention.  Query i of sequence b sits at position
 *   p = context_lens[b] - L_b + i (L_b its query count) and attends to positions <= p:
 *   o = softmax(scale * q . k_t) v_t over t <= p, dequantized inside the kernel.  Chunked
 *   prefill is one of the techniques [P-prod] "为什么长上下文更需要 KV Cache Quantization"
 *   names beside KV cache quantization.  No workspace.
 *   Supported: head_dim 128 with dense caches of block_size 16, and INT4 / INT2 caches
 *   (block_size 64).  For INT4 / INT2 the cache is read as it stands after the chunk was
 *   written: positions below Qb = 64*floor(max(context_lens[b] - residual_len, 0)/64) from
 *   blocks, the rest from ring sequence b.  GQA groups of 1, 2, 4, 8 (any divisor of 128)
 *   query heads per kv head run on the 5th-generation tensor cores (tiles of 128 query rows,
 *   each page dequantized once per tile); other groups of up to 8 on the dense tensor-core
 *   decode kernel's per-query mode (dense caches only).  Anything else returns
 *   KVQ_ERR_UNSUPPORTED.
 */
kvq_status kvq_prefill_attention(const kvq_cache_desc* cache, const void* q, int num_q_tokens,
                                 int batch, int num_q_heads, const int32_t* q_start,
                                 int max_q_len, const int32_t* block_tables,
                                 int max_blocks_per_seq, const int32_t* context_lens,
                                 int max_context, float softmax_scale, void* out,
                                 int32_t out_dtype, cudaStream_t stream);

/*
 * Size of the device scratch array used by kvq_decode_attention_noalloc (16 MiB).  Every
 * GPU that loads the library's device code reserves this much for the life of the process
 * (under CUDA's lazy module loading, at the first kvq_decode_attention_noalloc call on
 * that device rather than when the library is opened).
 */
#define KVQ_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/*
 * kvq_decode_attention_noalloc - kvq_decode_attention without a caller workspace.
 *   (No counterpart in the pages: this entry point exists for callers, not for the method.)
 *   Some callers cannot hand the library a workspace: a plugin running inside a host
 *   inference engine that plans all device memory itself and passes the plugin only its
 *   input and output buffers; a server that gives nearly all of HBM to the KV-cache pool up
 *   front, so a per-call allocation could fail mid-request; a decode loop that must not call
 *   the allocator on its hot path because cudaMalloc/cudaFree can synchronize the device.
 *   This variant takes the same arguments as kvq_decode_attention minus the workspace and
 *   uses a fixed, file-scope device array of KVQ_NOALLOC_SCRATCH_BYTES instead.  It calls no
 *   cudaMalloc, cudaFree or other allocating routine.
 *   - The scratch of the CURRENT device and context is used: make the device that owns
 *     `stream` current.  Every call with batch > 0 looks up the array's device address in
 *     the current context (nothing is cached, so a cudaDeviceReset or a switch of context
 *     between calls is safe).  Under lazy module loading the first look-up on a device loads
 *     the library's device code and reserves the array there; make that first call before
 *     any stream capture and while memory is still free.
 *   - Returns KVQ_ERR_INVALID_ARG, with nothing enqueued, when this shape needs more scratch
 *     than KVQ_NOALLOC_SCRATCH_BYTES (kvq_decode_workspace_size tells the need).  Returns
 *     KVQ_ERR_CUDA if the address look-up fails (for example when the first look-up cannot
 *     reserve the array because device memory is short).
 *   - All calls on a device share the one array, and it keeps whatever the last call left
 *     there (nothing in it needs to start at zero).  Calls that overlap on the GPU (for
 *     example on two streams without ordering between them) race on the array and give
 *     wrong results: serialize them.
 */
kvq_status kvq_decode_attention_noalloc(const kvq_cache_desc* cache, const void* q, int batch,
                                        int num_q_heads, const int32_t* block_tables,
                                        int max_blocks_per_seq, const int32_t* context_lens,
                                        const int32_t* seq_ids, int max_context,
                                        float softmax_scale, void* out, int32_t out_dtype,
                                        cudaStream_t stream);

/*
 * kvq_dequant - debug: expand whole blocks back to float32.
 *   block_ids  int32 [n_blocks], device.
 *   out        float32 [n_blocks][2][H][bs][D], device; index 0 of dim 1 is K, 1 is V.
 *   Each value is the dequantized value defined in the header comment.  An out-of-range
 *   block id leaves its output rows untouched (and is counted in the fault record).
 */
kvq_status kvq_dequant(const kvq_cache_desc* cache, const int32_t* block_ids, int n_blocks,
                       float* out, cudaStream_t stream);

/*
 * kvq_calibrate_fp8_scales - set-up step: per-kv-head scale from warm-up rows,
 *   scale_out[h] = (max over tokens and channels of |x[t][h][:]|) / 448, float32 division.
 *   x          act_dtype [n_tokens][num_kv_heads][head_dim], device.
 *   scale_out  float32 [num_kv_heads], device.  An all-zero head gives 0.
 *   ([P-prod] "vLLM：从 FP8 KV Cache 开始试点": scales from a random-token warm-up.)
 */
kvq_status kvq_calibrate_fp8_scales(const void* x, int n_tokens, int num_kv_heads,
                                    int head_dim, int32_t act_dtype, float* scale_out,
                                    cudaStream_t stream);

/*
 * kvq_calibrate_head_scales - set-up step: per-kv-head scale from warm-up rows,
 *   scale_out[h] = (max over tokens and channels of |x[t][h][:]|) / qmax, float32 division
 *   (kvq_calibrate_fp8_scales is this call with qmax = 448).
 *   x          act_dtype [n_tokens][num_kv_heads][head_dim], device.
 *   qmax       largest code magnitude: 127 for INT8, 448 for FP8 E4M3; finite and > 0.
 *   scale_out  float32 [num_kv_heads], device.  An all-zero head gives 0.
 *   The static scales of KVQ_SCALE_PER_HEAD ([P-mem] §3.2 动态量化策略: static quantization
 *   keeps fixed scales; [P-prod] "量化不是简单截断精度": a scale per tensor or per head).  A
 *   per-tensor scale is the largest of the per-head ones.
 */
kvq_status kvq_calibrate_head_scales(const void* x, int n_tokens, int num_kv_heads,
                                     int head_dim, int32_t act_dtype, float qmax,
                                     float* scale_out, cudaStream_t stream);

/*
 * kvq_calibrate_channel_scales - set-up step: per-(kv head, channel) scale from warm-up rows,
 *   scale_out[h][d] = (max over tokens of |x[t][h][d]|) / qmax, float32 division.
 *   x          act_dtype [n_tokens][num_kv_heads][head_dim], device.
 *   qmax       largest code magnitude: 127 for INT8, 448 for FP8 E4M3; finite and > 0.
 *   scale_out  float32 [num_kv_heads][head_dim], device.  An all-zero channel gives 0.
 *   The static scales of KVQ_SCALE_PER_CHANNEL ([P-vLLM] "vLLM引擎KV Cache量化配置与启动参数
 *   详解": INT8 scale factors generated offline from calibration data; [P-mem] §3.2
 *   动态量化策略: static quantization uses fixed scales).
 */
kvq_status kvq_calibrate_channel_scales(const void* x, int n_tokens, int num_kv_heads,
                                        int head_dim, int32_t act_dtype, float qmax,
                                        float* scale_out, cudaStream_t stream);

/*
 * kvq_read_device_fault - copy the descriptor's fault record into host `out[2]`
 *   (count, KVQ_FAULT_* bits), waiting for `stream` first.  If `reset` is non-zero the
 *   record is cleared afterwards (enqueued on `stream`).  Returns KVQ_ERR_DEVICE_FAULT
 *   when the count is non-zero, KVQ_OK otherwise, KVQ_ERR_INVALID_ARG if the
 *   descriptor has no fault record.
 */
kvq_status kvq_read_device_fault(const kvq_cache_desc* cache, int32_t* out, int reset,
                                 cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
