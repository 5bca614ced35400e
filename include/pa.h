/*
 * pa.h -- C ABI of libpa.so: paged KV-cache decode kernels for NVIDIA B200 (sm_100a).
 *
 * The method: a sequence's keys and values live in fixed-size physical blocks
 * (16 tokens) scattered through a global pool and located through a per-sequence
 * block table ("vLLM推理引擎PagedAttention原理与性能优化实战" sec 2.2; "vLLM 是什么：
 * PagedAttention 让大模型推理快 2-4 倍…" sec 2).  Attention over such a cache is the
 * standard softmax(q K^T / sqrt d) V with K and V gathered from the physical blocks
 * ("vLLM 推理优化技术深度调研报告" sec 3 formula 4, and dim. 1 sec 1 misconception 2).
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers unless stated otherwise.  The caller owns every
 *     buffer; the library allocates nothing and keeps no per-call state, so calls
 *     from several host threads are safe.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call only
 *     validates its host-visible arguments and enqueues work: it returns before
 *     the device has run it.  A return of PA_OK means "enqueued".
 *   - Work on a stream runs in stream order.  The decode kernels are launched as
 *     programmatic dependents (CUDA programmatic dependent launch).  Their CTAs
 *     may be scheduled while the kernel before them on the stream is still
 *     running, but they touch no memory until that kernel has completed and its
 *     writes are visible.  The order a caller observes is that of ordinary
 *     launches.
 *   - Tensors are dense, row-major (C order) with the shapes given below.
 *   - Data pointers must be 16-byte aligned (PA_ERR_INVALID_ARG otherwise).
 *   - Device data that the host cannot see (slots, block ids, sequence lengths) is
 *     range-checked on the device.  A bad value never faults: the access is
 *     clamped or skipped, the result of that item is unspecified, and a bit is set
 *     in a device error word that pa_get_device_error() reads and clears.
 *   - Two kernels (the E4M3 shared-prefix decode and the chunked prefill over two
 *     or more 128-row tiles per sequence and kv head) move registers between warp
 *     groups and check once that their build has the register count this assumes;
 *     otherwise the call takes a slower kernel of the same result (mma.sync, and
 *     one tile per CTA).  PA_FALLBACK_KERNELS=1 in the environment, read at each
 *     call, selects those kernels regardless.
 *
 * Cache layout (one layer): key_cache and value_cache are each
 *   [num_blocks][num_kv_heads][block_size][head_dim]
 * so token `o` of physical block `b` for kv head `h` is the row
 *   ((b * num_kv_heads + h) * block_size + o) * head_dim.
 * Logical token l of sequence s is in physical block block_tables[s][l / block_size]
 * at offset l % block_size ("vLLM 推理优化技术深度调研报告" sec 3 formula 3).
 * Query head h reads kv head h / (num_heads / num_kv_heads).
 *
 * FP8: PA_FP8_E4M3 is OCP E4M3 (bias 7, no infinities, max finite 448) with one
 * fp32 scale per cache tensor: stored code = round-nearest-even-saturating(
 * float(x) / scale) with IEEE fp32 division; read value = float(code) * scale
 * ("vLLM推理引擎PagedAttention原理与性能优化实战" sec 5.2, FP8 KV cache).
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_F16 = 0,      /* IEEE binary16 */
  PA_BF16 = 1,     /* bfloat16 */
  PA_F32 = 2,      /* IEEE binary32 (outputs only) */
  PA_FP8_E4M3 = 3  /* OCP E4M3 (caches only) */
} pa_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = -1,  /* null pointer, bad size, misalignment, inconsistent shapes */
  PA_ERR_UNSUPPORTED = -2,  /* valid but not implemented: dtype pair, head_dim, block_size */
  PA_ERR_WORKSPACE = -3,    /* workspace missing or smaller than the size function says */
  PA_ERR_CUDA = -4          /* a CUDA runtime call failed (e.g. launch error) */
} pa_status;

/* Bits of the device error word (see pa_get_device_error). */
#define PA_DEVERR_SLOT_RANGE 0x1u    /* reshape_and_cache: slot >= num_blocks * block_size */
#define PA_DEVERR_BLOCK_RANGE 0x2u   /* decode: block table entry outside [0, num_blocks) */
#define PA_DEVERR_SEQ_LEN 0x4u       /* decode: seq_len < 0, > max_seq_len or > table capacity */
#define PA_DEVERR_PIPE_TIMEOUT 0x8u  /* decode: a pipeline wait gave up after ~1 s */
#define PA_DEVERR_COPY_RANGE 0x10u   /* copy_blocks: block id outside [0, num_blocks) */
#define PA_DEVERR_PREFIX 0x20u       /* shared-prefix decode: prefix_len or tables break the promise */

/*
 * pa_reshape_and_cache -- write the new tokens' keys and values into their cache
 * slots.  The pages' memory flow "KV block request -> page-table registration ->
 * attention read -> release/reuse" ("vLLM 推理优化技术深度调研报告" sec 2): after
 * the block manager has registered a slot for each new token, this kernel stores
 * the token's K and V rows there.
 *
 *   key, value        [num_tokens][num_kv_heads][head_dim] of src_dtype (F16 or BF16)
 *   key_cache,
 *   value_cache       [num_blocks][num_kv_heads][block_size][head_dim] of cache_dtype
 *   slot_mapping      [num_tokens] int64; slot s -> block s / block_size, offset
 *                     s % block_size; s < 0 skips the token (padding)
 *   cache_dtype       == src_dtype (a bit copy) or PA_FP8_E4M3 (quantise with
 *                     k_scale / v_scale, which must then be finite and > 0)
 * Two tokens naming the same slot give an unspecified winner.  A slot at or past
 * num_blocks * block_size is skipped and sets PA_DEVERR_SLOT_RANGE.
 * Supported: block_size 16, 32, 64 or 128; head_dim a multiple of 8 up to 256.
 * num_tokens == 0 is a no-op returning PA_OK.
 */
int pa_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                         const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int64_t num_blocks, pa_dtype src_dtype,
                         pa_dtype cache_dtype, float k_scale, float v_scale, void* stream);

/*
 * pa_paged_attention_workspace_size -- bytes of device workspace that
 * pa_paged_attention_decode needs for these sizes (0 when every sequence fits in
 * one partition, i.e. max_seq_len <= the partition size).
 * partition_size: 0 = the library's default, else a positive multiple of 16
 * tokens.  The default keeps a sequence whole when the batch has at least
 * 2048 (sequence, head group) units, a head group being the largest of 8, 4, 2, 1
 * query heads dividing num_heads / num_kv_heads; otherwise it splits sequences
 * into enough partitions of at least 256 tokens to reach 2048 units.
 * Returns 0 also for invalid arguments.
 *
 * Workspace layout (fp32, each section 256-byte aligned), P = ceil(max_seq_len /
 * partition):  m[num_seqs][num_heads][P], l[num_seqs][num_heads][P],
 * o[num_seqs][num_heads][P][head_dim], holding for each token range the maximum
 * score m (natural-log units), the sum l of exp(score - m) and the normalised
 * partial output o.
 */
size_t pa_paged_attention_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                         int head_dim, int max_seq_len, int partition_size);

/*
 * pa_paged_attention_partition_size -- the partition length in tokens that
 * pa_paged_attention_decode uses for these sizes and this request (0 = default,
 * as described above).  Host only.  Returns 0 for invalid arguments.
 */
int pa_paged_attention_partition_size(int num_seqs, int num_heads, int num_kv_heads,
                                      int max_seq_len, int partition_size);

/*
 * pa_paged_attention_decode -- one query token per sequence attends over its
 * paged context: out[s][h] = softmax(scale * q[s][h] . K_s^T) V_s, with K_s, V_s
 * the first seq_lens[s] tokens gathered through block_tables[s] ("vLLM 推理优化
 * 技术深度调研报告" sec 3 formulas 3 and 4).  Softmax statistics and accumulation
 * are fp32.  Contexts longer than the partition size are split into partitions
 * whose results are merged by a log-sum-exp reduction (second kernel, same stream).
 *
 *   out           [num_seqs][num_heads][head_dim] of out_dtype (F16, BF16 or F32)
 *   query         [num_seqs][num_heads][head_dim] of q_dtype
 *   key_cache,
 *   value_cache   [num_blocks][num_kv_heads][block_size][head_dim] of cache_dtype
 *   block_tables  [num_seqs][max_blocks_per_seq] int32 physical block ids; entries
 *                 past ceil(seq_len / block_size) are never read
 *   seq_lens      [num_seqs] int32 context lengths (counting the new token);
 *                 0 gives a zero output; must be <= max_seq_len
 *   max_seq_len   host-side upper bound of seq_lens (sizes the launch)
 *   scale         the softmax scale (normally 1/sqrt(head_dim))
 *   k_scale,
 *   v_scale       FP8 dequantisation scales; ignored for F16/BF16 caches
 *   partition_size  0 = default (see the size function), else a positive
 *                 multiple of 16 tokens
 *   workspace     device buffer of at least pa_paged_attention_workspace_size()
 *                 bytes (may be NULL when that size is 0); contents on entry are
 *                 ignored, on exit unspecified
 * Supported: block_size 16, 32, 64 or 128 (the kernels stream 16-token tiles, so a
 * block is read as block_size / 16 contiguous tiles); head_dim 64 or 128;
 * num_heads % num_kv_heads == 0;
 * (q_dtype, cache_dtype) in {(F16,F16), (BF16,BF16), (F16,FP8), (BF16,FP8)}.
 */
int pa_paged_attention_decode(void* out, const void* query, const void* key_cache,
                              const void* value_cache, const int32_t* block_tables,
                              int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                              int max_seq_len, int num_heads, int num_kv_heads, int head_dim,
                              int block_size, int64_t num_blocks, float scale, pa_dtype q_dtype,
                              pa_dtype cache_dtype, pa_dtype out_dtype, float k_scale,
                              float v_scale, int partition_size, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * pa_paged_attention_decode_shared_prefix -- decode attention for groups of
 * sequences whose block tables share their first blocks: the beams of one prompt,
 * or parallel samples, after copy-on-write forking ("vLLM推理引擎PagedAttention原理
 * 与性能优化实战" sec 3.2: sharers' block tables point at the same physical blocks;
 * "vLLM 是什么…" sec 2: branches share the prompt's blocks).  The result is the
 * same as pa_paged_attention_decode on the same arguments; each shared block is
 * read from HBM, staged and widened once per group instead of once per sequence.
 *
 *   group_starts  [num_groups + 1] int32 (device): group g is the consecutive
 *                 sequences group_starts[g] .. group_starts[g+1] - 1
 *   prefix_lens   [num_groups] int32 (device): the group's shared prefix in tokens,
 *                 a multiple of block_size, at most its shortest seq_len; every
 *                 sequence of the group has the same block-table entries there
 *   max_group_size  host-side bound on the group sizes (sizes the launch)
 *   other arguments as for pa_paged_attention_decode (no partitions, no workspace)
 * A broken promise (prefix not block-aligned or too long, tables differing in the
 * prefix, a group larger than max_group_size) sets PA_DEVERR_PREFIX; the affected
 * outputs are then unspecified, and nothing faults.
 * Supported: block_size 16, 32, 64 or 128; head_dim 128; num_heads / num_kv_heads
 * <= 16; the same dtype pairs as pa_paged_attention_decode.
 */
int pa_paged_attention_decode_shared_prefix(
    void* out, const void* query, const void* key_cache, const void* value_cache,
    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
    int max_seq_len, const int32_t* group_starts, const int32_t* prefix_lens, int num_groups,
    int max_group_size, int num_heads, int num_kv_heads, int head_dim, int block_size,
    int64_t num_blocks, float scale, pa_dtype q_dtype, pa_dtype cache_dtype, pa_dtype out_dtype,
    float k_scale, float v_scale, void* stream);

/*
 * pa_paged_attention_prefill -- several query tokens per sequence attending
 * causally over the paged cache: a chunk of a long prompt processed between
 * decode steps ("vLLM推理引擎PagedAttention原理与性能优化实战" sec 6, chunked
 * prefill), or draft tokens checked in one pass.  The chunk's K/V are written by
 * pa_reshape_and_cache first; seq_lens count them.
 *
 *   out, query    [total_queries][num_heads][head_dim]; sequence i's rows are
 *                 query_start[i] .. query_start[i+1] - 1 (q_i rows)
 *   query_start   [num_seqs + 1] int32 (device), non-decreasing, query_start[0] = 0
 *   seq_lens      [num_seqs] int32: context lengths L_i including the chunk; row j of
 *                 sequence i sits at position L_i - q_i + j and attends to positions
 *                 0 .. L_i - q_i + j; q_i <= L_i (else PA_DEVERR_SEQ_LEN)
 *   max_query_len host-side bound on q_i (sizes the launch)
 *   other arguments as for pa_paged_attention_decode
 * Supported: head_dim 128; (q_dtype, cache_dtype) (F16, F16) or (BF16, BF16); out
 * F16, BF16 or F32; block_size 16, 32, 64 or 128.
 * Numerics: scores, softmax and accumulation in fp32; P enters the P.V product in
 * 16 bits (as two bf16 terms, hi and P - hi, when the cache is BF16 and out is F32).
 * Device data errors set bits in the device error word (pa_get_device_error):
 * PA_DEVERR_SEQ_LEN (length or chunk out of range; clamped), PA_DEVERR_BLOCK_RANGE
 * (block id outside the pool; block 0 read instead), PA_DEVERR_PIPE_TIMEOUT (an
 * internal wait gave up; the output is undefined).  Never a fault.
 */
int pa_paged_attention_prefill(void* out, const void* query, const void* key_cache,
                               const void* value_cache, const int32_t* block_tables,
                               int max_blocks_per_seq, const int32_t* seq_lens,
                               const int32_t* query_start, int num_seqs, int max_query_len,
                               int max_seq_len, int num_heads, int num_kv_heads, int head_dim,
                               int block_size, int64_t num_blocks, float scale,
                               pa_dtype q_dtype, pa_dtype cache_dtype, pa_dtype out_dtype,
                               void* stream);

/*
 * pa_copy_blocks -- the copy step of copy-on-write ("vLLM推理引擎PagedAttention原理
 * 与性能优化实战" sec 3.2): when a block shared by several sequences (e.g. beams
 * with a common prefix) must be written by one of them, the block manager gives
 * that sequence a fresh block and this call copies the old block's contents into it.
 *
 *   key_caches,
 *   value_caches   HOST arrays of num_layers DEVICE pointers, one cache per layer,
 *                  each [num_blocks][block_bytes] bytes
 *   block_mapping  [num_pairs][2] int64 (src, dst) physical block ids (device)
 *   block_bytes    bytes of one block of one layer (block_size * kv_heads *
 *                  head_dim * element size); a multiple of 16
 * Pairs run concurrently: a dst must not repeat or also appear as a src.  An id
 * outside [0, num_blocks) skips that pair and sets PA_DEVERR_COPY_RANGE.
 * num_pairs == 0 or num_layers == 0 is a no-op returning PA_OK.
 */
int pa_copy_blocks(void* const* key_caches, void* const* value_caches, int num_layers,
                   const int64_t* block_mapping, int num_pairs, size_t block_bytes,
                   int64_t num_blocks, void* stream);

/* Size of the library's own decode scratch (see below): 16 MiB per GPU. */
#define PA_STATIC_WORKSPACE_BYTES (16u * 1024u * 1024u)

/*
 * pa_paged_attention_decode_static_workspace -- pa_paged_attention_decode for
 * callers that cannot allocate device memory.  It computes the same decode
 * ("vLLM 推理优化技术深度调研报告" sec 3 formulas 3 and 4); the pages have no
 * counterpart to the fixed scratch, which exists for the library's users.
 *
 * Who needs it: a plugin inside a host process that owns every device allocation
 * and gives its plugins no allocator; a serving engine that has already reserved
 * nearly all HBM for its KV block pool, so that a late cudaMalloc would fail (and
 * cudaMalloc / cudaFree would also synchronise the device mid-step).
 *
 * Same arguments, layouts and results as pa_paged_attention_decode, minus the
 * workspace: the split-partition scratch lives in a fixed array of
 * PA_STATIC_WORKSPACE_BYTES in the library's own device memory, which every GPU
 * that uses it holds until the process exits.  This function allocates nothing
 * and calls no allocating routine.
 *   - Sizes whose pa_paged_attention_workspace_size() exceeds
 *     PA_STATIC_WORKSPACE_BYTES are rejected with PA_ERR_WORKSPACE.
 *   - Set-up: the first call on a device, whatever its sizes (num_seqs = 0
 *     included), looks up the array's device address (cudaGetSymbolAddress, with
 *     that device current) and caches it.  Under lazy module loading, the CUDA 12
 *     default, that lookup is also when the driver reserves the array on the
 *     device.  So make one call on each device before handing nearly all free
 *     memory to a KV pool (or run with CUDA_MODULE_LOADING=EAGER), and before any
 *     stream capture.  If the set-up fails the call returns PA_ERR_CUDA.
 *   - The cached address belongs to the device's context of that moment: after
 *     cudaDeviceReset it is stale, and this entry point must not be called on that
 *     device again in the same process.
 *   - Every call on a device shares the one array and it keeps the last call's
 *     contents (nothing in it needs to start at zero).  Calls whose work overlaps
 *     on the GPU (other streams, other host threads) race on it: serialise them.
 */
int pa_paged_attention_decode_static_workspace(
    void* out, const void* query, const void* key_cache, const void* value_cache,
    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
    int max_seq_len, int num_heads, int num_kv_heads, int head_dim, int block_size,
    int64_t num_blocks, float scale, pa_dtype q_dtype, pa_dtype cache_dtype, pa_dtype out_dtype,
    float k_scale, float v_scale, int partition_size, void* stream);

/*
 * pa_swap_blocks -- move whole blocks between two pools, e.g. out of GPU memory into
 * page-locked host memory when the pool runs out, and back when a preempted
 * sequence resumes ("vLLM 是什么…" sec 5, misconception 3: blocks are swapped to
 * CPU memory, or requests preempted).  One launch moves every pair of every layer:
 * the kernel reads and writes host memory through its device mapping, so scattered
 * blocks cost no per-block copy call.
 *
 *   dst_key_caches, dst_value_caches,
 *   src_key_caches, src_value_caches
 *                  HOST arrays of num_layers pointers; each pool is device memory or
 *                  page-locked host memory the device addresses at the same pointer
 *                  (cudaHostAlloc / cudaMallocHost / torch pin_memory);
 *                  [src_num_blocks or dst_num_blocks][block_bytes] bytes per layer
 *   block_mapping  [num_pairs][2] int64 (src block, dst block), device memory or
 *                  page-locked host memory
 *   block_bytes    bytes of one block of one layer; a multiple of 16
 * Pairs run concurrently: a dst must not repeat.  An id out of range skips the pair
 * and sets PA_DEVERR_COPY_RANGE.  Pageable (unregistered) host memory is rejected
 * with PA_ERR_INVALID_ARG.  num_pairs == 0 or num_layers == 0 is a no-op.
 */
int pa_swap_blocks(void* const* dst_key_caches, void* const* dst_value_caches,
                   const void* const* src_key_caches, const void* const* src_value_caches,
                   int num_layers, const int64_t* block_mapping, int num_pairs,
                   size_t block_bytes, int64_t src_num_blocks, int64_t dst_num_blocks,
                   void* stream);

/* Human-readable name of a pa_status value (static storage). */
const char* pa_status_string(int status);

/*
 * pa_get_device_error -- synchronise `stream`, store the OR of every device error
 * bit raised since the last call into *host_flag, and clear the word.
 * Returns PA_OK, PA_ERR_INVALID_ARG (host_flag NULL) or PA_ERR_CUDA.
 */
int pa_get_device_error(int* host_flag, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
