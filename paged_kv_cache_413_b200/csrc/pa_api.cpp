// pa_api.cpp -- the C ABI of libpa.so (declared in include/pa.h).
//
// Each entry point validates what the host can see (pointers, sizes, alignment,
// supported combinations), picks the launch configuration and enqueues the
// kernels on the caller's stream.  Nothing here allocates or keeps state.

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "pa.h"
#include "pa_internal.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_dtype(int t) { return t >= PA_F16 && t <= PA_FP8_E4M3; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? PA_OK : PA_ERR_CUDA; }

}  // namespace

extern "C" {

int pa_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                         const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int64_t num_blocks, pa_dtype src_dtype,
                         pa_dtype cache_dtype, float k_scale, float v_scale, void* stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_blocks <= 0 || !valid_dtype(src_dtype) || !valid_dtype(cache_dtype))
    return PA_ERR_INVALID_ARG;
  if (!pa::valid_block_size(block_size) || head_dim % 8 != 0 || head_dim > 256)
    return PA_ERR_UNSUPPORTED;
  if (src_dtype != PA_F16 && src_dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  const bool quant = cache_dtype == PA_FP8_E4M3;
  if (!quant && cache_dtype != src_dtype) return PA_ERR_UNSUPPORTED;
  if (quant && !(isfinite(k_scale) && k_scale > 0.f && isfinite(v_scale) && v_scale > 0.f))
    return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return PA_ERR_INVALID_ARG;
  return cuda_status(pa::launch_reshape_and_cache(
      key, value, key_cache, value_cache, slot_mapping, num_tokens, num_kv_heads, head_dim,
      block_size, num_blocks, src_dtype, cache_dtype, k_scale, v_scale,
      static_cast<cudaStream_t>(stream)));
}

size_t pa_paged_attention_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                         int head_dim, int max_seq_len, int partition_size) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 ||
      head_dim <= 0 || max_seq_len < 0 || partition_size < 0 ||
      partition_size % pa::kBlockSize != 0)
    return 0;
  const int part =
      pa::resolve_partition(partition_size, num_seqs, num_heads, num_kv_heads, max_seq_len);
  return pa::workspace_layout(num_seqs, num_heads, head_dim, max_seq_len, part).total;
}

int pa_paged_attention_partition_size(int num_seqs, int num_heads, int num_kv_heads,
                                      int max_seq_len, int partition_size) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 ||
      max_seq_len < 0 || partition_size < 0 || partition_size % pa::kBlockSize != 0)
    return 0;
  return pa::resolve_partition(partition_size, num_seqs, num_heads, num_kv_heads, max_seq_len);
}

int pa_paged_attention_decode(void* out, const void* query, const void* key_cache,
                              const void* value_cache, const int32_t* block_tables,
                              int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                              int max_seq_len, int num_heads, int num_kv_heads, int head_dim,
                              int block_size, int64_t num_blocks, float scale, pa_dtype q_dtype,
                              pa_dtype cache_dtype, pa_dtype out_dtype, float k_scale,
                              float v_scale, int partition_size, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (num_seqs < 0 || max_seq_len < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
      head_dim <= 0 || block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq < 0 ||
      partition_size < 0 || !valid_dtype(q_dtype) || !valid_dtype(cache_dtype) ||
      !valid_dtype(out_dtype) || !isfinite(scale))
    return PA_ERR_INVALID_ARG;
  if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  if (partition_size % pa::kBlockSize != 0) return PA_ERR_INVALID_ARG;
  if (!pa::valid_block_size(block_size) || (head_dim != 64 && head_dim != 128))
    return PA_ERR_UNSUPPORTED;
  if (out_dtype == PA_FP8_E4M3 || q_dtype == PA_FP8_E4M3 || q_dtype == PA_F32)
    return PA_ERR_UNSUPPORTED;
  if (cache_dtype != PA_FP8_E4M3 && cache_dtype != q_dtype) return PA_ERR_UNSUPPORTED;
  if (cache_dtype == PA_F32) return PA_ERR_UNSUPPORTED;
  if (cache_dtype == PA_FP8_E4M3 &&
      !(isfinite(k_scale) && k_scale > 0.f && isfinite(v_scale) && v_scale > 0.f))
    return PA_ERR_INVALID_ARG;
  if (int64_t(max_blocks_per_seq) * block_size < int64_t(max_seq_len))
    return PA_ERR_INVALID_ARG;  // the tables cannot hold the longest context
  if (num_seqs == 0) return PA_OK;
  if (!out || !query || !key_cache || !value_cache || !seq_lens ||
      (max_seq_len > 0 && !block_tables))
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3u))
    return PA_ERR_INVALID_ARG;
  const int part =
      pa::resolve_partition(partition_size, num_seqs, num_heads, num_kv_heads, max_seq_len);
  pa::DecodeArgs a{};
  a.ws = pa::workspace_layout(num_seqs, num_heads, head_dim, max_seq_len, part);
  if (a.ws.total > 0 && (!workspace || workspace_bytes < a.ws.total || !aligned16(workspace)))
    return PA_ERR_WORKSPACE;
  if (int64_t(num_seqs) * (a.ws.max_parts > 0 ? a.ws.max_parts : 1) > INT32_MAX ||
      int64_t(num_seqs) * num_heads > INT32_MAX || num_heads > 65535)
    return PA_ERR_UNSUPPORTED;  // grid limits
  a.out = out;
  a.query = query;
  a.key_cache = key_cache;
  a.value_cache = value_cache;
  a.block_tables = block_tables;
  a.seq_lens = seq_lens;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.max_seq_len = max_seq_len;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.scale = scale;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.q_dtype = q_dtype;
  a.cache_dtype = cache_dtype;
  a.out_dtype = out_dtype;
  a.partition = part;
  a.workspace = workspace;
  return pa::launch_decode(a, static_cast<cudaStream_t>(stream));
}

int pa_paged_attention_decode_shared_prefix(
    void* out, const void* query, const void* key_cache, const void* value_cache,
    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
    int max_seq_len, const int32_t* group_starts, const int32_t* prefix_lens, int num_groups,
    int max_group_size, int num_heads, int num_kv_heads, int head_dim, int block_size,
    int64_t num_blocks, float scale, pa_dtype q_dtype, pa_dtype cache_dtype, pa_dtype out_dtype,
    float k_scale, float v_scale, void* stream) {
  if (num_seqs < 0 || num_groups < 0 || max_group_size < 0 || max_seq_len < 0 ||
      num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_blocks <= 0 || max_blocks_per_seq < 0 || !valid_dtype(q_dtype) ||
      !valid_dtype(cache_dtype) || !valid_dtype(out_dtype) || !isfinite(scale))
    return PA_ERR_INVALID_ARG;
  if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  if (!pa::valid_block_size(block_size) || head_dim != 128 || num_heads / num_kv_heads > 16 ||
      num_heads > 65535)
    return PA_ERR_UNSUPPORTED;
  if (out_dtype == PA_FP8_E4M3 || q_dtype == PA_FP8_E4M3 || q_dtype == PA_F32 ||
      cache_dtype == PA_F32 || (cache_dtype != PA_FP8_E4M3 && cache_dtype != q_dtype))
    return PA_ERR_UNSUPPORTED;
  if (cache_dtype == PA_FP8_E4M3 &&
      !(isfinite(k_scale) && k_scale > 0.f && isfinite(v_scale) && v_scale > 0.f))
    return PA_ERR_INVALID_ARG;
  if (int64_t(max_blocks_per_seq) * block_size < int64_t(max_seq_len))
    return PA_ERR_INVALID_ARG;
  if (num_seqs == 0 || num_groups == 0) return PA_OK;
  if (max_group_size == 0) return PA_ERR_INVALID_ARG;
  if (!out || !query || !key_cache || !value_cache || !seq_lens || !group_starts ||
      !prefix_lens || (max_seq_len > 0 && !block_tables))
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
      (reinterpret_cast<uintptr_t>(group_starts) & 3u) ||
      (reinterpret_cast<uintptr_t>(prefix_lens) & 3u))
    return PA_ERR_INVALID_ARG;
  pa::DecodeArgs a{};
  a.out = out;
  a.query = query;
  a.key_cache = key_cache;
  a.value_cache = value_cache;
  a.block_tables = block_tables;
  a.seq_lens = seq_lens;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.max_seq_len = max_seq_len;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.scale = scale;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.q_dtype = q_dtype;
  a.cache_dtype = cache_dtype;
  a.out_dtype = out_dtype;
  return pa::launch_decode_shared_prefix(a, group_starts, prefix_lens, num_groups, max_group_size,
                                         static_cast<cudaStream_t>(stream));
}

int pa_paged_attention_prefill(void* out, const void* query, const void* key_cache,
                               const void* value_cache, const int32_t* block_tables,
                               int max_blocks_per_seq, const int32_t* seq_lens,
                               const int32_t* query_start, int num_seqs, int max_query_len,
                               int max_seq_len, int num_heads, int num_kv_heads, int head_dim,
                               int block_size, int64_t num_blocks, float scale,
                               pa_dtype q_dtype, pa_dtype cache_dtype, pa_dtype out_dtype,
                               void* stream) {
  if (num_seqs < 0 || max_query_len < 0 || max_seq_len < 0 || num_heads <= 0 ||
      num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0 ||
      max_blocks_per_seq < 0 || !valid_dtype(q_dtype) || !valid_dtype(cache_dtype) ||
      !valid_dtype(out_dtype) || !isfinite(scale))
    return PA_ERR_INVALID_ARG;
  if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  if (!pa::valid_block_size(block_size) || head_dim != 128 || num_heads > 65535 ||
      (q_dtype != PA_F16 && q_dtype != PA_BF16) || cache_dtype != q_dtype ||
      out_dtype == PA_FP8_E4M3)
    return PA_ERR_UNSUPPORTED;
  if (int64_t(max_blocks_per_seq) * block_size < int64_t(max_seq_len) ||
      max_query_len > max_seq_len)
    return PA_ERR_INVALID_ARG;
  if (num_seqs == 0 || max_query_len == 0) return PA_OK;
  if (!out || !query || !key_cache || !value_cache || !seq_lens || !query_start || !block_tables)
    return PA_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
      (reinterpret_cast<uintptr_t>(query_start) & 3u))
    return PA_ERR_INVALID_ARG;
  pa::DecodeArgs a{};
  a.out = out;
  a.query = query;
  a.key_cache = key_cache;
  a.value_cache = value_cache;
  a.block_tables = block_tables;
  a.seq_lens = seq_lens;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.max_seq_len = max_seq_len;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.scale = scale;
  a.q_dtype = q_dtype;
  a.cache_dtype = cache_dtype;
  a.out_dtype = out_dtype;
  return pa::launch_prefill(a, query_start, max_query_len, static_cast<cudaStream_t>(stream));
}

int pa_copy_blocks(void* const* key_caches, void* const* value_caches, int num_layers,
                   const int64_t* block_mapping, int num_pairs, size_t block_bytes,
                   int64_t num_blocks, void* stream) {
  if (num_layers < 0 || num_pairs < 0 || num_blocks <= 0) return PA_ERR_INVALID_ARG;
  if (num_layers == 0 || num_pairs == 0) return PA_OK;
  if (!key_caches || !value_caches || !block_mapping || block_bytes == 0 || block_bytes % 16)
    return PA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(block_mapping) & 7u) return PA_ERR_INVALID_ARG;
  if (num_pairs > 0x7fffffff) return PA_ERR_UNSUPPORTED;
  for (int l = 0; l < num_layers; ++l)
    if (!key_caches[l] || !value_caches[l] || !aligned16(key_caches[l]) ||
        !aligned16(value_caches[l]))
      return PA_ERR_INVALID_ARG;
  return cuda_status(pa::launch_copy_blocks(key_caches, value_caches, num_layers, block_mapping,
                                            num_pairs, block_bytes, num_blocks,
                                            static_cast<cudaStream_t>(stream)));
}

// Device memory, or page-locked host memory that the device can address directly
// at the same pointer (all cudaHostAlloc / pinned allocations under unified addressing).
static bool device_addressable(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return true;
  return a.type == cudaMemoryTypeHost && a.devicePointer == p;
}

int pa_swap_blocks(void* const* dst_key_caches, void* const* dst_value_caches,
                   const void* const* src_key_caches, const void* const* src_value_caches,
                   int num_layers, const int64_t* block_mapping, int num_pairs,
                   size_t block_bytes, int64_t src_num_blocks, int64_t dst_num_blocks,
                   void* stream) {
  if (num_layers < 0 || num_pairs < 0 || src_num_blocks <= 0 || dst_num_blocks <= 0)
    return PA_ERR_INVALID_ARG;
  if (num_layers == 0 || num_pairs == 0) return PA_OK;
  if (!dst_key_caches || !dst_value_caches || !src_key_caches || !src_value_caches ||
      !block_mapping || block_bytes == 0 || block_bytes % 16)
    return PA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(block_mapping) & 7u) || !device_addressable(block_mapping))
    return PA_ERR_INVALID_ARG;
  for (int l = 0; l < num_layers; ++l) {
    const void* ptrs[4] = {dst_key_caches[l], dst_value_caches[l], src_key_caches[l],
                           src_value_caches[l]};
    for (const void* q : ptrs)
      if (!q || !aligned16(q) || !device_addressable(q)) return PA_ERR_INVALID_ARG;
  }
  return cuda_status(pa::launch_swap_blocks(dst_key_caches, dst_value_caches, src_key_caches,
                                            src_value_caches, num_layers, block_mapping,
                                            num_pairs, block_bytes, src_num_blocks,
                                            dst_num_blocks, static_cast<cudaStream_t>(stream)));
}

const char* pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    default: return "PA_UNKNOWN_STATUS";
  }
}

int pa_get_device_error(int* host_flag, void* stream) {
  if (!host_flag) return PA_ERR_INVALID_ARG;
  unsigned bits = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = pa::read_and_clear_cache_errors(&bits, s);
  if (e == cudaSuccess) e = pa::read_and_clear_decode_errors(&bits, s);
  if (e == cudaSuccess) e = pa::read_and_clear_prefill_errors(&bits, s);
  if (e == cudaSuccess) e = pa::read_and_clear_shared_errors(&bits, s);
  *host_flag = static_cast<int>(bits);
  return cuda_status(e);
}

}  // extern "C"
