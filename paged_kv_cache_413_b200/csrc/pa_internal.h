// pa_internal.h -- host-side launchers shared between the kernel files and the
// C ABI layer (pa_api.cpp).  Arguments are already validated when these run.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

constexpr int kBlockSize = 16;            // tokens per streamed tile (and the smallest block)

// Physical block sizes the kernels take: multiples of the 16-token tile.
inline bool valid_block_size(int bs) { return bs == 16 || bs == 32 || bs == 64 || bs == 128; }
constexpr int kDefaultPartition = 512;     // tokens per split-K partition
constexpr int kMaxLayersPerLaunch = 64;    // copy_blocks: layer pointers per launch

struct WorkspaceLayout {
  size_t m_off, l_off, o_off, total;       // byte offsets of the m, l, o sections
  int max_parts;                           // partitions of the longest sequence
};

constexpr int kAutoTargetCtas = 2048;   // work units that keep a B200's 148 SMs streaming
constexpr int kAutoMinPartition = 256;  // smallest partition the default ever picks

// Query heads served by one CTA: the largest of 8, 4, 2, 1 dividing the group.
inline int heads_per_cta(int group) {
  return group % 8 == 0 ? 8 : group % 4 == 0 ? 4 : group % 2 == 0 ? 2 : 1;
}

// Partition size in tokens.  A positive request is taken as is.  The default (0)
// splits a sequence only when there are fewer than kAutoTargetCtas (sequence,
// head group) units to spread over the GPU: then into enough partitions of at
// least kAutoMinPartition tokens to reach that count.  Longer partitions amortise
// each CTA's pipeline fill and epilogue and avoid the merge pass.
inline int resolve_partition(int requested, int num_seqs, int num_heads, int num_kv_heads,
                             int max_seq_len) {
  if (requested > 0) return requested;
  const int whole = max_seq_len > 16 ? (max_seq_len + 15) / 16 * 16 : 16;
  const int64_t units =
      int64_t(num_seqs) * num_heads / heads_per_cta(num_kv_heads > 0 ? num_heads / num_kv_heads : 1);
  if (units >= kAutoTargetCtas) return whole;
  const int64_t splits = (kAutoTargetCtas + units - 1) / (units > 0 ? units : 1);
  int part = int((max_seq_len + splits - 1) / splits + 15) / 16 * 16;
  if (part < kAutoMinPartition) part = kAutoMinPartition;
  return part < whole ? part : whole;
}

inline WorkspaceLayout workspace_layout(int num_seqs, int num_heads, int head_dim,
                                        int max_seq_len, int partition) {
  WorkspaceLayout w{};
  w.max_parts = max_seq_len > 0 ? (max_seq_len + partition - 1) / partition : 0;
  if (w.max_parts <= 1) return w;  // no workspace needed
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t rows = size_t(num_seqs) * num_heads * w.max_parts;
  w.m_off = 0;
  w.l_off = up(rows * sizeof(float));
  w.o_off = w.l_off + up(rows * sizeof(float));
  w.total = w.o_off + up(rows * size_t(head_dim) * sizeof(float));
  return w;
}

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* key_cache,
                                     void* value_cache, const int64_t* slot_mapping,
                                     int num_tokens, int num_kv_heads, int head_dim,
                                     int block_size, int64_t num_blocks, pa_dtype src_dtype,
                                     pa_dtype cache_dtype, float k_scale, float v_scale,
                                     cudaStream_t stream);

cudaError_t launch_copy_blocks(void* const* key_caches, void* const* value_caches,
                               int num_layers, const int64_t* block_mapping, int num_pairs,
                               size_t block_bytes, int64_t num_blocks, cudaStream_t stream);

cudaError_t launch_swap_blocks(void* const* dst_key_caches, void* const* dst_value_caches,
                               const void* const* src_key_caches,
                               const void* const* src_value_caches, int num_layers,
                               const int64_t* block_mapping, int num_pairs, size_t block_bytes,
                               int64_t src_num_blocks, int64_t dst_num_blocks,
                               cudaStream_t stream);

struct DecodeArgs {
  void* out;
  const void* query;
  const void* key_cache;
  const void* value_cache;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  int max_blocks_per_seq, num_seqs, max_seq_len, num_heads, num_kv_heads, head_dim;
  int block_size;
  int64_t num_blocks;
  float scale, k_scale, v_scale;
  pa_dtype q_dtype, cache_dtype, out_dtype;
  int partition;                 // resolved, tokens
  WorkspaceLayout ws;
  void* workspace;
};

// PA_OK, PA_ERR_UNSUPPORTED (no kernel for the combination) or PA_ERR_CUDA.
int launch_decode(const DecodeArgs& a, cudaStream_t stream);

// Multi-query (chunked prefill) attention.
int launch_prefill(const DecodeArgs& a, const int32_t* query_start, int max_query_len,
                   cudaStream_t stream);

// Shared-prefix decode (groups of sequences sharing their first blocks).
int launch_decode_shared_prefix(const DecodeArgs& a, const int32_t* group_starts,
                                const int32_t* prefix_lens, int num_groups, int max_group_size,
                                cudaStream_t stream);

// Read and clear the device error words of the kernel files (synchronises stream).
cudaError_t read_and_clear_cache_errors(unsigned* bits, cudaStream_t stream);
cudaError_t read_and_clear_decode_errors(unsigned* bits, cudaStream_t stream);
cudaError_t read_and_clear_prefill_errors(unsigned* bits, cudaStream_t stream);
cudaError_t read_and_clear_shared_errors(unsigned* bits, cudaStream_t stream);

}  // namespace pa
