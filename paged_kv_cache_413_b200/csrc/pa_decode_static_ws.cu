// pa_decode_static_ws.cu -- decode attention for callers that cannot allocate.
//
// pa_paged_attention_decode needs a caller-provided device workspace when a
// sequence spans more than one partition.  Some callers cannot provide one: a
// plugin running inside a host process that owns every device allocation and
// hands its plugins no allocator, or a serving engine that has already reserved
// nearly all HBM for its KV block pool so that a late cudaMalloc would fail (and
// cudaMalloc / cudaFree would also synchronise the device in the middle of a
// step).  This entry point serves them: its scratch is a fixed array in the
// library's own device memory, held by every GPU that uses it until the process
// exits.
//
// The array's name is a device symbol.  In host code it is only a stand-in, not
// a device address, so the address is looked up with cudaGetSymbolAddress (with
// that device current) on the first call on each device, and passed to the
// kernels.  Under lazy module loading (the CUDA 12 default) that lookup is also
// the moment the driver reserves the array on the device.

#include <cuda_runtime.h>

#include <mutex>

#include "pa.h"
#include "pa_internal.h"

namespace {

constexpr int kMaxDevices = 64;

// The scratch shared by every call of pa_paged_attention_decode_static_workspace
// on a device.  Nothing in it needs to start at zero: every byte the kernels read
// was written earlier in the same call.
static __device__ __align__(256) unsigned char g_decode_scratch[PA_STATIC_WORKSPACE_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device: looked up on the
// first call on that device and kept (devices past kMaxDevices: every call).
int scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  const bool cached = dev >= 0 && dev < kMaxDevices;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!cached || g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
      return PA_ERR_CUDA;
    if (!cached) {
      *out = p;
      return PA_OK;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return PA_OK;
}

}  // namespace

extern "C" int pa_paged_attention_decode_static_workspace(
    void* out, const void* query, const void* key_cache, const void* value_cache,
    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
    int max_seq_len, int num_heads, int num_kv_heads, int head_dim, int block_size,
    int64_t num_blocks, float scale, pa_dtype q_dtype, pa_dtype cache_dtype, pa_dtype out_dtype,
    float k_scale, float v_scale, int partition_size, void* stream) {
  // The set-up comes first, whatever the sizes, so that any first call on a device
  // (num_seqs = 0 included) reserves the array there.
  void* scratch = nullptr;
  const int rc = scratch_on_current_device(&scratch);
  if (rc != PA_OK) return rc;
  const size_t need = pa_paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads,
                                                        head_dim, max_seq_len, partition_size);
  if (need > PA_STATIC_WORKSPACE_BYTES) return PA_ERR_WORKSPACE;  // beyond the fixed maximum
  return pa_paged_attention_decode(out, query, key_cache, value_cache, block_tables,
                                   max_blocks_per_seq, seq_lens, num_seqs, max_seq_len,
                                   num_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                   scale, q_dtype, cache_dtype, out_dtype, k_scale, v_scale,
                                   partition_size, scratch, PA_STATIC_WORKSPACE_BYTES, stream);
}
