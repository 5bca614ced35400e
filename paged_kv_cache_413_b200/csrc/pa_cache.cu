// pa_cache.cu -- cache-write and block-copy kernels (sm_100a).
//
// reshape_and_cache: the step of the memory flow that stores a new token's K and
// V rows into the slot the block manager registered for it ("vLLM 推理优化技术深度
// 调研报告" sec 2, memory flow; "vLLM 是什么…" sec 2, a new block only when the
// current one is full).  Optional fused FP8 E4M3 quantisation with a per-tensor
// scale ("vLLM推理引擎PagedAttention原理与性能优化实战" sec 5.2).
//
// copy_blocks: the copy step of copy-on-write ("vLLM推理引擎PagedAttention原理与
// 性能优化实战" sec 3.2).  swap_blocks: whole blocks between two pools, e.g. GPU
// memory and page-locked host memory when blocks are swapped out and back in
// ("vLLM 是什么…" sec 5, misconception 3); one kernel for all scattered blocks.
//
// All are pure data movement bound by HBM (or the host link); every access is a
// 16-byte vector (8-byte for the E4M3 stores), consecutive threads touch
// consecutive addresses.

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

__device__ unsigned int g_cache_err;

// Quantise 8 packed 16-bit values (one uint4) to 8 E4M3 bytes (one uint2):
// IEEE fp32 division by the scale, then round-nearest-even with saturation.
template <typename Tsrc>
__device__ __forceinline__ uint2 quantise8(uint4 x, float scale) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint16_t q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = unpack2(w[i], Tsrc{});
    q[i] = pack2_e4m3(__fdiv_rn(f.x, scale), __fdiv_rn(f.y, scale));
  }
  return make_uint2(uint32_t(q[0]) | (uint32_t(q[1]) << 16),
                    uint32_t(q[2]) | (uint32_t(q[3]) << 16));
}

// grid = (tokens, slices): the CTAs of a token split its row of 8-element chunks, so
// that every thread moves one chunk of K and one of V (one DRAM round trip) when
// the row has at most 128 x slices chunks.
template <typename Tsrc, bool kQuant>
__global__ void __launch_bounds__(128) reshape_and_cache_kernel(
    const uint16_t* __restrict__ key, const uint16_t* __restrict__ value,
    uint8_t* __restrict__ key_cache, uint8_t* __restrict__ value_cache,
    const int64_t* __restrict__ slot_mapping, int num_kv_heads, int head_dim, int block_size,
    int64_t num_slots, float k_scale, float v_scale) {
  // the decode that reads these slots is a programmatic dependent: let its CTAs be
  // scheduled now (it still waits for this grid to complete before reading)
  grid_dependents_may_launch();
  const int64_t t = blockIdx.x;
  const int64_t slot = slot_mapping[t];
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (threadIdx.x == 0 && blockIdx.y == 0) atomicOr(&g_cache_err, PA_DEVERR_SLOT_RANGE);
    return;
  }
  const int64_t blk = slot / block_size, off = slot % block_size;
  const int row = num_kv_heads * head_dim;  // elements of one token
  const int chunks = row >> 3;
  for (int c = blockIdx.y * blockDim.x + threadIdx.x; c < chunks; c += gridDim.y * blockDim.x) {
    const int e = c << 3;
    const int h = e / head_dim, d = e - h * head_dim;
    const int64_t src = t * row + e;
    const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim + d;
    const uint4 kx = __ldg(reinterpret_cast<const uint4*>(key + src));
    const uint4 vx = __ldg(reinterpret_cast<const uint4*>(value + src));
    if constexpr (!kQuant) {
      *reinterpret_cast<uint4*>(key_cache + dst * 2) = kx;
      *reinterpret_cast<uint4*>(value_cache + dst * 2) = vx;
    } else {
      *reinterpret_cast<uint2*>(key_cache + dst) = quantise8<Tsrc>(kx, k_scale);
      *reinterpret_cast<uint2*>(value_cache + dst) = quantise8<Tsrc>(vx, v_scale);
    }
  }
}

struct LayerPtrs {
  const uint8_t* src_k[kMaxLayersPerLaunch];
  const uint8_t* src_v[kMaxLayersPerLaunch];
  uint8_t* dst_k[kMaxLayersPerLaunch];
  uint8_t* dst_v[kMaxLayersPerLaunch];
};

// grid = (pairs, layers, 2): one CTA moves one block of one layer's K or V from the
// source pool to the destination pool (the same pool for copy-on-write copies).
// Either pool may be page-locked host memory mapped into the device address space.
__global__ void __launch_bounds__(256) move_blocks_kernel(LayerPtrs ptrs,
                                                          const int64_t* __restrict__ mapping,
                                                          int64_t block_bytes,
                                                          int64_t src_num_blocks,
                                                          int64_t dst_num_blocks) {
  const int64_t src = mapping[2 * blockIdx.x], dst = mapping[2 * blockIdx.x + 1];
  if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
      atomicOr(&g_cache_err, PA_DEVERR_COPY_RANGE);
    return;
  }
  const uint8_t* sbase = blockIdx.z ? ptrs.src_v[blockIdx.y] : ptrs.src_k[blockIdx.y];
  uint8_t* dbase = blockIdx.z ? ptrs.dst_v[blockIdx.y] : ptrs.dst_k[blockIdx.y];
  const uint4* s = reinterpret_cast<const uint4*>(sbase + src * block_bytes);
  uint4* d = reinterpret_cast<uint4*>(dbase + dst * block_bytes);
  const int64_t n = block_bytes >> 4;
  // four independent 16-byte loads in flight per thread before the stores
  int64_t i = threadIdx.x;
  for (; i + 3 * blockDim.x < n; i += 4 * blockDim.x) {
    const uint4 a = s[i], b = s[i + blockDim.x], c = s[i + 2 * blockDim.x],
                e = s[i + 3 * blockDim.x];
    d[i] = a;
    d[i + blockDim.x] = b;
    d[i + 2 * blockDim.x] = c;
    d[i + 3 * blockDim.x] = e;
  }
  for (; i < n; i += blockDim.x) d[i] = s[i];
}

cudaError_t launch_move_blocks(void* const* dst_k, void* const* dst_v, const void* const* src_k,
                               const void* const* src_v, int num_layers,
                               const int64_t* block_mapping, int num_pairs, size_t block_bytes,
                               int64_t src_num_blocks, int64_t dst_num_blocks,
                               cudaStream_t stream) {
  for (int l0 = 0; l0 < num_layers; l0 += kMaxLayersPerLaunch) {
    const int nl = num_layers - l0 < kMaxLayersPerLaunch ? num_layers - l0 : kMaxLayersPerLaunch;
    LayerPtrs p{};
    for (int i = 0; i < nl; ++i) {
      p.src_k[i] = static_cast<const uint8_t*>(src_k[l0 + i]);
      p.src_v[i] = static_cast<const uint8_t*>(src_v[l0 + i]);
      p.dst_k[i] = static_cast<uint8_t*>(dst_k[l0 + i]);
      p.dst_v[i] = static_cast<uint8_t*>(dst_v[l0 + i]);
    }
    move_blocks_kernel<<<dim3(num_pairs, nl, 2), 256, 0, stream>>>(
        p, block_mapping, static_cast<int64_t>(block_bytes), src_num_blocks, dst_num_blocks);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* key_cache,
                                     void* value_cache, const int64_t* slot_mapping,
                                     int num_tokens, int num_kv_heads, int head_dim,
                                     int block_size, int64_t num_blocks, pa_dtype src_dtype,
                                     pa_dtype cache_dtype, float k_scale, float v_scale,
                                     cudaStream_t stream) {
  // up to 8 slices a token (a row of 8192 elements), one chunk a thread
  const int chunks = (num_kv_heads * head_dim) >> 3;
  const int slices = (chunks + 127) / 128 < 8 ? (chunks + 127) / 128 : 8;
  const dim3 grid(unsigned(num_tokens), unsigned(slices > 0 ? slices : 1)), block(128);
  const int64_t num_slots = num_blocks * block_size;
  auto k = static_cast<const uint16_t*>(key);
  auto v = static_cast<const uint16_t*>(value);
  auto kc = static_cast<uint8_t*>(key_cache);
  auto vc = static_cast<uint8_t*>(value_cache);
  if (cache_dtype != PA_FP8_E4M3) {
    reshape_and_cache_kernel<__half, false><<<grid, block, 0, stream>>>(
        k, v, kc, vc, slot_mapping, num_kv_heads, head_dim, block_size, num_slots, k_scale,
        v_scale);
  } else if (src_dtype == PA_F16) {
    reshape_and_cache_kernel<__half, true><<<grid, block, 0, stream>>>(
        k, v, kc, vc, slot_mapping, num_kv_heads, head_dim, block_size, num_slots, k_scale,
        v_scale);
  } else {
    reshape_and_cache_kernel<__nv_bfloat16, true><<<grid, block, 0, stream>>>(
        k, v, kc, vc, slot_mapping, num_kv_heads, head_dim, block_size, num_slots, k_scale,
        v_scale);
  }
  return cudaGetLastError();
}

cudaError_t launch_copy_blocks(void* const* key_caches, void* const* value_caches,
                               int num_layers, const int64_t* block_mapping, int num_pairs,
                               size_t block_bytes, int64_t num_blocks, cudaStream_t stream) {
  return launch_move_blocks(key_caches, value_caches, key_caches, value_caches, num_layers,
                            block_mapping, num_pairs, block_bytes, num_blocks, num_blocks, stream);
}

cudaError_t launch_swap_blocks(void* const* dst_key_caches, void* const* dst_value_caches,
                               const void* const* src_key_caches,
                               const void* const* src_value_caches, int num_layers,
                               const int64_t* block_mapping, int num_pairs, size_t block_bytes,
                               int64_t src_num_blocks, int64_t dst_num_blocks,
                               cudaStream_t stream) {
  return launch_move_blocks(dst_key_caches, dst_value_caches, src_key_caches, src_value_caches,
                            num_layers, block_mapping, num_pairs, block_bytes, src_num_blocks,
                            dst_num_blocks, stream);
}

cudaError_t read_and_clear_cache_errors(unsigned* bits, cudaStream_t stream) {
  unsigned v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_cache_err, sizeof v, 0,
                                            cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  const unsigned zero = 0;
  e = cudaMemcpyToSymbolAsync(g_cache_err, &zero, sizeof zero, 0, cudaMemcpyHostToDevice,
                              stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  *bits |= v;
  return e;
}

}  // namespace pa
