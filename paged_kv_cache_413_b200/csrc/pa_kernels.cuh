// pa_kernels.cuh -- definitions shared by the attention kernels' translation units
// (decode, prefill): launch parameters, cache element traits, and the tensor-map
// encoder for the tiled TMA loads of the pool.
#pragma once

#include <cuda.h>  // CUtensorMap and its enums (types only; no driver library link)
#include <math.h>
#include <string.h>

#include <atomic>
#include <type_traits>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct Params {
  void* out;
  const uint8_t* query;
  const uint8_t* key_cache;
  const uint8_t* value_cache;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  float* ws_m;
  float* ws_l;
  float* ws_o;
  int max_blocks_per_seq;
  int block_size;       // tokens per physical block (a multiple of 16)
  int tiles_per_block;  // block_size / 16
  int max_seq_len;
  int cap;              // longest context the launch serves: min(max_seq_len, table width
                        // * block_size), computed on the host in 64 bits
  int num_heads;
  int num_kv_heads;
  int group;        // query heads per kv head
  int head_groups;  // CTAs per kv head (group / heads per CTA)
  int partition;    // tokens per partition (multiple of 16)
  int max_parts;
  int out_dtype;
  int64_t num_blocks;
  int num_seqs;     // sequences of the launch
  int lpt;          // decode: dispatch the longest sequences first (see decode_unit)
  float q_mult;     // scale * log2(e) [* k_scale]
  float v_mult;     // 1 or v_scale
};

template <typename CT>
struct CacheTraits;
template <>
struct CacheTraits<__half> {
  static constexpr int bytes = 2;
};
template <>
struct CacheTraits<__nv_bfloat16> {
  static constexpr int bytes = 2;
};
template <>
struct CacheTraits<fp8_e4m3> {
  static constexpr int bytes = 1;
};

// ---- tensor maps for the tensor-core kernel ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, fetched once through the runtime.
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// A pool [blocks][kv_heads][16][128] viewed as rows x 128 elements; boxes of 16 rows
// and 128 bytes (64 16-bit or 128 E4M3 elements), 128-byte swizzle.
bool encode_pool_map(CUtensorMap* m, const void* base, int64_t rows, bool fp8) {
  const cuuint64_t dims[2] = {128, cuuint64_t(rows)};
  const cuuint64_t strides[1] = {fp8 ? 128u : 256u};
  const cuuint32_t box[2] = {fp8 ? 128u : 64u, 16u};
  const cuuint32_t estr[2] = {1, 1};
  return encode_fn()(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2,
                     const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// Combine region layout: per warp and head the max (log2 units) and the sum, then
// the unnormalised accumulators with rows padded to D + 4 floats, which keeps the
// fragment-order writes of the four column groups on distinct banks.
template <int D>
constexpr int combine_row() {
  return D + 4;
}
template <int D, int GT>
constexpr size_t combine_bytes() {
  return (size_t(kConsumerWarps) * GT * 2 + size_t(kConsumerWarps) * GT * combine_row<D>() +
          size_t(GT) * (kConsumerWarps + 1)) *
         sizeof(float);
}

// Longest context a launch can serve: the host bound, or what the block tables
// can hold if that is less.  The product is taken in 64 bits, so wide tables of
// large blocks cannot overflow it; the result fits an int because max_seq_len does.
inline int context_cap(int max_seq_len, int max_blocks_per_seq, int block_size) {
  const int64_t table = int64_t(max_blocks_per_seq) * block_size;
  return table < max_seq_len ? int(table) : max_seq_len;
}

// Opt a kernel into `smem` bytes of dynamic shared memory on the current device,
// once per device and instantiation.  `done` records the devices set so far;
// fetch_or keeps concurrent host threads race-free (two of them may both make the
// idempotent call).  Devices past 63 are not recorded and get the call every time.
template <typename Kernel>
int set_smem_once(Kernel kern, size_t smem, std::atomic<unsigned long long>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return PA_OK;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
      cudaSuccess)
    return PA_ERR_CUDA;
  done.fetch_or(bit, std::memory_order_release);
  return PA_OK;
}

__device__ __forceinline__ void store_out(void* out, int64_t idx, float v, int dtype) {
  if (dtype == PA_F32)
    static_cast<float*>(out)[idx] = v;
  else if (dtype == PA_F16)
    static_cast<__half*>(out)[idx] = __float2half_rn(v);
  else
    static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
}

}  // namespace
}  // namespace pa
