// pa_decode.cu -- paged decode attention for sm_100a.
//
// out[s][h] = softmax(scale * q[s][h] . K_s^T) V_s where K_s and V_s are the first
// seq_len tokens of sequence s, gathered from 16-token physical blocks through its
// block table ("vLLM 推理优化技术深度调研报告" sec 3 formulas 3 and 4).  Decode is
// bound by HBM bandwidth (the same report, sec 3 formula 5: the decode stage is
// memory-bandwidth limited), so the kernel is built around moving every K/V byte
// exactly once at full bandwidth:
//
//   * one CTA per (sequence, partition of <= `partition` tokens, kv head group);
//     the CTA serves every query head that shares the kv head (GQA), so each K/V
//     block is read from HBM once for the whole group;
//   * a producer warp walks the block table and issues one 1-D bulk asynchronous
//     copy (TMA engine, cp.async.bulk) per K block and per V block of the kv head
//     (16 tokens x head_dim, contiguous in the pool layout) into a ring of
//     shared-memory stages guarded by mbarriers; no multicast;
//   * four consumer warps take blocks round-robin; each keeps its own fp32 online
//     softmax state (running max, running sum) and fp32 accumulator;
//   * at the end the warps' states are merged in shared memory; a sequence with
//     one partition writes its output directly, otherwise each partition writes
//     (m, l, o) to the workspace and a log-sum-exp reduce kernel merges them.
//
// Scores are kept in log2 units (q is pre-multiplied by scale * log2(e) and, for
// FP8 caches, by k_scale), so exponentials are exp2.

#include <math.h>

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

__device__ unsigned int g_decode_err;

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kStages = 8;
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
  int max_seq_len;
  int num_heads;
  int num_kv_heads;
  int group;        // query heads per kv head
  int head_groups;  // CTAs per kv head (group / heads per CTA)
  int partition;    // tokens per partition (multiple of 16)
  int max_parts;
  int out_dtype;
  int64_t num_blocks;
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

// This lane's DPL = D/32 consecutive elements of row `row` of a [16][D] tile.
template <typename CT, int D>
__device__ __forceinline__ void load_lane_row(const uint8_t* tile, int row, int lane,
                                              float (&f)[D / 32]) {
  constexpr int DPL = D / 32;
  if constexpr (CacheTraits<CT>::bytes == 2) {
    const uint8_t* p = tile + (row * D + lane * DPL) * 2;
    if constexpr (DPL == 4) {
      const uint2 w = *reinterpret_cast<const uint2*>(p);
      const float2 a = unpack2(w.x, CT{}), b = unpack2(w.y, CT{});
      f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    } else {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
      const float2 a = unpack2(w, CT{});
      f[0] = a.x; f[1] = a.y;
    }
  } else {
    const uint8_t* p = tile + row * D + lane * DPL;
    if constexpr (DPL == 4) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
      const float2 a = unpack2_e4m3(static_cast<uint16_t>(w & 0xffffu));
      const float2 b = unpack2_e4m3(static_cast<uint16_t>(w >> 16));
      f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    } else {
      const uint16_t w = *reinterpret_cast<const uint16_t*>(p);
      const float2 a = unpack2_e4m3(w);
      f[0] = a.x; f[1] = a.y;
    }
  }
}

// Sum N per-lane values over the 32 lanes of a warp so that lane l ends up with
// the total of value index (l >> (5 - log2 N)).  Recursive halving: at each level
// a lane keeps one half of its values and sends the other half to its partner.
template <int N>
__device__ __forceinline__ float transpose_reduce(float (&v)[N], int lane) {
  static_assert(N == 16 || N == 32, "N must be 16 or 32");
  int o = 16;
#pragma unroll
  for (int n = N; n > 1; n >>= 1, o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < n / 2; ++j) {
      const float send = upper ? v[j] : v[j + n / 2];
      const float keep = upper ? v[j + n / 2] : v[j];
      v[j] = keep + __shfl_xor_sync(kFullMask, send, o);
    }
  }
#pragma unroll
  for (; o >= 1; o >>= 1) v[0] += __shfl_xor_sync(kFullMask, v[0], o);
  return v[0];
}

template <typename QT, int D>
__device__ __forceinline__ void load_q_lane(const uint8_t* q, int lane, float mult,
                                            float (&f)[D / 32]) {
  constexpr int DPL = D / 32;
  const uint8_t* p = q + lane * DPL * 2;
  if constexpr (DPL == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    const float2 a = unpack2(w.x, QT{}), b = unpack2(w.y, QT{});
    f[0] = a.x * mult; f[1] = a.y * mult; f[2] = b.x * mult; f[3] = b.y * mult;
  } else {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    const float2 a = unpack2(w, QT{});
    f[0] = a.x * mult; f[1] = a.y * mult;
  }
}

__device__ __forceinline__ void store_out(void* out, int64_t idx, float v, int dtype) {
  if (dtype == PA_F32)
    static_cast<float*>(out)[idx] = v;
  else if (dtype == PA_F16)
    static_cast<__half*>(out)[idx] = __float2half_rn(v);
  else
    static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
}

template <int D, int GT, typename CT>
constexpr size_t smem_bytes() {
  constexpr size_t tile = size_t(kBlockSize) * D * CacheTraits<CT>::bytes;
  constexpr size_t pipe = 2 * kStages * tile;
  constexpr size_t combine = size_t(kConsumerWarps) * GT * (D + 2) * sizeof(float);
  constexpr size_t body = pipe > combine ? pipe : combine;
  return body + 2 * kStages * sizeof(uint64_t) + size_t(kConsumerWarps) * GT * 16 * sizeof(float);
}

// GT: query heads served by one CTA (a divisor of the GQA group, at most 8).
template <int D, int GT, typename CT, typename QT>
__global__ void __launch_bounds__(kThreads) decode_kernel(const Params p) {
  static_assert(D == 64 || D == 128, "head_dim");
  constexpr int DPL = D / 32;
  constexpr int TILE = kBlockSize * D * CacheTraits<CT>::bytes;
  constexpr int TC = GT >= 2 ? 32 / GT : 16;  // tokens per reduction chunk
  constexpr int NV = GT * TC;                 // values reduced together (16 or 32)
  constexpr int SHIFT = NV == 32 ? 0 : 1;     // lanes per reduced value = 1 << SHIFT
  constexpr int NCH = kBlockSize / TC;        // chunks per block
  constexpr int GROUP_LANES = 32 / GT;        // lanes holding one head's scores

  extern __shared__ __align__(128) uint8_t smem[];
  constexpr size_t tile_region = 2 * kStages * size_t(TILE);
  constexpr size_t combine_region = size_t(kConsumerWarps) * GT * (D + 2) * sizeof(float);
  constexpr size_t body = tile_region > combine_region ? tile_region : combine_region;
  uint8_t* kbuf = smem;
  uint8_t* vbuf = smem + kStages * TILE;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + body);
  uint64_t* empty = full + kStages;
  float* sp = reinterpret_cast<float*>(empty + kStages);  // [warps][GT][16] probabilities

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seq = blockIdx.x / p.max_parts;
  const int part = blockIdx.x - seq * p.max_parts;
  const int kvh = blockIdx.y / p.head_groups;
  const int hsub = blockIdx.y - kvh * p.head_groups;
  const int head0 = kvh * p.group + hsub * GT;  // first query head of this CTA

  // Sequence length, range-checked against the launch bound and the table width.
  int L = p.seq_lens[seq];
  const int cap = min(p.max_seq_len, p.max_blocks_per_seq * kBlockSize);
  if (L < 0 || L > cap) {
    if (tid == 0 && part == 0 && blockIdx.y == 0) atomicOr(&g_decode_err, PA_DEVERR_SEQ_LEN);
    L = L < 0 ? 0 : cap;
  }
  const int nparts = (L + p.partition - 1) / p.partition;
  if (part >= (nparts > 0 ? nparts : 1)) return;
  if (L == 0) {  // empty context: zero output
    for (int e = tid; e < GT * D; e += kThreads)
      store_out(p.out, (int64_t(seq) * p.num_heads + head0 + e / D) * D + e % D, 0.f,
                p.out_dtype);
    return;
  }
  const int tok_begin = part * p.partition;
  const int tok_end = min(L, tok_begin + p.partition);
  const int blk_begin = tok_begin / kBlockSize;
  const int nblk = (tok_end - tok_begin + kBlockSize - 1) / kBlockSize;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    fence_barrier_init();
  }
  __syncthreads();

  float m_run = -INFINITY, l_part = 0.f;
  float acc[GT][DPL];

  if (warp == kConsumerWarps) {
    // ---------------- producer: block table -> bulk copies ----------------
    const int32_t* table = p.block_tables + int64_t(seq) * p.max_blocks_per_seq + blk_begin;
    const uint64_t policy = l2_policy_evict_first();
    const size_t head_off = size_t(kvh) * TILE;
    const size_t block_stride = size_t(p.num_kv_heads) * TILE;
    int issued = 0;
    bool ok = true;
    for (int base = 0; base < nblk && ok; base += 32) {
      int32_t phys = 0;
      if (base + lane < nblk) {
        phys = table[base + lane];
        if (phys < 0 || phys >= p.num_blocks) {
          atomicOr(&g_decode_err, PA_DEVERR_BLOCK_RANGE);
          phys = 0;
        }
      }
      const int cnt = min(32, nblk - base);
      for (int j = 0; j < cnt; ++j) {
        const int32_t pb = __shfl_sync(kFullMask, phys, j);
        const int i = base + j, stage = i % kStages;
        if (lane == 0) {
          if (i >= kStages && !mbar_wait_bounded(&empty[stage], ((i / kStages) - 1) & 1)) {
            atomicOr(&g_decode_err, PA_DEVERR_PIPE_TIMEOUT);
            ok = false;
          }
          if (ok) {
            mbar_arrive_expect_tx(&full[stage], 2 * TILE);
            const size_t off = size_t(pb) * block_stride + head_off;
            bulk_copy_g2s(kbuf + stage * TILE, p.key_cache + off, TILE, &full[stage], policy);
            bulk_copy_g2s(vbuf + stage * TILE, p.value_cache + off, TILE, &full[stage], policy);
            ++issued;
          }
        }
        ok = __shfl_sync(kFullMask, ok, 0);
        if (!ok) break;
      }
    }
    // Drain: no copy may still be in flight when the CTA leaves or reuses smem.
    if (lane == 0) {
      const int first = issued > kStages ? issued - kStages : 0;
      for (int i = first; i < issued; ++i)
        if (!mbar_wait_bounded(&full[i % kStages], (i / kStages) & 1))
          atomicOr(&g_decode_err, PA_DEVERR_PIPE_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ---------------- consumers ----------------
    float q[GT][DPL];
#pragma unroll
    for (int g = 0; g < GT; ++g) {
      load_q_lane<QT, D>(p.query + (int64_t(seq) * p.num_heads + head0 + g) * D * 2, lane,
                         p.q_mult, q[g]);
#pragma unroll
      for (int i = 0; i < DPL; ++i) acc[g][i] = 0.f;
    }
    const int my_idx = lane >> SHIFT;
    const int my_g = my_idx / TC, my_t = my_idx % TC;
    const bool primary = (lane & ((1 << SHIFT) - 1)) == 0;
    float* wsp = sp + warp * GT * 16;

    for (int i = warp; i < nblk; i += kConsumerWarps) {
      const int stage = i % kStages;
      // every lane waits (acquire); the verdict is made warp-uniform so that no
      // lane can leave the loop while the others still shuffle inside it
      if (!__all_sync(kFullMask, mbar_wait_bounded(&full[stage], (i / kStages) & 1))) {
        if (lane == 0) atomicOr(&g_decode_err, PA_DEVERR_PIPE_TIMEOUT);
        break;
      }
      const uint8_t* kt = kbuf + stage * TILE;
      const uint8_t* vt = vbuf + stage * TILE;
      const int nvalid = min(kBlockSize, tok_end - (blk_begin + i) * kBlockSize);

      float s[NCH];
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        float part_v[NV];
#pragma unroll
        for (int t = 0; t < TC; ++t) {
          float kf[DPL];
          load_lane_row<CT, D>(kt, c * TC + t, lane, kf);
#pragma unroll
          for (int g = 0; g < GT; ++g) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) a = fmaf(q[g][e], kf[e], a);
            part_v[g * TC + t] = a;
          }
        }
        const float sc = transpose_reduce<NV>(part_v, lane);
        s[c] = (c * TC + my_t < nvalid) ? sc : -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < NCH; ++c) mx = fmaxf(mx, s[c]);
#pragma unroll
      for (int o = 1; o < GROUP_LANES; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, o));
      const float m_new = fmaxf(m_run, mx);
      const float alpha = exp2f(m_run - m_new);
      m_run = m_new;
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const float pr = exp2f(s[c] - m_new);
        psum += pr;
        if (primary) wsp[my_g * 16 + c * TC + my_t] = pr;
      }
      l_part = l_part * alpha + (primary ? psum : 0.f);
      float al[GT];
#pragma unroll
      for (int g = 0; g < GT; ++g) al[g] = __shfl_sync(kFullMask, alpha, g * GROUP_LANES);
      __syncwarp();
#pragma unroll
      for (int g = 0; g < GT; ++g)
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[g][e] *= al[g];
#pragma unroll
      for (int t = 0; t < kBlockSize; ++t) {
        if (t < nvalid) {  // never touch rows past the context (they may hold NaN)
          float vf[DPL];
          load_lane_row<CT, D>(vt, t, lane, vf);
#pragma unroll
          for (int g = 0; g < GT; ++g) {
            const float pg = wsp[g * 16 + t];
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[g][e] = fmaf(pg, vf[e], acc[g][e]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
    }
#pragma unroll
    for (int o = 1; o < GROUP_LANES; o <<= 1) l_part += __shfl_xor_sync(kFullMask, l_part, o);
  }

  __syncthreads();  // pipeline finished: the tile region becomes the combine region
  float* cm = reinterpret_cast<float*>(smem);             // [warps][GT]
  float* cl = cm + kConsumerWarps * GT;                    // [warps][GT]
  float* cacc = cl + kConsumerWarps * GT;                  // [warps][GT][D]
  if (warp < kConsumerWarps) {
    if ((lane % GROUP_LANES) == 0) {
      const int g = lane / GROUP_LANES;
      cm[warp * GT + g] = m_run;
      cl[warp * GT + g] = l_part;
    }
#pragma unroll
    for (int g = 0; g < GT; ++g)
#pragma unroll
      for (int e = 0; e < DPL; ++e) cacc[(warp * GT + g) * D + lane * DPL + e] = acc[g][e];
  }
  __syncthreads();
  for (int e = tid; e < GT * D; e += kThreads) {
    const int g = e / D, d = e - g * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, cm[w * GT + g]);
    float Ls = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float mw = cm[w * GT + g];
      if (mw == -INFINITY) continue;  // warp saw no block
      const float f = exp2f(mw - M);
      Ls += cl[w * GT + g] * f;
      O += cacc[(w * GT + g) * D + d] * f;
    }
    const float o = O / Ls * p.v_mult;
    const int64_t row = int64_t(seq) * p.num_heads + head0 + g;
    if (nparts == 1) {
      store_out(p.out, row * D + d, o, p.out_dtype);
    } else {
      const int64_t r = row * p.max_parts + part;
      p.ws_o[r * D + d] = o;
      if (d == 0) {
        p.ws_m[r] = M * kLn2;
        p.ws_l[r] = Ls;
      }
    }
  }
}

// Log-sum-exp merge of the partitions of sequences with more than one:
// M = max m_p, w_p = l_p exp(m_p - M), out = sum w_p o_p / sum w_p.
// grid = num_seqs * num_heads (one CTA per output row), one thread per element.
__global__ void lse_reduce_kernel(void* out, const float* __restrict__ ws_m,
                                  const float* __restrict__ ws_l, const float* __restrict__ ws_o,
                                  const int32_t* __restrict__ seq_lens, int num_heads,
                                  int head_dim, int max_parts, int partition, int cap,
                                  int out_dtype) {
  const int seq = blockIdx.x / num_heads, h = blockIdx.x - seq * num_heads;
  int L = seq_lens[seq];
  L = L < 0 ? 0 : (L > cap ? cap : L);
  const int nparts = (L + partition - 1) / partition;
  if (nparts <= 1) return;  // written by the decode kernel
  const int64_t row = int64_t(seq) * num_heads + h;
  const float* m = ws_m + row * max_parts;
  const float* l = ws_l + row * max_parts;
  float M = -INFINITY;
  for (int q = 0; q < nparts; ++q) M = fmaxf(M, m[q]);
  for (int d = threadIdx.x; d < head_dim; d += blockDim.x) {
    float W = 0.f, O = 0.f;
    for (int q = 0; q < nparts; ++q) {
      const float w = l[q] * exp2f((m[q] - M) * kLog2e);
      W += w;
      O += w * ws_o[(row * max_parts + q) * head_dim + d];
    }
    store_out(out, row * head_dim + d, O / W, out_dtype);
  }
}

template <int D, int GT, typename CT, typename QT>
int launch_typed(const Params& p, int num_seqs, cudaStream_t stream) {
  constexpr size_t smem = smem_bytes<D, GT, CT>();
  auto kern = decode_kernel<D, GT, CT, QT>;
  // The shared-memory opt-in is set once per device and instantiation; a race
  // only repeats an idempotent call.
  static unsigned long long attr_set_mask = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set_mask & bit)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
        cudaSuccess)
      return PA_ERR_CUDA;
    attr_set_mask |= bit;
  }
  const dim3 grid(unsigned(num_seqs) * unsigned(p.max_parts),
                  unsigned(p.num_kv_heads * p.head_groups));
  kern<<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <int D, typename CT, typename QT>
int dispatch_gt(const Params& p, int gt, int num_seqs, cudaStream_t s) {
  switch (gt) {
    case 1: return launch_typed<D, 1, CT, QT>(p, num_seqs, s);
    case 2: return launch_typed<D, 2, CT, QT>(p, num_seqs, s);
    case 4: return launch_typed<D, 4, CT, QT>(p, num_seqs, s);
    case 8: return launch_typed<D, 8, CT, QT>(p, num_seqs, s);
    default: return PA_ERR_UNSUPPORTED;
  }
}

template <typename CT, typename QT>
int dispatch_d(const Params& p, int d, int gt, int num_seqs, cudaStream_t s) {
  if (d == 128) return dispatch_gt<128, CT, QT>(p, gt, num_seqs, s);
  if (d == 64) return dispatch_gt<64, CT, QT>(p, gt, num_seqs, s);
  return PA_ERR_UNSUPPORTED;
}

}  // namespace

int launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  const int group = a.num_heads / a.num_kv_heads;
  const int gt = (group % 8 == 0) ? 8 : (group % 4 == 0) ? 4 : (group % 2 == 0) ? 2 : 1;
  Params p{};
  p.out = a.out;
  p.query = static_cast<const uint8_t*>(a.query);
  p.key_cache = static_cast<const uint8_t*>(a.key_cache);
  p.value_cache = static_cast<const uint8_t*>(a.value_cache);
  p.block_tables = a.block_tables;
  p.seq_lens = a.seq_lens;
  p.max_blocks_per_seq = a.max_blocks_per_seq;
  p.max_seq_len = a.max_seq_len;
  p.num_heads = a.num_heads;
  p.num_kv_heads = a.num_kv_heads;
  p.group = group;
  p.head_groups = group / gt;
  p.partition = a.partition;
  p.max_parts = a.ws.max_parts > 0 ? a.ws.max_parts : 1;
  p.out_dtype = a.out_dtype;
  p.num_blocks = a.num_blocks;
  const bool fp8 = a.cache_dtype == PA_FP8_E4M3;
  p.q_mult = a.scale * kLog2e * (fp8 ? a.k_scale : 1.f);
  p.v_mult = fp8 ? a.v_scale : 1.f;
  if (a.ws.max_parts > 1) {
    uint8_t* w = static_cast<uint8_t*>(a.workspace);
    p.ws_m = reinterpret_cast<float*>(w + a.ws.m_off);
    p.ws_l = reinterpret_cast<float*>(w + a.ws.l_off);
    p.ws_o = reinterpret_cast<float*>(w + a.ws.o_off);
  }
  int rc;
  if (a.cache_dtype == PA_F16 && a.q_dtype == PA_F16)
    rc = dispatch_d<__half, __half>(p, a.head_dim, gt, a.num_seqs, stream);
  else if (a.cache_dtype == PA_BF16 && a.q_dtype == PA_BF16)
    rc = dispatch_d<__nv_bfloat16, __nv_bfloat16>(p, a.head_dim, gt, a.num_seqs, stream);
  else if (fp8 && a.q_dtype == PA_F16)
    rc = dispatch_d<fp8_e4m3, __half>(p, a.head_dim, gt, a.num_seqs, stream);
  else if (fp8 && a.q_dtype == PA_BF16)
    rc = dispatch_d<fp8_e4m3, __nv_bfloat16>(p, a.head_dim, gt, a.num_seqs, stream);
  else
    rc = PA_ERR_UNSUPPORTED;
  if (rc != PA_OK || a.ws.max_parts <= 1) return rc;
  const int cap = a.max_seq_len < a.max_blocks_per_seq * kBlockSize
                      ? a.max_seq_len
                      : a.max_blocks_per_seq * kBlockSize;
  lse_reduce_kernel<<<unsigned(a.num_seqs) * unsigned(a.num_heads), a.head_dim, 0, stream>>>(
      a.out, p.ws_m, p.ws_l, p.ws_o, a.seq_lens, a.num_heads, a.head_dim, p.max_parts,
      a.partition, cap, a.out_dtype);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

cudaError_t read_and_clear_decode_errors(unsigned* bits, cudaStream_t stream) {
  unsigned v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_decode_err, sizeof v, 0,
                                            cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  const unsigned zero = 0;
  e = cudaMemcpyToSymbolAsync(g_decode_err, &zero, sizeof zero, 0, cudaMemcpyHostToDevice,
                              stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  *bits |= v;
  return e;
}

}  // namespace pa
