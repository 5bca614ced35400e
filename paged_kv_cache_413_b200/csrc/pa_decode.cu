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

#include "pa_kernels.cuh"

namespace pa {
namespace {

__device__ unsigned int g_decode_err;

// Ring depths.  Block i goes to stage i % stages and to consumer warp i % 4, so a
// stage count that is a multiple of the warp count gives every stage a single
// owning warp.  That matters: a parity wait cannot tell phase k from phase k - 2,
// so a warp must never wait on a stage whose previous phase another warp is still
// filling or reading.
#ifndef PA_MMA16_STAGES
#define PA_MMA16_STAGES 4
#endif
#ifndef PA_SIMT_STAGES
#define PA_SIMT_STAGES 4
#endif
constexpr int kStagesSimt = PA_SIMT_STAGES;     // 8 KB K+V per stage at D = 128, 16-bit;
                                                // 4 stages: 6 CTAs per SM
constexpr int kStagesMma16 = PA_MMA16_STAGES;   // 8 KB per stage; 4 CTAs per SM
constexpr int kStagesMmaFp8 = 8;                // 4 KB per stage
static_assert(kStagesSimt % kConsumerWarps == 0 && kStagesMma16 % kConsumerWarps == 0 &&
                  kStagesMmaFp8 % kConsumerWarps == 0,
              "each ring stage must belong to one consumer warp");

// ---------------------------------------------------------------------------
// Work order.  CTAs start roughly in linear block order, so handing out the
// longest sequences first (list scheduling, longest first) leaves the shortest
// units for the tail of the launch instead of whichever sequence came last.  The
// linear block index b is split into a rank (b / units per sequence), a partition
// and a (kv head, head group).  With p.lpt the sequence of a rank comes from a
// ranking of seq_lens by length in kLptBuckets buckets of 16-token tiles (longest
// first, ties by index), computed by one warp from one read of seq_lens; the
// launcher sets p.lpt only where that costs less than the tail it removes (long
// units, at most kLptMaxSeqs sequences).  Otherwise rank = sequence.
// ---------------------------------------------------------------------------
#ifndef PA_DECODE_LPT
#define PA_DECODE_LPT 1
#endif
constexpr int kLptBuckets = 256;
constexpr int kLptMaxSeqs = 256;      // lengths held in registers: 8 per lane
constexpr int kLptMinTokens = 1024;   // shortest unit (tokens) worth the ranking

struct LptScratch {
  int start[kLptBuckets];  // counts, then exclusive start offsets, per bucket
  int seq;
};

// Every thread of the CTA calls this once, before any role split.
__device__ __forceinline__ void decode_unit(const Params& p, LptScratch& sc, int& seq, int& part,
                                            int& hg) {
  const int HG = p.num_kv_heads * p.head_groups;
  const int64_t b = int64_t(blockIdx.y) * gridDim.x + blockIdx.x;
  const int per_seq = p.max_parts * HG;
  const int rank = int(b / per_seq);
  const int rem = int(b - int64_t(rank) * per_seq);
  part = rem / HG;
  hg = rem - part * HG;
  seq = rank;
#if PA_DECODE_LPT
  if (!p.lpt) return;  // uniform over the grid
  constexpr int kPer = kLptMaxSeqs / 32;
  static_assert(kLptBuckets == 32 * kPer, "one scan slice of buckets per lane");
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x, n = p.num_seqs;
    const int cap = p.cap;
    const int max_tiles = max(1, (cap + kBlockSize - 1) / kBlockSize);
    int bk[kPer];  // bucket of sequence lane + 32 k (0 = longest), -1 past the batch
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int i = lane + 32 * k;
      int L = i < n ? p.seq_lens[i] : 0;
      L = L < 0 ? 0 : (L > cap ? cap : L);
      const int tiles = (L + kBlockSize - 1) / kBlockSize;
      bk[k] = i < n ? (kLptBuckets - 1) - int(int64_t(tiles) * (kLptBuckets - 1) / max_tiles)
                    : -1;
      sc.start[lane * kPer + k] = 0;
    }
    __syncwarp();
#pragma unroll
    for (int k = 0; k < kPer; ++k)
      if (bk[k] >= 0) atomicAdd(&sc.start[bk[k]], 1);
    __syncwarp();
    // exclusive scan of the counts; this lane's buckets [kPer lane, kPer lane + kPer)
    int v[kPer], sum = 0;
#pragma unroll
    for (int k = 0; k < kPer; ++k) sum += (v[k] = sc.start[lane * kPer + k]);
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(kFullMask, incl, o);
      if (lane >= o) incl += t;
    }
    // the bucket holding `rank`, and rank's place inside it
    int run = incl - sum, kk = -1, j = 0;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      if (run <= rank && rank < run + v[k]) {
        kk = lane * kPer + k;
        j = rank - run;
      }
      run += v[k];
    }
    const unsigned own = __ballot_sync(kFullMask, kk >= 0);
    const int src = __ffs(own) - 1;  // exactly one lane holds it
    kk = __shfl_sync(kFullMask, kk, src);
    j = __shfl_sync(kFullMask, j, src);
    // the j-th sequence, by index, in bucket kk
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const unsigned bal = __ballot_sync(kFullMask, bk[k] == kk);
      const int c = __popc(bal);
      if (j < c) {
        if (bk[k] == kk && __popc(bal & ((1u << lane) - 1u)) == j) sc.seq = lane + 32 * k;
        break;
      }
      j -= c;
    }
  }
  __syncthreads();
  seq = sc.seq;
#endif
}

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

// Merge the consumer warps' softmax states (cm: max in log2 units, cl: sum,
// cacc: unnormalised accumulators, all in shared memory) and store the result:
// the output itself when the sequence has one partition, else this partition's
// (m, l, o) for the log-sum-exp reduce.  The per-head factors are computed once
// (cf: the weight of each warp divided by the total) before the element loop.
template <int D, int GT>
__device__ __forceinline__ void combine_and_store(const float* cm, const float* cl,
                                                  const float* cacc, float* cf, const Params& p,
                                                  int seq, int part, int head0, int nparts) {
  constexpr int R = combine_row<D>();
  if (threadIdx.x < GT) {
    const int g = threadIdx.x;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, cm[w * GT + g]);
    float f[kConsumerWarps];
    float Ls = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float mw = cm[w * GT + g];
      f[w] = mw == -INFINITY ? 0.f : exp2f(mw - M);  // a warp that saw no block weighs 0
      Ls += cl[w * GT + g] * f[w];
    }
    const float inv = p.v_mult / Ls;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) cf[g * (kConsumerWarps + 1) + w] = f[w] * inv;
    cf[g * (kConsumerWarps + 1) + kConsumerWarps] = Ls;
    if (nparts > 1) {
      const int64_t r = (int64_t(seq) * p.num_heads + head0 + g) * p.max_parts + part;
      p.ws_m[r] = M * kLn2;
      p.ws_l[r] = Ls;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < GT * D; e += kThreads) {
    const int g = e / D, d = e - g * D;
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w)
      o = fmaf(cacc[(w * GT + g) * R + d], cf[g * (kConsumerWarps + 1) + w], o);
    const int64_t row = int64_t(seq) * p.num_heads + head0 + g;
    if (nparts == 1)
      store_out(p.out, row * D + d, o, p.out_dtype);
    else
      p.ws_o[(row * p.max_parts + part) * D + d] = o;
  }
}

template <int D, int GT, typename CT, int S>
constexpr size_t smem_bytes() {
  constexpr size_t tile = size_t(kBlockSize) * D * CacheTraits<CT>::bytes;
  constexpr size_t pipe = 2 * S * tile;
  constexpr size_t combine = combine_bytes<D, GT>();
  constexpr size_t body = pipe > combine ? pipe : combine;
  return body + 2 * S * sizeof(uint64_t) + size_t(kConsumerWarps) * GT * 16 * sizeof(float);
}

// GT: query heads served by one CTA (a divisor of the GQA group, at most 8).
template <int D, int GT, typename CT, typename QT, int kStages>
__global__ void __launch_bounds__(kThreads) decode_kernel(const Params p) {
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(kStages % kConsumerWarps == 0, "each ring stage must belong to one warp");
  constexpr int DPL = D / 32;
  constexpr int TILE = kBlockSize * D * CacheTraits<CT>::bytes;
  constexpr int TC = GT >= 2 ? 32 / GT : 16;  // tokens per reduction chunk
  constexpr int NV = GT * TC;                 // values reduced together (16 or 32)
  constexpr int SHIFT = NV == 32 ? 0 : 1;     // lanes per reduced value = 1 << SHIFT
  constexpr int NCH = kBlockSize / TC;        // chunks per block
  constexpr int GROUP_LANES = 32 / GT;        // lanes holding one head's scores
  grid_dependency_wait();  // launched as a programmatic dependent

  extern __shared__ __align__(128) uint8_t smem[];
  constexpr size_t tile_region = 2 * kStages * size_t(TILE);
  constexpr size_t combine_region = combine_bytes<D, GT>();
  constexpr size_t body = tile_region > combine_region ? tile_region : combine_region;
  uint8_t* kbuf = smem;
  uint8_t* vbuf = smem + kStages * TILE;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + body);
  uint64_t* empty = full + kStages;
  float* sp = reinterpret_cast<float*>(empty + kStages);  // [warps][GT][16] probabilities

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __shared__ LptScratch lpt;
  int seq, part, hg;
  decode_unit(p, lpt, seq, part, hg);
  const int kvh = hg / p.head_groups;
  const int hsub = hg - kvh * p.head_groups;
  const int head0 = kvh * p.group + hsub * GT;  // first query head of this CTA

  // The producer starts the first block-table read before anything else; the row
  // has max_blocks_per_seq entries, so the speculative read stays inside it.
  const int32_t* table_row = p.block_tables + int64_t(seq) * p.max_blocks_per_seq;
  const int blk_begin = part * (p.partition / kBlockSize);
  int32_t phys_first = 0;
  if (warp == kConsumerWarps && (blk_begin + lane) / p.tiles_per_block < p.max_blocks_per_seq)
    phys_first = table_row[(blk_begin + lane) / p.tiles_per_block];
  // Sequence length, range-checked against the launch bound and the table width.
  int L = p.seq_lens[seq];
  const int cap = p.cap;
  if (L < 0 || L > cap) {
    if (tid == 0 && part == 0 && hg == 0) atomicOr(&g_decode_err, PA_DEVERR_SEQ_LEN);
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
    const uint64_t policy = l2_policy_evict_first();
    int issued = 0;
    bool ok = true;
    for (int base = 0; base < nblk && ok; base += 32) {
      // 16-token tile t of the sequence lives in block table_row[t / R] at sub-tile
      // t % R; its index in the pool viewed as [blocks][kv_heads][R] tiles:
      int tile = 0;
      if (base + lane < nblk) {
        const int t = blk_begin + base + lane, e = t / p.tiles_per_block;
        int32_t phys = base == 0 ? phys_first : table_row[e];
        if (phys < 0 || phys >= p.num_blocks) {
          atomicOr(&g_decode_err, PA_DEVERR_BLOCK_RANGE);
          phys = 0;
        }
        tile = (phys * p.num_kv_heads + kvh) * p.tiles_per_block + (t - e * p.tiles_per_block);
      }
      const int cnt = min(32, nblk - base);
      for (int j = 0; j < cnt; ++j) {
        const int tl = __shfl_sync(kFullMask, tile, j);
        const int i = base + j, stage = i % kStages;
        if (lane == 0) {
          if (i >= kStages && !mbar_wait_bounded(&empty[stage], ((i / kStages) - 1) & 1)) {
            atomicOr(&g_decode_err, PA_DEVERR_PIPE_TIMEOUT);
            ok = false;
          }
          if (ok) {
#ifdef PA_TEST_STALL_TILE
            // Failure-detection test build only: tile PA_TEST_STALL_TILE of every CTA
            // is neither announced nor copied, so its stage's phase never completes
            // and every wait on it must give up and report PA_DEVERR_PIPE_TIMEOUT.
            if (i != PA_TEST_STALL_TILE)
#endif
            {
              mbar_arrive_expect_tx(&full[stage], 2 * TILE);
              const size_t off = size_t(tl) * TILE;
              bulk_copy_g2s(kbuf + stage * TILE, p.key_cache + off, TILE, &full[stage], policy);
              bulk_copy_g2s(vbuf + stage * TILE, p.value_cache + off, TILE, &full[stage], policy);
            }
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
  constexpr int R = combine_row<D>();
  float* cm = reinterpret_cast<float*>(smem);             // [warps][GT]
  float* cl = cm + kConsumerWarps * GT;                    // [warps][GT]
  float* cacc = cl + kConsumerWarps * GT;                  // [warps][GT][R]
  float* cf = cacc + kConsumerWarps * GT * R;              // [GT][warps + 1]
  if (warp < kConsumerWarps) {
    if ((lane % GROUP_LANES) == 0) {
      const int g = lane / GROUP_LANES;
      cm[warp * GT + g] = m_run;
      cl[warp * GT + g] = l_part;
    }
#pragma unroll
    for (int g = 0; g < GT; ++g)
#pragma unroll
      for (int e = 0; e < DPL; ++e) cacc[(warp * GT + g) * R + lane * DPL + e] = acc[g][e];
  }
  __syncthreads();
  combine_and_store<D, GT>(cm, cl, cacc, cf, p, seq, part, head0, nparts);
  // let the merge kernel (launched as a programmatic dependent) get scheduled
  grid_dependents_may_launch();
}

// ---------------------------------------------------------------------------
// Tensor-core consumer for GQA groups of 4 or 8 query heads (head_dim 128).
//
// Per 16-token block the two contractions are warp-level MMAs (m16n8k16, fp32
// accumulate):  S^T[16 tokens x 8 heads] = K[16 x 128] . Q^T[128 x 8]  and
// O^T[128 x 8] += V^T[128 x 16] . P^T[16 x 8].  The GQA heads are the N side,
// so a group of 8 fills the instruction; P^T comes from the S^T accumulator by
// an in-register 8x8 transpose (movmatrix).  Softmax stays fp32.  K/V blocks are
// staged by tiled TMA with the 128-byte swizzle so that every ldmatrix is free
// of bank conflicts.  For bf16, P is split into bf16 hi + lo parts (two MMAs)
// so the probabilities keep ~16 significant bits.  E4M3 caches are widened to
// f16 exactly in registers; a bf16 query is then scaled by a power of two into
// f16 range (undone in the score multiplier).
// ---------------------------------------------------------------------------
struct TmaParams {
  CUtensorMap tmk;  // K pool as [rows = blocks * kv_heads * 16][128] elements
  CUtensorMap tmv;  // V pool, same view
  Params p;
};

template <typename CT, int kStages>
constexpr size_t mma_smem_bytes() {
  constexpr size_t tile = size_t(kBlockSize) * 128 * CacheTraits<CT>::bytes;
  constexpr size_t pipe = 2 * kStages * tile;
  constexpr size_t combine = combine_bytes<128, 8>();
  constexpr size_t body = pipe > combine ? pipe : combine;
  return 1024 + body + 2 * kStages * sizeof(uint64_t);
}

template <int GT, typename CT, typename QT, int kStages>
// Resident CTAs per SM the register budget must allow: 5 for groups of 8 (a few
// L1-cached spills; 0.903-0.910 -> 0.920 on the 70B-GQA workload), 4 for groups of
// 4, where 5 measured slightly slower.
#ifndef PA_MMA8_MIN_CTAS
#define PA_MMA8_MIN_CTAS 5  // 6 (64 registers, more spills) measured 0.82
#endif
__global__ void __launch_bounds__(kThreads, GT == 8 ? PA_MMA8_MIN_CTAS : 4) decode_mma_kernel(
    const __grid_constant__ TmaParams tp) {
  constexpr int D = 128;
  constexpr bool kFp8 = CacheTraits<CT>::bytes == 1;
  constexpr int TILE = kBlockSize * D * CacheTraits<CT>::bytes;
  using MT = typename std::conditional<kFp8, __half, CT>::type;  // MMA element type
  constexpr bool kSplitP = std::is_same<MT, __nv_bfloat16>::value;
  static_assert(GT == 4 || GT == 8, "heads per CTA");
  static_assert(kStages % kConsumerWarps == 0, "each ring stage must belong to one warp");
  const Params& p = tp.p;
  grid_dependency_wait();  // launched as a programmatic dependent

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  constexpr size_t tile_region = 2 * kStages * size_t(TILE);
  constexpr size_t combine_region = combine_bytes<D, GT>();
  constexpr size_t body = tile_region > combine_region ? tile_region : combine_region;
  uint8_t* kbuf = smem;
  uint8_t* vbuf = smem + kStages * TILE;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + body);
  uint64_t* empty = full + kStages;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __shared__ LptScratch lpt;
  int seq, part, hg;
  decode_unit(p, lpt, seq, part, hg);
  const int kvh = hg / p.head_groups;
  const int hsub = hg - kvh * p.head_groups;
  const int head0 = kvh * p.group + hsub * GT;

  const int32_t* table_row = p.block_tables + int64_t(seq) * p.max_blocks_per_seq;
  const int blk_begin = part * (p.partition / kBlockSize);
  int32_t phys_first = 0;
  if (warp == kConsumerWarps && (blk_begin + lane) / p.tiles_per_block < p.max_blocks_per_seq)
    phys_first = table_row[(blk_begin + lane) / p.tiles_per_block];
  int L = p.seq_lens[seq];
  const int cap = p.cap;
  if (L < 0 || L > cap) {
    if (tid == 0 && part == 0 && hg == 0) atomicOr(&g_decode_err, PA_DEVERR_SEQ_LEN);
    L = L < 0 ? 0 : cap;
  }
  const int nparts = (L + p.partition - 1) / p.partition;
  if (part >= (nparts > 0 ? nparts : 1)) return;
  if (L == 0) {
    for (int e = tid; e < GT * D; e += kThreads)
      store_out(p.out, (int64_t(seq) * p.num_heads + head0 + e / D) * D + e % D, 0.f,
                p.out_dtype);
    return;
  }
  const int tok_begin = part * p.partition;
  const int tok_end = min(L, tok_begin + p.partition);
  const int nblk = (tok_end - tok_begin + kBlockSize - 1) / kBlockSize;

  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);
    }
    fence_barrier_init();
  }
  __syncthreads();

  float acc[8][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int g = lane >> 2, c = lane & 3;   // fragment row group / column pair
  const int mi = lane >> 3, r = lane & 7;  // ldmatrix: matrix index / row

  if (warp == kConsumerWarps) {
    // ---------------- producer: block table -> tiled TMA loads ----------------
    const uint64_t policy = l2_policy_evict_first();
    int issued = 0;
    bool ok = true;
    for (int base = 0; base < nblk && ok; base += 32) {
      // 16-token tile t of the sequence lives in block table_row[t / R] at sub-tile
      // t % R; its index in the pool viewed as [blocks][kv_heads][R] tiles:
      int tile = 0;
      if (base + lane < nblk) {
        const int t = blk_begin + base + lane, e = t / p.tiles_per_block;
        int32_t phys = base == 0 ? phys_first : table_row[e];
        if (phys < 0 || phys >= p.num_blocks) {
          atomicOr(&g_decode_err, PA_DEVERR_BLOCK_RANGE);
          phys = 0;
        }
        tile = (phys * p.num_kv_heads + kvh) * p.tiles_per_block + (t - e * p.tiles_per_block);
      }
      const int cnt = min(32, nblk - base);
      for (int j = 0; j < cnt; ++j) {
        const int tl = __shfl_sync(kFullMask, tile, j);
        const int i = base + j, stage = i % kStages;
        if (lane == 0) {
          if (i >= kStages && !mbar_wait_bounded(&empty[stage], ((i / kStages) - 1) & 1)) {
            atomicOr(&g_decode_err, PA_DEVERR_PIPE_TIMEOUT);
            ok = false;
          }
          if (ok) {
            const int row = tl * kBlockSize;
            uint8_t* kd = kbuf + stage * TILE;
            uint8_t* vd = vbuf + stage * TILE;
            mbar_arrive_expect_tx(&full[stage], 2 * TILE);
            if constexpr (kFp8) {
              tma_load_2d(kd, &tp.tmk, 0, row, &full[stage], policy);
              tma_load_2d(vd, &tp.tmv, 0, row, &full[stage], policy);
            } else {
              tma_load_2d(kd, &tp.tmk, 0, row, &full[stage], policy);
              tma_load_2d(kd + TILE / 2, &tp.tmk, 64, row, &full[stage], policy);
              tma_load_2d(vd, &tp.tmv, 0, row, &full[stage], policy);
              tma_load_2d(vd + TILE / 2, &tp.tmv, 64, row, &full[stage], policy);
            }
            ++issued;
          }
        }
        ok = __shfl_sync(kFullMask, ok, 0);
        if (!ok) break;
      }
    }
    if (lane == 0) {
      const int first = issued > kStages ? issued - kStages : 0;
      for (int i = first; i < issued; ++i)
        if (!mbar_wait_bounded(&full[i % kStages], (i / kStages) & 1))
          atomicOr(&g_decode_err, PA_DEVERR_PIPE_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ---------------- consumers ----------------
    // Q^T as the B operand, one fragment pair per 16-wide k-step.  Heads past
    // the group (GT = 4) are zero columns.
    uint32_t qb[8][2];
    float mult = p.q_mult;
    const uint8_t* qrow = p.query + (int64_t(seq) * p.num_heads + head0 + (g < GT ? g : 0)) * D * 2;
    if constexpr (!kFp8) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        qb[ks][0] = g < GT ? *reinterpret_cast<const uint32_t*>(qrow + (16 * ks + 2 * c) * 2) : 0u;
        qb[ks][1] = g < GT ? *reinterpret_cast<const uint32_t*>(qrow + (16 * ks + 2 * c + 8) * 2) : 0u;
      }
    } else {
      // k-step ks covers dims 16 ks + 4c .. 4c+3 for this thread (see the K loads)
      uint2 raw[8];
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        raw[ks] = g < GT ? *reinterpret_cast<const uint2*>(qrow + (16 * ks + 4 * c) * 2)
                         : make_uint2(0u, 0u);
      if constexpr (std::is_same<QT, __half>::value) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          qb[ks][0] = raw[ks].x;
          qb[ks][1] = raw[ks].y;
        }
      } else {
        // bf16 -> f16: scale by 2^sq so that the largest |q| of the group lands in
        // [2^14, 2^15); the scores are multiplied back by 2^-sq.
        float qmax = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const float2 a = unpack2(raw[ks].x, QT{}), b = unpack2(raw[ks].y, QT{});
          qmax = fmaxf(qmax, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(b.x), fabsf(b.y))));
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) qmax = fmaxf(qmax, __shfl_xor_sync(kFullMask, qmax, o));
        int e = 0;
        if (qmax > 0.f && isfinite(qmax)) frexpf(qmax, &e);
        const int sq = min(max(15 - e, -100), 100);
        mult = ldexpf(mult, -sq);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const float2 a = unpack2(raw[ks].x, QT{}), b = unpack2(raw[ks].y, QT{});
          qb[ks][0] = pack2(ldexpf(a.x, sq), ldexpf(a.y, sq), __half{});
          qb[ks][1] = pack2(ldexpf(b.x, sq), ldexpf(b.y, sq), __half{});
        }
      }
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;

    for (int i = warp; i < nblk; i += kConsumerWarps) {
      const int stage = i % kStages;
      if (!__all_sync(kFullMask, mbar_wait_bounded(&full[stage], (i / kStages) & 1))) {
        if (lane == 0) atomicOr(&g_decode_err, PA_DEVERR_PIPE_TIMEOUT);
        break;
      }
      const uint32_t kt = smem_u32(kbuf + stage * TILE);
      const uint32_t vt = smem_u32(vbuf + stage * TILE);
      const int nvalid = min(kBlockSize, tok_end - (blk_begin + i) * kBlockSize);

      // ---- S^T = K . Q^T ----
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (!kFp8) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const int tok = r + 8 * (mi & 1), j = 2 * ks + (mi >> 1);
          uint32_t a[4];
          ldsm_x4(kt + (j >> 3) * (TILE / 2) + tok * 128 + (((j & 7) ^ r) << 4), a);
          mma_16816(sc, a, qb[ks][0], qb[ks][1], MT{});
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int tok = r + 8 * (mi & 1), j = 2 * u + (mi >> 1);
          uint32_t R[4];
          ldsm_x4(kt + tok * 128 + ((j ^ r) << 4), R);
          const uint32_t a0[4] = {e4m3x2_to_f16x2(R[0]), e4m3x2_to_f16x2(R[1]),
                                  e4m3x2_to_f16x2(R[0] >> 16), e4m3x2_to_f16x2(R[1] >> 16)};
          const uint32_t a1[4] = {e4m3x2_to_f16x2(R[2]), e4m3x2_to_f16x2(R[3]),
                                  e4m3x2_to_f16x2(R[2] >> 16), e4m3x2_to_f16x2(R[3] >> 16)};
          mma_16816(sc, a0, qb[2 * u][0], qb[2 * u][1], MT{});
          mma_16816(sc, a1, qb[2 * u + 1][0], qb[2 * u + 1][1], MT{});
        }
      }
      // sc = {S(g, 2c), S(g, 2c+1), S(g+8, 2c), S(g+8, 2c+1)} in log2 units
      const bool v0 = g < nvalid, v8 = g + 8 < nvalid;  // rows past the context -> -inf
      sc[0] = v0 ? sc[0] * mult : -INFINITY;
      sc[1] = v0 ? sc[1] * mult : -INFINITY;
      sc[2] = v8 ? sc[2] * mult : -INFINITY;
      sc[3] = v8 ? sc[3] * mult : -INFINITY;
      float mx0 = fmaxf(sc[0], sc[2]), mx1 = fmaxf(sc[1], sc[3]);
#pragma unroll
      for (int o = 4; o <= 16; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFullMask, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFullMask, mx1, o));
      }
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      const float p0 = exp2f(sc[0] - mn0), p1 = exp2f(sc[1] - mn1);
      const float p2 = exp2f(sc[2] - mn0), p3 = exp2f(sc[3] - mn1);
      l0 = l0 * al0 + (p0 + p2);
      l1 = l1 * al1 + (p1 + p3);
      // P^T fragments: the accumulator layout of S^T is an m8n8 fragment per 8
      // tokens; its transpose is the B operand of the P.V product.
      const uint32_t x0 = pack2(p0, p1, MT{}), x1 = pack2(p2, p3, MT{});
      const uint32_t bh0 = movmatrix_trans(x0), bh1 = movmatrix_trans(x1);
      uint32_t bl0 = 0, bl1 = 0;
      if constexpr (kSplitP) {
        const float2 h0 = unpack2(x0, MT{}), h1 = unpack2(x1, MT{});
        bl0 = movmatrix_trans(pack2(p0 - h0.x, p1 - h0.y, MT{}));
        bl1 = movmatrix_trans(pack2(p2 - h1.x, p3 - h1.y, MT{}));
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        acc[t][0] *= al0;
        acc[t][1] *= al1;
        acc[t][2] *= al0;
        acc[t][3] *= al1;
      }
      // zero V rows past the context: they may hold anything, even NaN
      uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
      if (nvalid < kBlockSize) {
        mlo = (2 * c < nvalid ? 0x0000ffffu : 0u) | (2 * c + 1 < nvalid ? 0xffff0000u : 0u);
        mhi = (2 * c + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * c + 9 < nvalid ? 0xffff0000u : 0u);
      }
      // ---- O^T += V^T . P^T ----
      if constexpr (!kFp8) {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int tok = r + 8 * (mi >> 1), j = 2 * t + (mi & 1);
          uint32_t a[4];
          ldsm_x4_trans(vt + (j >> 3) * (TILE / 2) + tok * 128 + (((j & 7) ^ r) << 4), a);
          a[0] &= mlo;
          a[1] &= mlo;
          a[2] &= mhi;
          a[3] &= mhi;
          mma_16816(acc[t], a, bh0, bh1, MT{});
          if constexpr (kSplitP) mma_16816(acc[t], a, bl0, bl1, MT{});
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int tok = r + 8 * (mi & 1), j = 2 * u + (mi >> 1);
          uint32_t R[4];
          ldsm_x4_trans(vt + tok * 128 + ((j ^ r) << 4), R);
          // R[q] bytes: (token 2c, dim d), (2c, d+1), (2c+1, d), (2c+1, d+1), d = 16 chunk + 2g
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t lo = R[2 * h], hi8 = R[2 * h + 1];
            uint32_t a[4] = {e4m3x2_to_f16x2(__byte_perm(lo, 0, 0x20)) & mlo,
                             e4m3x2_to_f16x2(__byte_perm(lo, 0, 0x31)) & mlo,
                             e4m3x2_to_f16x2(__byte_perm(hi8, 0, 0x20)) & mhi,
                             e4m3x2_to_f16x2(__byte_perm(hi8, 0, 0x31)) & mhi};
            mma_16816(acc[2 * u + h], a, bh0, bh1, MT{});
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
    }
#pragma unroll
    for (int o = 4; o <= 16; o <<= 1) {
      l0 += __shfl_xor_sync(kFullMask, l0, o);
      l1 += __shfl_xor_sync(kFullMask, l1, o);
    }
  }

  __syncthreads();  // pipeline finished: the tile region becomes the combine region
  constexpr int R = combine_row<D>();
  float* cm = reinterpret_cast<float*>(smem);
  float* cl = cm + kConsumerWarps * GT;
  float* cacc = cl + kConsumerWarps * GT;
  float* cf = cacc + kConsumerWarps * GT * R;
  if (warp < kConsumerWarps) {
    if (g == 0) {
      if (2 * c < GT) {
        cm[warp * GT + 2 * c] = m0;
        cl[warp * GT + 2 * c] = l0;
      }
      if (2 * c + 1 < GT) {
        cm[warp * GT + 2 * c + 1] = m1;
        cl[warp * GT + 2 * c + 1] = l1;
      }
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      // rows of the O^T fragment -> head dims
      const int d0 = kFp8 ? 16 * t + 2 * g : 16 * t + g;
      const int d1 = kFp8 ? d0 + 1 : d0 + 8;
      if (2 * c < GT) {
        cacc[(warp * GT + 2 * c) * R + d0] = acc[t][0];
        cacc[(warp * GT + 2 * c) * R + d1] = acc[t][2];
      }
      if (2 * c + 1 < GT) {
        cacc[(warp * GT + 2 * c + 1) * R + d0] = acc[t][1];
        cacc[(warp * GT + 2 * c + 1) * R + d1] = acc[t][3];
      }
    }
  }
  __syncthreads();
  combine_and_store<D, GT>(cm, cl, cacc, cf, p, seq, part, head0, nparts);
  // let the merge kernel (launched as a programmatic dependent) get scheduled
  grid_dependents_may_launch();
}

// Log-sum-exp merge of the partitions of sequences with more than one:
// M = max m_p, w_p = l_p exp(m_p - M), out = sum w_p o_p / sum w_p.
// One CTA of kReduceWarps warps per (sequence, head) row.  Warp w takes the
// partitions p = w, w + kReduceWarps, ..., four at a time with their loads in
// flight together; lanes own D/32 dims; the warps' sums meet in shared memory.
// Launched as a programmatic dependent of the decode kernel: it waits for that
// grid's results before reading the workspace.
constexpr int kReduceWarps = 4;

template <int D>
__global__ void __launch_bounds__(kReduceWarps * 32) lse_reduce_kernel(
    void* out, const float* __restrict__ ws_m, const float* __restrict__ ws_l,
    const float* __restrict__ ws_o, const int32_t* __restrict__ seq_lens, int num_rows,
    int num_heads, int max_parts, int partition, int cap, int out_dtype) {
  grid_dependency_wait();
  constexpr int DPL = D / 32;
  __shared__ float s_max[kReduceWarps];
  __shared__ float s_acc[kReduceWarps][D];
  __shared__ float s_w[kReduceWarps];
  const int row = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (row >= num_rows) return;
  int L = seq_lens[row / num_heads];
  L = L < 0 ? 0 : (L > cap ? cap : L);
  const int nparts = (L + partition - 1) / partition;
  if (nparts <= 1) return;  // written by the decode kernel (uniform over the CTA)
  const float* m = ws_m + int64_t(row) * max_parts;
  const float* l = ws_l + int64_t(row) * max_parts;
  const float* o = ws_o + int64_t(row) * max_parts * D + lane * DPL;
  float M = -INFINITY;
  for (int q = threadIdx.x; q < nparts; q += kReduceWarps * 32) M = fmaxf(M, m[q]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFullMask, M, off));
  if (lane == 0) s_max[warp] = M;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kReduceWarps; ++w) M = fmaxf(M, s_max[w]);
  float acc[DPL] = {};
  float W = 0.f;
  int q = warp;
  for (; q + 3 * kReduceWarps < nparts; q += 4 * kReduceWarps) {
    float w4[4];
    float v4[4][DPL];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int qq = q + u * kReduceWarps;
      w4[u] = l[qq] * exp2f((m[qq] - M) * kLog2e);
#pragma unroll
      for (int e = 0; e < DPL; ++e) v4[u][e] = o[int64_t(qq) * D + e];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      W += w4[u];
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(w4[u], v4[u][e], acc[e]);
    }
  }
  for (; q < nparts; q += kReduceWarps) {
    const float w = l[q] * exp2f((m[q] - M) * kLog2e);
    W += w;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = fmaf(w, o[int64_t(q) * D + e], acc[e]);
  }
#pragma unroll
  for (int e = 0; e < DPL; ++e) s_acc[warp][lane * DPL + e] = acc[e];
  if (lane == 0) s_w[warp] = W;
  __syncthreads();
  if (warp == 0) {
    float Wt = 0.f;
#pragma unroll
    for (int w = 0; w < kReduceWarps; ++w) Wt += s_w[w];
    const float inv = 1.f / Wt;
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
      float t = 0.f;
#pragma unroll
      for (int w = 0; w < kReduceWarps; ++w) t += s_acc[w][lane * DPL + e];
      store_out(out, int64_t(row) * D + lane * DPL + e, t * inv, out_dtype);
    }
  }
}

template <int D, int GT, typename CT, typename QT>
int launch_typed(const Params& p, int num_seqs, cudaStream_t stream) {
  constexpr size_t smem = smem_bytes<D, GT, CT, kStagesSimt>();
  auto kern = decode_kernel<D, GT, CT, QT, kStagesSimt>;
  static std::atomic<unsigned long long> smem_set{0};
  if (set_smem_once(kern, smem, smem_set) != PA_OK) return PA_ERR_CUDA;
  const dim3 grid(unsigned(num_seqs) * unsigned(p.max_parts),
                  unsigned(p.num_kv_heads * p.head_groups));
  const cudaError_t e = launch_dependent(kern, grid, dim3(kThreads), smem, stream, p);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
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

template <int GT, typename CT, typename QT>
int launch_mma_typed(const Params& p, const void* kc, const void* vc, int64_t rows, int num_seqs,
                     cudaStream_t stream) {
  constexpr bool fp8 = CacheTraits<CT>::bytes == 1;
  constexpr int stages = fp8 ? kStagesMmaFp8 : kStagesMma16;
  constexpr size_t smem = mma_smem_bytes<CT, stages>();
  auto kern = decode_mma_kernel<GT, CT, QT, stages>;
  static std::atomic<unsigned long long> smem_set{0};
  if (set_smem_once(kern, smem, smem_set) != PA_OK) return PA_ERR_CUDA;
  TmaParams tp;
  memset(&tp, 0, sizeof tp);
  tp.p = p;
  if (!encode_pool_map(&tp.tmk, kc, rows, fp8) || !encode_pool_map(&tp.tmv, vc, rows, fp8))
    return PA_ERR_CUDA;
  const dim3 grid(unsigned(num_seqs) * unsigned(p.max_parts),
                  unsigned(p.num_kv_heads * p.head_groups));
  const cudaError_t e = launch_dependent(kern, grid, dim3(kThreads), smem, stream, tp);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <typename CT, typename QT>
int dispatch_mma(const Params& p, int gt, const void* kc, const void* vc, int64_t rows,
                 int num_seqs, cudaStream_t s) {
  if (gt == 8) return launch_mma_typed<8, CT, QT>(p, kc, vc, rows, num_seqs, s);
  return launch_mma_typed<4, CT, QT>(p, kc, vc, rows, num_seqs, s);
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
  p.block_size = a.block_size;
  p.tiles_per_block = a.block_size / kBlockSize;
  p.max_seq_len = a.max_seq_len;
  p.cap = context_cap(a.max_seq_len, a.max_blocks_per_seq, a.block_size);
  p.num_heads = a.num_heads;
  p.num_kv_heads = a.num_kv_heads;
  p.group = group;
  p.head_groups = group / gt;
  p.partition = a.partition;
  p.max_parts = a.ws.max_parts > 0 ? a.ws.max_parts : 1;
  p.out_dtype = a.out_dtype;
  p.num_blocks = a.num_blocks;
  p.num_seqs = a.num_seqs;
  p.lpt = a.num_seqs <= kLptMaxSeqs && min(a.partition, a.max_seq_len) >= kLptMinTokens;
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
  const int64_t rows = a.num_blocks * a.num_kv_heads * a.block_size;
  const bool use_mma = a.head_dim == 128 && (gt == 4 || gt == 8) && rows < (int64_t(1) << 31) &&
                       encode_fn() != nullptr;
  if (use_mma) {
    const void* kc = a.key_cache;
    const void* vc = a.value_cache;
    if (a.cache_dtype == PA_F16 && a.q_dtype == PA_F16)
      rc = dispatch_mma<__half, __half>(p, gt, kc, vc, rows, a.num_seqs, stream);
    else if (a.cache_dtype == PA_BF16 && a.q_dtype == PA_BF16)
      rc = dispatch_mma<__nv_bfloat16, __nv_bfloat16>(p, gt, kc, vc, rows, a.num_seqs, stream);
    else if (fp8 && a.q_dtype == PA_F16)
      rc = dispatch_mma<fp8_e4m3, __half>(p, gt, kc, vc, rows, a.num_seqs, stream);
    else if (fp8 && a.q_dtype == PA_BF16)
      rc = dispatch_mma<fp8_e4m3, __nv_bfloat16>(p, gt, kc, vc, rows, a.num_seqs, stream);
    else
      rc = PA_ERR_UNSUPPORTED;
  } else if (a.cache_dtype == PA_F16 && a.q_dtype == PA_F16)
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
  const int cap = p.cap;
  const int out_rows = a.num_seqs * a.num_heads;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(out_rows));
  cfg.blockDim = dim3(kReduceWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float* wm = p.ws_m;
  const float* wl = p.ws_l;
  const float* wo = p.ws_o;
  cudaError_t e;
  if (a.head_dim == 128)
    e = cudaLaunchKernelEx(&cfg, lse_reduce_kernel<128>, a.out, wm, wl, wo, a.seq_lens, out_rows,
                           a.num_heads, p.max_parts, a.partition, cap, int(a.out_dtype));
  else
    e = cudaLaunchKernelEx(&cfg, lse_reduce_kernel<64>, a.out, wm, wl, wo, a.seq_lens, out_rows,
                           a.num_heads, p.max_parts, a.partition, cap, int(a.out_dtype));
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
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
