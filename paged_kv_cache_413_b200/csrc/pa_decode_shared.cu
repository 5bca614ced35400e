// pa_decode_shared.cu -- shared-prefix paged decode for copy-on-write groups.
//
// Sequences forked from one prompt (beams, parallel samples) share the physical
// blocks of their prefix ("vLLM推理引擎PagedAttention原理与性能优化实战" sec 3.2:
// sharers' block tables point at the same blocks, reference-counted).  Attention
// over such a group reads each shared block once for all of its members; the result
// is the per-sequence decode's ("vLLM 推理优化技术深度调研报告" sec 3 formulas 3, 4).

#include "pa_fallback.h"
#include "pa_kernels.cuh"
#include "pa_tcgen05.cuh"

namespace pa {
namespace {

__device__ unsigned int g_shared_err;

// Ring depths of the mma.sync kernel: 8 KB per stage for 16-bit caches, 4 KB for
// E4M3; a multiple of the consumer-warp count, so each stage has one owning warp.
constexpr int kSharedStages16 = 4;
constexpr int kSharedStagesFp8 = 8;

// ---------------------------------------------------------------------------
// Shared-prefix decode for copy-on-write groups (beams of one prompt, parallel
// samples): sequences whose block tables point at the same physical blocks for
// their first prefix_len tokens.  One CTA serves up to 16 query heads, i.e. the
// kv head's query heads of up to 16 / G sequences of a group.  It streams each
// shared prefix block once and applies it to all 16 heads (two n8 MMA tiles),
// then each sequence's own blocks with the other sequences' heads masked.  The
// online softmax of a head only ever sees its own sequence's tokens, so the
// result equals per-sequence decode while the shared blocks cross HBM and the
// SM once per group instead of once per sequence.
// ---------------------------------------------------------------------------
struct SharedParams {
  CUtensorMap tmk;
  CUtensorMap tmv;
  Params p;
  const int32_t* group_starts;  // [num_groups + 1]
  const int32_t* prefix_lens;   // [num_groups]
  int seqs_per_cta;             // SPB: sequences served by one CTA
  int ctas_per_group;           // ceil(max_group_size / SPB)
  int cluster;                  // CTAs splitting one unit's block stream (cluster size)
};

constexpr int kSharedCols = 16;  // query heads per CTA (two n8 tiles)
constexpr float kSharedRescaleLog2 = 8.f;  // lazy running max: largest weight 2^8

// 2^x by the MUFU approximation (inputs here are <= 8 or -inf; -inf gives 0)
__device__ __forceinline__ float ex2_approx_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
#ifndef PA_SHARED_MIN_CHUNK
#define PA_SHARED_MIN_CHUNK 128      // fewest blocks per CTA when a unit is split
#endif

template <typename CT, int kStages>
constexpr size_t shared_smem_bytes() {
  constexpr size_t tile = size_t(kBlockSize) * 128 * CacheTraits<CT>::bytes;
  constexpr size_t pipe = 2 * kStages * tile;
  constexpr size_t combine = combine_bytes<128, kSharedCols>();
  constexpr size_t body = pipe > combine ? pipe : combine;
  // + barriers, per-stage block info, Q^T fragments [8][2][32] x uint2, q multiplier
  // + cluster exchange: per column the CTA's max, sum and accumulator row
  return 1024 + body + 2 * kStages * sizeof(uint64_t) + kStages * sizeof(int) +
         8 * 2 * 32 * sizeof(uint2) + 16 +
         size_t(kSharedCols) * (2 + combine_row<128>()) * sizeof(float);
}

#ifndef PA_SHARED_MIN_CTAS
#define PA_SHARED_MIN_CTAS 4  // resident CTAs per SM the register budget must allow
#endif
template <typename CT, typename QT, int kStages>
__global__ void __launch_bounds__(kThreads, PA_SHARED_MIN_CTAS) decode_shared_prefix_kernel(
    const __grid_constant__ SharedParams sp) {
  constexpr int D = 128;
  constexpr int NT = 2;
  constexpr bool kFp8 = CacheTraits<CT>::bytes == 1;
  constexpr int TILE = kBlockSize * D * CacheTraits<CT>::bytes;
  using MT = typename std::conditional<kFp8, __half, CT>::type;
  constexpr bool kSplitP = std::is_same<MT, __nv_bfloat16>::value;
  static_assert(kStages % kConsumerWarps == 0, "each ring stage must belong to one warp");
  const Params& p = sp.p;
  grid_dependency_wait();  // launched as a programmatic dependent

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  constexpr size_t tile_region = 2 * kStages * size_t(TILE);
  constexpr size_t combine_region = combine_bytes<D, kSharedCols>();
  constexpr size_t body = tile_region > combine_region ? tile_region : combine_region;
  uint8_t* kbuf = smem;
  uint8_t* vbuf = smem + kStages * TILE;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + body);
  uint64_t* empty = full + kStages;
  int* info = reinterpret_cast<int*>(empty + kStages);          // owner << 8 | valid tokens
  uint2* qs = reinterpret_cast<uint2*>(info + kStages + (kStages & 1));  // [8][NT][32]
  float* qmult_s = reinterpret_cast<float*>(qs + 8 * NT * 32);
  float* xm = qmult_s + 4;                   // [16] this CTA's max per column (log2 units)
  float* xl = xm + kSharedCols;              // [16] its sum
  float* xo = xl + kSharedCols;              // [16][R] its accumulator rows

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // a cluster of `cluster` CTAs shares one (group part, kv head) unit and splits its
  // block stream into contiguous chunks
  const int unit = blockIdx.x / sp.cluster;
  const int crank = int(cluster_ctarank());
  const int grp = unit / sp.ctas_per_group;
  const int sub = unit - grp * sp.ctas_per_group;
  const int kvh = blockIdx.y;
  const int G = p.group;
  int gs0 = sp.group_starts[grp], gs1 = sp.group_starts[grp + 1];
  if (gs0 < 0 || gs1 > p.num_seqs || gs1 < gs0) {  // outside the batch: skip the group
    if (sub == 0 && threadIdx.x == 0 && blockIdx.y == 0) atomicOr(&g_shared_err, PA_DEVERR_PREFIX);
    gs0 = gs1 = 0;
  }
  if (sub == 0 && threadIdx.x == 0 && blockIdx.y == 0 &&
      gs1 - gs0 > sp.ctas_per_group * sp.seqs_per_cta)
    atomicOr(&g_shared_err, PA_DEVERR_PREFIX);  // a group the launch does not cover
  const int s0 = gs0 + sub * sp.seqs_per_cta;
  const int nseq = min(sp.seqs_per_cta, gs1 - s0);
  if (nseq <= 0) return;

  // lengths of the CTA's sequences and the shared prefix (device data: checked);
  // every read is issued before the first check, whose error report would order
  // the reads after it one by one
  const int cap = p.cap;
  int Lmin = cap;
  int Ls[kSharedCols];
#pragma unroll
  for (int j = 0; j < kSharedCols; ++j) Ls[j] = j < nseq ? p.seq_lens[s0 + j] : 0;
  int P = sp.prefix_lens[grp];
#pragma unroll
  for (int j = 0; j < kSharedCols; ++j) {
    int L = Ls[j];
    if (j < nseq && (L < 0 || L > cap)) {
      if (tid == 0) atomicOr(&g_shared_err, PA_DEVERR_SEQ_LEN);
      L = L < 0 ? 0 : cap;
    }
    Ls[j] = L;
    if (j < nseq) Lmin = min(Lmin, L);
  }
  if (P < 0 || P % p.block_size != 0 || P > Lmin) {
    if (tid == 0 && sub == 0 && kvh == 0) atomicOr(&g_shared_err, PA_DEVERR_PREFIX);
    P = P < 0 ? 0 : (min(P, Lmin) / p.block_size) * p.block_size;
  }
  const int pblk = P / kBlockSize;
  int ntotal = pblk;
#pragma unroll
  for (int j = 0; j < kSharedCols; ++j)
    if (j < nseq) ntotal += (Ls[j] + kBlockSize - 1) / kBlockSize - pblk;
  // this CTA's chunk [lo, hi) of the stream: prefix blocks, then each member's own
  const int chunk = (ntotal + sp.cluster - 1) / sp.cluster;
  const int lo = min(ntotal, crank * chunk), hi = min(ntotal, lo + chunk);
  const int nblk = hi - lo;

  const int g = lane >> 2, c = lane & 3;
  const int mi = lane >> 3, r = lane & 7;

  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);
    }
    fence_barrier_init();
  }
  __syncthreads();  // barriers initialised: the producer may start streaming

  float acc[8][NT][4];
  float m[NT][2], l[NT][2];

  if (warp == kConsumerWarps) {
    // ---------------- producer: prefix blocks, then every sequence's own blocks ------
    const uint64_t policy = l2_policy_evict_first();
    int issued = 0;
    bool ok = true;
    int gpos = 0;  // stream position of the current segment's first block
    for (int seg = 0; seg <= nseq && ok; ++seg) {
      const int owner = seg - 1;  // -1: the shared prefix
      const int32_t* row = p.block_tables + int64_t(s0 + (owner < 0 ? 0 : owner)) * p.max_blocks_per_seq;
      const int s_b0 = owner < 0 ? 0 : pblk;
      const int s_b1 = owner < 0 ? pblk : (Ls[owner] + kBlockSize - 1) / kBlockSize;
      const int Lown = owner < 0 ? P : Ls[owner];
      // the part of this segment inside [lo, hi)
      const int b0 = s_b0 + max(0, lo - gpos), b1 = s_b0 + min(s_b1 - s_b0, hi - gpos);
      gpos += s_b1 - s_b0;
      for (int base = b0; base < b1 && ok; base += 32) {
        int tile = 0;
        if (base + lane < b1) {
          const int t = base + lane, e = t / p.tiles_per_block;
          int32_t phys = row[e];
          if (owner < 0) {  // the promise: every sequence of the group has these blocks
            for (int j = 1; j < nseq; ++j)
              if (p.block_tables[int64_t(s0 + j) * p.max_blocks_per_seq + e] != phys)
                atomicOr(&g_shared_err, PA_DEVERR_PREFIX);
          }
          if (phys < 0 || phys >= p.num_blocks) {
            atomicOr(&g_shared_err, PA_DEVERR_BLOCK_RANGE);
            phys = 0;
          }
          tile = (phys * p.num_kv_heads + kvh) * p.tiles_per_block + (t - e * p.tiles_per_block);
        }
        const int cnt = min(32, b1 - base);
        for (int jj = 0; jj < cnt; ++jj) {
          const int tl = __shfl_sync(kFullMask, tile, jj);
          const int i = issued, stage = i % kStages;
          if (lane == 0) {
            if (i >= kStages && !mbar_wait_bounded(&empty[stage], ((i / kStages) - 1) & 1)) {
              atomicOr(&g_shared_err, PA_DEVERR_PIPE_TIMEOUT);
              ok = false;
            }
            if (ok) {
              const int nvalid = min(kBlockSize, Lown - (base + jj) * kBlockSize);
              info[stage] = ((owner + 1) << 8) | nvalid;
              const int trow = tl * kBlockSize;
              uint8_t* kd = kbuf + stage * TILE;
              uint8_t* vd = vbuf + stage * TILE;
              mbar_arrive_expect_tx(&full[stage], 2 * TILE);
              if constexpr (kFp8) {
                tma_load_2d(kd, &sp.tmk, 0, trow, &full[stage], policy);
                tma_load_2d(vd, &sp.tmv, 0, trow, &full[stage], policy);
              } else {
                tma_load_2d(kd, &sp.tmk, 0, trow, &full[stage], policy);
                tma_load_2d(kd + TILE / 2, &sp.tmk, 64, trow, &full[stage], policy);
                tma_load_2d(vd, &sp.tmv, 0, trow, &full[stage], policy);
                tma_load_2d(vd + TILE / 2, &sp.tmv, 64, trow, &full[stage], policy);
              }
            }
          }
          ok = __shfl_sync(kFullMask, ok, 0);
          if (!ok) break;
          ++issued;
        }
      }
    }
    if (lane == 0) {
      const int first = issued > kStages ? issued - kStages : 0;
      for (int i = first; i < issued; ++i)
        if (!mbar_wait_bounded(&full[i % kStages], (i / kStages) & 1))
          atomicOr(&g_shared_err, PA_DEVERR_PIPE_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ---------------- consumers ----------------
  // Q^T fragments of the CTA's 16 columns (column n = j * G + head-in-group),
    // prepared once by warp 0 into shared memory.
    if (warp == 0) {
      float mult = p.q_mult;
      uint32_t frag[8][NT][2];
      float qmax = 0.f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int n = nt * 8 + g, j = n / G, hi = n - j * G;
        const bool ok = n < nseq * G;
        const uint8_t* qrow =
            p.query + (int64_t(s0 + (ok ? j : 0)) * p.num_heads + kvh * G + (ok ? hi : 0)) * D * 2;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          if constexpr (!kFp8) {
            frag[ks][nt][0] = ok ? *reinterpret_cast<const uint32_t*>(qrow + (16 * ks + 2 * c) * 2) : 0u;
            frag[ks][nt][1] = ok ? *reinterpret_cast<const uint32_t*>(qrow + (16 * ks + 2 * c + 8) * 2) : 0u;
          } else {
            const uint2 w = ok ? *reinterpret_cast<const uint2*>(qrow + (16 * ks + 4 * c) * 2)
                               : make_uint2(0u, 0u);
            frag[ks][nt][0] = w.x;
            frag[ks][nt][1] = w.y;
            if constexpr (!std::is_same<QT, __half>::value) {
              const float2 a = unpack2(w.x, QT{}), b = unpack2(w.y, QT{});
              qmax = fmaxf(qmax, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(b.x), fabsf(b.y))));
            }
          }
        }
      }
      if constexpr (kFp8 && !std::is_same<QT, __half>::value) {
        // bf16 -> f16 with a power-of-two scale (see decode_mma_kernel)
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) qmax = fmaxf(qmax, __shfl_xor_sync(kFullMask, qmax, o));
        int e = 0;
        if (qmax > 0.f && isfinite(qmax)) frexpf(qmax, &e);
        const int sq = min(max(15 - e, -100), 100);
        mult = ldexpf(mult, -sq);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const float2 a = unpack2(frag[ks][nt][0], QT{}), b = unpack2(frag[ks][nt][1], QT{});
            frag[ks][nt][0] = pack2(ldexpf(a.x, sq), ldexpf(a.y, sq), __half{});
            frag[ks][nt][1] = pack2(ldexpf(b.x, sq), ldexpf(b.y, sq), __half{});
          }
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          qs[(ks * NT + nt) * 32 + lane] = make_uint2(frag[ks][nt][0], frag[ks][nt][1]);
      if (lane == 0) *qmult_s = mult;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");  // consumers only
    const float mult = *qmult_s;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m[nt][0] = m[nt][1] = -INFINITY;
      l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
      for (int t = 0; t < 8; ++t) acc[t][nt][0] = acc[t][nt][1] = acc[t][nt][2] = acc[t][nt][3] = 0.f;
    }
    for (int i = warp; i < nblk; i += kConsumerWarps) {
      const int stage = i % kStages;
      if (!__all_sync(kFullMask, mbar_wait_bounded(&full[stage], (i / kStages) & 1))) {
        if (lane == 0) atomicOr(&g_shared_err, PA_DEVERR_PIPE_TIMEOUT);
        break;
      }
      const int inf = info[stage];
      const int owner = (inf >> 8) - 1, nvalid = inf & 0xff;
      const uint32_t kt = smem_u32(kbuf + stage * TILE);
      const uint32_t vt = smem_u32(vbuf + stage * TILE);

      float sc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
      if constexpr (!kFp8) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const int tok = r + 8 * (mi & 1), j = 2 * ks + (mi >> 1);
          uint32_t a[4];
          ldsm_x4(kt + (j >> 3) * (TILE / 2) + tok * 128 + (((j & 7) ^ r) << 4), a);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const uint2 b = qs[(ks * NT + nt) * 32 + lane];
            mma_16816(sc[nt], a, b.x, b.y, MT{});
          }
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
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const uint2 b0 = qs[((2 * u) * NT + nt) * 32 + lane];
            const uint2 b1 = qs[((2 * u + 1) * NT + nt) * 32 + lane];
            mma_16816(sc[nt], a0, b0.x, b0.y, MT{});
            mma_16816(sc[nt], a1, b1.x, b1.y, MT{});
          }
        }
      }
      const bool v0 = g < nvalid, v8 = g + 8 < nvalid;
      uint32_t bh0[NT], bh1[NT], bl0[NT], bl1[NT];
      float al[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        // columns of this thread and whether the block belongs to them
        const int n0 = nt * 8 + 2 * c, n1 = n0 + 1;
        const bool a0 = owner < 0 || n0 / G == owner;
        const bool a1 = owner < 0 || n1 / G == owner;
        sc[nt][0] = (v0 && a0) ? sc[nt][0] * mult : -INFINITY;
        sc[nt][1] = (v0 && a1) ? sc[nt][1] * mult : -INFINITY;
        sc[nt][2] = (v8 && a0) ? sc[nt][2] * mult : -INFINITY;
        sc[nt][3] = (v8 && a1) ? sc[nt][3] * mult : -INFINITY;
        float mx0 = fmaxf(sc[nt][0], sc[nt][2]), mx1 = fmaxf(sc[nt][1], sc[nt][3]);
#pragma unroll
        for (int o = 4; o <= 16; o <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(kFullMask, mx0, o));
          mx1 = fmaxf(mx1, __shfl_xor_sync(kFullMask, mx1, o));
        }
        // lazy running max: it moves only when a tile's max passes it by more than
        // 2^8, so weights stay <= 256 and most tiles skip the accumulator rescale;
        // O and l are always relative to the same max, so the result is unchanged
        const float mn0 = mx0 > m[nt][0] + kSharedRescaleLog2 ? mx0 : m[nt][0];
        const float mn1 = mx1 > m[nt][1] + kSharedRescaleLog2 ? mx1 : m[nt][1];
        // a column that has seen no token yet keeps m = -inf: scale 1, weights 0
        al[nt][0] = mn0 == -INFINITY ? 1.f : ex2_approx_ftz(m[nt][0] - mn0);
        al[nt][1] = mn1 == -INFINITY ? 1.f : ex2_approx_ftz(m[nt][1] - mn1);
        m[nt][0] = mn0;
        m[nt][1] = mn1;
        const float p0 = mn0 == -INFINITY ? 0.f : ex2_approx_ftz(sc[nt][0] - mn0);
        const float p1 = mn1 == -INFINITY ? 0.f : ex2_approx_ftz(sc[nt][1] - mn1);
        const float p2 = mn0 == -INFINITY ? 0.f : ex2_approx_ftz(sc[nt][2] - mn0);
        const float p3 = mn1 == -INFINITY ? 0.f : ex2_approx_ftz(sc[nt][3] - mn1);
        l[nt][0] = l[nt][0] * al[nt][0] + (p0 + p2);
        l[nt][1] = l[nt][1] * al[nt][1] + (p1 + p3);
        const uint32_t x0 = pack2(p0, p1, MT{}), x1 = pack2(p2, p3, MT{});
        bh0[nt] = movmatrix_trans(x0);
        bh1[nt] = movmatrix_trans(x1);
        bl0[nt] = bl1[nt] = 0;
        if constexpr (kSplitP) {
          const float2 h0 = unpack2(x0, MT{}), h1 = unpack2(x1, MT{});
          bl0[nt] = movmatrix_trans(pack2(p0 - h0.x, p1 - h0.y, MT{}));
          bl1[nt] = movmatrix_trans(pack2(p2 - h1.x, p3 - h1.y, MT{}));
        }
      }
      if (__any_sync(kFullMask, al[0][0] != 1.f || al[0][1] != 1.f || al[1][0] != 1.f ||
                                    al[1][1] != 1.f))
#pragma unroll
        for (int t = 0; t < 8; ++t)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            acc[t][nt][0] *= al[nt][0];
            acc[t][nt][1] *= al[nt][1];
            acc[t][nt][2] *= al[nt][0];
            acc[t][nt][3] *= al[nt][1];
          }
      uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
      if (nvalid < kBlockSize) {
        mlo = (2 * c < nvalid ? 0x0000ffffu : 0u) | (2 * c + 1 < nvalid ? 0xffff0000u : 0u);
        mhi = (2 * c + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * c + 9 < nvalid ? 0xffff0000u : 0u);
      }
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
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mma_16816(acc[t][nt], a, bh0[nt], bh1[nt], MT{});
            if constexpr (kSplitP) mma_16816(acc[t][nt], a, bl0[nt], bl1[nt], MT{});
          }
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int tok = r + 8 * (mi & 1), j = 2 * u + (mi >> 1);
          uint32_t R[4];
          ldsm_x4_trans(vt + tok * 128 + ((j ^ r) << 4), R);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t lo = R[2 * h], hi8 = R[2 * h + 1];
            uint32_t a[4] = {e4m3x2_to_f16x2(__byte_perm(lo, 0, 0x20)) & mlo,
                             e4m3x2_to_f16x2(__byte_perm(lo, 0, 0x31)) & mlo,
                             e4m3x2_to_f16x2(__byte_perm(hi8, 0, 0x20)) & mhi,
                             e4m3x2_to_f16x2(__byte_perm(hi8, 0, 0x31)) & mhi};
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_16816(acc[2 * u + h][nt], a, bh0[nt], bh1[nt], MT{});
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int o = 4; o <= 16; o <<= 1) {
        l[nt][0] += __shfl_xor_sync(kFullMask, l[nt][0], o);
        l[nt][1] += __shfl_xor_sync(kFullMask, l[nt][1], o);
      }
  }

  __syncthreads();  // pipeline finished: the tile region becomes the combine region
  constexpr int GC = kSharedCols;
  constexpr int R = combine_row<D>();
  float* cm = reinterpret_cast<float*>(smem);
  float* cl = cm + kConsumerWarps * GC;
  float* cacc = cl + kConsumerWarps * GC;
  float* cf = cacc + kConsumerWarps * GC * R;
  if (warp < kConsumerWarps) {
    if (g == 0) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        cm[warp * GC + nt * 8 + 2 * c] = m[nt][0];
        cl[warp * GC + nt * 8 + 2 * c] = l[nt][0];
        cm[warp * GC + nt * 8 + 2 * c + 1] = m[nt][1];
        cl[warp * GC + nt * 8 + 2 * c + 1] = l[nt][1];
      }
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int d0 = kFp8 ? 16 * t + 2 * g : 16 * t + g;
      const int d1 = kFp8 ? d0 + 1 : d0 + 8;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int n0 = nt * 8 + 2 * c;
        cacc[(warp * GC + n0) * R + d0] = acc[t][nt][0];
        cacc[(warp * GC + n0) * R + d1] = acc[t][nt][2];
        cacc[(warp * GC + n0 + 1) * R + d0] = acc[t][nt][1];
        cacc[(warp * GC + n0 + 1) * R + d1] = acc[t][nt][3];
      }
    }
  }
  __syncthreads();
  if (sp.cluster == 1) {  // the whole unit in this CTA: finish the columns directly
    if (tid < GC) {
      const int n = tid;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, cm[w * GC + n]);
      float f[kConsumerWarps];
      float Lsum = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float mw = cm[w * GC + n];
        f[w] = mw == -INFINITY ? 0.f : exp2f(mw - M);
        Lsum += cl[w * GC + n] * f[w];
      }
      const float inv = Lsum > 0.f ? p.v_mult / Lsum : 0.f;  // an empty context gives zeros
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) cf[n * (kConsumerWarps + 1) + w] = f[w] * inv;
    }
    __syncthreads();
    for (int e = tid; e < nseq * G * D; e += kThreads) {
      const int n = e / D, d = e - n * D;
      float o = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w)
        o = fmaf(cacc[(w * GC + n) * R + d], cf[n * (kConsumerWarps + 1) + w], o);
      const int jseq = n / G, hi = n - jseq * G;
      store_out(p.out, (int64_t(s0 + jseq) * p.num_heads + kvh * G + hi) * D + d, o,
                p.out_dtype);
    }
    return;
  }
  // This CTA's state per column: max over its warps, sum and accumulator scaled to it.
  if (tid < GC) {
    const int n = tid;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, cm[w * GC + n]);
    float Lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float mw = cm[w * GC + n];
      const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);  // a warp that saw no block
      cf[n * (kConsumerWarps + 1) + w] = f;
      Lsum += cl[w * GC + n] * f;
    }
    xm[n] = M;
    xl[n] = Lsum;
  }
  __syncthreads();
  for (int e = tid; e < GC * D; e += kThreads) {
    const int n = e / D, d = e - n * D;
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w)
      o = fmaf(cacc[(w * GC + n) * R + d], cf[n * (kConsumerWarps + 1) + w], o);
    xo[n * R + d] = o;
  }
  // Merge across the cluster: CTA `crank` finishes the columns n = crank mod cluster,
  // one output element per thread, reading every CTA's state for it through
  // distributed shared memory (independent reads, issued together).
  cluster_sync();
  const int ncols = nseq * G;
  const int mycols = (ncols - crank + sp.cluster - 1) / sp.cluster;
  for (int e = tid; e < mycols * D; e += kThreads) {
    const int k = e / D, d = e - k * D;
    const int n = crank + k * sp.cluster;
    float mq[8], lq[8], oq[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (q < sp.cluster) {
        mq[q] = ld_dsmem_f32(xm + n, q);
        lq[q] = ld_dsmem_f32(xl + n, q);
        oq[q] = ld_dsmem_f32(xo + n * R + d, q);
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (q < sp.cluster) M = fmaxf(M, mq[q]);
    float Lsum = 0.f, o = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (q < sp.cluster && mq[q] != -INFINITY) {
        const float f = exp2f(mq[q] - M);
        Lsum = fmaf(lq[q], f, Lsum);
        o = fmaf(oq[q], f, o);
      }
    }
    const float inv = Lsum > 0.f ? p.v_mult / Lsum : 0.f;  // an empty context gives zeros
    const int jseq = n / G, hi = n - jseq * G;
    store_out(p.out, (int64_t(s0 + jseq) * p.num_heads + kvh * G + hi) * D + d, o * inv,
              p.out_dtype);
  }
  cluster_sync();  // keep every CTA's shared memory alive until all reads are done
}


// ---------------------------------------------------------------------------
// Shared-prefix decode on the 5th-generation tensor cores, for E4M3 caches.
//
// The same work unit as above (one CTA per group part and kv head, up to 16
// columns = the kv head's query heads of up to 16 / G members), but the stream
// of 16-token tiles -- the shared prefix first, then each member's own tiles --
// is cut into stages of 128 tokens with the tokens on the M axis, and both
// contractions run on E4M3 operands straight from the TMA-staged tiles:
//   S^T[128 tokens x 16 columns]  = K[128 x 128 dims] . Q^T     kind::f8f6f4
//   O^T[128 dims x 16 columns]   += V^T[128 dims x 128] . P^T   kind::f8f6f4
// Nothing is widened.  Q is split per column into E4M3 terms instead: scaled by
// a power of two so that its largest |q| lies in [128, 256), then
// q' = t_0 + 2^-4 t_1 (+ 2^-8 t_2), each t the E4M3 rounding of what is left.
// A bf16 value (8 significant bits) is exactly two such terms, an f16 value
// (11) exactly three, so S^T = sum 2^-4k K.T_k^T is the product with the exact
// query (each term's products are exact, accumulation is fp32).  P <= 2^8 (the
// lazy reference maximum below) is split the same way into three terms, about
// 12 significant bits, one more than the f16 P of the other kernels; O^T keeps
// one fp32 accumulator per term.  Rows past the context are zeroed in the staged
// V tile before P.V reads it.
//   * softmax warps 0-3: thread t owns token t of a stage (its row of S^T) and
//     dim t of O^T; every column keeps one reference maximum shared by all
//     threads, moved (with a rescale of l and of O^T's columns) only when some
//     score passes it by more than 2^8, which a vote and a named barrier detect;
//     each thread sums its own l and the sums meet once, at the end;
//   * warps 4 and 6 stream the raw K and V tiles (tiled TMA, 128-byte swizzle, no
//     multicast) into two rings of kStRing stages, K and V each with barriers of
//     their own: a K slot refills as soon as S has read it, so S and the softmax
//     of a stage can finish while its V is still landing; warp 5 issues each
//     stage's MMAs (S of stage st + 1 before P.V of stage st) and owns the TMEM
//     allocation; warp 7 idles.  setmaxnreg gives warps 4-7 72 registers a thread
//     and the softmax warps 184, so that two CTAs of 8 warps fit an SM.
// Every mbarrier a waiter could otherwise see two phases ahead is split per
// buffer.  All waits are bounded; after a failure the waits are skipped but every
// named barrier is still reached.
// ---------------------------------------------------------------------------
constexpr int kStTokens = 128;                          // tokens per stage (M of S^T)
constexpr int kStTiles = kStTokens / kBlockSize;        // pool tiles per stage
constexpr int kStQuads = 4;                             // softmax warps (TMEM lane quadrants)
constexpr int kStKWarp = kStQuads;        // streams the K tiles
constexpr int kStMmaWarp = kStQuads + 1;  // issues the MMAs, owns TMEM
constexpr int kStVWarp = kStQuads + 2;    // streams the V tiles; warp 7 idles
constexpr int kStThreads = (kStQuads + 4) * 32;
// Two CTAs per SM launch with 128 registers a thread; setmaxnreg then moves them
// from the loader/MMA warpgroup (72) to the softmax warpgroup (184).
constexpr int kStLaunchRegs = 128;
constexpr int kStLoadRegs = 72;      // the least that spills nothing (40 and 56 spill)
constexpr int kStSoftmaxRegs = 184;
static_assert(128 * kStLoadRegs + 128 * kStSoftmaxRegs <= kStThreads * kStLaunchRegs,
              "the split draws only on the registers the CTA was launched with");
#ifndef PA_SHARED_TC_RING
#define PA_SHARED_TC_RING 3
#endif
constexpr int kStRing = PA_SHARED_TC_RING;              // stages in flight, K and V each
constexpr int kStRawTile = kBlockSize * 128;            // one E4M3 tile of K or V: 2 KB
constexpr int kStRawHalf = kStTiles * kStRawTile;      // a stage's K (or V) tiles: 16 KB
constexpr int kStTerm = kSharedCols * 128;              // one E4M3 term of Q^T or P^T: 2 KB
constexpr int kStPTerms = 3;                            // terms of P
constexpr uint32_t kStTmemCols = 256;
constexpr uint32_t kStTmemS = 0;    // S^T buffers b = 0, 1: [terms of Q][16] fp32 columns
constexpr uint32_t kStTmemO = 128;  // O^T: [terms of P][16] fp32 columns
// kind::f8f6f4, E4M3 x E4M3 (format code 0), fp32 accumulate; S: both K-major;
// P.V: A = V^T and B = P^T both MN-major
constexpr uint32_t kStIdescPV = umma_idesc_f16_ab(0, 1, 1, 128, kSharedCols * kStPTerms);

template <int NQ>
constexpr size_t shared_tc_smem_bytes() {
  return 1024 + size_t(2 * kStRing) * kStRawHalf + size_t(NQ + kStPTerms) * kStTerm +
         (kStRing * 4 + 10) * sizeof(uint64_t) +
         (8 + 2 * kStQuads * kSharedCols + kStQuads * kSharedCols + kSharedCols) * 4 +
         (2 * (kSharedCols + 1) + 2) * 4;
}
static_assert(2 * (shared_tc_smem_bytes<3>() + 1024) <= 228 * 1024, "two CTAs per SM");

// D[tmem] (+)= A[smem desc] * B[smem desc] with 8-bit (E4M3) operands.
__device__ __forceinline__ void umma_f8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16 32-bit words into this warp's 32 TMEM lanes, columns taddr .. taddr + 15.
__device__ __forceinline__ void tmem_st16_f(uint32_t taddr, const float (&v)[16]) {
  uint32_t u[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(v[i]);
  tmem_st16(taddr, u);
}

// Split x0, x1 (|x| < 448) into `terms` E4M3 pairs: code k holds the E4M3 rounding
// of what the codes before it leave, times 16^k.
template <int terms>
__device__ __forceinline__ void split_e4m3x2(float x0, float x1, uint16_t (&code)[terms]) {
#pragma unroll
  for (int k = 0; k < terms; ++k) {
    code[k] = pack2_e4m3(x0, x1);
    if (k + 1 < terms) {
      const float2 back = unpack2_e4m3(code[k]);
      x0 = (x0 - back.x) * 16.f;  // exact: the difference has at most the bits left
      x1 = (x1 - back.y) * 16.f;
    }
  }
}

// The token of row r (0..127) of stage st: its member (-1 = shared prefix; the
// masked columns follow from it) and whether it lies inside that member's context.
struct StRow {
  int owner;
  bool valid;
};
__device__ __forceinline__ StRow st_row(int st, int r, int pblk, int ntotal, int nseq,
                                        const int* own_start, const int* own_len) {
  const int T = st * kStTiles + (r >> 4);
  StRow x{-1, T < ntotal};
  if (x.valid && T >= pblk) {
    x.owner = 0;
    while (x.owner + 1 < nseq && own_start[x.owner + 1] <= T) ++x.owner;
    x.valid = (pblk + (T - own_start[x.owner])) * kBlockSize + (r & 15) < own_len[x.owner];
  }
  return x;
}

template <typename QT>
__global__ void __launch_bounds__(kStThreads, 2) decode_shared_tc_kernel(
    const __grid_constant__ SharedParams sp) {
  constexpr int D = 128;
  constexpr int NQ = std::is_same<QT, __half>::value ? 3 : 2;  // terms of Q
  const Params& p = sp.p;
  grid_dependency_wait();  // launched as a programmatic dependent
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* rawk = smem;                                 // [kStRing][8 K tiles]
  uint8_t* rawv = rawk + kStRing * kStRawHalf;          // [kStRing][8 V tiles]
  uint8_t* qop = rawv + kStRing * kStRawHalf;           // Q^T terms: [NQ][16 rows][128 B] SW128
  uint8_t* pop = qop + NQ * kStTerm;                    // P^T terms: [3][128 tokens][16 B]
  // K and V of a stage have rings and barriers of their own: a K slot is free once
  // S has read it, a whole softmax and P.V before the V slot of the same stage
  uint64_t* fullk = reinterpret_cast<uint64_t*>(pop + kStPTerms * kStTerm);
  uint64_t* fullv = fullk + kStRing;
  uint64_t* emptyk = fullv + kStRing;
  uint64_t* emptyv = emptyk + kStRing;
  uint64_t* sfull = emptyv + kStRing;                    // [2] S buffer b of stage st written
  uint64_t* pready = sfull + 2;                         // P of stage st written, O rescaled
  uint64_t* odone = pready + 1;                         // P.V of stage st done
  uint64_t* qready = odone + 1;                         // Q^T terms written
  uint64_t* done = qready + 1;                          // every MMA done
  uint64_t* sread = done + 1;                           // [2] S buffer b read by the softmax
  int* flags = reinterpret_cast<int*>(sread + 3);       // [2][4] rescale votes
  float* wmax = reinterpret_cast<float*>(flags + 8);    // [2][4][16] warp column maxima
  float* lsum = wmax + 2 * kStQuads * kSharedCols;      // [4][16] warp column sums
  float* colmult = lsum + kStQuads * kSharedCols;       // [16] score multiplier per column
  int* own_start = reinterpret_cast<int*>(colmult + kSharedCols);  // [17] stream positions
  int* own_len = own_start + kSharedCols + 1;           // [16] member lengths
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(own_len + kSharedCols + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.x;
  const int kvh = blockIdx.y;
  const int grp = unit / sp.ctas_per_group;
  const int sub = unit - grp * sp.ctas_per_group;
  const int G = p.group;
  int gs0 = sp.group_starts[grp], gs1 = sp.group_starts[grp + 1];
  if (gs0 < 0 || gs1 > p.num_seqs || gs1 < gs0) {  // outside the batch: skip the group
    if (sub == 0 && tid == 0 && kvh == 0) atomicOr(&g_shared_err, PA_DEVERR_PREFIX);
    gs0 = gs1 = 0;
  }
  if (sub == 0 && tid == 0 && kvh == 0 && gs1 - gs0 > sp.ctas_per_group * sp.seqs_per_cta)
    atomicOr(&g_shared_err, PA_DEVERR_PREFIX);  // a group the launch does not cover
  const int s0 = gs0 + sub * sp.seqs_per_cta;
  const int nseq = min(sp.seqs_per_cta, gs1 - s0);
  if (nseq <= 0) return;  // uniform over the CTA, before any barrier or TMEM
  const int ncols = nseq * G;

  // The producer's block-table entries of the first group of 4 stages: lane l takes
  // stream tile l.  They are read now, before the lengths are known, on the guess
  // that the tile lies in the shared prefix (member 0's table, logical tile l, and
  // every member's entry for the promise check); a lane whose guess fails reads
  // its entry again once the stream layout is known.  The reads stay inside the
  // members' table rows.
  int32_t nx[kSharedCols];  // the fetched tile's entry in each member's table (prefix)
  const bool spec = (warp == kStKWarp || warp == kStVWarp) &&
                    lane / p.tiles_per_block < p.max_blocks_per_seq;
  if (spec) {
    const int e = lane / p.tiles_per_block;
#pragma unroll
    for (int jj = 0; jj < kSharedCols; ++jj)
      if (jj < nseq) nx[jj] = p.block_tables[int64_t(s0 + jj) * p.max_blocks_per_seq + e];
  }
  // Stage 0 leaves as soon as those entries are in.  The stream's first tiles are
  // member 0's logical tiles 0, 1, ... (its prefix tiles, then its own), so while
  // member 0 holds kStTiles tiles or more the first stage is its tiles 0 ..
  // kStTiles - 1 whatever the prefix length.  Each producer initialises its own
  // ring's barriers and issues that stage here, before the lengths are checked
  // and the CTA synchronises; its loop below skips the stage.  The checks of the
  // same entries (block range, the prefix promise) still run there.
  bool early = false;
  if (warp == kStKWarp || warp == kStVWarp) {
    const bool is_k = warp == kStKWarp;
    uint64_t* fullx = is_k ? fullk : fullv;
    uint64_t* emptyx = is_k ? emptyk : emptyv;
    if (lane == 0) {
      for (int i = 0; i < kStRing; ++i) {
        mbar_init(&fullx[i], 1);
        mbar_init(&emptyx[i], 1);
      }
      fence_barrier_init();
    }
    const int L0 = p.seq_lens[s0];
    const int32_t phys = spec ? nx[0] : -1;
    const bool in_range = lane >= kStTiles || (spec && phys >= 0 && phys < p.num_blocks);
    early = L0 > (kStTiles - 1) * kBlockSize && L0 <= p.cap && __all_sync(kFullMask, in_range);
    if (early) {
      const int e = lane / p.tiles_per_block;
      const int row =
          ((phys * p.num_kv_heads + kvh) * p.tiles_per_block + (lane - e * p.tiles_per_block)) *
          kBlockSize;
      if (lane == 0) mbar_arrive_expect_tx(&fullx[0], uint32_t(kStTiles) * kStRawTile);
      __syncwarp();
      if (lane < kStTiles)
        tma_load_2d((is_k ? rawk : rawv) + lane * kStRawTile, is_k ? &sp.tmk : &sp.tmv, 0, row,
                    &fullx[0], l2_policy_evict_first());
    }
  }
  // lengths and the shared prefix (device data: checked), as the mma.sync kernel;
  // every read is issued before the first check, whose error report would order
  // the reads after it one by one
  if (tid == 0) {
    const int cap = p.cap;
    int Lr[kSharedCols];
#pragma unroll
    for (int j = 0; j < kSharedCols; ++j) Lr[j] = j < nseq ? p.seq_lens[s0 + j] : 0;
    int P = sp.prefix_lens[grp];
    int Lmin = cap;
#pragma unroll
    for (int j = 0; j < kSharedCols; ++j) {
      int L = Lr[j];
      if (j < nseq && (L < 0 || L > cap)) {
        atomicOr(&g_shared_err, PA_DEVERR_SEQ_LEN);
        L = L < 0 ? 0 : cap;
      }
      own_len[j] = L;
      if (j < nseq) Lmin = min(Lmin, L);
    }
    if (P < 0 || P % p.block_size != 0 || P > Lmin) {
      if (sub == 0 && kvh == 0) atomicOr(&g_shared_err, PA_DEVERR_PREFIX);
      P = P < 0 ? 0 : (min(P, Lmin) / p.block_size) * p.block_size;
    }
    const int pb = P / kBlockSize;
    int pos = pb;
    for (int j = 0; j < kSharedCols; ++j) {
      own_start[j] = pos;
      if (j < nseq) pos += (own_len[j] + kBlockSize - 1) / kBlockSize - pb;
    }
    own_start[kSharedCols] = pos;
    mbar_init(&sfull[0], 1);
    mbar_init(&sfull[1], 1);
    mbar_init(pready, kStQuads);
    mbar_init(odone, 1);
    mbar_init(qready, kStQuads);
    mbar_init(done, 1);
    mbar_init(&sread[0], kStQuads);
    mbar_init(&sread[1], kStQuads);
    fence_barrier_init();
  }
  if (warp == kStMmaWarp) {  // the MMA warp owns the TMEM allocation
    tmem_alloc(tmem_slot, kStTmemCols);
    tmem_relinquish();
  }
  tcgen05_fence_before();
  __syncthreads();
  tcgen05_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int pblk = own_start[0];
  const int ntotal = own_start[kSharedCols];
  const int nstages = (ntotal + kStTiles - 1) / kStTiles;

  if (warp >= kStQuads) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kStLoadRegs));
  if (warp == kStKWarp || warp == kStVWarp) {
    // ---------------- producers: the raw E4M3 K (or V) tiles of each stage ----------------
    // Both warps walk the same stream and block-table entries; the K warp reports
    // bad entries.
    const bool is_k = warp == kStKWarp;
    uint64_t* fullx = is_k ? fullk : fullv;
    uint64_t* emptyx = is_k ? emptyk : emptyv;
    uint8_t* ring = is_k ? rawk : rawv;
    const CUtensorMap* map = is_k ? &sp.tmk : &sp.tmv;
    const uint64_t policy = l2_policy_evict_first();
    int issued = 0, ent = -1;
    bool ok = true;
    // Lane l takes stream tile 32 g + l of each group g of 4 stages.  The block-table
    // entries of group g + 1 are read while group g streams and are checked (the
    // prefix promise, the block range) when their group starts, so no table read
    // sits between a freed ring slot and its next load.
    int nx_T = 0, nx_lt = 0;  // the fetched tile (entries in nx); its logical tile
    auto fetch = [&](int T) {
      nx_T = T;
      if (T >= ntotal) return;
      int j = 0, lt = T;  // member whose table holds the tile, logical tile there
      if (T >= pblk) {
        while (j + 1 < nseq && own_start[j + 1] <= T) ++j;
        lt = pblk + (T - own_start[j]);
      }
      nx_lt = lt;
      const int e = lt / p.tiles_per_block;
      nx[0] = p.block_tables[int64_t(s0 + j) * p.max_blocks_per_seq + e];
      if (T < pblk) {
#pragma unroll
        for (int jj = 1; jj < kSharedCols; ++jj)
          if (jj < nseq) nx[jj] = p.block_tables[int64_t(s0 + jj) * p.max_blocks_per_seq + e];
      }
    };
    auto resolve = [&]() -> int {  // pool row of the fetched tile, -1 past the stream
      if (nx_T >= ntotal) return -1;
      int32_t phys = nx[0];
      if (nx_T < pblk) {  // the promise: every member has these blocks
        bool same = true;
#pragma unroll
        for (int jj = 1; jj < kSharedCols; ++jj)
          if (jj < nseq) same &= nx[jj] == phys;
        if (!same && is_k) atomicOr(&g_shared_err, PA_DEVERR_PREFIX);
      }
      if (phys < 0 || phys >= p.num_blocks) {
        if (is_k) atomicOr(&g_shared_err, PA_DEVERR_BLOCK_RANGE);
        phys = 0;
      }
      const int e = nx_lt / p.tiles_per_block;
      return ((phys * p.num_kv_heads + kvh) * p.tiles_per_block + (nx_lt - e * p.tiles_per_block)) *
             kBlockSize;
    };
    if (spec && lane < pblk && lane < ntotal) {  // the guess held: entries in nx already
      nx_T = lane;
      nx_lt = lane;
    } else {
      fetch(lane);
    }
    for (int st = 0; st < nstages && ok; ++st) {
      if ((st & 3) == 0) {
        ent = resolve();
        fetch((st + 4) * kStTiles + lane);
      }
      // lane i (< 8) loads tile i of the stage: the copies of a stage leave in one
      // instruction of 8 lanes (a copy costs its issuing thread far more than the
      // instruction does, so lanes issuing together keep many more in flight)
      const int row = __shfl_sync(kFullMask, ent, (st & 3) * kStTiles + (lane & (kStTiles - 1)));
      const int slot = st % kStRing;
      if (lane == 0 && st >= kStRing && !mbar_test(&emptyx[slot], ((st / kStRing) - 1) & 1) &&
          !mbar_wait_bounded(&emptyx[slot], ((st / kStRing) - 1) & 1)) {
        atomicOr(&g_shared_err, PA_DEVERR_PIPE_TIMEOUT);
        ok = false;
      }
      ok = __shfl_sync(kFullMask, ok, 0);
      if (!ok) break;
      const int n = min(kStTiles, ntotal - st * kStTiles);
      if (st > 0 || !early) {  // stage 0 may have left before the CTA synchronised
        if (lane == 0) mbar_arrive_expect_tx(&fullx[slot], uint32_t(n) * kStRawTile);
        __syncwarp();
        if (lane < n)
          tma_load_2d(ring + slot * kStRawHalf + lane * kStRawTile, map, 0, row, &fullx[slot],
                      policy);
      }
      ++issued;
    }
    if (lane == 0) {  // no copy may still be landing when the CTA exits
      for (int i = max(0, issued - kStRing); i < issued; ++i)
        if (!mbar_wait_bounded(&fullx[i % kStRing], (i / kStRing) & 1))
          atomicOr(&g_shared_err, PA_DEVERR_PIPE_TIMEOUT);
    }
    __syncwarp();
  } else if (warp == kStMmaWarp) {
    // ---------------- MMA issuer (one thread): S(st + 1), then P.V(st) ----------------
    if (lane == 0) {
      // K tiles of a stage: [128 token rows][128 B], 128-byte swizzle (K-major A);
      // V tiles: the same rows read as MN-major A (V^T).  The terms of Q^T and of P^T
      // sit side by side along N, so one MMA of N = 16 x terms covers them all and
      // reads each K or V tile once: Q^T terms [16 rows][128 B] K-major B, their
      // 8-row groups 1024 B apart, term after term; P^T terms [128 tokens][16 B]
      // MN-major B, 8-token core matrices 128 B apart along K, terms 2 KB apart
      // along N.
      const uint64_t kdesc = umma_smem_desc(smem_u32(rawk), 16, 1024, kUmmaSwizzle128B);
      const uint64_t vdesc = umma_smem_desc(smem_u32(rawv), 16, 1024, kUmmaSwizzle128B);
      const uint64_t qdesc = umma_smem_desc(smem_u32(qop), 16, 1024, kUmmaSwizzle128B);
      const uint64_t pdesc = umma_smem_desc(smem_u32(pop), 128, kStTerm, 0);
      constexpr uint32_t kIdescS = umma_idesc_f16(0, 0, kStTokens, kSharedCols * NQ);
      bool ok = mbar_wait_bounded(qready, 0);
      // Polls the barriers and issues S(ns) as soon as its stage has landed and its
      // S buffer is free (every softmax warp has loaded S(ns - 2)), and P.V(npv) as
      // soon as P(npv) is written; sleeps otherwise.
      int ns = 0, npv = 0, idle = 0;
      unsigned long long t_idle = 0;
      while (ok && npv < nstages) {
        bool prog = false;
        // S(ns) goes into the buffer of S(ns - 2) as soon as every softmax warp has
        // loaded that into its registers, not only once P.V(ns - 2) is issued
        if (ns < nstages && (ns < 2 || mbar_test(&sread[ns & 1], ((ns - 2) >> 1) & 1)) &&
            mbar_test(&fullk[ns % kStRing], (ns / kStRing) & 1)) {
          tcgen05_fence_after();
          const uint64_t kd = kdesc + uint64_t(((ns % kStRing) * kStRawHalf) >> 4);
          const uint32_t sb = tmem + kStTmemS + uint32_t(ns & 1) * (16 * 3);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)  // 32 dims per step, every Q term at once
            umma_f8_ss(sb, kd + uint64_t((ks * 32) >> 4), qdesc + uint64_t((ks * 32) >> 4),
                       kIdescS, ks > 0 ? 1u : 0u);
          umma_commit(&sfull[ns & 1]);
          umma_commit(&emptyk[ns % kStRing]);  // the K slot is read
          ++ns;
          prog = true;
        }
        if (npv < ns && mbar_test(pready, npv & 1) &&
            mbar_test(&fullv[npv % kStRing], (npv / kStRing) & 1)) {
          tcgen05_fence_after();
          const uint64_t vd = vdesc + uint64_t(((npv % kStRing) * kStRawHalf) >> 4);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)  // 32 tokens per step, every P term at once
            umma_f8_ss(tmem + kStTmemO, vd + uint64_t((ks * 4096) >> 4),
                       pdesc + uint64_t((ks * 512) >> 4), kStIdescPV,
                       (npv > 0 || ks > 0) ? 1u : 0u);
          umma_commit(odone);
          umma_commit(&emptyv[npv % kStRing]);  // the V slot is read
          ++npv;
          prog = true;
        }
        if (prog) {
          idle = 0;
          continue;
        }
        // sleep on the barrier the next step most likely waits for
        if (npv < ns)
          mbar_try_wait(pready, npv & 1, 500);
        else
          mbar_try_wait(&fullk[ns % kStRing], (ns / kStRing) & 1, 500);
        if (idle == 0) t_idle = global_timer_ns();
        if ((++idle & 63) == 0 && global_timer_ns() - t_idle > kWaitLimitNs) ok = false;
      }
      if (!ok) atomicOr(&g_shared_err, PA_DEVERR_PIPE_TIMEOUT);
      umma_commit(done);  // fires once every MMA issued above has completed
      if (!mbar_wait_bounded(done, 0)) atomicOr(&g_shared_err, PA_DEVERR_PIPE_TIMEOUT);
    }
    __syncwarp();
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kStSoftmaxRegs));
    // ---------------- softmax warps: token row r of S^T, dim row r of O^T ----------------
    const int r = tid;                                       // 0..127
    const uint32_t tl = tmem + (uint32_t(32 * warp) << 16);  // this warp's lane quadrant
    bool ok = true;
    // A phase that has completed is seen by a plain test, with no suspending try
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      if (ok) ok = __all_sync(kFullMask, mbar_test(bar, parity) || mbar_wait_bounded(bar, parity));
    };
    // ---- Q^T terms: thread t takes column n = t / 8, dims 16 (t % 8) .. + 15 ----
    {
      const int n = r >> 3, dc = r & 7;
      const int j = n / G, hi = n - j * G;
      uint4 w0 = make_uint4(0u, 0u, 0u, 0u), w1 = w0;
      if (n < ncols) {
        const uint4* src = reinterpret_cast<const uint4*>(
            p.query + (int64_t(s0 + j) * p.num_heads + kvh * G + hi) * D * 2 + dc * 32);
        w0 = src[0];
        w1 = src[1];
      }
      const uint32_t qw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      float qf[16];
      float qm = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 a = unpack2(qw[i], QT{});
        qf[2 * i] = a.x;
        qf[2 * i + 1] = a.y;
        qm = fmaxf(qm, fmaxf(fabsf(a.x), fabsf(a.y)));
      }
#pragma unroll
      for (int o = 4; o >= 1; o >>= 1) qm = fmaxf(qm, __shfl_xor_sync(kFullMask, qm, o));
      // the column's largest |q| goes to [128, 256): a power of two, exact
      int e = 0;
      if (qm > 0.f && isfinite(qm)) frexpf(qm, &e);
      const int sa = min(max(8 - e, -120), 120);
      if (dc == 0) colmult[n] = ldexpf(p.q_mult, -sa);
      uint32_t tw[NQ][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint16_t code[NQ];
        split_e4m3x2<NQ>(ldexpf(qf[2 * i], sa), ldexpf(qf[2 * i + 1], sa), code);
#pragma unroll
        for (int t = 0; t < NQ; ++t) {
          if (i & 1)
            tw[t][i >> 1] |= uint32_t(code[t]) << 16;
          else
            tw[t][i >> 1] = code[t];
        }
      }
      // K-major, 128-byte swizzle: the 16 dims of chunk dc of row n at chunk dc ^ (n % 8)
#pragma unroll
      for (int t = 0; t < NQ; ++t)
        *reinterpret_cast<uint4*>(qop + t * kStTerm + n * 128 + ((dc ^ (n & 7)) << 4)) =
            make_uint4(tw[t][0], tw[t][1], tw[t][2], tw[t][3]);
      fence_proxy_async_smem();  // the MMA reads them through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(qready);
      named_bar_sync(1, kStQuads * 32);  // colmult written
    }
    float cmul[kSharedCols];
#pragma unroll
    for (int n = 0; n < kSharedCols; ++n) cmul[n] = colmult[n];

    float mref[kSharedCols], lacc[kSharedCols];
#pragma unroll
    for (int n = 0; n < kSharedCols; ++n) {
      mref[n] = -INFINITY;
      lacc[n] = 0.f;
    }
    for (int st = 0; st < nstages; ++st) {
      const uint32_t b = uint32_t(st & 1);
      const StRow x = st_row(st, r, pblk, ntotal, nseq, own_start, own_len);
      const int lo = x.owner < 0 ? 0 : x.owner * G, hi = x.owner < 0 ? ncols : lo + G;
      // ---- scores of this row: the Q terms' products combined, masked, log2 units ----
      wait(&sfull[b], (st >> 1) & 1);
      tcgen05_fence_after();
      float sc[kSharedCols];
      {
        float st_[NQ][kSharedCols];
#pragma unroll
        for (int t = 0; t < NQ; ++t) tmem_ld16(tl + kStTmemS + b * (16 * 3) + 16 * t, st_[t]);
        tmem_wait_ld();
        // the S buffer is free for S(st + 2) once this warp's rows are in registers
        tcgen05_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sread[b]);
#pragma unroll
        for (int n = 0; n < kSharedCols; ++n) {
          float v = st_[NQ - 1][n];
#pragma unroll
          for (int t = NQ - 2; t >= 0; --t) v = fmaf(v, 0.0625f, st_[t][n]);
          sc[n] = v;
        }
      }
      bool up = false;
#pragma unroll
      for (int n = 0; n < kSharedCols; ++n) {
        sc[n] = (x.valid && n >= lo && n < hi) ? sc[n] * cmul[n] : -INFINITY;
        up |= sc[n] > mref[n] + kSharedRescaleLog2;
      }
      // ---- does any column's reference maximum move?  (vote, 128 threads) ----
      const int fb = (st & 1) * kStQuads;
      const unsigned vote = __ballot_sync(kFullMask, up);
      if (lane == 0) flags[fb + warp] = vote != 0u;
      named_bar_sync(1, kStQuads * 32);
      // P.V(st - 1) must be done before O^T is rescaled or the P^T buffer rewritten
      bool pv_done = st == 0;
      if (flags[fb] | flags[fb + 1] | flags[fb + 2] | flags[fb + 3]) {  // uniform
#pragma unroll
        for (int n = 0; n < kSharedCols; ++n) {
          float m = sc[n];
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
          if (lane == 0) wmax[(fb + warp) * kSharedCols + n] = m;
        }
        named_bar_sync(1, kStQuads * 32);
        float alpha[kSharedCols];
        bool moved = false;
#pragma unroll
        for (int n = 0; n < kSharedCols; ++n) {
          const float* wm = wmax + fb * kSharedCols + n;
          const float cm = fmaxf(fmaxf(wm[0], wm[kSharedCols]),
                                 fmaxf(wm[2 * kSharedCols], wm[3 * kSharedCols]));
          const float mn = cm > mref[n] + kSharedRescaleLog2 ? cm : mref[n];
          alpha[n] = mn == mref[n] ? 1.f : ex2_approx_ftz(mref[n] - mn);  // -inf -> 0
          moved |= mn != mref[n];
          mref[n] = mn;
          lacc[n] *= alpha[n];
        }
        if (st > 0 && moved) {  // O^T columns of this thread's dim row, every P term
          wait(odone, (st - 1) & 1);
          pv_done = true;
          tcgen05_fence_after();
#pragma unroll
          for (int t = 0; t < kStPTerms; ++t) {
            float o[kSharedCols];
            tmem_ld16(tl + kStTmemO + 16 * t, o);
            tmem_wait_ld();
#pragma unroll
            for (int n = 0; n < kSharedCols; ++n) o[n] *= alpha[n];
            tmem_st16_f(tl + kStTmemO + 16 * t, o);
          }
          tmem_wait_st();
        }
      }
      // ---- P^T row: three E4M3 terms of 16 bytes, token r of each ----
      uint32_t pw[kStPTerms][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int n0 = 2 * i, n1 = 2 * i + 1;
        const float p0 = sc[n0] > -INFINITY ? ex2_approx_ftz(sc[n0] - mref[n0]) : 0.f;
        const float p1 = sc[n1] > -INFINITY ? ex2_approx_ftz(sc[n1] - mref[n1]) : 0.f;
        lacc[n0] += p0;
        lacc[n1] += p1;
        uint16_t code[kStPTerms];
        split_e4m3x2<kStPTerms>(p0, p1, code);
#pragma unroll
        for (int t = 0; t < kStPTerms; ++t) {
          if (i & 1)
            pw[t][i >> 1] |= uint32_t(code[t]) << 16;
          else
            pw[t][i >> 1] = code[t];
        }
      }
      if (!pv_done) wait(odone, (st - 1) & 1);
#pragma unroll
      for (int t = 0; t < kStPTerms; ++t)
        *reinterpret_cast<uint4*>(pop + t * kStTerm + r * 16) =
            make_uint4(pw[t][0], pw[t][1], pw[t][2], pw[t][3]);
      // V rows past the context may hold anything, even NaN: zero them once the
      // stage's V has landed (its slot is not refilled before this P.V)
      if (__any_sync(kFullMask, !x.valid)) wait(&fullv[st % kStRing], (st / kStRing) & 1);
      if (!x.valid) {
        uint8_t* vrow = rawv + (st % kStRing) * kStRawHalf + (r >> 4) * kStRawTile + (r & 15) * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(vrow + 16 * c) = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
      tcgen05_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pready);
    }
    // ---- epilogue: column sums over the CTA, O^T row of this dim, outputs ----
    if (nstages > 0) wait(odone, (nstages - 1) & 1);
    tcgen05_fence_after();
    // column sums of the warp: halve the columns a lane holds at each step (16
    // shuffles); lanes 2c' and 2c' + 1 end with one column's sum
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool h = lane & 16;
      const float keep = h ? lacc[i + 8] : lacc[i], send = h ? lacc[i] : lacc[i + 8];
      lacc[i] = keep + __shfl_xor_sync(kFullMask, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool h = lane & 8;
      const float keep = h ? lacc[i + 4] : lacc[i], send = h ? lacc[i] : lacc[i + 4];
      lacc[i] = keep + __shfl_xor_sync(kFullMask, send, 8);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const bool h = lane & 4;
      const float keep = h ? lacc[i + 2] : lacc[i], send = h ? lacc[i] : lacc[i + 2];
      lacc[i] = keep + __shfl_xor_sync(kFullMask, send, 4);
    }
    {
      const bool h = lane & 2;
      const float keep = h ? lacc[1] : lacc[0], send = h ? lacc[0] : lacc[1];
      lacc[0] = keep + __shfl_xor_sync(kFullMask, send, 2);
    }
    lacc[0] += __shfl_xor_sync(kFullMask, lacc[0], 1);
    {
      const int c = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 +
                    ((lane >> 1) & 1);
      if ((lane & 1) == 0) lsum[warp * kSharedCols + c] = lacc[0];
    }
    named_bar_sync(1, kStQuads * 32);
    // per column, once: 1 / l (v_scale folded in) and the output row; the vote
    // arrays are free now
    float* einv = wmax;
    int64_t* ebase = reinterpret_cast<int64_t*>(wmax + 2 * kSharedCols);
    if (tid < kSharedCols) {
      const int n = tid;
      const float L = lsum[n] + lsum[kSharedCols + n] + lsum[2 * kSharedCols + n] +
                      lsum[3 * kSharedCols + n];
      einv[n] = L > 0.f ? p.v_mult / L : 0.f;  // an empty context gives zeros
      const int j = n / G, hh = n - j * G;
      ebase[n] = n < ncols ? (int64_t(s0 + j) * p.num_heads + kvh * G + hh) * D : -1;
    }
    named_bar_sync(1, kStQuads * 32);
    float o[kSharedCols];
#pragma unroll
    for (int n = 0; n < kSharedCols; ++n) o[n] = 0.f;
    if (nstages > 0) {
      float ot[kStPTerms][kSharedCols];
#pragma unroll
      for (int t = 0; t < kStPTerms; ++t) tmem_ld16(tl + kStTmemO + 16 * t, ot[t]);
      tmem_wait_ld();
#pragma unroll
      for (int n = 0; n < kSharedCols; ++n)
        o[n] = fmaf(fmaf(ot[2][n], 0.0625f, ot[1][n]), 0.0625f, ot[0][n]);
    }
    // Thread r holds dim r of every column.  The values go through shared memory
    // (the K ring: every S has completed, every K copy has landed) so that each
    // thread then writes 16-byte pieces of the columns' output rows instead of one
    // element of each (the entry point accepts only a 16-byte aligned output).
    {
      const int ob = p.out_dtype == PA_F32 ? 4 : 2;
      uint8_t* ost = rawk;
#pragma unroll
      for (int n = 0; n < kSharedCols; ++n) {
        const float v = o[n] * einv[n];
        if (p.out_dtype == PA_F32)
          reinterpret_cast<float*>(ost)[n * D + r] = v;
        else if (p.out_dtype == PA_F16)
          reinterpret_cast<__half*>(ost)[n * D + r] = __float2half_rn(v);
        else
          reinterpret_cast<__nv_bfloat16*>(ost)[n * D + r] = __float2bfloat16_rn(v);
      }
      named_bar_sync(1, kStQuads * 32);
      const int per_col = D * ob / 16;  // 16-byte pieces of one column's output row
      for (int c = r; c < kSharedCols * per_col; c += kStQuads * 32) {
        const int n = c / per_col, k = c - n * per_col;
        const int64_t base = ebase[n];
        if (base >= 0)
          *reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + base * ob + k * 16) =
              *reinterpret_cast<const uint4*>(ost + n * D * ob + k * 16);
      }
    }
    if (!ok && lane == 0) atomicOr(&g_shared_err, PA_DEVERR_PIPE_TIMEOUT);
  }
  tcgen05_fence_before();
  __syncthreads();
  if (warp == kStMmaWarp) {
    tcgen05_fence_after();
    tmem_dealloc(tmem, kStTmemCols);
  }
}

template <typename CT, typename QT>
int launch_shared_typed(const SharedParams& base, int grid_x, cudaStream_t stream) {
  constexpr bool fp8 = CacheTraits<CT>::bytes == 1;
  constexpr int stages = fp8 ? kSharedStagesFp8 : kSharedStages16;
  constexpr size_t smem = shared_smem_bytes<CT, stages>();
  auto kern = decode_shared_prefix_kernel<CT, QT, stages>;
  static std::atomic<unsigned long long> smem_set{0};
  if (set_smem_once(kern, smem, smem_set) != PA_OK) return PA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid_x) * unsigned(base.cluster), unsigned(base.p.num_kv_heads));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = unsigned(base.cluster);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, base);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

int launch_decode_shared_prefix(const DecodeArgs& a, const int32_t* group_starts,
                                const int32_t* prefix_lens, int num_groups, int max_group_size,
                                cudaStream_t stream) {
  const int group = a.num_heads / a.num_kv_heads;
  const int64_t rows = a.num_blocks * a.num_kv_heads * a.block_size;
  if (a.head_dim != 128 || group > kSharedCols || rows >= (int64_t(1) << 31) ||
      encode_fn() == nullptr)
    return PA_ERR_UNSUPPORTED;
  SharedParams sp;
  memset(&sp, 0, sizeof sp);
  Params& p = sp.p;
  p.out = a.out;
  p.query = static_cast<const uint8_t*>(a.query);
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
  p.head_groups = 1;
  p.partition = a.max_seq_len > 0 ? a.max_seq_len : 1;
  p.max_parts = 1;
  p.out_dtype = a.out_dtype;
  p.num_blocks = a.num_blocks;
  p.num_seqs = a.num_seqs;
  const bool fp8 = a.cache_dtype == PA_FP8_E4M3;
  p.q_mult = a.scale * kLog2e * (fp8 ? a.k_scale : 1.f);
  p.v_mult = fp8 ? a.v_scale : 1.f;
  sp.group_starts = group_starts;
  sp.prefix_lens = prefix_lens;
  sp.seqs_per_cta = kSharedCols / group;
  sp.ctas_per_group = (max_group_size + sp.seqs_per_cta - 1) / sp.seqs_per_cta;
  const int64_t grid_x = int64_t(num_groups) * sp.ctas_per_group;
  // Split each unit's block stream over a cluster of up to 8 CTAs when there are
  // too few units to keep the GPU streaming, keeping chunks of at least
  // PA_SHARED_MIN_CHUNK blocks.
  {
    const int64_t units = grid_x * a.num_kv_heads;
    int c = int((kAutoTargetCtas + units - 1) / (units > 0 ? units : 1));
    const int est_blocks = (a.max_seq_len + kBlockSize - 1) / kBlockSize;
    c = min(c, max(1, est_blocks / PA_SHARED_MIN_CHUNK));
    sp.cluster = max(1, min(c, 8));
  }
  if (grid_x * sp.cluster > INT32_MAX) return PA_ERR_UNSUPPORTED;
  if (!encode_pool_map(&sp.tmk, a.key_cache, rows, fp8) ||
      !encode_pool_map(&sp.tmv, a.value_cache, rows, fp8))
    return PA_ERR_CUDA;
  if (fp8 && (a.q_dtype == PA_F16 || a.q_dtype == PA_BF16) && !fallback_kernels_forced()) {
    // the tensor-core kernel: no cluster split.  Its register split assumes the CTA
    // is launched with kStLaunchRegs a thread (a split above the launch's registers
    // would wait forever); a build whose kernel has another count takes the
    // mma.sync kernel below.  Checked once per kernel.
    const dim3 grid(unsigned(grid_x), unsigned(a.num_kv_heads));
    auto launch_tc = [&](auto kern, size_t smem, std::atomic<unsigned long long>& mask,
                         std::atomic<int>& regs) -> int {
      int r = regs.load(std::memory_order_relaxed);
      if (r == 0) {
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return PA_ERR_CUDA;
        r = fa.numRegs == kStLaunchRegs ? 1 : -1;
        regs.store(r, std::memory_order_relaxed);
      }
      if (r < 0) return PA_ERR_UNSUPPORTED;
      SharedParams tcp = sp;
      tcp.cluster = 1;
      if (set_smem_once(kern, smem, mask) != PA_OK) return PA_ERR_CUDA;
      const cudaError_t e = launch_dependent(kern, grid, dim3(kStThreads), smem, stream, tcp);
      return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
    };
    static std::atomic<unsigned long long> done_h{0}, done_b{0};
    static std::atomic<int> regs_h{0}, regs_b{0};
    const int rc = a.q_dtype == PA_F16
                       ? launch_tc(decode_shared_tc_kernel<__half>, shared_tc_smem_bytes<3>(),
                                   done_h, regs_h)
                       : launch_tc(decode_shared_tc_kernel<__nv_bfloat16>,
                                   shared_tc_smem_bytes<2>(), done_b, regs_b);
    if (rc != PA_ERR_UNSUPPORTED) return rc;
  }
  if (a.cache_dtype == PA_F16 && a.q_dtype == PA_F16)
    return launch_shared_typed<__half, __half>(sp, int(grid_x), stream);
  if (a.cache_dtype == PA_BF16 && a.q_dtype == PA_BF16)
    return launch_shared_typed<__nv_bfloat16, __nv_bfloat16>(sp, int(grid_x), stream);
  if (fp8 && a.q_dtype == PA_F16) return launch_shared_typed<fp8_e4m3, __half>(sp, int(grid_x), stream);
  if (fp8 && a.q_dtype == PA_BF16)
    return launch_shared_typed<fp8_e4m3, __nv_bfloat16>(sp, int(grid_x), stream);
  return PA_ERR_UNSUPPORTED;
}

cudaError_t read_and_clear_shared_errors(unsigned* bits, cudaStream_t stream) {
  unsigned v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_shared_err, sizeof v, 0,
                                            cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  const unsigned zero = 0;
  e = cudaMemcpyToSymbolAsync(g_shared_err, &zero, sizeof zero, 0, cudaMemcpyHostToDevice,
                              stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  *bits |= v;
  return e;
}

}  // namespace pa
