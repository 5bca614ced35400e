// pa_prefill.cu -- multi-query (chunked prefill) attention over the paged cache
// for sm_100a: a 64-row mma.sync kernel for short chunks and a persistent
// 128-row tcgen05 kernel (TMEM accumulators) for the rest.

#include "pa_fallback.h"
#include "pa_kernels.cuh"
#include "pa_tcgen05.cuh"

namespace pa {
namespace {

__device__ unsigned int g_prefill_err;

// ---------------------------------------------------------------------------
// Multi-query attention over the paged cache (chunked prefill: several query
// tokens per sequence, each attending causally; "vLLM推理引擎PagedAttention原理与
// 性能优化实战" sec 6).  Sequence i's query rows are query_start[i] .. [i+1] - 1;
// row j sits at position L - q + j.  One CTA serves 64 (query token, head) rows of
// one kv head: row r is token r / G, head r % G of the group.  Each of the four
// consumer warps owns 16 rows for the whole pass (FlashAttention-2 layout over
// paged tiles): S = Q K^T and O += P V as mma.sync m16n8k16 per 16-token tile, P
// going straight from the S accumulator into the A operand, fp32 online softmax
// per row, causal and context masks.  Every staged tile is read by all four warps.
// ---------------------------------------------------------------------------
struct PrefillParams {
  CUtensorMap tmk;
  CUtensorMap tmv;
  Params p;
  const int32_t* query_start;  // [num_seqs + 1]
  int row_blocks;              // CTAs per (sequence, kv head): ceil(max rows / 64)
};

constexpr int kPrefillRows = kConsumerWarps * 16;

template <typename CT, int kStages>
constexpr size_t prefill_smem_bytes() {
  return 1024 + 2 * kStages * size_t(kBlockSize) * 128 * CacheTraits<CT>::bytes +
         2 * kStages * sizeof(uint64_t);
}

template <typename CT, int kStages>
__global__ void __launch_bounds__(kThreads) prefill_kernel(const __grid_constant__ PrefillParams pp) {
  constexpr int D = 128;
  constexpr int TILE = kBlockSize * D * CacheTraits<CT>::bytes;
  static_assert(CacheTraits<CT>::bytes == 2, "16-bit caches");
  using MT = CT;
  constexpr bool kSplitP = std::is_same<MT, __nv_bfloat16>::value;
  const Params& p = pp.p;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* kbuf = smem;
  uint8_t* vbuf = smem + kStages * TILE;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + 2 * kStages * TILE);
  uint64_t* empty = full + kStages;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seq = blockIdx.x / pp.row_blocks;
  const int rblk = blockIdx.x - seq * pp.row_blocks;
  const int kvh = blockIdx.y;
  const int G = p.group;
  const int32_t* table_row = p.block_tables + int64_t(seq) * p.max_blocks_per_seq;

  const int cap = p.cap;
  int L = p.seq_lens[seq];
  const int q0 = pp.query_start[seq];
  int nq = pp.query_start[seq + 1] - q0;
  if (L < 0 || L > cap || nq < 0 || nq > L) {
    if (tid == 0 && rblk == 0 && kvh == 0) atomicOr(&g_prefill_err, PA_DEVERR_SEQ_LEN);
    L = L < 0 ? 0 : (L > cap ? cap : L);
    nq = nq < 0 ? 0 : (nq > L ? L : nq);
  }
  const int rows = nq * G;
  const int row0 = rblk * kPrefillRows;
  if (row0 >= rows) return;
  // positions: row r -> token r / G at L - nq + r / G; tiles up to the CTA's last row
  const int pos_last = L - nq + (min(rows, row0 + kPrefillRows) - 1) / G;
  const int nblk = pos_last / kBlockSize + 1;

  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kConsumerWarps);  // every consumer warp reads every tile
    }
    fence_barrier_init();
  }
  __syncthreads();

  const int g = lane >> 2, c = lane & 3;
  const int mi = lane >> 3, r = lane & 7;

  if (warp == kConsumerWarps) {
    // ---------------- producer: tiles 0 .. nblk-1 of the sequence ----------------
    const uint64_t policy = l2_policy_evict_last();  // re-read by the other row blocks
    int issued = 0;
    bool ok = true;
    for (int base = 0; base < nblk && ok; base += 32) {
      int tile = 0;
      if (base + lane < nblk) {
        const int t = base + lane, e = t / p.tiles_per_block;
        int32_t phys = table_row[e];
        if (phys < 0 || phys >= p.num_blocks) {
          atomicOr(&g_prefill_err, PA_DEVERR_BLOCK_RANGE);
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
            atomicOr(&g_prefill_err, PA_DEVERR_PIPE_TIMEOUT);
            ok = false;
          }
          if (ok) {
            const int row = tl * kBlockSize;
            uint8_t* kd = kbuf + stage * TILE;
            uint8_t* vd = vbuf + stage * TILE;
            mbar_arrive_expect_tx(&full[stage], 2 * TILE);
            tma_load_2d(kd, &pp.tmk, 0, row, &full[stage], policy);
            tma_load_2d(kd + TILE / 2, &pp.tmk, 64, row, &full[stage], policy);
            tma_load_2d(vd, &pp.tmv, 0, row, &full[stage], policy);
            tma_load_2d(vd + TILE / 2, &pp.tmv, 64, row, &full[stage], policy);
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
          atomicOr(&g_prefill_err, PA_DEVERR_PIPE_TIMEOUT);
    }
    return;
  }

  // ---------------- consumers: 16 rows per warp ----------------
  const int ra = row0 + warp * 16 + g, rb = ra + 8;  // this thread's two rows
  const bool va = ra < rows, vb = rb < rows;
  const int pa_pos = L - nq + ra / G, pb_pos = L - nq + rb / G;
  const int wlast = min(rows, row0 + warp * 16 + 16) - 1;  // the warp's last row
  const int wpos = wlast >= row0 + warp * 16 ? L - nq + wlast / G : -1;
  auto qrow = [&](int rr) {
    return p.query + (int64_t(q0 + rr / G) * p.num_heads + kvh * G + rr % G) * D * 2;
  };
  uint32_t qa[8][4];
  {
    const uint8_t* ya = qrow(va ? ra : row0);
    const uint8_t* yb = qrow(vb ? rb : row0);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qa[ks][0] = va ? *reinterpret_cast<const uint32_t*>(ya + (16 * ks + 2 * c) * 2) : 0u;
      qa[ks][1] = vb ? *reinterpret_cast<const uint32_t*>(yb + (16 * ks + 2 * c) * 2) : 0u;
      qa[ks][2] = va ? *reinterpret_cast<const uint32_t*>(ya + (16 * ks + 2 * c + 8) * 2) : 0u;
      qa[ks][3] = vb ? *reinterpret_cast<const uint32_t*>(yb + (16 * ks + 2 * c + 8) * 2) : 0u;
    }
  }
  const float mult = p.q_mult;
  float acc[16][4];
#pragma unroll
  for (int t = 0; t < 16; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  float ma = -INFINITY, mb = -INFINITY, la = 0.f, lb = 0.f;

  for (int i = 0; i < nblk; ++i) {
    const int stage = i % kStages;
    if (!__all_sync(kFullMask, mbar_wait_bounded(&full[stage], (i / kStages) & 1))) {
      if (lane == 0) atomicOr(&g_prefill_err, PA_DEVERR_PIPE_TIMEOUT);
      break;
    }
    if (i * kBlockSize <= wpos) {  // some row of this warp sees part of this tile
      const uint32_t kt = smem_u32(kbuf + stage * TILE);
      const uint32_t vt = smem_u32(vbuf + stage * TILE);
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int tok = r + 8 * (mi >> 1), j = 2 * ks + (mi & 1);
        uint32_t b[4];
        ldsm_x4(kt + (j >> 3) * (TILE / 2) + tok * 128 + (((j & 7) ^ r) << 4), b);
        mma_16816(sc[0], qa[ks], b[0], b[1], MT{});
        mma_16816(sc[1], qa[ks], b[2], b[3], MT{});
      }
      // causal and context masks: token position tp is visible to a row at pos if tp <= pos
      float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int tp = i * kBlockSize + nt * 8 + 2 * c + e;
          sc[nt][e] = (va && tp <= pa_pos) ? sc[nt][e] * mult : -INFINITY;
          sc[nt][2 + e] = (vb && tp <= pb_pos) ? sc[nt][2 + e] * mult : -INFINITY;
          mxa = fmaxf(mxa, sc[nt][e]);
          mxb = fmaxf(mxb, sc[nt][2 + e]);
        }
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        mxa = fmaxf(mxa, __shfl_xor_sync(kFullMask, mxa, o));
        mxb = fmaxf(mxb, __shfl_xor_sync(kFullMask, mxb, o));
      }
      const float mna = fmaxf(ma, mxa), mnb = fmaxf(mb, mxb);
      const float ala = mna == -INFINITY ? 1.f : exp2f(ma - mna);
      const float alb = mnb == -INFINITY ? 1.f : exp2f(mb - mnb);
      ma = mna;
      mb = mnb;
      float pr[2][4];
      float suma = 0.f, sumb = 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          pr[nt][e] = mna == -INFINITY ? 0.f : exp2f(sc[nt][e] - mna);
          pr[nt][2 + e] = mnb == -INFINITY ? 0.f : exp2f(sc[nt][2 + e] - mnb);
          suma += pr[nt][e];
          sumb += pr[nt][2 + e];
        }
      la = la * ala + suma;
      lb = lb * alb + sumb;
      // P as the A operand (rows x 16 tokens): the S accumulator layout, repacked
      uint32_t ph[4] = {pack2(pr[0][0], pr[0][1], MT{}), pack2(pr[0][2], pr[0][3], MT{}),
                        pack2(pr[1][0], pr[1][1], MT{}), pack2(pr[1][2], pr[1][3], MT{})};
      uint32_t pl[4] = {0u, 0u, 0u, 0u};
      if constexpr (kSplitP) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int nt = q >> 1, hr = (q & 1) * 2;
          const float2 h = unpack2(ph[q], MT{});
          pl[q] = pack2(pr[nt][hr] - h.x, pr[nt][hr + 1] - h.y, MT{});
        }
      }
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        acc[t][0] *= ala;
        acc[t][1] *= ala;
        acc[t][2] *= alb;
        acc[t][3] *= alb;
      }
      // V rows past the context may hold anything (NaN): zero them in the B operand
      const int nvalid = min(kBlockSize, L - i * kBlockSize);
      uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
      if (nvalid < kBlockSize) {
        mlo = (2 * c < nvalid ? 0x0000ffffu : 0u) | (2 * c + 1 < nvalid ? 0xffff0000u : 0u);
        mhi = (2 * c + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * c + 9 < nvalid ? 0xffff0000u : 0u);
      }
#pragma unroll
      for (int dt = 0; dt < 8; ++dt) {
        const int tok = r + 8 * (mi & 1), j = 2 * dt + (mi >> 1);
        uint32_t b[4];
        ldsm_x4_trans(vt + (j >> 3) * (TILE / 2) + tok * 128 + (((j & 7) ^ r) << 4), b);
        b[0] &= mlo;
        b[1] &= mhi;
        b[2] &= mlo;
        b[3] &= mhi;
        mma_16816(acc[2 * dt], ph, b[0], b[1], MT{});
        mma_16816(acc[2 * dt + 1], ph, b[2], b[3], MT{});
        if constexpr (kSplitP) {
          mma_16816(acc[2 * dt], pl, b[0], b[1], MT{});
          mma_16816(acc[2 * dt + 1], pl, b[2], b[3], MT{});
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
  }
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    la += __shfl_xor_sync(kFullMask, la, o);
    lb += __shfl_xor_sync(kFullMask, lb, o);
  }
  const float ia = la > 0.f ? p.v_mult / la : 0.f, ib = lb > 0.f ? p.v_mult / lb : 0.f;
#pragma unroll
  for (int t = 0; t < 16; ++t) {
    const int d = 8 * t + 2 * c;
    if (va) {
      const int64_t o = (int64_t(q0 + ra / G) * p.num_heads + kvh * G + ra % G) * D + d;
      store_out(p.out, o, acc[t][0] * ia, p.out_dtype);
      store_out(p.out, o + 1, acc[t][1] * ia, p.out_dtype);
    }
    if (vb) {
      const int64_t o = (int64_t(q0 + rb / G) * p.num_heads + kvh * G + rb % G) * D + d;
      store_out(p.out, o, acc[t][2] * ib, p.out_dtype);
      store_out(p.out, o + 1, acc[t][3] * ib, p.out_dtype);
    }
  }
}

// ---------------------------------------------------------------------------
// Chunked prefill on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// For chunks with at least 128 (query token, head) rows per kv head the
// contraction is large enough for the CTA-wide MMA.  A tile is 128 rows of one kv
// head (one TMEM lane each); the kernel is persistent, one CTA per SM walking a
// round-robin share of the tiles, and each tile walks its sequence's KV in stages
// of kTcKv tokens (kTcKv / 16 pool tiles placed by TMA as 128-byte-swizzled
// operands):
//   S[128 x kTcKv] = Q[128 x 128] . K^T    A = Q from TMEM (stored once per tile, two
//                                          slots), B = K from shared memory; fp32 S
//                                          in TMEM, two buffers
//   O[128 x 128]  += P[128 x kTcKv] . V    A = P from TMEM (written over its own S),
//                                          B = V from shared memory (MN-major); O
//                                          stays in TMEM for the whole tile
// Shared memory therefore feeds only K and V.  K and V have rings and producer
// warps of their own, so a K slot refills as soon as its S is done and a V slot as
// soon as its P.V is done, straight on across tiles.  Eight softmax warps, two per
// TMEM lane quadrant, each take 32 rows x kTcKv / 2 columns (the row max of the
// two halves meets in shared memory behind a 64-thread named barrier): masks,
// fp32 online softmax in the exp2 domain, P as 16-bit pairs into TMEM.  P is taken
// relative to a per-row reference max that moves only when a new score exceeds it
// by more than 2^8, so O in TMEM is rescaled rarely.  The next tile's Q goes into
// its TMEM slot before this tile's epilogue, so the next S overlaps the epilogue.
// One thread polls the barriers and issues each S and P.V as soon as its inputs
// are ready (tcgen05.commit reports completion), sleeping in try_wait otherwise.
// All waits are bounded, and the named barriers are reached the same number of
// times on every path.
// kSplitP (bf16 operands with an fp32 output): P is held as two bf16 terms, hi
// and lo = P - hi (stored over the second half of the same S buffer), and P.V
// takes both, so the 16-bit rounding of P (relative 2^-9 in bf16) does not reach
// a full-precision output.
// ---------------------------------------------------------------------------
constexpr int kTcRows = 128;                   // query rows per CTA = TMEM lanes
#ifndef PA_TC_KV
#define PA_TC_KV 128
#endif
constexpr int kTcKv = PA_TC_KV;                // tokens per KV stage (N of the S MMA)
static_assert(kTcKv == 64 || kTcKv == 128, "stage of 64 or 128 tokens");
constexpr int kTcTiles = kTcKv / kBlockSize;   // 16-token pool tiles per stage
constexpr int kTcHalf = kTcKv / 2;             // S columns per softmax warp
#ifndef PA_TC_STAGES
#define PA_TC_STAGES (PA_TC_KV == 128 ? 2 : 4)
#endif
constexpr int kTcStages = PA_TC_STAGES;        // K and V rings
constexpr int kTcSoftmaxWarps = 8;             // two per TMEM lane quadrant
constexpr int kTcThreads = (kTcSoftmaxWarps + 3) * 32;  // + K loads, MMA, V loads
constexpr int kTcKWarp = kTcSoftmaxWarps;
constexpr int kTcMmaWarp = kTcSoftmaxWarps + 1;
constexpr int kTcVWarp = kTcSoftmaxWarps + 2;
constexpr uint32_t kTcTmemCols = 512;          // S (then P): 2 x kTcKv, O: 128, Q: 2 x 64
constexpr uint32_t kTcTmemO = 2 * kTcKv;       // first column of O
constexpr uint32_t kTcTmemQ = 2 * kTcKv + 128; // Q slot b at kTcTmemQ + 64 b (16-bit pairs)
static_assert(kTcTmemQ + 128 <= kTcTmemCols, "TMEM budget");
constexpr int kTcTileBytes = 2 * kTcKv * 128;  // K or V of a stage: [2 halves][kTcKv rows][128 B]
constexpr float kTcRescaleLog2 = 8.f;          // reference max moves beyond 2^8
constexpr uint32_t kTcPollNs = 500;            // MMA issuer's longest sleep per poll

// Packed fp32 pairs (sm_100): one instruction does the work of two, each lane
// IEEE round-to-nearest like fmaf / fadd; and the three-input maximum.
__device__ __forceinline__ unsigned long long f2_bits(float2 a) {
  unsigned long long u;
  asm("mov.b64 %0, {%1, %2};" : "=l"(u) : "f"(a.x), "f"(a.y));
  return u;
}
__device__ __forceinline__ float2 bits_f2(unsigned long long u) {
  float2 a;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a.x), "=f"(a.y) : "l"(u));
  return a;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)),
      "l"(f2_bits(c)));
  return bits_f2(r);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(r);
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

struct TcPrefillParams {
  CUtensorMap tmk;
  CUtensorMap tmv;
  Params p;
  const int32_t* query_start;
  int row_blocks;  // 128-row tiles per (sequence, kv head)
  int num_tiles;   // num_seqs * num_kv_heads * row_blocks
};

constexpr size_t tc_prefill_smem_bytes() {
  return 1024 + 2 * size_t(kTcStages) * kTcTileBytes + 6 * kTcRows * sizeof(float) +
         (4 * kTcStages + 9) * sizeof(uint64_t) + 16;
}

// One 128-row tile: tile = (seq * num_kv_heads + kvh) * row_blocks + row block, so
// consecutive tiles share a sequence's KV (read through L2).
struct TcTile {
  int seq, kvh, q0, nq, L, rows, row0, pos_last, ntiles, nkb;
};

__device__ __forceinline__ bool tc_tile(const TcPrefillParams& pp, int tile, TcTile& t,
                                        bool report) {
  const Params& p = pp.p;
  const int per_seq = p.num_kv_heads * pp.row_blocks;
  t.seq = tile / per_seq;
  const int rem = tile - t.seq * per_seq;
  t.kvh = rem / pp.row_blocks;
  const int rblk = rem - t.kvh * pp.row_blocks;
  const int cap = p.cap;
  int L = p.seq_lens[t.seq];
  t.q0 = pp.query_start[t.seq];
  int nq = pp.query_start[t.seq + 1] - t.q0;
  if (L < 0 || L > cap || nq < 0 || nq > L) {
    if (report && rblk == 0 && t.kvh == 0) atomicOr(&g_prefill_err, PA_DEVERR_SEQ_LEN);
    L = L < 0 ? 0 : (L > cap ? cap : L);
    nq = nq < 0 ? 0 : (nq > L ? L : nq);
  }
  t.L = L;
  t.nq = nq;
  t.rows = nq * p.group;
  t.row0 = rblk * kTcRows;
  if (t.row0 >= t.rows) return false;  // a short sequence's unused row block
  t.pos_last = L - nq + (min(t.rows, t.row0 + kTcRows) - 1) / p.group;
  t.ntiles = t.pos_last / kBlockSize + 1;
  t.nkb = (t.pos_last + kTcKv) / kTcKv;
  return true;
}

// The next non-empty tile of this CTA's round-robin share after `tile` (or the
// first one when tile < 0); false when none is left.
__device__ __forceinline__ bool tc_next_tile(const TcPrefillParams& pp, int& tile, TcTile& t,
                                             bool report) {
  for (tile = tile < 0 ? int(blockIdx.x) : tile + int(gridDim.x); tile < pp.num_tiles;
       tile += gridDim.x)
    if (tc_tile(pp, tile, t, report)) return true;
  return false;
}

// A walk over this CTA's stages in order: (tile, stage within the tile), plus the
// count of tiles begun (which selects the Q slot).
struct TcCursor {
  int tile = -1, jb = 0, nkb = 0, tcount = -1;
  bool valid = false;
  __device__ __forceinline__ void advance(const TcPrefillParams& pp) {
    if (valid && ++jb < nkb) return;
    TcTile t;
    valid = tc_next_tile(pp, tile, t, false);
    jb = 0;
    nkb = valid ? t.nkb : 0;
    ++tcount;
  }
};

static_assert(kTcStages >= 2 && tc_prefill_smem_bytes() <= 227 * 1024, "rings fit 227 KB");

// Q rows of a tile into TMEM slot `slot` as the A operand of S: thread (half h,
// row r) stores d in [64h, 64h + 64) as 32 columns of 16-bit pairs.  A negative
// scale is applied as |scale| to -Q (a sign flip is exact), so the softmax may
// take the row max before scaling.
__device__ __forceinline__ void tc_store_q(const Params& p, const TcTile& t, uint32_t tl,
                                           uint32_t slot, int r, int h) {
  constexpr int D = 128;
  const int gr = t.row0 + r;
  const bool valid = gr < t.rows;
  const int G = p.group;
  const uint4* src = reinterpret_cast<const uint4*>(
      p.query + (int64_t(t.q0 + (valid ? gr / G : 0)) * p.num_heads + t.kvh * G +
                 (valid ? gr % G : 0)) * D * 2) + 8 * h;
  const uint32_t flip = p.q_mult < 0.f ? 0x80008000u : 0u;
  float qv[32];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 v = valid ? src[c] : make_uint4(0u, 0u, 0u, 0u);
    qv[4 * c + 0] = __uint_as_float(v.x ^ flip);
    qv[4 * c + 1] = __uint_as_float(v.y ^ flip);
    qv[4 * c + 2] = __uint_as_float(v.z ^ flip);
    qv[4 * c + 3] = __uint_as_float(v.w ^ flip);
  }
  tmem_st32(tl + kTcTmemQ + 64 * slot + 32 * h, qv);
  tmem_wait_st();
}

template <typename CT, bool kSplitP>
__global__ void __launch_bounds__(kTcThreads, 1)
    prefill_tc_kernel(const __grid_constant__ TcPrefillParams pp) {
  constexpr int D = 128;
  static_assert(CacheTraits<CT>::bytes == 2, "16-bit caches");
  constexpr uint32_t kFmt = std::is_same<CT, __nv_bfloat16>::value ? 1u : 0u;
  constexpr uint32_t kIdescS = umma_idesc_f16(kFmt, 0, kTcRows, kTcKv);
  constexpr uint32_t kIdescPV = umma_idesc_f16(kFmt, 1, kTcRows, D);
  const Params& p = pp.p;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* ksm = smem;                                  // K ring
  uint8_t* vsm = ksm + kTcStages * kTcTileBytes;        // V ring
  float* xmax = reinterpret_cast<float*>(vsm + kTcStages * kTcTileBytes);  // [2][2 halves][128]
  float* lsum = xmax + 4 * kTcRows;                     // [2 halves][128]
  uint64_t* kfull = reinterpret_cast<uint64_t*>(lsum + 2 * kTcRows);
  uint64_t* kempty = kfull + kTcStages;
  uint64_t* vfull = kempty + kTcStages;
  uint64_t* vempty = vfull + kTcStages;
  uint64_t* s_full = vempty + kTcStages;  // [2]: S of stage g (buffer g & 1) written
  uint64_t* o_full = s_full + 2;          // [2]: P.V of stage g done
  uint64_t* p_ready = o_full + 2;         // [2]: P of stage g in TMEM, O rescaled
  uint64_t* q_ready = p_ready + 2;        // [2]: Q of this CTA's tile number c in slot c & 1
  uint64_t* done = q_ready + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int st = 0; st < kTcStages; ++st) {
      mbar_init(&kfull[st], 1);
      mbar_init(&kempty[st], 1);
      mbar_init(&vfull[st], 1);
      mbar_init(&vempty[st], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&o_full[b], 1);
      mbar_init(&p_ready[b], kTcSoftmaxWarps);
      mbar_init(&q_ready[b], kTcSoftmaxWarps);
    }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == kTcMmaWarp) {  // the MMA warp owns the TMEM allocation
    tmem_alloc(tmem_slot, kTcTmemCols);
    tmem_relinquish();
  }
  tcgen05_fence_before();
  __syncthreads();
  tcgen05_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kTcKWarp || warp == kTcVWarp) {
    // ---------------- TMA producers: stage = sequence tiles 16 j .. 16 j + 15 ----------------
    // one warp fills the K ring, the other the V ring, each at its own pace and
    // straight on into the next tile
    const bool is_k = warp == kTcKWarp;
    const CUtensorMap* map = is_k ? &pp.tmk : &pp.tmv;
    uint8_t* ring = is_k ? ksm : vsm;
    uint64_t* full = is_k ? kfull : vfull;
    uint64_t* empty = is_k ? kempty : vempty;
    const uint64_t policy = l2_policy_evict_last();  // other row blocks read it again
    constexpr int kPre = 32 / kTcTiles;  // stages covered by one table read per lane
    int g = 0;                           // stages issued by this CTA
    bool ok = true;
    int tile = -1;
    TcTile t;
    while (ok && tc_next_tile(pp, tile, t, is_k && lane == 0)) {
      const int32_t* table_row = p.block_tables + int64_t(t.seq) * p.max_blocks_per_seq;
      int ent = 0;  // this lane's pool tile of the current group of 32 tiles
      for (int jb = 0; jb < t.nkb && ok; ++jb, ++g) {
        const int stage = g % kTcStages;
        const int ntl = min(kTcTiles, t.ntiles - kTcTiles * jb);
        if (jb % kPre == 0) {
          const int tt = kTcTiles * jb + lane;
          ent = 0;
          if (tt < t.ntiles) {
            const int e = tt / p.tiles_per_block;
            int32_t phys = table_row[e];
            if (phys < 0 || phys >= p.num_blocks) {
              if (is_k) atomicOr(&g_prefill_err, PA_DEVERR_BLOCK_RANGE);
              phys = 0;
            }
            ent = (phys * p.num_kv_heads + t.kvh) * p.tiles_per_block +
                  (tt - e * p.tiles_per_block);
          }
        }
        int tls[kTcTiles];
#pragma unroll
        for (int i = 0; i < kTcTiles; ++i)
          tls[i] = __shfl_sync(kFullMask, ent, kTcTiles * (jb % kPre) + i);
        if (lane == 0) {
          if (g >= kTcStages && !mbar_wait_bounded(&empty[stage], ((g / kTcStages) - 1) & 1)) {
            atomicOr(&g_prefill_err, PA_DEVERR_PIPE_TIMEOUT);
            ok = false;
          }
          if (ok) {
            uint8_t* dst = ring + stage * kTcTileBytes;
            mbar_arrive_expect_tx(&full[stage], uint32_t(ntl) * 2 * 2048);
            for (int i = 0; i < ntl; ++i) {
              const int row = tls[i] * kBlockSize;
              tma_load_2d(dst + i * 2048, map, 0, row, &full[stage], policy);
              tma_load_2d(dst + kTcTileBytes / 2 + i * 2048, map, 64, row, &full[stage], policy);
            }
          }
        }
        ok = __shfl_sync(kFullMask, ok, 0);
        if (!ok) break;
      }
    }
    if (lane == 0) {  // no copy may still be landing when the CTA exits (one ring)
      for (int i = max(0, g - kTcStages); i < g; ++i)
        if (!mbar_wait_bounded(&full[i % kTcStages], (i / kTcStages) & 1))
          atomicOr(&g_prefill_err, PA_DEVERR_PIPE_TIMEOUT);
    }
  } else if (warp == kTcMmaWarp) {
    // ---------------- MMA issuer (one thread, polling) ----------------
    if (lane == 0) {
      // descriptors advance by a constant (byte offset >> 4) in the start-address field
      const uint64_t kdesc0 = umma_smem_desc(smem_u32(ksm), 16, 1024, kUmmaSwizzle128B);
      const uint64_t vdesc0 = umma_smem_desc(smem_u32(vsm), kTcTileBytes / 2, 1024,
                                             kUmmaSwizzle128B);
      TcCursor cs, cp;  // next S and next P.V
      cs.advance(pp);
      cp.advance(pp);
      int ns = 0, npv = 0, idle = 0;  // stages issued (global over this CTA's tiles)
      unsigned long long t_idle = 0;
      bool ok = true;
      while (cp.valid) {
        bool prog = false;
        // S(ns) into buffer ns & 1, whose P(ns - 2) went to P.V(ns - 2) already; the
        // first stage of a tile also needs that tile's Q
        if (cs.valid && ns <= npv + 1 &&
            (cs.jb > 0 || mbar_test(&q_ready[cs.tcount & 1], (cs.tcount >> 1) & 1)) &&
            mbar_test(&kfull[ns % kTcStages], (ns / kTcStages) & 1)) {
          tcgen05_fence_after();
          const uint64_t kd = kdesc0 + uint64_t(((ns % kTcStages) * kTcTileBytes) >> 4);
          const uint32_t d = tmem + uint32_t(ns & 1) * kTcKv;
          const uint32_t qa = tmem + kTcTmemQ + 64 * uint32_t(cs.tcount & 1);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            umma_f16_ts(d, qa + uint32_t(8 * ks),
                        kd + uint64_t(((ks >> 2) * (kTcTileBytes / 2) + (ks & 3) * 32) >> 4),
                        kIdescS, ks > 0 ? 1u : 0u);
          umma_commit(&s_full[ns & 1]);
          umma_commit(&kempty[ns % kTcStages]);
          ++ns;
          cs.advance(pp);
          prog = true;
        }
        // P.V(npv): P from TMEM over S buffer npv & 1, V from its ring slot; the
        // first stage of a tile writes O, the others accumulate
        if (npv < ns && mbar_test(&p_ready[npv & 1], (npv >> 1) & 1) &&
            mbar_test(&vfull[npv % kTcStages], (npv / kTcStages) & 1)) {
          tcgen05_fence_after();
          const uint64_t vd = vdesc0 + uint64_t(((npv % kTcStages) * kTcTileBytes) >> 4);
          const uint32_t pt = tmem + uint32_t(npv & 1) * kTcKv;
#pragma unroll
          for (int t = 0; t < (kSplitP ? 2 : 1); ++t) {
#pragma unroll
            for (int ks = 0; ks < kTcKv / 16; ++ks)
              umma_f16_ts(tmem + kTcTmemO, pt + uint32_t(t * (kTcKv / 2) + ks * 8),
                          vd + uint64_t((ks * 2048) >> 4), kIdescPV,
                          (cp.jb > 0 || t > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(&o_full[npv & 1]);
          umma_commit(&vempty[npv % kTcStages]);
          ++npv;
          cp.advance(pp);
          prog = true;
        }
        if (prog) {
          idle = 0;
          continue;
        }
        // sleep (no issue slots taken from the softmax warps) on the barrier the
        // next step most likely waits for: P of the oldest stage once its S is out
        if (npv < ns)
          mbar_try_wait(&p_ready[npv & 1], (npv >> 1) & 1, kTcPollNs);
        else
          mbar_try_wait(&kfull[ns % kTcStages], (ns / kTcStages) & 1, kTcPollNs);
        if (idle == 0) t_idle = global_timer_ns();
        if ((++idle & 63) == 0 && global_timer_ns() - t_idle > kWaitLimitNs) {
          ok = false;
          break;
        }
      }
      if (!ok) atomicOr(&g_prefill_err, PA_DEVERR_PIPE_TIMEOUT);
      umma_commit(done);  // fires once every MMA issued above has completed
    }
    __syncwarp();
  } else {
    // ---------------- softmax warps: thread = (row, column half) ----------------
    const int h = warp >> 2, qd = warp & 3;
    const int r = 32 * qd + lane;  // TMEM lane and row within a tile
    const uint32_t tl = tmem + (uint32_t(32 * qd) << 16);  // this warp's lane quadrant
    const uint32_t pair_bar = 1 + qd;                       // this warp and warp qd + 4*(1-h)
    const float mult = fabsf(p.q_mult);  // Q carries the sign
    bool ok = true;                      // warp-uniform; after a failure waits are skipped,
                                         // but every named barrier is still reached
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      if (ok) ok = __all_sync(kFullMask, mbar_wait_bounded(bar, parity));
    };
    auto arrive = [&](uint64_t* bar) {
      tcgen05_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    int tile = -1, g = 0, tc = 0;
    TcTile t;
    bool have = tc_next_tile(pp, tile, t, false);
    if (have) {
      tc_store_q(p, t, tl, 0, r, h);
      arrive(&q_ready[0]);
    }
    while (have) {
      const int gr = t.row0 + r;
      const bool valid = gr < t.rows;
      const int pos = valid ? t.L - t.nq + gr / p.group : -1;
      float m = -INFINITY, l = 0.f;  // reference max (exp2 domain), sum of this half
      for (int jb = 0; jb < t.nkb; ++jb, ++g) {
        const uint32_t sb = tl + uint32_t(g & 1) * kTcKv;  // S, then P, of this stage
        wait(&s_full[g & 1], (g >> 1) & 1);
        tcgen05_fence_after();
        float sv[kTcHalf];
#pragma unroll
        for (int q = 0; q < kTcHalf / 32; ++q) {
          float v[32];
          tmem_ld32(sb + kTcHalf * h + 32 * q, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[32 * q + i] = v[i];
        }
        tmem_wait_ld();
        // causal, context and padding mask: only stages that cross this row's last
        // visible position pay for it
        const int nvis = pos - jb * kTcKv - kTcHalf * h + 1;
        float me = mult;  // multiplier still to apply to sv
        if (nvis < kTcHalf) {
#pragma unroll
          for (int i = 0; i < kTcHalf; ++i) sv[i] = i < nvis ? sv[i] * mult : -INFINITY;
          me = 1.f;
        }
        float r8[8];  // 8 independent chains, two new columns per step
#pragma unroll
        for (int k = 0; k < 8; ++k) r8[k] = sv[k];
#pragma unroll
        for (int i = 8; i < kTcHalf; i += 2) r8[(i >> 1) & 7] = max3(r8[(i >> 1) & 7], sv[i], sv[i + 1]);
        const float pmax = fmaxf(fmaxf(fmaxf(r8[0], r8[1]), fmaxf(r8[2], r8[3])),
                                 fmaxf(fmaxf(r8[4], r8[5]), fmaxf(r8[6], r8[7]))) * me;
        float* xm = xmax + (g & 1) * 2 * kTcRows;
        xm[h * kTcRows + r] = pmax;
        named_bar_sync(pair_bar, 64);  // both halves have read S and posted their max
        const float mx = fmaxf(pmax, xm[(1 - h) * kTcRows + r]);
        if (jb == 0) {
          m = mx;  // O is written, not accumulated, by the tile's first P.V
        } else {
          const bool move = mx > m + kTcRescaleLog2;
          if (__any_sync(kFullMask, move)) {
            // rescale this warp's rows and columns of O once P.V(g - 1) has landed
            wait(&o_full[(g - 1) & 1], ((g - 1) >> 1) & 1);
            tcgen05_fence_after();
            const float f = move ? ex2_approx(m - mx) : 1.f;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              float v[32];
              tmem_ld32(tl + kTcTmemO + 64 * h + 32 * q, v);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] *= f;
              tmem_st32(tl + kTcTmemO + 64 * h + 32 * q, v);
            }
            l *= f;
            if (move) m = mx;
          }
        }
        const float mu = m == -INFINITY ? 0.f : m;
        const float2 me2 = make_float2(me, me), nmu2 = make_float2(-mu, -mu);
        float2 a4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};  // 4 chains of column pairs
#pragma unroll
        for (int c = 0; c < kTcHalf / 2; ++c) {
          const float2 x = fma2(make_float2(sv[2 * c], sv[2 * c + 1]), me2, nmu2);
          sv[2 * c] = ex2_approx(x.x);
          sv[2 * c + 1] = ex2_approx(x.y);
          a4[c & 3] = add2(a4[c & 3], make_float2(sv[2 * c], sv[2 * c + 1]));
        }
        const float2 a2 = add2(add2(a4[0], a4[1]), add2(a4[2], a4[3]));
        l += a2.x + a2.y;
        // P over the S columns both halves have read: this half's tokens as 16-bit
        // pairs in columns [h * kTcHalf / 2, (h + 1) * kTcHalf / 2), the lo term
        // kTcKv / 2 columns further on
#pragma unroll
        for (int q = 0; q < kTcHalf / 32; ++q) {
          uint32_t pw[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            pw[c] = pack2(sv[32 * q + 2 * c], sv[32 * q + 2 * c + 1], CT{});
          tmem_st16(sb + (kTcHalf / 2) * h + 16 * q, pw);
          if constexpr (kSplitP) {
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float2 hi = unpack2(pw[c], CT{});
              pw[c] = pack2(sv[32 * q + 2 * c] - hi.x, sv[32 * q + 2 * c + 1] - hi.y, CT{});
            }
            tmem_st16(sb + kTcKv / 2 + (kTcHalf / 2) * h + 16 * q, pw);
          }
        }
        if (jb == t.nkb - 1 && tid < 2 * kTcKv) {
          // V rows past the tile's last visible token may be stale or NaN: zero them
          wait(&vfull[g % kTcStages], (g / kTcStages) & 1);
          const int vr = tid >> 1, half = tid & 1;
          if (ok && jb * kTcKv + vr > t.pos_last) {
            uint8_t* vrow = vsm + (g % kTcStages) * kTcTileBytes + half * (kTcTileBytes / 2) +
                            vr * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(vrow + c * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        tmem_wait_st();
        arrive(&p_ready[g & 1]);
      }
      // the next tile's Q goes in before this tile's epilogue, so its first S can
      // run on the tensor core meanwhile (its slot's last reader, the S MMAs of the
      // tile before this one, finished before this tile's last S)
      const bool v_out = valid;
      const int64_t orow = (int64_t(t.q0 + (valid ? gr / p.group : 0)) * p.num_heads +
                            t.kvh * p.group + (valid ? gr % p.group : 0)) * D + 64 * h;
      have = tc_next_tile(pp, tile, t, false);
      if (have) {
        tc_store_q(p, t, tl, uint32_t((tc + 1) & 1), r, h);
        arrive(&q_ready[(tc + 1) & 1]);
      }
      // epilogue: O / l of this tile's rows, this warp's 64 columns
      wait(&o_full[(g - 1) & 1], ((g - 1) >> 1) & 1);
      lsum[h * kTcRows + r] = l;
      named_bar_sync(pair_bar, 64);
      const float lt = l + lsum[(1 - h) * kTcRows + r];
      named_bar_sync(pair_bar, 64);  // both read lsum before the next tile writes it
      if (ok) {
        tcgen05_fence_after();
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        uint8_t* dst = static_cast<uint8_t*>(p.out);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float v[32];
          tmem_ld32(tl + kTcTmemO + 64 * h + 32 * q, v);
          tmem_wait_ld();
          if (!v_out) continue;
          if (p.out_dtype == PA_F32) {
#pragma unroll
            for (int d = 0; d < 32; d += 4)
              *reinterpret_cast<float4*>(dst + (orow + 32 * q + d) * 4) =
                  make_float4(v[d] * inv, v[d + 1] * inv, v[d + 2] * inv, v[d + 3] * inv);
          } else if (p.out_dtype == PA_F16) {
#pragma unroll
            for (int d = 0; d < 32; d += 8)
              *reinterpret_cast<uint4*>(dst + (orow + 32 * q + d) * 2) =
                  make_uint4(pack2(v[d] * inv, v[d + 1] * inv, __half{}),
                             pack2(v[d + 2] * inv, v[d + 3] * inv, __half{}),
                             pack2(v[d + 4] * inv, v[d + 5] * inv, __half{}),
                             pack2(v[d + 6] * inv, v[d + 7] * inv, __half{}));
          } else {
#pragma unroll
            for (int d = 0; d < 32; d += 8)
              *reinterpret_cast<uint4*>(dst + (orow + 32 * q + d) * 2) =
                  make_uint4(pack2(v[d] * inv, v[d + 1] * inv, __nv_bfloat16{}),
                             pack2(v[d + 2] * inv, v[d + 3] * inv, __nv_bfloat16{}),
                             pack2(v[d + 4] * inv, v[d + 5] * inv, __nv_bfloat16{}),
                             pack2(v[d + 6] * inv, v[d + 7] * inv, __nv_bfloat16{}));
          }
        }
      }
      tcgen05_fence_before();  // O is read before the next tile's first P.V overwrites it
      ++tc;
    }
    if (!ok && lane == 0) atomicOr(&g_prefill_err, PA_DEVERR_PIPE_TIMEOUT);
  }
  // Free TMEM only after every MMA has completed and every TMEM access is done.
  __syncthreads();
  if (warp == kTcMmaWarp) {
    if (!__all_sync(kFullMask, mbar_wait_bounded(done, 0)) && lane == 0)
      atomicOr(&g_prefill_err, PA_DEVERR_PIPE_TIMEOUT);
    tcgen05_fence_after();
    tmem_dealloc(tmem, kTcTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Ping-pong form of the tcgen05 prefill: a CTA works on two 128-row tiles of one
// (sequence, kv head) at once -- row blocks 2k and 2k + 1, which share every KV
// stage -- with one softmax warpgroup per tile (warps 0-3 tile A, 4-7 tile B;
// thread = row, all 128 columns of S, read from TMEM once per stage into
// registers: setmaxnreg gives the softmax warpgroups 216 registers a thread and
// the load/MMA warpgroup 72).  TMEM holds S and O of both tiles (4 x 128
// columns); Q moves to shared memory (K-major, 128-byte swizzle) and S becomes an
// SS MMA.  The MMA thread issues, per stage j,
//     P.V_A(j), S_A(j + 1), P.V_B(j), S_B(j + 1)
// so each tile's softmax runs while the tensor core works on the other tile.  P is
// written over its own S as 16-bit pairs (two bf16 terms for kSplitP) and O stays
// in TMEM for the whole pair, rescaled per row only when the row's reference
// maximum moves by more than 2^8.  No barrier is shared between the two
// warpgroups, and a row never needs another thread.  K and V keep their rings and
// producer warps; a K stage is released after the last S that reads it, a V stage
// after the last P.V.
// ---------------------------------------------------------------------------
// Warpgroups: 0 and 1 softmax (tiles A and B), 2 the K loader, the MMA issuer, the
// V loader and one idle warp (setmaxnreg acts on whole warpgroups).  The split
// moves registers from warpgroup 2 to the softmax warpgroups, so that a thread
// holds its row's 128 scores; 72 / 216 spilled least of the splits that add up to
// the launch's registers (40 / 232: the loaders spill, 88 / 208: the softmax).
constexpr int kPpThreads = 12 * 32;
constexpr int kPpKWarp = 8;
constexpr int kPpMmaWarp = 9;
constexpr int kPpVWarp = 10;
constexpr int kPpLaunchRegs = 168;   // 65536 / 384, rounded down to 8
constexpr int kPpLoadRegs = 72;      // warpgroup 2 after setmaxnreg.dec
constexpr int kPpSoftmaxRegs = 216;  // warpgroups 0, 1 after setmaxnreg.inc
static_assert(128 * kPpLoadRegs + 256 * kPpSoftmaxRegs <= kPpThreads * kPpLaunchRegs,
              "the split draws only on the registers the CTA was launched with");
constexpr int kPpQBytes = kTcRows * 128 * 2;  // Q of a tile: [2 halves][128 rows][128 B]
constexpr uint32_t kPpTmemCols = 512;
__host__ __device__ constexpr uint32_t pp_tmem_s(int x) { return uint32_t(x) * 128; }
__host__ __device__ constexpr uint32_t pp_tmem_o(int x) { return 256 + uint32_t(x) * 128; }

constexpr size_t pp_prefill_smem_bytes() {
  return 1024 + 2 * size_t(kTcStages) * kTcTileBytes + 2 * size_t(kPpQBytes) +
         (4 * kTcStages + 11) * sizeof(uint64_t) + 16;
}
static_assert(kTcKv == 128, "one S buffer of 128 columns per tile");
static_assert(pp_prefill_smem_bytes() <= 227 * 1024, "rings and Q fit 227 KB");

// The pair of row blocks (2 pr, 2 pr + 1) of (sequence, kv head): both tiles' info.
struct PpPair {
  TcTile t[2];
  bool has[2];
  int nkb, ntiles, pos_last;  // stages, 16-token pool tiles, last visible position
};

__device__ __forceinline__ bool pp_pair(const TcPrefillParams& pp, int pair, PpPair& x,
                                        bool report) {
  const int pairs_per = (pp.row_blocks + 1) / 2;
  const int skv = pair / pairs_per, pr = pair - skv * pairs_per;  // skv = seq * Hkv + kvh
  const int base = skv * pp.row_blocks;
  x.has[0] = tc_tile(pp, base + 2 * pr, x.t[0], report);
  if (!x.has[0]) return false;
  x.has[1] = 2 * pr + 1 < pp.row_blocks && tc_tile(pp, base + 2 * pr + 1, x.t[1], false);
  const TcTile& last = x.has[1] ? x.t[1] : x.t[0];
  x.nkb = last.nkb;
  x.ntiles = last.ntiles;
  x.pos_last = last.pos_last;
  return true;
}

__device__ __forceinline__ bool pp_next(const TcPrefillParams& pp, int num_pairs, int& pair,
                                        PpPair& x, bool report) {
  for (pair = pair < 0 ? int(blockIdx.x) : pair + int(gridDim.x); pair < num_pairs;
       pair += gridDim.x)
    if (pp_pair(pp, pair, x, report)) return true;
  return false;
}

template <typename CT, bool kSplitP>
__global__ void __launch_bounds__(kPpThreads, 1)
    prefill_pp_kernel(const __grid_constant__ TcPrefillParams pp, int num_pairs) {
  constexpr int D = 128;
  static_assert(CacheTraits<CT>::bytes == 2, "16-bit caches");
  constexpr uint32_t kFmt = std::is_same<CT, __nv_bfloat16>::value ? 1u : 0u;
  constexpr uint32_t kIdescS = umma_idesc_f16(kFmt, 0, kTcRows, kTcKv);
  constexpr uint32_t kIdescPV = umma_idesc_f16(kFmt, 1, kTcRows, D);
  const Params& p = pp.p;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* ksm = smem;                                  // K ring
  uint8_t* vsm = ksm + kTcStages * kTcTileBytes;        // V ring
  uint8_t* qsm = vsm + kTcStages * kTcTileBytes;        // Q of tiles A, B
  uint64_t* kfull = reinterpret_cast<uint64_t*>(qsm + 2 * kPpQBytes);
  uint64_t* kempty = kfull + kTcStages;
  uint64_t* vfull = kempty + kTcStages;
  uint64_t* vempty = vfull + kTcStages;
  uint64_t* s_full = vempty + kTcStages;  // [2 tiles]: S of the tile's stage written
  uint64_t* o_full = s_full + 2;          // [2]: P.V of the tile's stage done
  uint64_t* p_ready = o_full + 2;         // [2]: P in TMEM, O rescaled (4 warps)
  uint64_t* q_ready = p_ready + 2;        // [2]: Q of the tile's pair in smem (4 warps)
  uint64_t* p_half = q_ready + 2;         // [2]: P of keys 0 .. 63 in TMEM (4 warps)
  uint64_t* done = p_half + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int st = 0; st < kTcStages; ++st) {
      mbar_init(&kfull[st], 1);
      mbar_init(&kempty[st], 1);
      mbar_init(&vfull[st], 1);
      mbar_init(&vempty[st], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&o_full[x], 1);
      mbar_init(&p_ready[x], 4);
      mbar_init(&q_ready[x], 4);
      mbar_init(&p_half[x], 4);
    }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == kPpMmaWarp) {  // the MMA warp owns the TMEM allocation
    tmem_alloc(tmem_slot, kPpTmemCols);
    tmem_relinquish();
  }
  tcgen05_fence_before();
  __syncthreads();
  tcgen05_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kPpLoadRegs));
  if (warp == kPpKWarp || warp == kPpVWarp) {
    // ---------------- TMA producers: stage j = pool tiles 8 j .. 8 j + 7 of the pair ----------------
    const bool is_k = warp == kPpKWarp;
    const CUtensorMap* map = is_k ? &pp.tmk : &pp.tmv;
    uint8_t* ring = is_k ? ksm : vsm;
    uint64_t* full = is_k ? kfull : vfull;
    uint64_t* empty = is_k ? kempty : vempty;
    const uint64_t policy = l2_policy_evict_last();  // the pair's other row blocks read it again
    constexpr int kPre = 32 / kTcTiles;
    int g = 0;
    bool ok = true;
    int pair = -1;
    PpPair x;
    while (ok && pp_next(pp, num_pairs, pair, x, is_k && lane == 0)) {
      const TcTile& t = x.t[0];
      const int32_t* table_row = p.block_tables + int64_t(t.seq) * p.max_blocks_per_seq;
      int ent = 0;
      for (int jb = 0; jb < x.nkb && ok; ++jb, ++g) {
        const int stage = g % kTcStages;
        const int ntl = min(kTcTiles, x.ntiles - kTcTiles * jb);
        if (jb % kPre == 0) {
          const int tt = kTcTiles * jb + lane;
          ent = 0;
          if (tt < x.ntiles) {
            const int e = tt / p.tiles_per_block;
            int32_t phys = table_row[e];
            if (phys < 0 || phys >= p.num_blocks) {
              if (is_k) atomicOr(&g_prefill_err, PA_DEVERR_BLOCK_RANGE);
              phys = 0;
            }
            ent = (phys * p.num_kv_heads + t.kvh) * p.tiles_per_block +
                  (tt - e * p.tiles_per_block);
          }
        }
        int tls[kTcTiles];
#pragma unroll
        for (int i = 0; i < kTcTiles; ++i)
          tls[i] = __shfl_sync(kFullMask, ent, kTcTiles * (jb % kPre) + i);
        if (lane == 0) {
          if (g >= kTcStages && !mbar_wait_bounded(&empty[stage], ((g / kTcStages) - 1) & 1)) {
            atomicOr(&g_prefill_err, PA_DEVERR_PIPE_TIMEOUT);
            ok = false;
          }
          if (ok) {
            uint8_t* dst = ring + stage * kTcTileBytes;
            mbar_arrive_expect_tx(&full[stage], uint32_t(ntl) * 2 * 2048);
            for (int i = 0; i < ntl; ++i) {
              const int row = tls[i] * kBlockSize;
              tma_load_2d(dst + i * 2048, map, 0, row, &full[stage], policy);
              tma_load_2d(dst + kTcTileBytes / 2 + i * 2048, map, 64, row, &full[stage], policy);
            }
          }
        }
        ok = __shfl_sync(kFullMask, ok, 0);
        if (!ok) break;
      }
    }
    if (lane == 0) {  // no copy may still be landing when the CTA exits (one ring)
      for (int i = max(0, g - kTcStages); i < g; ++i)
        if (!mbar_wait_bounded(&full[i % kTcStages], (i / kTcStages) & 1))
          atomicOr(&g_prefill_err, PA_DEVERR_PIPE_TIMEOUT);
    }
  } else if (warp == kPpMmaWarp) {
    // ---------------- MMA issuer (one thread) ----------------
    if (lane == 0) {
      const uint64_t kdesc0 = umma_smem_desc(smem_u32(ksm), 16, 1024, kUmmaSwizzle128B);
      const uint64_t vdesc0 = umma_smem_desc(smem_u32(vsm), kTcTileBytes / 2, 1024,
                                             kUmmaSwizzle128B);
      const uint64_t qdesc0 = umma_smem_desc(smem_u32(qsm), 16, 1024, kUmmaSwizzle128B);
      int g = 0;
      int cnt[2] = {0, 0};   // stages each tile has taken part in (phase counters)
      int nq[2] = {0, 0};    // pairs in which each tile was present (Q phases)
      bool ok = true;
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        if (ok && !mbar_wait_bounded(bar, parity)) ok = false;
        return ok;
      };
      auto issue_s = [&](int xt, int gs) {  // S of tile xt from K stage gs
        tcgen05_fence_after();
        const uint64_t kd = kdesc0 + uint64_t(((gs % kTcStages) * kTcTileBytes) >> 4);
        const uint64_t qd = qdesc0 + uint64_t((xt * kPpQBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t off = uint64_t(((ks >> 2) * (kTcTileBytes / 2) + (ks & 3) * 32) >> 4);
          umma_f16_ss(tmem + pp_tmem_s(xt), qd + off, kd + off, kIdescS, ks > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[xt]);
      };
      // O_xt += P_xt . V(stage gs) over keys 64 h .. 64 h + 63: the first half can
      // start while the softmax is still writing the second
      auto issue_pv = [&](int xt, int gs, int jb, int h) {
        tcgen05_fence_after();
        const uint64_t vd = vdesc0 + uint64_t(((gs % kTcStages) * kTcTileBytes) >> 4);
        const uint32_t pt = tmem + pp_tmem_s(xt);
#pragma unroll
        for (int t = 0; t < (kSplitP ? 2 : 1); ++t) {
#pragma unroll
          for (int kk = 0; kk < kTcKv / 32; ++kk) {
            const int ks = h * (kTcKv / 32) + kk;
            umma_f16_ts(tmem + pp_tmem_o(xt), pt + uint32_t(t * (kTcKv / 2) + ks * 8),
                        vd + uint64_t((ks * 2048) >> 4), kIdescPV,
                        (jb > 0 || t > 0 || ks > 0) ? 1u : 0u);
          }
        }
        if (h == 1) umma_commit(&o_full[xt]);
      };
      int pair = -1;
      PpPair x;
      while (ok && pp_next(pp, num_pairs, pair, x, false)) {
        const int nkb = x.nkb;
        auto in = [&](int xt, int jb) { return x.has[xt] && jb < x.t[xt].nkb; };
        // Q of the pair's tiles
        for (int xt = 0; xt < 2; ++xt)
          if (x.has[xt]) wait(&q_ready[xt], (nq[xt]++) & 1);
        // stage 0: S of both tiles
        if (!wait(&kfull[g % kTcStages], (g / kTcStages) & 1)) break;
        for (int xt = 0; xt < 2; ++xt)
          if (in(xt, 0)) issue_s(xt, g);
        umma_commit(&kempty[g % kTcStages]);
        for (int jb = 0; jb < nkb && ok; ++jb, ++g) {
          bool vwaited = false, kwaited = false;
          // P.V_A(jb), then S_A(jb + 1)
          if (in(0, jb)) {
            if (!wait(&p_half[0], cnt[0] & 1)) break;
            if (!wait(&vfull[g % kTcStages], (g / kTcStages) & 1)) break;
            vwaited = true;
            issue_pv(0, g, jb, 0);
            if (!wait(&p_ready[0], cnt[0] & 1)) break;
            issue_pv(0, g, jb, 1);
            ++cnt[0];
          }
          if (jb + 1 < nkb && in(0, jb + 1)) {
            if (!wait(&kfull[(g + 1) % kTcStages], ((g + 1) / kTcStages) & 1)) break;
            kwaited = true;
            issue_s(0, g + 1);
          }
          // P.V_B(jb), then S_B(jb + 1)
          if (in(1, jb)) {
            if (!wait(&p_half[1], cnt[1] & 1)) break;
            if (!vwaited && !wait(&vfull[g % kTcStages], (g / kTcStages) & 1)) break;
            issue_pv(1, g, jb, 0);
            if (!wait(&p_ready[1], cnt[1] & 1)) break;
            issue_pv(1, g, jb, 1);
            ++cnt[1];
          }
          umma_commit(&vempty[g % kTcStages]);  // the V stage's last P.V is issued
          if (jb + 1 < nkb) {
            if (in(1, jb + 1)) {
              if (!kwaited && !wait(&kfull[(g + 1) % kTcStages], ((g + 1) / kTcStages) & 1))
                break;
              issue_s(1, g + 1);
            }
            umma_commit(&kempty[(g + 1) % kTcStages]);  // its last S is issued
          }
        }
      }
      if (!ok) atomicOr(&g_prefill_err, PA_DEVERR_PIPE_TIMEOUT);
      umma_commit(done);  // fires once every MMA issued above has completed
    }
    __syncwarp();
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kPpSoftmaxRegs));
    // ---------------- softmax warpgroups: thread = row of tile xt ----------------
    const int xt = warp >> 2, qd = warp & 3;
    const int r = 32 * qd + lane;                           // TMEM lane and row of the tile
    const uint32_t tl = tmem + (uint32_t(32 * qd) << 16);  // this warp's lane quadrant
    const float mult = fabsf(p.q_mult);                     // Q carries the sign
    const uint32_t flip = p.q_mult < 0.f ? 0x80008000u : 0u;
    uint8_t* qx = qsm + xt * kPpQBytes;
    bool ok = true;  // warp-uniform; after a failure waits are skipped
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      if (ok) ok = __all_sync(kFullMask, mbar_wait_bounded(bar, parity));
    };
    auto arrive = [&](uint64_t* bar) {
      tcgen05_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    int g = 0, cnt = 0;  // stages of the CTA, stages of this tile
    int pair = -1;
    PpPair x;
    while (pp_next(pp, num_pairs, pair, x, false)) {
      const int gp = g;
      g += x.nkb;
      if (!x.has[xt]) continue;  // tile B of a pair with a single row block
      const TcTile& t = x.t[xt];
      const int gr = t.row0 + r;
      const bool valid = gr < t.rows;
      const int pos = valid ? t.L - t.nq + gr / p.group : -1;
      // ---- Q row into shared memory (K-major, 128-byte swizzle), sign carried ----
      {
        const uint4* src = reinterpret_cast<const uint4*>(
            p.query + (int64_t(t.q0 + (valid ? gr / p.group : 0)) * p.num_heads +
                       t.kvh * p.group + (valid ? gr % p.group : 0)) * D * 2);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          uint4 v = valid ? src[c] : make_uint4(0u, 0u, 0u, 0u);
          v.x ^= flip;
          v.y ^= flip;
          v.z ^= flip;
          v.w ^= flip;
          *reinterpret_cast<uint4*>(qx + (c >> 3) * (kPpQBytes / 2) + r * 128 +
                                    (((c & 7) ^ (r & 7)) << 4)) = v;
        }
        fence_proxy_async_smem();
        arrive(&q_ready[xt]);
      }
      float m = -INFINITY, l = 0.f;  // reference max (exp2 domain), row sum
      const uint32_t sb = tl + pp_tmem_s(xt);
      for (int jb = 0; jb < t.nkb; ++jb, ++cnt) {
        wait(&s_full[xt], cnt & 1);
        tcgen05_fence_after();
        // causal, context and padding mask: only stages that cross this row's last
        // visible position pay for it
        const int nvis = pos - jb * kTcKv + 1;
        const bool edge = nvis < kTcKv;
        // the row's 128 scores, one TMEM read
        float v[128];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32(sb + 32 * q, *reinterpret_cast<float(*)[32]>(v + 32 * q));
        tmem_wait_ld();
        // (an edge stage scales before masking, so that a zero scale never meets -inf)
        if (edge) {
#pragma unroll
          for (int i = 0; i < 128; ++i) v[i] = i < nvis ? v[i] * mult : -INFINITY;
        }
        float r8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) r8[k] = -INFINITY;
#pragma unroll
        for (int i = 0; i < 128; i += 2) r8[(i >> 1) & 7] = max3(r8[(i >> 1) & 7], v[i], v[i + 1]);
        const float mx = fmaxf(fmaxf(fmaxf(r8[0], r8[1]), fmaxf(r8[2], r8[3])),
                               fmaxf(fmaxf(r8[4], r8[5]), fmaxf(r8[6], r8[7]))) *
                         (edge ? 1.f : mult);
        if (jb == 0) {
          m = mx;  // O is written, not accumulated, by the tile's first P.V
        } else {
          const bool move = mx > m + kTcRescaleLog2;
          if (__any_sync(kFullMask, move)) {
            // rescale this warp's rows of O once P.V(jb - 1) of this tile has landed
            wait(&o_full[xt], (cnt - 1) & 1);
            tcgen05_fence_after();
            const float f = move ? ex2_approx(m - mx) : 1.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float o[32];
              tmem_ld32(tl + pp_tmem_o(xt) + 32 * q, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] *= f;
              tmem_st32(tl + pp_tmem_o(xt) + 32 * q, o);
            }
            l *= f;
            if (move) m = mx;
          }
        }
        const float mu = m == -INFINITY ? 0.f : m;
        const float me = edge ? 1.f : mult;  // multiplier still to apply
        const float2 me2 = make_float2(me, me), nmu2 = make_float2(-mu, -mu);
        float2 a4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
        // The pair's last stage: V rows past its last visible token may be stale or
        // NaN.  The tile whose P.V reads that stage first zeroes them (tile A if it
        // takes part in the stage), before any of its P is announced.
        if (jb == x.nkb - 1 && (xt == 0 || t.nkb != x.t[0].nkb || !x.has[0])) {
          const int gs = gp + jb;
          wait(&vfull[gs % kTcStages], (gs / kTcStages) & 1);
          if (ok && jb * kTcKv + r > x.pos_last) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint8_t* vrow = vsm + (gs % kTcStages) * kTcTileBytes + half * (kTcTileBytes / 2) +
                              r * 128;
#pragma unroll
              for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(vrow + c * 16) = make_uint4(0, 0, 0, 0);
            }
          }
          fence_proxy_async_smem();
        }
        // exponentials, then P over S as 16-bit pairs: chunk q's hi term into columns
        // [16 q, 16 q + 16), its lo term into [64 + 16 q, ...) (S is all in registers);
        // keys 0 .. 63 are announced on their own, so that their P.V can start
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t pw[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int i = 32 * q + 2 * c;
            const float2 e = fma2(make_float2(v[i], v[i + 1]), me2, nmu2);
            v[i] = ex2_approx(e.x);
            v[i + 1] = ex2_approx(e.y);
            a4[c & 3] = add2(a4[c & 3], make_float2(v[i], v[i + 1]));
            pw[c] = pack2(v[i], v[i + 1], CT{});
          }
          tmem_st16(sb + 16 * q, pw);
          if constexpr (kSplitP) {
            uint32_t lw[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int i = 32 * q + 2 * c;
              const float2 hi = unpack2(pw[c], CT{});
              lw[c] = pack2(v[i] - hi.x, v[i + 1] - hi.y, CT{});
            }
            tmem_st16(sb + kTcKv / 2 + 16 * q, lw);
          }
          if (q == 1) {
            tmem_wait_st();
            arrive(&p_half[xt]);
          }
        }
        const float2 a2 = add2(add2(a4[0], a4[1]), add2(a4[2], a4[3]));
        l += a2.x + a2.y;
        tmem_wait_st();
        arrive(&p_ready[xt]);
      }
      // epilogue: O / l of this tile's rows
      wait(&o_full[xt], (cnt - 1) & 1);
      if (ok) {
        tcgen05_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const int64_t orow = (int64_t(t.q0 + (valid ? gr / p.group : 0)) * p.num_heads +
                              t.kvh * p.group + (valid ? gr % p.group : 0)) * D;
        uint8_t* dst = static_cast<uint8_t*>(p.out);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v[32];
          tmem_ld32(tl + pp_tmem_o(xt) + 32 * q, v);
          tmem_wait_ld();
          if (!valid) continue;
          if (p.out_dtype == PA_F32) {
#pragma unroll
            for (int d = 0; d < 32; d += 4)
              *reinterpret_cast<float4*>(dst + (orow + 32 * q + d) * 4) =
                  make_float4(v[d] * inv, v[d + 1] * inv, v[d + 2] * inv, v[d + 3] * inv);
          } else if (p.out_dtype == PA_F16) {
#pragma unroll
            for (int d = 0; d < 32; d += 8)
              *reinterpret_cast<uint4*>(dst + (orow + 32 * q + d) * 2) =
                  make_uint4(pack2(v[d] * inv, v[d + 1] * inv, __half{}),
                             pack2(v[d + 2] * inv, v[d + 3] * inv, __half{}),
                             pack2(v[d + 4] * inv, v[d + 5] * inv, __half{}),
                             pack2(v[d + 6] * inv, v[d + 7] * inv, __half{}));
          } else {
#pragma unroll
            for (int d = 0; d < 32; d += 8)
              *reinterpret_cast<uint4*>(dst + (orow + 32 * q + d) * 2) =
                  make_uint4(pack2(v[d] * inv, v[d + 1] * inv, __nv_bfloat16{}),
                             pack2(v[d + 2] * inv, v[d + 3] * inv, __nv_bfloat16{}),
                             pack2(v[d + 4] * inv, v[d + 5] * inv, __nv_bfloat16{}),
                             pack2(v[d + 6] * inv, v[d + 7] * inv, __nv_bfloat16{}));
          }
        }
      }
      tcgen05_fence_before();  // O is read before the next pair's first P.V overwrites it
    }
    if (!ok && lane == 0) atomicOr(&g_prefill_err, PA_DEVERR_PIPE_TIMEOUT);
  }
  // Free TMEM only after every MMA has completed and every TMEM access is done.
  __syncthreads();
  if (warp == kPpMmaWarp) {
    if (!__all_sync(kFullMask, mbar_wait_bounded(done, 0)) && lane == 0)
      atomicOr(&g_prefill_err, PA_DEVERR_PIPE_TIMEOUT);
    tcgen05_fence_after();
    tmem_dealloc(tmem, kPpTmemCols);
  }
}

}  // namespace

int launch_prefill(const DecodeArgs& a, const int32_t* query_start, int max_query_len,
                   cudaStream_t stream) {
  const int group = a.num_heads / a.num_kv_heads;
  const int64_t rows = a.num_blocks * a.num_kv_heads * a.block_size;
  if (a.head_dim != 128 || a.cache_dtype == PA_FP8_E4M3 || a.cache_dtype != a.q_dtype ||
      rows >= (int64_t(1) << 31) || encode_fn() == nullptr)
    return PA_ERR_UNSUPPORTED;
  PrefillParams pp;
  memset(&pp, 0, sizeof pp);
  Params& p = pp.p;
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
  p.out_dtype = a.out_dtype;
  p.num_blocks = a.num_blocks;
  p.q_mult = a.scale * kLog2e;
  p.v_mult = 1.f;
  pp.query_start = query_start;
  pp.row_blocks = int((int64_t(max_query_len) * group + kPrefillRows - 1) / kPrefillRows);
  const int64_t grid_x = int64_t(a.num_seqs) * pp.row_blocks;
  if (pp.row_blocks == 0) return PA_OK;
  if (grid_x > INT32_MAX) return PA_ERR_UNSUPPORTED;
  if (!encode_pool_map(&pp.tmk, a.key_cache, rows, false) ||
      !encode_pool_map(&pp.tmv, a.value_cache, rows, false))
    return PA_ERR_CUDA;
  constexpr int stages = 4;
  auto run = [&](auto kern, size_t smem, std::atomic<unsigned long long>& mask) -> int {
    if (set_smem_once(kern, smem, mask) != PA_OK) return PA_ERR_CUDA;
    kern<<<dim3(unsigned(grid_x), unsigned(a.num_kv_heads)), kThreads, smem, stream>>>(pp);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
  };
  static std::atomic<unsigned long long> mask_h{0}, mask_b{0};
  if (int64_t(max_query_len) * group >= kTcRows) {
    // 128-row tiles for the 5th-generation tensor cores
    TcPrefillParams tp;
    memset(&tp, 0, sizeof tp);
    tp.tmk = pp.tmk;
    tp.tmv = pp.tmv;
    tp.p = pp.p;
    tp.query_start = pp.query_start;
    tp.row_blocks = int((int64_t(max_query_len) * group + kTcRows - 1) / kTcRows);
    const int64_t tiles = int64_t(a.num_seqs) * a.num_kv_heads * tp.row_blocks;
    if (tiles > INT32_MAX) return PA_ERR_UNSUPPORTED;
    tp.num_tiles = int(tiles);
    // persistent: one CTA per SM walks its round-robin share of the tiles
    int dev_sm = 0, sms = 0;
    if (cudaGetDevice(&dev_sm) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev_sm) != cudaSuccess)
      return PA_ERR_CUDA;
    // two 128-row tiles of one (sequence, kv head) per CTA at a time, when a
    // (sequence, kv head) has two: the other warpgroup would idle otherwise
    const int64_t pairs = int64_t(a.num_seqs) * a.num_kv_heads * ((tp.row_blocks + 1) / 2);
    if (tp.row_blocks >= 2 && pairs <= INT32_MAX && !fallback_kernels_forced()) {
      const unsigned grid_pp = unsigned(pairs < sms ? pairs : sms);
      constexpr size_t smem_pp = pp_prefill_smem_bytes();
      // The register split assumes the CTA is launched with kPpLaunchRegs a thread
      // (a split above the launch's registers would wait forever); a build whose
      // kernel has another count takes the one-tile kernel.  Checked once.
      auto launch_pp = [&](auto kern, std::atomic<unsigned long long>& mask,
                           std::atomic<int>& regs) -> int {
        int r = regs.load(std::memory_order_relaxed);
        if (r == 0) {
          cudaFuncAttributes fa;
          if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return PA_ERR_CUDA;
          r = fa.numRegs == kPpLaunchRegs ? 1 : -1;
          regs.store(r, std::memory_order_relaxed);
        }
        if (r < 0) return PA_ERR_UNSUPPORTED;
        if (set_smem_once(kern, smem_pp, mask) != PA_OK) return PA_ERR_CUDA;
        kern<<<grid_pp, kPpThreads, smem_pp, stream>>>(tp, int(pairs));
        return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
      };
      static std::atomic<unsigned long long> pmask_h{0}, pmask_b{0}, pmask_bs{0};
      static std::atomic<int> pregs_h{0}, pregs_b{0}, pregs_bs{0};
      int rc;
      if (a.cache_dtype == PA_F16)
        rc = launch_pp(prefill_pp_kernel<__half, false>, pmask_h, pregs_h);
      else if (a.out_dtype == PA_F32)
        rc = launch_pp(prefill_pp_kernel<__nv_bfloat16, true>, pmask_bs, pregs_bs);
      else
        rc = launch_pp(prefill_pp_kernel<__nv_bfloat16, false>, pmask_b, pregs_b);
      if (rc != PA_ERR_UNSUPPORTED) return rc;
    }
    const unsigned grid_tc = unsigned(tiles < sms ? tiles : sms);
    constexpr size_t smem = tc_prefill_smem_bytes();
    auto launch = [&](auto kern, std::atomic<unsigned long long>& mask) -> int {
      if (set_smem_once(kern, smem, mask) != PA_OK) return PA_ERR_CUDA;
      kern<<<grid_tc, kTcThreads, smem, stream>>>(tp);
      return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
    };
    static std::atomic<unsigned long long> tmask_h{0}, tmask_b{0}, tmask_bs{0};
    if (a.cache_dtype == PA_F16) return launch(prefill_tc_kernel<__half, false>, tmask_h);
    if (a.out_dtype == PA_F32) return launch(prefill_tc_kernel<__nv_bfloat16, true>, tmask_bs);
    return launch(prefill_tc_kernel<__nv_bfloat16, false>, tmask_b);
  }
  if (a.cache_dtype == PA_F16)
    return run(prefill_kernel<__half, stages>, prefill_smem_bytes<__half, stages>(), mask_h);
  return run(prefill_kernel<__nv_bfloat16, stages>, prefill_smem_bytes<__nv_bfloat16, stages>(),
             mask_b);
}

cudaError_t read_and_clear_prefill_errors(unsigned* bits, cudaStream_t stream) {
  unsigned v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_prefill_err, sizeof v, 0,
                                            cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  const unsigned zero = 0;
  e = cudaMemcpyToSymbolAsync(g_prefill_err, &zero, sizeof zero, 0, cudaMemcpyHostToDevice,
                              stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  *bits |= v;
  return e;
}

}  // namespace pa
