// Attention forward for sm_100a, two 128-query tiles (A and B) of one head
// per CTA.  Same operation, modes, masks and RoPE placement as
// attn_fwd_kernel (see attention.cuh); what changes is the schedule:
//
//   * one softmax warpgroup per query tile, each thread owning a whole row
//     of a score tile (no row-max exchange between warpgroups);
//   * scores are computed in 64-key sub-tiles, double-buffered in TMEM per
//     query tile, so S_X(j+1) = Q_X K_{j+1}^T runs on the tensor core while
//     the softmax of S_X(j) runs; each tile has its own MMA-issuing thread
//     and tile B starts some way into tile A's first sub-tile (two
//     softmax warpgroups sharing the tensor core, as in FlashAttention-4 on
//     Blackwell);
//   * every K and V stage (128 keys, two sub-tiles) is loaded into shared
//     memory once for both query tiles.
//
// The HYB instantiation adds MobileWan's linear read-out after the chunk's
// softmax part: phi(Q) replaces Q in shared memory, S_c (bf16 hi + lo) fills
// the freed K stages, phi(Q) S_c runs into the freed S buffers, and the
// epilogue joins both parts in one normalisation.
//
// Warp roles: warp 0 TMA Q_A, Q_B, then K stages; warp 1 TMEM allocation and
// tcgen05.mma issue for tile A; warp 2 TMA V stages; warp 3 tcgen05.mma issue
// for tile B; warps 4..7 softmax of tile A, warps 8..11 softmax of tile B
// (thread r owns query row r = TMEM lane r).
//
// TMEM columns (512): S_X buffer b at [128 x + 64 b, +64) fp32 for tiles
// x = A, B and b = 0, 1; O_A [256, 256+D), O_B [384, 384+D) fp32.  P (bf16
// pairs, 32 columns) overwrites the first half of its S buffer once the
// softmax holds the scores in registers; an issuer issues the scores of
// sub-tile j+2 into that buffer right after the P V of sub-tile j (one
// thread's tcgen05.mma operations run in issue order).
#pragma once
#include "attention.cuh"
#include "feature_map.cuh"

namespace vattn {
namespace attn {

template <int D>
struct PairCfg {
  static constexpr int kTileBytes = kTileM * D * 2;
  static constexpr int kBlocks = D / 64;
  // K and V stages of 128 keys.  K runs one stage deeper at head dim 128:
  // a K stage is refilled only after the lagging tile's last Q K^T on it,
  // and the refill's latency under load (about 3.6k cycles measured) is
  // longer than the two sub-tile periods two stages leave; V is read one
  // softmax later, which gives it that slack.
  static constexpr int kStagesK = D == 128 ? 3 : 4;
  static constexpr int kStagesV = D == 128 ? 2 : 4;
  static constexpr int kOffQ = 0;                          // Q_A, Q_B
  static constexpr int kOffK = 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kStagesK * kTileBytes;
  static constexpr int kOffBar = kOffV + kStagesV * kTileBytes;
  static constexpr int kNumBars = 4 + 2 * kStagesK + 2 * kStagesV + 12 + 2 + 5 + 4;
  // the misc words start on a 128-byte boundary whatever the barrier count,
  // so z_c (the destination of a bulk copy) stays 16-byte aligned
  static constexpr int kOffMisc = (kOffBar + kNumBars * 8 + 127) & ~127;
  static constexpr int kOffZ = kOffMisc + 64;        // hybrid: z_c, fp32 [D]
  static constexpr int kSmemBytes = kOffZ + D * 4;
  static_assert(kOffZ % 16 == 0, "bulk-copy destination must be 16-byte aligned");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory of one CTA");
};

constexpr int kPairThreads = 384;


// Rows of the two query tiles of pair `pr` and the key tiles they need
// (the union of both tiles' visible ranges; rows mask what they do not see).
struct PairGeom {
  int q0[2], q_end[2];
  bool hasB;
  TileGeom tg;   // q0 / q_end span both tiles; kbeg, kend: the union; n_tiles: this CTA's share
  int t0;        // the CTA's first key tile of the union (key split; 0 without)
};

// The pair's key tiles split into nsplit near-equal parts; part `split`.
__device__ __forceinline__ PairGeom pair_geom(const Params& p, int pr, int split, int nsplit) {
  PairGeom g;
  const int pps = (p.q_tiles_per_seg + 1) / 2;
  const int seg = pr / pps;
  const int t = pr - seg * pps;
  int e = (seg + 1) * p.q_seg_len;
  if (e > p.Lq) e = p.Lq;
  g.q0[0] = seg * p.q_seg_len + 2 * t * kTileM;
  g.q_end[0] = min(g.q0[0] + kTileM, e);
  g.q0[1] = g.q0[0] + kTileM;
  g.q_end[1] = min(g.q0[1] + kTileM, e);
  g.hasB = g.q0[1] < g.q_end[1];
  g.tg.q0 = g.q0[0];
  g.tg.q_end = g.hasB ? g.q_end[1] : g.q_end[0];
  g.t0 = 0;
  if (p.n_kseg == 0) {
    int lo0, hi0, lo1, hi1;
    key_range(p, g.tg.q0, lo0, hi0);
    key_range(p, g.tg.q_end - 1, lo1, hi1);
    g.tg.kbeg = lo0;
    g.tg.kend = hi1;
    const int total = g.tg.kend > g.tg.kbeg ? (g.tg.kend - g.tg.kbeg + kTileN - 1) / kTileN : 0;
    const int per = (total + nsplit - 1) / nsplit;
    g.t0 = min(total, split * per);
    g.tg.n_tiles = min(total, g.t0 + per) - g.t0;
  } else {
    g.tg.kbeg = g.tg.kend = 0;
    const KeySegment& last = p.kseg[p.n_kseg - 1];
    const int total = last.tile0 + (last.n_tok + kTileN - 1) / kTileN;
    const int per = nsplit > 1 ? p.split_tiles : total;
    g.t0 = min(total, split * per);
    g.tg.n_tiles = min(total, g.t0 + per) - g.t0;
  }
  return g;
}

// Where split `s`'s partial of query row `row` lives (row index into
// part_lse; times D into part_o): the streaming step's [split][B][H][Lq]
// layout, or the tail split's compact [tail item][split][256 pair rows].
__device__ __forceinline__ size_t part_row(const Params& p, const PairGeom& g, int b, int h, int s, int nsplit,
                                           int tail_item, int row) {
  if (p.tail_split)
    return (static_cast<size_t>(tail_item) * nsplit + s) * (2 * kTileM) + (row - g.q0[0]);
  return ((static_cast<size_t>(s) * p.B + b) * p.H + h) * p.Lq + row;
}

// A streaming step's append share: CTA `part` of the n_append leading CTAs
// copies its range of the frame's 16-byte chunks (raw K and V into the ring
// slot, K rotated at its (t, h, w) into the rotated ring), then counts
// itself done with a release; attention CTAs of the same launch wait for
// all shares before loading the rotated current frame.
template <int D>
__device__ __forceinline__ void append_share(const Params& p, int part) {
  const AppendWork& a = p.app;
  constexpr int D8 = D / 8;   // 16-byte chunks per head vector
  const long long cpr = static_cast<long long>(p.Hkv) * D8;
  const long long total = a.rows * cpr;
  const long long per = (total + p.n_append - 1) / p.n_append;
  const long long c0 = static_cast<long long>(part) * per;
  const long long c1 = min(total, c0 + per);
  const int Fr = p.rope_Hg * p.rope_Wg;
  const int pt = p.rope_pt, pth = p.rope_pt + p.rope_ph;
  constexpr int U = 4;   // chunks per thread and step: all loads before the stores
  for (long long base = c0 + threadIdx.x; base < c1; base += static_cast<long long>(blockDim.x) * U) {
    uint4 kv[U], vv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long i = base + static_cast<long long>(u) * blockDim.x;
      if (i < c1) {
        kv[u] = __ldg(a.k + i);
        vv[u] = __ldg(a.v + i);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long i = base + static_cast<long long>(u) * blockDim.x;
      if (i >= c1) continue;
      a.kr[i] = kv[u];
      a.vr[i] = vv[u];
      if (a.krot) {
        const int n = static_cast<int>((i / cpr) % a.F);   // token of the frame
        const int c16 = static_cast<int>(i % D8);          // chunk of the head vector
        const int in = n % Fr;
        const int pt_t = a.t0 + n / Fr, pt_h = in / p.rope_Wg, pt_w = in % p.rope_Wg;
        uint32_t w4[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = c16 * 4 + e;
          const int pos = j < pt ? pt_t : (j < pth ? pt_h : pt_w);
          const float2 cs = __ldg(p.rope_tab + pos * (D / 2) + j);
          const float x0 = bf16lo_to_f32(w4[e]), x1 = bf16hi_to_f32(w4[e]);
          w4[e] = pack_bf16x2(x0 * cs.x - x1 * cs.y, x0 * cs.y + x1 * cs.x);
        }
        a.krot[i] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    }
  }
  if (part == 0 && threadIdx.x == 0) a.ids[a.slot] = a.frame;
  // every thread's stores visible to the async proxy (TMA) and at gpu scope
  // before the CTA counts itself done
  fence_proxy_async_global();
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) atomicAdd(p.step_sync, 1u);
}

// The merge of a query-tile pair's key splits, by the pair's last CTA
// (ReGenVC Sec. 3.5's exact combination, here of splits of one CTA's keys):
// with lse_s = m_s + log2 l_s per split s, o = sum_s 2^(lse_s - M) o_s /
// sum_s 2^(lse_s - M), M = max_s lse_s.  Warp w of the softmax warpgroups
// merges 32 rows of its tile: each lane first forms its own row's weights,
// then the warp walks the rows, lane l reading and writing columns
// [l D/32, (l+1) D/32) (coalesced rows of the partials, from L2).
template <int D>
__device__ __forceinline__ void merge_splits(const Params& p, const PairGeom& g, int b, int h, int warp, int lane,
                                             int S, int tail_item) {
  const int x = (warp - 4) >> 2;
  if (x == 1 && !g.hasB) return;
  const int r0 = (x ? g.q0[1] : g.q0[0]) + (warp & 3) * 32;
  const int q_end = x ? g.q_end[1] : g.q_end[0];
  if (r0 >= q_end) return;
  const size_t bh = (static_cast<size_t>(b) * p.H + h) * p.Lq;
  const int myrow = r0 + lane;
  float wts[kMaxSplit];
  float M = -INFINITY;
#pragma unroll
  for (int s = 0; s < kMaxSplit; ++s) {
    wts[s] = (s < S && myrow < q_end) ? __ldcg(p.part_lse + part_row(p, g, b, h, s, S, tail_item, myrow))
                                      : -INFINITY;
    M = fmaxf(M, wts[s]);
  }
  float W = 0.f;
#pragma unroll
  for (int s = 0; s < kMaxSplit; ++s) {
    wts[s] = M == -INFINITY ? 0.f : ex2_approx(wts[s] - M);   // 0 for an empty split
    W += wts[s];
  }
  const float invW = W > 0.f ? 1.f / W : 0.f;
  if (p.lse && myrow < q_end)
    p.lse[bh + myrow] = W > 0.f ? (M + __log2f(W)) * 0.69314718055994531f : -INFINITY;
  constexpr int CPL = D / 32;   // columns per lane
  const int nrows = min(32, q_end - r0);
#pragma unroll 1
  for (int rr = 0; rr < nrows; ++rr) {
    float acc[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[e] = 0.f;
#pragma unroll
    for (int s = 0; s < kMaxSplit; ++s) {
      if (s < S) {
        const float w = __shfl_sync(0xffffffffu, wts[s], rr);
        const float* src = p.part_o + part_row(p, g, b, h, s, S, tail_item, r0 + rr) * D + lane * CPL;
        if constexpr (CPL == 2) {
          const float2 v = __ldcg(reinterpret_cast<const float2*>(src));
          acc[0] = fmaf(w, v.x, acc[0]);
          acc[1] = fmaf(w, v.y, acc[1]);
        } else {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(src));
          acc[0] = fmaf(w, v.x, acc[0]);
          acc[1] = fmaf(w, v.y, acc[1]);
          acc[2] = fmaf(w, v.z, acc[2]);
          acc[3] = fmaf(w, v.w, acc[3]);
        }
      }
    }
    const float iw = __shfl_sync(0xffffffffu, invW, rr);
    __nv_bfloat16* dst = p.o + ((static_cast<size_t>(b) * p.Lq + r0 + rr) * p.H + h) * D + lane * CPL;
    if constexpr (CPL == 2) {
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * iw, acc[1] * iw);
    } else {
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc[0] * iw, acc[1] * iw),
                                                  pack_bf16x2(acc[2] * iw, acc[3] * iw));
    }
  }
}

// Last act of every CTA of a streaming step: count the exit; the last CTA
// puts both counters back to zero for the next launch.
__device__ __forceinline__ void step_exit(const Params& p) {
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(p.step_sync + 1, 1u);
    if (old == static_cast<uint32_t>(p.total_ctas) - 1u) {
      p.step_sync[0] = 0u;
      p.step_sync[1] = 0u;
      __threadfence();
    }
  }
}

// Keep the 32 registers of r after every earlier volatile statement (the
// TMEM load wait): later uses cannot be scheduled above it.
__device__ __forceinline__ void reg_tie32(uint32_t (&r)[32]) {
  asm volatile("" : VATTN_RW8(0), VATTN_RW8(8), VATTN_RW8(16), VATTN_RW8(24));
}

template <int D, int ROPE, bool HYB>
__global__ void __launch_bounds__(kPairThreads, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmK2,
                     const __grid_constant__ CUtensorMap tmV2, const __grid_constant__ CUtensorMap tmO,
                     const Params p) {
  static_assert(ROPE == kRopeNone || ROPE == kRopeQ, "keys are rotated before this kernel");
  static_assert(!HYB || (D == 128 && ROPE == kRopeNone), "hybrid: head dim 128, no RoPE");
  using C = PairCfg<D>;
  constexpr int NSK = C::kStagesK, NSV = C::kStagesV;
  constexpr int kSub = kTileN / 2;                 // keys per score sub-tile
  constexpr uint32_t kSubBytes = kSub * 128;       // sub-tile offset inside a 64-column block
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t sbase = smem_addr(smem);
  const bool stepping = p.linear_grid && p.step_sync;
  if (sbase & 1023u) {   // 128B-swizzled operand tiles need 1024-byte alignment
    if (threadIdx.x == 0 && p.status) atomicCAS(p.status, 0u, kStatusSmemAlign);
    if (stepping) step_exit(p);
    return;
  }
  // which work this CTA does: (pair, head, batch) of a 3-D grid, or an
  // append share / (pair, head, batch, split) of a streaming step's 1-D grid
  int pr, h, b, split = 0, nsplit = 1, tail_item = 0;
  if (p.linear_grid && p.tail_split) {
    // whole items first, then the split items' parts
    const int idx = static_cast<int>(blockIdx.x);
    int item = idx;
    if (idx >= p.n_normal) {
      const int rel = idx - p.n_normal;
      tail_item = rel / p.n_split;
      split = rel - tail_item * p.n_split;
      nsplit = p.n_split;
      item = p.n_normal + tail_item;
    }
    pr = item % p.n_pairs;
    item /= p.n_pairs;
    h = item % p.H;
    b = item / p.H;
  } else if (p.linear_grid) {
    int idx = static_cast<int>(blockIdx.x);
    if (idx < p.n_append) {
      append_share<D>(p, idx);
      step_exit(p);
      return;
    }
    idx -= p.n_append;
    pr = idx % p.n_pairs;
    idx /= p.n_pairs;
    h = idx % p.H;
    idx /= p.H;
    b = idx % p.B;
    split = idx / p.B;
    nsplit = p.n_split > 1 ? p.n_split : 1;
  } else {
    h = blockIdx.y;
    b = blockIdx.z;
    pr = p.reverse_q ? static_cast<int>(gridDim.x - 1 - blockIdx.x) : static_cast<int>(blockIdx.x);
  }
  const uint32_t sQ = sbase + C::kOffQ, sK = sbase + C::kOffK, sV = sbase + C::kOffV;
  const uint32_t bar0 = sbase + C::kOffBar;
  auto bQFull = [&](int x) { return bar0 + 8 * x; };
  auto bQReady = [&](int x) { return bar0 + 16 + 8 * x; };
  auto bKFull = [&](int s) { return bar0 + 32 + 8 * s; };
  auto bKEmpty = [&](int s) { return bar0 + 32 + 8 * (NSK + s); };
  auto bVFull = [&](int s) { return bar0 + 32 + 8 * (2 * NSK + s); };
  auto bVEmpty = [&](int s) { return bar0 + 32 + 8 * (2 * NSK + NSV + s); };
  const uint32_t bx = bar0 + 32 + 16 * NSK + 16 * NSV;
  auto bSFull = [&](int x, int b) { return bx + 8 * (2 * x + b); };
  auto bPFull = [&](int x, int b) { return bx + 32 + 8 * (2 * x + b); };
  auto bPvDone = [&](int x) { return bx + 64 + 8 * x; };
  auto bODone = [&](int x) { return bx + 80 + 8 * x; };   // last P V of the tile complete
  auto bFinal = [&](int x) { return bx + 96 + 8 * x; };     // all MMAs of issuer x complete
  // hybrid read-out: phi(Q_x) in place of Q_x, S_c (bf16 hi / lo) in the K stages, phi(Q_x) S_c
  auto bPhiReady = [&](int x) { return bx + 112 + 8 * x; };
  const uint32_t bScReady = bx + 128;
  auto bLinDone = [&](int x) { return bx + 136 + 8 * x; };
  // hybrid: each tile's last Q K^T complete (Q_x and, with both, the K
  // stages free); z_c landed in shared memory
  auto bQKDone = [&](int x) { return bx + 152 + 8 * x; };
  const uint32_t bZFull = bx + 168;
  const uint32_t bStartB = bx + 176;   // tile A's softmax has its first row maxima
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile uint32_t* tmem_slot = misc;
  volatile uint32_t* abort_flag = misc + 1;
  Abort ab{abort_flag, p.status, p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kvh = h / (p.H / p.Hkv);
  const PairGeom g = pair_geom(p, pr, split, nsplit);
  if (g.q0[0] >= g.q_end[0]) {   // pair past the end of a short last segment
    if (stepping) step_exit(p);
    return;
  }
  const int nk = g.tg.n_tiles;          // 128-key stages
  const int ns = 2 * nk;                // 64-key score sub-tiles
  const bool hasB = g.hasB;

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(bQFull(x), 1);
      mbar_init(bQReady(x), 4);
      mbar_init(bPvDone(x), 1);
      mbar_init(bODone(x), 1);
      for (int bb = 0; bb < 2; ++bb) {
        mbar_init(bSFull(x, bb), 1);
        mbar_init(bPFull(x, bb), 4);
      }
    }
    // a stage is released once by the MMA issuer of each query tile
    for (int s = 0; s < NSK; ++s) {
      mbar_init(bKFull(s), 1);
      mbar_init(bKEmpty(s), hasB ? 2 : 1);
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(bVFull(s), 1);
      mbar_init(bVEmpty(s), hasB ? 2 : 1);
    }
    mbar_init(bFinal(0), 1);
    mbar_init(bFinal(1), 1);
    mbar_init(bPhiReady(0), 4);
    mbar_init(bPhiReady(1), 4);
    mbar_init(bScReady, 4);
    mbar_init(bQKDone(0), 1);
    mbar_init(bQKDone(1), 1);
    mbar_init(bZFull, 1);
    mbar_init(bStartB, 4);
    mbar_init(bLinDone(0), 1);
    mbar_init(bLinDone(1), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(const_cast<uint32_t*>(tmem_slot)), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------ producer: Q_A, Q_B, then K
    if (lane == 0) {
      for (int x = 0; x < (hasB ? 2 : 1); ++x) {
        mbar_arrive_expect_tx(bQFull(x), C::kTileBytes);
#pragma unroll
        for (int blk = 0; blk < C::kBlocks; ++blk)
          tma_load_4d(sQ + x * C::kTileBytes + blk * (kTileM * 128), &tmQ, bQFull(x), blk * 64, h,
                      x ? g.q0[1] : g.q0[0], b);
      }
      int j = 0;
      bool waited = p.wait_tile < 0 || !stepping;
      for (; j < nk; ++j) {
        const int s = j % NSK;
        if (j >= NSK && !mbar_wait(bKEmpty(s), ((j / NSK) - 1) & 1, ab, kStatusTimeoutProducer)) break;
        if (!waited && g.t0 + j >= p.wait_tile) {
          // this tile's keys are written by the step's append CTAs
          if (!wait_counter(p.step_sync, static_cast<uint32_t>(p.n_append), ab, kStatusTimeoutStep)) break;
          fence_proxy_async_global();
          waited = true;
        }
        const KeyTile kt = key_tile(p, g.tg, g.t0 + j);
        const CUtensorMap* m = kt.kmap ? &tmK2 : &tmK;
        mbar_arrive_expect_tx(bKFull(s), C::kTileBytes);
#pragma unroll
        for (int blk = 0; blk < C::kBlocks; ++blk)
          tma_load_4d(sK + s * C::kTileBytes + blk * (kTileM * 128), m, bKFull(s), blk * 64, kvh, kt.k0,
                      kt.kc3 + b);
      }
      // drain: every load issued so far has landed before the CTA exits
      for (int i = max(0, j - NSK); i < j; ++i) {
        mbar_drain(bKFull(i % NSK), (i / NSK) & 1, ab.limit_ns);
      }
      for (int x = 0; x < (hasB ? 2 : 1); ++x) {
        mbar_drain(bQFull(x), 0, ab.limit_ns);
      }
    }
  } else if (warp == 2) {
    // ----------------------------------------------------- producer: V
    if (lane == 0) {
      if constexpr (HYB) {
        // z_c (the pair's chunk state, 512 bytes) for the read-out, now
        const int c = g.q0[0] / p.q_seg_len;
        mbar_arrive_expect_tx(bZFull, D * 4);
        bulk_load(sbase + C::kOffZ, p.hyb_z + ((static_cast<size_t>(c) * p.B + b) * p.H + h) * D, D * 4, bZFull);
      }
      int j = 0;
      for (; j < nk; ++j) {
        const int s = j % NSV;
        if (j >= NSV && !mbar_wait(bVEmpty(s), ((j / NSV) - 1) & 1, ab, kStatusTimeoutProducer)) break;
        const KeyTile kt = key_tile(p, g.tg, g.t0 + j);
        const CUtensorMap* m = kt.vmap ? &tmV2 : &tmV;
        mbar_arrive_expect_tx(bVFull(s), C::kTileBytes);
#pragma unroll
        for (int blk = 0; blk < C::kBlocks; ++blk)
          tma_load_4d(sV + s * C::kTileBytes + blk * (kTileM * 128), m, bVFull(s), blk * 64, kvh, kt.k0,
                      kt.vc3 + b);
      }
      for (int i = max(0, j - NSV); i < j; ++i) {
        mbar_drain(bVFull(i % NSV), (i / NSV) & 1, ab.limit_ns);
      }
      if constexpr (HYB) mbar_drain(bZFull, 0, ab.limit_ns);
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------- MMA
    // one issuing thread per query tile: warp 1 for A, warp 3 for B
    const int x = warp == 1 ? 0 : 1;
    if (lane == 0 && (x == 0 || hasB)) {
      constexpr uint32_t idQK = idesc_bf16_f32(kTileM, kSub, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(kTileM, D, false, true);
      // descriptors built once; a K step or a sub-tile adds a constant to
      // the start-address field (address >> 4, 14 bits), which cannot carry
      // out of the field (shared memory < 256 KB)
      const uint64_t dQx = sdesc_sw128(sQ + x * C::kTileBytes, 16, 1024);
      const uint64_t dK = sdesc_sw128(sK, 16, 1024);
      const uint64_t dV = sdesc_sw128(sV, kTileM * 128, 1024);
      const uint32_t tSx = tmem + static_cast<uint32_t>(x * 128);
      const uint32_t tOx = tmem + 256u + static_cast<uint32_t>(x * 128);
      // start-address step (>> 4) of sub-tile u: stage (u / 2) % stages, half u % 2
      auto sub_step = [](int u, int stages) -> uint64_t {
        return static_cast<uint64_t>(((u >> 1) % stages) * (C::kTileBytes >> 4) + (u & 1) * (kSubBytes >> 4));
      };
      // S_x(u) = Q_x K(u)^T into S buffer u & 1
      auto issue_qk = [&](int u) {
        const uint64_t dk = dK + sub_step(u, NSK);
        const uint32_t tS = tSx + static_cast<uint32_t>((u & 1) * kSub);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * (kTileM * 128) + (kk & 3) * 32) >> 4;
          umma_ss(tS, dQx + off, dk + off, idQK, kk > 0);
        }
        umma_commit(bSFull(x, u & 1));
      };
      // O_x += P_x(u) V(u), P_x(u) in the first half of S buffer u & 1
      auto issue_pv = [&](int u) {
        const uint64_t dv = dV + sub_step(u, NSV);
        const uint32_t tP = tSx + static_cast<uint32_t>((u & 1) * kSub);
        const uint32_t acc0 = u > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < kSub / 16; ++kk)
          umma_ts(tOx, tP + kk * 8, dv + static_cast<uint64_t>(kk * (2048 >> 4)), idPV, kk > 0 ? 1u : acc0);
        umma_commit(bPvDone(x));
      };
      bool ok = mbar_wait(ROPE == kRopeQ ? bQReady(x) : bQFull(x), 0, ab, kStatusTimeoutMma);
      // tile B starts after tile A, so the two softmax warpgroups do not run
      // in lockstep (2-3 % faster than both at once): at head dim 64 and in
      // the hybrid's short loops once tile A has the row maxima of its first
      // sub-tile (2.4 % and 2.8 % faster than the alternative), in the long
      // head-dim-128 loops once tile A has published its first P (2.5 %
      // faster than the early start), measured on B200
      constexpr bool kEarlyB = D == 64 || HYB;
      if (x == 1 && ok && nk > 0)
        ok = mbar_wait(kEarlyB ? bStartB : bPFull(0, 0), 0, ab, kStatusTimeoutMma);
      // S_x(j) once its K stage has landed (a stage is waited for at its
      // first sub-tile only, and released once its second one is issued)
      auto qk_step = [&](int j) -> bool {
        const int stj = (j >> 1) % NSK;
        if (!(j & 1) && !mbar_wait(bKFull(stj), ((j >> 1) / NSK) & 1, ab, kStatusTimeoutMma)) return false;
        tc_fence_after();
        issue_qk(j);
        if (HYB && j == ns - 1) umma_commit(bQKDone(x));
        if (j & 1) umma_commit(bKEmpty(stj));   // both sub-tiles of the stage issued
        return true;
      };
      // both S buffers first (ns = 2 nk is even)
      if (ok && nk > 0) ok = qk_step(0) && qk_step(1);
      // per sub-tile u: O_x += P_x(u) V(u) once the softmax has published
      // P_x(u), then at once S_x(u + 2) into the same buffer.  tcgen05.mma
      // operations issued by one thread run in issue order, so the P V reads
      // P before the next scores overwrite it; not waiting for the P V to
      // complete keeps its latency off the softmax's path to S_x(u + 2).
      int u = 0;
      for (; ok && u < ns; ++u) {
        const int st = (u >> 1) % NSV;
        if (!(u & 1) && !mbar_wait(bVFull(st), ((u >> 1) / NSV) & 1, ab, kStatusTimeoutMma)) break;
        if (!mbar_wait(bPFull(x, u & 1), (u >> 1) & 1, ab, kStatusTimeoutMma)) break;
        tc_fence_after();
        issue_pv(u);
        if (u == ns - 1) umma_commit(bODone(x));
        if (u & 1) umma_commit(bVEmpty(st));
        if (u + 2 < ns && !qk_step(u + 2)) break;
      }
      if constexpr (HYB) {
        // linear read-out phi(Q_x) S_c into the S buffers of tile x (free
        // after the last P V): A = phi(Q_x) K-major in place of Q_x, B = S_c
        // split into bf16 hi and lo parts, MN-major, in the K stages
        if (ok && u == ns && mbar_wait(bPhiReady(x), 0, ab, kStatusTimeoutMma) &&
            mbar_wait(bScReady, 0, ab, kStatusTimeoutMma)) {
          tc_fence_after();
          const uint64_t dHi = sdesc_sw128(sK, D * 128, 1024);
          const uint64_t dLo = sdesc_sw128(sK + D * D * 2, D * 128, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * (kTileM * 128) + (kk & 3) * 32) >> 4;
            umma_ss(tSx, dQx + off, dHi + static_cast<uint64_t>(kk * (2048 >> 4)), idPV, kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * (kTileM * 128) + (kk & 3) * 32) >> 4;
            umma_ss(tSx, dQx + off, dLo + static_cast<uint64_t>(kk * (2048 >> 4)), idPV, 1u);
          }
          umma_commit(bLinDone(x));
        }
      }
      // all issued MMAs complete before teardown
      umma_commit(bFinal(x));
      mbar_drain(bFinal(x), 0, ab.limit_ns);
    }
  } else if (warp >= 4 && warp < 12) {
    // ---------------------------------------------------------- softmax
    const int x = (warp - 4) >> 2;                   // query tile of this warpgroup
    if (x == 0 || hasB) {
      const int r = (threadIdx.x - 128) & 127;       // row of the tile = TMEM lane
      const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
      const uint32_t tO = trow + 256u + static_cast<uint32_t>(x * 128);
      const int q_end = x ? g.q_end[1] : g.q_end[0];
      const int qn = (x ? g.q0[1] : g.q0[0]) + r;
      const bool row_valid = qn < q_end;
      const bool full_tile = q_end - (x ? g.q0[1] : g.q0[0]) == kTileM;   // uniform in the warpgroup
      int lo = 0, hi = 0;
      if (p.n_kseg == 0) key_range(p, row_valid ? qn : q_end - 1, lo, hi);
      float m_run = -INFINITY, l_run = 0.f;
      const float sl2 = p.scale_log2;
      bool ok = true;
      int pv_seen = 0;   // completions of bPvDone(x) known to this thread
      if constexpr (ROPE == kRopeQ) {
        // rotate this thread's query row of Q_x in place, once
        ok = mbar_wait(bQFull(x), 0, ab, kStatusTimeoutSoftmax);
        const int Fr = p.rope_Hg * p.rope_Wg;
        RopePos pos{0, 0, 0};
        if (row_valid) {
          const int in = qn % Fr;
          pos = RopePos{p.qoff + qn / Fr, in / p.rope_Wg, in % p.rope_Wg};
        }
        rope_row_inplace<D>(smem + C::kOffQ + x * C::kTileBytes, r, pos, p);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bQReady(x));
      }
      // segment mode with equal segments: the valid keys of each tile follow
      // from the tile's index inside its segment, kept as a running count
      const int seg_tiles = p.seg_tok > 0 ? (p.seg_tok + kTileN - 1) / kTileN : 1;
      int seg_t = p.seg_tok > 0 ? g.t0 % seg_tiles : 0;
      // No early exit: a failed wait only happens after the CTA aborted,
      // when every later wait fails at once; the warp stays converged for
      // the warp-collective TMEM accesses.
      for (int u = 0; u < ns; ++u) {
        const int bb = u & 1;
        if (!mbar_wait(bSFull(x, bb), (u >> 1) & 1, ab, kStatusTimeoutSoftmax)) ok = false;
        tc_fence_after();
        const uint32_t tS = trow + static_cast<uint32_t>(x * 128 + bb * kSub);
        int col_lo = 0, col_hi = kSub;
        if (p.n_kseg == 0) {
          const int k0 = g.tg.kbeg + g.t0 * kTileN + u * kSub;
          col_lo = lo - k0;
          col_hi = hi - k0;
        } else if (p.seg_tok > 0) {
          col_hi = min(kTileN, p.seg_tok - seg_t * kTileN) - bb * kSub;
          if (bb && ++seg_t == seg_tiles) seg_t = 0;
        } else {
          col_hi = key_tile(p, g.tg, g.t0 + (u >> 1)).valid - bb * kSub;
        }
        const bool masked = col_lo > 0 || col_hi < kSub;
        uint32_t s0[32], s1[32];
        tmem_ld32(tS, s0);
        tmem_ld32(tS + 32, s1);
        tmem_ld_wait_dep(s0);
        reg_tie32(s1);
        // row max over all 64 columns of an unmasked sub-tile
        auto row_max = [&]() {
          float mx8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
#pragma unroll
          for (int c = 0; c < 32; ++c)
            mx8[c & 7] = fmax3(mx8[c & 7], __uint_as_float(s0[c]), __uint_as_float(s1[c]));
          return fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        };
        // P = exp2(s * scale * log2e + nm) of an unmasked sub-tile into the
        // first half of the S buffer, 16 columns (32 keys) at a time; returns
        // the row sum (packed fp32x2 partial sums).  CLAMP caps the
        // polynomial's argument at 64, where its exponent insertion would
        // otherwise wrap (MUFU ex2 saturates to inf by itself).
        auto exps = [&](float nm, auto clamp) {
          constexpr bool CLAMP = decltype(clamp)::value;
          float rs2[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const uint32_t* sq = q == 0 ? s0 : s1;
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              float x0, x1, p0, p1;
              ffma2(x0, x1, __uint_as_float(sq[c]), __uint_as_float(sq[c + 1]), sl2, sl2, nm, nm);
              if ((PolyMask<D>::value >> ((c >> 1) & 7)) & 1u) {
                if constexpr (CLAMP) {
                  x0 = fminf(x0, 64.f);
                  x1 = fminf(x1, 64.f);
                }
                ex2_poly2(p0, p1, x0, x1);
              } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
              }
              fadd2(rs2[(c >> 1) & 1][0], rs2[(c >> 1) & 1][1], p0, p1);
              pk[c / 2] = pack_bf16x2(p0, p1);
            }
            tmem_st16(tS + q * 16, pk);
          }
          return (rs2[0][0] + rs2[0][1]) + (rs2[1][0] + rs2[1][1]);
        };
        float factor = 1.f;
        bool resc = false;
        float rs;
        // Every tcgen05.st below (and each full-mask vote) is warp-collective,
        // so both branches are taken by the whole warp: the speculative one
        // only when no row of the warp is masked in this sub-tile (masks
        // differ per row in the chunk-causal and sliding modes).
        const bool spec = SpecExp<D, ROPE, HYB>::value && u > 0 && !__any_sync(0xffffffffu, masked);
        if (spec) {
          // exponentials against the current reference max before this
          // sub-tile's max is known.  The row sum bounds every term, so a sum
          // of at most 2^threshold proves each exponent argument is at most
          // the threshold, which is all the reference needs: the max is then
          // never taken.  Otherwise take it, move the reference if it grew by
          // more than the threshold, and redo the sub-tile.
          rs = exps(m_run == -INFINITY ? 0.f : -m_run, std::true_type{});
          // a row with no visible key before this sub-tile has no reference
          // yet (its terms above were taken against 0): it sets one now;
          // !(rs <= bound) also catches inf and NaN
          const bool need = m_run == -INFINITY || !(rs <= kSpecSumBound);
          if (__any_sync(0xffffffffu, need)) {
            if (need) {   // per lane; no collective operation inside
              const float m_new = fmaxf(m_run, row_max() * sl2);
              if (m_new > m_run + kRescaleThreshold) {
                factor = ex2_approx(m_run - m_new);   // 0 when m_run = -inf
                m_run = m_new;
                resc = true;
              }
            }
            if (__any_sync(0xffffffffu, resc)) {
              tmem_st_wait();   // the first stores land before they are replaced
              rs = exps(m_run == -INFINITY ? 0.f : -m_run, std::false_type{});
            }
          }
        } else {
          // row max over the visible columns (per lane; no collective inside)
          float mx;
          if (!masked) {
            mx = row_max();
          } else {
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float v0 = (c >= col_lo && c < col_hi) ? __uint_as_float(s0[c]) : -INFINITY;
              const float v1 = (c + 32 >= col_lo && c + 32 < col_hi) ? __uint_as_float(s1[c]) : -INFINITY;
              mx8[c & 7] = fmax3(mx8[c & 7], v0, v1);
            }
            mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
          }
          if (x == 0 && u == 0 && lane == 0) mbar_arrive(bStartB);   // every CTA has sub-tile 0 (ns >= 2)
          const float m_new = fmaxf(m_run, mx * sl2);
          if (m_new > m_run + kRescaleThreshold) {
            factor = ex2_approx(m_run - m_new);   // 0 when m_run = -inf
            m_run = m_new;
            resc = true;
          }
          const float nm = (m_run == -INFINITY) ? 0.f : -m_run;
          // P = exp2(s * scale * log2e - m) into the first half of the S
          // buffer, 16 columns (32 keys) at a time; the per-lane branch only
          // picks the values, the stores run converged after it
          float rs2[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const uint32_t* sq = q == 0 ? s0 : s1;
            uint32_t pk[16];
            if (!masked) {
#pragma unroll
              for (int c = 0; c < 32; c += 2) {
                float x0, x1, p0, p1;
                ffma2(x0, x1, __uint_as_float(sq[c]), __uint_as_float(sq[c + 1]), sl2, sl2, nm, nm);
                if ((PolyMask<D>::value >> ((c >> 1) & 7)) & 1u) {
                  ex2_poly2(p0, p1, x0, x1);
                } else {
                  p0 = ex2_approx(x0);
                  p1 = ex2_approx(x1);
                }
                fadd2(rs2[(c >> 1) & 1][0], rs2[(c >> 1) & 1][1], p0, p1);
                pk[c / 2] = pack_bf16x2(p0, p1);
              }
            } else {
#pragma unroll
              for (int c = 0; c < 32; c += 2) {
                const int col = q * 32 + c;
                float p0 = ex2_approx(fmaf(__uint_as_float(sq[c]), sl2, nm));
                float p1 = ex2_approx(fmaf(__uint_as_float(sq[c + 1]), sl2, nm));
                p0 = (col >= col_lo && col < col_hi) ? p0 : 0.f;
                p1 = (col + 1 >= col_lo && col + 1 < col_hi) ? p1 : 0.f;
                rs2[(c >> 1) & 1][0] += p0;
                rs2[(c >> 1) & 1][1] += p1;
                pk[c / 2] = pack_bf16x2(p0, p1);
              }
            }
            tmem_st16(tS + q * 16, pk);
          }
          rs = (rs2[0][0] + rs2[0][1]) + (rs2[1][0] + rs2[1][1]);
        }
        // O_x rescale: wait until the P V of the previous sub-tile (which
        // accumulates into O_x) has completed; the next one waits for P below.
        // The single-phase parity wait is sound because S_x(u), issued after
        // P_x(u - 2) V, has completed: bPvDone is at most one phase behind.
        if (__any_sync(0xffffffffu, resc && u > 0)) {
          if (pv_seen < u) {
            if (!mbar_wait(bPvDone(x), (u - 1) & 1, ab, kStatusTimeoutSoftmax)) ok = false;
            pv_seen = u;
            tc_fence_after();
          }
          const float f = (resc && u > 0) ? factor : 1.f;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t orr[32];
            tmem_ld32(tO + c * 32, orr);
            tmem_ld_wait_dep(orr);
#pragma unroll
            for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * f);
            tmem_st32(tO + c * 32, orr);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        // (self-test only: the first warp of tile A withholds its arrival for
        // sub-tile 1, so tile A's issuer waits until its bound runs out)
        const bool withhold = p.test_withhold && x == 0 && warp == 4 && u == 1;
        if (lane == 0 && !withhold) mbar_arrive(bPFull(x, bb));
        l_run = l_run * factor + rs;
      }
      float dl = 0.f;   // hybrid: phi(q_r) . z_c
      if constexpr (HYB) {
        // Q_x is free as soon as this tile's last scores are in: every MMA
        // reading it has completed.  z_c was copied into shared memory at
        // the start.
        bool okh = ok && mbar_wait(bZFull, 0, ab, kStatusTimeoutSoftmax);
        const int c = g.q0[0] / p.q_seg_len;   // the pair's chunk
        // phi(q_r) in place of row r of Q_x (bf16), and phi(q_r) . z_c in fp32
        const fmap::Poly aq = fmap::load_poly(p.hyb_coef, 0, p.H, h);
        const uint32_t qrow = sQ + static_cast<uint32_t>(x * C::kTileBytes);
        const uint32_t sz = sbase + C::kOffZ;
        // one loop per feature map (the map is uniform over the launch); four
        // partial sums keep the dot product's dependency chain short
        auto phi_rows = [&](auto kind) {
          constexpr int K = decltype(kind)::value;
          float d4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
          for (int blk = 0; blk < D / 64; ++blk) {
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
              const uint32_t addr = qrow + blk * (kTileM * 128) + sw128_offset(r, c8);
              const uint4 v = lds128(addr);
              const uint4 z0 = lds128(sz + (blk * 64 + c8 * 8) * 4);
              const uint4 z1 = lds128(sz + (blk * 64 + c8 * 8 + 4) * 4);
              const uint32_t zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
              uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float x0 = bf16lo_to_f32(w4[e]), x1 = bf16hi_to_f32(w4[e]);
                x0 = fmap::feature(K, aq, x0);
                x1 = fmap::feature(K, aq, x1);
                w4[e] = pack_bf16x2(x0, x1);
                // the denominator takes the same bf16 values the read-out MMA multiplies
                d4[e] = fmaf(bf16lo_to_f32(w4[e]), __uint_as_float(zz[2 * e]), d4[e]);
                d4[e] = fmaf(bf16hi_to_f32(w4[e]), __uint_as_float(zz[2 * e + 1]), d4[e]);
              }
              sts128(addr, make_uint4(w4[0], w4[1], w4[2], w4[3]));
            }
          }
          return (d4[0] + d4[1]) + (d4[2] + d4[3]);
        };
        dl = p.hyb_fmap == fmap::kFmapPoly3 ? phi_rows(std::integral_constant<int, fmap::kFmapPoly3>{})
                                            : phi_rows(std::integral_constant<int, fmap::kFmapElu1>{});
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bPhiReady(x));
        if (x == 0) {
          // S_c (fp32 [D][D], row a = key feature) -> bf16 hi + lo, MN-major
          // 128B-swizzled B operand tiles (64-column blocks of D rows) in the
          // K stages, which are free once tile B's last Q K^T has completed
          // too.  Tile A's warpgroup converts all of it, so tile A's read-out
          // does not wait for tile B's loop to end; consecutive threads take
          // consecutive 32-byte pieces of S_c (coalesced loads).
          if (hasB) okh = okh && mbar_wait(bQKDone(1), 0, ab, kStatusTimeoutSoftmax);
          tc_fence_after();
          const float* src = p.hyb_S + ((static_cast<size_t>(c) * p.B + b) * p.H + h) * D * D;
#pragma unroll 8
          for (int i = 0; i < D * D / (8 * kTileM); ++i) {
            const int id = i * kTileM + r;        // 8-float piece: row id / 16, piece id % 16
            const int a = id >> 4, cc = id & 15;
            const float4 a0 = __ldg(reinterpret_cast<const float4*>(src + a * D + cc * 8));
            const float4 a1 = __ldg(reinterpret_cast<const float4*>(src + a * D + cc * 8 + 4));
            const float xs[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            uint32_t hi4[4], lo4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              hi4[e] = pack_bf16x2(xs[2 * e], xs[2 * e + 1]);
              lo4[e] = pack_bf16x2(xs[2 * e] - bf16lo_to_f32(hi4[e]), xs[2 * e + 1] - bf16hi_to_f32(hi4[e]));
            }
            const uint32_t off = (cc >> 3) * (D * 128) + sw128_offset(a, cc & 7);
            sts128(sK + off, make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]));
            sts128(sK + D * D * 2 + off, make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(bScReady);
        }
        okh = okh && mbar_wait(bLinDone(x), 0, ab, kStatusTimeoutSoftmax);
        tc_fence_after();
        ok = okh;
      }
      // epilogue: O_x / l -> bf16, lse
      if (ok && ns > 0) {
        // bPvDone may still be two completions short here; bODone completes
        // exactly once, after the last P V of this tile
        ok = mbar_wait(bODone(x), 0, ab, kStatusTimeoutSoftmax);
        tc_fence_after();
      }
      ok = __all_sync(0xffffffffu, ok);   // the TMEM loads below are warp-collective
      if (ok && !HYB && nsplit > 1) {
        // key split: this CTA's partial result, o / l in fp32 and m + log2 l,
        // for the pair's merging CTA
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        const size_t prow = part_row(p, g, b, h, split, nsplit, tail_item, qn);
        float* dst = p.part_o + prow * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orr[32];
          tmem_ld32(tO + c * 32, orr);
          tmem_ld_wait_dep(orr);
          if (row_valid) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
              __stcg(reinterpret_cast<float4*>(dst + c * 32) + e,
                     make_float4(__uint_as_float(orr[4 * e]) * inv, __uint_as_float(orr[4 * e + 1]) * inv,
                                 __uint_as_float(orr[4 * e + 2]) * inv, __uint_as_float(orr[4 * e + 3]) * inv));
          }
        }
        if (row_valid) __stcg(p.part_lse + prow, l_run > 0.f ? m_run + __log2f(l_run) : -INFINITY);
      } else if (ok) {
        // hybrid: o = (2^m O + lin) / (2^m l + phi(q).z) with O, l relative
        // to the softmax's reference max m; scaled by 2^-m when m > 0, so
        // neither factor overflows
        const float as = (HYB && m_run <= 0.f) ? ex2_approx(m_run) : 1.f;   // 0 when m = -inf
        const float fl = HYB ? (m_run > 0.f ? ex2_approx(-m_run) : 1.f) : 0.f;
        const float den = as * l_run + fl * dl;
        const float inv = den > 0.f ? 1.f / den : 0.f;
        __nv_bfloat16* orow = p.o + ((static_cast<size_t>(b) * p.Lq + qn) * p.H + h) * D;
        // a full tile's rows go through its Q buffer (free: every MMA reading
        // it has completed) and leave with one TMA store per 64-column block;
        // a partial tile's rows past its end may belong to the next segment,
        // so its threads store their own rows
        const uint32_t stage = sQ + static_cast<uint32_t>(x * C::kTileBytes);
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orr[32];
          if (ns > 0) {
            tmem_ld32(tO + c * 32, orr);
            tmem_ld_wait_dep(orr);
            if constexpr (HYB) {
              uint32_t lin[32];
              tmem_ld32(trow + static_cast<uint32_t>(x * 128 + c * 32), lin);
              tmem_ld_wait_dep(lin);
#pragma unroll
              for (int e = 0; e < 32; ++e)
                orr[e] = __float_as_uint(fmaf(fl, __uint_as_float(lin[e]), as * __uint_as_float(orr[e])));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) orr[e] = 0u;
          }
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * inv, __uint_as_float(orr[2 * e + 1]) * inv);
          if (full_tile) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              sts128(stage + (c >> 1) * (kTileM * 128) + sw128_offset(r, (c & 1) * 4 + e),
                     make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]));
          } else if (row_valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
          }
        }
        if (p.lse && row_valid) {
          const float lse = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
          p.lse[(static_cast<size_t>(b) * p.H + h) * p.Lq + qn] = lse;
        }
      }
      if (full_tile && (HYB || nsplit <= 1)) {
        // every thread of the warpgroup takes part (no early exit above), so
        // the barrier completes; the store runs only if all rows were staged
        fence_proxy_async_smem();
        const bool all_ok = x ? bar_and<4, 128>(ok) : bar_and<3, 128>(ok);
        if (all_ok && threadIdx.x == 128 + 128 * x) {
#pragma unroll
          for (int blk = 0; blk < D / 64; ++blk)
            tma_store_4d(&tmO, sQ + x * C::kTileBytes + blk * (kTileM * 128), blk * 64, h, x ? g.q0[1] : g.q0[0],
                         b);
          bulk_commit();
          bulk_wait_read_all();
        }
      }
    }
  }

  if (!HYB && nsplit > 1 && warp >= 4 && warp < 12) {
    // key split: count this CTA's partial in; the pair's last CTA merges
    __threadfence();
    asm volatile("bar.sync 2, 256;" ::: "memory");
    volatile uint32_t* last = misc + 2;
    const size_t pc = p.tail_split ? static_cast<size_t>(tail_item)
                                   : (static_cast<size_t>(b) * p.H + h) * p.n_pairs + pr;
    if (threadIdx.x == 128) {
      const uint32_t old = atomicAdd(p.pair_count + pc, 1u);
      *last = old == static_cast<uint32_t>(nsplit) - 1u ? 1u : 0u;
      __threadfence();
    }
    asm volatile("bar.sync 2, 256;" ::: "memory");
    if (*last) {
      merge_splits<D>(p, g, b, h, warp, lane, nsplit, tail_item);
      if (threadIdx.x == 128) p.pair_count[pc] = 0u;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (stepping) step_exit(p);
}

}  // namespace attn
}  // namespace vattn
