// Attention forward for sm_100a with the key rotation fused in: one CTA per
// 128-query tile of one head, every K tile rotated in shared memory.
//
// What it computes (per query row i, visible key set A(i) given by the
// mode): o_i = sum_{j in A(i)} softmax_j(scale * q_i . k_j) v_j, with q and
// k rotated by 3D-RoPE at their (t, h, w) positions — the spatiotemporal
// self-attention of Wan-style DiTs and of FlashDecoder ("Transformer
// Backbone Design" Sec. 3.2; "Streaming with Rolling KV Cache" Sec. 3.3).
// This kernel serves calls that give RoPE but no key workspace (and
// streaming over a raw, un-rotated ring); every other attention call runs
// the two-tile kernel of attention_pair.cuh.  This header also holds the
// parameter block, the mask geometry and the key-segment walk both kernels
// share.
//
// Warp roles (one elected lane issues for the single-thread roles):
//   warp 0        TMA producer: Q tile once, then K tiles (multi-stage ring)
//   warp 1        TMEM allocation + tcgen05.mma issue
//   warp 2        TMA producer: V tiles
//   warps 4..11   two softmax warpgroups: thread r of either owns query row
//                 r of the tile (TMEM lane r); warpgroup 0 takes score
//                 columns 0-63 of every key tile, warpgroup 1 columns 64-127
//                 (row max exchanged in shared memory each tile, row sums
//                 combined at the end); P (bf16) into TMEM, O rescale,
//                 epilogue.
//   warps 12..15  RoPE of the Q tile and of every K tile in shared memory
//
// TMEM columns (512 allocated): S double buffer [0,128) and [128,256) fp32,
// O [256, 256+D) fp32, P [384, 448) bf16 pairs.
// S = Q K^T is an SS MMA (both operands K-major, 128B swizzle);
// O += P V is a TS MMA (P from TMEM, V MN-major in shared memory).
#pragma once
#include <type_traits>

#include "common.cuh"

namespace vattn {
namespace attn {

using namespace sm100;

constexpr int kTileM = 128;   // query rows per CTA
constexpr int kTileN = 128;   // keys per tile
constexpr int kMaxKeySegments = 8;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP = 384;
constexpr uint32_t kTmemCols = 512;
// Rescale O only when the running max grows by more than this (log2
// units): stale maxima keep every exp2 argument below it, so fp32 stays
// far from overflow while most tiles skip the O correction.
constexpr float kRescaleThreshold = 8.0f;
// Speculative exponentials in the two-tile kernel: an unmasked sub-tile
// after a CTA's first is exponentiated against the current reference max,
// and its own max is taken only when the row sum exceeds 2^threshold.  On
// for head dim 64 (+2.3 % measured on B200), for the instantiation that
// rotates Q in the kernel (+2.0 % and +1.6 % on the 1.3B- and 14B-like
// calls) and for the hybrid (+1.2 %); off for head dim 128 without RoPE,
// where its extra live registers cost more than the row max saves (-0.9 %).
template <int D, int ROPE, bool HYB>
struct SpecExp {
  static constexpr bool value = D == 64 || ROPE != 0 || HYB;
};
constexpr float kSpecSumBound = 256.0f;   // 2^kRescaleThreshold
// Which of every 8 consecutive score pairs take the FMA-pipe polynomial
// exp2 instead of MUFU ex2 (bit i set: pair i mod 8).  At head dim 128 the
// MUFU keeps pace with the tensor core and the polynomial only adds issue
// pressure; at head dim 64 the MMA work per score halves and a quarter of
// the exponentials move to the FMA pipe (measured on B200).
template <int D>
struct PolyMask {
  static constexpr uint32_t value = D == 64 ? 0x88u : 0x00u;
};

enum Mode : int { kFull = 0, kChunkCausal = 1, kSliding = 2 };

struct KeySegment {
  int kmap;     // K source: 0 = tmK, 1 = tmK2
  int kc3;      // K fourth TMA coordinate = kc3 + batch index
  int vmap;     // V source: 0 = tmV, 1 = tmV2
  int vc3;      // V fourth TMA coordinate = vc3 + batch index
  int tok0;     // first token of the segment along the token axis
  int n_tok;    // tokens in the segment
  int frame;    // absolute frame index (RoPE t of every key in it)
  int tile0;    // number of key tiles in earlier segments
};

// The frame a streaming step appends, copied by the step's first CTAs
// (raw K and V into the ring slot, K rotated at its frame into the rotated
// ring) while the attention CTAs of the same launch run.
struct AppendWork {
  const uint4* k;           // frame K, V: bf16 [B][F][Hkv][D]
  const uint4* v;
  uint4* kr;                // raw ring slot
  uint4* vr;
  uint4* krot;              // rotated ring slot (nullable: no rotation)
  int32_t* ids;             // frame id table: ids[slot] = frame
  int slot, frame;
  long long rows;           // B * F
  int F;                    // tokens per stream frame
  int t0;                   // RoPE t of the frame's first token
};

constexpr int kMaxSplit = 16;   // key splits per query-tile pair

struct Params {
  __nv_bfloat16* o;
  float* lse;
  uint32_t* status;
  int B, Lq, Lk, H, Hkv;
  float scale_log2;         // scale * log2(e)
  int mode, F, chunk, wb, wf, qoff, koff;
  int q_seg_len;            // query tiles restart at multiples of this
  int q_tiles_per_seg;
  int n_q_tiles;
  int reverse_q;            // heaviest tiles first (chunk-causal)
  int n_kseg;               // 0: contiguous keys with the mode's masks
  KeySegment kseg[kMaxKeySegments];
  int seg_tok;              // segment mode: every segment holds this many tokens (0: lengths differ)
  // RoPE
  const float2* rope_tab;   // [max_pos][D/2] (cos, sin)
  int rope_Hg, rope_Wg, rope_pt, rope_ph, rope_maxpos;
  // hybrid chunk attention: per-chunk exclusive state prefix
  const float* hyb_S;       // [C][B][H][D][D]
  const float* hyb_z;       // [C][B][H][D]
  int hyb_fmap;             // feature map of the read-out (fmap::kFmapElu1 / kFmapPoly3)
  const float* hyb_coef;    // [2][H][4] polynomial coefficients (map 0 = q is used here)
  int lead;                 // SLIDING only: the key window also reaches this many tokens back
  // self-test knobs (zero in every attention call): a bound on each wait
  // other than the default, and withholding one softmax arrival so that a
  // wait of the MMA issuer runs out
  uint64_t wait_limit_ns;
  int test_withhold;
  // two-tile kernel only: a 1-D grid over (append CTAs, pairs, heads,
  // batch, split) instead of (pairs, heads, batch)
  int linear_grid;
  int n_pairs;              // query-tile pairs per (batch, head)
  // key split (segment mode): split s walks key tiles
  // [s * split_tiles, (s + 1) * split_tiles); with n_split > 1 every CTA
  // writes its partial result and the last CTA of a pair merges them
  int n_split;
  int split_tiles;
  float* part_o;            // [n_split][B][H][Lq][D] fp32: the split's o (normalised by its own l)
  float* part_lse;          // [n_split][B][H][Lq] fp32: m + log2 l of the split (log2 domain)
  uint32_t* pair_count;     // [B][H][n_pairs] arrivals; the merging CTA puts it back to 0
  // streaming step: CTAs [0, n_append) of the linear grid copy the frame
  int n_append;
  AppendWork app;
  uint32_t* step_sync;      // [0] append shares done, [1] CTAs exited; back to 0 at the last exit
  int wait_tile;            // key tiles >= this read keys the append CTAs write (-1: none)
  int total_ctas;
  // tail split (linear grid): the first n_normal (pair, head, batch) items
  // run whole, each later item as n_split CTAs over parts of its key
  // range, with partials in a compact layout ([item - n_normal][split][256
  // rows of the pair])
  int tail_split;
  int n_normal;
};

template <int D>
struct Cfg {
  static constexpr int kTileBytes = kTileM * D * 2;  // one 128 x D bf16 tile
  static constexpr int kBlocks = D / 64;             // 64-column swizzle blocks per tile
  static constexpr int kStages = (D == 128) ? 3 : 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  static constexpr int kNumBars = 2 + 5 * kStages + 4 + 2 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffXchg = kOffMisc + 64;   // row max exchange [2 parities][2 wg][128] fp32
  // The dynamic shared-memory window starts 1024-byte aligned (checked at
  // kernel entry), so no alignment slack is reserved.
  static constexpr int kSmemBytes = kOffXchg + 2048;
};

// Visible key range [lo, hi) of query token n (contiguous keys).  For all
// three modes the visible keys of one query are an interval and both ends
// are non-decreasing in n.
__device__ __forceinline__ void key_range(const Params& p, int n, int& lo, int& hi) {
  if (p.mode == kFull) {
    lo = 0;
    hi = p.Lk;
    return;
  }
  const long long fq = p.qoff + n / p.F;
  long long a, b;
  if (p.mode == kChunkCausal) {
    a = 0;
    b = ((fq / p.chunk) + 1) * p.chunk - p.koff;
  } else {
    a = fq - p.wb - p.koff;
    b = fq + p.wf + 1 - p.koff;
  }
  a *= p.F;
  b *= p.F;
  if (p.mode == kSliding) a -= p.lead;
  lo = static_cast<int>(a < 0 ? 0 : (a > p.Lk ? p.Lk : a));
  hi = static_cast<int>(b < 0 ? 0 : (b > p.Lk ? p.Lk : b));
}

struct TileGeom {
  int q0, q_end;      // query rows [q0, q_end) of this CTA
  int kbeg, kend;     // contiguous key range covered by tiles
  int n_tiles;
};

__device__ __forceinline__ TileGeom tile_geom(const Params& p, int qt) {
  TileGeom g;
  const int seg = qt / p.q_tiles_per_seg;
  const int t = qt - seg * p.q_tiles_per_seg;
  g.q0 = seg * p.q_seg_len + t * kTileM;
  int e = (seg + 1) * p.q_seg_len;
  if (e > p.Lq) e = p.Lq;
  g.q_end = min(g.q0 + kTileM, e);
  if (p.n_kseg == 0) {
    int lo0, hi0, lo1, hi1;
    key_range(p, g.q0, lo0, hi0);
    key_range(p, g.q_end - 1, lo1, hi1);
    g.kbeg = lo0;
    g.kend = hi1;
    g.n_tiles = g.kend > g.kbeg ? (g.kend - g.kbeg + kTileN - 1) / kTileN : 0;
  } else {
    g.kbeg = g.kend = 0;
    const KeySegment& last = p.kseg[p.n_kseg - 1];
    g.n_tiles = last.tile0 + (last.n_tok + kTileN - 1) / kTileN;
  }
  return g;
}

struct KeyTile {
  int kmap, kc3, vmap, vc3;   // TMA sources and 4th coordinates (minus batch)
  int k0;             // token start
  int valid;          // keys in this tile that exist (segment mode)
  int frame;          // segment frame (segment mode)
};

__device__ __forceinline__ KeyTile key_tile(const Params& p, const TileGeom& g, int j) {
  KeyTile kt;
  if (p.n_kseg == 0) {
    kt.kmap = kt.vmap = 0;
    kt.kc3 = kt.vc3 = 0;
    kt.k0 = g.kbeg + j * kTileN;
    kt.valid = min(kTileN, g.kend - kt.k0);
    kt.frame = 0;
  } else {
    int s = 0;
#pragma unroll 1
    for (int i = 1; i < p.n_kseg; ++i)
      if (p.kseg[i].tile0 <= j) s = i;
    const KeySegment& sg = p.kseg[s];
    const int t = j - sg.tile0;
    kt.kmap = sg.kmap;
    kt.kc3 = sg.kc3;
    kt.vmap = sg.vmap;
    kt.vc3 = sg.vc3;
    kt.k0 = sg.tok0 + t * kTileN;
    kt.valid = min(kTileN, sg.n_tok - t * kTileN);
    kt.frame = sg.frame;
  }
  return kt;
}

// (t, h, w) -> table rows for the rotation of one token.
struct RopePos {
  int t, h, w;
};

// Rotate one 128-byte-swizzled 128 x D bf16 tile row in place: channel pair
// j of the row turns by the angle of its axis position.  Row r of a tile is
// contiguous 64-element blocks, one per swizzle block.
template <int D>
__device__ __forceinline__ void rope_row_inplace(uint8_t* tile, uint32_t r, RopePos pos, const Params& p) {
  const float2* row_t = p.rope_tab + pos.t * (D / 2);
  const float2* row_h = p.rope_tab + pos.h * (D / 2);
  const float2* row_w = p.rope_tab + pos.w * (D / 2);
  const int pt = p.rope_pt, pth = p.rope_pt + p.rope_ph;
#pragma unroll 2
  for (int g = 0; g < D / 32; ++g) {   // 4 chunks of 16 bytes = 16 channel pairs per group
    uint4 v[4];
    float2 cs[16];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c16 = g * 4 + u;
      v[u] = *reinterpret_cast<const uint4*>(tile + (c16 >> 3) * (kTileM * 128) + sw128_offset(r, c16 & 7));
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int j = g * 16 + e;
      const float2* src = j < pt ? row_t : (j < pth ? row_h : row_w);
      cs[e] = __ldg(src + j);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint32_t w4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 c2 = cs[u * 4 + e];
        const float x0 = bf16lo_to_f32(w4[e]), x1 = bf16hi_to_f32(w4[e]);
        w4[e] = pack_bf16x2(x0 * c2.x - x1 * c2.y, x0 * c2.y + x1 * c2.x);
      }
      const int c16 = g * 4 + u;
      *reinterpret_cast<uint4*>(tile + (c16 >> 3) * (kTileM * 128) + sw128_offset(r, c16 & 7)) =
          make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
  }
}

// RoPE modes: 0 none; 1 Q rotated in the kernel (once per CTA), K already
// rotated by the caller path; 2 Q and every K tile rotated in the kernel.
constexpr int kRopeNone = 0, kRopeQ = 1, kRopeQK = 2;

constexpr int kFusedThreads = 512;

template <int D>
__global__ void __launch_bounds__(kFusedThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmK2,
                    const __grid_constant__ CUtensorMap tmV2, const Params p) {
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t sbase = smem_addr(smem);
  if (sbase & 1023u) {   // 128B-swizzled operand tiles need 1024-byte alignment
    if (threadIdx.x == 0 && p.status) atomicCAS(p.status, 0u, kStatusSmemAlign);
    return;
  }
  const uint32_t sQ = sbase + C::kOffQ, sK = sbase + C::kOffK, sV = sbase + C::kOffV;
  const uint32_t bar0 = sbase + C::kOffBar;
  // barrier map
  const uint32_t bQFull = bar0, bQReady = bar0 + 8;
  auto bKFull = [&](int s) { return bar0 + 16 + 8 * s; };
  auto bKReady = [&](int s) { return bar0 + 16 + 8 * (NS + s); };
  auto bKEmpty = [&](int s) { return bar0 + 16 + 8 * (2 * NS + s); };
  auto bVFull = [&](int s) { return bar0 + 16 + 8 * (3 * NS + s); };
  auto bVEmpty = [&](int s) { return bar0 + 16 + 8 * (4 * NS + s); };
  const uint32_t bx = bar0 + 16 + 8 * 5 * NS;
  auto bSFull = [&](int b) { return bx + 8 * b; };
  auto bSFree = [&](int b) { return bx + 16 + 8 * b; };
  const uint32_t bPFull = bx + 32, bPvDone = bx + 40;
  const uint32_t bFinal = bx + 48;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile uint32_t* tmem_slot = misc;
  volatile uint32_t* abort_flag = misc + 1;
  Abort ab{abort_flag, p.status};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (p.H / p.Hkv);
  const int qt = p.reverse_q ? (p.n_q_tiles - 1 - blockIdx.x) : blockIdx.x;
  const TileGeom g = tile_geom(p, qt);
  if (g.q0 >= g.q_end) return;   // tile past the end of a short last segment
  const int nk = g.n_tiles;

  if (threadIdx.x == 0) {
    mbar_init(bQFull, 1);
    mbar_init(bQReady, 4);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bKFull(s), 1);
      mbar_init(bKReady(s), 4);
      mbar_init(bKEmpty(s), 1);
      mbar_init(bVFull(s), 1);
      mbar_init(bVEmpty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bSFull(i), 1);
      mbar_init(bSFree(i), 8);
    }
    mbar_init(bPFull, 8);
    mbar_init(bPvDone, 1);
    mbar_init(bFinal, 1);
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
    // ------------------------------------------------ producer: Q, then K
    if (lane == 0) {
      mbar_arrive_expect_tx(bQFull, C::kTileBytes);
#pragma unroll
      for (int blk = 0; blk < C::kBlocks; ++blk)
        tma_load_4d(sQ + blk * (kTileM * 128), &tmQ, bQFull, blk * 64, h, g.q0, b);
      int j = 0;
      for (; j < nk; ++j) {
        const int s = j % NS;
        if (j >= NS && !mbar_wait(bKEmpty(s), ((j / NS) - 1) & 1, ab, kStatusTimeoutProducer)) break;
        const KeyTile kt = key_tile(p, g, j);
        const CUtensorMap* m = kt.kmap ? &tmK2 : &tmK;
        mbar_arrive_expect_tx(bKFull(s), C::kTileBytes);
#pragma unroll
        for (int blk = 0; blk < C::kBlocks; ++blk)
          tma_load_4d(sK + s * C::kTileBytes + blk * (kTileM * 128), m, bKFull(s), blk * 64, kvh, kt.k0,
                      kt.kc3 + b);
      }
      // drain: wait until every load issued so far has landed
      for (int i = max(0, j - NS); i < j; ++i) {
        mbar_drain(bKFull(i % NS), (i / NS) & 1, ab.limit_ns);
      }
      mbar_drain(bQFull, 0, ab.limit_ns);
    }
  } else if (warp == 2) {
    // ----------------------------------------------------- producer: V
    if (lane == 0) {
      int j = 0;
      for (; j < nk; ++j) {
        const int s = j % NS;
        if (j >= NS && !mbar_wait(bVEmpty(s), ((j / NS) - 1) & 1, ab, kStatusTimeoutProducer)) break;
        const KeyTile kt = key_tile(p, g, j);
        const CUtensorMap* m = kt.vmap ? &tmV2 : &tmV;
        mbar_arrive_expect_tx(bVFull(s), C::kTileBytes);
#pragma unroll
        for (int blk = 0; blk < C::kBlocks; ++blk)
          tma_load_4d(sV + s * C::kTileBytes + blk * (kTileM * 128), m, bVFull(s), blk * 64, kvh, kt.k0,
                      kt.vc3 + b);
      }
      for (int i = max(0, j - NS); i < j; ++i) {
        mbar_drain(bVFull(i % NS), (i / NS) & 1, ab.limit_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idQK = idesc_bf16_f32(kTileM, kTileN, false, false);
      constexpr uint32_t idPV = idesc_bf16_f32(kTileM, D, false, true);
      const uint32_t tO = tmem + kColO, tP = tmem + kColP;
      bool ok = mbar_wait(bQReady, 0, ab, kStatusTimeoutMma);
      tc_fence_after();
      auto issue_pv = [&](int i) -> bool {
        if (!mbar_wait(bPFull, i & 1, ab, kStatusTimeoutMma)) return false;
        const int s = i % NS;
        if (!mbar_wait(bVFull(s), (i / NS) & 1, ab, kStatusTimeoutMma)) return false;
        tc_fence_after();
        const uint64_t dVs = sdesc_sw128(sV + s * C::kTileBytes, kTileM * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < kTileN / 16; ++kk)
          umma_ts(tO, tP + kk * 8, dVs + static_cast<uint64_t>(kk * (2048 >> 4)), idPV,
                  (i > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bPvDone);
        umma_commit(bVEmpty(s));
        return true;
      };
      // shared-memory descriptors, built once: the start-address field
      // (address >> 4, 14 bits) is advanced by adding (offset >> 4) to the
      // low word, which cannot carry past the field (shared memory < 256 KB)
      const uint64_t dQ = sdesc_sw128(sQ, 16, 1024);
      const uint64_t dK = sdesc_sw128(sK, 16, 1024);
      // S = Q K^T for tile t into S buffer t & 1; it needs K tile t and the
      // buffer's previous tile (t - 2) consumed by the softmax, which is
      // signalled right after that tile's row max, long before its P.
      auto issue_qk = [&](int t) -> bool {
        const int s = t % NS, buf = t & 1;
        if (!mbar_wait(bKReady(s), (t / NS) & 1, ab, kStatusTimeoutMma)) return false;
        if (t >= 2 && !mbar_wait(bSFree(buf), ((t - 2) >> 1) & 1, ab, kStatusTimeoutMma))
          return false;
        tc_fence_after();
        const uint64_t dKs = dK + static_cast<uint64_t>((s * C::kTileBytes) >> 4);
        const uint32_t tS = tmem + (buf ? kColS1 : kColS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * (kTileM * 128) + (kk & 3) * 32) >> 4;
          umma_ss(tS, dQ + off, dKs + off, idQK, kk > 0);
        }
        umma_commit(bSFull(buf));
        umma_commit(bKEmpty(s));
        return true;
      };
      // issue order: QK(0), QK(1), then per tile j: QK(j + 2), PV(j)
      for (int t = 0; ok && t < 2 && t < nk; ++t) ok = issue_qk(t);
      for (int j = 0; ok && j < nk; ++j) {
        if (j + 2 < nk && !issue_qk(j + 2)) {
          ok = false;
          break;
        }
        if (!issue_pv(j)) {
          ok = false;
          break;
        }
      }
      // all issued MMAs complete before teardown
      umma_commit(bFinal);
      mbar_drain(bFinal, 0, ab.limit_ns);
    }
  } else if (warp >= 4 && warp < 12) {
    // ---------------------------------------------------------- softmax
    // Two warpgroups share every row: wg 0 owns score columns [0, 64), wg 1
    // columns [64, 128) of each 128-key tile (and the matching halves of P
    // and of the O columns).  The row max is exchanged through shared memory
    // once per tile; the row sums stay per warpgroup until the epilogue.
    const int wg = (warp - 4) >> 2;
    const int r = (threadIdx.x - 128) & 127;         // row of the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t trow = tmem + lane_base;
    const int qn = g.q0 + r;
    const bool row_valid = qn < g.q_end;
    int lo = 0, hi = 0;
    if (p.n_kseg == 0) key_range(p, row_valid ? qn : g.q_end - 1, lo, hi);
    float* xmax = reinterpret_cast<float*>(smem + C::kOffXchg);   // [2 parities][2 wg][128]
    float m_run = -INFINITY, l_run = 0.f;
    const float sl2 = p.scale_log2;
    bool ok = true;
    int pv_phase = 0;   // completions of bPvDone observed so far
    const int cbase = wg * 64;    // first score column of this warpgroup
    // No early exit: after a failed wait (which only happens once the CTA has
    // aborted, when every later wait fails at once) the remaining tiles run
    // on garbage, so both warpgroups execute the same row-max barriers and
    // meet the epilogue barrier exactly once.
    for (int j = 0; j < nk; ++j) {
      const int buf = j & 1;
      if (!mbar_wait(bSFull(buf), (j >> 1) & 1, ab, kStatusTimeoutSoftmax)) ok = false;
      tc_fence_after();
      const uint32_t tS = trow + (buf ? kColS1 : kColS0) + cbase;
      int col_lo = 0, col_hi = kTileN;
      if (p.n_kseg == 0) {
        const int k0 = g.kbeg + j * kTileN;
        col_lo = lo - k0 - cbase;
        col_hi = hi - k0 - cbase;
      } else {
        const KeyTile kt = key_tile(p, g, j);
        col_hi = kt.valid - cbase;
      }
      const bool masked = col_lo > 0 || col_hi < 64;
      // pass 1: max over this warpgroup's 64 visible columns
      uint32_t a[32], bb[32];
      tmem_ld32(tS, a);
      tmem_ld32(tS + 32, bb);
      tmem_ld_wait_dep2(a, bb);
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
      if (!masked) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          mx8[c & 7] = fmax3(mx8[c & 7], __uint_as_float(a[c]), __uint_as_float(bb[c]));
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          mx8[c & 7] = fmaxf(mx8[c & 7], (c >= col_lo && c < col_hi) ? __uint_as_float(a[c]) : -INFINITY);
          mx8[c & 7] = fmaxf(mx8[c & 7],
                             (c + 32 >= col_lo && c + 32 < col_hi) ? __uint_as_float(bb[c]) : -INFINITY);
        }
      }
      float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      // exchange with the other warpgroup (double-buffered by tile parity)
      xmax[(buf * 2 + wg) * 128 + r] = mx;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      mx = fmaxf(mx, xmax[(buf * 2 + (wg ^ 1)) * 128 + r]);
      // the S buffer is consumed once both halves have their registers
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bSFree(buf));
      const float m_tile = mx * sl2;
      const float m_new = fmaxf(m_run, m_tile);
      float factor = 1.f;
      bool resc = false;
      if (m_new > m_run + kRescaleThreshold) {
        factor = ex2_approx(m_run - m_new);   // 0 when m_run = -inf
        m_run = m_new;
        resc = true;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      // pass 2 on the registers of pass 1: P = exp2(s*scale*log2e - m) on the
      // MUFU ex2; scale-and-subtract and the row sum run as packed fp32x2.
      // Unmasked tiles (all but the edges of a key range) take a loop with
      // no per-element visibility test.
      uint32_t pk[32];
      float rs2[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
      const float nm = -m_use;
      if (!masked) {
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const uint32_t u0 = hq ? bb[c] : a[c], u1 = hq ? bb[c + 1] : a[c + 1];
            float x0, x1, p0, p1;
            ffma2(x0, x1, __uint_as_float(u0), __uint_as_float(u1), sl2, sl2, nm, nm);
            if ((PolyMask<D>::value >> ((c >> 1) & 7)) & 1u) {
              ex2_poly2(p0, p1, x0, x1);
            } else {
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
            }
            fadd2(rs2[(c >> 1) & 3][0], rs2[(c >> 1) & 3][1], p0, p1);
            pk[hq * 16 + c / 2] = pack_bf16x2(p0, p1);
          }
        }
      } else {
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const int col = hq * 32 + c;
            const uint32_t u0 = hq ? bb[c] : a[c], u1 = hq ? bb[c + 1] : a[c + 1];
            float p0 = ex2_approx(fmaf(__uint_as_float(u0), sl2, nm));
            float p1 = ex2_approx(fmaf(__uint_as_float(u1), sl2, nm));
            p0 = (col >= col_lo && col < col_hi) ? p0 : 0.f;
            p1 = (col + 1 >= col_lo && col + 1 < col_hi) ? p1 : 0.f;
            rs2[(c >> 1) & 3][0] += p0;
            rs2[(c >> 1) & 3][1] += p1;
            pk[hq * 16 + c / 2] = pack_bf16x2(p0, p1);
          }
        }
      }
      const float rs = ((rs2[0][0] + rs2[0][1]) + (rs2[1][0] + rs2[1][1])) +
                       ((rs2[2][0] + rs2[2][1]) + (rs2[3][0] + rs2[3][1]));
      // the previous P V reads the P columns and accumulates into O: it must
      // be complete before either is touched
      if (pv_phase < j) {
        if (!mbar_wait(bPvDone, (j - 1) & 1, ab, kStatusTimeoutSoftmax)) ok = false;
        pv_phase = j;
        tc_fence_after();
      }
      const bool o_valid = j > 0;
      if (__any_sync(0xffffffffu, resc && o_valid)) {
        const float f = (resc && o_valid) ? factor : 1.f;
#pragma unroll 1
        for (int c = wg * (D / 64); c < (wg + 1) * (D / 64); ++c) {
          uint32_t orr[32];
          tmem_ld32(trow + kColO + c * 32, orr);
          tmem_ld_wait_dep(orr);
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * f);
          tmem_st32(trow + kColO + c * 32, orr);
        }
      }
      tmem_st32(trow + kColP + wg * 32, pk);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bPFull);
      l_run = l_run * factor + rs;
    }
    // epilogue: O / l -> bf16 (each warpgroup writes its half of the
    // columns), lse from warpgroup 0
    const int need = nk;
    if (ok && need > 0 && pv_phase < need) {
      ok = mbar_wait(bPvDone, (need - 1) & 1, ab, kStatusTimeoutSoftmax);
      tc_fence_after();
    }
    ok = __all_sync(0xffffffffu, ok);   // the epilogue's TMEM loads are warp-collective
    // row sums through the exchange slot of parity nk & 1: its last reads
    // (tile nk - 2) finished before the barrier of tile nk - 1
    float* xl = reinterpret_cast<float*>(smem + C::kOffXchg) + (nk & 1) * 256;   // [2 wg][128]
    xl[wg * 128 + r] = l_run;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    const float l_all = l_run + xl[(wg ^ 1) * 128 + r];
    if (ok) {
      const float inv = l_all > 0.f ? 1.f / l_all : 0.f;
      __nv_bfloat16* orow = p.o + ((static_cast<size_t>(b) * p.Lq + qn) * p.H + h) * D;
#pragma unroll 1
      for (int c = wg * (D / 64); c < (wg + 1) * (D / 64); ++c) {
        uint32_t orr[32];
        if (need > 0) {
          tmem_ld32(trow + kColO + c * 32, orr);
          tmem_ld_wait_dep(orr);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = 0u;
        }
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * inv, __uint_as_float(orr[2 * e + 1]) * inv);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
      if (wg == 0 && p.lse && row_valid) {
        const float lse = l_all > 0.f ? (m_run + __log2f(l_all)) * 0.69314718055994531f : -INFINITY;
        p.lse[(static_cast<size_t>(b) * p.H + h) * p.Lq + qn] = lse;
      }
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------ aux warpgroup
    // RoPE of the Q tile and of every K tile, in shared memory, in place.
    const int r = threadIdx.x - 384;
    {
      const int Fr = p.rope_Hg * p.rope_Wg;
      bool ok = mbar_wait(bQFull, 0, ab, kStatusTimeoutAux);
      if (ok) {
        const int n = g.q0 + r;
        RopePos pos{0, 0, 0};
        if (n < g.q_end) {
          const int in = n % Fr;
          pos = RopePos{p.qoff + n / Fr, in / p.rope_Wg, in % p.rope_Wg};
        }
        rope_row_inplace<D>(smem + C::kOffQ, r, pos, p);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bQReady);
      }
      for (int j = 0; ok && j < nk; ++j) {
        const int s = j % NS;
        if (!mbar_wait(bKFull(s), (j / NS) & 1, ab, kStatusTimeoutAux)) break;
        const KeyTile kt = key_tile(p, g, j);
        RopePos pos{0, 0, 0};
        if (p.n_kseg == 0) {
          const int n = kt.k0 + r;
          if (n < p.Lk) {
            const int in = n % Fr;
            pos = RopePos{p.koff + n / Fr, in / p.rope_Wg, in % p.rope_Wg};
          }
        } else if (r < kt.valid) {
          const int in = kt.k0 + r;   // token index inside its frame
          pos = RopePos{kt.frame, in / p.rope_Wg, in % p.rope_Wg};
        }
        rope_row_inplace<D>(smem + C::kOffK + s * C::kTileBytes, r, pos, p);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bKReady(s));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace attn
}  // namespace vattn
