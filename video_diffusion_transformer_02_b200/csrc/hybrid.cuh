// Hybrid chunk attention, state part (MobileWan recurrence distillation:
// causal linear attention across chunks carried in a running state (s, z),
// feature map phi = elu + 1 or a per-head degree-3 polynomial, see
// feature_map.cuh).
//
//   dS_c = sum_{j in range c} phi(k_j) v_j^T   (D x D, fp32)   -- tcgen05 MMA
//   dz_c = sum_{j in range c} phi(k_j)          (D, fp32)       -- tcgen05 MMA
//                                                  (phi(K)^T times a ones block)
//   S_c  = S_in + sum_{c' < c} dS_c'  (exclusive scan over ranges), same for z
//
// Range c holds the tokens [c ct - ov, (c + 1) ct - ov) clipped to [0, L):
// with softmax chunks that reach ov tokens back into the previous chunk, the
// state read by chunk c covers exactly the keys before its softmax window,
// and the last range ends at L, so the total is the state after all L
// tokens.  ov = 0: ranges are the chunks.
//
// The attention part (softmax inside the chunk plus the linear read-out of
// S_c, z_c) is the HYBRID variant of the attention kernel.
#pragma once
#include "common.cuh"
#include "feature_map.cuh"
#include "grid_dep.cuh"

namespace vattn {
namespace hyb {

using namespace sm100;

struct DeltaParams {
  float* wsS;        // [C][B][H][D][D]
  float* wsz;        // [C][B][H][D]
  uint32_t* status;
  int B, L, H, chunk;
  int overlap;       // ov: ranges are shifted back by it
  int fmap;          // fmap::kFmapElu1 or kFmapPoly3
  const float* coef; // [2][H][4] polynomial coefficients (map 1 = k is used here)
};

// Tokens per stage: 64-row K and V tiles keep a CTA at 97 KB of shared
// memory and 128 TMEM columns, so two CTAs share an SM and the whole grid
// (chunks x heads, 264 CTAs for the MobileWan-style workload) is resident at
// once: no second wave, HBM streamed by every CTA together.
constexpr int kRows = 64;

template <int D>
struct DeltaCfg {
  static constexpr int kTileBytes = kRows * D * 2;
  static constexpr int kStages = 3;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kStages * kTileBytes;
  static constexpr int kOffOnes = 2 * kStages * kTileBytes;   // bf16 ones, one 64-column block of kRows rows
  static constexpr int kOnesBytes = kRows * 128;
  static constexpr int kOffBar = kOffOnes + kOnesBytes;
  static constexpr int kNumBars = 3 * kStages + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;
  static constexpr int kTmemCols = 256;                       // dS in [0, D), dz in [D, D + 16)
};

// grid (H, C, B), 384 threads: warp 0 TMA, warp 1 TMEM + MMA, warps 4..11
// feature map and epilogue.  Feature-map thread t owns the 16-byte chunk
// t % 16 (eight features) of rows t / 16 + 16 i of every tile; the eight
// warps release a stage with one arrive each, with no block-wide barrier
// per tile.  The column sums dz come from the tensor core as well: per
// stage, phi(K)^T times a block of ones (N = 16) accumulates them next to
// dS in TMEM, from the same bf16 values the dS product multiplies.
constexpr int kDeltaThreads = 384;
constexpr int kPhiThreads = 256;

template <int D, int FMAP>
__global__ void __launch_bounds__(kDeltaThreads, 2)
    delta_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const DeltaParams p) {
  static_assert(D == 128, "state delta supports head_dim 128");
  pdl::grid_dep_wait();
  pdl::grid_dep_launch();
  using C = DeltaCfg<D>;
  constexpr int NS = C::kStages;
  constexpr int kChunks = D / 8;                       // 16-byte chunks per row
  constexpr int kRowGroups = kPhiThreads / kChunks;    // rows handled in parallel
  constexpr int kRowsPerThread = kRows / kRowGroups;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t sK = sbase + C::kOffK, sV = sbase + C::kOffV, bar0 = sbase + C::kOffBar;
  auto bFull = [&](int s) { return bar0 + 8 * s; };
  auto bPhi = [&](int s) { return bar0 + 8 * (NS + s); };
  auto bEmpty = [&](int s) { return bar0 + 8 * (2 * NS + s); };
  const uint32_t bDone = bar0 + 8 * 3 * NS;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile uint32_t* tmem_slot = misc;
  volatile uint32_t* abort_flag = misc + 1;
  Abort ab{abort_flag, p.status};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, c = blockIdx.y, b = blockIdx.z;   // heads fastest: CTAs running together read whole token rows
  const int c0 = max(0, c * p.chunk - p.overlap);
  const int c1 = max(c0, min(p.L, (c + 1) * p.chunk - p.overlap));
  const int nt = (c1 - c0 + kRows - 1) / kRows;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bFull(s), 1);
      mbar_init(bPhi(s), kPhiThreads / 32);
      mbar_init(bEmpty(s), 1);
    }
    mbar_init(bDone, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(const_cast<uint32_t*>(tmem_slot)), C::kTmemCols);
    tmem_relinquish();
  }
  if (warp >= 4) {
    // the ones block (bf16 1.0 pairs), an operand of the async proxy
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + C::kOffOnes);
    for (int i = threadIdx.x - 128; i < C::kOnesBytes / 4; i += kPhiThreads) ones[i] = 0x3F803F80u;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int t = 0;
      for (; t < nt; ++t) {
        const int s = t % NS;
        if (t >= NS && !mbar_wait(bEmpty(s), ((t / NS) - 1) & 1, ab, kStatusTimeoutProducer)) break;
        mbar_arrive_expect_tx(bFull(s), 2 * C::kTileBytes);
        const int r0 = c0 + t * kRows;
#pragma unroll
        for (int blk = 0; blk < D / 64; ++blk) {
          tma_load_4d(sK + s * C::kTileBytes + blk * (kRows * 128), &tmK, bFull(s), blk * 64, h, r0, b);
          tma_load_4d(sV + s * C::kTileBytes + blk * (kRows * 128), &tmV, bFull(s), blk * 64, h, r0, b);
        }
      }
      for (int i = max(0, t - NS); i < t; ++i) {
        mbar_drain(bFull(i % NS), (i / NS) & 1, ab.limit_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // D[a][e] += sum_tokens phiK[token][a] * V[token][e]: A = phiK^T and
      // B = V are both MN-major (tokens are the K dimension of the MMA).
      constexpr uint32_t id = idesc_bf16_f32(D, D, true, true);
      constexpr uint32_t idz = idesc_bf16_f32(D, 16, true, true);
      const uint32_t ob = sbase + C::kOffOnes;
      for (int t = 0; t < nt; ++t) {
        const int s = t % NS;
        if (!mbar_wait(bPhi(s), (t / NS) & 1, ab, kStatusTimeoutMma)) break;
        tc_fence_after();
        const uint32_t kb = sK + s * C::kTileBytes, vb = sV + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          umma_ss(tmem, sdesc_sw128(kb + kk * 2048, kRows * 128, 1024),
                  sdesc_sw128(vb + kk * 2048, kRows * 128, 1024), id, (t > 0 || kk > 0) ? 1u : 0u);
        // dz: every column of the ones block is 1, so each of the 16 result
        // columns is the column sum of phi(K) over the stage's rows
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          umma_ss(tmem + D, sdesc_sw128(kb + kk * 2048, kRows * 128, 1024),
                  sdesc_sw128(ob + kk * 2048, kRows * 128, 1024), idz, (t > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bEmpty(s));
      }
      umma_commit(bDone);
      mbar_drain(bDone, 0, ab.limit_ns);
    }
  } else if (warp >= 4) {
    const int tid = threadIdx.x - 128;
    const int ch = tid % kChunks, rg = tid / kChunks;
    // address of this thread's chunk in row rg of a tile; row rg + 16 i adds
    // 16 i * 128 bytes and keeps the swizzle phase (16 i is a multiple of 8)
    const uint32_t off0 = (ch >> 3) * (kRows * 128) + sw128_offset(rg, ch & 7);
    const fmap::Poly ak = fmap::load_poly(p.coef, 1, p.H, h);
    bool ok = true;
    // No early exit (a failed wait only follows an abort): every thread
    // reaches the reduction barrier below.
    for (int t = 0; t < nt; ++t) {
      const int s = t % NS;
      if (!mbar_wait(bFull(s), (t / NS) & 1, ab, kStatusTimeoutAux)) ok = false;
      const uint32_t kb = sK + s * C::kTileBytes + off0;
      const int row_end = c1 - (c0 + t * kRows);    // rows at or past it belong to the next chunk
      uint4 v[kRowsPerThread];
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) v[i] = lds128(kb + i * (kRowGroups * 128));
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const bool valid = rg + i * kRowGroups < row_end;
        uint32_t w4[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float x0 = bf16lo_to_f32(w4[e]), x1 = bf16hi_to_f32(w4[e]);
          x0 = valid ? fmap::feature(FMAP, ak, x0) : 0.f;
          x1 = valid ? fmap::feature(FMAP, ak, x1) : 0.f;
          w4[e] = pack_bf16x2(x0, x1);
        }
        sts128(kb + i * (kRowGroups * 128), make_uint4(w4[0], w4[1], w4[2], w4[3]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bPhi(s));
    }
    if (ok && nt > 0) {
      ok = mbar_wait(bDone, 0, ab, kStatusTimeoutAux);
      tc_fence_after();
    }
    ok = __all_sync(0xffffffffu, ok);   // the TMEM loads below are warp-collective
    // S rows from TMEM: warp w reads lanes 32 (w % 4) ..; warps 4..7 take
    // columns 0..63, warps 8..11 columns 64..127
    const int r = (warp & 3) * 32 + lane;
    const int cb = (warp >= 8) ? D / 2 : 0;
    float* dst = p.wsS + ((((static_cast<size_t>(c) * p.B + b) * p.H + h) * D) + r) * D + cb;
    const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + cb;
#pragma unroll 1
    for (int q = 0; q < D / 64; ++q) {
      uint32_t v[32];
      if (ok && nt > 0) {
        tmem_ld32(trow + q * 32, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      float4* d4 = reinterpret_cast<float4*>(dst + q * 32);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        d4[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                            __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
    }
    if (warp < 8) {
      // dz[r] from TMEM lane r, column D (the 16 dz columns are equal)
      uint32_t v[32];
      if (ok && nt > 0) {
        tmem_ld32(trow - cb + D, v);
        tmem_ld_wait();
      } else {
        v[0] = 0u;
      }
      p.wsz[((static_cast<size_t>(c) * p.B + b) * p.H + h) * D + r] = __uint_as_float(v[0]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Exclusive scan over chunks, in place in the workspace, starting from the
// caller's state; the caller's state leaves as the total.  One float4 per
// thread and element; the loads of up to kScanBatch chunks are issued before
// their stores (coalesced 16-byte accesses, many in flight).
constexpr int kScanBatch = 12;

__global__ void __launch_bounds__(256, 2) scan_kernel(float4* __restrict__ wsS, float4* __restrict__ S, long long nS4,
                                                      float4* __restrict__ wsz, float4* __restrict__ z, long long nz4,
                                                      int C) {
  pdl::grid_dep_wait();
  pdl::grid_dep_launch();
  const long long total = nS4 + nz4;
  for (long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const bool isS = idx < nS4;
    const long long e = isS ? idx : idx - nS4;
    const long long n = isS ? nS4 : nz4;
    float4* col = (isS ? wsS : wsz) + e;   // chunk c's element at col[c * n]
    float4* st = (isS ? S : z) + e;
    float4 run = *st;
    for (int c0 = 0; c0 < C; c0 += kScanBatch) {
      float4* base = col + c0 * n;
      float4 d[kScanBatch];
#pragma unroll
      for (int u = 0; u < kScanBatch; ++u)
        if (c0 + u < C) d[u] = base[u * n];
#pragma unroll
      for (int u = 0; u < kScanBatch; ++u) {
        if (c0 + u < C) {
          base[u * n] = run;
          run.x += d[u].x;
          run.y += d[u].y;
          run.z += d[u].z;
          run.w += d[u].w;
        }
      }
    }
    *st = run;
  }
}

}  // namespace hyb
}  // namespace vattn
