// Exact combination of partial attentions (the step that joins the key
// shards of Ring attention, ReGenVC "Unified sequence parallelism", Sec.
// 3.5: each shard's attention is a softmax over its keys only; knowing each
// partial's log-sum-exp makes the combination exact up to rounding):
//
//   M = max_r lse_r,  w_r = exp(lse_r - M),  o = sum_r w_r o_r / sum_r w_r,
//   lse = M + ln sum_r w_r
//
// (a part whose keys were all invisible has lse = -inf and weight 0).  Pure
// HBM pass: every 16-byte chunk of every part is read once, the result
// written once, with 16-byte vectors.
#pragma once
#include "common.cuh"

namespace vattn {
namespace merge {

using namespace sm100;

constexpr int kMaxParts = 64;

struct MergeParams {
  const uint4* __restrict__ o_parts;   // bf16 [R][B][L][H][D], 8 channels per uint4
  const float* __restrict__ lse_parts; // fp32 [R][B][H][L] (natural log)
  uint4* __restrict__ o;               // bf16 [B][L][H][D]
  float* __restrict__ lse;             // fp32 [B][H][L] (nullable)
  int R, B, L, H, D;
};

// Thread = one 16-byte chunk (8 channels) of one (b, token, head) row; the
// chunks of a row are consecutive threads, so every load and store of a
// warp is one contiguous span.
__global__ void __launch_bounds__(256) merge_kernel(const MergeParams p) {
  const int cpr = p.D / 8;   // chunks per row
  const long long rows = static_cast<long long>(p.B) * p.L * p.H;
  const long long n = rows * cpr;
  const long long part = n;   // uint4 chunks per part
  const long long lse_part = rows;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = i / cpr;          // (b * L + t) * H + h
    const int h = static_cast<int>(row % p.H);
    const long long bt = row / p.H;
    const int t = static_cast<int>(bt % p.L);
    const int b = static_cast<int>(bt / p.L);
    const long long li = (static_cast<long long>(b) * p.H + h) * p.L + t;
    float m = -INFINITY;
    for (int r = 0; r < p.R; ++r) m = fmaxf(m, __ldg(p.lse_parts + r * lse_part + li));
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float wsum = 0.f;
    if (m > -INFINITY) {
      for (int r = 0; r < p.R; ++r) {
        const float w = __expf(__ldg(p.lse_parts + r * lse_part + li) - m);
        const uint4 v = __ldg(p.o_parts + r * part + i);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] = fmaf(w, bf16lo_to_f32(u[e]), acc[2 * e]);
          acc[2 * e + 1] = fmaf(w, bf16hi_to_f32(u[e]), acc[2 * e + 1]);
        }
        wsum += w;
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    uint32_t w4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) w4[e] = pack_bf16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
    p.o[i] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    if (p.lse && (i % cpr) == 0) p.lse[li] = wsum > 0.f ? m + __logf(wsum) : -INFINITY;
  }
}

}  // namespace merge
}  // namespace vattn
