// Rolling KV cache append (FlashDecoder "Streaming with Rolling KV Cache",
// Sec. 3.3): frame f's K and V are copied bit for bit into ring slot
// f mod capacity and the slot's frame id is set.  Pure HBM copy with
// 16-byte vectors, both tensors' loads in flight before the stores.
#pragma once
#include "common.cuh"

namespace vattn {
namespace kv {

__global__ void __launch_bounds__(256) append_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                     uint4* __restrict__ kr, uint4* __restrict__ vr,
                                                     long long n16, int32_t* ids, int slot, int frame) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + stride < n16; i += 2 * stride) {
    const uint4 a0 = __ldg(k + i), b0 = __ldg(v + i);
    const uint4 a1 = __ldg(k + i + stride), b1 = __ldg(v + i + stride);
    kr[i] = a0;
    vr[i] = b0;
    kr[i + stride] = a1;
    vr[i + stride] = b1;
  }
  if (i < n16) {
    const uint4 a0 = __ldg(k + i), b0 = __ldg(v + i);
    kr[i] = a0;
    vr[i] = b0;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) ids[slot] = frame;
}

// Append with rotated keys: one pass copies K and V into the raw ring slot
// (bit-exact) and writes K rotated by 3D-RoPE at its absolute frame into the
// rotated-key ring slot.  Inputs are one frame, [B][F][Hkv][d]; token n of
// the frame sits at (h, w) = (n / Wg, n % Wg).  Channel pair j turns by the
// table angle of its axis position (t = frame for pairs < pt, h for the next
// ph, w for the rest).
struct AppendRopeParams {
  const uint4* k;
  const uint4* v;
  uint4* kr;        // raw K slot (nullable: rotate only)
  uint4* vr;        // raw V slot (nullable with kr)
  uint4* krot;      // rotated K slot
  long long n16;    // 16-byte chunks per tensor
  int32_t* ids;     // frame id table (nullable)
  int slot, frame;
  int F, Hkv, d, Wg, pt, ph;
  const float2* tab;
};

__global__ void __launch_bounds__(256) append_rope_kernel(const AppendRopeParams p) {
  const int cpr = p.d / 8;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < p.n16; i += stride) {
    const uint4 kv = __ldg(p.k + i);
    if (p.kr) {
      const uint4 vv = __ldg(p.v + i);
      p.kr[i] = kv;
      p.vr[i] = vv;
    }
    const int c16 = static_cast<int>(i % cpr);
    const int n = static_cast<int>(((i / cpr) / p.Hkv) % p.F);
    const int hh = n / p.Wg, w = n % p.Wg;
    uint32_t w4[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = c16 * 4 + e;
      const int pos = j < p.pt ? p.frame : (j < p.pt + p.ph ? hh : w);
      const float2 cs = __ldg(p.tab + static_cast<long long>(pos) * (p.d / 2) + j);
      const float x0 = sm100::bf16lo_to_f32(w4[e]), x1 = sm100::bf16hi_to_f32(w4[e]);
      w4[e] = sm100::pack_bf16x2(x0 * cs.x - x1 * cs.y, x0 * cs.y + x1 * cs.x);
    }
    p.krot[i] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
  if (p.ids && blockIdx.x == 0 && threadIdx.x == 0) p.ids[p.slot] = p.frame;
}

}  // namespace kv
}  // namespace vattn
