// Feature maps of the hybrid chunk attention's causal linear part
// (MobileWan review: phi applied elementwise to q and k).
//   kFmapElu1: phi(x) = elu(x) + 1 (Katharopoulos et al., positive, the
//              workload configuration);
//   kFmapPoly3: phi(x) = a0 + a1 x + a2 x^2 + a3 x^3 with caller-given
//              coefficients per head and per map (the page variant's
//              learnable degree-3 polynomial feature maps, App. A.3.1).
#pragma once
#include "common.cuh"

namespace vattn {
namespace fmap {

enum : int { kFmapElu1 = 0, kFmapPoly3 = 1 };

struct Poly {
  float a0, a1, a2, a3;
};

// coef: fp32 [2][H][4] (map 0 = q, 1 = k); unused for elu + 1.
__device__ __forceinline__ Poly load_poly(const float* coef, int map, int H, int h) {
  if (!coef) return Poly{0.f, 0.f, 0.f, 0.f};
  const float4 c = __ldg(reinterpret_cast<const float4*>(coef + (static_cast<size_t>(map) * H + h) * 4));
  return Poly{c.x, c.y, c.z, c.w};
}

__device__ __forceinline__ float feature(int kind, const Poly& a, float x) {
  if (kind == kFmapPoly3) return fmaf(fmaf(fmaf(a.a3, x, a.a2), x, a.a1), x, a.a0);
  return x > 0.f ? x + 1.f : __expf(x);
}

}  // namespace fmap
}  // namespace vattn
