// 3D rotary position embedding: the cos/sin table and the standalone rotate.
//
// Channel pair j = (2j, 2j+1) of a head vector turns by angle
// pos * theta^(-i / n_axis): pairs [0, n_t) use the frame index t, the next
// n_h the row h, the last n_w the column w; i is the pair's index inside its
// axis group (FlashDecoder "Transformer Backbone Design", Sec. 3.2, 3D-RoPE
// applied separately on the temporal and spatial axes; t/x/y channel groups
// as in the Kaleido review; RoFormer frequencies).
#pragma once
#include "common.cuh"

namespace vattn {
namespace rope {

using namespace sm100;

// table[pos][j] = (cos, sin)(pos * omega_j), angle and trig in double,
// rounded once to fp32.
__global__ void table_kernel(float2* tab, int max_pos, int pairs, int pt, int ph, int pw,
                             double theta) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= max_pos * pairs) return;
  const int pos = i / pairs, j = i - (i / pairs) * pairs;
  int ii, n;
  if (j < pt) {
    ii = j;
    n = pt;
  } else if (j < pt + ph) {
    ii = j - pt;
    n = ph;
  } else {
    ii = j - pt - ph;
    n = pw;
  }
  const double omega = pow(theta, -static_cast<double>(ii) / static_cast<double>(n));
  double s, c;
  sincos(static_cast<double>(pos) * omega, &s, &c);
  tab[i] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

struct QKParams {
  const uint4* src[2];
  uint4* dst[2];
  long long n16[2];   // 16-byte chunks per tensor
  int heads[2];       // H for q, Hkv for k
  int L, d, Hg, Wg, pt, ph, frame_offset;
  const float2* tab;
};

// One 16-byte chunk (4 channel pairs) per thread and iteration.
__global__ void __launch_bounds__(256) rope_qk_kernel(const QKParams p) {
  const long long total = p.n16[0] + p.n16[1];
  const int cpr = p.d / 8;   // chunks per head vector
  const int F = p.Hg * p.Wg;
  for (long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int which = idx < p.n16[0] ? 0 : 1;
    const long long local = which ? idx - p.n16[0] : idx;
    const int c16 = static_cast<int>(local % cpr);
    const long long vec = local / cpr;
    const int tok = static_cast<int>((vec / p.heads[which]) % p.L);
    const int in = tok % F;
    const int t = p.frame_offset + tok / F, hh = in / p.Wg, w = in % p.Wg;
    const uint4 v = __ldg(p.src[which] + local);
    uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = c16 * 4 + e;
      const int pos = j < p.pt ? t : (j < p.pt + p.ph ? hh : w);
      const float2 cs = __ldg(p.tab + static_cast<long long>(pos) * (p.d / 2) + j);
      const float x0 = bf16lo_to_f32(w4[e]), x1 = bf16hi_to_f32(w4[e]);
      w4[e] = pack_bf16x2(x0 * cs.x - x1 * cs.y, x0 * cs.y + x1 * cs.x);
    }
    p.dst[which][local] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
}

}  // namespace rope
}  // namespace vattn
