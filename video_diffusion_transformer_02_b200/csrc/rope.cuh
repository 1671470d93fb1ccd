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
#include "grid_dep.cuh"

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

// Rotation of a token-major tensor [B][L][heads][d] (16-byte chunks, 4
// channel pairs each).  Thread layout: a block owns a contiguous range of
// (batch, token) rows; thread c of a row owns chunk c (head c / (d/8),
// channel chunk c % (d/8)) for every row of the range, so one row is read
// and written as one contiguous, coalesced block, and the token position
// (t, h, w) advances incrementally from row to row (no division in the
// loop).  Optionally the raw input (and a second tensor) is copied to other
// outputs in the same pass (ring append).
struct RotParams {
  const uint4* __restrict__ src;      // tensor to rotate
  uint4* __restrict__ dst;            // rotated output
  const uint4* __restrict__ src2;     // second tensor copied verbatim (nullable)
  uint4* __restrict__ raw_dst;        // raw copy of src (nullable)
  uint4* __restrict__ raw_dst2;       // raw copy of src2 (nullable)
  long long rows;                     // B * L
  int L, heads, d;
  int frame_offset, Hg, Wg, pt, ph;   // token n of a row: t = frame_offset + n / (Hg*Wg)
  const float2* __restrict__ tab;
  int32_t* ids;                       // frame id to set (nullable)
  int slot, frame;
};

template <bool COPY>
__global__ void __launch_bounds__(512) rotate_rows_kernel(const RotParams p) {
  pdl::grid_dep_wait();
  pdl::grid_dep_launch();
  const int cpt = p.heads * (p.d / 8);                 // chunks per row
  const long long rows_per_block = (p.rows + gridDim.x - 1) / gridDim.x;
  const long long r0 = static_cast<long long>(blockIdx.x) * rows_per_block;
  const long long r1 = r0 + rows_per_block < p.rows ? r0 + rows_per_block : p.rows;
  const int F = p.Hg * p.Wg;
  for (int c = threadIdx.x; c < cpt; c += blockDim.x) {
    const int c16 = c % (p.d / 8);
    // this chunk's four pairs: axis of each pair (0 t, 1 h, 2 w)
    uint32_t axis = 0;   // 2 bits per pair: 0 t, 1 h, 2 w
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = c16 * 4 + e;
      axis |= static_cast<uint32_t>(j < p.pt ? 0 : (j < p.pt + p.ph ? 1 : 2)) << (2 * e);
    }
    // position of row r0
    const int n0 = static_cast<int>(r0 % p.L);
    int t = p.frame_offset + n0 / F, in = n0 % F;
    int hh = in / p.Wg, w = in % p.Wg;
    int n = n0;
    constexpr int U = 4;   // rows per step: their loads are issued before any store
    for (long long rb = r0; rb < r1; rb += U) {
      uint4 v[U], v2[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (rb + u < r1) {
          const long long i = (rb + u) * cpt + c;
          v[u] = __ldg(p.src + i);
          if (COPY) v2[u] = __ldg(p.src2 + i);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (rb + u >= r1) continue;
        const long long i = (rb + u) * cpt + c;
        if (COPY) {
          p.raw_dst[i] = v[u];
          p.raw_dst2[i] = v2[u];
        }
        uint32_t w4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = c16 * 4 + e;
          const uint32_t ax = (axis >> (2 * e)) & 3u;
          const int pos = ax == 0 ? t : (ax == 1 ? hh : w);
          const float2 cs = __ldg(p.tab + pos * (p.d / 2) + j);
          const float x0 = bf16lo_to_f32(w4[e]), x1 = bf16hi_to_f32(w4[e]);
          w4[e] = pack_bf16x2(x0 * cs.x - x1 * cs.y, x0 * cs.y + x1 * cs.x);
        }
        p.dst[i] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        // next token: w, then h, then t; a new batch row restarts at token 0
        if (++n == p.L) {
          n = 0;
          t = p.frame_offset;
          hh = 0;
          w = 0;
        } else if (++w == p.Wg) {
          w = 0;
          if (++hh == p.Hg) {
            hh = 0;
            ++t;
          }
        }
      }
    }
  }
  if (p.ids && blockIdx.x == 0 && threadIdx.x == 0) p.ids[p.slot] = p.frame;
}

}  // namespace rope
}  // namespace vattn
