// fp64 CPU oracle for spatiotemporal attention with 3D rotary embedding.
//
// TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, direct definition
// of what the CUDA library computes.  Only the tests, the smoke check and the
// benchmark's CPU-baseline leg load it.  It shares no code, header, table or
// constant with the CUDA path: every cosine, exponential and sum here is
// evaluated from the definitions in double precision.
//
// Inputs are bfloat16 bit patterns (uint16), widened exactly to double.
// Layout of q/k/v/o: [B][L][H][d], contiguous.  Token n of a T x Hg x Wg
// latent grid sits at (t, h, w) = (n / (Hg*Wg), (n / Wg) % Hg, n % Wg)
// (row-major over the latent order B x C x T x H x W of FlashDecoder,
// "Preliminaries: Latent Diffusion Model", Sec. 3.1).
//
// Sources of each definition (page title, section):
//  * 3D-RoPE: FlashDecoder, "Transformer Backbone Design" (Sec. 3.2): rotary
//    embedding applied separately to the temporal and spatial axes; the
//    channel pairs fall into t / h / w groups (Kaleido review, "What carries
//    the argument"); per-pair frequencies as in RoFormer (FlashDecoder ref.
//    [53]): omega_i = theta^(-i / n_axis) for the i-th pair of an axis group.
//  * masked softmax attention in three modes: FlashDecoder "Streaming with
//    Rolling KV Cache" (Sec. 3.3, per-frame sliding window, no in-frame mask),
//    "Effectiveness of Each Component" (Sec. 4.2, full block-causal baseline).
//  * hybrid chunk attention with state (s, z): MobileWan review ("The pith",
//    "What carries the argument", axiom ledger): softmax inside a chunk,
//    causal linear attention across chunks, feature map elu(x)+1
//    (Katharopoulos et al., "Transformers are RNNs", cited there).
#include <cmath>
#include <cstdint>
#include <cstring>
#include <cstdlib>
#include <limits>
#include <vector>
#include <algorithm>
#include <thread>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

inline double bf16_to_double(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return static_cast<double>(f);
}

struct Rope {
  int Hg, Wg;           // spatial grid of a frame
  int pairs_t, pairs_h, pairs_w;
  double theta;
};

// Rotate one head vector x[d] (doubles) in place for grid position (t,h,w).
// Pair j = channels (2j, 2j+1).  Pairs [0, pt) use t, [pt, pt+ph) use h,
// the rest use w; within an axis group the i-th pair turns at angle
// pos * theta^(-i / n_axis).
void rope_rotate(double* x, int d, const Rope& r, long t, long h, long w) {
  const int pairs = d / 2;
  for (int j = 0; j < pairs; ++j) {
    long pos;
    int i, n;
    if (j < r.pairs_t) { pos = t; i = j; n = r.pairs_t; }
    else if (j < r.pairs_t + r.pairs_h) { pos = h; i = j - r.pairs_t; n = r.pairs_h; }
    else { pos = w; i = j - r.pairs_t - r.pairs_h; n = r.pairs_w; }
    const double omega = std::pow(r.theta, -static_cast<double>(i) / static_cast<double>(n));
    const double a = static_cast<double>(pos) * omega;
    const double c = std::cos(a), s = std::sin(a);
    const double x0 = x[2 * j], x1 = x[2 * j + 1];
    x[2 * j] = x0 * c - x1 * s;
    x[2 * j + 1] = x0 * s + x1 * c;
  }
}

inline void token_position(long n, long frame_offset, const Rope& r, long* t, long* h, long* w) {
  const long F = static_cast<long>(r.Hg) * r.Wg;
  *t = frame_offset + n / F;
  *h = (n / r.Wg) % r.Hg;
  *w = n % r.Wg;
}

// Load head vector [b][n][h][:] of a [B][L][H][d] bf16 tensor as doubles.
inline void load_vec(const uint16_t* x, long L, long H, long d, long b, long n, long h, double* out) {
  const uint16_t* p = x + ((b * L + n) * H + h) * d;
  for (long c = 0; c < d; ++c) out[c] = bf16_to_double(p[c]);
}

enum { MODE_FULL = 0, MODE_CHUNK_CAUSAL = 1, MODE_SLIDING = 2 };

// Is key token nk (frame fk) visible from query token nq (frame fq)?
// FULL: always.  CHUNK_CAUSAL(c): floor(fk/c) <= floor(fq/c) (bidirectional
// inside a chunk of c frames, causal across chunks).  SLIDING(wb, wf):
// fq - wb <= fk <= fq + wf (the query's own frame plus wb earlier and wf
// later frames; no mask inside a frame).
inline bool allowed(int mode, long fq, long fk, int chunk, int wb, int wf) {
  switch (mode) {
    case MODE_FULL: return true;
    case MODE_CHUNK_CAUSAL: return (fk / chunk) <= (fq / chunk);
    case MODE_SLIDING: return fk >= fq - wb && fk <= fq + wf;
  }
  return false;
}

int n_threads() {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// softmax attention for one query row given the full key set of its head,
// restricted to the allowed keys.  q: rotated query (double[d]); K: rotated
// keys [Lk][d] (double); V: values [Lk][d] (double).  Two passes: row max,
// then sum of exp(s - max) and the weighted sum of values.
void attend_row(const double* q, const double* K, const double* V, long Lk, int d,
                double scale, const std::vector<char>& mask_row, double* o, double* lse) {
  double m = -std::numeric_limits<double>::infinity();
  std::vector<double> s(Lk);
  for (long j = 0; j < Lk; ++j) {
    if (!mask_row[j]) continue;
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += q[c] * K[j * d + c];
    s[j] = scale * acc;
    if (s[j] > m) m = s[j];
  }
  for (int c = 0; c < d; ++c) o[c] = 0.0;
  if (m == -std::numeric_limits<double>::infinity()) {   // no visible key
    *lse = m;
    return;
  }
  double l = 0.0;
  for (long j = 0; j < Lk; ++j) {
    if (!mask_row[j]) continue;
    const double p = std::exp(s[j] - m);
    l += p;
    for (int c = 0; c < d; ++c) o[c] += p * V[j * d + c];
  }
  for (int c = 0; c < d; ++c) o[c] /= l;
  *lse = m + std::log(l);
}

}  // namespace

extern "C" {

int oracle_num_threads() { return n_threads(); }

// 3D-RoPE of a [B][L][H][d] tensor; out is double [B][L][H][d].
// Token n sits at frame t = t_offset + n / (Hg*Wg).
int oracle_rope(const uint16_t* x, double* out, int B, int L, int H, int d,
                int Hg, int Wg, int pairs_t, int pairs_h, int pairs_w, double theta,
                int t_offset) {
  if (d % 2 || pairs_t + pairs_h + pairs_w != d / 2) return 1;
  Rope r{Hg, Wg, pairs_t, pairs_h, pairs_w, theta};
#pragma omp parallel for schedule(static)
  for (long bn = 0; bn < static_cast<long>(B) * L; ++bn) {
    const long n = bn % L;
    long t, h, w;
    token_position(n, t_offset, r, &t, &h, &w);
    for (long hd = 0; hd < H; ++hd) {
      double* o = out + (bn * H + hd) * d;
      for (int c = 0; c < d; ++c) o[c] = bf16_to_double(x[(bn * H + hd) * d + c]);
      rope_rotate(o, d, r, t, h, w);
    }
  }
  return 0;
}

// Masked softmax attention.  q [B][Lq][H][d], k/v [B][Lk][Hkv][d].
// Query token n is in frame q_frame_offset + n / F, key token n in frame
// k_frame_offset + n / F (F = tokens per frame; unused by FULL).
// rope_cfg (nullable) = {Hg, Wg, pairs_t, pairs_h, pairs_w} and theta:
// queries and keys are rotated at their own (t, h, w), t = absolute frame.
// rows: n_rows triples (b, h, i) of query rows to evaluate; rows == NULL
// means all B*H*Lq rows in [b][i][h] order.  o: double [n_rows][d] (or
// [B][Lq][H][d]); lse: double [n_rows] (or [B][H][Lq]), natural log of the
// softmax denominator of the scaled scores; -inf for a row with no key.
int oracle_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     int B, int Lq, int Lk, int H, int Hkv, int d, double scale,
                     int mode, int F, int chunk, int wb, int wf,
                     int q_frame_offset, int k_frame_offset,
                     const int* rope_cfg, double theta,
                     const int32_t* rows, long n_rows, double* o, double* lse) {
  if (H % Hkv) return 1;
  if (mode != MODE_FULL && F <= 0) return 1;
  if (mode == MODE_CHUNK_CAUSAL && chunk <= 0) return 1;
  const bool use_rope = rope_cfg != nullptr;
  Rope r{};
  if (use_rope) {
    r = Rope{rope_cfg[0], rope_cfg[1], rope_cfg[2], rope_cfg[3], rope_cfg[4], theta};
    if (r.pairs_t + r.pairs_h + r.pairs_w != d / 2) return 1;
  }
  const int group = H / Hkv;
  std::vector<int32_t> all;
  if (!rows) {
    n_rows = static_cast<long>(B) * H * Lq;
    all.resize(n_rows * 3);
    long idx = 0;
    for (int b = 0; b < B; ++b)
      for (int i = 0; i < Lq; ++i)
        for (int h = 0; h < H; ++h) { all[idx++] = b; all[idx++] = h; all[idx++] = i; }
    rows = all.data();
  }
  // Process rows grouped by (b, kv head): rotate that head's keys once.
  std::vector<long> order(n_rows);
  for (long i = 0; i < n_rows; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(), [&](long a, long b2) {
    const long ka = static_cast<long>(rows[3 * a]) * Hkv + rows[3 * a + 1] / group;
    const long kb = static_cast<long>(rows[3 * b2]) * Hkv + rows[3 * b2 + 1] / group;
    return ka < kb;
  });
  std::vector<double> K(static_cast<size_t>(Lk) * d), V(static_cast<size_t>(Lk) * d);
  long start = 0;
  while (start < n_rows) {
    const long r0 = order[start];
    const int b = rows[3 * r0];
    const int kvh = rows[3 * r0 + 1] / group;
    long end = start;
    while (end < n_rows && rows[3 * order[end]] == b && rows[3 * order[end] + 1] / group == kvh) ++end;
#pragma omp parallel for schedule(static)
    for (long n = 0; n < Lk; ++n) {
      load_vec(k, Lk, Hkv, d, b, n, kvh, &K[n * d]);
      load_vec(v, Lk, Hkv, d, b, n, kvh, &V[n * d]);
      if (use_rope) {
        long t, hh, w;
        token_position(n, k_frame_offset, r, &t, &hh, &w);
        rope_rotate(&K[n * d], d, r, t, hh, w);
      }
    }
#pragma omp parallel
    {
      std::vector<double> qv(d);
      std::vector<char> mask(Lk);
#pragma omp for schedule(dynamic, 4)
      for (long s = start; s < end; ++s) {
        const long ri = order[s];
        const int h = rows[3 * ri + 1];
        const long i = rows[3 * ri + 2];
        load_vec(q, Lq, H, d, b, i, h, qv.data());
        if (use_rope) {
          long t, hh, w;
          token_position(i, q_frame_offset, r, &t, &hh, &w);
          rope_rotate(qv.data(), d, r, t, hh, w);
        }
        const long fq = mode == MODE_FULL ? 0 : q_frame_offset + i / F;
        for (long j = 0; j < Lk; ++j) {
          const long fk = mode == MODE_FULL ? 0 : k_frame_offset + j / F;
          mask[j] = allowed(mode, fq, fk, chunk, wb, wf) ? 1 : 0;
        }
        double* orow;
        double* lrow;
        if (all.empty()) {
          orow = o + ri * d;
          lrow = lse + ri;
        } else {
          orow = o + ((static_cast<long>(b) * Lq + i) * H + h) * d;
          lrow = lse + (static_cast<long>(b) * H + h) * Lq + i;
        }
        attend_row(qv.data(), K.data(), V.data(), Lk, d, scale, mask, orow, lrow);
      }
    }
    start = end;
  }
  return 0;
}

// Streaming decode (FlashDecoder Sec. 3.3): frame f's F query tokens attend
// to all tokens of frames max(0, f - wb) .. f, taken from the full key and
// value sequences of n_frames frames.  Keys are gathered per frame (the
// frame-by-frame processing order), not masked.  rows: (b, h, i) triples
// over the whole sequence (i = f * F + token); o [n_rows][d], lse [n_rows].
//
// RoPE positions (rope_cfg given): a stream frame holds r = F / (Hg*Wg)
// latent frames of Hg x Wg tokens (r = 1 for the backbone; r = r_t for the
// temporal-refinement layers, which see r_t * L_frm tokens per step,
// FlashDecoder "Complexity Analysis", Sec. 3.3).  Token n of stream frame
// fr sits at t = r * (fr - base) + n / (Hg*Wg), h = (n / Wg) % Hg,
// w = n % Wg, where base = 0 (absolute frame index) or, with
// window_relative, base = max(0, f - wb), the first frame of the query's
// window (positions relative to the current window, "Long Video Decoding",
// Sec. 4.3).
int oracle_stream(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                  int B, int n_frames, int F, int H, int Hkv, int d, double scale, int wb,
                  const int* rope_cfg, double theta,
                  const int32_t* rows, long n_rows, double* o, double* lse, int window_relative) {
  if (H % Hkv) return 1;
  const bool use_rope = rope_cfg != nullptr;
  Rope r{};
  long sub = 1;   // latent frames per stream frame
  if (use_rope) {
    r = Rope{rope_cfg[0], rope_cfg[1], rope_cfg[2], rope_cfg[3], rope_cfg[4], theta};
    const long fr_tokens = static_cast<long>(r.Hg) * r.Wg;
    if (F % fr_tokens) return 1;
    sub = F / fr_tokens;
  }
  const long L = static_cast<long>(n_frames) * F;
  const int group = H / Hkv;
#pragma omp parallel
  {
    std::vector<double> qv(d), K, V;
    std::vector<char> mask;
#pragma omp for schedule(dynamic, 1)
    for (long s = 0; s < n_rows; ++s) {
      const int b = rows[3 * s], h = rows[3 * s + 1];
      const long i = rows[3 * s + 2];
      const long f = i / F;
      const long f0 = std::max(0L, f - wb);
      const long base = window_relative ? f0 : 0;
      const long nk = (f - f0 + 1) * F;
      K.assign(nk * d, 0.0);
      V.assign(nk * d, 0.0);
      mask.assign(nk, 1);
      for (long fr = f0; fr <= f; ++fr) {
        for (long tkn = 0; tkn < F; ++tkn) {
          const long j = (fr - f0) * F + tkn;
          load_vec(k, L, Hkv, d, b, fr * F + tkn, h / group, &K[j * d]);
          load_vec(v, L, Hkv, d, b, fr * F + tkn, h / group, &V[j * d]);
          if (use_rope) {
            long t, hh, w;
            token_position(tkn, sub * (fr - base), r, &t, &hh, &w);
            rope_rotate(&K[j * d], d, r, t, hh, w);
          }
        }
      }
      load_vec(q, L, H, d, b, i, h, qv.data());
      if (use_rope) {
        long t, hh, w;
        token_position(i % F, sub * (f - base), r, &t, &hh, &w);
        rope_rotate(qv.data(), d, r, t, hh, w);
      }
      attend_row(qv.data(), K.data(), V.data(), nk, d, scale, mask, o + s * d, lse + s);
    }
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Hybrid chunk attention (MobileWan).  Tokens are split into chunks of
// chunk_tokens consecutive tokens (the last may be shorter).  For query i in
// chunk c, with s_ij = scale * q_i . k_j and phi(x) = elu(x) + 1 applied
// elementwise to the raw q and k:
//   num_i = sum_{j in c} exp(s_ij) v_j + sum_{j in chunks < c} (phi(q_i).phi(k_j)) v_j
//   den_i = sum_{j in c} exp(s_ij)     + sum_{j in chunks < c}  phi(q_i).phi(k_j)
//   o_i = num_i / den_i   (one joint normalisation)
// An optional incoming state (S0 [d][d], z0 [d]) stands for keys before token
// 0 and enters both sums as phi(q_i)^T S0 and phi(q_i)^T z0.
// ---------------------------------------------------------------------------
static inline double phi(double x) { return x > 0.0 ? x + 1.0 : std::exp(x); }

// Parallel (masked) form: every earlier key is visited explicitly.
// rows: (b, h, i) triples; o [n_rows][d].  S0/z0 per (b, h): [B][H][d][d],
// [B][H][d] (nullable = zero state).
int oracle_hybrid_parallel(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           int B, int L, int H, int d, int chunk_tokens, double scale,
                           const double* S0, const double* z0,
                           const int32_t* rows, long n_rows, double* o) {
  if (chunk_tokens <= 0) return 1;
#pragma omp parallel
  {
    std::vector<double> qv(d), pq(d), kv(d), vv(d), num(d);
#pragma omp for schedule(dynamic, 1)
    for (long s = 0; s < n_rows; ++s) {
      const int b = rows[3 * s], h = rows[3 * s + 1];
      const long i = rows[3 * s + 2];
      const long c = i / chunk_tokens;
      const long c0 = c * chunk_tokens, c1 = std::min<long>(L, c0 + chunk_tokens);
      load_vec(q, L, H, d, b, i, h, qv.data());
      for (int x = 0; x < d; ++x) pq[x] = phi(qv[x]);
      std::fill(num.begin(), num.end(), 0.0);
      double den = 0.0;
      if (S0) {
        const double* Sb = S0 + (static_cast<long>(b) * H + h) * d * d;
        const double* zb = z0 + (static_cast<long>(b) * H + h) * d;
        for (int a = 0; a < d; ++a) {
          den += pq[a] * zb[a];
          for (int e = 0; e < d; ++e) num[e] += pq[a] * Sb[a * d + e];
        }
      }
      for (long j = 0; j < c0; ++j) {           // earlier chunks: linear
        load_vec(k, L, H, d, b, j, h, kv.data());
        load_vec(v, L, H, d, b, j, h, vv.data());
        double w = 0.0;
        for (int x = 0; x < d; ++x) w += pq[x] * phi(kv[x]);
        den += w;
        for (int x = 0; x < d; ++x) num[x] += w * vv[x];
      }
      for (long j = c0; j < c1; ++j) {          // own chunk: softmax weights
        load_vec(k, L, H, d, b, j, h, kv.data());
        load_vec(v, L, H, d, b, j, h, vv.data());
        double acc = 0.0;
        for (int x = 0; x < d; ++x) acc += qv[x] * kv[x];
        const double w = std::exp(scale * acc);
        den += w;
        for (int x = 0; x < d; ++x) num[x] += w * vv[x];
      }
      for (int x = 0; x < d; ++x) o[s * d + x] = num[x] / den;
    }
  }
  return 0;
}

// Recurrent form (the model run as an RNN over chunks): state S [d][d]
// (S[a][e] = sum phi(k_j)[a] v_j[e]) and z [d] (sum phi(k_j)) over all keys of
// earlier chunks.  Chunk c's queries read phi(q)^T S and phi(q)^T z, then the
// chunk's keys are folded into the state.
// S_io/z_io (nullable): incoming state per (b, h), overwritten with the
// outgoing state; o: double [B][L][H][d]; row_mask (nullable, [B][H][L] char)
// limits which outputs are evaluated (the state is always advanced fully).
int oracle_hybrid_recurrent(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                            int B, int L, int H, int d, int chunk_tokens, double scale,
                            double* S_io, double* z_io, const char* row_mask, double* o) {
  if (chunk_tokens <= 0) return 1;
  const long n_chunks = (L + chunk_tokens - 1) / chunk_tokens;
  const long BH = static_cast<long>(B) * H;
#pragma omp parallel
  {
    std::vector<double> S(static_cast<size_t>(d) * d), z(d), qv(d), pq(d), kv(d), vv(d), num(d);
    std::vector<double> Kc, Vc;
#pragma omp for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
      const int b = static_cast<int>(bh / H), h = static_cast<int>(bh % H);
      if (S_io) {
        std::copy(S_io + bh * d * d, S_io + (bh + 1) * d * d, S.begin());
        std::copy(z_io + bh * d, z_io + (bh + 1) * d, z.begin());
      } else {
        std::fill(S.begin(), S.end(), 0.0);
        std::fill(z.begin(), z.end(), 0.0);
      }
      for (long c = 0; c < n_chunks; ++c) {
        const long c0 = c * chunk_tokens, c1 = std::min<long>(L, c0 + chunk_tokens);
        const long n = c1 - c0;
        Kc.resize(n * d);
        Vc.resize(n * d);
        for (long j = 0; j < n; ++j) {
          load_vec(k, L, H, d, b, c0 + j, h, &Kc[j * d]);
          load_vec(v, L, H, d, b, c0 + j, h, &Vc[j * d]);
        }
        for (long i = c0; i < c1; ++i) {
          if (row_mask && !row_mask[bh * L + i]) continue;
          load_vec(q, L, H, d, b, i, h, qv.data());
          for (int x = 0; x < d; ++x) pq[x] = phi(qv[x]);
          double den = 0.0;
          std::fill(num.begin(), num.end(), 0.0);
          for (int a = 0; a < d; ++a) {
            den += pq[a] * z[a];
            for (int e = 0; e < d; ++e) num[e] += pq[a] * S[a * d + e];
          }
          for (long j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int x = 0; x < d; ++x) acc += qv[x] * Kc[j * d + x];
            const double w = std::exp(scale * acc);
            den += w;
            for (int x = 0; x < d; ++x) num[x] += w * Vc[j * d + x];
          }
          double* orow = o + ((static_cast<long>(b) * L + i) * H + h) * d;
          for (int x = 0; x < d; ++x) orow[x] = num[x] / den;
        }
        for (long j = 0; j < n; ++j) {           // fold chunk c into the state
          for (int a = 0; a < d; ++a) {
            const double pk = phi(Kc[j * d + a]);
            z[a] += pk;
            for (int e = 0; e < d; ++e) S[a * d + e] += pk * Vc[j * d + e];
          }
        }
      }
      if (S_io) {
        std::copy(S.begin(), S.end(), S_io + bh * d * d);
        std::copy(z.begin(), z.end(), z_io + bh * d);
      }
    }
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Hybrid chunk attention, general form: the feature map of the MobileWan page
// variant and softmax chunks that overlap the previous chunk (MobileWan
// review, axiom ledger / App. A.3.1: learnable polynomial feature maps of
// degree 3 for phi_q and phi_k; chunk overlap T_o).
//   fmap 0: phi(x) = elu(x) + 1 (coef unused);
//   fmap 1: phi_q(x) = a0 + a1 x + a2 x^2 + a3 x^3 with (a0..a3) =
//           coef[(0 * H + h) * 4 ..], phi_k likewise with coef[(1 * H + h) * 4 ..]
//           (one polynomial per head and map; coefficients are caller data).
// With overlap ov >= 0 tokens, the softmax part of chunk c covers keys
// [max(0, c * ct - ov), min(L, (c + 1) * ct)) -- the chunk plus the last ov
// tokens before it -- and the linear part the keys j < c * ct - ov (plus the
// incoming state); every key before the end of the query's chunk is counted
// once.  The overlap reaches back inside this call only (chunk 0 has none);
// the outgoing state covers all L tokens.  ov = 0 is the form above.
// ---------------------------------------------------------------------------
static inline double feature(int fmap, const double* a, double x) {
  if (fmap == 0) return x > 0.0 ? x + 1.0 : std::exp(x);
  return a[0] + x * (a[1] + x * (a[2] + x * a[3]));
}

// Parallel form: rows (b, h, i); o [n_rows][d]; S0/z0 nullable as above.
int oracle_hybrid2_parallel(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                            int B, int L, int H, int d, int chunk_tokens, int overlap, double scale,
                            int fmap, const double* coef, const double* S0, const double* z0,
                            const int32_t* rows, long n_rows, double* o) {
  if (chunk_tokens <= 0 || overlap < 0 || (fmap == 1 && !coef) || fmap < 0 || fmap > 1) return 1;
#pragma omp parallel
  {
    std::vector<double> qv(d), pq(d), kv(d), vv(d), num(d);
#pragma omp for schedule(dynamic, 1)
    for (long s = 0; s < n_rows; ++s) {
      const int b = rows[3 * s], h = rows[3 * s + 1];
      const long i = rows[3 * s + 2];
      const double* aq = fmap == 1 ? coef + (0L * H + h) * 4 : nullptr;
      const double* ak = fmap == 1 ? coef + (1L * H + h) * 4 : nullptr;
      const long c = i / chunk_tokens;
      const long w0 = std::max(0L, c * chunk_tokens - overlap);      // softmax window start
      const long w1 = std::min<long>(L, (c + 1) * chunk_tokens);     // and end
      load_vec(q, L, H, d, b, i, h, qv.data());
      for (int x = 0; x < d; ++x) pq[x] = feature(fmap, aq, qv[x]);
      std::fill(num.begin(), num.end(), 0.0);
      double den = 0.0;
      if (S0) {
        const double* Sb = S0 + (static_cast<long>(b) * H + h) * d * d;
        const double* zb = z0 + (static_cast<long>(b) * H + h) * d;
        for (int a = 0; a < d; ++a) {
          den += pq[a] * zb[a];
          for (int e = 0; e < d; ++e) num[e] += pq[a] * Sb[a * d + e];
        }
      }
      for (long j = 0; j < w0; ++j) {           // before the window: linear
        load_vec(k, L, H, d, b, j, h, kv.data());
        load_vec(v, L, H, d, b, j, h, vv.data());
        double w = 0.0;
        for (int x = 0; x < d; ++x) w += pq[x] * feature(fmap, ak, kv[x]);
        den += w;
        for (int x = 0; x < d; ++x) num[x] += w * vv[x];
      }
      for (long j = w0; j < w1; ++j) {          // the window: softmax weights
        load_vec(k, L, H, d, b, j, h, kv.data());
        load_vec(v, L, H, d, b, j, h, vv.data());
        double acc = 0.0;
        for (int x = 0; x < d; ++x) acc += qv[x] * kv[x];
        const double w = std::exp(scale * acc);
        den += w;
        for (int x = 0; x < d; ++x) num[x] += w * vv[x];
      }
      for (int x = 0; x < d; ++x) o[s * d + x] = num[x] / den;
    }
  }
  return 0;
}

// Recurrent form: per (b, h) the state (S, z) is advanced in chunk order;
// chunk c's queries read the state of keys j < c * ct - ov, then the keys
// [c * ct - ov, (c + 1) * ct - ov) are folded in; after the last chunk the
// remaining keys are folded so that the outgoing state covers all L tokens.
int oracle_hybrid2_recurrent(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             int B, int L, int H, int d, int chunk_tokens, int overlap, double scale,
                             int fmap, const double* coef, double* S_io, double* z_io,
                             const char* row_mask, double* o) {
  if (chunk_tokens <= 0 || overlap < 0 || (fmap == 1 && !coef) || fmap < 0 || fmap > 1) return 1;
  const long n_chunks = (L + chunk_tokens - 1) / chunk_tokens;
  const long BH = static_cast<long>(B) * H;
#pragma omp parallel
  {
    std::vector<double> S(static_cast<size_t>(d) * d), z(d), qv(d), pq(d), kv(d), vv(d), num(d);
#pragma omp for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
      const int b = static_cast<int>(bh / H), h = static_cast<int>(bh % H);
      const double* aq = fmap == 1 ? coef + (0L * H + h) * 4 : nullptr;
      const double* ak = fmap == 1 ? coef + (1L * H + h) * 4 : nullptr;
      if (S_io) {
        std::copy(S_io + bh * d * d, S_io + (bh + 1) * d * d, S.begin());
        std::copy(z_io + bh * d, z_io + (bh + 1) * d, z.begin());
      } else {
        std::fill(S.begin(), S.end(), 0.0);
        std::fill(z.begin(), z.end(), 0.0);
      }
      long folded = 0;   // keys [0, folded) are in the state
      auto fold_to = [&](long end) {
        for (; folded < end; ++folded) {
          load_vec(k, L, H, d, b, folded, h, kv.data());
          load_vec(v, L, H, d, b, folded, h, vv.data());
          for (int a = 0; a < d; ++a) {
            const double pk = feature(fmap, ak, kv[a]);
            z[a] += pk;
            for (int e = 0; e < d; ++e) S[a * d + e] += pk * vv[e];
          }
        }
      };
      for (long c = 0; c < n_chunks; ++c) {
        const long w0 = std::max(0L, c * chunk_tokens - overlap);
        const long w1 = std::min<long>(L, (c + 1) * chunk_tokens);
        fold_to(w0);
        for (long i = c * chunk_tokens; i < w1; ++i) {
          if (row_mask && !row_mask[bh * L + i]) continue;
          load_vec(q, L, H, d, b, i, h, qv.data());
          for (int x = 0; x < d; ++x) pq[x] = feature(fmap, aq, qv[x]);
          double den = 0.0;
          std::fill(num.begin(), num.end(), 0.0);
          for (int a = 0; a < d; ++a) {
            den += pq[a] * z[a];
            for (int e = 0; e < d; ++e) num[e] += pq[a] * S[a * d + e];
          }
          for (long j = w0; j < w1; ++j) {
            load_vec(k, L, H, d, b, j, h, kv.data());
            load_vec(v, L, H, d, b, j, h, vv.data());
            double acc = 0.0;
            for (int x = 0; x < d; ++x) acc += qv[x] * kv[x];
            const double w = std::exp(scale * acc);
            den += w;
            for (int x = 0; x < d; ++x) num[x] += w * vv[x];
          }
          double* orow = o + ((static_cast<long>(b) * L + i) * H + h) * d;
          for (int x = 0; x < d; ++x) orow[x] = num[x] / den;
        }
      }
      fold_to(L);
      if (S_io) {
        std::copy(S.begin(), S.end(), S_io + bh * d * d);
        std::copy(z.begin(), z.end(), z_io + bh * d);
      }
    }
  }
  return 0;
}

// Exact combination of R partial attentions of the same rows over disjoint
// key sets (the join of Ring attention's key shards, ReGenVC "Unified
// sequence parallelism", Sec. 3.5): the softmax over the union of the key
// sets, written through each part's log-sum-exp.
//   o_parts [R][n][d], lse_parts [R][n] (natural log; -inf = no key) ->
//   o [n][d], lse [n].
int oracle_merge(const double* o_parts, const double* lse_parts, int R, long n, int d, double* o, double* lse) {
  if (R < 1) return 1;
  for (long i = 0; i < n; ++i) {
    double m = -std::numeric_limits<double>::infinity();
    for (int r = 0; r < R; ++r) m = std::max(m, lse_parts[r * n + i]);
    for (int c = 0; c < d; ++c) o[i * d + c] = 0.0;
    if (m == -std::numeric_limits<double>::infinity()) {
      lse[i] = m;
      continue;
    }
    double wsum = 0.0;
    for (int r = 0; r < R; ++r) {
      const double w = std::exp(lse_parts[r * n + i] - m);
      wsum += w;
      for (int c = 0; c < d; ++c) o[i * d + c] += w * o_parts[(r * n + i) * d + c];
    }
    for (int c = 0; c < d; ++c) o[i * d + c] /= wsum;
    lse[i] = m + std::log(wsum);
  }
  return 0;
}

}  // extern "C"
