// C ABI of libvattn: argument checks, TMA descriptors, launch
// configuration.  All kernels live in this one translation unit.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/vattn.h"
#include "attention.cuh"
#include "attention_pair.cuh"
#include "hybrid.cuh"
#include "kvcache.cuh"
#include "merge.cuh"
#include "feature_map.cuh"
#include "rope.cuh"
#include "selftest.cuh"

// Device status word: a kernel that gives up on a bounded wait records a
// nonzero code here (first code wins); vattn_check() reads and clears it.
__device__ uint32_t g_vattn_status;

namespace {

thread_local std::string t_last_error;

vattn_status fail(vattn_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
vattn_status fail(vattn_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

vattn_status cuda_fail(cudaError_t e, const char* where) {
  return fail(VATTN_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define VATTN_CUDA(call)                              \
  do {                                                \
    cudaError_t e_ = (call);                          \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
  int sms = 148, dev;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Launch with programmatic stream serialisation (the memory-bound kernels):
// the grid may be scheduled while the previous grid on the stream is still
// running, and its first act is griddepcontrol.wait, so it reads and writes
// nothing before that grid has completed; it then releases the next grid.
// Back-to-back launches (a CUDA graph of appends, the hybrid's delta and
// scan) thereby hide their launch gaps.
template <typename... KArgs, typename... Args>
cudaError_t launch_after(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Tail split of a FULL attention call: with `items` (pair, head, batch)
// work units on `sms` SMs (one two-tile CTA per SM), the last partial wave of
// r items leaves sms - r SMs idle for a whole item; when r <= sms / 2 those
// items run as s = min(sms / r, 16, key tiles) CTAs each (fewer when some
// would get no key tile), over parts of their keys, merged in the kernel.
// Workspace: r arrival counters, then the partials (lse fp32 and o fp32) of
// r * s CTAs x 256 query rows.
struct TailLayout {
  long long n_normal = 0;
  int n_split = 1, tail_items = 0;
  size_t off_count = 0, off_lse = 0, off_o = 0, bytes = 0;
};

TailLayout tail_layout(int B, int Lq, int Lk, int H, int d) {
  TailLayout t;
  if (B < 1 || Lq < 1 || Lk < 1 || H < 1 || d < 1) return t;
  const long long pairs = ((Lq + 127) / 128 + 1) / 2;
  const long long items = pairs * H * B;
  const int sms = sm_count();
  const long long waves = items / sms, r = items - waves * sms;
  const int key_tiles = (Lk + 127) / 128;
  if (waves < 1 || r == 0 || 2 * r > sms || key_tiles < 2) return t;
  int sp = static_cast<int>(sms / r);
  sp = std::min(sp, vattn::attn::kMaxSplit);
  sp = std::min(sp, key_tiles);
  // the kernel gives each split ceil(key_tiles / sp) key tiles: drop the
  // splits that would be left with none
  const int per = (key_tiles + sp - 1) / sp;
  sp = (key_tiles + per - 1) / per;
  if (sp < 2) return t;
  t.n_split = sp;
  t.tail_items = static_cast<int>(r);
  t.n_normal = items - r;
  t.off_count = 0;
  t.off_lse = round256(static_cast<size_t>(r) * 4);
  t.off_o = t.off_lse + round256(static_cast<size_t>(r) * sp * 256 * 4);
  t.bytes = t.off_o + static_cast<size_t>(r) * sp * 256 * d * 4;
  return t;
}

// ---------------------------------------------------------------- devices
constexpr int kMaxDevices = 64;
uint32_t* g_status_ptr[kMaxDevices];
std::mutex g_mu;

vattn_status current_device(int* dev) {
  VATTN_CUDA(cudaGetDevice(dev));
  if (*dev < 0 || *dev >= kMaxDevices) return fail(VATTN_ERR_UNSUPPORTED, "device index %d", *dev);
  return VATTN_OK;
}

vattn_status status_ptr(uint32_t** out) {
  int dev;
  vattn_status st = current_device(&dev);
  if (st) return st;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    VATTN_CUDA(cudaGetSymbolAddress(&p, g_vattn_status));
    g_status_ptr[dev] = static_cast<uint32_t*>(p);
  }
  *out = g_status_ptr[dev];
  return VATTN_OK;
}

// Opt a kernel into its dynamic shared memory size once per device.
template <typename K>
vattn_status ensure_smem(K kernel, int bytes, uint64_t* done_mask) {
  int dev;
  vattn_status st = current_device(&dev);
  if (st) return st;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!(done_mask[dev / 64] & (1ull << (dev % 64)))) {
    VATTN_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
    done_mask[dev / 64] |= 1ull << (dev % 64);
  }
  return VATTN_OK;
}

// ------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

vattn_status get_encode(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    VATTN_CUDA(cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q));
    if (q != cudaDriverEntryPointSuccess || !p)
      return fail(VATTN_ERR_CUDA, "cuTensorMapEncodeTiled not available from the driver");
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  *fn = g_encode;
  return VATTN_OK;
}

// bf16 tensor [n3][n2][n1][d] (d innermost) as a 4-D TMA map whose box is
// 64 channels x 1 x `rows` x 1, 128-byte swizzle, zero fill out of range.
vattn_status make_map(CUtensorMap* m, const void* base, int d, int n1, int n2, int n3, int rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  vattn_status st = get_encode(&enc);
  if (st) return st;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n1),
                              static_cast<cuuint64_t>(n2), static_cast<cuuint64_t>(n3)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(d) * 2 * n1,
                                 static_cast<cuuint64_t>(d) * 2 * n1 * n2};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(rows), 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(VATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return VATTN_OK;
}

// ------------------------------------------------------------------ rope
vattn_status check_rope(const vattn_rope* r, int d) {
  if (!r) return fail(VATTN_ERR_INVALID_ARG, "rope is NULL");
  if (d % 2) return fail(VATTN_ERR_INVALID_ARG, "odd head dim");
  if (r->Hg < 1 || r->Wg < 1) return fail(VATTN_ERR_INVALID_ARG, "rope grid Hg=%d Wg=%d", r->Hg, r->Wg);
  if (r->pairs_t < 0 || r->pairs_h < 0 || r->pairs_w < 0 || r->pairs_t + r->pairs_h + r->pairs_w != d / 2)
    return fail(VATTN_ERR_INVALID_ARG, "rope pairs %d+%d+%d != d/2=%d", r->pairs_t, r->pairs_h, r->pairs_w,
                d / 2);
  if (r->max_pos < 1 || r->max_pos > (1 << 20)) return fail(VATTN_ERR_INVALID_ARG, "rope max_pos %d", r->max_pos);
  if (r->Hg > r->max_pos || r->Wg > r->max_pos)
    return fail(VATTN_ERR_INVALID_ARG, "rope max_pos %d smaller than the grid", r->max_pos);
  if (!(r->theta > 0.0) || !std::isfinite(r->theta)) return fail(VATTN_ERR_INVALID_ARG, "rope theta");
  return VATTN_OK;
}

bool supported_d(int d) { return d == 64 || d == 128; }

uint64_t g_fused_smem_done[2][1];

// One query tile per CTA, Q and every K tile rotated in the kernel
// (attention.cuh): grid = query tiles x heads x batch.
template <int D>
vattn_status launch_fused(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& k2,
                          const CUtensorMap& v2, const vattn::attn::Params& p, cudaStream_t s) {
  using Cfg = vattn::attn::Cfg<D>;
  auto kern = vattn::attn::attn_fwd_kernel<D>;
  vattn_status st = ensure_smem(kern, Cfg::kSmemBytes, g_fused_smem_done[D == 64 ? 0 : 1]);
  if (st) return st;
  const dim3 grid(p.n_q_tiles, p.H, p.B);
  kern<<<grid, vattn::attn::kFusedThreads, Cfg::kSmemBytes, s>>>(q, k, v, k2, v2, p);
  VATTN_CUDA(cudaGetLastError());
  return VATTN_OK;
}

uint64_t g_pair_smem_done[5][1];

// Two query tiles per CTA (attention_pair.cuh): grid = tile pairs x heads x
// batch.
template <int D, int ROPE, bool HYB = false>
vattn_status launch_pair(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& k2,
                         const CUtensorMap& v2, const CUtensorMap& o, const vattn::attn::Params& p, cudaStream_t s) {
  using Cfg = vattn::attn::PairCfg<D>;
  constexpr int slot = HYB ? 4 : (D == 64 ? 0 : 2) + (ROPE == vattn::attn::kRopeQ ? 1 : 0);
  auto kern = vattn::attn::attn_pair_kernel<D, ROPE, HYB>;
  vattn_status st = ensure_smem(kern, Cfg::kSmemBytes, g_pair_smem_done[slot]);
  if (st) return st;
  const int segs = p.n_q_tiles / p.q_tiles_per_seg;
  const long long pairs = static_cast<long long>(segs) * ((p.q_tiles_per_seg + 1) / 2);
  if (pairs > 0x7fffffffLL) return fail(VATTN_ERR_UNSUPPORTED, "too many query tiles");
  const dim3 grid = p.linear_grid ? dim3(static_cast<unsigned>(p.total_ctas))
                                  : dim3(static_cast<unsigned>(pairs), p.H, p.B);
  kern<<<grid, vattn::attn::kPairThreads, Cfg::kSmemBytes, s>>>(q, k, v, k2, v2, o, p);
  VATTN_CUDA(cudaGetLastError());
  return VATTN_OK;
}

vattn_status dispatch_attention(int d, int rope_mode, const CUtensorMap& q, const CUtensorMap& k,
                                const CUtensorMap& v, const CUtensorMap& k2, const CUtensorMap& v2,
                                const CUtensorMap& o, const vattn::attn::Params& p, cudaStream_t s) {
  using namespace vattn::attn;
  // keys rotated inside the kernel: the one-tile kernel with the RoPE warpgroup
  if (rope_mode == kRopeQK)
    return d == 64 ? launch_fused<64>(q, k, v, k2, v2, p, s) : launch_fused<128>(q, k, v, k2, v2, p, s);
  // keys already rotated (or no RoPE): the two-tile kernel
  if (d == 64)
    return rope_mode == kRopeQ ? launch_pair<64, kRopeQ>(q, k, v, k2, v2, o, p, s)
                               : launch_pair<64, kRopeNone>(q, k, v, k2, v2, o, p, s);
  return rope_mode == kRopeQ ? launch_pair<128, kRopeQ>(q, k, v, k2, v2, o, p, s)
                             : launch_pair<128, kRopeNone>(q, k, v, k2, v2, o, p, s);
}

// Rotate K once into k_out (the standalone RoPE kernel on keys only).
vattn_status launch_rope_k(const void* k, void* k_out, int B, int L, int Hkv, int d, const vattn_rope* rope,
                           const float* table, int frame_offset, cudaStream_t stream) {
  return vattn_rope_qk(nullptr, k, nullptr, k_out, B, L, 1, Hkv, d, rope, table, frame_offset, stream);
}

void fill_rope_params(vattn::attn::Params& p, const vattn_rope* r, const float* table) {
  if (!r) return;
  p.rope_tab = reinterpret_cast<const float2*>(table);
  p.rope_Hg = r->Hg;
  p.rope_Wg = r->Wg;
  p.rope_pt = r->pairs_t;
  p.rope_ph = r->pairs_h;
  p.rope_maxpos = r->max_pos;
}

// Threads cover the chunks of one row in as few equal passes of at most
// 512 as possible; each block takes 4..16 consecutive rows (about 4 blocks
// per SM for small tensors, 16 rows per block for large ones), so a thread
// has several independent rows in flight.
template <bool COPY>
cudaError_t launch_rotate_rows(const vattn::rope::RotParams& p, cudaStream_t stream) {
  int sms = 148, dev;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int cpt = p.heads * (p.d / 8);
  const int passes = (cpt + 511) / 512;
  const int threads = (((cpt + passes - 1) / passes + 31) / 32) * 32;
  long long rpb = p.rows / (4LL * sms);
  rpb = rpb < 4 ? 4 : (rpb > 16 ? 16 : rpb);
  long long blocks = (p.rows + rpb - 1) / rpb;
  if (blocks > p.rows) blocks = p.rows;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  return launch_after(vattn::rope::rotate_rows_kernel<COPY>, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, stream, p);
}

}  // namespace

// ============================================================ C interface
struct vattn_kvcache {
  void* k_ring;
  void* v_ring;
  int32_t* frame_ids;
  int capacity, B, F, Hkv, d;
  std::vector<int32_t> host_ids;
  CUtensorMap map_k, map_v;
  // optional rotated-key ring: capacity + 1 slots, frame f in slot f % (capacity + 1)
  void* k_rot = nullptr;
  vattn_rope rope{};
  const float* table = nullptr;
  CUtensorMap map_krot;
  // the last vattn_attention_stream call rotated these keys of this frame
  // into the rotated ring (host-side record; cleared by restore/enable_rope)
  const void* rotated_k = nullptr;
  int rotated_frame = -1;
  int sub = 1;              // latent frames (Hg x Wg tokens) per cache frame
  // positions of the rotated ring: -1 absolute frame index; otherwise the
  // window start frame of the last window-relative step
  int rot_base = -1;
};

namespace {
size_t frame_bytes(const vattn_kvcache* c) { return static_cast<size_t>(c->B) * c->F * c->Hkv * c->d * 2; }

// Launch the append / rotate pass for one frame: rotated K into slot
// frame % (capacity + 1) of the rotated ring, the frame's first token at
// RoPE t = t0.  kr/vr null: rotate only.
vattn_status launch_append_rope(const vattn_kvcache* c, const void* k, const void* v, void* kr, void* vr,
                                int32_t* ids, int slot, int frame, int t0, cudaStream_t stream) {
  vattn::rope::RotParams p{};
  p.src = static_cast<const uint4*>(k);
  p.dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(c->k_rot) +
                                   static_cast<size_t>(frame % (c->capacity + 1)) * frame_bytes(c));
  p.src2 = static_cast<const uint4*>(v);
  p.raw_dst = static_cast<uint4*>(kr);
  p.raw_dst2 = static_cast<uint4*>(vr);
  p.rows = static_cast<long long>(c->B) * c->F;
  p.L = c->F;
  p.heads = c->Hkv;
  p.d = c->d;
  p.frame_offset = t0;
  p.Hg = c->rope.Hg;
  p.Wg = c->rope.Wg;
  p.pt = c->rope.pairs_t;
  p.ph = c->rope.pairs_h;
  p.tab = reinterpret_cast<const float2*>(c->table);
  p.ids = ids;
  p.slot = slot;
  p.frame = frame;
  VATTN_CUDA(kr ? launch_rotate_rows<true>(p, stream) : launch_rotate_rows<false>(p, stream));
  return VATTN_OK;
}

// Rotate every frame present in the raw ring into the rotated-key ring at
// its absolute frame index.
vattn_status rerotate_present(vattn_kvcache* c, cudaStream_t stream) {
  const size_t bytes = frame_bytes(c);
  for (int i = 0; i < c->capacity; ++i) {
    const int fr = c->host_ids[i];
    if (fr < 0) continue;
    if (static_cast<long long>(c->sub) * (fr + 1) > c->rope.max_pos)
      return fail(VATTN_ERR_INVALID_ARG, "frame %d beyond rope max_pos", fr);
    const uint8_t* kraw = static_cast<const uint8_t*>(c->k_ring) + static_cast<size_t>(i) * bytes;
    const uint8_t* vraw = static_cast<const uint8_t*>(c->v_ring) + static_cast<size_t>(i) * bytes;
    if (vattn_status st = launch_append_rope(c, kraw, vraw, nullptr, nullptr, nullptr, 0, fr, c->sub * fr, stream))
      return st;
  }
  c->rot_base = -1;
  return VATTN_OK;
}

// Put the rotated ring back at absolute positions after window-relative
// steps (which leave it rotated relative to their last window).
vattn_status to_absolute(vattn_kvcache* c, cudaStream_t stream) {
  if (!c->k_rot || c->rot_base < 0) return VATTN_OK;
  return rerotate_present(c, stream);
}

bool same_rope(const vattn_rope& a, const vattn_rope& b) {
  return a.Hg == b.Hg && a.Wg == b.Wg && a.pairs_t == b.pairs_t && a.pairs_h == b.pairs_h &&
         a.pairs_w == b.pairs_w && a.theta == b.theta && a.max_pos == b.max_pos;
}
}  // namespace

extern "C" {

const char* vattn_status_string(vattn_status s) {
  switch (s) {
    case VATTN_OK: return "ok";
    case VATTN_ERR_INVALID_ARG: return "invalid argument";
    case VATTN_ERR_UNSUPPORTED: return "unsupported";
    case VATTN_ERR_CUDA: return "CUDA error";
    case VATTN_ERR_TIMEOUT: return "kernel wait timed out";
  }
  return "unknown status";
}

const char* vattn_last_error(void) { return t_last_error.c_str(); }

vattn_status vattn_check(vattn_stream stream) {
  VATTN_CUDA(cudaStreamSynchronize(stream));
  uint32_t v = 0;
  VATTN_CUDA(cudaMemcpyFromSymbol(&v, g_vattn_status, sizeof(v)));
  if (v) {
    const uint32_t zero = 0;
    VATTN_CUDA(cudaMemcpyToSymbol(g_vattn_status, &zero, sizeof(zero)));
    if (v == vattn::sm100::kStatusSmemAlign)
      return fail(VATTN_ERR_CUDA, "dynamic shared memory was not 1024-byte aligned; the kernel did not run");
    return fail(VATTN_ERR_TIMEOUT, "a kernel gave up on a bounded wait (code %u)", v);
  }
  return VATTN_OK;
}

size_t vattn_rope_table_bytes(const vattn_rope* rope, int d) {
  if (check_rope(rope, d)) return 0;
  return static_cast<size_t>(rope->max_pos) * (d / 2) * sizeof(float2);
}

vattn_status vattn_rope_table_build(const vattn_rope* rope, int d, float* table, vattn_stream stream) {
  if (vattn_status st = check_rope(rope, d)) return st;
  if (!table || (reinterpret_cast<uintptr_t>(table) & 7u))
    return fail(VATTN_ERR_INVALID_ARG, "table must be a non-NULL 8-byte aligned device pointer");
  const int n = rope->max_pos * (d / 2);
  vattn::rope::table_kernel<<<(n + 255) / 256, 256, 0, stream>>>(
      reinterpret_cast<float2*>(table), rope->max_pos, d / 2, rope->pairs_t, rope->pairs_h, rope->pairs_w,
      rope->theta);
  VATTN_CUDA(cudaGetLastError());
  return VATTN_OK;
}

vattn_status vattn_rope_qk(const void* q, const void* k, void* q_out, void* k_out, int B, int L, int H, int Hkv,
                           int d, const vattn_rope* rope, const float* table, int frame_offset,
                           vattn_stream stream) {
  if (B < 1 || L < 1 || H < 1 || Hkv < 1) return fail(VATTN_ERR_INVALID_ARG, "sizes must be >= 1");
  if (d < 8 || d % 8) return fail(VATTN_ERR_UNSUPPORTED, "head dim %d (multiple of 8 required)", d);
  if (vattn_status st = check_rope(rope, d)) return st;
  if (!table) return fail(VATTN_ERR_INVALID_ARG, "table is NULL");
  if ((q == nullptr) != (q_out == nullptr) || (k == nullptr) != (k_out == nullptr))
    return fail(VATTN_ERR_INVALID_ARG, "q/q_out and k/k_out must be given together");
  if ((q && (!aligned16(q) || !aligned16(q_out))) || (k && (!aligned16(k) || !aligned16(k_out))))
    return fail(VATTN_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if (frame_offset < 0) return fail(VATTN_ERR_INVALID_ARG, "frame_offset < 0");
  const long long F = static_cast<long long>(rope->Hg) * rope->Wg;
  if (frame_offset + (L - 1) / F >= rope->max_pos)
    return fail(VATTN_ERR_INVALID_ARG, "frame index beyond rope max_pos");
  for (int which = 0; which < 2; ++which) {
    const void* src = which ? k : q;
    void* dst = which ? k_out : q_out;
    if (!src) continue;
    vattn::rope::RotParams p{};
    p.src = static_cast<const uint4*>(src);
    p.dst = static_cast<uint4*>(dst);
    p.rows = static_cast<long long>(B) * L;
    p.L = L;
    p.heads = which ? Hkv : H;
    p.d = d;
    p.frame_offset = frame_offset;
    p.Hg = rope->Hg;
    p.Wg = rope->Wg;
    p.pt = rope->pairs_t;
    p.ph = rope->pairs_h;
    p.tab = reinterpret_cast<const float2*>(table);
    VATTN_CUDA(launch_rotate_rows<false>(p, stream));
  }
  return VATTN_OK;
}

size_t vattn_attention_workspace_bytes(int B, int Lk, int Hkv, int d, const vattn_rope* rope) {
  if (!rope || B < 1 || Lk < 1 || Hkv < 1 || d < 1) return 0;
  return static_cast<size_t>(B) * Lk * Hkv * d * 2;
}

size_t vattn_attention_workspace_bytes_ex(int B, int Lq, int Lk, int H, int Hkv, int d, vattn_mode mode,
                                          const vattn_rope* rope) {
  const size_t rot = vattn_attention_workspace_bytes(B, Lk, Hkv, d, rope);
  if (mode != VATTN_FULL) return rot;
  const TailLayout t = tail_layout(B, Lq, Lk, H, d);
  if (t.n_split <= 1) return rot;
  return (rope ? round256(rot) : 0) + t.bytes;
}

// vattn_attention with the two self-test knobs of the parameter block (a
// wait bound other than the default, one withheld softmax arrival).
static vattn_status attention_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                                   int Lq, int Lk, int H, int Hkv, int d, float scale, vattn_mode mode,
                                   int tokens_per_frame, int chunk_frames, int window_back, int window_fwd,
                                   int q_frame_offset, int k_frame_offset, const vattn_rope* rope,
                                   const float* table, void* workspace, size_t workspace_bytes,
                                   vattn_stream stream, uint64_t wait_limit_ns, int withhold) {
  if (!q || !k || !v || !o) return fail(VATTN_ERR_INVALID_ARG, "q, k, v, o must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(VATTN_ERR_INVALID_ARG, "q, k, v, o must be 16-byte aligned");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return fail(VATTN_ERR_INVALID_ARG, "lse misaligned");
  if (B < 1 || Lq < 1 || Lk < 1 || H < 1 || Hkv < 1) return fail(VATTN_ERR_INVALID_ARG, "sizes must be >= 1");
  if (B > 65535 || H > 65535) return fail(VATTN_ERR_UNSUPPORTED, "B or H above 65535");
  if (H % Hkv) return fail(VATTN_ERR_INVALID_ARG, "H=%d not a multiple of Hkv=%d", H, Hkv);
  if (!supported_d(d)) return fail(VATTN_ERR_UNSUPPORTED, "head dim %d (64 or 128 supported)", d);
  if (!std::isfinite(scale)) return fail(VATTN_ERR_INVALID_ARG, "scale not finite");
  if (mode != VATTN_FULL && mode != VATTN_CHUNK_CAUSAL && mode != VATTN_SLIDING)
    return fail(VATTN_ERR_INVALID_ARG, "mode %d", static_cast<int>(mode));
  if (q_frame_offset < 0 || k_frame_offset < 0) return fail(VATTN_ERR_INVALID_ARG, "negative frame offset");
  if (mode != VATTN_FULL && tokens_per_frame < 1)
    return fail(VATTN_ERR_INVALID_ARG, "tokens_per_frame must be >= 1 for masked modes");
  if (mode == VATTN_CHUNK_CAUSAL && chunk_frames < 1) return fail(VATTN_ERR_INVALID_ARG, "chunk_frames < 1");
  if (mode == VATTN_SLIDING && (window_back < 0 || window_fwd < 0))
    return fail(VATTN_ERR_INVALID_ARG, "negative window");
  if ((rope == nullptr) != (table == nullptr)) return fail(VATTN_ERR_INVALID_ARG, "rope and table go together");
  if (rope) {
    if (vattn_status st = check_rope(rope, d)) return st;
    const long long Fr = static_cast<long long>(rope->Hg) * rope->Wg;
    if (mode != VATTN_FULL && tokens_per_frame != Fr)
      return fail(VATTN_ERR_INVALID_ARG, "tokens_per_frame %d != Hg*Wg %lld", tokens_per_frame, Fr);
    if (q_frame_offset + (Lq - 1) / Fr >= rope->max_pos || k_frame_offset + (Lk - 1) / Fr >= rope->max_pos)
      return fail(VATTN_ERR_INVALID_ARG, "frame index beyond rope max_pos");
  }
  if (workspace) {
    if (!aligned16(workspace)) return fail(VATTN_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    if (rope && workspace_bytes < vattn_attention_workspace_bytes(B, Lk, Hkv, d, rope))
      return fail(VATTN_ERR_INVALID_ARG, "workspace %zu bytes < %zu required", workspace_bytes,
                  vattn_attention_workspace_bytes(B, Lk, Hkv, d, rope));
  }
  const int wb = window_back > (1 << 24) ? (1 << 24) : window_back;
  const int wf = window_fwd > (1 << 24) ? (1 << 24) : window_fwd;

  vattn::attn::Params p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  if (vattn_status st = status_ptr(&p.status)) return st;
  p.B = B;
  p.Lq = Lq;
  p.Lk = Lk;
  p.H = H;
  p.Hkv = Hkv;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.mode = static_cast<int>(mode);
  p.F = tokens_per_frame > 0 ? tokens_per_frame : 1;
  p.chunk = chunk_frames > 0 ? chunk_frames : 1;
  p.wb = wb;
  p.wf = wf;
  p.qoff = q_frame_offset;
  p.koff = k_frame_offset;
  p.q_seg_len = Lq;
  p.q_tiles_per_seg = (Lq + 127) / 128;
  p.n_q_tiles = p.q_tiles_per_seg;
  p.reverse_q = mode == VATTN_CHUNK_CAUSAL ? 1 : 0;
  p.n_kseg = 0;
  p.wait_limit_ns = wait_limit_ns;
  p.test_withhold = withhold;
  fill_rope_params(p, rope, table);

  CUtensorMap mq, mk, mv, mo;
  if (vattn_status st = make_map(&mq, q, d, H, Lq, B, 128)) return st;
  if (vattn_status st = make_map(&mk, k, d, Hkv, Lk, B, 128)) return st;
  if (vattn_status st = make_map(&mv, v, d, Hkv, Lk, B, 128)) return st;
  if (vattn_status st = make_map(&mo, o, d, H, Lq, B, 128)) return st;
  // tail split (FULL mode, two-tile kernel, workspace of the _ex size)
  if (workspace && mode == VATTN_FULL) {
    const size_t base = rope ? round256(vattn_attention_workspace_bytes(B, Lk, Hkv, d, rope)) : 0;
    const TailLayout t = tail_layout(B, Lq, Lk, H, d);
    if (t.n_split > 1 && workspace_bytes >= base + t.bytes) {
      uint8_t* ws = static_cast<uint8_t*>(workspace) + base;
      p.linear_grid = 1;
      p.tail_split = 1;
      p.n_split = t.n_split;
      p.n_normal = static_cast<int>(t.n_normal);
      p.n_pairs = (p.q_tiles_per_seg + 1) / 2;
      p.pair_count = reinterpret_cast<uint32_t*>(ws + t.off_count);
      p.part_lse = reinterpret_cast<float*>(ws + t.off_lse);
      p.part_o = reinterpret_cast<float*>(ws + t.off_o);
      const long long total = t.n_normal + static_cast<long long>(t.tail_items) * t.n_split;
      if (total > 0x7fffffffLL) return fail(VATTN_ERR_UNSUPPORTED, "grid too large");
      p.total_ctas = static_cast<int>(total);
    }
  }
  if (rope && workspace) {
    // rotate K once into the workspace; the kernel rotates Q tiles itself
    if (vattn_status st = launch_rope_k(k, workspace, B, Lk, Hkv, d, rope, table, k_frame_offset, stream))
      return st;
    CUtensorMap mkr;
    if (vattn_status st = make_map(&mkr, workspace, d, Hkv, Lk, B, 128)) return st;
    return dispatch_attention(d, vattn::attn::kRopeQ, mq, mkr, mv, mkr, mv, mo, p, stream);
  }
  return dispatch_attention(d, rope ? vattn::attn::kRopeQK : vattn::attn::kRopeNone, mq, mk, mv, mk, mv, mo, p,
                            stream);
}

vattn_status vattn_attention(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Lq,
                             int Lk, int H, int Hkv, int d, float scale, vattn_mode mode, int tokens_per_frame,
                             int chunk_frames, int window_back, int window_fwd, int q_frame_offset,
                             int k_frame_offset, const vattn_rope* rope, const float* table,
                             void* workspace, size_t workspace_bytes, vattn_stream stream) {
  return attention_impl(q, k, v, o, lse, B, Lq, Lk, H, Hkv, d, scale, mode, tokens_per_frame, chunk_frames,
                        window_back, window_fwd, q_frame_offset, k_frame_offset, rope, table, workspace,
                        workspace_bytes, stream, 0, 0);
}

// ------------------------------------------------------------- KV cache
vattn_status vattn_kvcache_init(vattn_kvcache** cache, void* k_ring, void* v_ring, int32_t* frame_ids,
                                int capacity, int B, int F, int Hkv, int d, vattn_stream stream) {
  if (!cache || !k_ring || !v_ring || !frame_ids) return fail(VATTN_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(k_ring) || !aligned16(v_ring) || (reinterpret_cast<uintptr_t>(frame_ids) & 3u))
    return fail(VATTN_ERR_INVALID_ARG, "ring buffers must be 16-byte aligned");
  if (capacity < 1 || capacity > vattn::attn::kMaxKeySegments - 1)
    return fail(VATTN_ERR_UNSUPPORTED, "capacity %d (1..%d)", capacity, vattn::attn::kMaxKeySegments - 1);
  if (B < 1 || F < 1 || Hkv < 1) return fail(VATTN_ERR_INVALID_ARG, "sizes must be >= 1");
  if (!supported_d(d)) return fail(VATTN_ERR_UNSUPPORTED, "head dim %d", d);
  if (static_cast<long long>(capacity) * B > 65535) return fail(VATTN_ERR_UNSUPPORTED, "capacity*B too large");
  vattn_kvcache* c = new vattn_kvcache();
  c->k_ring = k_ring;
  c->v_ring = v_ring;
  c->frame_ids = frame_ids;
  c->capacity = capacity;
  c->B = B;
  c->F = F;
  c->Hkv = Hkv;
  c->d = d;
  c->host_ids.assign(capacity, -1);
  vattn_status st = make_map(&c->map_k, k_ring, d, Hkv, F, capacity * B, 128);
  if (!st) st = make_map(&c->map_v, v_ring, d, Hkv, F, capacity * B, 128);
  if (st) {
    delete c;
    return st;
  }
  cudaError_t e = cudaMemsetAsync(frame_ids, 0xFF, sizeof(int32_t) * capacity, stream);
  if (e != cudaSuccess) {
    delete c;
    return cuda_fail(e, "cudaMemsetAsync(frame_ids)");
  }
  *cache = c;
  return VATTN_OK;
}

vattn_status vattn_kvcache_append(vattn_kvcache* c, const void* k, const void* v, int frame_idx,
                                  vattn_stream stream) {
  if (!c || !k || !v) return fail(VATTN_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(k) || !aligned16(v)) return fail(VATTN_ERR_INVALID_ARG, "k, v must be 16-byte aligned");
  if (frame_idx < 0) return fail(VATTN_ERR_INVALID_ARG, "frame_idx < 0");
  const int slot = frame_idx % c->capacity;
  const long long bytes = static_cast<long long>(c->B) * c->F * c->Hkv * c->d * 2;
  const long long n16 = bytes / 16;
  uint4* kr = reinterpret_cast<uint4*>(static_cast<uint8_t*>(c->k_ring) + slot * bytes);
  uint4* vr = reinterpret_cast<uint4*>(static_cast<uint8_t*>(c->v_ring) + slot * bytes);
  const bool rotated = c->k_rot && c->rotated_k == k && c->rotated_frame == frame_idx;
  c->rotated_k = nullptr;
  c->rotated_frame = -1;
  if (c->k_rot && !rotated) {
    if (static_cast<long long>(c->sub) * (frame_idx + 1) > c->rope.max_pos)
      return fail(VATTN_ERR_INVALID_ARG, "frame index beyond rope max_pos");
    if (vattn_status st = to_absolute(c, stream)) return st;
    if (vattn_status st = launch_append_rope(c, k, v, kr, vr, c->frame_ids, slot, frame_idx, c->sub * frame_idx,
                                             stream))
      return st;
    c->host_ids[slot] = frame_idx;
    return VATTN_OK;
  }
  // plain copy (also when the stream call already rotated these keys)
  int sms = 148, dev;
  if (current_device(&dev) == VATTN_OK) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // an equal share for every SM: a multiple of the SM count (at most two
  // blocks per SM, the fastest measured for one frame), each thread moving
  // kUnroll vectors per tensor and step
  const long long want = (n16 + 256LL * vattn::kv::kUnroll - 1) / (256LL * vattn::kv::kUnroll);
  const long long per_sm = (want + sms - 1) / sms;
  const int blocks = static_cast<int>(sms * (per_sm < 2 ? per_sm : 2));
  VATTN_CUDA(launch_after(vattn::kv::append_kernel, dim3(blocks), dim3(256), 0, stream, static_cast<const uint4*>(k),
                          static_cast<const uint4*>(v), kr, vr, n16, c->frame_ids, slot, frame_idx));
  c->host_ids[slot] = frame_idx;
  return VATTN_OK;
}

vattn_status vattn_attention_stream(vattn_kvcache* c, const void* q, const void* k_cur, const void* v_cur, void* o,
                                    float* lse, int H, int frame_idx, int window_back, float scale,
                                    const vattn_rope* rope, const float* table, vattn_stream stream) {
  if (!c || !q || !k_cur || !v_cur || !o) return fail(VATTN_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(q) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(o))
    return fail(VATTN_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return fail(VATTN_ERR_INVALID_ARG, "lse misaligned");
  if (H < 1 || H % c->Hkv) return fail(VATTN_ERR_INVALID_ARG, "H=%d vs Hkv=%d", H, c->Hkv);
  if (H > 65535) return fail(VATTN_ERR_UNSUPPORTED, "H above 65535");
  if (frame_idx < 0) return fail(VATTN_ERR_INVALID_ARG, "frame_idx < 0");
  if (window_back < 0 || window_back > c->capacity)
    return fail(VATTN_ERR_INVALID_ARG, "window_back %d outside 0..capacity(%d)", window_back, c->capacity);
  if (!std::isfinite(scale)) return fail(VATTN_ERR_INVALID_ARG, "scale not finite");
  if ((rope == nullptr) != (table == nullptr)) return fail(VATTN_ERR_INVALID_ARG, "rope and table go together");
  const bool rot_ring = rope && c->k_rot;
  if (rope) {
    if (vattn_status st = check_rope(rope, c->d)) return st;
    const long long Fr = static_cast<long long>(rope->Hg) * rope->Wg;
    // keys rotated in the kernel (no rotated ring) need one latent frame
    // per cache frame; the rotated ring allows several
    if (rot_ring ? (c->F % Fr) : (Fr != c->F))
      return fail(VATTN_ERR_INVALID_ARG, "rope grid Hg*Wg does not fit frame tokens %d", c->F);
    if ((c->F / Fr) * (static_cast<long long>(frame_idx) + 1) > rope->max_pos)
      return fail(VATTN_ERR_INVALID_ARG, "frame index beyond rope max_pos");
  }
  vattn::attn::Params p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  if (vattn_status st = status_ptr(&p.status)) return st;
  p.B = c->B;
  p.Lq = c->F;
  p.Lk = c->F;
  p.H = H;
  p.Hkv = c->Hkv;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.mode = 0;
  p.F = c->F;
  p.chunk = 1;
  p.qoff = rot_ring ? c->sub * frame_idx : frame_idx;
  p.q_seg_len = c->F;
  p.q_tiles_per_seg = (c->F + 127) / 128;
  p.n_q_tiles = p.q_tiles_per_seg;
  p.reverse_q = 0;
  // Keys come from the rotated-key ring (rotated once per frame) when the
  // cache has one and the call rotates; otherwise from the raw ring, rotated
  // tile by tile in the kernel when rope is given.
  if (rot_ring) {
    if (!same_rope(*rope, c->rope) || table != c->table)
      return fail(VATTN_ERR_INVALID_ARG, "rope/table differ from those given to vattn_kvcache_enable_rope");
    if (vattn_status st = to_absolute(c, stream)) return st;
    // the current frame's rotated keys: slot frame_idx % (capacity + 1),
    // which holds a frame outside the window
    if (vattn_status st = launch_append_rope(c, k_cur, v_cur, nullptr, nullptr, nullptr, 0, frame_idx,
                                             c->sub * frame_idx, stream))
      return st;
    c->rotated_k = k_cur;
    c->rotated_frame = frame_idx;
  }
  int n = 0, tiles = 0;
  const int per = (c->F + 127) / 128;
  const int rcap = c->capacity + 1;
  for (int fr = frame_idx - window_back; fr < frame_idx; ++fr) {
    if (fr < 0) continue;
    const int slot = fr % c->capacity;
    if (c->host_ids[slot] != fr) continue;
    const int kc3 = rot_ring ? (fr % rcap) * c->B : slot * c->B;
    p.kseg[n] = vattn::attn::KeySegment{0, kc3, 0, slot * c->B, 0, c->F, fr, tiles};
    tiles += per;
    ++n;
  }
  if (rot_ring)
    p.kseg[n] = vattn::attn::KeySegment{0, (frame_idx % rcap) * c->B, 1, 0, 0, c->F, frame_idx, tiles};
  else
    p.kseg[n] = vattn::attn::KeySegment{1, 0, 1, 0, 0, c->F, frame_idx, tiles};
  ++n;
  p.n_kseg = n;
  p.seg_tok = c->F;
  fill_rope_params(p, rope, table);
  CUtensorMap mq, mk2, mv2, mo;
  if (vattn_status st = make_map(&mq, q, c->d, H, c->F, c->B, 128)) return st;
  if (vattn_status st = make_map(&mk2, k_cur, c->d, c->Hkv, c->F, c->B, 128)) return st;
  if (vattn_status st = make_map(&mv2, v_cur, c->d, c->Hkv, c->F, c->B, 128)) return st;
  if (vattn_status st = make_map(&mo, o, c->d, H, c->F, c->B, 128)) return st;
  if (rot_ring)
    return dispatch_attention(c->d, vattn::attn::kRopeQ, mq, c->map_krot, c->map_v, c->map_krot, mv2, mo, p,
                              stream);
  return dispatch_attention(c->d, rope ? vattn::attn::kRopeQK : vattn::attn::kRopeNone, mq, c->map_k,
                            c->map_v, mk2, mv2, mo, p, stream);
}

vattn_status vattn_kvcache_frame_ids(const vattn_kvcache* c, int32_t* host_ids) {
  if (!c || !host_ids) return fail(VATTN_ERR_INVALID_ARG, "NULL pointer");
  std::memcpy(host_ids, c->host_ids.data(), sizeof(int32_t) * c->capacity);
  return VATTN_OK;
}



vattn_status vattn_kvcache_restore(vattn_kvcache* c, const int32_t* host_ids, vattn_stream stream) {
  if (!c || !host_ids) return fail(VATTN_ERR_INVALID_ARG, "NULL pointer");
  for (int i = 0; i < c->capacity; ++i)
    if (host_ids[i] >= 0 && host_ids[i] % c->capacity != i)
      return fail(VATTN_ERR_INVALID_ARG, "frame %d cannot sit in slot %d", host_ids[i], i);
  std::memcpy(c->host_ids.data(), host_ids, sizeof(int32_t) * c->capacity);
  c->rotated_k = nullptr;
  c->rotated_frame = -1;
  if (c->k_rot) return rerotate_present(c, stream);
  return VATTN_OK;
}

vattn_status vattn_kvcache_enable_rope(vattn_kvcache* c, void* k_ring_rot, const vattn_rope* rope,
                                       const float* table, vattn_stream stream) {
  if (!c || !k_ring_rot || !table) return fail(VATTN_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(k_ring_rot)) return fail(VATTN_ERR_INVALID_ARG, "k_ring_rot must be 16-byte aligned");
  if (vattn_status st = check_rope(rope, c->d)) return st;
  const long long Fr = static_cast<long long>(rope->Hg) * rope->Wg;
  if (c->F % Fr) return fail(VATTN_ERR_INVALID_ARG, "frame tokens %d not a multiple of Hg*Wg=%lld", c->F, Fr);
  if (static_cast<long long>(c->capacity + 1) * c->B > 65535)
    return fail(VATTN_ERR_UNSUPPORTED, "(capacity+1)*B too large");
  CUtensorMap m;
  if (vattn_status st = make_map(&m, k_ring_rot, c->d, c->Hkv, c->F, (c->capacity + 1) * c->B, 128)) return st;
  c->k_rot = k_ring_rot;
  c->sub = static_cast<int>(c->F / Fr);
  c->rope = *rope;
  c->table = table;
  c->map_krot = m;
  c->rotated_k = nullptr;
  c->rotated_frame = -1;
  return rerotate_present(c, stream);
}

vattn_status vattn_kvcache_destroy(vattn_kvcache* c) {
  delete c;
  return VATTN_OK;
}

}  // extern "C"

// ------------------------------------------------- fused streaming step
namespace {

// Key splits for `items` (pair, head, batch) work units of n_tiles key tiles
// each on `sms` SMs (one CTA per SM): the count minimising
//   waves * (tiles per split + 5 + merge) + merge,
// where 5 tiles stand for a CTA's prologue and epilogue (a CTA's fixed part
// is several thousand cycles, about two 128-key tiles' worth each way) and
// a split's partial write and merge read cost about 0.1 tile each.  Counts
// that would leave a split empty are skipped.  Against 1.5 tiles, 5 chose
// fewer splits for the XL-shaped 480p streams and measured 10-12 % faster
// there, with the other streams unchanged.
int choose_splits(long long items, int n_tiles, int sms) {
  double best = 1e300;
  int best_s = 1;
  for (int s = 1; s <= vattn::attn::kMaxSplit && s <= n_tiles; ++s) {
    const int per = (n_tiles + s - 1) / s;
    if ((n_tiles + per - 1) / per != s) continue;
    const double waves = std::ceil(static_cast<double>(items) * s / sms);
    const double cost = waves * (per + 5.0 + (s > 1 ? 0.1 : 0.0)) + (s > 1 ? 0.1 * s : 0.0);
    if (cost < best - 1e-9) {
      best = cost;
      best_s = s;
    }
  }
  return best_s;
}

struct StepLayout {
  int pairs, per_tiles, n_split_max;
  size_t off_count, off_lse, off_o, bytes;
};

// Workspace of vattn_kvcache_step: [0, 256) the step counters; then the
// pairs' arrival counters; then split partials (lse, o) for the largest
// split count any frame of this window can use.
StepLayout step_layout(const vattn_kvcache* c, int H, int window_back) {
  StepLayout L{};
  const int qt = (c->F + 127) / 128;
  L.pairs = (qt + 1) / 2;
  L.per_tiles = (c->F + 127) / 128;
  const int sms = sm_count();
  const long long items = static_cast<long long>(L.pairs) * H * c->B;
  L.n_split_max = 1;
  for (int nseg = 1; nseg <= window_back + 1; ++nseg) {
    const int s = choose_splits(items, nseg * L.per_tiles, sms);
    if (s > L.n_split_max) L.n_split_max = s;
  }
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  L.off_count = 256;
  L.off_lse = L.off_count + up(static_cast<size_t>(c->B) * H * L.pairs * 4);
  const size_t rows = static_cast<size_t>(c->B) * H * c->F;
  L.off_o = L.off_lse + (L.n_split_max > 1 ? up(L.n_split_max * rows * 4) : 0);
  L.bytes = L.off_o + (L.n_split_max > 1 ? L.n_split_max * rows * c->d * 4 : 0);
  return L;
}

uint64_t g_step_smem_done[4][1];

template <int D, int ROPE>
vattn_status launch_step(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& k2,
                         const CUtensorMap& v2, const CUtensorMap& o, const vattn::attn::Params& p, cudaStream_t s) {
  using Cfg = vattn::attn::PairCfg<D>;
  auto kern = vattn::attn::attn_pair_kernel<D, ROPE, false>;
  vattn_status st = ensure_smem(kern, Cfg::kSmemBytes,
                                g_step_smem_done[(D == 64 ? 0 : 2) + (ROPE == vattn::attn::kRopeQ ? 1 : 0)]);
  if (st) return st;
  kern<<<p.total_ctas, vattn::attn::kPairThreads, Cfg::kSmemBytes, s>>>(q, k, v, k2, v2, o, p);
  VATTN_CUDA(cudaGetLastError());
  return VATTN_OK;
}
}  // namespace

extern "C" {

size_t vattn_kvcache_step_workspace_bytes(const vattn_kvcache* c, int H, int window_back) {
  if (!c || H < 1 || window_back < 0 || window_back >= c->capacity) return 0;
  return step_layout(c, H, window_back).bytes;
}

vattn_status vattn_kvcache_step(vattn_kvcache* c, const void* q, const void* k_cur, const void* v_cur, void* o,
                                float* lse, int H, int frame_idx, int window_back, float scale,
                                const vattn_rope* rope, const float* table, int window_relative, void* workspace,
                                size_t workspace_bytes, vattn_stream stream) {
  if (!c || !q || !k_cur || !v_cur || !o || !workspace) return fail(VATTN_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(q) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(o) || !aligned16(workspace))
    return fail(VATTN_ERR_INVALID_ARG, "tensors and workspace must be 16-byte aligned");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return fail(VATTN_ERR_INVALID_ARG, "lse misaligned");
  if (H < 1 || H % c->Hkv) return fail(VATTN_ERR_INVALID_ARG, "H=%d vs Hkv=%d", H, c->Hkv);
  if (frame_idx < 0) return fail(VATTN_ERR_INVALID_ARG, "frame_idx < 0");
  if (window_back < 0 || window_back >= c->capacity)
    return fail(VATTN_ERR_INVALID_ARG,
                "window_back %d: the step appends into slot frame %% capacity, so capacity (%d) must exceed it",
                window_back, c->capacity);
  if (!std::isfinite(scale)) return fail(VATTN_ERR_INVALID_ARG, "scale not finite");
  if ((rope == nullptr) != (table == nullptr)) return fail(VATTN_ERR_INVALID_ARG, "rope and table go together");
  if (rope && !c->k_rot)
    return fail(VATTN_ERR_INVALID_ARG, "a step with RoPE needs the rotated-key ring (vattn_kvcache_enable_rope)");
  if (rope && (!same_rope(*rope, c->rope) || table != c->table))
    return fail(VATTN_ERR_INVALID_ARG, "rope/table differ from those given to vattn_kvcache_enable_rope");
  if (window_relative && !rope) return fail(VATTN_ERR_INVALID_ARG, "window_relative needs rope");
  const StepLayout Ly = step_layout(c, H, window_back);
  if (workspace_bytes < Ly.bytes)
    return fail(VATTN_ERR_INVALID_ARG, "workspace %zu bytes < %zu required", workspace_bytes, Ly.bytes);
  const int cap = c->capacity, rcap = cap + 1, sub = c->sub;
  const int base = window_relative ? std::max(0, frame_idx - window_back) : 0;
  if (rope && static_cast<long long>(sub) * (frame_idx - base + 1) > rope->max_pos)
    return fail(VATTN_ERR_INVALID_ARG, "frame position beyond rope max_pos");
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  // the window's earlier frames present in the ring
  std::vector<int> past;
  for (int fr = frame_idx - window_back; fr < frame_idx; ++fr)
    if (fr >= 0 && c->host_ids[fr % cap] == fr) past.push_back(fr);

  // positions of the rotated ring for this step
  if (rope) {
    if (window_relative) {
      // every earlier frame of the window again, relative to its start
      const size_t bytes = frame_bytes(c);
      for (int fr : past) {
        const uint8_t* kraw = static_cast<const uint8_t*>(c->k_ring) + static_cast<size_t>(fr % cap) * bytes;
        if (vattn_status st = launch_append_rope(c, kraw, nullptr, nullptr, nullptr, nullptr, 0, fr,
                                                 sub * (fr - base), stream))
          return st;
      }
      c->rot_base = base;
    } else if (vattn_status st = to_absolute(c, stream)) {
      return st;
    }
  }

  vattn::attn::Params p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  if (vattn_status st = status_ptr(&p.status)) return st;
  p.B = c->B;
  p.Lq = c->F;
  p.Lk = c->F;
  p.H = H;
  p.Hkv = c->Hkv;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.mode = 0;
  p.F = c->F;
  p.chunk = 1;
  p.qoff = sub * (frame_idx - base);
  p.q_seg_len = c->F;
  p.q_tiles_per_seg = (c->F + 127) / 128;
  p.n_q_tiles = p.q_tiles_per_seg;
  const int per = Ly.per_tiles;
  int n = 0, tiles = 0;
  for (int fr : past) {
    const int kc3 = rope ? (fr % rcap) * c->B : (fr % cap) * c->B;
    p.kseg[n++] = vattn::attn::KeySegment{0, kc3, 0, (fr % cap) * c->B, 0, c->F, fr, tiles};
    tiles += per;
  }
  const int cur_tile = tiles;
  if (rope)   // the current frame's keys: rotated into its spare-ring slot by this launch
    p.kseg[n++] = vattn::attn::KeySegment{0, (frame_idx % rcap) * c->B, 1, 0, 0, c->F, frame_idx, tiles};
  else
    p.kseg[n++] = vattn::attn::KeySegment{1, 0, 1, 0, 0, c->F, frame_idx, tiles};
  tiles += per;
  p.n_kseg = n;
  p.seg_tok = c->F;
  fill_rope_params(p, rope, table);

  // the append: raw K and V into slot frame % capacity (outside the window),
  // K rotated into the rotated ring, by the launch's first CTAs; attention
  // CTAs wait for them only before the current frame's rotated keys.  When
  // the window holds no earlier frame every CTA would wait at once: then
  // the append runs as its own launch first.
  const size_t fb = frame_bytes(c);
  const int slot = frame_idx % cap;
  uint8_t* kr = static_cast<uint8_t*>(c->k_ring) + static_cast<size_t>(slot) * fb;
  uint8_t* vr = static_cast<uint8_t*>(c->v_ring) + static_cast<size_t>(slot) * fb;
  uint8_t* krot = rope ? static_cast<uint8_t*>(c->k_rot) + static_cast<size_t>(frame_idx % rcap) * fb : nullptr;
  const int t0 = sub * (frame_idx - base);
  const bool fold = !rope || cur_tile > 0;
  if (!fold) {
    if (vattn_status st = launch_append_rope(c, k_cur, v_cur, kr, vr, c->frame_ids, slot, frame_idx, t0, stream))
      return st;
  }
  const long long chunks = static_cast<long long>(c->B) * c->F * c->Hkv * (c->d / 8);
  p.n_append = fold ? static_cast<int>(std::min<long long>(16, (chunks + 384 * 4 - 1) / (384 * 4))) : 0;
  p.app = vattn::attn::AppendWork{static_cast<const uint4*>(k_cur), static_cast<const uint4*>(v_cur),
                                  reinterpret_cast<uint4*>(kr), reinterpret_cast<uint4*>(vr),
                                  reinterpret_cast<uint4*>(krot), c->frame_ids, slot, frame_idx,
                                  static_cast<long long>(c->B) * c->F, c->F, t0};
  p.wait_tile = (fold && rope) ? cur_tile : -1;
  // key splits
  const long long items = static_cast<long long>(Ly.pairs) * H * c->B;
  p.n_split = choose_splits(items, tiles, sm_count());
  if (p.n_split > Ly.n_split_max) p.n_split = Ly.n_split_max;
  p.split_tiles = (tiles + p.n_split - 1) / p.n_split;
  p.n_split = (tiles + p.split_tiles - 1) / p.split_tiles;
  p.pair_count = reinterpret_cast<uint32_t*>(ws + Ly.off_count);
  p.part_lse = reinterpret_cast<float*>(ws + Ly.off_lse);
  p.part_o = reinterpret_cast<float*>(ws + Ly.off_o);
  p.step_sync = reinterpret_cast<uint32_t*>(ws);
  p.linear_grid = 1;
  p.n_pairs = Ly.pairs;
  const long long total = p.n_append + items * p.n_split;
  if (total > 0x7fffffffLL) return fail(VATTN_ERR_UNSUPPORTED, "grid too large");
  p.total_ctas = static_cast<int>(total);

  CUtensorMap mq, mk2, mv2, mo;
  if (vattn_status st = make_map(&mq, q, c->d, H, c->F, c->B, 128)) return st;
  if (vattn_status st = make_map(&mk2, k_cur, c->d, c->Hkv, c->F, c->B, 128)) return st;
  if (vattn_status st = make_map(&mv2, v_cur, c->d, c->Hkv, c->F, c->B, 128)) return st;
  if (vattn_status st = make_map(&mo, o, c->d, H, c->F, c->B, 128)) return st;
  const CUtensorMap& mk = rope ? c->map_krot : c->map_k;
  vattn_status st;
  if (c->d == 64)
    st = rope ? launch_step<64, vattn::attn::kRopeQ>(mq, mk, c->map_v, mk2, mv2, mo, p, stream)
              : launch_step<64, vattn::attn::kRopeNone>(mq, mk, c->map_v, mk2, mv2, mo, p, stream);
  else
    st = rope ? launch_step<128, vattn::attn::kRopeQ>(mq, mk, c->map_v, mk2, mv2, mo, p, stream)
              : launch_step<128, vattn::attn::kRopeNone>(mq, mk, c->map_v, mk2, mv2, mo, p, stream);
  if (st) return st;
  c->host_ids[slot] = frame_idx;
  c->rotated_k = nullptr;
  c->rotated_frame = -1;
  return VATTN_OK;
}

// ---------------------------------------------------------------- hybrid
size_t vattn_hybrid_workspace_bytes(int B, int L, int H, int d, int chunk_tokens) {
  if (B < 1 || L < 1 || H < 1 || d < 1 || chunk_tokens < 1) return 0;
  const size_t C = (static_cast<size_t>(L) + chunk_tokens - 1) / chunk_tokens;
  return C * B * H * (static_cast<size_t>(d) * d + d) * sizeof(float);
}

}  // extern "C"

namespace {
// Shared argument checks of the hybrid calls; C = number of chunks.
vattn_status check_hybrid(int B, int L, int H, int d, int chunk_tokens, const void* workspace,
                          size_t workspace_bytes, int* C) {
  if (!workspace) return fail(VATTN_ERR_INVALID_ARG, "NULL workspace");
  if (!aligned16(workspace)) return fail(VATTN_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if (B < 1 || L < 1 || H < 1 || chunk_tokens < 1) return fail(VATTN_ERR_INVALID_ARG, "sizes must be >= 1");
  if (B > 65535 || H > 65535) return fail(VATTN_ERR_UNSUPPORTED, "B or H above 65535");
  if (d != 128) return fail(VATTN_ERR_UNSUPPORTED, "hybrid supports head dim 128 (got %d)", d);
  const size_t need = vattn_hybrid_workspace_bytes(B, L, H, d, chunk_tokens);
  if (workspace_bytes < need)
    return fail(VATTN_ERR_INVALID_ARG, "workspace %zu bytes < %zu required", workspace_bytes, need);
  *C = (L + chunk_tokens - 1) / chunk_tokens;
  if (*C > 65535) return fail(VATTN_ERR_UNSUPPORTED, "more than 65535 chunks");
  return VATTN_OK;
}

// Launch 1 of the hybrid call: per-range state deltas into the workspace.
vattn_status launch_delta(const CUtensorMap& mk, const CUtensorMap& mv, float* wsS, float* wsz, uint32_t* status,
                          int B, int L, int H, int C, int chunk_tokens, cudaStream_t stream, int overlap = 0,
                          int fmap = vattn::fmap::kFmapElu1, const float* coef = nullptr) {
  static uint64_t done[2][1];
  const bool poly = fmap == vattn::fmap::kFmapPoly3;
  auto kern = poly ? vattn::hyb::delta_kernel<128, vattn::fmap::kFmapPoly3>
                   : vattn::hyb::delta_kernel<128, vattn::fmap::kFmapElu1>;
  const int smem = vattn::hyb::DeltaCfg<128>::kSmemBytes;
  if (vattn_status st = ensure_smem(kern, smem, done[poly ? 1 : 0])) return st;
  vattn::hyb::DeltaParams dp{wsS, wsz, status, B, L, H, chunk_tokens, overlap, fmap, coef};
  VATTN_CUDA(launch_after(kern, dim3(H, C, B), dim3(vattn::hyb::kDeltaThreads), smem, stream, mk, mv, dp));
  return VATTN_OK;
}

// Launch 2: exclusive scan over chunks, in place, plus the state out.
vattn_status launch_scan(float* wsS, float* wsz, float* S, float* z, int B, int H, int d, int C,
                         cudaStream_t stream) {
  const long long nS4 = static_cast<long long>(B) * H * d * d / 4, nz4 = static_cast<long long>(B) * H * d / 4;
  int sms = 148, dev;
  if (current_device(&dev) == VATTN_OK) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (nS4 + nz4 + 255) / 256;
  const int blocks = static_cast<int>(want < sms * 4LL ? want : sms * 4LL);
  VATTN_CUDA(launch_after(vattn::hyb::scan_kernel, dim3(blocks), dim3(256), 0, stream, reinterpret_cast<float4*>(wsS),
                          reinterpret_cast<float4*>(S), nS4, reinterpret_cast<float4*>(wsz),
                          reinterpret_cast<float4*>(z), nz4, C));
  return VATTN_OK;
}
}  // namespace

extern "C" {

vattn_status vattn_hybrid_delta(const void* k, const void* v, int B, int L, int H, int d, int chunk_tokens,
                                void* workspace, size_t workspace_bytes, vattn_stream stream) {
  if (!k || !v) return fail(VATTN_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(k) || !aligned16(v)) return fail(VATTN_ERR_INVALID_ARG, "k, v must be 16-byte aligned");
  int C;
  if (vattn_status st = check_hybrid(B, L, H, d, chunk_tokens, workspace, workspace_bytes, &C)) return st;
  float* wsS = static_cast<float*>(workspace);
  float* wsz = wsS + static_cast<size_t>(C) * B * H * d * d;
  uint32_t* status;
  if (vattn_status st = status_ptr(&status)) return st;
  CUtensorMap mk, mv;
  if (vattn_status st = make_map(&mk, k, d, H, L, B, vattn::hyb::kRows)) return st;
  if (vattn_status st = make_map(&mv, v, d, H, L, B, vattn::hyb::kRows)) return st;
  return launch_delta(mk, mv, wsS, wsz, status, B, L, H, C, chunk_tokens, stream);
}

vattn_status vattn_hybrid_scan(float* S, float* z, int B, int L, int H, int d, int chunk_tokens, void* workspace,
                               size_t workspace_bytes, vattn_stream stream) {
  if (!S || !z) return fail(VATTN_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(S) || !aligned16(z)) return fail(VATTN_ERR_INVALID_ARG, "S, z must be 16-byte aligned");
  int C;
  if (vattn_status st = check_hybrid(B, L, H, d, chunk_tokens, workspace, workspace_bytes, &C)) return st;
  float* wsS = static_cast<float*>(workspace);
  float* wsz = wsS + static_cast<size_t>(C) * B * H * d * d;
  return launch_scan(wsS, wsz, S, z, B, H, d, C, stream);
}

size_t vattn_hybrid_workspace_bytes_ex(int B, int L, int H, int d, int chunk_tokens, int overlap_tokens) {
  if (overlap_tokens < 0) return 0;
  return vattn_hybrid_workspace_bytes(B, L + overlap_tokens, H, d, chunk_tokens);
}

}  // extern "C"

namespace {
// The three launches of a hybrid call.  With overlap ov the state deltas
// cover the ranges [c ct - ov, (c + 1) ct - ov) (R = ceil((L + ov) / ct)
// of them) and each query chunk's softmax window starts ov tokens early.
vattn_status hybrid_impl(const void* q, const void* k, const void* v, void* o, float* S, float* z, int B, int L,
                         int H, int d, int chunk_tokens, int overlap, float scale, int fmap, const float* coef,
                         void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!q || !k || !v || !o || !S || !z) return fail(VATTN_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(S) || !aligned16(z))
    return fail(VATTN_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (!std::isfinite(scale)) return fail(VATTN_ERR_INVALID_ARG, "scale not finite");
  if (overlap < 0 || overlap > (1 << 30) - L) return fail(VATTN_ERR_INVALID_ARG, "overlap %d", overlap);
  if (fmap != vattn::fmap::kFmapElu1 && fmap != vattn::fmap::kFmapPoly3)
    return fail(VATTN_ERR_INVALID_ARG, "feature map %d", fmap);
  if (fmap == vattn::fmap::kFmapPoly3 && (!coef || !aligned16(coef)))
    return fail(VATTN_ERR_INVALID_ARG, "the polynomial feature map needs 16-byte aligned coefficients");
  int C, R;
  if (vattn_status st = check_hybrid(B, L, H, d, chunk_tokens, workspace, workspace_bytes, &C)) return st;
  if (vattn_status st = check_hybrid(B, L + overlap, H, d, chunk_tokens, workspace, workspace_bytes, &R)) return st;
  float* wsS = static_cast<float*>(workspace);
  float* wsz = wsS + static_cast<size_t>(R) * B * H * d * d;
  uint32_t* status;
  if (vattn_status st = status_ptr(&status)) return st;

  CUtensorMap mq, mk, mv, mo;
  if (vattn_status st = make_map(&mq, q, d, H, L, B, 128)) return st;
  if (vattn_status st = make_map(&mk, k, d, H, L, B, 128)) return st;
  if (vattn_status st = make_map(&mv, v, d, H, L, B, 128)) return st;
  if (vattn_status st = make_map(&mo, o, d, H, L, B, 128)) return st;

  // (1) per-range state deltas (tiles of vattn::hyb::kRows tokens), (2)
  // exclusive scan over ranges (+ state out)
  CUtensorMap mkd, mvd;
  if (vattn_status st = make_map(&mkd, k, d, H, L, B, vattn::hyb::kRows)) return st;
  if (vattn_status st = make_map(&mvd, v, d, H, L, B, vattn::hyb::kRows)) return st;
  if (vattn_status st = launch_delta(mkd, mvd, wsS, wsz, status, B, L, H, R, chunk_tokens, stream, overlap, fmap,
                                     coef))
    return st;
  if (vattn_status st = launch_scan(wsS, wsz, S, z, B, H, d, R, stream)) return st;
  // (3) attention with linear-state initialisation
  vattn::attn::Params p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = nullptr;
  p.status = status;
  p.B = B;
  p.Lq = L;
  p.Lk = L;
  p.H = H;
  p.Hkv = H;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.mode = vattn::attn::kSliding;   // keys = the query's own chunk
  p.F = chunk_tokens;
  p.chunk = 1;
  p.wb = 0;
  p.wf = 0;
  p.q_seg_len = chunk_tokens;
  p.q_tiles_per_seg = (chunk_tokens + 127) / 128;
  p.n_q_tiles = C * p.q_tiles_per_seg;
  p.hyb_S = wsS;
  p.hyb_z = wsz;
  p.hyb_fmap = fmap;
  p.hyb_coef = coef;
  p.lead = overlap;
  return launch_pair<128, vattn::attn::kRopeNone, true>(mq, mk, mv, mk, mv, mo, p, stream);
}
}  // namespace

extern "C" {

vattn_status vattn_hybrid_chunk(const void* q, const void* k, const void* v, void* o, float* S, float* z, int B,
                                int L, int H, int d, int chunk_tokens, float scale, void* workspace,
                                size_t workspace_bytes, vattn_stream stream) {
  return hybrid_impl(q, k, v, o, S, z, B, L, H, d, chunk_tokens, 0, scale, vattn::fmap::kFmapElu1, nullptr,
                     workspace, workspace_bytes, stream);
}

vattn_status vattn_hybrid_chunk_ex(const void* q, const void* k, const void* v, void* o, float* S, float* z, int B,
                                   int L, int H, int d, int chunk_tokens, int overlap_tokens, float scale,
                                   vattn_feature_map fmap, const float* coef, void* workspace,
                                   size_t workspace_bytes, vattn_stream stream) {
  return hybrid_impl(q, k, v, o, S, z, B, L, H, d, chunk_tokens, overlap_tokens, scale, static_cast<int>(fmap),
                     coef, workspace, workspace_bytes, stream);
}

// ------------------------------------------------- hybrid without workspace
// Scratch of vattn_hybrid_chunk_noalloc, for callers that cannot allocate
// device memory themselves.  The host code below must not hand the symbol
// itself to a kernel (in host code it names a host-side stand-in); it passes
// the device address that cudaGetSymbolAddress returns for the current
// device.
static __device__ __align__(256) unsigned char g_hybrid_noalloc_scratch[VATTN_HYBRID_NOALLOC_MAX_BYTES];

namespace {
void* g_noalloc_ptr[kMaxDevices];

// Device address of the static scratch on the current device, looked up
// once per device.
vattn_status noalloc_scratch(void** out) {
  int dev;
  if (vattn_status st = current_device(&dev)) return st;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_hybrid_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_hybrid_noalloc_scratch)");
    if (!p) return fail(VATTN_ERR_CUDA, "no device address for the static scratch");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return VATTN_OK;
}
}  // namespace

vattn_status vattn_hybrid_chunk_noalloc(const void* q, const void* k, const void* v, void* o, float* S,
                                        float* z, int B, int L, int H, int d, int chunk_tokens, float scale,
                                        vattn_stream stream) {
  const size_t need = vattn_hybrid_workspace_bytes(B, L, H, d, chunk_tokens);
  if (need == 0) return fail(VATTN_ERR_INVALID_ARG, "sizes must be >= 1");
  if (need > VATTN_HYBRID_NOALLOC_MAX_BYTES)
    return fail(VATTN_ERR_UNSUPPORTED,
                "this shape needs %zu bytes of scratch; the static scratch of "
                "vattn_hybrid_chunk_noalloc holds %zu (use vattn_hybrid_chunk with a workspace)",
                need, static_cast<size_t>(VATTN_HYBRID_NOALLOC_MAX_BYTES));
  void* scratch = nullptr;
  if (vattn_status st = noalloc_scratch(&scratch)) return st;
  return vattn_hybrid_chunk(q, k, v, o, S, z, B, L, H, d, chunk_tokens, scale, scratch,
                            VATTN_HYBRID_NOALLOC_MAX_BYTES, stream);
}

// ----------------------------------------------------------------- merge
vattn_status vattn_attention_merge(const void* o_parts, const float* lse_parts, int R, void* o, float* lse, int B,
                                   int L, int H, int d, vattn_stream stream) {
  if (!o_parts || !lse_parts || !o) return fail(VATTN_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(o_parts) || !aligned16(o) || (reinterpret_cast<uintptr_t>(lse_parts) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return fail(VATTN_ERR_INVALID_ARG, "o_parts and o must be 16-byte aligned, lse 4-byte aligned");
  if (R < 1 || R > vattn::merge::kMaxParts) return fail(VATTN_ERR_INVALID_ARG, "R=%d (1..%d)", R,
                                                         vattn::merge::kMaxParts);
  if (B < 1 || L < 1 || H < 1) return fail(VATTN_ERR_INVALID_ARG, "sizes must be >= 1");
  if (d < 8 || d % 8) return fail(VATTN_ERR_UNSUPPORTED, "head dim %d (multiple of 8 required)", d);
  vattn::merge::MergeParams mp{static_cast<const uint4*>(o_parts), lse_parts, static_cast<uint4*>(o), lse,
                               R, B, L, H, d};
  const long long n = static_cast<long long>(B) * L * H * (d / 8);
  int sms = 148, dev;
  if (current_device(&dev) == VATTN_OK) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long want = (n + 255) / 256;
  const int blocks = static_cast<int>(want < sms * 8LL ? want : sms * 8LL);
  vattn::merge::merge_kernel<<<blocks, 256, 0, stream>>>(mp);
  VATTN_CUDA(cudaGetLastError());
  return VATTN_OK;
}

// ------------------------------------------------------------- self-test
// Not part of the attention interface: checks the tensor-core operand
// layouts (see include/vattn_selftest.h).
vattn_status vattn_selftest_umma(int variant, const void* a, const void* b, float* out, vattn_stream stream) {
  if (variant < 0 || variant > 3) return fail(VATTN_ERR_INVALID_ARG, "variant %d", variant);
  if (!a || !b || !out || !aligned16(a) || !aligned16(b) || !aligned16(out))
    return fail(VATTN_ERR_INVALID_ARG, "pointers must be non-NULL and 16-byte aligned");
  uint32_t* status;
  if (vattn_status st = status_ptr(&status)) return st;
  CUtensorMap ma, mb;
  if (vattn_status st = make_map(&ma, a, 128, 1, 128, 1, 128)) return st;
  if (vattn_status st = make_map(&mb, b, 128, 1, 128, 1, 128)) return st;
  static uint64_t done[1];
  const int smem = 65536 + 64 + 1024;
  if (vattn_status st = ensure_smem(vattn::selftest::umma_kernel, smem, done)) return st;
  vattn::selftest::umma_kernel<<<1, 128, smem, stream>>>(ma, mb, out, variant, status);
  VATTN_CUDA(cudaGetLastError());
  return VATTN_OK;
}

// Not part of the attention interface: drives a bounded wait to its limit
// to check the timeout reporting path (see include/vattn_selftest.h).
vattn_status vattn_selftest_wait_timeout(uint32_t limit_us, vattn_stream stream) {
  if (limit_us == 0 || limit_us > 2000000) return fail(VATTN_ERR_INVALID_ARG, "limit_us must be 1..2000000");
  uint32_t* status;
  if (vattn_status st = status_ptr(&status)) return st;
  vattn::selftest::wait_timeout_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(limit_us) * 1000ull, status);
  VATTN_CUDA(cudaGetLastError());
  return VATTN_OK;
}

// Not part of the attention interface: the two-tile attention kernel with
// one softmax arrival withheld and a short wait bound (see
// include/vattn_selftest.h).
vattn_status vattn_selftest_attention_timeout(const void* q, const void* k, const void* v, void* o, int L, int H,
                                              int d, uint32_t limit_us, vattn_stream stream) {
  if (limit_us == 0 || limit_us > 2000000) return fail(VATTN_ERR_INVALID_ARG, "limit_us must be 1..2000000");
  if (L < 2 * vattn::attn::kTileN)
    return fail(VATTN_ERR_INVALID_ARG, "L=%d: at least two key tiles are needed to withhold sub-tile 1", L);
  return attention_impl(q, k, v, o, nullptr, 1, L, L, H, H, d, d == 64 ? 0.125f : 0.08838834764831845f,
                        VATTN_FULL, 0, 1, 0, 0, 0, 0, nullptr, nullptr, nullptr, 0, stream,
                        static_cast<uint64_t>(limit_us) * 1000ull, 1);
}

// Not part of the attention interface: the softmax's exponentials element
// by element (see include/vattn_selftest.h).
vattn_status vattn_selftest_ex2(int variant, const float* x, float* y, int n, vattn_stream stream) {
  if (variant < 0 || variant > 2) return fail(VATTN_ERR_INVALID_ARG, "variant %d", variant);
  if (!x || !y || n < 1 || (variant == 1 && (n & 1)))
    return fail(VATTN_ERR_INVALID_ARG, "x, y non-NULL, n >= 1 (even for variant 1)");
  int blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  vattn::selftest::ex2_kernel<<<blocks, 256, 0, stream>>>(x, y, n, variant);
  VATTN_CUDA(cudaGetLastError());
  return VATTN_OK;
}

}  // extern "C"
