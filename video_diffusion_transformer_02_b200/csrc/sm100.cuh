// sm_100a device primitives written as inline PTX: shared-memory mbarriers
// with time-bounded waits, TMA tiled loads (no multicast), and the tcgen05
// tensor-core path (TMEM allocation, MMA issue, commit, TMEM <-> register
// moves).  Everything here is a thin, named wrapper around one PTX
// instruction; the kernels compose them.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace vattn {
namespace sm100 {

// ------------------------------------------------------------------ status
// A kernel that gives up on a wait records a code in the library's device
// status word and returns; the host reads it through vattn_check().
enum : uint32_t {
  kStatusOk = 0,
  kStatusTimeoutProducer = 1,
  kStatusTimeoutMma = 2,
  kStatusTimeoutSoftmax = 3,
  kStatusTimeoutAux = 4,
  kStatusSmemAlign = 5,   // dynamic shared memory not 1024-byte aligned
  kStatusTimeoutStep = 6, // a streaming step's attention CTA waited too long for the frame's keys
};
// Wall-clock bound of a single wait (nanoseconds of %globaltimer).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// --------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
// Make initialised barriers visible to the async proxy (TMA, tcgen05).
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Shared abort flag of a CTA plus the global status word.  A role that times
// out sets both; every other role polls the shared flag while it waits and
// leaves its loop, so the CTA reaches its teardown and returns.
struct Abort {
  volatile uint32_t* flag;   // shared memory
  uint32_t* status;          // global memory (may be null)
  uint64_t limit_ns = kWaitLimitNs;   // bound of each wait
};

__device__ __forceinline__ void raise_abort(const Abort& ab, uint32_t code) {
  *ab.flag = 1u;
  if (ab.status) atomicCAS(ab.status, 0u, code);
}

// As mbar_wait below, with an explicit time limit (ns) and no back-off.
__device__ __forceinline__ bool mbar_wait_limit(uint32_t bar, uint32_t parity, const Abort& ab, uint32_t code,
                                                uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*ab.flag) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        raise_abort(ab, code);
        return false;
      }
    }
  }
}

// Wait until phase `parity` of `bar` has completed.  Returns false if the
// CTA aborted or the wait exceeded ab.limit_ns (then the abort is raised
// with `code`).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const Abort& ab, uint32_t code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*ab.flag) return false;
      if (global_timer_ns() - t0 > ab.limit_ns) {
        raise_abort(ab, code);
        return false;
      }
    }
  }
}

// Poll `bar` until phase `parity` completes or limit_ns passes, without
// raising anything: the teardown drains of a CTA (loads and MMAs already in
// flight) that must end whether or not the CTA aborted.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity) && global_timer_ns() - t0 < limit_ns) {
  }
}

// ------------------------------------------------- cross-CTA signalling
// Generic-proxy global writes made visible to later async-proxy (TMA) reads,
// by this thread or (after a release/acquire pair) by another CTA.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Wait until *counter >= target (another CTA of the same launch counts up
// with a release), bounded like mbar_wait.  Returns false on abort or when
// ab.limit_ns passes (the abort is then raised with `code`).
__device__ __forceinline__ bool wait_counter(const uint32_t* counter, uint32_t target, const Abort& ab,
                                             uint32_t code) {
  if (ld_acquire_gpu(counter) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(64);
    if (ld_acquire_gpu(counter) >= target) return true;
    if ((it & 15u) == 0u) {
      if (*ab.flag) return false;
      if (global_timer_ns() - t0 > ab.limit_ns) {
        raise_abort(ab, code);
        return false;
      }
    }
  }
}

// -------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 4-D tiled bulk tensor load into shared memory, completing transaction
// bytes on `bar`.  c0 is the innermost coordinate (elements).
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* m, uint32_t bar, int c0,
                                            int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

// 4-D tiled bulk tensor store from shared memory (one bulk group; the
// coordinates must not be negative).
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* m, uint32_t src, int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
// Plain (untiled) bulk copy global -> shared, completing transaction bytes
// on `bar` (both addresses 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk store of this thread has finished reading
// shared memory.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// Named barrier ID over COUNT threads that also ANDs a predicate across them.
template <uint32_t ID, uint32_t COUNT>
__device__ __forceinline__ bool bar_and(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "n"(ID), "n"(COUNT)
      : "memory");
  return r != 0;
}

// Order generic-proxy shared-memory writes before later async-proxy reads
// (tcgen05.mma operands written by threads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// TMEM address: lane in bits [31:16], column in bits [15:0].
__device__ __forceinline__ uint32_t tmem_lane_col(uint32_t base, uint32_t lane, uint32_t col) {
  return base + (lane << 16) + col;
}

#define VATTN_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                    "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define VATTN_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
                    "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// Warp-collective load of 32 consecutive 32-bit columns of this warp's 32
// TMEM lanes: thread i receives lane (base lane + i), columns col..col+31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : VATTN_R8(0), VATTN_R8(8), VATTN_R8(16), VATTN_R8(24)
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
#define VATTN_RW8(i) "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), \
                     "+r"(r[i + 4]), "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7])
// Wait for this thread's TMEM loads and tie the destination registers to the
// wait, so no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_ld_wait_dep(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : VATTN_RW8(0), VATTN_RW8(8), VATTN_RW8(16), VATTN_RW8(24)::"memory");
}
__device__ __forceinline__ void tmem_ld_wait_dep2(uint32_t (&r)[32], uint32_t (&s)[32]) {
  tmem_ld_wait_dep(r);
  asm volatile("" : "+r"(s[0]), "+r"(s[1]), "+r"(s[2]), "+r"(s[3]), "+r"(s[4]), "+r"(s[5]), "+r"(s[6]),
               "+r"(s[7]), "+r"(s[8]), "+r"(s[9]), "+r"(s[10]), "+r"(s[11]), "+r"(s[12]), "+r"(s[13]),
               "+r"(s[14]), "+r"(s[15]), "+r"(s[16]), "+r"(s[17]), "+r"(s[18]), "+r"(s[19]), "+r"(s[20]),
               "+r"(s[21]), "+r"(s[22]), "+r"(s[23]), "+r"(s[24]), "+r"(s[25]), "+r"(s[26]), "+r"(s[27]),
               "+r"(s[28]), "+r"(s[29]), "+r"(s[30]), "+r"(s[31]));
}
// Warp-collective store of 32 consecutive columns (same lane mapping).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      VATTN_W8(0), VATTN_W8(8), VATTN_W8(16), VATTN_W8(24)
      : "memory");
}
// Warp-collective store of 16 consecutive columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      VATTN_W8(0), VATTN_W8(8)
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------- UMMA
// Shared-memory matrix descriptor for a 128-byte-swizzled operand tile
// (sm_100 layout: start>>4 in [0,14), leading byte offset>>4 in [16,30),
// stride byte offset>>4 in [32,46), version 1 in [46,48), swizzle mode 2
// (128B) in [61,64)).  K-major tiles: rows of 128 B, 8-row groups `sbo`
// apart.  MN-major tiles: 64-element atoms along MN `lbo` apart, 8-row K
// groups `sbo` apart.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor of kind::f16 with bf16 A/B and fp32 D:
// D format [4,6)=1 (f32), A format [7,10)=1 (bf16), B format [10,13)=1,
// A major [15], B major [16] (1 = MN-major), N>>3 in [17,23), M>>4 in [24,29).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// D(tmem) (+)= A(smem) * B(smem)
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D(tmem) (+)= A(tmem) * B(smem); A is K-major, two 16-bit values per column.
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when every tcgen05 operation this thread issued so
// far has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// Per-warpgroup register budget (all four warps of a warpgroup execute the
// same instruction).  The launch reserves threads x launch registers; the
// decreases must free at least what the increases take.
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// --------------------------------------------------- packed fp32 / 3-input
// d = a * b + c on two lanes at once (fma.rn.f32x2).
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                      float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
// (d0, d1) += (a0, a1) with add.rn.f32x2.
__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1) {
  asm("{\n\t.reg .b64 ra, rd;\n\t"
      "mov.b64 rd, {%0, %1};\n\tmov.b64 ra, {%2, %3};\n\t"
      "add.rn.f32x2 rd, rd, ra;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1));
}
// max of three fp32 values (one instruction).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// ------------------------------------------------------------ conversions
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float bf16lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// 2^x on the FMA pipe (offloads the MUFU unit): Cody-Waite reduction
// x = j + f with j = round(x) (via the 1.5*2^23 shifter), f in [-0.5, 0.5],
// degree-3 minimax polynomial for 2^f (max relative error 7.5e-5 for
// x >= -125, below 7.6e-5 with fp32 evaluation; the coefficients come from
// fit_exp2_poly.py), then j added to the exponent field.  Arguments below
// -125 return a value in [0, 2^-124] (the softmax's probabilities there are
// zero to every digit that counts).
__device__ __forceinline__ float ex2_poly(float x) {
  x = fmaxf(x, -126.0f);
  const float t = x + 12582912.0f;
  const float f = x - (t - 12582912.0f);
  float p = fmaf(5.517166853e-02f, f, 2.426111251e-01f);
  p = fmaf(p, f, 6.932609677e-01f);
  p = fmaf(p, f, 9.999280572e-01f);
  // t's low mantissa bits hold j (two's complement); shifted by 23 they land
  // in the exponent field (unsigned arithmetic: the wrap is defined)
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

// Two lanes of ex2_poly with packed fp32x2 arithmetic: the same reduction,
// polynomial and exponent insertion (j * 2^23 added onto the polynomial's
// bits in unsigned 32-bit arithmetic).
__device__ __forceinline__ void ex2_poly2(float& y0, float& y1, float x0, float x1) {
  x0 = fmaxf(x0, -126.0f);
  x1 = fmaxf(x1, -126.0f);
  float t0, t1, j0, j1, f0, f1, p0, p1;
  ffma2(t0, t1, x0, x1, 1.0f, 1.0f, 12582912.0f, 12582912.0f);     // x + 1.5*2^23
  ffma2(j0, j1, t0, t1, 1.0f, 1.0f, -12582912.0f, -12582912.0f);   // round(x)
  ffma2(f0, f1, j0, j1, -1.0f, -1.0f, x0, x1);                     // x - round(x)
  ffma2(p0, p1, f0, f1, 5.517166853e-02f, 5.517166853e-02f, 2.426111251e-01f, 2.426111251e-01f);
  ffma2(p0, p1, p0, p1, f0, f1, 6.932609677e-01f, 6.932609677e-01f);
  ffma2(p0, p1, p0, p1, f0, f1, 9.999280572e-01f, 9.999280572e-01f);
  y0 = __uint_as_float((__float_as_uint(t0) << 23) + __float_as_uint(p0));
  y1 = __uint_as_float((__float_as_uint(t1) << 23) + __float_as_uint(p1));
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// Byte offset of 16-byte chunk `c` (0..7) of row `r` inside a 128B-swizzled
// [rows][64 x 16-bit] block (TMA SWIZZLE_128B pattern, 1024-byte aligned).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t r, uint32_t c) {
  return r * 128u + ((c ^ (r & 7u)) << 4);
}

}  // namespace sm100
}  // namespace vattn
