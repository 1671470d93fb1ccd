// Tensor-core operand-layout self-test: one 128x128x128 bf16 product per
// launch through exactly the TMA maps, shared-memory descriptors, TMEM
// packing and instruction descriptors that the attention and state kernels
// use.  The host compares the fp32 result with a plain product.
//   variant 0: D = A B^T, A [m][k], B [n][k] both K-major (S = Q K^T form)
//   variant 1: D = A B,   A [m][k] staged in TMEM, B [k][n] MN-major (O += P V)
//   variant 2: D = A B,   A [m][k] K-major smem, B [k][n] MN-major
//   variant 3: D = A^T B, A [k][m] and B [k][n] both MN-major (state delta)
#pragma once
#include "common.cuh"

namespace vattn {
namespace selftest {

using namespace sm100;

__global__ void __launch_bounds__(128, 1)
    umma_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, float* out,
                int variant, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sA = smem_addr(smem), sB = sA + 32768, bar = sA + 65536, bar2 = bar + 8;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + 65536 + 16);
  volatile uint32_t* tmem_slot = misc;
  volatile uint32_t* abort_flag = misc + 1;
  Abort ab{abort_flag, status};
  const int warp = threadIdx.x >> 5, r = threadIdx.x;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_init(bar2, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_addr(const_cast<uint32_t*>(tmem_slot)), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar, 65536);
    for (int blk = 0; blk < 2; ++blk) {
      tma_load_4d(sA + blk * 16384, &tmA, bar, blk * 64, 0, 0, 0);
      tma_load_4d(sB + blk * 16384, &tmB, bar, blk * 64, 0, 0, 0);
    }
  }
  bool ok = mbar_wait(bar, 0, ab, kStatusTimeoutAux);
  if (variant == 1) {
    // row r of A -> TMEM lane r, columns [128, 192): two bf16 per column
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16) + 128;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t pk[32];
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        const uint4 v = lds128(sA + half * 16384 + sw128_offset(r, c8));
        pk[c8 * 4 + 0] = v.x;
        pk[c8 * 4 + 1] = v.y;
        pk[c8 * 4 + 2] = v.z;
        pk[c8 * 4 + 3] = v.w;
      }
      tmem_st32(trow + half * 32, pk);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && ok) {
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t kmaj = (kk >> 2) * 16384 + (kk & 3) * 32;   // K-major step
      const uint32_t mnmaj = kk * 2048;                           // MN-major step
      if (variant == 0)
        umma_ss(tmem, sdesc_sw128(sA + kmaj, 16, 1024), sdesc_sw128(sB + kmaj, 16, 1024),
                idesc_bf16_f32(128, 128, false, false), kk > 0);
      else if (variant == 1)
        umma_ts(tmem, tmem + 128 + kk * 8, sdesc_sw128(sB + mnmaj, 16384, 1024),
                idesc_bf16_f32(128, 128, false, true), kk > 0);
      else if (variant == 2)
        umma_ss(tmem, sdesc_sw128(sA + kmaj, 16, 1024), sdesc_sw128(sB + mnmaj, 16384, 1024),
                idesc_bf16_f32(128, 128, false, true), kk > 0);
      else
        umma_ss(tmem, sdesc_sw128(sA + mnmaj, 16384, 1024), sdesc_sw128(sB + mnmaj, 16384, 1024),
                idesc_bf16_f32(128, 128, true, true), kk > 0);
    }
    umma_commit(bar2);
  }
  __syncwarp();
  ok = ok && mbar_wait(bar2, 0, ab, kStatusTimeoutAux);
  tc_fence_after();
  if (ok) {
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    for (int q = 0; q < 4; ++q) {
      uint32_t v[32];
      tmem_ld32(trow + q * 32, v);
      tmem_ld_wait();
      for (int e = 0; e < 32; ++e) out[r * 128 + q * 32 + e] = __uint_as_float(v[e]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// A wait that runs out: thread 0 arms an mbarrier that nothing ever
// arrives on; every thread's bounded wait gives up after limit_ns, the
// abort is raised (status word set) and the kernel returns normally.
__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(uint64_t limit_ns, uint32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  const uint32_t b = smem_addr(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  Abort ab{&abort_flag, status};
  mbar_wait_limit(b, 0, ab, kStatusTimeoutAux, limit_ns);
}

// The exponentials of the softmax, element by element:
//   variant 0: y = ex2_poly(x)       (FMA-pipe polynomial)
//   variant 1: (y[2i], y[2i+1]) = ex2_poly2(x[2i], x[2i+1])   (packed form; n even)
//   variant 2: y = ex2_approx(x)     (MUFU ex2.approx.ftz)
__global__ void ex2_kernel(const float* __restrict__ x, float* __restrict__ y, int n, int variant) {
  const int stride = gridDim.x * blockDim.x;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    if (variant == 0) {
      y[i] = ex2_poly(x[i]);
    } else if (variant == 1) {
      if (2 * i + 1 < n) ex2_poly2(y[2 * i], y[2 * i + 1], x[2 * i], x[2 * i + 1]);
    } else {
      y[i] = ex2_approx(x[i]);
    }
  }
}

}  // namespace selftest
}  // namespace vattn
