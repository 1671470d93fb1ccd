// Rolling KV cache append (FlashDecoder "Streaming with Rolling KV Cache",
// Sec. 3.3): frame f's K and V are copied bit for bit into ring slot
// f mod capacity and the slot's frame id is set.  Pure HBM copy with
// 16-byte vectors, both tensors' loads in flight before the stores.
#pragma once
#include "common.cuh"
#include "grid_dep.cuh"

namespace vattn {
namespace kv {

// Each thread moves kUnroll 16-byte vectors of K and of V per step, all
// loads issued before any store (8 loads in flight per thread).
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(256) append_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                     uint4* __restrict__ kr, uint4* __restrict__ vr,
                                                     long long n16, int32_t* ids, int slot, int frame) {
  pdl::grid_dep_wait();
  pdl::grid_dep_launch();
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (long long base = tid; base < n16; base += stride * kUnroll) {
    uint4 ka[kUnroll], va[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long i = base + u * stride;
      if (i < n16) {
        ka[u] = __ldg(k + i);
        va[u] = __ldg(v + i);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long i = base + u * stride;
      if (i < n16) {
        kr[i] = ka[u];
        vr[i] = va[u];
      }
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) ids[slot] = frame;
}

// Appends to a cache with a rotated-key ring use rope::rotate_rows_kernel
// with raw copies (one pass: raw K, raw V and rotated K).

}  // namespace kv
}  // namespace vattn
