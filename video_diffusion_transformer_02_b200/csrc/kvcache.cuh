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

}  // namespace kv
}  // namespace vattn
