/*
 * Tensor-core layout self-test of libvattn.  The pages have no counterpart:
 * this entry point exists to check, on the device, the operand layouts the
 * attention and state kernels rely on (TMA 128-byte swizzle, shared-memory
 * matrix descriptors, TMEM operand packing, instruction descriptors).
 *
 * One 128x128x128 product, bf16 inputs, fp32 result, on `stream`:
 *   variant 0: out[m][n] = sum_k a[m][k] * b[n][k]      (a, b K-major)
 *   variant 1: out[m][n] = sum_k a[m][k] * b[k][n]      (a staged in TMEM)
 *   variant 2: out[m][n] = sum_k a[m][k] * b[k][n]      (a K-major, b MN-major)
 *   variant 3: out[m][n] = sum_k a[k][m] * b[k][n]      (both MN-major)
 * a, b: device bf16 [128][128] row-major; out: device fp32 [128][128].
 * All pointers 16-byte aligned.  Returns VATTN_ERR_INVALID_ARG on a bad
 * variant or pointer; errors of the launch as VATTN_ERR_CUDA.
 */
#ifndef VATTN_SELFTEST_H_
#define VATTN_SELFTEST_H_
#include "vattn.h"
#ifdef __cplusplus
extern "C" {
#endif
vattn_status vattn_selftest_umma(int variant, const void* a, const void* b, float* out, vattn_stream stream);
#ifdef __cplusplus
}
#endif
#endif
