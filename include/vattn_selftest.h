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

/*
 * Timeout reporting check (no counterpart in the pages).  Launches one warp
 * that waits, with a bound of limit_us microseconds (1..2000000), on a
 * shared-memory barrier that nothing ever arrives on.  The wait gives up,
 * records a code in the device status word and the kernel returns normally:
 * the following vattn_check() reports VATTN_ERR_TIMEOUT and clears the word,
 * and the context stays usable.  Nothing faults, traps or hangs.
 */
vattn_status vattn_selftest_wait_timeout(uint32_t limit_us, vattn_stream stream);
#ifdef __cplusplus
}
#endif
#endif
