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

/*
 * The same check inside the two-tile attention kernel (no counterpart in the
 * pages).  One full-attention call without RoPE (B = 1, Hkv = H, scale
 * 1/sqrt(d)) on q, k, v, o bf16 [1][L][H][d] (device, 16-byte aligned),
 * L >= 256, with every wait bounded by limit_us microseconds (1..2000000)
 * instead of two seconds, and with the first softmax warp of each CTA's
 * first query tile withholding its arrival for score sub-tile 1.  That
 * tile's MMA issuer waits for it until the bound runs out, raises the CTA's
 * abort and records a code in the status word; every other role leaves its
 * loop, waits (bounded) for its copies and MMAs in flight, the CTA frees its
 * TMEM and returns.  The following vattn_check() reports VATTN_ERR_TIMEOUT;
 * o is left partly unwritten.  Nothing faults, traps or hangs.
 */
vattn_status vattn_selftest_attention_timeout(const void* q, const void* k, const void* v, void* o, int L,
                                              int H, int d, uint32_t limit_us, vattn_stream stream);

/*
 * The softmax exponentials, element by element (no counterpart in the
 * pages; checks the exp2 the kernels use):
 *   variant 0: y[i] = 2^x[i] by the FMA-pipe polynomial (Cody-Waite
 *              reduction, degree-3 minimax, relative error < 7.6e-5 for
 *              x >= -125; arguments below -125 give a value in
 *              [0, 2^-124]);
 *   variant 1: the same on pairs (x[2i], x[2i+1]) in packed fp32x2 form
 *              (n even);
 *   variant 2: y[i] = ex2.approx.ftz(x[i]) (MUFU).
 * x, y: device fp32 [n].
 */
vattn_status vattn_selftest_ex2(int variant, const float* x, float* y, int n, vattn_stream stream);
#ifdef __cplusplus
}
#endif
#endif
