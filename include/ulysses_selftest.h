/*
 * ulysses_selftest.h -- test hooks, exported by libulysses_selftest.so (a
 * library of its own, built beside libulysses.so; not part of the layer).
 *
 * These entry points run single device helpers of the kernels on their own,
 * so tests can compare them with reference values.
 */
#ifndef ULYSSES_SELFTEST_H_
#define ULYSSES_SELFTEST_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * y[i] = 2^x[i] computed with the FMA-pipe exponential the attention softmax
 * uses for part of its probabilities (round-to-nearest range reduction plus a
 * degree-3 minimax polynomial; maximum relative error 7.5e-5 for
 * -125 <= x <= 64; inputs below -125 return 2^-125).  x and y are device
 * arrays of n floats, 4-byte aligned; asynchronous on `stream`.
 * Returns 0, 1 for a bad argument, 6 for a CUDA launch error.
 */
int ulysses_selftest_exp2_poly(const float* x, float* y, int64_t n, void* stream);

/*
 * Failure-path check of the kernels' bounded waits: one CTA waits on an
 * mbarrier phase that nothing completes, first with the single-thread wait,
 * then with the warp-collective wait, each limited to limit_us microseconds
 * (1 .. 1,000,000).  Each wait gives up, sets bit 1 (wait timeout) of
 * *dev_err, and the kernel also sets 0x100 / 0x200 for the two waits and
 * returns; the context stays usable.  dev_err is a caller-owned device word.
 * Returns 0, 1 for a bad argument, 6 for a CUDA launch error.
 */
int ulysses_selftest_wait_timeout(unsigned int* dev_err, int64_t limit_us, void* stream);

/*
 * The range check of the bounds-checked build (-DULYSSES_DEBUG), forced on
 * in this hook: offsets 0, -8 and 96 of 8 elements against an extent of 100.
 * The first is inside and sets 0x10 in *dev_err; the other two are refused,
 * each setting bit 4 (out of bounds) and 0x20 / 0x40 respectively.  No memory
 * but *dev_err is touched.  Returns 0, 1 for a bad argument, 6 for a CUDA
 * launch error.
 */
int ulysses_selftest_bounds_check(unsigned int* dev_err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ULYSSES_SELFTEST_H_ */
