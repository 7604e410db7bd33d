/*
 * fp8gemm_testing.h -- test hook of libfp8gemm.so.  Not for production use.
 *
 * Every pipeline wait inside the GEMM kernels is bounded: a wait that does
 * not complete within its limit (1 s by default) records FP8G_DEVERR_TIMEOUT
 * in the device error word (fp8g_get_device_error), stops every role of the
 * CTA, drains the copies and MMAs the CTA has in flight, frees its tensor
 * memory and returns.  The pages have no counterpart; this hook exists so
 * that a test can make such a wait run out on a healthy GPU, without a fault
 * and without an unbounded wait.
 */
#ifndef FP8GEMM_TESTING_H
#define FP8GEMM_TESTING_H

#ifdef __cplusplus
extern "C" {
#endif

/*
 * From the next call on, the TMA producers of the single-CTA kernel variants
 * skip the loads of pipeline iteration `iteration` (counted per CTA from 0),
 * so the stage that iteration fills never completes, and every wait of those
 * kernels gives up after `wait_limit_us` microseconds (100 .. 1000000)
 * instead of 1 s.  The calls that hit the withheld stage therefore record
 * FP8G_DEVERR_TIMEOUT and leave their outputs undefined.  CTA-pair variants
 * and fp8_gemm_nt_no_alloc are not affected.  A negative `iteration` turns
 * the hook off and restores the 1 s limit.  Process-wide.
 * Returns FP8G_OK, or FP8G_ERR_INVALID_ARG for a limit out of range.
 */
int fp8g_testing_withhold_stage(int iteration, unsigned wait_limit_us);

#ifdef __cplusplus
}
#endif

#endif /* FP8GEMM_TESTING_H */
