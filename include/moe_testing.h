/*
 * fp8_moe — entry points of two test and profiling builds of the library (fp8_moe_layer_b200/
 * build.py), which the production library (libfp8moe.so) does not export. The pages describing
 * the method have no counterpart to this header.
 *  - the wait-test build (libfp8moe_waittest.so, -DMOE_WAIT_TEST): every bounded wait inside a
 *    kernel gives up after 2 ms instead of about 1 s, and moe_test_withhold_gemm_commit below,
 *    so that the status path of include/moe.h (MOE_ERR_DEVICE_TIMEOUT, moe_device_status) can be
 *    exercised without faulting the GPU;
 *  - the role-counter build (libfp8moe_roles.so, -DMOE_ROLE_COUNTERS): the grouped GEMMs add up,
 *    per CTA, the cycles each warp role spends waiting (moe_role_counters_* below).
 */
#ifndef FP8_MOE_TESTING_H
#define FP8_MOE_TESTING_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Host only. When `on` is non-zero, every CTA of the gate/up GEMM launched by the following
 * moe_forward / moe_grouped_ffn_fp8 calls issues its first tile's MMAs but withholds the signal
 * that the tile's accumulators are ready. The epilogue warps' bounded wait for that signal then
 * expires (2 ms): they record MOE_ERR_DEVICE_TIMEOUT with where-code 4 (gate/up GEMM) in the
 * workspace status word, and every warp of the kernel unwinds through its own bounded waits,
 * lets its in-flight copies and MMAs land, frees its tensor memory and returns. The call itself
 * still returns MOE_OK (the launches succeeded); moe_device_status reports the timeout. Pass 0
 * to restore normal operation. Not thread-safe: set it while no other host thread calls the
 * library. */
void moe_test_withhold_gemm_commit(int on);

/* Role-counter build only. Copies the counters to `out` (host, 3 * 256 * 8 uint64): for GEMM mode
 * m (0 gate/up with the SwiGLU epilogue, 1 down, 2 gate/up K-split partials) and CTA c, entries
 * [(m * 256 + c) * 8 + i]: i = 0 cycles the TMA producer waited for a free stage, 1 cycles the MMA
 * issuer waited for a free accumulator, 2 cycles it waited for a stage's data, 3 K blocks it
 * issued, 4 cycles the first epilogue warp waited for an accumulator, 5 cycles from the kernel's
 * set-up to its end, 6 tiles. Returns 0, or MOE_ERR_CUDA if the copy fails. Synchronous. */
int moe_role_counters_read(uint64_t* out);

/* Role-counter build only. Zeroes the counters (synchronous). Returns 0 or MOE_ERR_CUDA. */
int moe_role_counters_reset(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8_MOE_TESTING_H */
