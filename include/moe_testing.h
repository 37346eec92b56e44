/*
 * fp8_moe — entry points of the wait-test build only (libfp8moe_waittest.so, compiled with
 * -DMOE_WAIT_TEST by fp8_moe_layer_b200/build.py). That build is the library with two changes
 * for testing the device-timeout path without faulting the GPU: every bounded wait inside a
 * kernel gives up after 2 ms instead of about 1 s, and the switch below. The production library
 * (libfp8moe.so) exports none of these symbols. The pages describing the method have no
 * counterpart to this header: it exists so that the status path of include/moe.h
 * (MOE_ERR_DEVICE_TIMEOUT, moe_device_status) can be exercised.
 */
#ifndef FP8_MOE_TESTING_H
#define FP8_MOE_TESTING_H

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

#ifdef __cplusplus
}
#endif

#endif /* FP8_MOE_TESTING_H */
