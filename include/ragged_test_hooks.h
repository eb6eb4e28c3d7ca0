/*
 * ragged_test_hooks.h - test-only entry point of libragged_testhooks.so.
 *
 * That library is built from the same sources as libragged.so with
 * RAGGED_TEST_HOOKS defined; the product library does not contain this
 * function or the switches it sets.  The pages have no counterpart: it exists
 * so that a test can make the tcgen05 kernels' bounded waits expire on a GPU
 * without any fault, and check what the failure path leaves behind.
 */
#ifndef RAGGED_TEST_HOOKS_H
#define RAGGED_TEST_HOOKS_H

#include "ragged.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * ragged_test_set_hooks - set the test switches of the current device
 * (synchronous copies to device globals; call between launches).
 *   hook        0 = none; 1 = the persistent tcgen05 kernel's load warp issues
 *               no load, so the MMA and softmax waits on its tiles expire;
 *               2 = the per-tile tcgen05 kernel's MMA thread issues no
 *               product, so the softmax waits on its scores expire.
 *   spin_limit  polls per bounded mbarrier wait (the product value is 2^22);
 *               must be positive.
 * A kernel whose wait expires sets RAGGED_DEV_TIMEOUT in the status word,
 * writes no output row, frees its TMEM and returns.
 * Returns RAGGED_ERR_INVALID_ARG for an unknown hook or a zero limit.
 */
RAGGED_API ragged_status ragged_test_set_hooks(int32_t hook, uint32_t spin_limit);

#ifdef __cplusplus
}
#endif

#endif /* RAGGED_TEST_HOOKS_H */
