/*
 * fa_test.h - test hooks of libfa (not for production use).
 *
 * The watchdog test needs a kernel whose wait can never be satisfied. This
 * hook makes the forward producer skip the load of the first K tile, so the
 * MMA thread's first wait runs out, the CTA aborts cleanly (it drains its
 * copies and frees its tensor memory) and fa_check_device_error returns
 * FA_ERR_TIMEOUT. No memory fault, trap or endless loop is involved.
 *
 *   code 0: normal operation (default)
 *   code 1: forward producer never loads the first K tile
 *
 * Applies to launches made after the call, from any thread.
 */
#ifndef FA_TEST_H_
#define FA_TEST_H_

#ifdef __cplusplus
extern "C" {
#endif

void fa_test_set_fault(int code);

#ifdef __cplusplus
}
#endif

#endif /* FA_TEST_H_ */
