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

#include "fa.h"

#ifdef __cplusplus
extern "C" {
#endif

void fa_test_set_fault(int code);

/*
 * Evaluates, for n device floats x (each <= 0), the forward kernel's
 * FMA-pipe exponential into y_poly and the exponential unit's ex2.approx
 * into y_ex2 (device buffers of n floats), asynchronously on `stream`.
 * Returns FA_OK, FA_ERR_INVALID_ARGUMENT (null pointer, n < 0) or
 * FA_ERR_CUDA.
 */
int fa_test_exp2(const float* x, float* y_poly, float* y_ex2, int n, void* stream);

/*
 * Evaluates, for n device floats x (each <= 0), the forward kernel's
 * float32-accurate FMA-pipe exponential (the one it uses for the O rescale
 * factor) into y (n device floats), asynchronously on `stream`. Returns
 * FA_OK, FA_ERR_INVALID_ARGUMENT (null pointer, n < 0) or FA_ERR_CUDA.
 */
int fa_test_exp2_accurate(const float* x, float* y, int n, void* stream);

/*
 * Host only (no device call): the stream-K work partition fa_decode would
 * use for this shape with num_ctas CTAs, as eight integers in out[0..7]:
 * W (key tiles over all units), T (128-key tiles per unit), G (CTAs = runs),
 * MS (most units one run may touch), R (query rows per KV head), rho (row
 * replication over the 128 tensor-memory lanes), rv (stored rows per copy),
 * n_chunks (row chunks per KV head). A unit is (batch, KV head, row chunk);
 * run c covers tiles [c*W/G, (c+1)*W/G) in unit order. Returns FA_OK,
 * FA_ERR_INVALID_ARGUMENT (null out, num_ctas < 1, bad shape) or
 * FA_ERR_UNSUPPORTED, as fa_decode would for the shape.
 */
int fa_test_decode_plan(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_ctas, long long* out);

#ifdef __cplusplus
}
#endif

#endif /* FA_TEST_H_ */
