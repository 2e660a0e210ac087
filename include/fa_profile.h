/*
 * fa_profile.h - optional timing hook of libfa.
 *
 * fa_bwd runs three kernels in order on its stream: a preprocess (row sums
 * D and zeroing of the dQ accumulator), the main backward kernel, and a
 * postprocess (dQ conversion). To time the main kernel alone with CUDA
 * events on the launching stream, a caller may hand the library two events
 * (cudaEvent_t, created by the caller on the current device); fa_bwd then
 * records `after_pre` right after the preprocess launch and `after_main`
 * right after the main launch. Passing NULL for both turns the hook off.
 * The setting is process-wide and applies to later fa_bwd calls from any
 * thread; it is meant for benchmarks, not for concurrent production use.
 *
 * fa_decode runs two kernels: the split decode kernel and the merge of its
 * partial results. fa_profile_set_decode_event hands it one event that it
 * records right after the decode kernel's launch (NULL turns it off), with
 * the same scope as above.
 */
#ifndef FA_PROFILE_H_
#define FA_PROFILE_H_

#ifdef __cplusplus
extern "C" {
#endif

void fa_profile_set_bwd_events(void* after_pre, void* after_main);
void fa_profile_set_decode_event(void* after_main);

#ifdef __cplusplus
}
#endif

#endif /* FA_PROFILE_H_ */
