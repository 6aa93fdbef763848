/*
 * kvq_testing.h -- test hooks of libkvq. Not part of the method: they exist so that the
 * tests can make a kernel's bounded wait give up without faulting or hanging the GPU.
 */
#ifndef KVQ_TESTING_H_
#define KVQ_TESTING_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * kvq_testing_set_fused_wait -- for the calling thread's later quantize and append calls
 *   that compute the amax in one launch: each quantize tile waits for extra_a_tiles amax
 *   tiles more than the launch has (arrivals that never come), and gives up after
 *   wait_ns nanoseconds (0: the library's 2 s). (0, 0) restores normal operation. With
 *   extra_a_tiles > 0 every such call times out: its outputs stay unwritten, its amax
 *   becomes NaN and kvq_device_status() returns KVQ_ERR_TIMEOUT.
 */
void kvq_testing_set_fused_wait(uint32_t extra_a_tiles, uint64_t wait_ns);

/*
 * kvq_testing_set_attention_wait -- for the current device: with wait_ns > 0, the MMA warp
 *   of every later kvq_attention call first waits on an mbarrier that nothing arrives on,
 *   and every data-path wait gives up after wait_ns nanoseconds. So the MMA warp issues
 *   nothing, the other warps' waits give up in turn, the call lets whatever it issued
 *   drain (that last wait keeps the library's 1 s bound), frees its tensor memory and
 *   sets *status to 1. wait_ns == 0 restores normal operation. Call it while no
 *   attention kernel runs on the device.
 */
void kvq_testing_set_attention_wait(uint64_t wait_ns);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_TESTING_H_ */
