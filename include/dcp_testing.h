/*
 * dcp_testing.h -- test hook of libdcpcombine.so: makes the timeout path of the pack
 * kernel's bounded wait run, so that a test can check it without faulting or hanging a
 * GPU.  Not part of the combine; no page has a counterpart.
 */
#ifndef DCP_TESTING_H
#define DCP_TESTING_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * dcp_pack (same arguments, same validation and status codes) with two changes: each
 * CTA's wait for the bulk copies of its first tile expects 16 bytes that never arrive,
 * and every wait gives up after 20 ms instead of one second.  Every copy still completes;
 * only the wait runs out.  Each CTA therefore stops at its first tile, after waiting
 * (bounded) for all the copies it has issued, and is counted once in dcp_wait_timeouts;
 * send_buf is left incomplete.  The kernel returns normally, and the device stays usable.
 */
int32_t dcp_testing_pack_stalled(const void *cp_attn_out, const float *cp_attn_lse, void *send_buf,
                                 int64_t B, int64_t H, int64_t D, int32_t world_size, int32_t dtype,
                                 int64_t out_stride_b, int64_t out_stride_h, int64_t lse_stride_b,
                                 void *cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* DCP_TESTING_H */
