/*
 * dcp_testing.h -- test hooks of libdcpcombine.so: one makes the timeout path of the pack
 * kernels' bounded waits run, so that a test can check it without faulting or hanging a
 * GPU; one reports the launch shape the host picks for a split-layout combine, so that the
 * shape rules can be checked without a GPU; two report which pack kernel ran and the tensor
 * pack's tile shape.  Not part of the combine; no page has a counterpart.
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

/*
 * The shape the host picks for a split-layout combine of N shards whose rows are `chunks`
 * 16-byte chunks (D * elemsize / 16): kind 0 = dcp_lse_combine (and its strided form),
 * 1 = dcp_lse_combine_varlen, 2 = the per-row path of dcp_combine_pack.  Writes out[0] =
 * lanes per row, out[1] = chunk slots per lane per pass, out[2] = shards per batch, out[3] =
 * 1 if phase 1's LSE reads are prefetched (for kind 0 before the short-launch rule, which
 * also depends on the row count).  The lanes per row decide the result bits: the weights are
 * summed by lane j of G over shards j, j + G, ..., then by halving over the G lanes.  Needs
 * no GPU.  Returns DCP_OK, or DCP_ERR_INVALID_ARG for a kind outside 0..2, N outside
 * [1, DCP_MAX_SHARDS], chunks < 1 or a null `out`.
 */
int32_t dcp_testing_split_shape(int32_t kind, int32_t N, int32_t chunks, int32_t *out);

/*
 * Which kernel the calling host thread's last dcp_pack (or dcp_testing_pack_stalled) launched,
 * so that a test can check the path it covers: 0 = none yet (or an empty call), 1 = pack_kernel
 * with one bulk copy per row, 2 = pack_kernel copying a token's contiguous heads as runs,
 * 3 = pack_kernel with tiles in rank-fastest order, 4 = pack_tma_kernel with a 3-dimensional
 * tensor map (rows of at most 256 elements), 5 = pack_tma_kernel with each row split into
 * pieces (4 dimensions).  Needs no arguments and cannot fail.
 */
int32_t dcp_testing_last_pack_kernel(void);

/*
 * The tile shape dcp_pack's tensor copies would take for Hr heads per rank of D elements of
 * `dtype` and B tokens, without encoding a map (needs no GPU): out[0] = k, the tokens per tile
 * (at most 256 and at most B, k x Hr rows within 64 KiB, the largest such k); out[1] = m, the
 * pieces each row is split into (the fewest with D a multiple of m, at most 256 elements and a
 * multiple of 16 bytes each); out[2] = the tensor map's dimensions (3 when m = 1, else 4).
 * All three are 0 when no tile suits the shape (more than 256 heads, or one token's heads over
 * 64 KiB).  Which launches use the shape also depends on the device (see dcp_pack).  Returns
 * DCP_OK, or DCP_ERR_INVALID_ARG for a dtype outside 0..2, Hr, D or B < 1, or a null `out`.
 */
int32_t dcp_testing_pack_tensor_shape(int64_t Hr, int64_t D, int32_t dtype, int64_t B, int32_t *out);

#ifdef __cplusplus
}
#endif

#endif /* DCP_TESTING_H */
