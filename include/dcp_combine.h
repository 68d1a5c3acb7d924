/*
 * dcp_combine.h -- C ABI of libdcpcombine.so: the decode-context-parallel (DCP)
 * LSE-weighted combine of partial attention outputs on NVIDIA B200 (sm_100a).
 *
 * Decode context parallelism shards the KV cache of each request over N ranks.
 * Each shard attends to its part of the context and returns a partial output
 * [B, H, D] with its log-sum-exp (LSE) [B, H]; the exact attention result is
 * the LSE-weighted combine of the N partials.  This library runs the three
 * device steps of that combine, all inside one GPU's memory:
 *
 *   dcp_pack                 partial output + fp32 LSE -> one packed send buffer
 *   dcp_lse_combine          combine of separate output / LSE receive buffers
 *   dcp_lse_combine_strided  the same with any token / head layout
 *   dcp_lse_combine_varlen   the same per request: shards without KV are skipped
 *   dcp_combine_pack         a producer's split merge written straight into the send buffer
 *   dcp_unpack_combine       combine read straight out of the packed buffer
 *
 * Defining passages (web pages, by title and section):
 *   [COMBINE] vLLM API docs, vllm.v1.attention.ops.dcp_alltoall,
 *             _lse_weighted_combine: the combine rules.
 *   [A2A]     same page, dcp_a2a_lse_reduce: the packed buffer
 *             [N, B, H/N, D + lse_pack_dim] in the output dtype, the head
 *             scatter (rank r receives heads [r*H/N, (r+1)*H/N)), and the
 *             unpack+combine that follows the All-to-All.
 *   [DIRECT]  vLLM API docs, vllm.v1.attention.ops.dcp, DirectDCPA2AWorkspace:
 *             split receive buffers received_output [N, T_max, H/N, D] and
 *             received_lse [N, T_max, H/N] (fp32), i.e. a shard stride that
 *             may exceed B*H*D.
 *   [ASCEND]  vllm-ascend, vllm_ascend/attention/context_parallel/sfa_cp.py,
 *             _merge_dcp_outputs_with_torch: the same merge as a softmax over
 *             the shard axis, on head- or token-scattered receive layouts.
 *
 * The combine, per token b and head h, over shards n = 0..N-1 ([COMBINE]):
 *   l_n <- -inf if l_n is NaN or +-inf
 *   m    = max_n l_n, and m <- 0 if m == -inf
 *   w_n  = exp(l_n - m) (base e) or 2^(l_n - m) (base 2); NaN -> 0
 *   S    = sum_n w_n;  w_n <- w_n / max(S, 1e-10)
 *   out[b,h,:]    = sum_n w_n * o_n[b,h,:]   (fp32 accumulation, one rounding)
 *   global_lse[b,h] = ln(S) + m   (log2(S) + m in base 2; S unclamped, so an
 *                                  all-empty row gives -inf)
 *
 * Conventions shared by every entry point:
 *   - All buffer pointers are DEVICE pointers on the device that is current on
 *     the calling thread; the caller owns every buffer.  The library allocates
 *     nothing.
 *   - Calls are asynchronous on `cuda_stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and never synchronise (dcp_wait_timeouts, which
 *     reads a device counter, is the one exception).  Inputs must stay valid
 *     and outputs untouched until the stream reaches the call.
 *   - Outputs must not overlap inputs.
 *   - Sizes and strides are in ELEMENTS of the named array's type.
 *   - Every argument is validated on the host before any launch; a non-zero
 *     dcp_status is returned and nothing is launched.  dcp_last_error() then
 *     describes the problem.  A failed launch returns DCP_ERR_CUDA.
 *   - B == 0 is a valid no-op.
 *   - Thread-safe: no global mutable state besides the per-thread error text and the
 *     device's count of timed-out waits (dcp_wait_timeouts).
 */
#ifndef DCP_COMBINE_H
#define DCP_COMBINE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element type of the attention outputs and of the packed buffer.  LSEs are
 * always fp32, as [A2A] specifies for the partial LSE. */
typedef enum {
    DCP_BF16 = 0,
    DCP_FP16 = 1,
    DCP_FP32 = 2
} dcp_dtype;

typedef enum {
    DCP_OK = 0,
    DCP_ERR_INVALID_ARG = 1,       /* null pointer, count out of range, bad stride */
    DCP_ERR_UNSUPPORTED_DTYPE = 2, /* dtype not one of dcp_dtype */
    DCP_ERR_MISALIGNED = 3,        /* pointer / row / stride alignment not met */
    DCP_ERR_SHAPE = 4,             /* H not divisible by world_size */
    DCP_ERR_CUDA = 5               /* the kernel launch failed */
} dcp_status;

/* Largest number of shards (DCP ranks) one call combines. */
#define DCP_MAX_SHARDS 64

/*
 * Number of output-dtype slots that carry one fp32 LSE in a packed row
 * ([A2A], _dcp_a2a_lse_pack_dim): 4 bytes / element size, i.e. 2 for bf16
 * and fp16, 1 for fp32.  Returns -1 for an unknown dtype.
 */
int32_t dcp_lse_pack_dim(int32_t dtype);

/*
 * Pack step of [A2A] dcp_a2a_lse_reduce.
 *
 * cp_attn_out  [B, H, D] of `dtype`; element (b, h, d) at
 *              b*out_stride_b + h*out_stride_h + d.
 * cp_attn_lse  [B, H] fp32; element (b, h) at b*lse_stride_b + h.
 * send_buf     [world_size, B, H/world_size, D + P] of `dtype`, contiguous,
 *              P = dcp_lse_pack_dim(dtype).  Row (r, b, h) receives
 *              cp_attn_out[b, r*H/world_size + h, 0:D] unchanged, then the 4
 *              bytes of cp_attn_lse[b, r*H/world_size + h] in memory order
 *              (slot D = low half-word for 16-bit dtypes).  Bit-exact: no
 *              rounding, NaN payloads preserved.
 *
 * Requirements: world_size in [1, DCP_MAX_SHARDS]; H % world_size == 0
 * (else DCP_ERR_SHAPE); B >= 0; H, D >= 1; D*elemsize a multiple of 16
 * (D % 8 == 0 for 16-bit types, D % 4 == 0 for fp32); cp_attn_out and
 * send_buf 16-byte aligned, out_stride_b / out_stride_h multiples of
 * 16/elemsize and >= 1 (else DCP_ERR_MISALIGNED / DCP_ERR_INVALID_ARG);
 * cp_attn_lse 4-byte aligned, lse_stride_b >= H.
 *
 * Long calls load each tile (consecutive tokens x all heads of one rank, about
 * 64 KiB) with one tensor copy, through a tensor map the call encodes with the
 * driver's cuTensorMapEncodeTiled (found through cudaGetDriverEntryPoint; the
 * library does not link the driver); such a call may launch two kernels, the
 * second for each rank's last B mod (tokens per tile) tokens.  Other calls, and
 * any whose map the driver refuses, copy rows with bulk copies.  Same result.
 *
 * The kernels wait for their copies with a time limit; a wait that runs out
 * (never, while the copies work) leaves this call's send_buf incomplete and
 * is counted by dcp_wait_timeouts, and the call still returns DCP_OK (it
 * returns before the kernel runs).  A caller that must be sure of send_buf
 * reads dcp_wait_timeouts (which synchronises) before trusting it.
 */
int32_t dcp_pack(const void *cp_attn_out, const float *cp_attn_lse, void *send_buf,
                 int64_t B, int64_t H, int64_t D, int32_t world_size, int32_t dtype,
                 int64_t out_stride_b, int64_t out_stride_h, int64_t lse_stride_b,
                 void *cuda_stream);

/*
 * Combine of split receive buffers ([COMBINE] on the [DIRECT] layout).
 *
 * outputs     [N, B, H, D] of `dtype`; element (n, b, h, d) at
 *             n*out_stride_n + (b*H + h)*D + d, out_stride_n >= B*H*D.
 * lses        [N, B, H] fp32; element (n, b, h) at n*lse_stride_n + b*H + h,
 *             lse_stride_n >= B*H.
 * result      [B, H, D] of `dtype`, contiguous.
 * global_lse  [B, H] fp32, contiguous; written only when return_lse != 0
 *             (may be NULL otherwise).
 * is_lse_base_on_e  nonzero: LSEs are natural logs; zero: base-2 logs.
 *
 * Requirements: N in [1, DCP_MAX_SHARDS]; B >= 0; H, D >= 1; D*elemsize a
 * multiple of 16; outputs and result 16-byte aligned; out_stride_n a
 * multiple of 16/elemsize; lses and global_lse 4-byte aligned.
 */
int32_t dcp_lse_combine(const void *outputs, const float *lses, void *result, float *global_lse,
                        int32_t N, int64_t B, int64_t H, int64_t D,
                        int64_t out_stride_n, int64_t lse_stride_n, int32_t dtype,
                        int32_t is_lse_base_on_e, int32_t return_lse, void *cuda_stream);

/*
 * The same combine with every layout stride explicit: split receive buffers in
 * any token / head order.  This covers the layouts in which the vllm-ascend
 * sfa_cp.py merge (_merge_dcp_outputs_with_torch, _merge_dcp_outputs) receives
 * the shards: head-scattered [N, H/N, T, D] with LSEs [N, H/N, T]
 * ("token_dim = 2"), and token-scattered [N, T/N, H, D] ("token_dim = 1"),
 * as well as capacity-strided [DIRECT] buffers.
 *
 * outputs     element (n, b, h, d) at n*out_stride_n + b*out_stride_b +
 *             h*out_stride_h + d.
 * lses        fp32; element (n, b, h) at n*lse_stride_n + b*lse_stride_b +
 *             h*lse_stride_h.
 * result      element (b, h, d) at b*result_stride_b + h*result_stride_h + d.
 * global_lse  fp32; element (b, h) at b*glse_stride_b + h*glse_stride_h;
 *             written only when return_lse != 0 (may be NULL otherwise).
 * Strides are in elements of each array and >= 0; inputs may overlap one
 * another (they are only read); result rows must not overlap.
 *
 * Requirements: as dcp_lse_combine, and out_stride_* and result_stride_*
 * multiples of 16 bytes (else DCP_ERR_MISALIGNED); B*H < 2^32.
 */
int32_t dcp_lse_combine_strided(const void *outputs, const float *lses, void *result, float *global_lse,
                                int32_t N, int64_t B, int64_t H, int64_t D,
                                int64_t out_stride_n, int64_t out_stride_b, int64_t out_stride_h,
                                int64_t lse_stride_n, int64_t lse_stride_b, int64_t lse_stride_h,
                                int64_t result_stride_b, int64_t result_stride_h,
                                int64_t glse_stride_b, int64_t glse_stride_h, int32_t dtype,
                                int32_t is_lse_base_on_e, int32_t return_lse, void *cuda_stream);

/*
 * Variable-length combine of split receive buffers: the receive-side reduce of
 * [DIRECT] (DirectDCPA2AWorkspace.lse_reduce), which also takes the batch's
 * seq_lens and query_start_loc.  The page does not define what the reduce does
 * with them; this library reads them as follows.
 *   - Token b belongs to request r when query_start_loc[r] <= b <
 *     query_start_loc[r + 1].  A token outside every request (padding) has no
 *     context: its result row is 0 and its global LSE -inf.
 *   - Shard n holds KV of request r when n * interleave < seq_lens[r]
 *     (blocks of `interleave` KV positions dealt round-robin to the N ranks, as
 *     in [ASCEND] AscendSFACPMetadataBuilder._get_dcp_local_seq_lens).  A shard
 *     that holds none counts as LSE -inf and its output row is NOT read: it may
 *     hold anything, NaN included.
 *   - Everything else is the [COMBINE] rule set, as dcp_lse_combine.
 *
 * outputs, lses, result, global_lse, out_stride_n, lse_stride_n: as
 *             dcp_lse_combine.
 * seq_lens    [num_reqs] int32 DEVICE array: KV length of each request.  Shard n
 *             holds KV when its local length is positive (n * interleave <
 *             seq_lens[r]); 0 and negative values are accepted and mean that no
 *             shard holds KV of the request.
 * query_start_loc  [num_reqs + 1] int32 DEVICE array, non-decreasing: the first
 *             token of each request, then the end of the last one.  Values that
 *             are not non-decreasing give unspecified results but no access
 *             outside the two arrays.
 * num_reqs    >= 0; with 0 every token is padding and the arrays may be NULL.
 * interleave  >= 1: KV positions per round-robin block (1 = token interleave).
 *
 * Requirements: as dcp_lse_combine; seq_lens and query_start_loc non-NULL
 * (when num_reqs > 0 and B > 0) and 4-byte aligned, else DCP_ERR_INVALID_ARG /
 * DCP_ERR_MISALIGNED.
 */
int32_t dcp_lse_combine_varlen(const void *outputs, const float *lses, void *result, float *global_lse,
                               int32_t N, int64_t B, int64_t H, int64_t D,
                               int64_t out_stride_n, int64_t lse_stride_n,
                               const int32_t *seq_lens, const int32_t *query_start_loc,
                               int32_t num_reqs, int32_t interleave, int32_t dtype,
                               int32_t is_lse_base_on_e, int32_t return_lse, void *cuda_stream);

/*
 * Combine fused with the pack: the producer's epilogue.  A split-KV (flash-decoding)
 * producer ends by merging its S partial results over its own KV splits, by the same
 * [COMBINE] rules; this call does that merge and writes the merged rows straight into the
 * [A2A] send buffer, so cp_attn_out is never written and dcp_pack never runs.
 * Equivalent to dcp_lse_combine(..., return_lse = 1) into [B, H, D] + [B, H], then
 * dcp_pack of those into send_buf, with the same bits.
 *
 * partial_outputs  [S, B, H, D] of `dtype`; element (s, b, h, d) at
 *             s*out_stride_s + (b*H + h)*D + d, out_stride_s >= B*H*D.
 * partial_lses     [S, B, H] fp32; element (s, b, h) at s*lse_stride_s + b*H + h,
 *             lse_stride_s >= B*H.
 * send_buf    [world_size, B, H/world_size, D + P] of `dtype`, contiguous (as written
 *             by dcp_pack): row (r, b, h) receives the merged row of head r*H/world_size
 *             + h, then the 4 bytes of its merged fp32 LSE (ln S + m, or log2 S + m).
 *
 * Requirements: S in [1, DCP_MAX_SHARDS]; world_size in [1, DCP_MAX_SHARDS]; H %
 * world_size == 0 (else DCP_ERR_SHAPE); B >= 0; H, D >= 1; D*elemsize a multiple of 16;
 * partial_outputs and send_buf 16-byte aligned; out_stride_s a multiple of 16/elemsize;
 * partial_lses 4-byte aligned.
 */
int32_t dcp_combine_pack(const void *partial_outputs, const float *partial_lses, void *send_buf,
                         int32_t S, int64_t B, int64_t H, int64_t D,
                         int64_t out_stride_s, int64_t lse_stride_s, int32_t world_size,
                         int32_t dtype, int32_t is_lse_base_on_e, void *cuda_stream);

/*
 * Fused unpack + combine over the packed receive buffer ([A2A], the step
 * after the All-to-All): one pass over the buffer, the LSE read out of each
 * row's last P slots.
 *
 * recv_buf    [N, B, Hr, D + P] of `dtype`; row (n, b, h) starts at element
 *             n*stride_n + (b*Hr + h)*(D + P); stride_n >= B*Hr*(D + P).
 * result      [B, Hr, D] of `dtype`, contiguous.
 * global_lse  [B, Hr] fp32, contiguous; written only when return_lse != 0.
 *
 * Requirements: N in [1, DCP_MAX_SHARDS]; B >= 0; Hr, D >= 1; D*elemsize a
 * multiple of 16; recv_buf and result 16-byte aligned; stride_n*elemsize a
 * multiple of 4; global_lse 4-byte aligned.
 */
int32_t dcp_unpack_combine(const void *recv_buf, void *result, float *global_lse,
                           int32_t N, int64_t B, int64_t Hr, int64_t D, int64_t stride_n,
                           int32_t dtype, int32_t is_lse_base_on_e, int32_t return_lse,
                           void *cuda_stream);

/*
 * Pack CTAs whose wait timed out on the current device since the last reset.  dcp_pack
 * waits for its bulk and tensor copies with a limit of one second per wait; when a wait runs
 * out the CTA is counted here and stops (after waiting, bounded, for the copies it has
 * issued), so the send buffer of that call is incomplete.  A tensor-copy CTA whose shared
 * memory cannot be placed on a 128-byte boundary is counted too and copies nothing (the
 * launch reserves the room to align it, so this does not happen).  A nonzero count therefore means a result is
 * invalid (it never happens when the copies work).  Synchronises the device (the counter is
 * read from device memory); with reset != 0 the counter is cleared afterwards.  Returns
 * DCP_ERR_CUDA if the read fails.
 */
int32_t dcp_wait_timeouts(uint64_t *count, int32_t reset);

/* Text of the last non-OK status returned on the calling thread ("" if none). */
const char *dcp_last_error(void);

/* Library version, major*10000 + minor*100 + patch. */
int32_t dcp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DCP_COMBINE_H */
