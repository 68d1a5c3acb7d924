// dcp_combine_launch.cuh -- choice of the combine kernel instance for a call and its
// launch; included by the per-element-type translation units only.
#pragma once

#include "dcp_host.h"

namespace dcp_host {

template <class T, int G, int CPL, int NB, bool PACKED, int MIN_CTAS, bool UNIFORM, bool VARLEN, bool PACK_OUT,
          bool PREFETCH>
int32_t launch_combine(const dcp::CombineArgs &a, cudaStream_t stream) {
    const char *fn = PACKED ? "dcp_unpack_combine" : PACK_OUT ? "dcp_combine_pack" : "dcp_lse_combine";
    auto kernel = dcp::combine_kernel<T, G, CPL, NB, PACKED, MIN_CTAS, UNIFORM, VARLEN, PACK_OUT, PREFETCH>;
    static InstanceCache ic;
    constexpr int kUnitsPerWarp = 32 / G;
    constexpr int kWarps = dcp::kCombineThreads / 32;
    const size_t smem = dcp::combine_smem_bytes(kUnitsPerWarp, a.N, PACKED, PREFETCH);
    if (!reserve_smem(kernel, ic, dcp::combine_smem_bytes(kUnitsPerWarp, DCP_MAX_SHARDS, PACKED, PREFETCH)))
        return fail(DCP_ERR_CUDA, "%s: cannot reserve shared memory", fn);
    const int per_sm = cached_resident_ctas(kernel, ic, dcp::kCombineThreads, smem);
    const int64_t tasks = (a.units + kUnitsPerWarp - 1) / kUnitsPerWarp;
    const int64_t want = (tasks + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)sm_count() * per_sm;
    const int grid = (int)(want < cap ? want : cap);
    kernel<<<grid, dcp::kCombineThreads, smem, stream>>>(a);
    return launch_status(fn);
}

// The single-pass packed combine (online_unpack_kernel), one pass per row.
template <class T, int G, int CPL, int NB, int MIN_CTAS>
int32_t launch_online(const dcp::CombineArgs &a, cudaStream_t stream) {
    auto kernel = dcp::online_unpack_kernel<T, G, CPL, NB, MIN_CTAS>;
    static InstanceCache ic;
    if (a.slots > CPL) return fail(DCP_ERR_INVALID_ARG, "dcp_unpack_combine: internal shape error");
    constexpr int kUnitsPerWarp = 32 / G;
    constexpr int kWarps = dcp::kCombineThreads / 32;
    const int per_sm = cached_resident_ctas(kernel, ic, dcp::kCombineThreads, 0);
    const int64_t tasks = (a.units + kUnitsPerWarp - 1) / kUnitsPerWarp;
    const int64_t want = (tasks + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)sm_count() * per_sm;
    const int grid = (int)(want < cap ? want : cap);
    kernel<<<grid, dcp::kCombineThreads, 0, stream>>>(a);
    return launch_status("dcp_unpack_combine");
}

// Occupancy: the kernel keeps NB * CPL 16-byte loads in flight per lane, so the
// bytes in flight per SM are set by how many warps fit.  Capping registers so
// that 3 CTAs fit (2 for the four-slot shapes, which spill otherwise) measured
// best on B200 for every shape.
template <class T, int G, bool PACKED, bool UNIFORM, bool VARLEN, bool PACK_OUT, bool PREFETCH>
int32_t launch_cpl(dcp::CombineArgs a, int cpl, cudaStream_t stream) {
    switch (cpl) {
        case 1: return launch_combine<T, G, 1, 8, PACKED, 3, UNIFORM, VARLEN, PACK_OUT, PREFETCH>(a, stream);
        case 2: return launch_combine<T, G, 2, 4, PACKED, 3, UNIFORM, VARLEN, PACK_OUT, PREFETCH>(a, stream);
        default: return launch_combine<T, G, 4, 2, PACKED, 2, UNIFORM, VARLEN, PACK_OUT, PREFETCH>(a, stream);
    }
}

template <class T, bool PACKED, bool UNIFORM, bool VARLEN, bool PACK_OUT, bool PREFETCH>
int32_t launch_g(dcp::CombineArgs a, int G, int cpl, cudaStream_t stream) {
    switch (G) {
        case 4: return launch_cpl<T, 4, PACKED, UNIFORM, VARLEN, PACK_OUT, PREFETCH>(a, cpl, stream);
        case 8: return launch_cpl<T, 8, PACKED, UNIFORM, VARLEN, PACK_OUT, PREFETCH>(a, cpl, stream);
        case 16: return launch_cpl<T, 16, PACKED, UNIFORM, VARLEN, PACK_OUT, PREFETCH>(a, cpl, stream);
        default: return launch_cpl<T, 32, PACKED, UNIFORM, VARLEN, PACK_OUT, PREFETCH>(a, cpl, stream);
    }
}

// Shape of the work per lane.  Each lane should keep about eight 16-byte loads
// in flight: chunk slots per lane (CPL) times shards per batch (NB = 8 / CPL),
// so fewer shards ask for more chunks per lane, i.e. fewer lanes per row (G).
// When all shards of the packed buffer put a row at the same offset from a
// 16-byte boundary (the shard stride is a multiple of 16 bytes) and one pass
// covers a row, the sums are realigned once per output chunk ("uniform");
// otherwise every shard's chunk is realigned, and that path keeps at least two
// slots per lane.
struct CombineShape {
    int G;    // lanes per row
    int cpl;  // chunk slots per lane per pass
};

inline CombineShape combine_shape(bool packed, bool uniform, int N, int chunks) {
    int cpl_target = N >= 8 ? 1 : N >= 4 ? 2 : 4;
    if (packed && !uniform && cpl_target < 2) cpl_target = 2;
    // split layout, 8 or more shards, rows of at most 256 bytes: two chunk slots per lane
    // (four rows per warp) measured 3-6% faster than one with 8-15 shards, 2% with 16
    if (!packed && N >= 8 && chunks <= 16) cpl_target = 2;
    const int per_lane = (chunks + cpl_target - 1) / cpl_target;
    int G = 4;
    while (G < per_lane && G < 32) G *= 2;
    const int slots = (chunks + G - 1) / G;
    return {G, slots >= 3 ? 4 : slots};  // one pass whenever slots <= 4
}

// The fused pack's 4-row group kernel: packed rows of D' = 32 C data words, C = 2 or 4, with
// heads per rank a multiple of 4.  Tasks are 4-row groups, one per warp at a time.
template <class K>
int32_t launch_group(K kernel, InstanceCache &ic, const dcp::CombineArgs &a, size_t smem, const char *fn,
                     cudaStream_t stream) {
    if (!reserve_smem(kernel, ic, smem)) return fail(DCP_ERR_CUDA, "%s: cannot reserve shared memory", fn);
    const int per_sm = cached_resident_ctas(kernel, ic, dcp::kCombineThreads, smem);
    constexpr int kWarps = dcp::kCombineThreads / 32;
    const int64_t groups = (a.units + 3) / 4;
    const int64_t want = (groups + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)sm_count() * per_sm;
    const int grid = (int)(want < cap ? want : cap);
    kernel<<<grid, dcp::kCombineThreads, smem, stream>>>(a);
    return launch_status(fn);
}

template <class T, int C, int NB, int MIN_CTAS>
int32_t launch_group_pack(const dcp::CombineArgs &a, cudaStream_t stream) {
    if (a.data_w != 32 * C || a.pack_hr % 4 != 0) return fail(DCP_ERR_INVALID_ARG, "dcp_combine_pack: internal shape error");
    static InstanceCache ic;
    if (!reserve_smem(dcp::group_pack_kernel<T, C, NB, MIN_CTAS>, ic,
                      dcp::group_pack_smem_bytes(DCP_MAX_SHARDS, 32 * C)))
        return fail(DCP_ERR_CUDA, "dcp_combine_pack: cannot reserve shared memory");
    return launch_group(dcp::group_pack_kernel<T, C, NB, MIN_CTAS>, ic, a, dcp::group_pack_smem_bytes(a.N, a.data_w),
                        "dcp_combine_pack", stream);
}

// NB = 2 splits in flight: measured best or equal for S = 4 and 8 (D' = 64: 0.89-0.94 of the
// measured peak at B = 16384, against 0.75-0.81 for the per-row packed stores).
template <class T>
int32_t dispatch_group_pack(const dcp::CombineArgs &a, cudaStream_t stream) {
    switch (a.data_w) {
        case 64: return launch_group_pack<T, 2, 2, 3>(a, stream);
        case 128: return launch_group_pack<T, 4, 2, 3>(a, stream);
        default: return fail(DCP_ERR_INVALID_ARG, "dcp_combine_pack: internal shape error");
    }
}

template <class T, bool PACKED>
int32_t dispatch_combine(dcp::CombineArgs a, cudaStream_t stream) {
    const int chunks = a.chunks;
    const bool uniform = PACKED && (a.N == 1 || a.shard_stride_w % 4 == 0) && chunks <= 4 * 32;
    // the fused pack's group kernel: D' = 64 or 128 (at 32 the per-row path measured faster)
    const bool group_rows = a.data_w == 64 || a.data_w == 128;
    const CombineShape sh = combine_shape(PACKED, uniform, a.N, chunks);
    const int G = sh.G, cpl = sh.cpl;
    a.slots = (chunks + G - 1) / G;
    // Phase 1's reads one task ahead: measured worth it where phase 1's latency is exposed
    // (two shards, or packed rows of 1 KiB and more), and 2-4% slower where the stream
    // already hides it.
    const bool prefetch = a.N <= 2 || (PACKED && chunks >= 64);
    if constexpr (PACKED) {
        if (uniform && chunks <= 32 && a.N >= 3) {
            // rows of at most 512 bytes and 3 or more shards: the single-pass kernel, whose LSEs
            // come with each batch's data.  Measured at B = 16384 (fractions of the measured
            // peak, single-pass against two-phase): D = 64 N = 8, 16: 0.91, 0.99 vs 0.74, 0.77;
            // D = 128 N = 3, 4, 8, 16: 0.86, 0.96, 0.99, 1.03 vs 0.71, 0.77, 0.94, 0.91;
            // D = 256 N = 4, 8: 0.96, 0.98 vs 0.82, 0.81.  At N = 2 the two kinds tie.
            if (chunks <= 8) {
                a.slots = (chunks + 3) / 4;
                return launch_online<T, 4, 2, 4, 3>(a, stream);
            }
            if (chunks <= 16) {
                if (a.N >= 8) {
                    a.slots = (chunks + 7) / 8;
                    return launch_online<T, 8, 2, 4, 3>(a, stream);
                }
                a.slots = (chunks + 3) / 4;
                return launch_online<T, 4, 4, 4, 2>(a, stream);
            }
            a.slots = (chunks + 7) / 8;
            return launch_online<T, 8, 4, 4, 2>(a, stream);
        }
        if (uniform) {
            if (prefetch) return launch_g<T, true, true, false, false, true>(a, G, cpl, stream);
            return launch_g<T, true, true, false, false, false>(a, G, cpl, stream);
        }
        return launch_g<T, true, false, false, false, false>(a, G, cpl, stream);
    } else {
        if (a.varlen) {
            if (G == 8 && chunks > 8 && chunks <= 16 && a.N >= 8) {
                // the plain combine's shape (G = 8, so the weights are summed alike) with all 8
                // shards of a batch in flight: D = 128, B = 16384, N = 8 / 16 took 1.09 / 1.03 of the
                // plain combine's time per byte read, against 1.11 / 1.05 with 4
                return launch_combine<T, 8, 2, 8, false, 2, false, true, false, true>(a, stream);
            }
            return launch_g<T, false, false, true, false, true>(a, G, cpl, stream);
        }
        if (a.pack_b > 0) {
            if (group_rows && a.pack_hr % 4 == 0) {
                // the weights summed as the split combine would (same lanes per row)
                a.red_lanes = G;
                return dispatch_group_pack<T>(a, stream);
            }
            return launch_g<T, false, false, false, true, false>(a, G, cpl, stream);
        }
        if (prefetch) return launch_g<T, false, false, false, false, true>(a, G, cpl, stream);
        return launch_g<T, false, false, false, false, false>(a, G, cpl, stream);
    }
}

}  // namespace dcp_host
