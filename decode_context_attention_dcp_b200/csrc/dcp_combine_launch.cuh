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
template <class T, int G, int CPL, int NB, int MIN_CTAS, bool SINGLE = false>
int32_t launch_online_as(const dcp::CombineArgs &a, cudaStream_t stream) {
    auto kernel = dcp::online_unpack_kernel<T, G, CPL, NB, MIN_CTAS, SINGLE>;
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

// ... with the single-batch instance when every shard fits one batch
template <class T, int G, int CPL, int NB, int MIN_CTAS>
int32_t launch_online(const dcp::CombineArgs &a, cudaStream_t stream) {
    if (a.N <= NB) return launch_online_as<T, G, CPL, NB, MIN_CTAS, true>(a, stream);
    return launch_online_as<T, G, CPL, NB, MIN_CTAS, false>(a, stream);
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

// Shape of the packed two-phase combine.  Each lane should keep about eight 16-byte loads
// in flight: chunk slots per lane (CPL) times shards per batch (NB = 8 / CPL), so fewer
// shards ask for more chunks per lane, i.e. fewer lanes per row (G).  When all shards of the
// packed buffer put a row at the same offset from a 16-byte boundary (the shard stride is a
// multiple of 16 bytes) and one pass covers a row, the sums are realigned once per output
// chunk ("uniform"); otherwise every shard's chunk is realigned, and that path keeps at least
// two slots per lane.
struct CombineShape {
    int G;    // lanes per row
    int cpl;  // chunk slots per lane per pass
};

inline CombineShape combine_shape(bool uniform, int N, int chunks) {
    int cpl_target = N >= 8 ? 1 : N >= 4 ? 2 : 4;
    if (!uniform && cpl_target < 2) cpl_target = 2;
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

// The packed receive layout (dcp_unpack_combine).
template <class T>
int32_t dispatch_packed(dcp::CombineArgs a, cudaStream_t stream) {
    const int chunks = a.chunks;
    const bool uniform = (a.N == 1 || a.shard_stride_w % 4 == 0) && chunks <= 4 * 32;
    const CombineShape sh = combine_shape(uniform, a.N, chunks);
    const int G = sh.G, cpl = sh.cpl;
    a.slots = (chunks + G - 1) / G;
    // Phase 1's reads one task ahead: measured worth it where phase 1's latency is exposed
    // (two shards, or packed rows of 1 KiB and more), and 2-4% slower where the stream
    // already hides it.
    const bool prefetch = a.N <= 2 || chunks >= 64;
    if (uniform && a.N == 2 && chunks <= 16) {
        // two shards, rows of at most 256 bytes: the single-pass kernel with both shards in one
        // batch (B = 16384, D = 128: 0.84 of the measured peak against 0.76 two-phase; D = 64:
        // 0.64 against 0.51)
        if (chunks <= 8) {
            a.slots = (chunks + 3) / 4;
            return launch_online<T, 4, 2, 4, 3>(a, stream);
        }
        a.slots = (chunks + 3) / 4;
        return launch_online<T, 4, 4, 2, 2>(a, stream);
    }
    if (uniform && chunks <= 32 && a.N >= 3) {
        // rows of at most 512 bytes and 3 or more shards: the single-pass kernel, whose LSEs
        // come with each batch's data (with N <= 4 one batch holds them all).  Measured at
        // B = 16384 (fractions of the measured peak, single-pass against two-phase): D = 64
        // N = 4, 8, 16: 0.85, 0.91, 0.99 vs -, 0.74, 0.77; D = 128 N = 3, 4, 8, 16: 0.92,
        // 0.97, 1.01, 1.03 vs 0.71, 0.77, 0.94, 0.91; D = 256 N = 3, 4, 8: 0.96, 0.99, 0.95
        // vs -, 0.82, 0.81.
        if (chunks <= 8) {
            a.slots = (chunks + 3) / 4;
            return launch_online<T, 4, 2, 4, 3>(a, stream);
        }
        if (chunks <= 16) {
            if (a.N >= 8) {
                a.slots = (chunks + 7) / 8;
                return launch_online_as<T, 8, 2, 4, 3>(a, stream);
            }
            a.slots = (chunks + 3) / 4;
            return launch_online<T, 4, 4, 4, 2>(a, stream);
        }
        a.slots = (chunks + 7) / 8;
        return launch_online<T, 8, 4, 4, 2>(a, stream);
    }
    if (uniform) {
        if (chunks > 32 && chunks <= 64 && a.N <= 4) {
            // rows of 513 bytes to 1 KiB and at most 4 shards: the single-pass kernel, one batch
            // holding every shard (16 lanes per row).  Measured at D = 512 (fractions of the
            // measured peak, against the two-phase kernel): B = 16384, N = 2, 3, 4: 0.92, 0.99,
            // 0.97 against 0.885, 0.94, 0.95; B = 4096, N = 2, 4: 0.84, 1.00 against 0.79, 0.965.
            a.slots = (chunks + 15) / 16;
            if (a.N <= 2) return launch_online_as<T, 16, 4, 2, 2, true>(a, stream);
            return launch_online_as<T, 16, 4, 4, 2, true>(a, stream);
        }
        if (chunks > 32 && chunks <= 64 && a.N >= 5 && a.N < 16) {
            // rows of 513 bytes to 1 KiB and 5-15 shards: 16 lanes per row (a quarter of the
            // row's chunks per lane), 4 shards per batch (16 loads in flight per lane).
            // Measured at D = 512 (fractions of the measured peak, against 32 lanes per row):
            // B = 16384, N = 6, 8: 0.96, 0.96 against 0.92, 0.93; B = 4096, N = 8: 1.03 against
            // 1.00; B = 1024, N = 8: 0.81 against 0.81.  The single-pass kernel (8 shards per
            // batch) did not beat it at N = 5-8.  With 16 shards the 32-lane shape stays ahead
            // (B = 4096: 1.03 against 0.98).
            a.slots = (chunks + 15) / 16;
            return launch_combine<T, 16, 4, 4, true, 2, true, false, false, true>(a, stream);
        }
        if (prefetch) return launch_g<T, true, true, false, false, true>(a, G, cpl, stream);
        return launch_g<T, true, true, false, false, false>(a, G, cpl, stream);
    }
    return launch_g<T, true, false, false, false, false>(a, G, cpl, stream);
}

// Shape of the split-layout combine (dcp_lse_combine and its strided, variable-length and
// fused-pack forms).  Lanes per row G: the row's chunks over about 2 slots per lane with 8
// or more shards (one pass, CPL = 2, 4 shards per batch; rows of at most 8 chunks with 16 or
// more shards: one slot, 8 shards per batch), about 4 with 4-7 shards and 8 with fewer
// (passes of CPL = 4, 2 shards per batch, or all 3).  Phase 1's LSE words are copied one
// task ahead wherever there are fewer than 8 shards or rows of at most 256 bytes.  Measured
// on B200 (split bf16, B = 16384, 16 heads; fractions of the measured copy peak, this shape
// against the previous one):
//   D = 64:  N = 3, 6, 32: 0.89, 1.01, 1.04 against 0.84, 0.84, 0.92
//   D = 128: N = 3, 4, 8, 12: 1.07, 1.06, 1.09, 1.08 against 0.86, 0.94, 1.06, 1.03
//   D = 256: N = 3, 8, 12: 1.03, 1.04, 1.06 against 0.91, 0.94, 0.95
//   D = 512: N = 2, 4: 1.00, 1.04 against 0.98, 1.01
// and within 2% of the best of 22 shapes at every other N in 2-32.  Only G decides the
// result bits (the lanes that sum a row's weights); CPL and the batch only order the loads.
struct SplitShape {
    int G;          // lanes per row
    int cpl;        // chunk slots per lane per pass: 1, 2 or 4
    int nb;         // shards per batch: cpl * nb 16-byte loads in flight per lane
    bool prefetch;  // phase 1's LSE words copied into shared memory one task ahead
};

inline SplitShape split_shape(int N, int chunks) {
    const int per_lane = (N >= 16 && chunks <= 8) ? 1 : N >= 8 ? 2 : N >= 4 ? 4 : 8;
    int G = 4;
    while (G * per_lane < chunks && G < 32) G *= 2;
    const int slots = (chunks + G - 1) / G;
    const int cpl = slots <= 2 ? slots : N >= 8 ? 2 : 4;
    const int nb = cpl == 1 ? 8 : cpl == 2 ? (N <= 2 ? 2 : 4) : (N == 3 ? 4 : 2);
    return {G, cpl, nb, N < 8 || chunks <= 16};
}

// The variable-length combine's shape.  A row whose request reaches only some shards issues
// fewer loads in the same time, so with 4 or more shards each lane keeps 16 loads in flight:
// G = about a quarter of the row's chunks, 4 slots of 4 shards.  The weights must be summed as
// the plain combine sums them (so that a batch whose requests reach every shard gives the
// same bits): lane j of G sums shards j, j + G, ... and the G lanes then reduce by halves, so
// two lane counts agree whenever N <= 2 * the smaller one; otherwise the plain shape is
// kept, as it is with fewer than 4 shards.  Measured at B = 16384, split bf16, time against
// the plain combine's time scaled by the bytes read (about 30% of the requests reaching only
// some shards), this shape against the plain one:
//   D = 128, N = 4, 8: 1.11, 1.07 against 1.18, 1.10
//   D = 256, N = 4, 8, 16: 1.04, 1.04, 1.04 against 1.11, 1.09, 1.05
//   D = 512, N = 4, 8, 16: 1.03, 1.05, 1.03 against 1.08, 1.08, 1.03
inline SplitShape varlen_shape(int N, int chunks, const SplitShape &plain) {
    const SplitShape kept = {plain.G, plain.cpl, plain.nb, true};  // the varlen kernel always prefetches
    if (N < 4) return kept;
    int G = 4;
    while (G * 4 < chunks && G < 32) G *= 2;
    const int lo = G < plain.G ? G : plain.G;
    if (G != plain.G && N > 2 * lo) return kept;
    const int slots = (chunks + G - 1) / G;
    const int cpl = slots <= 2 ? slots : 4;
    return {G, cpl, cpl == 1 ? 8 : 4, true};
}

// The variable-length combine of 8 or more shards with 8 lanes per row of 144-256 bytes keeps
// all 8 shards of a batch in flight: D = 128, B = 16384, N = 16 took 1.03 of the plain
// combine's time per byte read, against 1.05 with 4.
inline bool varlen_all_in_flight(const SplitShape &v, int N, int chunks) {
    return v.G == 8 && v.cpl == 2 && chunks > 8 && chunks <= 16 && N >= 8;
}

// The fused pack's per-row shape (rows that the 4-row group kernel does not take).  Its
// packed-row stores favour more loads in flight per lane and no LSE prefetch: with 4-7
// splits the variable-length shape (16 loads per lane), with 8 or more two slots of 8 splits,
// both with the plain combine's lanes per row (so the result equals dcp_lse_combine +
// dcp_pack bit for bit).  Measured at D = 512, B = 16384 (fractions of the measured peak, this
// shape against the plain one): S = 4, 2-16 ranks: 0.97-0.98 against 0.85-0.89; S = 8:
// 1.01 against 0.99; S = 16 (B = 4096): 1.03 against 1.00.
inline SplitShape pack_shape(int N, int chunks, const SplitShape &plain) {
    if (N >= 8 && plain.cpl == 2) return {plain.G, 2, 8, false};
    if (N >= 4) {
        const SplitShape v = varlen_shape(N, chunks, plain);
        if (v.G == plain.G) return {v.G, v.cpl, v.nb, false};
    }
    return {plain.G, plain.cpl, plain.nb, false};
}

// Registers are capped so that 3 CTAs fit (8 loads in flight per lane), 4 for the 4-load
// shape and 2 for the four-slot shapes, which spill otherwise.  Single-slot shapes only
// arise with G = 4 or 8 and the 2 x 2 shape with G = 4 (rows of at most 8 chunks); a shape
// with a G it does not arise with takes the two-slot instance, which computes the same
// result.
template <class T, int G, bool VARLEN, bool PACK_OUT, bool PREFETCH>
int32_t launch_split_g(const dcp::CombineArgs &a, const SplitShape &s, cudaStream_t stream) {
    if (s.cpl == 4) {
        if (s.nb == 4) return launch_combine<T, G, 4, 4, false, 2, false, VARLEN, PACK_OUT, PREFETCH>(a, stream);
        return launch_combine<T, G, 4, 2, false, 2, false, VARLEN, PACK_OUT, PREFETCH>(a, stream);
    }
    if constexpr (G <= 8) {
        if (s.cpl == 1) return launch_combine<T, G, 1, 8, false, 3, false, VARLEN, PACK_OUT, PREFETCH>(a, stream);
    }
    if constexpr (PACK_OUT) {
        if (s.nb == 8) return launch_combine<T, G, 2, 8, false, 2, false, VARLEN, PACK_OUT, PREFETCH>(a, stream);
    }
    if constexpr (G == 4) {
        if (s.nb == 2) return launch_combine<T, 4, 2, 2, false, 4, false, VARLEN, PACK_OUT, PREFETCH>(a, stream);
    }
    return launch_combine<T, G, 2, 4, false, 3, false, VARLEN, PACK_OUT, PREFETCH>(a, stream);
}

template <class T, bool VARLEN, bool PACK_OUT, bool PREFETCH>
int32_t launch_split(const dcp::CombineArgs &a, const SplitShape &s, cudaStream_t stream) {
    switch (s.G) {
        case 4: return launch_split_g<T, 4, VARLEN, PACK_OUT, PREFETCH>(a, s, stream);
        case 8: return launch_split_g<T, 8, VARLEN, PACK_OUT, PREFETCH>(a, s, stream);
        case 16: return launch_split_g<T, 16, VARLEN, PACK_OUT, PREFETCH>(a, s, stream);
        default: return launch_split_g<T, 32, VARLEN, PACK_OUT, PREFETCH>(a, s, stream);
    }
}

// The split layout: dcp_lse_combine, dcp_lse_combine_strided, dcp_lse_combine_varlen and
// dcp_combine_pack.
template <class T>
int32_t dispatch_split(dcp::CombineArgs a, cudaStream_t stream) {
    SplitShape s = split_shape(a.N, a.chunks);
    // A short launch (at most ~8 tasks per resident warp of a 3-CTA-per-SM shape) exposes
    // phase 1's round trip at the start of every task: there the LSE prefetch pays for any
    // row length (N = 8, B = 1024, 16 heads, D = 512: 0.87 of the measured peak against 0.81;
    // N = 16: 0.97 against 0.95; at B = 16384 it lost, 1.00 against 1.04).
    if (!s.prefetch) {
        const int64_t tasks = (a.units + 32 / s.G - 1) / (32 / s.G);
        if (tasks <= (int64_t)8 * sm_count() * 3 * (dcp::kCombineThreads / 32)) s.prefetch = true;
    }
    a.slots = (a.chunks + s.G - 1) / s.G;
    if (a.varlen) {
        const SplitShape v = varlen_shape(a.N, a.chunks, s);
        a.slots = (a.chunks + v.G - 1) / v.G;
        if (varlen_all_in_flight(v, a.N, a.chunks))
            return launch_combine<T, 8, 2, 8, false, 2, false, true, false, true>(a, stream);
        return launch_split<T, true, false, true>(a, v, stream);
    }
    if (a.pack_b > 0) {
        // the fused pack's group kernel: D' = 64 or 128 (at 32 the per-row path measured faster)
        if ((a.data_w == 64 || a.data_w == 128) && a.pack_hr % 4 == 0) {
            a.red_lanes = s.G;  // the weights summed as the split combine would (same lanes per row)
            return dispatch_group_pack<T>(a, stream);
        }
        return launch_split<T, false, true, false>(a, pack_shape(a.N, a.chunks, s), stream);
    }
    if (s.prefetch) return launch_split<T, false, false, true>(a, s, stream);
    return launch_split<T, false, false, false>(a, s, stream);
}

}  // namespace dcp_host
