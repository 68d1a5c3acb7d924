// dcp_kernels.cuh -- sm_100a kernels of the DCP LSE-weighted combine.
//
// Memory-bound kernels (no tensor cores: the combine is a weighted sum over N
// shards, ~1 FMA per 2 bytes moved):
//
//   combine_kernel<..., PACKED=false>  combine of split receive buffers (any strides)
//     VARLEN=true                      ... per request: shards without KV are not read
//     PACK_OUT=true                    ... written as packed send rows (split merge + pack)
//   combine_kernel<..., PACKED=true>   fused unpack + combine of the packed buffer (two phases)
//     PREFETCH=true (either layout)    phase 1's reads copied one task ahead
//   online_unpack_kernel               the same in one pass, LSEs arriving with each batch's
//                                      data (packed rows of at most 1 KiB)
//   group_pack_kernel                  split merge written as 4-row spans of packed send rows
//   pack_kernel                        output rows + fp32 LSE -> packed rows (bulk copies)
//   pack_tma_kernel                    the same for long launches, each tile of tokens x a
//                                      rank's heads loaded by one tensor copy
//
// The combine follows vLLM API docs, vllm.v1.attention.ops.dcp_alltoall,
// _lse_weighted_combine; the packed layout [N, B, H/N, D + P] follows the same
// page's dcp_a2a_lse_reduce.
//
// Data are handled as 32-bit words throughout: a bf16/fp16 word holds two
// elements, an fp32 word one.  Every row of D elements is a whole number of
// 16-byte chunks (host-checked), and a packed row is that plus one word (the
// fp32 LSE), so packed rows are 4-byte aligned but in general not 16-byte
// aligned.
#pragma once

#include <cuda.h>  // CUtensorMap (a type only; the library does not link the driver)
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dcp {

constexpr int kMaxShards = 64;
constexpr int kCombineThreads = 256;
constexpr int kPackThreads = 256;

// ---------------------------------------------------------------------------
// element types: decode one 32-bit word into floats, encode floats into a word
struct Bf16 {
    static constexpr int kPerWord = 2;
    __device__ __forceinline__ static void decode(uint32_t w, float *f) {
        f[0] = __uint_as_float(w << 16);
        f[1] = __uint_as_float(w & 0xffff0000u);
    }
    __device__ __forceinline__ static uint32_t encode(const float *f) {
        __nv_bfloat162 v = __floats2bfloat162_rn(f[0], f[1]);  // .x = low half
        return *reinterpret_cast<uint32_t *>(&v);
    }
};

struct Fp16 {
    static constexpr int kPerWord = 2;
    __device__ __forceinline__ static void decode(uint32_t w, float *f) {
        __half2 h = *reinterpret_cast<__half2 *>(&w);
        float2 v = __half22float2(h);
        f[0] = v.x;
        f[1] = v.y;
    }
    __device__ __forceinline__ static uint32_t encode(const float *f) {
        __half2 v = __floats2half2_rn(f[0], f[1]);
        return *reinterpret_cast<uint32_t *>(&v);
    }
};

struct Fp32 {
    static constexpr int kPerWord = 1;
    __device__ __forceinline__ static void decode(uint32_t w, float *f) { f[0] = __uint_as_float(w); }
    __device__ __forceinline__ static uint32_t encode(const float *f) { return __float_as_uint(f[0]); }
};

// ---------------------------------------------------------------------------
// memory access helpers.  Inputs are read-only for the whole kernel, so loads
// take the non-coherent path and do not allocate in L1 (each byte is used once).
template <int VW>
struct Words {
    uint32_t w[VW];
};

template <int VW>
__device__ __forceinline__ Words<VW> load_stream(const uint32_t *p);

template <>
__device__ __forceinline__ Words<4> load_stream<4>(const uint32_t *p) {
    Words<4> r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3])
        : "l"(p));
    return r;
}

template <>
__device__ __forceinline__ Words<1> load_stream<1>(const uint32_t *p) {
    Words<1> r;
    asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r.w[0]) : "l"(p));
    return r;
}

template <int VW>
__device__ __forceinline__ void store_words(uint32_t *p, const Words<VW> &v);

// Stores carry no "memory" clobber: nothing in these kernels reads what they
// write, and a clobber would make the compiler reload every kernel argument
// after each store.
template <>
__device__ __forceinline__ void store_words<4>(uint32_t *p, const Words<4> &v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.w[0]), "r"(v.w[1]), "r"(v.w[2]),
                 "r"(v.w[3]));
}

template <>
__device__ __forceinline__ void store_words<1>(uint32_t *p, const Words<1> &v) {
    asm volatile("st.global.u32 [%0], %1;" ::"l"(p), "r"(v.w[0]));
}

__device__ __forceinline__ uint32_t load_word(const uint32_t *p) {
    uint32_t r;
    asm("ld.global.nc.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Asynchronous copies into shared memory.  They need no "memory" clobber: reads
// of the copied words are ordered by cp.async.wait_group (which has one) and the
// barrier after it.
__device__ __forceinline__ void cp_async_word(uint32_t *s, const uint32_t *g) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(s)), "l"(g));
}

__device__ __forceinline__ void cp_async_chunk(void *s, const uint32_t *g) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(s)), "l"(g));
}

// The 16-byte chunk at word w of a 16-byte aligned buffer into shared memory, copying
// only the words below `limit` (the rest of the destination is zero-filled, and nothing
// at or past `limit` is read).  At least one word must lie below `limit`.
__device__ __forceinline__ void cp_async_chunk_bounded(void *s, const uint32_t *base, int64_t w, int64_t limit) {
    const int64_t left = limit - w;
    const uint32_t bytes = left >= 4 ? 16u : (uint32_t)(4 * left);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(s)), "l"(base + w), "r"(bytes));
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int PENDING>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(PENDING) : "memory");
}

// mbarrier and bulk-copy helpers (shared-memory barrier objects, 8 bytes each).
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the copy engine.
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

// Orders this thread's earlier shared-memory accesses before its later bulk copies.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Pack CTAs whose wait for a tile's copies timed out: counted here, read (and cleared) by
// the host with dcp_wait_timeouts.
// Internal to each translation unit: the pack kernel and dcp_wait_timeouts share one.
static __device__ unsigned long long g_wait_timeouts = 0;

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // one second

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits for the barrier's phase with the given parity; false when limit_ns pass (or the
// iteration cap is reached) first.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t spin = 0; spin < (1u << 26); ++spin) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > limit_ns) break;
    }
    return false;
}

// Global -> shared bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned),
// completing as transaction bytes on `bar`.
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(dst)),
                 "l"(src), "r"(bytes), "r"(smem_addr(bar))
                 : "memory");
}

// n / d for n < 2^32 and d <= 2^32, with magic = ceil(2^64 / d) (0 meaning d == 1).
__device__ __forceinline__ uint64_t div_magic(uint64_t n, uint64_t magic) {
    return magic ? __umul64hi(n, magic) : n;
}

// An LSE that is NaN or +-inf becomes -inf; classified on the exponent bits so
// the rule holds under any compiler math flags.
__device__ __forceinline__ float sanitize_lse(uint32_t bits) {
    return ((bits & 0x7f800000u) == 0x7f800000u) ? -INFINITY : __uint_as_float(bits);
}

template <int G>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <int G>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// ---------------------------------------------------------------------------
// combine
struct CombineArgs {
    const uint32_t *src;     // split: outputs; packed: receive buffer (as words)
    const float *lses;       // split layout only
    uint32_t *result;        // result rows (as words)
    float *glse;             // global LSEs, written when return_lse
    int64_t units;           // rows of the result (B * heads)
    int64_t shard_stride_w;  // words between consecutive shards
    int64_t lse_stride_n;    // split layout: floats between consecutive shards
    int64_t row_pitch_w;     // packed layout: words between consecutive rows of one shard
    int64_t total_w;         // packed layout: words of the buffer that may be read
    // split layout: row (b, h) of a shard at b*src_sb_w + h*src_sh_w, its LSE at
    // b*lse_sb + h*lse_sh, the result row at b*res_sb_w + h*res_sh_w and the global
    // LSE at b*glse_sb + h*glse_sh.  The packed layout's result is [units, data_w]
    // and its global LSE [units], contiguous.
    int64_t heads;           // H: unit u is (b, h) = (u / H, u mod H)
    uint64_t heads_magic;    // ceil(2^64 / H), 0 when H == 1
    int64_t src_sb_w, src_sh_w;
    int64_t lse_sb, lse_sh;
    int64_t res_sb_w, res_sh_w;
    int64_t glse_sb, glse_sh;
    int32_t data_w;          // words of data per row (D * elemsize / 4), a multiple of 4
    int32_t chunks;          // data_w / 4: 16-byte chunks per row
    int32_t slots;           // ceil(chunks / G): chunk slots per lane
    int32_t N;
    int32_t base_e;
    int32_t return_lse;
    // split layout, variable length (varlen != 0, the VARLEN kernels): token b belongs to the request r
    // with qsl[r] <= b < qsl[r + 1] (num_reqs + 1 non-decreasing entries); shard n
    // holds KV of that request iff n * interleave < seq_lens[r].  A shard without
    // KV counts as LSE -inf and its row is not read; a token outside every request
    // combines no shard at all.
    // PACK_OUT (split layout in, the packed send layout out): unit (b, h) of the H = heads
    // input heads is written as packed row ((h / pack_hr) * pack_b + b) * pack_hr + h mod
    // pack_hr, data_w + 1 words per row, the merged fp32 LSE in its last word.
    int64_t pack_b;
    int64_t pack_hr;
    uint64_t pack_hr_magic;  // ceil(2^64 / pack_hr), 0 when pack_hr == 1
    int32_t red_lanes;       // group_pack_kernel: lanes that reduce one row's LSEs (4, 8, 16, 32)
    int32_t varlen;
    int32_t num_reqs;
    int32_t interleave;
    const int32_t *seq_lens;
    const int32_t *qsl;
};

// Variable-length combine: the shards that hold KV for a token are shards [0, k) of its
// request, k = ceil(seq / interleave) capped at N (under interleaved sharding, blocks of
// `interleave` positions dealt round-robin, shard n holds positions iff
// n * interleave < seq); a token outside every request has none.
__device__ __forceinline__ int varlen_held_shards(const CombineArgs &a, int32_t seq) {
    if (seq <= 0) return 0;
    // interleave 1 (token-by-token sharding, the default) needs no division
    const int32_t k = a.interleave == 1 ? seq : (seq - 1) / a.interleave + 1;
    return k < a.N ? k : a.N;
}

__device__ __forceinline__ int clamp_req(int64_t q, int R) { return (int)(q < 0 ? 0 : q > R - 1 ? R - 1 : q); }

// The request a token's position interpolates to: b * R / qsl[R] (r_per_token = R / qsl[R]),
// clamped to [0, R - 1].  Exact for plain decode (request r is token r) and for any batch
// whose requests all have the same number of query tokens.
__device__ __forceinline__ int varlen_guess(int64_t b, int R, int64_t qsl_end, float r_per_token) {
    return clamp_req(b < qsl_end ? (int64_t)((float)b * r_per_token) : (int64_t)R - 1, R);
}

// The request r with qsl[r] <= b < qsl[r + 1] for the rows whose `active` is set (-1 if
// none), and its seq_lens entry.  The G lanes of a row search together.  Each round every
// lane probes one position (reading qsl and seq_lens there), a vote counts the probes <= b,
// and the range left for the first start > b shrinks to the gap between two neighbouring
// probes.  Round 0 probes the G consecutive requests around varlen_guess; later rounds split
// the range evenly, (G+1)-ary.  The seq_lens entry comes from the lane that probed r last
// (else it is read).  All 32 lanes call this (it votes); every read stays inside
// qsl[0..R - 1] and seq_lens[0..R), and it ends after at most 64 rounds whatever qsl holds.
// An active row needs b < qsl_end = qsl[R].
template <int G>
__device__ __forceinline__ int varlen_search(const CombineArgs &a, int64_t b, bool active_row, int j,
                                            int64_t qsl_end, float r_per_token, int32_t &seq) {
    const int R = a.num_reqs;
    const int lane = threadIdx.x & 31;
    const unsigned gmask = (G == 32 ? 0xffffffffu : ((1u << G) - 1u)) << (lane & (32 - G));
    const int64_t window = (int64_t)varlen_guess(b, R, qsl_end, r_per_token) - (G / 2 - 1);
    // the first r in [0, R) with qsl[r] > b (R if none) lies in [lo, hi]
    int lo = 0, hi = active_row ? R : 0;
    int last_p = -1;
    int32_t last_s = 0;
    for (int round = 0; round < 64 && __any_sync(0xffffffffu, lo < hi); ++round) {
        const bool active = lo < hi;  // the same for the G lanes of a row
        auto probe = [&](int jj) -> int {
            if (round == 0) return clamp_req(window + jj, R);  // lo = 0, hi = R
            const int64_t q = lo + ((int64_t)(jj + 1) * (hi - lo)) / (G + 1);
            return (int)(q > hi - 1 ? hi - 1 : q);
        };
        bool le = false;
        if (active) {
            last_p = probe(j);
            le = (int64_t)__ldg(a.qsl + last_p) <= b;
            last_s = __ldg(a.seq_lens + last_p);
        }
        const int c = __popc(__ballot_sync(0xffffffffu, le) & gmask);
        if (active) {
            const int nlo = c == 0 ? lo : probe(c - 1) + 1;
            const int nhi = c == G ? hi : probe(c);
            hi = nhi;
            lo = nlo < nhi ? nlo : nhi;  // nlo > nhi only when qsl is not non-decreasing
        }
    }
    // b < qsl_end, so lo >= 1 means b lies in request lo - 1
    const int r = active_row ? lo - 1 : -1;
    const unsigned hit = __ballot_sync(0xffffffffu, r >= 0 && last_p == r) & gmask;
    seq = __shfl_sync(0xffffffffu, last_s, hit ? __ffs(hit) - 1 : lane);
    if (r >= 0 && !hit) seq = __ldg(a.seq_lens + r);
    return r;
}

// Shards holding KV for token b (0 for an inactive row): shards [0, k) of its request,
// k = ceil(seq / interleave) capped at N; 0 when b lies in no request.  q_lo, q_hi, s_g are
// qsl[g], qsl[g + 1] and seq_lens[g] for g = varlen_guess(b), fetched one task ahead: when
// request g holds b nothing else is read; otherwise the row's lanes run varlen_search.  All
// 32 lanes call this.  full_seq = (N - 1) * interleave.
template <int G>
__device__ __forceinline__ int varlen_shards(const CombineArgs &a, int64_t b, bool active_row, int j, int64_t qsl_end,
                                             float r_per_token, int64_t full_seq, int32_t q_lo, int32_t q_hi,
                                             int32_t s_g) {
    const bool searched = active_row && a.num_reqs > 0 && b < qsl_end;
    bool found = searched && (int64_t)q_lo <= b && b < (int64_t)q_hi;
    int32_t seq = s_g;
    const bool need = searched && !found;
    if (__any_sync(0xffffffffu, need)) {
        int32_t s_r;
        const int r = varlen_search<G>(a, b, need, j, qsl_end, r_per_token, s_r);
        if (need) {
            found = r >= 0;
            seq = s_r;
        }
    }
    if (!found) return 0;
    if ((int64_t)seq > full_seq) return a.N;  // the usual case: KV on every shard
    return varlen_held_shards(a, seq);
}

// The 4 words that start at word q (0..3) of the 8-word window (lo, hi).
__device__ __forceinline__ Words<4> funnel_words(const Words<4> &lo, const Words<4> &hi, int q) {
    uint32_t a0 = lo.w[0], a1 = lo.w[1], a2 = lo.w[2], a3 = lo.w[3], a4 = hi.w[0], a5 = hi.w[1], a6 = hi.w[2];
    if (q & 2) {
        a0 = a2; a1 = a3; a2 = a4; a3 = a5; a4 = a6;
    }
    if (q & 1) {
        a0 = a1; a1 = a2; a2 = a3; a3 = a4;
    }
    Words<4> r;
    r.w[0] = a0; r.w[1] = a1; r.w[2] = a2; r.w[3] = a3;
    return r;
}

// The 16-byte chunk at word w of a 16-byte aligned buffer, reading no word at or
// beyond `limit` (those come back as 0): the buffer's last row may end inside a chunk.
__device__ __forceinline__ Words<4> load_chunk_bounded(const uint32_t *base, int64_t w, int64_t limit) {
    if (w + 4 <= limit) return load_stream<4>(base + w);
    Words<4> r;
#pragma unroll
    for (int e = 0; e < 4; ++e) r.w[e] = (w + e < limit) ? load_word(base + w + e) : 0u;
    return r;
}

// Shared memory of one combine CTA: per warp and per row in flight, the N normalised
// weights and what phase 1 reads for N shards: the rows' aligned tail chunks (packed
// layout), and with `prefetch` two buffers of them (or of the LSE words, split layout),
// filled one task ahead.
__host__ __device__ constexpr size_t combine_smem_bytes(int units_per_warp, int N, bool packed, bool prefetch) {
    return (size_t)(kCombineThreads / 32) * units_per_warp * N *
           (sizeof(float) + (prefetch ? 2 : 1) * (packed ? 16 : 0) + (prefetch && !packed ? 2 * 4 : 0));
}

// One warp works on 32/G result rows at a time, G lanes per row; lane j of a row
// owns its 16-byte chunks j, j+G, j+2G, ... (slots), CPL slots per pass.
//   1. The loads of the first NB shards' chunks are issued.
//   2. Phase 1 (weights): lane j takes shards j, j+G, ...; it reads each LSE
//      (split: from the LSE array; packed: from the row's tail chunk, which is
//      kept in shared memory; with PREFETCH both were copied there while the
//      previous task ran), sanitises it by exponent bits, and the G lanes
//      reduce max and sum with xor-shuffles.  The normalised weights go to
//      shared memory; lane 0 writes the global LSE (PACK_OUT: into the packed
//      row's last word).
//   3. Phase 2 (weighted sum): fp32 FMAs over all N shards, NB shards' loads
//      in flight at a time, then one rounding and a 16-byte store per chunk
//      (PACK_OUT: realigned to the packed row, see below).
// VARLEN: before step 1 the row's lanes find the number of shards holding KV
// (varlen_shards); loads and LSE reads of the other shards are skipped.
// Packed rows are 2D+4 bytes, so a row starts q = 0..3 words past a 16-byte
// boundary.  Lanes load aligned chunks; output chunk c is the 4 words at offset
// q of aligned chunks c and c+1, and aligned chunk c+1 comes from the next lane
// by shuffle (lane G-1 takes lane 0's next slot), or from the tail chunk in
// shared memory for the row's last chunk.
// UNIFORM (packed, every shard's rows at the same offset q -- shard strides a
// multiple of 16 bytes -- and one pass): the lanes accumulate the aligned chunks
// as they are, and only the fp32 sums are realigned, once per output chunk:
// output chunk c is elements 2q/e.. of sum c and the first ones of sum c+1 (from
// the next lane, or, for the last chunk, the weighted sum of the tail chunks,
// formed in phase 1 and reduced over the lane group).
template <class T, int G, int CPL, int NB, bool PACKED, int MIN_CTAS = 1, bool UNIFORM = false, bool VARLEN = false,
          bool PACK_OUT = false, bool PREFETCH = false>
__global__ void __launch_bounds__(kCombineThreads, MIN_CTAS) combine_kernel(const CombineArgs a) {
    static_assert(!VARLEN || PREFETCH, "the variable-length combine prefetches its request guesses");
    constexpr int kUnitsPerWarp = 32 / G;
    constexpr int kWarps = kCombineThreads / 32;
    constexpr int kElems = 4 * T::kPerWord;
    extern __shared__ uint4 s_dyn[];

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int ul = lane / G;
    const int j = lane % G;
    const int next_lane = (lane & ~(G - 1)) | ((j + 1) & (G - 1));
    const int slot_base = warp * kUnitsPerWarp + ul;
    constexpr int kRows = kWarps * kUnitsPerWarp;  // rows in flight per CTA
    constexpr int kBufs = PREFETCH ? 2 : 1;
    // packed: tail chunks [kBufs][kRows][N] (uint4); split with PREFETCH: LSE words
    // [2][kRows][N]; then the weights [kRows][N]
    uint4 *s_tail_all = s_dyn;
    uint32_t *s_lse = reinterpret_cast<uint32_t *>(s_dyn);
    float *sw = reinterpret_cast<float *>(s_dyn) +
                (size_t)kRows * a.N * (PACKED ? 4 * kBufs : (PREFETCH ? 2 : 0)) + (size_t)slot_base * a.N;
    const int64_t tasks = (a.units + kUnitsPerWarp - 1) / kUnitsPerWarp;
    // What phase 1 reads for each row's next task -- the LSE words (split layout) or the
    // rows' aligned tail chunks, which hold the LSE (packed layout) -- is copied into shared
    // memory one task ahead (two buffers, alternating), so phase 1 waits on no global read.
    // VARLEN: lane 0 of the row also copies qsl[g], qsl[g + 1] and seq_lens[g]
    // (g = varlen_guess) of the next token.  One copy group per task.
    __shared__ int32_t s_probe[VARLEN ? 2 : 1][VARLEN ? 3 * kRows : 1];
    int64_t qsl_end = 0;
    float r_per_token = 0.0f;
    const int64_t full_seq = (int64_t)(a.N - 1) * a.interleave;
    int buf = 0;
    auto prefetch = [&](int64_t t, int into) {
        const int64_t uu = t * kUnitsPerWarp + ul;
        if (uu < a.units) {
            if constexpr (PACKED) {
                uint4 *dst = s_tail_all + ((size_t)into * kRows + slot_base) * a.N;
                const int64_t rw = uu * a.row_pitch_w;  // the row's first word in shard 0
                for (int n = j; n < a.N; n += G) {
                    const int64_t wa = ((int64_t)n * a.shard_stride_w + rw) & ~int64_t(3);
                    cp_async_chunk_bounded(dst + n, a.src, wa + 4 * (int64_t)a.chunks, a.total_w);
                }
            } else {
                uint32_t *dst = s_lse + ((size_t)into * kRows + slot_base) * a.N;
                const int64_t bb = (int64_t)div_magic((uint64_t)uu, a.heads_magic);
                const int64_t lo = bb * a.lse_sb + (uu - bb * a.heads) * a.lse_sh;
                const uint32_t *lses = reinterpret_cast<const uint32_t *>(a.lses);
                for (int n = j; n < a.N; n += G) cp_async_word(dst + n, lses + n * a.lse_stride_n + lo);
                if constexpr (VARLEN) {
                    if (j == 0 && a.num_reqs > 0) {
                        const int g = varlen_guess(bb, a.num_reqs, qsl_end, r_per_token);
                        uint32_t *d = reinterpret_cast<uint32_t *>(&s_probe[into][3 * slot_base]);
                        cp_async_word(d, reinterpret_cast<const uint32_t *>(a.qsl + g));
                        cp_async_word(d + 1, reinterpret_cast<const uint32_t *>(a.qsl + g + 1));
                        cp_async_word(d + 2, reinterpret_cast<const uint32_t *>(a.seq_lens + g));
                    }
                }
            }
        }
        cp_async_commit();
    };
    if constexpr (VARLEN) {
        if (a.num_reqs > 0) {
            qsl_end = __ldg(a.qsl + a.num_reqs);
            if (qsl_end > 0) r_per_token = (float)a.num_reqs / (float)qsl_end;
        }
    }
    if constexpr (PREFETCH) prefetch((int64_t)blockIdx.x * kWarps + warp, 0);

    for (int64_t task = (int64_t)blockIdx.x * kWarps + warp; task < tasks; task += (int64_t)gridDim.x * kWarps) {
        const int64_t u = task * kUnitsPerWarp + ul;
        const bool valid = u < a.units;
        int64_t row, res_off, glse_off, lse_off = 0;
        int nk = a.N;  // shards [0, nk) are read; the rest weigh 0
        if constexpr (PACKED) {
            row = u * a.row_pitch_w;
            res_off = u * a.data_w;
            glse_off = u;
        } else {
            const int64_t b = (int64_t)div_magic((uint64_t)u, a.heads_magic);
            const int64_t h = u - b * a.heads;
            row = b * a.src_sb_w + h * a.src_sh_w;
            lse_off = b * a.lse_sb + h * a.lse_sh;
            res_off = b * a.res_sb_w + h * a.res_sh_w;
            glse_off = b * a.glse_sb + h * a.glse_sh;
            if constexpr (PACK_OUT) {
                const int64_t rank = (int64_t)div_magic((uint64_t)h, a.pack_hr_magic);
                res_off = ((rank * a.pack_b + b) * a.pack_hr + (h - rank * a.pack_hr)) * (int64_t)(a.data_w + 1);
            }
            if constexpr (VARLEN) {
                cp_async_wait<0>();  // this task's prefetch (lane 0's guess copies among them)
                __syncwarp();
                const int32_t *pr = &s_probe[buf][3 * slot_base];
                nk = varlen_shards<G>(a, b, valid, j, qsl_end, r_per_token, full_seq, pr[0], pr[1], pr[2]);
            }
        }

        int c[CPL];
        bool act[CPL];
        Words<4> x[NB][CPL];
        int qv[NB];

        auto set_pass = [&](int s0) {
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                c[k] = j + G * (s0 + k);
                act[k] = valid && c[k] < a.chunks;
            }
        };
        auto issue = [&](int n0) {
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                const int64_t w0 = (int64_t)(n0 + i) * a.shard_stride_w + row;
                const int64_t wa = PACKED ? (w0 & ~int64_t(3)) : w0;
                qv[i] = (int)(w0 & 3);
#pragma unroll
                for (int k = 0; k < CPL; ++k) {
                    if (n0 + i < nk && act[k]) {
                        x[i][k] = load_stream<4>(a.src + wa + 4 * c[k]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) x[i][k].w[e] = 0u;
                    }
                }
            }
        };

        set_pass(0);
        issue(0);
        if constexpr (PREFETCH) prefetch(task + (int64_t)gridDim.x * kWarps, buf ^ 1);
        uint4 *s_tail = s_tail_all + ((size_t)buf * kRows + slot_base) * a.N;  // packed: this task's tails

        // ---- phase 1: weights of the N shards --------------------------------
        if constexpr (PREFETCH) cp_async_wait<1>();  // this task's copies (each lane reads the ones it made)
        const uint32_t *lse_now = s_lse + ((size_t)buf * kRows + slot_base) * a.N;
        float lmax = -INFINITY;
        for (int n = j; n < a.N; n += G) {
            float l = -INFINITY;
            if (valid && n < nk) {
                uint32_t bits;
                const int64_t w0 = (int64_t)n * a.shard_stride_w + row;
                if constexpr (PACKED) {
                    uint4 t;
                    if constexpr (PREFETCH) {
                        t = s_tail[n];
                    } else {
                        const Words<4> v = load_chunk_bounded(a.src, (w0 & ~int64_t(3)) + 4 * (int64_t)a.chunks, a.total_w);
                        t = make_uint4(v.w[0], v.w[1], v.w[2], v.w[3]);
                        s_tail[n] = t;
                    }
                    const int q = (int)(w0 & 3);
                    bits = q == 0 ? t.x : q == 1 ? t.y : q == 2 ? t.z : t.w;
                } else {
                    if constexpr (PREFETCH) {
                        bits = lse_now[n];
                    } else {
                        bits = load_word(reinterpret_cast<const uint32_t *>(a.lses) + n * a.lse_stride_n + lse_off);
                    }
                }
                l = sanitize_lse(bits);
            }
            sw[n] = l;
            lmax = fmaxf(lmax, l);
        }
        lmax = group_max<G>(lmax);
        const float m = (lmax == -INFINITY) ? 0.0f : lmax;
        float wsum = 0.0f;
        for (int n = j; n < a.N; n += G) {
            const float x1 = sw[n] - m;
            float w = a.base_e ? expf(x1) : exp2f(x1);
            if (w != w) w = 0.0f;
            sw[n] = w;
            wsum += w;
        }
        wsum = group_sum<G>(wsum);
        const float denom = fmaxf(wsum, 1e-10f);
        for (int n = j; n < a.N; n += G) sw[n] = sw[n] / denom;
        if constexpr (PACK_OUT) {
            if (valid && j == 0) {
                Words<1> lw;
                lw.w[0] = __float_as_uint((a.base_e ? logf(wsum) : log2f(wsum)) + m);
                store_words<1>(a.result + res_off + a.data_w, lw);
            }
        } else {
            if (a.return_lse && valid && j == 0) a.glse[glse_off] = (a.base_e ? logf(wsum) : log2f(wsum)) + m;
        }

        // UNIFORM: weighted sum of the shards' tail chunks.  With few shards the lane
        // that owns the row's last chunk sums them itself; otherwise each lane sums its
        // shards and the group reduces.
        __syncwarp();  // lanes read the weights and tail chunks other lanes wrote
        float tacc[kElems];
        if constexpr (PACKED && UNIFORM) {
#pragma unroll
            for (int e = 0; e < kElems; ++e) tacc[e] = 0.0f;
            const bool few = a.N <= 4;  // the same for the whole warp
            const int n_first = few ? 0 : j;
            const int n_step = few ? 1 : G;
            const bool owner = j == (a.chunks - 1) % G;
            for (int n = n_first; n < a.N && (!few || owner); n += n_step) {
                const uint4 t = s_tail[n];
                const float w = sw[n];
                const uint32_t tw[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float f[T::kPerWord];
                    T::decode(tw[e], f);
#pragma unroll
                    for (int h = 0; h < T::kPerWord; ++h)
                        tacc[e * T::kPerWord + h] = fmaf(w, f[h], tacc[e * T::kPerWord + h]);
                }
            }
            // only the first 3 words (the most a row can leave in its tail chunk) matter
            if (!few) {
#pragma unroll
                for (int e = 0; e < 3 * T::kPerWord; ++e) tacc[e] = group_sum<G>(tacc[e]);
            }
        }
        __syncwarp();

        // ---- phase 2: weighted sum of the N rows -------------------------------
        for (int s0 = 0; s0 < a.slots; s0 += CPL) {
            if (s0 > 0) {
                set_pass(s0);
                issue(0);
            }
            float acc[CPL][kElems];
#pragma unroll
            for (int k = 0; k < CPL; ++k)
#pragma unroll
                for (int e = 0; e < kElems; ++e) acc[k][e] = 0.0f;
            const bool more_passes = s0 + CPL < a.slots;
            for (int n0 = 0; n0 < a.N; n0 += NB) {
                if (n0 > 0) issue(n0);
#pragma unroll
                for (int i = 0; i < NB; ++i) {
                    if (n0 + i >= a.N) break;  // uniform across the warp
                    const int n = n0 + i;
                    const float w = sw[n];
#pragma unroll
                    for (int k = 0; k < CPL; ++k) {
                        Words<4> v = x[i][k];
                        if constexpr (PACKED && !UNIFORM) {
                            // aligned chunk c+1: lane j+1's slot k, or lane 0's slot k+1 for lane G-1
                            Words<4> send = x[i][k];
                            if (k + 1 < CPL && j == 0) send = x[i][k + 1];
                            Words<4> nx;
#pragma unroll
                            for (int e = 0; e < 4; ++e) nx.w[e] = __shfl_sync(0xffffffffu, send.w[e], next_lane);
                            if (act[k] && c[k] == a.chunks - 1) {
                                const uint4 t = s_tail[n];
                                nx.w[0] = t.x; nx.w[1] = t.y; nx.w[2] = t.z; nx.w[3] = t.w;
                            } else if (act[k] && k == CPL - 1 && j == G - 1 && more_passes) {
                                const int64_t wa = ((int64_t)n * a.shard_stride_w + row) & ~int64_t(3);
                                nx = load_stream<4>(a.src + wa + 4 * (c[k] + 1));
                            }
                            v = funnel_words(v, nx, qv[i]);
                        }
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float f[T::kPerWord];
                            T::decode(v.w[e], f);
#pragma unroll
                            for (int h = 0; h < T::kPerWord; ++h)
                                acc[k][e * T::kPerWord + h] = fmaf(w, f[h], acc[k][e * T::kPerWord + h]);
                        }
                    }
                }
            }
            if constexpr (PACKED && UNIFORM) {
                // Round the aligned sums to output words first (rounding is per element,
                // so it commutes with a whole-word shift), then funnel by q words: output
                // chunk c = words q.. of sums c and c+1; sum c+1 comes from the next lane
                // (lane 0's next slot for lane G-1, the tail sum for the row's last chunk).
                const int q = qv[0];  // the same for every shard
                Words<4> enc[CPL];
#pragma unroll
                for (int k = 0; k < CPL; ++k)
#pragma unroll
                    for (int e = 0; e < 4; ++e) enc[k].w[e] = T::encode(&acc[k][e * T::kPerWord]);
                Words<4> tenc;
#pragma unroll
                for (int e = 0; e < 3; ++e) tenc.w[e] = T::encode(&tacc[e * T::kPerWord]);
                tenc.w[3] = 0u;
#pragma unroll
                for (int k = 0; k < CPL; ++k) {
                    Words<4> send = enc[k];
                    if (k + 1 < CPL && j == 0) send = enc[k + 1 < CPL ? k + 1 : k];
                    Words<4> nx;
#pragma unroll
                    for (int e = 0; e < 3; ++e) nx.w[e] = __shfl_sync(0xffffffffu, send.w[e], next_lane);
                    nx.w[3] = 0u;
                    if (act[k] && c[k] == a.chunks - 1) nx = tenc;
                    if (act[k]) store_words<4>(a.result + res_off + 4 * (int64_t)c[k], funnel_words(enc[k], nx, q));
                }
            } else if constexpr (PACK_OUT) {
                // The packed row starts q = res_off mod 4 words past a 16-byte boundary.
                // Interior: the aligned chunk at row word 4c + 4 - q is words 4 - q.. of
                // output chunk c and the first q words of chunk c + 1 (from the next lane,
                // lane 0's next slot for lane G-1).  The row's first 4 - q and last q words
                // are written one by one, so no store touches a neighbouring row.  Rows that
                // take more than one pass are written word by word.
                const int q = (int)(res_off & 3);
                uint32_t *rowp = a.result + res_off;
                Words<4> enc[CPL];
#pragma unroll
                for (int k = 0; k < CPL; ++k)
#pragma unroll
                    for (int e = 0; e < 4; ++e) enc[k].w[e] = T::encode(&acc[k][e * T::kPerWord]);
                if (a.slots <= CPL) {  // one pass: every chunk of the row is in registers
#pragma unroll
                    for (int k = 0; k < CPL; ++k) {
                        Words<4> send = enc[k];
                        if (k + 1 < CPL && j == 0) send = enc[k + 1 < CPL ? k + 1 : k];
                        Words<4> nx;
#pragma unroll
                        for (int e = 0; e < 3; ++e) nx.w[e] = __shfl_sync(0xffffffffu, send.w[e], next_lane);
                        nx.w[3] = 0u;
                        if (!act[k]) continue;
                        const int cc = c[k];
                        if (q == 0) {
                            store_words<4>(rowp + 4 * cc, enc[k]);
                            continue;
                        }
                        if (cc + 1 < a.chunks) store_words<4>(rowp + 4 * cc + 4 - q, funnel_words(enc[k], nx, 4 - q));
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const bool head = cc == 0 && e < 4 - q;
                            const bool tail = cc + 1 == a.chunks && e >= 4 - q;
                            if (head || tail) {
                                Words<1> wv;
                                wv.w[0] = enc[k].w[e];
                                store_words<1>(rowp + 4 * cc + e, wv);
                            }
                        }
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < CPL; ++k) {
                        if (!act[k]) continue;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            Words<1> wv;
                            wv.w[0] = enc[k].w[e];
                            store_words<1>(rowp + 4 * c[k] + e, wv);
                        }
                    }
                }
            } else {
#pragma unroll
                for (int k = 0; k < CPL; ++k) {
                    if (act[k]) {
                        Words<4> o;
#pragma unroll
                        for (int e = 0; e < 4; ++e) o.w[e] = T::encode(&acc[k][e * T::kPerWord]);
                        store_words<4>(a.result + res_off + 4 * (int64_t)c[k], o);
                    }
                }
            }
        }
        __syncwarp();
        if constexpr (PREFETCH) buf ^= 1;
    }
    if constexpr (PREFETCH) cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// single-pass unpack + combine of packed rows (uniform shard stride, one pass per row)
//
// The two-phase kernel must read every shard's LSE (the row's tail chunk) before it can weight
// any data, and with the LSE inside the data stream that read is a DRAM round trip of its own
// per task.  Here each batch of NB shards brings its LSEs with its data: lane j < NB of a row
// also loads shard n0 + j's tail chunk, which holds the row's LSE (word q, q = the row's word
// offset from a 16-byte boundary) and up to 3 of its last data words.  The combine rules are
// applied to the running state (m, S, sums) batch by batch:
//   l_n <- -inf if NaN or +-inf;  m' = max(m, max over the batch);
//   c = exp(m - m') (1 while m' is still -inf);  w_n = exp(l_n - m'), NaN -> 0;
//   S <- c S + sum w_n;  sums <- c sums + sum w_n o_n.
// At the end the sums are divided by max(S, 1e-10) and the global LSE is ln S + m (log2 in
// base 2; m taken as 0 when every LSE was -inf).  This is the page's arithmetic with the
// weights formed against the running maximum and rescaled to the final one, so it differs from
// the two-phase result by fp32 rounding only.  Row layout, realignment and stores are those of
// combine_kernel's uniform packed path (G lanes per row, CPL chunk slots per lane).
// SINGLE (N <= NB, so one batch holds every shard): the batch's maximum is the row's, its weight
// sum is the row's S, and the weights are normalised before the weighted sum, in the page's
// order, instead of rescaling the sums at the end.
template <class T, int G, int CPL, int NB, int MIN_CTAS, bool SINGLE = false>
__global__ void __launch_bounds__(kCombineThreads, MIN_CTAS) online_unpack_kernel(const CombineArgs a) {
    static_assert(NB <= G, "each shard of a batch needs a lane to read its tail chunk");
    constexpr int kUnitsPerWarp = 32 / G;
    constexpr int kWarps = kCombineThreads / 32;
    constexpr int kE = 4 * T::kPerWord;
    const int lane = threadIdx.x & 31;
    const int ul = lane / G;
    const int j = lane % G;
    const int row_lane0 = lane - j;
    const int next_lane = (lane & ~(G - 1)) | ((j + 1) & (G - 1));
    const int64_t tasks = (a.units + kUnitsPerWarp - 1) / kUnitsPerWarp;
    const bool base_e = a.base_e != 0;

    for (int64_t task = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); task < tasks;
         task += (int64_t)gridDim.x * kWarps) {
        const int64_t u = task * kUnitsPerWarp + ul;
        const bool valid = u < a.units;
        const int64_t row = u * a.row_pitch_w;  // the row's first word in shard 0
        const int q = (int)(row & 3);             // the same in every shard (uniform stride)
        const int64_t wa0 = row - q;              // the row's aligned window in shard 0
        int c[CPL];
        bool act[CPL];
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
            c[k] = j + G * k;
            act[k] = valid && c[k] < a.chunks;
        }
        Words<4> x[NB][CPL];
        Words<4> t;  // lane j < NB: the tail chunk of shard n0 + j
        auto issue = [&](int n0) {
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                const int64_t wa = (int64_t)(n0 + i) * a.shard_stride_w + wa0;
#pragma unroll
                for (int k = 0; k < CPL; ++k) {
                    if (n0 + i < a.N && act[k]) {
                        x[i][k] = load_stream<4>(a.src + wa + 4 * c[k]);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) x[i][k].w[e] = 0u;
                    }
                }
            }
            if (valid && j < NB && n0 + j < a.N) {
                t = load_chunk_bounded(a.src, (int64_t)(n0 + j) * a.shard_stride_w + wa0 + 4 * (int64_t)a.chunks, a.total_w);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) t.w[e] = 0u;
            }
        };
        issue(0);

        float m = -INFINITY, S = 0.0f;
        float acc[CPL][kE];
#pragma unroll
        for (int k = 0; k < CPL; ++k)
#pragma unroll
            for (int e = 0; e < kE; ++e) acc[k][e] = 0.0f;
        float tacc[3 * T::kPerWord];  // this lane's shards: weighted sum of the tail chunks' first 3 words
#pragma unroll
        for (int e = 0; e < 3 * T::kPerWord; ++e) tacc[e] = 0.0f;
        // the tail chunk's first 3 words, weighted into tacc
        auto add_tail = [&](float w) {
            const uint32_t tw[3] = {t.w[0], t.w[1], t.w[2]};
#pragma unroll
            for (int e = 0; e < 3; ++e) {
                float f[T::kPerWord];
                T::decode(tw[e], f);
#pragma unroll
                for (int h = 0; h < T::kPerWord; ++h)
                    tacc[e * T::kPerWord + h] = fmaf(w, f[h], tacc[e * T::kPerWord + h]);
            }
        };
        auto add_rows = [&](int i, float wi) {
#pragma unroll
            for (int k = 0; k < CPL; ++k)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float f[T::kPerWord];
                    T::decode(x[i][k].w[e], f);
#pragma unroll
                    for (int h = 0; h < T::kPerWord; ++h)
                        acc[k][e * T::kPerWord + h] = fmaf(wi, f[h], acc[k][e * T::kPerWord + h]);
                }
        };
        float r = 1.0f;  // the normalisation still to apply to the sums (1: already in the weights)
        if constexpr (SINGLE) {
            const bool mine = valid && j < a.N;
            const uint32_t lbits = q == 0 ? t.w[0] : q == 1 ? t.w[1] : q == 2 ? t.w[2] : t.w[3];
            const float l = mine ? sanitize_lse(lbits) : -INFINITY;
            m = group_max<G>(l);
            float w = base_e ? expf(l - m) : exp2f(l - m);
            if (w != w) w = 0.0f;
            if (!mine) w = 0.0f;
            float wv[NB];
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                wv[i] = 0.0f;
                if (i >= a.N) break;  // the same for the whole warp
                wv[i] = __shfl_sync(0xffffffffu, w, row_lane0 + i);
                S += wv[i];
            }
            const float rn = 1.0f / fmaxf(S, 1e-10f);
            add_tail(w * rn);
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                if (i >= a.N) break;  // the same for the whole warp
                add_rows(i, wv[i] * rn);
            }
        } else {
            for (int n0 = 0; n0 < a.N; n0 += NB) {
                if (n0 > 0) issue(n0);
                // the batch's LSEs, its maximum and the rescaling of the running state
                const bool mine = valid && j < NB && n0 + j < a.N;
                const uint32_t lbits = q == 0 ? t.w[0] : q == 1 ? t.w[1] : q == 2 ? t.w[2] : t.w[3];
                const float l = mine ? sanitize_lse(lbits) : -INFINITY;
                const float bmax = group_max<G>(l);
                const float mn = fmaxf(m, bmax);
                const float scale = mn == -INFINITY ? 1.0f : (base_e ? expf(m - mn) : exp2f(m - mn));
                float w = base_e ? expf(l - mn) : exp2f(l - mn);
                if (w != w) w = 0.0f;
                if (!mine) w = 0.0f;
                m = mn;
                // the running sums are still +0 in the first batch, where scaling them changes nothing
                if (n0 > 0) {
#pragma unroll
                    for (int k = 0; k < CPL; ++k)
#pragma unroll
                        for (int e = 0; e < kE; ++e) acc[k][e] *= scale;
#pragma unroll
                    for (int e = 0; e < 3 * T::kPerWord; ++e) tacc[e] *= scale;
                    S *= scale;
                }
                add_tail(w);
#pragma unroll
                for (int i = 0; i < NB; ++i) {
                    if (n0 + i >= a.N) break;  // the same for the whole warp
                    const float wi = __shfl_sync(0xffffffffu, w, row_lane0 + i);
                    S += wi;
                    add_rows(i, wi);
                }
            }
            r = 1.0f / fmaxf(S, 1e-10f);
        }
        // the tail sums over the row's lanes, normalised
#pragma unroll
        for (int e = 0; e < 3 * T::kPerWord; ++e) {
            tacc[e] = group_sum<G>(tacc[e]);
            if constexpr (!SINGLE) tacc[e] *= r;
        }
        if (a.return_lse && valid && j == 0) a.glse[u] = (base_e ? logf(S) : log2f(S)) + (m == -INFINITY ? 0.0f : m);
        // round, then realign: result chunk c = words q.. of sums c and c + 1 (the next lane's, lane
        // 0's next slot for lane G - 1, the tail sums for the row's last chunk)
        Words<4> enc[CPL];
#pragma unroll
        for (int k = 0; k < CPL; ++k)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float f[T::kPerWord];
#pragma unroll
                for (int h = 0; h < T::kPerWord; ++h) f[h] = SINGLE ? acc[k][e * T::kPerWord + h] : acc[k][e * T::kPerWord + h] * r;
                enc[k].w[e] = T::encode(f);
            }
        Words<4> tenc;
#pragma unroll
        for (int e = 0; e < 3; ++e) tenc.w[e] = T::encode(&tacc[e * T::kPerWord]);
        tenc.w[3] = 0u;
        uint32_t *res = a.result + u * a.data_w;
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
            Words<4> send = enc[k];
            if (k + 1 < CPL && j == 0) send = enc[k + 1 < CPL ? k + 1 : k];
            Words<4> nx;
#pragma unroll
            for (int e = 0; e < 3; ++e) nx.w[e] = __shfl_sync(0xffffffffu, send.w[e], next_lane);
            nx.w[3] = 0u;
            if (act[k] && c[k] == a.chunks - 1) nx = tenc;
            if (act[k]) store_words<4>(res + 4 * (int64_t)c[k], funnel_words(enc[k], nx, q));
        }
    }
}

// ---------------------------------------------------------------------------
// split merge written as 4-row groups of packed send rows (dcp_combine_pack, D' = 32 C,
// C = 1, 2, 4, heads per rank a multiple of 4)
//
// Packed rows [4 g, 4 g + 4) of the send buffer [ranks, B, Hr, D' + 1] are 4 consecutive
// heads of one (rank, token), i.e. the consecutive input rows u0 .. u0 + 3 of the split
// partials, and one aligned span of D' + 1 chunks of the send buffer.  A warp merges one
// group at a time.  Lane l = 8 r + j loads chunks j + 8 k (k < C) of input row r, so each
// load instruction reads 128 consecutive bytes of every row (split rows are aligned).
// Phase 1 reduces each row's S LSEs over `red_lanes` lanes (the split combine's grouping, so
// that the weights, hence the bits, equal those of dcp_lse_combine), phase 2 runs fp32 FMAs
// over the splits with NB splits in flight.  The rounded words and the merged LSEs are placed
// in a copy of the span in shared memory (row r at word r (D' + 1)), from which lane l stores
// chunks l + 32 k, and lane 31 the span's last chunk: 16-byte stores of 512 consecutive bytes,
// every word of the span written once.
__host__ __device__ constexpr size_t group_pack_smem_bytes(int N, int data_w) {
    // per warp: the span copy (4 (D' + 1) words) and the weights [N][4] floats
    return (size_t)(kCombineThreads / 32) * (4 * (data_w + 1) + N * 4) * 4;
}

template <class T, int C, int NB, int MIN_CTAS>
__global__ void __launch_bounds__(kCombineThreads, MIN_CTAS) group_pack_kernel(const CombineArgs a) {
    constexpr int kE = T::kPerWord;
    constexpr int kWarps = kCombineThreads / 32;
    extern __shared__ uint4 s_dyn[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int N = a.N;
    const int data_w = a.data_w;  // 32 C
    const int pitch = data_w + 1;
    const int span_w = 4 * pitch;  // a multiple of 4
    uint32_t *s_span = reinterpret_cast<uint32_t *>(s_dyn) + (size_t)warp * span_w;
    float *sw = reinterpret_cast<float *>(s_dyn) + (size_t)kWarps * span_w + (size_t)warp * N * 4;
    __shared__ uint32_t s_glse_all[kWarps][4];
    uint32_t *s_glse = s_glse_all[warp];
    const int r = lane >> 3;  // the input row of this lane in phase 2
    const int j = lane & 7;
    const uint32_t *lses = reinterpret_cast<const uint32_t *>(a.lses);
    const int64_t per_rank = a.pack_b * a.pack_hr;
    const int64_t groups = (a.units + 3) >> 2;  // units = ranks * B * Hr packed rows, a multiple of 4

    for (int64_t g = (int64_t)blockIdx.x * kWarps + warp; g < groups; g += (int64_t)gridDim.x * kWarps) {
        const int64_t p0 = g * 4;
        const int64_t rank = p0 / per_rank;
        const int64_t rem = p0 - rank * per_rank;
        const int64_t b = rem / a.pack_hr;
        const int64_t u0 = b * a.heads + rank * a.pack_hr + (rem - b * a.pack_hr);
        const int64_t row = (u0 + r) * data_w + 4 * j;  // this lane's first input word in split 0
        Words<4> x[NB][C];
        auto issue = [&](int n0) {
#pragma unroll
            for (int i = 0; i < NB; ++i)
#pragma unroll
                for (int k = 0; k < C; ++k) {
                    if (n0 + i < N) {
                        x[i][k] = load_stream<4>(a.src + (int64_t)(n0 + i) * a.shard_stride_w + row + 32 * k);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) x[i][k].w[e] = 0u;
                    }
                }
        };
        issue(0);

        // ---- phase 1: weights of each row over the splits ---------------------------------------
        // `red` lanes per row, 32 / red rows per pass: the lane grouping of the split combine
        // for the same S and D', so that the weights are summed in the same order and the
        // result equals dcp_lse_combine + dcp_pack bit for bit.
        // (any other value is taken as 8, so that every loop below ends whatever the argument)
        const int red = (a.red_lanes == 4 || a.red_lanes == 16 || a.red_lanes == 32) ? a.red_lanes : 8;
        for (int rb = 0; rb < 4; rb += 32 / red) {
            const int rr = rb + lane / red;  // >= 4 on idle lanes (red = 4)
            const int jj = lane % red;
            const bool act = rr < 4;
            float lmax = -INFINITY;
            for (int n = jj; act && n < N; n += red) {
                const float l = sanitize_lse(load_word(lses + (int64_t)n * a.lse_stride_n + u0 + rr));
                sw[n * 4 + rr] = l;
                lmax = fmaxf(lmax, l);
            }
            for (int o = red / 2; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
            const float m = (lmax == -INFINITY) ? 0.0f : lmax;
            float wsum = 0.0f;
            for (int n = jj; act && n < N; n += red) {
                const float x1 = sw[n * 4 + rr] - m;
                float w = a.base_e ? expf(x1) : exp2f(x1);
                if (w != w) w = 0.0f;
                sw[n * 4 + rr] = w;
                wsum += w;
            }
            for (int o = red / 2; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
            const float denom = fmaxf(wsum, 1e-10f);
            for (int n = jj; act && n < N; n += red) sw[n * 4 + rr] = sw[n * 4 + rr] / denom;
            if (act && jj == 0) s_glse[rr] = __float_as_uint((a.base_e ? logf(wsum) : log2f(wsum)) + m);
        }
        __syncwarp();

        // ---- phase 2: weighted sum over the splits --------------------------------------------
        float acc[C][4][kE];
#pragma unroll
        for (int k = 0; k < C; ++k)
#pragma unroll
            for (int e = 0; e < 4; ++e)
#pragma unroll
                for (int h = 0; h < kE; ++h) acc[k][e][h] = 0.0f;
        for (int n0 = 0; n0 < N; n0 += NB) {
            if (n0 > 0) issue(n0);
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                if (n0 + i >= N) break;  // the same for the whole warp
                const float w = sw[(n0 + i) * 4 + r];
#pragma unroll
                for (int k = 0; k < C; ++k)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float f[kE];
                        T::decode(x[i][k].w[e], f);
#pragma unroll
                        for (int h = 0; h < kE; ++h) acc[k][e][h] = fmaf(w, f[h], acc[k][e][h]);
                    }
            }
        }
        // the packed span in shared memory: row r's words at r (D' + 1), its LSE after them
        uint32_t *srow = s_span + r * pitch + 4 * j;
#pragma unroll
        for (int k = 0; k < C; ++k)
#pragma unroll
            for (int e = 0; e < 4; ++e) srow[32 * k + e] = T::encode(acc[k][e]);
        if (j == 0) s_span[r * pitch + data_w] = s_glse[r];
        __syncwarp();
        uint32_t *span = a.result + p0 * pitch;
        const uint4 *sv = reinterpret_cast<const uint4 *>(s_span);
#pragma unroll
        for (int k = 0; k < C; ++k) {
            const uint4 v = sv[lane + 32 * k];
            Words<4> o;
            o.w[0] = v.x; o.w[1] = v.y; o.w[2] = v.z; o.w[3] = v.w;
            store_words<4>(span + 4 * (lane + 32 * k), o);
        }
        if (lane == 31) {
            const uint4 v = sv[32 * C];
            Words<4> o;
            o.w[0] = v.x; o.w[1] = v.y; o.w[2] = v.z; o.w[3] = v.w;
            store_words<4>(span + 4 * 32 * C, o);
        }
        __syncwarp();  // shared memory is reused by the next group
    }
}

// ---------------------------------------------------------------------------
// pack
constexpr int kPackStages = 3;            // shared-memory tiles in flight per CTA
constexpr int kPackMinStageWords = 8192;  // up to 32 KiB per tile (more when one row needs it)
constexpr int kPackMaxTileRows = 64;      // rows per tile (row tables in shared memory)

struct PackArgs {
    const uint32_t *src;      // cp_attn_out as words
    const uint32_t *lse;      // cp_attn_lse as raw 32-bit words
    uint32_t *dst;            // send buffer as words (16-byte aligned)
    int64_t rows;             // N * B * Hr packed rows
    int64_t B;
    int64_t Hr;
    int64_t src_stride_b_w;   // words between tokens of cp_attn_out
    int64_t src_stride_h_w;   // words between heads of cp_attn_out
    int64_t lse_stride_b;     // words between tokens of cp_attn_lse
    uint64_t per_rank_magic;  // ceil(2^64 / (B * Hr)), 0 when B * Hr == 1
    uint64_t hr_magic;        // ceil(2^64 / Hr), 0 when Hr == 1
    uint32_t pitch_magic;     // ceil(2^32 / row_pitch_w): t / row_pitch_w == umulhi(t, magic) when t * row_pitch_w < 2^32
    int32_t data_w;           // words of data per row (a multiple of 4)
    int32_t row_pitch_w;      // data_w + 1: words per packed row
    int32_t tile_rows;        // packed rows per tile
    int32_t stage_w;          // words per shared-memory stage (a multiple of 4)
    int32_t max_run;          // rows per bulk copy, at most: 1, or more when the heads of a token
                              // are contiguous (src_stride_h_w == data_w)
    uint64_t wait_limit_ns;   // limit of each wait for a tile's copies (kWaitLimitNs)
    uint32_t stall_bytes;     // added to the byte count a CTA's first tile waits for: 0, except
                              // in the check of the timeout path (its wait then runs out)
    // pack_tma_kernel only: tokens per box of the tensor map; tiles per rank; and, in the launch
    // of each rank's last B mod tile_tokens tokens (one tile per rank), their first token and count
    int32_t tile_tokens;
    int32_t store_tokens;
    int64_t tiles_per_rank;
    int64_t first_token;
};

// Stores one landed tile: packed rows [i0, i0 + nrows) form the send range of words
// [d0, d0 + nrows * pitch).  The stage holds the tile's source rows one after another
// (data_w words each), then their LSE words from word lse_base.  Packed word t of the
// range is row r = t / pitch, word kk = t mod pitch, i.e. stage word t - r when kk < data_w,
// else LSE r.  Pass 1 writes every whole 16-byte chunk that lies inside one row's data as
// two aligned 16-byte shared loads and a word funnel.  Pass 2 writes, one thread per row,
// the chunk that holds the row's LSE word (rows are >= 5 words, so a chunk holds at most
// one LSE).  The partial chunks at the two ends of the range use 4-byte stores.  Threads
// tid = 0 .. nthreads - 1 (nthreads >= 8) share the work.
__device__ __forceinline__ void pack_store_tile(const uint32_t *stage, uint32_t *dst, int64_t d0, int nrows, int data_w,
                                                int pitch, int lse_base, uint32_t pitch_magic, int tid, int nthreads) {
    const int len = nrows * pitch;
    const uint4 *stage_v4 = reinterpret_cast<const uint4 *>(stage);
    auto word_of = [&](int r, int kk) -> uint32_t {  // word kk of packed row r of the tile
        return kk < data_w ? stage[r * data_w + kk] : stage[lse_base + r];
    };
    const int lead = (int)((4 - (d0 & 3)) & 3);  // words before the first 16-byte boundary
    const int full = (len - lead) >> 2;           // whole 16-byte chunks of the range
    uint32_t *dst_full = dst + d0 + lead;         // 16-byte aligned; chunk g = words lead+4g .. +3

    // pass 1: chunks inside one row's data
    for (int g = tid; g < full; g += nthreads) {
        const int t0 = lead + 4 * g;
        const int r = (int)__umulhi((uint32_t)t0, pitch_magic);
        const int kk = t0 - r * pitch;
        if (kk + 3 < data_w) {
            const int base = t0 - r;  // stage word of packed word t0
            const uint4 lo4 = stage_v4[base >> 2];
            const uint4 hi4 = stage_v4[(base >> 2) + 1];
            Words<4> lo, hi;
            lo.w[0] = lo4.x; lo.w[1] = lo4.y; lo.w[2] = lo4.z; lo.w[3] = lo4.w;
            hi.w[0] = hi4.x; hi.w[1] = hi4.y; hi.w[2] = hi4.z; hi.w[3] = hi4.w;
            store_words<4>(dst_full + 4 * g, funnel_words(lo, hi, base & 3));
        }
    }
    // pass 2: the chunk holding each row's LSE word
    for (int r = tid; r < nrows; r += nthreads) {
        const int t_row = r * pitch;
        const int t_lse = t_row + data_w;
        const int g = (t_lse - lead) >> 2;
        if (t_lse >= lead && g < full) {
            Words<4> o;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int kk = lead + 4 * g + e - t_row;
                o.w[e] = kk < pitch ? word_of(r, kk) : word_of(r + 1, kk - pitch);
            }
            store_words<4>(dst_full + 4 * g, o);
        }
    }
    // the partial chunks at the two ends of the range (a range has >= 5 words)
    auto word_at = [&](int t) -> uint32_t {
        const int r = (int)__umulhi((uint32_t)t, pitch_magic);
        return word_of(r, t - r * pitch);
    };
    if (tid < lead) {
        Words<1> o;
        o.w[0] = word_at(tid);
        store_words<1>(dst + d0 + tid, o);
    } else if (tid >= 4 && tid < 8) {
        const int t = lead + 4 * full + (tid - 4);
        if (t < len) {
            Words<1> o;
            o.w[0] = word_at(t);
            store_words<1>(dst + d0 + t, o);
        }
    }
}

// A CTA packs tiles of `tile_rows` consecutive packed rows (one contiguous word
// range of the send buffer), kPackStages tiles in flight.
//   Row table: for each tile, one thread per row computes the row's source
//   offset and LSE index (one tile ahead of its copies).
//   Loads: the tile's source rows (16-byte aligned, whole 16-byte chunks) are
//   copied with 16-byte cp.async into a stage, row after row, a group of lanes
//   per row; each row's LSE word goes behind the rows.
//   Stores, once a tile has landed: packed word t of the tile is row
//   r = t / (D'+1), word k = t mod (D'+1) (D' = data words per row), i.e. stage
//   word t - r when k < D', else LSE r.  Pass 1 writes every whole 16-byte
//   chunk that lies inside one row's data as two aligned 16-byte shared loads
//   and a word funnel.  Pass 2 writes, one thread per row, the chunk that holds
//   the row's LSE word (rows are >= 5 words, so a chunk holds at most one LSE).
//   The partial chunks at the two ends of the range use 4-byte stores.
// Every word of the send buffer is written once, by one CTA.
template <int STAGES = kPackStages, int THREADS = kPackThreads, int MAX_ROWS = kPackMaxTileRows, bool RANK_FAST = false>
__global__ void __launch_bounds__(THREADS) pack_kernel(const PackArgs a) {
    constexpr int kPackStages = STAGES;
    constexpr int kPackThreads = THREADS;
    constexpr int kPackMaxTileRows = MAX_ROWS;
    extern __shared__ uint4 s_stage_v4[];
    uint32_t *s_stage = reinterpret_cast<uint32_t *>(s_stage_v4);
    __shared__ int64_t s_row_src[kPackStages][kPackMaxTileRows];  // word offset of each source row
    __shared__ int64_t s_row_lse[kPackStages][kPackMaxTileRows];  // index of each row's LSE
    __shared__ int32_t s_row_run[kPackStages][kPackMaxTileRows];  // rows copied from this row on (0: none)
    __shared__ uint64_t s_full[kPackStages];                      // a stage's rows have landed
    __shared__ int s_abort;                                       // a wait timed out
    const int tid = threadIdx.x;
    // RANK_FAST: tiles never straddle a rank, and tile t is the (t / ranks)-th tile of rank
    // t mod ranks, so the tiles in flight at once cover all ranks of the same tokens
    const int64_t per_rank = a.B * a.Hr;
    const int64_t ranks = a.rows / per_rank;
    const int64_t tiles_per_rank = (per_rank + a.tile_rows - 1) / a.tile_rows;
    const int64_t tiles = RANK_FAST ? ranks * tiles_per_rank : (a.rows + a.tile_rows - 1) / a.tile_rows;
    const int64_t my_tiles = tiles > blockIdx.x ? (tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int tile_rows = a.tile_rows;
    const int data_w = a.data_w;
    const int pitch = a.row_pitch_w;
    const int stage_w = a.stage_w;
    const int lse_base = tile_rows * data_w;  // LSE words follow the rows in a stage
    const uint32_t pitch_magic = a.pitch_magic;
    const uint32_t *__restrict__ src = a.src;
    const uint32_t *__restrict__ lse = a.lse;

    auto tile_start = [&](int64_t k) -> int64_t {  // the first packed row of this CTA's k-th tile
        const int64_t t = blockIdx.x + k * gridDim.x;
        if constexpr (RANK_FAST) {
            const int64_t j = t / ranks;
            return (t - j * ranks) * per_rank + j * tile_rows;
        }
        return t * tile_rows;
    };
    auto tile_rows_of = [&](int64_t k) -> int {
        const int64_t i0 = tile_start(k);
        if constexpr (RANK_FAST) return (int)min((int64_t)tile_rows, per_rank - i0 % per_rank);
        return (int)min((int64_t)tile_rows, a.rows - i0);
    };
    // row table of this CTA's k-th tile, into slot k % kPackStages: rows are
    // ordered [rank][token][head], row (rank, b, h) holds cp_attn_out[b, rank*Hr + h]
    auto fill_table = [&](int64_t k) {
        const int64_t i0 = tile_start(k);
        const int nrows = tile_rows_of(k);
        const int slot = (int)(k % kPackStages);
        for (int r = tid; r < nrows; r += kPackThreads) {
            const uint64_t i = (uint64_t)(i0 + r);
            const uint64_t rank = div_magic(i, a.per_rank_magic);
            const uint64_t rem = i - rank * (uint64_t)(a.B * a.Hr);
            const uint64_t b = div_magic(rem, a.hr_magic);
            const uint64_t hh = rem - b * (uint64_t)a.Hr;  // head within the rank
            const uint64_t head = rank * (uint64_t)a.Hr + hh;
            s_row_src[slot][r] = (int64_t)b * a.src_stride_b_w + (int64_t)head * a.src_stride_h_w;
            s_row_lse[slot][r] = (int64_t)b * a.lse_stride_b + (int64_t)head;
            // with contiguous heads, rows r .. r + run - 1 (heads hh .. of this rank and token b,
            // up to the next multiple of max_run and within the tile) are one run of source
            // words, copied by the run's first row
            int run = 1;
            if (a.max_run > 1) {
                const int pos = (int)(hh % (uint64_t)a.max_run);
                run = (r == 0 || pos == 0)
                          ? (int)min(min((int64_t)(a.max_run - pos), (int64_t)a.Hr - (int64_t)hh), (int64_t)(nrows - r))
                          : 0;
            }
            s_row_run[slot][r] = run;
        }
    };
    // each run of source rows is one bulk copy (16-byte aligned, a multiple of 16 bytes)
    // that completes on the stage's barrier; the LSE words are 4-byte cp.async copies
    const uint32_t row_bytes = (uint32_t)data_w * 4u;
    auto issue = [&](int64_t k) {
        const int nrows = tile_rows_of(k);
        const int slot = (int)(k % kPackStages);
        uint32_t *stage = s_stage + slot * stage_w;
        if (tid == 0) mbar_arrive_expect_tx(&s_full[slot], (uint32_t)nrows * row_bytes + (k == 0 ? a.stall_bytes : 0u));
        for (int r = tid; r < nrows; r += kPackThreads) {
            const int run = s_row_run[slot][r];
            if (run > 0) {
                fence_proxy_async();
                bulk_copy_g2s(stage + r * data_w, src + s_row_src[slot][r], (uint32_t)run * row_bytes, &s_full[slot]);
            }
            cp_async_word(stage + lse_base + r, lse + s_row_lse[slot][r]);
        }
    };

    if (tid == 0) {
        for (int st = 0; st < kPackStages; ++st) mbar_init(&s_full[st], 1);
        mbar_fence_init();
        s_abort = 0;
    }
    for (int64_t k = 0; k < kPackStages && k < my_tiles; ++k) fill_table(k);
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kPackStages - 1; ++k) {
        if (k < my_tiles) issue(k);
        cp_async_commit();
    }
    __syncthreads();  // every thread is done reading the table slots of tiles 0 .. kPackStages-2
    for (int64_t k = 0; k < my_tiles; ++k) {
        if (k + kPackStages - 1 < my_tiles) issue(k + kPackStages - 1);
        cp_async_commit();
        // tile k's table slot was last read when tile k's copies were issued: fill it
        // for tile k + kPackStages while the copies are in flight
        if (k + kPackStages < my_tiles) fill_table(k + kPackStages);
        cp_async_wait<kPackStages - 1>();  // this thread's LSE copies of tile k have landed
        // the rows of tile k
        if (!mbar_wait_bounded(&s_full[(int)(k % kPackStages)], (uint32_t)((k / kPackStages) & 1), a.wait_limit_ns))
            s_abort = 1;
        __syncthreads();                   // ... and everyone else's (and the table)
        if (s_abort) {
            // A wait ran out: the CTA is counted and stops, its tiles unwritten.  Copies of
            // tiles k .. k + kPackStages - 1 may still be in flight into this CTA's shared
            // memory, so thread 0 first waits (bounded) for each of those tiles, which keeps
            // the CTA resident until they land; every thread waits for its own word copies.
            if (tid == 0) {
                atomicAdd(&g_wait_timeouts, 1ull);
                for (int64_t kk = k; kk < k + kPackStages && kk < my_tiles; ++kk)
                    mbar_wait_bounded(&s_full[(int)(kk % kPackStages)], (uint32_t)((kk / kPackStages) & 1),
                                      a.wait_limit_ns);
            }
            cp_async_wait<0>();
            return;
        }

        const int64_t i0 = tile_start(k);
        pack_store_tile(s_stage + (int)(k % kPackStages) * stage_w, a.dst, i0 * pitch, tile_rows_of(k), data_w, pitch,
                        lse_base, pitch_magic, tid, kPackThreads);
        __syncthreads();  // stage k % kPackStages is free for tile k + kPackStages
    }
    cp_async_wait<0>();
}

// The pack with each tile loaded by one tensor copy.  A tile is tile_tokens consecutive tokens
// b0 .. of one rank, all Hr of its heads: a box [tile_tokens][Hr][D] of cp_attn_out, which the
// tensor map `tmap` describes (3 dimensions {D, H, B}, or 4 {D/m, m, H, B} when a row is split
// into m pieces of at most 256 elements), and packed rows [(rank B + b0) Hr, ...), one
// contiguous range of the send buffer.  The box lands as rows back to back, as pack_store_tile
// expects; the LSE words follow with 4-byte cp.async copies.  The whole-tile launch (TAIL =
// false) covers tokens [0, B - B mod tile_tokens) of every rank, tile_tokens tokens a tile.  A
// second launch (TAIL = true), one tile per rank, covers the tokens left: its tiles start at
// first_token and store store_tokens tokens, and the box reaches past token B - 1, which the copy
// fills with zeros and still counts.  Waits, the abort path and the stall hook are those of
// pack_kernel.  STAGES tiles in flight per CTA; tiles of about 64 KiB with 2 stages measured best
// (one CTA per SM).
template <int STAGES, int THREADS, int DIMS, bool TAIL>
__global__ void __launch_bounds__(THREADS) pack_tma_kernel(const __grid_constant__ CUtensorMap tmap, const PackArgs a) {
    extern __shared__ __align__(128) uint4 s_tma_stage_v4[];
    // the launch adds 128 bytes, so the stages can start on a 128-byte boundary
    uint32_t *s_stage = reinterpret_cast<uint32_t *>(s_tma_stage_v4) + ((128u - (smem_addr(s_tma_stage_v4) & 127u)) & 127u) / 4;
    __shared__ uint64_t s_full[STAGES];
    __shared__ int s_abort;
    const int tid = threadIdx.x;
    const int Hr = (int)a.Hr;
    const int ranks = (int)(a.rows / (a.B * a.Hr));
    const int64_t tiles = (int64_t)ranks * a.tiles_per_rank;
    const int64_t my_tiles = tiles > blockIdx.x ? (tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int k = a.tile_tokens;
    const int box_rows = k * Hr;
    const int nrows = TAIL ? a.store_tokens * Hr : box_rows;  // rows each tile stores
    const int data_w = a.data_w, pitch = a.row_pitch_w, stage_w = a.stage_w;
    const int lse_base = box_rows * data_w;  // LSE words follow the box in a stage
    const uint32_t box_bytes = (uint32_t)box_rows * (uint32_t)data_w * 4u;
    const uint64_t tmap_addr = reinterpret_cast<uint64_t>(&tmap);

    // (an offset added to b0 in the whole-tile launch cost about 7% at 1 KiB rows, measured)
    auto tile_of = [&](int64_t kk, int &rank, int64_t &b0) {
        const int64_t t = blockIdx.x + kk * gridDim.x;
        rank = (int)(t / a.tiles_per_rank);
        if constexpr (TAIL)
            b0 = a.first_token;  // one tile per rank
        else
            b0 = (t - (int64_t)rank * a.tiles_per_rank) * k;
    };
    auto issue = [&](int64_t kk) {
        int rank;
        int64_t b0;
        tile_of(kk, rank, b0);
        const int slot = (int)(kk % STAGES);
        uint32_t *stage = s_stage + slot * stage_w;
        if (tid == 0) {
            fence_proxy_async();
            mbar_arrive_expect_tx(&s_full[slot], box_bytes + (kk == 0 ? a.stall_bytes : 0u));
            if constexpr (DIMS == 3) {
                asm volatile(
                    "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
                    "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(stage)),
                    "l"(tmap_addr), "r"(0), "r"(rank * Hr), "r"((int)b0), "r"(smem_addr(&s_full[slot]))
                    : "memory");
            } else {
                asm volatile(
                    "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
                    "[%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_addr(stage)),
                    "l"(tmap_addr), "r"(0), "r"(0), "r"(rank * Hr), "r"((int)b0), "r"(smem_addr(&s_full[slot]))
                    : "memory");
            }
        }
        for (int r = tid; r < nrows; r += THREADS) {
            const int64_t b = b0 + r / Hr;
            cp_async_word(stage + lse_base + r, a.lse + b * a.lse_stride_b + rank * Hr + r % Hr);
        }
    };

    if (tid == 0) {
        for (int st = 0; st < STAGES; ++st) mbar_init(&s_full[st], 1);
        mbar_fence_init();
        s_abort = 0;
    }
    __syncthreads();
    if (smem_addr(s_stage) & 127u) {  // a tensor copy needs a 128-byte aligned destination: none issued
        if (tid == 0) atomicAdd(&g_wait_timeouts, 1ull);
        return;
    }
#pragma unroll
    for (int kk = 0; kk < STAGES - 1; ++kk) {
        if (kk < my_tiles) issue(kk);
        cp_async_commit();
    }
    for (int64_t kk = 0; kk < my_tiles; ++kk) {
        if (kk + STAGES - 1 < my_tiles) issue(kk + STAGES - 1);
        cp_async_commit();
        cp_async_wait<STAGES - 1>();  // this thread's LSE copies of tile kk have landed
        if (!mbar_wait_bounded(&s_full[(int)(kk % STAGES)], (uint32_t)((kk / STAGES) & 1), a.wait_limit_ns))
            s_abort = 1;
        __syncthreads();
        if (s_abort) {
            // as in pack_kernel: counted once, then wait (bounded) for every tile in flight
            if (tid == 0) {
                atomicAdd(&g_wait_timeouts, 1ull);
                for (int64_t q = kk; q < kk + STAGES && q < my_tiles; ++q)
                    mbar_wait_bounded(&s_full[(int)(q % STAGES)], (uint32_t)((q / STAGES) & 1), a.wait_limit_ns);
            }
            cp_async_wait<0>();
            return;
        }
        int rank;
        int64_t b0;
        tile_of(kk, rank, b0);
        const int64_t i0 = ((int64_t)rank * a.B + b0) * Hr;
        pack_store_tile(s_stage + (int)(kk % STAGES) * stage_w, a.dst, i0 * pitch, nrows, data_w, pitch, lse_base,
                        a.pitch_magic, tid, THREADS);
        __syncthreads();  // stage kk % STAGES is free for tile kk + STAGES
    }
    cp_async_wait<0>();
}

}  // namespace dcp
