// dcp_kernels.cuh -- sm_100a kernels of the DCP LSE-weighted combine.
//
// Three memory-bound kernels (no tensor cores: the combine is a weighted sum
// over N shards, ~1 FMA per 2 bytes moved):
//
//   combine_kernel<..., PACKED=false>  combine of split receive buffers
//   combine_kernel<..., PACKED=true>   fused unpack + combine of the packed buffer
//   pack_kernel                         output rows + fp32 LSE -> packed rows
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

template <>
__device__ __forceinline__ void store_words<4>(uint32_t *p, const Words<4> &v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.w[0]), "r"(v.w[1]), "r"(v.w[2]),
                 "r"(v.w[3])
                 : "memory");
}

template <>
__device__ __forceinline__ void store_words<1>(uint32_t *p, const Words<1> &v) {
    asm volatile("st.global.u32 [%0], %1;" ::"l"(p), "r"(v.w[0]) : "memory");
}

__device__ __forceinline__ uint32_t load_word(const uint32_t *p) {
    uint32_t r;
    asm("ld.global.nc.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
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
    uint32_t *result;        // [units, data_w] words
    float *glse;             // [units], written when return_lse
    int64_t units;           // rows of the result (B * heads)
    int64_t shard_stride_w;  // words between consecutive shards
    int64_t lse_stride_n;    // split layout: floats between consecutive shards
    int64_t row_pitch_w;     // words between consecutive rows of one shard
    int32_t data_w;          // words of data per row (D * elemsize / 4)
    int32_t chunks;          // data_w / VW
    int32_t slots;           // ceil(chunks / G): chunk slots per lane
    int32_t N;
    int32_t base_e;
    int32_t return_lse;
};

// One warp works on 32/G result rows at a time, G lanes per row.  Phase 1: the
// G lanes of a row read the N LSEs (lane j takes shards j, j+G, ...), reduce
// max and sum with shuffles, and leave the normalised weights in shared memory.
// Phase 2: lane j accumulates chunks j, j+G, ... of the row over all N shards,
// with NB shards' loads issued before their FMAs, and stores the rounded row.
template <class T, int VW, int G, int CPL, int NB, bool PACKED>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineArgs a) {
    constexpr int kUnitsPerWarp = 32 / G;
    constexpr int kWarps = kCombineThreads / 32;
    constexpr int kElems = VW * T::kPerWord;
    __shared__ float s_w[kWarps][kUnitsPerWarp][kMaxShards];

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int ul = lane / G;
    const int j = lane % G;
    float *sw = s_w[warp][ul];
    const int64_t tasks = (a.units + kUnitsPerWarp - 1) / kUnitsPerWarp;

    for (int64_t task = (int64_t)blockIdx.x * kWarps + warp; task < tasks; task += (int64_t)gridDim.x * kWarps) {
        const int64_t u = task * kUnitsPerWarp + ul;
        const bool valid = u < a.units;
        const int64_t row = u * a.row_pitch_w;

        // ---- phase 1: weights of the N shards --------------------------------
        float lmax = -INFINITY;
        for (int n = j; n < a.N; n += G) {
            float l = -INFINITY;
            if (valid) {
                const uint32_t bits =
                    PACKED ? load_word(a.src + n * a.shard_stride_w + row + a.data_w)
                           : load_word(reinterpret_cast<const uint32_t *>(a.lses) + n * a.lse_stride_n + u);
                l = sanitize_lse(bits);
            }
            sw[n] = l;
            lmax = fmaxf(lmax, l);
        }
        lmax = group_max<G>(lmax);
        const float m = (lmax == -INFINITY) ? 0.0f : lmax;
        float wsum = 0.0f;
        for (int n = j; n < a.N; n += G) {
            const float x = sw[n] - m;
            float w = a.base_e ? expf(x) : exp2f(x);
            if (w != w) w = 0.0f;
            sw[n] = w;
            wsum += w;
        }
        wsum = group_sum<G>(wsum);
        const float denom = fmaxf(wsum, 1e-10f);
        for (int n = j; n < a.N; n += G) sw[n] = sw[n] / denom;
        if (a.return_lse && valid && j == 0) a.glse[u] = (a.base_e ? logf(wsum) : log2f(wsum)) + m;
        __syncwarp();

        // ---- phase 2: weighted sum of the N rows -------------------------------
        for (int s0 = 0; s0 < a.slots; s0 += CPL) {
            int c[CPL];
            bool act[CPL];
            float acc[CPL][kElems];
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                c[k] = j + G * (s0 + k);
                act[k] = valid && c[k] < a.chunks;
#pragma unroll
                for (int e = 0; e < kElems; ++e) acc[k][e] = 0.0f;
            }
            for (int n0 = 0; n0 < a.N; n0 += NB) {
                Words<VW> x[NB][CPL];
#pragma unroll
                for (int i = 0; i < NB; ++i) {
                    const int64_t base = (int64_t)(n0 + i) * a.shard_stride_w + row;
#pragma unroll
                    for (int k = 0; k < CPL; ++k) {
                        if (n0 + i < a.N && act[k]) {
                            x[i][k] = load_stream<VW>(a.src + base + (int64_t)c[k] * VW);
                        } else {
#pragma unroll
                            for (int v = 0; v < VW; ++v) x[i][k].w[v] = 0u;
                        }
                    }
                }
#pragma unroll
                for (int i = 0; i < NB; ++i) {
                    if (n0 + i < a.N) {
                        const float w = sw[n0 + i];
#pragma unroll
                        for (int k = 0; k < CPL; ++k) {
#pragma unroll
                            for (int v = 0; v < VW; ++v) {
                                float f[T::kPerWord];
                                T::decode(x[i][k].w[v], f);
#pragma unroll
                                for (int e = 0; e < T::kPerWord; ++e)
                                    acc[k][v * T::kPerWord + e] = fmaf(w, f[e], acc[k][v * T::kPerWord + e]);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                if (act[k]) {
                    Words<VW> o;
#pragma unroll
                    for (int v = 0; v < VW; ++v) o.w[v] = T::encode(&acc[k][v * T::kPerWord]);
                    store_words<VW>(a.result + u * a.data_w + (int64_t)c[k] * VW, o);
                }
            }
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// pack
struct PackArgs {
    const uint32_t *src;      // cp_attn_out as words
    const uint32_t *lse;      // cp_attn_lse as raw 32-bit words
    uint32_t *dst;            // send buffer as words
    int64_t rows;             // N * B * Hr packed rows
    int64_t B;
    int64_t Hr;
    int64_t src_stride_b_w;   // words between tokens of cp_attn_out
    int64_t src_stride_h_w;   // words between heads of cp_attn_out
    int64_t lse_stride_b;     // words between tokens of cp_attn_lse
    int32_t data_w;           // words of data per row
    int32_t chunks;           // data_w / 4 (16-byte chunks per source row)
    uint64_t chunks_magic;    // ceil(2^32 / chunks): n / chunks == (n * magic) >> 32 whenever n * chunks < 2^32
    int32_t row_pitch_w;      // data_w + 1
    int32_t tile_rows;        // packed rows per tile
};

// A CTA packs tiles of `tile_rows` consecutive packed rows, i.e. one contiguous
// word range of the send buffer.  It gathers the source rows (16-byte loads)
// and their LSE words into shared memory laid out exactly as that range, with
// the same alignment modulo 16 bytes, then writes the range back with 16-byte
// stores (4-byte stores only for the partial chunks at its two ends).  Every
// word of the send buffer is written once, by one CTA.
__global__ void __launch_bounds__(kPackThreads) pack_kernel(const PackArgs a) {
    extern __shared__ uint4 s_tile_v4[];
    uint32_t *s_tile = reinterpret_cast<uint32_t *>(s_tile_v4);
    __shared__ int64_t s_src_row[kPackThreads];

    const int tid = threadIdx.x;
    const int64_t tiles = (a.rows + a.tile_rows - 1) / a.tile_rows;
    const int64_t per_rank = a.B * a.Hr;

    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int64_t i0 = tile * a.tile_rows;
        const int nrows = (int)min((int64_t)a.tile_rows, a.rows - i0);
        const int64_t dst_w0 = i0 * a.row_pitch_w;
        const int q = (int)(dst_w0 & 3);  // alignment of the range start, in words

        // source row offsets and LSE words, one thread per packed row
        for (int r = tid; r < nrows; r += kPackThreads) {
            const int64_t i = i0 + r;
            const int64_t rank = i / per_rank;
            const int64_t rem = i - rank * per_rank;
            const int64_t b = rem / a.Hr;
            const int64_t head = rank * a.Hr + (rem - b * a.Hr);
            s_src_row[r] = b * a.src_stride_b_w + head * a.src_stride_h_w;
            s_tile[q + r * a.row_pitch_w + a.data_w] = load_word(a.lse + b * a.lse_stride_b + head);
        }
        __syncthreads();

        // gather: 16-byte loads from the source rows, 4-byte shared stores; the
        // store order is rotated by lane/8 so the 32 lanes hit 32 distinct banks
        const int total_chunks = nrows * a.chunks;
        const int rot = (tid >> 3) & 3;
        for (int idx = tid; idx < total_chunks; idx += kPackThreads) {
            const int r = (int)(((uint64_t)idx * a.chunks_magic) >> 32);
            const int c = idx - r * a.chunks;
            const Words<4> v = load_stream<4>(a.src + s_src_row[r] + 4 * c);
            uint32_t *s = s_tile + q + r * a.row_pitch_w + 4 * c;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int e = (k + rot) & 3;
                const uint32_t val = e == 0 ? v.w[0] : e == 1 ? v.w[1] : e == 2 ? v.w[2] : v.w[3];
                s[e] = val;
            }
        }
        __syncthreads();

        // scatter: shared word s <-> send-buffer word dst_w0 - q + s
        const int end = q + nrows * a.row_pitch_w;  // one past the last shared word in use
        uint32_t *dst = a.dst + (dst_w0 - q);
        const int first_full = q ? 1 : 0;           // first 16-byte chunk fully inside the range
        const int full_end = end >> 2;              // one past the last full chunk
        for (int t = first_full + tid; t < full_end; t += kPackThreads) {
            const uint4 v = s_tile_v4[t];
            Words<4> o;
            o.w[0] = v.x;
            o.w[1] = v.y;
            o.w[2] = v.z;
            o.w[3] = v.w;
            store_words<4>(dst + 4 * t, o);
        }
        // A range holds at least one packed row of >= 5 words, so end >= 5: the
        // head words [q, 4) and the tail words [4 * full_end, end) never overlap.
        if (tid < 4) {  // the partial chunk at the head of the range
            const int s = tid;
            if (s >= q && q > 0) {
                Words<1> o;
                o.w[0] = s_tile[s];
                store_words<1>(dst + s, o);
            }
        } else if (tid < 8) {  // the partial chunk at the tail
            const int s = 4 * full_end + (tid - 4);
            if (s < end) {
                Words<1> o;
                o.w[0] = s_tile[s];
                store_words<1>(dst + s, o);
            }
        }
        __syncthreads();
    }
}

}  // namespace dcp
