// dcp_api.cu -- the extern "C" entry points of libdcpcombine.so (see
// include/dcp_combine.h for the contract of each call).
//
// Host side only: argument validation (before any CUDA call), choice of the
// kernel instance for the row width, grid sizing, launch, and launch-error
// reporting.  Nothing here allocates device memory or synchronises.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include <atomic>

#include "dcp_combine_launch.cuh"
#include "dcp_host.h"
#include "dcp_testing.h"

namespace dcp_host {

namespace {
thread_local char g_error[512] = "";
}  // namespace

const char *last_error() { return g_error; }

int32_t fail(int32_t status, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_error, sizeof g_error, fmt, ap);
    va_end(ap);
    return status;
}

int32_t ok() {
    g_error[0] = '\0';
    return DCP_OK;
}

// Multiprocessor count of the current device (cached per device).
int sm_count() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64) {
        int v = cache[dev].load(std::memory_order_relaxed);
        if (v > 0) return v;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

int32_t launch_status(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(DCP_ERR_CUDA, "%s: kernel launch failed: %s", what, cudaGetErrorString(e));
    return ok();
}

}  // namespace dcp_host

namespace {

using dcp_host::cached_resident_ctas;
using dcp_host::fail;
using dcp_host::InstanceCache;
using dcp_host::launch_status;
using dcp_host::ok;
using dcp_host::reserve_smem;
using dcp_host::resident_ctas;
using dcp_host::sm_count;

int elem_size(int32_t dtype) {
    switch (dtype) {
        case DCP_BF16:
        case DCP_FP16: return 2;
        case DCP_FP32: return 4;
        default: return 0;
    }
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

constexpr int64_t kMaxD = 8192;            // elements per row
constexpr int64_t kMaxRows = int64_t(1) << 40;



// ceil(2^64 / d) for d >= 2; 0 stands for d == 1 (n / 1 == n).
uint64_t magic64(uint64_t d) {
    if (d <= 1) return 0;
    const unsigned __int128 one = 1;
    return (uint64_t)(((one << 64) + d - 1) / d);
}

// The pack kernel's dynamic shared memory can exceed the default 48 KiB: opt in
// once per device, for the largest stage any accepted row width needs.
// The pack kernel this host thread launched last (dcp_testing_last_pack_kernel).
thread_local int32_t t_last_pack_kernel = 0;

// One pack kernel instance: its dynamic shared memory is reserved once per device (enough for
// a stage of `max_stage_w` words), and its resident CTAs per SM are cached per device for the
// last dynamic shared-memory size asked.
template <int STAGES, int MAX_ROWS, bool RANK_FAST>
struct PackInstance {
    static constexpr auto kernel = dcp::pack_kernel<STAGES, dcp::kPackThreads, MAX_ROWS, RANK_FAST>;
    static bool reserve(int max_stage_w) {
        static std::atomic<int> done[64];
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return false;
        if (dev < 64 && done[dev].load(std::memory_order_acquire)) return true;
        const size_t bytes = (size_t)STAGES * max_stage_w * 4;
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
            return false;
        if (dev < 64) done[dev].store(1, std::memory_order_release);
        return true;
    }
    static int resident(size_t smem) {
        static std::atomic<uint64_t> cache[64];  // per device: (smem << 16) | ctas
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
            return resident_ctas(kernel, dcp::kPackThreads, smem);
        const uint64_t c = cache[dev].load(std::memory_order_relaxed);
        if (c && (c >> 16) == smem) return (int)(c & 0xffff);
        const int n = resident_ctas(kernel, dcp::kPackThreads, smem);
        cache[dev].store(((uint64_t)smem << 16) | (uint64_t)n, std::memory_order_relaxed);
        return n;
    }
};

// Geometry of a pack instance for one call.  A stage holds about `stage_words` words of
// source rows (at least one row, at most MAX_ROWS) and their LSE words, plus 4 words of slack
// for the second aligned read of the last chunk.
struct PackGeom {
    int tile_rows = 0;
    int stage_w = 0;
    size_t smem = 0;
    int64_t tiles = 0;  // tiles of the call
    int64_t cap = 0;    // CTAs resident at once
};

template <int STAGES, int MAX_ROWS, bool RANK_FAST = false>
bool pack_geometry(const dcp::PackArgs &a, int stage_words, PackGeom &g) {
    using I = PackInstance<STAGES, MAX_ROWS, RANK_FAST>;
    g.tile_rows = (stage_words - 8) / a.row_pitch_w;
    if (g.tile_rows < 1) g.tile_rows = 1;
    if (g.tile_rows > MAX_ROWS) g.tile_rows = MAX_ROWS;
    g.stage_w = ((g.tile_rows * a.row_pitch_w + 3) & ~3) + 4;
    const int max_stage_w = (int)(((kMaxD + 1 + 3) & ~int64_t(3)) + 4);  // one fp32 row of kMaxD words
    if (!I::reserve(stage_words + 8 > max_stage_w ? stage_words + 8 : max_stage_w)) return false;
    g.smem = (size_t)STAGES * g.stage_w * 4;
    const int64_t per_rank = a.B * a.Hr;
    g.tiles = RANK_FAST ? (a.rows / per_rank) * ((per_rank + g.tile_rows - 1) / g.tile_rows)
                        : (a.rows + g.tile_rows - 1) / g.tile_rows;
    g.cap = (int64_t)sm_count() * I::resident(g.smem);
    return true;
}

// `runs`: where a token's heads are contiguous, the rows of one (rank, token) in a tile are
// copied as one run.
template <int STAGES, int MAX_ROWS, bool RANK_FAST = false>
int32_t launch_pack(const char *fn, dcp::PackArgs a, const PackGeom &g, bool runs, cudaStream_t stream) {
    a.tile_rows = g.tile_rows;
    a.stage_w = g.stage_w;
    const bool contiguous = a.src_stride_h_w == a.data_w;
    a.max_run = runs && contiguous ? (int32_t)(a.Hr < (int64_t(1) << 20) ? a.Hr : (int64_t(1) << 20)) : 1;
    const int grid = (int)(g.tiles < g.cap ? g.tiles : g.cap);
    PackInstance<STAGES, MAX_ROWS, RANK_FAST>::kernel<<<grid, dcp::kPackThreads, g.smem, stream>>>(a);
    t_last_pack_kernel = RANK_FAST ? 3 : a.max_run > 1 ? 2 : 1;
    return launch_status(fn);
}

// ---- the tensor-copy pack (pack_tma_kernel) ----

// cuTensorMapEncodeTiled, found once through the runtime (the library does not link the driver).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
    static std::atomic<int> tried{0};
    PFN_cuTensorMapEncodeTiled_v12000 f = fn.load(std::memory_order_acquire);
    if (f || tried.load(std::memory_order_acquire)) return f;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    fn.store(f, std::memory_order_release);
    tried.store(1, std::memory_order_release);
    return f;
}

constexpr int kPackTmaStages = 2;
constexpr int kPackTmaBoxBytes = 65536;  // about 64 KiB of rows per tile
// the largest stage: 64 KiB of rows of at least 16 bytes (4096 rows), their LSE words, slack
constexpr int kPackTmaMaxStageW = ((kPackTmaBoxBytes / 4 + kPackTmaBoxBytes / 16 + 4) + 31) & ~31;

// A tensor map and tile shape for pack_tma_kernel, or false when the shape does not suit it
// (more than 256 heads per rank, a token's heads over 64 KiB, B or H beyond a 32-bit
// coordinate, no row split into pieces of at most 256 elements and a multiple of 16 bytes, or
// an encoding the driver refuses).
// The tile shape alone: k tokens per tile (at most 256, at most B, k Hr rows within 64 KiB) and
// the row split into m pieces (the fewest of at most 256 elements each, D a multiple of m, a
// piece a multiple of 16 bytes); false when no such shape exists.
bool pack_tma_shape(int64_t Hr, int64_t D, int es, int64_t B, int64_t &k, int64_t &m) {
    const int64_t row_bytes = D * es;
    if (Hr < 1 || B < 1 || D < 1 || Hr > 256 || Hr * row_bytes > kPackTmaBoxBytes) return false;
    k = kPackTmaBoxBytes / (Hr * row_bytes);
    if (k > 256) k = 256;
    if (k > B) k = B;
    m = (D + 255) / 256;
    while (m <= 256 && (D % m != 0 || ((D / m) * es) % 16 != 0)) ++m;
    return m <= 256;
}

bool pack_tma_plan(dcp::PackArgs &a, const void *cp_attn_out, int64_t H, int64_t D, int es, int64_t out_stride_b,
                   int64_t out_stride_h, CUtensorMap &map, int &dims) {
    if (a.B > INT32_MAX || H > INT32_MAX) return false;  // tensor-copy coordinates are 32-bit
    int64_t k = 0, m = 0;
    if (!pack_tma_shape(a.Hr, D, es, a.B, k, m)) return false;
    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (!encode) return false;
    const CUtensorMapDataType type = es == 4 ? CU_TENSOR_MAP_DATA_TYPE_UINT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
    const cuuint32_t one[4] = {1, 1, 1, 1};
    CUresult r;
    if (m == 1) {
        const cuuint64_t dim[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)a.B};
        const cuuint64_t stride[2] = {(cuuint64_t)(out_stride_h * es), (cuuint64_t)(out_stride_b * es)};
        const cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)a.Hr, (cuuint32_t)k};
        r = encode(&map, type, 3, const_cast<void *>(cp_attn_out), dim, stride, box, one, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        dims = 3;
    } else {
        const cuuint64_t dim[4] = {(cuuint64_t)(D / m), (cuuint64_t)m, (cuuint64_t)H, (cuuint64_t)a.B};
        const cuuint64_t stride[3] = {(cuuint64_t)((D / m) * es), (cuuint64_t)(out_stride_h * es),
                                      (cuuint64_t)(out_stride_b * es)};
        const cuuint32_t box[4] = {(cuuint32_t)(D / m), (cuuint32_t)m, (cuuint32_t)a.Hr, (cuuint32_t)k};
        r = encode(&map, type, 4, const_cast<void *>(cp_attn_out), dim, stride, box, one, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        dims = 4;
    }
    if (r != CUDA_SUCCESS) return false;
    a.tile_tokens = (int32_t)k;
    const int box_rows = (int)(k * a.Hr);
    a.stage_w = ((box_rows * a.data_w + box_rows + 4) + 31) & ~31;  // 128-byte aligned stages
    return true;
}

template <int DIMS>
int32_t launch_pack_tma(const char *fn, const dcp::PackArgs &a, const CUtensorMap &map, cudaStream_t stream) {
    auto kernel = dcp::pack_tma_kernel<kPackTmaStages, dcp::kPackThreads, DIMS, false>;
    auto tail_kernel = dcp::pack_tma_kernel<kPackTmaStages, dcp::kPackThreads, DIMS, true>;
    static std::atomic<int> reserved[64];
    static std::atomic<uint64_t> occupancy[64];  // per device: (smem << 16) | ctas
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return fail(DCP_ERR_CUDA, "%s: no device", fn);
    if (!reserved[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kPackTmaStages * kPackTmaMaxStageW * 4 + 128) != cudaSuccess ||
            cudaFuncSetAttribute(tail_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kPackTmaStages * kPackTmaMaxStageW * 4 + 128) != cudaSuccess)
            return fail(DCP_ERR_CUDA, "%s: cannot reserve shared memory for the pack kernel", fn);
        reserved[dev].store(1, std::memory_order_release);
    }
    const size_t smem = (size_t)kPackTmaStages * a.stage_w * 4 + 128;  // + room to align the stages
    int per_sm;
    const uint64_t c = occupancy[dev].load(std::memory_order_relaxed);
    if (c && (c >> 16) == smem) {
        per_sm = (int)(c & 0xffff);
    } else {
        per_sm = resident_ctas(kernel, dcp::kPackThreads, smem);
        occupancy[dev].store(((uint64_t)smem << 16) | (uint64_t)per_sm, std::memory_order_relaxed);
    }
    // whole tiles of tile_tokens tokens (B >= tile_tokens), then one tile per rank for the
    // B mod tile_tokens tokens left
    const int64_t ranks = a.rows / (a.B * a.Hr);
    const int64_t cap = (int64_t)sm_count() * per_sm;
    dcp::PackArgs m = a;
    m.store_tokens = a.tile_tokens;
    m.tiles_per_rank = a.B / a.tile_tokens;
    m.first_token = 0;
    const int64_t tiles = ranks * m.tiles_per_rank;
    kernel<<<(int)(tiles < cap ? tiles : cap), dcp::kPackThreads, smem, stream>>>(map, m);
    const int64_t rem = a.B % a.tile_tokens;
    if (rem) {
        m.store_tokens = (int32_t)rem;
        m.tiles_per_rank = 1;
        m.first_token = a.B - rem;
        tail_kernel<<<(int)(ranks < cap ? ranks : cap), dcp::kPackThreads, smem, stream>>>(map, m);
    }
    t_last_pack_kernel = DIMS == 3 ? 4 : 5;
    return launch_status(fn);
}

template <bool PACKED>
int32_t dispatch_dtype(int32_t dtype, const dcp::CombineArgs &a, cudaStream_t stream) {
    switch (dtype) {
        case DCP_BF16: return dcp_host::dispatch_combine_bf16(a, PACKED, stream);
        case DCP_FP16: return dcp_host::dispatch_combine_fp16(a, PACKED, stream);
        default: return dcp_host::dispatch_combine_fp32(a, PACKED, stream);
    }
}

int32_t check_common(const char *fn, int32_t dtype, int32_t N, int64_t B, int64_t H, int64_t D) {
    if (elem_size(dtype) == 0) return fail(DCP_ERR_UNSUPPORTED_DTYPE, "%s: unsupported dtype %d", fn, (int)dtype);
    if (N < 1 || N > DCP_MAX_SHARDS)
        return fail(DCP_ERR_INVALID_ARG, "%s: shard count %d outside [1, %d]", fn, (int)N, DCP_MAX_SHARDS);
    if (B < 0) return fail(DCP_ERR_INVALID_ARG, "%s: negative token count %lld", fn, (long long)B);
    if (H < 1) return fail(DCP_ERR_INVALID_ARG, "%s: head count %lld < 1", fn, (long long)H);
    if (D < 1 || D > kMaxD) return fail(DCP_ERR_INVALID_ARG, "%s: head dim %lld outside [1, %lld]", fn, (long long)D,
                                        (long long)kMaxD);
    if ((D * elem_size(dtype)) % 16 != 0)
        return fail(DCP_ERR_MISALIGNED, "%s: a row of D=%lld elements is not a multiple of 16 bytes", fn,
                    (long long)D);
    if (B > 0 && (B > kMaxRows / H || B * H > kMaxRows / (int64_t)N))
        return fail(DCP_ERR_INVALID_ARG, "%s: problem too large", fn);
    return DCP_OK;
}

}  // namespace

extern "C" {

int32_t dcp_version(void) { return 10000; }

int32_t dcp_wait_timeouts(uint64_t *count, int32_t reset) {
    if (!count) return fail(DCP_ERR_INVALID_ARG, "dcp_wait_timeouts: count is null");
    unsigned long long v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, dcp::g_wait_timeouts, sizeof(v));
    if (e == cudaSuccess && reset) {
        const unsigned long long zero = 0;
        e = cudaMemcpyToSymbol(dcp::g_wait_timeouts, &zero, sizeof(zero));
    }
    if (e != cudaSuccess) return fail(DCP_ERR_CUDA, "dcp_wait_timeouts: %s", cudaGetErrorString(e));
    *count = v;
    return ok();
}

const char *dcp_last_error(void) { return dcp_host::last_error(); }

int32_t dcp_lse_pack_dim(int32_t dtype) {
    const int es = elem_size(dtype);
    return es ? 4 / es : -1;
}

namespace {

// Request metadata of a variable-length combine (on == false: every shard is read).
struct Varlen {
    bool on = false;
    const int32_t *seq_lens = nullptr;
    const int32_t *qsl = nullptr;
    int32_t num_reqs = 0;
    int32_t interleave = 1;
};

// Packed output of a combine (dcp_combine_pack): B and heads per rank; on == false: plain rows.
struct PackOut {
    bool on = false;
    int64_t B = 0;
    int64_t Hr = 1;
};

// The split-layout combine with every stride explicit (elements of each array).
int32_t lse_combine_impl(const char *fn, const void *outputs, const float *lses, void *result, float *global_lse,
                         int32_t N, int64_t B, int64_t H, int64_t D, int64_t os_n, int64_t os_b, int64_t os_h,
                         int64_t ls_n, int64_t ls_b, int64_t ls_h, int64_t rs_b, int64_t rs_h, int64_t gs_b,
                         int64_t gs_h, int32_t dtype, int32_t is_lse_base_on_e, int32_t return_lse,
                         void *cuda_stream, const Varlen &vl = Varlen{}, const PackOut &po = PackOut{}) {
    int32_t st = check_common(fn, dtype, N, B, H, D);
    if (st != DCP_OK) return st;
    const int es = elem_size(dtype);
    const int64_t vec = 16 / es;  // elements per 16 bytes
    if (os_n < 0 || os_b < 0 || os_h < 0 || ls_n < 0 || ls_b < 0 || ls_h < 0 || rs_b < 0 || rs_h < 0 || gs_b < 0 ||
        gs_h < 0)
        return fail(DCP_ERR_INVALID_ARG, "%s: negative stride", fn);
    if (os_n % vec || os_b % vec || os_h % vec || rs_b % vec || rs_h % vec)
        return fail(DCP_ERR_MISALIGNED, "%s: output and result strides must be multiples of 16 bytes", fn);
    if (B == 0) return ok();
    if (!outputs || !lses || !result) return fail(DCP_ERR_INVALID_ARG, "%s: null buffer pointer", fn);
    if (return_lse && !global_lse) return fail(DCP_ERR_INVALID_ARG, "%s: return_lse set but global_lse is null", fn);
    if (!aligned(outputs, 16) || !aligned(result, 16))
        return fail(DCP_ERR_MISALIGNED, "%s: outputs and result must be 16-byte aligned", fn);
    if (!aligned(lses, 4) || (return_lse && !aligned(global_lse, 4)))
        return fail(DCP_ERR_MISALIGNED, "%s: lses and global_lse must be 4-byte aligned", fn);
    if (B * H >= (int64_t(1) << 32)) return fail(DCP_ERR_INVALID_ARG, "%s: more than 2^32 result rows", fn);

    dcp::CombineArgs a{};
    a.src = static_cast<const uint32_t *>(outputs);
    a.lses = lses;
    a.result = static_cast<uint32_t *>(result);
    a.glse = global_lse;
    a.units = B * H;
    a.shard_stride_w = os_n * es / 4;
    a.lse_stride_n = ls_n;
    a.data_w = (int32_t)(D * es / 4);
    a.row_pitch_w = a.data_w;
    a.chunks = a.data_w / 4;
    a.heads = H;
    a.heads_magic = magic64((uint64_t)H);
    a.src_sb_w = os_b * es / 4;
    a.src_sh_w = os_h * es / 4;
    a.lse_sb = ls_b;
    a.lse_sh = ls_h;
    a.res_sb_w = rs_b * es / 4;
    a.res_sh_w = rs_h * es / 4;
    a.glse_sb = gs_b;
    a.glse_sh = gs_h;
    a.N = N;
    a.base_e = is_lse_base_on_e ? 1 : 0;
    a.return_lse = return_lse ? 1 : 0;
    a.pack_b = po.on ? B : 0;
    a.pack_hr = po.Hr;
    a.pack_hr_magic = magic64((uint64_t)po.Hr);
    a.varlen = vl.on ? 1 : 0;
    a.num_reqs = vl.num_reqs;
    a.interleave = vl.interleave;
    a.seq_lens = vl.seq_lens;
    a.qsl = vl.qsl;
    return dispatch_dtype<false>(dtype, a, static_cast<cudaStream_t>(cuda_stream));
}

// Layout checks of dcp_lse_combine (canonical [N, B, H, D] shards, shard strides free).
int32_t check_split_layout(const char *fn, int32_t N, int64_t B, int64_t H, int64_t D, int64_t out_stride_n,
                           int64_t lse_stride_n, int32_t dtype) {
    int32_t st = check_common(fn, dtype, N, B, H, D);
    if (st != DCP_OK) return st;
    if (out_stride_n < B * H * D)
        return fail(DCP_ERR_INVALID_ARG, "%s: out_stride_n %lld < B*H*D = %lld", fn, (long long)out_stride_n,
                    (long long)(B * H * D));
    if (lse_stride_n < B * H)
        return fail(DCP_ERR_INVALID_ARG, "%s: lse_stride_n %lld < B*H = %lld", fn, (long long)lse_stride_n,
                    (long long)(B * H));
    if ((out_stride_n * elem_size(dtype)) % 16 != 0)
        return fail(DCP_ERR_MISALIGNED, "%s: out_stride_n %lld elements is not a multiple of 16 bytes", fn,
                    (long long)out_stride_n);
    return DCP_OK;
}

}  // namespace

int32_t dcp_lse_combine(const void *outputs, const float *lses, void *result, float *global_lse, int32_t N, int64_t B,
                        int64_t H, int64_t D, int64_t out_stride_n, int64_t lse_stride_n, int32_t dtype,
                        int32_t is_lse_base_on_e, int32_t return_lse, void *cuda_stream) {
    const char *fn = "dcp_lse_combine";
    int32_t st = check_split_layout(fn, N, B, H, D, out_stride_n, lse_stride_n, dtype);
    if (st != DCP_OK) return st;
    return lse_combine_impl(fn, outputs, lses, result, global_lse, N, B, H, D, out_stride_n, H * D, D, lse_stride_n,
                            H, 1, H * D, D, H, 1, dtype, is_lse_base_on_e, return_lse, cuda_stream);
}

int32_t dcp_lse_combine_strided(const void *outputs, const float *lses, void *result, float *global_lse, int32_t N,
                                int64_t B, int64_t H, int64_t D, int64_t out_stride_n, int64_t out_stride_b,
                                int64_t out_stride_h, int64_t lse_stride_n, int64_t lse_stride_b,
                                int64_t lse_stride_h, int64_t result_stride_b, int64_t result_stride_h,
                                int64_t glse_stride_b, int64_t glse_stride_h, int32_t dtype, int32_t is_lse_base_on_e,
                                int32_t return_lse, void *cuda_stream) {
    return lse_combine_impl("dcp_lse_combine_strided", outputs, lses, result, global_lse, N, B, H, D, out_stride_n,
                            out_stride_b, out_stride_h, lse_stride_n, lse_stride_b, lse_stride_h, result_stride_b,
                            result_stride_h, glse_stride_b, glse_stride_h, dtype, is_lse_base_on_e, return_lse,
                            cuda_stream);
}

int32_t dcp_lse_combine_varlen(const void *outputs, const float *lses, void *result, float *global_lse, int32_t N,
                               int64_t B, int64_t H, int64_t D, int64_t out_stride_n, int64_t lse_stride_n,
                               const int32_t *seq_lens, const int32_t *query_start_loc, int32_t num_reqs,
                               int32_t interleave, int32_t dtype, int32_t is_lse_base_on_e, int32_t return_lse,
                               void *cuda_stream) {
    const char *fn = "dcp_lse_combine_varlen";
    int32_t st = check_split_layout(fn, N, B, H, D, out_stride_n, lse_stride_n, dtype);
    if (st != DCP_OK) return st;
    if (num_reqs < 0) return fail(DCP_ERR_INVALID_ARG, "%s: negative request count %d", fn, (int)num_reqs);
    if (interleave < 1) return fail(DCP_ERR_INVALID_ARG, "%s: interleave %d < 1", fn, (int)interleave);
    if (num_reqs > 0 && B > 0) {
        if (!seq_lens || !query_start_loc)
            return fail(DCP_ERR_INVALID_ARG, "%s: seq_lens and query_start_loc are needed for %d requests", fn,
                        (int)num_reqs);
        if (!aligned(seq_lens, 4) || !aligned(query_start_loc, 4))
            return fail(DCP_ERR_MISALIGNED, "%s: seq_lens and query_start_loc must be 4-byte aligned", fn);
    }
    Varlen vl;
    vl.on = true;
    vl.seq_lens = seq_lens;
    vl.qsl = query_start_loc;
    vl.num_reqs = num_reqs;
    vl.interleave = interleave;
    return lse_combine_impl(fn, outputs, lses, result, global_lse, N, B, H, D, out_stride_n, H * D, D, lse_stride_n,
                            H, 1, H * D, D, H, 1, dtype, is_lse_base_on_e, return_lse, cuda_stream, vl);
}

int32_t dcp_combine_pack(const void *partial_outputs, const float *partial_lses, void *send_buf, int32_t S, int64_t B,
                         int64_t H, int64_t D, int64_t out_stride_s, int64_t lse_stride_s, int32_t world_size,
                         int32_t dtype, int32_t is_lse_base_on_e, void *cuda_stream) {
    const char *fn = "dcp_combine_pack";
    int32_t st = check_split_layout(fn, S, B, H, D, out_stride_s, lse_stride_s, dtype);
    if (st != DCP_OK) return st;
    if (world_size < 1 || world_size > DCP_MAX_SHARDS)
        return fail(DCP_ERR_INVALID_ARG, "%s: world_size %d outside [1, %d]", fn, (int)world_size, DCP_MAX_SHARDS);
    if (H % world_size != 0)
        return fail(DCP_ERR_SHAPE, "%s: H=%lld heads do not split evenly over %d ranks", fn, (long long)H,
                    (int)world_size);
    if (B == 0) return ok();
    if (!send_buf) return fail(DCP_ERR_INVALID_ARG, "%s: null buffer pointer", fn);
    if (!aligned(send_buf, 16)) return fail(DCP_ERR_MISALIGNED, "%s: send_buf must be 16-byte aligned", fn);
    PackOut po;
    po.on = true;
    po.B = B;
    po.Hr = H / world_size;
    // the result pointer is the send buffer; rows are placed by the kernel
    return lse_combine_impl(fn, partial_outputs, partial_lses, send_buf, nullptr, S, B, H, D, out_stride_s, H * D, D,
                            lse_stride_s, H, 1, H * D, D, H, 1, dtype, is_lse_base_on_e, 0, cuda_stream, Varlen{}, po);
}

int32_t dcp_unpack_combine(const void *recv_buf, void *result, float *global_lse, int32_t N, int64_t B, int64_t Hr,
                           int64_t D, int64_t stride_n, int32_t dtype, int32_t is_lse_base_on_e, int32_t return_lse,
                           void *cuda_stream) {
    const char *fn = "dcp_unpack_combine";
    int32_t st = check_common(fn, dtype, N, B, Hr, D);
    if (st != DCP_OK) return st;
    const int es = elem_size(dtype);
    const int64_t W = D + 4 / es;
    if (stride_n < B * Hr * W)
        return fail(DCP_ERR_INVALID_ARG, "%s: stride_n %lld < B*Hr*(D+P) = %lld", fn, (long long)stride_n,
                    (long long)(B * Hr * W));
    if ((stride_n * es) % 4 != 0)
        return fail(DCP_ERR_MISALIGNED, "%s: stride_n %lld elements is not a multiple of 4 bytes", fn,
                    (long long)stride_n);
    if (B == 0) return ok();
    if (!recv_buf || !result) return fail(DCP_ERR_INVALID_ARG, "%s: null buffer pointer", fn);
    if (return_lse && !global_lse) return fail(DCP_ERR_INVALID_ARG, "%s: return_lse set but global_lse is null", fn);
    if (!aligned(recv_buf, 16) || !aligned(result, 16))
        return fail(DCP_ERR_MISALIGNED, "%s: recv_buf and result must be 16-byte aligned", fn);
    if (return_lse && !aligned(global_lse, 4))
        return fail(DCP_ERR_MISALIGNED, "%s: global_lse must be 4-byte aligned", fn);

    dcp::CombineArgs a{};
    a.src = static_cast<const uint32_t *>(recv_buf);
    a.lses = nullptr;
    a.result = static_cast<uint32_t *>(result);
    a.glse = global_lse;
    a.units = B * Hr;
    a.shard_stride_w = stride_n * es / 4;
    a.lse_stride_n = 0;
    a.data_w = (int32_t)(D * es / 4);
    a.row_pitch_w = a.data_w + 1;
    a.chunks = a.data_w / 4;
    a.total_w = (int64_t)(N - 1) * a.shard_stride_w + a.units * a.row_pitch_w;
    a.N = N;
    a.base_e = is_lse_base_on_e ? 1 : 0;
    a.return_lse = return_lse ? 1 : 0;
    return dispatch_dtype<true>(dtype, a, static_cast<cudaStream_t>(cuda_stream));
}

}  // extern "C"

namespace {

// dcp_pack with the wait limit and the first-tile stall of the timeout check explicit.
int32_t pack_impl(const char *fn, const void *cp_attn_out, const float *cp_attn_lse, void *send_buf, int64_t B,
                  int64_t H, int64_t D, int32_t world_size, int32_t dtype, int64_t out_stride_b, int64_t out_stride_h,
                  int64_t lse_stride_b, void *cuda_stream, uint64_t wait_limit_ns, uint32_t stall_bytes) {
    t_last_pack_kernel = 0;
    int32_t st = check_common(fn, dtype, world_size, B, H, D);
    if (st != DCP_OK) return st;
    if (H % world_size != 0)
        return fail(DCP_ERR_SHAPE, "%s: H=%lld heads do not split evenly over %d ranks", fn, (long long)H,
                    (int)world_size);
    const int es = elem_size(dtype);
    if (out_stride_b < 1 || out_stride_h < 1)
        return fail(DCP_ERR_INVALID_ARG, "%s: output strides must be >= 1", fn);
    if ((out_stride_b * es) % 16 != 0 || (out_stride_h * es) % 16 != 0)
        return fail(DCP_ERR_MISALIGNED, "%s: output strides (%lld, %lld) are not multiples of 16 bytes", fn,
                    (long long)out_stride_b, (long long)out_stride_h);
    if (lse_stride_b < H)
        return fail(DCP_ERR_INVALID_ARG, "%s: lse_stride_b %lld < H = %lld", fn, (long long)lse_stride_b,
                    (long long)H);
    if (B == 0) return ok();
    if (!cp_attn_out || !cp_attn_lse || !send_buf) return fail(DCP_ERR_INVALID_ARG, "%s: null buffer pointer", fn);
    if (!aligned(cp_attn_out, 16) || !aligned(send_buf, 16))
        return fail(DCP_ERR_MISALIGNED, "%s: cp_attn_out and send_buf must be 16-byte aligned", fn);
    if (!aligned(cp_attn_lse, 4)) return fail(DCP_ERR_MISALIGNED, "%s: cp_attn_lse must be 4-byte aligned", fn);

    dcp::PackArgs a{};
    a.src = static_cast<const uint32_t *>(cp_attn_out);
    a.lse = reinterpret_cast<const uint32_t *>(cp_attn_lse);
    a.dst = static_cast<uint32_t *>(send_buf);
    a.B = B;
    a.Hr = H / world_size;
    a.rows = (int64_t)world_size * B * a.Hr;
    a.src_stride_b_w = out_stride_b * es / 4;
    a.src_stride_h_w = out_stride_h * es / 4;
    a.lse_stride_b = lse_stride_b;
    a.data_w = (int32_t)(D * es / 4);
    a.row_pitch_w = a.data_w + 1;
    if (a.rows >= (int64_t(1) << 32))
        return fail(DCP_ERR_INVALID_ARG, "%s: more than 2^32 packed rows", fn);
    a.per_rank_magic = magic64((uint64_t)(B * a.Hr));
    a.hr_magic = magic64((uint64_t)a.Hr);
    a.pitch_magic = (uint32_t)(((uint64_t(1) << 32) + (uint64_t)a.row_pitch_w - 1) / (uint64_t)a.row_pitch_w);
    a.wait_limit_ns = wait_limit_ns;
    a.stall_bytes = stall_bytes;
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    // Shapes measured on B200 (bf16, fractions of the measured copy peak).
    // * Rows of at most 128 bytes: 2 stages of up to 256 rows (about 32 KiB), copied as runs
    //   (D = 64: 0.84, against 0.72 for 3 stages of 64 rows with runs and 0.57 without).
    // * Otherwise 3 stages of up to 64 rows or 32 KiB (the best of 2-6 stages of 16-48 KiB and
    //   64-256 rows; at D = 128 the 64-row tile keeps 4 CTAs on an SM).  Runs of a token's
    //   contiguous heads win in launches of at most ~24 tiles per CTA (N = 8, B = 1024,
    //   D = 512: 0.91 against 0.85; N = 2, B = 16384, D = 128: 0.88 against 0.80) and lose in
    //   longer ones, where one copy per row keeps more copies in flight (N = 16, B = 16384:
    //   D = 512 0.94 against 0.87, D = 128 0.91 against 0.85).
    // * Longer launches: one tensor copy per tile of about 64 KiB (tokens x all heads of a rank),
    //   2 stages, one CTA per SM: N = 16, B = 16384: D = 512 1.00 against 0.94 for one copy per
    //   row, D = 128 0.94 against 0.91; N = 8, B = 16384: D = 512 0.98, D = 256 0.97, D = 128
    //   0.96 against 0.89; N = 3 / 4, B = 16384, D = 512: 0.98 / 0.94 against 0.92 / 0.91 for
    //   the rank-fast order below; D = 64: 0.84-0.91 against 0.83.
    // * Except rows of 1 KiB and more for 3 or 4 ranks in under ~64 tensor tiles per SM: 2 stages
    //   of up to 48 KiB, tiles in rank-fastest order, so that the tiles in flight read all ranks
    //   of the same tokens (N = 4, B = 4096, D = 512: 0.93 against 0.89 for the tensor copies).
    //   Shapes the tensor copy does not suit also take the kernels above or this one.
    PackGeom g;
    if (!pack_geometry<dcp::kPackStages, dcp::kPackMaxTileRows>(a, dcp::kPackMinStageWords, g))
        return fail(DCP_ERR_CUDA, "%s: cannot reserve shared memory", fn);
    const bool is_short = g.tiles <= 24 * g.cap;
    if (!is_short) {
        CUtensorMap map;
        int dims = 0;
        dcp::PackArgs t = a;
        if (pack_tma_plan(t, cp_attn_out, H, D, es, out_stride_b, out_stride_h, map, dims)) {
            const int64_t tma_tiles = (int64_t)world_size * ((a.B + t.tile_tokens - 1) / t.tile_tokens);
            const bool rank_fast = a.data_w >= 256 && (world_size == 3 || world_size == 4) &&
                                   tma_tiles < 64 * (int64_t)sm_count();
            if (!rank_fast)
                return dims == 3 ? launch_pack_tma<3>(fn, t, map, stream) : launch_pack_tma<4>(fn, t, map, stream);
        }
    }
    if (a.data_w <= 32) {
        if (!pack_geometry<2, 256>(a, 12288, g)) return fail(DCP_ERR_CUDA, "%s: cannot reserve shared memory", fn);
        return launch_pack<2, 256>(fn, a, g, true, stream);
    }
    if (is_short) return launch_pack<dcp::kPackStages, dcp::kPackMaxTileRows>(fn, a, g, true, stream);
    if (a.data_w >= 256 && world_size <= 4) {
        PackGeom r;
        if (!pack_geometry<2, 256, true>(a, 12288, r)) return fail(DCP_ERR_CUDA, "%s: cannot reserve shared memory", fn);
        return launch_pack<2, 256, true>(fn, a, r, false, stream);
    }
    return launch_pack<dcp::kPackStages, dcp::kPackMaxTileRows>(fn, a, g, false, stream);
}

}  // namespace

extern "C" {

int32_t dcp_pack(const void *cp_attn_out, const float *cp_attn_lse, void *send_buf, int64_t B, int64_t H, int64_t D,
                 int32_t world_size, int32_t dtype, int64_t out_stride_b, int64_t out_stride_h, int64_t lse_stride_b,
                 void *cuda_stream) {
    return pack_impl("dcp_pack", cp_attn_out, cp_attn_lse, send_buf, B, H, D, world_size, dtype, out_stride_b,
                     out_stride_h, lse_stride_b, cuda_stream, dcp::kWaitLimitNs, 0u);
}

int32_t dcp_testing_split_shape(int32_t kind, int32_t N, int32_t chunks, int32_t *out) {
    if (kind < 0 || kind > 2 || N < 1 || N > DCP_MAX_SHARDS || chunks < 1 || !out)
        return fail(DCP_ERR_INVALID_ARG, "dcp_testing_split_shape: kind %d, N %d, chunks %d", (int)kind, (int)N,
                    (int)chunks);
    const dcp_host::SplitShape plain = dcp_host::split_shape(N, chunks);
    dcp_host::SplitShape s = plain;
    if (kind == 1) {
        s = dcp_host::varlen_shape(N, chunks, plain);
        if (dcp_host::varlen_all_in_flight(s, N, chunks)) s.nb = 8;
    } else if (kind == 2) {
        s = dcp_host::pack_shape(N, chunks, plain);
    }
    out[0] = s.G;
    out[1] = s.cpl;
    out[2] = s.nb;
    out[3] = s.prefetch ? 1 : 0;
    return ok();
}

int32_t dcp_testing_last_pack_kernel(void) { return t_last_pack_kernel; }

int32_t dcp_testing_pack_tensor_shape(int64_t Hr, int64_t D, int32_t dtype, int64_t B, int32_t *out) {
    if (dtype < 0 || dtype > 2 || Hr < 1 || D < 1 || B < 1 || !out)
        return fail(DCP_ERR_INVALID_ARG, "dcp_testing_pack_tensor_shape: Hr %lld, D %lld, dtype %d, B %lld",
                    (long long)Hr, (long long)D, (int)dtype, (long long)B);
    int64_t k = 0, m = 0;
    if (pack_tma_shape(Hr, D, elem_size(dtype), B, k, m)) {
        out[0] = (int32_t)k;
        out[1] = (int32_t)m;
        out[2] = m == 1 ? 3 : 4;
    } else {
        out[0] = out[1] = out[2] = 0;
    }
    return ok();
}

int32_t dcp_testing_pack_stalled(const void *cp_attn_out, const float *cp_attn_lse, void *send_buf, int64_t B,
                                 int64_t H, int64_t D, int32_t world_size, int32_t dtype, int64_t out_stride_b,
                                 int64_t out_stride_h, int64_t lse_stride_b, void *cuda_stream) {
    // 16 bytes that never arrive keep each CTA's first tile waiting until the 20 ms limit
    return pack_impl("dcp_testing_pack_stalled", cp_attn_out, cp_attn_lse, send_buf, B, H, D, world_size, dtype,
                     out_stride_b, out_stride_h, lse_stride_b, cuda_stream, 20000000ull, 16u);
}

}  // extern "C"
