/*
 * dcp_oracle.c -- plain, slow, fp64 CPU oracle for the decode-context-parallel
 * (DCP) LSE-weighted combine, its pack step and its unpack+combine step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the smoke check and the bench's CPU-baseline
 * leg use it.  It shares no code, header, table or constant with the CUDA
 * library; its sole job is to say what the right answer is.
 *
 * Sources (web pages, cited by title and section):
 *   [A2A]   vLLM API docs, module vllm.v1.attention.ops.dcp_alltoall:
 *           function _lse_weighted_combine (the CPU reference of the combine)
 *           and function dcp_a2a_lse_reduce (pack -> All-to-All -> unpack+combine).
 *   [ASC]   vllm-ascend, vllm_ascend/attention/context_parallel/sfa_cp.py:
 *           _merge_dcp_outputs_with_torch (the same merge written as a softmax
 *           over the shard axis) and _get_dcp_local_seq_lens (KV sharding).
 *   [DIRECT] vLLM API docs, module vllm.v1.attention.ops.dcp:
 *           DirectDCPA2AWorkspace.lse_reduce, which also takes seq_lens and
 *           query_start_loc; oracle_lse_combine_varlen implements a stated
 *           reading of them (parity of that reading is unpinned).
 *
 * Everything is written as the definition, step by step, in double precision.
 * Loops run in the natural index order; there is no blocking, fusion or
 * reordering.  Build with -O2 -fno-fast-math so isnan/isinf keep their meaning.
 *
 * Dtype codes used by this file (its own, not the library's):
 *   0 = bfloat16, 1 = IEEE binary16, 2 = IEEE binary32, 3 = IEEE binary64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_BF16 0
#define ORC_FP16 1
#define ORC_FP32 2
#define ORC_F64 3

static int elem_size(int dtype) {
    switch (dtype) {
        case ORC_BF16: return 2;
        case ORC_FP16: return 2;
        case ORC_FP32: return 4;
        case ORC_F64: return 8;
        default: return 0;
    }
}

/* bfloat16 is the upper half of an IEEE binary32: put the 16 bits on top. */
static double decode_bf16(uint16_t bits) {
    uint32_t w = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* IEEE 754 binary16 from its definition: 1 sign bit, 5 exponent bits
 * (bias 15), 10 fraction bits; exponent 0 = zero/subnormal, 31 = inf/NaN. */
static double decode_fp16(uint16_t bits) {
    int sign = (bits >> 15) & 1;
    int expo = (bits >> 10) & 0x1f;
    int frac = bits & 0x3ff;
    double v;
    if (expo == 0) {
        v = ldexp((double)frac, -24);            /* frac * 2^-10 * 2^-14 */
    } else if (expo == 31) {
        v = frac ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + frac), expo - 25); /* (1 + frac/1024) * 2^(expo-15) */
    }
    return sign ? -v : v;
}

/* Element i of an array of the given dtype, as a double. */
static double load_elem(const void *base, int dtype, int64_t i) {
    switch (dtype) {
        case ORC_BF16: return decode_bf16(((const uint16_t *)base)[i]);
        case ORC_FP16: return decode_fp16(((const uint16_t *)base)[i]);
        case ORC_FP32: return (double)((const float *)base)[i];
        case ORC_F64: return ((const double *)base)[i];
        default: return NAN;
    }
}

double oracle_decode(const void *base, int dtype, int64_t i) { return load_elem(base, dtype, i); }

/* Number of output-dtype slots that hold one fp32 LSE in a packed row.
 * [A2A] dcp_a2a_lse_reduce sends each output row and its fp32 LSE together in
 * one buffer of the output dtype; the plainest lossless reading is
 * 4 bytes / itemsize. */
int oracle_lse_pack_dim(int dtype) {
    if (dtype == ORC_BF16 || dtype == ORC_FP16) return 2;
    if (dtype == ORC_FP32) return 1;
    return -1;
}

/*
 * Pack step of [A2A] dcp_a2a_lse_reduce: the send buffer has shape
 * [world_size, B, H/world_size, D + lse_pack_dim] in the output dtype, and
 * chunk r of dim 0 goes to rank r, so rank r receives heads
 * [r*Hr, (r+1)*Hr).  Row (r, b, h) holds out[b, r*Hr + h, 0:D] followed by the
 * 4 bytes of lse[b, r*Hr + h] (its bit pattern, in memory order).
 * Strides are in elements; the innermost dimension of out is contiguous.
 * Returns 0, or -1 on a bad argument.
 */
int oracle_pack(const void *cp_attn_out, const float *cp_attn_lse, void *send_buf,
                int64_t B, int64_t H, int64_t D, int world_size, int dtype,
                int64_t out_stride_b, int64_t out_stride_h, int64_t lse_stride_b) {
    int es = elem_size(dtype);
    int pack = oracle_lse_pack_dim(dtype);
    if (es == 0 || pack < 0 || world_size < 1 || H % world_size != 0) return -1;
    int64_t Hr = H / world_size;
    int64_t W = D + pack;
    const unsigned char *src = (const unsigned char *)cp_attn_out;
    unsigned char *dst = (unsigned char *)send_buf;
    for (int64_t r = 0; r < world_size; ++r) {
        for (int64_t b = 0; b < B; ++b) {
            for (int64_t h = 0; h < Hr; ++h) {
                int64_t head = r * Hr + h;
                int64_t dst_row = (r * B + b) * Hr + h;
                unsigned char *d = dst + dst_row * W * es;
                const unsigned char *s = src + (b * out_stride_b + head * out_stride_h) * es;
                memcpy(d, s, (size_t)(D * es));
                memcpy(d + D * es, &cp_attn_lse[b * lse_stride_b + head], 4);
            }
        }
    }
    return 0;
}

/*
 * Split a packed receive buffer [N, B, Hr, D + pack] (shard stride stride_n
 * elements) into outputs [N, B, Hr, D] (raw elements, contiguous) and
 * lses [N, B, Hr] (fp32, contiguous).  Inverse of the row layout above.
 */
int oracle_unpack(const void *recv_buf, void *outputs, float *lses,
                  int N, int64_t B, int64_t Hr, int64_t D, int64_t stride_n, int dtype) {
    int es = elem_size(dtype);
    int pack = oracle_lse_pack_dim(dtype);
    if (es == 0 || pack < 0 || N < 1) return -1;
    int64_t W = D + pack;
    const unsigned char *src = (const unsigned char *)recv_buf;
    unsigned char *dst = (unsigned char *)outputs;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < B; ++b) {
            for (int64_t h = 0; h < Hr; ++h) {
                const unsigned char *row = src + (n * stride_n + (b * Hr + h) * W) * es;
                int64_t unit = (n * B + b) * Hr + h;
                memcpy(dst + unit * D * es, row, (size_t)(D * es));
                memcpy(&lses[unit], row + D * es, 4);
            }
        }
    }
    return 0;
}

/*
 * One (b, h) row of the combine, the [COMBINE] rules in their order.  `empty`
 * (NULL = none) marks shards whose row holds no context: their LSE counts as
 * -inf and their output row is never read.  l and w are N-entry scratch.
 */
static void combine_row(const void *outputs, int out_dtype, const void *lses, int lse_dtype,
                        double *result, double *global_lse, int N, int64_t b, int64_t h,
                        int64_t B, int64_t H, int64_t D, int64_t out_stride_n, int64_t lse_stride_n,
                        int is_lse_base_on_e, int return_lse, const int *empty,
                        double *l, double *w) {
    (void)B; /* rows are addressed (b * H + h); B is the layout's extent */
    /* step 1: sanitise */
    for (int n = 0; n < N; ++n) {
        double v = (empty && empty[n]) ? -INFINITY
                                       : load_elem(lses, lse_dtype, n * lse_stride_n + b * H + h);
        l[n] = (isnan(v) || isinf(v)) ? -INFINITY : v;
    }
    /* step 2: max over shards, an all -inf max becomes 0 */
    double m = l[0];
    for (int n = 1; n < N; ++n)
        if (l[n] > m) m = l[n];
    if (m == -INFINITY) m = 0.0;
    /* step 3: weights */
    for (int n = 0; n < N; ++n) {
        w[n] = is_lse_base_on_e ? exp(l[n] - m) : pow(2.0, l[n] - m);
        if (isnan(w[n])) w[n] = 0.0;
    }
    /* step 4: normalise by the clamped sum */
    double S = 0.0;
    for (int n = 0; n < N; ++n) S += w[n];
    double denom = S < 1e-10 ? 1e-10 : S;
    for (int n = 0; n < N; ++n) w[n] = w[n] / denom;
    /* step 5: weighted sum over shards */
    for (int64_t d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int n = 0; n < N; ++n)
            if (!(empty && empty[n]))
                acc += load_elem(outputs, out_dtype, n * out_stride_n + (b * H + h) * D + d) * w[n];
        result[(b * H + h) * D + d] = acc;
    }
    /* step 6: global LSE from the unclamped sum */
    if (return_lse)
        global_lse[b * H + h] = (is_lse_base_on_e ? log(S) : log2(S)) + m;
}

/*
 * The combine, following [A2A] _lse_weighted_combine step by step, for every
 * token b and head h:
 *   1. an LSE that is NaN or +-inf becomes -inf;
 *   2. m = max over shards of the LSE; if m is -inf it becomes 0;
 *   3. w_n = exp(l_n - m) (base e) or 2^(l_n - m) (base 2); a NaN weight is 0;
 *   4. S = sum_n w_n, and each weight is divided by max(S, 1e-10);
 *   5. result[b,h,:] = sum_n w_n * outputs[n,b,h,:];
 *   6. global_lse[b,h] = log(S) + m (natural log, or log2 for base 2), with
 *      the unclamped S.
 * outputs: [N, B, H, D] of out_dtype, shard stride out_stride_n elements;
 * lses: [N, B, H] of lse_dtype (fp32 or f64), shard stride lse_stride_n.
 * result: [B, H, D] f64; global_lse: [B, H] f64 (written when return_lse).
 */
int oracle_lse_combine(const void *outputs, int out_dtype, const void *lses, int lse_dtype,
                       double *result, double *global_lse,
                       int N, int64_t B, int64_t H, int64_t D,
                       int64_t out_stride_n, int64_t lse_stride_n,
                       int is_lse_base_on_e, int return_lse) {
    if (N < 1 || elem_size(out_dtype) == 0) return -1;
    if (lse_dtype != ORC_FP32 && lse_dtype != ORC_F64) return -1;
    double *l = (double *)malloc(sizeof(double) * (size_t)N);
    double *w = (double *)malloc(sizeof(double) * (size_t)N);
    if (!l || !w) { free(l); free(w); return -1; }
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h)
            combine_row(outputs, out_dtype, lses, lse_dtype, result, global_lse, N, b, h, B, H, D,
                        out_stride_n, lse_stride_n, is_lse_base_on_e, return_lse, NULL, l, w);
    free(l);
    free(w);
    return 0;
}

/*
 * Unpack + combine of the receive buffer [N, B, Hr, D + pack] of [A2A]
 * dcp_a2a_lse_reduce, done the plain way: unpack into separate arrays, then
 * run the combine above on them.  Output [B, Hr, D] f64 (+ [B, Hr] f64).
 */
int oracle_unpack_combine(const void *recv_buf, int dtype, double *result, double *global_lse,
                          int N, int64_t B, int64_t Hr, int64_t D, int64_t stride_n,
                          int is_lse_base_on_e, int return_lse) {
    int es = elem_size(dtype);
    if (es == 0 || N < 1) return -1;
    size_t units = (size_t)N * (size_t)B * (size_t)Hr;
    void *outs = malloc(units * (size_t)D * (size_t)es + 1);
    float *lses = (float *)malloc(units * sizeof(float) + 1);
    if (!outs || !lses) { free(outs); free(lses); return -1; }
    int rc = oracle_unpack(recv_buf, outs, lses, N, B, Hr, D, stride_n, dtype);
    if (rc == 0)
        rc = oracle_lse_combine(outs, dtype, lses, ORC_FP32, result, global_lse, N, B, Hr, D,
                                B * Hr * D, B * Hr, is_lse_base_on_e, return_lse);
    free(outs);
    free(lses);
    return rc;
}

/*
 * The same merge as stated in [ASC] _merge_dcp_outputs_with_torch, kept as an
 * independent second expression of the method: non-finite LSEs are masked to
 * -inf, the weights are a softmax over the shard axis (max-shifted exp divided
 * by the sum), a NaN weight becomes 0, and the output is the weighted sum.
 * This form has no clamp and no LSE output; an all -inf row gives NaN weights
 * (-inf minus -inf), which the NaN rule turns into 0.
 * Same argument layout as oracle_lse_combine (base e only).
 */
int oracle_softmax_merge(const void *outputs, int out_dtype, const void *lses, int lse_dtype,
                         double *result, int N, int64_t B, int64_t H, int64_t D,
                         int64_t out_stride_n, int64_t lse_stride_n) {
    if (N < 1 || elem_size(out_dtype) == 0) return -1;
    if (lse_dtype != ORC_FP32 && lse_dtype != ORC_F64) return -1;
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    if (!p) return -1;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            double mx = -INFINITY;
            for (int n = 0; n < N; ++n) {
                double v = load_elem(lses, lse_dtype, n * lse_stride_n + b * H + h);
                p[n] = isfinite(v) ? v : -INFINITY;
                if (p[n] > mx) mx = p[n];
            }
            double z = 0.0;
            for (int n = 0; n < N; ++n) {
                p[n] = exp(p[n] - mx);
                z += p[n];
            }
            for (int n = 0; n < N; ++n) {
                p[n] = p[n] / z;
                if (isnan(p[n])) p[n] = 0.0;
            }
            for (int64_t d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int n = 0; n < N; ++n)
                    acc += load_elem(outputs, out_dtype, n * out_stride_n + (b * H + h) * D + d) * p[n];
                result[(b * H + h) * D + d] = acc;
            }
        }
    }
    free(p);
    return 0;
}

/*
 * Brute-force softmax attention for one decode token over the KV positions
 * listed in pos[0..npos-1] -- the quantity a DCP shard produces before the
 * combine ([ASC]: each rank attends over its own KV shard and returns its
 * output with its LSE).
 * q: [H, D]; k, v: [L, H, D] (all of dtype); scale multiplies q.k.
 * out: [H, D] f64 = sum_p softmax_p(s) v_p, with s_p = scale * q.k_p;
 * lse: [H] f64 = log(sum_p exp(s_p)) (base e) or that value / ln 2 (base 2).
 * An empty position list gives lse = -inf and out = 0.
 */
int oracle_attention(const void *q, const void *k, const void *v, int dtype,
                     double *out, double *lse, int64_t H, int64_t D,
                     const int64_t *pos, int64_t npos, double scale, int is_lse_base_on_e) {
    if (elem_size(dtype) == 0) return -1;
    double *s = (double *)malloc(sizeof(double) * (size_t)(npos > 0 ? npos : 1));
    if (!s) return -1;
    for (int64_t h = 0; h < H; ++h) {
        double mx = -INFINITY;
        for (int64_t i = 0; i < npos; ++i) {
            double dot = 0.0;
            for (int64_t d = 0; d < D; ++d)
                dot += load_elem(q, dtype, h * D + d) * load_elem(k, dtype, (pos[i] * H + h) * D + d);
            s[i] = scale * dot;
            if (s[i] > mx) mx = s[i];
        }
        double z = 0.0;
        for (int64_t i = 0; i < npos; ++i) z += exp(s[i] - mx);
        for (int64_t d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int64_t i = 0; i < npos; ++i)
                acc += exp(s[i] - mx) * load_elem(v, dtype, (pos[i] * H + h) * D + d);
            out[h * D + d] = npos > 0 ? acc / z : 0.0;
        }
        double lse_e = npos > 0 ? log(z) + mx : -INFINITY;
        lse[h] = is_lse_base_on_e ? lse_e : lse_e / log(2.0);
    }
    free(s);
    return 0;
}

/*
 * KV tokens held by one rank under interleaved sharding, following [ASC]
 * _get_dcp_local_seq_lens: blocks of `interleave` consecutive positions are
 * dealt round-robin to the cp_size ranks.
 */
int64_t oracle_local_seq_len(int64_t seq_len, int64_t cp_size, int64_t rank, int64_t interleave) {
    int64_t base = seq_len / interleave / cp_size * interleave;
    int64_t rem = seq_len - base * cp_size - rank * interleave;
    if (rem < 0) rem = 0;
    if (rem > interleave) rem = interleave;
    return base + rem;
}

/*
 * Variable-length combine: the receive-side reduce of [vLLM API docs,
 * vllm.v1.attention.ops.dcp, DirectDCPA2AWorkspace.lse_reduce], which takes
 * optional seq_lens and query_start_loc.  The pages do not say what the op does
 * with them; the reading taken here (parity of this reading is unpinned):
 *   - token t belongs to request r when query_start_loc[r] <= t <
 *     query_start_loc[r + 1] (num_reqs + 1 entries); tokens outside every
 *     request have no context at all;
 *   - shard n holds oracle_local_seq_len(seq_lens[r], N, n, interleave) KV
 *     positions of request r ([ASC] _get_dcp_local_seq_lens); a shard that
 *     holds none (a local length <= 0, which a negative seq_lens entry gives) is
 *     empty: its LSE counts as -inf and its output row is not
 *     read (it may never have been written);
 *   - everything else is oracle_lse_combine.
 * Same layouts as oracle_lse_combine (split layout, shard strides).
 */
int oracle_lse_combine_varlen(const void *outputs, int out_dtype, const void *lses, int lse_dtype,
                              double *result, double *global_lse, int N, int64_t B, int64_t H, int64_t D,
                              int64_t out_stride_n, int64_t lse_stride_n, const int32_t *seq_lens,
                              const int32_t *query_start_loc, int num_reqs, int interleave,
                              int is_lse_base_on_e, int return_lse) {
    if (N < 1 || elem_size(out_dtype) == 0 || interleave < 1 || num_reqs < 0) return -1;
    if (lse_dtype != ORC_FP32 && lse_dtype != ORC_F64) return -1;
    double *l = (double *)malloc(sizeof(double) * (size_t)N);
    double *w = (double *)malloc(sizeof(double) * (size_t)N);
    int *empty = (int *)malloc(sizeof(int) * (size_t)N);
    if (!l || !w || !empty) { free(l); free(w); free(empty); return -1; }
    for (int64_t b = 0; b < B; ++b) {
        int req = -1;
        for (int r = 0; r < num_reqs; ++r)
            if (query_start_loc[r] <= b && b < query_start_loc[r + 1]) req = r;
        for (int n = 0; n < N; ++n)
            empty[n] = req < 0 || oracle_local_seq_len(seq_lens[req], N, n, interleave) <= 0;
        for (int64_t h = 0; h < H; ++h)
            combine_row(outputs, out_dtype, lses, lse_dtype, result, global_lse, N, b, h, B, H, D,
                        out_stride_n, lse_stride_n, is_lse_base_on_e, return_lse, empty, l, w);
    }
    free(l);
    free(w);
    free(empty);
    return 0;
}
