/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the fused per-token operators
 * of a packed audio-video diffusion-transformer block.
 *
 * TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check and the
 * benchmark's CPU-baseline leg; never by the product path.  It shares no code
 * with the CUDA library.  Each function below is the textbook definition of
 * its operator written out with scalar loops, in the order the definition
 * states it; the only parallelism is an OpenMP loop over independent rows.
 *
 * Pages: "Why Real-Time MiniMax H3 Serving Requires More Than a Faster DiT",
 * "Key takeaways" bullets 1-2; "MiniMax H3 通过 vLLM-Omni 实现 FastH3 实时推理",
 * "vLLM-Omni 中的系统级优化" bullets 1-2.  Those passages name the operators
 * and the padding-free packed sequence but print no formula, so every formula
 * here is the plainest standard reading (see the per-function comments).
 *
 * Parity pins: every function is pinned by the CPU tests (closed forms,
 * invariants, library special cases); none is "parity unpinned".
 */
#include "oracle.h"

#include <math.h>
#include <stddef.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ bf16 */

double oracle_bf16_to_f64(uint16_t h)
{
    /* A bf16 value is the upper half of an IEEE binary32 value. */
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

uint16_t oracle_f64_to_bf16(double x)
{
    /* bf16: 1 sign bit, 8 exponent bits (bias 127), 7 stored mantissa bits.
     * Between 2^e and 2^(e+1) (e >= -126) the spacing is 2^(e-7); below the
     * smallest normal 2^-126 the spacing stays 2^-133 (subnormals).  Round
     * |x| to the nearest multiple of that spacing with ties to even
     * (nearbyint in the default rounding mode), then read off the bits of
     * the now exactly representable value. */
    if (isnan(x))
        return signbit(x) ? 0xFFC0u : 0x7FC0u;
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double ax = fabs(x);
    if (isinf(ax))
        return sign | 0x7F80u;
    if (ax == 0.0)
        return sign;
    int e = ilogb(ax);
    if (e < -126)
        e = -126;
    double spacing = ldexp(1.0, e - 7);
    double r = nearbyint(ax / spacing) * spacing;
    if (r >= ldexp(1.0, 128))
        return sign | 0x7F80u; /* rounds past the largest finite bf16 */
    float f = (float)r;        /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return sign | (uint16_t)(u >> 16);
}

static double ld(const uint16_t* p) { return oracle_bf16_to_f64(*p); }

/* Element idx of a per-sequence modulation vector stored as bf16 bits or as
 * fp32 (f32 != 0), widened exactly. */
static double ldm(const void* base, int64_t idx, int f32)
{
    if (f32)
        return (double)((const float*)base)[idx];
    return oracle_bf16_to_f64(((const uint16_t*)base)[idx]);
}

/* -------------------------------------------------------- packed rows */

/* Offset of the per-sequence vectors that valid row r of sequence b uses.
 * One vector set per sequence: b * seq_stride.  With per-stream vectors
 * (rope_grid != NULL) the joint audio-video sequence holds its T*H*W video
 * rows first and its audio rows after them; video rows use the set at
 * b * seq_stride, audio rows the set audio_offset elements further on.  A row's
 * index in its whole sequence is its local index plus the sequence's position
 * offset (pos_offset NULL: 0). */
static int64_t vec_offset(int32_t b, int64_t r, int64_t seq_stride, const int32_t* rope_grid,
                          const int32_t* pos_offset, int64_t audio_offset)
{
    int64_t off = (int64_t)b * seq_stride;
    if (rope_grid) {
        int64_t thw = (int64_t)rope_grid[3 * b] * rope_grid[3 * b + 1] * rope_grid[3 * b + 2];
        int64_t g = r + (pos_offset ? pos_offset[b] : 0); /* index in the whole sequence */
        if (g >= thw)
            off += audio_offset;
    }
    return off;
}

/* The padded buffer holds num_seqs sequences; sequence b owns padded rows
 * [cu_seqlens_padded[b], cu_seqlens_padded[b+1]) and its first
 * cu_seqlens[b+1] - cu_seqlens[b] rows are valid (the rest is structural
 * suffix padding, which is neither read nor written).  Returns 1 and fills
 * (*seq, *local) for a valid row, 0 for padding. */
static int locate_row(const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                      int32_t num_seqs, int64_t row, int32_t* seq, int64_t* local)
{
    for (int32_t b = 0; b < num_seqs; ++b) {
        if (row >= cu_seqlens_padded[b] && row < cu_seqlens_padded[b + 1]) {
            int64_t r = row - cu_seqlens_padded[b];
            int64_t len = (int64_t)cu_seqlens[b + 1] - cu_seqlens[b];
            if (r < len) {
                *seq = b;
                *local = r;
                return 1;
            }
            return 0;
        }
    }
    return 0;
}

static int64_t row_at(const int64_t* rows, int64_t i) { return rows ? rows[i] : i; }

static int seqlens_ok(const int32_t* cs, const int32_t* cp, int32_t num_seqs, int64_t num_rows_padded)
{
    if (num_seqs < 0 || num_rows_padded < 0)
        return 0;
    if (num_seqs == 0)
        return 1;
    if (!cs || !cp || cs[0] != 0 || cp[0] != 0)
        return 0;
    for (int32_t b = 0; b < num_seqs; ++b) {
        if (cs[b + 1] < cs[b] || cp[b + 1] < cp[b])
            return 0;
        if (cs[b + 1] - cs[b] > cp[b + 1] - cp[b])
            return 0;
    }
    return cp[num_seqs] <= num_rows_padded;
}

static void put(uint16_t* out_bits, double* out_f64, int64_t idx, double v)
{
    out_bits[idx] = oracle_f64_to_bf16(v);
    if (out_f64)
        out_f64[idx] = v;
}

/* ------------------------------------------------------------ rotary */

/* Rotation angle of pair j (elements 2j, 2j+1) of a head of width head_dim.
 * 1D rows: angle = p * theta^(-2j/head_dim), the standard rotary frequency.
 * 3D rows: head_dim is split into sections of sec_t, sec_h, sec_w elements
 * (in that order); pair j lies in the section of axis s with width d_s and
 * local pair index j', and rotates by p_s * theta^(-2j'/d_s). */
static double rope_angle(int j, int head_dim, int is3d, const int64_t pos3[3], int64_t pos1,
                         const int32_t sec[3], double theta)
{
    if (!is3d)
        return (double)pos1 * pow(theta, -2.0 * (double)j / (double)head_dim);
    int first = 0; /* first pair of the current section */
    for (int s = 0; s < 3; ++s) {
        int npairs = sec[s] / 2;
        if (j < first + npairs) {
            int jl = j - first;
            return (double)pos3[s] * pow(theta, -2.0 * (double)jl / (double)sec[s]);
        }
        first += npairs;
    }
    return 0.0; /* unreachable when the sections sum to head_dim */
}

/* One head: RMSNorm over head_dim, times the weight, then rotate every
 * pair of elements (i0, i1) of pair index j by its angle:
 *   ms    = (1/D) * sum_i x_i^2
 *   y_i   = x_i / sqrt(ms + eps) * w_i
 *   o_i0  = y_i0 cos(a_j) - y_i1 sin(a_j)
 *   o_i1  = y_i0 sin(a_j) + y_i1 cos(a_j)
 * Pair j is (2j, 2j+1) for interleaved rotary embedding, (j, j + D/2) for the
 * half-split ("rotate half") layout; with no rotary embedding o = y. */
static void rmsnorm_rope_head(const uint16_t* x, const uint16_t* w, int D, double eps,
                              int is3d, const int64_t pos3[3], int64_t pos1,
                              const int32_t sec[3], double theta, int rope_mode,
                              uint16_t* out_bits, double* out_f64, double* y)
{
    double ms = 0.0;
    for (int i = 0; i < D; ++i)
        ms += ld(&x[i]) * ld(&x[i]);
    ms /= (double)D;
    double inv_rms = 1.0 / sqrt(ms + eps);
    for (int i = 0; i < D; ++i)
        y[i] = ld(&x[i]) * inv_rms * ld(&w[i]);
    if (rope_mode == ORACLE_ROPE_NONE) {
        for (int i = 0; i < D; ++i)
            put(out_bits, out_f64, i, y[i]);
        return;
    }
    for (int j = 0; j < D / 2; ++j) {
        double a = rope_angle(j, D, is3d, pos3, pos1, sec, theta);
        double c = cos(a), s = sin(a);
        int i0 = rope_mode == ORACLE_ROPE_HALF ? j : 2 * j;
        int i1 = rope_mode == ORACLE_ROPE_HALF ? j + D / 2 : 2 * j + 1;
        double y0 = y[i0], y1 = y[i1];
        put(out_bits, out_f64, i0, y0 * c - y1 * s);
        put(out_bits, out_f64, i1, y0 * s + y1 * c);
    }
}

int oracle_qk_rmsnorm_rope(
    const uint16_t* q, int64_t q_row_stride,
    const uint16_t* k, int64_t k_row_stride,
    const uint16_t* q_weight, const uint16_t* k_weight,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded,
    int32_t num_q_heads, int32_t num_k_heads, int32_t head_dim,
    const int32_t* rope_grid, int32_t sec_t, int32_t sec_h, int32_t sec_w,
    double rope_theta, double eps,
    uint16_t* q_out, uint16_t* k_out, double* q_out_f64, double* k_out_f64,
    const int64_t* rows, int64_t num_rows)
{
    return oracle_qk_rmsnorm_rope_ex(q, q_row_stride, k, k_row_stride, q_weight, k_weight, cu_seqlens,
                                     cu_seqlens_padded, num_seqs, num_rows_padded, num_q_heads, num_k_heads,
                                     head_dim, rope_grid, sec_t, sec_h, sec_w, rope_theta, eps,
                                     ORACLE_ROPE_INTERLEAVED, q_out, k_out, q_out_f64, k_out_f64, rows, num_rows);
}

int oracle_qk_rmsnorm_rope_ex(
    const uint16_t* q, int64_t q_row_stride,
    const uint16_t* k, int64_t k_row_stride,
    const uint16_t* q_weight, const uint16_t* k_weight,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded,
    int32_t num_q_heads, int32_t num_k_heads, int32_t head_dim,
    const int32_t* rope_grid, int32_t sec_t, int32_t sec_h, int32_t sec_w,
    double rope_theta, double eps, int32_t rope_mode,
    uint16_t* q_out, uint16_t* k_out, double* q_out_f64, double* k_out_f64,
    const int64_t* rows, int64_t num_rows)
{
    return oracle_qk_rmsnorm_rope_shard(q, q_row_stride, k, k_row_stride, q_weight, k_weight, cu_seqlens,
                                        cu_seqlens_padded, num_seqs, num_rows_padded, num_q_heads, num_k_heads,
                                        head_dim, rope_grid, sec_t, sec_h, sec_w, rope_theta, eps, rope_mode, NULL,
                                        q_out, k_out, q_out_f64, k_out_f64, rows, num_rows);
}

int oracle_qk_rmsnorm_rope_shard(
    const uint16_t* q, int64_t q_row_stride,
    const uint16_t* k, int64_t k_row_stride,
    const uint16_t* q_weight, const uint16_t* k_weight,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded,
    int32_t num_q_heads, int32_t num_k_heads, int32_t head_dim,
    const int32_t* rope_grid, int32_t sec_t, int32_t sec_h, int32_t sec_w,
    double rope_theta, double eps, int32_t rope_mode, const int32_t* pos_offset,
    uint16_t* q_out, uint16_t* k_out, double* q_out_f64, double* k_out_f64,
    const int64_t* rows, int64_t num_rows)
{
    if (!q || !k || !q_weight || !k_weight || !q_out || !k_out)
        return -1;
    if (rope_mode != ORACLE_ROPE_INTERLEAVED && rope_mode != ORACLE_ROPE_HALF && rope_mode != ORACLE_ROPE_NONE)
        return -1;
    if (head_dim <= 0 || head_dim % 2 || head_dim > 1024 || num_q_heads < 0 || num_k_heads < 0)
        return -1;
    if (q_row_stride < (int64_t)num_q_heads * head_dim || k_row_stride < (int64_t)num_k_heads * head_dim)
        return -1;
    const int32_t sec[3] = {sec_t, sec_h, sec_w};
    if (rope_grid) {
        for (int s = 0; s < 3; ++s)
            if (sec[s] < 0 || sec[s] % 2)
                return -1;
        if (sec_t + sec_h + sec_w != head_dim)
            return -1;
    }
    if (!seqlens_ok(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded))
        return -1;
    int64_t n = rows ? num_rows : num_rows_padded;

#pragma omp parallel
    {
        double y[1024];
#pragma omp for schedule(dynamic, 8)
        for (int64_t i = 0; i < n; ++i) {
            int64_t row = row_at(rows, i), r;
            int32_t b;
            if (row < 0 || row >= num_rows_padded)
                continue;
            if (!locate_row(cu_seqlens, cu_seqlens_padded, num_seqs, row, &b, &r))
                continue;
            /* Positions: the row's index in its whole sequence is g = r plus
             * the sequence's position offset (non-zero when this buffer holds
             * one rank's slice of a longer sequence).  A row inside the
             * sequence's T x H x W video grid (t-major, then h, then w) takes
             * 3D positions; every other row takes the 1D position counted
             * from the end of the grid. */
            const int64_t g = r + (pos_offset ? pos_offset[b] : 0);
            int is3d = 0;
            int64_t pos3[3] = {0, 0, 0}, pos1 = g;
            if (rope_grid) {
                int64_t T = rope_grid[3 * b], H = rope_grid[3 * b + 1], W = rope_grid[3 * b + 2];
                int64_t thw = T * H * W;
                if (g < thw) {
                    is3d = 1;
                    pos3[0] = g / (H * W);
                    pos3[1] = (g / W) % H;
                    pos3[2] = g % W;
                } else {
                    pos1 = g - thw;
                }
            }
            for (int32_t h = 0; h < num_q_heads; ++h) {
                int64_t off = row * q_row_stride + (int64_t)h * head_dim;
                rmsnorm_rope_head(q + off, q_weight, head_dim, eps, is3d, pos3, pos1, sec, rope_theta, rope_mode,
                                  q_out + off, q_out_f64 ? q_out_f64 + off : NULL, y);
            }
            for (int32_t h = 0; h < num_k_heads; ++h) {
                int64_t off = row * k_row_stride + (int64_t)h * head_dim;
                rmsnorm_rope_head(k + off, k_weight, head_dim, eps, is3d, pos3, pos1, sec, rope_theta, rope_mode,
                                  k_out + off, k_out_f64 ? k_out_f64 + off : NULL, y);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------- adaLN */

int oracle_adaln_modulate(
    const uint16_t* x, int64_t x_row_stride,
    const uint16_t* shift, const uint16_t* scale, int64_t mod_seq_stride,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, double eps,
    uint16_t* out, int64_t out_row_stride, double* out_f64,
    const int64_t* rows, int64_t num_rows)
{
    return oracle_adaln_modulate_ex(x, x_row_stride, shift, scale, mod_seq_stride, 0, cu_seqlens,
                                    cu_seqlens_padded, num_seqs, num_rows_padded, hidden, eps, out,
                                    out_row_stride, out_f64, rows, num_rows);
}

int oracle_adaln_modulate_ex(
    const uint16_t* x, int64_t x_row_stride,
    const void* shift, const void* scale, int64_t mod_seq_stride, int32_t mod_f32,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, double eps,
    uint16_t* out, int64_t out_row_stride, double* out_f64,
    const int64_t* rows, int64_t num_rows)
{
    return oracle_adaln_modulate_av(x, x_row_stride, shift, scale, mod_seq_stride, mod_f32, NULL, NULL, 0, cu_seqlens,
                                    cu_seqlens_padded, num_seqs, num_rows_padded, hidden, eps, out,
                                    out_row_stride, out_f64, rows, num_rows);
}

int oracle_adaln_modulate_av(
    const uint16_t* x, int64_t x_row_stride,
    const void* shift, const void* scale, int64_t mod_seq_stride, int32_t mod_f32,
    const int32_t* rope_grid, const int32_t* pos_offset, int64_t audio_offset,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, double eps,
    uint16_t* out, int64_t out_row_stride, double* out_f64,
    const int64_t* rows, int64_t num_rows)
{
    if (!x || !shift || !scale || !out || hidden <= 0)
        return -1;
    if (x_row_stride < hidden || out_row_stride < hidden || mod_seq_stride < 0)
        return -1;
    if (!seqlens_ok(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded))
        return -1;
    int64_t n = rows ? num_rows : num_rows_padded;

#pragma omp parallel for schedule(dynamic, 8)
    for (int64_t i = 0; i < n; ++i) {
        int64_t row = row_at(rows, i), r;
        int32_t b;
        if (row < 0 || row >= num_rows_padded)
            continue;
        if (!locate_row(cu_seqlens, cu_seqlens_padded, num_seqs, row, &b, &r))
            continue;
        const uint16_t* xr = x + row * x_row_stride;
        const int64_t mb = vec_offset(b, r, mod_seq_stride, rope_grid, pos_offset, audio_offset);
        /* LayerNorm without affine: mean, then the biased variance about it. */
        double mean = 0.0;
        for (int32_t c = 0; c < hidden; ++c)
            mean += ld(&xr[c]);
        mean /= (double)hidden;
        double var = 0.0;
        for (int32_t c = 0; c < hidden; ++c)
            var += (ld(&xr[c]) - mean) * (ld(&xr[c]) - mean);
        var /= (double)hidden;
        double inv_std = 1.0 / sqrt(var + eps);
        /* Modulation: x_hat * (1 + scale) + shift. */
        for (int32_t c = 0; c < hidden; ++c) {
            double xhat = (ld(&xr[c]) - mean) * inv_std;
            double v = xhat * (1.0 + ldm(scale, mb + c, mod_f32)) + ldm(shift, mb + c, mod_f32);
            put(out, out_f64, row * out_row_stride + c, v);
        }
    }
    return 0;
}

/* ---------------------------------------------------- gated residual */

int oracle_gated_residual(
    const uint16_t* x, int64_t x_row_stride,
    const uint16_t* y, int64_t y_row_stride,
    const uint16_t* gate, int64_t gate_seq_stride,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden,
    uint16_t* out, int64_t out_row_stride, double* out_f64,
    const int64_t* rows, int64_t num_rows)
{
    return oracle_gated_residual_ex(x, x_row_stride, y, y_row_stride, gate, gate_seq_stride, 0, cu_seqlens,
                                    cu_seqlens_padded, num_seqs, num_rows_padded, hidden, out, out_row_stride,
                                    out_f64, rows, num_rows);
}

int oracle_gated_residual_ex(
    const uint16_t* x, int64_t x_row_stride,
    const uint16_t* y, int64_t y_row_stride,
    const void* gate, int64_t gate_seq_stride, int32_t gate_f32,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden,
    uint16_t* out, int64_t out_row_stride, double* out_f64,
    const int64_t* rows, int64_t num_rows)
{
    return oracle_gated_residual_av(x, x_row_stride, y, y_row_stride, gate, gate_seq_stride, gate_f32, NULL, NULL, 0,
                                    cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded, hidden, out,
                                    out_row_stride, out_f64, rows, num_rows);
}

int oracle_gated_residual_av(
    const uint16_t* x, int64_t x_row_stride,
    const uint16_t* y, int64_t y_row_stride,
    const void* gate, int64_t gate_seq_stride, int32_t gate_f32,
    const int32_t* rope_grid, const int32_t* pos_offset, int64_t audio_offset,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden,
    uint16_t* out, int64_t out_row_stride, double* out_f64,
    const int64_t* rows, int64_t num_rows)
{
    if (!x || !y || !gate || !out || hidden <= 0)
        return -1;
    if (x_row_stride < hidden || y_row_stride < hidden || out_row_stride < hidden || gate_seq_stride < 0)
        return -1;
    if (!seqlens_ok(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded))
        return -1;
    int64_t n = rows ? num_rows : num_rows_padded;

#pragma omp parallel for schedule(dynamic, 8)
    for (int64_t i = 0; i < n; ++i) {
        int64_t row = row_at(rows, i), r;
        int32_t b;
        if (row < 0 || row >= num_rows_padded)
            continue;
        if (!locate_row(cu_seqlens, cu_seqlens_padded, num_seqs, row, &b, &r))
            continue;
        const int64_t gb = vec_offset(b, r, gate_seq_stride, rope_grid, pos_offset, audio_offset);
        for (int32_t c = 0; c < hidden; ++c) {
            double v = ld(&x[row * x_row_stride + c]) + ldm(gate, gb + c, gate_f32) * ld(&y[row * y_row_stride + c]);
            put(out, out_f64, row * out_row_stride + c, v);
        }
    }
    return 0;
}

/* ------------------------------------- gated residual + next adaLN */

/* The residual update of one sublayer and the modulated normalization that
 * opens the next one ("Why Real-Time MiniMax H3 Serving Requires More Than a
 * Faster DiT", "Key takeaways", bullet 2 groups residual updates with
 * modulation and normalization).  Step 1 is the gated residual, rounded to
 * bf16 because that is the value the residual stream stores; step 2 is the
 * adaLN modulation of those stored values. */
int oracle_gated_residual_adaln(
    const uint16_t* x, int64_t x_row_stride,
    const uint16_t* y, int64_t y_row_stride,
    const uint16_t* gate, int64_t gate_seq_stride,
    const uint16_t* shift, const uint16_t* scale, int64_t mod_seq_stride,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, double eps,
    uint16_t* res_out, int64_t res_row_stride,
    uint16_t* norm_out, int64_t norm_row_stride, double* norm_out_f64,
    const int64_t* rows, int64_t num_rows)
{
    return oracle_gated_residual_adaln_ex(x, x_row_stride, y, y_row_stride, gate, gate_seq_stride, shift, scale,
                                          mod_seq_stride, 0, cu_seqlens, cu_seqlens_padded, num_seqs,
                                          num_rows_padded, hidden, eps, res_out, res_row_stride, norm_out,
                                          norm_row_stride, norm_out_f64, rows, num_rows);
}

int oracle_gated_residual_adaln_ex(
    const uint16_t* x, int64_t x_row_stride,
    const uint16_t* y, int64_t y_row_stride,
    const void* gate, int64_t gate_seq_stride,
    const void* shift, const void* scale, int64_t mod_seq_stride, int32_t mod_f32,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, double eps,
    uint16_t* res_out, int64_t res_row_stride,
    uint16_t* norm_out, int64_t norm_row_stride, double* norm_out_f64,
    const int64_t* rows, int64_t num_rows)
{
    return oracle_gated_residual_adaln_av(x, x_row_stride, y, y_row_stride, gate, gate_seq_stride, shift, scale,
                                          mod_seq_stride, mod_f32, NULL, NULL, 0, 0, cu_seqlens, cu_seqlens_padded,
                                          num_seqs, num_rows_padded, hidden, eps, res_out, res_row_stride,
                                          norm_out, norm_row_stride, norm_out_f64, rows, num_rows);
}

int oracle_gated_residual_adaln_av(
    const uint16_t* x, int64_t x_row_stride,
    const uint16_t* y, int64_t y_row_stride,
    const void* gate, int64_t gate_seq_stride,
    const void* shift, const void* scale, int64_t mod_seq_stride, int32_t mod_f32,
    const int32_t* rope_grid, const int32_t* pos_offset, int64_t gate_audio_offset, int64_t mod_audio_offset,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, double eps,
    uint16_t* res_out, int64_t res_row_stride,
    uint16_t* norm_out, int64_t norm_row_stride, double* norm_out_f64,
    const int64_t* rows, int64_t num_rows)
{
    if (!x || !y || !gate || !shift || !scale || !res_out || !norm_out || hidden <= 0)
        return -1;
    if (x_row_stride < hidden || y_row_stride < hidden || res_row_stride < hidden || norm_row_stride < hidden ||
        gate_seq_stride < 0 || mod_seq_stride < 0)
        return -1;
    if (!seqlens_ok(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded))
        return -1;
    int64_t n = rows ? num_rows : num_rows_padded;

#pragma omp parallel for schedule(dynamic, 8)
    for (int64_t i = 0; i < n; ++i) {
        int64_t row = row_at(rows, i), r;
        int32_t b;
        if (row < 0 || row >= num_rows_padded)
            continue;
        if (!locate_row(cu_seqlens, cu_seqlens_padded, num_seqs, row, &b, &r))
            continue;
        const int64_t gb = vec_offset(b, r, gate_seq_stride, rope_grid, pos_offset, gate_audio_offset);
        uint16_t* rr = res_out + row * res_row_stride;
        /* step 1: residual update, stored as bf16 */
        for (int32_t c = 0; c < hidden; ++c) {
            double v = ld(&x[row * x_row_stride + c]) + ldm(gate, gb + c, mod_f32) * ld(&y[row * y_row_stride + c]);
            rr[c] = oracle_f64_to_bf16(v);
        }
        /* step 2: adaLN of the stored residual */
        const int64_t mb = vec_offset(b, r, mod_seq_stride, rope_grid, pos_offset, mod_audio_offset);
        double mean = 0.0;
        for (int32_t c = 0; c < hidden; ++c)
            mean += ld(&rr[c]);
        mean /= (double)hidden;
        double var = 0.0;
        for (int32_t c = 0; c < hidden; ++c)
            var += (ld(&rr[c]) - mean) * (ld(&rr[c]) - mean);
        var /= (double)hidden;
        double inv_std = 1.0 / sqrt(var + eps);
        for (int32_t c = 0; c < hidden; ++c) {
            double xhat = (ld(&rr[c]) - mean) * inv_std;
            double v = xhat * (1.0 + ldm(scale, mb + c, mod_f32)) + ldm(shift, mb + c, mod_f32);
            put(norm_out, norm_out_f64, row * norm_row_stride + c, v);
        }
    }
    return 0;
}

/* ------------------------------------------------------------- SwiGLU */

int oracle_swiglu(
    const uint16_t* a, int64_t a_row_stride,
    const uint16_t* b, int64_t b_row_stride,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t inner,
    uint16_t* out, int64_t out_row_stride, double* out_f64,
    const int64_t* rows, int64_t num_rows)
{
    if (!a || !b || !out || inner <= 0)
        return -1;
    if (a_row_stride < inner || b_row_stride < inner || out_row_stride < inner)
        return -1;
    if (!seqlens_ok(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded))
        return -1;
    int64_t n = rows ? num_rows : num_rows_padded;

#pragma omp parallel for schedule(dynamic, 8)
    for (int64_t i = 0; i < n; ++i) {
        int64_t row = row_at(rows, i), r;
        int32_t s;
        if (row < 0 || row >= num_rows_padded)
            continue;
        if (!locate_row(cu_seqlens, cu_seqlens_padded, num_seqs, row, &s, &r))
            continue;
        for (int32_t c = 0; c < inner; ++c) {
            double av = ld(&a[row * a_row_stride + c]);
            double bv = ld(&b[row * b_row_stride + c]);
            double silu = av / (1.0 + exp(-av));
            put(out, out_f64, row * out_row_stride + c, silu * bv);
        }
    }
    return 0;
}

/* ------------------------------------------------ frames -> uint8 */

/* "Why Real-Time MiniMax H3 Serving Requires More Than a Faster DiT", "Key
 * takeaways", bullet 3: decoded frames are converted on the GPU into compact
 * uint8 BTHWC data once, and the encoder reads planar paths from it.  The page
 * gives no value mapping; the reading taken is the usual one for decoder
 * output in [-1, 1]: scale to [0, 255], clamp, round to nearest even. */
static uint8_t frame_value_to_u8(float x)
{
    float t = x + 1.0f;
    float u = t * 127.5f;
    if (!(u > 0.0f)) /* also NaN */
        return 0;
    if (u >= 255.0f)
        return 255;
    return (uint8_t)nearbyintf(u);
}

int oracle_frames_to_u8(const float* x, int64_t batch, int64_t channels, int64_t frames, int64_t height,
                        int64_t width, int32_t layout, uint8_t* out)
{
    if (!x || !out || batch < 0 || channels < 0 || frames < 0 || height < 0 || width < 0)
        return -1;
    if (layout != 0 && layout != 1)
        return -1;
    int64_t planes = batch * frames;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bt = 0; bt < planes; ++bt) {
        int64_t b = bt / frames, t = bt % frames;
        for (int64_t c = 0; c < channels; ++c)
            for (int64_t h = 0; h < height; ++h)
                for (int64_t w = 0; w < width; ++w) {
                    int64_t src = (((b * channels + c) * frames + t) * height + h) * width + w;
                    int64_t dst = layout == 0
                        ? (((b * frames + t) * height + h) * width + w) * channels + c
                        : (((b * frames + t) * channels + c) * height + h) * width + w;
                    out[dst] = frame_value_to_u8(x[src]);
                }
    }
    return 0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Thread count for the following calls (harness control for timing the
 * oracle on one core; the arithmetic does not depend on it). */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}
