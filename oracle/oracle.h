/*
 * oracle.h -- plain CPU oracle for the fused per-token operators of a packed
 * audio-video diffusion-transformer block.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library,
 * its C ABI or its Python binding) may include, link or call this code; only
 * the tests, the package entry point's smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no source with the CUDA path.
 *
 * Sources.  The operators are named in "Why Real-Time MiniMax H3 Serving
 * Requires More Than a Faster DiT", section "Key takeaways", bullets 1 and 2
 * (packed audio-video sequence with valid lengths, structural suffix padding
 * removed; Q/K RMSNorm with RoPE, modulation and normalization, residual
 * updates and SwiGLU fused), and in "MiniMax H3 通过 vLLM-Omni 实现 FastH3
 * 实时推理", section "vLLM-Omni 中的系统级优化", bullets 1 and 2.  The pages
 * give no formulas; the readings used here (listed in the repository's design
 * notes) are the textbook definitions of each operator.
 *
 * Conventions shared by every function:
 *   - every activation is bf16, passed as its raw 16-bit pattern (uint16_t),
 *     row-major, with a row stride in elements;
 *   - arithmetic is fp64; each output element is rounded once to bf16
 *     (round to nearest, ties to even) and, if an fp64 output buffer is given,
 *     also stored unrounded;
 *   - the packed sequence is described by cu_seqlens[B+1] (cumulative VALID
 *     lengths, cu_seqlens[0] = 0) and cu_seqlens_padded[B+1] (row offset of
 *     each sequence in the padded buffer); row cu_seqlens_padded[b] + r is a
 *     valid row iff r < cu_seqlens[b+1] - cu_seqlens[b];
 *   - outputs are written on valid rows only: padding rows are left untouched;
 *   - rows == NULL means "every padded row"; otherwise only the listed padded
 *     row indices are computed (padding rows in the list are skipped);
 *   - the return value is 0 on success and -1 on an invalid argument.
 */
#ifndef DIT_ORACLE_H
#define DIT_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* bf16 bit pattern -> fp64 (exact). */
double oracle_bf16_to_f64(uint16_t h);

/* fp64 -> bf16 bit pattern, round to nearest, ties to even; overflow -> inf. */
uint16_t oracle_f64_to_bf16(double x);

/* Per-head Q/K RMSNorm fused with rotary position embedding.
 * q: [rows][num_q_heads][head_dim] (row stride q_row_stride), k likewise.
 * q_weight, k_weight: bf16[head_dim], shared by all heads of q (resp. k).
 * rope_grid: NULL (every row 1D, position = index within its sequence) or
 *   int32[num_seqs][3] = (T, H, W): the first T*H*W rows of sequence b take
 *   3D positions (t, h, w); later rows take 1D position r - T*H*W.
 * sec_t, sec_h, sec_w: even section widths (elements) of head_dim used by the
 *   t, h and w axes on 3D rows; they must sum to head_dim when rope_grid is
 *   given.
 * q_out/k_out: same layout and strides as q/k.  *_f64 may be NULL. */
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
    const int64_t* rows, int64_t num_rows);

/* The same with a choice of rotary layout:
 *   ORACLE_ROPE_INTERLEAVED  pairs (2j, 2j+1)            (what oracle_qk_rmsnorm_rope does)
 *   ORACLE_ROPE_HALF         pairs (j, j + head_dim/2)   ("rotate half" layout)
 *   ORACLE_ROPE_NONE         no rotation: per-head RMSNorm times the weight only
 * Pair j has the same angle in both rotary layouts. */
#define ORACLE_ROPE_INTERLEAVED 0
#define ORACLE_ROPE_HALF 1
#define ORACLE_ROPE_NONE 2
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
    const int64_t* rows, int64_t num_rows);

/* oracle_qk_rmsnorm_rope_ex on one rank's slice of longer sequences: the
 * rows of sequence b are the rows pos_offset[b], pos_offset[b] + 1, ... of
 * the whole sequence, and take that sequence's positions (3D inside its grid,
 * 1D after it).  The pages restrict each rank's rotary work to its own rows
 * ("Why Real-Time MiniMax H3 Serving Requires More Than a Faster DiT", "Key
 * takeaways", bullet 1).  pos_offset NULL is the _ex function. */
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
    const int64_t* rows, int64_t num_rows);

/* Adaptive LayerNorm modulation: out = LN(x) * (1 + scale_b) + shift_b.
 * shift/scale: bf16[num_seqs][hidden] with a per-sequence stride of
 * mod_seq_stride elements. */
int oracle_adaln_modulate(
    const uint16_t* x, int64_t x_row_stride,
    const uint16_t* shift, const uint16_t* scale, int64_t mod_seq_stride,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, double eps,
    uint16_t* out, int64_t out_row_stride, double* out_f64,
    const int64_t* rows, int64_t num_rows);

/* Gated residual update: out = x + gate_b * y. */
int oracle_gated_residual(
    const uint16_t* x, int64_t x_row_stride,
    const uint16_t* y, int64_t y_row_stride,
    const uint16_t* gate, int64_t gate_seq_stride,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden,
    uint16_t* out, int64_t out_row_stride, double* out_f64,
    const int64_t* rows, int64_t num_rows);

/* Gated residual update followed by the next sublayer's adaLN, as one op:
 *   res_out  = bf16(x + gate_b * y)                      (the updated residual stream)
 *   norm_out = bf16(LN(res_out) * (1 + scale_b) + shift_b)
 * LN reads the residual as stored (bf16), so the pair equals
 * oracle_gated_residual followed by oracle_adaln_modulate on its output. */
int oracle_gated_residual_adaln(
    const uint16_t* x, int64_t x_row_stride,
    const uint16_t* y, int64_t y_row_stride,
    const uint16_t* gate, int64_t gate_seq_stride,
    const uint16_t* shift, const uint16_t* scale, int64_t mod_seq_stride,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, double eps,
    uint16_t* res_out, int64_t res_row_stride,
    uint16_t* norm_out, int64_t norm_row_stride, double* norm_out_f64,
    const int64_t* rows, int64_t num_rows);

/* The modulated ops with their per-sequence vectors (gate, shift, scale) in
 * either bf16 bits (f32 == 0) or fp32 (f32 != 0); everything else as above. */
int oracle_adaln_modulate_ex(
    const uint16_t* x, int64_t x_row_stride,
    const void* shift, const void* scale, int64_t mod_seq_stride, int32_t mod_f32,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, double eps,
    uint16_t* out, int64_t out_row_stride, double* out_f64,
    const int64_t* rows, int64_t num_rows);
int oracle_gated_residual_ex(
    const uint16_t* x, int64_t x_row_stride,
    const uint16_t* y, int64_t y_row_stride,
    const void* gate, int64_t gate_seq_stride, int32_t gate_f32,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden,
    uint16_t* out, int64_t out_row_stride, double* out_f64,
    const int64_t* rows, int64_t num_rows);
int oracle_gated_residual_adaln_ex(
    const uint16_t* x, int64_t x_row_stride,
    const uint16_t* y, int64_t y_row_stride,
    const void* gate, int64_t gate_seq_stride,
    const void* shift, const void* scale, int64_t mod_seq_stride, int32_t mod_f32,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, double eps,
    uint16_t* res_out, int64_t res_row_stride,
    uint16_t* norm_out, int64_t norm_row_stride, double* norm_out_f64,
    const int64_t* rows, int64_t num_rows);

/* Per-stream modulation of the joint audio-video sequence (the pages pack
 * the audio and video tokens of a request into one sequence, "Why Real-Time
 * MiniMax H3 Serving Requires More Than a Faster DiT", "Key takeaways",
 * bullet 1; they do not say whether the two streams share modulation
 * vectors).  Sequence b holds rope_grid[b] = (T, H, W): its first T*H*W valid
 * rows are video and use the vectors at b * stride; the remaining valid rows
 * are audio and use the vectors audio_offset elements further on.  A row's
 * index in its whole sequence is its local index plus pos_offset[b]
 * (pos_offset NULL: 0), as in oracle_qk_rmsnorm_rope_shard.  With rope_grid
 * NULL every row uses b * stride (the _ex functions). */
int oracle_adaln_modulate_av(
    const uint16_t* x, int64_t x_row_stride,
    const void* shift, const void* scale, int64_t mod_seq_stride, int32_t mod_f32,
    const int32_t* rope_grid, const int32_t* pos_offset, int64_t audio_offset,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, double eps,
    uint16_t* out, int64_t out_row_stride, double* out_f64,
    const int64_t* rows, int64_t num_rows);
int oracle_gated_residual_av(
    const uint16_t* x, int64_t x_row_stride,
    const uint16_t* y, int64_t y_row_stride,
    const void* gate, int64_t gate_seq_stride, int32_t gate_f32,
    const int32_t* rope_grid, const int32_t* pos_offset, int64_t audio_offset,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden,
    uint16_t* out, int64_t out_row_stride, double* out_f64,
    const int64_t* rows, int64_t num_rows);
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
    const int64_t* rows, int64_t num_rows);

/* SwiGLU activation: out = silu(a) * b, silu(a) = a / (1 + exp(-a)). */
int oracle_swiglu(
    const uint16_t* a, int64_t a_row_stride,
    const uint16_t* b, int64_t b_row_stride,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
    int32_t num_seqs, int64_t num_rows_padded, int32_t inner,
    uint16_t* out, int64_t out_row_stride, double* out_f64,
    const int64_t* rows, int64_t num_rows);

/* Decoded video frames -> uint8, converted once on the device before the
 * media encoder.  x: fp32 [batch][channels][frames][height][width]
 * (channels first, contiguous).  Each value becomes
 *   u = rint(clamp((x + 1) * 127.5, 0, 255))
 * in fp32 arithmetic, one IEEE operation at a time (x + 1, then * 127.5),
 * ties to even, NaN -> 0.  The float decides an integer here, so this function
 * computes in fp32 exactly as the device does, not in fp64.
 * layout 0: out [batch][frames][height][width][channels]  (interleaved, "BTHWC")
 * layout 1: out [batch][frames][channels][height][width]  (one plane per channel) */
int oracle_frames_to_u8(const float* x, int64_t batch, int64_t channels, int64_t frames, int64_t height,
                        int64_t width, int32_t layout, uint8_t* out);

/* Number of OpenMP threads the oracle's row loops use (1 without OpenMP). */
int oracle_num_threads(void);
void oracle_set_num_threads(int n);

#ifdef __cplusplus
}
#endif

#endif /* DIT_ORACLE_H */
