/*
 * dit_token.h -- C ABI of the fused per-token operators of a packed
 * audio-video diffusion-transformer (DiT) block, for NVIDIA B200 (sm_100a).
 *
 * The operators are the ones named in "Why Real-Time MiniMax H3 Serving
 * Requires More Than a Faster DiT", section "Key takeaways", bullet 2 (Q/K
 * RMSNorm with RoPE, modulation and normalization, residual updates and
 * SwiGLU, fused to cut repeated small launches) and in "MiniMax H3 通过
 * vLLM-Omni 实现 FastH3 实时推理", section "vLLM-Omni 中的系统级优化",
 * bullet 2.  They run over a packed sequence whose valid lengths come from
 * cu_seqlens, so structural suffix padding is never touched (first page,
 * "Key takeaways", bullet 1; third page, same section, bullet 1).  The pages
 * print no formulas; each entry point states the standard definition it
 * computes.
 *
 * Common conventions
 * ------------------
 * Data type   every activation and weight is bf16 (IEEE binary32 upper
 *             half), row-major; modulation vectors are bf16, or fp32 through
 *             the _ex entry points; decoded frames are fp32.  Arithmetic is
 *             fp32 and every output element is rounded once, to
 *             nearest-even.
 * Pointers    all tensor pointers are DEVICE pointers, owned by the caller;
 *             they must be 16-byte aligned.  Strides are in ELEMENTS and must
 *             be multiples of 8 (16 bytes; fp32 vector strides multiples of
 *             4); so must hidden, inner and head_dim.
 * Packing     cu_seqlens[num_seqs+1] (device, int32): cumulative VALID lengths,
 *             cu_seqlens[0] = 0.  cu_seqlens_padded[num_seqs+1] (device,
 *             int32): first padded row of every sequence, the last entry the
 *             end of the used rows (<= num_rows_padded).  Row
 *             cu_seqlens_padded[b] + r is valid iff
 *             r < cu_seqlens[b+1] - cu_seqlens[b]; every other row (suffix
 *             padding) is neither read nor written.  The device arrays are
 *             trusted but never followed out of bounds: a row index outside
 *             [0, num_rows_padded) or past a sequence's padded slot is
 *             skipped.  dit_validate_seqlens checks them on the device.
 * Aliasing    in-place use is allowed only as exact aliasing (same pointer
 *             and stride): out == x for dit_adaln_modulate and
 *             dit_gated_residual, res_out == x for dit_gated_residual_adaln;
 *             q and k are always updated in place.
 *             Partial overlap is undefined.
 * Stream      `stream` is a cudaStream_t (NULL = the legacy default stream).
 *             Calls only enqueue work: they never synchronize or allocate,
 *             and are safe to call from several host threads.  The only
 *             state is per host thread: the last CUDA error.
 * Launches    every kernel is launched with programmatic stream
 *             serialization and waits for the previous kernel on the stream
 *             to complete before its first memory access, so back-to-back
 *             calls overlap launch latency (not work); this is invisible to
 *             the caller, and a kernel launched after one of these starts
 *             as usual unless it opts in the same way.
 * Errors      argument errors are returned BEFORE anything is launched; a
 *             failed launch returns DIT_ERR_CUDA (dit_last_cuda_error gives
 *             the CUDA error code seen by this thread).  No entry point traps
 *             on the device.
 */
#ifndef DIT_TOKEN_H
#define DIT_TOKEN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t dit_status;
enum {
    DIT_OK = 0,
    DIT_ERR_NULL = 1,        /* a required pointer is NULL */
    DIT_ERR_SHAPE = 2,       /* negative/zero size, stride too small, bad sections */
    DIT_ERR_ALIGN = 3,       /* pointer not 16-byte aligned or size/stride not a multiple of 8 */
    DIT_ERR_UNSUPPORTED = 4, /* e.g. head_dim other than 64 or 128 */
    DIT_ERR_SEQLENS = 5,     /* dit_validate_seqlens found a malformed descriptor */
    DIT_ERR_CUDA = 6         /* the kernel launch failed */
};

#define DIT_ABI_VERSION 1

#if defined(__GNUC__)
#define DIT_API __attribute__((visibility("default")))
#else
#define DIT_API
#endif

/* Per-head Q/K RMSNorm fused with rotary position embedding (RoPE), in place.
 *
 * Pages: first page "Key takeaways" bullet 2 (the Q/K normalization fused
 * with the rotary embedding) and bullet 1 (rotary rows are computed only for
 * the rows a rank needs).  For every valid row and every head h of q (weight
 * q_weight) and of k (weight k_weight):
 *   ms   = (1/D) sum_i x_i^2
 *   y_i  = x_i * rsqrt(ms + eps) * w_i
 *   (o_2j, o_2j+1) = (y_2j c - y_2j+1 s, y_2j s + y_2j+1 c),  c, s = cos, sin(angle_j)
 * with interleaved pairs (2j, 2j+1).  Angles:
 *   rope_grid == NULL: angle_j = p * theta^(-2j/D), p = row index within its sequence;
 *   rope_grid[b] = (T, H, W): rows r < T*H*W of sequence b are video latents at
 *     (t, h, w) = (r / (H W), (r / W) mod H, r mod W); head_dim is split into
 *     sections of sec_t, sec_h, sec_w elements (in that order) and pair j' of
 *     the section of axis s (width d_s) turns by p_s * theta^(-2j'/d_s);
 *     rows r >= T*H*W (audio) use the 1D angle with p = r - T*H*W.
 *
 * q            device bf16 [num_rows_padded][num_q_heads * head_dim], row stride q_row_stride
 *              (>= num_q_heads * head_dim; may be a slice of a fused QKV buffer)
 * k            likewise with num_k_heads (num_k_heads may differ from num_q_heads)
 * q_weight     device bf16 [head_dim], shared by all q heads; k_weight likewise for k
 * rope_grid    device int32 [num_seqs][3] or NULL
 * sec_*        even, >= 0, summing to head_dim when rope_grid != NULL (ignored otherwise)
 * head_dim     64 or 128 (else DIT_ERR_UNSUPPORTED)
 */
DIT_API dit_status dit_qk_rmsnorm_rope(void* q, int64_t q_row_stride, void* k, int64_t k_row_stride,
                               const void* q_weight, const void* k_weight,
                               const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                               int32_t num_seqs, int64_t num_rows_padded,
                               int32_t num_q_heads, int32_t num_k_heads, int32_t head_dim,
                               const int32_t* rope_grid, int32_t sec_t, int32_t sec_h, int32_t sec_w,
                               float rope_theta, float eps, void* stream);

/* dit_qk_rmsnorm_rope with a choice of rotary layout and head_dim 64, 128 or
 * 256.  No counterpart on the pages beyond the operator itself: they do not
 * say how Q/K are laid out, so the layout is a parameter.
 *   DIT_ROPE_INTERLEAVED  pairs (2j, 2j+1)       -- what dit_qk_rmsnorm_rope does
 *   DIT_ROPE_HALF         pairs (j, j + D/2)     ("rotate half" layout); same angles
 *   DIT_ROPE_NONE         per-head RMSNorm times the weight, no rotation (rope_grid
 *                         and sections are ignored) -- the Q/K normalization of
 *                         attention blocks without positional rotation, e.g. the
 *                         VAE's (third page, "vLLM-Omni 中的系统级优化", bullet 3)
 * Every other argument is as for dit_qk_rmsnorm_rope; an unknown mode or a
 * head_dim outside {64, 128, 256} returns DIT_ERR_UNSUPPORTED. */
#define DIT_ROPE_INTERLEAVED 0
#define DIT_ROPE_HALF 1
#define DIT_ROPE_NONE 2
DIT_API dit_status dit_qk_rmsnorm_rope_ex(void* q, int64_t q_row_stride, void* k, int64_t k_row_stride,
                                          const void* q_weight, const void* k_weight,
                                          const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                                          int32_t num_seqs, int64_t num_rows_padded,
                                          int32_t num_q_heads, int32_t num_k_heads, int32_t head_dim,
                                          const int32_t* rope_grid, int32_t sec_t, int32_t sec_h,
                                          int32_t sec_w, float rope_theta, float eps, int32_t rope_mode,
                                          void* stream);

/* dit_qk_rmsnorm_rope_ex on one rank's slice of longer sequences.
 *
 * Pages: first page "Key takeaways" bullet 1 (each rank's rotary work is
 * restricted to its own rows of the packed sequence).  The rows of sequence b
 * in this buffer are rows pos_offset[b], pos_offset[b] + 1, ... of the whole
 * sequence b, and take that sequence's positions: with rope_grid[b] =
 * (T, H, W), whole-sequence rows below T*H*W are 3D, the rest 1D counted from
 * the end of the grid.  pos_offset: device int32 [num_seqs] (>= 0), or NULL
 * (every offset 0: the _ex call).  Ignored when rope_mode is DIT_ROPE_NONE.
 * The offsets are trusted like cu_seqlens: a negative entry, outside the
 * documented range, is read as 0 (no fault and no flag). */
DIT_API dit_status dit_qk_rmsnorm_rope_shard(void* q, int64_t q_row_stride, void* k, int64_t k_row_stride,
                                             const void* q_weight, const void* k_weight,
                                             const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                                             int32_t num_seqs, int64_t num_rows_padded, int32_t num_q_heads,
                                             int32_t num_k_heads, int32_t head_dim, const int32_t* rope_grid,
                                             int32_t sec_t, int32_t sec_h, int32_t sec_w, float rope_theta,
                                             float eps, int32_t rope_mode, const int32_t* pos_offset,
                                             void* stream);

/* Adaptive LayerNorm modulation: out = LN(x) * (1 + scale_b) + shift_b.
 *
 * Pages: first page "Key takeaways" bullet 2 (the modulation and the
 * normalization are fused).  LN has no affine: mean and biased variance over the hidden axis,
 * x_hat = (x - mean) * rsqrt(var + eps).  shift/scale are per sequence b.
 *
 * x, out       device bf16 [num_rows_padded][hidden], row strides >= hidden (out may be x)
 * shift, scale device bf16, vector of sequence b at shift + b * mod_seq_stride
 *              (mod_seq_stride >= 0, a multiple of 8; e.g. 6*hidden for a [B][6][hidden]
 *              modulation tensor)
 */
DIT_API dit_status dit_adaln_modulate(const void* x, int64_t x_row_stride, void* out, int64_t out_row_stride,
                              const void* shift, const void* scale, int64_t mod_seq_stride,
                              const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                              int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, float eps,
                              void* stream);

/* Gated residual update: out = x + gate_b * y (one fp32 fused multiply-add,
 * one rounding).
 *
 * Pages: first page "Key takeaways" bullet 2 (the residual update is fused).
 * x, y, out    device bf16 [num_rows_padded][hidden] with their own row strides (out may be x)
 * gate         device bf16, vector of sequence b at gate + b * gate_seq_stride
 */
DIT_API dit_status dit_gated_residual(const void* x, int64_t x_row_stride, const void* y, int64_t y_row_stride,
                              const void* gate, int64_t gate_seq_stride, void* out, int64_t out_row_stride,
                              const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                              int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, void* stream);

/* Gated residual update fused with the next sublayer's adaLN modulation:
 *   res_out  = bf16(x + gate_b * y)
 *   norm_out = bf16(LN(res_out) * (1 + scale_b) + shift_b)
 * LN (no affine, biased variance) reads the residual as stored in bf16, so the
 * pair equals dit_gated_residual followed by dit_adaln_modulate on its output,
 * while x and y are read once and res_out and norm_out written once.
 *
 * Pages: first page "Key takeaways" bullet 2 (residual updates fused together
 * with the modulation and normalization work).
 * x, y         device bf16 [num_rows_padded][hidden] with their own row strides
 * gate         device bf16, vector of sequence b at gate + b * gate_seq_stride
 * shift, scale device bf16, vectors of sequence b at + b * mod_seq_stride
 * res_out      device bf16 [num_rows_padded][hidden] (may be x)
 * norm_out     device bf16 [num_rows_padded][hidden] (must not overlap the others)
 * hidden       a multiple of 8, at most 16384
 */
DIT_API dit_status dit_gated_residual_adaln(const void* x, int64_t x_row_stride, const void* y,
                                            int64_t y_row_stride, const void* gate, int64_t gate_seq_stride,
                                            const void* shift, const void* scale, int64_t mod_seq_stride,
                                            void* res_out, int64_t res_row_stride, void* norm_out,
                                            int64_t norm_row_stride, const int32_t* cu_seqlens,
                                            const int32_t* cu_seqlens_padded, int32_t num_seqs,
                                            int64_t num_rows_padded, int32_t hidden, float eps, void* stream);

/* Element types of the per-sequence modulation vectors (gate, shift, scale)
 * accepted by the _ex entry points below.  The pages fix no precision for
 * them; a modulation head may emit them in bf16 or keep them in fp32.  The
 * activations stay bf16 either way, and every op computes in fp32, so an fp32
 * vector only removes the rounding of the vector itself. */
#define DIT_DTYPE_BF16 0
#define DIT_DTYPE_F32 1

/* dit_adaln_modulate with shift and scale of element type mod_dtype
 * (DIT_DTYPE_BF16 or DIT_DTYPE_F32).  For fp32 vectors mod_seq_stride must be a
 * multiple of 4 (16-byte aligned vectors); for bf16 a multiple of 8.  An
 * unknown mod_dtype returns DIT_ERR_UNSUPPORTED. */
DIT_API dit_status dit_adaln_modulate_ex(const void* x, int64_t x_row_stride, void* out, int64_t out_row_stride,
                                         const void* shift, const void* scale, int64_t mod_seq_stride,
                                         const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                                         int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, float eps,
                                         int32_t mod_dtype, void* stream);

/* dit_gated_residual with a gate of element type gate_dtype (same codes and
 * stride rule as above). */
DIT_API dit_status dit_gated_residual_ex(const void* x, int64_t x_row_stride, const void* y, int64_t y_row_stride,
                                         const void* gate, int64_t gate_seq_stride, void* out,
                                         int64_t out_row_stride, const int32_t* cu_seqlens,
                                         const int32_t* cu_seqlens_padded, int32_t num_seqs,
                                         int64_t num_rows_padded, int32_t hidden, int32_t gate_dtype, void* stream);

/* dit_gated_residual_adaln with gate, shift and scale all of element type
 * mod_dtype (same codes; gate_seq_stride and mod_seq_stride follow the stride
 * rule above). */
DIT_API dit_status dit_gated_residual_adaln_ex(const void* x, int64_t x_row_stride, const void* y,
                                               int64_t y_row_stride, const void* gate, int64_t gate_seq_stride,
                                               const void* shift, const void* scale, int64_t mod_seq_stride,
                                               void* res_out, int64_t res_row_stride, void* norm_out,
                                               int64_t norm_row_stride, const int32_t* cu_seqlens,
                                               const int32_t* cu_seqlens_padded, int32_t num_seqs,
                                               int64_t num_rows_padded, int32_t hidden, float eps,
                                               int32_t mod_dtype, void* stream);

/* SwiGLU activation: out = silu(a) * b, silu(a) = a / (1 + exp(-a)).
 *
 * Pages: first page "Key takeaways" bullet 2 and third page "vLLM-Omni 中的
 * 系统级优化" bullet 2 (the SwiGLU activation is fused).
 * a, b         device bf16 [num_rows_padded][inner] with their own row strides; for a
 *              chunked [rows][2*inner] projection pass a = base, b = base + inner and
 *              both row strides 2*inner
 * out          device bf16 [num_rows_padded][inner], row stride out_row_stride
 */
DIT_API dit_status dit_swiglu(const void* a, int64_t a_row_stride, const void* b, int64_t b_row_stride,
                      void* out, int64_t out_row_stride,
                      const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                      int32_t num_seqs, int64_t num_rows_padded, int32_t inner, void* stream);

/* Decoded video frames (fp32) -> uint8, converted once on the device before
 * the media encoder.
 *
 * Pages: first page "Key takeaways" bullet 3 (frames are converted on the GPU
 * to compact uint8 BTHWC data, and the encoder reads planar paths); third
 * page "vLLM-Omni 中的系统级优化" bullet 4 (the FP32 frames are converted to
 * contiguous uint8 only once).  The pages give no value mapping; each value
 * becomes u = rint(clamp((x + 1) * 127.5, 0, 255)) computed in fp32 (x + 1
 * rounded, then * 127.5 rounded), ties to even, NaN -> 0.
 *
 * x       device fp32 [batch][channels][frames][height][width], contiguous, 4-byte aligned
 * layout  DIT_FRAMES_BTHWC: out [batch][frames][height][width][channels] (interleaved)
 *         DIT_FRAMES_BTCHW: out [batch][frames][channels][height][width] (planes)
 * out     device uint8, batch*channels*frames*height*width bytes, contiguous
 * Fast path when width % 16 == 0, channels is 1, 3 or 4 and both pointers are
 * 16-byte aligned; any other shape takes a per-value path with the same result.
 */
#define DIT_FRAMES_BTHWC 0
#define DIT_FRAMES_BTCHW 1
DIT_API dit_status dit_frames_to_u8(const float* x, int64_t batch, int64_t channels, int64_t frames,
                                    int64_t height, int64_t width, int32_t layout, uint8_t* out, void* stream);

/* Device-side check of a packing descriptor; no counterpart on the pages (it
 * guards the padding-free packing of the first page, "Key takeaways" bullet 1).
 * Writes flag[0] = 0 if cu_seqlens[0] == 0, cu_seqlens_padded[0] == 0, both
 * are non-decreasing, every valid length fits its padded slot and
 * cu_seqlens_padded[num_seqs] <= num_rows_padded; otherwise flag[0] = 1 and
 * flag[1] = the first offending sequence index (0 also when a leading entry
 * is not 0, even for num_seqs == 0).  flag: device int32[2].  The
 * kernel never traps; the host reads the flag when it chooses to (e.g. with
 * cudaMemcpy after the stream) and maps 1 to DIT_ERR_SEQLENS. */
DIT_API dit_status dit_validate_seqlens(const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                                int32_t num_seqs, int64_t num_rows_padded, int32_t* flag, void* stream);

/* Per-stream packing descriptor of joint audio-video sequences.
 *
 * Pages: first page "Key takeaways" bullet 1 (a request's audio and video
 * tokens are packed into one sequence); whether the two streams share
 * modulation vectors is left open, and this call lets them differ.
 * Sequence b of (cu_seqlens, cu_seqlens_padded) holds v_b = clamp(T*H*W, 0,
 * min(L_b, padded_b)) video rows (rope_grid[b] = (T, H, W)) and then its audio
 * rows and suffix padding.  The output describes 2*num_seqs sequences:
 *   2b     the video rows of b:       valid v_b, padded v_b
 *   2b + 1 the audio rows of b:       valid L_b - v_b, padded padded_b - v_b
 * over the same buffer rows.  Passing it to dit_adaln_modulate(_ex),
 * dit_gated_residual(_ex) or dit_gated_residual_adaln(_ex) with vectors laid out
 * [num_seqs][2 streams][...] (sequence stride of the output = the stride
 * between the two streams' sets) applies the video set to video rows and the
 * audio set to audio rows.  RoPE keeps the original descriptor (positions are
 * per request).
 *
 * For one rank's slice of longer sequences (pos_offset[b] = the whole-sequence
 * index of b's first row, as in dit_qk_rmsnorm_rope_shard) v_b counts the grid
 * rows past that start: clamp(T*H*W - pos_offset[b], 0, min(L_b, padded_b)).
 *
 * cu_seqlens, cu_seqlens_padded  device int32 [num_seqs + 1]
 * rope_grid                      device int32 [num_seqs][3] (may be NULL only if num_seqs == 0)
 * pos_offset                     device int32 [num_seqs], or NULL (all 0)
 * out_cu_seqlens, out_cu_seqlens_padded  device int32 [2 * num_seqs + 1], written
 * One small kernel on `stream`; no synchronization.  Entries 0 are copied. */
DIT_API dit_status dit_av_stream_seqlens(const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                                         const int32_t* rope_grid, const int32_t* pos_offset, int32_t num_seqs,
                                         int32_t* out_cu_seqlens, int32_t* out_cu_seqlens_padded, void* stream);

/* Human-readable name of a status code (static storage; never NULL). */
DIT_API const char* dit_status_string(dit_status s);

/* The CUDA error code (cudaError_t value) behind the last DIT_ERR_CUDA
 * returned on the calling thread, 0 if none. */
DIT_API int32_t dit_last_cuda_error(void);

/* DIT_ABI_VERSION of the library. */
DIT_API int32_t dit_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DIT_TOKEN_H */
