// api.cu -- the C ABI declared in include/dit_token.h: host-side argument
// checks, the rotary frequency bases, and the launches.  Nothing here
// allocates or synchronizes; the only state is thread-local: the last CUDA
// error.
#include <cmath>
#include <cstdint>

#include <cuda_runtime.h>

#include "dit_token.h"
#include "launch.h"

static_assert(DIT_ROPE_INTERLEAVED == dit::kRopeInterleaved && DIT_ROPE_HALF == dit::kRopeHalf &&
                  DIT_ROPE_NONE == dit::kRopeNone,
              "rotary mode codes");

namespace {

thread_local int32_t g_last_cuda_error = 0;

// The rotary frequency bases of p, in fp64: theta^(-2/D) for 1D rows (pair j
// turns at its j-th power, theta^(-2j/D)); on 3D rows pair j lies in the t, h
// or w section of d_s elements (d_s / 2 pairs) and turns at
// theta^(-2j'/d_s), the j'-th power of theta^(-2/d_s), j' its index inside
// the section.  The kernel forms each pair's frequency from these.
void rope_bases(dit::QkParams& p, float rope_theta, int32_t head_dim, int32_t sec_t, int32_t sec_h, int32_t sec_w,
                bool grid)
{
    const double theta = (double)rope_theta;
    const int32_t sec[3] = {sec_t, sec_h, sec_w};
    p.base_1d = std::pow(theta, -2.0 / head_dim);
    for (int s = 0; s < 3; ++s) {
        const bool used = grid && sec[s] > 0;
        p.base_3d[s] = used ? std::pow(theta, -2.0 / sec[s]) : 0.0;
        p.sec_pairs[s] = grid ? sec[s] / 2 : 0;
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool mult8(int64_t v) { return (v & 7) == 0; }

// A per-sequence vector stride keeps every sequence's vector 16-byte aligned:
// a multiple of 8 bf16 or of 4 fp32 elements.
bool mod_stride_ok(int64_t v, bool f32) { return f32 ? (v & 3) == 0 : mult8(v); }

bool known_dtype(int32_t d) { return d == DIT_DTYPE_BF16 || d == DIT_DTYPE_F32; }

dit_status from_cuda(cudaError_t e)
{
    if (e == cudaSuccess)
        return DIT_OK;
    g_last_cuda_error = (int32_t)e;
    return DIT_ERR_CUDA;
}

// Checks shared by every operator: sizes, then the descriptor pointers.
// Returns DIT_OK and sets *nothing_to_do when the batch is empty.
dit_status check_packing(const int32_t* cs, const int32_t* cp, int32_t num_seqs, int64_t num_rows_padded,
                         bool* nothing_to_do)
{
    if (num_seqs < 0 || num_rows_padded < 0 || num_rows_padded > INT32_MAX)
        return DIT_ERR_SHAPE;
    *nothing_to_do = (num_seqs == 0 || num_rows_padded == 0);
    if (*nothing_to_do)
        return DIT_OK;
    if (!cs || !cp)
        return DIT_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(cs) & 3u) || (reinterpret_cast<uintptr_t>(cp) & 3u))
        return DIT_ERR_ALIGN;
    return DIT_OK;
}

dit::Packing packing(const int32_t* cs, const int32_t* cp, int32_t num_seqs, int64_t num_rows_padded)
{
    return dit::Packing{cs, cp, num_seqs, (int32_t)num_rows_padded};
}

}  // namespace

extern "C" {

dit_status dit_qk_rmsnorm_rope(void* q, int64_t q_row_stride, void* k, int64_t k_row_stride,
                               const void* q_weight, const void* k_weight,
                               const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                               int32_t num_seqs, int64_t num_rows_padded,
                               int32_t num_q_heads, int32_t num_k_heads, int32_t head_dim,
                               const int32_t* rope_grid, int32_t sec_t, int32_t sec_h, int32_t sec_w,
                               float rope_theta, float eps, void* stream)
{
    if (head_dim != 64 && head_dim != 128 && head_dim > 0)
        return DIT_ERR_UNSUPPORTED;  // the original entry point keeps its documented range
    return dit_qk_rmsnorm_rope_ex(q, q_row_stride, k, k_row_stride, q_weight, k_weight, cu_seqlens,
                                  cu_seqlens_padded, num_seqs, num_rows_padded, num_q_heads, num_k_heads,
                                  head_dim, rope_grid, sec_t, sec_h, sec_w, rope_theta, eps,
                                  DIT_ROPE_INTERLEAVED, stream);
}

dit_status dit_qk_rmsnorm_rope_ex(void* q, int64_t q_row_stride, void* k, int64_t k_row_stride,
                                  const void* q_weight, const void* k_weight,
                                  const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                                  int32_t num_seqs, int64_t num_rows_padded,
                                  int32_t num_q_heads, int32_t num_k_heads, int32_t head_dim,
                                  const int32_t* rope_grid, int32_t sec_t, int32_t sec_h, int32_t sec_w,
                                  float rope_theta, float eps, int32_t rope_mode, void* stream)
{
    return dit_qk_rmsnorm_rope_shard(q, q_row_stride, k, k_row_stride, q_weight, k_weight, cu_seqlens,
                                     cu_seqlens_padded, num_seqs, num_rows_padded, num_q_heads, num_k_heads,
                                     head_dim, rope_grid, sec_t, sec_h, sec_w, rope_theta, eps, rope_mode, nullptr,
                                     stream);
}

dit_status dit_qk_rmsnorm_rope_shard(void* q, int64_t q_row_stride, void* k, int64_t k_row_stride,
                                     const void* q_weight, const void* k_weight,
                                     const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                                     int32_t num_seqs, int64_t num_rows_padded,
                                     int32_t num_q_heads, int32_t num_k_heads, int32_t head_dim,
                                     const int32_t* rope_grid, int32_t sec_t, int32_t sec_h, int32_t sec_w,
                                     float rope_theta, float eps, int32_t rope_mode, const int32_t* pos_offset,
                                     void* stream)
{
    bool empty = false;
    dit_status st = check_packing(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded, &empty);
    if (st != DIT_OK)
        return st;
    if (num_q_heads < 0 || num_k_heads < 0 || head_dim <= 0)
        return DIT_ERR_SHAPE;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256)
        return DIT_ERR_UNSUPPORTED;
    if (rope_mode != DIT_ROPE_INTERLEAVED && rope_mode != DIT_ROPE_HALF && rope_mode != DIT_ROPE_NONE)
        return DIT_ERR_UNSUPPORTED;
    if (q_row_stride < (int64_t)num_q_heads * head_dim || k_row_stride < (int64_t)num_k_heads * head_dim)
        return DIT_ERR_SHAPE;
    if (!(rope_theta > 0.f) || !(eps >= 0.f) || !std::isfinite(rope_theta) || !std::isfinite(eps))
        return DIT_ERR_SHAPE;
    if (rope_grid && rope_mode != DIT_ROPE_NONE) {
        if (sec_t < 0 || sec_h < 0 || sec_w < 0 || (sec_t | sec_h | sec_w) & 1 ||
            (int64_t)sec_t + sec_h + sec_w != head_dim)
            return DIT_ERR_SHAPE;
    }
    if (empty || num_q_heads + num_k_heads == 0)
        return DIT_OK;
    if (!q || !k || !q_weight || !k_weight)
        return DIT_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(q_weight) || !aligned16(k_weight) ||
        !mult8(q_row_stride) || !mult8(k_row_stride) ||
        (rope_grid && (reinterpret_cast<uintptr_t>(rope_grid) & 3u)) ||
        (pos_offset && (reinterpret_cast<uintptr_t>(pos_offset) & 3u)))
        return DIT_ERR_ALIGN;

    dit::QkParams p{};
    p.q = static_cast<uint16_t*>(q);
    p.k = static_cast<uint16_t*>(k);
    p.q_weight = static_cast<const uint16_t*>(q_weight);
    p.k_weight = static_cast<const uint16_t*>(k_weight);
    p.rope_grid = rope_mode == DIT_ROPE_NONE ? nullptr : rope_grid;
    p.pos_offset = rope_mode == DIT_ROPE_NONE ? nullptr : pos_offset;
    p.q_row_stride = q_row_stride;
    p.k_row_stride = k_row_stride;
    p.pk = packing(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded);
    p.num_q_heads = num_q_heads;
    p.num_k_heads = num_k_heads;
    p.eps = eps;
    rope_bases(p, rope_theta, head_dim, sec_t, sec_h, sec_w, p.rope_grid != nullptr);
    return from_cuda(dit::launch_qk_rmsnorm_rope(p, head_dim, rope_mode, static_cast<cudaStream_t>(stream)));
}

dit_status dit_adaln_modulate(const void* x, int64_t x_row_stride, void* out, int64_t out_row_stride,
                              const void* shift, const void* scale, int64_t mod_seq_stride,
                              const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                              int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, float eps,
                              void* stream)
{
    return dit_adaln_modulate_ex(x, x_row_stride, out, out_row_stride, shift, scale, mod_seq_stride, cu_seqlens,
                                 cu_seqlens_padded, num_seqs, num_rows_padded, hidden, eps, DIT_DTYPE_BF16,
                                 stream);
}

dit_status dit_adaln_modulate_ex(const void* x, int64_t x_row_stride, void* out, int64_t out_row_stride,
                                 const void* shift, const void* scale, int64_t mod_seq_stride,
                                 const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                                 int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, float eps,
                                 int32_t mod_dtype, void* stream)
{
    if (!known_dtype(mod_dtype))
        return DIT_ERR_UNSUPPORTED;
    const bool f32 = mod_dtype == DIT_DTYPE_F32;
    bool empty = false;
    dit_status st = check_packing(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded, &empty);
    if (st != DIT_OK)
        return st;
    if (hidden <= 0 || x_row_stride < hidden || out_row_stride < hidden || mod_seq_stride < 0 ||
        !(eps >= 0.f) || !std::isfinite(eps))
        return DIT_ERR_SHAPE;
    if (hidden > dit::kMaxAdalnHidden)
        return DIT_ERR_UNSUPPORTED;
    if (empty)
        return DIT_OK;
    if (!x || !out || !shift || !scale)
        return DIT_ERR_NULL;
    if (!aligned16(x) || !aligned16(out) || !aligned16(shift) || !aligned16(scale) || !mult8(hidden) ||
        !mult8(x_row_stride) || !mult8(out_row_stride) || !mod_stride_ok(mod_seq_stride, f32))
        return DIT_ERR_ALIGN;
    dit::AdalnParams p{static_cast<const uint16_t*>(x), static_cast<uint16_t*>(out), shift, scale,
                       x_row_stride, out_row_stride, mod_seq_stride,
                       packing(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded), hidden, eps,
                       f32 ? 1 : 0};
    return from_cuda(dit::launch_adaln_modulate(p, static_cast<cudaStream_t>(stream)));
}

dit_status dit_gated_residual(const void* x, int64_t x_row_stride, const void* y, int64_t y_row_stride,
                              const void* gate, int64_t gate_seq_stride, void* out, int64_t out_row_stride,
                              const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                              int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, void* stream)
{
    return dit_gated_residual_ex(x, x_row_stride, y, y_row_stride, gate, gate_seq_stride, out, out_row_stride,
                                 cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded, hidden, DIT_DTYPE_BF16,
                                 stream);
}

dit_status dit_gated_residual_ex(const void* x, int64_t x_row_stride, const void* y, int64_t y_row_stride,
                                 const void* gate, int64_t gate_seq_stride, void* out, int64_t out_row_stride,
                                 const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                                 int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, int32_t gate_dtype,
                                 void* stream)
{
    if (!known_dtype(gate_dtype))
        return DIT_ERR_UNSUPPORTED;
    const bool f32 = gate_dtype == DIT_DTYPE_F32;
    bool empty = false;
    dit_status st = check_packing(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded, &empty);
    if (st != DIT_OK)
        return st;
    if (hidden <= 0 || x_row_stride < hidden || y_row_stride < hidden || out_row_stride < hidden ||
        gate_seq_stride < 0)
        return DIT_ERR_SHAPE;
    if (empty)
        return DIT_OK;
    if (!x || !y || !gate || !out)
        return DIT_ERR_NULL;
    if (!aligned16(x) || !aligned16(y) || !aligned16(gate) || !aligned16(out) || !mult8(hidden) ||
        !mult8(x_row_stride) || !mult8(y_row_stride) || !mult8(out_row_stride) ||
        !mod_stride_ok(gate_seq_stride, f32))
        return DIT_ERR_ALIGN;
    dit::GatedParams p{static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(y), gate,
                       static_cast<uint16_t*>(out), x_row_stride, y_row_stride, gate_seq_stride, out_row_stride,
                       packing(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded), hidden, f32 ? 1 : 0};
    return from_cuda(dit::launch_gated_residual(p, static_cast<cudaStream_t>(stream)));
}

dit_status dit_gated_residual_adaln(const void* x, int64_t x_row_stride, const void* y, int64_t y_row_stride,
                                    const void* gate, int64_t gate_seq_stride,
                                    const void* shift, const void* scale, int64_t mod_seq_stride,
                                    void* res_out, int64_t res_row_stride, void* norm_out, int64_t norm_row_stride,
                                    const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                                    int32_t num_seqs, int64_t num_rows_padded, int32_t hidden, float eps,
                                    void* stream)
{
    return dit_gated_residual_adaln_ex(x, x_row_stride, y, y_row_stride, gate, gate_seq_stride, shift, scale,
                                       mod_seq_stride, res_out, res_row_stride, norm_out, norm_row_stride,
                                       cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded, hidden, eps,
                                       DIT_DTYPE_BF16, stream);
}

dit_status dit_gated_residual_adaln_ex(const void* x, int64_t x_row_stride, const void* y, int64_t y_row_stride,
                                       const void* gate, int64_t gate_seq_stride,
                                       const void* shift, const void* scale, int64_t mod_seq_stride,
                                       void* res_out, int64_t res_row_stride, void* norm_out,
                                       int64_t norm_row_stride, const int32_t* cu_seqlens,
                                       const int32_t* cu_seqlens_padded, int32_t num_seqs,
                                       int64_t num_rows_padded, int32_t hidden, float eps, int32_t mod_dtype,
                                       void* stream)
{
    if (!known_dtype(mod_dtype))
        return DIT_ERR_UNSUPPORTED;
    const bool f32 = mod_dtype == DIT_DTYPE_F32;
    bool empty = false;
    dit_status st = check_packing(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded, &empty);
    if (st != DIT_OK)
        return st;
    if (hidden <= 0 || x_row_stride < hidden || y_row_stride < hidden || res_row_stride < hidden ||
        norm_row_stride < hidden || gate_seq_stride < 0 || mod_seq_stride < 0 || !(eps >= 0.f) ||
        !std::isfinite(eps))
        return DIT_ERR_SHAPE;
    if (hidden > dit::kMaxAdalnHidden)
        return DIT_ERR_UNSUPPORTED;
    if (empty)
        return DIT_OK;
    if (!x || !y || !gate || !shift || !scale || !res_out || !norm_out)
        return DIT_ERR_NULL;
    if (!aligned16(x) || !aligned16(y) || !aligned16(gate) || !aligned16(shift) || !aligned16(scale) ||
        !aligned16(res_out) || !aligned16(norm_out) || !mult8(hidden) || !mult8(x_row_stride) ||
        !mult8(y_row_stride) || !mult8(res_row_stride) || !mult8(norm_row_stride) ||
        !mod_stride_ok(gate_seq_stride, f32) || !mod_stride_ok(mod_seq_stride, f32))
        return DIT_ERR_ALIGN;
    dit::FusedParams p{static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(y), gate, shift, scale,
                       static_cast<uint16_t*>(res_out), static_cast<uint16_t*>(norm_out), x_row_stride,
                       y_row_stride, gate_seq_stride, mod_seq_stride, res_row_stride, norm_row_stride,
                       packing(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded), hidden, eps,
                       f32 ? 1 : 0};
    return from_cuda(dit::launch_gated_residual_adaln(p, static_cast<cudaStream_t>(stream)));
}

dit_status dit_swiglu(const void* a, int64_t a_row_stride, const void* b, int64_t b_row_stride,
                      void* out, int64_t out_row_stride,
                      const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                      int32_t num_seqs, int64_t num_rows_padded, int32_t inner, void* stream)
{
    bool empty = false;
    dit_status st = check_packing(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded, &empty);
    if (st != DIT_OK)
        return st;
    if (inner <= 0 || a_row_stride < inner || b_row_stride < inner || out_row_stride < inner)
        return DIT_ERR_SHAPE;
    if (empty)
        return DIT_OK;
    if (!a || !b || !out)
        return DIT_ERR_NULL;
    if (!aligned16(a) || !aligned16(b) || !aligned16(out) || !mult8(inner) || !mult8(a_row_stride) ||
        !mult8(b_row_stride) || !mult8(out_row_stride))
        return DIT_ERR_ALIGN;
    dit::SwigluParams p{static_cast<const uint16_t*>(a), static_cast<const uint16_t*>(b),
                        static_cast<uint16_t*>(out), a_row_stride, b_row_stride, out_row_stride,
                        packing(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded), inner};
    return from_cuda(dit::launch_swiglu(p, static_cast<cudaStream_t>(stream)));
}

dit_status dit_frames_to_u8(const float* x, int64_t batch, int64_t channels, int64_t frames, int64_t height,
                            int64_t width, int32_t layout, uint8_t* out, void* stream)
{
    if (batch < 0 || channels < 0 || frames < 0 || height < 0 || width < 0)
        return DIT_ERR_SHAPE;
    if (layout != DIT_FRAMES_BTHWC && layout != DIT_FRAMES_BTCHW)
        return DIT_ERR_UNSUPPORTED;
    if (batch == 0 || channels == 0 || frames == 0 || height == 0 || width == 0)
        return DIT_OK;
    const double total = (double)batch * channels * frames * height * width;
    if (total > 9.0e15)
        return DIT_ERR_SHAPE;
    if (!x || !out)
        return DIT_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(x) & 3u)
        return DIT_ERR_ALIGN;
    dit::FramesParams p{x, out, batch, channels, frames, height, width, layout};
    return from_cuda(dit::launch_frames_to_u8(p, static_cast<cudaStream_t>(stream)));
}

dit_status dit_validate_seqlens(const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                                int32_t num_seqs, int64_t num_rows_padded, int32_t* flag, void* stream)
{
    if (num_seqs < 0 || num_rows_padded < 0 || num_rows_padded > INT32_MAX)
        return DIT_ERR_SHAPE;
    if (!cu_seqlens || !cu_seqlens_padded || !flag)
        return DIT_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens_padded) & 3u) ||
        (reinterpret_cast<uintptr_t>(flag) & 3u))
        return DIT_ERR_ALIGN;
    dit::Packing pk = packing(cu_seqlens, cu_seqlens_padded, num_seqs, num_rows_padded);
    return from_cuda(dit::launch_validate_seqlens(pk, num_rows_padded, flag, static_cast<cudaStream_t>(stream)));
}

dit_status dit_av_stream_seqlens(const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                                 const int32_t* rope_grid, const int32_t* pos_offset, int32_t num_seqs,
                                 int32_t* out_cu_seqlens, int32_t* out_cu_seqlens_padded, void* stream)
{
    if (num_seqs < 0 || num_seqs > (INT32_MAX - 1) / 2)
        return DIT_ERR_SHAPE;
    if (!cu_seqlens || !cu_seqlens_padded || !out_cu_seqlens || !out_cu_seqlens_padded ||
        (num_seqs > 0 && !rope_grid))
        return DIT_ERR_NULL;
    const uintptr_t any = reinterpret_cast<uintptr_t>(cu_seqlens) | reinterpret_cast<uintptr_t>(cu_seqlens_padded) |
                          reinterpret_cast<uintptr_t>(rope_grid) | reinterpret_cast<uintptr_t>(pos_offset) |
                          reinterpret_cast<uintptr_t>(out_cu_seqlens) |
                          reinterpret_cast<uintptr_t>(out_cu_seqlens_padded);
    if (any & 3u)
        return DIT_ERR_ALIGN;
    return from_cuda(dit::launch_av_stream_seqlens(cu_seqlens, cu_seqlens_padded, rope_grid, pos_offset, num_seqs,
                                                   out_cu_seqlens, out_cu_seqlens_padded,
                                                   static_cast<cudaStream_t>(stream)));
}

const char* dit_status_string(dit_status s)
{
    switch (s) {
    case DIT_OK: return "DIT_OK";
    case DIT_ERR_NULL: return "DIT_ERR_NULL: a required pointer is NULL";
    case DIT_ERR_SHAPE: return "DIT_ERR_SHAPE: invalid size, stride or rope sections";
    case DIT_ERR_ALIGN: return "DIT_ERR_ALIGN: pointer not 16-byte aligned or size/stride not a multiple of 8";
    case DIT_ERR_UNSUPPORTED: return "DIT_ERR_UNSUPPORTED: unsupported head_dim or hidden size";
    case DIT_ERR_SEQLENS: return "DIT_ERR_SEQLENS: malformed cu_seqlens / cu_seqlens_padded";
    case DIT_ERR_CUDA: return "DIT_ERR_CUDA: kernel launch failed";
    default: return "unknown dit_status";
    }
}

int32_t dit_last_cuda_error(void) { return g_last_cuda_error; }

int32_t dit_abi_version(void) { return DIT_ABI_VERSION; }

}  // extern "C"
