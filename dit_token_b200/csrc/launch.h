// launch.h -- internal interface between the C ABI (api.cu) and the kernel
// translation units.  Arguments reaching these launchers are already
// validated; every launcher only enqueues and returns cudaGetLastError().
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace dit {

struct Packing {
    const int32_t* cu_seqlens;
    const int32_t* cu_seqlens_padded;
    int32_t num_seqs;
    int32_t num_rows_padded;
};

constexpr int kMaxPairs = 128;  // head_dim <= 256

// Rotary layouts of dit_qk_rmsnorm_rope_ex (the DIT_ROPE_* values of the ABI).
constexpr int kRopeInterleaved = 0;
constexpr int kRopeHalf = 1;
constexpr int kRopeNone = 2;

struct QkParams {
    uint16_t* q;
    uint16_t* k;
    const uint16_t* q_weight;
    const uint16_t* k_weight;
    const int32_t* rope_grid;
    const int32_t* pos_offset;  // [num_seqs] start of each sequence's rows in the whole sequence, or null
    int64_t q_row_stride;
    int64_t k_row_stride;
    Packing pk;
    int32_t num_q_heads;
    int32_t num_k_heads;
    float eps;
    // Per-pair rotary frequencies, computed once on the host in fp64:
    // inv_freq_1d[j] = theta^(-2j/D); inv_freq_3d[j] = theta^(-2j'/d_s) for the
    // section s = axis[j] that pair j falls in, j' its index in that section.
    double inv_freq_1d[kMaxPairs];
    double inv_freq_3d[kMaxPairs];
    int8_t axis[kMaxPairs];
};

struct AdalnParams {
    const uint16_t* x;
    uint16_t* out;
    const void* shift;  // bf16 or fp32 (mod_f32)
    const void* scale;
    int64_t x_row_stride;
    int64_t out_row_stride;
    int64_t mod_seq_stride;
    Packing pk;
    int32_t hidden;
    float eps;
    int32_t mod_f32;
};

struct GatedParams {
    const uint16_t* x;
    const uint16_t* y;
    const void* gate;  // bf16 or fp32 (gate_f32)
    uint16_t* out;
    int64_t x_row_stride;
    int64_t y_row_stride;
    int64_t gate_seq_stride;
    int64_t out_row_stride;
    Packing pk;
    int32_t hidden;
    int32_t gate_f32;
};

struct FusedParams {
    const uint16_t* x;
    const uint16_t* y;
    const void* gate;  // gate, shift, scale: bf16 or fp32 (mod_f32)
    const void* shift;
    const void* scale;
    uint16_t* res_out;
    uint16_t* norm_out;
    int64_t x_row_stride;
    int64_t y_row_stride;
    int64_t gate_seq_stride;
    int64_t mod_seq_stride;
    int64_t res_row_stride;
    int64_t norm_row_stride;
    Packing pk;
    int32_t hidden;
    float eps;
    int32_t mod_f32;
};

struct SwigluParams {
    const uint16_t* a;
    const uint16_t* b;
    uint16_t* out;
    int64_t a_row_stride;
    int64_t b_row_stride;
    int64_t out_row_stride;
    Packing pk;
    int32_t inner;
};

struct FramesParams {
    const float* x;
    uint8_t* out;
    int64_t B, C, T, H, W;
    int32_t layout;
};

cudaError_t launch_frames_to_u8(const FramesParams& p, cudaStream_t stream);
cudaError_t launch_qk_rmsnorm_rope(const QkParams& p, int head_dim, int rope_mode, cudaStream_t stream);
cudaError_t launch_adaln_modulate(const AdalnParams& p, cudaStream_t stream);
cudaError_t launch_gated_residual(const GatedParams& p, cudaStream_t stream);
cudaError_t launch_swiglu(const SwigluParams& p, cudaStream_t stream);
cudaError_t launch_gated_residual_adaln(const FusedParams& p, cudaStream_t stream);
cudaError_t launch_av_stream_seqlens(const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                                     const int32_t* rope_grid, const int32_t* pos_offset, int32_t num_seqs,
                                     int32_t* out_cu_seqlens, int32_t* out_cu_seqlens_padded, cudaStream_t stream);
cudaError_t launch_validate_seqlens(const Packing& pk, int64_t num_rows_padded, int32_t* flag,
                                    cudaStream_t stream);

// Largest hidden size dit_adaln_modulate supports (8 warps x 8 vectors x 32 lanes x 8).
constexpr int kMaxAdalnHidden = 16384;

}  // namespace dit
