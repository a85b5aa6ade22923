// launch.h -- internal interface between the C ABI (api.cu) and the kernel
// translation units.  Arguments reaching these launchers are already
// validated; every launcher only enqueues and returns cudaGetLastError().
#pragma once

#include <cstdint>
#include <utility>

#include <cuda_runtime.h>

namespace dit {

// Programmatic dependent launch.  Every kernel of the library starts with
// grid_dependency_wait() (common.cuh) before its first global-memory access
// -- the packing descriptors included -- and then lets its own dependents
// launch.  So each launch may carry the programmatic-serialization attribute:
// when the previous kernel on the stream lets it, this kernel's CTAs are
// placed and resident while that kernel drains, and start the moment it
// completes (its writes visible), instead of after a full launch gap.  A
// kernel launched after one that does not take part simply starts when that
// one completes, as without the attribute.  DIT_PDL=0 at build time launches
// plainly (for comparison).
#ifndef DIT_PDL
#define DIT_PDL 1
#endif

// A 32-byte boundary (the 256-bit row accesses need one).
inline bool aligned32(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 31u) == 0; }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t stream, Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = DIT_PDL ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

struct Packing {
    const int32_t* cu_seqlens;
    const int32_t* cu_seqlens_padded;
    int32_t num_seqs;
    int32_t num_rows_padded;
};


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
    // Rotary frequency bases, fp64 from the host: pair j of a 1D row turns
    // at base_1d^j = theta^(-2j/D); on a 3D row pair j lies in section s (the
    // first sec_pairs[0] pairs t, the next sec_pairs[1] h, the rest w) and
    // turns at base_3d[s]^j' = theta^(-2j'/d_s), j' its index in the section.
    double base_1d;
    double base_3d[3];
    int32_t sec_pairs[3];
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

// How dit_adaln_modulate lays a row out: 2, 4 or 8 words (8-, 16- or 32-byte
// accesses) per lane vector, a row per warp (team 1) or per CTA of 2, 4 or 8
// warps, and whether the per-sequence vectors are read 32 bytes at a time.
// adaln_shape picks it for a call; launch_adaln_shape runs a given one (every
// shape computes the same result up to the order of the row statistics).
struct AdalnShape {
    int row_words;
    int team;
    bool wide_vectors;
};
AdalnShape adaln_shape(const AdalnParams& p);
cudaError_t launch_adaln_shape(const AdalnParams& p, const AdalnShape& shape, cudaStream_t stream);
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
