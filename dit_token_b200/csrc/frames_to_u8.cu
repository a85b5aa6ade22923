// frames_to_u8.cu -- decoded video frames (fp32, channels first) to uint8,
// converted once on the device before the media encoder ("Why Real-Time
// MiniMax H3 Serving Requires More Than a Faster DiT", "Key takeaways",
// bullet 3: compact uint8 BTHWC data built on the GPU, planar paths for the
// encoder; "MiniMax H3 通过 vLLM-Omni 实现 FastH3 实时推理",
// "vLLM-Omni 中的系统级优化", bullet 4: the FP32 frames are converted to
// contiguous uint8 only once).
//
//   u = rint(clamp((x + 1) * 127.5, 0, 255)), fp32, ties to even, NaN -> 0
//   layout 0: [B][C][T][H][W] fp32 -> [B][T][H][W][C] uint8 (interleaved)
//   layout 1: [B][C][T][H][W] fp32 -> [B][T][C][H][W] uint8 (planes)
//
// One thread converts 16 consecutive pixels of one (b, t, h) row: per channel
// four 16-byte loads (all issued before any conversion), then the bytes are
// interleaved in registers and leave as 16-byte stores (48 bytes per thread
// for RGB).  HBM traffic: 4 bytes in and 1 byte out per value.
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

__device__ __forceinline__ uint32_t to_u8(float x)
{
    const float t = __fadd_rn(x, 1.0f);  // two separately rounded steps, no contraction
    const float u = __fmul_rn(t, 127.5f);
    if (!(u > 0.0f))
        return 0u;  // also NaN
    if (u >= 255.0f)
        return 255u;
    return (uint32_t)__float2int_rn(u);  // round to nearest, ties to even
}

__device__ __forceinline__ float4 ld_stream_f4(const float* p)
{
    return __ldcs(reinterpret_cast<const float4*>(p));
}

// 16 values of one channel -> 16 bytes (4 words, byte k of word i = value 4i + k).
__device__ __forceinline__ void convert16(const float4 (&v)[4], uint32_t (&b)[4])
{
#pragma unroll
    for (int i = 0; i < 4; ++i)
        b[i] = to_u8(v[i].x) | (to_u8(v[i].y) << 8) | (to_u8(v[i].z) << 16) | (to_u8(v[i].w) << 24);
}

__device__ __forceinline__ uint32_t byte_of(const uint32_t (&b)[4], int k)
{
    return (b[k >> 2] >> (8 * (k & 3))) & 0xffu;
}

// Vector path: width % 16 == 0, C in {1, 3, 4}, 16-byte aligned pointers.
template <int C, int LAYOUT>
__global__ void __launch_bounds__(kCtaThreads)
frames_vec_kernel(const float* __restrict__ x, uint8_t* __restrict__ out, int64_t T, int64_t H, int64_t W,
                  int64_t items)
{
    grid_dependency_wait();
    const int64_t groups = W / 16;
    for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items;
         it += (int64_t)gridDim.x * blockDim.x) {
        const int64_t g = it % groups;
        const int64_t row = it / groups;  // (b * T + t) * H + h
        const int64_t h = row % H;
        const int64_t bt = row / H;
        const int64_t t = bt % T;
        const int64_t b = bt / T;
        const int64_t w0 = 16 * g;
        float4 v[C][4];
#pragma unroll
        for (int c = 0; c < C; ++c) {
            const float* src = x + (((b * C + c) * T + t) * H + h) * W + w0;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                v[c][i] = ld_stream_f4(src + 4 * i);
        }
        uint32_t bytes[C][4];
#pragma unroll
        for (int c = 0; c < C; ++c)
            convert16(v[c], bytes[c]);
        if (LAYOUT == 1) {
#pragma unroll
            for (int c = 0; c < C; ++c) {
                uint8_t* dst = out + (((bt * C + c) * H + h) * W + w0);
                __stcs(reinterpret_cast<uint4*>(dst), make_uint4(bytes[c][0], bytes[c][1], bytes[c][2], bytes[c][3]));
            }
        } else {
            // interleave: output byte k = 16 pixels x C channels, k = C * p + c
            uint32_t o[4 * C];
#pragma unroll
            for (int wd = 0; wd < 4 * C; ++wd) {
                uint32_t word = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int byte = 4 * wd + k;
                    word |= byte_of(bytes[byte % C], byte / C) << (8 * k);
                }
                o[wd] = word;
            }
            uint8_t* dst = out + (row * W + w0) * C;
#pragma unroll
            for (int q = 0; q < C; ++q)
                __stcs(reinterpret_cast<uint4*>(dst) + q, make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]));
        }
    }
}

// General path: any channel count and width, one value per thread.
__global__ void __launch_bounds__(kCtaThreads)
frames_scalar_kernel(const float* __restrict__ x, uint8_t* __restrict__ out, int64_t C, int64_t T, int64_t H,
                     int64_t W, int32_t layout, int64_t items)
{
    grid_dependency_wait();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < items;
         i += (int64_t)gridDim.x * blockDim.x) {
        // i enumerates the output in its own order, so stores are coalesced
        int64_t w, h, c, t, b;
        if (layout == 0) {
            c = i % C;
            int64_t r = i / C;
            w = r % W;
            r /= W;
            h = r % H;
            r /= H;
            t = r % T;
            b = r / T;
        } else {
            w = i % W;
            int64_t r = i / W;
            h = r % H;
            r /= H;
            c = r % C;
            r /= C;
            t = r % T;
            b = r / T;
        }
        out[i] = (uint8_t)to_u8(x[(((b * C + c) * T + t) * H + h) * W + w]);
    }
}

unsigned grid_for(int64_t items)
{
    const int64_t blocks = (items + kCtaThreads - 1) / kCtaThreads;
    return (unsigned)(blocks < (1 << 20) ? (blocks > 0 ? blocks : 1) : (1 << 20));
}

}  // namespace

cudaError_t launch_frames_to_u8(const FramesParams& p, cudaStream_t stream)
{
    const bool vec = (p.W % 16 == 0) && (p.C == 1 || p.C == 3 || p.C == 4) &&
                     ((reinterpret_cast<uintptr_t>(p.x) | reinterpret_cast<uintptr_t>(p.out)) & 15u) == 0;
    if (vec) {
        const int64_t items = p.B * p.T * p.H * (p.W / 16);
        const unsigned grid = grid_for(items);
#define DIT_FRAMES_CASE(CC)                                                                                  \
    if (p.C == CC) {                                                                                         \
        if (p.layout == 0)                                                                                   \
            return launch_kernel(frames_vec_kernel<CC, 0>, grid, kCtaThreads, 0, stream, p.x, p.out, p.T, p.H, \
                                 p.W, items);                                                                \
        return launch_kernel(frames_vec_kernel<CC, 1>, grid, kCtaThreads, 0, stream, p.x, p.out, p.T, p.H, p.W, \
                             items);                                                                         \
    }
        DIT_FRAMES_CASE(1)
        DIT_FRAMES_CASE(3)
        DIT_FRAMES_CASE(4)
#undef DIT_FRAMES_CASE
    }
    const int64_t items = p.B * p.C * p.T * p.H * p.W;
    return launch_kernel(frames_scalar_kernel, grid_for(items), kCtaThreads, 0, stream, p.x, p.out, p.C, p.T, p.H,
                         p.W, (int32_t)p.layout, items);
}

}  // namespace dit
