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
// two 32-byte loads (16-byte ones when the frames are not 32-byte aligned),
// all issued before any conversion, then the bytes are interleaved in
// registers and leave as 16-byte stores (48 bytes per thread for RGB).  HBM
// traffic: 4 bytes in and 1 byte out per value.  Per value: the two rounded
// steps on fp32 pairs, a clamp, and one add of 1.5 * 2^23, which rounds to
// the nearest integer (ties to even: the sum's spacing is 1) and leaves that
// integer in the low byte of the sum's bits; byte permutes pack four values
// into a word.  Indices are 32-bit where they fit (two divisions a thread).
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

// u -> rint(clamp(u, 0, 255)), ties to even, NaN -> 0, in the low byte of
// the result: fmaxf returns the non-NaN operand, and adding 1.5 * 2^23 (where
// the float spacing is 1) rounds to the nearest integer, ties to even.
__device__ __forceinline__ uint32_t u8_bits(float u)
{
    return __float_as_uint(__fadd_rn(fminf(fmaxf(u, 0.0f), 255.0f), 12582912.0f));
}

__device__ __forceinline__ uint32_t to_u8(float x)
{
    // two separately rounded steps, no contraction
    return u8_bits(__fmul_rn(__fadd_rn(x, 1.0f), 127.5f)) & 0xffu;
}

// The low bytes of a, b, c, d as one word (a in byte 0).
__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// 16 consecutive fp32 values of a streamed frame row, evict-first: two
// 32-byte loads (W32, 32-byte aligned address) or four 16-byte ones.
// volatile: the loads keep their program order, so all of a thread's loads
// are in flight before its first conversion.
template <bool W32>
__device__ __forceinline__ void ld_frames16(const float* p, float4 (&v)[4])
{
    if constexpr (W32) {
#pragma unroll
        for (int i = 0; i < 4; i += 2) {
            uint32_t w[8];
            asm volatile("ld.global.cs.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                         : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]),
                           "=r"(w[7])
                         : "l"(p + 4 * i));
            v[i] = make_float4(__uint_as_float(w[0]), __uint_as_float(w[1]), __uint_as_float(w[2]),
                               __uint_as_float(w[3]));
            v[i + 1] = make_float4(__uint_as_float(w[4]), __uint_as_float(w[5]), __uint_as_float(w[6]),
                                   __uint_as_float(w[7]));
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            v[i] = __ldcs(reinterpret_cast<const float4*>(p + 4 * i));
    }
}

// 16 values of one channel -> their bytes in the low bytes of u[0..15].
__device__ __forceinline__ void convert16(const float4 (&v)[4], uint32_t (&u)[16])
{
    const float2 one2 = make_float2(1.0f, 1.0f), s2 = make_float2(127.5f, 127.5f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = __fmul2_rn(__fadd2_rn(make_float2(v[i].x, v[i].y), one2), s2);
        const float2 b = __fmul2_rn(__fadd2_rn(make_float2(v[i].z, v[i].w), one2), s2);
        u[4 * i] = u8_bits(a.x);
        u[4 * i + 1] = u8_bits(a.y);
        u[4 * i + 2] = u8_bits(b.x);
        u[4 * i + 3] = u8_bits(b.y);
    }
}

// Vector path: width % 16 == 0, C in {1, 3, 4}, 16-byte aligned pointers.
// I: the index type (32-bit when every index fits); W32: 32-byte loads.
template <int C, int LAYOUT, typename I, bool W32>
__global__ void __launch_bounds__(kCtaThreads)
frames_vec_kernel(const float* __restrict__ x, uint8_t* __restrict__ out, int64_t T, int64_t H, int64_t W,
                  int64_t items)
{
    grid_dependency_wait();
    const I groups = (I)(W / 16);
    const I TH = (I)(T * H);
    const int64_t plane = T * H * W;  // one channel of one batch entry
    for (I it = (I)blockIdx.x * (I)blockDim.x + (I)threadIdx.x; it < (I)items; it += (I)gridDim.x * (I)blockDim.x) {
        const I row = it / groups;  // (b * T + t) * H + h
        const I w0 = 16 * (it - row * groups);
        const I b = row / TH;
        const I th = row - b * TH;  // t * H + h
        const float* src = x + (int64_t)b * C * plane + (int64_t)th * W + w0;
        float4 v[C][4];
#pragma unroll
        for (int c = 0; c < C; ++c)
            ld_frames16<W32>(src + c * plane, v[c]);
        uint32_t u[C][16];
#pragma unroll
        for (int c = 0; c < C; ++c)
            convert16(v[c], u[c]);
        if (LAYOUT == 1) {
            const I bt = row / (I)H;
            const I h = row - bt * (I)H;
#pragma unroll
            for (int c = 0; c < C; ++c) {
                uint8_t* dst = out + (((int64_t)bt * C + c) * H + h) * W + w0;
                __stcs(reinterpret_cast<uint4*>(dst),
                       make_uint4(pack4(u[c][0], u[c][1], u[c][2], u[c][3]), pack4(u[c][4], u[c][5], u[c][6], u[c][7]),
                                  pack4(u[c][8], u[c][9], u[c][10], u[c][11]),
                                  pack4(u[c][12], u[c][13], u[c][14], u[c][15])));
            }
        } else {
            // interleave: output byte k of the 16 pixels x C channels is
            // channel k % C of pixel k / C
            uint32_t o[4 * C];
#pragma unroll
            for (int wd = 0; wd < 4 * C; ++wd) {
                const int k = 4 * wd;
                o[wd] = pack4(u[k % C][k / C], u[(k + 1) % C][(k + 1) / C], u[(k + 2) % C][(k + 2) / C],
                              u[(k + 3) % C][(k + 3) / C]);
            }
            uint8_t* dst = out + ((int64_t)row * W + w0) * C;
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

template <int C, int LAYOUT, typename I>
cudaError_t launch_vec(const FramesParams& p, unsigned grid, int64_t items, cudaStream_t stream)
{
    // W % 16 == 0 puts every row and channel plane 64 bytes apart, so the
    // frames' base address alone decides whether 32-byte loads are aligned
    if (aligned32(p.x))
        return launch_kernel(frames_vec_kernel<C, LAYOUT, I, true>, grid, kCtaThreads, 0, stream, p.x, p.out, p.T,
                             p.H, p.W, items);
    return launch_kernel(frames_vec_kernel<C, LAYOUT, I, false>, grid, kCtaThreads, 0, stream, p.x, p.out, p.T, p.H,
                         p.W, items);
}

template <int C, int LAYOUT>
cudaError_t launch_vec_index(const FramesParams& p, unsigned grid, int64_t items, cudaStream_t stream)
{
    // 32-bit indices when the items (plus one grid stride) and the rows fit
    const bool i32 = items + (int64_t)grid * kCtaThreads < (int64_t)INT32_MAX && p.B * p.T * p.H < INT32_MAX;
    return i32 ? launch_vec<C, LAYOUT, int32_t>(p, grid, items, stream)
               : launch_vec<C, LAYOUT, int64_t>(p, grid, items, stream);
}

template <int C>
cudaError_t launch_vec_layout(const FramesParams& p, unsigned grid, int64_t items, cudaStream_t stream)
{
    return p.layout == 0 ? launch_vec_index<C, 0>(p, grid, items, stream)
                         : launch_vec_index<C, 1>(p, grid, items, stream);
}

}  // namespace

cudaError_t launch_frames_to_u8(const FramesParams& p, cudaStream_t stream)
{
    const bool vec = (p.W % 16 == 0) && (p.C == 1 || p.C == 3 || p.C == 4) &&
                     ((reinterpret_cast<uintptr_t>(p.x) | reinterpret_cast<uintptr_t>(p.out)) & 15u) == 0;
    if (vec) {
        const int64_t items = p.B * p.T * p.H * (p.W / 16);
        const unsigned grid = grid_for(items);
        switch (p.C) {
        case 1: return launch_vec_layout<1>(p, grid, items, stream);
        case 3: return launch_vec_layout<3>(p, grid, items, stream);
        default: return launch_vec_layout<4>(p, grid, items, stream);
        }
    }
    const int64_t items = p.B * p.C * p.T * p.H * p.W;
    return launch_kernel(frames_scalar_kernel, grid_for(items), kCtaThreads, 0, stream, p.x, p.out, p.C, p.T, p.H,
                         p.W, (int32_t)p.layout, items);
}

}  // namespace dit
