// swiglu.cu -- out = silu(a) * b, silu(a) = a / (1 + exp(-a)), over the valid
// rows of a packed sequence ("Why Real-Time MiniMax H3 Serving Requires More
// Than a Faster DiT", "Key takeaways", bullet 2; "MiniMax H3 通过 vLLM-Omni
// 实现 FastH3 实时推理", "vLLM-Omni 中的系统级优化", bullet 2).
//
// One warp per valid row in CTAs of 4 warps, 4 vectors of a and of b in
// flight per lane (fewer for narrow rows, below), 32 bytes per lane access
// where the rows allow it: 838 us
// on batched varlen (inner 13824, 5.79 GB; 107 % of the measured 6458 GB/s
// copy bandwidth, which reads and writes equally) against 875 us with 16-byte
// accesses and 8-warp CTAs; 57.4 against 63.5 us on one rank's slice of the
// long video (7,736 rows of 8192).  The activation costs one exp2 and one
// reciprocal on the SFU per element (__expf, __fdividef); with 6 bytes of HBM
// traffic per element that stays under the SFU's throughput at B200 clocks.
// For a -> -inf, exp(-a) overflows to +inf and the quotient is a signed zero,
// as in the definition.
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

__device__ __forceinline__ float silu_mul(float a, float b)
{
    return __fdividef(a * b, 1.0f + __expf(-a));
}

// One warp per valid row, WARPS rows per CTA, UNR vectors of NW words
// (2 * NW elements) of a and of b in flight per lane.
template <int NW, int UNR, int WARPS>
__global__ void __launch_bounds__(WARPS * kWarp)
swiglu_kernel(const SwigluParams p)
{
    constexpr int EPV = 2 * NW;
    grid_dependency_wait();
    const int lane = threadIdx.x & (kWarp - 1);
    const int v = blockIdx.x * WARPS + (threadIdx.x >> 5);
    RowSlot s;
    if (!map_valid_row(v, p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs,
                       p.pk.num_rows_padded, lane, s))
        return;
    const uint16_t* ar = p.a + (int64_t)s.row * p.a_row_stride;
    const uint16_t* br = p.b + (int64_t)s.row * p.b_row_stride;
    uint16_t* orow = p.out + (int64_t)s.row * p.out_row_stride;
    const int nvec = p.inner / EPV;

    for (int c0 = 0; c0 < nvec; c0 += kWarp * UNR) {
        uint32_t av[UNR][NW], bv[UNR][NW];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int j = c0 + u * kWarp + lane;
            if (j < nvec) {
                ld_stream_words<NW>(ar + EPV * j, av[u]);
                ld_stream_words<NW>(br + EPV * j, bv[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int j = c0 + u * kWarp + lane;
            if (j < nvec) {
                uint32_t o[NW];
#pragma unroll
                for (int e = 0; e < NW; ++e)
                    o[e] = pack2(silu_mul(bf16_lo(av[u][e]), bf16_lo(bv[u][e])),
                                 silu_mul(bf16_hi(av[u][e]), bf16_hi(bv[u][e])));
                st_stream_words<NW>(orow + EPV * j, o);
            }
        }
    }
}

template <int NW, int UNR, int WARPS>
cudaError_t launch_shape(const SwigluParams& p, cudaStream_t stream)
{
    const unsigned grid = (unsigned)((p.pk.num_rows_padded + WARPS - 1) / WARPS);
    return launch_kernel(swiglu_kernel<NW, UNR, WARPS>, grid, WARPS * kWarp, 0, stream, p);
}

// Vectors in flight per lane: 4 for wide rows (4-warp CTAs), but no more than
// a lane has: a row of one vector per lane (inner 512 with 32-byte accesses:
// VAE-like shapes, 2^20 rows) runs 452.7 us with one in flight and 8-warp
// CTAs, 471.1 with two and 622.7 with four (4-warp CTAs).
template <int NW>
cudaError_t launch_width(const SwigluParams& p, cudaStream_t stream)
{
    const int per_lane = (p.inner / (2 * NW) + kWarp - 1) / kWarp;
    if (per_lane <= 1)
        return launch_shape<NW, 1, 8>(p, stream);
    if (per_lane <= 2)
        return launch_shape<NW, 2, 4>(p, stream);
    return launch_shape<NW, 4, 4>(p, stream);
}

}  // namespace

// 32-byte accesses when a, b and out are 32-byte aligned and inner and the
// row strides are multiples of 16 elements (every row then starts on a
// 32-byte boundary; the halves of a chunked [rows, 2 * inner] projection
// qualify whenever inner is a multiple of 16), else 16-byte ones.
cudaError_t launch_swiglu(const SwigluParams& p, cudaStream_t stream)
{
    const bool wide = aligned32(p.a) && aligned32(p.b) && aligned32(p.out) && p.inner % 16 == 0 &&
                      p.a_row_stride % 16 == 0 && p.b_row_stride % 16 == 0 && p.out_row_stride % 16 == 0;
    return wide ? launch_width<8>(p, stream) : launch_width<4>(p, stream);
}

}  // namespace dit
