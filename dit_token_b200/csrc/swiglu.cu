// swiglu.cu -- out = silu(a) * b, silu(a) = a / (1 + exp(-a)), over the valid
// rows of a packed sequence ("Why Real-Time MiniMax H3 Serving Requires More
// Than a Faster DiT", "Key takeaways", bullet 2; "MiniMax H3 通过 vLLM-Omni
// 实现 FastH3 实时推理", "vLLM-Omni 中的系统级优化", bullet 2).
//
// One warp per valid row in CTAs of 4 warps, 4 vectors of a and of b in
// flight per lane, 32 bytes per lane access where the rows allow it: 838 us
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

constexpr int kSwigluWarps = 4;  // rows (warps) per CTA

__device__ __forceinline__ float silu_mul(float a, float b)
{
    return __fdividef(a * b, 1.0f + __expf(-a));
}

// One warp per valid row, UNR vectors of NW words (2 * NW elements) of a and
// of b in flight per lane.
template <int NW, int UNR>
__global__ void __launch_bounds__(kSwigluWarps * kWarp)
swiglu_kernel(const SwigluParams p)
{
    constexpr int EPV = 2 * NW;
    grid_dependency_wait();
    const int lane = threadIdx.x & (kWarp - 1);
    const int v = blockIdx.x * kSwigluWarps + (threadIdx.x >> 5);
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

}  // namespace

// 32-byte accesses when a, b and out are 32-byte aligned and inner and the
// row strides are multiples of 16 elements (every row then starts on a
// 32-byte boundary; the halves of a chunked [rows, 2 * inner] projection
// qualify whenever inner is a multiple of 16), else 16-byte ones.
cudaError_t launch_swiglu(const SwigluParams& p, cudaStream_t stream)
{
    const unsigned grid = (unsigned)((p.pk.num_rows_padded + kSwigluWarps - 1) / kSwigluWarps);
    const bool wide = aligned32(p.a) && aligned32(p.b) && aligned32(p.out) && p.inner % 16 == 0 &&
                      p.a_row_stride % 16 == 0 && p.b_row_stride % 16 == 0 && p.out_row_stride % 16 == 0;
    return wide ? launch_kernel(swiglu_kernel<8, 4>, grid, kSwigluWarps * kWarp, 0, stream, p)
                : launch_kernel(swiglu_kernel<4, 4>, grid, kSwigluWarps * kWarp, 0, stream, p);
}

}  // namespace dit
