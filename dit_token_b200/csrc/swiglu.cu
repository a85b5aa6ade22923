// swiglu.cu -- out = silu(a) * b, silu(a) = a / (1 + exp(-a)), over the valid
// rows of a packed sequence ("Why Real-Time MiniMax H3 Serving Requires More
// Than a Faster DiT", "Key takeaways", bullet 2; "MiniMax H3 通过 vLLM-Omni
// 实现 FastH3 实时推理", "vLLM-Omni 中的系统级优化", bullet 2).
//
// One warp per valid row, U 16-byte vectors of a and of b in flight per lane.
// The activation costs one exp2 and one reciprocal on the SFU per element
// (__expf, __fdividef); with 6 bytes of HBM traffic per element that stays
// under the SFU's throughput at B200 clocks.  For a -> -inf, exp(-a)
// overflows to +inf and the quotient is a signed zero, as in the definition.
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

#ifndef DIT_EW_UNROLL
#define DIT_EW_UNROLL 4
#endif
constexpr int kUnroll = DIT_EW_UNROLL;  // 16-byte vectors per lane and input in flight

__device__ __forceinline__ float silu_mul(float a, float b)
{
    return __fdividef(a * b, 1.0f + __expf(-a));
}

__global__ void __launch_bounds__(kCtaThreads)
swiglu_kernel(const SwigluParams p)
{
    const int lane = threadIdx.x & (kWarp - 1);
    const int v = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    RowSlot s;
    if (!map_valid_row(v, p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs,
                       p.pk.num_rows_padded, lane, s))
        return;
    const uint16_t* ar = p.a + (int64_t)s.row * p.a_row_stride;
    const uint16_t* br = p.b + (int64_t)s.row * p.b_row_stride;
    uint16_t* orow = p.out + (int64_t)s.row * p.out_row_stride;
    const int nvec = p.inner / 8;

    for (int c0 = 0; c0 < nvec; c0 += kWarp * kUnroll) {
        uint4 av[kUnroll], bv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int j = c0 + u * kWarp + lane;
            if (j < nvec) {
                av[u] = ld_stream(ar + 8 * j);
                bv[u] = ld_stream(br + 8 * j);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int j = c0 + u * kWarp + lane;
            if (j < nvec) {
                float af[8], bf[8], o[8];
                unpack8(av[u], af);
                unpack8(bv[u], bf);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    o[e] = silu_mul(af[e], bf[e]);
                st_stream(orow + 8 * j, pack8(o));
            }
        }
    }
}

}  // namespace

cudaError_t launch_swiglu(const SwigluParams& p, cudaStream_t stream)
{
    const unsigned grid = (unsigned)((p.pk.num_rows_padded + kWarpsPerCta - 1) / kWarpsPerCta);
    swiglu_kernel<<<grid, kCtaThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace dit
