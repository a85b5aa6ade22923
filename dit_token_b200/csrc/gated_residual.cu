// gated_residual.cu -- out = x + gate_b * y over the valid rows of a packed
// sequence ("Why Real-Time MiniMax H3 Serving Requires More Than a Faster
// DiT", "Key takeaways", bullet 2: the residual update is one of the fused
// operators).
//
// One warp per valid row; each lane streams U 16-byte vectors of x and y per
// step (all loads of a step are issued before any arithmetic), adds
// gate * y with one fp32 FMA per element and rounds once.  The gate vector
// (bf16, or fp32 as the modulation head may emit it) is read through the
// read-only path: it is shared by every row of a sequence and stays in L1/L2.
// HBM traffic: 6 bytes per element (x, y in; out out).
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

#ifndef DIT_EW_UNROLL
#define DIT_EW_UNROLL 4
#endif
constexpr int kUnroll = DIT_EW_UNROLL;  // 16-byte vectors per lane and input in flight

template <bool F32>
__global__ void __launch_bounds__(kCtaThreads)
gated_residual_kernel(const GatedParams p)
{
    const int lane = threadIdx.x & (kWarp - 1);
    const int v = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    RowSlot s;
    if (!map_valid_row(v, p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs,
                       p.pk.num_rows_padded, lane, s))
        return;
    const uint16_t* xr = p.x + (int64_t)s.row * p.x_row_stride;
    const uint16_t* yr = p.y + (int64_t)s.row * p.y_row_stride;
    const int64_t goff = (int64_t)s.seq * p.gate_seq_stride;
    uint16_t* orow = p.out + (int64_t)s.row * p.out_row_stride;
    const int nvec = p.hidden / 8;

    for (int c0 = 0; c0 < nvec; c0 += kWarp * kUnroll) {
        uint4 xv[kUnroll], yv[kUnroll];
        Vec8Raw<F32> gv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int j = c0 + u * kWarp + lane;
            if (j < nvec) {
                xv[u] = ld_stream(xr + 8 * j);
                yv[u] = ld_stream(yr + 8 * j);
                gv[u] = vec8_load<F32>(p.gate, goff + 8 * j);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int j = c0 + u * kWarp + lane;
            if (j < nvec) {
                const uint32_t xw[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
                const uint32_t yw[4] = {yv[u].x, yv[u].y, yv[u].z, yv[u].w};
                f32x2 g[4];
                vec8_unpack<F32>(gv[u], g);
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    o[e] = f2_to_bf16x2(f2_fma(g[e], f2_from_bf16x2(yw[e]), f2_from_bf16x2(xw[e])));
                st_stream(orow + 8 * j, make_uint4(o[0], o[1], o[2], o[3]));
            }
        }
    }
}

}  // namespace

cudaError_t launch_gated_residual(const GatedParams& p, cudaStream_t stream)
{
    const unsigned grid = (unsigned)((p.pk.num_rows_padded + kWarpsPerCta - 1) / kWarpsPerCta);
    if (p.gate_f32)
        gated_residual_kernel<true><<<grid, kCtaThreads, 0, stream>>>(p);
    else
        gated_residual_kernel<false><<<grid, kCtaThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace dit
