// gated_residual.cu -- out = x + gate_b * y over the valid rows of a packed
// sequence ("Why Real-Time MiniMax H3 Serving Requires More Than a Faster
// DiT", "Key takeaways", bullet 2: the residual update is one of the fused
// operators).
//
// One warp per valid row; each lane streams U 16-byte vectors of x and y per
// step (all loads of a step are issued before any arithmetic), adds
// gate * y with one fp32 FMA per element and rounds once.  The gate vector is
// read through the read-only path: it is shared by every row of a sequence and
// stays in L1/L2.  HBM traffic: 6 bytes per element (x, y in; out out).
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

#ifndef DIT_EW_UNROLL
#define DIT_EW_UNROLL 4
#endif
constexpr int kUnroll = DIT_EW_UNROLL;  // 16-byte vectors per lane and input in flight

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
    const uint16_t* gr = p.gate + (int64_t)s.seq * p.gate_seq_stride;
    uint16_t* orow = p.out + (int64_t)s.row * p.out_row_stride;
    const int nvec = p.hidden / 8;

    for (int c0 = 0; c0 < nvec; c0 += kWarp * kUnroll) {
        uint4 xv[kUnroll], yv[kUnroll], gv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int j = c0 + u * kWarp + lane;
            if (j < nvec) {
                xv[u] = ld_stream(xr + 8 * j);
                yv[u] = ld_stream(yr + 8 * j);
                gv[u] = ld_shared_vec(gr + 8 * j);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int j = c0 + u * kWarp + lane;
            if (j < nvec) {
                float xf[8], yf[8], gf[8], o[8];
                unpack8(xv[u], xf);
                unpack8(yv[u], yf);
                unpack8(gv[u], gf);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    o[e] = fmaf(gf[e], yf[e], xf[e]);
                st_stream(orow + 8 * j, pack8(o));
            }
        }
    }
}

}  // namespace

cudaError_t launch_gated_residual(const GatedParams& p, cudaStream_t stream)
{
    const unsigned grid = (unsigned)((p.pk.num_rows_padded + kWarpsPerCta - 1) / kWarpsPerCta);
    gated_residual_kernel<<<grid, kCtaThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace dit
