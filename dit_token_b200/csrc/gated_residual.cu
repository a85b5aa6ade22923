// gated_residual.cu -- out = x + gate_b * y over the valid rows of a packed
// sequence ("Why Real-Time MiniMax H3 Serving Requires More Than a Faster
// DiT", "Key takeaways", bullet 2: the residual update is one of the fused
// operators).
//
// One warp per valid row in CTAs of 4 warps; each lane streams UNR vectors of
// x and y per step (all loads of a step are issued before any arithmetic),
// adds gate * y with one fp32 FMA per element and rounds once.  The gate
// vector (bf16, or fp32 as the modulation head may emit it) is read through
// the read-only path: it is shared by every row of a sequence and stays in
// L1/L2.  With a bf16 gate and rows on 32-byte boundaries a lane moves 32
// bytes per access (2 vectors in flight): 308 us on batched varlen (hidden
// 5120, 2.15 GB) against 314 us with 16-byte accesses, and 22.5 against 24.6
// us on one rank's slice of the long video (7,736 rows of 3072).  An fp32
// gate keeps 16-byte activation accesses, so that a lane's share of the gate
// is one contiguous 32-byte piece.  HBM traffic: 6 bytes per element (x, y
// in; out out).
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

constexpr int kResWarps = 4;  // rows (warps) per CTA

template <int NW, int UNR, bool F32>
__global__ void __launch_bounds__(kResWarps * kWarp)
gated_residual_kernel(const GatedParams p)
{
    constexpr int EPV = 2 * NW;
    constexpr int NG = NW < 4 ? NW : 4;  // words per read of the gate
    grid_dependency_wait();
    const int lane = threadIdx.x & (kWarp - 1);
    const int v = blockIdx.x * kResWarps + (threadIdx.x >> 5);
    RowSlot s;
    if (!map_valid_row(v, p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs,
                       p.pk.num_rows_padded, lane, s))
        return;
    const uint16_t* xr = p.x + (int64_t)s.row * p.x_row_stride;
    const uint16_t* yr = p.y + (int64_t)s.row * p.y_row_stride;
    const int64_t goff = (int64_t)s.seq * p.gate_seq_stride;
    uint16_t* orow = p.out + (int64_t)s.row * p.out_row_stride;
    const int nvec = p.hidden / EPV;

    for (int c0 = 0; c0 < nvec; c0 += kWarp * UNR) {
        uint32_t xv[UNR][NW], yv[UNR][NW];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int j = c0 + u * kWarp + lane;
            if (j < nvec) {
                ld_stream_words<NW>(xr + EPV * j, xv[u]);
                ld_stream_words<NW>(yr + EPV * j, yv[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int j = c0 + u * kWarp + lane;
            if (j < nvec) {
                uint32_t o[NW];
#pragma unroll
                for (int h = 0; h < NW / NG; ++h) {
                    f32x2 g[NG];
                    vec_pairs<F32, NG>(p.gate, goff + EPV * j + 2 * NG * h, g);
#pragma unroll
                    for (int e = 0; e < NG; ++e)
                        o[NG * h + e] = f2_to_bf16x2(
                            f2_fma(g[e], f2_from_bf16x2(yv[u][NG * h + e]), f2_from_bf16x2(xv[u][NG * h + e])));
                }
                st_stream_words<NW>(orow + EPV * j, o);
            }
        }
    }
}

}  // namespace

cudaError_t launch_gated_residual(const GatedParams& p, cudaStream_t stream)
{
    const unsigned grid = (unsigned)((p.pk.num_rows_padded + kResWarps - 1) / kResWarps);
    const dim3 block(kResWarps * kWarp);
    if (p.gate_f32)
        return launch_kernel(gated_residual_kernel<4, 4, true>, grid, block, 0, stream, p);
    const bool wide = aligned32(p.x) && aligned32(p.y) && aligned32(p.out) && p.hidden % 16 == 0 &&
                      p.x_row_stride % 16 == 0 && p.y_row_stride % 16 == 0 && p.out_row_stride % 16 == 0;
    return wide ? launch_kernel(gated_residual_kernel<8, 2, false>, grid, block, 0, stream, p)
                : launch_kernel(gated_residual_kernel<4, 4, false>, grid, block, 0, stream, p);
}

}  // namespace dit
