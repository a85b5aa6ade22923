// adaln_modulate.cu -- out = LN(x) * (1 + scale_b) + shift_b over the valid rows
// of a packed sequence ("Why Real-Time MiniMax H3 Serving Requires More Than a
// Faster DiT", "Key takeaways", bullet 2: the adaptive normalization and its
// modulation are one of the fused operators).  LN has no affine; the variance is the biased one.
//
// A team of TEAM warps owns one row and keeps the whole row in registers
// (VPT 16-byte vectors per lane), so x is read from HBM once: a warp-shuffle
// sum gives the mean, a second pass over the registers the sum of squared
// deviations (exact two-pass variance), and a third pass writes the
// modulated output.  Teams of more than one warp combine their partial sums
// through shared memory.  HBM traffic: 4 bytes per element.
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

template <int VPT, int TEAM>
__global__ void __launch_bounds__(kCtaThreads)
adaln_kernel(const AdalnParams p)
{
    constexpr int kRowsPerCta = kWarpsPerCta / TEAM;
    constexpr int kTeamThreads = TEAM * kWarp;
    __shared__ float red[2][kWarpsPerCta];

    const int lane = threadIdx.x & (kWarp - 1);
    const int warp = threadIdx.x >> 5;
    const int team = warp / TEAM;
    const int tt = (warp % TEAM) * kWarp + lane;  // thread index within the team
    const int v = blockIdx.x * kRowsPerCta + team;
    RowSlot s;
    const bool active = map_valid_row(v, p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs,
                                      p.pk.num_rows_padded, lane, s);
    if (TEAM == 1 && !active)
        return;  // single-warp teams never meet a CTA barrier
    const int nvec = p.hidden / 8;
    const uint16_t* xr = active ? p.x + (int64_t)s.row * p.x_row_stride : p.x;

    uint4 xv[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = i * kTeamThreads + tt;
        xv[i] = (active && j < nvec) ? ld_stream(xr + 8 * j) : make_uint4(0u, 0u, 0u, 0u);
    }

    // mean
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        float f[8];
        unpack8(xv[i], f);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            sum += f[e];
    }
    sum = group_sum<kWarp>(sum);
    if (TEAM > 1) {
        if (lane == 0)
            red[0][warp] = sum;
        __syncthreads();
        sum = 0.f;
#pragma unroll
        for (int w = 0; w < TEAM; ++w)
            sum += red[0][team * TEAM + w];
    }
    const float inv_n = 1.0f / (float)p.hidden;
    const float mean = sum * inv_n;

    // biased variance about the mean (padding lanes hold zeros: skip them)
    float sq = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = i * kTeamThreads + tt;
        if (j < nvec) {
            float f[8];
            unpack8(xv[i], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float d = f[e] - mean;
                sq = fmaf(d, d, sq);
            }
        }
    }
    sq = group_sum<kWarp>(sq);
    if (TEAM > 1) {
        if (lane == 0)
            red[1][warp] = sq;
        __syncthreads();
        sq = 0.f;
#pragma unroll
        for (int w = 0; w < TEAM; ++w)
            sq += red[1][team * TEAM + w];
    }
    if (!active)
        return;  // after the last barrier
    const float rstd = rsqrtf(sq * inv_n + p.eps);

    const uint16_t* sh = p.shift + (int64_t)s.seq * p.mod_seq_stride;
    const uint16_t* sc = p.scale + (int64_t)s.seq * p.mod_seq_stride;
    uint16_t* orow = p.out + (int64_t)s.row * p.out_row_stride;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = i * kTeamThreads + tt;
        if (j < nvec) {
            float f[8], shf[8], scf[8], o[8];
            unpack8(xv[i], f);
            unpack8(ld_shared_vec(sh + 8 * j), shf);
            unpack8(ld_shared_vec(sc + 8 * j), scf);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                o[e] = fmaf((f[e] - mean) * rstd, 1.0f + scf[e], shf[e]);
            st_stream(orow + 8 * j, pack8(o));
        }
    }
}

template <int TEAM>
cudaError_t launch_team(const AdalnParams& p, int vpt, cudaStream_t stream)
{
    const int rows_per_cta = kWarpsPerCta / TEAM;
    const unsigned grid = (unsigned)((p.pk.num_rows_padded + rows_per_cta - 1) / rows_per_cta);
    switch (vpt) {
    case 1: adaln_kernel<1, TEAM><<<grid, kCtaThreads, 0, stream>>>(p); break;
    case 2: adaln_kernel<2, TEAM><<<grid, kCtaThreads, 0, stream>>>(p); break;
    case 3: adaln_kernel<3, TEAM><<<grid, kCtaThreads, 0, stream>>>(p); break;
    case 4: adaln_kernel<4, TEAM><<<grid, kCtaThreads, 0, stream>>>(p); break;
    case 5: adaln_kernel<5, TEAM><<<grid, kCtaThreads, 0, stream>>>(p); break;
    case 6: adaln_kernel<6, TEAM><<<grid, kCtaThreads, 0, stream>>>(p); break;
    case 7: adaln_kernel<7, TEAM><<<grid, kCtaThreads, 0, stream>>>(p); break;
    case 8: adaln_kernel<8, TEAM><<<grid, kCtaThreads, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

// Team size: the smallest of 1, 2, 4, 8 warps that holds the row in at most 8
// vectors per lane (hidden 2048 -> 1 warp, 3072 -> 2, 5120 -> 4).
cudaError_t launch_adaln_modulate(const AdalnParams& p, cudaStream_t stream)
{
    const int nvec = p.hidden / 8;
    for (int team = 1; team <= kWarpsPerCta; team *= 2) {
        const int per = team * kWarp;
        const int vpt = (nvec + per - 1) / per;
        if (vpt <= 8) {
            switch (team) {
            case 1: return launch_team<1>(p, vpt, stream);
            case 2: return launch_team<2>(p, vpt, stream);
            case 4: return launch_team<4>(p, vpt, stream);
            default: return launch_team<8>(p, vpt, stream);
            }
        }
    }
    return cudaErrorInvalidValue;  // hidden > kMaxAdalnHidden, rejected by the ABI first
}

}  // namespace dit
