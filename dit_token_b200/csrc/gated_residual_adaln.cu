// gated_residual_adaln.cu -- the residual update of one DiT sublayer fused with
// the modulated normalization that opens the next one:
//   res  = bf16(x + gate_b * y)                        (written: the residual stream)
//   norm = bf16(LN(res) * (1 + scale_b) + shift_b)     (written: the next sublayer's input)
// "Why Real-Time MiniMax H3 Serving Requires More Than a Faster DiT", "Key
// takeaways", bullet 2 lists residual updates next to modulation and
// normalization among the fused work.  LN reads the residual as stored
// (rounded to bf16), so the pair equals the two separate ops back to back,
// bit for bit up to the fp32 reduction order -- while HBM sees x and y read
// once and res and norm written once: 8 bytes per element instead of the
// 10 of the unfused pair.
//
// Layout as in adaln_modulate.cu: a team of TEAM warps owns a row and keeps
// the rounded residual in registers (VPT 16-byte vectors per lane).
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

template <int VPT, int TEAM>
__global__ void __launch_bounds__(kCtaThreads, MinCtas<VPT, 2>::value)
gated_residual_adaln_kernel(const FusedParams p)
{
    constexpr int kRowsPerCta = kWarpsPerCta / TEAM;
    constexpr int kTeamThreads = TEAM * kWarp;
    __shared__ float red[2][kWarpsPerCta];

    const int lane = threadIdx.x & (kWarp - 1);
    const int warp = threadIdx.x >> 5;
    const int team = warp / TEAM;
    const int tt = (warp % TEAM) * kWarp + lane;
    const int v = blockIdx.x * kRowsPerCta + team;
    RowSlot s;
    const bool active = map_valid_row(v, p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs,
                                      p.pk.num_rows_padded, lane, s);
    if (!active)
        return;  // the whole team leaves: its barriers involve only its own warps
    const int nvec = p.hidden / 8;

    // residual update, rounded once, kept packed
    uint4 rv[VPT];
    {
        uint4 xv[VPT], yv[VPT];
        const uint16_t* xr = p.x + (int64_t)s.row * p.x_row_stride;
        const uint16_t* yr = p.y + (int64_t)s.row * p.y_row_stride;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int j = i * kTeamThreads + tt;
            const bool in = j < nvec;
            xv[i] = in ? ld_stream(xr + 8 * j) : make_uint4(0u, 0u, 0u, 0u);
            yv[i] = in ? ld_stream(yr + 8 * j) : make_uint4(0u, 0u, 0u, 0u);
        }
        const uint16_t* gr = p.gate + (int64_t)s.seq * p.gate_seq_stride;
        uint16_t* res = p.res_out + (int64_t)s.row * p.res_row_stride;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int j = i * kTeamThreads + tt;
            if (j < nvec) {
                float xf[8], yf[8], gf[8], o[8];
                unpack8(xv[i], xf);
                unpack8(yv[i], yf);
                unpack8(ld_shared_vec(gr + 8 * j), gf);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    o[e] = fmaf(gf[e], yf[e], xf[e]);
                rv[i] = pack8(o);
                st_stream(res + 8 * j, rv[i]);
            } else {
                rv[i] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    }

    // LN statistics of the stored residual
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        float f[8];
        unpack8(rv[i], f);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            sum += f[e];
    }
    sum = group_sum<kWarp>(sum);
    if (TEAM > 1) {
        if (lane == 0)
            red[0][warp] = sum;
        team_barrier<TEAM>(team);
        sum = 0.f;
#pragma unroll
        for (int w = 0; w < TEAM; ++w)
            sum += red[0][team * TEAM + w];
    }
    const float inv_n = 1.0f / (float)p.hidden;
    const float mean = sum * inv_n;
    float sq = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = i * kTeamThreads + tt;
        if (j < nvec) {
            float f[8];
            unpack8_again(rv[i], f);
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
        team_barrier<TEAM>(team);
        sq = 0.f;
#pragma unroll
        for (int w = 0; w < TEAM; ++w)
            sq += red[1][team * TEAM + w];
    }
    const float rstd = rsqrtf(sq * inv_n + p.eps);

    const uint16_t* sh = p.shift + (int64_t)s.seq * p.mod_seq_stride;
    const uint16_t* sc = p.scale + (int64_t)s.seq * p.mod_seq_stride;
    uint16_t* nrow = p.norm_out + (int64_t)s.row * p.norm_row_stride;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = i * kTeamThreads + tt;
        if (j < nvec) {
            float f[8], shf[8], scf[8], o[8];
            unpack8_again(rv[i], f);
            unpack8(ld_shared_vec(sh + 8 * j), shf);
            unpack8(ld_shared_vec(sc + 8 * j), scf);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                o[e] = fmaf((f[e] - mean) * rstd, 1.0f + scf[e], shf[e]);
            st_stream(nrow + 8 * j, pack8(o));
        }
    }
}

template <int TEAM, int VPT>
void launch_one(const FusedParams& p, cudaStream_t stream)
{
    const int rows_per_cta = kWarpsPerCta / TEAM;
    const unsigned grid = (unsigned)((p.pk.num_rows_padded + rows_per_cta - 1) / rows_per_cta);
    gated_residual_adaln_kernel<VPT, TEAM><<<grid, kCtaThreads, 0, stream>>>(p);
}

template <int TEAM>
cudaError_t launch_team(const FusedParams& p, int vpt, cudaStream_t stream)
{
    switch (vpt) {
    case 1: launch_one<TEAM, 1>(p, stream); break;
    case 2: launch_one<TEAM, 2>(p, stream); break;
    case 3: launch_one<TEAM, 3>(p, stream); break;
    case 4: launch_one<TEAM, 4>(p, stream); break;
    case 5: launch_one<TEAM, 5>(p, stream); break;
    case 6: launch_one<TEAM, 6>(p, stream); break;
    case 7: launch_one<TEAM, 7>(p, stream); break;
    case 8: launch_one<TEAM, 8>(p, stream); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

// Team size: the smallest of 1, 2, 4, 8 warps that holds the row in at most 8
// vectors per lane (hidden 2048 -> 1 warp, 3072 -> 2, 5120 -> 4).
cudaError_t launch_gated_residual_adaln(const FusedParams& p, cudaStream_t stream)
{
    const int nvec = p.hidden / 8;
    for (int team = 1; team <= kWarpsPerCta; team *= 2) {
        const int per = team * kWarp;
        const int vpt = (nvec + per - 1) / per;
        if (vpt > 8)
            continue;
        switch (team) {
        case 1: return launch_team<1>(p, vpt, stream);
        case 2: return launch_team<2>(p, vpt, stream);
        case 4: return launch_team<4>(p, vpt, stream);
        default: return launch_team<8>(p, vpt, stream);
        }
    }
    return cudaErrorInvalidValue;  // hidden > kMaxAdalnHidden, rejected by the ABI first
}

}  // namespace dit
