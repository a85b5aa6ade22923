// gated_residual_adaln.cu -- the residual update of one DiT sublayer fused with
// the modulated normalization that opens the next one:
//   res  = bf16(x + gate_b * y)                        (written: the residual stream)
//   norm = bf16(LN(res) * (1 + scale_b) + shift_b)     (written: the next sublayer's input)
// "Why Real-Time MiniMax H3 Serving Requires More Than a Faster DiT", "Key
// takeaways", bullet 2 lists residual updates next to modulation and
// normalization among the fused work.  LN reads the residual as stored
// (rounded to bf16), so the pair equals the two separate ops back to back
// (the residual bit for bit; the normalization up to the order in which the
// row statistics are merged) -- while HBM sees x and y read once and res and
// norm written once: 8 bytes per element instead of the 10 of the unfused
// pair.
//
// Layout as in adaln_modulate.cu: a team of TEAM warps owns a row and keeps
// the rounded residual in registers (VPT 16-byte vectors per lane); one-pass
// moments for the statistics, packed fp32 pairs for the arithmetic.  gate,
// shift and scale are bf16, or all three fp32.  One short-lived CTA per two
// to four rows: a persistent form (each team a fixed run of rows, the
// vectors staged once per CTA in shared memory as fp32) measured slower,
// 569 against 455 us on batched varlen (hidden 5120) and 322 against 234 us
// on 61,888 rows of hidden 3072, even with fp32 vectors (591 against 527 us).
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

template <int VPT, int TEAM, bool F32>
__global__ void __launch_bounds__(kCtaThreads, MinCtas<VPT, 2>::value)
gated_residual_adaln_kernel(const FusedParams p)
{
    constexpr int kRowsPerCta = kWarpsPerCta / TEAM;
    constexpr int kTeamThreads = TEAM * kWarp;
    __shared__ Moments red[kWarpsPerCta];

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
        const int64_t goff = (int64_t)s.seq * p.gate_seq_stride;
        uint16_t* res = p.res_out + (int64_t)s.row * p.res_row_stride;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int j = i * kTeamThreads + tt;
            if (j < nvec) {
                f32x2 g[4];
                vec8_pairs<F32>(p.gate, goff + 8 * j, g);
                const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
                const uint32_t yw[4] = {yv[i].x, yv[i].y, yv[i].z, yv[i].w};
                uint32_t o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    o[e] = f2_to_bf16x2(f2_fma(g[e], f2_from_bf16x2(yw[e]), f2_from_bf16x2(xw[e])));
                rv[i] = make_uint4(o[0], o[1], o[2], o[3]);
                st_stream(res + 8 * j, rv[i]);
            } else {
                rv[i] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    }

    // LN statistics of the stored residual: shifted sums, merged as moments
    const float k = bf16_lo(rv[0].x);
    const f32x2 kk = f2_make(k, k);
    f32x2 s2 = f2_make(0.f, 0.f), q2 = f2_make(0.f, 0.f);
    float cnt = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = i * kTeamThreads + tt;
        if (j < nvec) {
            const uint32_t w[4] = {rv[i].x, rv[i].y, rv[i].z, rv[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const f32x2 d = f2_sub(f2_from_bf16x2(w[e]), kk);
                s2 = f2_add(s2, d);
                q2 = f2_fma(d, d, q2);
            }
            cnt += 8.f;
        }
    }
    float s0, s1, q0, q1;
    f2_split(s2, s0, s1);
    f2_split(q2, q0, q1);
    Moments m = moments_warp(moments_from_sums(cnt, k, s0 + s1, q0 + q1));
    if (TEAM > 1) {
        if (lane == 0)
            red[warp] = m;
        team_barrier<TEAM>(team);
        m = red[team * TEAM];
#pragma unroll
        for (int w = 1; w < TEAM; ++w)
            m = moments_merge(m, red[team * TEAM + w]);
    }
    const float rstd = rsqrtf(m.m2 * (1.0f / (float)p.hidden) + p.eps);  // as in adaln_modulate.cu
    const f32x2 r2 = f2_make(rstd, rstd);
    const float nb = -m.mean * rstd;
    const f32x2 b2 = f2_make(nb, nb);
    const f32x2 one2 = f2_make(1.f, 1.f);

    const int64_t moff = (int64_t)s.seq * p.mod_seq_stride;
    uint16_t* nrow = p.norm_out + (int64_t)s.row * p.norm_row_stride;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = i * kTeamThreads + tt;
        if (j < nvec) {
            f32x2 hv[4], cv[4];
            vec8_pairs<F32>(p.shift, moff + 8 * j, hv);
            vec8_pairs<F32>(p.scale, moff + 8 * j, cv);
            const uint32_t rw[4] = {rv[i].x, rv[i].y, rv[i].z, rv[i].w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const f32x2 t = f2_fma(f2_from_bf16x2(rw[e]), r2, b2);
                o[e] = f2_to_bf16x2(f2_fma(t, f2_add(cv[e], one2), hv[e]));
            }
            st_stream(nrow + 8 * j, make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
}

template <int TEAM, int VPT>
void launch_one(const FusedParams& p, cudaStream_t stream)
{
    const int rows_per_cta = kWarpsPerCta / TEAM;
    const unsigned grid = (unsigned)((p.pk.num_rows_padded + rows_per_cta - 1) / rows_per_cta);
    if (p.mod_f32)
        gated_residual_adaln_kernel<VPT, TEAM, true><<<grid, kCtaThreads, 0, stream>>>(p);
    else
        gated_residual_adaln_kernel<VPT, TEAM, false><<<grid, kCtaThreads, 0, stream>>>(p);
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

// Team size: the smallest of 2, 4, 8 warps that holds the row in at most 8
// vectors per lane (hidden 2048 -> 2 warps, 3072 -> 2, 5120 -> 4).  A single
// warp per row was measured slower on short rows (hidden 2048: 36.9 against
// 29.9 us for 8192 rows), and at most 4 vectors per lane slower on long ones
// (hidden 5120: 568 against 456 us).
cudaError_t launch_gated_residual_adaln(const FusedParams& p, cudaStream_t stream)
{
    const int nvec = p.hidden / 8;
    for (int team = 2; team <= kWarpsPerCta; team *= 2) {
        const int per = team * kWarp;
        const int vpt = (nvec + per - 1) / per;
        if (vpt > 8)
            continue;
        switch (team) {
        case 2: return launch_team<2>(p, vpt, stream);
        case 4: return launch_team<4>(p, vpt, stream);
        default: return launch_team<8>(p, vpt, stream);
        }
    }
    return cudaErrorInvalidValue;  // hidden > kMaxAdalnHidden, rejected by the ABI first
}

}  // namespace dit
