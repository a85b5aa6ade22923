// adaln_modulate.cu -- out = LN(x) * (1 + scale_b) + shift_b over the valid rows
// of a packed sequence ("Why Real-Time MiniMax H3 Serving Requires More Than a
// Faster DiT", "Key takeaways", bullet 2: the adaptive normalization and its
// modulation are one of the fused operators).  LN has no affine; the variance
// is the biased one.
//
// Shape, for rows of up to 6144 elements: one warp owns a row and holds it in
// registers (x is read from HBM once), short-lived CTAs of 4 warps, one row
// each, so the hardware keeps every SM filled with new rows as old ones
// finish.  A lane holds VPT vectors of 16 elements (32-byte accesses, when
// the row pointers allow) or of 8 elements (16-byte accesses).  Statistics
// in one pass: per-lane sums about the lane's first value, merged over the
// warp as (count, mean, M2) moments by shuffles.  Output pass: per element
// (x * rstd - mean * rstd) * (1 + scale) + shift in packed fp32 pairs, the
// per-sequence vectors read through the read-only path (they stay in L1/L2:
// every row of a sequence reads the same 2 * hidden values).  Wider rows (to
// 16384 elements) use a team of 2-8 warps per row with a named barrier per
// team.  HBM traffic: 4 bytes per element.
//
// Measured (batched varlen, hidden 5120, 1.43 GB per launch, L2 clean; the
// B200's measured copy bandwidth 6458 GB/s): this kernel 228.9 us (96.7 %);
// the same with 16-byte accesses 268 us, with 8-warp CTAs 241.8 us.  The
// earlier persistent design (2 CTAs of 8 warps per SM, contiguous per-warp
// row runs, the CTA's modulation staged in shared memory as fp32) ran 241.7
// us: ncu on a full-size launch showed 24 % of warp slots active (128
// registers) and short-scoreboard stalls on the staged vectors as the
// largest stall (3.1 per issued instruction); it also lost to this kernel at
// every other shape (61,888 rows of 3072: 129.3 against 115.6 us; 7,736 rows
// of 3072: 24.6 against 23.6 us; 8,192 rows of 2048: 21.4 against 18.5 us).
// Persistent variants with fewer staged sequences, grid-stride or
// interleaved row order, 16-warp CTAs or 32-byte accesses all measured
// between 236 and 420 us.
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

constexpr int kRowWarps = 4;                 // rows (warps) per CTA of the row kernel
constexpr int kRowCtaThreads = kRowWarps * kWarp;
constexpr int kMaxRowElems = 6144;           // widest row one warp holds

// Statistics of the VPT vectors of NW words a lane holds (vectors at or past
// nvec are empty), merged over the warp.  Vector i of the lane is vector
// i * STRIDE + lane_vec0 of the row.
template <int VPT, int NW, int STRIDE>
__device__ __forceinline__ Moments lane_row_moments(const uint32_t (&xv)[VPT][NW], int lane_vec0, int nvec)
{
    const float k = bf16_lo(xv[0][0]);
    const f32x2 kk = f2_make(k, k);
    f32x2 s2 = f2_make(0.f, 0.f), q2 = f2_make(0.f, 0.f);
    float cnt = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        if (i * STRIDE + lane_vec0 < nvec) {
#pragma unroll
            for (int e = 0; e < NW; ++e) {
                const f32x2 d = f2_sub(f2_from_bf16x2(xv[i][e]), kk);
                s2 = f2_add(s2, d);
                q2 = f2_fma(d, d, q2);
            }
            cnt += (float)(2 * NW);
        }
    }
    return moments_warp(moments_from_sums(cnt, k, s2.x + s2.y, q2.x + q2.y));
}

// 2 * NP output elements (NP words, NP = 2 or 4): (x * rstd + nb) *
// (1 + scale) + shift, with the sequence's vectors read at element
// `moff_elem`.
template <bool F32, int NP>
__device__ __forceinline__ void modulate_words(const uint32_t* x, uint32_t* o, f32x2 r2, f32x2 b2,
                                               const AdalnParams& p, int64_t moff_elem)
{
    f32x2 A[NP], B[NP];
    vec_pairs<F32, NP>(p.scale, moff_elem, A);
    vec_pairs<F32, NP>(p.shift, moff_elem, B);
    const f32x2 one2 = f2_make(1.f, 1.f);
#pragma unroll
    for (int e = 0; e < NP; ++e)
        o[e] = f2_to_bf16x2(f2_fma(f2_fma(f2_from_bf16x2(x[e]), r2, b2), f2_add(A[e], one2), B[e]));
}

// Words of a row vector modulated together: a vector of NW words is done in
// groups of NG (the per-sequence vectors are read 4 or 8 elements at a time).
template <int NW>
constexpr int kGroupWords = NW < 4 ? NW : 4;

// ------------------------------------------------------------ warp per row

template <int VPT, int NW, bool F32>
__global__ void __launch_bounds__(kRowCtaThreads)
adaln_row_kernel(const AdalnParams p)
{
    constexpr int EPV = 2 * NW;  // elements per vector
    grid_dependency_wait();
    const int lane = threadIdx.x & (kWarp - 1);
    const int v = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
    RowSlot s;
    if (!map_valid_row(v, p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs, p.pk.num_rows_padded, lane, s))
        return;  // uniform over the warp
    const int nvec = p.hidden / EPV;
    const uint16_t* xr = p.x + (int64_t)s.row * p.x_row_stride + EPV * lane;
    uint32_t xv[VPT][NW];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        if (i * kWarp + lane < nvec) {
            ld_stream_words<NW>(xr + EPV * kWarp * i, xv[i]);
        } else {
#pragma unroll
            for (int e = 0; e < NW; ++e)
                xv[i][e] = 0u;
        }
    }
    const Moments m = lane_row_moments<VPT, NW, kWarp>(xv, lane, nvec);
    const float rstd = rsqrtf(m.m2 * (1.0f / (float)p.hidden) + p.eps);
    const f32x2 r2 = f2_make(rstd, rstd);
    const float nb = -m.mean * rstd;
    const f32x2 b2 = f2_make(nb, nb);
    uint16_t* orow = p.out + (int64_t)s.row * p.out_row_stride + EPV * lane;
    const int64_t moff = (int64_t)s.seq * p.mod_seq_stride + EPV * lane;
    constexpr int NG = kGroupWords<NW>;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        if (i * kWarp + lane < nvec) {
            uint32_t o[NW];
#pragma unroll
            for (int h = 0; h < NW / NG; ++h)
                modulate_words<F32, NG>(xv[i] + NG * h, o + NG * h, r2, b2, p, moff + EPV * kWarp * i + 2 * NG * h);
            st_stream_words<NW>(orow + EPV * kWarp * i, o);
        }
    }
}

template <int VPT, int NW>
cudaError_t launch_row_t(const AdalnParams& p, cudaStream_t stream)
{
    const unsigned grid = (unsigned)((p.pk.num_rows_padded + kRowWarps - 1) / kRowWarps);
    return p.mod_f32 ? launch_kernel(adaln_row_kernel<VPT, NW, true>, grid, kRowCtaThreads, 0, stream, p)
                     : launch_kernel(adaln_row_kernel<VPT, NW, false>, grid, kRowCtaThreads, 0, stream, p);
}

// VPT rounded up to an instantiated count (the bounds checks cover the rest).
template <int NW>
cudaError_t launch_row(const AdalnParams& p, cudaStream_t stream)
{
    const int vpt = (p.hidden / (2 * NW) + kWarp - 1) / kWarp;
    if (vpt <= 4) {
        switch (vpt) {
        case 1: return launch_row_t<1, NW>(p, stream);
        case 2: return launch_row_t<2, NW>(p, stream);
        case 3: return launch_row_t<3, NW>(p, stream);
        default: return launch_row_t<4, NW>(p, stream);
        }
    }
    if constexpr (NW == 2) {  // at most 48 vectors of 4
        if (vpt <= 6)
            return launch_row_t<6, NW>(p, stream);
        if (vpt <= 8)
            return launch_row_t<8, NW>(p, stream);
        if (vpt <= 12)
            return launch_row_t<12, NW>(p, stream);
        if (vpt <= 16)
            return launch_row_t<16, NW>(p, stream);
        if (vpt <= 24)
            return launch_row_t<24, NW>(p, stream);
        if (vpt <= 32)
            return launch_row_t<32, NW>(p, stream);
        if (vpt <= 40)
            return launch_row_t<40, NW>(p, stream);
        return launch_row_t<48, NW>(p, stream);
    } else if constexpr (NW == 8) {  // rows of up to 6144 elements: at most 12 vectors of 16
        if (vpt <= 5)
            return launch_row_t<5, NW>(p, stream);
        if (vpt <= 6)
            return launch_row_t<6, NW>(p, stream);
        if (vpt <= 8)
            return launch_row_t<8, NW>(p, stream);
        if (vpt <= 10)
            return launch_row_t<10, NW>(p, stream);
        return launch_row_t<12, NW>(p, stream);
    } else {  // at most 24 vectors of 8
        if (vpt <= 6)
            return launch_row_t<6, NW>(p, stream);
        if (vpt <= 8)
            return launch_row_t<8, NW>(p, stream);
        if (vpt <= 12)
            return launch_row_t<12, NW>(p, stream);
        if (vpt <= 16)
            return launch_row_t<16, NW>(p, stream);
        if (vpt <= 20)
            return launch_row_t<20, NW>(p, stream);
        return launch_row_t<24, NW>(p, stream);
    }
}

// ------------------------------------------------------------ team per row

template <int VPT, int TEAM, bool F32>
__global__ void __launch_bounds__(kCtaThreads, MinCtas<VPT>::value)
adaln_team_kernel(const AdalnParams p)
{
    constexpr int kRowsPerCta = kWarpsPerCta / TEAM;
    constexpr int kTeamThreads = TEAM * kWarp;
    __shared__ Moments red[kWarpsPerCta];
    grid_dependency_wait();
    const int lane = threadIdx.x & (kWarp - 1);
    const int warp = threadIdx.x >> 5;
    const int team = warp / TEAM;
    const int tt = (warp % TEAM) * kWarp + lane;
    const int v = blockIdx.x * kRowsPerCta + team;
    RowSlot s;
    if (!map_valid_row(v, p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs, p.pk.num_rows_padded, lane, s))
        return;  // the whole team leaves: its barrier involves only its own warps
    const int nvec = p.hidden / 8;
    const uint16_t* xr = p.x + (int64_t)s.row * p.x_row_stride;
    uint32_t xv[VPT][4];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = i * kTeamThreads + tt;
        if (j < nvec) {
            ld_stream_words<4>(xr + 8 * j, xv[i]);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                xv[i][e] = 0u;
        }
    }
    Moments m = lane_row_moments<VPT, 4, kTeamThreads>(xv, tt, nvec);
    if (lane == 0)
        red[warp] = m;
    team_barrier<TEAM>(team);
    m = red[team * TEAM];
#pragma unroll
    for (int w = 1; w < TEAM; ++w)
        m = moments_merge(m, red[team * TEAM + w]);
    const float rstd = rsqrtf(m.m2 * (1.0f / (float)p.hidden) + p.eps);
    const f32x2 r2 = f2_make(rstd, rstd);
    const float nb = -m.mean * rstd;
    const f32x2 b2 = f2_make(nb, nb);
    const int64_t moff = (int64_t)s.seq * p.mod_seq_stride;
    uint16_t* orow = p.out + (int64_t)s.row * p.out_row_stride;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = i * kTeamThreads + tt;
        if (j < nvec) {
            uint32_t o[4];
            modulate_words<F32, 4>(xv[i], o, r2, b2, p, moff + 8 * j);
            st_stream_words<4>(orow + 8 * j, o);
        }
    }
}

template <int TEAM>
cudaError_t launch_team(const AdalnParams& p, cudaStream_t stream)
{
    const int nvec = p.hidden / 8;
    const int vpt = (nvec + TEAM * kWarp - 1) / (TEAM * kWarp);
    const int rows_per_cta = kWarpsPerCta / TEAM;
    const unsigned grid = (unsigned)((p.pk.num_rows_padded + rows_per_cta - 1) / rows_per_cta);
#define DIT_TEAM_CASE(V)                                                                                     \
    case V:                                                                                                  \
        return p.mod_f32 ? launch_kernel(adaln_team_kernel<V, TEAM, true>, grid, kCtaThreads, 0, stream, p)  \
                         : launch_kernel(adaln_team_kernel<V, TEAM, false>, grid, kCtaThreads, 0, stream, p);
    switch (vpt) {
        DIT_TEAM_CASE(4)
        DIT_TEAM_CASE(5)
        DIT_TEAM_CASE(6)
        DIT_TEAM_CASE(7)
        DIT_TEAM_CASE(8)
    default: return cudaErrorInvalidValue;
    }
#undef DIT_TEAM_CASE
}

}  // namespace

// Rows of up to 6144 elements: one warp per row.  With bf16 vectors, 32-byte
// accesses when x and out are 32-byte aligned and hidden and both row strides
// are multiples of 16 elements (every row then starts on a 32-byte
// boundary), else 16-byte ones.  With fp32 vectors, 8-byte accesses: a
// lane's share of each vector is then one 16-byte piece and a warp's vector
// loads are contiguous (with 16- or 32-byte accesses each warp load
// instruction spans 1 or 2 KB of the vector and the L1 throughput, not HBM,
// sets the pace: batched varlen 319.6 / 407.6 us against 264.3 us; 61,888
// rows of 3072: 143.4 / 217.1 against 129.1 us).  Wider rows (to 16384): the
// smallest team of 2, 4 or 8 warps that holds the row in at most 8 vectors
// per lane.
cudaError_t launch_adaln_modulate(const AdalnParams& p, cudaStream_t stream)
{
    const int nvec = p.hidden / 8;
    if (p.hidden <= kMaxRowElems) {
        if (p.mod_f32)
            return launch_row<2>(p, stream);
        const bool wide = aligned32(p.x) && aligned32(p.out) && p.hidden % 16 == 0 && p.x_row_stride % 16 == 0 &&
                          p.out_row_stride % 16 == 0;
        return wide ? launch_row<8>(p, stream) : launch_row<4>(p, stream);
    }
    if (nvec <= 2 * kWarp * 8)
        return launch_team<2>(p, stream);
    if (nvec <= 4 * kWarp * 8)
        return launch_team<4>(p, stream);
    if (nvec <= 8 * kWarp * 8)
        return launch_team<8>(p, stream);
    return cudaErrorInvalidValue;  // hidden > kMaxAdalnHidden, rejected by the ABI first
}

}  // namespace dit
