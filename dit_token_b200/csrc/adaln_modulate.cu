// adaln_modulate.cu -- out = LN(x) * (1 + scale_b) + shift_b over the valid rows
// of a packed sequence ("Why Real-Time MiniMax H3 Serving Requires More Than a
// Faster DiT", "Key takeaways", bullet 2: the adaptive normalization and its
// modulation are one of the fused operators).  LN has no affine; the variance
// is the biased one.
//
// A row is held in registers (x is read from HBM once) by one warp, or by a
// team of 2-8 warps for wide rows, in short-lived CTAs, so the hardware keeps
// every SM filled with new rows as old ones finish.  A lane holds VPT vectors
// of 4, 8 or 16 elements (8-, 16- or 32-byte accesses).  Statistics in one
// pass: per-lane sums of x and x^2, added over the warp by shuffles and
// turned into (count, mean, M2) moments, which a team merges through shared
// memory behind one barrier; a row whose mean lies more than 4 deviations
// from 0 (where those sums lose digits) is summed again about its mean.
// Output pass: per element (x * rstd - mean * rstd) *
// (1 + scale) + shift in packed fp32 pairs, the per-sequence vectors read
// through the read-only path (they stay in L1/L2: every row of a sequence
// reads the same 2 * hidden values), 16 or 32 bytes per lane at a time.  HBM
// traffic: 4 bytes per element.
//
// The shape (access width, team size, vector-read width) is chosen per call
// from measurements; see adaln_shape.  The design replaced a persistent
// kernel (2 CTAs of 8 warps per SM, contiguous per-warp row runs, the CTA's
// modulation staged in shared memory as fp32): 241.7 us on batched varlen
// against 228.9 us for a warp per row with 32-byte accesses in 4-warp CTAs;
// ncu on a full-size launch of the persistent kernel showed 24 % of warp
// slots active (128 registers) and short-scoreboard stalls on the staged
// vectors as the largest stall (3.1 per issued instruction).  Persistent
// variants with fewer staged sequences, grid-stride or interleaved row order,
// 16-warp CTAs or 32-byte accesses all measured between 236 and 420 us.
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

constexpr int kRowWarps = 4;                 // rows (warps) per CTA of the warp-per-row kernel
constexpr int kRowCtaThreads = kRowWarps * kWarp;

// 2 * NP output elements (NP words): (x * rstd + nb) * (1 + scale) + shift,
// with the sequence's vectors read at element `moff_elem`: 32 bytes at a time
// (WV: NP = 8 bf16 or 4 fp32 pairs) or 8/16 bytes (NP = 2 or 4).
template <bool F32, int NP, bool WV>
__device__ __forceinline__ void modulate_words(const uint32_t* x, uint32_t* o, f32x2 r2, f32x2 b2,
                                               const AdalnParams& p, int64_t moff_elem)
{
    f32x2 A[NP], B[NP];
    if constexpr (WV) {
        vec_pairs_wide<F32, NP>(p.scale, moff_elem, A);
        vec_pairs_wide<F32, NP>(p.shift, moff_elem, B);
    } else {
        vec_pairs<F32, NP>(p.scale, moff_elem, A);
        vec_pairs<F32, NP>(p.shift, moff_elem, B);
    }
    const f32x2 one2 = f2_make(1.f, 1.f);
#pragma unroll
    for (int e = 0; e < NP; ++e)
        o[e] = f2_to_bf16x2(f2_fma(f2_fma(f2_from_bf16x2(x[e]), r2, b2), f2_add(A[e], one2), B[e]));
}

// Words of a row vector per read of the per-sequence vectors.
template <int NW, bool F32, bool WV>
constexpr int kGroupWords = WV ? (F32 ? 4 : 8) : (NW < 4 ? NW : 4);

template <int VPT, int NW, int STRIDE>
__device__ __forceinline__ void load_row(const uint16_t* xr, int lane_vec0, int nvec, uint32_t (&xv)[VPT][NW])
{
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = i * STRIDE + lane_vec0;
        if (j < nvec) {
            ld_stream_words<NW>(xr + 2 * NW * j, xv[i]);
        } else {
#pragma unroll
            for (int e = 0; e < NW; ++e)
                xv[i][e] = 0u;
        }
    }
}

// The output pass of one row: the lane's VPT vectors, vector i at row vector
// i * STRIDE + lane_vec0.
template <int VPT, int NW, int STRIDE, bool F32, bool WV>
__device__ __forceinline__ void modulate_row(const uint32_t (&xv)[VPT][NW], int lane_vec0, int nvec, float rstd,
                                             float mean, const AdalnParams& p, const RowSlot& s)
{
    constexpr int EPV = 2 * NW;
    constexpr int NG = kGroupWords<NW, F32, WV>;
    static_assert(NG <= NW, "a vector read covers at most one row vector");
    const f32x2 r2 = f2_make(rstd, rstd);
    const float nb = -mean * rstd;
    const f32x2 b2 = f2_make(nb, nb);
    uint16_t* orow = p.out + (int64_t)s.row * p.out_row_stride;
    const int64_t moff = (int64_t)s.seq * p.mod_seq_stride;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = i * STRIDE + lane_vec0;
        if (j < nvec) {
            uint32_t o[NW];
#pragma unroll
            for (int h = 0; h < NW / NG; ++h)
                modulate_words<F32, NG, WV>(xv[i] + NG * h, o + NG * h, r2, b2, p, moff + EPV * j + 2 * NG * h);
            st_stream_words<NW>(orow + EPV * j, o);
        }
    }
}

// ------------------------------------------------------------ warp per row

template <int VPT, int NW, bool F32, bool WV>
__global__ void __launch_bounds__(kRowCtaThreads)
adaln_row_kernel(const AdalnParams p)
{
    grid_dependency_wait();
    const int lane = threadIdx.x & (kWarp - 1);
    const int v = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
    RowSlot s;
    if (!map_valid_row(v, p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs, p.pk.num_rows_padded, lane, s))
        return;  // uniform over the warp
    const int nvec = p.hidden / (2 * NW);
    uint32_t xv[VPT][NW];
    load_row<VPT, NW, kWarp>(p.x + (int64_t)s.row * p.x_row_stride, lane, nvec, xv);
    const Moments m = row_moments<VPT, NW, 1>(xv, nvec, nullptr, nullptr, nullptr);
    const float rstd = rsqrtf(m.m2 * (1.0f / (float)p.hidden) + p.eps);
    modulate_row<VPT, NW, kWarp, F32, WV>(xv, lane, nvec, rstd, m.mean, p, s);
}

// ------------------------------------------------------------ team per row

// One row per CTA of TEAM warps.
template <int VPT, int NW, int TEAM, bool F32, bool WV>
__global__ void __launch_bounds__(TEAM * kWarp)
adaln_team_kernel(const AdalnParams p)
{
    constexpr int kTeamThreads = TEAM * kWarp;
    __shared__ Moments red[TEAM], red2[TEAM];
    __shared__ int far_w[TEAM];
    grid_dependency_wait();
    const int lane = threadIdx.x & (kWarp - 1);
    const int tt = threadIdx.x;
    RowSlot s;
    if (!map_valid_row(blockIdx.x, p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs, p.pk.num_rows_padded,
                       lane, s))
        return;  // uniform over the CTA: every warp maps the same row
    const int nvec = p.hidden / (2 * NW);
    uint32_t xv[VPT][NW];
    load_row<VPT, NW, kTeamThreads>(p.x + (int64_t)s.row * p.x_row_stride, tt, nvec, xv);
    const Moments m = row_moments<VPT, NW, TEAM>(xv, nvec, red, red2, far_w);
    const float rstd = rsqrtf(m.m2 * (1.0f / (float)p.hidden) + p.eps);
    modulate_row<VPT, NW, kTeamThreads, F32, WV>(xv, tt, nvec, rstd, m.mean, p, s);
}

// ------------------------------------------------------------ launch

// The smallest instantiated vector count >= vpt: every count to 8, then 10
// and 12 for one warp per row (the bounds checks cover the vectors a lane
// does not have); teams hold at most 8.
template <int NW, int TEAM, bool F32, bool WV, int V = 1>
cudaError_t launch_vpt(const AdalnParams& p, int vpt, cudaStream_t stream)
{
    if constexpr (V > (TEAM == 1 ? 12 : 8)) {
        return cudaErrorInvalidValue;
    } else {
        if (vpt <= V) {
            if constexpr (TEAM == 1) {
                const unsigned grid = (unsigned)((p.pk.num_rows_padded + kRowWarps - 1) / kRowWarps);
                return launch_kernel(adaln_row_kernel<V, NW, F32, WV>, grid, kRowCtaThreads, 0, stream, p);
            } else {
                const unsigned grid = (unsigned)p.pk.num_rows_padded;  // one row per CTA
                return launch_kernel(adaln_team_kernel<V, NW, TEAM, F32, WV>, grid, TEAM * kWarp, 0, stream, p);
            }
        }
        constexpr int kNext = V < 8 ? V + 1 : V + 2;
        return launch_vpt<NW, TEAM, F32, WV, kNext>(p, vpt, stream);
    }
}

template <int NW, bool F32, bool WV>
cudaError_t launch_team(const AdalnParams& p, int team, cudaStream_t stream)
{
    const int vpt = (p.hidden / (2 * NW) + team * kWarp - 1) / (team * kWarp);
    switch (team) {
    case 1: return launch_vpt<NW, 1, F32, WV>(p, vpt, stream);
    case 2: return launch_vpt<NW, 2, F32, WV>(p, vpt, stream);
    case 4: return launch_vpt<NW, 4, F32, WV>(p, vpt, stream);
    case 8: return launch_vpt<NW, 8, F32, WV>(p, vpt, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_adaln_shape(const AdalnParams& p, const AdalnShape& sh, cudaStream_t stream)
{
    if (p.mod_f32) {
        if (sh.row_words == 4)
            return sh.wide_vectors ? launch_team<4, true, true>(p, sh.team, stream)
                                   : launch_team<4, true, false>(p, sh.team, stream);
        if (sh.row_words == 2 && !sh.wide_vectors)
            return launch_team<2, true, false>(p, sh.team, stream);
        return cudaErrorInvalidValue;
    }
    if (sh.row_words == 8)
        return sh.wide_vectors ? launch_team<8, false, true>(p, sh.team, stream)
                               : launch_team<8, false, false>(p, sh.team, stream);
    if (sh.row_words == 4 && !sh.wide_vectors)
        return launch_team<4, false, false>(p, sh.team, stream);
    return cudaErrorInvalidValue;
}

AdalnShape adaln_shape(const AdalnParams& p)
{
    AdalnShape sh{};
    const bool rows32 = aligned32(p.x) && aligned32(p.out) && p.hidden % 16 == 0 && p.x_row_stride % 16 == 0 &&
                        p.out_row_stride % 16 == 0;
    // 32-byte vector reads need every sequence's vectors on a 32-byte boundary
    const bool vec32 = aligned32(p.shift) && aligned32(p.scale) && p.mod_seq_stride % (p.mod_f32 ? 8 : 16) == 0;
    if (p.mod_f32) {
        // fp32 vectors: a lane's share of each vector must be contiguous across
        // the warp (16-byte row accesses with 32-byte vector reads, else 8-byte
        // row accesses with 16-byte vector reads)
        sh.row_words = vec32 ? 4 : 2;
        sh.wide_vectors = vec32;
    } else {
        sh.row_words = rows32 ? 8 : 4;
        sh.wide_vectors = rows32 && vec32;
    }
    // one warp per row up to 8 vectors per lane, else the smallest team of
    // 2, 4 or 8 warps holding the row in at most 8 (8-byte accesses cannot
    // hold rows beyond 8192 elements that way: those take 16-byte ones)
    auto fit = [&](int words) {
        const int nvec = p.hidden / (2 * words);
        int team = 1;
        while (team < 8 && (nvec + team * kWarp - 1) / (team * kWarp) > 8)
            team *= 2;
        return (nvec + team * kWarp - 1) / (team * kWarp) <= 8 ? team : 0;
    };
    sh.team = fit(sh.row_words);
    if (sh.team == 0) {
        sh.row_words = 4;
        sh.wide_vectors = false;
        sh.team = fit(4);
    }
    // A warp holding 6-8 vectors of 32 bytes per lane (rows of 3072-4096
    // elements) runs at 82-98 registers, so 16-20 warps fit on an SM; a team
    // of 2 holds 3-4 each at 54-63 registers, 32-36 warps.  Measured per call
    // in a chain of launches (clean L2 before the chain, 1965 MHz), the team
    // is 8-13 % faster at 4-8 K rows, 2-5 % at 16-32 K and about 1 % at 61,888
    // (3072) or 65,536 (4096) rows, and 1.2 % slower at 131,072 rows of 3072.
    // At 4-5 vectors (2048-2560) the team was behind at every row count but
    // one (8 K rows of 2048: 2 % ahead), so those keep one warp per row.
    if (sh.team == 1 && sh.row_words == 8 && p.pk.num_rows_padded <= 65536) {
        const int nvec = p.hidden / 16;
        if ((nvec + kWarp - 1) / kWarp >= 6)
            sh.team = 2;
    }
    return sh;
}

cudaError_t launch_adaln_modulate(const AdalnParams& p, cudaStream_t stream)
{
    return launch_adaln_shape(p, adaln_shape(p), stream);
}

}  // namespace dit
