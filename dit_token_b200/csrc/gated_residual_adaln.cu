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
// Layout: one short-lived CTA per row, a team of TEAM warps (1-8) that keeps
// the rounded residual in registers (VPT vectors of NW words per lane);
// one-pass moments per warp, merged across the team through shared memory
// behind one barrier; packed fp32 pairs for the arithmetic.  gate, shift and
// scale are bf16, or all three fp32.  The access width per lane and the team
// size come from a sweep over both (batched varlen, hidden 5120, L2 clean,
// the B200's measured copy bandwidth 6458 GB/s):
//  * bf16 vectors: 32-byte accesses, the smallest team that holds the row in
//    at most 3 vectors per lane (5120: 4 warps, 3072 and 2048: 2 warps):
//    424.9 us (104 %), against 456.7 us for the earlier kernel (16-byte
//    accesses, 2-4 rows per 8-warp CTA); 61,888 rows of 3072: 227.4 against
//    235.5 us;
//  * fp32 vectors: a lane's share of each fp32 vector is contiguous only
//    with 8- or 16-byte activation accesses (with 32-byte ones each warp
//    load instruction spans 2 KB of the vector: 56-66 %); 16-byte ones with
//    the vectors read 32 bytes at a time: 456.7 us (97 %).
// A persistent form (each team a fixed run of rows, the vectors staged once
// per CTA in shared memory as fp32) measured slower: 569 against 455 us on
// batched varlen, 322 against 234 us on 61,888 rows of 3072, and 591 against
// 527 us with fp32 vectors.
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

// A group of NG pairs of a per-sequence vector: 32-byte reads (WV: 8 bf16 or
// 4 fp32 pairs) or 8/16-byte ones.
template <bool F32, int NG, bool WV>
__device__ __forceinline__ void seq_pairs(const void* base, int64_t elem, f32x2 (&v)[NG])
{
    if constexpr (WV)
        vec_pairs_wide<F32, NG>(base, elem, v);
    else
        vec_pairs<F32, NG>(base, elem, v);
}

template <int VPT, int NW, int TEAM, bool F32, bool WV = false>
__global__ void __launch_bounds__(TEAM * kWarp)
gated_residual_adaln_kernel(const FusedParams p)
{
    constexpr int EPV = 2 * NW;                  // elements per vector
    // words per group of per-sequence vector reads
    constexpr int NG = WV ? (F32 ? 4 : 8) : (NW < 4 ? NW : 4);
    static_assert(NG <= NW, "a vector read covers at most one row vector");
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
    const int nvec = p.hidden / EPV;

    // residual update, rounded once, kept packed
    uint32_t rv[VPT][NW];
    {
        uint32_t xv[VPT][NW], yv[VPT][NW];
        const uint16_t* xr = p.x + (int64_t)s.row * p.x_row_stride;
        const uint16_t* yr = p.y + (int64_t)s.row * p.y_row_stride;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int j = i * kTeamThreads + tt;
            if (j < nvec) {
                ld_stream_words<NW>(xr + EPV * j, xv[i]);
                ld_stream_words<NW>(yr + EPV * j, yv[i]);
            } else {
#pragma unroll
                for (int e = 0; e < NW; ++e)
                    xv[i][e] = yv[i][e] = 0u;
            }
        }
        const int64_t goff = (int64_t)s.seq * p.gate_seq_stride;
        uint16_t* res = p.res_out + (int64_t)s.row * p.res_row_stride;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int j = i * kTeamThreads + tt;
            if (j < nvec) {
#pragma unroll
                for (int h = 0; h < NW / NG; ++h) {
                    f32x2 g[NG];
                    seq_pairs<F32, NG, WV>(p.gate, goff + EPV * j + 2 * NG * h, g);
#pragma unroll
                    for (int e = 0; e < NG; ++e)
                        rv[i][NG * h + e] = f2_to_bf16x2(
                            f2_fma(g[e], f2_from_bf16x2(yv[i][NG * h + e]), f2_from_bf16x2(xv[i][NG * h + e])));
                }
                st_stream_words<NW>(res + EPV * j, rv[i]);
            } else {
#pragma unroll
                for (int e = 0; e < NW; ++e)
                    rv[i][e] = 0u;
            }
        }
    }

    // LN statistics of the stored residual (as adaLN's)
    const Moments m = row_moments<VPT, NW, TEAM>(rv, nvec, red, red2, far_w);
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
            uint32_t o[NW];
#pragma unroll
            for (int h = 0; h < NW / NG; ++h) {
                f32x2 hv[NG], cv[NG];
                seq_pairs<F32, NG, WV>(p.shift, moff + EPV * j + 2 * NG * h, hv);
                seq_pairs<F32, NG, WV>(p.scale, moff + EPV * j + 2 * NG * h, cv);
#pragma unroll
                for (int e = 0; e < NG; ++e) {
                    const f32x2 t = f2_fma(f2_from_bf16x2(rv[i][NG * h + e]), r2, b2);
                    o[NG * h + e] = f2_to_bf16x2(f2_fma(t, f2_add(cv[e], one2), hv[e]));
                }
            }
            st_stream_words<NW>(nrow + EPV * j, o);
        }
    }
}

template <int VPT, int NW, int TEAM, bool F32, bool WV>
cudaError_t launch_one(const FusedParams& p, cudaStream_t stream)
{
    const unsigned grid = (unsigned)p.pk.num_rows_padded;  // one row per CTA
    return launch_kernel(gated_residual_adaln_kernel<VPT, NW, TEAM, F32, WV>, grid, TEAM * kWarp, 0, stream, p);
}

// VPT (1..MAXV) as a template argument.
template <int NW, int TEAM, bool F32, bool WV, int MAXV, int V = 1>
cudaError_t launch_vpt(const FusedParams& p, int vpt, cudaStream_t stream)
{
    if constexpr (V > MAXV) {
        return cudaErrorInvalidValue;
    } else {
        if (vpt == V)
            return launch_one<V, NW, TEAM, F32, WV>(p, stream);
        return launch_vpt<NW, TEAM, F32, WV, MAXV, V + 1>(p, vpt, stream);
    }
}

// The smallest team of 1, 2, 4 or 8 warps that holds the row in at most
// MAXV vectors of NW words per lane (the widest rows: 8 warps, up to 8
// vectors).
template <int NW, bool F32, int MAXV, bool WV = false>
cudaError_t launch_width(const FusedParams& p, cudaStream_t stream)
{
    const int nvec = p.hidden / (2 * NW);
    auto vpt_for = [&](int team) { return (nvec + team * kWarp - 1) / (team * kWarp); };
    if (vpt_for(1) <= MAXV)
        return launch_vpt<NW, 1, F32, WV, MAXV>(p, vpt_for(1), stream);
    if (vpt_for(2) <= MAXV)
        return launch_vpt<NW, 2, F32, WV, MAXV>(p, vpt_for(2), stream);
    if (vpt_for(4) <= MAXV)
        return launch_vpt<NW, 4, F32, WV, MAXV>(p, vpt_for(4), stream);
    return launch_vpt<NW, 8, F32, WV, 8>(p, vpt_for(8), stream);
}

}  // namespace

// Access width: bf16 vectors take 32-byte accesses when all four row buffers
// are 32-byte aligned and hidden and every row stride are multiples of 16
// elements (each row then starts on a 32-byte boundary), else 16-byte ones;
// fp32 vectors take 16-byte accesses (teams of at most 5 vectors per lane),
// with the vectors read 32 bytes per lane at a time when every sequence's
// vectors start on a 32-byte boundary (batched varlen 501.7 -> 456.7 us,
// long video 255.9 -> 244.8 us: each warp load instruction then covers
// contiguous memory).
cudaError_t launch_gated_residual_adaln(const FusedParams& p, cudaStream_t stream)
{
    if (p.mod_f32) {
        const bool vec32 = aligned32(p.gate) && aligned32(p.shift) && aligned32(p.scale) &&
                           p.gate_seq_stride % 8 == 0 && p.mod_seq_stride % 8 == 0;
        return vec32 ? launch_width<4, true, 5, true>(p, stream) : launch_width<4, true, 5>(p, stream);
    }
    const bool wide = aligned32(p.x) && aligned32(p.y) && aligned32(p.res_out) && aligned32(p.norm_out) &&
                      p.hidden % 16 == 0 && p.x_row_stride % 16 == 0 && p.y_row_stride % 16 == 0 &&
                      p.res_row_stride % 16 == 0 && p.norm_row_stride % 16 == 0;
    return wide ? launch_width<8, false, 3>(p, stream) : launch_width<4, false, 5>(p, stream);
}

}  // namespace dit
