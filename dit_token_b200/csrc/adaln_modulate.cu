// adaln_modulate.cu -- out = LN(x) * (1 + scale_b) + shift_b over the valid rows
// of a packed sequence ("Why Real-Time MiniMax H3 Serving Requires More Than a
// Faster DiT", "Key takeaways", bullet 2: the adaptive normalization and its
// modulation are one of the fused operators).  LN has no affine; the variance
// is the biased one.
//
// Why this shape.  With only 4 bytes of HBM traffic per element, this op is
// paced by instruction issue, not by HBM, unless every per-row and
// per-element cost is cut (ncu on a team-per-row kernel: 20.6 thread
// instructions per element, 70 % of issue slots busy, 48 % of DRAM peak; the
// per-row costs -- finding the row, merging statistics across warps -- were
// ~450 instructions per warp-row).  So, for rows of up to 6144 elements:
//  * one warp owns a whole row (VPT 16-byte vectors per lane, x read from HBM
//    once and kept in registers); no cross-warp merge, no barrier per row;
//  * persistent CTAs of 8 warps, each warp walking a contiguous run of valid
//    rows: the row mapping advances incrementally instead of being searched;
//  * the modulation of the (at most two) sequences a CTA touches is staged
//    once in shared memory as fp32 A = 1 + scale and B = shift, so the output
//    pass is (x * rstd - mean * rstd) * A + B with packed fp32 FMAs and no
//    per-row unpacking of the vectors (rows of any third sequence read them
//    from global memory instead);
//  * statistics in one pass (per-lane shifted sums merged as count/mean/M2
//    moments by warp shuffles), arithmetic on packed fp32 pairs.
// Wider rows (up to 16384) use a team of 2-8 warps per row with the same
// statistics and a named barrier per team.  HBM traffic: 4 bytes per element.
//
// Measured alternatives (batched varlen, hidden 5120, 1.43 GB per launch):
// team of 4 warps per row 299 us; 2 warps 263 us; CTA-wide smem ring fed by
// cp.async 370-450 us; persistent 4-warp CTAs with 3 rows prefetched in
// registers 352 us; the row streamed twice (second read from L2) 339 us;
// one warp per row with the next row prefetched into shared memory by
// cp.async (modulation then from global) 316 us; one warp per row fed by 1-D
// bulk copies (TMA) into a 2-slot shared-memory ring per warp with mbarrier
// completion, 8 warps and 205 KB of shared memory per SM, 523 us (ncu: 26 %
// of DRAM peak, SM activity very uneven -- active cycles min / mean / max
// 2k / 132k / 203k of 210k -- with the copy engine's pipe nearly idle); this
// kernel with each register vector refilled with the next row's during the
// output pass 248 us against 244 us without (both with a clean L2); the
// next row (or the one after) pulled into L2 by a 1-D bulk prefetch
// (cp.async.bulk.prefetch.L2) issued by one lane per row 260 / 303 us against
// 242 us; this kernel 242-264 us.
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

constexpr int kMaxWarpVpt = 24;    // widest row a single warp holds: 24 * 256 = 6144 elements
constexpr int kSmemBudget = 104 * 1024;

// Statistics of the VPT vectors a lane holds (vectors past nvec are empty),
// merged over the warp.  Vector i of the lane is vector i * STRIDE + lane_vec0
// of the row.
template <int VPT, int STRIDE>
__device__ __forceinline__ Moments lane_row_moments(const uint4 (&xv)[VPT], int lane_vec0, int nvec)
{
    const float k = bf16_lo(xv[0].x);
    const f32x2 kk = f2_make(k, k);
    f32x2 s2 = f2_make(0.f, 0.f), q2 = f2_make(0.f, 0.f);
    float cnt = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        if (i * STRIDE + lane_vec0 < nvec) {
            const uint32_t w[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const f32x2 d = f2_sub(f2_from_bf16x2(w[e]), kk);
                s2 = f2_add(s2, d);
                q2 = f2_fma(d, d, q2);
            }
            cnt += 8.f;
        }
    }
    return moments_warp(moments_from_sums(cnt, k, s2.x + s2.y, q2.x + q2.y));
}

// One output vector: (x * rstd + nb) * A + B for the 8 elements of x.
__device__ __forceinline__ uint4 modulate8(uint4 x, f32x2 r2, f32x2 b2, const f32x2 (&A)[4], const f32x2 (&B)[4])
{
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
        o[e] = f2_to_bf16x2(f2_fma(f2_fma(f2_from_bf16x2(w[e]), r2, b2), A[e], B[e]));
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// A = 1 + scale and B = shift of the 8 elements at element `elem` of a
// sequence's vectors, from global memory (bf16 or fp32).
template <bool F32>
__device__ __forceinline__ void mod_from_global(const void* shift, const void* scale, int64_t elem, f32x2 (&A)[4],
                                                f32x2 (&B)[4])
{
    vec8_pairs<F32>(scale, elem, A);
    vec8_pairs<F32>(shift, elem, B);
    const f32x2 one2 = f2_make(1.f, 1.f);
#pragma unroll
    for (int e = 0; e < 4; ++e)
        A[e] = f2_add(A[e], one2);
}

// ------------------------------------------------------------ warp per row

template <int VPT, bool F32>
__global__ void __launch_bounds__(kCtaThreads)
adaln_warp_kernel(const AdalnParams p, int slots)
{
    extern __shared__ __align__(16) float mod_smem[];  // [slots][2][hidden]: A, then B
    const int nvec = p.hidden / 8;
    const int C = p.hidden;
    const int tid = threadIdx.x;
    const int lane = tid & (kWarp - 1), warp = tid >> 5;

    // this CTA's contiguous run of valid-row ordinals, then this warp's share
    const int total = min(max(__ldg(p.pk.cu_seqlens + p.pk.num_seqs), 0), p.pk.num_rows_padded);
    const int per = (total + (int)gridDim.x - 1) / (int)gridDim.x;
    const int c0 = min(total, (int)blockIdx.x * per);
    const int c1 = min(total, c0 + per);
    if (c1 <= c0)
        return;  // uniform over the CTA

    // stage the modulation of the first and the last sequence of the run
    int staged[2] = {-1, -1};
    {
        const int b0 = find_seq(c0, p.pk.cu_seqlens, p.pk.num_seqs, lane);
        const int b1 = find_seq(c1 - 1, p.pk.cu_seqlens, p.pk.num_seqs, lane);
        staged[0] = slots > 0 ? b0 : -1;
        staged[1] = (slots > 1 && b1 != b0) ? b1 : -1;
#pragma unroll
        for (int sidx = 0; sidx < 2; ++sidx) {
            const int b = staged[sidx];
            if (b < 0)
                continue;  // uniform
            float* A = mod_smem + (size_t)sidx * 2 * C;
            float* B = A + C;
            const int64_t moff = (int64_t)b * p.mod_seq_stride;
            for (int j = tid; j < nvec; j += kCtaThreads) {
                f32x2 a[4], bb[4];
                mod_from_global<F32>(p.shift, p.scale, moff + 8 * j, a, bb);
                float4* A4 = reinterpret_cast<float4*>(A + 8 * j);
                float4* B4 = reinterpret_cast<float4*>(B + 8 * j);
                A4[0] = make_float4(a[0].x, a[0].y, a[1].x, a[1].y);
                A4[1] = make_float4(a[2].x, a[2].y, a[3].x, a[3].y);
                B4[0] = make_float4(bb[0].x, bb[0].y, bb[1].x, bb[1].y);
                B4[1] = make_float4(bb[2].x, bb[2].y, bb[3].x, bb[3].y);
            }
        }
        __syncthreads();
    }

    const int wper = (c1 - c0 + kWarpsPerCta - 1) / kWarpsPerCta;
    const int w0 = min(c1, c0 + warp * wper);
    const int w1 = min(c1, w0 + wper);
    if (w1 <= w0)
        return;  // no barrier follows
    RowCursor cur{p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs, p.pk.num_rows_padded};
    {
        const int b = find_seq(w0, p.pk.cu_seqlens, p.pk.num_seqs, lane);
        cur.load(b < 0 ? 0 : b);
    }
    const float inv_n = 1.0f / (float)C;

    for (int v = w0; v < w1; ++v) {
        const int row = cur.row(v);
        if (row < 0)
            continue;  // uniform over the warp
        const int seq = cur.b;
        const uint16_t* xr = p.x + (int64_t)row * p.x_row_stride + 8 * lane;
        uint4 xv[VPT];
#pragma unroll
        for (int i = 0; i < VPT; ++i)
            xv[i] = i * kWarp + lane < nvec ? ld_stream(xr + 8 * kWarp * i) : make_uint4(0u, 0u, 0u, 0u);

        const Moments m = lane_row_moments<VPT, kWarp>(xv, lane, nvec);
        const float rstd = rsqrtf(m.m2 * inv_n + p.eps);
        const f32x2 r2 = f2_make(rstd, rstd);
        const float nb = -m.mean * rstd;
        const f32x2 b2 = f2_make(nb, nb);

        uint16_t* orow = p.out + (int64_t)row * p.out_row_stride + 8 * lane;
        const int sidx = seq == staged[0] ? 0 : (seq == staged[1] ? 1 : -1);
        if (sidx >= 0) {
            const float* A = mod_smem + (size_t)sidx * 2 * C + 8 * lane;
            const float* B = A + C;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                if (i * kWarp + lane < nvec) {
                    const float4* A4 = reinterpret_cast<const float4*>(A + 8 * kWarp * i);
                    const float4* B4 = reinterpret_cast<const float4*>(B + 8 * kWarp * i);
                    const float4 a0 = A4[0], a1 = A4[1], q0 = B4[0], q1 = B4[1];
                    const f32x2 Av[4] = {f2_make(a0.x, a0.y), f2_make(a0.z, a0.w), f2_make(a1.x, a1.y),
                                         f2_make(a1.z, a1.w)};
                    const f32x2 Bv[4] = {f2_make(q0.x, q0.y), f2_make(q0.z, q0.w), f2_make(q1.x, q1.y),
                                         f2_make(q1.z, q1.w)};
                    st_stream(orow + 8 * kWarp * i, modulate8(xv[i], r2, b2, Av, Bv));
                }
            }
        } else {
            const int64_t moff = (int64_t)seq * p.mod_seq_stride;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int j = i * kWarp + lane;
                if (j < nvec) {
                    f32x2 Av[4], Bv[4];
                    mod_from_global<F32>(p.shift, p.scale, moff + 8 * j, Av, Bv);
                    st_stream(orow + 8 * kWarp * i, modulate8(xv[i], r2, b2, Av, Bv));
                }
            }
        }
    }
}

template <int VPT, bool F32>
cudaError_t launch_warp_t(const AdalnParams& p, cudaStream_t stream)
{
    const size_t slot_bytes = (size_t)2 * p.hidden * sizeof(float);
    const int slots = 2 * slot_bytes <= (size_t)kSmemBudget ? 2 : (slot_bytes <= (size_t)kSmemBudget ? 1 : 0);
    const size_t smem = slots * slot_bytes;
    cudaError_t e;
    if (smem > 48 * 1024 &&
        (e = cudaFuncSetAttribute(adaln_warp_kernel<VPT, F32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)) != cudaSuccess)
        return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, adaln_warp_kernel<VPT, F32>, kCtaThreads,
                                                           smem)) != cudaSuccess)
        return e;
    const long long want = (long long)sms * (per_sm > 0 ? per_sm : 1);
    const long long rows_cap = (p.pk.num_rows_padded + kWarpsPerCta - 1) / kWarpsPerCta;
    const unsigned grid = (unsigned)(want < rows_cap ? want : rows_cap);
    adaln_warp_kernel<VPT, F32><<<grid, kCtaThreads, smem, stream>>>(p, slots);
    return cudaGetLastError();
}

template <int VPT>
cudaError_t launch_warp(const AdalnParams& p, cudaStream_t stream)
{
    return p.mod_f32 ? launch_warp_t<VPT, true>(p, stream) : launch_warp_t<VPT, false>(p, stream);
}

// ------------------------------------------------------------ team per row

template <int VPT, int TEAM, bool F32>
__global__ void __launch_bounds__(kCtaThreads, MinCtas<VPT>::value)
adaln_team_kernel(const AdalnParams p)
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
    if (!map_valid_row(v, p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs, p.pk.num_rows_padded, lane, s))
        return;  // the whole team leaves: its barrier involves only its own warps
    const int nvec = p.hidden / 8;
    const uint16_t* xr = p.x + (int64_t)s.row * p.x_row_stride;
    uint4 xv[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = i * kTeamThreads + tt;
        xv[i] = j < nvec ? ld_stream(xr + 8 * j) : make_uint4(0u, 0u, 0u, 0u);
    }
    Moments m = lane_row_moments<VPT, kTeamThreads>(xv, tt, nvec);
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
            f32x2 Av[4], Bv[4];
            mod_from_global<F32>(p.shift, p.scale, moff + 8 * j, Av, Bv);
            st_stream(orow + 8 * j, modulate8(xv[i], r2, b2, Av, Bv));
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
        if (p.mod_f32)                                                                                       \
            adaln_team_kernel<V, TEAM, true><<<grid, kCtaThreads, 0, stream>>>(p);                           \
        else                                                                                                 \
            adaln_team_kernel<V, TEAM, false><<<grid, kCtaThreads, 0, stream>>>(p);                          \
        break;
    switch (vpt) {
        DIT_TEAM_CASE(4)
        DIT_TEAM_CASE(5)
        DIT_TEAM_CASE(6)
        DIT_TEAM_CASE(7)
        DIT_TEAM_CASE(8)
    default: return cudaErrorInvalidValue;
    }
#undef DIT_TEAM_CASE
    return cudaGetLastError();
}

}  // namespace

// Rows of up to 6144 elements: one warp per row, VPT = ceil(hidden / 256)
// vectors per lane rounded up to an instantiated count.  Wider rows (to
// 16384): the smallest team of 2, 4 or 8 warps that holds the row in at most
// 8 vectors per lane.
cudaError_t launch_adaln_modulate(const AdalnParams& p, cudaStream_t stream)
{
    const int nvec = p.hidden / 8;
    const int vpt = (nvec + kWarp - 1) / kWarp;
    // Rows of 2304-3072 elements with bf16 vectors: two warps per row measured
    // faster than one (hidden 3072: 61,888 rows 129.2 against 135.4 us, 16,256
    // rows 41.0 against 42.3 us); with fp32 vectors, and at other widths
    // (2048: 22.6 against 21.5 us; 5120: 268.9 against 243.9 us), slower.
    if (!p.mod_f32 && vpt > 8 && vpt <= 12)
        return launch_team<2>(p, stream);
    if (vpt <= kMaxWarpVpt) {
        switch (vpt) {
        case 1: return launch_warp<1>(p, stream);
        case 2: return launch_warp<2>(p, stream);
        case 3: return launch_warp<3>(p, stream);
        case 4: return launch_warp<4>(p, stream);
        case 5: return launch_warp<5>(p, stream);
        case 6: return launch_warp<6>(p, stream);
        case 7: return launch_warp<7>(p, stream);
        case 8: return launch_warp<8>(p, stream);
        default: break;
        }
        if (vpt <= 10)
            return launch_warp<10>(p, stream);
        if (vpt <= 12)
            return launch_warp<12>(p, stream);
        if (vpt <= 16)
            return launch_warp<16>(p, stream);
        if (vpt <= 20)
            return launch_warp<20>(p, stream);
        return launch_warp<24>(p, stream);
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
