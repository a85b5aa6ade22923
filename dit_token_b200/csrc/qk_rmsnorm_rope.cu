// qk_rmsnorm_rope.cu -- per-head RMSNorm of q and k fused with rotary position
// embedding, in place, over the valid rows of a packed sequence ("Why
// Real-Time MiniMax H3 Serving Requires More Than a Faster DiT", "Key
// takeaways", bullet 2: the Q/K normalization is fused with the rotary
// embedding; bullet 1: rotary rows are computed only where needed).
//
// Layout.  One warp per valid row.  A head of D = 8*LPH elements (D = 64,
// 128 or 256) is held by a group of LPH lanes, 8 elements (one 16-byte vector)
// per lane, so the per-head sum of squares is a log2(LPH)-step xor-shuffle
// reduction.  A lane always sits at the same offset inside a head, so it
// needs the cos/sin of only its own pairs (4 interleaved, 8 half-split): it
// computes them once per row (angle reduced in fp64, then sincosf) and reuses
// them for all num_q_heads + num_k_heads heads of that row -- cos/sin are
// never re-read or recomputed per head.  Each step issues U head vectors per lane before any
// arithmetic.  HBM traffic: q and k are each read once and written once, 4
// bytes per element.
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

#ifndef DIT_QK_UNROLL
#define DIT_QK_UNROLL 4
#endif
constexpr int kUnroll = DIT_QK_UNROLL;  // head vectors per lane in flight

// angle mod 2*pi in fp64, then single precision: keeps the angle exact to
// ~1e-7 rad for any position, and lets sincosf take its short path.
__device__ __forceinline__ void pair_cos_sin(double angle, float& c, float& s)
{
    constexpr double kTwoPi = 6.283185307179586476925286766559;
    constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
    const double red = angle - kTwoPi * rint(angle * kInvTwoPi);
    sincosf((float)red, &s, &c);
}

// Rotary layouts (template MODE): pair j of a head is (2j, 2j+1) when
// interleaved -- all four of a lane's pairs are inside its own 8 elements --
// or (j, j + D/2) when half-split -- a lane then holds one side of 8 pairs and
// the lane LPH/2 away holds the other side, fetched with one xor shuffle per
// element.  MODE none applies the RMSNorm and the weight only.
//
// Interleaved (the common case) folds the weight into the rotation: per lane
// and per pair the four coefficients w0 cos, -w1 sin, w0 sin, w1 cos are formed
// once per row (for q and for k), so a pair costs 2 multiplies and 2 FMAs plus
// the RMS scale: (o0, o1) = r * (x0 w0 c - x1 w1 s, x0 w0 s + x1 w1 c).

struct PairCoef {
    float c00[4], c01[4], c10[4], c11[4];  // o0 = x0 c00 + x1 c01; o1 = x0 c10 + x1 c11
};

template <int D, int MODE, int NP>
__device__ __forceinline__ void rms_rotate_heads(uint16_t* base, int H, int sub, float eps, const float (&w)[8],
                                                 const PairCoef& pc, const float (&cs)[NP], const float (&sn)[NP],
                                                 bool upper)
{
    constexpr int LPH = D / 8;
    constexpr int HPW = kWarp / LPH;
    const float inv_d = 1.0f / (float)D;
    for (int h0 = 0; h0 < H; h0 += HPW * kUnroll) {
        uint4 xv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int h = h0 + u * HPW + sub;
            xv[u] = h < H ? ld_stream(base + (int64_t)h * D) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int h = h0 + u * HPW + sub;
            const uint32_t wd[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
            f32x2 ss2 = f2_make(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const f32x2 xx = f2_from_bf16x2(wd[e]);
                ss2 = f2_fma(xx, xx, ss2);
            }
            const float ss = group_sum<LPH>(ss2.x + ss2.y);  // every lane of the warp takes part
            const float r = rsqrtf(ss * inv_d + eps);
            float o[8];
            if (MODE == kRopeInterleaved) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float x0 = bf16_lo(wd[e]), x1 = bf16_hi(wd[e]);
                    o[2 * e] = r * fmaf(x1, pc.c01[e], x0 * pc.c00[e]);
                    o[2 * e + 1] = r * fmaf(x1, pc.c11[e], x0 * pc.c10[e]);
                }
            } else {
                float y[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    y[2 * e] = bf16_lo(wd[e]) * (r * w[2 * e]);
                    y[2 * e + 1] = bf16_hi(wd[e]) * (r * w[2 * e + 1]);
                }
                if (MODE == kRopeHalf) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float partner = __shfl_xor_sync(0xffffffffu, y[e], LPH / 2);  // all lanes take part
                        o[e] = upper ? partner * sn[e % NP] + y[e] * cs[e % NP]
                                     : y[e] * cs[e % NP] - partner * sn[e % NP];
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        o[e] = y[e];
                }
            }
            if (h < H)
                st_stream(base + (int64_t)h * D, pack8(o));
        }
    }
}

template <int D, int MODE>
__global__ void __launch_bounds__(kCtaThreads)
qk_rmsnorm_rope_kernel(const __grid_constant__ QkParams p)  // read in place: the tables are indexed per lane
{
    constexpr int LPH = D / 8;          // lanes per head
    constexpr int NP = MODE == kRopeHalf ? 8 : (MODE == kRopeInterleaved ? 4 : 1);  // pairs per lane
    const int lane = threadIdx.x & (kWarp - 1);
    const int v = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    RowSlot s;
    if (!map_valid_row(v, p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs,
                       p.pk.num_rows_padded, lane, s))
        return;
    const int sub = lane / LPH;  // which head of the step
    const int li = lane % LPH;   // position inside the head: elements 8*li .. 8*li+7
    const bool upper = MODE == kRopeHalf && li >= LPH / 2;  // holds the j + D/2 side

    float cs[NP], sn[NP];
#pragma unroll
    for (int e = 0; e < NP; ++e) {
        cs[e] = 1.f;
        sn[e] = 0.f;
    }
    if (MODE != kRopeNone) {
        // Positions of this row: a row inside the sequence's T x H x W video
        // grid (t-major, then h, then w) is 3D; every later row is 1D, counted
        // from the end of the grid.  Without a grid every row is 1D.
        bool is3d = false;
        long long pt = 0, ph = 0, pw = 0;
        long long pos1 = s.local;
        if (p.rope_grid != nullptr) {
            const long long T = __ldg(p.rope_grid + 3 * s.seq);
            const long long H = __ldg(p.rope_grid + 3 * s.seq + 1);
            const long long W = __ldg(p.rope_grid + 3 * s.seq + 2);
            const long long thw = T * H * W;
            if (s.local < thw) {
                is3d = true;
                pt = s.local / (H * W);
                ph = (s.local / W) % H;
                pw = s.local % W;
            } else {
                pos1 = s.local - thw;
            }
        }
#pragma unroll
        for (int e = 0; e < NP; ++e) {
            const int j = MODE == kRopeHalf ? 8 * (li % (LPH / 2)) + e : 4 * li + e;
            const int ax = p.axis[j];
            const long long pj = is3d ? (ax == 0 ? pt : (ax == 1 ? ph : pw)) : pos1;
            const double ang = (double)pj * (is3d ? p.inv_freq_3d[j] : p.inv_freq_1d[j]);
            pair_cos_sin(ang, cs[e], sn[e]);
        }
    }
    float wq[8], wk[8];
    unpack8(ld_shared_vec(p.q_weight + 8 * li), wq);
    unpack8(ld_shared_vec(p.k_weight + 8 * li), wk);
    PairCoef pq{}, pk{};
    if (MODE == kRopeInterleaved) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float c = cs[e % NP], sv = sn[e % NP];
            pq.c00[e] = wq[2 * e] * c;
            pq.c01[e] = -wq[2 * e + 1] * sv;
            pq.c10[e] = wq[2 * e] * sv;
            pq.c11[e] = wq[2 * e + 1] * c;
            pk.c00[e] = wk[2 * e] * c;
            pk.c01[e] = -wk[2 * e + 1] * sv;
            pk.c10[e] = wk[2 * e] * sv;
            pk.c11[e] = wk[2 * e + 1] * c;
        }
    }
    uint16_t* qrow = p.q + (int64_t)s.row * p.q_row_stride + 8 * li;
    uint16_t* krow = p.k + (int64_t)s.row * p.k_row_stride + 8 * li;
    rms_rotate_heads<D, MODE, NP>(qrow, p.num_q_heads, sub, p.eps, wq, pq, cs, sn, upper);
    rms_rotate_heads<D, MODE, NP>(krow, p.num_k_heads, sub, p.eps, wk, pk, cs, sn, upper);
}

template <int D>
cudaError_t launch_d(const QkParams& p, int mode, unsigned grid, cudaStream_t stream)
{
    switch (mode) {
    case kRopeInterleaved: qk_rmsnorm_rope_kernel<D, kRopeInterleaved><<<grid, kCtaThreads, 0, stream>>>(p); break;
    case kRopeHalf: qk_rmsnorm_rope_kernel<D, kRopeHalf><<<grid, kCtaThreads, 0, stream>>>(p); break;
    case kRopeNone: qk_rmsnorm_rope_kernel<D, kRopeNone><<<grid, kCtaThreads, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qk_rmsnorm_rope(const QkParams& p, int head_dim, int rope_mode, cudaStream_t stream)
{
    const unsigned grid = (unsigned)((p.pk.num_rows_padded + kWarpsPerCta - 1) / kWarpsPerCta);
    switch (head_dim) {
    case 64: return launch_d<64>(p, rope_mode, grid, stream);
    case 128: return launch_d<128>(p, rope_mode, grid, stream);
    case 256: return launch_d<256>(p, rope_mode, grid, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace dit
