// qk_rmsnorm_rope.cu -- per-head RMSNorm of q and k fused with rotary position
// embedding, in place, over the valid rows of a packed sequence ("Why
// Real-Time MiniMax H3 Serving Requires More Than a Faster DiT", "Key
// takeaways", bullet 2: the Q/K normalization is fused with the rotary
// embedding; bullet 1: rotary rows are computed only where needed).
//
// Layout.  One warp per valid row.  A head of D = 8*LPH elements (D = 64,
// 128 or 256) is held by a group of LPH lanes, 8 elements per lane, so the
// per-head sum of squares is a log2(LPH)-step xor-shuffle reduction.  A lane
// always sits at the same place inside a head, so it needs the cos/sin of
// only its own 4 pairs: it computes them once per row (angle reduced in fp64,
// then the hardware sine and cosine) and reuses them for all num_q_heads +
// num_k_heads heads of that row -- cos/sin are never re-read or recomputed
// per head.  The heads go in batches of U steps, software-pipelined: a
// batch's loads are issued before the previous batch is computed, and the
// first batch's before the row's angles, so a warp always has loads in flight
// (measured on batched varlen, 40x128 heads: 452 -> 429 us; with 8 K heads
// 300 -> 261 us).  HBM traffic: q and k are each read once and written once,
// 4 bytes per element.
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

// Rows (warps) per CTA: 4.  Against 8, measured equal on wide rows (40 + 40
// heads of 128: 430.5 against 430.9 us) and faster on narrow ones (24 q + 4 k
// heads: 147.4 against 151.6 us).
constexpr int kQkWarps = 4;

// Steps per head batch (head vectors per lane in one batch): 4, or 2 when
// 4-step batches would leave over a quarter of their head slots empty (see
// launch_d).

// angle mod 2*pi in fp64, then single precision: keeps the angle exact to
// ~1e-7 rad for any position.  On the reduced angle, in [-pi, pi], the
// hardware sine and cosine (__sincosf, absolute error ~1e-6 there) replace
// the full-range sincosf: with 24 q + 4 k heads of 128 per row the per-row
// setup is a large share of the work (long video 143.8 -> 141.3 us), and the
// outputs move by at most one bf16 unit in ~1e-4 of the elements.
__device__ __forceinline__ void pair_cos_sin(double angle, float& c, float& s)
{
    constexpr double kTwoPi = 6.283185307179586476925286766559;
    constexpr double kInvTwoPi = 0.15915494309189533576888376337251;
    const double red = angle - kTwoPi * rint(angle * kInvTwoPi);
    __sincosf((float)red, &s, &c);
}

// b^k for 0 <= k < 128 (a pair index) by repeated squaring: the fp64 product
// stays within ~1e-14 (relative) of theta^(-2j/d), far below what the fp32
// reduced angle can resolve.
__device__ __forceinline__ double pow_index(double b, int k)
{
    double r = 1.0;
#pragma unroll
    for (int i = 0; i < 7; ++i) {
        if ((k >> i) & 1)
            r *= b;
        b *= b;
    }
    return r;
}

// Frequencies of the lane's NP pairs j = 4 li .. 4 li + NP - 1 and, on a 3D
// row, their sections: 1D base_1d^j; 3D the section's base to the pair's
// index inside the section.  The bases are read with warp-uniform indices
// only: a parameter read whose address differs across the lanes of a warp is
// served one address at a time (with 24 q + 4 k heads per row, reading
// per-pair tables that way cost 4 % of the kernel on the long video and 16 %
// on one rank's slice of it).
template <int NP>
__device__ __forceinline__ void pair_frequencies(const QkParams& p, int li, bool is3d, double (&f)[NP],
                                                 int (&ax)[NP])
{
    const int j0 = 4 * li;
    if (!is3d) {
        f[0] = pow_index(p.base_1d, j0);
#pragma unroll
        for (int e = 0; e < NP; ++e) {
            if (e > 0)
                f[e] = f[e - 1] * p.base_1d;
            ax[e] = 0;
        }
        return;
    }
    const int n0 = p.sec_pairs[0], n01 = n0 + p.sec_pairs[1];
#pragma unroll
    for (int e = 0; e < NP; ++e)
        ax[e] = j0 + e < n0 ? 0 : (j0 + e < n01 ? 1 : 2);
    auto base = [&](int sct) { return sct == 0 ? p.base_3d[0] : (sct == 1 ? p.base_3d[1] : p.base_3d[2]); };
    f[0] = pow_index(base(ax[0]), j0 - (ax[0] == 0 ? 0 : (ax[0] == 1 ? n0 : n01)));
#pragma unroll
    for (int e = 1; e < NP; ++e)  // a pair that opens a new section is its index 0
        f[e] = ax[e] == ax[e - 1] ? f[e - 1] * base(ax[e]) : 1.0;
}

// Rotary layouts (template MODE).  In both rotating layouts a lane owns the
// four pairs j = 4*li .. 4*li+3 of its head:
//   interleaved  pair j = elements (2j, 2j+1): the lane's 16-byte vector
//                 8*li .. 8*li+7 holds all four pairs;
//   half-split   pair j = elements (j, j + D/2): the lane loads two 8-byte
//                 vectors, elements 4*li .. 4*li+3 and D/2 + 4*li .. +3, so
//                 both sides of each pair are its own and no lane exchange is
//                 needed (a warp's 8-byte accesses still cover whole
//                 128-byte lines).
// Either way the weight is folded into the rotation: per lane and per pair the
// four coefficients w0 cos, -w1 sin, w0 sin, w1 cos are formed once per row
// (for q and for k), so a pair costs 2 multiplies and 2 FMAs plus the RMS
// scale: (o0, o1) = r * (x0 w0 c - x1 w1 s, x0 w0 s + x1 w1 c), where w0, w1
// are the weights of the pair's two elements.  MODE none applies the RMSNorm
// and the weight only.

struct PairCoef {
    float c00[4], c01[4], c10[4], c11[4];  // o0 = x0 c00 + x1 c01; o1 = x0 c10 + x1 c11
};

// Element offset (from the head's start) of the lane's first / second access.
template <int D, int MODE>
__device__ __forceinline__ int lane_off(int li, int part)
{
    if (MODE == kRopeHalf)
        return part * (D / 2) + 4 * li;
    return 8 * li;
}

template <int D, int MODE>
__device__ __forceinline__ uint4 load_head(const uint16_t* head, int li)
{
    if (MODE == kRopeHalf) {
        const uint2 a = __ldcs(reinterpret_cast<const uint2*>(head + lane_off<D, MODE>(li, 0)));
        const uint2 b = __ldcs(reinterpret_cast<const uint2*>(head + lane_off<D, MODE>(li, 1)));
        return make_uint4(a.x, a.y, b.x, b.y);
    }
    return ld_stream(head + lane_off<D, MODE>(li, 0));
}

template <int D, int MODE>
__device__ __forceinline__ void store_head(uint16_t* head, int li, uint4 v)
{
    if (MODE == kRopeHalf) {
        __stcs(reinterpret_cast<uint2*>(head + lane_off<D, MODE>(li, 0)), make_uint2(v.x, v.y));
        __stcs(reinterpret_cast<uint2*>(head + lane_off<D, MODE>(li, 1)), make_uint2(v.z, v.w));
        return;
    }
    st_stream(head + lane_off<D, MODE>(li, 0), v);
}

// The lane's 8 elements in register order: interleaved (and none) = the
// vector's own order; half-split = 4 elements of the first half, then the 4
// matching elements of the second half.  Pair e of the lane is
//   interleaved: registers (2e, 2e+1);  half-split: registers (e, 4+e).
template <int MODE>
__device__ __forceinline__ void pair_regs(int e, int& a, int& b)
{
    if (MODE == kRopeHalf) {
        a = e;
        b = 4 + e;
    } else {
        a = 2 * e;
        b = 2 * e + 1;
    }
}

// The heads of a row are handled in batches of U steps (HPW heads per
// step): first the q heads, then the k heads.  Batch b's loads are issued
// before batch b-1 is computed, and batch 0's before the row's angles are
// computed, so a warp always has a batch in flight.
template <int D, int U>
struct Batches {
    static constexpr int kHeads = (kWarp / (D / 8)) * U;  // heads per batch
    int nq, n;
    __device__ __forceinline__ Batches(int Hq, int Hk)
        : nq((Hq + kHeads - 1) / kHeads), n(nq + (Hk + kHeads - 1) / kHeads)
    {
    }
};

template <int D, int MODE, int U>
__device__ __forceinline__ void load_batch(const uint16_t* row, int H, int h0, int sub, int li, uint4 (&xv)[U])
{
    constexpr int HPW = kWarp / (D / 8);
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int h = h0 + u * HPW + sub;
        xv[u] = h < H ? load_head<D, MODE>(row + (int64_t)h * D, li) : make_uint4(0u, 0u, 0u, 0u);
    }
}

template <int D, int MODE, int U>
__device__ __forceinline__ void rms_rotate_batch(uint16_t* row, int H, int h0, int sub, int li, float eps,
                                                 const float (&w)[8], const PairCoef& pc, const uint4 (&xv)[U])
{
    constexpr int LPH = D / 8;
    constexpr int HPW = kWarp / LPH;
    const float inv_d = 1.0f / (float)D;
#pragma unroll
    for (int u = 0; u < U; ++u) {
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
        float x[8], o[8];
        unpack8(xv[u], x);
        if (MODE == kRopeNone) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
                o[e] = x[e] * (r * w[e]);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                int a, b;
                pair_regs<MODE>(e, a, b);
                o[a] = r * fmaf(x[b], pc.c01[e], x[a] * pc.c00[e]);
                o[b] = r * fmaf(x[b], pc.c11[e], x[a] * pc.c10[e]);
            }
        }
        if (h < H)
            store_head<D, MODE>(row + (int64_t)h * D, li, pack8(o));
    }
}

template <int D, int MODE, int U>
__global__ void __launch_bounds__(kQkWarps * kWarp)
qk_rmsnorm_rope_kernel(const __grid_constant__ QkParams p)  // read in place, never copied
{
    constexpr int LPH = D / 8;          // lanes per head
    constexpr int NP = MODE == kRopeNone ? 1 : 4;  // pairs per lane
    grid_dependency_wait();
    const int lane = threadIdx.x & (kWarp - 1);
    const int v = blockIdx.x * kQkWarps + (threadIdx.x >> 5);
    RowSlot s;
    if (!map_valid_row(v, p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs,
                       p.pk.num_rows_padded, lane, s))
        return;
    const int sub = lane / LPH;  // which head of the step
    const int li = lane % LPH;   // position inside the head: pairs 4*li .. 4*li+3
    uint16_t* qrow = p.q + (int64_t)s.row * p.q_row_stride;
    uint16_t* krow = p.k + (int64_t)s.row * p.k_row_stride;
    constexpr int kBatchHeads = Batches<D, U>::kHeads;
    const Batches<D, U> nb(p.num_q_heads, p.num_k_heads);

    // batch 0 travels while the row's angles are computed
    uint4 cur[U];
    if (nb.nq > 0)
        load_batch<D, MODE, U>(qrow, p.num_q_heads, 0, sub, li, cur);
    else
        load_batch<D, MODE, U>(krow, p.num_k_heads, 0, sub, li, cur);

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
        // g: the row's index in its whole sequence (the buffer may hold one
        // rank's slice of it, starting at row pos_offset[seq])
        // (a negative offset, outside the documented range, is read as 0, so
        // every position stays >= 0 and the grid divisions below only run for
        // a non-empty grid)
        const int off = p.pos_offset != nullptr ? max(__ldg(p.pos_offset + s.seq), 0) : 0;
        const long long g = (long long)s.local + off;
        bool is3d = false;
        long long pt = 0, ph = 0, pw = 0;
        long long pos1 = g;
        if (p.rope_grid != nullptr) {
            const long long T = __ldg(p.rope_grid + 3 * s.seq);
            const long long H = __ldg(p.rope_grid + 3 * s.seq + 1);
            const long long W = __ldg(p.rope_grid + 3 * s.seq + 2);
            const long long thw = T * H * W;
            if (g < thw) {  // g >= 0, so the grid is non-empty here
                is3d = true;
                const long long hw = H * W;
                if (hw > 0 && hw <= 0xffffffffLL) {
                    // 32-bit divisions (g < 2^32 always): the row setup is a
                    // large share of a narrow row's work (24 q + 4 k heads:
                    // 146.4 -> 144.2 us, results unchanged)
                    const unsigned gu = (unsigned)g, hwu = (unsigned)hw, wu = (unsigned)W;
                    const unsigned t = gu / hwu, rem = gu - t * hwu, h = rem / wu;
                    pt = t;
                    ph = h;
                    pw = rem - h * wu;
                } else {
                    pt = g / hw;
                    ph = (g / W) % H;
                    pw = g % W;
                }
            } else {
                pos1 = g - thw;
            }
        }
        double f[NP];
        int ax[NP];
        pair_frequencies<NP>(p, li, is3d, f, ax);
#pragma unroll
        for (int e = 0; e < NP; ++e) {
            const long long pj = is3d ? (ax[e] == 0 ? pt : (ax[e] == 1 ? ph : pw)) : pos1;
            pair_cos_sin((double)pj * f[e], cs[e], sn[e]);
        }
    }
    // the weights of the lane's 8 elements, in register order
    float wq[8], wk[8];
    if (MODE == kRopeHalf) {
        const uint2 q0 = __ldg(reinterpret_cast<const uint2*>(p.q_weight + lane_off<D, MODE>(li, 0)));
        const uint2 q1 = __ldg(reinterpret_cast<const uint2*>(p.q_weight + lane_off<D, MODE>(li, 1)));
        const uint2 k0 = __ldg(reinterpret_cast<const uint2*>(p.k_weight + lane_off<D, MODE>(li, 0)));
        const uint2 k1 = __ldg(reinterpret_cast<const uint2*>(p.k_weight + lane_off<D, MODE>(li, 1)));
        unpack8(make_uint4(q0.x, q0.y, q1.x, q1.y), wq);
        unpack8(make_uint4(k0.x, k0.y, k1.x, k1.y), wk);
    } else {
        unpack8(ld_readonly(p.q_weight + 8 * li), wq);
        unpack8(ld_readonly(p.k_weight + 8 * li), wk);
    }
    PairCoef pq{}, pk{};
    if (MODE != kRopeNone) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int a, b;
            pair_regs<MODE>(e, a, b);
            const float c = cs[e % NP], sv = sn[e % NP];
            pq.c00[e] = wq[a] * c;
            pq.c01[e] = -wq[b] * sv;
            pq.c10[e] = wq[a] * sv;
            pq.c11[e] = wq[b] * c;
            pk.c00[e] = wk[a] * c;
            pk.c01[e] = -wk[b] * sv;
            pk.c10[e] = wk[a] * sv;
            pk.c11[e] = wk[b] * c;
        }
    }
    for (int b = 0; b < nb.n; ++b) {
        uint4 nxt[U];
        const int bn = b + 1;
        if (bn < nb.nq)
            load_batch<D, MODE, U>(qrow, p.num_q_heads, bn * kBatchHeads, sub, li, nxt);
        else if (bn < nb.n)
            load_batch<D, MODE, U>(krow, p.num_k_heads, (bn - nb.nq) * kBatchHeads, sub, li, nxt);
        if (b < nb.nq)
            rms_rotate_batch<D, MODE, U>(qrow, p.num_q_heads, b * kBatchHeads, sub, li, p.eps, wq, pq, cur);
        else
            rms_rotate_batch<D, MODE, U>(krow, p.num_k_heads, (b - nb.nq) * kBatchHeads, sub, li, p.eps, wk, pk, cur);
#pragma unroll
        for (int u = 0; u < U; ++u)
            cur[u] = nxt[u];
    }
}

template <int D, int U>
cudaError_t launch_du(const QkParams& p, int mode, unsigned grid, cudaStream_t stream)
{
    switch (mode) {
    case kRopeInterleaved: return launch_kernel(qk_rmsnorm_rope_kernel<D, kRopeInterleaved, U>, grid, kQkWarps * kWarp, 0, stream, p);
    case kRopeHalf: return launch_kernel(qk_rmsnorm_rope_kernel<D, kRopeHalf, U>, grid, kQkWarps * kWarp, 0, stream, p);
    case kRopeNone: return launch_kernel(qk_rmsnorm_rope_kernel<D, kRopeNone, U>, grid, kQkWarps * kWarp, 0, stream, p);
    default: return cudaErrorInvalidValue;
    }
}

// Batch depth: 4 steps, unless 4-step batches would leave more than a quarter
// of their head slots empty and 2 fills them better -- a batch of 4 steps
// spans 4 * 32 / (D / 8) heads, and a row with, say, 8 q and 8 k heads of 64
// would leave half of each batch's lanes without a head (2 steps: 888 -> 639
// us there), while 24 q + 4 k heads of 128 fill 7/8 of 4-step batches and run
// faster with them (141.3 against 144.2 us on the long video).
template <int D>
cudaError_t launch_d(const QkParams& p, int mode, unsigned grid, cudaStream_t stream)
{
    auto slots = [&](int heads_per_batch) {
        return ((p.num_q_heads + heads_per_batch - 1) / heads_per_batch +
                (p.num_k_heads + heads_per_batch - 1) / heads_per_batch) * heads_per_batch;
    };
    constexpr int kHpw = kWarp / (D / 8);
    const int heads = p.num_q_heads + p.num_k_heads;
    const bool shallow = 4 * heads < 3 * slots(4 * kHpw) && slots(2 * kHpw) < slots(4 * kHpw);
    return shallow ? launch_du<D, 2>(p, mode, grid, stream) : launch_du<D, 4>(p, mode, grid, stream);
}

}  // namespace

cudaError_t launch_qk_rmsnorm_rope(const QkParams& p, int head_dim, int rope_mode, cudaStream_t stream)
{
    const unsigned grid = (unsigned)((p.pk.num_rows_padded + kQkWarps - 1) / kQkWarps);
    switch (head_dim) {
    case 64: return launch_d<64>(p, rope_mode, grid, stream);
    case 128: return launch_d<128>(p, rope_mode, grid, stream);
    case 256: return launch_d<256>(p, rope_mode, grid, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace dit
