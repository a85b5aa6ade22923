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
// through shared memory behind a named barrier of their own, so the teams of
// a CTA run independently.  The register budget is capped so that enough
// CTAs stay resident to keep ~10 rows of loads in flight per SM: the kernel
// is bound by bytes in flight, not by arithmetic.  HBM traffic: 4 bytes per
// element.
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

template <int VPT, int TEAM>
__global__ void __launch_bounds__(kCtaThreads, MinCtas<VPT>::value)
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
    if (!active)
        return;  // the whole team leaves: its barriers involve only its own warps
    const int nvec = p.hidden / 8;
    const uint16_t* xr = p.x + (int64_t)s.row * p.x_row_stride;

    uint4 xv[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = i * kTeamThreads + tt;
        xv[i] = j < nvec ? ld_stream(xr + 8 * j) : make_uint4(0u, 0u, 0u, 0u);
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
        team_barrier<TEAM>(team);
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
            unpack8_again(xv[i], f);
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
    uint16_t* orow = p.out + (int64_t)s.row * p.out_row_stride;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int j = i * kTeamThreads + tt;
        if (j < nvec) {
            float f[8], shf[8], scf[8], o[8];
            unpack8_again(xv[i], f);
            unpack8(ld_shared_vec(sh + 8 * j), shf);
            unpack8(ld_shared_vec(sc + 8 * j), scf);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                o[e] = fmaf((f[e] - mean) * rstd, 1.0f + scf[e], shf[e]);
            st_stream(orow + 8 * j, pack8(o));
        }
    }
}

// Pipelined variant: persistent CTAs, each owning one contiguous range of
// valid-row ordinals.  An S-stage shared-memory ring filled by cp.async keeps
// S - 1 rows per CTA in flight while the current row is reduced and written;
// the ordinal -> padded-row mapping advances incrementally (global loads only
// when a sequence boundary is crossed), and the current sequence's shift and
// scale vectors sit in shared memory.  The whole CTA works on one row: two
// block reductions (mean, then squared deviations), then the output pass.
__device__ __forceinline__ float block_sum(float v, float* red, int warp, int lane)
{
    v = group_sum<kWarp>(v);
    if (lane == 0)
        red[warp] = v;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kWarpsPerCta; ++w)
        t += red[w];
    return t;
}

// Walks valid-row ordinals upward; every thread holds the same state.
struct RowCursor {
    const int32_t* cs;
    const int32_t* cp;
    int B;
    int rows_padded;
    int b;       // current sequence
    int cs0, cs1, cp0, cp1;

    __device__ void load(int bb)
    {
        b = bb;
        cs0 = __ldg(cs + b);
        cs1 = __ldg(cs + b + 1);
        cp0 = __ldg(cp + b);
        cp1 = __ldg(cp + b + 1);
    }
    // Padded row of ordinal v (v never decreases between calls), or -1.
    __device__ int row(int v)
    {
        while (v >= cs1 && b + 1 < B)
            load(b + 1);
        const int r = v - cs0;
        if (r < 0 || r >= cs1 - cs0 || r >= cp1 - cp0)
            return -1;
        const long long rr = (long long)cp0 + r;
        return rr < rows_padded ? (int)rr : -1;
    }
};

template <int S>
__global__ void __launch_bounds__(kCtaThreads)
adaln_pipelined_kernel(const AdalnParams p)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int nvec = p.hidden / 8;
    uint4* stage = reinterpret_cast<uint4*>(smem_raw);  // [S][nvec]
    uint4* mod_sh = stage + S * nvec;                    // shift of the current sequence
    uint4* mod_sc = mod_sh + nvec;                       // scale of the current sequence
    __shared__ float red[2][kWarpsPerCta];
    __shared__ int slot_row[S];
    __shared__ int slot_seq[S];

    const int tid = threadIdx.x;
    const int lane = tid & (kWarp - 1), warp = tid >> 5;
    const int total = min(max(__ldg(p.pk.cu_seqlens + p.pk.num_seqs), 0), p.pk.num_rows_padded);
    const int per = (total + (int)gridDim.x - 1) / (int)gridDim.x;
    const int v0 = min(total, (int)blockIdx.x * per);
    const int n = min(total, v0 + per) - v0;
    if (n <= 0)
        return;  // uniform: the whole CTA leaves before any barrier

    RowCursor cur{p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs, p.pk.num_rows_padded};
    RowSlot first;
    const bool ok0 = map_valid_row(v0, p.pk.cu_seqlens, p.pk.cu_seqlens_padded, p.pk.num_seqs,
                                   p.pk.num_rows_padded, lane, first);
    cur.load(ok0 ? first.seq : 0);

    auto issue = [&](int i) {
        const int st = i % S;
        const int row = cur.row(v0 + i);
        if (tid == 0) {
            slot_row[st] = row;
            slot_seq[st] = cur.b;
        }
        if (row >= 0) {
            const uint16_t* src = p.x + (int64_t)row * p.x_row_stride;
            uint4* dst = stage + st * nvec;
            for (int j = tid; j < nvec; j += kCtaThreads)
                cp_async16(dst + j, src + 8 * j);
        }
        cp_async_commit();
    };

#pragma unroll
    for (int i = 0; i < S - 1; ++i) {
        if (i < n)
            issue(i);
        else
            cp_async_commit();  // keep one group per ring slot
    }
    const float inv_n = 1.0f / (float)p.hidden;
    int mod_seq = -1;
    for (int i = 0; i < n; ++i) {
        if (i + S - 1 < n)
            issue(i + S - 1);
        else
            cp_async_commit();
        cp_async_wait<S - 1>();  // this thread's copies of row i have landed
        __syncthreads();         // ... and everyone else's
        const int st = i % S;
        const int row = slot_row[st];
        if (row >= 0) {  // uniform across the CTA
            const int seq = slot_seq[st];
            if (seq != mod_seq) {  // uniform; rare (sequence boundary)
                const uint16_t* sh = p.shift + (int64_t)seq * p.mod_seq_stride;
                const uint16_t* sc = p.scale + (int64_t)seq * p.mod_seq_stride;
                for (int j = tid; j < nvec; j += kCtaThreads) {
                    mod_sh[j] = ld_shared_vec(sh + 8 * j);
                    mod_sc[j] = ld_shared_vec(sc + 8 * j);
                }
                mod_seq = seq;
                // visibility: the block_sum barriers below come before any read
            }
            const uint4* xs = stage + st * nvec;
            float sum = 0.f;
            for (int j = tid; j < nvec; j += kCtaThreads) {
                float f[8];
                unpack8(xs[j], f);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    sum += f[e];
            }
            const float mean = block_sum(sum, red[0], warp, lane) * inv_n;
            float sq = 0.f;
            for (int j = tid; j < nvec; j += kCtaThreads) {
                float f[8];
                unpack8(xs[j], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float d = f[e] - mean;
                    sq = fmaf(d, d, sq);
                }
            }
            const float rstd = rsqrtf(block_sum(sq, red[1], warp, lane) * inv_n + p.eps);
            uint16_t* orow = p.out + (int64_t)row * p.out_row_stride;
            for (int j = tid; j < nvec; j += kCtaThreads) {
                float f[8], shf[8], scf[8], o[8];
                unpack8(xs[j], f);
                unpack8(mod_sh[j], shf);
                unpack8(mod_sc[j], scf);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    o[e] = fmaf((f[e] - mean) * rstd, 1.0f + scf[e], shf[e]);
                st_stream(orow + 8 * j, pack8(o));
            }
        }
        __syncthreads();  // ring slot st (and the shift/scale copy) may be rewritten next
    }
    cp_async_wait<0>();
}

template <int S>
cudaError_t launch_pipelined(const AdalnParams& p, cudaStream_t stream)
{
    const size_t smem = (size_t)(S + 2) * (p.hidden / 8) * sizeof(uint4);
    cudaError_t e = cudaFuncSetAttribute(adaln_pipelined_kernel<S>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess)
        return e;
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, adaln_pipelined_kernel<S>, kCtaThreads,
                                                           smem)) != cudaSuccess)
        return e;
    const long long want = (long long)sms * (per_sm > 0 ? per_sm : 1);
    const unsigned grid = (unsigned)(want < p.pk.num_rows_padded ? want : p.pk.num_rows_padded);
    adaln_pipelined_kernel<S><<<grid, kCtaThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

#ifndef DIT_ADALN_PIPELINED
#define DIT_ADALN_PIPELINED 0
#endif
#ifndef DIT_ADALN_MAX_VPT
#define DIT_ADALN_MAX_VPT 8
#endif

// Vectors per lane that have an instantiation; a row needing another count
// uses the next larger one (the extra slots are predicated off).
constexpr int kVptSteps[] = {1, 2, 3, 4, 5, 6, 7, 8, 10, 12, 16, 20, 24};

template <int TEAM, int VPT>
void launch_one(const AdalnParams& p, cudaStream_t stream)
{
    const int rows_per_cta = kWarpsPerCta / TEAM;
    const unsigned grid = (unsigned)((p.pk.num_rows_padded + rows_per_cta - 1) / rows_per_cta);
    adaln_kernel<VPT, TEAM><<<grid, kCtaThreads, 0, stream>>>(p);
}

template <int TEAM>
cudaError_t launch_team(const AdalnParams& p, int vpt, cudaStream_t stream)
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
#if DIT_ADALN_MAX_VPT > 8
    case 10: launch_one<TEAM, 10>(p, stream); break;
    case 12: launch_one<TEAM, 12>(p, stream); break;
    case 16: launch_one<TEAM, 16>(p, stream); break;
    case 20: launch_one<TEAM, 20>(p, stream); break;
    case 24: launch_one<TEAM, 24>(p, stream); break;
#endif
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

// Team size: the smallest of 1, 2, 4, 8 warps that holds the row in at most
// DIT_ADALN_MAX_VPT vectors per lane.
cudaError_t launch_adaln_modulate(const AdalnParams& p, cudaStream_t stream)
{
    const int nvec = p.hidden / 8;
#if DIT_ADALN_PIPELINED
    {
#ifdef DIT_ADALN_STAGES
        return launch_pipelined<DIT_ADALN_STAGES>(p, stream);
#else
        const int row_bytes = nvec * 16;
        if (row_bytes <= 6 * 1024)
            return launch_pipelined<8>(p, stream);
        if (row_bytes <= 12 * 1024)
            return launch_pipelined<4>(p, stream);
        return launch_pipelined<2>(p, stream);
#endif
    }
#endif
    for (int team = 1; team <= kWarpsPerCta; team *= 2) {
        const int per = team * kWarp;
        int vpt = (nvec + per - 1) / per;
        if (vpt > DIT_ADALN_MAX_VPT && team < kWarpsPerCta)
            continue;
        for (int s : kVptSteps)
            if (s >= vpt && s <= DIT_ADALN_MAX_VPT) {
                vpt = s;
                break;
            }
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
