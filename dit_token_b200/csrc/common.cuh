// common.cuh -- device helpers shared by the fused DiT token kernels:
// packed-row mapping, 128-bit bf16 vector I/O and bf16 <-> fp32 conversion.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace dit {

constexpr int kWarp = 32;
constexpr int kCtaThreads = 256;          // 8 warps

// ---------------------------------------------- dependent launches
// Called first in every kernel, before any global-memory access: waits until
// the kernel this one depends on (the previous one on the stream, when the
// launch carries the programmatic-serialization attribute) has completed and
// its writes are visible, then lets this kernel's own dependents be
// scheduled.  Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void grid_dependency_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------ packed rows
//
// The packed batch holds num_seqs sequences; sequence b owns padded rows
// [cp[b], cp[b+1]) and its first cs[b+1] - cs[b] rows are valid.  Work is
// indexed by the VALID-row ordinal v in [0, cs[B]) so that padding costs no
// thread: v lives in sequence b = max{b : cs[b] <= v} at padded row
// cp[b] + (v - cs[b]).  "Why Real-Time MiniMax H3 Serving Requires More Than
// a Faster DiT", "Key takeaways", bullet 1: work follows each sequence's
// valid length, so the padding rows at its end cost nothing.

struct RowSlot {
    int32_t row;    // padded row index
    int32_t seq;    // sequence index b
    int32_t local;  // index of the row within its sequence (RoPE position)
};

// Largest b in [0, B) with cs[b] <= v, or -1.  Warp-collective (every lane
// passes the same v): a 32-way search, one ballot per level, so B <= 32 costs
// a single round of loads and B <= 1024 two.
__device__ __forceinline__ int find_seq(int v, const int32_t* __restrict__ cs, int B, int lane)
{
    int lo = 0, n = B;
    while (n > kWarp) {
        const int step = (n + kWarp - 1) / kWarp;
        const int idx = lane * step;
        const bool ok = idx < n && __ldg(cs + lo + idx) <= v;
        const unsigned m = __ballot_sync(0xffffffffu, ok);
        if (m == 0u)
            return -1;
        const int kk = 31 - __clz(m);
        lo += kk * step;
        n = min(step, n - kk * step);
    }
    const bool ok = lane < n && __ldg(cs + lo + lane) <= v;
    const unsigned m = __ballot_sync(0xffffffffu, ok);
    return m == 0u ? -1 : lo + 31 - __clz(m);
}

// Maps valid-row ordinal v to its padded row.  Warp-collective; returns false
// (for the whole warp) when v is past the last valid row or when the device
// descriptor points outside the buffer -- such rows are skipped, never
// followed out of bounds.
__device__ __forceinline__ bool map_valid_row(int v, const int32_t* __restrict__ cs,
                                              const int32_t* __restrict__ cp, int B,
                                              int rows_padded, int lane, RowSlot& s)
{
    const int b = find_seq(v, cs, B, lane);
    if (b < 0)
        return false;
    const int cs0 = __ldg(cs + b), cs1 = __ldg(cs + b + 1);
    const int cp0 = __ldg(cp + b), cp1 = __ldg(cp + b + 1);
    const int r = v - cs0;
    if (r < 0 || r >= cs1 - cs0 || r >= cp1 - cp0)
        return false;
    const long long row = (long long)cp0 + r;
    if (row < 0 || row >= rows_padded)
        return false;
    s.row = (int32_t)row;
    s.seq = b;
    s.local = r;
    return true;
}

// ---------------------------------------------------------- vector I/O
// Streamed activations are touched once: load and store them with the
// evict-first (".cs") policy so they do not push the small per-sequence
// vectors (gates, shifts, scales, norm weights) out of L2.  Those go through
// the read-only path (__ldg) instead.

__device__ __forceinline__ uint4 ld_stream(const uint16_t* p)
{
    return __ldcs(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ void st_stream(uint16_t* p, uint4 v)
{
    __stcs(reinterpret_cast<uint4*>(p), v);
}

// NW 32-bit words (NW = 4: 16 bytes, NW = 8: 32 bytes) of a streamed row,
// evict-first.  The 32-byte form (one 256-bit access per lane, sm_100) halves
// the load and store instructions of a row; it needs a 32-byte aligned
// address.
template <int NW>
__device__ __forceinline__ void ld_stream_words(const uint16_t* p, uint32_t (&w)[NW])
{
    static_assert(NW == 2 || NW == 4 || NW == 8, "8-, 16- or 32-byte accesses");
    if constexpr (NW == 2) {
        const uint2 v = __ldcs(reinterpret_cast<const uint2*>(p));
        w[0] = v.x;
        w[1] = v.y;
    } else if constexpr (NW == 4) {
        const uint4 v = __ldcs(reinterpret_cast<const uint4*>(p));
        w[0] = v.x;
        w[1] = v.y;
        w[2] = v.z;
        w[3] = v.w;
    } else {
        // volatile: kept in program order with the other volatile asm, so
        // never above the grid-dependency wait
        asm volatile("ld.global.cs.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
            : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
            : "l"(p));
    }
}

// The 32-byte store is inline assembly whose memory effect the compiler does
// not see: use it only for output the kernel never reads back.
template <int NW>
__device__ __forceinline__ void st_stream_words(uint16_t* p, const uint32_t (&w)[NW])
{
    static_assert(NW == 2 || NW == 4 || NW == 8, "8-, 16- or 32-byte accesses");
    if constexpr (NW == 2) {
        __stcs(reinterpret_cast<uint2*>(p), make_uint2(w[0], w[1]));
    } else if constexpr (NW == 4) {
        __stcs(reinterpret_cast<uint4*>(p), make_uint4(w[0], w[1], w[2], w[3]));
    } else {
        asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]),
                     "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]));
    }
}

// 8 elements of a small vector that many rows share (norm weights, gates,
// shifts, scales): read-only path, kept in L1/L2.
__device__ __forceinline__ uint4 ld_readonly(const uint16_t* p)
{
    return __ldg(reinterpret_cast<const uint4*>(p));
}

// ------------------------------------------------------ bf16 <-> fp32
// A bf16 value is the upper half of a binary32 value, so widening is a shift.

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ void unpack8(uint4 v, float (&f)[8])
{
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
    f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// ------------------------------------------------ packed fp32 pairs
// sm_100 executes add/mul/fma on two fp32 lanes of a 64-bit register pair in
// one instruction (PTX .f32x2); the row kernels that are bound by instruction
// issue rather than by HBM use these for their element-wise arithmetic.
// The pairs are float2 values operated on with the sm_100 packed builtins
// (__fadd2_rn, __ffma2_rn ...), so the compiler allocates register pairs itself.
typedef float2 f32x2;

__device__ __forceinline__ f32x2 f2_make(float lo, float hi) { return make_float2(lo, hi); }

// bf16x2 word (element 0 in the low half) -> the two values as an fp32 pair.
__device__ __forceinline__ f32x2 f2_from_bf16x2(uint32_t w)
{
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ f32x2 f2_add(f32x2 a, f32x2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ f32x2 f2_sub(f32x2 a, f32x2 b) { return __fadd2_rn(a, make_float2(-b.x, -b.y)); }
__device__ __forceinline__ f32x2 f2_fma(f32x2 a, f32x2 b, f32x2 c) { return __ffma2_rn(a, b, c); }

// Eight consecutive elements, starting at element `elem`, of a per-sequence
// vector stored as bf16 (F32 false) or fp32 (F32 true).  These vectors are
// shared by every row of a sequence: read-only path.  vec8_load only issues
// the load(s) and keeps the raw words, so a loop can put every load of a step
// in flight before the first conversion; vec8_unpack widens them to four fp32
// pairs.
template <bool F32>
struct Vec8Raw;
template <>
struct Vec8Raw<false> {
    uint4 u;
};
template <>
struct Vec8Raw<true> {
    float4 a, b;
};

template <bool F32>
__device__ __forceinline__ Vec8Raw<F32> vec8_load(const void* base, int64_t elem)
{
    Vec8Raw<F32> r;
    if constexpr (F32) {
        const float4* f = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem);
        r.a = __ldg(f);
        r.b = __ldg(f + 1);
    } else {
        r.u = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + elem));
    }
    return r;
}

template <bool F32>
__device__ __forceinline__ void vec8_unpack(const Vec8Raw<F32>& r, f32x2 (&v)[4])
{
    if constexpr (F32) {
        v[0] = make_float2(r.a.x, r.a.y);
        v[1] = make_float2(r.a.z, r.a.w);
        v[2] = make_float2(r.b.x, r.b.y);
        v[3] = make_float2(r.b.z, r.b.w);
    } else {
        v[0] = f2_from_bf16x2(r.u.x);
        v[1] = f2_from_bf16x2(r.u.y);
        v[2] = f2_from_bf16x2(r.u.z);
        v[3] = f2_from_bf16x2(r.u.w);
    }
}

template <bool F32>
__device__ __forceinline__ void vec8_pairs(const void* base, int64_t elem, f32x2 (&v)[4])
{
    vec8_unpack<F32>(vec8_load<F32>(base, elem), v);
}

// 32 bytes of a per-sequence vector (16 bf16 or 8 fp32 elements) through the
// read-only path in one 256-bit load (sm_100); the address must be 32-byte
// aligned.  With a lane's share of a vector this wide, a warp's vector loads
// cover contiguous memory, so each 128-byte line is fetched once per load
// instruction instead of twice.
__device__ __forceinline__ void ld_vec32(const void* p, uint32_t (&w)[8])
{
    asm("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
        : "l"(p));
}

// NP pairs of a per-sequence vector at element `elem` as fp32 pairs, read 32
// bytes at a time: bf16 takes NP = 8 (16 elements), fp32 NP = 4 (8 elements).
template <bool F32, int NP>
__device__ __forceinline__ void vec_pairs_wide(const void* base, int64_t elem, f32x2 (&v)[NP])
{
    static_assert(NP == (F32 ? 4 : 8), "32 bytes: 16 bf16 or 8 fp32 elements");
    uint32_t w[8];
    if constexpr (F32) {
        ld_vec32(static_cast<const float*>(base) + elem, w);
#pragma unroll
        for (int e = 0; e < 4; ++e)
            v[e] = make_float2(__uint_as_float(w[2 * e]), __uint_as_float(w[2 * e + 1]));
    } else {
        ld_vec32(static_cast<const uint16_t*>(base) + elem, w);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            v[e] = f2_from_bf16x2(w[e]);
    }
}

// NP consecutive pairs (2 * NP elements, NP = 2 or 4) of a per-sequence
// vector starting at element `elem`, as fp32 pairs: one 8- or 16-byte load
// (bf16) or one or two 16-byte loads (fp32) through the read-only path.
template <bool F32, int NP>
__device__ __forceinline__ void vec_pairs(const void* base, int64_t elem, f32x2 (&v)[NP])
{
    static_assert(NP == 2 || NP == 4, "4 or 8 elements");
    if constexpr (NP == 4) {
        vec8_pairs<F32>(base, elem, v);
    } else if constexpr (F32) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem));
        v[0] = make_float2(a.x, a.y);
        v[1] = make_float2(a.z, a.w);
    } else {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + elem));
        v[0] = f2_from_bf16x2(u.x);
        v[1] = f2_from_bf16x2(u.y);
    }
}

// fp32 pair -> bf16x2 word, round to nearest even.
__device__ __forceinline__ uint32_t f2_to_bf16x2(f32x2 v)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(v.y), "f"(v.x));
    return r;
}

// Two fp32 values -> one bf16x2 word (round to nearest, ties to even).
__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8])
{
    return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
}

// ----------------------------------------------- row mean / variance
// LayerNorm statistics: the lanes of a warp accumulate s = sum(x - k) and
// q = sum((x - k)^2) about one shift k common to the warp (first k = 0; again
// about the row's mean where that pass lost digits, see row_moments), the
// sums are added over the warp, and become (count, mean, M2 = sum of squared
// deviations).  Warps that share a row merge their moments pairwise (Chan,
// Golub and LeVeque's update):
//   n = na + nb,  d = mb - ma,  mean = ma + d nb / n,  M2 = Ma + Mb + d^2 na nb / n.
// The summation and merge orders are fixed, so the result is bitwise
// reproducible.
struct Moments {
    float n, mean, m2;
};

__device__ __forceinline__ Moments moments_merge(Moments a, Moments b)
{
    const float n = a.n + b.n;
    if (n == 0.f)
        return a;
    const float d = b.mean - a.mean;
    const float wb = __fdividef(b.n, n);  // a weight in [0, 1]: the fast quotient is ample
    return Moments{n, fmaf(d, wb, a.mean), a.m2 + b.m2 + d * d * a.n * wb};
}

__device__ __forceinline__ Moments moments_from_sums(float n, float k, float s, float q)
{
    if (n == 0.f)
        return Moments{0.f, 0.f, 0.f};
    const float m = __fdividef(s, n);
    return Moments{n, k + m, fmaxf(q - s * m, 0.f)};
}

// Moments of a warp's n values from each lane's sums s2 (of x - k) and q2 (of
// (x - k)^2), kept as fp32 pairs, about the warp's common shift k: the sums
// are added over the 32 lanes by an xor butterfly (both lanes of a pair add
// the same two operands, so every lane ends with the same totals).
// M2 = q - s^2 / n (and the mean, k + s / n) cancel when k lies far from the
// mean: `far` reports a shift more than 4 standard deviations away
// (s^2 / n > 16 M2), where up to 4 of fp32's 24 bits are lost; the caller
// then sums the row again about the mean just found (within a small fraction
// of a deviation of the true one).
__device__ __forceinline__ Moments warp_moments(float n, float k, f32x2 s2, f32x2 q2, bool& far)
{
    f32x2 sq = f2_make(s2.x + s2.y, q2.x + q2.y);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        sq = f2_add(sq, f2_make(__shfl_xor_sync(0xffffffffu, sq.x, o), __shfl_xor_sync(0xffffffffu, sq.y, o)));
    const Moments m = moments_from_sums(n, k, sq.x, sq.y);
    far = sq.x * (m.mean - k) > 16.f * m.m2;
    return m;
}

// How many of the vectors i * STRIDE + warp_vec0 + lane (i < VPT, lane < 32)
// fall below nvec: the vectors a warp holds of a row.
template <int VPT, int STRIDE>
__device__ __forceinline__ int warp_vector_count(int warp_vec0, int nvec)
{
    int n = 0;
#pragma unroll
    for (int i = 0; i < VPT; ++i)
        n += min(max(nvec - (i * STRIDE + warp_vec0), 0), kWarp);
    return n;
}

// Statistics of the warp's share of a row: the VPT vectors of NW words each
// lane holds (vectors at or past nvec are empty), about the shift k (common
// to the warp; SHIFT false: k = 0, the values summed as they are).  Vector i
// of the lane is vector i * STRIDE + lane_vec0 of the row.
template <int VPT, int NW, int STRIDE, bool SHIFT>
__device__ __forceinline__ Moments lane_row_moments(const uint32_t (&xv)[VPT][NW], int lane_vec0, int nvec,
                                                    float k, bool& far)
{
    const int lane = threadIdx.x & (kWarp - 1);
    const f32x2 kk = f2_make(k, k);
    f32x2 s2 = f2_make(0.f, 0.f), q2 = f2_make(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        if (i * STRIDE + lane_vec0 < nvec) {
#pragma unroll
            for (int e = 0; e < NW; ++e) {
                const f32x2 d = SHIFT ? f2_sub(f2_from_bf16x2(xv[i][e]), kk) : f2_from_bf16x2(xv[i][e]);
                s2 = f2_add(s2, d);
                q2 = f2_fma(d, d, q2);
            }
        }
    }
    const int nv = warp_vector_count<VPT, STRIDE>(lane_vec0 - lane, nvec);
    return warp_moments((float)(2 * NW * nv), SHIFT ? k : 0.f, s2, q2, far);
}

// The row's moments: sums of the values and their squares as they are (about
// 0), merged across a team of TEAM warps (TEAM > 1: through shared memory,
// behind a barrier); summed again about the mean found when a warp's mean lay
// more than 4 deviations from 0, where the first sums lose digits.  A row
// whose mean is small against its spread -- the usual case, massive
// activations in a few channels included -- takes one pass.  red, red2 and
// far_w: TEAM entries of shared memory.
template <int VPT, int NW, int TEAM>
__device__ __forceinline__ Moments row_moments(const uint32_t (&xv)[VPT][NW], int nvec, Moments* red,
                                               Moments* red2, int* far_w)
{
    constexpr int STRIDE = TEAM * kWarp;
    const int lane = threadIdx.x & (kWarp - 1);
    const int warp = threadIdx.x >> 5;
    // the lane's first vector: a warp per row (several rows per CTA) or a
    // team per row (one row per CTA)
    const int tt = TEAM == 1 ? lane : (int)threadIdx.x;
    bool far;
    Moments m = lane_row_moments<VPT, NW, STRIDE, false>(xv, tt, nvec, 0.f, far);
    if constexpr (TEAM > 1) {
        if (lane == 0) {
            red[warp] = m;
            far_w[warp] = far;
        }
        __syncthreads();
        m = red[0];
        far = far_w[0] != 0;
#pragma unroll
        for (int w = 1; w < TEAM; ++w) {
            m = moments_merge(m, red[w]);
            far = far || far_w[w] != 0;
        }
    }
    if (far) {  // uniform over the warp (TEAM 1) or the CTA
        bool unused;
        m = lane_row_moments<VPT, NW, STRIDE, true>(xv, tt, nvec, m.mean, unused);
        if constexpr (TEAM > 1) {
            if (lane == 0)
                red2[warp] = m;
            __syncthreads();
            m = red2[0];
#pragma unroll
            for (int w = 1; w < TEAM; ++w)
                m = moments_merge(m, red2[w]);
        }
    }
    return m;
}

template <int WIDTH>
__device__ __forceinline__ float group_sum(float v)
{
#pragma unroll
    for (int o = WIDTH / 2; o >= 1; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace dit
