// validate.cu -- device-side check of a packing descriptor (cu_seqlens,
// cu_seqlens_padded).  It writes a flag word and never traps, so a malformed
// descriptor is reported to the host instead of faulting the context.
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

__global__ void validate_seqlens_kernel(const int32_t* __restrict__ cs, const int32_t* __restrict__ cp,
                                        int B, long long rows_padded, int32_t* flag)
{
    // One warp; lanes stride over sequences and the first failure wins.  The
    // leading entries are checked whatever the sequence count, so an empty
    // batch whose descriptor does not start at 0 is reported too.
    constexpr int kNone = 0x7fffffff;
    grid_dependency_wait();
    const int lane = threadIdx.x;
    int first_bad = kNone;
    if (lane == 0 && (cs[0] != 0 || cp[0] != 0))
        first_bad = 0;
    for (int b = lane; b < B; b += kWarp) {
        const int c0 = cs[b], c1 = cs[b + 1], p0 = cp[b], p1 = cp[b + 1];
        const bool bad = c1 < c0 || p1 < p0 || (c1 - c0) > (p1 - p0) || (long long)p1 > rows_padded;
        if (bad)
            first_bad = min(first_bad, b);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
        first_bad = min(first_bad, __shfl_xor_sync(0xffffffffu, first_bad, o));
    if (lane == 0) {
        flag[0] = first_bad != kNone ? 1 : 0;
        flag[1] = first_bad != kNone ? first_bad : -1;
    }
}

}  // namespace

cudaError_t launch_validate_seqlens(const Packing& pk, int64_t num_rows_padded, int32_t* flag,
                                    cudaStream_t stream)
{
    return launch_kernel(validate_seqlens_kernel, 1, kWarp, 0, stream, pk.cu_seqlens, pk.cu_seqlens_padded,
                         (int)pk.num_seqs, (long long)num_rows_padded, flag);
}

}  // namespace dit
