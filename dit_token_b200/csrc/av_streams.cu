// av_streams.cu -- the per-stream packing descriptor of joint audio-video
// sequences.  A request packs its video latents (T*H*W rows, from rope_grid)
// and then its audio tokens into one sequence, followed by suffix padding
// ("Why Real-Time MiniMax H3 Serving Requires More Than a Faster DiT", "Key
// takeaways", bullet 1).  Sequence b of the input descriptor becomes two
// sequences of the output:
//   2b     the video rows of b (valid = padded = min(T*H*W, L_b); for a slice
//          of a longer sequence starting at row pos_offset[b], the grid rows
//          past that start)
//   2b + 1 the audio rows of b, then all of b's padding
// Every per-sequence operator run on the output descriptor, with its
// per-sequence vectors laid out [B][2][...], applies one vector set to the
// video rows and another to the audio rows -- per-stream modulation with no
// change to the operators' kernels and no extra per-row branch in them.
#include "common.cuh"
#include "launch.h"

namespace dit {
namespace {

__global__ void __launch_bounds__(kCtaThreads)
av_stream_seqlens_kernel(const int32_t* __restrict__ cs, const int32_t* __restrict__ cp,
                         const int32_t* __restrict__ grid, const int32_t* __restrict__ pos_offset, int B,
                         int32_t* __restrict__ out_cs, int32_t* __restrict__ out_cp)
{
    grid_dependency_wait();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i == 0) {
        out_cs[0] = cs[0];
        out_cp[0] = cp[0];
    }
    for (int b = i; b < B; b += gridDim.x * blockDim.x) {
        const int32_t c0 = cs[b], c1 = cs[b + 1], p0 = cp[b], p1 = cp[b + 1];
        // the video part never exceeds the valid rows nor the padded extent,
        // so a well-formed descriptor stays well-formed
        long long cap = (long long)c1 - c0;
        const long long room = (long long)p1 - p0;
        cap = cap < room ? cap : room;
        cap = cap > 0 ? cap : 0;
        // video rows left in this slice: the grid's rows past the slice's start
        const long long off = pos_offset ? pos_offset[b] : 0;
        const long long thw = (long long)grid[3 * b] * grid[3 * b + 1] * grid[3 * b + 2] - off;
        const int32_t v = (int32_t)(thw <= 0 ? 0 : (thw < cap ? thw : cap));
        out_cs[2 * b + 1] = c0 + v;
        out_cs[2 * b + 2] = c1;
        out_cp[2 * b + 1] = p0 + v;
        out_cp[2 * b + 2] = p1;
    }
}

}  // namespace

cudaError_t launch_av_stream_seqlens(const int32_t* cu_seqlens, const int32_t* cu_seqlens_padded,
                                     const int32_t* rope_grid, const int32_t* pos_offset, int32_t num_seqs,
                                     int32_t* out_cu_seqlens, int32_t* out_cu_seqlens_padded, cudaStream_t stream)
{
    const int blocks = num_seqs / kCtaThreads + 1;
    const unsigned grid = (unsigned)(blocks < 1024 ? blocks : 1024);
    return launch_kernel(av_stream_seqlens_kernel, grid, kCtaThreads, 0, stream, cu_seqlens, cu_seqlens_padded,
                         rope_grid, pos_offset, (int)num_seqs, out_cu_seqlens, out_cu_seqlens_padded);
}

}  // namespace dit
