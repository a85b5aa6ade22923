/*
 * abi_demo.c -- the C ABI used from plain C, with no Python: device buffers
 * from the CUDA runtime, the library's entry points called with raw
 * pointers.  Checks results that have exact closed forms:
 *   dit_gated_residual with gate 0            -> out == x, bit for bit
 *   dit_gated_residual with gate 1, y = -x    -> out == 0
 *   dit_adaln_modulate with scale -1          -> out == shift, bit for bit
 *   dit_swiglu with b = 0                     -> out == +-0
 * and that a NULL pointer is reported before any launch.  Padding rows must
 * keep their fill.  Prints "abi_demo: ok" and exits 0 on success.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "dit_token.h"

#define ROWS 24      /* two sequences: 9 valid of 16 padded rows, 5 valid of 8 */
#define C 264        /* hidden = inner: a multiple of 8 that is not a multiple of 256 */
#define FILL 0x7FC1u /* bf16 NaN on padding rows */

static uint32_t lcg = 12345u;
static uint16_t rand_bf16(void)
{
    lcg = lcg * 1664525u + 1013904223u;
    /* sign, exponent 120..134 (|x| in [2^-7, 2^8)), 7 mantissa bits */
    uint16_t sign = (uint16_t)((lcg >> 31) << 15);
    uint16_t exp = (uint16_t)(120u + ((lcg >> 16) % 15u));
    uint16_t man = (uint16_t)((lcg >> 8) & 0x7Fu);
    return (uint16_t)(sign | (exp << 7) | man);
}

static int fail(const char* what)
{
    fprintf(stderr, "abi_demo: FAILED: %s\n", what);
    return 1;
}

#define CK(call)                                                              \
    do {                                                                      \
        if ((call) != cudaSuccess)                                            \
            return fail(#call);                                               \
    } while (0)

int main(void)
{
    const int32_t cs[3] = {0, 9, 14}, cp[3] = {0, 16, 24};
    static uint16_t hx[ROWS * C], hneg[ROWS * C], hout[ROWS * C], hvec[2 * C], hfill[ROWS * C];
    for (int i = 0; i < ROWS * C; ++i) {
        hx[i] = rand_bf16();
        hneg[i] = (uint16_t)(hx[i] ^ 0x8000u);
        hfill[i] = (uint16_t)FILL;
    }
    uint16_t *x, *y, *out, *vec, *zero;
    int32_t *dcs, *dcp;
    const size_t nb = sizeof(uint16_t) * ROWS * C;
    CK(cudaMalloc((void**)&x, nb));
    CK(cudaMalloc((void**)&y, nb));
    CK(cudaMalloc((void**)&out, nb));
    CK(cudaMalloc((void**)&vec, sizeof(uint16_t) * 2 * C));
    CK(cudaMalloc((void**)&zero, nb));
    CK(cudaMalloc((void**)&dcs, sizeof cs));
    CK(cudaMalloc((void**)&dcp, sizeof cp));
    CK(cudaMemcpy(x, hx, nb, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(dcs, cs, sizeof cs, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(dcp, cp, sizeof cp, cudaMemcpyHostToDevice));
    CK(cudaMemset(zero, 0, nb));

    /* gate 0: out == x (two sequences share one gate vector: sequence stride 0) */
    CK(cudaMemset(vec, 0, sizeof(uint16_t) * 2 * C));
    CK(cudaMemcpy(out, hfill, nb, cudaMemcpyHostToDevice));
    if (dit_gated_residual(x, C, zero, C, vec, 0, out, C, dcs, dcp, 2, ROWS, C, NULL) != DIT_OK)
        return fail("dit_gated_residual (gate 0)");
    CK(cudaMemcpy(hout, out, nb, cudaMemcpyDeviceToHost));
    for (int b = 0; b < 2; ++b)
        for (int r = cp[b]; r < cp[b + 1]; ++r)
            for (int c = 0; c < C; ++c) {
                const uint16_t want = r - cp[b] < cs[b + 1] - cs[b] ? hx[r * C + c] : (uint16_t)FILL;
                if (hout[r * C + c] != want)
                    return fail("gate 0 must return x on valid rows and leave padding alone");
            }

    /* gate 1, y = -x: out == 0 */
    for (int i = 0; i < C; ++i)
        hvec[i] = 0x3F80u; /* 1.0 */
    CK(cudaMemcpy(vec, hvec, sizeof(uint16_t) * C, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(y, hneg, nb, cudaMemcpyHostToDevice));
    if (dit_gated_residual(x, C, y, C, vec, 0, out, C, dcs, dcp, 2, ROWS, C, NULL) != DIT_OK)
        return fail("dit_gated_residual (gate 1)");
    CK(cudaMemcpy(hout, out, nb, cudaMemcpyDeviceToHost));
    for (int r = 0; r < 9; ++r)
        for (int c = 0; c < C; ++c)
            if ((hout[r * C + c] & 0x7FFFu) != 0)
                return fail("x + 1 * (-x) must be zero");

    /* adaLN with scale -1: LN(x) * 0 + shift == shift */
    for (int i = 0; i < C; ++i) {
        hvec[i] = rand_bf16();      /* shift */
        hvec[C + i] = 0xBF80u;      /* scale = -1.0 */
    }
    CK(cudaMemcpy(vec, hvec, sizeof(uint16_t) * 2 * C, cudaMemcpyHostToDevice));
    if (dit_adaln_modulate(x, C, out, C, vec, vec + C, 0, dcs, dcp, 2, ROWS, C, 1e-6f, NULL) != DIT_OK)
        return fail("dit_adaln_modulate");
    CK(cudaMemcpy(hout, out, nb, cudaMemcpyDeviceToHost));
    for (int r = 16; r < 21; ++r)
        for (int c = 0; c < C; ++c)
            if (hout[r * C + c] != hvec[c])
                return fail("scale -1 must return the shift");

    /* SwiGLU with b = 0: silu(a) * 0 == +-0 */
    if (dit_swiglu(x, C, zero, C, out, C, dcs, dcp, 2, ROWS, C, NULL) != DIT_OK)
        return fail("dit_swiglu");
    CK(cudaMemcpy(hout, out, nb, cudaMemcpyDeviceToHost));
    for (int r = 0; r < 9; ++r)
        for (int c = 0; c < C; ++c)
            if ((hout[r * C + c] & 0x7FFFu) != 0)
                return fail("silu(a) * 0 must be zero");

    /* argument errors come back before any launch */
    if (dit_swiglu(NULL, C, zero, C, out, C, dcs, dcp, 2, ROWS, C, NULL) != DIT_ERR_NULL)
        return fail("a NULL input must give DIT_ERR_NULL");
    if (strncmp(dit_status_string(DIT_ERR_NULL), "DIT_ERR_NULL", 12) != 0)
        return fail("dit_status_string");
    CK(cudaDeviceSynchronize());
    printf("abi_demo: ok (ABI version %d)\n", dit_abi_version());
    return 0;
}
