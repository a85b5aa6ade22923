"""Pins of the oracle's fused gated residual + adaLN: the pair is exactly the
gated residual followed by adaLN of the stored (bf16) residual; at gate 0 the
normalization is torch's layer_norm of x (weight 1 + scale, bias shift); at
scale = -1 it returns shift exactly; the residual output is independent of
the modulation vectors."""
import numpy as np
import torch
import torch.nn.functional as F

import oracle
from _util import bits, cu, f64, packed

SENT = 0x7FC1


def inputs(lengths, padded, C, rng):
    x, valid = packed(lengths, padded, C, rng)
    y, _ = packed(lengths, padded, C, rng)
    B = len(lengths)
    mod = bits(rng.standard_normal((B, 6, C)) * 0.1)
    return x, y, mod, valid


def test_equals_residual_then_adaln_bit_exactly():
    rng = np.random.default_rng(0)
    lengths, padded, C = [7, 0, 12], [8, 4, 16], 256
    x, y, mod, valid = inputs(lengths, padded, C, rng)
    flat = np.ascontiguousarray(mod.reshape(-1))
    cs, cp = cu(lengths), cu(padded)
    res, norm = oracle.gated_residual_adaln(x, y, flat[2 * C:], flat, flat[C:], cs, cp, hidden=C,
                                            gate_seq_stride=6 * C, mod_seq_stride=6 * C,
                                            res_init=np.full_like(x, SENT), norm_init=np.full_like(x, SENT))
    r2 = oracle.gated_residual(x, y, flat[2 * C:], cs, cp, hidden=C, gate_seq_stride=6 * C,
                               out_init=np.full_like(x, SENT))
    n2 = oracle.adaln_modulate(r2, flat, flat[C:], cs, cp, hidden=C, mod_seq_stride=6 * C,
                               out_init=np.full_like(x, SENT))
    assert np.array_equal(res, r2) and np.array_equal(norm, n2)
    pad = np.setdiff1d(np.arange(x.shape[0]), valid)
    assert np.all(res[pad] == SENT) and np.all(norm[pad] == SENT)


def test_zero_gate_normalizes_x_like_torch_layer_norm():
    rng = np.random.default_rng(1)
    L, C, eps = 9, 512, 1e-6
    x = bits(rng.standard_normal((L, C)) * 2 + 0.3)
    y = bits(rng.standard_normal((L, C)))
    g = bits(np.zeros((1, C)))
    sh = bits(rng.standard_normal((1, C)) * 0.1)
    sc = bits(rng.standard_normal((1, C)) * 0.1)
    res, norm, n64 = oracle.gated_residual_adaln(x, y, g, sh, sc, [0, L], [0, L], hidden=C, eps=eps,
                                                 want_f64=True)
    assert np.array_equal(res, x)
    ref = F.layer_norm(torch.from_numpy(f64(x)), (C,), weight=torch.from_numpy(1 + f64(sc[0])),
                       bias=torch.from_numpy(f64(sh[0])), eps=eps).numpy()
    np.testing.assert_allclose(n64, ref, rtol=1e-12, atol=1e-12)


def test_scale_minus_one_returns_shift_and_residual_ignores_modulation():
    rng = np.random.default_rng(2)
    L, C = 4, 64
    x, y = bits(rng.standard_normal((L, C))), bits(rng.standard_normal((L, C)))
    g = bits(rng.standard_normal((1, C)) * 0.1)
    sh = bits(rng.standard_normal((1, C)))
    res1, norm1 = oracle.gated_residual_adaln(x, y, g, sh, bits(np.full((1, C), -1.0)), [0, L], [0, L], hidden=C)
    res2, _ = oracle.gated_residual_adaln(x, y, g, bits(np.zeros((1, C))), bits(np.zeros((1, C))),
                                          [0, L], [0, L], hidden=C)
    assert np.array_equal(norm1, np.broadcast_to(sh, (L, C)))
    assert np.array_equal(res1, res2)
