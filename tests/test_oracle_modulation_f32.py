"""Pins of the oracle's fp32 modulation vectors: values that bf16 represents
give the bf16 path's results bit for bit; general fp32 values follow
torch's layer_norm affine (adaLN) and the exact-gate cases (residual); the
fused op is still the two ops back to back."""
import numpy as np
import torch
import torch.nn.functional as F

import oracle
from _util import bits, cu, f64, packed


def test_bf16_representable_fp32_vectors_match_the_bf16_path():
    rng = np.random.default_rng(0)
    lengths, padded, C = [5, 9], [8, 12], 256
    x, valid = packed(lengths, padded, C, rng)
    y, _ = packed(lengths, padded, C, rng)
    m16 = bits(rng.standard_normal((2, 3, C)) * 0.1)
    m32 = f64(m16).astype(np.float32)
    cs, cp = cu(lengths), cu(padded)
    f16, f32 = np.ascontiguousarray(m16.reshape(-1)), np.ascontiguousarray(m32.reshape(-1))
    a = oracle.adaln_modulate(x, f16, f16[C:], cs, cp, hidden=C, mod_seq_stride=3 * C)
    b = oracle.adaln_modulate(x, f32, f32[C:], cs, cp, hidden=C, mod_seq_stride=3 * C)
    assert np.array_equal(a[valid], b[valid])
    a = oracle.gated_residual(x, y, f16[2 * C:], cs, cp, hidden=C, gate_seq_stride=3 * C)
    b = oracle.gated_residual(x, y, f32[2 * C:], cs, cp, hidden=C, gate_seq_stride=3 * C)
    assert np.array_equal(a[valid], b[valid])
    a = oracle.gated_residual_adaln(x, y, f16[2 * C:], f16, f16[C:], cs, cp, hidden=C, gate_seq_stride=3 * C,
                                    mod_seq_stride=3 * C)
    b = oracle.gated_residual_adaln(x, y, f32[2 * C:], f32, f32[C:], cs, cp, hidden=C, gate_seq_stride=3 * C,
                                    mod_seq_stride=3 * C)
    assert np.array_equal(a[0][valid], b[0][valid]) and np.array_equal(a[1][valid], b[1][valid])


def test_general_fp32_modulation_follows_layer_norm_affine():
    rng = np.random.default_rng(1)
    L, C, eps = 7, 512, 1e-6
    x = bits(rng.standard_normal((L, C)))
    sh = (rng.standard_normal((1, C)) * 0.1).astype(np.float32)   # not bf16-representable
    sc = (rng.standard_normal((1, C)) * 0.1).astype(np.float32)
    _, o64 = oracle.adaln_modulate(x, sh, sc, [0, L], [0, L], hidden=C, eps=eps, want_f64=True)
    ref = F.layer_norm(torch.from_numpy(f64(x)), (C,), weight=torch.from_numpy(1 + sc[0].astype(np.float64)),
                       bias=torch.from_numpy(sh[0].astype(np.float64)), eps=eps).numpy()
    np.testing.assert_allclose(o64, ref, rtol=1e-12, atol=1e-12)


def test_fp32_gate_exact_cases_and_fused_composition():
    rng = np.random.default_rng(2)
    L, C = 6, 128
    xv = rng.standard_normal((L, C))
    x, y = bits(xv), bits(rng.standard_normal((L, C)))
    out = oracle.gated_residual(x, y, np.zeros((1, C), np.float32), [0, L], [0, L], hidden=C)
    assert np.array_equal(out, x)
    out, o64 = oracle.gated_residual(x, bits(-xv), np.ones((1, C), np.float32), [0, L], [0, L], hidden=C,
                                     want_f64=True)
    assert np.all(o64 == 0.0)
    g = (rng.standard_normal((1, C)) * 0.1).astype(np.float32)
    _, o64 = oracle.gated_residual(x, y, g, [0, L], [0, L], hidden=C, want_f64=True)
    np.testing.assert_allclose(o64, f64(x) + g.astype(np.float64) * f64(y), rtol=0, atol=0)
    sh = (rng.standard_normal((1, C)) * 0.1).astype(np.float32)
    sc = (rng.standard_normal((1, C)) * 0.1).astype(np.float32)
    res, norm = oracle.gated_residual_adaln(x, y, g, sh, sc, [0, L], [0, L], hidden=C)
    r2 = oracle.gated_residual(x, y, g, [0, L], [0, L], hidden=C)
    n2 = oracle.adaln_modulate(r2, sh, sc, [0, L], [0, L], hidden=C)
    assert np.array_equal(res, r2) and np.array_equal(norm, n2)
