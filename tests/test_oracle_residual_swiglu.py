"""Pins of the oracle's gated residual (exact cases, linearity, per-sequence
gate) and SwiGLU (40-digit closed forms, scipy's expit, the odd-part
identity silu(a) - silu(-a) = a, the large-a limit)."""
import numpy as np
import pytest
from scipy.special import expit

import oracle
from _util import bits, cu, f64, golden, packed


# ---------------------------------------------------------- gated residual

def res(x, y, g, lengths, padded, C, gss=None):
    return oracle.gated_residual(x, y, g, cu(lengths), cu(padded), hidden=C, gate_seq_stride=gss,
                                 want_f64=True)


def test_zero_gate_returns_x_bit_exactly():
    rng = np.random.default_rng(0)
    L, C = 7, 256
    x, y = bits(rng.standard_normal((L, C))), bits(rng.standard_normal((L, C)))
    out, _ = res(x, y, bits(np.zeros((1, C))), [L], [L], C)
    assert np.array_equal(out, x)


def test_unit_gate_with_negated_y_is_zero():
    rng = np.random.default_rng(1)
    L, C = 7, 64
    xv = rng.standard_normal((L, C))
    out, o64 = res(bits(xv), bits(-xv), bits(np.ones((1, C))), [L], [L], C)
    assert np.all(o64 == 0.0) and np.all(out == 0)


def test_linear_in_gate_and_exact_small_case():
    rng = np.random.default_rng(2)
    L, C = 5, 64
    x, y = bits(rng.standard_normal((L, C))), bits(rng.standard_normal((L, C)))
    g = rng.standard_normal((1, C)) * 0.1
    _, a = res(x, y, bits(g), [L], [L], C)
    _, b = res(x, y, bits(2 * f64(bits(g))), [L], [L], C)  # exactly twice the bf16 gate
    np.testing.assert_allclose(b - f64(x), 2 * (a - f64(x)), rtol=1e-14, atol=1e-15)
    _, e = res(bits(np.ones((1, 8))), bits(np.full((1, 8), 3.0)), bits(np.full((1, 8), 0.5)), [1], [1], 8)
    assert np.all(e == 2.5)


def test_gate_is_per_sequence():
    rng = np.random.default_rng(3)
    lengths, padded, C = [3, 5], [4, 8], 64
    x, valid = packed(lengths, padded, C, rng)
    y = x.copy()
    y[valid] = bits(-f64(x[valid]))
    gate = bits(np.stack([np.zeros(C), np.ones(C)]))
    out, _ = res(x, y, gate, lengths, padded, C)
    assert np.array_equal(out[:3], x[:3])       # sequence 0: gate 0
    assert np.all(out[4:9] == 0)                 # sequence 1: x - x


# ------------------------------------------------------------------ SwiGLU

def sw(a, b, lengths, padded, I):
    return oracle.swiglu(a, b, cu(lengths), cu(padded), inner=I, want_f64=True)


def test_closed_forms():
    cases = golden("silu_closed_forms.json")["cases"]
    a = bits([[c["a"] for c in cases]])
    assert np.array_equal(f64(a)[0], [c["a"] for c in cases])  # all exactly representable
    _, o = sw(a, bits(np.ones((1, len(cases)))), [1], [1], len(cases))
    np.testing.assert_allclose(o[0], [c["silu"] for c in cases], rtol=2e-16, atol=0)


def test_matches_scipy_expit():
    rng = np.random.default_rng(4)
    L, I = 33, 512
    a = bits(rng.standard_normal((L, I)) * 4)
    b = bits(rng.standard_normal((L, I)))
    _, o = sw(a, b, [L], [L], I)
    A, B = f64(a), f64(b)
    np.testing.assert_allclose(o, A * expit(A) * B, rtol=1e-14, atol=1e-300)


def test_odd_part_identity_and_operand_order():
    rng = np.random.default_rng(5)
    I = 256
    av = f64(bits(rng.standard_normal((1, I)) * 3))
    a = bits(np.concatenate([av, -av]))
    _, o = sw(a, bits(np.ones((2, I))), [2], [2], I)
    np.testing.assert_allclose(o[0] - o[1], av[0], rtol=1e-14, atol=1e-15)
    # silu applies to a, not b: silu(1) * 2 != silu(2) * 1
    _, o = sw(bits([[1.0]]), bits([[2.0]]), [1], [1], 1)
    assert abs(o[0, 0] - 2 * 0.7310585786300049) < 1e-15


def test_zero_operands_and_large_a():
    I = 8
    _, o = sw(bits(np.zeros((1, I))), bits(np.ones((1, I)) * 5), [1], [1], I)
    assert np.all(o == 0)
    _, o = sw(bits(np.ones((1, I)) * 3), bits(np.zeros((1, I))), [1], [1], I)
    assert np.all(o == 0)
    _, o = sw(bits(np.full((1, I), 20.0)), bits(np.full((1, I), -1.5)), [1], [1], I)
    np.testing.assert_allclose(o, 20.0 * -1.5, rtol=3e-9)
    _, o = sw(bits(np.full((1, I), -200.0)), bits(np.ones((1, I))), [1], [1], I)
    assert np.all(np.abs(o) < 1e-80)


@pytest.mark.parametrize("I", [8, 24])
def test_padding_untouched(I):
    rng = np.random.default_rng(6)
    lengths, padded = [2, 0, 3], [4, 2, 5]
    a, valid = packed(lengths, padded, I, rng)
    b, _ = packed(lengths, padded, I, rng)
    out, _ = sw(a, b, lengths, padded, I)
    pad = np.setdiff1d(np.arange(a.shape[0]), valid)
    assert np.all(out[pad] == 0x7FC1)
