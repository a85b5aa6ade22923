"""Pins of the oracle's rotary layouts beyond the interleaved one.

half-split: a one-hot pair (j, j + D/2) turns by the closed-form angle; the
complex form z_j = y_j + i y_{j+D/2} times exp(i p w_j); and the layout
identity -- permuting elements (and weights) from the half-split order to
the interleaved order maps the two operators onto each other.  none: the
output is torch's rms_norm times the weight at every position."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from _util import bits, f64, golden


def run(q, w, L, H, D, mode, grid=None, sections=(0, 0, 0), eps=1e-6):
    return oracle.qk_rmsnorm_rope(q, q, w, w, [0, L], [0, L], num_q_heads=H, num_k_heads=H, head_dim=D,
                                  rope_grid=grid, sections=sections, eps=eps, want_f64=True, rope_mode=mode)


@pytest.mark.parametrize("case", [c for c in golden("rope_frequencies.json")["cases"] if c["d"] in (64, 128)])
def test_half_split_one_hot_closed_form(case):
    D, j, freq = case["d"], case["j"], case["freq"]
    p = int(round(1 / freq))
    L = p + 1
    x = np.zeros((L, D), np.float32)
    x[:, j] = 0.5
    one = bits(np.ones(D))
    _, _, q64, _ = run(bits(x), one, L, 1, D, "half", eps=0.0)
    assert abs(q64[p][j] - math.sqrt(D) * math.cos(1.0)) < 1e-9
    assert abs(q64[p][j + D // 2] - math.sqrt(D) * math.sin(1.0)) < 1e-9
    others = np.delete(q64[p], [j, j + D // 2])
    assert np.all(others == 0.0)


def test_half_split_complex_form():
    rng = np.random.default_rng(0)
    L, D = 40, 128
    q = bits(rng.standard_normal((L, D)))
    one = bits(np.ones(D))
    _, _, q64, _ = run(q, one, L, 1, D, "half")
    y = F.rms_norm(torch.from_numpy(f64(q)), (D,), eps=1e-6).numpy()
    z = y[:, : D // 2] + 1j * y[:, D // 2:]
    ang = np.arange(L)[:, None] * np.power(10000.0, -np.arange(D // 2) * 2.0 / D)[None, :]
    r = z * np.exp(1j * ang)
    np.testing.assert_allclose(q64[:, : D // 2], r.real, atol=1e-12)
    np.testing.assert_allclose(q64[:, D // 2:], r.imag, atol=1e-12)


@pytest.mark.parametrize("grid", [None, np.array([[2, 3, 4]], np.int32)])
def test_half_split_is_interleaved_under_a_permutation(grid):
    rng = np.random.default_rng(1)
    D, H = 128, 2
    L = 24 + 5
    sections = (44, 42, 42) if grid is not None else (0, 0, 0)
    xh = rng.standard_normal((L, H, D)).astype(np.float32)
    wh = (1 + 0.02 * rng.standard_normal(D)).astype(np.float32)
    perm = np.empty(D, dtype=np.int64)          # interleaved slot 2j <- half j, 2j+1 <- half j + D/2
    perm[0::2] = np.arange(D // 2)
    perm[1::2] = np.arange(D // 2) + D // 2
    xi = xh[..., perm]
    wi = wh[perm]
    _, _, h64, _ = run(bits(xh.reshape(L, -1)), bits(wh), L, H, D, "half", grid, sections)
    _, _, i64, _ = run(bits(xi.reshape(L, -1)), bits(wi), L, H, D, "interleaved", grid, sections)
    np.testing.assert_allclose(h64.reshape(L, H, D)[..., perm], i64.reshape(L, H, D), rtol=1e-13, atol=1e-13)


def test_no_rotation_is_rms_norm_times_weight():
    rng = np.random.default_rng(2)
    L, H, D = 9, 3, 64
    q = bits(rng.standard_normal((L, H * D)))
    w = bits(1 + 0.02 * rng.standard_normal(D))
    _, _, q64, _ = run(q, w, L, H, D, "none", grid=np.array([[1, 3, 3]], np.int32), sections=(22, 22, 20))
    ref = F.rms_norm(torch.from_numpy(f64(q).reshape(L, H, D)), (D,), weight=torch.from_numpy(f64(w)),
                     eps=1e-6).numpy()
    np.testing.assert_allclose(q64.reshape(L, H, D), ref, rtol=1e-13, atol=1e-13)
