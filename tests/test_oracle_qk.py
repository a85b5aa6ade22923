"""Pins of the oracle's Q/K RMSNorm + RoPE against facts fixed by the mathematics.

RMSNorm: unit weight gives RMS 1 per head; the weight scales the RMS; the
epsilon enters as sqrt(ms / (ms + eps)); torch.nn.functional.rms_norm agrees
where the rotation is the identity.  RoPE: closed-form frequencies rotate a
one-hot pair by exactly 1 rad at the chosen positions; pairs are interleaved;
pair norms are preserved; q.k depends only on the position offset; the
complex-exponential form agrees; 3D positions decompose t-major with per-axis
section frequencies; rows after the video grid use 1D positions restarting at
0 with full-head_dim frequencies.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from _util import bits, cu, f64, golden, packed

SQ = math.sqrt


def run(q, k, wq, wk, lengths, padded, Hq, Hk, D, grid=None, sections=(0, 0, 0), eps=1e-6,
        theta=10000.0, rows=None):
    return oracle.qk_rmsnorm_rope(
        q, k, wq, wk, cu(lengths), cu(padded), num_q_heads=Hq, num_k_heads=Hk, head_dim=D,
        rope_grid=grid, sections=sections, rope_theta=theta, eps=eps, rows=rows, want_f64=True)


def one_hot_rows(n, H, D, index, value=0.5):
    x = np.zeros((n, H * D), dtype=np.float32)
    for h in range(H):
        x[:, h * D + index] = value
    return bits(x)


def test_unit_weight_rms_is_one_per_head():
    rng = np.random.default_rng(0)
    L, Hq, Hk, D = 37, 3, 2, 64
    x = rng.standard_normal((L, Hq, D)) * np.array([0.01, 1.0, 30.0])[None, :, None]
    q = bits(x.reshape(L, -1))
    k = bits(rng.standard_normal((L, Hk * D)) * 5)
    one = bits(np.ones(D))
    _, _, q64, k64 = run(q, k, one, one, [L], [L], Hq, Hk, D, eps=0.0)
    for t, H in ((q64, Hq), (k64, Hk)):
        rms = np.sqrt(np.mean(t.reshape(L, H, D) ** 2, axis=-1))
        np.testing.assert_allclose(rms, 1.0, rtol=0, atol=1e-12)


def test_weights_scale_rms_separately_for_q_and_k():
    rng = np.random.default_rng(1)
    L, H, D = 9, 2, 128
    q = bits(rng.standard_normal((L, H * D)))
    k = bits(rng.standard_normal((L, H * D)))
    _, _, q64, k64 = run(q, k, bits(np.full(D, 2.0)), bits(np.full(D, 0.5)), [L], [L], H, H, D, eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(q64.reshape(L, H, D) ** 2, -1)), 2.0, atol=1e-12)
    np.testing.assert_allclose(np.sqrt(np.mean(k64.reshape(L, H, D) ** 2, -1)), 0.5, atol=1e-12)


def test_eps_enters_as_ms_over_ms_plus_eps():
    rng = np.random.default_rng(2)
    L, H, D, eps = 11, 2, 64, 0.75
    q = bits(rng.standard_normal((L, H * D)) * 0.6)
    one = bits(np.ones(D))
    _, _, q64, _ = run(q, q, one, one, [L], [L], H, H, D, eps=eps)
    ms = np.mean(f64(q).reshape(L, H, D) ** 2, -1)
    rms = np.sqrt(np.mean(q64.reshape(L, H, D) ** 2, -1))
    np.testing.assert_allclose(rms, np.sqrt(ms / (ms + eps)), atol=1e-12)


def test_position_zero_matches_torch_rms_norm():
    rng = np.random.default_rng(3)
    L, H, D, eps = 4, 3, 128, 1e-6
    q = bits(rng.standard_normal((L, H * D)))
    w = bits(1 + 0.02 * rng.standard_normal(D))
    _, _, q64, _ = run(q, q, w, w, [L], [L], H, H, D, eps=eps)
    ref = F.rms_norm(torch.from_numpy(f64(q[0]).reshape(H, D)), (D,),
                     weight=torch.from_numpy(f64(w)), eps=eps).numpy()
    np.testing.assert_allclose(q64[0].reshape(H, D), ref, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("case", golden("rope_frequencies.json")["cases"])
def test_one_hot_pair_rotates_by_closed_form_angle(case):
    # One-hot at element 2j: RMSNorm (eps = 0, w = 1) makes it sqrt(D); at the
    # position p = 1 / freq the pair turns by exactly 1 rad.
    d, j, freq = case["d"], case["j"], case["freq"]
    if d not in (64, 128):
        pytest.skip("3D section widths are covered by the 3D tests")
    p = int(round(1.0 / freq))
    L = p + 1
    x = one_hot_rows(L, 1, d, 2 * j)
    one = bits(np.ones(d))
    _, _, q64, _ = run(x, x, one, one, [L], [L], 1, 1, d, eps=0.0)
    out = q64[p]
    assert abs(out[2 * j] - SQ(d) * math.cos(1.0)) < 1e-9
    assert abs(out[2 * j + 1] - SQ(d) * math.sin(1.0)) < 1e-9
    others = np.delete(out, [2 * j, 2 * j + 1])
    assert np.all(np.abs(others) < 1e-300)


def test_pairs_are_interleaved_and_rotation_is_counterclockwise():
    # (x0, x1) = (1, 0) at p = 1 must become sqrt(D) (cos 1, sin 1): the pair is
    # elements (2j, 2j+1), not (j, j + D/2), and the sign is + for sin on x1.
    D = 64
    x = one_hot_rows(2, 1, D, 0)
    one = bits(np.ones(D))
    _, _, q64, _ = run(x, x, one, one, [2], [2], 1, 1, D, eps=0.0)
    assert q64[1][1] > 0 and abs(q64[1][1] - SQ(D) * math.sin(1.0)) < 1e-12
    assert abs(q64[1][D // 2]) == 0.0


def test_pair_norm_is_preserved():
    rng = np.random.default_rng(4)
    L, H, D = 300, 2, 128
    q = bits(rng.standard_normal((L, H * D)))
    one = bits(np.ones(D))
    _, _, q64, _ = run(q, q, one, one, [L], [L], H, H, D, eps=1e-6)
    y = F.rms_norm(torch.from_numpy(f64(q).reshape(L, H, D)), (D,), eps=1e-6).numpy()
    n_in = np.hypot(y[..., 0::2], y[..., 1::2])
    o = q64.reshape(L, H, D)
    n_out = np.hypot(o[..., 0::2], o[..., 1::2])
    np.testing.assert_allclose(n_out, n_in, rtol=1e-12, atol=1e-14)


def test_matches_complex_exponential_form():
    # RoPE of a pair = (y_2j + i y_2j+1) * exp(i p theta^(-2j/D)).
    rng = np.random.default_rng(5)
    L, D, theta = 50, 64, 10000.0
    q = bits(rng.standard_normal((L, D)))
    one = bits(np.ones(D))
    _, _, q64, _ = run(q, q, one, one, [L], [L], 1, 1, D, eps=1e-6)
    y = F.rms_norm(torch.from_numpy(f64(q)), (D,), eps=1e-6).numpy()
    z = y[:, 0::2] + 1j * y[:, 1::2]
    ang = np.arange(L)[:, None] * np.power(theta, -np.arange(D // 2) * 2.0 / D)[None, :]
    w = z * np.exp(1j * ang)
    np.testing.assert_allclose(q64[:, 0::2], w.real, atol=1e-12)
    np.testing.assert_allclose(q64[:, 1::2], w.imag, atol=1e-12)


@pytest.mark.parametrize("grid", [None, (3, 4, 5)])
def test_qk_dot_depends_only_on_offset(grid):
    rng = np.random.default_rng(6)
    D, H = 128, 1
    if grid is None:
        L, m, n, s = 40, 3, 11, 17
        sections = (0, 0, 0)
        rows_pairs = [(m, n), (m + s, n + s)]
        G = None
    else:
        T, Hh, W = grid
        L = T * Hh * W
        sections = (44, 42, 42)
        # shift every axis by one: (0,1,2)->(1,2,3) for q and (1,0,1)->(2,1,2) for k
        def r(t, h, w):
            return t * Hh * W + h * W + w
        rows_pairs = [(r(0, 1, 2), r(1, 0, 1)), (r(1, 2, 3), r(2, 1, 2))]
        G = np.array([grid], dtype=np.int32)
    qv = rng.standard_normal(D)
    kv = rng.standard_normal(D)
    q = np.zeros((L, D))
    k = np.zeros((L, D))
    for mq, nk in rows_pairs:
        q[mq] = qv
        k[nk] = kv
    one = bits(np.ones(D))
    _, _, q64, k64 = run(bits(q), bits(k), one, one, [L], [L], H, H, D, grid=G, sections=sections, eps=1e-6)
    d0 = np.dot(q64[rows_pairs[0][0]], k64[rows_pairs[0][1]])
    d1 = np.dot(q64[rows_pairs[1][0]], k64[rows_pairs[1][1]])
    assert abs(d0 - d1) < 1e-10 * max(1.0, abs(d0))


def test_3d_positions_decompose_t_major_by_section():
    # One-hot at the first pair of each section (elements 0, 44, 86) rotates
    # by t, h and w respectively (first-pair frequency is 1).
    T, H, W, D = 3, 4, 5, 128
    L = T * H * W
    one = bits(np.ones(D))
    G = np.array([[T, H, W]], dtype=np.int32)
    for elem, axis in ((0, 0), (44, 1), (86, 2)):
        x = one_hot_rows(L, 1, D, elem)
        _, _, q64, _ = run(x, x, one, one, [L], [L], 1, 1, D, grid=G, sections=(44, 42, 42), eps=0.0)
        for r in range(L):
            pos = (r // (H * W), (r // W) % H, r % W)[axis]
            assert abs(q64[r][elem] - SQ(D) * math.cos(pos)) < 1e-12
            assert abs(q64[r][elem + 1] - SQ(D) * math.sin(pos)) < 1e-12


def test_3d_section_frequency_uses_section_width():
    # t-section of 44 elements: local pair 11 has frequency 10000^(-22/44) = 0.01,
    # so at t = 100 it turns by 1 rad.  A whole-head_dim reading would give
    # 10000^(-22/128) instead.
    freq = [c for c in golden("rope_frequencies.json")["cases"] if c["d"] == 44][0]["freq"]
    T, D = 101, 128
    x = one_hot_rows(T, 1, D, 22)
    one = bits(np.ones(D))
    G = np.array([[T, 1, 1]], dtype=np.int32)
    _, _, q64, _ = run(x, x, one, one, [T], [T], 1, 1, D, grid=G, sections=(44, 42, 42), eps=0.0)
    t = int(round(1 / freq))
    assert abs(q64[t][22] - SQ(D) * math.cos(1.0)) < 1e-9
    assert abs(q64[t][23] - SQ(D) * math.sin(1.0)) < 1e-9


def test_rows_after_grid_use_1d_positions_with_full_head_dim():
    # Audio rows after a 2x2x2 grid: position restarts at 0; pair 32 of a
    # 128-wide head has the 1D frequency 0.01 (it would be an h-section pair
    # on a 3D row).
    T = H = W = 2
    thw, D, audio = 8, 128, 101
    L = thw + audio
    one = bits(np.ones(D))
    G = np.array([[T, H, W]], dtype=np.int32)
    for elem, freq in ((0, 1.0), (64, 0.01)):
        x = one_hot_rows(L, 1, D, elem)
        _, _, q64, _ = run(x, x, one, one, [L], [L], 1, 1, D, grid=G, sections=(44, 42, 42), eps=0.0)
        for r in range(thw, L):
            p = r - thw
            assert abs(q64[r][elem] - SQ(D) * math.cos(p * freq)) < 1e-9
            assert abs(q64[r][elem + 1] - SQ(D) * math.sin(p * freq)) < 1e-9


@pytest.mark.parametrize("axis", [0, 1, 2])
def test_unit_axis_leaves_its_section_unrotated(axis):
    rng = np.random.default_rng(7)
    dims = [3, 4, 5]
    dims[axis] = 1
    T, H, W = dims
    D, L = 128, T * H * W
    sec = (44, 42, 42)
    lo = sum(sec[:axis])
    q = bits(rng.standard_normal((L, D)))
    one = bits(np.ones(D))
    G = np.array([dims], dtype=np.int32)
    _, _, q64, _ = run(q, q, one, one, [L], [L], 1, 1, D, grid=G, sections=sec, eps=1e-6)
    y = F.rms_norm(torch.from_numpy(f64(q)), (D,), eps=1e-6).numpy()
    np.testing.assert_allclose(q64[:, lo:lo + sec[axis]], y[:, lo:lo + sec[axis]], atol=1e-14)


def test_grid_1x1xW_with_one_section_equals_1d():
    rng = np.random.default_rng(8)
    W, D = 33, 64
    q = bits(rng.standard_normal((W, 2 * D)))
    k = bits(rng.standard_normal((W, 2 * D)))
    w = bits(1 + 0.02 * rng.standard_normal(D))
    a = run(q, k, w, w, [W], [W], 2, 2, D)
    b = run(q, k, w, w, [W], [W], 2, 2, D, grid=np.array([[1, 1, W]], np.int32), sections=(0, 0, D))
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_gqa_shapes_and_invalid_sections():
    rng = np.random.default_rng(9)
    L, D = 5, 64
    q = bits(rng.standard_normal((L, 4 * D)))
    k = bits(rng.standard_normal((L, 2 * D)))
    one = bits(np.ones(D))
    qo, ko, q64, k64 = run(q, k, one, one, [L], [L], 4, 2, D, eps=0.0)
    assert q64.shape == (L, 4 * D) and k64.shape == (L, 2 * D)
    np.testing.assert_allclose(np.sqrt(np.mean(k64.reshape(L, 2, D) ** 2, -1)), 1.0, atol=1e-12)
    with pytest.raises(ValueError):
        run(q, k, one, one, [L], [L], 4, 2, D, grid=np.array([[1, 1, L]], np.int32), sections=(20, 20, 20))
    with pytest.raises(ValueError):
        run(q, k, one, one, [L], [L], 4, 2, D, grid=np.array([[1, 1, L]], np.int32), sections=(21, 21, 22))


def test_padding_rows_untouched_and_bf16_is_rounded_f64():
    rng = np.random.default_rng(10)
    lengths, padded, H, D = [5, 0, 9], [8, 4, 16], 2, 64
    q, valid = packed(lengths, padded, H * D, rng)
    k, _ = packed(lengths, padded, H * D, rng)
    one = bits(np.ones(D))
    qo, ko, q64, _ = run(q, k, one, one, lengths, padded, H, H, D)
    pad = np.setdiff1d(np.arange(q.shape[0]), valid)
    assert np.array_equal(qo[pad], q[pad]) and np.array_equal(ko[pad], k[pad])
    assert np.all(np.isnan(q64[pad]))
    assert np.array_equal(qo[valid], oracle.f64_to_bf16_array(q64[valid]))
