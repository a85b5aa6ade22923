"""Pins of the oracle's adaLN modulation: torch.nn.functional.layer_norm (an
independent library routine, with and without its affine standing in for the
modulation), the statistics module, and the exact case scale = -1."""
import statistics

import numpy as np
import torch
import torch.nn.functional as F

import oracle
from _util import bits, cu, f64, packed


def run(x, shift, scale, lengths, padded, C, eps=1e-6, mss=None):
    return oracle.adaln_modulate(x, shift, scale, cu(lengths), cu(padded), hidden=C, eps=eps,
                                 mod_seq_stride=mss, want_f64=True)


def test_identity_modulation_is_layer_norm():
    rng = np.random.default_rng(0)
    L, C, eps = 17, 256, 1e-6
    x = bits(rng.standard_normal((L, C)) * 3 + 0.5)
    z = bits(np.zeros((1, C)))
    _, o64 = run(x, z, z, [L], [L], C, eps)
    ref = F.layer_norm(torch.from_numpy(f64(x)), (C,), eps=eps).numpy()
    np.testing.assert_allclose(o64, ref, rtol=1e-12, atol=1e-12)


def test_modulation_matches_layer_norm_affine():
    # LN(x) * (1 + scale) + shift is layer_norm with weight 1 + scale, bias shift.
    rng = np.random.default_rng(1)
    L, C, eps = 9, 512, 1e-6
    x = bits(rng.standard_normal((L, C)))
    sh = bits(rng.standard_normal((1, C)) * 0.1)
    sc = bits(rng.standard_normal((1, C)) * 0.1)
    _, o64 = run(x, sh, sc, [L], [L], C, eps)
    ref = F.layer_norm(torch.from_numpy(f64(x)), (C,), weight=torch.from_numpy(1 + f64(sc[0])),
                       bias=torch.from_numpy(f64(sh[0])), eps=eps).numpy()
    np.testing.assert_allclose(o64, ref, rtol=1e-12, atol=1e-12)


def test_scale_minus_one_returns_shift_exactly():
    rng = np.random.default_rng(2)
    L, C = 6, 128
    x = bits(rng.standard_normal((L, C)))
    sh = bits(rng.standard_normal((1, C)))
    sc = bits(np.full((1, C), -1.0))
    out, _ = run(x, sh, sc, [L], [L], C)
    assert np.array_equal(out, np.broadcast_to(sh, (L, C)))


def test_mean_zero_and_variance_with_large_eps():
    rng = np.random.default_rng(3)
    L, C, eps = 5, 64, 0.5
    x = bits(rng.standard_normal((L, C)) * 0.7 - 2.0)
    z = bits(np.zeros((1, C)))
    _, o64 = run(x, z, z, [L], [L], C, eps)
    for r in range(L):
        xr = [float(v) for v in f64(x[r])]
        var = statistics.pvariance(xr)
        assert abs(statistics.fmean(o64[r])) < 1e-12
        assert abs(statistics.pvariance(o64[r]) - var / (var + eps)) < 1e-12


def test_each_sequence_uses_its_own_vectors():
    # Two sequences, shift = 0 / 1 and scale = 0 / -1 with a stride of 2C
    # between sequences: rows of sequence 1 become exactly 1.
    rng = np.random.default_rng(4)
    lengths, padded, C = [3, 4], [4, 4], 64
    x, valid = packed(lengths, padded, C, rng)
    mod = np.zeros((2, 2, C), dtype=np.float32)  # [seq, (shift, scale), C]
    mod[1, 0] = 1.0
    mod[1, 1] = -1.0
    m = bits(mod)
    out, o64 = oracle.adaln_modulate(x, m[:, 0].copy(), m[:, 1].copy(), cu(lengths), cu(padded),
                                     hidden=C, want_f64=True)
    assert np.all(o64[4:8] == 1.0)
    ref = F.layer_norm(torch.from_numpy(f64(x[:3])), (C,), eps=1e-6).numpy()
    np.testing.assert_allclose(o64[:3], ref, atol=1e-12)
    # the strided form reads the same vectors: one [seq][shift | scale] buffer,
    # scale starting C elements in, 2C elements between sequences
    flat = np.ascontiguousarray(m.reshape(-1))
    out2 = oracle.adaln_modulate(x, flat, flat[C:], cu(lengths), cu(padded), hidden=C,
                                 mod_seq_stride=2 * C)
    assert np.array_equal(out2[valid], out[valid])
