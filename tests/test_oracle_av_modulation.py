"""Pins of the oracle's per-stream modulation: in a joint audio-video sequence
the first T*H*W valid rows (video) use one vector set and the remaining rows
(audio) another.  The selection is checked against torch's layer_norm with
the affine weight and bias picked per row here, against the plain gated
residual on each stream's rows, and the fused op against the two ops back to
back; audio_offset 0 must give the single-set result."""
import numpy as np
import torch
import torch.nn.functional as F

import oracle
from _util import bits, cu, f64, packed

LENGTHS = [31, 5, 6, 12]
PADDED = [32, 8, 8, 16]
GRID = np.array([[2, 3, 4], [1, 1, 5], [0, 0, 0], [3, 1, 3]], dtype=np.int32)  # video rows 24, 5, 0, 9


def stream_of_rows(lengths, padded, grid):
    """(padded row, sequence, is_audio) of every valid row."""
    out, base = [], 0
    for b, (L, P) in enumerate(zip(lengths, padded)):
        thw = int(grid[b, 0]) * int(grid[b, 1]) * int(grid[b, 2])
        out += [(base + r, b, r >= thw) for r in range(L)]
        base += P
    return out


def vectors(rng, B, C, dtype):
    """[B][2 streams][3 (shift, scale, gate)][C]; returns the flat array."""
    v = rng.standard_normal((B, 2, 3, C)) * 0.1
    return np.ascontiguousarray((bits(v) if dtype == "bf16" else v.astype(np.float32)).reshape(-1))


def value(flat, dtype):
    return f64(flat) if dtype == "bf16" else flat.astype(np.float64)


def test_adaln_per_stream_vectors_follow_layer_norm():
    rng = np.random.default_rng(0)
    C, eps = 128, 1e-6
    x, valid = packed(LENGTHS, PADDED, C, rng)
    for dtype in ("bf16", "f32"):
        flat = vectors(rng, len(LENGTHS), C, dtype)
        vals = value(flat, dtype).reshape(len(LENGTHS), 2, 3, C)
        _, o64 = oracle.adaln_modulate(x, flat, flat[C:], cu(LENGTHS), cu(PADDED), hidden=C, eps=eps,
                                       mod_seq_stride=6 * C, rope_grid=GRID, audio_offset=3 * C, want_f64=True)
        rows = stream_of_rows(LENGTHS, PADDED, GRID)
        assert sum(a for _, _, a in rows) == 7 + 0 + 6 + 3
        for row, b, audio in rows:
            s = int(audio)
            ref = F.layer_norm(torch.from_numpy(f64(x[row])), (C,),
                               weight=torch.from_numpy(1.0 + vals[b, s, 1]),
                               bias=torch.from_numpy(vals[b, s, 0]), eps=eps).numpy()
            np.testing.assert_allclose(o64[row], ref, rtol=1e-12, atol=1e-12)


def test_gated_residual_per_stream_gate():
    rng = np.random.default_rng(1)
    C = 64
    x, _ = packed(LENGTHS, PADDED, C, rng)
    y, _ = packed(LENGTHS, PADDED, C, rng)
    flat = vectors(rng, len(LENGTHS), C, "f32")
    vals = value(flat, "f32").reshape(len(LENGTHS), 2, 3, C)
    out = oracle.gated_residual(x, y, flat[2 * C:], cu(LENGTHS), cu(PADDED), hidden=C, gate_seq_stride=6 * C,
                                rope_grid=GRID, audio_offset=3 * C)
    for row, b, audio in stream_of_rows(LENGTHS, PADDED, GRID):
        # one stream's gate on one row: the single-sequence op on that row alone
        g = np.ascontiguousarray(flat.reshape(len(LENGTHS), 2, 3, C)[b, int(audio), 2][None, :])
        one = oracle.gated_residual(x[row][None, :], y[row][None, :], g, [0, 1], [0, 1], hidden=C)
        assert np.array_equal(out[row], one[0])
        # and the gate really differs between the streams of this sequence
        assert not np.array_equal(vals[b, 0, 2], vals[b, 1, 2])


def test_fused_is_the_two_per_stream_ops_back_to_back():
    rng = np.random.default_rng(2)
    C = 96
    x, valid = packed(LENGTHS, PADDED, C, rng)
    y, _ = packed(LENGTHS, PADDED, C, rng)
    flat = vectors(rng, len(LENGTHS), C, "bf16")
    cs, cp = cu(LENGTHS), cu(PADDED)
    kw = dict(hidden=C, rope_grid=GRID)
    res, norm = oracle.gated_residual_adaln(x, y, flat[2 * C:], flat, flat[C:], cs, cp, gate_seq_stride=6 * C,
                                            mod_seq_stride=6 * C, gate_audio_offset=3 * C,
                                            mod_audio_offset=3 * C, **kw)
    r2 = oracle.gated_residual(x, y, flat[2 * C:], cs, cp, gate_seq_stride=6 * C, audio_offset=3 * C, **kw)
    n2 = oracle.adaln_modulate(r2, flat, flat[C:], cs, cp, mod_seq_stride=6 * C, audio_offset=3 * C, **kw)
    assert np.array_equal(res[valid], r2[valid])
    assert np.array_equal(norm[valid], n2[valid])


def test_zero_audio_offset_is_the_single_set():
    rng = np.random.default_rng(3)
    C = 64
    x, valid = packed(LENGTHS, PADDED, C, rng)
    flat = vectors(rng, len(LENGTHS), C, "bf16")
    cs, cp = cu(LENGTHS), cu(PADDED)
    a = oracle.adaln_modulate(x, flat, flat[C:], cs, cp, hidden=C, mod_seq_stride=6 * C, rope_grid=GRID,
                              audio_offset=0)
    b = oracle.adaln_modulate(x, flat, flat[C:], cs, cp, hidden=C, mod_seq_stride=6 * C)
    assert np.array_equal(a[valid], b[valid])
    # and a non-zero offset changes exactly the audio rows
    c = oracle.adaln_modulate(x, flat, flat[C:], cs, cp, hidden=C, mod_seq_stride=6 * C, rope_grid=GRID,
                              audio_offset=3 * C)
    for row, _, audio in stream_of_rows(LENGTHS, PADDED, GRID):
        assert np.array_equal(c[row], b[row]) != audio
