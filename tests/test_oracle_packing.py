"""Pins of the oracle's packed-sequence handling: padding rows are left alone,
a batch equals its sequences run one by one (concatenation invariance,
positions restart per sequence), zero-length sequences are no-ops, a row
subset gives the same rows as the full run, malformed descriptors are
rejected."""
import numpy as np
import pytest

import oracle
from _util import bits, cu, packed

SENT = 0x7FC1


def all_ops(lengths, padded, rng, grid=None, rows=None):
    H, D, C, I = 2, 64, 128, 64
    q, valid = packed(lengths, padded, H * D, rng)
    k, _ = packed(lengths, padded, H * D, rng)
    x, _ = packed(lengths, padded, C, rng)
    y, _ = packed(lengths, padded, C, rng)
    a, _ = packed(lengths, padded, I, rng)
    b, _ = packed(lengths, padded, I, rng)
    B = len(lengths)
    w = bits(1 + 0.02 * rng.standard_normal(D))
    mod = bits(rng.standard_normal((B, 3, C)) * 0.1)
    cs, cp = cu(lengths), cu(padded)
    sec = (22, 22, 20) if grid is not None else (0, 0, 0)
    qo, ko = oracle.qk_rmsnorm_rope(q, k, w, w, cs, cp, num_q_heads=H, num_k_heads=H, head_dim=D,
                                    rope_grid=grid, sections=sec, rows=rows)
    ao = oracle.adaln_modulate(x, mod[:, 0].copy(), mod[:, 1].copy(), cs, cp, hidden=C, rows=rows,
                               out_init=np.full_like(x, SENT))
    go = oracle.gated_residual(x, y, mod[:, 2].copy(), cs, cp, hidden=C, rows=rows,
                               out_init=np.full_like(x, SENT))
    so = oracle.swiglu(a, b, cs, cp, inner=I, rows=rows)
    inputs = dict(q=q, k=k, x=x, y=y, a=a, b=b, w=w, mod=mod)
    return inputs, valid, (qo, ko, ao, go, so)


def test_padding_rows_are_left_alone():
    rng = np.random.default_rng(0)
    lengths, padded = [5, 0, 3, 7], [8, 2, 3, 9]
    inp, valid, outs = all_ops(lengths, padded, rng)
    pad = np.setdiff1d(np.arange(sum(padded)), valid)
    qo, ko, ao, go, so = outs
    assert np.array_equal(qo[pad], inp["q"][pad]) and np.array_equal(ko[pad], inp["k"][pad])
    for o in (ao, go, so):
        assert np.all(o[pad] == SENT)
        assert not np.any(o[valid] == SENT)


@pytest.mark.parametrize("with_grid", [False, True])
def test_batch_equals_sequences_run_alone(with_grid):
    rng = np.random.default_rng(1)
    lengths, padded = [6, 13, 4], [8, 16, 4]
    grid = np.array([[1, 2, 2], [2, 2, 3], [0, 0, 0]], np.int32) if with_grid else None
    inp, valid, outs = all_ops(lengths, padded, rng, grid=grid)
    cp = cu(padded)
    H, D, C, I = 2, 64, 128, 64
    sec = (22, 22, 20) if with_grid else (0, 0, 0)
    for s, L in enumerate(lengths):
        r = slice(cp[s], cp[s] + L)
        one = [0, L]
        g = None if grid is None else grid[s:s + 1]
        qo, ko = oracle.qk_rmsnorm_rope(inp["q"][r], inp["k"][r], inp["w"], inp["w"], one, one,
                                        num_q_heads=H, num_k_heads=H, head_dim=D, rope_grid=g, sections=sec)
        assert np.array_equal(qo, outs[0][r]) and np.array_equal(ko, outs[1][r])
        m = inp["mod"][s:s + 1]
        ao = oracle.adaln_modulate(inp["x"][r], m[:, 0].copy(), m[:, 1].copy(), one, one, hidden=C)
        go = oracle.gated_residual(inp["x"][r], inp["y"][r], m[:, 2].copy(), one, one, hidden=C)
        so = oracle.swiglu(inp["a"][r], inp["b"][r], one, one, inner=I)
        assert np.array_equal(ao, outs[2][r]) and np.array_equal(go, outs[3][r])
        assert np.array_equal(so, outs[4][r])


def test_zero_length_sequences_and_empty_batch():
    rng = np.random.default_rng(2)
    lengths, padded = [0, 4, 0], [0, 4, 3]
    inp, valid, outs = all_ops(lengths, padded, rng)
    assert list(valid) == [0, 1, 2, 3]
    assert np.all(outs[4][4:] == SENT)
    # no sequences at all: nothing is computed, nothing is written
    e = np.zeros((0, 64), np.uint16)
    assert oracle.swiglu(e, e, [0], [0], inner=64).shape == (0, 64)


def test_row_subset_matches_full_run():
    rng = np.random.default_rng(3)
    lengths, padded = [9, 5], [12, 8]
    full = all_ops(lengths, padded, np.random.default_rng(3))
    rows = np.array([0, 8, 10, 12, 16, 19], dtype=np.int64)  # includes padding rows 10, 19
    sub = all_ops(lengths, padded, np.random.default_rng(3), rows=rows)
    valid_sel = [0, 8, 12, 16]
    for f, s in zip(full[2], sub[2]):
        assert np.array_equal(f[valid_sel], s[valid_sel])


def test_malformed_descriptors_are_rejected():
    x = np.zeros((4, 8), np.uint16)
    g = np.zeros((1, 8), np.uint16)
    for cs, cp in [([0, 5], [0, 4]),      # longer than its padded slot
                   ([1, 3], [0, 4]),      # does not start at 0
                   ([0, 3, 2], [0, 2, 4]),  # decreasing
                   ([0, 3], [0, 5])]:     # beyond the buffer
        with pytest.raises(ValueError):
            oracle.gated_residual(x, x, g, cs, cp, hidden=8)
