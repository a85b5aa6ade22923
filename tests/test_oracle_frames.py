"""Pins of the oracle's frame conversion: hand-checked values of the mapping
(ends, midpoint tie, clamps, NaN), agreement with numpy's IEEE float32
arithmetic on random values including every tie, and the two layouts as
numpy transposes of the element-wise conversion."""
import numpy as np
import pytest

import oracle


def frames(vals):
    v = np.asarray(vals, dtype=np.float32)
    return v.reshape(1, 1, 1, 1, -1)


def test_hand_checked_values():
    x = frames([-1.0, 1.0, 0.0, -0.5, 0.5, 5.0, -3.0, np.nan, np.inf, -np.inf, 1.0 / 255.0 * 2 - 1])
    got = oracle.frames_to_u8(x).reshape(-1)
    # (x+1)*127.5: 0, 255, 127.5 -> 128 (tie to even), 63.75 -> 64, 191.25 -> 191,
    # clamps 255 / 0, NaN -> 0, +inf -> 255, -inf -> 0, (2/255)*127.5 ~ 1 -> 1
    assert got.tolist() == [0, 255, 128, 64, 191, 255, 0, 0, 255, 0, 1]


def test_ties_go_to_even():
    # x = k/127.5 - 1 + 1/255 lands on k + 0.5 only approximately in fp32;
    # build exact ties instead from u = k + 0.5 with x + 1 = u / 127.5 exactly:
    # u = 127.5 * (x + 1) is exact for x + 1 = m / 2^8 when 127.5 m / 2^8 has
    # few enough bits; pick x + 1 in {1/255 * ...} by scanning exact binary values.
    xs = np.arange(0, 512, dtype=np.float32) / np.float32(256.0) - np.float32(1.0)   # exact
    u = (xs + np.float32(1.0)) * np.float32(127.5)
    ties = np.abs(u - np.floor(u) - 0.5) == 0
    assert ties.any()
    got = oracle.frames_to_u8(frames(xs[ties])).reshape(-1).astype(np.int64)
    want = np.where(np.floor(u[ties]).astype(np.int64) % 2 == 0, np.floor(u[ties]), np.ceil(u[ties]))
    assert np.array_equal(got, want.astype(np.int64))


def test_matches_numpy_float32_arithmetic():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-1.2, 1.2, 200_000), rng.standard_normal(50_000) * 3,
                        np.arange(-1, 1.0001, 1 / 1024)]).astype(np.float32)
    t = (x + np.float32(1.0)).astype(np.float32)
    u = (t * np.float32(127.5)).astype(np.float32)
    want = np.rint(np.clip(u, 0, 255)).astype(np.uint8)
    got = oracle.frames_to_u8(frames(x)).reshape(-1)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("shape", [(1, 3, 2, 4, 16), (2, 3, 3, 5, 7), (1, 1, 2, 3, 4), (1, 4, 1, 2, 20)])
def test_layouts_are_transposes_of_the_elementwise_map(shape):
    rng = np.random.default_rng(1)
    x = rng.uniform(-1.1, 1.1, shape).astype(np.float32)
    flat = oracle.frames_to_u8(x.reshape(1, 1, 1, 1, -1)).reshape(shape)   # element-wise, same layout
    assert np.array_equal(oracle.frames_to_u8(x, layout=0), np.transpose(flat, (0, 2, 3, 4, 1)))
    assert np.array_equal(oracle.frames_to_u8(x, layout=1), np.transpose(flat, (0, 2, 1, 3, 4)))
