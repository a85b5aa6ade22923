"""Pins of the oracle's bf16 conversions against the IEEE definition and torch."""
import math

import numpy as np
import torch

import oracle
from _util import golden


def test_roundtrip_every_finite_pattern():
    # bf16 -> f64 is exact, so every non-NaN pattern must come back unchanged.
    for h in range(1 << 16):
        if (h & 0x7F80) == 0x7F80 and (h & 0x007F):
            continue  # NaN payloads
        assert oracle.f64_to_bf16(oracle.bf16_to_f64(h)) == h, hex(h)


def test_widening_is_upper_half_of_binary32():
    rng = np.random.default_rng(0)
    for h in rng.integers(0, 1 << 16, 2000):
        h = int(h)
        if (h & 0x7F80) == 0x7F80 and (h & 0x007F):
            continue
        f = np.array([h << 16], dtype=np.uint32).view(np.float32)[0]
        assert oracle.bf16_to_f64(h) == float(f)


def test_golden_ties_and_edges():
    for c in golden("bf16_rounding.json")["cases"]:
        assert oracle.f64_to_bf16(float.fromhex(c["x"])) == c["bits"], c["what"]


def test_matches_torch_rne_on_binary32_values():
    # For a value that is exactly a binary32 number, one rounding to bf16 is
    # what torch's float32 -> bfloat16 conversion does (RNE).
    rng = np.random.default_rng(1)
    u = rng.integers(0, 1 << 32, 100_000, dtype=np.uint64).astype(np.uint32)
    f = u.view(np.float32)
    f = f[np.isfinite(f)]
    f = np.concatenate([f, (rng.standard_normal(50_000) * 10.0 ** rng.integers(-40, 38, 50_000)).astype(np.float32)])
    f = f[np.isfinite(f)]
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f64_to_bf16_array(f.astype(np.float64))
    assert np.array_equal(got, want)


def test_nan_and_inf():
    assert oracle.f64_to_bf16(math.inf) == 0x7F80
    assert oracle.f64_to_bf16(-math.inf) == 0xFF80
    n = oracle.f64_to_bf16(math.nan)
    assert (n & 0x7F80) == 0x7F80 and (n & 0x7F)
