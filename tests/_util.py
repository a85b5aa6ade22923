"""Small helpers shared by the tests (input construction only, no operator math)."""
import json
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
SENTINEL = 0x7FC1


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def bits(values) -> np.ndarray:
    """float values -> bf16 bit patterns (uint16) by torch's round-to-nearest-even."""
    t = torch.as_tensor(np.asarray(values, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def tbits(t: torch.Tensor) -> np.ndarray:
    """A bf16 torch tensor's bit patterns as a numpy uint16 array."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(b) -> np.ndarray:
    """bf16 bit patterns -> exact fp64 values."""
    b = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def cu(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


def packed(lengths, padded, width, rng, scale=1.0, fill=SENTINEL):
    """A [sum(padded), width] bf16 bit buffer: N(0, scale^2) on valid rows,
    ``fill`` on padding rows.  Returns (bits, valid_row_indices)."""
    rows = int(sum(padded))
    buf = np.full((rows, width), fill, dtype=np.uint16)
    cp = cu(padded)
    valid = []
    for b, L in enumerate(lengths):
        r = np.arange(cp[b], cp[b] + L)
        buf[r] = bits(rng.standard_normal((L, width)) * scale)
        valid.extend(r.tolist())
    return buf, np.asarray(valid, dtype=np.int64)
