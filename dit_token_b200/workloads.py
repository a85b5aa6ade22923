"""Seeded synthetic workloads for the fused per-token DiT operators.

This module holds shapes, the packed-sequence descriptors (``cu_seqlens``,
``cu_seqlens_padded``, per-sequence rope grids) and seeded random draws --
and none of the operators' arithmetic.  It is the one module that both the
CUDA path's tests/benchmark and the CPU oracle's checks take inputs from.

The workloads stand in for the MiniMax H3 DiT requests described in "Why
Real-Time MiniMax H3 Serving Requires More Than a Faster DiT" (a packed
audio-video sequence with valid lengths and structural suffix padding, "Key
takeaways", bullet 1); the pages print no tensor shapes, so the shapes below
are the five stated workload configurations:

=================  ====  ======================  =======  ======  ======  =====
name               seqs  valid rows              padded   hidden  heads   inner
=================  ====  ======================  =======  ======  ======  =====
tiny               1     200                     256      256     4x64    512
single_stream      1     8192                    8320     2048    16x128  5632
video              1     16x24x42 + 128 audio    16384    3072    24x128  8192
long_video         1     61x24x42 + 400 audio    61952    3072    24x128  8192
batched_varlen     4     U[1024, 30000] each     x128     5120    40x128  13824
long_video_slice   1     7336 video + 400 audio  7800     3072    24x128  8192
=================  ====  ======================  =======  ======  ======  =====

``long_video_slice`` is the share one rank holds when long_video's rows are
split over 8 ranks (the serving configuration runs 8-way sequence
parallelism, "MiniMax H3 通过 vLLM-Omni 实现 FastH3 实时推理", "FastH3
推理配置"): rank 7 of 8 in ``shard.shard_packing``, i.e. whole-sequence rows
54152 .. 61887 (the last 7336 video rows, the 400 audio rows) and the 64
padding rows, with ``pos_offset`` = 54152 so its rows keep their
whole-sequence rotary positions.

Value distributions: activations N(0, 1); RMSNorm weights 1 + N(0, 0.02);
modulation vectors (shift, scale, gate) N(0, 0.1).  Draws are fp32 normals
from numpy's PCG64, split into fixed 4 Mi-element chunks with one child seed
each (so the values do not depend on the thread count), then rounded to bf16
by torch.  Padding rows and two canary rows before and after every
row-indexed buffer hold the bf16 quiet NaN 0x7FC1.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass
from typing import Optional, Tuple

import numpy as np
import torch

SENTINEL = 0x7FC1  # bf16 quiet NaN with a payload: padding and canary rows
CANARY_ROWS = 2
_CHUNK = 1 << 22

# Child-seed slots: one per tensor, so building one operator's inputs never
# shifts another's values.
_SLOT = {"q": 0, "k": 1, "q_weight": 2, "k_weight": 3, "adaln_x": 4, "mod": 5,
         "res_x": 6, "res_y": 7, "ab": 8, "mod_av": 9}

WORKLOAD_NAMES = ("tiny", "single_stream", "video", "long_video", "batched_varlen", "long_video_slice")

# The rank whose share of long_video is long_video_slice, and the rank count.
SLICE_RANK, SLICE_WORLD = 7, 8

# Video latent frame of the video-shaped workloads: H x W = 24 x 42.
_FRAME_H, _FRAME_W = 24, 42


@dataclass(frozen=True)
class Workload:
    """One packed, suffix-padded batch of sequences and the operator shapes."""
    name: str
    lengths: Tuple[int, ...]            # valid rows per sequence
    padded: Tuple[int, ...]             # padded rows per sequence (>= lengths)
    hidden: int
    num_q_heads: int
    num_k_heads: int
    head_dim: int
    inner: int
    grids: Optional[Tuple[Tuple[int, int, int], ...]] = None  # (T, H, W) per sequence
    sections: Tuple[int, int, int] = (0, 0, 0)                # t/h/w widths of head_dim
    rope_theta: float = 10000.0
    eps: float = 1e-6
    seed: int = 0
    # whole-sequence index of each sequence's first row (one rank's slice of
    # longer sequences), or None: every sequence starts at its row 0
    pos_offset: Optional[Tuple[int, ...]] = None

    @property
    def num_seqs(self) -> int:
        return len(self.lengths)

    @property
    def num_valid(self) -> int:
        return int(sum(self.lengths))

    @property
    def num_rows_padded(self) -> int:
        return int(sum(self.padded))

    @property
    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.lengths)]).astype(np.int32)

    @property
    def cu_seqlens_padded(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.padded)]).astype(np.int32)

    @property
    def rope_grid(self) -> Optional[np.ndarray]:
        if self.grids is None:
            return None
        return np.asarray(self.grids, dtype=np.int32).reshape(-1, 3)

    @property
    def pos_offsets(self) -> Optional[np.ndarray]:
        return None if self.pos_offset is None else np.asarray(self.pos_offset, dtype=np.int32)

    @property
    def qk_width(self) -> Tuple[int, int]:
        return self.num_q_heads * self.head_dim, self.num_k_heads * self.head_dim

    def valid_rows(self) -> np.ndarray:
        """Padded row indices of every valid row, in order."""
        cp = self.cu_seqlens_padded
        return np.concatenate([np.arange(cp[b], cp[b] + L, dtype=np.int64)
                               for b, L in enumerate(self.lengths)]) if self.lengths else \
            np.zeros(0, np.int64)

    def padding_rows(self) -> np.ndarray:
        cp = self.cu_seqlens_padded
        parts = [np.arange(cp[b] + L, cp[b + 1], dtype=np.int64) for b, L in enumerate(self.lengths)]
        return np.concatenate(parts) if parts else np.zeros(0, np.int64)


def _round_up(n: int, m: int) -> int:
    return -(-n // m) * m


def workload(name: str, seed: int = 0) -> Workload:
    """The named workload; ``seed`` also draws the batched-varlen lengths."""
    if name == "tiny":
        return Workload(name, (200,), (256,), 256, 4, 4, 64, 512, seed=seed)
    if name == "single_stream":
        return Workload(name, (8192,), (8320,), 2048, 16, 16, 128, 5632, seed=seed)
    if name in ("video", "long_video"):
        T, audio = (16, 128) if name == "video" else (61, 400)
        n = T * _FRAME_H * _FRAME_W + audio
        return Workload(name, (n,), (_round_up(n, 256),), 3072, 24, 24, 128, 8192,
                        grids=((T, _FRAME_H, _FRAME_W),), sections=(44, 42, 42), seed=seed)
    if name == "batched_varlen":
        lengths = tuple(int(v) for v in np.random.default_rng(seed).integers(1024, 30001, 4))
        padded = tuple(_round_up(L, 128) for L in lengths)
        # Each request: floor(L / 1008) video frames of 24 x 42 latents, the
        # remaining rows a 1D (audio) tail.
        grids = tuple((L // (_FRAME_H * _FRAME_W), _FRAME_H, _FRAME_W) for L in lengths)
        return Workload(name, lengths, padded, 5120, 40, 40, 128, 13824,
                        grids=grids, sections=(44, 42, 42), seed=seed)
    if name == "long_video_slice":
        from .shard import shard_packing
        full = workload("long_video", seed)
        sh = shard_packing(full.cu_seqlens, full.cu_seqlens_padded, full.rope_grid, SLICE_RANK, SLICE_WORLD)
        return Workload(name, tuple(int(v) for v in np.diff(sh.cu_seqlens)),
                        tuple(int(v) for v in np.diff(sh.cu_seqlens_padded)), full.hidden, full.num_q_heads,
                        full.num_k_heads, full.head_dim, full.inner,
                        grids=tuple(tuple(int(t) for t in g) for g in sh.rope_grid), sections=full.sections,
                        seed=seed, pos_offset=tuple(int(v) for v in sh.pos_offset))
    raise KeyError(f"unknown workload {name!r}; known: {WORKLOAD_NAMES}")


def scaled(w: Workload, factor: float) -> Workload:
    """The same workload with every sequence's valid length scaled by
    ``factor`` (a smaller or larger batch of the same shapes): padding keeps
    the workload's granularity and video grids keep their 24 x 42 frames."""
    if factor == 1.0:
        return w
    gran = {"tiny": 256, "single_stream": 128, "video": 256, "long_video": 256, "batched_varlen": 128}
    g = gran.get(w.name.split("@")[0], 8)
    lengths = tuple(max(1, int(round(L * factor))) for L in w.lengths)
    padded = tuple(_round_up(L, g) for L in lengths)
    grids = None
    if w.grids is not None:
        frame = _FRAME_H * _FRAME_W
        if w.name.startswith("batched_varlen"):
            grids = tuple((L // frame, _FRAME_H, _FRAME_W) for L in lengths)
        else:  # keep the audio tail, shrink the frames
            grids = tuple((max(0, (L - (L0 - T * H * Wd)) // frame), _FRAME_H, _FRAME_W)
                          for L, L0, (T, H, Wd) in zip(lengths, w.lengths, w.grids))
    if w.pos_offset is not None:
        raise ValueError(f"{w.name} is a slice of longer sequences and cannot be scaled")
    return Workload(f"{w.name}@{factor:g}", lengths, padded, w.hidden, w.num_q_heads, w.num_k_heads,
                    w.head_dim, w.inner, grids, w.sections, w.rope_theta, w.eps, w.seed)


def custom(name: str, lengths, padded, *, hidden, num_q_heads, num_k_heads, head_dim, inner,
           grids=None, sections=(0, 0, 0), rope_theta=10000.0, eps=1e-6, seed=0) -> Workload:
    """A workload with explicit shapes (edge cases, small ragged tests)."""
    return Workload(name, tuple(int(v) for v in lengths), tuple(int(v) for v in padded), hidden,
                    num_q_heads, num_k_heads, head_dim, inner,
                    None if grids is None else tuple(tuple(int(t) for t in g) for g in grids),
                    tuple(sections), float(rope_theta), float(eps), seed)


# ------------------------------------------------------------ random draws

def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def normal_bf16(shape, seed_seq: np.random.SeedSequence, mean: float = 0.0,
                std: float = 1.0, dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """A CPU bf16 tensor of N(mean, std^2) draws, deterministic in seed_seq.
    With dtype=torch.float32 the same draws are returned unrounded (the bf16
    tensor is their round-to-nearest-even image)."""
    n = int(math.prod(shape))
    out = torch.empty(n, dtype=dtype)
    nchunks = max(1, -(-n // _CHUNK))
    children = seed_seq.spawn(nchunks)

    def fill(i):
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        if lo >= hi:
            return
        z = np.random.Generator(np.random.PCG64(children[i])).standard_normal(hi - lo, dtype=np.float32)
        if std != 1.0:
            z *= np.float32(std)
        if mean != 0.0:
            z += np.float32(mean)
        out[lo:hi] = torch.from_numpy(z)

    if nchunks == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nchunks)))
    return out.view(*shape)


def _seed(w: Workload, slot: str) -> np.random.SeedSequence:
    return np.random.SeedSequence(w.seed).spawn(len(_SLOT))[_SLOT[slot]]


def sentinel_like(shape) -> torch.Tensor:
    t = torch.empty(shape, dtype=torch.int16)
    t.fill_(SENTINEL)
    return t.view(torch.bfloat16)


def _row_buffer(w: Workload, width: int, slot: Optional[str]) -> torch.Tensor:
    """[canary + padded rows + canary, width]: seeded normals on valid rows
    (``slot`` given) or the sentinel everywhere (``slot`` None)."""
    rows = w.num_rows_padded + 2 * CANARY_ROWS
    if slot is None:
        return sentinel_like((rows, width))
    buf = normal_bf16((rows, width), _seed(w, slot))
    mask = np.ones(rows, dtype=bool)
    mask[CANARY_ROWS + w.valid_rows()] = False
    idx = torch.from_numpy(np.nonzero(mask)[0])
    buf.view(torch.int16)[idx] = SENTINEL
    return buf


def rows_view(buf: torch.Tensor) -> torch.Tensor:
    """The padded-row part of a buffer with canary rows on both ends."""
    return buf[CANARY_ROWS: buf.shape[0] - CANARY_ROWS]


def qk_inputs(w: Workload) -> dict:
    """q, k buffers [canary + rows + canary, heads * head_dim] (in place) and
    the two RMSNorm weight vectors."""
    qw, kw = w.qk_width
    return {
        "q": _row_buffer(w, qw, "q"),
        "k": _row_buffer(w, kw, "k"),
        "q_weight": normal_bf16((w.head_dim,), _seed(w, "q_weight"), mean=1.0, std=0.02),
        "k_weight": normal_bf16((w.head_dim,), _seed(w, "k_weight"), mean=1.0, std=0.02),
    }


def modulation(w: Workload, dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """Per-sequence modulation vectors [num_seqs, 6, hidden] ~ N(0, 0.1):
    (shift, scale, gate) of the attention sublayer, then of the MLP sublayer.
    Operators receive one slice with a sequence stride of 6 * hidden.  dtype
    float32 gives the same draws unrounded (a modulation head kept in fp32)."""
    return normal_bf16((w.num_seqs, 6, w.hidden), _seed(w, "mod"), std=0.1, dtype=dtype)


def modulation_av(w: Workload, dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """Per-stream modulation vectors [num_seqs, 2, 6, hidden] ~ N(0, 0.1):
    stream 0 for a request's video rows, stream 1 for its audio rows."""
    return normal_bf16((w.num_seqs, 2, 6, w.hidden), _seed(w, "mod_av"), std=0.1, dtype=dtype)


def adaln_inputs(w: Workload) -> dict:
    mod = modulation(w)
    return {"x": _row_buffer(w, w.hidden, "adaln_x"), "out": _row_buffer(w, w.hidden, None),
            "mod": mod, "shift": mod[:, 0], "scale": mod[:, 1], "mod_seq_stride": 6 * w.hidden}


def residual_inputs(w: Workload) -> dict:
    mod = modulation(w)
    return {"x": _row_buffer(w, w.hidden, "res_x"), "y": _row_buffer(w, w.hidden, "res_y"),
            "out": _row_buffer(w, w.hidden, None), "mod": mod, "gate": mod[:, 2],
            "gate_seq_stride": 6 * w.hidden}


def swiglu_inputs(w: Workload) -> dict:
    """A chunked [rows, 2 * inner] buffer: a = columns [0, inner), b = the rest."""
    ab = _row_buffer(w, 2 * w.inner, "ab")
    return {"ab": ab, "a": ab[:, : w.inner], "b": ab[:, w.inner:], "out": _row_buffer(w, w.inner, None)}


# Decoded-video frames of the pages' 10-second request: 243 frames of
# 1344 x 768 RGB ("MiniMax H3 通过 vLLM-Omni 实现 FastH3 实时推理", results and
# duration-sweep tables), in the decoder's channels-first layout.
FRAMES_SHAPE = (1, 3, 243, 768, 1344)


def frames_input(shape=FRAMES_SHAPE, seed: int = 0) -> torch.Tensor:
    """fp32 [B, C, T, H, W] decoder output: uniform in [-1.05, 1.05] (slightly
    past the nominal [-1, 1] so the clamps are exercised), seeded, chunked
    like the normal draws."""
    n = int(math.prod(shape))
    out = torch.empty(n, dtype=torch.float32)
    nchunks = max(1, -(-n // _CHUNK))
    children = np.random.SeedSequence(seed).spawn(nchunks)

    def fill(i):
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        g = np.random.Generator(np.random.PCG64(children[i]))
        out[lo:hi] = torch.from_numpy(g.uniform(-1.05, 1.05, hi - lo).astype(np.float32))

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(fill, range(nchunks)))
    return out.view(*shape)


def sample_rows(w: Workload, per_seq: int, seed: int = 1234) -> np.ndarray:
    """Padded indices of a seeded sample of valid rows: each sequence's first
    and last valid row, for a sequence with a T x H x W grid the rows at the
    grid's edges (local W - 1, H*W - 1, T*H*W - 1 -- the largest 3D position --
    and T*H*W, the first row after the grid), plus up to ``per_seq`` others."""
    rng = np.random.default_rng(seed)
    cp = w.cu_seqlens_padded
    picks = []
    for b, L in enumerate(w.lengths):
        if L == 0:
            continue
        local = {0, L - 1}
        if w.grids is not None:
            T, H, Wd = w.grids[b]
            off = 0 if w.pos_offset is None else w.pos_offset[b]
            local.update(r - off for r in (Wd - 1, H * Wd - 1, T * H * Wd - 1, T * H * Wd) if 0 <= r - off < L)
        local.update(int(v) for v in rng.choice(L, size=min(per_seq, L), replace=False))
        picks.extend(cp[b] + np.array(sorted(local), dtype=np.int64))
    return np.asarray(picks, dtype=np.int64)
