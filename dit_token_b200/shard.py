"""Row and head sharding of a packed batch across ranks (host logic, numpy only).

The operators are row-local, so a packed batch splits across ranks with no
exchange: rank r takes a contiguous range of the valid tokens, balanced by
count.  A sequence cut by a range boundary becomes a piece on each side; a
piece's rows keep their whole-sequence positions through `pos_offset` (the
index of its first row in the whole sequence), so rotary embedding sees the
same positions as the unsharded batch -- each rank computes only its own
rotary rows ("Why Real-Time MiniMax H3 Serving Requires More Than a Faster
DiT", "Key takeaways", bullet 1).  A sequence's suffix padding goes with the
piece that ends it, so every shard is again a suffix-padded packing.

`shard_packing` returns the shard's descriptors plus `rows`, the padded row of
the full buffer that each shard row comes from; the shards' `rows` partition
the full buffer's rows.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class Shard:
    rank: int
    world: int
    seq: np.ndarray                 # int32 [n]: the full batch's sequence index of each piece
    pos_offset: np.ndarray          # int32 [n]: whole-sequence index of each piece's first row
    cu_seqlens: np.ndarray          # int32 [n + 1]
    cu_seqlens_padded: np.ndarray   # int32 [n + 1]
    rope_grid: Optional[np.ndarray]  # int32 [n, 3] (the pieces' sequences' grids) or None
    rows: np.ndarray                # int64 [num_rows_padded]: source row in the full buffer

    @property
    def num_seqs(self) -> int:
        return int(self.seq.size)

    @property
    def num_rows_padded(self) -> int:
        return int(self.rows.size)

    @property
    def num_valid(self) -> int:
        return int(self.cu_seqlens[-1])


def token_range(total: int, rank: int, world: int) -> tuple:
    """[t0, t1): the valid-token ordinals rank `rank` of `world` owns."""
    return rank * total // world, (rank + 1) * total // world


def shard_packing(cu_seqlens, cu_seqlens_padded, rope_grid, rank: int, world: int) -> Shard:
    cs = np.asarray(cu_seqlens, dtype=np.int64)
    cp = np.asarray(cu_seqlens_padded, dtype=np.int64)
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if cs.ndim != 1 or cs.shape != cp.shape or cs.size < 1:
        raise ValueError("cu_seqlens and cu_seqlens_padded must be vectors of num_seqs + 1 entries")
    B = cs.size - 1
    grid = None if rope_grid is None else np.asarray(rope_grid, dtype=np.int64).reshape(B, 3)
    total = int(cs[-1])
    t0, t1 = token_range(total, rank, world)

    def owner(pos: int) -> int:
        # the rank whose token range holds ordinal pos (the last rank for pos == total)
        for r in range(world):
            a, e = token_range(total, r, world)
            if a <= pos < e:
                return r
        return world - 1

    seq, off, n_valid, n_pad, rows = [], [], [], [], []
    for b in range(B):
        L = int(cs[b + 1] - cs[b])
        P = int(cp[b + 1] - cp[b])
        if L == 0:
            if owner(int(cs[b])) != rank:
                continue
            a, e = int(cs[b]), int(cs[b])
        else:
            a, e = max(int(cs[b]), t0), min(int(cs[b + 1]), t1)
            if a >= e:
                continue
        o = a - int(cs[b])
        n = e - a
        pad = (P - L) if e == int(cs[b + 1]) else 0
        seq.append(b)
        off.append(o)
        n_valid.append(n)
        n_pad.append(n + pad)
        rows.append(np.arange(int(cp[b]) + o, int(cp[b]) + o + n + pad, dtype=np.int64))
    cu = np.zeros(len(seq) + 1, dtype=np.int32)
    cu_p = np.zeros(len(seq) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(n_valid, dtype=np.int64)
    cu_p[1:] = np.cumsum(n_pad, dtype=np.int64)
    return Shard(rank, world, np.asarray(seq, dtype=np.int32), np.asarray(off, dtype=np.int32), cu, cu_p,
                 None if grid is None else grid[np.asarray(seq, dtype=np.int64)].astype(np.int32),
                 np.concatenate(rows) if rows else np.zeros(0, dtype=np.int64))


def head_range(num_q_heads: int, num_k_heads: int, rank: int, world: int) -> tuple:
    """(q_first, q_count, k_first, k_count): the heads rank `rank` of `world`
    holds when Q/K are split by heads instead of rows (the layout after a
    sequence-to-head all-to-all).  Every rank keeps all rows, so positions
    need no offsets; the per-head normalisation and rotation are independent
    of the other heads, and a rank's call on its heads (a column slice of the
    whole buffer, or its own contiguous buffer) equals those columns of the
    whole call.  q heads split evenly; k heads split evenly when there are at
    least as many as ranks, else each is replicated on world / num_k_heads
    ranks -- either way the rank holds exactly the k heads its q heads attend
    with under grouped-query attention (q head h uses k head
    h // (num_q_heads / num_k_heads))."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if num_q_heads < 1 or num_k_heads < 1 or num_q_heads % num_k_heads:
        raise ValueError("num_q_heads must be a positive multiple of num_k_heads")
    if num_q_heads % world:
        raise ValueError(f"{num_q_heads} q heads do not split over {world} ranks")
    if num_k_heads >= world:
        if num_k_heads % world:
            raise ValueError(f"{num_k_heads} k heads do not split over {world} ranks")
        kc = num_k_heads // world
        return rank * (num_q_heads // world), num_q_heads // world, rank * kc, kc
    if world % num_k_heads:
        raise ValueError(f"{num_k_heads} k heads do not replicate evenly over {world} ranks")
    return rank * (num_q_heads // world), num_q_heads // world, rank * num_k_heads // world, 1
