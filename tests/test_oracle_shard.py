"""Pins of the oracle's position offsets (one rank's slice of longer
sequences) and of the host sharding helper: cutting a packed batch into
contiguous per-rank slices, with each slice's rows keeping their
whole-sequence positions, must reproduce the unsharded results row for row
for every operator, at several world sizes; the slices' rows partition the
buffer."""
import numpy as np
import pytest

import oracle
from dit_token_b200.shard import head_range, shard_packing
from _util import bits, cu

# sequences: 3D video (24 rows) + 9 audio rows, a 1D one, an empty one, 3D only
LENGTHS = [33, 17, 0, 12]
PADDED = [40, 24, 8, 16]
GRID = np.array([[2, 3, 4], [0, 0, 0], [0, 0, 0], [2, 2, 3]], dtype=np.int32)
H, D = 2, 64
SEC = (24, 20, 20)


def batch(C, seed):
    rng = np.random.default_rng(seed)
    rows = sum(PADDED)
    x = bits(rng.standard_normal((rows, C)))
    y = bits(rng.standard_normal((rows, C)))
    mod = bits(rng.standard_normal((len(LENGTHS), 2, 6, C)) * 0.1)   # per-stream sets
    return x, y, mod


def valid_rows(cs, cp):
    return np.concatenate([np.arange(cp[b], cp[b] + cs[b + 1] - cs[b]) for b in range(len(cs) - 1)])


def run_all(x, y, mod, cs, cp, grid, pos_offset, C):
    """Every operator on one packing; returns a dict of output bit arrays."""
    flat = np.ascontiguousarray(mod.reshape(-1))
    out = {}
    out["q"], out["k"] = oracle.qk_rmsnorm_rope(x[:, : H * D], y[:, : H * D], bits(np.linspace(0.5, 1.5, D)),
                                                bits(np.linspace(1.5, 0.5, D)), cs, cp, num_q_heads=H,
                                                num_k_heads=H, head_dim=D, rope_grid=grid, sections=SEC,
                                                q_row_stride=C, k_row_stride=C, pos_offset=pos_offset)
    out["qh"], _ = oracle.qk_rmsnorm_rope(x[:, : H * D], y[:, : H * D], bits(np.ones(D)), bits(np.ones(D)), cs, cp,
                                          num_q_heads=H, num_k_heads=H, head_dim=D, rope_grid=grid, sections=SEC,
                                          q_row_stride=C, k_row_stride=C, pos_offset=pos_offset, rope_mode="half")
    av = dict(rope_grid=grid, pos_offset=pos_offset)
    out["adaln"] = oracle.adaln_modulate(x, flat, flat[C:], cs, cp, hidden=C, mod_seq_stride=12 * C,
                                         audio_offset=6 * C, **av)
    out["res"] = oracle.gated_residual(x, y, flat[2 * C:], cs, cp, hidden=C, gate_seq_stride=12 * C,
                                       audio_offset=6 * C, **av)
    out["fres"], out["fnorm"] = oracle.gated_residual_adaln(
        x, y, flat[2 * C:], flat[3 * C:], flat[4 * C:], cs, cp, hidden=C, gate_seq_stride=12 * C,
        mod_seq_stride=12 * C, gate_audio_offset=6 * C, mod_audio_offset=6 * C, **av)
    out["swiglu"] = oracle.swiglu(x, y, cs, cp, inner=C)
    return out


@pytest.mark.parametrize("world", [2, 3, 5])
def test_shards_reproduce_the_whole_batch(world):
    C = 128
    x, y, mod = batch(C, world)
    cs, cp = cu(LENGTHS), cu(PADDED)
    full = run_all(x, y, mod, cs, cp, GRID, None, C)
    full_valid = set(valid_rows(cs, cp).tolist())
    seen = []
    for rank in range(world):
        sh = shard_packing(cs, cp, GRID, rank, world)
        seen.append(sh.rows)
        if sh.num_rows_padded == 0:
            continue
        part = run_all(x[sh.rows], y[sh.rows], mod[sh.seq], sh.cu_seqlens, sh.cu_seqlens_padded, sh.rope_grid,
                       sh.pos_offset, C)
        local_valid = valid_rows(sh.cu_seqlens, sh.cu_seqlens_padded)
        assert all(int(sh.rows[i]) in full_valid for i in local_valid)
        for name, arr in part.items():
            assert np.array_equal(arr[local_valid], full[name][sh.rows[local_valid]]), (world, rank, name)
    # the shards' rows, in rank order, are the buffer's rows, each once
    assert np.array_equal(np.concatenate(seen), np.arange(sum(PADDED)))


def test_shard_boundaries_and_offsets():
    cs, cp = cu(LENGTHS), cu(PADDED)
    total = cs[-1]
    sizes = [shard_packing(cs, cp, GRID, r, 4).num_valid for r in range(4)]
    assert sum(sizes) == total and max(sizes) - min(sizes) <= 1
    sh = shard_packing(cs, cp, GRID, 1, 4)            # tokens 15 .. 30: the middle of sequence 0
    assert sh.seq.tolist() == [0] and sh.pos_offset.tolist() == [15] and sh.num_valid == 16
    assert sh.num_rows_padded == 16                    # sequence 0 goes on: no padding here
    last = shard_packing(cs, cp, GRID, 3, 4)
    assert last.seq.tolist() == [1, 2, 3]             # the empty sequence rides with its neighbour
    assert last.pos_offset.tolist() == [13, 0, 0]     # tokens 46 .. 49 are rows 13 .. 16 of sequence 1
    assert last.cu_seqlens_padded[-1] == last.num_rows_padded


def test_offset_zero_is_the_plain_call():
    C = 128
    x, y, mod = batch(C, 9)
    cs, cp = cu(LENGTHS), cu(PADDED)
    a = run_all(x, y, mod, cs, cp, GRID, None, C)
    b = run_all(x, y, mod, cs, cp, GRID, np.zeros(len(LENGTHS), np.int32), C)
    for name in a:
        assert np.array_equal(a[name], b[name]), name


def test_more_ranks_than_tokens_and_empty_batches():
    cs, cp = cu([2, 0, 1]), cu([8, 8, 8])
    shards = [shard_packing(cs, cp, None, r, 8) for r in range(8)]
    assert sum(s.num_valid for s in shards) == 3
    assert np.array_equal(np.concatenate([s.rows for s in shards]), np.arange(24))
    assert all(s.rope_grid is None for s in shards)
    for s in shards:                                   # every shard is a well-formed packing
        assert s.cu_seqlens[0] == 0 and s.cu_seqlens_padded[0] == 0
        assert np.all(np.diff(s.cu_seqlens) <= np.diff(s.cu_seqlens_padded))
        assert s.cu_seqlens_padded[-1] == s.num_rows_padded
    empty = [shard_packing(cu([0, 0]), cu([4, 4]), None, r, 3) for r in range(3)]
    assert [e.num_seqs for e in empty] == [0, 0, 2]    # padding-only sequences go to the last rank
    assert np.array_equal(empty[2].rows, np.arange(8))
    with pytest.raises(ValueError):
        shard_packing(cs, cp, None, 3, 3)


@pytest.mark.parametrize("Hq,Hk,world", [(8, 8, 2), (8, 2, 2), (8, 2, 4), (8, 2, 8), (24, 4, 8), (40, 8, 4), (6, 1, 3)])
def test_head_range_covers_every_head_with_its_group(Hq, Hk, world):
    """q heads partition over the ranks; a rank holds exactly the k heads its
    q heads use under grouped-query attention (q head h -> k head h // (Hq/Hk))."""
    seen = []
    for r in range(world):
        q0, qc, k0, kc = head_range(Hq, Hk, r, world)
        seen += list(range(q0, q0 + qc))
        assert set(range(k0, k0 + kc)) == {h // (Hq // Hk) for h in range(q0, q0 + qc)}
    assert seen == list(range(Hq))


def test_head_range_rejects_uneven_splits():
    for args in [(8, 2, 3), (8, 3, 2), (6, 2, 4), (12, 4, 8), (8, 2, 2 * 8)]:
        with pytest.raises(ValueError):
            head_range(*args[:2], 0, args[2])
    with pytest.raises(ValueError):
        head_range(8, 2, 2, 2)


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("mode", ["interleaved", "half"])
def test_head_slices_reproduce_the_whole_call(world, mode):
    """The normalisation and rotation of one head read no other head: each
    rank's oracle call on its heads (every row, its own columns) equals those
    columns of the call on all heads.  A norm taken over the whole row instead
    of per head fails this."""
    Hq, Hk = 4, 2
    rng = np.random.default_rng(21)
    rows = sum(PADDED)
    q = bits(rng.standard_normal((rows, Hq * D)) * np.repeat(rng.uniform(0.2, 5.0, Hq), D))
    k = bits(rng.standard_normal((rows, Hk * D)) * np.repeat(rng.uniform(0.2, 5.0, Hk), D))
    wq, wk = bits(np.linspace(0.5, 1.5, D)), bits(np.linspace(1.5, 0.5, D))
    cs, cp = cu(LENGTHS), cu(PADDED)
    kw = dict(head_dim=D, rope_grid=GRID, sections=SEC, rope_mode=mode)
    qf, kf = oracle.qk_rmsnorm_rope(q, k, wq, wk, cs, cp, num_q_heads=Hq, num_k_heads=Hk, **kw)
    for r in range(world):
        q0, qc, k0, kc = head_range(Hq, Hk, r, world)
        qsl, ksl = slice(q0 * D, (q0 + qc) * D), slice(k0 * D, (k0 + kc) * D)
        qo, ko = oracle.qk_rmsnorm_rope(np.ascontiguousarray(q[:, qsl]), np.ascontiguousarray(k[:, ksl]), wq, wk,
                                        cs, cp, num_q_heads=qc, num_k_heads=kc, **kw)
        assert np.array_equal(qo, qf[:, qsl]), (r, "q")
        assert np.array_equal(ko, kf[:, ksl]), (r, "k")
