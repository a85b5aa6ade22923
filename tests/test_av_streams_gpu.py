"""Per-stream (video / audio) modulation on the GPU: the descriptor kernel
behind dit_av_stream_seqlens is checked bit for bit against its definition,
and the modulated ops run on that descriptor are checked against the
oracle's per-stream modulation, which works from the original descriptor
and the grid (it shares nothing with the descriptor trick)."""
import numpy as np
import pytest
import torch

import dit_token_b200 as dit
from dit_token_b200 import workloads as W
import _parity as P
from _util import tbits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dit_token_b200 import build
    build.build()


def expected_split(cs, cp, grid):
    B = len(cs) - 1
    o_cs = np.zeros(2 * B + 1, np.int64)
    o_cp = np.zeros(2 * B + 1, np.int64)
    o_cs[0], o_cp[0] = cs[0], cp[0]
    for b in range(B):
        L, room = cs[b + 1] - cs[b], cp[b + 1] - cp[b]
        thw = int(grid[b, 0]) * int(grid[b, 1]) * int(grid[b, 2])
        v = min(max(thw, 0), max(min(L, room), 0))
        o_cs[2 * b + 1], o_cs[2 * b + 2] = cs[b] + v, cs[b + 1]
        o_cp[2 * b + 1], o_cp[2 * b + 2] = cp[b] + v, cp[b + 1]
    return o_cs.astype(np.int32), o_cp.astype(np.int32)


def run_split(cs, cp, grid):
    a, b = dit.dit_av_stream_seqlens(torch.from_numpy(np.asarray(cs, np.int32)).cuda(),
                                     torch.from_numpy(np.asarray(cp, np.int32)).cuda(),
                                     torch.from_numpy(np.ascontiguousarray(grid, np.int32)).cuda())
    return a.cpu().numpy(), b.cpu().numpy()


def test_descriptor_matches_its_definition():
    cases = []
    for name in ("video", "long_video", "batched_varlen"):
        w = W.workload(name)
        cases.append((w.cu_seqlens, w.cu_seqlens_padded, w.rope_grid))
    rng = np.random.default_rng(9)
    B = 2500
    lengths = rng.integers(0, 300, B)
    padded = lengths + rng.integers(0, 20, B)
    grid = rng.integers(0, 9, (B, 3))            # T*H*W below, at and above the length
    cases.append((np.concatenate([[0], np.cumsum(lengths)]), np.concatenate([[0], np.cumsum(padded)]), grid))
    cases.append(([0, 5, 5, 12], [0, 8, 8, 16], [[1, 2, 2], [3, 3, 3], [100, 1, 1]]))
    for cs, cp, grid in cases:
        grid = np.asarray(grid, np.int32)
        got = run_split(cs, cp, grid)
        want = expected_split(np.asarray(cs, np.int64), np.asarray(cp, np.int64), grid)
        assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1])
    # an empty batch still yields the one-entry descriptor
    a, b = dit.dit_av_stream_seqlens(torch.zeros(1, dtype=torch.int32, device="cuda"),
                                     torch.zeros(1, dtype=torch.int32, device="cuda"),
                                     torch.zeros((0, 3), dtype=torch.int32, device="cuda"))
    assert a.tolist() == [0] and b.tolist() == [0]


def boundary_rows(w):
    """Padded indices of the last video row and the first audio row of every
    sequence that has both."""
    out = []
    for b, L in enumerate(w.lengths):
        thw = int(np.prod(w.rope_grid[b]))
        for r in (thw - 1, thw):
            if 0 <= r < L:
                out.append(int(w.cu_seqlens_padded[b]) + r)
    return np.asarray(out, np.int64)


def av_case(name, per_seq):
    w = W.workload(name)
    rows = np.unique(np.concatenate([W.sample_rows(w, per_seq=per_seq), boundary_rows(w)]))
    return w, rows


@pytest.mark.parametrize("name", ["video", "long_video", "batched_varlen"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_per_stream_modulation_matches_the_oracle(name, dtype):
    w, rows = av_case(name, 24)
    C, B = w.hidden, w.num_seqs
    cs, cp, grid = P.device_packing(w)
    cs2, cp2 = dit.dit_av_stream_seqlens(cs, cp, grid)
    m = W.modulation_av(w, dtype)
    mv = m.cuda().view(2 * B, 6, C)
    flat = P.mod_flat(m)
    keep = P.untouched_rows(w)
    av = dict(rope_grid=w.rope_grid)

    inp = W.adaln_inputs(w)
    out = inp["out"].cuda()
    dit.dit_adaln_modulate(W.rows_view(inp["x"].cuda()), mv[:, 0], mv[:, 1], cs2, cp2, out=W.rows_view(out),
                           eps=w.eps)
    import oracle
    ref = oracle.adaln_modulate(tbits(W.rows_view(inp["x"])), flat, flat[C:], w.cu_seqlens, w.cu_seqlens_padded,
                                hidden=C, eps=w.eps, mod_seq_stride=12 * C, audio_offset=6 * C, rows=rows, **av)
    P.assert_close(P.gather_rows(out, rows), ref[rows], f"{name} adaln av")
    P.assert_untouched(out, inp["out"], keep, f"{name} adaln av")

    inp = W.residual_inputs(w)
    x, y = inp["x"].cuda(), inp["y"].cuda()
    out = inp["out"].cuda()
    dit.dit_gated_residual(W.rows_view(x), W.rows_view(y), mv[:, 2], cs2, cp2, out=W.rows_view(out))
    xb, yb = tbits(W.rows_view(inp["x"])), tbits(W.rows_view(inp["y"]))
    ref = oracle.gated_residual(xb, yb, flat[2 * C:], w.cu_seqlens, w.cu_seqlens_padded, hidden=C,
                                gate_seq_stride=12 * C, audio_offset=6 * C, rows=rows, **av)
    P.assert_close(P.gather_rows(out, rows), ref[rows], f"{name} residual av")
    P.assert_untouched(out, inp["out"], keep, f"{name} residual av")

    res = inp["out"].cuda()
    norm = W.sentinel_like(inp["out"].shape).cuda()
    dit.dit_gated_residual_adaln(W.rows_view(x), W.rows_view(y), mv[:, 2], mv[:, 3], mv[:, 4], cs2, cp2,
                                 res_out=W.rows_view(res), norm_out=W.rows_view(norm), eps=w.eps)
    r_ref, n_ref = oracle.gated_residual_adaln(xb, yb, flat[2 * C:], flat[3 * C:], flat[4 * C:], w.cu_seqlens,
                                               w.cu_seqlens_padded, hidden=C, eps=w.eps, gate_seq_stride=12 * C,
                                               mod_seq_stride=12 * C, gate_audio_offset=6 * C,
                                               mod_audio_offset=6 * C, rows=rows, **av)
    P.assert_close(P.gather_rows(res, rows), r_ref[rows], f"{name} fused residual av")
    P.assert_close(P.gather_rows(norm, rows), n_ref[rows], f"{name} fused norm av")
    assert torch.equal(res.view(torch.int16), out.view(torch.int16))
    P.assert_untouched(norm, inp["out"], keep, f"{name} fused norm av")


def test_same_vectors_on_both_streams_equal_the_single_set():
    w = W.workload("video")
    C, B = w.hidden, w.num_seqs
    cs, cp, grid = P.device_packing(w)
    cs2, cp2 = dit.dit_av_stream_seqlens(cs, cp, grid)
    m1 = W.modulation(w).cuda()                               # [B, 6, C]
    m2 = torch.stack([m1, m1], dim=1).contiguous().view(2 * B, 6, C)
    inp = W.adaln_inputs(w)
    x = W.rows_view(inp["x"].cuda())
    a = dit.dit_adaln_modulate(x, m1[:, 0], m1[:, 1], cs, cp, eps=w.eps)
    b = dit.dit_adaln_modulate(x, m2[:, 0], m2[:, 1], cs2, cp2, eps=w.eps)
    rows = torch.from_numpy(w.valid_rows()).cuda()
    assert torch.equal(a[rows].view(torch.int16), b[rows].view(torch.int16))
