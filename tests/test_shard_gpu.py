"""One batch split into per-rank slices (dit_token_b200.shard), each slice run
on the GPU with its own descriptors and whole-sequence position offsets: every
operator's slice outputs equal the unsharded GPU run bit for bit, and the
Q/K slice outputs match the oracle's slice call.  The slices run one after
another on one GPU (no rank waits on another)."""
import numpy as np
import pytest
import torch

import dit_token_b200 as dit
from dit_token_b200 import workloads as W
from dit_token_b200.shard import head_range, shard_packing
import _parity as P
import oracle
from _util import tbits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dit_token_b200 import build
    build.build()


def ragged():
    return W.custom("sp", (700, 45, 0, 300), (704, 48, 8, 304), hidden=256, num_q_heads=3, num_k_heads=1,
                    head_dim=64, inner=264, grids=((4, 6, 25), (0, 0, 0), (0, 0, 0), (3, 5, 10)),
                    sections=(24, 20, 20), seed=2)


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def run_ops(w, x, y, q, k, wq, wk, mod, mav, cs, cp, grid, po):
    """All operators on one packing; q, k updated in place; returns outputs."""
    out = {}
    dit.dit_qk_rmsnorm_rope(q, k, wq, wk, cs, cp, num_q_heads=w.num_q_heads, num_k_heads=w.num_k_heads,
                            head_dim=w.head_dim, rope_grid=grid, sections=w.sections, rope_theta=w.rope_theta,
                            eps=w.eps, pos_offset=po)
    out["q"], out["k"] = q, k
    out["adaln"] = dit.dit_adaln_modulate(x, mod[:, 0], mod[:, 1], cs, cp, eps=w.eps)
    out["res"] = dit.dit_gated_residual(x, y, mod[:, 2], cs, cp)
    out["fres"], out["fnorm"] = dit.dit_gated_residual_adaln(x, y, mod[:, 2], mod[:, 3], mod[:, 4], cs, cp,
                                                             eps=w.eps)
    out["swiglu"] = dit.dit_swiglu(x, y, cs, cp)  # x, y as the two halves (inner = hidden)
    B = cs.numel() - 1
    cs2, cp2 = dit.dit_av_stream_seqlens(cs, cp, grid, pos_offset=po)
    mv = mav.view(2 * B, 6, w.hidden)
    out["adaln_av"] = dit.dit_adaln_modulate(x, mv[:, 0], mv[:, 1], cs2, cp2, eps=w.eps)
    return out


@pytest.mark.parametrize("name,world", [("ragged", 2), ("ragged", 3), ("batched_varlen", 4)])
def test_slices_equal_the_whole_batch(name, world):
    w = ragged() if name == "ragged" else W.workload(name)
    rv = W.rows_view
    qi, ri = W.qk_inputs(w), W.residual_inputs(w)
    x, y = rv(ri["x"]).cuda(), rv(ri["y"]).cuda()
    q0, k0 = rv(qi["q"]).cuda(), rv(qi["k"]).cuda()
    wq, wk = qi["q_weight"].cuda(), qi["k_weight"].cuda()
    mod = ri["mod"].cuda()
    mav = W.modulation_av(w).cuda()
    cs, cp, grid = P.device_packing(w)
    full = run_ops(w, x, y, q0.clone(), k0.clone(), wq, wk, mod, mav, cs, cp, grid, None)
    for rank in range(world):
        sh = shard_packing(w.cu_seqlens, w.cu_seqlens_padded, w.rope_grid, rank, world)
        if sh.num_rows_padded == 0:
            continue
        rows = torch.from_numpy(sh.rows).cuda()
        seqs = torch.from_numpy(sh.seq.astype(np.int64)).cuda()
        part = run_ops(w, x[rows], y[rows], q0[rows].contiguous(), k0[rows].contiguous(), wq, wk,
                       mod[seqs], mav[seqs].contiguous(), dev_i32(sh.cu_seqlens), dev_i32(sh.cu_seqlens_padded),
                       dev_i32(sh.rope_grid), dev_i32(sh.pos_offset))
        valid = torch.from_numpy(np.concatenate(
            [np.arange(sh.cu_seqlens_padded[i], sh.cu_seqlens_padded[i] + sh.cu_seqlens[i + 1] - sh.cu_seqlens[i])
             for i in range(sh.num_seqs)]).astype(np.int64)).cuda()
        for key, t in part.items():
            a = t[valid].view(torch.int16)
            b = full[key][rows[valid]].view(torch.int16)
            assert torch.equal(a, b), (name, world, rank, key)


def test_slice_qk_matches_the_oracle_slice_call():
    w = ragged()
    rv = W.rows_view
    qi = W.qk_inputs(w)
    q0, k0 = tbits(rv(qi["q"])), tbits(rv(qi["k"]))
    for rank in range(3):
        sh = shard_packing(w.cu_seqlens, w.cu_seqlens_padded, w.rope_grid, rank, 3)
        q = torch.from_numpy(q0[sh.rows].view(np.int16)).view(torch.bfloat16).cuda()
        k = torch.from_numpy(k0[sh.rows].view(np.int16)).view(torch.bfloat16).cuda()
        dit.dit_qk_rmsnorm_rope(q, k, qi["q_weight"].cuda(), qi["k_weight"].cuda(), dev_i32(sh.cu_seqlens),
                                dev_i32(sh.cu_seqlens_padded), num_q_heads=w.num_q_heads,
                                num_k_heads=w.num_k_heads, head_dim=w.head_dim, rope_grid=dev_i32(sh.rope_grid),
                                sections=w.sections, rope_theta=w.rope_theta, eps=w.eps,
                                pos_offset=dev_i32(sh.pos_offset))
        qo, ko = oracle.qk_rmsnorm_rope(q0[sh.rows], k0[sh.rows], tbits(qi["q_weight"]), tbits(qi["k_weight"]),
                                        sh.cu_seqlens, sh.cu_seqlens_padded, num_q_heads=w.num_q_heads,
                                        num_k_heads=w.num_k_heads, head_dim=w.head_dim, rope_grid=sh.rope_grid,
                                        sections=w.sections, rope_theta=w.rope_theta, eps=w.eps,
                                        pos_offset=sh.pos_offset)
        valid = np.concatenate([np.arange(sh.cu_seqlens_padded[i],
                                          sh.cu_seqlens_padded[i] + sh.cu_seqlens[i + 1] - sh.cu_seqlens[i])
                                for i in range(sh.num_seqs)])
        P.assert_close(tbits(q)[valid], qo[valid], f"slice {rank} q")
        P.assert_close(tbits(k)[valid], ko[valid], f"slice {rank} k")


def heads():
    return W.custom("hs", (700, 45, 0, 300), (704, 48, 8, 304), hidden=256, num_q_heads=8, num_k_heads=2,
                    head_dim=128, inner=264, grids=((4, 6, 25), (0, 0, 0), (0, 0, 0), (3, 5, 10)),
                    sections=(32, 48, 48), seed=3)


@pytest.mark.parametrize("world", [2, 4, 8])
@pytest.mark.parametrize("rope_mode", ["interleaved", "half"])
@pytest.mark.parametrize("layout", ["view", "copy"])
def test_head_slices_equal_the_whole_call(world, rope_mode, layout):
    """Sharding by heads (the layout after a sequence-to-head all-to-all):
    rank r holds every row but only its q heads and the k head(s) they use
    (dit_token_b200.shard.head_range; k heads are replicated when there are
    fewer than ranks).  Each rank's call on its heads, either in place on a
    column view of the whole buffer (row stride of all heads) or on its own
    contiguous buffer, equals the unsharded call's columns bit for bit, though
    the kernel's batching of heads per CTA changes with the head count."""
    w = heads()
    rv = W.rows_view
    qi = W.qk_inputs(w)
    q0, k0 = rv(qi["q"]).cuda(), rv(qi["k"]).cuda()
    wq, wk = qi["q_weight"].cuda(), qi["k_weight"].cuda()
    cs, cp, grid = P.device_packing(w)
    D, Hq, Hk = w.head_dim, w.num_q_heads, w.num_k_heads
    kw = dict(head_dim=D, rope_grid=grid, sections=w.sections, rope_theta=w.rope_theta, eps=w.eps,
              rope_mode=rope_mode)
    qf, kf = q0.clone(), k0.clone()
    dit.dit_qk_rmsnorm_rope(qf, kf, wq, wk, cs, cp, num_q_heads=Hq, num_k_heads=Hk, **kw)
    qs = q0.clone()
    for rank in range(world):
        qh0, hq, kh0, hk = head_range(Hq, Hk, rank, world)
        qcols, kcols = slice(qh0 * D, (qh0 + hq) * D), slice(kh0 * D, (kh0 + hk) * D)
        q = qs[:, qcols] if layout == "view" else q0[:, qcols].contiguous()
        k = k0[:, kcols].contiguous()
        dit.dit_qk_rmsnorm_rope(q, k, wq, wk, cs, cp, num_q_heads=hq, num_k_heads=hk, **kw)
        if layout == "copy":
            assert torch.equal(q.view(torch.int16), qf[:, qcols].view(torch.int16)), (world, rank, "q")
        assert torch.equal(k.view(torch.int16), kf[:, kcols].view(torch.int16)), (world, rank, "k")
    if layout == "view":
        assert torch.equal(qs.view(torch.int16), qf.view(torch.int16)), world
