"""The operators only enqueue work (no allocation, no synchronization), so a
whole step can be captured in a CUDA graph and replayed; the replay must be
bitwise identical to eager execution."""
import pytest
import torch

import dit_token_b200 as dit
from dit_token_b200 import workloads as W
import _parity as P

pytestmark = pytest.mark.gpu


def test_step_captures_and_replays_bitwise():
    from dit_token_b200 import build
    build.build()
    w = W.workload("single_stream")
    qk, ad, rs, sw = W.qk_inputs(w), W.adaln_inputs(w), W.residual_inputs(w), W.swiglu_inputs(w)
    cs, cp, grid = P.device_packing(w)
    rv = W.rows_view

    def buffers():
        return {"q": qk["q"].cuda(), "k": qk["k"].cuda(), "ax": ad["x"].cuda(), "aout": ad["out"].cuda(),
                "rx": rs["x"].cuda(), "ry": rs["y"].cuda(), "rout": rs["out"].cuda(), "norm": ad["out"].cuda(),
                "ab": sw["ab"].cuda(), "sout": sw["out"].cuda()}

    wq, wk, mod = qk["q_weight"].cuda(), qk["k_weight"].cuda(), ad["mod"].cuda()

    def step(b):
        dit.dit_qk_rmsnorm_rope(rv(b["q"]), rv(b["k"]), wq, wk, cs, cp, num_q_heads=w.num_q_heads,
                                num_k_heads=w.num_k_heads, head_dim=w.head_dim, rope_grid=grid,
                                sections=w.sections, eps=w.eps)
        dit.dit_adaln_modulate(rv(b["ax"]), mod[:, 0], mod[:, 1], cs, cp, out=rv(b["aout"]), eps=w.eps)
        dit.dit_gated_residual(rv(b["rx"]), rv(b["ry"]), mod[:, 2], cs, cp, out=rv(b["rout"]))
        dit.dit_gated_residual_adaln(rv(b["rx"]), rv(b["ry"]), mod[:, 2], mod[:, 3], mod[:, 4], cs, cp,
                                     res_out=rv(b["rout"]), norm_out=rv(b["norm"]), eps=w.eps)
        ab = rv(b["ab"])
        dit.dit_swiglu(ab[:, : w.inner], ab[:, w.inner:], cs, cp, out=rv(b["sout"]))

    eager = buffers()
    step(eager)
    graphed = buffers()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step(buffers())  # warm-up on the side stream (first launches set kernel attributes)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(graphed)
    g.replay()
    torch.cuda.synchronize()
    for name in eager:
        assert torch.equal(eager[name].view(torch.int16), graphed[name].view(torch.int16)), name
