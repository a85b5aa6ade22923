"""The entry points called from several host threads at once, each thread on
its own CUDA stream and buffers (the header promises that calls only enqueue
work and keep no state): every thread's results equal a serial run bit for
bit."""
import threading

import pytest
import torch

import dit_token_b200 as dit
from dit_token_b200 import workloads as W
import _parity as P

pytestmark = pytest.mark.gpu


def run_all(w, inp, stream):
    cs, cp, grid = P.device_packing(w)
    rv = W.rows_view
    # the inputs were copied on this thread's current stream: the op stream
    # (a non-blocking pool stream) must wait for those copies
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        q, k = rv(inp["q"]), rv(inp["k"])
        dit.dit_qk_rmsnorm_rope(q, k, inp["q_weight"], inp["k_weight"], cs, cp, num_q_heads=w.num_q_heads,
                                num_k_heads=w.num_k_heads, head_dim=w.head_dim, rope_grid=grid, sections=w.sections,
                                rope_theta=w.rope_theta, eps=w.eps)
        a = dit.dit_adaln_modulate(rv(inp["x"]), inp["mod"][:, 0], inp["mod"][:, 1], cs, cp, eps=w.eps)
        r, n = dit.dit_gated_residual_adaln(rv(inp["x"]), rv(inp["y"]), inp["mod"][:, 2], inp["mod"][:, 3],
                                            inp["mod"][:, 4], cs, cp, eps=w.eps)
        s = dit.dit_swiglu(rv(inp["x"]), rv(inp["y"]), cs, cp)
    stream.synchronize()
    rows = torch.from_numpy(w.valid_rows()).cuda()
    return [t[rows].view(torch.int16).clone() for t in (q, k, a, r, n, s)]


def inputs(w):
    qk, res = W.qk_inputs(w), W.residual_inputs(w)
    return {"q": qk["q"].cuda(), "k": qk["k"].cuda(), "q_weight": qk["q_weight"].cuda(),
            "k_weight": qk["k_weight"].cuda(), "x": res["x"].cuda(), "y": res["y"].cuda(), "mod": res["mod"].cuda()}


def test_four_threads_four_streams():
    from dit_token_b200 import build
    build.build()
    w = W.custom("thr", (300, 77, 500), (304, 80, 512), hidden=512, num_q_heads=4, num_k_heads=2, head_dim=128,
                 inner=512, grids=((2, 5, 10), (0, 0, 0), (3, 6, 20)), sections=(44, 42, 42), seed=6)
    serial = run_all(w, inputs(w), torch.cuda.Stream())
    results, errors = [None] * 4, []

    def worker(i):
        try:
            inp = inputs(w)           # each thread its own buffers
            for _ in range(3):
                out = run_all(w, {k: v.clone() for k, v in inp.items()}, torch.cuda.Stream())
            results[i] = out
        except Exception as e:        # reported below, on the main thread
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(4)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for out in results:
        for a, b in zip(out, serial):
            assert torch.equal(a, b)
