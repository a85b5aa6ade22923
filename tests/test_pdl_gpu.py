"""Ordering of dependent launches.  The library launches its kernels so that
each may be scheduled while the previous kernel on the stream drains, and
every kernel waits for that kernel's completion before its first memory
access.  A chain in which every stage depends on the one before -- gated
residual, adaLN of its output, SwiGLU of that output's two halves, then Q/K
RMSNorm + RoPE in place on the same buffer (which must not start writing it
while SwiGLU still reads it) -- runs twelve rounds back to back on one
stream, eagerly and as a replayed CUDA graph.  Every round refills the
intermediate buffers with NaN sentinels (ordinary torch kernels, which do
not take part in dependent launches, so the chain's first kernel also
follows a plain one) and swaps the inputs, so a stage that ran early would
read sentinels or the previous round's data.  The chain's results must equal
bit for bit those of the same four calls with a device synchronization after
each (no overlap possible); each stage of that reference run is compared
with the oracle applied to the reference's own previous stage."""
import dataclasses

import pytest
import torch

import dit_token_b200 as dit
import oracle
from dit_token_b200 import workloads as W
import _parity as P
from _util import tbits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def chain():
    from dit_token_b200 import build
    build.build()
    w = W.custom("chain", (9000, 4500, 2601), (9088, 4608, 2688), hidden=3072, num_q_heads=24, num_k_heads=4,
                 head_dim=128, inner=1536, grids=((8, 24, 42), (0, 0, 0), (2, 24, 42)), sections=(44, 42, 42),
                 seed=77)
    res = W.residual_inputs(w)
    qk = W.qk_inputs(dataclasses.replace(w, num_q_heads=w.hidden // w.head_dim, num_k_heads=4))
    cs, cp, grid = P.device_packing(w)
    rv = W.rows_view
    C = w.hidden
    d = {"x0": res["x"].cuda(), "y0": res["y"].cuda(), "mod": res["mod"].cuda(), "qw": qk["q_weight"].cuda(),
         "kw": qk["k_weight"].cuda(), "k0": qk["k"].cuda(), "sentinel": W.sentinel_like(res["out"].shape).cuda()}
    d["xin"], d["yin"] = d["x0"].clone(), d["y0"].clone()
    d["r"], d["a"] = d["sentinel"].clone(), d["sentinel"].clone()
    d["k"] = d["k0"].clone()
    d["s"] = W.sentinel_like((res["out"].shape[0], C // 2)).cuda()

    def stages(sync):
        """The four dependent calls (after refilling the intermediates); with
        sync, a device synchronization after each and a snapshot of the adaLN
        output (which the Q/K stage then rotates in place)."""
        snaps = {}
        d["r"].copy_(d["sentinel"])
        d["a"].copy_(d["sentinel"])
        d["s"].fill_(float("nan"))
        d["k"].copy_(d["k0"])
        dit.dit_gated_residual(rv(d["xin"]), rv(d["yin"]), d["mod"][:, 2], cs, cp, out=rv(d["r"]))
        if sync:
            torch.cuda.synchronize()
        dit.dit_adaln_modulate(rv(d["r"]), d["mod"][:, 0], d["mod"][:, 1], cs, cp, out=rv(d["a"]), eps=w.eps)
        if sync:
            torch.cuda.synchronize()
            snaps["a"] = d["a"].clone()
        dit.dit_swiglu(rv(d["a"])[:, : C // 2], rv(d["a"])[:, C // 2:], cs, cp, out=rv(d["s"]))
        if sync:
            torch.cuda.synchronize()
        dit.dit_qk_rmsnorm_rope(rv(d["a"]), rv(d["k"]), d["qw"], d["kw"], cs, cp, num_q_heads=C // w.head_dim,
                                num_k_heads=4, head_dim=w.head_dim, rope_grid=grid, sections=w.sections,
                                rope_theta=w.rope_theta, eps=w.eps)
        if sync:
            torch.cuda.synchronize()
        return snaps

    def set_inputs(i):
        src = (d["x0"], d["y0"]) if i % 2 == 0 else (d["y0"], d["x0"])
        d["xin"].copy_(src[0])
        d["yin"].copy_(src[1])

    refs = []
    for i in range(2):
        set_inputs(i)
        snaps = stages(sync=True)
        refs.append({"r": d["r"].clone(), "a": snaps["a"], "s": d["s"].clone(), "q": d["a"].clone(),
                     "k": d["k"].clone()})
    yield w, d, stages, set_inputs, refs, res, qk


def test_reference_stages_match_oracle(chain):
    """Each stage of the synchronized run against the oracle applied to that
    run's own previous stage (no compounding of rounding across stages)."""
    w, d, _, _, refs, res, qk = chain
    rv = W.rows_view
    C, rows = w.hidden, w.valid_rows()
    cs, cp = w.cu_seqlens, w.cu_seqlens_padded
    flat = P.mod_flat(res["mod"])
    for i, ref in enumerate(refs):
        xb, yb = (res["x"], res["y"]) if i % 2 == 0 else (res["y"], res["x"])
        r_or = oracle.gated_residual(tbits(rv(xb)), tbits(rv(yb)), flat[2 * C:], cs, cp, hidden=C,
                                     gate_seq_stride=6 * C)
        P.assert_close(P.gather_rows(ref["r"], rows), r_or[rows], f"input set {i} residual")
        r_gpu = tbits(rv(ref["r"]))
        a_or = oracle.adaln_modulate(r_gpu, flat, flat[C:], cs, cp, hidden=C, eps=w.eps, mod_seq_stride=6 * C)
        P.assert_close(P.gather_rows(ref["a"], rows), a_or[rows], f"input set {i} adaln")
        a_gpu = tbits(rv(ref["a"]))
        half = C // 2
        s_or = oracle.swiglu(a_gpu, a_gpu.reshape(-1)[half:], cs, cp, inner=half, a_row_stride=C,
                             b_row_stride=C, nrows=a_gpu.shape[0])
        P.assert_close(P.gather_rows(ref["s"], rows), s_or[rows], f"input set {i} swiglu")
        q_or, k_or = oracle.qk_rmsnorm_rope(a_gpu, tbits(rv(qk["k"])), tbits(qk["q_weight"]),
                                            tbits(qk["k_weight"]), cs, cp, num_q_heads=C // w.head_dim,
                                            num_k_heads=4, head_dim=w.head_dim, rope_grid=w.rope_grid,
                                            sections=w.sections, rope_theta=w.rope_theta, eps=w.eps)
        P.assert_close(P.gather_rows(ref["q"], rows), q_or[rows], f"input set {i} q")
        P.assert_close(P.gather_rows(ref["k"], rows), k_or[rows], f"input set {i} k")


@pytest.mark.parametrize("graphed", [False, True])
def test_dependent_chain_equals_synchronized_run(chain, graphed):
    """Eager: the chain is launched round after round.  Graphed: one round
    is captured in a CUDA graph (the dependent launches become programmatic
    edges of the graph) and replayed round after round."""
    w, d, stages, set_inputs, refs, _, _ = chain
    run = lambda: stages(sync=False)  # noqa: E731
    if graphed:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            stages(sync=False)  # warm-up off the capture
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            stages(sync=False)
        run = g.replay
    rounds = 12
    for i in range(rounds):
        set_inputs(i)
        run()
        if i >= rounds - 2:
            ref = refs[i % 2]
            for name, t in (("r", d["r"]), ("s", d["s"]), ("q", d["a"]), ("k", d["k"])):
                assert torch.equal(t.view(torch.int16), ref[name].view(torch.int16)), f"round {i} {name}"
    torch.cuda.synchronize()


@pytest.mark.parametrize("graphed", [False, True])
def test_descriptor_written_by_the_previous_kernel(graphed):
    """A kernel's first reads are the packing descriptors, which the
    previous kernel on the stream may have just written: dit_av_stream_seqlens
    writes the per-stream descriptor into buffers that are reset every round
    (to an empty descriptor, which would make adaLN write nothing) and the
    per-stream adaLN reads it right away.  Twelve rounds back to back, eagerly
    and as a replayed graph; the outputs equal the synchronized run's bit for
    bit, and the oracle's per-stream adaLN."""
    w = W.custom("desc", (6100, 900, 3000), (6144, 1024, 3072), hidden=2048, num_q_heads=1, num_k_heads=1,
                 head_dim=64, inner=8, grids=((5, 24, 42), (0, 0, 0), (2, 24, 42)), seed=91)
    C, B = w.hidden, w.num_seqs
    rows = w.valid_rows()
    cs, cp, grid = P.device_packing(w)
    m = W.modulation_av(w)
    mv = m.cuda().view(2 * B, 6, C)
    inp = W.adaln_inputs(w)
    x = W.rows_view(inp["x"].cuda())
    out = W.sentinel_like(inp["out"].shape).cuda()
    cs2 = torch.zeros(2 * B + 1, dtype=torch.int32, device="cuda")
    cp2 = torch.zeros_like(cs2)
    sentinel = W.sentinel_like(inp["out"].shape).cuda()

    def one_round(sync=False):
        out.copy_(sentinel)
        cs2.zero_()
        cp2.zero_()
        dit.dit_av_stream_seqlens(cs, cp, grid, out=(cs2, cp2))
        if sync:
            torch.cuda.synchronize()
        dit.dit_adaln_modulate(x, mv[:, 0], mv[:, 1], cs2, cp2, out=W.rows_view(out), eps=w.eps)
        if sync:
            torch.cuda.synchronize()

    one_round(sync=True)
    ref = out.clone()
    import oracle
    flat = P.mod_flat(m)
    o = oracle.adaln_modulate(tbits(W.rows_view(inp["x"])), flat, flat[C:], w.cu_seqlens, w.cu_seqlens_padded,
                              hidden=C, eps=w.eps, mod_seq_stride=12 * C, audio_offset=6 * C, rows=rows,
                              rope_grid=w.rope_grid)
    P.assert_close(P.gather_rows(ref, rows), o[rows], "per-stream adaln, synchronized")
    run = one_round
    if graphed:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            one_round()
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            one_round()
        run = g.replay
    for i in range(12):
        run()
        # (the comparison synchronizes between rounds, never inside one)
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"round {i}"
