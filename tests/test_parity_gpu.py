"""GPU parity of the four operators against the CPU oracle on the five seeded
workloads, at full size and in the launch configuration the benchmark times.

Every valid row of every workload is compared element by element with the
oracle (which computes the whole batch), every padding row and the canary
rows around each buffer are checked bit-exactly at full size, and a second
run must be bitwise identical.
"""
import pytest
import torch

from dit_token_b200 import workloads as W
import _parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=W.WORKLOAD_NAMES)
def case(request):
    from dit_token_b200 import build
    build.build()
    w = W.workload(request.param)
    inputs = {"qk": W.qk_inputs(w), "adaln": W.adaln_inputs(w), "residual": W.residual_inputs(w),
              "swiglu": W.swiglu_inputs(w)}
    rows = w.valid_rows()
    yield w, inputs, rows
    del inputs
    torch.cuda.empty_cache()


def test_qk_rmsnorm_rope(case):
    w, inp, rows = case[0], case[1]["qk"], case[2]
    q, k = P.gpu_qk(w, inp)
    torch.cuda.synchronize()
    qo, ko = P.oracle_qk(w, inp, rows)
    P.assert_close(P.gather_rows(q, rows), qo[rows], f"{w.name} q")
    P.assert_close(P.gather_rows(k, rows), ko[rows], f"{w.name} k")
    keep = P.untouched_rows(w)
    P.assert_untouched(q, inp["q"], keep, f"{w.name} q")
    P.assert_untouched(k, inp["k"], keep, f"{w.name} k")
    q2, k2 = P.gpu_qk(w, inp)
    assert torch.equal(q.view(torch.int16), q2.view(torch.int16))
    assert torch.equal(k.view(torch.int16), k2.view(torch.int16))


def test_adaln_modulate(case):
    w, inp, rows = case[0], case[1]["adaln"], case[2]
    out = P.gpu_adaln(w, inp)
    torch.cuda.synchronize()
    ref = P.oracle_adaln(w, inp, rows)
    P.assert_close(P.gather_rows(out, rows), ref[rows], f"{w.name} adaln")
    P.assert_untouched(out, inp["out"], P.untouched_rows(w), f"{w.name} adaln out")
    out2 = P.gpu_adaln(w, inp)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def test_gated_residual(case):
    w, inp, rows = case[0], case[1]["residual"], case[2]
    out = P.gpu_residual(w, inp)
    torch.cuda.synchronize()
    ref = P.oracle_residual(w, inp, rows)
    P.assert_close(P.gather_rows(out, rows), ref[rows], f"{w.name} residual")
    P.assert_untouched(out, inp["out"], P.untouched_rows(w), f"{w.name} residual out")
    out2 = P.gpu_residual(w, inp)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def test_swiglu(case):
    w, inp, rows = case[0], case[1]["swiglu"], case[2]
    out = P.gpu_swiglu(w, inp)
    torch.cuda.synchronize()
    ref = P.oracle_swiglu(w, inp, rows)
    P.assert_close(P.gather_rows(out, rows), ref[rows], f"{w.name} swiglu")
    P.assert_untouched(out, inp["out"], P.untouched_rows(w), f"{w.name} swiglu out")
    out2 = P.gpu_swiglu(w, inp)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def test_gated_residual_adaln(case):
    w, inp, rows = case[0], case[1]["residual"], case[2]
    res, norm = P.gpu_fused(w, inp)
    torch.cuda.synchronize()
    r_ref, n_ref = P.oracle_fused(w, inp, rows)
    P.assert_close(P.gather_rows(res, rows), r_ref[rows], f"{w.name} fused residual")
    P.assert_close(P.gather_rows(norm, rows), n_ref[rows], f"{w.name} fused norm")
    keep = P.untouched_rows(w)
    P.assert_untouched(res, inp["out"], keep, f"{w.name} fused res")
    P.assert_untouched(norm, inp["out"], keep, f"{w.name} fused norm")
    # the fused op's residual is the separate kernel's bit for bit; its
    # normalization agrees with the separate adaLN kernel (whose statistics are
    # merged in another order) within the same tolerance
    import dit_token_b200 as dit
    cs, cp, _ = P.device_packing(w)
    mod = inp["mod"].cuda()
    r2 = P.gpu_residual(w, inp)
    n2 = W.sentinel_like(inp["out"].shape).cuda()
    dit.dit_adaln_modulate(W.rows_view(r2), mod[:, 3], mod[:, 4], cs, cp, out=W.rows_view(n2), eps=w.eps)
    assert torch.equal(res.view(torch.int16), r2.view(torch.int16))
    P.assert_close(P.gather_rows(norm, rows), P.gather_rows(n2, rows), f"{w.name} fused vs separate adaLN")
