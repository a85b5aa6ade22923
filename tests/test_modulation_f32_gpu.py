"""fp32 per-sequence modulation vectors (gate, shift, scale) on the GPU, through
the _ex entry points, against the oracle's fp32 path.

The activations stay bf16; the vectors are the unrounded N(0, 0.1) draws whose
rounding is the bf16 modulation of the same workload.  Three checks:
parity with the oracle at every adaLN team shape and on many short sequences
(more sequences per CTA than the adaLN kernel stages in shared memory); bit
equality with the bf16 path when the fp32 vectors hold bf16 values; and
sampled rows of the full batched-varlen workload.
"""
import numpy as np
import pytest
import torch

import dit_token_b200 as dit
from dit_token_b200 import workloads as W
import _parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dit_token_b200 import build
    build.build()


def with_f32_mod(w, inp):
    out = dict(inp)
    out["mod"] = W.modulation(w, torch.float32)
    return out


def check_three_ops(w, rows, tag):
    keep = P.untouched_rows(w)
    inp = with_f32_mod(w, W.adaln_inputs(w))
    out = P.gpu_adaln(w, inp)
    P.assert_close(P.gather_rows(out, rows), P.oracle_adaln(w, inp, rows)[rows], f"{tag} adaln f32")
    P.assert_untouched(out, inp["out"], keep, f"{tag} adaln f32")
    inp = with_f32_mod(w, W.residual_inputs(w))
    out = P.gpu_residual(w, inp)
    P.assert_close(P.gather_rows(out, rows), P.oracle_residual(w, inp, rows)[rows], f"{tag} residual f32")
    P.assert_untouched(out, inp["out"], keep, f"{tag} residual f32")
    res, norm = P.gpu_fused(w, inp)
    r_ref, n_ref = P.oracle_fused(w, inp, rows)
    P.assert_close(P.gather_rows(res, rows), r_ref[rows], f"{tag} fused residual f32")
    P.assert_close(P.gather_rows(norm, rows), n_ref[rows], f"{tag} fused norm f32")
    P.assert_untouched(res, inp["out"], keep, f"{tag} fused res f32")
    P.assert_untouched(norm, inp["out"], keep, f"{tag} fused norm f32")
    # the fused residual is the separate residual kernel's, bit for bit
    assert torch.equal(res.view(torch.int16), out.view(torch.int16))


@pytest.mark.parametrize("hidden", [8, 264, 2048, 3072, 5120, 6152, 8192, 16384])
def test_f32_modulation_every_team_shape(hidden):
    w = W.custom("mod32", (13, 6), (16, 8), hidden=hidden, num_q_heads=1, num_k_heads=1, head_dim=64,
                 inner=8, seed=hidden + 1)
    check_three_ops(w, w.valid_rows(), f"hidden {hidden}")


def test_f32_modulation_many_short_sequences():
    rng = np.random.default_rng(11)
    lengths = rng.integers(0, 7, 400)
    padded = [int(L) + int(rng.integers(0, 3)) for L in lengths]
    w = W.custom("mod32many", lengths, padded, hidden=1024, num_q_heads=1, num_k_heads=1, head_dim=64,
                 inner=8, seed=4)
    check_three_ops(w, w.valid_rows(), "many")


@pytest.mark.parametrize("hidden", [264, 5120, 8192])
def test_bf16_valued_f32_vectors_match_the_bf16_path(hidden):
    """fp32 vectors holding bf16 values give the bf16 path's results: the
    element-wise residuals bit for bit; the normalizations (whose row
    statistics the two paths sum in different lane layouts -- they use
    different access widths) within the tolerance and almost all bit for
    bit."""
    w = W.custom("same", (37, 5, 90), (40, 8, 96), hidden=hidden, num_q_heads=1, num_k_heads=1, head_dim=64,
                 inner=8, seed=7)
    cs, cp, _ = P.device_packing(w)
    inp = W.residual_inputs(w)
    x, y = W.rows_view(inp["x"].cuda()), W.rows_view(inp["y"].cuda())
    m16 = inp["mod"].cuda()
    m32 = m16.float()
    a = dit.dit_adaln_modulate(x, m16[:, 0], m16[:, 1], cs, cp, eps=w.eps)
    b = dit.dit_adaln_modulate(x, m32[:, 0], m32[:, 1], cs, cp, eps=w.eps)
    rows = torch.from_numpy(w.valid_rows()).cuda()

    def close(u, v, what):
        ub, vb = u[rows].view(torch.int16), v[rows].view(torch.int16)
        P.assert_close(ub.cpu().numpy().view(np.uint16), vb.cpu().numpy().view(np.uint16), what)
        assert (ub == vb).float().mean().item() >= 0.999, what

    close(a, b, "adaln")
    a = dit.dit_gated_residual(x, y, m16[:, 2], cs, cp)
    b = dit.dit_gated_residual(x, y, m32[:, 2], cs, cp)
    assert torch.equal(a[rows].view(torch.int16), b[rows].view(torch.int16))
    ra, na = dit.dit_gated_residual_adaln(x, y, m16[:, 2], m16[:, 3], m16[:, 4], cs, cp, eps=w.eps)
    rb, nb = dit.dit_gated_residual_adaln(x, y, m32[:, 2], m32[:, 3], m32[:, 4], cs, cp, eps=w.eps)
    assert torch.equal(ra[rows].view(torch.int16), rb[rows].view(torch.int16))
    close(na, nb, "fused norm")


def test_f32_modulation_batched_varlen_sampled():
    w = W.workload("batched_varlen")
    check_three_ops(w, W.sample_rows(w, per_seq=32), "batched_varlen")


def test_mixed_dtypes_are_rejected():
    w = W.custom("mix", (5,), (8,), hidden=64, num_q_heads=1, num_k_heads=1, head_dim=64, inner=8)
    cs, cp, _ = P.device_packing(w)
    x = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    g16 = torch.zeros(1, 64, dtype=torch.bfloat16, device="cuda")
    g32 = torch.zeros(1, 64, dtype=torch.float32, device="cuda")
    with pytest.raises(TypeError):
        dit.dit_adaln_modulate(x, g16, g32, cs, cp)
    with pytest.raises(TypeError):
        dit.dit_gated_residual_adaln(x, x, g32, g16, g16, cs, cp)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("hidden", [2048, 5120])
def test_vectors_off_a_32_byte_boundary(dtype, hidden):
    """Per-sequence vectors are read 32 bytes per lane at a time only when
    every sequence's vectors start on a 32-byte boundary; vectors 16 bytes
    off one (a legal layout) take the 16-byte reads and give the same
    results against the oracle, for adaLN and the fused op."""
    w = W.custom("offvec", (300, 77), (304, 80), hidden=hidden, num_q_heads=1, num_k_heads=1, head_dim=64,
                 inner=8, seed=hidden + 5)
    rows = w.valid_rows()
    inp = W.residual_inputs(w)
    mod = inp["mod"].to(dtype)
    per = 16 // mod.element_size()                  # elements in 16 bytes
    wide = torch.zeros(w.num_seqs, 6 * hidden + 2 * per, dtype=dtype)
    wide[:, per:per + 6 * hidden] = mod.reshape(w.num_seqs, -1)
    shifted = wide.cuda()[:, per:per + 6 * hidden].view(w.num_seqs, 6, hidden)   # 16 bytes past the start
    assert shifted.data_ptr() % 32 == 16
    cs, cp, _ = P.device_packing(w)
    x, y = W.rows_view(inp["x"].cuda()), W.rows_view(inp["y"].cuda())
    ref_inp = dict(inp, mod=mod)
    out = W.sentinel_like(inp["out"].shape).cuda()
    dit.dit_adaln_modulate(x, shifted[:, 0], shifted[:, 1], cs, cp, out=W.rows_view(out), eps=w.eps)
    a_ref = P.oracle_adaln(w, dict(ref_inp, x=inp["x"]), rows)
    P.assert_close(P.gather_rows(out, rows), a_ref[rows], f"adaln {dtype} off 32 B")
    res = W.sentinel_like(inp["out"].shape).cuda()
    norm = W.sentinel_like(inp["out"].shape).cuda()
    dit.dit_gated_residual_adaln(x, y, shifted[:, 2], shifted[:, 3], shifted[:, 4], cs, cp,
                                 res_out=W.rows_view(res), norm_out=W.rows_view(norm), eps=w.eps)
    r_ref, n_ref = P.oracle_fused(w, ref_inp, rows)
    P.assert_close(P.gather_rows(res, rows), r_ref[rows], f"fused residual {dtype} off 32 B")
    P.assert_close(P.gather_rows(norm, rows), n_ref[rows], f"fused norm {dtype} off 32 B")
