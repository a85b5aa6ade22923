"""How close the kernels come to the oracle, beyond the agreement tolerance: on
sampled rows of the video and batched varlen workloads, the share of output
elements that are bit-identical to the oracle's result (fp64, rounded once to
bf16) and the largest distance in bf16 units in the last place.  fp32
arithmetic against fp64 can only move a result across a rounding boundary, so
at least 99.95 % of the elements must match exactly (measured: 99.996-100 %)
and none may be more than 1 ulp away,
except where the result is tiny (|ref| < 1e-3), where a fp32 absolute error
of ~1e-7 is many ulps of a small number."""
import numpy as np
import pytest
import torch

import dit_token_b200 as dit
from dit_token_b200 import workloads as W
import _parity as P

pytestmark = pytest.mark.gpu


def ulp_distance(gpu_bits, ref_bits):
    """|a - b| in bf16 units in the last place (bit patterns mapped to a
    monotonic integer line; +0 and -0 coincide)."""
    def line(b):
        b = np.asarray(b, dtype=np.uint16).astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(line(gpu_bits) - line(ref_bits))


def check(name, gpu_bits, ref_bits, exact_share=0.9995):
    d = ulp_distance(gpu_bits, ref_bits)
    ref = (np.asarray(ref_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    big = np.abs(ref) >= 1e-3
    share = float(np.mean(d == 0))
    worst = int(d[big].max()) if big.any() else 0
    assert share >= exact_share, f"{name}: only {share:.4f} of elements bit-identical to the oracle"
    assert worst <= 1, f"{name}: an element with |ref| >= 1e-3 is {worst} ulps from the oracle"
    print(f"{name}: {share:.5f} of {d.size} elements bit-identical, max {worst} ulp (|ref| >= 1e-3), "
          f"max {int(d.max())} ulp overall")
    return share, worst


@pytest.mark.parametrize("name", ["video", "batched_varlen"])
def test_outputs_are_within_one_ulp_of_the_oracle(name):
    w = W.workload(name)
    rows = W.sample_rows(w, per_seq=16)
    inp = W.qk_inputs(w)
    q, k = P.gpu_qk(w, inp)
    qo, ko = P.oracle_qk(w, inp, rows)
    check(f"{name} q", P.gather_rows(q, rows), qo[rows])
    check(f"{name} k", P.gather_rows(k, rows), ko[rows])
    del q, k, inp
    inp = W.adaln_inputs(w)
    check(f"{name} adaln", P.gather_rows(P.gpu_adaln(w, inp), rows), P.oracle_adaln(w, inp, rows)[rows])
    del inp
    inp = W.residual_inputs(w)
    check(f"{name} residual", P.gather_rows(P.gpu_residual(w, inp), rows), P.oracle_residual(w, inp, rows)[rows],
          exact_share=1.0)   # one fp32 FMA of bf16 values, rounded once: exact in fp64 too
    res, norm = P.gpu_fused(w, inp)
    r_ref, n_ref = P.oracle_fused(w, inp, rows)
    check(f"{name} fused residual", P.gather_rows(res, rows), r_ref[rows], exact_share=1.0)
    check(f"{name} fused norm", P.gather_rows(norm, rows), n_ref[rows])
    del inp, res, norm
    inp = W.swiglu_inputs(w)
    check(f"{name} swiglu", P.gather_rows(P.gpu_swiglu(w, inp), rows), P.oracle_swiglu(w, inp, rows)[rows])
    torch.cuda.empty_cache()


HARD_KINDS = ("N(0,1)", "channel 0 = 300", "channels 0 and 512 = 3000", "channel 77 = 3000", "mean 256",
              "mean 1, std 0.01", "constant")
# least share of elements bit-identical to the oracle, per kind: rows whose mean is far
# from zero in units of their spread lose digits of the mean in fp32 (and constant rows
# come out as shift plus an fp32 rounding residue of x * rstd), so those kinds get only
# the error bound below
HARD_EXACT = {"N(0,1)": 0.995, "channel 0 = 300": 0.995, "channels 0 and 512 = 3000": 0.995,
              "channel 77 = 3000": 0.995, "mean 256": 0.9, "mean 1, std 0.01": 0.95, "constant": 0.0}


def hard_rows(n_per_kind, C, seed):
    """Rows that strain one-pass statistics: massive activations in fixed channels
    (channel 0 is the first element of warp 0's lane 0; 512 that of the second
    warp of a 2-warp team with 32-byte vectors), large means, tiny spreads,
    constant rows; then the bf16 rounding of each value."""
    g = torch.Generator().manual_seed(seed)
    blocks = []
    for kind in HARD_KINDS:
        x = torch.randn(n_per_kind, C, generator=g, dtype=torch.float64)
        if kind == "channel 0 = 300":
            x[:, 0] = 300.0
        elif kind == "channels 0 and 512 = 3000":
            x[:, 0] = 3000.0
            x[:, 512] = 3000.0
        elif kind == "channel 77 = 3000":
            x[:, 77] = 3000.0
        elif kind == "mean 256":
            x += 256.0
        elif kind == "mean 1, std 0.01":
            x = 1.0 + 0.01 * x
        elif kind == "constant":
            x = (3.0 * torch.randn(n_per_kind, 1, generator=g, dtype=torch.float64)).expand(-1, C)
        blocks.append(x)
    return torch.cat(blocks).to(torch.bfloat16)


def check_hard(what, gpu_bits, ref_bits, n_per_kind):
    """Per kind: |gpu - ref| within one bf16 unit in the last place of max(|ref|, 1)
    (the output's own scale: LN output is O(1)), and the kind's bit-identical share."""
    g = (np.asarray(gpu_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    r = (np.asarray(ref_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(r), 1.0))) - 7)
    d = ulp_distance(gpu_bits, ref_bits)
    for i, kind in enumerate(HARD_KINDS):
        sl = slice(i * n_per_kind, (i + 1) * n_per_kind)
        err = np.abs(g[sl] - r[sl])
        assert np.all(err <= ulp[sl]), f"{what} {kind}: error {err.max()} above one unit of max(|ref|, 1)"
        share = float(np.mean(d[sl] == 0))
        assert share >= HARD_EXACT[kind], f"{what} {kind}: only {share:.4f} bit-identical to the oracle"
        print(f"{what} {kind}: {share:.5f} bit-identical, max error {err.max():.3g}")


@pytest.mark.parametrize("hidden", [2048, 3072, 5120, 8192, 16384])
def test_adaln_statistics_on_hard_rows(hidden):
    """adaLN and the fused residual + adaLN on rows built to defeat one-pass
    statistics; 2048 and 3072 take a warp per row, 5120 and wider a team of
    warps (2 at 5120 and 8192, 4 at 16384; the fused op's teams are wider)."""
    n = 24
    nrows = n * len(HARD_KINDS)
    w = W.custom("hard", (nrows // 2, nrows // 2), (nrows // 2 + 4, nrows // 2 + 4), hidden=hidden,
                 num_q_heads=1, num_k_heads=1, head_dim=64, inner=8, seed=hidden)
    rows = w.valid_rows()
    x = hard_rows(n, hidden, seed=hidden)
    inp = W.adaln_inputs(w)
    W.rows_view(inp["x"])[torch.from_numpy(rows)] = x
    out = P.gpu_adaln(w, inp)
    check_hard(f"adaln {hidden}", P.gather_rows(out, rows), P.oracle_adaln(w, inp, rows)[rows], n)
    inp = W.residual_inputs(w)
    W.rows_view(inp["x"])[torch.from_numpy(rows)] = x
    inp["y"].zero_()  # the residual is then x itself, and the norm is adaLN of the hard rows
    res, norm = P.gpu_fused(w, inp)
    r_ref, n_ref = P.oracle_fused(w, inp, rows)
    assert np.array_equal(P.gather_rows(res, rows), r_ref[rows])
    check_hard(f"fused {hidden}", P.gather_rows(norm, rows), n_ref[rows], n)


@pytest.mark.parametrize("hidden", [3072, 5120])
@pytest.mark.parametrize("layout", ["rows on a 16-byte boundary", "fp32 vectors"])
def test_adaln_statistics_on_hard_rows_other_layouts(hidden, layout):
    """The same rows through the kernels' other instantiations: 16-byte row
    accesses (rows starting 8 elements into a wider buffer, so not on a
    32-byte boundary) and fp32 modulation vectors."""
    n = 24
    nrows = n * len(HARD_KINDS)
    w = W.custom("hard", (nrows // 2, nrows // 2), (nrows // 2 + 4, nrows // 2 + 4), hidden=hidden,
                 num_q_heads=1, num_k_heads=1, head_dim=64, inner=8, seed=hidden + 1)
    rows = w.valid_rows()
    x = hard_rows(n, hidden, seed=hidden + 1)
    inp = W.adaln_inputs(w)
    res_inp = W.residual_inputs(w)
    for d in (inp, res_inp):
        W.rows_view(d["x"])[torch.from_numpy(rows)] = x
    res_inp["y"].zero_()
    if layout == "fp32 vectors":
        inp["mod"] = W.modulation(w, torch.float32)
        res_inp["mod"] = inp["mod"]
        out = P.gpu_adaln(w, inp)
        res, norm = P.gpu_fused(w, res_inp)
        got_a, got_r, got_n = (P.gather_rows(t, rows) for t in (out, res, norm))
    else:
        cs, cp, _ = P.device_packing(w)
        mod = inp["mod"].cuda()
        C, off = hidden, 8

        def wide(src=None):
            buf = W.sentinel_like((inp["x"].shape[0], C + 16)).cuda()
            if src is not None:
                buf[:, off:off + C] = src.cuda()
            return buf, W.rows_view(buf)[:, off:off + C]

        (_, xa), (ob, oa) = wide(inp["x"]), wide()
        dit.dit_adaln_modulate(xa, mod[:, 0], mod[:, 1], cs, cp, out=oa, eps=w.eps)
        (_, xf), (_, yf), (rb, rf), (nb, nf) = wide(res_inp["x"]), wide(res_inp["y"]), wide(), wide()
        dit.dit_gated_residual_adaln(xf, yf, mod[:, 2], mod[:, 3], mod[:, 4], cs, cp, res_out=rf, norm_out=nf,
                                     eps=w.eps)
        torch.cuda.synchronize()
        got_a, got_r, got_n = (P.gather_rows(t[:, off:off + C].contiguous(), rows) for t in (ob, rb, nb))
    check_hard(f"adaln {hidden} {layout}", got_a, P.oracle_adaln(w, inp, rows)[rows], n)
    r_ref, n_ref = P.oracle_fused(w, res_inp, rows)
    assert np.array_equal(got_r, r_ref[rows])
    check_hard(f"fused {hidden} {layout}", got_n, n_ref[rows], n)
