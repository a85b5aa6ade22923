"""GPU edge cases, every valid row compared with the oracle: ragged shapes
(rows not a multiple of a CTA, widths not a multiple of a warp step),
zero-length and length-1 sequences, a sequence that fills its padded slot,
GQA, head_dim 64 with 3D sections, unit grid axes, strided (fused QKV)
buffers, in-place use, hundreds of sequences, every adaLN team/vector
variant up to the largest supported hidden size, empty batches, and
malformed device descriptors (skipped rows, nothing written out of bounds,
flagged by dit_validate_seqlens)."""
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


def ragged(head_dim=128, sections=(44, 42, 42), hq=3, hk=1, hidden=2056, inner=1032, seed=3):
    lengths = (1, 0, 37, 136, 300, 64)
    padded = (8, 8, 40, 136, 304, 64)
    grids = ((1, 1, 1), (0, 0, 0), (2, 3, 5), (4, 1, 6), (3, 7, 1), (0, 0, 0))
    return W.custom("ragged", lengths, padded, hidden=hidden, num_q_heads=hq, num_k_heads=hk,
                    head_dim=head_dim, inner=inner, grids=grids, sections=sections, seed=seed)


def all_ops_full(w, in_place=False):
    rows = w.valid_rows()
    keep = P.untouched_rows(w)
    inp = W.qk_inputs(w)
    q, k = P.gpu_qk(w, inp)
    qo, ko = P.oracle_qk(w, inp, rows)
    P.assert_close(P.gather_rows(q, rows), qo[rows], "q")
    P.assert_close(P.gather_rows(k, rows), ko[rows], "k")
    P.assert_untouched(q, inp["q"], keep, "q")
    P.assert_untouched(k, inp["k"], keep, "k")

    inp = W.adaln_inputs(w)
    out = P.gpu_adaln(w, inp, in_place=in_place)
    P.assert_close(P.gather_rows(out, rows), P.oracle_adaln(w, inp, rows)[rows], "adaln")
    P.assert_untouched(out, inp["x"] if in_place else inp["out"], keep, "adaln")

    inp = W.residual_inputs(w)
    out = P.gpu_residual(w, inp, in_place=in_place)
    P.assert_close(P.gather_rows(out, rows), P.oracle_residual(w, inp, rows)[rows], "residual")
    P.assert_untouched(out, inp["x"] if in_place else inp["out"], keep, "residual")

    inp = W.swiglu_inputs(w)
    out = P.gpu_swiglu(w, inp)
    P.assert_close(P.gather_rows(out, rows), P.oracle_swiglu(w, inp, rows)[rows], "swiglu")
    P.assert_untouched(out, inp["out"], keep, "swiglu")

    inp = W.residual_inputs(w)
    res, norm = P.gpu_fused(w, inp, in_place=in_place)
    r_ref, n_ref = P.oracle_fused(w, inp, rows)
    P.assert_close(P.gather_rows(res, rows), r_ref[rows], "fused residual")
    P.assert_close(P.gather_rows(norm, rows), n_ref[rows], "fused norm")
    P.assert_untouched(res, inp["x"] if in_place else inp["out"], keep, "fused residual")
    P.assert_untouched(norm, inp["out"], keep, "fused norm")


@pytest.mark.parametrize("in_place", [False, True])
def test_ragged_batch(in_place):
    all_ops_full(ragged(), in_place=in_place)


def test_head_dim_64_with_3d_sections_and_gqa():
    all_ops_full(ragged(head_dim=64, sections=(24, 20, 20), hq=4, hk=2, hidden=264, inner=520))


@pytest.mark.parametrize("mode", ["interleaved", "half", "none"])
@pytest.mark.parametrize("head_dim,sections", [(64, (24, 20, 20)), (128, (44, 42, 42)), (256, (88, 84, 84))])
def test_rope_modes_and_head_dims(mode, head_dim, sections):
    w = ragged(head_dim=head_dim, sections=sections, hq=3, hk=2, hidden=264, inner=264, seed=head_dim)
    rows = w.valid_rows()
    inp = W.qk_inputs(w)
    q, k = P.gpu_qk(w, inp, rope_mode=mode)
    qo, ko = P.oracle_qk(w, inp, rows, rope_mode=mode)
    P.assert_close(P.gather_rows(q, rows), qo[rows], f"q {mode} {head_dim}")
    P.assert_close(P.gather_rows(k, rows), ko[rows], f"k {mode} {head_dim}")
    keep = P.untouched_rows(w)
    P.assert_untouched(q, inp["q"], keep, "q")
    P.assert_untouched(k, inp["k"], keep, "k")


@pytest.mark.parametrize("sections", [(64, 0, 64), (0, 64, 64), (64, 64, 0), (2, 124, 2)])
@pytest.mark.parametrize("mode", ["interleaved", "half"])
def test_rope_sections_with_empty_or_tiny_sections(sections, mode):
    """Each pair's frequency is formed on the device from its section's base:
    sections of size 0 (so a lane's pairs jump from the t to the w section) or
    of one pair agree with the oracle."""
    w = ragged(head_dim=128, sections=sections, hq=3, hk=2, hidden=264, inner=264, seed=sum(sections[:2]) + 7)
    rows = w.valid_rows()
    inp = W.qk_inputs(w)
    q, k = P.gpu_qk(w, inp, rope_mode=mode)
    qo, ko = P.oracle_qk(w, inp, rows, rope_mode=mode)
    P.assert_close(P.gather_rows(q, rows), qo[rows], f"q {mode} {sections}")
    P.assert_close(P.gather_rows(k, rows), ko[rows], f"k {mode} {sections}")


def test_rope_grid_beyond_32_bit_planes():
    """A grid whose H x W plane passes 2^32 (1 x 70000 x 70000): the row's 3D
    position takes the 64-bit divisions instead of the 32-bit ones, and rows
    past W wrap to the next h; against the oracle, in both rotating layouts."""
    lengths, padded = (300, 77000), (304, 77056)
    w = W.custom("wide", lengths, padded, hidden=264, num_q_heads=2, num_k_heads=1, head_dim=128, inner=264,
                 grids=((2, 3, 5), (1, 70000, 70000)), sections=(44, 42, 42), seed=12)
    rows = W.sample_rows(w, per_seq=256)
    for mode in ("interleaved", "half"):
        inp = W.qk_inputs(w)
        q, k = P.gpu_qk(w, inp, rope_mode=mode)
        qo, ko = P.oracle_qk(w, inp, rows, rope_mode=mode)
        P.assert_close(P.gather_rows(q, rows), qo[rows], f"q {mode}")
        P.assert_close(P.gather_rows(k, rows), ko[rows], f"k {mode}")


def test_half_split_video_full_size_sampled():
    w = W.workload("video")
    rows = W.sample_rows(w, per_seq=64)
    inp = W.qk_inputs(w)
    q, k = P.gpu_qk(w, inp, rope_mode="half")
    qo, ko = P.oracle_qk(w, inp, rows, rope_mode="half")
    P.assert_close(P.gather_rows(q, rows), qo[rows], "q half video")
    P.assert_close(P.gather_rows(k, rows), ko[rows], "k half video")


def test_1d_only_and_degenerate_sections():
    w = W.custom("1d", (77, 3), (80, 8), hidden=512, num_q_heads=2, num_k_heads=2, head_dim=128, inner=256)
    all_ops_full(w)
    # a 1 x 1 x W grid whose only section is w reproduces the 1D rotation
    w3 = W.custom("1d", (77, 3), (80, 8), hidden=512, num_q_heads=2, num_k_heads=2, head_dim=128, inner=256,
                  grids=((1, 1, 77), (1, 1, 3)), sections=(0, 0, 128))
    inp = W.qk_inputs(w)
    a = P.gpu_qk(w, inp)
    b = P.gpu_qk(w3, inp)
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))


def test_many_sequences():
    rng = np.random.default_rng(11)
    lengths = rng.integers(0, 21, 300)
    padded = [-(-int(L) // 8) * 8 + 8 * int(rng.integers(0, 2)) for L in lengths]
    grids = [(int(L) // 4, 2, 2) if L >= 4 else (0, 0, 0) for L in lengths]
    w = W.custom("many", lengths, padded, hidden=256, num_q_heads=2, num_k_heads=2, head_dim=64, inner=264,
                 grids=grids, sections=(22, 22, 20))
    all_ops_full(w)


def test_fused_qkv_slices_and_wide_out_stride():
    w = ragged()
    inp = W.qk_inputs(w)
    qw, kw = w.qk_width
    # [rows, q | k | v] buffer: q and k are column slices with row stride qw + 2 kw
    qkv = torch.cat([inp["q"], inp["k"], inp["k"]], dim=1).cuda()
    cs, cp, grid = P.device_packing(w)
    rv = W.rows_view(qkv)
    dit.dit_qk_rmsnorm_rope(rv[:, :qw], rv[:, qw:qw + kw], inp["q_weight"].cuda(), inp["k_weight"].cuda(),
                            cs, cp, num_q_heads=w.num_q_heads, num_k_heads=w.num_k_heads, head_dim=w.head_dim,
                            rope_grid=grid, sections=w.sections, rope_theta=w.rope_theta, eps=w.eps)
    q, k = P.gpu_qk(w, inp)
    assert torch.equal(qkv[:, :qw].contiguous().view(torch.int16), q.view(torch.int16))
    assert torch.equal(qkv[:, qw:qw + kw].contiguous().view(torch.int16), k.view(torch.int16))
    assert torch.equal(qkv[:, qw + kw:].cpu().view(torch.int16), inp["k"].view(torch.int16))  # v untouched
    # adaLN into a wider output buffer (row stride 3 * hidden)
    inp = W.adaln_inputs(w)
    wide = W.sentinel_like((inp["x"].shape[0], 3 * w.hidden)).cuda()
    mod = inp["mod"].cuda()
    dit.dit_adaln_modulate(W.rows_view(inp["x"].cuda()), mod[:, 0], mod[:, 1], cs, cp,
                           out=W.rows_view(wide)[:, w.hidden:2 * w.hidden], eps=w.eps)
    ref = P.gpu_adaln(w, inp)
    assert torch.equal(wide[:, w.hidden:2 * w.hidden].contiguous().view(torch.int16), ref.view(torch.int16))
    assert torch.all(wide[:, :w.hidden].view(torch.int16) == W.SENTINEL)


@pytest.mark.parametrize("hidden", [8, 256, 264, 2048, 2056, 3072, 4096, 5120, 6136, 6144, 6152, 8192, 16384])
def test_adaln_every_team_shape(hidden):
    w = W.custom("adaln", (13, 6), (16, 8), hidden=hidden, num_q_heads=1, num_k_heads=1, head_dim=64,
                 inner=8, seed=hidden)
    rows = w.valid_rows()
    inp = W.adaln_inputs(w)
    out = P.gpu_adaln(w, inp)
    P.assert_close(P.gather_rows(out, rows), P.oracle_adaln(w, inp, rows)[rows], f"adaln {hidden}")
    P.assert_untouched(out, inp["out"], P.untouched_rows(w), "adaln")
    inp = W.residual_inputs(w)
    res, norm = P.gpu_fused(w, inp)
    r_ref, n_ref = P.oracle_fused(w, inp, rows)
    P.assert_close(P.gather_rows(res, rows), r_ref[rows], f"fused residual {hidden}")
    P.assert_close(P.gather_rows(norm, rows), n_ref[rows], f"fused norm {hidden}")


@pytest.mark.parametrize("offset", [0, 8, 16])
def test_adaln_row_alignment(offset):
    """adaLN reads and writes 32 bytes per lane access when every row starts
    on a 32-byte boundary and 16 bytes otherwise: rows starting `offset`
    elements into a wider buffer (8: 16-byte aligned only) agree with the
    oracle either way, in place too."""
    w = W.custom("adaln_al", (300, 77), (304, 80), hidden=3072, num_q_heads=1, num_k_heads=1, head_dim=64,
                 inner=8, seed=41)
    C, rows = w.hidden, w.valid_rows()
    inp = W.adaln_inputs(w)
    ref = P.oracle_adaln(w, inp, rows)
    cs, cp, _ = P.device_packing(w)
    mod = inp["mod"].cuda()
    buf = W.sentinel_like((inp["x"].shape[0], C + 32)).cuda()
    buf[:, offset:offset + C] = inp["x"].cuda()
    x = W.rows_view(buf)[:, offset:offset + C]
    out = W.sentinel_like((inp["x"].shape[0], C + 32)).cuda()
    o = W.rows_view(out)[:, offset:offset + C]
    dit.dit_adaln_modulate(x, mod[:, 0], mod[:, 1], cs, cp, out=o, eps=w.eps)
    dit.dit_adaln_modulate(x, mod[:, 0], mod[:, 1], cs, cp, out=x, eps=w.eps)   # in place
    torch.cuda.synchronize()
    for name, t in (("out", out), ("in place", buf)):
        got = P.gather_rows(t[:, offset:offset + C].contiguous(), rows)
        P.assert_close(got, ref[rows], f"adaln offset {offset} {name}")
        # columns outside the row slice are untouched
        assert torch.all(t[:, :offset].view(torch.int16) == W.SENTINEL)
        assert torch.all(t[:, offset + C:].view(torch.int16) == W.SENTINEL)


@pytest.mark.parametrize("width", [8, 64, 504, 512, 520, 1024, 1032, 2048, 5632, 13824])
def test_swiglu_and_residual_every_width(width):
    """Every launch shape of SwiGLU and the gated residual: one, two or more
    vectors per lane, 32-byte accesses (widths that are multiples of 16) and
    16-byte ones (the others), against the oracle."""
    w = W.custom("widths", (37, 5, 90), (40, 8, 96), hidden=width, num_q_heads=1, num_k_heads=1, head_dim=64,
                 inner=width, seed=width + 3)
    rows = w.valid_rows()
    inp = W.swiglu_inputs(w)
    out = P.gpu_swiglu(w, inp)
    P.assert_close(P.gather_rows(out, rows), P.oracle_swiglu(w, inp, rows)[rows], f"swiglu {width}")
    P.assert_untouched(out, inp["out"], P.untouched_rows(w), f"swiglu {width}")
    inp = W.residual_inputs(w)
    out = P.gpu_residual(w, inp)
    P.assert_close(P.gather_rows(out, rows), P.oracle_residual(w, inp, rows)[rows], f"residual {width}")
    P.assert_untouched(out, inp["out"], P.untouched_rows(w), f"residual {width}")


def test_swiglu_extreme_activations():
    w = W.custom("sw", (5,), (8,), hidden=8, num_q_heads=1, num_k_heads=1, head_dim=64, inner=64)
    inp = W.swiglu_inputs(w)
    vals = torch.tensor([0.0, -0.0, 1.0, -1.0, 20.0, -20.0, 88.0, -88.0, 100.0, -100.0, 1e-3, -1e-3,
                         3.0e4, -3.0e4, 0.5, -0.5] * 4, dtype=torch.float32)
    ab = W.rows_view(inp["ab"])
    ab[:5, :64] = vals.to(torch.bfloat16)
    rows = w.valid_rows()
    out = P.gpu_swiglu(w, inp)
    P.assert_close(P.gather_rows(out, rows), P.oracle_swiglu(w, inp, rows)[rows], "swiglu extremes")


def test_empty_batches():
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    cs = torch.zeros(1, dtype=torch.int32, device="cuda")
    g = torch.zeros(1, 64, dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(x, 7.0)
    dit.dit_gated_residual(x, x, g, cs, cs, out=out)          # num_seqs = 0
    dit.dit_swiglu(x, x, cs, cs, out=out)
    w = W.custom("zero", (0, 0), (4, 4), hidden=64, num_q_heads=1, num_k_heads=1, head_dim=64, inner=64)
    inp = W.residual_inputs(w)
    o = P.gpu_residual(w, inp)                               # all sequences empty
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)
    assert torch.equal(o.cpu().view(torch.int16), inp["out"].view(torch.int16))


def test_malformed_device_descriptors_are_skipped_and_flagged():
    w = W.custom("bad", (10, 6), (8, 8), hidden=64, num_q_heads=1, num_k_heads=1, head_dim=64, inner=64)
    # sequence 0 claims 10 valid rows in an 8-row slot; the second slot ends
    # past the 16-row buffer (cu_seqlens_padded = [0, 8, 20]).
    inp = W.residual_inputs(w)
    x, y, out = inp["x"].cuda(), inp["y"].cuda(), inp["out"].cuda()
    mod = inp["mod"].cuda()
    cs = torch.tensor([0, 10, 16], dtype=torch.int32, device="cuda")
    cp = torch.tensor([0, 8, 20], dtype=torch.int32, device="cuda")
    dit.dit_gated_residual(W.rows_view(x), W.rows_view(y), mod[:, 2], cs, cp, out=W.rows_view(out))
    flag = dit.dit_validate_seqlens(cs, cp, 16)
    torch.cuda.synchronize()
    assert flag.tolist() == [1, 0]
    o = out.cpu()
    assert torch.all(o[:W.CANARY_ROWS].view(torch.int16) == W.SENTINEL)
    assert torch.all(o[-W.CANARY_ROWS:].view(torch.int16) == W.SENTINEL)
    # rows 0..7 (sequence 0, clamped to its slot) and 8..13 (sequence 1) are written
    assert not torch.any(o[W.CANARY_ROWS:W.CANARY_ROWS + 14].view(torch.int16) == W.SENTINEL)
    assert torch.all(o[W.CANARY_ROWS + 14:W.CANARY_ROWS + 16].view(torch.int16) == W.SENTINEL)
    good = dit.dit_validate_seqlens(torch.tensor([0, 6, 12], dtype=torch.int32, device="cuda"),
                                    torch.tensor([0, 8, 16], dtype=torch.int32, device="cuda"), 16)
    cp2 = torch.tensor([0, 8, 16], dtype=torch.int32, device="cuda")
    cs2 = torch.tensor([0, 5, 4], dtype=torch.int32, device="cuda")   # decreasing
    bad2 = dit.dit_validate_seqlens(cs2, cp2, 16)
    torch.cuda.synchronize()
    assert good.tolist()[0] == 0 and bad2.tolist() == [1, 1]
    # an empty batch is still checked for its leading entries
    z = torch.zeros(1, dtype=torch.int32, device="cuda")
    one = torch.ones(1, dtype=torch.int32, device="cuda")
    empty_ok = dit.dit_validate_seqlens(z, z, 0)
    empty_bad = dit.dit_validate_seqlens(one, z, 0)
    empty_bad_p = dit.dit_validate_seqlens(z, one, 4)
    torch.cuda.synchronize()
    assert empty_ok.tolist() == [0, -1]
    assert empty_bad.tolist() == [1, 0] and empty_bad_p.tolist() == [1, 0]


def test_check_seqlens_raises_on_malformed_descriptors():
    ok_cs = torch.tensor([0, 6, 12], dtype=torch.int32, device="cuda")
    ok_cp = torch.tensor([0, 8, 16], dtype=torch.int32, device="cuda")
    dit.check_seqlens(ok_cs, ok_cp, 16)
    with pytest.raises(dit.DitError) as e:
        dit.check_seqlens(torch.tensor([0, 9, 12], dtype=torch.int32, device="cuda"), ok_cp, 16)
    assert e.value.status == 5
    with pytest.raises(dit.DitError):
        dit.check_seqlens(ok_cs, ok_cp, 12)   # the descriptor runs past the buffer


def test_gqa_at_scale_and_thousands_of_sequences():
    # 40 query heads sharing 8 key heads over a 16k-row batch of the big shapes
    lengths = [4000, 7000, 5000]
    padded = [-(-L // 128) * 128 for L in lengths]
    w = W.custom("gqa", lengths, padded, hidden=5120, num_q_heads=40, num_k_heads=8, head_dim=128, inner=8,
                 grids=[(L // 1008, 24, 42) for L in lengths], sections=(44, 42, 42), seed=21)
    rows = W.sample_rows(w, per_seq=48)
    inp = W.qk_inputs(w)
    q, k = P.gpu_qk(w, inp)
    qo, ko = P.oracle_qk(w, inp, rows)
    P.assert_close(P.gather_rows(q, rows), qo[rows], "q gqa")
    P.assert_close(P.gather_rows(k, rows), ko[rows], "k gqa")
    # 2500 sequences: the sequence search takes three 32-way levels
    rng = np.random.default_rng(5)
    lengths = rng.integers(0, 6, 2500)
    padded = [int(L) + int(rng.integers(0, 3)) for L in lengths]
    w = W.custom("many2", lengths, padded, hidden=64, num_q_heads=1, num_k_heads=1, head_dim=64, inner=64, seed=3)
    all_ops_full(w)


def test_vae_like_shapes():
    """Q/K normalization without rotation and SwiGLU at VAE-like shapes: one
    sequence of 2^18 tokens, 512 channels as 8 heads of 64, SwiGLU inner 512."""
    n = 1 << 18
    w = W.custom("vae", (n,), (n,), hidden=512, num_q_heads=8, num_k_heads=8, head_dim=64, inner=512, seed=4)
    rows = W.sample_rows(w, per_seq=2000)
    inp = W.qk_inputs(w)
    q, k = P.gpu_qk(w, inp, rope_mode="none")
    qo, ko = P.oracle_qk(w, inp, rows, rope_mode="none")
    P.assert_close(P.gather_rows(q, rows), qo[rows], "vae q")
    P.assert_close(P.gather_rows(k, rows), ko[rows], "vae k")
    sw = W.swiglu_inputs(w)
    out = P.gpu_swiglu(w, sw)
    P.assert_close(P.gather_rows(out, rows), P.oracle_swiglu(w, sw, rows)[rows], "vae swiglu")


@pytest.mark.parametrize("mode", ["interleaved", "half"])
@pytest.mark.parametrize("sliced", [False, True])
def test_small_rows_many_sequences(mode, sliced):
    """Rows of 256 bytes (one q and one k head of 64) in the tens of
    thousands, ragged 3D grids with 1D tails, empty sequences, and (when
    sliced) per-sequence position offsets, all against the oracle."""
    rng = np.random.default_rng(21 if sliced else 20)
    B = 160
    lengths = rng.integers(0, 400, B)
    lengths[::37] = 0
    padded = lengths + rng.integers(0, 9, B)
    grids = np.stack([rng.integers(0, 4, B), rng.integers(1, 7, B), rng.integers(1, 9, B)], axis=1)
    w = W.custom("small", lengths, padded, hidden=64, num_q_heads=1, num_k_heads=1, head_dim=64, inner=64,
                 grids=grids, sections=(24, 20, 20), seed=9)
    po = rng.integers(0, 60, B).astype(np.int32) if sliced else None
    inp = W.qk_inputs(w)
    cs, cp, grid = P.device_packing(w)
    q, k = inp["q"].cuda(), inp["k"].cuda()
    dit.dit_qk_rmsnorm_rope(W.rows_view(q), W.rows_view(k), inp["q_weight"].cuda(), inp["k_weight"].cuda(), cs, cp,
                            num_q_heads=1, num_k_heads=1, head_dim=64, rope_grid=grid, sections=w.sections,
                            rope_theta=w.rope_theta, eps=w.eps, rope_mode=mode,
                            pos_offset=None if po is None else torch.from_numpy(po).cuda())
    rows = w.valid_rows()
    import oracle
    from _util import tbits
    qo, ko = oracle.qk_rmsnorm_rope(tbits(W.rows_view(inp["q"])), tbits(W.rows_view(inp["k"])),
                                    tbits(inp["q_weight"]), tbits(inp["k_weight"]), w.cu_seqlens,
                                    w.cu_seqlens_padded, num_q_heads=1, num_k_heads=1, head_dim=64,
                                    rope_grid=w.rope_grid, sections=w.sections, rope_theta=w.rope_theta,
                                    eps=w.eps, rope_mode=mode, pos_offset=po)
    P.assert_close(P.gather_rows(q, rows), qo[rows], f"small rows q {mode}")
    P.assert_close(P.gather_rows(k, rows), ko[rows], f"small rows k {mode}")
    keep = P.untouched_rows(w)
    P.assert_untouched(q, inp["q"], keep, "small rows q")
    P.assert_untouched(k, inp["k"], keep, "small rows k")


def test_negative_position_offset_reads_as_zero():
    """pos_offset entries are documented as >= 0; a negative one is read as 0
    (whole-sequence positions from the slice's own first row), including with
    an empty grid, and nothing outside the valid rows is written."""
    w = W.custom("negoff", (40, 30), (48, 32), hidden=256, num_q_heads=1, num_k_heads=1, head_dim=128, inner=64,
                 grids=((1, 4, 5), (0, 0, 7)), sections=(44, 42, 42), seed=31)
    inp = W.qk_inputs(w)
    cs, cp, grid = P.device_packing(w)
    outs = []
    for offs in ([0, 0], [-5, -1000]):
        q, k = inp["q"].cuda(), inp["k"].cuda()
        dit.dit_qk_rmsnorm_rope(W.rows_view(q), W.rows_view(k), inp["q_weight"].cuda(), inp["k_weight"].cuda(),
                                cs, cp, num_q_heads=1, num_k_heads=1, head_dim=128, rope_grid=grid,
                                sections=w.sections, rope_theta=w.rope_theta, eps=w.eps,
                                pos_offset=torch.tensor(offs, dtype=torch.int32, device="cuda"))
        outs.append((q, k))
    torch.cuda.synchronize()
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    keep = P.untouched_rows(w)
    P.assert_untouched(outs[1][0], inp["q"], keep, "negative offset q")
    P.assert_untouched(outs[1][1], inp["k"], keep, "negative offset k")
