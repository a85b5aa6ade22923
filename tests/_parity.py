"""Shared parity machinery: run an operator through the C ABI on the GPU and
through the CPU oracle on the same seeded inputs, compare element by element,
and check that padding and canary rows are bit-identical afterwards."""
import numpy as np
import torch

import dit_token_b200 as dit
import oracle
from dit_token_b200 import workloads as W
from _util import f64, tbits

ABS_TOL, REL_TOL = 2e-2, 1e-2


def _values(b: np.ndarray) -> torch.Tensor:
    """bf16 bit patterns (uint16) -> exact fp64 values, as a CPU tensor."""
    t = torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).to(torch.int32) << 16
    return t.view(torch.float32).to(torch.float64)


def assert_close(gpu_bits, ref_bits, what="", chunk=1 << 26):
    """|gpu - ref| <= max(2e-2, 1e-2 |ref|) elementwise, ref = the oracle's
    fp64 result rounded once to bf16; both must be finite.  Works through the
    arrays in chunks (multi-threaded torch CPU arithmetic), so whole
    full-size outputs can be compared.  Returns the largest |gpu - ref|."""
    g_all = np.asarray(gpu_bits, dtype=np.uint16).reshape(-1)
    r_all = np.asarray(ref_bits, dtype=np.uint16).reshape(-1)
    assert np.shape(gpu_bits) == np.shape(ref_bits), f"{what}: shapes differ"
    worst = 0.0
    for lo in range(0, g_all.size, chunk):
        g, r = _values(g_all[lo:lo + chunk]), _values(r_all[lo:lo + chunk])
        assert bool(torch.isfinite(r).all()), f"{what}: oracle produced non-finite values"
        if not bool(torch.isfinite(g).all()):
            idx = torch.nonzero(~torch.isfinite(g))[:5].flatten() + lo
            raise AssertionError(f"{what}: GPU produced non-finite values at flat indices {idx.tolist()}")
        err = (g - r).abs()
        tol = torch.clamp(REL_TOL * r.abs(), min=ABS_TOL)
        bad = err > tol
        if bool(bad.any()):
            idx = torch.nonzero(bad)[:5].flatten()
            shape = np.shape(gpu_bits)
            raise AssertionError(
                f"{what}: {int(bad.sum())} elements of chunk {lo // chunk} out of tolerance, e.g. "
                + ", ".join(f"{np.unravel_index(int(i) + lo, shape)}: gpu {float(g[i])} ref {float(r[i])}"
                            for i in idx))
        if err.numel():
            worst = max(worst, float(err.max()))
    return worst


def untouched_rows(w: W.Workload) -> np.ndarray:
    """Indices, in a canary-framed buffer, of every row an operator must not
    touch: the canary rows at both ends and every padding row."""
    n = w.num_rows_padded + 2 * W.CANARY_ROWS
    keep = np.ones(n, dtype=bool)
    keep[W.CANARY_ROWS + w.valid_rows()] = False
    return np.nonzero(keep)[0]


def assert_untouched(dev_buf: torch.Tensor, host_before: torch.Tensor, rows: np.ndarray, what=""):
    idx = torch.from_numpy(rows).to(dev_buf.device)
    after = dev_buf.index_select(0, idx).view(torch.int16)
    before = host_before.index_select(0, torch.from_numpy(rows)).view(torch.int16).to(dev_buf.device)
    assert torch.equal(after, before), f"{what}: a padding or canary row changed"


def device_packing(w: W.Workload):
    cs = torch.from_numpy(w.cu_seqlens).cuda()
    cp = torch.from_numpy(w.cu_seqlens_padded).cuda()
    grid = None if w.rope_grid is None else torch.from_numpy(w.rope_grid).cuda()
    return cs, cp, grid


# ------------------------------------------------------------ GPU runs

def gpu_qk(w, inp, rope_mode="interleaved"):
    cs, cp, grid = device_packing(w)
    q = inp["q"].cuda()
    k = inp["k"].cuda()
    po = None if w.pos_offset is None else torch.from_numpy(w.pos_offsets).cuda()
    dit.dit_qk_rmsnorm_rope(W.rows_view(q), W.rows_view(k), inp["q_weight"].cuda(), inp["k_weight"].cuda(),
                            cs, cp, num_q_heads=w.num_q_heads, num_k_heads=w.num_k_heads,
                            head_dim=w.head_dim, rope_grid=grid, sections=w.sections,
                            rope_theta=w.rope_theta, eps=w.eps, rope_mode=rope_mode, pos_offset=po)
    return q, k


def gpu_adaln(w, inp, in_place=False):
    cs, cp, _ = device_packing(w)
    x = inp["x"].cuda()
    mod = inp["mod"].cuda()
    out = x if in_place else inp["out"].cuda()
    dit.dit_adaln_modulate(W.rows_view(x), mod[:, 0], mod[:, 1], cs, cp, out=W.rows_view(out), eps=w.eps)
    return out


def gpu_residual(w, inp, in_place=False):
    cs, cp, _ = device_packing(w)
    x = inp["x"].cuda()
    y = inp["y"].cuda()
    mod = inp["mod"].cuda()
    out = x if in_place else inp["out"].cuda()
    dit.dit_gated_residual(W.rows_view(x), W.rows_view(y), mod[:, 2], cs, cp, out=W.rows_view(out))
    return out


def gpu_fused(w, inp, in_place=False):
    """Gated residual (gate = mod[:, 2]) fused with the MLP sublayer's adaLN
    (shift = mod[:, 3], scale = mod[:, 4]); returns (res, norm) buffers."""
    cs, cp, _ = device_packing(w)
    x = inp["x"].cuda()
    y = inp["y"].cuda()
    mod = inp["mod"].cuda()
    res = x if in_place else inp["out"].cuda()
    norm = W.sentinel_like(inp["out"].shape).cuda()
    dit.dit_gated_residual_adaln(W.rows_view(x), W.rows_view(y), mod[:, 2], mod[:, 3], mod[:, 4], cs, cp,
                                 res_out=W.rows_view(res), norm_out=W.rows_view(norm), eps=w.eps)
    return res, norm


def gpu_swiglu(w, inp):
    cs, cp, _ = device_packing(w)
    ab = W.rows_view(inp["ab"].cuda())
    out = inp["out"].cuda()
    dit.dit_swiglu(ab[:, : w.inner], ab[:, w.inner:], cs, cp, out=W.rows_view(out))
    return out


# ------------------------------------------------------------ oracle runs

def oracle_qk(w, inp, rows, rope_mode="interleaved"):
    q = tbits(W.rows_view(inp["q"]))
    k = tbits(W.rows_view(inp["k"]))
    return oracle.qk_rmsnorm_rope(q, k, tbits(inp["q_weight"]), tbits(inp["k_weight"]), w.cu_seqlens,
                                  w.cu_seqlens_padded, num_q_heads=w.num_q_heads,
                                  num_k_heads=w.num_k_heads, head_dim=w.head_dim, rope_grid=w.rope_grid,
                                  sections=w.sections, rope_theta=w.rope_theta, eps=w.eps, rows=rows,
                                  rope_mode=rope_mode, pos_offset=w.pos_offsets)


def mod_flat(mod: torch.Tensor) -> np.ndarray:
    """The [num_seqs, 6, hidden] modulation tensor flattened for the oracle:
    bf16 bit patterns (uint16) or fp32 values, as the tensor holds them."""
    if mod.dtype == torch.float32:
        return np.ascontiguousarray(mod.detach().cpu().numpy().reshape(-1))
    return np.ascontiguousarray(tbits(mod).reshape(-1))


def oracle_adaln(w, inp, rows):
    x = tbits(W.rows_view(inp["x"]))
    flat = mod_flat(inp["mod"])
    return oracle.adaln_modulate(x, flat, flat[w.hidden:], w.cu_seqlens, w.cu_seqlens_padded,
                                 hidden=w.hidden, eps=w.eps, mod_seq_stride=6 * w.hidden, rows=rows)


def oracle_residual(w, inp, rows):
    x = tbits(W.rows_view(inp["x"]))
    y = tbits(W.rows_view(inp["y"]))
    flat = mod_flat(inp["mod"])
    return oracle.gated_residual(x, y, flat[2 * w.hidden:], w.cu_seqlens, w.cu_seqlens_padded,
                                 hidden=w.hidden, gate_seq_stride=6 * w.hidden, rows=rows)


def oracle_fused(w, inp, rows):
    x = tbits(W.rows_view(inp["x"]))
    y = tbits(W.rows_view(inp["y"]))
    flat = mod_flat(inp["mod"])
    C = w.hidden
    return oracle.gated_residual_adaln(x, y, flat[2 * C:], flat[3 * C:], flat[4 * C:], w.cu_seqlens,
                                       w.cu_seqlens_padded, hidden=C, eps=w.eps, gate_seq_stride=6 * C,
                                       mod_seq_stride=6 * C, rows=rows)


def oracle_swiglu(w, inp, rows):
    ab = tbits(W.rows_view(inp["ab"]))              # [rows, 2I], no copy of the halves
    flat = ab.reshape(-1)
    return oracle.swiglu(ab, flat[w.inner:], w.cu_seqlens, w.cu_seqlens_padded, inner=w.inner,
                         a_row_stride=2 * w.inner, b_row_stride=2 * w.inner, nrows=ab.shape[0], rows=rows)


def gather_rows(dev_buf: torch.Tensor, rows: np.ndarray) -> np.ndarray:
    """Bits of padded rows ``rows`` of a canary-framed device buffer."""
    idx = torch.from_numpy(rows + W.CANARY_ROWS).to(dev_buf.device)
    return tbits(dev_buf.index_select(0, idx))
