"""ctypes front end of the CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY.  Only the tests, the package entry point's smoke
check and the benchmark's CPU-baseline leg import this module; the product
path (dit_token_b200) never does.

Every function takes numpy arrays of raw bf16 bit patterns (uint16) and
returns new output arrays: the bf16 result (uint16, same layout as the input,
padding rows left as given by ``out_init``) and, when asked for, the fp64
result before rounding.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        # DIT_ORACLE_LIB lets the mutation tests load a deliberately broken copy.
        path = os.environ.get("DIT_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        i32p = ctypes.POINTER(ctypes.c_int32)
        i64p = ctypes.POINTER(ctypes.c_int64)
        f64p = ctypes.POINTER(ctypes.c_double)
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        L.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f64.restype = f64
        L.oracle_f64_to_bf16.argtypes = [f64]
        L.oracle_f64_to_bf16.restype = ctypes.c_uint16
        L.oracle_qk_rmsnorm_rope.argtypes = [
            u16p, i64, u16p, i64, u16p, u16p, i32p, i32p, i32, i64, i32, i32, i32,
            i32p, i32, i32, i32, f64, f64, u16p, u16p, f64p, f64p, i64p, i64]
        L.oracle_qk_rmsnorm_rope_ex.argtypes = [
            u16p, i64, u16p, i64, u16p, u16p, i32p, i32p, i32, i64, i32, i32, i32,
            i32p, i32, i32, i32, f64, f64, i32, u16p, u16p, f64p, f64p, i64p, i64]
        L.oracle_qk_rmsnorm_rope_shard.argtypes = [
            u16p, i64, u16p, i64, u16p, u16p, i32p, i32p, i32, i64, i32, i32, i32,
            i32p, i32, i32, i32, f64, f64, i32, i32p, u16p, u16p, f64p, f64p, i64p, i64]
        L.oracle_adaln_modulate.argtypes = [
            u16p, i64, u16p, u16p, i64, i32p, i32p, i32, i64, i32, f64, u16p, i64, f64p, i64p, i64]
        L.oracle_gated_residual.argtypes = [
            u16p, i64, u16p, i64, u16p, i64, i32p, i32p, i32, i64, i32, u16p, i64, f64p, i64p, i64]
        L.oracle_gated_residual_adaln.argtypes = [
            u16p, i64, u16p, i64, u16p, i64, u16p, u16p, i64, i32p, i32p, i32, i64, i32, f64,
            u16p, i64, u16p, i64, f64p, i64p, i64]
        vp = ctypes.c_void_p
        L.oracle_adaln_modulate_ex.argtypes = [
            u16p, i64, vp, vp, i64, i32, i32p, i32p, i32, i64, i32, f64, u16p, i64, f64p, i64p, i64]
        L.oracle_gated_residual_ex.argtypes = [
            u16p, i64, u16p, i64, vp, i64, i32, i32p, i32p, i32, i64, i32, u16p, i64, f64p, i64p, i64]
        L.oracle_gated_residual_adaln_ex.argtypes = [
            u16p, i64, u16p, i64, vp, i64, vp, vp, i64, i32, i32p, i32p, i32, i64, i32, f64,
            u16p, i64, u16p, i64, f64p, i64p, i64]
        L.oracle_adaln_modulate_av.argtypes = [
            u16p, i64, vp, vp, i64, i32, i32p, i32p, i64, i32p, i32p, i32, i64, i32, f64, u16p, i64, f64p, i64p, i64]
        L.oracle_gated_residual_av.argtypes = [
            u16p, i64, u16p, i64, vp, i64, i32, i32p, i32p, i64, i32p, i32p, i32, i64, i32, u16p, i64, f64p, i64p,
            i64]
        L.oracle_gated_residual_adaln_av.argtypes = [
            u16p, i64, u16p, i64, vp, i64, vp, vp, i64, i32, i32p, i32p, i64, i64, i32p, i32p, i32, i64, i32, f64,
            u16p, i64, u16p, i64, f64p, i64p, i64]
        L.oracle_swiglu.argtypes = [
            u16p, i64, u16p, i64, i32p, i32p, i32, i64, i32, u16p, i64, f64p, i64p, i64]
        L.oracle_frames_to_u8.argtypes = [ctypes.POINTER(ctypes.c_float), i64, i64, i64, i64, i64, i32,
                                          ctypes.POINTER(ctypes.c_uint8)]
        for name in ("oracle_qk_rmsnorm_rope", "oracle_qk_rmsnorm_rope_ex", "oracle_adaln_modulate",
                     "oracle_frames_to_u8",
                     "oracle_gated_residual", "oracle_gated_residual_adaln", "oracle_swiglu",
                     "oracle_adaln_modulate_ex", "oracle_gated_residual_ex", "oracle_gated_residual_adaln_ex",
                     "oracle_adaln_modulate_av", "oracle_gated_residual_av", "oracle_gated_residual_adaln_av",
                     "oracle_qk_rmsnorm_rope_shard",
                     "oracle_num_threads"):
            getattr(L, name).restype = ctypes.c_int
        L.oracle_set_num_threads.argtypes = [i32]
        L.oracle_set_num_threads.restype = None
        _lib = L
    return _lib


def _ptr(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _u16(a):
    a = np.asarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected raw bf16 bits as uint16, got {a.dtype}")
    return a


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: invalid arguments (oracle returned {rc})")


def _rows(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, r.size


def _seqlens(cu_seqlens, cu_seqlens_padded):
    cs = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    cp = np.ascontiguousarray(np.asarray(cu_seqlens_padded, dtype=np.int32))
    return cs, cp


def _flat_view(a, row_stride, rows_padded):
    """The array as a flat uint16 buffer plus its row stride in elements."""
    a = np.ascontiguousarray(_u16(a))
    if row_stride is None:
        row_stride = int(np.prod(a.shape[1:])) if a.ndim > 1 else 1
    return a, row_stride


def _mod(a):
    """Per-sequence modulation vectors: raw bf16 bits (uint16) or fp32 values.
    Returns (contiguous array, is_fp32)."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return np.ascontiguousarray(a), 0
    if a.dtype == np.float32:
        return np.ascontiguousarray(a), 1
    raise TypeError(f"modulation vectors must be uint16 (bf16 bits) or float32, got {a.dtype}")


def _vptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def bf16_to_f64(bits: int) -> float:
    return lib().oracle_bf16_to_f64(int(bits))


def f64_to_bf16(x: float) -> int:
    return int(lib().oracle_f64_to_bf16(float(x)))


def f64_to_bf16_array(x) -> np.ndarray:
    f = lib().oracle_f64_to_bf16
    x = np.asarray(x, dtype=np.float64)
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint16).reshape(x.shape)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns (bits << 16 is the binary32 value)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    """OpenMP threads for the following oracle calls (results do not depend on it)."""
    lib().oracle_set_num_threads(int(n))


def qk_rmsnorm_rope(q, k, q_weight, k_weight, cu_seqlens, cu_seqlens_padded, *,
                    num_q_heads, num_k_heads, head_dim, rope_grid=None,
                    sections=(0, 0, 0), rope_theta=10000.0, eps=1e-6,
                    q_row_stride=None, k_row_stride=None, rows=None,
                    q_out_init=None, k_out_init=None, want_f64=False, q_out=None, k_out=None,
                    rope_mode="interleaved", pos_offset=None):
    """Per-head Q/K RMSNorm fused with 1D / 3D rotary embedding.

    rope_mode: "interleaved" (pairs 2j, 2j+1), "half" (pairs j, j + D/2) or
    "none" (RMSNorm only).  pos_offset: int32 [num_seqs] or None -- the rows
    of sequence b are rows pos_offset[b], ... of the whole sequence (one
    rank's slice).

    q, k: uint16 arrays whose first axis is the padded row; row strides
    default to the product of the remaining axes.  Returns (q_out, k_out) or,
    with want_f64, (q_out, k_out, q_f64, k_f64)."""
    cs, cp = _seqlens(cu_seqlens, cu_seqlens_padded)
    B = cs.size - 1
    q, qs = _flat_view(q, q_row_stride, None)
    k, ks = _flat_view(k, k_row_stride, None)
    nrows = q.shape[0]
    if q_out is None:
        q_out = np.array(q if q_out_init is None else q_out_init, dtype=np.uint16, copy=True)
    if k_out is None:
        k_out = np.array(k if k_out_init is None else k_out_init, dtype=np.uint16, copy=True)
    q64 = np.full(q.shape, np.nan) if want_f64 else None
    k64 = np.full(k.shape, np.nan) if want_f64 else None
    grid = None if rope_grid is None else np.ascontiguousarray(np.asarray(rope_grid, dtype=np.int32))
    wq = np.ascontiguousarray(_u16(q_weight))
    wk = np.ascontiguousarray(_u16(k_weight))
    r, nr = _rows(rows)
    L = lib()
    mode = {"interleaved": 0, "half": 1, "none": 2}[rope_mode]
    po = _int32(pos_offset)
    rc = L.oracle_qk_rmsnorm_rope_shard(
        _ptr(q, ctypes.c_uint16), qs, _ptr(k, ctypes.c_uint16), ks,
        _ptr(wq, ctypes.c_uint16), _ptr(wk, ctypes.c_uint16),
        _ptr(cs, ctypes.c_int32), _ptr(cp, ctypes.c_int32), B, nrows,
        num_q_heads, num_k_heads, head_dim,
        _ptr(grid, ctypes.c_int32), *[int(s) for s in sections], float(rope_theta), float(eps), mode,
        _ptr(po, ctypes.c_int32),
        _ptr(q_out, ctypes.c_uint16), _ptr(k_out, ctypes.c_uint16),
        _ptr(q64, ctypes.c_double), _ptr(k64, ctypes.c_double),
        _ptr(r, ctypes.c_int64), nr)
    _check(rc, "qk_rmsnorm_rope")
    if want_f64:
        return q_out, k_out, q64, k64
    return q_out, k_out


def _int32(a):
    """A contiguous int32 copy of an optional integer array (grids, offsets)."""
    return None if a is None else np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def adaln_modulate(x, shift, scale, cu_seqlens, cu_seqlens_padded, *, hidden, eps=1e-6,
                   mod_seq_stride=None, x_row_stride=None, rows=None, out_init=None,
                   want_f64=False, out=None, rope_grid=None, audio_offset=0, pos_offset=None):
    """out = LayerNorm(x) * (1 + scale_b) + shift_b on valid rows.

    shift, scale: uint16 (bf16 bits) or float32 arrays [num_seqs, ...] read
    with mod_seq_stride elements between sequences (default: hidden).
    Per-stream vectors: with rope_grid [num_seqs][3] given, the audio rows of
    sequence b (local index >= T*H*W) read their vectors audio_offset
    elements after the video rows' ones; pos_offset [num_seqs] (or None) is
    where each sequence's rows start in the whole sequence."""
    cs, cp = _seqlens(cu_seqlens, cu_seqlens_padded)
    B = cs.size - 1
    x, xs = _flat_view(x, x_row_stride, None)
    nrows = x.shape[0]
    if out is None:
        out = np.array(x if out_init is None else out_init, dtype=np.uint16, copy=True)
    o64 = np.full(out.shape, np.nan) if want_f64 else None
    sh, f1 = _mod(shift)
    sc, f2 = _mod(scale)
    if f1 != f2:
        raise TypeError("shift and scale must have the same dtype")
    mss = hidden if mod_seq_stride is None else mod_seq_stride
    r, nr = _rows(rows)
    grid = _int32(rope_grid)
    rc = lib().oracle_adaln_modulate_av(
        _ptr(x, ctypes.c_uint16), xs, _vptr(sh), _vptr(sc), mss, f1, _ptr(grid, ctypes.c_int32),
        _ptr(_int32(pos_offset), ctypes.c_int32), audio_offset,
        _ptr(cs, ctypes.c_int32), _ptr(cp, ctypes.c_int32), B, nrows, hidden, float(eps),
        _ptr(out, ctypes.c_uint16), xs, _ptr(o64, ctypes.c_double), _ptr(r, ctypes.c_int64), nr)
    _check(rc, "adaln_modulate")
    return (out, o64) if want_f64 else out


def gated_residual(x, y, gate, cu_seqlens, cu_seqlens_padded, *, hidden, gate_seq_stride=None,
                   x_row_stride=None, y_row_stride=None, rows=None, out_init=None,
                   want_f64=False, out=None, rope_grid=None, audio_offset=0, pos_offset=None):
    """out = x + gate_b * y on valid rows (per-stream gates as in
    adaln_modulate)."""
    cs, cp = _seqlens(cu_seqlens, cu_seqlens_padded)
    B = cs.size - 1
    x, xs = _flat_view(x, x_row_stride, None)
    y, ys = _flat_view(y, y_row_stride, None)
    nrows = x.shape[0]
    if out is None:
        out = np.array(x if out_init is None else out_init, dtype=np.uint16, copy=True)
    o64 = np.full(out.shape, np.nan) if want_f64 else None
    g, gf = _mod(gate)
    gss = hidden if gate_seq_stride is None else gate_seq_stride
    r, nr = _rows(rows)
    grid = _int32(rope_grid)
    rc = lib().oracle_gated_residual_av(
        _ptr(x, ctypes.c_uint16), xs, _ptr(y, ctypes.c_uint16), ys, _vptr(g), gss, gf,
        _ptr(grid, ctypes.c_int32), _ptr(_int32(pos_offset), ctypes.c_int32), audio_offset,
        _ptr(cs, ctypes.c_int32), _ptr(cp, ctypes.c_int32), B, nrows, hidden,
        _ptr(out, ctypes.c_uint16), xs, _ptr(o64, ctypes.c_double), _ptr(r, ctypes.c_int64), nr)
    _check(rc, "gated_residual")
    return (out, o64) if want_f64 else out


def gated_residual_adaln(x, y, gate, shift, scale, cu_seqlens, cu_seqlens_padded, *, hidden, eps=1e-6,
                        gate_seq_stride=None, mod_seq_stride=None, x_row_stride=None, y_row_stride=None,
                        rows=None, res_init=None, norm_init=None, want_f64=False, res_out=None,
                        norm_out=None, rope_grid=None, gate_audio_offset=0, mod_audio_offset=0,
                        pos_offset=None):
    """res = x + gate_b * y (bf16), norm = LN(res) * (1 + scale_b) + shift_b on
    valid rows (per-stream vectors as in adaln_modulate, with one audio
    offset for the gate and one for shift/scale).  Returns (res, norm) or,
    with want_f64, (res, norm, norm_f64)."""
    cs, cp = _seqlens(cu_seqlens, cu_seqlens_padded)
    B = cs.size - 1
    x, xs = _flat_view(x, x_row_stride, None)
    y, ys = _flat_view(y, y_row_stride, None)
    nrows = x.shape[0]
    if res_out is None:
        res_out = np.array(x if res_init is None else res_init, dtype=np.uint16, copy=True)
    if norm_out is None:
        norm_out = np.array(x if norm_init is None else norm_init, dtype=np.uint16, copy=True)
    n64 = np.full(norm_out.shape, np.nan) if want_f64 else None
    g, f0 = _mod(gate)
    sh, f1 = _mod(shift)
    sc, f2 = _mod(scale)
    if not (f0 == f1 == f2):
        raise TypeError("gate, shift and scale must have the same dtype")
    gss = hidden if gate_seq_stride is None else gate_seq_stride
    mss = hidden if mod_seq_stride is None else mod_seq_stride
    r, nr = _rows(rows)
    grid = _int32(rope_grid)
    rc = lib().oracle_gated_residual_adaln_av(
        _ptr(x, ctypes.c_uint16), xs, _ptr(y, ctypes.c_uint16), ys, _vptr(g), gss,
        _vptr(sh), _vptr(sc), mss, f1, _ptr(grid, ctypes.c_int32), _ptr(_int32(pos_offset), ctypes.c_int32),
        gate_audio_offset, mod_audio_offset,
        _ptr(cs, ctypes.c_int32), _ptr(cp, ctypes.c_int32), B, nrows, hidden, float(eps),
        _ptr(res_out, ctypes.c_uint16), xs, _ptr(norm_out, ctypes.c_uint16), xs, _ptr(n64, ctypes.c_double),
        _ptr(r, ctypes.c_int64), nr)
    _check(rc, "gated_residual_adaln")
    return (res_out, norm_out, n64) if want_f64 else (res_out, norm_out)


def swiglu(a, b, cu_seqlens, cu_seqlens_padded, *, inner, a_row_stride=None, b_row_stride=None,
           out_row_stride=None, nrows=None, rows=None, out_init=None, want_f64=False, out=None):
    """out = silu(a) * b on valid rows.

    a, b: uint16 arrays whose first axis is the padded row (for a chunked
    [rows, 2*inner] buffer pass its two column halves).  The output has
    ``out_row_stride`` (default ``inner``) elements per row; rows the oracle
    does not write keep ``out_init`` (default: the bf16 NaN 0x7FC1)."""
    cs, cp = _seqlens(cu_seqlens, cu_seqlens_padded)
    B = cs.size - 1
    a, as_ = _flat_view(a, a_row_stride, None)
    b, bs = _flat_view(b, b_row_stride, None)
    n = a.shape[0] if nrows is None else nrows
    ostride = inner if out_row_stride is None else out_row_stride
    if out is not None:
        pass
    elif out_init is None:
        out = np.full((n, ostride), 0x7FC1, dtype=np.uint16)
    else:
        out = np.array(out_init, dtype=np.uint16, copy=True)
    o64 = np.full(out.shape, np.nan) if want_f64 else None
    r, nr = _rows(rows)
    rc = lib().oracle_swiglu(
        _ptr(a, ctypes.c_uint16), as_, _ptr(b, ctypes.c_uint16), bs,
        _ptr(cs, ctypes.c_int32), _ptr(cp, ctypes.c_int32), B, n, inner,
        _ptr(out, ctypes.c_uint16), ostride, _ptr(o64, ctypes.c_double), _ptr(r, ctypes.c_int64), nr)
    _check(rc, "swiglu")
    return (out, o64) if want_f64 else out


def frames_to_u8(x, layout: int = 0) -> np.ndarray:
    """fp32 frames [B, C, T, H, W] -> uint8 [B, T, H, W, C] (layout 0) or
    [B, T, C, H, W] (layout 1)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    if x.ndim != 5:
        raise ValueError("expected [batch, channels, frames, height, width]")
    B, C, T, H, W = x.shape
    shape = (B, T, H, W, C) if layout == 0 else (B, T, C, H, W)
    out = np.zeros(shape, dtype=np.uint8)
    rc = lib().oracle_frames_to_u8(_ptr(x, ctypes.c_float), B, C, T, H, W, layout, _ptr(out, ctypes.c_uint8))
    _check(rc, "frames_to_u8")
    return out
