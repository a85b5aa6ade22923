"""Fused per-token operators of a packed audio-video DiT block, for B200.

Python binding of the C ABI in ``include/dit_token.h`` (``libdit_token.so``,
built in-tree by ``python -m dit_token_b200.build``).  Each function has the
name of its C entry point and only marshals arguments: it reads pointers,
row strides and the current CUDA stream from torch tensors and calls the
library through ctypes.  Every step of the computation runs in the CUDA
kernels; there is no CPU or PyTorch fallback -- a missing library raises.

The operators (see the header for the exact definitions):

* ``dit_qk_rmsnorm_rope``  per-head Q/K RMSNorm fused with 1D / 3D RoPE, in place
* ``dit_adaln_modulate``   LN(x) * (1 + scale_b) + shift_b
* ``dit_gated_residual``   x + gate_b * y
* ``dit_swiglu``           silu(a) * b
* ``dit_gated_residual_adaln``  res = x + gate_b * y, then LN(res) * (1 + scale_b) + shift_b
* ``dit_frames_to_u8``     decoded fp32 frames [B, C, T, H, W] -> uint8 BTHWC (or planar BTCHW)

All run over a packed sequence described by ``cu_seqlens`` (cumulative valid
lengths) and ``cu_seqlens_padded`` (row offsets), touching valid rows only.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = ["dit_qk_rmsnorm_rope", "dit_adaln_modulate", "dit_gated_residual", "dit_swiglu",
           "dit_gated_residual_adaln", "dit_frames_to_u8",
           "dit_validate_seqlens", "check_seqlens", "DitError", "library", "LIB_PATH", "STATUS"]

# DIT_TOKEN_LIB may point at another build of the same library.
LIB_PATH = os.environ.get("DIT_TOKEN_LIB") or os.path.join(os.path.dirname(os.path.abspath(__file__)),
                                                          "libdit_token.so")

STATUS = {0: "DIT_OK", 1: "DIT_ERR_NULL", 2: "DIT_ERR_SHAPE", 3: "DIT_ERR_ALIGN",
          4: "DIT_ERR_UNSUPPORTED", 5: "DIT_ERR_SEQLENS", 6: "DIT_ERR_CUDA"}


class DitError(RuntimeError):
    def __init__(self, func: str, status: int, message: str):
        super().__init__(f"{func}: {message} (status {status})")
        self.status = status


_lib: Optional[ctypes.CDLL] = None

_VP = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_F32 = ctypes.c_float

_SIGNATURES = {
    "dit_qk_rmsnorm_rope": [_VP, _I64, _VP, _I64, _VP, _VP, _VP, _VP, _I32, _I64, _I32, _I32, _I32,
                            _VP, _I32, _I32, _I32, _F32, _F32, _VP],
    "dit_qk_rmsnorm_rope_ex": [_VP, _I64, _VP, _I64, _VP, _VP, _VP, _VP, _I32, _I64, _I32, _I32, _I32,
                               _VP, _I32, _I32, _I32, _F32, _F32, _I32, _VP],
    "dit_qk_rmsnorm_rope_shard": [_VP, _I64, _VP, _I64, _VP, _VP, _VP, _VP, _I32, _I64, _I32, _I32, _I32,
                                  _VP, _I32, _I32, _I32, _F32, _F32, _I32, _VP, _VP],
    "dit_adaln_modulate": [_VP, _I64, _VP, _I64, _VP, _VP, _I64, _VP, _VP, _I32, _I64, _I32, _F32, _VP],
    "dit_adaln_modulate_ex": [_VP, _I64, _VP, _I64, _VP, _VP, _I64, _VP, _VP, _I32, _I64, _I32, _F32, _I32,
                              _VP],
    "dit_gated_residual": [_VP, _I64, _VP, _I64, _VP, _I64, _VP, _I64, _VP, _VP, _I32, _I64, _I32, _VP],
    "dit_gated_residual_ex": [_VP, _I64, _VP, _I64, _VP, _I64, _VP, _I64, _VP, _VP, _I32, _I64, _I32, _I32,
                              _VP],
    "dit_swiglu": [_VP, _I64, _VP, _I64, _VP, _I64, _VP, _VP, _I32, _I64, _I32, _VP],
    "dit_gated_residual_adaln": [_VP, _I64, _VP, _I64, _VP, _I64, _VP, _VP, _I64, _VP, _I64, _VP, _I64,
                                 _VP, _VP, _I32, _I64, _I32, _F32, _VP],
    "dit_gated_residual_adaln_ex": [_VP, _I64, _VP, _I64, _VP, _I64, _VP, _VP, _I64, _VP, _I64, _VP, _I64,
                                    _VP, _VP, _I32, _I64, _I32, _F32, _I32, _VP],
    "dit_validate_seqlens": [_VP, _VP, _I32, _I64, _VP, _VP],
    "dit_av_stream_seqlens": [_VP, _VP, _VP, _VP, _I32, _VP, _VP, _VP],
    "dit_frames_to_u8": [_VP, _I64, _I64, _I64, _I64, _I64, _I32, _VP, _VP],
    "dit_status_string": [_I32],
    "dit_last_cuda_error": [],
    "dit_abi_version": [],
}


def library() -> ctypes.CDLL:
    """The loaded libdit_token.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m dit_token_b200.build` "
                               "(the operators have no fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_char_p if name == "dit_status_string" else ctypes.c_int32
        _lib = L
    return _lib


def _call(name: str, *args) -> None:
    L = library()
    st = getattr(L, name)(*args)
    if st != 0:
        msg = L.dit_status_string(st).decode()
        if st == 6:
            msg += f" (cudaError {L.dit_last_cuda_error()})"
        raise DitError(name, st, msg)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _rows(t: torch.Tensor, what: str) -> tuple:
    """(pointer, row stride in elements) of a bf16 CUDA tensor whose first axis
    is the padded row and whose remaining axes are contiguous."""
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{what}: expected bfloat16, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{what}: expected a CUDA tensor")
    if t.dim() < 2:
        raise ValueError(f"{what}: expected [rows, ...]")
    expect = 1
    for d in range(t.dim() - 1, 0, -1):
        if t.size(d) != 1 and t.stride(d) != expect:
            raise ValueError(f"{what}: the per-row axes must be contiguous")
        expect *= t.size(d)
    return t.data_ptr(), t.stride(0)


def _vec(t: torch.Tensor, what: str) -> int:
    if t.dtype != torch.bfloat16 or not t.is_cuda:
        raise TypeError(f"{what}: expected a bfloat16 CUDA tensor")
    return t.data_ptr()


# element-type codes of the per-sequence vectors (DIT_DTYPE_* in dit_token.h)
_DTYPE_CODES = {torch.bfloat16: 0, torch.float32: 1}


def _seq_vectors(t: torch.Tensor, hidden: int, what: str) -> tuple:
    """(pointer, per-sequence stride, dtype code) of per-sequence vectors
    [num_seqs, hidden], bf16 or fp32 (any sequence stride, contiguous last axis)."""
    if t.dtype not in _DTYPE_CODES or not t.is_cuda:
        raise TypeError(f"{what}: expected a bfloat16 or float32 CUDA tensor")
    if t.dim() != 2 or t.size(1) != hidden or (t.stride(1) != 1 and hidden > 1):
        raise ValueError(f"{what}: expected [num_seqs, {hidden}] with a contiguous last axis")
    return t.data_ptr(), t.stride(0), _DTYPE_CODES[t.dtype]


def _one_dtype(codes, what: str) -> int:
    if len(set(codes)) != 1:
        raise TypeError(f"{what} must all be bfloat16 or all float32")
    return codes[0]


def _packing(cu_seqlens: torch.Tensor, cu_seqlens_padded: torch.Tensor):
    for t, n in ((cu_seqlens, "cu_seqlens"), (cu_seqlens_padded, "cu_seqlens_padded")):
        if t.dtype != torch.int32 or not t.is_cuda or t.dim() != 1 or not t.is_contiguous():
            raise TypeError(f"{n}: expected a contiguous int32 CUDA vector")
    if cu_seqlens.numel() != cu_seqlens_padded.numel() or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens and cu_seqlens_padded must both have num_seqs + 1 entries")
    return cu_seqlens.data_ptr(), cu_seqlens_padded.data_ptr(), cu_seqlens.numel() - 1


def dit_qk_rmsnorm_rope(q: torch.Tensor, k: torch.Tensor, q_weight: torch.Tensor, k_weight: torch.Tensor,
                        cu_seqlens: torch.Tensor, cu_seqlens_padded: torch.Tensor, *,
                        num_q_heads: int, num_k_heads: int, head_dim: int,
                        rope_grid: Optional[torch.Tensor] = None,
                        sections: Sequence[int] = (0, 0, 0), rope_theta: float = 10000.0,
                        eps: float = 1e-6, rope_mode: str = "interleaved",
                        pos_offset: Optional[torch.Tensor] = None, stream=None) -> None:
    """In place: q, k <- RoPE(RMSNorm_head(q) * q_weight), RoPE(RMSNorm_head(k) * k_weight).

    q: [rows, num_q_heads * head_dim] (or [rows, heads, head_dim]) bf16, any
    row stride; k likewise.  rope_grid: int32 [num_seqs, 3] (T, H, W) or None
    (every row 1D); sections: t/h/w widths of head_dim on 3D rows.
    rope_mode: "interleaved" (pairs 2j, 2j+1; the C entry dit_qk_rmsnorm_rope),
    "half" (pairs j, j + D/2) or "none" (RMSNorm only) -- the latter two, and
    head_dim 256, go through dit_qk_rmsnorm_rope_ex.  pos_offset: int32
    [num_seqs] or None -- this buffer holds a slice of longer sequences whose
    rows start at row pos_offset[b] of sequence b (dit_qk_rmsnorm_rope_shard)."""
    qp, qs = _rows(q, "q")
    kp, ks = _rows(k, "k")
    if k.size(0) != q.size(0):
        raise ValueError("q and k must have the same number of rows")
    cs, cp, B = _packing(cu_seqlens, cu_seqlens_padded)
    gp = 0
    if rope_grid is not None:
        if rope_grid.dtype != torch.int32 or not rope_grid.is_cuda or not rope_grid.is_contiguous() \
                or tuple(rope_grid.shape) != (B, 3):
            raise TypeError("rope_grid: expected a contiguous int32 CUDA tensor [num_seqs, 3]")
        gp = rope_grid.data_ptr()
    st, sh, sw = (int(s) for s in sections)
    args = (qp, qs, kp, ks, _vec(q_weight, "q_weight"), _vec(k_weight, "k_weight"), cs, cp, B, q.size(0),
            num_q_heads, num_k_heads, head_dim, gp or None, st, sh, sw, float(rope_theta), float(eps))
    mode = {"interleaved": 0, "half": 1, "none": 2}[rope_mode]
    if pos_offset is not None:
        _call("dit_qk_rmsnorm_rope_shard", *args, mode, _offsets(pos_offset, B), _stream(stream))
    elif mode == 0 and head_dim in (64, 128):
        _call("dit_qk_rmsnorm_rope", *args, _stream(stream))
    else:
        _call("dit_qk_rmsnorm_rope_ex", *args, mode, _stream(stream))


def _offsets(pos_offset: torch.Tensor, B: int) -> int:
    if pos_offset.dtype != torch.int32 or not pos_offset.is_cuda or not pos_offset.is_contiguous() or \
            tuple(pos_offset.shape) != (B,):
        raise TypeError("pos_offset: expected a contiguous int32 CUDA vector [num_seqs]")
    return pos_offset.data_ptr() or None


def dit_adaln_modulate(x: torch.Tensor, shift: torch.Tensor, scale: torch.Tensor,
                       cu_seqlens: torch.Tensor, cu_seqlens_padded: torch.Tensor, *,
                       out: Optional[torch.Tensor] = None, eps: float = 1e-6, stream=None) -> torch.Tensor:
    """out = LayerNorm(x) * (1 + scale_b) + shift_b on valid rows.

    x: [rows, hidden]; shift, scale: [num_seqs, hidden] (any sequence stride,
    e.g. slices of a [num_seqs, 6, hidden] modulation tensor -- both must
    share it), both bf16 (dit_adaln_modulate) or both fp32
    (dit_adaln_modulate_ex).  ``out`` may be x; if None a new tensor is
    returned whose padding rows are left uninitialised."""
    hidden = x.size(-1)
    if out is None:
        out = torch.empty_like(x)
    xp, xs = _rows(x, "x")
    op, os_ = _rows(out, "out")
    shp, sst, shd = _seq_vectors(shift, hidden, "shift")
    scp, cst, scd = _seq_vectors(scale, hidden, "scale")
    dt = _one_dtype((shd, scd), "shift and scale")
    cs, cp, B = _packing(cu_seqlens, cu_seqlens_padded)
    if B > 1 and sst != cst:
        raise ValueError("shift and scale must share one sequence stride")
    args = (xp, xs, op, os_, shp, scp, sst if B > 1 else hidden, cs, cp, B, x.size(0), hidden, float(eps))
    if dt == 0:
        _call("dit_adaln_modulate", *args, _stream(stream))
    else:
        _call("dit_adaln_modulate_ex", *args, dt, _stream(stream))
    return out


def dit_gated_residual(x: torch.Tensor, y: torch.Tensor, gate: torch.Tensor,
                       cu_seqlens: torch.Tensor, cu_seqlens_padded: torch.Tensor, *,
                       out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out = x + gate_b * y on valid rows (``out`` may be x).  gate: bf16
    (dit_gated_residual) or fp32 (dit_gated_residual_ex) [num_seqs, hidden]."""
    hidden = x.size(-1)
    if out is None:
        out = torch.empty_like(x)
    xp, xs = _rows(x, "x")
    yp, ys = _rows(y, "y")
    op, os_ = _rows(out, "out")
    gp, gst, dt = _seq_vectors(gate, hidden, "gate")
    cs, cp, B = _packing(cu_seqlens, cu_seqlens_padded)
    args = (xp, xs, yp, ys, gp, gst if B > 1 else hidden, op, os_, cs, cp, B, x.size(0), hidden)
    if dt == 0:
        _call("dit_gated_residual", *args, _stream(stream))
    else:
        _call("dit_gated_residual_ex", *args, dt, _stream(stream))
    return out


def dit_gated_residual_adaln(x: torch.Tensor, y: torch.Tensor, gate: torch.Tensor, shift: torch.Tensor,
                             scale: torch.Tensor, cu_seqlens: torch.Tensor, cu_seqlens_padded: torch.Tensor, *,
                             res_out: Optional[torch.Tensor] = None, norm_out: Optional[torch.Tensor] = None,
                             eps: float = 1e-6, stream=None):
    """res = x + gate_b * y; norm = LayerNorm(res) * (1 + scale_b) + shift_b,
    on valid rows, in one pass.  ``res_out`` may be x.  gate, shift and scale
    all bf16 (dit_gated_residual_adaln) or all fp32 (dit_gated_residual_adaln_ex).
    Returns (res, norm)."""
    hidden = x.size(-1)
    if res_out is None:
        res_out = torch.empty_like(x)
    if norm_out is None:
        norm_out = torch.empty_like(x)
    xp, xs = _rows(x, "x")
    yp, ys = _rows(y, "y")
    rp, rs = _rows(res_out, "res_out")
    np_, ns = _rows(norm_out, "norm_out")
    gp, gst, gd = _seq_vectors(gate, hidden, "gate")
    shp, sst, shd = _seq_vectors(shift, hidden, "shift")
    scp, cst, scd = _seq_vectors(scale, hidden, "scale")
    dt = _one_dtype((gd, shd, scd), "gate, shift and scale")
    cs, cp, B = _packing(cu_seqlens, cu_seqlens_padded)
    if B > 1 and sst != cst:
        raise ValueError("shift and scale must share one sequence stride")
    args = (xp, xs, yp, ys, gp, gst if B > 1 else hidden, shp, scp, sst if B > 1 else hidden, rp, rs, np_, ns,
            cs, cp, B, x.size(0), hidden, float(eps))
    if dt == 0:
        _call("dit_gated_residual_adaln", *args, _stream(stream))
    else:
        _call("dit_gated_residual_adaln_ex", *args, dt, _stream(stream))
    return res_out, norm_out


def dit_swiglu(a: torch.Tensor, b: torch.Tensor, cu_seqlens: torch.Tensor, cu_seqlens_padded: torch.Tensor,
               *, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out = silu(a) * b on valid rows.  a, b: [rows, inner] (e.g. the two
    column halves of a [rows, 2 * inner] projection)."""
    inner = a.size(-1)
    if b.size(-1) != inner:
        raise ValueError("a and b must have the same width")
    if out is None:
        out = torch.empty((a.size(0), inner), dtype=a.dtype, device=a.device)
    ap, as_ = _rows(a, "a")
    bp, bs = _rows(b, "b")
    op, os_ = _rows(out, "out")
    cs, cp, B = _packing(cu_seqlens, cu_seqlens_padded)
    _call("dit_swiglu", ap, as_, bp, bs, op, os_, cs, cp, B, a.size(0), inner, _stream(stream))
    return out


def dit_frames_to_u8(x: torch.Tensor, *, layout: str = "bthwc", out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """Decoded frames fp32 [B, C, T, H, W] -> uint8 [B, T, H, W, C] ("bthwc") or
    [B, T, C, H, W] ("btchw"): u = rint(clamp((x + 1) * 127.5, 0, 255))."""
    if x.dtype != torch.float32 or not x.is_cuda or x.dim() != 5 or not x.is_contiguous():
        raise TypeError("x: expected a contiguous float32 CUDA tensor [B, C, T, H, W]")
    B, C, T, H, Wd = x.shape
    code = {"bthwc": 0, "btchw": 1}[layout]
    shape = (B, T, H, Wd, C) if code == 0 else (B, T, C, H, Wd)
    if out is None:
        out = torch.empty(shape, dtype=torch.uint8, device=x.device)
    if out.dtype != torch.uint8 or not out.is_cuda or tuple(out.shape) != shape or not out.is_contiguous():
        raise TypeError(f"out: expected a contiguous uint8 CUDA tensor {shape}")
    _call("dit_frames_to_u8", x.data_ptr(), B, C, T, H, Wd, code, out.data_ptr(), _stream(stream))
    return out


def dit_validate_seqlens(cu_seqlens: torch.Tensor, cu_seqlens_padded: torch.Tensor, num_rows_padded: int,
                         *, flag: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Enqueue the device-side descriptor check; returns the int32[2] flag
    tensor (flag[0] == 1: malformed, flag[1]: first bad sequence)."""
    cs, cp, B = _packing(cu_seqlens, cu_seqlens_padded)
    if flag is None:
        flag = torch.empty(2, dtype=torch.int32, device=cu_seqlens.device)
    _call("dit_validate_seqlens", cs, cp, B, int(num_rows_padded), flag.data_ptr(), _stream(stream))
    return flag


def dit_av_stream_seqlens(cu_seqlens: torch.Tensor, cu_seqlens_padded: torch.Tensor, rope_grid: torch.Tensor,
                          *, pos_offset: Optional[torch.Tensor] = None, out: Optional[tuple] = None,
                          stream=None) -> tuple:
    """Per-stream descriptor of joint audio-video sequences: sequence b becomes
    sequences 2b (its T*H*W video rows) and 2b + 1 (its audio rows and
    padding).  Returns (cu_seqlens_av, cu_seqlens_padded_av), int32
    [2 * num_seqs + 1] on the device.  Pass them to the modulated ops with
    vectors laid out [num_seqs, 2, ...] viewed as [2 * num_seqs, ...], e.g. for
    mod [B, 2, 6, C]: shift = mod.view(2 * B, 6, C)[:, 0].  pos_offset: as in
    dit_qk_rmsnorm_rope, for one rank's slice of longer sequences."""
    cs, cp, B = _packing(cu_seqlens, cu_seqlens_padded)
    if rope_grid.dtype != torch.int32 or not rope_grid.is_cuda or not rope_grid.is_contiguous() or \
            tuple(rope_grid.shape) != (B, 3):
        raise TypeError("rope_grid: expected a contiguous int32 CUDA tensor [num_seqs, 3]")
    if out is None:
        out = (torch.empty(2 * B + 1, dtype=torch.int32, device=cu_seqlens.device),
               torch.empty(2 * B + 1, dtype=torch.int32, device=cu_seqlens.device))
    for t in out:
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous() or t.numel() != 2 * B + 1:
            raise TypeError(f"out: expected two contiguous int32 CUDA vectors of {2 * B + 1} entries")
    po = None if pos_offset is None else _offsets(pos_offset, B)
    _call("dit_av_stream_seqlens", cs, cp, rope_grid.data_ptr() or None, po, B, out[0].data_ptr(),
          out[1].data_ptr(), _stream(stream))
    return out


def check_seqlens(cu_seqlens: torch.Tensor, cu_seqlens_padded: torch.Tensor, num_rows_padded: int,
                  stream=None) -> None:
    """Validate a packing descriptor on the device and raise DitError
    (DIT_ERR_SEQLENS) if it is malformed.  Synchronizes with the stream to
    read the flag, so call it where a host round trip is acceptable (e.g. once
    per batch layout), not inside a captured or latency-critical sequence."""
    flag = dit_validate_seqlens(cu_seqlens, cu_seqlens_padded, num_rows_padded, stream=stream)
    bad, first = (int(v) for v in flag.tolist())
    if bad:
        raise DitError("dit_validate_seqlens", 5,
                       f"{library().dit_status_string(5).decode()}: first bad sequence {first}")
