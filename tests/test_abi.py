"""C-ABI checks that need no GPU: the library loads, exports every entry point
the header declares, and rejects bad arguments with the documented status
before launching anything."""
import os
import re

import pytest

import dit_token_b200 as dit
from dit_token_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dit_token.h")

OK, NULL, SHAPE, ALIGN, UNSUP = 0, 1, 2, 3, 4
P = 0x10000  # an aligned, never dereferenced fake device address


@pytest.fixture(scope="module")
def L():
    build.build()
    return dit.library()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DIT_API\s+[\w\s\*]+?\b(dit_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) == 16, names
    for n in names:
        assert hasattr(L, n), n
    assert L.dit_abi_version() == 1


def test_status_strings(L):
    for s in range(7):
        assert L.dit_status_string(s).decode().startswith(dit.STATUS[s])
    assert L.dit_status_string(99) == b"unknown dit_status"


def qk(L, **kw):
    a = dict(q=P, qs=256, k=P, ks=256, wq=P, wk=P, cs=P, cp=P, B=1, rows=16, hq=2, hk=2, d=128,
             grid=None, st=0, sh=0, sw=0, theta=10000.0, eps=1e-6)
    a.update(kw)
    return L.dit_qk_rmsnorm_rope(a["q"], a["qs"], a["k"], a["ks"], a["wq"], a["wk"], a["cs"], a["cp"], a["B"],
                                 a["rows"], a["hq"], a["hk"], a["d"], a["grid"], a["st"], a["sh"], a["sw"],
                                 a["theta"], a["eps"], None)


def test_qk_argument_checks(L):
    assert qk(L, q=None) == NULL
    assert qk(L, wk=None) == NULL
    assert qk(L, cs=None) == NULL
    assert qk(L, d=96) == UNSUP
    assert qk(L, d=0) == SHAPE
    assert qk(L, qs=255) == SHAPE            # stride smaller than heads * head_dim
    assert qk(L, qs=264, q=P + 2) == ALIGN   # pointer not 16-byte aligned
    assert qk(L, qs=260) == ALIGN            # stride not a multiple of 8
    assert qk(L, B=-1) == SHAPE
    assert qk(L, rows=-5) == SHAPE
    assert qk(L, rows=1 << 31) == SHAPE
    assert qk(L, grid=P, st=44, sh=42, sw=40) == SHAPE   # sections do not sum to head_dim
    assert qk(L, grid=P, st=43, sh=43, sw=42) == SHAPE   # odd section
    assert qk(L, grid=P, st=-2, sh=66, sw=64) == SHAPE
    assert qk(L, theta=0.0) == SHAPE
    assert qk(L, eps=float("nan")) == SHAPE
    assert qk(L, grid=P + 2, st=44, sh=42, sw=42) == ALIGN


def test_qk_ex_argument_checks(L):
    def ex(mode, d=128, **kw):
        a = dict(q=P, qs=512, k=P, ks=512, grid=None, st=0, sh=0, sw=0)
        a.update(kw)
        return L.dit_qk_rmsnorm_rope_ex(a["q"], a["qs"], a["k"], a["ks"], P, P, P, P, 1, 16, 2, 2, d, a["grid"],
                                        a["st"], a["sh"], a["sw"], 10000.0, 1e-6, mode, None)
    assert ex(3) == UNSUP and ex(-1) == UNSUP
    assert ex(0, d=512, qs=1024, ks=1024) == UNSUP
    assert ex(1, d=256, qs=500) == SHAPE
    assert ex(1, grid=P, st=44, sh=42, sw=40) == SHAPE
    assert ex(2, grid=P, st=44, sh=42, sw=40, q=None) == NULL   # sections are ignored without rotation
    assert qk(L, d=256, qs=512, ks=512) == UNSUP                # the original entry keeps 64/128


def test_empty_batches_launch_nothing(L):
    # nothing to do -> DIT_OK even with NULL tensors, and no CUDA call is made
    assert qk(L, B=0, q=None, k=None, cs=None, cp=None) == OK
    assert qk(L, rows=0, q=None, k=None) == OK
    assert qk(L, hq=0, hk=0) == OK
    assert L.dit_swiglu(None, 8, None, 8, None, 8, None, None, 0, 0, 8, None) == OK
    assert L.dit_gated_residual(None, 8, None, 8, None, 8, None, 8, P, P, 3, 0, 8, None) == OK
    assert L.dit_adaln_modulate(None, 8, None, 8, None, None, 8, P, P, 0, 64, 8, 1e-6, None) == OK


def test_adaln_argument_checks(L):
    def call(**kw):
        a = dict(x=P, xs=64, o=P, os=64, sh=P, sc=P, ms=64, B=1, rows=4, C=64, eps=1e-6)
        a.update(kw)
        return L.dit_adaln_modulate(a["x"], a["xs"], a["o"], a["os"], a["sh"], a["sc"], a["ms"], P, P,
                                    a["B"], a["rows"], a["C"], a["eps"], None)
    assert call(x=None) == NULL and call(sc=None) == NULL
    assert call(C=0) == SHAPE and call(xs=56) == SHAPE and call(ms=-8) == SHAPE
    assert call(C=60, xs=64, os=64) == ALIGN
    assert call(ms=12) == ALIGN
    assert call(o=P + 8) == ALIGN
    assert call(C=16392, xs=16392, os=16392) == UNSUP
    assert call(eps=-1.0) == SHAPE


def test_residual_and_swiglu_argument_checks(L):
    def res(**kw):
        a = dict(x=P, xs=64, y=P, ys=64, g=P, gs=64, o=P, os=64, B=2, rows=4, C=64)
        a.update(kw)
        return L.dit_gated_residual(a["x"], a["xs"], a["y"], a["ys"], a["g"], a["gs"], a["o"], a["os"], P, P,
                                    a["B"], a["rows"], a["C"], None)
    assert res(y=None) == NULL and res(g=None) == NULL
    assert res(ys=32) == SHAPE and res(gs=-8) == SHAPE and res(C=-8) == SHAPE
    assert res(gs=4) == ALIGN and res(y=P + 4) == ALIGN and res(C=36, xs=64, ys=64, os=64) == ALIGN

    def sw(**kw):
        a = dict(a=P, as_=128, b=P, bs=128, o=P, os=64, B=1, rows=4, I=64)
        a.update(kw)
        return L.dit_swiglu(a["a"], a["as_"], a["b"], a["bs"], a["o"], a["os"], P, P, a["B"], a["rows"], a["I"],
                            None)
    assert sw(b=None) == NULL and sw(o=None) == NULL
    assert sw(os=32) == SHAPE and sw(I=0) == SHAPE
    assert sw(b=P + 64 * 2 + 2) == ALIGN and sw(as_=132) == ALIGN


def test_fused_residual_adaln_argument_checks(L):
    def call(**kw):
        a = dict(x=P, xs=64, y=P, ys=64, g=P, gs=64, sh=P, sc=P, ms=64, r=P, rs=64, n=P, ns=64, B=1, rows=4,
                 C=64, eps=1e-6)
        a.update(kw)
        return L.dit_gated_residual_adaln(a["x"], a["xs"], a["y"], a["ys"], a["g"], a["gs"], a["sh"], a["sc"],
                                          a["ms"], a["r"], a["rs"], a["n"], a["ns"], P, P, a["B"], a["rows"],
                                          a["C"], a["eps"], None)
    assert call(n=None) == NULL and call(sh=None) == NULL and call(g=None) == NULL
    assert call(ns=32) == SHAPE and call(ms=-8) == SHAPE and call(eps=-1.0) == SHAPE
    assert call(C=16392, xs=16392, ys=16392, rs=16392, ns=16392) == UNSUP
    assert call(r=P + 8) == ALIGN and call(gs=12) == ALIGN
    assert call(B=0, x=None, n=None) == OK


def test_modulation_dtype_entries(L):
    """The _ex entries take a dtype code (0 bf16, 1 fp32); fp32 vectors need a
    sequence stride that is a multiple of 4, bf16 ones a multiple of 8."""
    def ada(dt, ms=64):
        return L.dit_adaln_modulate_ex(P, 64, P, 64, P, P, ms, P, P, 0, 4, 64, 1e-6, dt, None)
    def res(dt, gs=64, B=0):
        return L.dit_gated_residual_ex(P, 64, P, 64, P, gs, P, 64, P, P, B, 4, 64, dt, None)
    def fused(dt, gs=64, ms=64, g=P):
        return L.dit_gated_residual_adaln_ex(P, 64, P, 64, g, gs, P, P, ms, P, 64, P, 64, P, P, 0, 4, 64, 1e-6,
                                             dt, None)
    for f in (ada, res, fused):
        assert f(2) == UNSUP and f(-1) == UNSUP
        assert f(0) == OK and f(1) == OK     # empty batches: checks only, no launch
    assert ada(1, ms=68) == OK and ada(0, ms=68) == OK            # empty: strides unchecked
    assert fused(1, g=None) == OK                                  # empty batch: no pointer needed
    # non-empty calls stop at the alignment check, before any launch
    assert L.dit_adaln_modulate_ex(P, 64, P, 64, P, P, 68, P, P, 1, 4, 64, 1e-6, 0, None) == ALIGN
    assert L.dit_adaln_modulate_ex(P, 64, P, 64, P, P, 66, P, P, 1, 4, 64, 1e-6, 1, None) == ALIGN
    assert L.dit_gated_residual_ex(P, 64, P, 64, P, 12, P, 64, P, P, 2, 4, 64, 0, None) == ALIGN
    assert L.dit_gated_residual_ex(P, 64, P, 64, P, 10, P, 64, P, P, 2, 4, 64, 1, None) == ALIGN
    assert L.dit_gated_residual_adaln_ex(P, 64, P, 64, P, 64, P, P, 66, P, 64, P, 64, P, P, 1, 4, 64, 1e-6, 1,
                                         None) == ALIGN
    assert L.dit_gated_residual_adaln_ex(P, 64, P, 64, None, 64, P, P, 64, P, 64, P, 64, P, P, 1, 4, 64, 1e-6,
                                         1, None) == NULL


def test_av_stream_seqlens_argument_checks(L):
    f = L.dit_av_stream_seqlens
    assert f(P, P, P, None, -1, P, P, None) == SHAPE
    assert f(P, P, P, None, 1 << 30, P, P, None) == SHAPE
    assert f(None, P, P, None, 2, P, P, None) == NULL
    assert f(P, P, None, None, 2, P, P, None) == NULL        # the split needs the grid
    assert f(P, P, P, None, 2, P, None, None) == NULL
    assert f(P, P, P + 2, None, 2, P, P, None) == ALIGN
    assert f(P, P, P, P + 2, 2, P, P, None) == ALIGN


def test_qk_shard_argument_checks(L):
    def sh(po, **kw):
        a = dict(q=P, B=1, mode=0)
        a.update(kw)
        return L.dit_qk_rmsnorm_rope_shard(a["q"], 256, P, 256, P, P, P, P, a["B"], 16, 2, 2, 128, None, 0, 0, 0,
                                           10000.0, 1e-6, a["mode"], po, None)
    assert sh(P + 2) == ALIGN
    assert sh(None, q=None) == NULL
    assert sh(P, mode=7) == UNSUP
    assert sh(P + 2, B=0) == OK          # empty batch: nothing checked past the shapes


def test_frames_argument_checks(L):
    assert L.dit_frames_to_u8(P, 1, 3, 2, 4, 16, 2, P, None) == UNSUP
    assert L.dit_frames_to_u8(P, 1, -3, 2, 4, 16, 0, P, None) == SHAPE
    assert L.dit_frames_to_u8(None, 1, 3, 2, 4, 16, 0, P, None) == NULL
    assert L.dit_frames_to_u8(P, 1, 3, 2, 4, 16, 0, None, None) == NULL
    assert L.dit_frames_to_u8(P + 2, 1, 3, 2, 4, 16, 0, P, None) == ALIGN
    assert L.dit_frames_to_u8(None, 0, 3, 2, 4, 16, 0, None, None) == OK    # empty
    assert L.dit_frames_to_u8(P, 1 << 40, 1 << 20, 1, 1, 1, 0, P, None) == SHAPE


def test_validate_argument_checks(L):
    flag = P
    assert L.dit_validate_seqlens(None, P, 1, 4, flag, None) == NULL
    assert L.dit_validate_seqlens(P, P, 1, 4, None, None) == NULL
    assert L.dit_validate_seqlens(P, P, -1, 4, flag, None) == SHAPE
    assert L.dit_validate_seqlens(P + 2, P, 1, 4, flag, None) == ALIGN


def test_binding_rejects_cpu_tensors_before_the_library():
    import torch
    x = torch.zeros(4, 8, dtype=torch.bfloat16)
    cs = torch.zeros(2, dtype=torch.int32)
    with pytest.raises((TypeError, ValueError)):
        dit.dit_gated_residual(x, x, torch.zeros(1, 8, dtype=torch.bfloat16), cs, cs)
    with pytest.raises(TypeError):
        dit.dit_swiglu(x.float(), x.float(), cs, cs)
    with pytest.raises(TypeError):   # fp16 modulation vectors are not accepted
        dit._seq_vectors(torch.zeros(1, 8, dtype=torch.float16), 8, "gate")
    with pytest.raises(TypeError):   # mixed bf16 / fp32 vectors in one call
        dit._one_dtype((0, 1, 0), "gate, shift and scale")


def test_switched_build_never_replaces_the_in_tree_library():
    """A build with compile-time switches (e.g. DIT_PDL=0) must name its own
    output file; the in-tree library is left as it is."""
    before = os.path.getmtime(build.LIB) if os.path.exists(build.LIB) else None
    for out in (None, build.LIB):
        with pytest.raises(ValueError):
            build.build(out=out, defines=["DIT_PDL=0"])
    after = os.path.getmtime(build.LIB) if os.path.exists(build.LIB) else None
    assert before == after
