"""GPU frame conversion (fp32 BCTHW -> uint8 BTHWC / BTCHW) against the CPU
oracle, bit for bit: the vector path (width % 16 == 0, 1/3/4 channels), the
per-value path (other widths and channel counts), special values (ties,
clamps, NaN, infinities), and the pages' 10-second 1344x768 request at full
size on sampled frames, in the launch configuration the benchmark times."""
import numpy as np
import pytest
import torch

import dit_token_b200 as dit
import oracle
from dit_token_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from dit_token_b200 import build
    build.build()


def check(x_cpu, layout):
    x = x_cpu.cuda()
    got = dit.dit_frames_to_u8(x, layout=layout).cpu().numpy()
    want = oracle.frames_to_u8(x_cpu.numpy(), layout=0 if layout == "bthwc" else 1)
    assert got.shape == want.shape
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} bytes differ, first at {bad[:3].tolist()}"


@pytest.mark.parametrize("layout", ["bthwc", "btchw"])
@pytest.mark.parametrize("shape", [(1, 3, 2, 5, 16), (2, 3, 3, 7, 48), (1, 1, 2, 3, 32), (1, 4, 2, 4, 64),
                                   (1, 3, 2, 5, 7), (1, 2, 3, 4, 16), (2, 5, 1, 3, 20), (1, 3, 1, 1, 1)])
def test_shapes(shape, layout):
    check(W.frames_input(shape, seed=sum(shape)), layout)


@pytest.mark.parametrize("layout", ["bthwc", "btchw"])
def test_special_values(layout):
    x = W.frames_input((1, 3, 2, 4, 32), seed=5)
    specials = torch.tensor([-1.0, 1.0, 0.0, -0.5, 0.5, 5.0, -3.0, float("nan"), float("inf"), float("-inf"),
                             -0.9921875, 0.00390625, -0.0, 1e-30, -1e-30, 0.99609375])
    flat = x.view(-1)
    flat[: specials.numel()] = specials
    xs = torch.arange(0, 512, dtype=torch.float32) / 256.0 - 1.0   # contains exact ties
    flat[64: 64 + 512] = xs[: min(512, flat.numel() - 64)]
    check(x, layout)


def test_empty_and_pages_request_sampled_frames():
    empty = torch.zeros((1, 3, 0, 4, 16), dtype=torch.float32, device="cuda")
    assert dit.dit_frames_to_u8(empty).numel() == 0
    x_cpu = W.frames_input(W.FRAMES_SHAPE, seed=0)
    x = x_cpu.cuda()
    for layout in ("bthwc", "btchw"):
        got = dit.dit_frames_to_u8(x, layout=layout)
        for t0 in (0, 121, 242):
            sl = x_cpu[:, :, t0:t0 + 1].contiguous().numpy()
            want = oracle.frames_to_u8(sl, layout=0 if layout == "bthwc" else 1)
            assert np.array_equal(got[:, t0:t0 + 1].cpu().numpy(), want), (layout, t0)
        got2 = dit.dit_frames_to_u8(x, layout=layout)
        assert torch.equal(got, got2)


@pytest.mark.parametrize("layout", ["bthwc", "btchw"])
def test_frames_not_32_byte_aligned(layout):
    """Frames starting 16 bytes past a 32-byte boundary take the 16-byte loads
    of the fast path (32-byte ones need the boundary); the bytes are the same."""
    x_cpu = W.frames_input((1, 3, 3, 5, 32), seed=6)
    buf = torch.zeros(x_cpu.numel() + 8, dtype=torch.float32, device="cuda")
    x = buf[4:4 + x_cpu.numel()].view(x_cpu.shape)
    x.copy_(x_cpu.cuda())
    assert x.data_ptr() % 32 == 16 and x.is_contiguous()
    got = dit.dit_frames_to_u8(x, layout=layout).cpu().numpy()
    want = oracle.frames_to_u8(x_cpu.numpy(), layout=0 if layout == "bthwc" else 1)
    assert np.array_equal(got, want)
