"""Outputs at a 16-byte but not 32-byte aligned address.

The final fp32 states (fused forward, state pass) and the decode front end's
history rows go out as 32-byte stores when the destination allows it and as
16-byte stores otherwise (the boundary asks for 16-byte alignment only).
Each case runs the same call twice, once into a 32-byte aligned tensor and
once into one placed 16 bytes past a 32-byte boundary, and asks for the same
bits; the aligned results themselves are checked against the oracle by the
other test files.
"""
import pytest
import torch

import linear_attention_simple_b200 as gla
from linear_attention_simple_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from linear_attention_simple_b200 import build
    build.build()
    gla.lib()


def off16(shape, fill=None):
    """fp32 tensor of `shape` whose data starts 16 bytes past a 32-byte
    boundary (a view 4 floats into a larger allocation)."""
    n = 1
    for s in shape:
        n *= s
    buf = torch.zeros(n + 16, dtype=torch.float32, device="cuda")
    base = buf.data_ptr() % 32 // 4           # floats past the last 32-byte boundary
    start = (8 - base) % 8 + 4
    t = buf[start:start + n].view(shape)
    assert t.data_ptr() % 32 == 16
    if fill is not None:
        t.copy_(fill)
    return t


# (2, 300, 40): one CTA per head, the fused kernel writes S_T;
# (1, 1000, 2): the segmented path, whose last segment's fused pass writes it
@pytest.mark.parametrize("B,T,H", [(2, 300, 40), (1, 1000, 2)])
def test_chunk_fwd_final_state_16_byte_aligned(B, T, H):
    d = inputs.chunk_inputs(B, T, H, seed=900 + T, device="cuda", s0_std=0.1)
    o1, s1 = gla.gla_chunk_fwd(d["q"], d["k"], d["v"], d["a"], s0=d["s0"])
    assert s1.data_ptr() % 32 == 0
    s2 = off16(s1.shape)
    o2, _ = gla.gla_chunk_fwd(d["q"], d["k"], d["v"], d["a"], s0=off16(d["s0"].shape, d["s0"]), s_final=s2)
    assert gla.gla_get_device_status() == 0
    assert torch.equal(s1, s2)
    assert torch.equal(o1, o2)


def test_segment_state_16_byte_aligned():
    """B*H = 80: one state-pass CTA per head writes the segment's state."""
    d = inputs.chunk_inputs(2, 300, 40, seed=910, device="cuda")
    s1, g1 = gla.gla_segment_state_fwd(d["k"], d["v"], d["a"])
    assert s1.data_ptr() % 32 == 0
    s2 = off16(s1.shape)
    gla.gla_segment_state_fwd(d["k"], d["v"], d["a"], s_seg=s2)
    assert gla.gla_get_device_status() == 0
    assert torch.equal(s1, s2)


@pytest.mark.parametrize("N,D", [(7, 256), (33, 3072)])
def test_decode_front_history_16_byte_aligned(N, D):
    x = inputs.randn((N, D), 920 + N, "cuda", dtype=torch.bfloat16)
    w = inputs.randn((D, 4), 921, "cuda", std=0.5)
    pool0 = inputs.randn((N, 3, D), 922, "cuda")
    p1 = pool0.clone()
    assert p1.data_ptr() % 32 == 0
    p2 = off16(pool0.shape, pool0)
    y1 = gla.conv1d_silu_decode_step(x, w, p1)
    y2 = gla.conv1d_silu_decode_step(x, w, p2)
    assert gla.gla_get_device_status() == 0
    assert torch.equal(y1, y2)
    assert torch.equal(p1, p2)
