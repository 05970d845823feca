"""GPU parity of the streamed-weight path: layers whose weights (128 output
channels x the whole fan-in) do not fit in shared memory beside the rings.
Each ring stage then carries its K blocks' weights next to its activations.

Covers the 3x3 of ResNet50's later stages (Res4.x: 256 channels at 14x14,
Res5.x: 512 at 7x7) in the halo form, the stride-2 3x3 of Res4.1 (per-tap
form), 1x1 layers beyond the resident fan-in with and without a shortcut,
the Res5.1 projection (Conv3 + projection: 512 + 1024 channels of fan-in),
and the Res4.x bottleneck block.  Byte-for-byte against the CPU oracle.
"""
import pytest
import torch

import x1_conv_bn_b200 as X
from x1_conv_bn_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from x1_conv_bn_b200 import _build

    _build.build()
    X.lib()
    X.x1cb_last_device_error(clear=True)


def _nhwc(t):
    B, C1, H, W, _ = t.shape
    return t.permute(0, 2, 3, 1, 4).reshape(B, H, W, C1 * 32)


def _ok():
    torch.cuda.synchronize()
    st, bits = X.x1cb_last_device_error(clear=True)
    assert st == 0, bits


def _spread(ref):
    assert (ref == 0).float().mean() < 0.95 and ref.unique().numel() > 20


def _streams(B, H, W, Ic, Oc, R, res):
    return "wstream=1" in X.x1cb_describe_plan(B, H, W, Ic, Oc, R, int(res))


STREAM_3X3 = [
    (6, 14, 14, 256, 256),     # Res4.x conv2
    (3, 7, 7, 512, 512),       # Res5.x conv2
    (2, 9, 13, 192, 128),      # odd channel-block count, ragged tiles
    (1, 3, 130, 160, 128),     # per-tap form (W + 2 > 128) with streamed weights
]


@pytest.mark.parametrize("shape", STREAM_3X3, ids=[str(s) for s in STREAM_3X3])
def test_streamed_3x3_parity(oracle, shape):
    B, H, W, Ic, Oc = shape
    assert _streams(B, H, W, Ic, Oc, 3, False)
    s = synth.ConvShape(B, H, W, Ic, Oc, 3, False)
    inp = synth.conv_inputs(s, sum(shape))
    out = X.conv3x3_bn_relu_i8(X.x1cb_pack_act(inp.x.to(DEV)), X.x1cb_pack_weight(inp.w.to(DEV)),
                               inp.bias.to(DEV), inp.m.to(DEV), inp.S)
    _ok()
    ref = oracle.conv(inp.x, inp.w, inp.bias, inp.m, inp.S)
    got = _nhwc(out.cpu())
    assert torch.equal(got, ref), int((got != ref).sum())
    _spread(ref)


def test_streamed_3x3_full_int8_range(oracle):
    s = synth.ConvShape(2, 14, 14, 256, 256, 3, False)
    inp = synth.full_range_conv_inputs(s, 23, S=35)
    out = X.conv3x3_bn_relu_i8(X.x1cb_pack_act(inp.x.to(DEV)), X.x1cb_pack_weight(inp.w.to(DEV)),
                               inp.bias.to(DEV), inp.m.to(DEV), inp.S)
    _ok()
    assert torch.equal(_nhwc(out.cpu()), oracle.conv(inp.x, inp.w, inp.bias, inp.m, inp.S))


def test_streamed_3x3_stride2_res41(oracle):
    """Res4.1's conv2: 3x3 stride 2, 256 channels, 28x28 -> 14x14."""
    s = synth.ConvShape(4, 28, 28, 256, 256, 3, False)
    inp = synth.conv_inputs(s, 411)
    out = X.conv3x3s2_bn_relu_i8(X.x1cb_pack_act(inp.x.to(DEV)),
                                 X.x1cb_pack_weight(inp.w.to(DEV)), inp.bias.to(DEV),
                                 inp.m.to(DEV), inp.S)
    _ok()
    ref = oracle.conv_strided(inp.x, inp.w, inp.bias, inp.m, inp.S, 2)
    assert torch.equal(_nhwc(out.cpu()), ref)
    _spread(ref)


STREAM_1X1 = [
    (3, 14, 14, 1152, 256, True),
    (2, 7, 7, 2048, 512, False),
    (5, 5, 7, 4096, 128, True),
]


@pytest.mark.parametrize("shape", STREAM_1X1, ids=[str(s) for s in STREAM_1X1])
def test_streamed_1x1_parity(oracle, shape):
    B, H, W, Ic, Oc, res = shape
    assert _streams(B, H, W, Ic, Oc, 1, res)
    s = synth.ConvShape(B, H, W, Ic, Oc, 1, res)
    inp = synth.conv_inputs(s, Ic + Oc)
    r = X.x1cb_pack_act(inp.r.to(DEV)) if res else None
    out = X.conv1x1_bn_add_relu_i8(X.x1cb_pack_act(inp.x.to(DEV)),
                                   X.x1cb_pack_weight(inp.w.to(DEV)), inp.bias.to(DEV),
                                   inp.m.to(DEV), inp.m_r, inp.S, r)
    _ok()
    ref = oracle.conv(inp.x, inp.w, inp.bias, inp.m, inp.S, inp.r, inp.m_r)
    assert torch.equal(_nhwc(out.cpu()), ref)
    _spread(ref)


def test_streamed_projection_res51(oracle):
    """Res5.1's Conv3 + projection: y 512 channels at 7x7, block input 1024
    channels at 14x14, 2048 outputs; 1536 channels of fan-in stream."""
    B, H, W, Cy, Cx, Oc = 2, 7, 7, 512, 1024, 2048
    assert "wstream=1" in X.x1cb_describe_plan_ex(B, H, W, Cy, Oc, 1, 1, Cx)
    g = torch.Generator().manual_seed(51)
    y = torch.randint(0, 128, (B, H, W, Cy), generator=g, dtype=torch.int8)
    x = torch.randint(0, 128, (B, 2 * H, 2 * W, Cx), generator=g, dtype=torch.int8)
    w3 = torch.randint(-127, 128, (Oc, Cy, 1, 1), generator=g, dtype=torch.int8)
    wp = torch.randint(-127, 128, (Oc, Cx, 1, 1), generator=g, dtype=torch.int8)
    bias = torch.randint(-(1 << 14), (1 << 14) + 1, (Oc,), generator=g, dtype=torch.int32)
    c = synth.multiplier_center(Cy + Cx)
    m = torch.randint(int(0.9 * c), int(1.1 * c) + 1, (Oc,), generator=g, dtype=torch.int32)
    out = X.conv1x1_proj_bn_relu_i8(X.x1cb_pack_act(y.to(DEV)), X.x1cb_pack_weight(w3.to(DEV)),
                                    X.x1cb_pack_act(x.to(DEV)), X.x1cb_pack_weight(wp.to(DEV)),
                                    bias.to(DEV), m.to(DEV), 24)
    _ok()
    ref = oracle.conv_proj(y, w3, x, wp, bias, m, 24)
    assert torch.equal(_nhwc(out.cpu()), ref)
    _spread(ref)


def test_res4_bottleneck_block(oracle):
    """Res4.x: 1024 -> 256 -> 256 (3x3, streamed) -> 1024 + shortcut, 14x14."""
    s = synth.BlockShape(8, 14, 14, 1024, 256)
    inp = synth.block_inputs(s, 44)
    x = X.x1cb_pack_act(inp.x.to(DEV))
    ws = [X.x1cb_pack_weight(w.to(DEV)) for w in inp.w]
    bs = [b.to(DEV) for b in inp.bias]
    ms = [m.to(DEV) for m in inp.m]
    out = X.bottleneck_i8(x, ws[0], bs[0], ms[0], ws[1], bs[1], ms[1], ws[2], bs[2], ms[2],
                          inp.m_r, inp.S)
    _ok()
    ref = oracle.bottleneck(inp.x, inp.w, inp.bias, inp.m, inp.m_r, inp.S)
    assert torch.equal(_nhwc(out.cpu()), ref)
    _spread(ref)
