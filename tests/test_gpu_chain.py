"""GPU parity of the fused Conv2 -> Conv3 kernel (pairs of CTAs sharing each
MMA; Conv2's int8 output stays in shared memory as Conv3's A operand).

bottleneck_i8 takes the fused form for Cmid = 128; these tests compare it
byte for byte with the oracle's three composed layers and with the
three-launch form of the same library, over shapes whose halo tiling has an
odd tile count (the last pair's second CTA has no tile), ragged image rows
and batches, both I/O stage forms (4-pixel groups and whole 8-byte rows),
Cout from 128 to 1024, and many launches back to back.
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
    X.x1cb_set_block_fusion(True)
    X.x1cb_last_device_error(clear=True)
    yield
    X.x1cb_set_block_fusion(False)  # the library's default


def _nhwc(t):
    B, C1, H, W, _ = t.shape
    return t.permute(0, 2, 3, 1, 4).reshape(B, H, W, C1 * 32)


def _packed(inp):
    x = X.x1cb_pack_act(inp.x.to(DEV))
    args = []
    for w, b, m in zip(inp.w, inp.bias, inp.m):
        args += [X.x1cb_pack_weight(w.to(DEV)), b.to(DEV), m.to(DEV)]
    return x, args


def _run(x, args, inp, fused):
    X.x1cb_set_block_fusion(fused)
    try:
        out = X.bottleneck_i8(x, *args, inp.m_r, inp.S)
        torch.cuda.synchronize()
    finally:
        X.x1cb_set_block_fusion(True)  # this module's setting
    st, bits = X.x1cb_last_device_error(clear=True)
    assert st == 0, hex(bits)
    return out


CHAIN = [
    # B, H, W, Cin (= Cout), Cmid
    (1, 28, 28, 512, 128),     # 7 halo tiles: the last pair is half empty
    (2, 28, 28, 512, 128),
    (3, 9, 4, 384, 128),       # 4-pixel groups, several images per tile
    (1, 6, 5, 256, 128),       # 5-wide rows: whole-row I/O stages
    (5, 14, 14, 1024, 128),    # Cout = 1024 (8 output chunks), 14-wide rows
    (2, 7, 7, 128, 128),       # one output chunk
    (4, 30, 28, 512, 128),     # ragged in H
]


@pytest.mark.parametrize("shape", CHAIN, ids=[str(s) for s in CHAIN])
def test_fused_block_parity(oracle, shape):
    inp = synth.block_inputs(synth.BlockShape(*shape), 77)
    x, args = _packed(inp)
    X.x1cb_last_epilogue_forms(clear=True)
    got = _nhwc(_run(x, args, inp, True).cpu())
    assert X.x1cb_last_epilogue_forms(clear=True) != 0
    ref = oracle.bottleneck(inp.x, inp.w, inp.bias, inp.m, inp.m_r, inp.S)
    assert torch.equal(got, ref), int((got != ref).sum())
    assert (ref == 0).float().mean() < 0.95 and ref.unique().numel() > 20


def test_fused_equals_three_launches():
    inp = synth.block_inputs(synth.BlockShape(9, 28, 28, 512, 128), 5)
    x, args = _packed(inp)
    a = _run(x, args, inp, True)
    b = _run(x, args, inp, False)
    assert torch.equal(a, b)


def test_fused_block_full_int8_range(oracle):
    """Full-range activations and weights with wide biases and multipliers:
    Conv2's and Conv3's forms differ from the benchmark's."""
    s = synth.BlockShape(2, 12, 12, 256, 128)
    g = torch.Generator().manual_seed(9)
    inp = synth.block_inputs(s, 9)
    inp.x = torch.randint(-128, 128, inp.x.shape, generator=g, dtype=torch.int8)
    for k in range(3):
        inp.w[k] = torch.randint(-128, 128, inp.w[k].shape, generator=g, dtype=torch.int8)
        inp.bias[k] = torch.randint(-(1 << 20), 1 << 20, inp.bias[k].shape, generator=g,
                                    dtype=torch.int32)
        inp.m[k] = torch.randint(-(1 << 12), 1 << 12, inp.m[k].shape, generator=g,
                                 dtype=torch.int32)
    inp.S = 30
    inp.m_r = -(3 << 20)
    x, args = _packed(inp)
    got = _nhwc(_run(x, args, inp, True).cpu())
    ref = oracle.bottleneck(inp.x, inp.w, inp.bias, inp.m, inp.m_r, inp.S)
    assert torch.equal(got, ref), int((got != ref).sum())


def test_fused_block_repeated_launches(oracle):
    """300 back-to-back fused blocks: the pair protocol's barrier phases
    (cross-CTA arrivals, multicast commits) stay exact launch after launch."""
    inp = synth.block_inputs(synth.BlockShape(64, 28, 28, 512, 128), 13)
    x, args = _packed(inp)
    X.x1cb_last_device_error(clear=True)
    outs = []
    for i in range(300):
        o = X.bottleneck_i8(x, *args, inp.m_r, inp.S)
        if i % 100 == 0 or i == 299:
            outs.append(o)
    torch.cuda.synchronize()
    st, bits = X.x1cb_last_device_error(clear=True)
    assert st == 0, hex(bits)
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    pix = torch.arange(0, 64 * 784, 97)
    ref = oracle.bottleneck_pixels(inp.x, inp.w, inp.bias, inp.m, inp.m_r, inp.S, pix)
    got = _nhwc(outs[-1].cpu()).reshape(-1, 512)[pix]
    assert torch.equal(got, ref)


def test_fused_entry_point_equals_the_two_layers():
    """conv3x3_conv1x1_bn_add_relu_i8 against conv3x3_bn_relu_i8 followed by
    conv1x1_bn_add_relu_i8 (both oracle-checked elsewhere), bit for bit."""
    s = synth.BlockShape(6, 28, 28, 512, 128)
    inp = synth.block_inputs(s, 17)
    x, args = _packed(inp)
    y1 = X.conv1x1_bn_add_relu_i8(x, args[0], args[1], args[2], 0, inp.S)
    fused = X.conv3x3_conv1x1_bn_add_relu_i8(y1, args[3], args[4], args[5], args[6], args[7],
                                             args[8], inp.m_r, inp.S, x)
    y2 = X.conv3x3_bn_relu_i8(y1, args[3], args[4], args[5], inp.S)
    two = X.conv1x1_bn_add_relu_i8(y2, args[6], args[7], args[8], inp.m_r, inp.S, x)
    torch.cuda.synchronize()
    assert X.x1cb_last_device_error(clear=True)[0] == 0
    assert torch.equal(fused, two)
    assert "resident_clusters=" in X.x1cb_describe_chain(6, 28, 28)
