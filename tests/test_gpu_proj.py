"""GPU parity of the projection-block path (Res3.1): the stride-2 3x3 (phase
planes of the input, or one strided box per tap for very wide images), the
Conv3 + projection shortcut in one accumulator, and the three-layer block,
each through the C ABI against the CPU oracle, byte for byte.

Inputs are drawn by x1_conv_bn_b200.synth; each side packs with its own code.
Ragged and odd extents are covered: an odd input (7 x 9 -> 4 x 5), a batch
tail, tiles of fewer than 128 GEMM rows.
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


def _status_ok():
    torch.cuda.synchronize()
    st, bits = X.x1cb_last_device_error(clear=True)
    assert st == 0, bits


def _spread(ref):
    assert (ref == 0).float().mean() < 0.95 and ref.unique().numel() > 20


S2_SHAPES = [
    # B, H, W, Ic, Oc  (input extent; output (H-1)//2+1 x (W-1)//2+1)
    (2, 56, 56, 128, 128),
    (3, 7, 9, 64, 128),
    (1, 5, 5, 32, 128),
    (5, 30, 20, 96, 384),
    (1, 2, 3, 32, 256),
    (1, 3, 260, 32, 128),   # 130 output columns: one box per tap instead of phase planes
]


@pytest.mark.parametrize("shape", S2_SHAPES, ids=[str(s) for s in S2_SHAPES])
def test_conv3x3_stride2_parity(oracle, shape):
    B, H, W, Ic, Oc = shape
    inp = synth.conv_inputs(synth.ConvShape(B, H, W, Ic, Oc, 3, False), sum(shape))
    x = X.x1cb_pack_act(inp.x.to(DEV))
    w = X.x1cb_pack_weight(inp.w.to(DEV))
    out = X.conv3x3s2_bn_relu_i8(x, w, inp.bias.to(DEV), inp.m.to(DEV), inp.S)
    _status_ok()
    ref = oracle.conv_strided(inp.x, inp.w, inp.bias, inp.m, inp.S, 2)
    got = _nhwc(out.cpu())
    assert got.shape == ref.shape
    assert torch.equal(got, ref), int((got != ref).sum())
    _spread(ref)


# The 128 -> 128 3x3 at stride 2 runs on CTA pairs (phase planes as above):
# several images per tile, odd input extents, an odd tile count, one pixel.
PAIR_S2 = [(2, 56, 56), (3, 9, 13), (5, 8, 8), (2, 57, 57), (1, 1, 1), (7, 28, 20)]


@pytest.mark.parametrize("shape", PAIR_S2, ids=[str(s) for s in PAIR_S2])
def test_conv3x3_stride2_on_cta_pairs(oracle, shape):
    B, H, W = shape
    assert " pair=1 " in X.x1cb_describe_plan_ex(B, H, W, 128, 128, 3, 2)
    inp = synth.conv_inputs(synth.ConvShape(B, H, W, 128, 128, 3, False), 900 + sum(shape))
    x = X.x1cb_pack_act(inp.x.to(DEV))
    w = X.x1cb_pack_weight(inp.w.to(DEV))
    out = X.conv3x3s2_bn_relu_i8(x, w, inp.bias.to(DEV), inp.m.to(DEV), inp.S)
    _status_ok()
    ref = oracle.conv_strided(inp.x, inp.w, inp.bias, inp.m, inp.S, 2)
    got = _nhwc(out.cpu())
    assert got.shape == ref.shape
    assert torch.equal(got, ref), int((got != ref).sum())


def test_conv3x3_stride2_on_cta_pairs_full_int8_range(oracle):
    s = synth.ConvShape(3, 13, 11, 128, 128, 3, False)
    inp = synth.full_range_conv_inputs(s, 23, S=33)
    x = X.x1cb_pack_act(inp.x.to(DEV))
    w = X.x1cb_pack_weight(inp.w.to(DEV))
    out = X.conv3x3s2_bn_relu_i8(x, w, inp.bias.to(DEV), inp.m.to(DEV), inp.S)
    _status_ok()
    ref = oracle.conv_strided(inp.x, inp.w, inp.bias, inp.m, inp.S, 2)
    assert torch.equal(_nhwc(out.cpu()), ref)


def test_conv3x3_stride2_full_int8_range(oracle):
    s = synth.ConvShape(2, 13, 11, 64, 128, 3, False)
    inp = synth.full_range_conv_inputs(s, 17, S=33)
    x = X.x1cb_pack_act(inp.x.to(DEV))
    w = X.x1cb_pack_weight(inp.w.to(DEV))
    out = X.conv3x3s2_bn_relu_i8(x, w, inp.bias.to(DEV), inp.m.to(DEV), inp.S)
    _status_ok()
    ref = oracle.conv_strided(inp.x, inp.w, inp.bias, inp.m, inp.S, 2)
    assert torch.equal(_nhwc(out.cpu()), ref)


def _proj_case(B, H, W, Cy, Cx, Oc, Hx, Wx, seed, full=False):
    g = torch.Generator().manual_seed(seed)
    lo = -128 if full else 0
    y = torch.randint(lo, 128, (B, H, W, Cy), generator=g, dtype=torch.int8)
    x = torch.randint(lo, 128, (B, Hx, Wx, Cx), generator=g, dtype=torch.int8)
    w3 = torch.randint(-127, 128, (Oc, Cy, 1, 1), generator=g, dtype=torch.int8)
    wp = torch.randint(-127, 128, (Oc, Cx, 1, 1), generator=g, dtype=torch.int8)
    if full:
        bias = torch.randint(-(1 << 20), 1 << 20, (Oc,), generator=g, dtype=torch.int32)
        m = torch.randint(-(1 << 20), 1 << 20, (Oc,), generator=g, dtype=torch.int32)
        S = 31
    else:
        bias = torch.randint(-(1 << 14), (1 << 14) + 1, (Oc,), generator=g, dtype=torch.int32)
        c = synth.multiplier_center(Cy + Cx)
        m = torch.randint(int(0.9 * c), int(1.1 * c) + 1, (Oc,), generator=g, dtype=torch.int32)
        S = 24
    return y, x, w3, wp, bias, m, S


PROJ_SHAPES = [
    # B, H, W, Cy, Cx, Oc, Hx, Wx
    (2, 28, 28, 128, 256, 512, 56, 56),
    (3, 7, 9, 64, 96, 256, 14, 18),
    (2, 5, 6, 32, 64, 128, 9, 11),     # odd block input: x read at (2h, 2w) up to 8, 10
    (9, 3, 4, 128, 128, 384, 6, 8),
]


@pytest.mark.parametrize("shape", PROJ_SHAPES, ids=[str(s) for s in PROJ_SHAPES])
@pytest.mark.parametrize("full", [False, True], ids=["bench", "full_range"])
def test_conv1x1_projection_parity(oracle, shape, full):
    y, x, w3, wp, bias, m, S = _proj_case(*shape, seed=sum(shape), full=full)
    ref = oracle.conv_proj(y, w3, x, wp, bias, m, S)
    out = X.conv1x1_proj_bn_relu_i8(X.x1cb_pack_act(y.to(DEV)), X.x1cb_pack_weight(w3.to(DEV)),
                                    X.x1cb_pack_act(x.to(DEV)), X.x1cb_pack_weight(wp.to(DEV)),
                                    bias.to(DEV), m.to(DEV), S)
    _status_ok()
    got = _nhwc(out.cpu())
    assert torch.equal(got, ref), int((got != ref).sum())
    if not full:
        _spread(ref)


def _run_proj_block(inp):
    x = X.x1cb_pack_act(inp.x.to(DEV))
    ws = [X.x1cb_pack_weight(w.to(DEV)) for w in inp.w]
    wp = X.x1cb_pack_weight(inp.wp.to(DEV))
    bs = [b.to(DEV) for b in inp.bias]
    ms = [m.to(DEV) for m in inp.m]
    out = X.bottleneck_proj_i8(x, ws[0], bs[0], ms[0], ws[1], bs[1], ms[1], ws[2], wp, bs[2],
                               ms[2], inp.S)
    _status_ok()
    return _nhwc(out.cpu())


@pytest.mark.parametrize("shape", [(2, 56, 56, 256, 128, 512), (1, 9, 7, 128, 128, 256),
                                   (3, 14, 12, 256, 128, 384)])
def test_projection_block_parity(oracle, shape):
    inp = synth.proj_block_inputs(synth.ProjBlockShape(*shape), 41)
    ref = oracle.bottleneck_proj(inp.x, inp.w, inp.wp, inp.bias, inp.m, inp.S)
    got = _run_proj_block(inp)
    assert torch.equal(got, ref), int((got != ref).sum())
    _spread(ref)


def test_projection_block_full_size_every_output(oracle):
    """Res3.1 at B=256 (56x56x256 in, 28x28x512 out): every output byte."""
    s = synth.CONFIGS["p31"]
    inp = synth.proj_block_inputs(s, synth.CONFIG_SEEDS["p31"])
    got = _run_proj_block(inp)
    ref = oracle.bottleneck_proj(inp.x, inp.w, inp.wp, inp.bias, inp.m, inp.S)
    assert torch.equal(got, ref), int((got != ref).sum())
    _spread(ref)
