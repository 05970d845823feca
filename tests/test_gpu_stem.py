"""GPU parity of the stem kernel: conv (7x7 stride 2 pad 3 in ResNet50, also
3x3 and 1x1 forms) + BN + ReLU + 3x3 stride-2 max pooling in one launch,
64 output channels, against the CPU oracle byte for byte.

The image's 3 channels travel as one 32-channel block whose other channels
are zero (on the GPU side only; the oracle computes with the 3 channels).
Odd image extents exercise the pooled tiles' ragged edges and the conv
pixels outside the image that the pooling must ignore.
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


def _stem_case(B, H, W, Cin, R, seed, full=False):
    g = torch.Generator().manual_seed(seed)
    lo = -128 if full else 0
    x = torch.randint(lo, 128, (B, H, W, Cin), generator=g, dtype=torch.int8)
    w = torch.randint(-127, 128, (64, Cin, R, R), generator=g, dtype=torch.int8)
    if full:
        bias = torch.randint(-(1 << 20), 1 << 20, (64,), generator=g, dtype=torch.int32)
        m = torch.randint(-(1 << 16), 1 << 16, (64,), generator=g, dtype=torch.int32)
        S = 30
    else:
        bias = torch.randint(-(1 << 14), (1 << 14) + 1, (64,), generator=g, dtype=torch.int32)
        c = synth.multiplier_center(R * R * Cin)
        m = torch.randint(int(0.9 * c), int(1.1 * c) + 1, (64,), generator=g, dtype=torch.int32)
        S = 24
    return x, w, bias, m, S


def _gpu_stem(x, w, bias, m, S, R, stride):
    B, H, W, Cin = x.shape
    C = (Cin + 31) // 32 * 32
    xp = torch.zeros(B, H, W, C, dtype=torch.int8)
    xp[..., :Cin] = x
    wp = torch.zeros(64, C, R, R, dtype=torch.int8)
    wp[:, :Cin] = w
    out = X.conv_bn_relu_maxpool_i8(X.x1cb_pack_act(xp.to(DEV)), X.x1cb_pack_weight(wp.to(DEV)),
                                    bias.to(DEV), m.to(DEV), S, R=R, stride=stride)
    torch.cuda.synchronize()
    st, bits = X.x1cb_last_device_error(clear=True)
    assert st == 0, hex(bits)
    return _nhwc(out.cpu())


STEM = [
    # B, H, W, Cin, R, stride
    (2, 224, 224, 3, 7, 2),    # ResNet50's stem: 112x112 conv, 56x56 pooled
    (1, 37, 29, 3, 7, 2),      # odd extents: ragged pooled tiles
    (3, 30, 26, 64, 3, 1),     # 3x3 stride 1 + pool
    (2, 17, 21, 32, 1, 2),     # 1x1 stride 2 + pool
    (1, 5, 3, 3, 7, 2),        # one pooled tile smaller than the tile shape
]


@pytest.mark.parametrize("shape", STEM, ids=[str(s) for s in STEM])
def test_stem_parity(oracle, shape):
    B, H, W, Cin, R, stride = shape
    x, w, bias, m, S = _stem_case(B, H, W, Cin, R, sum(shape))
    got = _gpu_stem(x, w, bias, m, S, R, stride)
    ref = oracle.conv_pool(x, w, bias, m, S, stride=stride)
    assert got.shape == ref.shape
    assert torch.equal(got, ref), int((got != ref).sum())
    assert ref.unique().numel() > 10


def test_stem_full_int8_range(oracle):
    x, w, bias, m, S = _stem_case(2, 45, 38, 32, 7, 3, full=True)
    got = _gpu_stem(x, w, bias, m, S, 7, 2)
    ref = oracle.conv_pool(x, w, bias, m, S, stride=2)
    assert torch.equal(got, ref), int((got != ref).sum())


def test_stem_full_size_every_output(oracle):
    """ResNet50's stem at B=64 (224x224x3 -> 56x56x64), every output byte."""
    x, w, bias, m, S = _stem_case(64, 224, 224, 3, 7, 2024)
    got = _gpu_stem(x, w, bias, m, S, 7, 2)
    ref = oracle.conv_pool(x, w, bias, m, S, stride=2)
    assert torch.equal(got, ref), int((got != ref).sum())
    assert (ref == 0).float().mean() < 0.9


def _gpu_folded_stem(x, w, bias, m, S, R):
    folded = X.x1cb_pack_stem(x.to(DEV).contiguous(), R=R)
    wf = X.x1cb_pack_stem_weight(w.to(DEV).contiguous())
    out = X.stem_conv_bn_relu_maxpool_i8(folded, wf, bias.to(DEV), m.to(DEV), S, R=R,
                                         W=x.shape[2])
    torch.cuda.synchronize()
    st, bits = X.x1cb_last_device_error(clear=True)
    assert st == 0, hex(bits)
    return _nhwc(out.cpu())


FOLDED = [
    (2, 224, 224, 3, 7),
    (1, 37, 29, 3, 7),
    (3, 20, 18, 4, 7),     # 28 of 32 channels used
    (2, 15, 17, 10, 3),    # 3x3 over 10 channels: 30 of 32
    (1, 6, 5, 3, 5),
]


@pytest.mark.parametrize("shape", FOLDED, ids=[str(s) for s in FOLDED])
def test_folded_stem_parity(oracle, shape):
    """The width-folded stem (R x 1 over the folded image) against the
    oracle's R x R stem on the plain image."""
    B, H, W, Cin, R = shape
    x, w, bias, m, S = _stem_case(B, H, W, Cin, R, 7 * sum(shape))
    got = _gpu_folded_stem(x, w, bias, m, S, R)
    ref = oracle.conv_pool(x, w, bias, m, S, stride=2)
    assert got.shape == ref.shape
    assert torch.equal(got, ref), int((got != ref).sum())
    assert ref.unique().numel() > 10


@pytest.mark.parametrize("W", [9, 10])
def test_pack_stem_layout(W):
    """Folded pixel (h, c), channel ds*Cin + ci = image pixel (h, 2c - 3 + ds),
    channel ci (zero outside); channels from R*Cin on are zero; Wc = the
    stride-2 convolution's output columns."""
    g = torch.Generator().manual_seed(4 + W)
    x = torch.randint(-128, 128, (2, 5, W, 3), generator=g, dtype=torch.int8)
    Wc = (W + 6 - 7) // 2 + 1
    got = X.x1cb_pack_stem(x.to(DEV), R=7).cpu()
    assert got.shape == (2, 1, 5, Wc, 32)
    got = got.reshape(2, 5, Wc, 32)
    ref = torch.zeros(2, 5, Wc, 32, dtype=torch.int8)
    xp = torch.nn.functional.pad(x, (0, 0, 3, 3 + 2))  # pad W by 3 (and 2 for the last column)
    for ds in range(7):
        ref[..., ds * 3:ds * 3 + 3] = xp[:, :, ds:ds + 2 * Wc:2, :]
    assert torch.equal(got, ref)


def test_folded_stem_full_size_every_output(oracle):
    """ResNet50's stem at B=64 through the folded path, every output byte."""
    x, w, bias, m, S = _stem_case(64, 224, 224, 3, 7, 2025)
    got = _gpu_folded_stem(x, w, bias, m, S, 7)
    ref = oracle.conv_pool(x, w, bias, m, S, stride=2)
    assert torch.equal(got, ref), int((got != ref).sum())
