"""Pins for the oracle's stem: 3x3 stride-2 max pooling and the fused
conv (7x7, stride 2, pad 3) + BN + ReLU + max pooling, plus the blocked
weight layout of a 64-channel layer.

* max pooling against torch's ``max_pool2d`` (its padding never wins) on
  float64 copies, odd and even extents, and a pure-Python brute force;
* the whole stem against float64 ``conv2d`` (stride 2, pad 3; exact while
  |acc| < 2^53), the requantisation written with ``torch.div(...,
  rounding_mode='floor')`` and ``max_pool2d``;
* zero-padding the image's 3 channels to the 32 of one channel block changes
  nothing;
* the 64-channel blocked layout [1, R, R, Ic/32, 64, 32] as a torch permute.
"""
import pytest
import torch
import torch.nn.functional as F

from x1_conv_bn_b200 import synth


def _pool_torch(y):
    t = F.max_pool2d(y.permute(0, 3, 1, 2).double(), 3, stride=2, padding=1)
    return t.permute(0, 2, 3, 1).to(torch.int8)


@pytest.mark.parametrize("shape", [(2, 112, 112, 64), (1, 7, 5, 32), (3, 1, 1, 8), (1, 2, 9, 4)])
def test_maxpool_vs_torch(oracle, shape):
    g = torch.Generator().manual_seed(sum(shape))
    y = torch.randint(-128, 128, shape, generator=g, dtype=torch.int8)
    got = oracle.maxpool3s2(y)
    assert torch.equal(got, _pool_torch(y))


def test_maxpool_brute_force(oracle):
    g = torch.Generator().manual_seed(3)
    y = torch.randint(-128, 128, (1, 5, 6, 3), generator=g, dtype=torch.int8)
    got = oracle.maxpool3s2(y).tolist()
    Y = y.tolist()
    for i in range(3):
        for j in range(3):
            for c in range(3):
                vals = [Y[0][2 * i + r - 1][2 * j + s - 1][c] for r in range(3) for s in range(3)
                        if 0 <= 2 * i + r - 1 < 5 and 0 <= 2 * j + s - 1 < 6]
                assert got[0][i][j][c] == max(vals)


def _requant(acc, bias, m, S):
    t = (acc + bias.long()) * m.long() + (1 << (S - 1))
    return torch.div(t, 1 << S, rounding_mode="floor").clamp(0, 127).to(torch.int8)


def _stem_inputs(B, H, W, Cin, Oc, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randint(0, 128, (B, H, W, Cin), generator=g, dtype=torch.int8)
    w = torch.randint(-127, 128, (Oc, Cin, 7, 7), generator=g, dtype=torch.int8)
    bias = torch.randint(-(1 << 14), (1 << 14) + 1, (Oc,), generator=g, dtype=torch.int32)
    c = synth.multiplier_center(49 * Cin)
    m = torch.randint(int(0.9 * c), int(1.1 * c) + 1, (Oc,), generator=g, dtype=torch.int32)
    return x, w, bias, m


def test_stem_vs_float64_conv_and_pool(oracle):
    x, w, bias, m = _stem_inputs(2, 56, 56, 3, 64, 7)
    acc = F.conv2d(x.permute(0, 3, 1, 2).double(), w.double(), stride=2, padding=3)
    acc = acc.permute(0, 2, 3, 1).round().long()
    y = _requant(acc, bias, m, 24)
    exp = _pool_torch(y)
    got = oracle.conv_pool(x, w, bias, m, 24, stride=2)
    assert got.shape == (2, 14, 14, 64)
    assert torch.equal(got, exp)
    assert exp.unique().numel() > 30 and (exp == 0).float().mean() < 0.9


def test_stem_channel_padding_changes_nothing(oracle):
    x, w, bias, m = _stem_inputs(1, 23, 17, 3, 64, 8)
    xp = torch.zeros(1, 23, 17, 32, dtype=torch.int8)
    xp[..., :3] = x
    wp = torch.zeros(64, 32, 7, 7, dtype=torch.int8)
    wp[:, :3] = w
    assert torch.equal(oracle.conv_pool(x, w, bias, m, 24), oracle.conv_pool(xp, wp, bias, m, 24))


def test_stem_is_conv_then_pool(oracle):
    x, w, bias, m = _stem_inputs(2, 20, 18, 32, 64, 9)
    y = oracle.conv_strided(x, w, bias, m, 24, 2)
    assert torch.equal(oracle.conv_pool(x, w, bias, m, 24), oracle.maxpool3s2(y))


def test_64_channel_weight_layout(oracle):
    w = torch.randint(-128, 128, (64, 32, 7, 7), dtype=torch.int8)
    blk = oracle.pack_weight(w)
    ref = w.reshape(1, 64, 1, 32, 7, 7).permute(0, 4, 5, 2, 1, 3).contiguous()
    assert blk.shape == (1, 7, 7, 1, 64, 32)
    assert torch.equal(blk, ref)
    assert torch.equal(oracle.unpack_weight(blk, 64, 32, 7), w)
