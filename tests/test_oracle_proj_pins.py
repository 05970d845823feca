"""Pins for the oracle's strided convolution and the projection block
(Res3.1: conv1 1x1, conv2 3x3 stride 2, conv3 1x1 with the stride-2 1x1
projection of the block input in the same accumulator).

Each function is checked against something other than itself:
* a pure-Python brute force with a stride (tests/brute.py) on tiny shapes,
  full int8 range and extreme parameters;
* library special cases: float64 ``conv2d`` with ``stride=2`` (exact while
  |acc| < 2^53) and, for the projection, the sum of two int64 matmuls, one of
  them over the block input sliced ``[:, ::2, ::2]``;
* invariants: stride 1 equals the stride-1 oracle; the projection with zero
  projection weights equals the plain 1x1; the block equals its three
  composed layers.
"""
import pytest
import torch
import torch.nn.functional as F

from tests.brute import brute_conv_strided
from x1_conv_bn_b200 import synth


def _requant_torch(acc, bias, m, S):
    t = (acc + bias.long()) * m.long() + (1 << (S - 1))
    return torch.div(t, 1 << S, rounding_mode="floor").clamp(0, 127).to(torch.int8)


STRIDED = [
    # B, H, W, Ic, Oc, R, pad, stride
    (1, 5, 5, 32, 4, 3, 1, 2),
    (2, 4, 6, 32, 3, 3, 1, 2),
    (1, 7, 4, 32, 5, 1, 0, 2),
    (1, 6, 6, 64, 3, 3, 1, 3),
    (2, 3, 3, 32, 2, 3, 1, 1),
]


@pytest.mark.parametrize("shape", STRIDED, ids=[str(s) for s in STRIDED])
def test_strided_vs_brute_force(oracle, shape):
    B, H, W, Ic, Oc, R, pad, stride = shape
    g = torch.Generator().manual_seed(sum(shape))
    x = torch.randint(-128, 128, (B, H, W, Ic), generator=g, dtype=torch.int8)
    w = torch.randint(-128, 128, (Oc, Ic, R, R), generator=g, dtype=torch.int8)
    bias = torch.randint(-(1 << 20), 1 << 20, (Oc,), generator=g, dtype=torch.int32)
    m = torch.randint(-(1 << 16), 1 << 16, (Oc,), generator=g, dtype=torch.int32)
    m[0] = (1 << 31) - 1
    for S in (1, 24, 37):
        got = oracle.conv_strided(x, w, bias, m, S, stride, pad=pad)
        exp = brute_conv_strided(x.tolist(), w.tolist(), bias.tolist(), m.tolist(), S, stride,
                                 pad)
        assert got.tolist() == exp


def test_stride2_3x3_vs_float64_conv2d(oracle):
    s = synth.ConvShape(2, 56, 56, 128, 128, 3, False)
    inp = synth.conv_inputs(s, 314)
    acc = F.conv2d(inp.x.permute(0, 3, 1, 2).double(), inp.w.double(), stride=2, padding=1)
    assert acc.shape[-2:] == (28, 28)
    acc = acc.permute(0, 2, 3, 1).reshape(-1, s.Oc).round().long()
    exp = _requant_torch(acc, inp.bias, inp.m, inp.S)
    got = oracle.conv_strided(inp.x, inp.w, inp.bias, inp.m, inp.S, 2)
    assert got.shape == (2, 28, 28, 128)
    assert torch.equal(got.reshape(-1, s.Oc), exp)
    assert exp.unique().numel() > 60


def test_odd_extent_stride2(oracle):
    """H = 7 with pad 1, stride 2: (7 + 2 - 3) // 2 + 1 = 4 output rows; the
    last row's bottom taps fall outside the image."""
    g = torch.Generator().manual_seed(5)
    x = torch.randint(-128, 128, (1, 7, 9, 32), generator=g, dtype=torch.int8)
    w = torch.randint(-128, 128, (128, 32, 3, 3), generator=g, dtype=torch.int8)
    bias = torch.randint(-1000, 1000, (128,), generator=g, dtype=torch.int32)
    m = torch.full((128,), 1 << 12, dtype=torch.int32)
    acc = F.conv2d(x.permute(0, 3, 1, 2).double(), w.double(), stride=2, padding=1)
    acc = acc.permute(0, 2, 3, 1).reshape(-1, 128).round().long()
    got = oracle.conv_strided(x, w, bias, m, 24, 2)
    assert got.shape == (1, 4, 5, 128)
    assert torch.equal(got.reshape(-1, 128), _requant_torch(acc, bias, m, 24))


def test_stride1_equals_the_plain_oracle(oracle):
    s = synth.ConvShape(2, 9, 7, 64, 128, 3, False)
    inp = synth.conv_inputs(s, 8)
    a = oracle.conv(inp.x, inp.w, inp.bias, inp.m, inp.S)
    b = oracle.conv_strided(inp.x, inp.w, inp.bias, inp.m, inp.S, 1)
    assert torch.equal(a, b)


def _proj_inputs(B, H, W, Cy, Cx, Oc, seed, full=False):
    g = torch.Generator().manual_seed(seed)
    lo = -128 if full else 0
    y = torch.randint(lo, 128, (B, H, W, Cy), generator=g, dtype=torch.int8)
    x = torch.randint(lo, 128, (B, 2 * H, 2 * W, Cx), generator=g, dtype=torch.int8)
    w3 = torch.randint(-127, 128, (Oc, Cy, 1, 1), generator=g, dtype=torch.int8)
    wp = torch.randint(-127, 128, (Oc, Cx, 1, 1), generator=g, dtype=torch.int8)
    bias = torch.randint(-(1 << 14), (1 << 14) + 1, (Oc,), generator=g, dtype=torch.int32)
    c = synth.multiplier_center(Cy + Cx)
    m = torch.randint(int(0.9 * c), int(1.1 * c) + 1, (Oc,), generator=g, dtype=torch.int32)
    return y, x, w3, wp, bias, m


def test_projection_vs_two_int64_matmuls(oracle):
    B, H, W, Cy, Cx, Oc = 2, 28, 28, 128, 256, 512
    y, x, w3, wp, bias, m = _proj_inputs(B, H, W, Cy, Cx, Oc, 77)
    xs = x[:, ::2, ::2, :]
    acc = (y.reshape(-1, Cy).long() @ w3.reshape(Oc, Cy).long().T
           + xs.reshape(-1, Cx).long() @ wp.reshape(Oc, Cx).long().T)
    exp = _requant_torch(acc, bias, m, 24)
    got = oracle.conv_proj(y, w3, x, wp, bias, m, 24)
    assert torch.equal(got.reshape(-1, Oc), exp)
    assert 0.05 < (exp == 0).float().mean() < 0.95 and exp.unique().numel() > 60


def test_projection_full_range_vs_brute_force(oracle):
    """Full int8 range and extreme multipliers through a pure-Python sum over
    both sources (tiny shape)."""
    B, H, W, Cy, Cx, Oc = 1, 2, 3, 32, 64, 3
    y, x, w3, wp, bias, m = _proj_inputs(B, H, W, Cy, Cx, Oc, 9, full=True)
    m[0], m[1] = (1 << 31) - 1, -(1 << 31)
    S = 40
    got = oracle.conv_proj(y, w3, x, wp, bias, m, S).tolist()
    Y, X_, W3, WP = y.tolist(), x.tolist(), w3.tolist(), wp.tolist()
    for h in range(H):
        for w in range(W):
            for o in range(Oc):
                acc = sum(Y[0][h][w][i] * W3[o][i][0][0] for i in range(Cy))
                acc += sum(X_[0][2 * h][2 * w][j] * WP[o][j][0][0] for j in range(Cx))
                t = (acc + int(bias[o])) * int(m[o]) + (1 << (S - 1))
                assert got[0][h][w][o] == min(max(t >> S, 0), 127)


def test_projection_with_zero_projection_is_the_1x1(oracle):
    y, x, w3, wp, bias, m = _proj_inputs(2, 5, 6, 64, 96, 128, 11)
    a = oracle.conv_proj(y, w3, x, torch.zeros_like(wp), bias, m, 24)
    b = oracle.conv(y, w3, bias, m, 24)
    assert torch.equal(a, b)


def test_projection_block_is_its_layers(oracle):
    B, H, W, Cin, Cmid, Cout = 2, 12, 10, 256, 128, 512
    g = torch.Generator().manual_seed(3)
    x = torch.randint(0, 128, (B, H, W, Cin), generator=g, dtype=torch.int8)
    shapes = [(Cmid, Cin, 1), (Cmid, Cmid, 3), (Cout, Cmid, 1)]
    ws, bs, ms = [], [], []
    for (o, i, R), K in zip(shapes, [Cin, 9 * Cmid, Cmid + Cin]):
        ws.append(torch.randint(-127, 128, (o, i, R, R), generator=g, dtype=torch.int8))
        bs.append(torch.randint(-(1 << 14), (1 << 14) + 1, (o,), generator=g, dtype=torch.int32))
        c = synth.multiplier_center(K)
        ms.append(torch.randint(int(0.9 * c), int(1.1 * c) + 1, (o,), generator=g,
                                dtype=torch.int32))
    wp = torch.randint(-127, 128, (Cout, Cin, 1, 1), generator=g, dtype=torch.int8)
    blk = oracle.bottleneck_proj(x, ws, wp, bs, ms, 24)
    y1 = oracle.conv_strided(x, ws[0], bs[0], ms[0], 24, 1)
    y2 = oracle.conv_strided(y1, ws[1], bs[1], ms[1], 24, 2)
    y3 = oracle.conv_proj(y2, ws[2], x, wp, bs[2], ms[2], 24)
    assert blk.shape == (B, 6, 5, Cout)
    assert torch.equal(blk, y3)
    for t in (y1, y2, y3):
        assert t.unique().numel() > 20
