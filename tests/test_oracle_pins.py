"""Pins for the CPU oracle: it is checked against things other than itself.

* hand-computed requantisation cases (tests/golden/requant_hand_cases.txt);
* a pure-Python brute force on tiny shapes, full int8 range, extreme params;
* library special cases: the 1x1 conv is an int64 matmul and the 3x3 conv a
  float64 ``conv2d`` (exact while |acc| < 2^53), each followed by a
  requantisation written with ``torch.div(..., rounding_mode='floor')``;
* the layout definitions of the Inspur article (section 3.1) re-expressed as
  torch reshapes/permutes;
* invariants: zero weights, identity weights, centre-tap 3x3 == 1x1, batch
  independence, block == three composed layers, pixel-sampled == full.
"""
import os

import pytest
import torch
import torch.nn.functional as F

from tests.brute import brute_conv
from x1_conv_bn_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "requant_hand_cases.txt")


def _hand_cases():
    rows = []
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        acc, bias, m, r, m_r, S, exp = line.split()
        rows.append((int(acc), int(bias), int(m), None if r == "-" else int(r), int(m_r), int(S),
                     int(exp)))
    return rows


HAND = _hand_cases()


def test_golden_file_is_non_trivial():
    assert len(HAND) >= 20
    assert {e for *_, e in HAND} >= {0, 1, 5, 6, 64, 127}


@pytest.mark.parametrize("case", HAND, ids=[f"hand{i}" for i in range(len(HAND))])
def test_requant_hand_cases(oracle, case):
    acc, bias, m, r, m_r, S, exp = case
    assert oracle.requant(acc, bias, m, r, m_r, S) == exp


@pytest.mark.parametrize("case", HAND[:14], ids=[f"hand{i}" for i in range(14)])
def test_hand_cases_through_conv(oracle, case):
    """The same cases reached through a real 1x1 convolution: acc is built as
    x . w with x = (a, 0, ...), w = (1, 0, ...) or spread over channels."""
    acc, bias, m, r, m_r, S, exp = case
    if abs(acc) > 127 * 32:
        pytest.skip("acc not reachable with one unit weight per channel")
    Ic, Oc = 32, 128
    x = torch.zeros(1, 1, 1, Ic, dtype=torch.int8)
    # spread acc over channels in chunks of at most 127 in magnitude
    rem, i = acc, 0
    while rem != 0:
        step = max(-127, min(127, rem))
        x[0, 0, 0, i] = step
        rem -= step
        i += 1
    w = torch.zeros(Oc, Ic, 1, 1, dtype=torch.int8)
    w[:, :, 0, 0] = 1
    b = torch.full((Oc,), bias, dtype=torch.int32)
    mm = torch.full((Oc,), m, dtype=torch.int32)
    rr = None if r is None else torch.full((1, 1, 1, Oc), r, dtype=torch.int8)
    out = oracle.conv(x, w, b, mm, S, rr, m_r)
    assert (out == exp).all()


def _lists(t):
    return t.tolist()


SHAPES = [
    # B, H, W, Ic, Oc, R
    (1, 1, 1, 32, 8, 1),
    (2, 3, 5, 32, 8, 1),
    (1, 2, 2, 64, 4, 1),
    (2, 3, 3, 32, 6, 3),
    (1, 5, 2, 32, 5, 3),
    (1, 1, 1, 32, 3, 3),
    (2, 2, 3, 64, 3, 3),
]


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
@pytest.mark.parametrize("has_res", [True, False])
def test_oracle_vs_brute_force(oracle, shape, has_res):
    B, H, W, Ic, Oc, R = shape
    g = torch.Generator().manual_seed(hash((shape, has_res)) & 0xFFFF)
    x = torch.randint(-128, 128, (B, H, W, Ic), generator=g, dtype=torch.int8)
    w = torch.randint(-128, 128, (Oc, Ic, R, R), generator=g, dtype=torch.int8)
    bias = torch.randint(-(1 << 20), 1 << 20, (Oc,), generator=g, dtype=torch.int32)
    m = torch.randint(-(1 << 16), 1 << 16, (Oc,), generator=g, dtype=torch.int32)
    m[0] = (1 << 31) - 1  # extreme multipliers
    m[-1] = -(1 << 31)
    r = torch.randint(-128, 128, (B, H, W, Oc), generator=g, dtype=torch.int8) if has_res else None
    m_r = -(1 << 27) + 12345
    for S in (1, 24, 30, 45):
        got = oracle.conv(x, w, bias, m, S, r, m_r)
        exp = brute_conv(_lists(x), _lists(w), _lists(bias), _lists(m), S,
                         _lists(r) if r is not None else None, m_r)
        assert got.tolist() == exp


def _requant_torch(acc, bias, m, S, r=None, m_r=0):
    """Requantisation with torch int64 ops; floor division by the library."""
    t = (acc + bias.long()) * m.long()
    if r is not None:
        t = t + r.long() * m_r
    t = t + (1 << (S - 1))
    y = torch.div(t, 1 << S, rounding_mode="floor")
    return y.clamp(0, 127).to(torch.int8)


@pytest.mark.parametrize("cfg", ["1"])
def test_1x1_vs_int64_matmul(oracle, cfg):
    s = synth.CONFIGS[cfg]
    inp = synth.conv_inputs(s, synth.CONFIG_SEEDS[cfg])
    acc = inp.x.reshape(-1, s.Ic).long() @ inp.w.reshape(s.Oc, s.Ic).long().T
    exp = _requant_torch(acc, inp.bias, inp.m, inp.S, inp.r.reshape(-1, s.Oc), inp.m_r)
    got = oracle.conv(inp.x, inp.w, inp.bias, inp.m, inp.S, inp.r, inp.m_r)
    assert torch.equal(got.reshape(-1, s.Oc), exp)
    # the check is meaningful: outputs are spread, not all clamped
    assert 0.05 < (exp == 0).float().mean() < 0.95
    assert exp.unique().numel() > 60


def test_3x3_vs_float64_conv2d(oracle):
    s = synth.ConvShape(2, 28, 28, 128, 128, 3, False)
    inp = synth.conv_inputs(s, 4242)
    xf = inp.x.permute(0, 3, 1, 2).double()
    acc = F.conv2d(xf, inp.w.double(), padding=1)  # exact: |acc| < 2^53
    acc = acc.permute(0, 2, 3, 1).reshape(-1, s.Oc).round().long()
    exp = _requant_torch(acc, inp.bias, inp.m, inp.S)
    got = oracle.conv(inp.x, inp.w, inp.bias, inp.m, inp.S)
    assert torch.equal(got.reshape(-1, s.Oc), exp)
    assert exp.unique().numel() > 60


def test_full_range_1x1_vs_int64_matmul(oracle):
    s = synth.ConvShape(2, 7, 9, 96, 256, 1, True)
    inp = synth.full_range_conv_inputs(s, 77, S=34)
    acc = inp.x.reshape(-1, s.Ic).long() @ inp.w.reshape(s.Oc, s.Ic).long().T
    exp = _requant_torch(acc, inp.bias, inp.m, inp.S, inp.r.reshape(-1, s.Oc), inp.m_r)
    got = oracle.conv(inp.x, inp.w, inp.bias, inp.m, inp.S, inp.r, inp.m_r)
    assert torch.equal(got.reshape(-1, s.Oc), exp)
    assert 0.1 < (exp == 0).float().mean() < 0.9


# ---- layouts (Inspur article, section 3.1) ---------------------------------

def test_pack_act_matches_layout_definition(oracle):
    B, H, W, C = 2, 5, 3, 96
    x = torch.randint(-128, 128, (B, H, W, C), dtype=torch.int8)
    packed = oracle.pack_act(x)
    # [B, H, W, C] -> [B, C/32, H, W, 32]
    ref = x.reshape(B, H, W, C // 32, 32).permute(0, 3, 1, 2, 4).contiguous()
    assert torch.equal(packed, ref)
    assert torch.equal(oracle.unpack_act(packed), x)


@pytest.mark.parametrize("R", [1, 3])
def test_pack_weight_matches_layout_definition(oracle, R):
    Oc, Ic = 256, 64
    w = torch.randint(-128, 128, (Oc, Ic, R, R), dtype=torch.int8)
    blk = oracle.pack_weight(w)
    # [Oc, Ic, R, S] -> [O1, R, S, I1, O2=128, I2=32]
    ref = w.reshape(Oc // 128, 128, Ic // 32, 32, R, R).permute(0, 4, 5, 2, 1, 3).contiguous()
    assert torch.equal(blk, ref)
    assert torch.equal(oracle.unpack_weight(blk, Oc, Ic, R), w)


def test_pack_weight_1x1_is_o1_i1_o2_i2(oracle):
    """For 1x1 the blocked weight is the article's [O1, I1, O2, I2] = [4, 4, 128, 32]
    for the Conv3 shape Oc=512, Ic=128."""
    w = torch.randint(-128, 128, (512, 128, 1, 1), dtype=torch.int8)
    blk = oracle.pack_weight(w).reshape(4, 4, 128, 32)
    o, i = 300, 77
    assert blk[o // 128, i // 32, o % 128, i % 32] == w[o, i, 0, 0]


# ---- invariants --------------------------------------------------------------

def test_zero_weights_gives_half_residual(oracle):
    s = synth.ConvShape(2, 4, 4, 32, 128, 1, True)
    inp = synth.conv_inputs(s, 5)
    zero_w = torch.zeros_like(inp.w)
    zero_b = torch.zeros_like(inp.bias)
    got = oracle.conv(inp.x, zero_w, zero_b, inp.m, inp.S, inp.r, inp.m_r)
    # m_r = 2^(S-1): out = floor((r + 1) / 2) for r >= 0
    assert torch.equal(got, torch.div(inp.r.long() + 1, 2, rounding_mode="floor").to(torch.int8))


def test_identity_weight(oracle):
    C = 128
    x = torch.randint(-128, 128, (2, 3, 5, C), dtype=torch.int8)
    w = torch.eye(C, dtype=torch.int8).reshape(C, C, 1, 1)
    S = 24
    got = oracle.conv(x, w, torch.zeros(C, dtype=torch.int32),
                      torch.full((C,), 1 << S, dtype=torch.int32), S)
    assert torch.equal(got, x.clamp(min=0))


def test_centre_tap_3x3_equals_1x1(oracle):
    s1 = synth.ConvShape(2, 6, 7, 64, 128, 1, False)
    inp = synth.conv_inputs(s1, 9)
    w3 = torch.zeros(128, 64, 3, 3, dtype=torch.int8)
    w3[:, :, 1, 1] = inp.w[:, :, 0, 0]
    a = oracle.conv(inp.x, inp.w, inp.bias, inp.m, inp.S)
    b = oracle.conv(inp.x, w3, inp.bias, inp.m, inp.S)
    assert torch.equal(a, b)


def test_batch_independence(oracle):
    s = synth.ConvShape(2, 5, 5, 32, 128, 3, False)
    inp = synth.conv_inputs(s, 11)
    full = oracle.conv(inp.x, inp.w, inp.bias, inp.m, inp.S)
    for b in range(2):
        one = oracle.conv(inp.x[b:b + 1], inp.w, inp.bias, inp.m, inp.S)
        assert torch.equal(full[b:b + 1], one)


def test_block_is_three_layers(oracle):
    s = synth.BlockShape(2, 6, 5, 256, 128)
    inp = synth.block_inputs(s, 21)
    blk = oracle.bottleneck(inp.x, inp.w, inp.bias, inp.m, inp.m_r, inp.S)
    y1 = oracle.conv(inp.x, inp.w[0], inp.bias[0], inp.m[0], inp.S)
    y2 = oracle.conv(y1, inp.w[1], inp.bias[1], inp.m[1], inp.S)
    y3 = oracle.conv(y2, inp.w[2], inp.bias[2], inp.m[2], inp.S, inp.x, inp.m_r)
    assert torch.equal(blk, y3)
    assert y1.unique().numel() > 20 and y2.unique().numel() > 20 and y3.unique().numel() > 20
    pix = torch.tensor([0, 5, 29, 30, 47, 59])
    rows = oracle.bottleneck_pixels(inp.x, inp.w, inp.bias, inp.m, inp.m_r, inp.S, pix)
    assert torch.equal(rows, blk.reshape(-1, 256)[pix])


def test_conv_pixels_matches_full(oracle):
    s = synth.ConvShape(3, 5, 4, 64, 128, 3, True)
    inp = synth.conv_inputs(s, 13)
    full = oracle.conv(inp.x, inp.w, inp.bias, inp.m, inp.S, inp.r, inp.m_r)
    pix = torch.tensor([0, 1, 19, 20, 33, 59])
    rows = oracle.conv_pixels(inp.x, inp.w, inp.bias, inp.m, inp.S, pix, inp.r, inp.m_r)
    assert torch.equal(rows, full.reshape(-1, 128)[pix])


def test_planted_mistakes_are_caught():
    """A pin must fail when the oracle's arithmetic is wrong.  Plant mistakes
    in a Python copy of the requantisation (on the CPU) and check that the
    hand cases reject every one of them."""
    def rq(acc, bias, m, r, m_r, S, mistake):
        if mistake == "drop_bias":
            t = acc * m
        elif mistake == "bias_after_mul":
            t = acc * m + bias
        else:
            t = (acc + bias) * m
        if r is not None and mistake != "drop_res":
            t += (r * m_r) if mistake != "res_sign" else -(r * m_r)
        if mistake != "no_round":
            t += 1 << (S - 1)
        if mistake == "logical_shift":
            y = (t % (1 << 64)) >> S
        elif mistake == "int32_wrap":
            t32 = ((t + (1 << 31)) % (1 << 32)) - (1 << 31)
            y = t32 >> S
        else:
            y = t >> S
        hi = 255 if mistake == "u8_clamp" else 127
        return min(max(y, 0), hi)

    for mistake in ["drop_bias", "bias_after_mul", "drop_res", "res_sign", "no_round",
                    "logical_shift", "int32_wrap", "u8_clamp"]:
        bad = [c for c in HAND if rq(*c[:6], mistake) != c[6]]
        assert bad, f"hand cases do not catch mistake {mistake}"
    # the unmodified rule passes every hand case
    assert all(rq(*c[:6], None) == c[6] for c in HAND)
