"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Integer arithmetic has a unique result, so every comparison is bit-exact.
Inputs come from the seeded generators in x1_conv_bn_b200.synth; the GPU side
packs them with its own pack kernels, the oracle computes from the logical
NHWC/OIHW tensors with its own code, and the packed GPU output is compared
with the oracle output packed by the oracle.
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
    X.x1cb_debug_inject(0)
    X.x1cb_set_wait_limit_ns(0)
    st, bits = X.x1cb_last_device_error(clear=True)


def _gpu_conv(inp: synth.ConvInputs):
    s = inp.shape
    x = X.x1cb_pack_act(inp.x.to(DEV).contiguous())
    w = X.x1cb_pack_weight(inp.w.to(DEV).contiguous())
    bias, m = inp.bias.to(DEV), inp.m.to(DEV)
    if s.R == 1:
        r = X.x1cb_pack_act(inp.r.to(DEV).contiguous()) if inp.r is not None else None
        out = X.conv1x1_bn_add_relu_i8(x, w, bias, m, inp.m_r, inp.S, r)
    else:
        assert inp.r is None
        out = X.conv3x3_bn_relu_i8(x, w, bias, m, inp.S)
    torch.cuda.synchronize()
    st, bits = X.x1cb_last_device_error(clear=True)
    assert st == 0, bits
    return out.cpu()


def _oracle_conv(oracle, inp):
    return oracle.conv(inp.x, inp.w, inp.bias, inp.m, inp.S, inp.r, inp.m_r)


def _assert_spread(ref):
    # the case exercises the arithmetic, not only the clamps
    frac0 = (ref == 0).float().mean().item()
    assert frac0 < 0.95 and (ref == 127).float().mean().item() < 0.95


# ---- layout kernels -----------------------------------------------------------

@pytest.mark.parametrize("shape", [(1, 1, 1, 32), (2, 5, 7, 96), (3, 28, 28, 128), (1, 3, 130, 64)])
def test_pack_unpack_act(oracle, shape):
    g = torch.Generator().manual_seed(1)
    x = torch.randint(-128, 128, shape, generator=g, dtype=torch.int8)
    got = X.x1cb_pack_act(x.to(DEV)).cpu()
    assert torch.equal(got, oracle.pack_act(x))
    back = X.x1cb_unpack_act(X.x1cb_pack_act(x.to(DEV))).cpu()
    assert torch.equal(back, x)


@pytest.mark.parametrize("shape", [(128, 32, 1), (512, 128, 1), (256, 64, 3), (128, 128, 3)])
def test_pack_weight(oracle, shape):
    Oc, Ic, R = shape
    g = torch.Generator().manual_seed(2)
    w = torch.randint(-128, 128, (Oc, Ic, R, R), generator=g, dtype=torch.int8)
    got = X.x1cb_pack_weight(w.to(DEV)).cpu()
    assert torch.equal(got, oracle.pack_weight(w))


# ---- fused 1x1 ------------------------------------------------------------------

SMALL_1X1 = [
    # B, H, W, Ic, Oc   (several tiles, ragged pixel and batch tails)
    (1, 1, 1, 32, 128),
    (1, 28, 28, 128, 512),
    (3, 28, 28, 128, 512),
    (9, 28, 28, 128, 512),
    (2, 7, 9, 64, 256),
    (5, 14, 14, 256, 1024),
    (7, 7, 7, 512, 2048),
    (3, 56, 56, 64, 256),
    (2, 3, 5, 1024, 128),
    (17, 2, 3, 32, 384),
]


@pytest.mark.parametrize("shape", SMALL_1X1, ids=[str(s) for s in SMALL_1X1])
@pytest.mark.parametrize("has_res", [True, False], ids=["res", "nores"])
def test_conv1x1_parity(oracle, shape, has_res):
    s = synth.ConvShape(*shape, R=1, has_res=has_res)
    inp = synth.conv_inputs(s, seed=hash(shape) & 0xFFFF)
    ref = oracle.pack_act(_oracle_conv(oracle, inp))
    got = _gpu_conv(inp)
    assert torch.equal(got, ref), (got != ref).sum().item()
    _assert_spread(ref)


# Shapes whose plans once went wrong: 384- and 768-channel layers large enough
# for wide channel groups (a group must be whole N = 256 MMAs), and a 512 -> 256
# layer with a shortcut whose 4-K-block boxes did not fit beside its weights.
WIDE_GROUPS = [(96, 16, 16, 128, 384), (48, 16, 16, 128, 768), (26, 28, 28, 512, 256)]


@pytest.mark.parametrize("shape", WIDE_GROUPS, ids=[str(s) for s in WIDE_GROUPS])
def test_conv1x1_channel_groups(oracle, shape):
    s = synth.ConvShape(*shape, R=1, has_res=True)
    inp = synth.conv_inputs(s, 77 + shape[4])
    got = _nhwc(_gpu_conv(inp))
    ref = _oracle_conv(oracle, inp)
    assert torch.equal(got, ref), _first_mismatch(got, ref)


# Shortcut layers whose resident weights take more than 96 KB and whose
# channel group is not one N = 256 MMA stage the shortcut and result in 8 KB
# pieces (two 32-channel chunks): N = 128 groups (four accumulator slots)
# with one K block per box on 125-row tiles.
NARROW_IO = [(9, 7, 7, 1024, 256)]


@pytest.mark.parametrize("shape", NARROW_IO, ids=[str(s) for s in NARROW_IO])
def test_conv1x1_narrow_io_stages(oracle, shape):
    assert "stage_ch=2" in X.x1cb_describe_plan(*shape, 1, True)
    s = synth.ConvShape(*shape, R=1, has_res=True)
    inp = synth.conv_inputs(s, 91 + shape[0])
    got = _nhwc(_gpu_conv(inp))
    ref = _oracle_conv(oracle, inp)
    assert torch.equal(got, ref), _first_mismatch(got, ref)
    _assert_spread(oracle.pack_act(ref))


# Shortcut layers whose 256-channel groups take more than 96 KB of weights run
# on CTA pairs sharing each MMA (M = 256): an even and an odd tile count (the
# second CTA of the last pair has no tile), a batch tail, and one channel group
# over many pairs.
PAIR_1X1 = [(43, 7, 7, 512, 2048), (41, 7, 7, 512, 2048), (26, 28, 28, 512, 256)]


@pytest.mark.parametrize("shape", PAIR_1X1, ids=[str(s) for s in PAIR_1X1])
def test_conv1x1_on_cta_pairs(oracle, shape):
    assert "cta_pair=1" in X.x1cb_describe_plan(*shape, 1, True)
    s = synth.ConvShape(*shape, R=1, has_res=True)
    inp = synth.conv_inputs(s, 71 + shape[0])
    got = _nhwc(_gpu_conv(inp))
    ref = _oracle_conv(oracle, inp)
    assert torch.equal(got, ref), _first_mismatch(got, ref)
    _assert_spread(oracle.pack_act(ref))


@pytest.mark.parametrize("S", [12, 24, 40])
def test_conv1x1_on_cta_pairs_full_int8_range(oracle, S):
    """Full-range operands at three shifts: the epilogue forms with and
    without the bias folded into the pair's MMAs."""
    s = synth.ConvShape(41, 7, 7, 512, 2048, R=1, has_res=True)
    inp = synth.full_range_conv_inputs(s, 300 + S, S=S)
    got = _nhwc(_gpu_conv(inp))
    ref = _oracle_conv(oracle, inp)
    assert torch.equal(got, ref), _first_mismatch(got, ref)


@pytest.mark.parametrize("S", [12, 24, 31, 40])
def test_conv1x1_full_int8_range(oracle, S):
    """x, w, r over [-128, 127], negative multipliers, wide bias, several shifts."""
    s = synth.ConvShape(4, 9, 13, 96, 256, 1, True)
    inp = synth.full_range_conv_inputs(s, 90 + S, S=S)
    ref = oracle.pack_act(_oracle_conv(oracle, inp))
    got = _gpu_conv(inp)
    assert torch.equal(got, ref), (got != ref).sum().item()


def test_conv1x1_hand_cases(oracle):
    """The golden requantisation cases through the full kernel: channel o gets
    acc = a_o (x = (a, 0, ...), w = 1 on channel 0), bias, m and residual of case o."""
    from tests.test_oracle_pins import HAND

    cases = [c for c in HAND if abs(c[0]) <= 127 and c[5] == 24]
    Oc = 128
    Ic = 32
    x = torch.zeros(1, 1, 1, Ic, dtype=torch.int8)
    w = torch.zeros(Oc, Ic, 1, 1, dtype=torch.int8)
    bias = torch.zeros(Oc, dtype=torch.int32)
    m = torch.zeros(Oc, dtype=torch.int32)
    r = torch.zeros(1, 1, 1, Oc, dtype=torch.int8)
    # one pixel: x[0] = 1 so acc_o = w[o, 0]
    x[0, 0, 0, 0] = 1
    exp = []
    m_r = 1 << 23
    for acc, b, mm, rr, mr, S, e in cases:
        if rr is not None and mr != m_r:
            continue
        w[len(exp), 0, 0, 0] = acc
        bias[len(exp)] = b
        m[len(exp)] = mm
        r[0, 0, 0, len(exp)] = 0 if rr is None else rr
        exp.append(e)
    n = len(exp)
    inp = synth.ConvInputs(synth.ConvShape(1, 1, 1, Ic, Oc, 1, True), x, w, bias, m, r, m_r, 24)
    got = X.x1cb_unpack_act(_gpu_conv(inp).to(DEV)).cpu()
    assert got.reshape(-1)[:n].tolist() == exp
    assert torch.equal(got, _oracle_conv(oracle, inp))


def test_conv1x1_bias_too_large_to_fold(oracle):
    """Biases beyond the range the MMA can fold (|bias| > 2^18) take the
    all-32-bit form with the bias added in the epilogue."""
    s = synth.ConvShape(3, 14, 14, 128, 256, 1, True)
    inp = synth.conv_inputs(s, 71)
    g = torch.Generator().manual_seed(72)
    inp.bias = torch.randint(-(1 << 20), (1 << 20) + 1, (s.Oc,), generator=g, dtype=torch.int32)
    inp.bias[0] = (1 << 18) + 1
    ref = oracle.pack_act(_oracle_conv(oracle, inp))
    got = _gpu_conv(inp)
    assert torch.equal(got, ref)
    assert 0.05 < (ref == 0).float().mean().item() < 0.95


def test_conv1x1_mixed_epilogue_forms_across_ctas(oracle):
    """B=1 splits the 512 output channels over 4 CTA groups; group 1 gets a
    bias too large to fold, group 2 a multiplier too large for the 32-bit
    forms, group 3 stays in the folded form: every CTA picks its own exact form."""
    s = synth.CONFIGS["1"]
    inp = synth.conv_inputs(s, 73)
    inp.bias[128:256] = inp.bias[128:256] * 64  # |bias| up to 2^20: no fold
    inp.m[256:384] = inp.m[256:384] * 4096      # m * 2^9 beyond int32: 64-bit form
    assert "groups=4" in X.x1cb_describe_plan(1, 28, 28, 128, 512, 1, 1)
    ref = oracle.pack_act(_oracle_conv(oracle, inp))
    got = _gpu_conv(inp)
    assert torch.equal(got, ref)


# The all-32-bit forms fold the shortcut in as y2 = hi32((acc + bias) * m'') + 1
# + r * k with k = m_r / 2^(S-1).  These cases drive k != 1 (negative, odd,
# and the extremes the form admits), with the bias folded into the MMA and
# added in the epilogue, and check that the intended form really ran.
K_CASES = [(2, -1), (2, 3), (2, -(1 << 23) + 1), (2, 1 << 23),
           (24, -1), (24, 3), (24, -256), (24, 255)]


@pytest.mark.parametrize("S,k", K_CASES, ids=[f"S{S}_k{k}" for S, k in K_CASES])
@pytest.mark.parametrize("fold", [True, False], ids=["fold", "nofold"])
@pytest.mark.parametrize("mag", ["full", "small"])
def test_all32_forms_with_shortcut_scale(oracle, S, k, fold, mag):
    s = synth.ConvShape(3, 9, 13, 96, 256, 1, True)
    g = torch.Generator().manual_seed(S * 7 + (k & 0xFFFF) + (1000 if fold else 0))
    lo, hi = (-128, 127) if mag == "full" else (-3, 3)
    x = torch.randint(lo, hi + 1, (s.B, s.H, s.W, s.Ic), generator=g, dtype=torch.int8)
    w = torch.randint(-128, 128, (s.Oc, s.Ic, 1, 1), generator=g, dtype=torch.int8)
    r = torch.randint(-128, 128, (s.B, s.H, s.W, s.Oc), generator=g, dtype=torch.int8)
    if fold:
        bias = torch.randint(-(1 << 12), (1 << 12) + 1, (s.Oc,), generator=g, dtype=torch.int32)
    else:  # every channel beyond the foldable range
        mag_b = torch.randint((1 << 18) + 1, 1 << 20, (s.Oc,), generator=g, dtype=torch.int32)
        sign = torch.randint(0, 2, (s.Oc,), generator=g, dtype=torch.int32) * 2 - 1
        bias = mag_b * sign
    if S == 2:  # m * 2^31 must fit int32
        m = torch.randint(-1, 1, (s.Oc,), generator=g, dtype=torch.int32)
    else:
        m = torch.randint(-(1 << 21), (1 << 21) + 1, (s.Oc,), generator=g, dtype=torch.int32)
    m_r = k * (1 << (S - 1))
    assert -(1 << 31) <= m_r < (1 << 31)
    inp = synth.ConvInputs(s, x, w, bias, m, r, m_r, S)
    ref = _oracle_conv(oracle, inp)
    X.x1cb_last_epilogue_forms(clear=True)
    got = _nhwc(_gpu_conv(inp))
    forms = X.x1cb_last_epilogue_forms(clear=True)
    assert forms == (1 << (3 if fold else 2)), forms
    assert torch.equal(got, ref), _first_mismatch(got, ref)
    assert ref.unique().numel() >= 2


@pytest.mark.parametrize("k,form", [(-(1 << 23), 0), (-(1 << 23) + 1, 2)])
def test_all32_form_bound_on_the_shortcut_scale(oracle, k, form):
    """At S = 9, m_r = k * 2^8.  With (acc + bias) near -2^31 and m'' = -2^31
    the high word is near 2^30; r = -128 adds -128 * k.  For k = -2^23 that
    sum is 2^31, outside int32, so the all-32-bit form must not be taken (the
    generic form runs); k = -2^23 + 1 still fits and keeps the form.  Either
    way every output is the exact 127."""
    s = synth.ConvShape(1, 2, 4, 32, 128, 1, True)
    x = torch.zeros(s.B, s.H, s.W, s.Ic, dtype=torch.int8)
    x[..., 0] = 1
    w = torch.zeros(s.Oc, s.Ic, 1, 1, dtype=torch.int8)
    w[:, 0, 0, 0] = -128                     # acc = -128
    bias = torch.full((s.Oc,), -(1 << 31) + (1 << 21), dtype=torch.int32)
    m = torch.full((s.Oc,), -128, dtype=torch.int32)  # m * 2^(33-9) = -2^31
    r = torch.full((s.B, s.H, s.W, s.Oc), -128, dtype=torch.int8)
    inp = synth.ConvInputs(s, x, w, bias, m, r, k * 256, 9)
    ref = _oracle_conv(oracle, inp)
    assert (ref == 127).all()
    X.x1cb_last_epilogue_forms(clear=True)
    got = _nhwc(_gpu_conv(inp))
    assert X.x1cb_last_epilogue_forms(clear=True) == 1 << form
    assert torch.equal(got, ref), _first_mismatch(got, ref)


# ---- fused 3x3 ------------------------------------------------------------------

# The halo form covers W+2 <= 128 (tiles of th rows x tg images, ragged in H
# and B); (1, 3, 130, ...) takes the per-tap form.
SMALL_3X3 = [
    (1, 1, 1, 32, 128),
    (2, 28, 28, 128, 128),
    (3, 5, 7, 64, 256),
    (1, 3, 130, 32, 128),
    (11, 6, 6, 128, 128),
    (2, 30, 28, 128, 128),
    (5, 3, 5, 64, 128),
    (4, 13, 21, 96, 384),
]


@pytest.mark.parametrize("shape", SMALL_3X3, ids=[str(s) for s in SMALL_3X3])
def test_conv3x3_parity(oracle, shape):
    s = synth.ConvShape(*shape, R=3, has_res=False)
    inp = synth.conv_inputs(s, seed=hash(shape) & 0xFFFF)
    ref = oracle.pack_act(_oracle_conv(oracle, inp))
    got = _gpu_conv(inp)
    assert torch.equal(got, ref), (got != ref).sum().item()


# The 128 -> 128 3x3 runs on CTA pairs (each CTA holds half the weights):
# several images per tile, a ragged last row of tiles, an odd tile count (the
# second CTA of the last pair has no tile), unswizzled output rows (W = 14),
# wide rows (two image rows per tile) and a single pixel.
PAIR_3X3 = [(11, 6, 6), (2, 30, 28), (3, 9, 12), (4, 14, 14), (5, 56, 56), (1, 1, 1), (7, 28, 28)]


@pytest.mark.parametrize("shape", PAIR_3X3, ids=[str(s) for s in PAIR_3X3])
def test_conv3x3_on_cta_pairs(oracle, shape):
    B, H, W = shape
    assert " pair=1 " in X.x1cb_describe_plan(B, H, W, 128, 128, 3, False)
    s = synth.ConvShape(B, H, W, 128, 128, R=3, has_res=False)
    inp = synth.conv_inputs(s, seed=500 + B * H + W)
    ref = oracle.pack_act(_oracle_conv(oracle, inp))
    got = _gpu_conv(inp)
    assert torch.equal(got, ref), (got != ref).sum().item()


@pytest.mark.parametrize("S", [12, 33])
def test_conv3x3_on_cta_pairs_full_int8_range(oracle, S):
    """Full-range operands and wide biases and multipliers at two shifts (the
    pair kernel picks its exact form from them at run time)."""
    s = synth.ConvShape(3, 9, 12, 128, 128, 3, False)
    inp = synth.full_range_conv_inputs(s, 17 + S, S=S)
    ref = oracle.pack_act(_oracle_conv(oracle, inp))
    got = _gpu_conv(inp)
    assert torch.equal(got, ref), (got != ref).sum().item()


def test_conv3x3_full_int8_range(oracle):
    s = synth.ConvShape(2, 9, 11, 64, 128, 3, False)
    inp = synth.full_range_conv_inputs(s, 7, S=33)
    ref = oracle.pack_act(_oracle_conv(oracle, inp))
    got = _gpu_conv(inp)
    assert torch.equal(got, ref)


def test_centre_tap_3x3_equals_1x1():
    s = synth.ConvShape(3, 10, 12, 64, 128, 1, False)
    inp = synth.conv_inputs(s, 5)
    w3 = torch.zeros(128, 64, 3, 3, dtype=torch.int8)
    w3[:, :, 1, 1] = inp.w[:, :, 0, 0]
    a = _gpu_conv(inp)
    inp3 = synth.ConvInputs(synth.ConvShape(3, 10, 12, 64, 128, 3, False), inp.x, w3, inp.bias,
                            inp.m, None, 0, inp.S)
    assert torch.equal(a, _gpu_conv(inp3))


# ---- bottleneck block -------------------------------------------------------------

@pytest.mark.parametrize("shape", [(2, 28, 28, 512, 128), (1, 6, 5, 256, 128), (3, 9, 4, 384, 128)])
def test_bottleneck_parity(oracle, shape):
    s = synth.BlockShape(*shape)
    inp = synth.block_inputs(s, seed=31)
    ref = oracle.pack_act(oracle.bottleneck(inp.x, inp.w, inp.bias, inp.m, inp.m_r, inp.S))
    x = X.x1cb_pack_act(inp.x.to(DEV))
    ws = [X.x1cb_pack_weight(w.to(DEV)) for w in inp.w]
    bs = [b.to(DEV) for b in inp.bias]
    ms = [m.to(DEV) for m in inp.m]
    out = X.bottleneck_i8(x, ws[0], bs[0], ms[0], ws[1], bs[1], ms[1], ws[2], bs[2], ms[2],
                          inp.m_r, inp.S)
    torch.cuda.synchronize()
    assert torch.equal(out.cpu(), ref)
    _assert_spread(ref)


# ---- full-size workloads, every output byte -------------------------------------

def _sample_pixels(B, H, W, n, seed):
    g = torch.Generator().manual_seed(seed)
    P = B * H * W
    pix = torch.randint(0, P, (n,), generator=g)
    edges = torch.tensor([0, W - 1, (H - 1) * W, H * W - 1, P - 1, P - H * W, P // 2])
    return torch.unique(torch.cat([pix, edges.clamp(0, P - 1)]))


def _gather_nc32(t_nc32_cpu, pix, H, W):
    """Rows [n, C] of a packed [B, C/32, H, W, 32] tensor at flattened pixels."""
    B, C1 = t_nc32_cpu.shape[:2]
    flat = t_nc32_cpu.permute(0, 2, 3, 1, 4).reshape(B * H * W, C1 * 32)
    return flat[pix]


def _nhwc(t_nc32_cpu):
    """[B, C/32, H, W, 32] -> [B, H, W, C] (a layout view, no arithmetic)."""
    B, C1, H, W, _ = t_nc32_cpu.shape
    return t_nc32_cpu.permute(0, 2, 3, 1, 4).reshape(B, H, W, C1 * 32)


def _first_mismatch(got, ref):
    bad = (got != ref).nonzero()
    return f"{bad.shape[0]} bytes differ, first at {bad[0].tolist()}" if bad.numel() else ""


@pytest.mark.parametrize("cfg", ["1", "2", "3", "4a", "4b", "4c"])
def test_full_size_1x1_every_output(oracle, cfg):
    """The benchmark workloads at full size, compared byte for byte with the
    whole oracle output (B=2048: 822 MB of results, 12544 tiles over the
    persistent grid, including the last partial wave)."""
    s = synth.CONFIGS[cfg]
    inp = synth.conv_inputs(s, synth.CONFIG_SEEDS[cfg])
    got = _nhwc(_gpu_conv(inp))
    ref = _oracle_conv(oracle, inp)
    assert torch.equal(got, ref), _first_mismatch(got, ref)
    _assert_spread(ref)


# ---- many launches back to back -----------------------------------------------------
# The kernel's warps hand ring slots and accumulators to one another through
# mbarrier phases; an ordering mistake there shows up only now and then, as a
# wait that runs out (device status) or as a launch that differs from the rest.

STRESS = [
    (256, 28, 28, 128, 512, 1, True),   # Res3.2 Conv3 (I/O ring of 7 stages)
    (96, 28, 28, 512, 128, 1, False),   # Res3.2 conv1 (3 stages)
    (96, 28, 28, 128, 128, 3, False),   # Res3.2 conv2 on CTA pairs (4 stages)
    (96, 28, 28, 64, 128, 3, False),    # a 3x3 of one CTA, halo form (2 stages)
]


@pytest.mark.parametrize("shape", STRESS, ids=[str(s) for s in STRESS])
def test_repeated_launches_stay_exact(oracle, shape):
    s = synth.ConvShape(*shape)
    inp = synth.conv_inputs(s, 91)
    x = X.x1cb_pack_act(inp.x.to(DEV))
    w = X.x1cb_pack_weight(inp.w.to(DEV))
    bias, m = inp.bias.to(DEV), inp.m.to(DEV)
    r = X.x1cb_pack_act(inp.r.to(DEV)) if s.has_res else None
    X.x1cb_last_device_error(clear=True)
    outs = []
    for i in range(300):
        if s.R == 1:
            out = X.conv1x1_bn_add_relu_i8(x, w, bias, m, inp.m_r, inp.S, r)
        else:
            out = X.conv3x3_bn_relu_i8(x, w, bias, m, inp.S)
        if i % 50 == 0 or i == 299:
            outs.append(out)
    torch.cuda.synchronize()
    st, bits = X.x1cb_last_device_error(clear=True)
    assert st == 0 and bits == 0, bits
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    pix = _sample_pixels(s.B, s.H, s.W, 600, 3)
    ref = oracle.conv_pixels(inp.x, inp.w, inp.bias, inp.m, inp.S, pix, inp.r, inp.m_r)
    assert torch.equal(_gather_nc32(outs[0].cpu(), pix, s.H, s.W), ref)


def test_full_size_block_every_output(oracle):
    """The Res3.2 bottleneck block at B=1024, every output byte against the
    oracle's three composed layers."""
    s = synth.CONFIGS["5"]
    inp = synth.block_inputs(s, synth.CONFIG_SEEDS["5"])
    x = X.x1cb_pack_act(inp.x.to(DEV))
    ws = [X.x1cb_pack_weight(w.to(DEV)) for w in inp.w]
    bs = [b.to(DEV) for b in inp.bias]
    ms = [m.to(DEV) for m in inp.m]
    X.x1cb_last_device_error(clear=True)
    out = X.bottleneck_i8(x, ws[0], bs[0], ms[0], ws[1], bs[1], ms[1], ws[2], bs[2], ms[2],
                          inp.m_r, inp.S)
    torch.cuda.synchronize()
    st, bits = X.x1cb_last_device_error(clear=True)
    assert st == 0, bits
    got = _nhwc(out.cpu())
    del out, x
    ref = oracle.bottleneck(inp.x, inp.w, inp.bias, inp.m, inp.m_r, inp.S)
    assert torch.equal(got, ref), _first_mismatch(got, ref)
    _assert_spread(ref)


# ---- safety properties ----------------------------------------------------------------

def test_guard_bands_untouched():
    s = synth.ConvShape(3, 7, 9, 64, 256, 1, True)
    inp = synth.conv_inputs(s, 3)
    x = X.x1cb_pack_act(inp.x.to(DEV))
    w = X.x1cb_pack_weight(inp.w.to(DEV))
    r = X.x1cb_pack_act(inp.r.to(DEV))
    n = s.pixels * s.Oc
    pad = 4096
    buf = torch.full((n + 2 * pad,), 0x5A, dtype=torch.int8, device=DEV)
    out = buf[pad:pad + n].view(s.B, s.Oc // 32, s.H, s.W, 32)
    X.conv1x1_bn_add_relu_i8(x, w, inp.bias.to(DEV), inp.m.to(DEV), inp.m_r, inp.S, r, out=out)
    torch.cuda.synchronize()
    assert (buf[:pad] == 0x5A).all() and (buf[pad + n:] == 0x5A).all()


def test_repeatable_and_stream_ordered(oracle):
    s = synth.ConvShape(16, 28, 28, 128, 512, 1, True)
    inp = synth.conv_inputs(s, 12)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        a = _gpu_conv(inp)
        b = _gpu_conv(inp)
    assert torch.equal(a, b)


def test_bounded_wait_reports_timeout_and_context_survives(oracle):
    """A wait that nothing satisfies (test hook) runs out after 50 ms; the
    kernel returns, the status word says timeout, and the next call is exact."""
    s = synth.ConvShape(4, 28, 28, 128, 512, 1, True)
    inp = synth.conv_inputs(s, 44)
    x = X.x1cb_pack_act(inp.x.to(DEV))
    w = X.x1cb_pack_weight(inp.w.to(DEV))
    r = X.x1cb_pack_act(inp.r.to(DEV))
    bias, m = inp.bias.to(DEV), inp.m.to(DEV)
    X.x1cb_last_device_error(clear=True)
    try:
        X.x1cb_set_wait_limit_ns(50_000_000)
        X.x1cb_debug_inject(1)
        X.conv1x1_bn_add_relu_i8(x, w, bias, m, inp.m_r, inp.S, r)
        st, bits = X.x1cb_last_device_error(clear=True)
    finally:
        X.x1cb_debug_inject(0)
        X.x1cb_set_wait_limit_ns(0)
    assert st == X.X1CB_ERR_TIMEOUT
    assert bits & 2  # the MMA warp's wait ran out
    assert not bits & 8  # every copy in flight landed before exit
    out = X.conv1x1_bn_add_relu_i8(x, w, bias, m, inp.m_r, inp.S, r)
    torch.cuda.synchronize()
    assert X.x1cb_last_device_error(clear=True)[0] == 0
    assert torch.equal(out.cpu(), oracle.pack_act(_oracle_conv(oracle, inp)))


def test_empty_batch_is_noop():
    x = torch.empty((0, 4, 28, 28, 32), dtype=torch.int8, device=DEV)
    w = torch.zeros((4, 4, 128, 32), dtype=torch.int8, device=DEV)
    b = torch.zeros(512, dtype=torch.int32, device=DEV)
    out = X.conv1x1_bn_add_relu_i8(x, w, b, b, 0, 24, None)
    assert out.shape == (0, 16, 28, 28, 32)


def test_two_threads_on_one_device_stay_exact(oracle):
    """Two host threads call the library at once, each on its own stream, on
    shapes whose plans differ (the plan cache and the per-device kernel set-up
    are shared); both results stay bit-exact."""
    import threading

    cases = [synth.conv_inputs(synth.ConvShape(8, 28, 28, 128, 512, 1, True), 61),
             synth.conv_inputs(synth.ConvShape(6, 14, 14, 256, 1024, 1, True), 62),
             synth.conv_inputs(synth.ConvShape(5, 28, 28, 128, 128, 3, False), 63)]
    refs = [_oracle_conv(oracle, c) for c in cases]
    got = [[None] * 20 for _ in cases]
    errors = []

    def worker(i):
        try:
            torch.cuda.set_device(0)
            c = cases[i]
            st = torch.cuda.Stream()
            with torch.cuda.stream(st):
                x = X.x1cb_pack_act(c.x.to(DEV))
                w = X.x1cb_pack_weight(c.w.to(DEV))
                b, m = c.bias.to(DEV), c.m.to(DEV)
                r = X.x1cb_pack_act(c.r.to(DEV)) if c.r is not None else None
                for j in range(20):
                    if c.shape.R == 1:
                        got[i][j] = X.conv1x1_bn_add_relu_i8(x, w, b, m, c.m_r, c.S, r)
                    else:
                        got[i][j] = X.conv3x3_bn_relu_i8(x, w, b, m, c.S)
            st.synchronize()
        except Exception as e:  # reported on the main thread
            errors.append(e)

    ts = [threading.Thread(target=worker, args=(i,)) for i in range(len(cases))]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not errors, errors
    torch.cuda.synchronize()
    assert X.x1cb_last_device_error(clear=True)[0] == 0
    for i, ref in enumerate(refs):
        for o in got[i]:
            assert torch.equal(_nhwc(o.cpu()), ref)


def test_operands_must_be_memory_of_the_current_device():
    """Host memory handed to the C ABI is refused before anything launches."""
    import ctypes

    s = synth.ConvShape(1, 4, 4, 32, 128, 1, False)
    inp = synth.conv_inputs(s, 5)
    x = X.x1cb_pack_act(inp.x.to(DEV))
    w = X.x1cb_pack_weight(inp.w.to(DEV))
    b, m = inp.bias.to(DEV), inp.m.to(DEV)
    out = torch.empty((1, 4, 4, 4, 32), dtype=torch.int8, device=DEV)
    host = torch.empty_like(out, device="cpu").pin_memory()
    v = ctypes.c_void_p
    L = X.lib()
    args = lambda xp, op: (v(xp), v(w.data_ptr()), v(b.data_ptr()), v(m.data_ptr()), 0, 24,
                           None, v(op), 1, 4, 4, 32, 128, None)
    assert L.conv1x1_bn_add_relu_i8(*args(x.data_ptr(), host.data_ptr())) == X.X1CB_ERR_DEVICE
    hx = x.cpu().pin_memory()
    assert L.conv1x1_bn_add_relu_i8(*args(hx.data_ptr(), out.data_ptr())) == X.X1CB_ERR_DEVICE
    assert L.conv1x1_bn_add_relu_i8(*args(x.data_ptr(), out.data_ptr())) == X.X1CB_OK
    torch.cuda.synchronize()
    with pytest.raises(ValueError):
        X.conv1x1_bn_add_relu_i8(x, w.cpu(), b, m, 0, 24)
