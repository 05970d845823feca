"""The C ABI loads, exports every function include/x1cb.h declares, and its
host-side argument checks reject bad calls before touching any device.  No
call here launches work: pointers are fake, aligned addresses that are never
dereferenced because validation fails (or the problem is empty) first."""
import ctypes

import pytest

import x1_conv_bn_b200 as X


@pytest.fixture(scope="module")
def L():
    from x1_conv_bn_b200 import _build

    _build.build()
    return X.lib()


def test_header_declares_the_boundary():
    names = X.header_functions()
    for n in ["conv1x1_bn_add_relu_i8", "conv3x3_bn_relu_i8", "bottleneck_i8",
              "bottleneck_i8_workspace_size", "x1cb_pack_act", "x1cb_unpack_act",
              "x1cb_pack_weight", "x1cb_status_string", "x1cb_last_device_error"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    missing = [n for n in X.header_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_python_binding_has_same_names(L):
    for n in X.header_functions():
        assert callable(getattr(X, n)), n


def test_status_strings(L):
    assert X.x1cb_status_string(0) == "ok"
    for code in range(-9, 0):
        assert X.x1cb_status_string(code) != "unknown status"
    assert "sm_100a" in X.x1cb_version()


P = 1 << 20  # fake 16-byte aligned "device" addresses, never dereferenced


def _conv(L, x=P, w=2 * P, bias=3 * P, m=4 * P, r=5 * P, out=6 * P, B=2, H=28, W=28, Ic=128,
          Oc=512, S=24):
    v = ctypes.c_void_p
    return L.conv1x1_bn_add_relu_i8(v(x), v(w), v(bias), v(m), 1 << 23, S,
                                    v(r) if r else None, v(out), B, H, W, Ic, Oc, None)


def test_conv1x1_argument_checks(L):
    big = 1 << 34  # far apart so nothing overlaps
    kw = dict(x=big, w=2 * big, bias=3 * big, m=4 * big, r=5 * big, out=6 * big)
    assert _conv(L, **{**kw, "x": 0}) == X.X1CB_ERR_NULL
    assert _conv(L, **{**kw, "out": 0}) == X.X1CB_ERR_NULL
    assert _conv(L, **kw, Ic=48) == X.X1CB_ERR_SHAPE
    assert _conv(L, **kw, Ic=0) == X.X1CB_ERR_SHAPE
    assert _conv(L, **kw, Oc=192) == X.X1CB_ERR_SHAPE
    assert _conv(L, **kw, S=0) == X.X1CB_ERR_SHAPE
    assert _conv(L, **kw, S=61) == X.X1CB_ERR_SHAPE
    assert _conv(L, **kw, B=-1) == X.X1CB_ERR_SHAPE
    assert _conv(L, **{**kw, "x": big + 8}) == X.X1CB_ERR_ALIGN
    assert _conv(L, **{**kw, "r": 5 * big + 4}) == X.X1CB_ERR_ALIGN
    # output overlapping the input or the shortcut
    assert _conv(L, **{**kw, "out": big}) == X.X1CB_ERR_OVERLAP
    assert _conv(L, **{**kw, "out": 5 * big + 4096}) == X.X1CB_ERR_OVERLAP
    # empty problems are a no-op that succeeds without a device
    assert _conv(L, **kw, B=0) == X.X1CB_OK
    assert _conv(L, **kw, H=0) == X.X1CB_OK


def test_conv3x3_and_block_argument_checks(L):
    v = ctypes.c_void_p
    big = 1 << 34
    assert L.conv3x3_bn_relu_i8(v(big), v(2 * big), v(3 * big), v(4 * big), 24, v(6 * big),
                                2, 28, 28, 128, 128, 0, None) == X.X1CB_ERR_SHAPE  # pad != 1
    assert L.conv3x3_bn_relu_i8(v(big), v(2 * big), v(3 * big), v(4 * big), 24, v(6 * big),
                                0, 28, 28, 128, 128, 1, None) == X.X1CB_OK
    ws = L.bottleneck_i8_workspace_size(4, 28, 28, 128)
    assert ws >= 2 * 4 * 28 * 28 * 128
    args = [v((k + 1) * big) for k in range(10)]
    # workspace too small
    assert L.bottleneck_i8(*args, 1 << 23, 24, v(20 * big), v(30 * big), ws - 1,
                           4, 28, 28, 512, 128, None) == X.X1CB_ERR_WORKSPACE
    assert L.bottleneck_i8(*args, 1 << 23, 24, v(20 * big), None, 0,
                           4, 28, 28, 512, 128, None) == X.X1CB_ERR_WORKSPACE
    # out == x
    assert L.bottleneck_i8(*args, 1 << 23, 24, args[0], v(30 * big), ws,
                           4, 28, 28, 512, 128, None) == X.X1CB_ERR_OVERLAP
    # Cmid not a multiple of 128
    assert L.bottleneck_i8(*args, 1 << 23, 24, v(20 * big), v(30 * big), ws,
                           4, 28, 28, 512, 96, None) == X.X1CB_ERR_SHAPE


def test_pack_argument_checks(L):
    v = ctypes.c_void_p
    assert L.x1cb_pack_act(None, v(P), 1, 2, 2, 32, None) == X.X1CB_ERR_NULL
    assert L.x1cb_pack_act(None, None, 0, 2, 2, 32, None) == X.X1CB_OK
    assert L.x1cb_pack_act(v(P), v(2 * P), 1, 2, 2, 40, None) == X.X1CB_ERR_SHAPE
    assert L.x1cb_pack_act(v(P + 1), v(2 * P), 1, 2, 2, 32, None) == X.X1CB_ERR_ALIGN
    assert L.x1cb_pack_weight(v(P), v(2 * P), 128, 32, 4, None) == X.X1CB_ERR_SHAPE
    assert L.x1cb_pack_weight(v(P), v(2 * P), 192, 32, 3, None) == X.X1CB_ERR_SHAPE
    assert L.x1cb_pack_weight(v(P), v(P), 128, 32, 1, None) == X.X1CB_ERR_OVERLAP


@pytest.mark.parametrize("shape,expect", [
    ((2048, 28, 28, 128, 512, 1, 1), "tile=16x1x8 rows=128 m_tiles=12544 NC=512"),
    ((1, 28, 28, 128, 512, 1, 1), "rows=128 m_tiles=7 NC=128 groups=4"),
    ((1024, 28, 28, 128, 128, 3, 0), "NC=128"),
])
def test_plans(L, shape, expect):
    assert expect in X.x1cb_describe_plan(*shape)


def _plan(shape):
    return dict(kv.split("=") for kv in X.x1cb_describe_plan(*shape).split())


@pytest.mark.parametrize("B,Ic,R,res", [(1, 128, 1, 1), (1024, 128, 1, 1), (2048, 256, 1, 0),
                                        (512, 128, 3, 0), (64, 512, 1, 1)])
def test_channel_groups_are_whole_mmas(L, B, Ic, R, res):
    """Every output width (multiples of 128): a CTA's NC channels are n_subs
    whole MMAs of nmma columns, and the groups tile Oc exactly (a 384-channel
    group of one 256-column MMA would leave a third uncomputed)."""
    for Oc in range(128, 2049, 128):
        p = _plan((B, 28, 28, Ic, Oc, R, res))
        NC, nmma, subs, groups = (int(p[k]) for k in ("NC", "nmma", "subs", "groups"))
        assert nmma * subs == NC and NC * groups == Oc, (Oc, p)


def test_large_resident_weights_take_whole_boxes_and_cta_pairs(L):
    """7x7 512 -> 2048 expand conv with shortcut (B = 512): 128 KB of weights
    per 256-channel group.  The tile's rows are a multiple of 8 so that each
    activation box carries four K blocks, and the layer runs on CTA pairs
    (64 KB of weights each) with four 16 KB shortcut/result stages; a layer
    whose group is not one N = 256 MMA (1024 -> 256: N = 128 groups) stages
    the shortcut in 8 KB pieces instead."""
    p = _plan((512, 7, 7, 512, 2048, 1, 1))
    assert int(p["rows"]) % 8 == 0 and p["kc"] == "4", p
    assert p["cta_pair"] == "1" and int(p["grid"]) % 2 == 0, p
    assert p["stage_ch"] == "4" and int(p["r_stages"]) >= 4 and int(p["a_stages"]) >= 5, p
    q = _plan((9, 7, 7, 1024, 256, 1, 1))
    assert q["cta_pair"] == "0" and q["stage_ch"] == "2" and int(q["r_stages"]) >= 4, q
    # the Res3.2 conv3 (64 KB of weights) keeps 16 KB stages, six of them
    q = _plan((2048, 28, 28, 128, 512, 1, 1))
    assert q["stage_ch"] == "4" and int(q["r_stages"]) >= 6, q


@pytest.mark.parametrize("shape,tile", [
    ((1024, 28, 28, 128, 128, 3, 0), "28x4x1"),   # Res3.2 conv2: 4 rows + frame = 120 GEMM rows
    ((2, 30, 28, 128, 128, 3, 0), "28x4x1"),      # ragged in H: 8 tiles per image, last one 2 rows
    ((5, 3, 5, 64, 128, 3, 0), "5x3x3"),          # three framed images in one tile
    ((11, 6, 6, 128, 128, 3, 0), "6x6x2"),
    ((1, 1, 1, 32, 128, 3, 0), "1x1x1"),
])
def test_halo_tiles(L, shape, tile):
    """3x3 with W+2 <= 128 uses the halo form: every pixel of the tile lands in
    the 128 GEMM rows, m = (g*(th+2) + y)*(W+2) + x."""
    p = _plan(shape)
    assert p["halo"] == "1" and p["tile"] == tile and p["kc"] == "1"
    tw, th, tg = (int(v) for v in tile.split("x"))
    W = shape[2]
    assert tw == W
    assert (tg - 1) * (th + 2) * (W + 2) + (th - 1) * (W + 2) + (W - 1) < 128
    assert int(p["rows"]) == tw * th * tg


def test_wide_images_take_the_per_tap_form(L):
    p = _plan((1, 3, 130, 32, 128, 3, 0))
    assert p["halo"] == "0"


@pytest.mark.parametrize("shape,swz", [
    ((2048, 28, 28, 128, 512, 1, 1), "1"),    # tw 16, row length 784
    ((512, 56, 56, 64, 256, 1, 1), "1"),
    ((1024, 28, 28, 128, 128, 3, 0), "1"),    # halo tile 28 wide
    ((512, 14, 14, 256, 1024, 1, 1), "1"),    # 16-pixel tiles of the 196-pixel image rows
    ((512, 7, 7, 512, 2048, 1, 1), "0"),      # 49-pixel rows: not whole 4-pixel groups
    ((17, 2, 3, 32, 384, 1, 1), "0"),
])
def test_swizzled_io_stages_only_for_whole_pixel_groups(L, shape, swz):
    p = _plan(shape)
    assert p["swz"] == swz
    if swz == "1":
        assert int(p["tile"].split("x")[0]) % 4 == 0


@pytest.mark.parametrize("shape", [(2048, 28, 28, 128, 512, 1, 1), (1024, 28, 28, 512, 128, 1, 0),
                                   (1024, 28, 28, 128, 128, 3, 0), (3, 14, 14, 256, 1024, 1, 1)])
def test_plans_fit_shared_memory(L, shape):
    p = _plan(shape)
    assert int(p["smem"]) <= 232448
    assert int(p["r_stages"]) >= (4 if shape[-1] else 2)
    assert int(p["a_stages"]) >= 2


def _stream(shape):
    return _plan(shape)["wstream"]


@pytest.mark.parametrize("R,res,max_ic", [(1, 1, 1120), (1, 0, 1376), (3, 0, 128)])
def test_weights_stay_resident_up_to_the_stated_fan_in(L, R, res, max_ic):
    """Up to these fan-ins the weights of 128 output channels stay resident in
    shared memory; beyond them they are streamed with the activations."""
    assert _stream((4, 28, 28, max_ic, 128, R, res)) == "0"
    assert _stream((4, 28, 28, max_ic + 32, 128, R, res)) == "1"


@pytest.mark.parametrize("shape", [(8, 14, 14, 1024, 256, 3, 0), (512, 7, 7, 512, 512, 3, 0),
                                   (4, 28, 28, 4096, 128, 1, 1), (2, 7, 7, 4096, 128, 3, 0)])
def test_large_fan_in_streams_weights(L, shape):
    p = _plan(shape)
    assert p["wstream"] == "1" and p["NC"] == "128" and p["subs"] == "1"
    assert int(p["smem"]) <= 232448 and int(p["a_stages"]) >= 2


def _header_param_counts():
    import re

    text = open(X.HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(\w+)\s*\(([^()]*)\)\s*;", text):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argtypes_match_the_header(L):
    """Every declared function's ctypes signature has as many arguments as
    its C declaration (a missing or extra one would shift every later
    argument)."""
    counts = _header_param_counts()
    assert len(counts) == len(X.header_functions())
    for name, n in counts.items():
        at = getattr(L, name).argtypes
        if at is None:  # argument-less helpers
            assert n == 0, name
        else:
            assert len(at) == n, (name, len(at), n)
