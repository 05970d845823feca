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
    for code in range(-8, 0):
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
    assert L.x1cb_pack_weight(v(P), v(2 * P), 128, 32, 5, None) == X.X1CB_ERR_SHAPE
    assert L.x1cb_pack_weight(v(P), v(P), 128, 32, 1, None) == X.X1CB_ERR_OVERLAP


@pytest.mark.parametrize("shape,expect", [
    ((2048, 28, 28, 128, 512, 1, 1), "tile=16x1x8 rows=128 m_tiles=12544 NC=512"),
    ((1, 28, 28, 128, 512, 1, 1), "rows=128 m_tiles=7 NC=128 groups=4"),
    ((1024, 28, 28, 128, 128, 3, 0), "NC=128"),
])
def test_plans(L, shape, expect):
    assert expect in X.x1cb_describe_plan(*shape)


def test_plan_rejects_weights_that_do_not_fit(L):
    with pytest.raises(X.X1cbError):
        X.x1cb_describe_plan(8, 14, 14, 1024, 256, 3, 0)
