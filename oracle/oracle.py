"""ctypes wrapper and build step for the plain C oracle (x1cb_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg use this module; the library never does.  It shares no code with
the CUDA path.  Inputs are torch CPU tensors in logical layouts (NHWC
activations, OIHW weights); results come back as NHWC int8 tensors.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "x1cb_oracle.c")
_LIB = os.path.join(_HERE, "libx1cb_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP over output rows)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-o", _LIB, _SRC]
        subprocess.check_call(cmd)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        c_i8p = ctypes.c_void_p
        L.x1o_requant.restype = ctypes.c_int8
        L.x1o_requant.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int,
                                  ctypes.c_int32, ctypes.c_int32, ctypes.c_int]
        for name in ("x1o_pack_act", "x1o_unpack_act"):
            getattr(L, name).argtypes = [c_i8p, c_i8p] + [ctypes.c_int] * 4
        for name in ("x1o_pack_weight", "x1o_unpack_weight"):
            getattr(L, name).argtypes = [c_i8p, c_i8p] + [ctypes.c_int] * 3
        L.x1o_conv.argtypes = ([c_i8p] * 4 + [ctypes.c_int, c_i8p, ctypes.c_int32, c_i8p]
                               + [ctypes.c_int] * 7)
        L.x1o_conv_pixels.argtypes = ([c_i8p] * 4 + [ctypes.c_int, c_i8p, ctypes.c_int32, c_i8p,
                                       ctypes.c_int64, c_i8p] + [ctypes.c_int] * 7)
        L.x1o_bottleneck.argtypes = ([c_i8p] * 10 + [ctypes.c_int32, ctypes.c_int, c_i8p]
                                     + [ctypes.c_int] * 5)
        L.x1o_bottleneck_pixels.argtypes = ([c_i8p] * 10 + [ctypes.c_int32, ctypes.c_int, c_i8p,
                                             ctypes.c_int64, c_i8p] + [ctypes.c_int] * 5)
        L.x1o_conv_strided.argtypes = ([c_i8p] * 4 + [ctypes.c_int, c_i8p, ctypes.c_int32, c_i8p]
                                       + [ctypes.c_int] * 8)
        L.x1o_conv_proj.argtypes = [c_i8p] * 6 + [ctypes.c_int, c_i8p] + [ctypes.c_int] * 9
        L.x1o_bottleneck_proj.argtypes = [c_i8p] * 11 + [ctypes.c_int, c_i8p] + [ctypes.c_int] * 6
        L.x1o_maxpool3s2.argtypes = [c_i8p, c_i8p] + [ctypes.c_int] * 4
        L.x1o_conv_pool.argtypes = [c_i8p] * 4 + [ctypes.c_int, c_i8p] + [ctypes.c_int] * 8
        L.x1o_set_threads.argtypes = [ctypes.c_int]
        L.x1o_set_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(t):
    if t is None:
        return None
    assert t.device.type == "cpu" and t.is_contiguous()
    return ctypes.c_void_p(t.data_ptr())


def _cpu(t, dtype):
    return None if t is None else t.detach().to("cpu", dtype).contiguous()


def set_threads(n: int = 0) -> int:
    """Set the OpenMP thread count (0 keeps the current one); returns it."""
    return lib().x1o_set_threads(n)


def requant(acc: int, bias: int, m: int, r: int | None, m_r: int, S: int) -> int:
    return int(lib().x1o_requant(acc, bias, m, int(r is not None), 0 if r is None else r, m_r, S))


def pack_act(nhwc: torch.Tensor) -> torch.Tensor:
    B, H, W, C = nhwc.shape
    x = _cpu(nhwc, torch.int8)
    out = torch.empty((B, C // 32, H, W, 32), dtype=torch.int8)
    lib().x1o_pack_act(_p(x), _p(out), B, H, W, C)
    return out


def unpack_act(nc32: torch.Tensor) -> torch.Tensor:
    B, C1, H, W, _ = nc32.shape
    x = _cpu(nc32, torch.int8)
    out = torch.empty((B, H, W, C1 * 32), dtype=torch.int8)
    lib().x1o_unpack_act(_p(x), _p(out), B, H, W, C1 * 32)
    return out


def pack_weight(oihw: torch.Tensor) -> torch.Tensor:
    Oc, Ic, R, _ = oihw.shape
    w = _cpu(oihw, torch.int8)
    O2 = min(Oc, 128)
    out = torch.empty((Oc // O2, R, R, Ic // 32, O2, 32), dtype=torch.int8)
    lib().x1o_pack_weight(_p(w), _p(out), Oc, Ic, R)
    return out


def unpack_weight(blk: torch.Tensor, Oc: int, Ic: int, R: int) -> torch.Tensor:
    w = _cpu(blk, torch.int8)
    out = torch.empty((Oc, Ic, R, R), dtype=torch.int8)
    lib().x1o_unpack_weight(_p(w), _p(out), Oc, Ic, R)
    return out


def conv(x, w, bias, m, S, r=None, m_r=0, pad=None):
    """Fused conv + BN (+ residual Sum) + ReLU + requant.  NHWC in, NHWC out."""
    B, H, W, Ic = x.shape
    Oc, Ic2, R, _ = w.shape
    assert Ic2 == Ic
    pad = (R - 1) // 2 if pad is None else pad
    x, w = _cpu(x, torch.int8), _cpu(w, torch.int8)
    bias, m = _cpu(bias, torch.int32), _cpu(m, torch.int32)
    r = _cpu(r, torch.int8)
    out = torch.empty((B, H, W, Oc), dtype=torch.int8)
    lib().x1o_conv(_p(x), _p(w), _p(bias), _p(m), S, _p(r), int(m_r), _p(out),
                   B, H, W, Ic, Oc, R, pad)
    return out


def conv_pixels(x, w, bias, m, S, pix, r=None, m_r=0, pad=None):
    """The fused conv at chosen flattened pixels (b*H + h)*W + w -> [n, Oc]."""
    B, H, W, Ic = x.shape
    Oc, _, R, _ = w.shape
    pad = (R - 1) // 2 if pad is None else pad
    x, w = _cpu(x, torch.int8), _cpu(w, torch.int8)
    bias, m = _cpu(bias, torch.int32), _cpu(m, torch.int32)
    r = _cpu(r, torch.int8)
    pix = _cpu(torch.as_tensor(pix), torch.int64)
    out = torch.empty((pix.numel(), Oc), dtype=torch.int8)
    lib().x1o_conv_pixels(_p(x), _p(w), _p(bias), _p(m), S, _p(r), int(m_r), _p(pix),
                          pix.numel(), _p(out), B, H, W, Ic, Oc, R, pad)
    return out


def bottleneck(x, ws, bs, ms, m_r, S):
    B, H, W, Cin = x.shape
    Cmid = ws[0].shape[0]
    args = [_cpu(x, torch.int8)]
    for w, b, m in zip(ws, bs, ms):
        args += [_cpu(w, torch.int8), _cpu(b, torch.int32), _cpu(m, torch.int32)]
    out = torch.empty((B, H, W, Cin), dtype=torch.int8)
    lib().x1o_bottleneck(*[_p(a) for a in args], int(m_r), S, _p(out), B, H, W, Cin, Cmid)
    return out


def bottleneck_pixels(x, ws, bs, ms, m_r, S, pix):
    B, H, W, Cin = x.shape
    Cmid = ws[0].shape[0]
    args = [_cpu(x, torch.int8)]
    for w, b, m in zip(ws, bs, ms):
        args += [_cpu(w, torch.int8), _cpu(b, torch.int32), _cpu(m, torch.int32)]
    pix = _cpu(torch.as_tensor(pix), torch.int64)
    out = torch.empty((pix.numel(), Cin), dtype=torch.int8)
    lib().x1o_bottleneck_pixels(*[_p(a) for a in args], int(m_r), S, _p(pix), pix.numel(),
                                _p(out), B, H, W, Cin, Cmid)
    return out


def out_extent(n: int, R: int, pad: int, stride: int) -> int:
    return (n + 2 * pad - R) // stride + 1


def conv_strided(x, w, bias, m, S, stride, r=None, m_r=0, pad=None):
    """Fused conv of any stride + BN (+ residual) + ReLU + requant.  NHWC in,
    NHWC out of (H + 2 pad - R) / stride + 1 rows and columns."""
    B, H, W, Ic = x.shape
    Oc, _, R, _ = w.shape
    pad = (R - 1) // 2 if pad is None else pad
    Ho, Wo = out_extent(H, R, pad, stride), out_extent(W, R, pad, stride)
    x, w = _cpu(x, torch.int8), _cpu(w, torch.int8)
    bias, m = _cpu(bias, torch.int32), _cpu(m, torch.int32)
    r = _cpu(r, torch.int8)
    out = torch.empty((B, Ho, Wo, Oc), dtype=torch.int8)
    lib().x1o_conv_strided(_p(x), _p(w), _p(bias), _p(m), S, _p(r), int(m_r), _p(out),
                           B, H, W, Ic, Oc, R, pad, stride)
    return out


def conv_proj(y, w3, x, wp, bias, m, S, stride=2):
    """Projection block's Conv3: 1x1 of y plus the stride-`stride` 1x1 of x in
    one accumulator, + BN + ReLU + requant.  y [B,H,W,Cy], x [B,Hx,Wx,Cx]."""
    B, H, W, Cy = y.shape
    _, Hx, Wx, Cx = x.shape
    Oc = w3.shape[0]
    y, x = _cpu(y, torch.int8), _cpu(x, torch.int8)
    w3, wp = _cpu(w3, torch.int8), _cpu(wp, torch.int8)
    bias, m = _cpu(bias, torch.int32), _cpu(m, torch.int32)
    out = torch.empty((B, H, W, Oc), dtype=torch.int8)
    lib().x1o_conv_proj(_p(y), _p(w3), _p(x), _p(wp), _p(bias), _p(m), S, _p(out),
                        B, H, W, Cy, Cx, Oc, Hx, Wx, stride)
    return out


def bottleneck_proj(x, ws, wp, bs, ms, S):
    """Res3.1 projection block.  ws = (w1, w2, w3) OIHW, wp the projection
    weight [Cout, Cin, 1, 1]; bs, ms the three layers' bias and multiplier
    (the third shared by Conv3 and the projection)."""
    B, H, W, Cin = x.shape
    Cmid, Cout = ws[0].shape[0], ws[2].shape[0]
    Ho, Wo = out_extent(H, 3, 1, 2), out_extent(W, 3, 1, 2)
    args = [_cpu(x, torch.int8)]
    for w, b, mm in zip(ws[:2], bs[:2], ms[:2]):
        args += [_cpu(w, torch.int8), _cpu(b, torch.int32), _cpu(mm, torch.int32)]
    args += [_cpu(ws[2], torch.int8), _cpu(wp, torch.int8), _cpu(bs[2], torch.int32),
             _cpu(ms[2], torch.int32)]
    out = torch.empty((B, Ho, Wo, Cout), dtype=torch.int8)
    lib().x1o_bottleneck_proj(*[_p(a) for a in args], S, _p(out), B, H, W, Cin, Cmid, Cout)
    return out


def maxpool3s2(y):
    """3x3 stride-2 max pooling (pad 1, padding never wins).  NHWC in and out."""
    B, H, W, C = y.shape
    y = _cpu(y, torch.int8)
    out = torch.empty((B, out_extent(H, 3, 1, 2), out_extent(W, 3, 1, 2), C), dtype=torch.int8)
    lib().x1o_maxpool3s2(_p(y), _p(out), B, H, W, C)
    return out


def conv_pool(x, w, bias, m, S, stride=2, pad=None):
    """Stem: conv (R x R, pad (R-1)/2, stride) + BN + ReLU, then 3x3 stride-2
    max pooling.  NHWC in and out."""
    B, H, W, Ic = x.shape
    Oc, _, R, _ = w.shape
    pad = (R - 1) // 2 if pad is None else pad
    Hc, Wc = out_extent(H, R, pad, stride), out_extent(W, R, pad, stride)
    x, w = _cpu(x, torch.int8), _cpu(w, torch.int8)
    bias, m = _cpu(bias, torch.int32), _cpu(m, torch.int32)
    out = torch.empty((B, out_extent(Hc, 3, 1, 2), out_extent(Wc, 3, 1, 2), Oc),
                      dtype=torch.int8)
    lib().x1o_conv_pool(_p(x), _p(w), _p(bias), _p(m), S, _p(out), B, H, W, Ic, Oc, R, pad,
                        stride)
    return out
