"""Python binding of the x1cb C ABI (include/x1cb.h).

Argument marshalling only: tensors become device pointers and sizes, the
current torch CUDA stream becomes the ``void *stream`` argument, and every
step of the computation runs in the library's CUDA kernels.  There is no
fallback: if libx1cb.so is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libx1cb.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "x1cb.h")

X1CB_OK = 0
X1CB_ERR_NULL = -1
X1CB_ERR_SHAPE = -2
X1CB_ERR_ALIGN = -3
X1CB_ERR_ARCH = -4
X1CB_ERR_CUDA = -5
X1CB_ERR_TIMEOUT = -6
X1CB_ERR_WORKSPACE = -7
X1CB_ERR_OVERLAP = -8


class X1cbError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {x1cb_status_string(status)} ({status})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libx1cb.so (raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libx1cb.so is not built ({LIB_PATH}); run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int32, ctypes.c_size_t
        L.conv1x1_bn_add_relu_i8.argtypes = [vp, vp, vp, vp, i32, i32, vp, vp, i, i, i, i, i, vp]
        L.conv3x3_bn_relu_i8.argtypes = [vp, vp, vp, vp, i32, vp, i, i, i, i, i, i, vp]
        L.bottleneck_i8_workspace_size.argtypes = [i, i, i, i]
        L.bottleneck_i8_workspace_size.restype = sz
        L.bottleneck_i8.argtypes = [vp] * 10 + [i32, i32, vp, vp, sz, i, i, i, i, i, vp]
        L.bottleneck_i8_noalloc.argtypes = [vp] * 10 + [i32, i32, vp, i, i, i, i, i, vp]
        L.x1cb_pack_act.argtypes = [vp, vp, i, i, i, i, vp]
        L.x1cb_unpack_act.argtypes = [vp, vp, i, i, i, i, vp]
        L.x1cb_pack_weight.argtypes = [vp, vp, i, i, i, vp]
        L.x1cb_status_string.argtypes = [i]
        L.x1cb_status_string.restype = ctypes.c_char_p
        L.x1cb_last_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint), i]
        L.x1cb_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
        L.x1cb_set_wait_limit_ns.restype = None
        L.x1cb_debug_inject.argtypes = [i]
        L.x1cb_debug_inject.restype = None
        L.x1cb_describe_plan.argtypes = [i, i, i, i, i, i, i, ctypes.c_char_p, sz]
        L.x1cb_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def header_functions() -> list:
    """Names of every function declared in include/x1cb.h."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[\w ]+?\**\s*\b(\w+)\s*\(", text, flags=re.M)


def _check(status: int, what: str):
    if status != X1CB_OK:
        raise X1cbError(status, what)


def _dev(t: Optional[torch.Tensor], dtype, name: str):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _act_shape(x: torch.Tensor, name: str):
    if x.dim() != 5 or x.shape[-1] != 32:
        raise ValueError(f"{name} must be NC/32HW32 [B, C/32, H, W, 32], got {tuple(x.shape)}")
    B, C1, H, W, _ = x.shape
    return B, C1 * 32, H, W


def conv1x1_bn_add_relu_i8(x, w, bias, m, m_r: int, S: int, r=None, out=None, stream=None):
    """Fused 1x1 conv + BN (+ shortcut Sum when r is given) + ReLU + int8.

    x [B, Ic/32, H, W, 32] int8; w blocked [Oc/128, Ic/32, 128, 32] int8;
    bias, m [Oc] int32; r, out [B, Oc/32, H, W, 32] int8."""
    B, Ic, H, W = _act_shape(x, "x")
    Oc = bias.numel()
    if out is None:
        out = torch.empty((B, Oc // 32, H, W, 32), dtype=torch.int8, device=x.device)
    st = lib().conv1x1_bn_add_relu_i8(
        _dev(x, torch.int8, "x"), _dev(w, torch.int8, "w"), _dev(bias, torch.int32, "bias"),
        _dev(m, torch.int32, "m"), int(m_r), int(S), _dev(r, torch.int8, "r"),
        _dev(out, torch.int8, "out"), B, H, W, Ic, Oc, _stream(stream))
    _check(st, "conv1x1_bn_add_relu_i8")
    return out


def conv3x3_bn_relu_i8(x, w, bias, m, S: int, out=None, pad: int = 1, stream=None):
    """Fused 3x3 conv (stride 1, pad 1) + BN + ReLU + int8.

    x [B, Ic/32, H, W, 32]; w [Oc/128, 3, 3, Ic/32, 128, 32]; out [B, Oc/32, H, W, 32]."""
    B, Ic, H, W = _act_shape(x, "x")
    Oc = bias.numel()
    if out is None:
        out = torch.empty((B, Oc // 32, H, W, 32), dtype=torch.int8, device=x.device)
    st = lib().conv3x3_bn_relu_i8(
        _dev(x, torch.int8, "x"), _dev(w, torch.int8, "w"), _dev(bias, torch.int32, "bias"),
        _dev(m, torch.int32, "m"), int(S), _dev(out, torch.int8, "out"), B, H, W, Ic, Oc,
        int(pad), _stream(stream))
    _check(st, "conv3x3_bn_relu_i8")
    return out


def bottleneck_i8_workspace_size(B: int, H: int, W: int, Cmid: int) -> int:
    return int(lib().bottleneck_i8_workspace_size(B, H, W, Cmid))


def bottleneck_i8(x, w1, b1, m1, w2, b2, m2, w3, b3, m3, m_r: int, S: int, out=None,
                  workspace=None, stream=None):
    """Res3.x bottleneck: 1x1 (+BN+ReLU), 3x3 (+BN+ReLU), 1x1 (+BN+Sum(x)+ReLU)."""
    B, Cin, H, W = _act_shape(x, "x")
    Cmid = b1.numel()
    if out is None:
        out = torch.empty_like(x)
    need = bottleneck_i8_workspace_size(B, H, W, Cmid)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.int8, device=x.device)
    st = lib().bottleneck_i8(
        _dev(x, torch.int8, "x"), _dev(w1, torch.int8, "w1"), _dev(b1, torch.int32, "b1"),
        _dev(m1, torch.int32, "m1"), _dev(w2, torch.int8, "w2"), _dev(b2, torch.int32, "b2"),
        _dev(m2, torch.int32, "m2"), _dev(w3, torch.int8, "w3"), _dev(b3, torch.int32, "b3"),
        _dev(m3, torch.int32, "m3"), int(m_r), int(S), _dev(out, torch.int8, "out"),
        _dev(workspace, torch.int8, "workspace"), workspace.numel(), B, H, W, Cin, Cmid,
        _stream(stream))
    _check(st, "bottleneck_i8")
    return out


def bottleneck_i8_noalloc(x, w1, b1, m1, w2, b2, m2, w3, b3, m3, m_r: int, S: int, out=None,
                          stream=None):
    """bottleneck_i8 without a workspace argument, for callers that cannot
    allocate device memory: the library keeps the two intermediates in a
    built-in 32 MiB device array (problems that need more are rejected).
    Calls share that array, so calls that overlap on the GPU race."""
    B, Cin, H, W = _act_shape(x, "x")
    Cmid = b1.numel()
    if out is None:
        out = torch.empty_like(x)
    st = lib().bottleneck_i8_noalloc(
        _dev(x, torch.int8, "x"), _dev(w1, torch.int8, "w1"), _dev(b1, torch.int32, "b1"),
        _dev(m1, torch.int32, "m1"), _dev(w2, torch.int8, "w2"), _dev(b2, torch.int32, "b2"),
        _dev(m2, torch.int32, "m2"), _dev(w3, torch.int8, "w3"), _dev(b3, torch.int32, "b3"),
        _dev(m3, torch.int32, "m3"), int(m_r), int(S), _dev(out, torch.int8, "out"),
        B, H, W, Cin, Cmid, _stream(stream))
    _check(st, "bottleneck_i8_noalloc")
    return out


def x1cb_pack_act(nhwc, out=None, stream=None):
    """[B, H, W, C] int8 -> NC/32HW32 [B, C/32, H, W, 32] on the device."""
    B, H, W, C = nhwc.shape
    if out is None:
        out = torch.empty((B, C // 32, H, W, 32), dtype=torch.int8, device=nhwc.device)
    _check(lib().x1cb_pack_act(_dev(nhwc, torch.int8, "nhwc"), _dev(out, torch.int8, "out"),
                               B, H, W, C, _stream(stream)), "x1cb_pack_act")
    return out


def x1cb_unpack_act(nc32, out=None, stream=None):
    B, C, H, W = _act_shape(nc32, "nc32")
    if out is None:
        out = torch.empty((B, H, W, C), dtype=torch.int8, device=nc32.device)
    _check(lib().x1cb_unpack_act(_dev(nc32, torch.int8, "nc32"), _dev(out, torch.int8, "out"),
                                 B, H, W, C, _stream(stream)), "x1cb_unpack_act")
    return out


def x1cb_pack_weight(oihw, out=None, stream=None):
    """[Oc, Ic, R, R] int8 -> blocked [Oc/128, R, R, Ic/32, 128, 32]."""
    Oc, Ic, R, R2 = oihw.shape
    if out is None:
        out = torch.empty((Oc // 128, R, R, Ic // 32, 128, 32), dtype=torch.int8,
                          device=oihw.device)
    _check(lib().x1cb_pack_weight(_dev(oihw, torch.int8, "oihw"), _dev(out, torch.int8, "out"),
                                  Oc, Ic, R, _stream(stream)), "x1cb_pack_weight")
    return out


def x1cb_status_string(status: int) -> str:
    return lib().x1cb_status_string(int(status)).decode()


def x1cb_last_device_error(clear: bool = True):
    """(status, bits) of the sticky device status word; synchronises."""
    bits = ctypes.c_uint(0)
    st = lib().x1cb_last_device_error(ctypes.byref(bits), int(clear))
    return st, bits.value


def x1cb_set_wait_limit_ns(ns: int):
    lib().x1cb_set_wait_limit_ns(int(ns))


def x1cb_debug_inject(mode: int):
    lib().x1cb_debug_inject(int(mode))


def x1cb_describe_plan(B, H, W, Ic, Oc, R=1, has_res=True) -> str:
    buf = ctypes.create_string_buffer(512)
    _check(lib().x1cb_describe_plan(B, H, W, Ic, Oc, R, int(has_res), buf, 512),
           "x1cb_describe_plan")
    return buf.value.decode()


def x1cb_version() -> str:
    return lib().x1cb_version().decode()
