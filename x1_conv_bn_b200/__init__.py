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
X1CB_ERR_DEVICE = -9


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
        L.x1cb_last_epilogue_forms.argtypes = [ctypes.POINTER(ctypes.c_uint), i]
        L.x1cb_trace_copy.argtypes = [vp, ctypes.c_longlong, i]
        L.x1cb_trace_copy.restype = ctypes.c_longlong
        L.x1cb_set_block_fusion.argtypes = [i]
        L.x1cb_set_block_fusion.restype = None
        L.x1cb_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
        L.x1cb_set_wait_limit_ns.restype = None
        L.x1cb_debug_inject.argtypes = [i]
        L.x1cb_debug_inject.restype = None
        L.x1cb_describe_plan.argtypes = [i, i, i, i, i, i, i, ctypes.c_char_p, sz]
        L.x1cb_version.restype = ctypes.c_char_p
        L.conv3x3s2_bn_relu_i8.argtypes = [vp] * 4 + [i32, vp] + [i] * 5 + [vp]
        L.conv1x1_proj_bn_relu_i8.argtypes = [vp] * 6 + [i32, vp] + [i] * 8 + [vp]
        L.bottleneck_proj_i8_workspace_size.argtypes = [i, i, i, i]
        L.bottleneck_proj_i8_workspace_size.restype = sz
        L.bottleneck_proj_i8.argtypes = [vp] * 11 + [i32, vp, vp, sz] + [i] * 6 + [vp]
        L.x1cb_describe_plan_ex.argtypes = [i] * 10 + [ctypes.c_char_p, sz]
        L.conv_bn_relu_maxpool_i8.argtypes = [vp] * 4 + [i32, vp] + [i] * 7 + [vp]
        L.x1cb_describe_chain.argtypes = [i] * 5 + [ctypes.c_char_p, sz]
        L.conv3x3_conv1x1_bn_add_relu_i8.argtypes = [vp] * 7 + [i32, i32, vp, vp] + [i] * 5 + [vp]
        L.stem_conv_bn_relu_maxpool_i8.argtypes = [vp] * 4 + [i32, vp] + [i] * 4 + [vp]
        L.x1cb_pack_stem.argtypes = [vp, vp] + [i] * 5 + [vp]
        L.x1cb_pack_stem_weight.argtypes = [vp, vp] + [i] * 3 + [vp]
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


def _stream(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif isinstance(stream, torch.cuda.Stream) and stream.device != device:
        raise ValueError(f"stream is on {stream.device}, operands on {device}")
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _same_device(first: torch.Tensor, *others):
    """Every operand must live on the first one's GPU; the call then runs with
    that GPU current (the library launches on the current device)."""
    if not isinstance(first, torch.Tensor) or first.device.type != "cuda":
        raise ValueError("operands must be CUDA tensors")
    for t in others:
        if t is not None and isinstance(t, torch.Tensor) and t.device != first.device:
            raise ValueError(f"operand on {t.device}, expected {first.device}")
    return torch.cuda.device(first.device)


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
    with _same_device(x, w, bias, m, r, out):
        st = lib().conv1x1_bn_add_relu_i8(
            _dev(x, torch.int8, "x"), _dev(w, torch.int8, "w"), _dev(bias, torch.int32, "bias"),
            _dev(m, torch.int32, "m"), int(m_r), int(S), _dev(r, torch.int8, "r"),
            _dev(out, torch.int8, "out"), B, H, W, Ic, Oc, _stream(stream, x.device))
    _check(st, "conv1x1_bn_add_relu_i8")
    return out


def conv3x3_bn_relu_i8(x, w, bias, m, S: int, out=None, pad: int = 1, stream=None):
    """Fused 3x3 conv (stride 1, pad 1) + BN + ReLU + int8.

    x [B, Ic/32, H, W, 32]; w [Oc/128, 3, 3, Ic/32, 128, 32]; out [B, Oc/32, H, W, 32]."""
    B, Ic, H, W = _act_shape(x, "x")
    Oc = bias.numel()
    if out is None:
        out = torch.empty((B, Oc // 32, H, W, 32), dtype=torch.int8, device=x.device)
    with _same_device(x, w, bias, m, out):
        st = lib().conv3x3_bn_relu_i8(
            _dev(x, torch.int8, "x"), _dev(w, torch.int8, "w"), _dev(bias, torch.int32, "bias"),
            _dev(m, torch.int32, "m"), int(S), _dev(out, torch.int8, "out"), B, H, W, Ic, Oc,
            int(pad), _stream(stream, x.device))
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
    with _same_device(x, w1, b1, m1, w2, b2, m2, w3, b3, m3, out, workspace):
        st = lib().bottleneck_i8(
            _dev(x, torch.int8, "x"), _dev(w1, torch.int8, "w1"), _dev(b1, torch.int32, "b1"),
            _dev(m1, torch.int32, "m1"), _dev(w2, torch.int8, "w2"), _dev(b2, torch.int32, "b2"),
            _dev(m2, torch.int32, "m2"), _dev(w3, torch.int8, "w3"), _dev(b3, torch.int32, "b3"),
            _dev(m3, torch.int32, "m3"), int(m_r), int(S), _dev(out, torch.int8, "out"),
            _dev(workspace, torch.int8, "workspace"), workspace.numel(), B, H, W, Cin, Cmid,
            _stream(stream, x.device))
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
    with _same_device(x, w1, b1, m1, w2, b2, m2, w3, b3, m3, out):
        st = lib().bottleneck_i8_noalloc(
            _dev(x, torch.int8, "x"), _dev(w1, torch.int8, "w1"), _dev(b1, torch.int32, "b1"),
            _dev(m1, torch.int32, "m1"), _dev(w2, torch.int8, "w2"), _dev(b2, torch.int32, "b2"),
            _dev(m2, torch.int32, "m2"), _dev(w3, torch.int8, "w3"), _dev(b3, torch.int32, "b3"),
            _dev(m3, torch.int32, "m3"), int(m_r), int(S), _dev(out, torch.int8, "out"),
            B, H, W, Cin, Cmid, _stream(stream, x.device))
    _check(st, "bottleneck_i8_noalloc")
    return out


def _half(n: int) -> int:
    """Output extent of a stride-2 3x3 (pad 1) over n pixels."""
    return (n - 1) // 2 + 1 if n > 0 else 0


def conv3x3_conv1x1_bn_add_relu_i8(y1, w2, b2, m2, w3, b3, m3, m_r: int, S: int, r,
                                   out=None, stream=None):
    """Conv2 (3x3 + BN + ReLU) -> Conv3 (1x1 + BN + shortcut r + ReLU) of the
    bottleneck in one launch; conv2's output stays on chip.
    y1 [B, Cmid/32, H, W, 32]; r, out [B, Cout/32, H, W, 32]."""
    B, Cmid, H, W = _act_shape(y1, "y1")
    Cout = b3.numel()
    if out is None:
        out = torch.empty((B, Cout // 32, H, W, 32), dtype=torch.int8, device=y1.device)
    with _same_device(y1, w2, b2, m2, w3, b3, m3, r, out):
        st = lib().conv3x3_conv1x1_bn_add_relu_i8(
            _dev(y1, torch.int8, "y1"), _dev(w2, torch.int8, "w2"), _dev(b2, torch.int32, "b2"),
            _dev(m2, torch.int32, "m2"), _dev(w3, torch.int8, "w3"), _dev(b3, torch.int32, "b3"),
            _dev(m3, torch.int32, "m3"), int(m_r), int(S), _dev(r, torch.int8, "r"),
            _dev(out, torch.int8, "out"), B, H, W, Cmid, Cout, _stream(stream, y1.device))
    _check(st, "conv3x3_conv1x1_bn_add_relu_i8")
    return out


def conv3x3s2_bn_relu_i8(x, w, bias, m, S: int, out=None, stream=None):
    """Fused 3x3 stride-2 conv (pad 1) + BN + ReLU + int8 (a projection
    block's Conv2).  x [B, Ic/32, H, W, 32] -> out [B, Oc/32, Ho, Wo, 32]."""
    B, Ic, H, W = _act_shape(x, "x")
    Oc = bias.numel()
    if out is None:
        out = torch.empty((B, Oc // 32, _half(H), _half(W), 32), dtype=torch.int8,
                          device=x.device)
    with _same_device(x, w, bias, m, out):
        st = lib().conv3x3s2_bn_relu_i8(
            _dev(x, torch.int8, "x"), _dev(w, torch.int8, "w"), _dev(bias, torch.int32, "bias"),
            _dev(m, torch.int32, "m"), int(S), _dev(out, torch.int8, "out"), B, H, W, Ic, Oc,
            _stream(stream, x.device))
    _check(st, "conv3x3s2_bn_relu_i8")
    return out


def conv1x1_proj_bn_relu_i8(y, w3, x, wp, bias, m, S: int, out=None, stream=None):
    """Projection block's Conv3: 1x1 of y plus the stride-2 1x1 of the block
    input x in one accumulator, + BN + ReLU + int8.
    y [B, Cy/32, H, W, 32]; x [B, Cx/32, Hx, Wx, 32]; out [B, Oc/32, H, W, 32]."""
    B, Cy, H, W = _act_shape(y, "y")
    B2, Cx, Hx, Wx = _act_shape(x, "x")
    if B2 != B:
        raise ValueError("y and x must have the same batch")
    Oc = bias.numel()
    if out is None:
        out = torch.empty((B, Oc // 32, H, W, 32), dtype=torch.int8, device=y.device)
    with _same_device(y, w3, x, wp, bias, m, out):
        st = lib().conv1x1_proj_bn_relu_i8(
            _dev(y, torch.int8, "y"), _dev(w3, torch.int8, "w3"), _dev(x, torch.int8, "x"),
            _dev(wp, torch.int8, "wp"), _dev(bias, torch.int32, "bias"),
            _dev(m, torch.int32, "m"), int(S), _dev(out, torch.int8, "out"),
            B, H, W, Cy, Hx, Wx, Cx, Oc, _stream(stream, y.device))
    _check(st, "conv1x1_proj_bn_relu_i8")
    return out


def conv_bn_relu_maxpool_i8(x, w, bias, m, S: int, R: int = 7, stride: int = 2, out=None,
                            stream=None):
    """The stem's conv (R x R, pad (R-1)/2, stride) + BN + ReLU + 3x3 stride-2
    max pooling in one launch; 64 output channels.
    x [B, Ic/32, H, W, 32] -> out [B, 2, Hp, Wp, 32]."""
    B, Ic, H, W = _act_shape(x, "x")
    Oc = bias.numel()
    pad = (R - 1) // 2
    Hc, Wc = (H + 2 * pad - R) // stride + 1, (W + 2 * pad - R) // stride + 1
    if out is None:
        out = torch.empty((B, Oc // 32, _half(Hc), _half(Wc), 32), dtype=torch.int8,
                          device=x.device)
    with _same_device(x, w, bias, m, out):
        st = lib().conv_bn_relu_maxpool_i8(
            _dev(x, torch.int8, "x"), _dev(w, torch.int8, "w"), _dev(bias, torch.int32, "bias"),
            _dev(m, torch.int32, "m"), int(S), _dev(out, torch.int8, "out"), B, H, W, Ic, Oc,
            int(R), int(stride), _stream(stream, x.device))
    _check(st, "conv_bn_relu_maxpool_i8")
    return out


def stem_fold_width(W: int, R: int = 7) -> int:
    """Columns of the folded stem tensor: the stride-2 convolution's outputs."""
    pad = (R - 1) // 2
    return (W + 2 * pad - R) // 2 + 1 if W + 2 * pad >= R else 0


def x1cb_pack_stem(nhwc, R: int = 7, out=None, stream=None):
    """Image [B, H, W, Cin] -> width-folded [B, 1, H, Wc, 32] (R*Cin <= 32),
    Wc = stem_fold_width(W, R)."""
    B, H, W, Cin = nhwc.shape
    if out is None:
        out = torch.empty((B, 1, H, stem_fold_width(W, R), 32), dtype=torch.int8,
                          device=nhwc.device)
    with _same_device(nhwc, out):
        st = lib().x1cb_pack_stem(_dev(nhwc, torch.int8, "nhwc"), _dev(out, torch.int8, "out"),
                                  B, H, W, Cin, int(R), _stream(stream, nhwc.device))
    _check(st, "x1cb_pack_stem")
    return out


def x1cb_pack_stem_weight(oihw, out=None, stream=None):
    """[64, Cin, R, R] -> folded [1, R, 1, 1, 64, 32]."""
    Oc, Cin, R, _ = oihw.shape
    if out is None:
        out = torch.empty((1, R, 1, 1, Oc, 32), dtype=torch.int8, device=oihw.device)
    with _same_device(oihw, out):
        st = lib().x1cb_pack_stem_weight(_dev(oihw, torch.int8, "oihw"),
                                         _dev(out, torch.int8, "out"), Oc, Cin, R,
                                         _stream(stream, oihw.device))
    _check(st, "x1cb_pack_stem_weight")
    return out


def stem_conv_bn_relu_maxpool_i8(folded, wf, bias, m, S: int, R: int = 7, out=None,
                                 stream=None, W: Optional[int] = None):
    """The stem on a width-folded image: R x R stride-2 conv + BN + ReLU +
    3x3 stride-2 max pooling, 64 outputs.  folded [B, 1, H, Wc, 32] from
    x1cb_pack_stem; W is the image width (any width whose folded width is Wc
    gives the same result; default 2*Wc)."""
    B, C, H, Wc = _act_shape(folded, "folded")
    pad = (R - 1) // 2
    if W is None:
        W = 2 * Wc
    if stem_fold_width(W, R) != Wc:
        raise X1cbError(X1CB_ERR_SHAPE, "stem_conv_bn_relu_maxpool_i8: W does not fold to Wc")
    Hc = (H + 2 * pad - R) // 2 + 1
    if out is None:
        out = torch.empty((B, 2, _half(Hc), _half(Wc), 32), dtype=torch.int8,
                          device=folded.device)
    with _same_device(folded, wf, bias, m, out):
        st = lib().stem_conv_bn_relu_maxpool_i8(
            _dev(folded, torch.int8, "folded"), _dev(wf, torch.int8, "wf"),
            _dev(bias, torch.int32, "bias"), _dev(m, torch.int32, "m"), int(S),
            _dev(out, torch.int8, "out"), B, H, W, int(R), _stream(stream, folded.device))
    _check(st, "stem_conv_bn_relu_maxpool_i8")
    return out


def bottleneck_proj_i8_workspace_size(B: int, H: int, W: int, Cmid: int) -> int:
    return int(lib().bottleneck_proj_i8_workspace_size(B, H, W, Cmid))


def bottleneck_proj_i8(x, w1, b1, m1, w2, b2, m2, w3, wp, b3, m3, S: int, out=None,
                       workspace=None, stream=None):
    """Projection bottleneck (Res3.1): 1x1, 3x3 stride 2, 1x1 + stride-2 1x1
    projection of x in one accumulator; BN + ReLU after each."""
    B, Cin, H, W = _act_shape(x, "x")
    Cmid, Cout = b1.numel(), b3.numel()
    if out is None:
        out = torch.empty((B, Cout // 32, _half(H), _half(W), 32), dtype=torch.int8,
                          device=x.device)
    need = bottleneck_proj_i8_workspace_size(B, H, W, Cmid)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.int8, device=x.device)
    with _same_device(x, w1, b1, m1, w2, b2, m2, w3, wp, b3, m3, out, workspace):
        st = lib().bottleneck_proj_i8(
            _dev(x, torch.int8, "x"), _dev(w1, torch.int8, "w1"), _dev(b1, torch.int32, "b1"),
            _dev(m1, torch.int32, "m1"), _dev(w2, torch.int8, "w2"), _dev(b2, torch.int32, "b2"),
            _dev(m2, torch.int32, "m2"), _dev(w3, torch.int8, "w3"), _dev(wp, torch.int8, "wp"),
            _dev(b3, torch.int32, "b3"), _dev(m3, torch.int32, "m3"), int(S),
            _dev(out, torch.int8, "out"), _dev(workspace, torch.int8, "workspace"),
            workspace.numel(), B, H, W, Cin, Cmid, Cout, _stream(stream, x.device))
    _check(st, "bottleneck_proj_i8")
    return out


def x1cb_pack_act(nhwc, out=None, stream=None):
    """[B, H, W, C] int8 -> NC/32HW32 [B, C/32, H, W, 32] on the device."""
    B, H, W, C = nhwc.shape
    if out is None:
        out = torch.empty((B, C // 32, H, W, 32), dtype=torch.int8, device=nhwc.device)
    with _same_device(nhwc, out):
        st = lib().x1cb_pack_act(_dev(nhwc, torch.int8, "nhwc"), _dev(out, torch.int8, "out"),
                                 B, H, W, C, _stream(stream, nhwc.device))
    _check(st, "x1cb_pack_act")
    return out


def x1cb_unpack_act(nc32, out=None, stream=None):
    B, C, H, W = _act_shape(nc32, "nc32")
    if out is None:
        out = torch.empty((B, H, W, C), dtype=torch.int8, device=nc32.device)
    with _same_device(nc32, out):
        st = lib().x1cb_unpack_act(_dev(nc32, torch.int8, "nc32"), _dev(out, torch.int8, "out"),
                                   B, H, W, C, _stream(stream, nc32.device))
    _check(st, "x1cb_unpack_act")
    return out


def x1cb_pack_weight(oihw, out=None, stream=None):
    """[Oc, Ic, R, R] int8 -> blocked [Oc/O2, R, R, Ic/32, O2, 32], O2 = min(Oc, 128)."""
    Oc, Ic, R, R2 = oihw.shape
    O2 = min(Oc, 128)
    if out is None:
        out = torch.empty((Oc // O2, R, R, Ic // 32, O2, 32), dtype=torch.int8,
                          device=oihw.device)
    with _same_device(oihw, out):
        st = lib().x1cb_pack_weight(_dev(oihw, torch.int8, "oihw"),
                                    _dev(out, torch.int8, "out"), Oc, Ic, R,
                                    _stream(stream, oihw.device))
    _check(st, "x1cb_pack_weight")
    return out


def x1cb_status_string(status: int) -> str:
    return lib().x1cb_status_string(int(status)).decode()


def x1cb_last_device_error(clear: bool = True):
    """(status, bits) of the sticky device status word; synchronises."""
    bits = ctypes.c_uint(0)
    st = lib().x1cb_last_device_error(ctypes.byref(bits), int(clear))
    return st, bits.value


def x1cb_last_epilogue_forms(clear: bool = True) -> int:
    """Bit set of the exact epilogue forms run since the last clear (bit 0
    generic, 1 64-bit high word, 2 all-32-bit, 3 all-32-bit with the bias in
    the MMA); synchronises."""
    bits = ctypes.c_uint(0)
    _check(lib().x1cb_last_epilogue_forms(ctypes.byref(bits), int(clear)),
           "x1cb_last_epilogue_forms")
    return bits.value


TRACE_SHAPE = (4, 16, 1024)  # [cta][event][n] of SM clock values


def x1cb_trace_copy(clear: bool = True):
    """Timeline table of a trace build as an int64 tensor of TRACE_SHAPE
    (None when the library was built without the trace)."""
    import numpy as np

    words = TRACE_SHAPE[0] * TRACE_SHAPE[1] * TRACE_SHAPE[2]
    buf = np.zeros(words, dtype=np.uint64)
    n = lib().x1cb_trace_copy(buf.ctypes.data, words, int(clear))
    if n < 0:
        raise X1cbError(int(n), "x1cb_trace_copy")
    if n == 0:
        return None
    return torch.from_numpy(buf.view(np.int64).reshape(TRACE_SHAPE).copy())


def x1cb_set_block_fusion(enable: bool):
    """On: bottleneck_i8 runs conv2 -> conv3 as one fused launch where the
    shape allows.  Off (the default, measured faster on B200): separate
    launches.  Same results either way."""
    lib().x1cb_set_block_fusion(int(bool(enable)))


def x1cb_set_wait_limit_ns(ns: int):
    lib().x1cb_set_wait_limit_ns(int(ns))


def x1cb_debug_inject(mode: int):
    lib().x1cb_debug_inject(int(mode))


def x1cb_describe_plan(B, H, W, Ic, Oc, R=1, has_res=True) -> str:
    buf = ctypes.create_string_buffer(512)
    _check(lib().x1cb_describe_plan(B, H, W, Ic, Oc, R, int(has_res), buf, 512),
           "x1cb_describe_plan")
    return buf.value.decode()


def x1cb_describe_plan_ex(B, Hin, Win, Ic, Oc, R=1, stride=1, Ic2=0, has_res=False,
                          pool=False) -> str:
    buf = ctypes.create_string_buffer(512)
    _check(lib().x1cb_describe_plan_ex(B, Hin, Win, Ic, Oc, R, stride, Ic2, int(has_res),
                                       int(pool), buf, 512), "x1cb_describe_plan_ex")
    return buf.value.decode()


def x1cb_describe_chain(B, H, W, Cmid=128, Cout=512) -> str:
    buf = ctypes.create_string_buffer(512)
    _check(lib().x1cb_describe_chain(B, H, W, Cmid, Cout, buf, 512), "x1cb_describe_chain")
    return buf.value.decode()


def x1cb_version() -> str:
    return lib().x1cb_version().decode()
