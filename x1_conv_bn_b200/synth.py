"""Seeded synthetic inputs for the fused INT8 bottleneck convolutions.

This module only draws random tensors. It holds none of the arithmetic of the
convolution or of its epilogue, so that the CPU oracle and the CUDA path can
both be fed from it without sharing any of the method.

Workload recipe (the pages measure on ImageNet through MLPerf and DAWNBench;
no dataset is used here, these synthetic tensors stand in for it):

* Shapes follow the Inspur page "卷积合并计算算法" (MLPerf v2.0 ResNet50), section 3
  (Res3.2 parameters): 28x28, Conv3 Ic=128 -> Oc=512, shortcut with 512
  channels, batch 2048 in section 4.
* Activations and residual: uniform integers in [0, 127].  Weights: uniform in
  [-127, 127].  Bias: uniform in [-2^14, 2^14].  All ranges inclusive.
* Per-channel multiplier m_c: uniform integer in [round(0.9 c), round(1.1 c)]
  with c = round(2^S * 32 / (sqrt(K) * sigma_x * sigma_w)), where sigma_x and
  sigma_w are the analytic standard deviations of the discrete uniform
  distributions above and K is the layer's fan-in R*S*Ic.
* Residual multiplier m_r = 2^(S-1), S = 24.

Tensors are drawn in a fixed order from one ``torch.Generator`` per case
(seed = 1000 + config index by default) and returned in logical NHWC
(activations) and OIHW (weights) layouts.  Packing into NC/32HW32 and the
blocked weight layout is part of the method and is done by each side with
its own code.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, Optional

import torch

S_DEFAULT = 24
X_LO, X_HI = 0, 127
W_LO, W_HI = -127, 127
BIAS_LO, BIAS_HI = -(1 << 14), 1 << 14
# Analytic standard deviation of a discrete uniform distribution over n values.
SIGMA_X = math.sqrt(((X_HI - X_LO + 1) ** 2 - 1) / 12.0)
SIGMA_W = math.sqrt(((W_HI - W_LO + 1) ** 2 - 1) / 12.0)


def multiplier_center(fan_in: int, S: int = S_DEFAULT) -> int:
    """Centre of the m_c distribution for a layer of fan-in ``fan_in``."""
    return int(round((2 ** S) * 32.0 / (math.sqrt(fan_in) * SIGMA_X * SIGMA_W)))


def _randint(g: torch.Generator, lo: int, hi: int, shape, dtype, device) -> torch.Tensor:
    return torch.randint(lo, hi + 1, tuple(shape), generator=g, dtype=dtype, device=device)


@dataclass(frozen=True)
class ConvShape:
    """One fused convolution layer: stride 1, 'same' padding (R-1)/2."""

    B: int
    H: int
    W: int
    Ic: int
    Oc: int
    R: int = 1
    has_res: bool = True

    @property
    def pad(self) -> int:
        return (self.R - 1) // 2

    @property
    def fan_in(self) -> int:
        return self.R * self.R * self.Ic

    @property
    def pixels(self) -> int:
        return self.B * self.H * self.W

    def ops(self) -> int:
        """Multiply-adds counted as 2 ops: 2*M*N*K."""
        return 2 * self.pixels * self.Oc * self.fan_in

    def bytes_moved(self) -> int:
        """Algorithmic HBM bytes: every tensor read or written once."""
        n = self.pixels * (self.Ic + self.Oc)  # x read + out written
        if self.has_res:
            n += self.pixels * self.Oc  # residual read
        n += self.Oc * self.fan_in  # weights
        n += self.Oc * 8  # bias + multiplier (int32 each)
        return n


@dataclass(frozen=True)
class BlockShape:
    """Res3.x bottleneck: 1x1 Cin->Cmid, 3x3 Cmid->Cmid, 1x1 Cmid->Cin + shortcut."""

    B: int
    H: int
    W: int
    Cin: int
    Cmid: int

    def stages(self):
        return (
            ConvShape(self.B, self.H, self.W, self.Cin, self.Cmid, 1, False),
            ConvShape(self.B, self.H, self.W, self.Cmid, self.Cmid, 3, False),
            ConvShape(self.B, self.H, self.W, self.Cmid, self.Cin, 1, True),
        )

    def ops(self) -> int:
        return sum(s.ops() for s in self.stages())

    def bytes_moved(self) -> int:
        return sum(s.bytes_moved() for s in self.stages())


@dataclass(frozen=True)
class ProjBlockShape:
    """Res3.1-style projection bottleneck on an H x W input: 1x1 Cin->Cmid,
    3x3 stride 2 Cmid->Cmid, 1x1 Cmid->Cout plus the stride-2 1x1 projection
    Cin->Cout of the block input in the same accumulator."""

    B: int
    H: int
    W: int
    Cin: int
    Cmid: int
    Cout: int

    @property
    def Ho(self) -> int:
        return (self.H - 1) // 2 + 1

    @property
    def Wo(self) -> int:
        return (self.W - 1) // 2 + 1

    def ops(self) -> int:
        px_in, px_out = self.B * self.H * self.W, self.B * self.Ho * self.Wo
        return 2 * (px_in * self.Cmid * self.Cin + px_out * self.Cmid * 9 * self.Cmid
                    + px_out * self.Cout * (self.Cmid + self.Cin))

    def bytes_moved(self) -> int:
        px_in, px_out = self.B * self.H * self.W, self.B * self.Ho * self.Wo
        n = px_in * (self.Cin + self.Cmid)                      # conv1: x in, y1 out
        n += px_in * self.Cmid + px_out * self.Cmid             # conv2: y1 in, y2 out
        n += px_out * (self.Cmid + self.Cin + self.Cout)        # conv3: y2, strided x, out
        n += self.Cmid * self.Cin + 9 * self.Cmid ** 2 + self.Cout * (self.Cmid + self.Cin)
        n += 8 * (2 * self.Cmid + self.Cout)
        return n


@dataclass
class ProjBlockInputs:
    shape: ProjBlockShape
    x: torch.Tensor  # [B, H, W, Cin] int8
    w: list = field(default_factory=list)  # conv1, conv2, conv3 OIHW
    wp: Optional[torch.Tensor] = None      # projection [Cout, Cin, 1, 1]
    bias: list = field(default_factory=list)
    m: list = field(default_factory=list)
    S: int = S_DEFAULT


def proj_block_inputs(s: ProjBlockShape, seed: int, device="cpu",
                      S: int = S_DEFAULT) -> ProjBlockInputs:
    """Draw x, then (w, bias, m) of conv1 and conv2, then w3, wp, bias3, m3.
    The third layer's multiplier uses the fan-in of both sources (Cmid + Cin)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = _randint(g, X_LO, X_HI, (s.B, s.H, s.W, s.Cin), torch.int8, device)
    out = ProjBlockInputs(s, x, S=S)
    for st in (ConvShape(s.B, s.H, s.W, s.Cin, s.Cmid, 1, False),
               ConvShape(s.B, s.H, s.W, s.Cmid, s.Cmid, 3, False)):
        w, bias, m = _draw_layer(g, st, S, device)
        out.w.append(w)
        out.bias.append(bias)
        out.m.append(m)
    out.w.append(_randint(g, W_LO, W_HI, (s.Cout, s.Cmid, 1, 1), torch.int8, device))
    out.wp = _randint(g, W_LO, W_HI, (s.Cout, s.Cin, 1, 1), torch.int8, device)
    out.bias.append(_randint(g, BIAS_LO, BIAS_HI, (s.Cout,), torch.int32, device))
    c = multiplier_center(s.Cmid + s.Cin, S)
    out.m.append(_randint(g, int(round(0.9 * c)), int(round(1.1 * c)), (s.Cout,), torch.int32,
                          device))
    return out


@dataclass(frozen=True)
class StemShape:
    """The network's stem: R x R convolution (pad (R-1)/2, stride) of an image
    of Cin channels (carried in one 32-channel block), BN, ReLU, then 3x3
    stride-2 max pooling; Oc = 64 output channels."""

    B: int
    H: int
    W: int
    Cin: int = 3
    Oc: int = 64
    R: int = 7
    stride: int = 2

    @property
    def Hc(self) -> int:
        return (self.H + 2 * ((self.R - 1) // 2) - self.R) // self.stride + 1

    @property
    def Wc(self) -> int:
        return (self.W + 2 * ((self.R - 1) // 2) - self.R) // self.stride + 1

    @property
    def Hp(self) -> int:
        return (self.Hc - 1) // 2 + 1

    @property
    def Wp(self) -> int:
        return (self.Wc - 1) // 2 + 1

    def ops(self) -> int:
        """2 x MACs of the convolution over the image's real channels."""
        return 2 * self.B * self.Hc * self.Wc * self.Oc * self.R * self.R * self.Cin

    def bytes_moved(self) -> int:
        """The stem's input as the kernel reads it -- the width-folded image,
        one 32-byte block per image row and output column (H x Wc) -- plus the
        pooled output, the folded weights (R K blocks of 64 x 32) and the
        per-channel constants."""
        return (self.B * self.H * self.Wc * 32 + self.B * self.Hp * self.Wp * self.Oc
                + self.Oc * 32 * self.R + 8 * self.Oc)


def stem_inputs(s: StemShape, seed: int, device="cpu", S: int = S_DEFAULT) -> ConvInputs:
    """Image x in [0, 127] (Cin channels), weights, bias, multiplier (fan-in
    R*R*Cin)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = _randint(g, X_LO, X_HI, (s.B, s.H, s.W, s.Cin), torch.int8, device)
    w, bias, m = _draw_layer(g, ConvShape(s.B, s.H, s.W, s.Cin, s.Oc, s.R, False), S, device)
    return ConvInputs(ConvShape(s.B, s.H, s.W, s.Cin, s.Oc, s.R, False), x, w, bias, m, None, 0,
                      S)


# Named workloads.  Index 1..5 as in the benchmark plan; "4a".."4c" are the
# three expand convolutions of the sweep.
CONFIGS: Dict[str, object] = {
    "1": ConvShape(1, 28, 28, 128, 512, 1, True),
    "2": ConvShape(256, 28, 28, 128, 512, 1, True),
    "3": ConvShape(2048, 28, 28, 128, 512, 1, True),
    "4a": ConvShape(512, 56, 56, 64, 256, 1, True),
    "4b": ConvShape(512, 14, 14, 256, 1024, 1, True),
    "4c": ConvShape(512, 7, 7, 512, 2048, 1, True),
    "5": BlockShape(1024, 28, 28, 512, 128),
    # Res3.1 (the stage's projection block), 56x56x256 in, 28x28x512 out.
    "p31": ProjBlockShape(256, 56, 56, 256, 128, 512),
    # Res4.x conv2: 3x3 256 -> 256 at 14x14 (weights streamed).
    "r4c2": ConvShape(512, 14, 14, 256, 256, 3, False),
    # The stem: 7x7 stride 2 of a 224x224 RGB image, BN, ReLU, 3x3/2 max pool.
    "stem": StemShape(256, 224, 224),
}
CONFIG_SEEDS = {"1": 1001, "2": 1002, "3": 1003, "4a": 1004, "4b": 1004, "4c": 1004, "5": 1005,
                "p31": 1031, "r4c2": 1042, "stem": 1050}
WORKLOAD_NAMES = {
    "1": "res3.2-conv3 1x1 128->512 +bn+sum+relu, 28x28, B=1",
    "2": "res3.2-conv3 1x1 128->512 +bn+sum+relu, 28x28, B=256",
    "3": "res3.2-conv3 1x1 128->512 +bn+sum+relu, 28x28, B=2048",
    "4a": "expand 1x1 64->256 +bn+sum+relu, 56x56, B=512",
    "4b": "expand 1x1 256->1024 +bn+sum+relu, 14x14, B=512",
    "4c": "expand 1x1 512->2048 +bn+sum+relu, 7x7, B=512",
    "5": "res3.2 bottleneck block 512->128->128->512, 28x28, B=1024",
    "p31": "res3.1 projection block 256->128->128(s2)->512 + proj 256->512(s2), 56x56->28x28, "
           "B=256",
    "r4c2": "res4.x conv2 3x3 256->256 +bn+relu, 14x14, B=512",
    "stem": "stem 7x7/2 3->64 +bn+relu+maxpool 3x3/2, 224x224->56x56, B=256",
}


@dataclass
class ConvInputs:
    shape: ConvShape
    x: torch.Tensor  # [B, H, W, Ic] int8
    w: torch.Tensor  # [Oc, Ic, R, R] int8
    bias: torch.Tensor  # [Oc] int32
    m: torch.Tensor  # [Oc] int32
    r: Optional[torch.Tensor]  # [B, H, W, Oc] int8 or None
    m_r: int
    S: int


@dataclass
class BlockInputs:
    shape: BlockShape
    x: torch.Tensor  # [B, H, W, Cin] int8 (also the residual)
    w: list = field(default_factory=list)  # three OIHW weights
    bias: list = field(default_factory=list)
    m: list = field(default_factory=list)
    m_r: int = 1 << (S_DEFAULT - 1)
    S: int = S_DEFAULT


def _draw_layer(g, s: ConvShape, S: int, device):
    w = _randint(g, W_LO, W_HI, (s.Oc, s.Ic, s.R, s.R), torch.int8, device)
    bias = _randint(g, BIAS_LO, BIAS_HI, (s.Oc,), torch.int32, device)
    c = multiplier_center(s.fan_in, S)
    m = _randint(g, int(round(0.9 * c)), int(round(1.1 * c)), (s.Oc,), torch.int32, device)
    return w, bias, m


def conv_inputs(s: ConvShape, seed: int, device="cpu", S: int = S_DEFAULT) -> ConvInputs:
    """Draw x, w, bias, m, r (in that order) for one fused layer."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = _randint(g, X_LO, X_HI, (s.B, s.H, s.W, s.Ic), torch.int8, device)
    w, bias, m = _draw_layer(g, s, S, device)
    r = _randint(g, X_LO, X_HI, (s.B, s.H, s.W, s.Oc), torch.int8, device) if s.has_res else None
    return ConvInputs(s, x, w, bias, m, r, 1 << (S - 1), S)


def block_inputs(s: BlockShape, seed: int, device="cpu", S: int = S_DEFAULT) -> BlockInputs:
    """Draw x, then (w, bias, m) for conv1, conv2, conv3."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = _randint(g, X_LO, X_HI, (s.B, s.H, s.W, s.Cin), torch.int8, device)
    out = BlockInputs(s, x, S=S, m_r=1 << (S - 1))
    for st in s.stages():
        w, bias, m = _draw_layer(g, st, S, device)
        out.w.append(w)
        out.bias.append(bias)
        out.m.append(m)
    return out


def full_range_conv_inputs(s: ConvShape, seed: int, S: int, device="cpu") -> ConvInputs:
    """Stress inputs: x, w, r over the full int8 range; bias, m, m_r over wide
    int32 ranges.  Used for edge-case parity (the method must be exact for any
    int8 data, not only the benchmark distributions)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = _randint(g, -128, 127, (s.B, s.H, s.W, s.Ic), torch.int8, device)
    w = _randint(g, -128, 127, (s.Oc, s.Ic, s.R, s.R), torch.int8, device)
    bias = _randint(g, -(1 << 20), (1 << 20), (s.Oc,), torch.int32, device)
    m = _randint(g, -(1 << 20), (1 << 20), (s.Oc,), torch.int32, device)
    r = _randint(g, -128, 127, (s.B, s.H, s.W, s.Oc), torch.int8, device) if s.has_res else None
    m_r = int(_randint(g, -(1 << 26), (1 << 26), (1,), torch.int32, device).item())
    return ConvInputs(s, x, w, bias, m, r, m_r, S)
